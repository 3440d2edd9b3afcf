"""The C-ABI library loads on a machine without a GPU, exports every function that
include/fa.h declares, and rejects bad arguments on the host before any CUDA call."""

import ctypes
import os
import re

import pytest

from exact_io_aware_63_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_0-9]+\s*\*?\s*(fa_[a-z_0-9]+)\s*\(",
                                 text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ["fa_fwd", "fa_fwd_traced", "fa_bwd", "fa_bwd_traced", "fa_bwd_phase",
              "fa_bwd_deterministic", "fa_fwd_dropout", "fa_bwd_dropout",
              "fa_selftest_wait_timeout", "fa_selftest_ex2", "fa_fwd_varlen", "fa_bwd_varlen",
              "fa_bwd_workspace_size",
              "fa_get_device_status", "fa_status_string", "fa_version"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(binding.library_path() if os.path.exists(binding.library_path())
                      else binding.load()._name)
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert binding.fa_version() == 10000
    for code in [0, -1, -2, -3, -4, -5, -6, -7, -8]:
        assert binding.fa_status_string(code) != "unknown status"
    assert binding.fa_status_string(12345) == "unknown status"


def test_workspace_size():
    B, H, N, d = 16, 16, 512, 64
    R = B * H * N
    ws = binding.fa_bwd_workspace_size(B, H, N, d)
    assert ws >= 4 * R + 4 * R + 4 * R * d
    assert ws % 256 == 0
    assert binding.fa_bwd_workspace_size(1, 1, 100, 64) >= 4 * 100 * 66   # any N >= 1
    assert binding.fa_bwd_workspace_size(1, 1, -128, 64) == 0     # negative
    assert binding.fa_bwd_workspace_size(1, 1, 128, 80) == 0      # d
    # d = 32 and 96 run on the 64 / 128 kernels; their scratch is sized by d
    assert binding.fa_bwd_workspace_size(1, 1, 128, 96) >= 4 * 128 * 96
    assert binding.fa_bwd_workspace_size(1, 1, 128, 96) < binding.fa_bwd_workspace_size(
        1, 1, 128, 128)
    assert binding.fa_bwd_workspace_size(0, 1, 128, 64) == 0      # empty


# Fake, well-aligned device addresses: validation fails before they are touched.
P = 1 << 40


def fwd(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=128, d=64, scale=0.125, causal=0,
             block_mask=None, kv_len=None)
    a.update(kw)
    lib = binding.load()
    return lib.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"],
                      a["scale"], a["causal"], a["block_mask"], a["kv_len"], None)


def bwd(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=1, H=1, N=128, d=64,
             scale=0.125, causal=0, block_mask=None, kv_len=None, ws=P, ws_bytes=1 << 30)
    a.update(kw)
    lib = binding.load()
    return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"], a["dk"],
                      a["dv"], a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"],
                      a["block_mask"], a["kv_len"], a["ws"], a["ws_bytes"], None)


def bwd_det(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=1, H=1, N=128, d=64,
             scale=0.125, causal=0, block_mask=None, kv_len=None, ws=P, ws_bytes=1 << 30)
    a.update(kw)
    lib = binding.load()
    return lib.fa_bwd_deterministic(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"],
                                    a["dk"], a["dv"], a["B"], a["H"], a["N"], a["d"], a["scale"],
                                    a["causal"], a["block_mask"], a["kv_len"], a["ws"],
                                    a["ws_bytes"], None)


def fwd_drop(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, N=128, d=64, scale=0.125, causal=0,
             block_mask=None, kv_len=None, p_drop=0.1, seed=1, offset=0)
    a.update(kw)
    lib = binding.load()
    return lib.fa_fwd_dropout(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"],
                              a["d"], a["scale"], a["causal"], a["block_mask"], a["kv_len"],
                              a["p_drop"], a["seed"], a["offset"], None)


def bwd_drop(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=1, H=1, N=128, d=64,
             scale=0.125, causal=0, block_mask=None, kv_len=None, p_drop=0.1, seed=1, offset=0,
             ws=P, ws_bytes=1 << 30)
    a.update(kw)
    lib = binding.load()
    return lib.fa_bwd_dropout(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"],
                              a["dk"], a["dv"], a["B"], a["H"], a["N"], a["d"], a["scale"],
                              a["causal"], a["block_mask"], a["kv_len"], a["p_drop"], a["seed"],
                              a["offset"], a["ws"], a["ws_bytes"], None)


ALL_CALLS = [fwd, bwd, bwd_det, fwd_drop, bwd_drop]
FWD_CALLS = (fwd, fwd_drop)


@pytest.mark.parametrize("call", ALL_CALLS)
def test_shape_errors(call):
    assert call(N=-128) == -3
    assert call(N=-1) == -3
    assert call(B=-1) == -3
    assert call(B=1 << 16, H=1 << 8, N=1 << 8) == -3   # B*H*N >= 2^31
    assert call(d=80) == -4
    assert call(d=192) == -4
    assert call(d=16) == -4


@pytest.mark.parametrize("call", ALL_CALLS)
def test_empty_problems_are_no_ops(call):
    assert call(B=0) == 0
    assert call(H=0) == 0
    assert call(N=0) == 0
    # nothing is dereferenced for an empty problem, not even NULL pointers
    assert call(B=0, q=None, k=None) == 0


@pytest.mark.parametrize("call", ALL_CALLS)
def test_null_and_alignment(call):
    assert call(q=None) == -1
    assert call(o=None) == -1 if call in FWD_CALLS else call(dq=None) == -1
    assert call(k=P + 8) == -2
    assert call(lse=P + 2) == -2
    assert call(kv_len=P + 1) == -2


@pytest.mark.parametrize("call", ALL_CALLS)
def test_scale_errors(call):
    assert call(scale=0.0) == -8
    assert call(scale=-1.0) == -8
    assert call(scale=float("inf")) == -8
    assert call(scale=float("nan")) == -8


@pytest.mark.parametrize("call", [bwd, bwd_det, bwd_drop])
def test_backward_workspace_errors(call):
    assert call(ws=None) == -5
    assert call(ws_bytes=16) == -5
    assert call(ws=P + 16) == -2


def test_traced_variants_need_the_visit_buffer():
    lib = binding.load()
    rc = lib.fa_fwd_traced(P, P, P, P, P, 1, 1, 128, 64, 0.125, 0, None, None, None, None)
    assert rc == -1
    rc = lib.fa_bwd_traced(P, P, P, P, P, P, P, P, P, 1, 1, 128, 64, 0.125, 0, None, None, P,
                           1 << 30, None, None)
    assert rc == -1


def test_backward_phase_number_is_checked():
    lib = binding.load()
    for ph in (-1, 4):
        rc = lib.fa_bwd_phase(ph, P, P, P, P, P, P, P, P, P, 1, 1, 128, 64, 0.125, 0, None, None, P,
                              1 << 30, None)
        assert rc == -8


@pytest.mark.parametrize("call", [fwd_drop, bwd_drop])
def test_dropout_probability_is_checked(call):
    for bad in (-0.1, 1.0, 1.5, float("nan"), float("inf")):
        assert call(p_drop=bad) == -8
    # checked before anything else, even for an empty problem
    assert call(p_drop=1.0, B=0) == -8
    # valid probabilities pass the dropout check and reach the shape checks
    for good in (0.0, 0.1, 0.5, 0.999):
        assert call(p_drop=good, d=80) == -4


def test_selftest_arguments_are_checked():
    lib = binding.load()
    assert lib.fa_selftest_wait_timeout(0, 1000, None, None) == -1
    assert lib.fa_selftest_wait_timeout(0, 1000, P + 2, None) == -2
    assert lib.fa_selftest_wait_timeout(0, 0, P, None) == -8
    assert lib.fa_selftest_wait_timeout(0, 2_000_001, P, None) == -8
    assert lib.fa_selftest_ex2(P, P, -1, 0, None) == -3
    assert lib.fa_selftest_ex2(None, None, 0, 0, None) == 0
    assert lib.fa_selftest_ex2(None, P, 8, 1, None) == -1
    assert lib.fa_selftest_ex2(P + 2, P, 8, 0, None) == -2


def fwd_varlen(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, cu=P, B=2, H=1, max_seqlen=128, T=200, d=64, scale=0.125,
             causal=0, p_drop=0.0)
    a.update(kw)
    return binding.load().fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu"], a["B"],
                                        a["H"], a["max_seqlen"], a["T"], a["d"], a["scale"],
                                        a["causal"], a["p_drop"], 0, 0, None)


def bwd_varlen(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, dout=P, dq=P, dk=P, dv=P, cu=P, B=2, H=1, max_seqlen=128,
             T=200, d=64, scale=0.125, causal=0, p_drop=0.0, ws=P, ws_bytes=1 << 30)
    a.update(kw)
    return binding.load().fa_bwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"],
                                        a["dq"], a["dk"], a["dv"], a["cu"], a["B"], a["H"],
                                        a["max_seqlen"], a["T"], a["d"], a["scale"], a["causal"],
                                        a["p_drop"], 0, 0, a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("call", [fwd_varlen, bwd_varlen])
def test_varlen_argument_checks(call):
    assert call(B=-1) == -3
    assert call(T=-5) == -3
    assert call(max_seqlen=-1) == -3
    assert call(T=300) == -3                   # more tokens than B * max_seqlen
    assert call(d=80) == -4
    assert call(cu=None) == -1
    assert call(cu=P + 2) == -2
    assert call(q=None) == -1
    assert call(k=P + 8) == -2
    assert call(scale=0.0) == -8
    assert call(p_drop=1.0) == -8
    # empty problems do nothing
    assert call(B=0, cu=None) == 0
    assert call(T=0, cu=None) == 0
    assert call(max_seqlen=0, T=0, cu=None) == 0
    assert call(H=0) == 0


def test_varlen_backward_workspace_checks():
    assert bwd_varlen(ws=None) == -5
    assert bwd_varlen(ws_bytes=64) == -5
    assert bwd_varlen(ws=P + 16) == -2


def test_binding_has_every_declared_function():
    # the Python binding carries the C ABI under the same names, each with a wrapper
    declared = set(declared_functions())
    assert set(binding._SIGS) == declared
    for name in declared:
        assert callable(getattr(binding, name)), name


def test_ordered_dq_takes_head_dimensions_64_and_128_only():
    # d = 32 and 96 are accepted by fa_bwd but not by the ordered dQ kernel; the
    # check comes before any launch
    assert bwd_det(d=96) == -4
    assert bwd_det(d=32) == -4
    lib = binding.load()
    rc = lib.fa_bwd_phase(3, P, P, P, P, P, P, P, P, P, 1, 1, 128, 96, 0.125, 0, None, None, P,
                          1 << 30, None)
    assert rc == -4


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "fa.h"

int main(void) {
    /* host-side paths only: no GPU is needed for any of these calls */
    if (fa_version() <= 0) return 1;
    if (strlen(fa_status_string(FA_ERR_SHAPE)) == 0) return 2;
    if (fa_bwd_workspace_size(2, 3, 300, 64) == 0) return 3;
    if (fa_bwd_workspace_size(-1, 3, 300, 64) != 0) return 4;
    /* argument errors come back before any CUDA call */
    if (fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 80, 0.125f, 0, NULL, NULL, NULL)
        != FA_ERR_UNSUPPORTED_D) return 5;
    if (fa_fwd(NULL, NULL, NULL, NULL, NULL, 1, 1, 128, 64, 0.125f, 0, NULL, NULL, NULL)
        != FA_ERR_NULL) return 6;
    if (fa_fwd(NULL, NULL, NULL, NULL, NULL, 0, 1, 128, 64, 0.125f, 0, NULL, NULL, NULL)
        != FA_OK) return 7;
    printf("ok %d\n", fa_version());
    return 0;
}
"""


def test_plain_c_program_links_and_calls_the_library(tmp_path):
    # the boundary is a C ABI: a C99 program with no C++ or Python links against it
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not installed")
    binding.load()  # builds the library if it is missing
    lib_dir = os.path.dirname(binding.library_path())
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src),
                    "-L", lib_dir, "-lfa_b200", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                   check=True, timeout=120)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, (r.returncode, r.stderr)
    assert r.stdout.startswith("ok ")


def test_status_codes_agree_between_header_binding_and_library():
    # every fa_status enumerator of the header: its value, the binding's name for it, and a
    # distinct description from fa_status_string
    text = open(HEADER).read()
    body = re.search(r"typedef enum \{(.*?)\} fa_status;", text, flags=re.S).group(1)
    body = re.sub(r"/\*.*?\*/", "", body, flags=re.S)
    codes = {name: int(val) for name, val in re.findall(r"(FA_[A-Z_]+)\s*=\s*(-?\d+)", body)}
    assert codes["FA_OK"] == 0 and len(codes) == len(set(codes.values()))
    assert {v: k for k, v in codes.items()} == binding.STATUS_NAMES
    texts = [binding.fa_status_string(v) for v in codes.values()]
    assert len(set(texts)) == len(texts) and "unknown status" not in texts


def _c_type(param):
    """ctypes type a C parameter declaration is marshalled as."""
    p = re.sub(r"\bconst\b", "", param).strip()
    if "*" in p:
        return ctypes.c_void_p
    base = " ".join(p.split()[:-1])  # drop the parameter name
    return {"int": ctypes.c_int, "float": ctypes.c_float, "size_t": ctypes.c_size_t,
            "uint64_t": ctypes.c_uint64, "uint32_t": ctypes.c_uint32,
            "unsigned int": ctypes.c_uint}[base]


def test_binding_signatures_match_the_header():
    # a wrong count or kind of argtypes would shift every later argument silently
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    protos = dict(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(([^()]*)\)\s*;", text))
    assert set(protos) == set(binding._SIGS)
    for name, params in protos.items():
        params = [] if params.strip() in ("", "void") else [q.strip() for q in params.split(",")]
        want = [_c_type(q) for q in params]
        got = binding._SIGS[name][1]
        assert len(got) == len(want), name
        for i, (g, w) in enumerate(zip(got, want)):
            assert ctypes.sizeof(g) == ctypes.sizeof(w) and g._type_ == w._type_, (name, i)


def test_binding_return_types_match_the_header():
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    rets = dict((n, r.strip()) for r, n in
                re.findall(r"^\s*((?:const\s+)?[a-z_0-9]+\s*\**)\s*(fa_[a-z_0-9]+)\s*\(", text,
                           flags=re.M))
    kinds = {"int": ctypes.c_int, "size_t": ctypes.c_size_t, "const char*": ctypes.c_char_p}
    assert set(rets) == set(binding._SIGS)
    for name, ret in rets.items():
        assert binding._SIGS[name][0] is kinds[re.sub(r"\s*\*", "*", ret)], name


def test_head_dimension_256_has_no_dropout_or_packed_form():
    lib = binding.load()
    # dropout at d = 256 is refused before any pointer is looked at
    assert lib.fa_fwd_dropout(P, P, P, P, P, 1, 1, 128, 256, 0.0625, 0, None, None, 0.1, 1, 0,
                              None) == -4
    assert lib.fa_bwd_dropout(P, P, P, P, P, P, P, P, P, 1, 1, 128, 256, 0.0625, 0, None, None,
                              0.1, 1, 0, P, 1 << 30, None) == -4
    assert fwd_varlen(d=256) == -4
    assert bwd_varlen(d=256) == -4
    # the plain passes accept it: their next check is the NULL pointer
    assert lib.fa_fwd(None, P, P, P, P, 1, 1, 128, 256, 0.0625, 0, None, None, None) == -1
    # no float32 dQ accumulator at d = 256: -D and -LSE2 (4 bytes each per row, rows
    # padded to 384) and the 256-byte counter only
    assert binding.fa_bwd_workspace_size(1, 1, 300, 256) == 4 * 384 + 4 * 384 + 256
