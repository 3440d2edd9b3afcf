"""Shared helpers for the GPU tests: run the CUDA path through the C ABI and the FP64
oracle on the same seeded inputs, and compare.

Tolerances (stated for BF16 inputs with FP32 accumulation):
  O     max-abs error <= 1e-2
  dQ, dK, dV  relative L2 error <= 1e-2 per tensor
  LSE   max-abs error <= 1e-3 (LSE is FP32 from FP32 row max and sum; the
        only rounding is in the FP32 accumulations and the hardware exp2 /
        log2, each far below 1e-4 for scores of order 10)
"""

import warnings

import numpy as np
import torch

import oracle
from exact_io_aware_63_b200 import binding

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_TOL = 1e-2


def to_dev(x):
    dev = torch.device("cuda", 0)
    bm = None if x.block_mask is None else x.block_mask.to(dev)
    kl = None if x.kv_len is None else x.kv_len.to(dev)
    return (x.q.to(dev), x.k.to(dev), x.v.to(dev), x.dout.to(dev), bm, kl)


def run_gpu(x, backward=True, traced=False):
    q, k, v, do, bm, kl = to_dev(x)
    B, H, N, d = q.shape
    n_t = -(-N // 128)  # ceil: a last, partial tile counts
    out = {}
    vis_f = torch.zeros((B, H, n_t, n_t), dtype=torch.uint8, device=q.device) if traced else None
    o, lse = binding.attention_forward(q, k, v, x.scale, x.causal, bm, kl, visited=vis_f)
    out["o"], out["lse"] = o, lse
    if backward:
        vis_b = torch.zeros_like(vis_f) if traced else None
        dq, dk, dv = binding.attention_backward(q, k, v, o, lse, do, x.scale, x.causal, bm, kl,
                                                visited=vis_b)
        out["dq"], out["dk"], out["dv"] = dq, dk, dv
        out["vis_b"] = vis_b
    out["vis_f"] = vis_f
    torch.cuda.synchronize()
    status = binding.fa_get_device_status()
    assert status == 0, binding.fa_status_string(status)
    return out


def f64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def head_slices(x, heads):
    """Stack the chosen (b, h) heads as a batch of single-head problems."""
    sel = lambda t: np.stack([f64(t[b, h]) for b, h in heads])[:, None]
    kl = None if x.kv_len is None else np.array([int(x.kv_len[b]) for b, _ in heads], np.int32)
    bm = None if x.block_mask is None else x.block_mask.numpy()
    return sel(x.q), sel(x.k), sel(x.v), sel(x.dout), bm, kl


def rel_l2(a, b):
    den = np.linalg.norm(b)
    return np.linalg.norm(a - b) / (den if den > 0 else 1.0)


def compare_forward(o_gpu, lse_gpu, o_ref, lse_ref, where=""):
    o_gpu = np.asarray(o_gpu, np.float64)
    lse_gpu = np.asarray(lse_gpu, np.float64)
    empty = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse_gpu), empty), f"{where}: -inf LSE rows differ"
    assert np.all(o_gpu[empty] == 0.0), f"{where}: rows with no key must be exactly 0"
    err = np.abs(o_gpu - o_ref)
    worst = float(err.max()) if err.size else 0.0
    if worst > O_TOL:
        idx = np.unravel_index(np.argmax(err), err.shape)
        raise AssertionError(f"{where}: O max-abs {worst:.3e} > {O_TOL} at {idx}: "
                             f"gpu {o_gpu[idx]:.6f} ref {o_ref[idx]:.6f}")
    fin = ~empty
    lerr = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert lerr <= LSE_TOL, f"{where}: LSE max-abs {lerr:.3e} > {LSE_TOL}"
    return worst, lerr


BF16_U = 2.0 ** -8   # unit roundoff of bfloat16 (8-bit significand)


def forward_error_bound(x, heads, o_ref):
    """Element-wise bound on |O_gpu - O_ref| from the arithmetic of the kernel: P enters
    the P V product rounded to bfloat16 (relative error <= u each, so the output moves by
    at most u * sum_c P_rc |V_cx|) and O is rounded to bfloat16 once (<= u |O|).
    sum_c P_rc |V_cx| is the oracle's output for values |V|."""
    q, k, v, _, bm, kl = head_slices(x, heads)
    pv_abs, _ = oracle.attention_forward(q, k, np.abs(v), x.scale, x.causal, bm, kl)
    return BF16_U * pv_abs + BF16_U * (1 + BF16_U) * np.abs(o_ref) + 1e-5


class BeyondOTol(UserWarning):
    """Elements of O whose error exceeds O_TOL (allowed only where a test's bound, derived
    from the kernel's bfloat16 roundings, is wider than O_TOL)."""


def bf16_ulp(a):
    """Spacing of bfloat16 values at |a| (8 significand bits: 2^(e - 7) for |a| in
    [2^e, 2^(e+1))); the smallest normal spacing below 2^-126."""
    a = np.maximum(np.abs(np.asarray(a, np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def report_beyond_o_tol(o_gpu, o_ref, where=""):
    """Every element of O whose error exceeds O_TOL, with |O_ref| and the error in bfloat16
    ulps of |O_ref|, issued as a BeyondOTol warning (listed in pytest's warning summary).
    Returns the rows (index, |O_ref|, error, error in ulps)."""
    err = np.abs(np.asarray(o_gpu, np.float64) - o_ref)
    hits = np.argwhere(err > O_TOL)
    rows = []
    for idx in map(tuple, hits):
        e = float(err[idx])
        rows.append((idx, float(abs(o_ref[idx])), e, e / float(bf16_ulp(o_ref[idx]))))
    if rows:
        worst = max(rows, key=lambda r: r[3])
        shown = "; ".join(f"{i} |O_ref| {a:.4f} err {e:.3e} = {u:.2f} ulp"
                          for i, a, e, u in rows[:8])
        warnings.warn(BeyondOTol(
            f"{where}: {len(rows)} of {err.size} O elements above O_TOL {O_TOL}, worst "
            f"{worst[3]:.2f} bf16 ulp of |O_ref| ({worst[2]:.3e} at |O_ref| {worst[1]:.4f}): "
            f"{shown}"))
    return rows


def dq_edge_bound(do_rows, o_gpu, o_ref, pk_abs, dq_ref, scale, v_abs_max):
    """Element-wise bound on |dQ_gpu - dQ_ref| for rows with few keys.  The kernels take
    D_r = sum_x dO_rx O_rx from the bf16 output O (the reading of the D formula), so D_r
    is off by at most dD_r = sum_x |dO_rx| |O_gpu,rx - O_rx|, which moves dQ_r by
    scale * dD_r * sum_c P_rc K_c, at most scale * dD_r * sum_c P_rc |K_cx| (pk_abs: the
    oracle's forward with values |K|).  In a row with few keys and one dominant key
    dP - D nearly cancels and this term dominates.  The roundings of P, dS and dQ to
    bf16 add at most a few bf16 units of the row: 2^-6 of |dQ_ref,x| and of the row's
    root mean square.  D_r and each dP_rc are float32 sums of d products, summed in
    different orders: each within d * 2^-24 of the sum of the products' magnitudes
    (|dO_r| |O_r| for D, at most |dO_r| v_abs_max for dP)."""
    d = do_rows.shape[1]
    dd = np.sum(np.abs(do_rows) * np.abs(o_gpu - o_ref), axis=1, keepdims=True)
    dd += d * 2.0 ** -24 * np.sum(np.abs(do_rows) * (np.abs(o_ref) + v_abs_max), axis=1,
                                  keepdims=True)
    rms = np.sqrt(np.mean(dq_ref ** 2, axis=1, keepdims=True))
    return scale * dd * pk_abs + 2.0 ** -6 * (np.abs(dq_ref) + rms) + 1e-6


def compare_grads(gpu, ref, where=""):
    errs = {}
    for name in ("dq", "dk", "dv"):
        e = rel_l2(np.asarray(gpu[name], np.float64), ref[name])
        errs[name] = e
        assert e <= GRAD_TOL, f"{where}: {name} rel-L2 {e:.3e} > {GRAD_TOL}"
    return errs


def check_all_heads(x, heads=None, backward=True):
    """Full comparison of every output of the chosen heads (default: all heads)."""
    B, H = x.q.shape[:2]
    if heads is None:
        heads = [(b, h) for b in range(B) for h in range(H)]
    out = run_gpu(x, backward=backward)
    q, k, v, do, bm, kl = head_slices(x, heads)
    o_ref, lse_ref = oracle.attention_forward(q, k, v, x.scale, x.causal, bm, kl)
    pick = lambda t: np.stack([f64(t[b, h]) for b, h in heads])[:, None]
    res = {"fwd": compare_forward(pick(out["o"]), pick(out["lse"]), o_ref, lse_ref, "forward")}
    if backward:
        dq, dk, dv, _ = oracle.attention_backward(q, k, v, do, x.scale, x.causal, bm, kl)
        res["bwd"] = compare_grads({n: pick(out[n]) for n in ("dq", "dk", "dv")},
                                   {"dq": dq, "dk": dk, "dv": dv}, "backward")
    return res, out
