"""CPU tests of bench.py's host-side helpers (no GPU)."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from exact_io_aware_63_b200 import inputs  # noqa: E402


def _allowed_by_definition(x):
    """Element by element from the mask definition: causal (c <= r), key padding
    (c < kv_len[b]) and the 128 x 128 block mask, combined by AND."""
    B, H, N, d = x.q.shape
    out = torch.zeros((B, N, N), dtype=torch.bool)
    for b in range(B):
        for r in range(N):
            for c in range(N):
                ok = True
                if x.causal and c > r:
                    ok = False
                if x.kv_len is not None and c >= int(x.kv_len[b]):
                    ok = False
                if x.block_mask is not None and not bool(x.block_mask[r // 128, c // 128]):
                    ok = False
                out[b, r, c] = ok
    return out


def test_standard_attention_mask_matches_the_definition():
    x = inputs.make_inputs(2, 1, 256, 64, causal=True, seed=7, key_padding=(100, 256),
                           block_keep=0.5)
    got = bench.standard_allowed(x, torch.device("cpu"))
    want = _allowed_by_definition(x)
    assert torch.equal(got.expand(2, 1, 256, 256)[:, 0], want)


def test_standard_attention_mask_without_masks_is_all_true():
    x = inputs.make_inputs(1, 1, 128, 64, seed=3)
    got = bench.standard_allowed(x, torch.device("cpu"))
    assert bool(got.all())


def _count_allowed(x):
    return int(_allowed_by_definition(x).sum()) * x.q.shape[1]


def test_metric_flops_count_the_allowed_products():
    # 4 d FLOPs per allowed (row, key) pair of every head: causal counts half the
    # matrix (the metric's convention, which includes the diagonal's half), key
    # padding counts its kept keys for every row, block masks their kept tiles
    x = inputs.make_inputs(2, 3, 256, 64, seed=5, key_padding=(100, 256))
    assert bench.flops_fwd(x) == 4.0 * 64 * _count_allowed(x)
    x = inputs.make_inputs(1, 2, 256, 64, seed=6, block_keep=0.5)
    assert bench.flops_fwd(x) == 4.0 * 64 * _count_allowed(x)
    x = inputs.make_inputs(1, 1, 256, 64, causal=True, seed=7)
    assert bench.flops_fwd(x) == 4.0 * 64 * 256 * 256 / 2


def test_packed_batch_flops_are_each_sequence_alone():
    x = inputs.make_inputs(3, 2, 512, 64, seed=8, key_padding=(200, 512))
    lens = bench.packed_lengths(x)
    assert lens == [int(v) for v in x.kv_len]
    assert bench.flops_fwd_packed(x) == sum(4.0 * 2 * 64 * L * L for L in lens)
    # no key padding: every sequence has N tokens, and the packed count is the dense one
    y = inputs.make_inputs(2, 2, 256, 64, seed=9)
    assert bench.packed_lengths(y) == [256, 256]
    assert bench.flops_fwd_packed(y) == bench.flops_fwd(y)


def test_ideal_bytes_follow_the_rows():
    # forward: Q, K, V read and O written once (bf16, 2E each) plus LSE (4R); main
    # backward kernel: Q, K, V, dO read (8E), -LSE2 and -D read (8R), dK and dV
    # written (4E), the float32 dQ accumulator read and written once by its
    # reduce-adds (8E)
    x = inputs.make_inputs(2, 3, 256, 64, seed=10)
    for R in (2 * 3 * 256, 100):
        E = R * 64
        got = bench.ideal_bytes(x) if R == 2 * 3 * 256 else bench.ideal_bytes(x, rows=R)
        assert got == (8 * E + 4 * R, 20 * E + 8 * R)


def test_launches_per_step():
    # forward, preprocess, main and a dQ kernel; d = 256 has two main passes
    for d in (32, 64, 96, 128):
        assert bench.launches_per_step(d) == 4
    assert bench.launches_per_step(256) == 5


def test_oracle_sample_flops_cover_the_workload_when_the_sample_is_everything():
    # the CPU baseline counts a sample's FLOPs as the metric counts the whole workload,
    # pro rata to allowed entries: a sample of every head and row is the whole count
    x = inputs.make_inputs(2, 2, 256, 64, causal=True, seed=11, key_padding=(100, 256))
    _, flops, heads = bench.time_oracle(x, 4, 256, threads=2)
    assert len(heads) == 4
    assert abs(flops - 3.5 * bench.flops_fwd(x)) <= 1e-9 * flops
    # half the heads (both of batch 0): batch 0's share of the allowed entries
    _, half, heads = bench.time_oracle(x, 2, 256, threads=2)
    assert heads == [(0, 0), (0, 1)]
    share = bench.allowed_entries(x, range(256))
    assert abs(half - 3.5 * bench.flops_fwd(x) * share[0] / share.sum()) <= 1e-9 * half


def _bench(*argv, env=None):
    import json
    import subprocess
    e = dict(os.environ)
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        *argv], capture_output=True, text=True, timeout=300, env=e)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


def test_reference_arm_prints_one_contract_line():
    (line,) = _bench("--impl", "reference", "--shape", "1,2,256,64", "--steps", "2",
                     "--warmup", "1")
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["steps"] == 2 and line["warmup"] == 1
    assert line["value"] > 0 and line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert line["config"]["N"] == 256 and line["config"]["H"] == 2
    # the keys naming the workload are the ones the GPU arm's line carries
    ap = type("A", (), {"workload": "long16k_causal", "shape": "1,2,256,64"})()
    x = bench.workload_or_shape(ap)
    want = bench.workload_config(ap, inputs.WORKLOADS["long16k_causal"], x)
    assert {k: line["config"][k] for k in want} == want
    assert want["causal"] is True and want["flop_density"] == bench.density(x)


def test_reference_arm_runs_on_rank_zero_only():
    assert _bench("--impl", "reference", "--shape", "1,1,128,64", "--steps", "1", "--warmup", "1",
                  env={"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_gpu_count_must_match_the_launched_processes():
    import subprocess
    env = dict(os.environ)
    env.update({"WORLD_SIZE": "2", "RANK": "0"})
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        "--gpus", "3", "--steps", "1"], capture_output=True, text=True, timeout=120,
                       env=env)
    assert r.returncode != 0 and "one process per GPU" in r.stderr


def test_gpus_without_a_launcher_start_one_rank_per_gpu():
    # `--gpus 2` run as a plain command starts two ranks itself (torch.distributed.run,
    # rendezvous on 127.0.0.1); the reference arm then runs on rank 0 alone and prints
    # one line for the two-process job
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    import json
    import subprocess
    r = subprocess.run([sys.executable, os.path.join(os.path.dirname(bench.__file__), "bench.py"),
                        "--gpus", "2", "--impl", "reference", "--shape", "1,1,128,64",
                        "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    # bench.py reports ncu DRAM bytes only while the benchmarked kernels' sources hash to
    # the value recorded beside them; any change to those sources turns it into null
    import json
    csrc = tmp_path / "exact_io_aware_63_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.BENCHED_KERNEL_SOURCES:
        (csrc / name).write_text(f"// {name}\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h = bench.kernel_source_hash()
    (tmp_path / "profiles").mkdir()
    rec = {"bert": {"fa_bwd_kernel": {"dram_bytes_per_launch": 123, "source_hash": h}}}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    assert bench.ncu_traffic("fa_bwd_kernel", "bert") == 123
    assert bench.ncu_traffic("fa_fwd_kernel", "bert") is None
    assert bench.ncu_traffic("fa_bwd_kernel", "gpt2") is None
    (csrc / bench.BENCHED_KERNEL_SOURCES[0]).write_text("// changed\n")
    assert bench.kernel_source_hash() != h
    assert bench.ncu_traffic("fa_bwd_kernel", "bert") is None
