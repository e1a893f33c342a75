"""Host-side logic of bench.py on the CPU: the multi-rank plumbing over gloo
(world size 2), the reference arm's JSON line (the float64 oracle, launched as
the driver launches it), and the workload bookkeeping.  No GPU is used."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        got = bench.max_over_ranks(float(10 * rank + 1), world)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2(tmp_path):
    """Every rank gets the largest per-rank time (the slowest rank's), after a
    barrier, on two gloo processes."""
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    vals = [float(open(tmp_path / f"r{r}.txt").read()) for r in range(2)]
    assert vals == [11.0, 11.0]


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5


def _check_reference_line(d, workload, steps, warmup, world):
    assert d["impl"] == "reference" and d["metric"] == "QLoRA linear fwd+bwd tokens/s"
    assert d["unit"] == "tokens/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["n_gpus"] == world and d["steps"] == steps and d["warmup"] == warmup
    assert d["dtype"] == "f64" and d["vs_baseline"] is None and d["scaling"] == "weak"
    assert d["config"]["workload"] == workload
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_in_process():
    """The reference arm times the oracle on a bounded sample and fills every key
    of the contract."""
    args = bench.argparse.Namespace(workload="linear256_m64_r8", steps=2, warmup=1, gpus=1)
    d = bench.arm_reference(args, 1, 0)
    _check_reference_line(d, "linear256_m64_r8", 2, 1, 1)
    assert bench.arm_reference(args, 2, 1) is None          # only rank 0 runs it


def test_reference_arm_torchrun_world2():
    """Launched as the driver launches N > 1 (torch.distributed.run, 127.0.0.1):
    exactly one JSON line, from rank 0, and every rank exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--workload", "linear256_m64_r8", "--steps", "1", "--warmup", "0"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    p = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, p.stdout
    _check_reference_line(json.loads(lines[0]), "linear256_m64_r8", 1, 0, 2)


def test_workload_defaults_and_bytes(monkeypatch):
    """Per-workload defaults (the Llama-7B stack is the default workload, with
    every row), and the stack's activation bytes counting each shared X once
    (q, k, v share one input, gate and up another)."""
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "attn4096_m4096_r16"])
    a = bench.parse()
    assert (a.steps, a.warmup, a.rows) == (2000, 10, "all")
    monkeypatch.setattr(sys, "argv", ["bench.py"])
    a = bench.parse()
    assert (a.steps, a.warmup, a.rows, a.workload) == (20, 3, "all", "llama7b_stack_m2048_r16")
    assert set(bench.ROW_NAMES) >= {"quantize", "gemv", "mlp_m8192"}
    assert bench.weight_row_shape(bench.WORKLOADS["llama7b_stack_m2048_r16"]) == (4096, 11008)
    wl = bench.WORKLOADS["llama7b_stack_m2048_r16"]
    assert len(wl["shapes"]) == 224
    M = wl["M"]
    unshared = dict(wl)
    unshared.pop("layer")
    # k and v read q's X and up reads gate's: three fewer 4096-wide X reads per layer
    saved = 2 * M * 4096 * (2 + 1) * wl["layers"]
    assert bench.set_bytes(unshared) - bench.set_bytes(wl) == saved


@pytest.mark.parametrize("name", sorted(bench.WORKLOADS))
def test_workload_config_names_the_workload(name):
    c = bench.workload_config(name)
    assert c["workload"] == name and c["M"] == bench.WORKLOADS[name]["M"]


def test_code_hash_ignores_comments_not_code():
    """The traffic record's source hash: comments and whitespace do not change
    it, code (including string literals that contain comment markers) does."""
    a = 'int f(int x) {  // add one\n  return x + 1; /* done */ }\nconst char* s = "a // b";\n'
    b = 'int f(int x) { return x + 1; }\n/* header */ const char* s = "a // b";'
    c = 'int f(int x) { return x + 2; }\nconst char* s = "a // b";'
    assert bench.code_tokens(a) == bench.code_tokens(b)
    assert bench.code_tokens(a) != bench.code_tokens(c)
    assert '"a // b"' in bench.code_tokens(a)


def test_gemm_peak_rule():
    """The headline GEMM's denominator: burst for a short region at full clock,
    sustained once the region is long or the power cap shows in the clock record."""
    pk = {"bf16_tflops": 1648.3, "bf16_tflops_sustained": 1398.5}
    assert bench.gemm_peak(pk, 0.5, []) == (1648.3, False, False)
    assert bench.gemm_peak(pk, 0.5, None) == (1648.3, False, False)
    assert bench.gemm_peak(pk, 1.1, ["sw_power_cap"]) == (1398.5, True, True)
    assert bench.gemm_peak(pk, 2.5, []) == (1398.5, True, False)
    assert bench.gemm_peak(pk, 0.5, ["hw_slowdown"]) == (1648.3, False, False)
