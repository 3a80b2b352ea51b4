"""Host-side logic of bench.py without a GPU: the reference arm (the CPU
oracle timed on a bounded sample) and the multi-rank aggregation used when
torchrun launches one rank per GPU (weak scaling, max-over-ranks time),
exercised with the gloo backend on two CPU processes."""
import json
import os
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--workload", "tiny"],
                         capture_output=True, text=True, env=env, timeout=300, check=True)
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--workload", "tiny"],
                         capture_output=True, text=True, env=env, timeout=300)
    assert out.returncode == 0 and out.stdout.strip() == ""


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench
    ms = 10.0 + 5.0 * rank                 # the slower rank decides the step time
    t = bench.max_over_ranks(ms)
    v = bench.weak_scaling_value(1e12, world, t)
    q.put((rank, t, v))
    dist.barrier()
    dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in res:
        assert t == pytest.approx(15.0)
        assert v == pytest.approx(2 * 1e12 / 15e-3 / 1e12)


def test_workload_overrides_and_flop_counts():
    """The gradient-mode override, the operator workloads and the algorithmic
    flop count: 8U, 9U with Prob-STE, 7U for exact softmax (one S in the
    forward), 8U for the rounded-exponential baselines (they need the final
    row maximum, so two passes over S)."""
    sys.path.insert(0, ROOT)
    import bench
    from quantized_softmax_attention_b200 import workloads as W
    w = bench.workload("gpt2_fwm", "projection")
    assert w.grad == W.GRAD_PROJECT and w.cal == W.CAL_FWM
    assert bench.config_dict(w, 1)["grad"] == "projection"
    U = bench.gemm_units(w)
    assert bench.algorithmic_flops(w) == 9 * U
    assert bench.algorithmic_flops(bench.workload("gpt2_heavy")) == 8 * U
    assert bench.algorithmic_flops(bench.workload("gpt2_bf16exp")) == 8 * U
    sm = W.Workload(**{**w.__dict__, "operator": 1})
    assert bench.algorithmic_flops(sm) == 7 * U
    assert bench.config_dict(bench.workload("gpt2_fp8exp"), 1)["operator"].endswith("FP8-rounded exp")
    assert bench.workload("gpt2_fixed").cal == W.CAL_FIXED
