"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The layer does not shard: under torchrun every rank runs an independent
replica, the ranks meet at barriers, the reported time is the slowest
rank's and the throughput counts every replica's work.  These checks run
that plumbing with the gloo backend, without a GPU.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local, pg = bench.dist_setup(world, backend="gloo")
    assert (w, r, local) == (world, rank, rank) and pg is not None
    bench.barrier(pg)
    # rank r took (r + 1) ms per step: the job's time is the slowest rank's
    slowest = bench.max_over_ranks(pg, float(rank + 1), device="cpu")
    value = bench.whole_job_tflops(w, 2.0e12, slowest * 10, 10)
    bench.barrier(pg)
    pg.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(f"{slowest} {value}\n")


def test_two_gloo_ranks_take_the_slowest_time_and_sum_the_work(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        slowest, value = map(float, (tmp_path / f"rank{rank}.txt").read_text().split())
        assert slowest == pytest.approx(2.0)               # max over ranks of 1 and 2 ms
        assert value == pytest.approx(2 * 2.0e12 / 2e-3 / 1e12)  # both replicas' FLOPs over 2 ms


def test_single_process_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(None, 3.5) == 3.5
    assert bench.whole_job_tflops(1, 1e12, 10.0, 10) == pytest.approx(1000.0)


def test_reference_arm_prints_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "tiny"])
    assert capsys.readouterr().out == ""


def test_algorithmic_work_of_the_decode_step():
    """Roofline numerators: 21 hit experts of the decode shape stream their
    gate/up ([2*768, 2048]) and down ([2048, 768]) bf16 weights once."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from grouped_gemm_gating_b200 import workloads as W
    cfg = W.CONFIGS["decode"]
    ids = (np.arange(cfg.T * cfg.k, dtype=np.int32) % 21).reshape(cfg.T, cfg.k)   # 21 distinct experts
    a = bench.algorithmic(cfg, ids)
    per_expert = (2 * 768 * 2048 + 2048 * 768) * 2
    assert a["U"] == 21 and a["weight_bytes"] == 21 * per_expert
    assert a["fused_bytes"] == 21 * per_expert + 2 * 3 * 2048 * 2          # + x in, out
    assert a["flops_routed"] == 2 * 3 * 8 * 3 * 2048 * 768                  # 2*T*k*3*d*F (SwiGLU)
    gu, dn = a["gate_up_gemm"][0], a["down_gemm"][0]
    assert gu + dn == a["flops_routed"]


def test_algorithmic_counts_the_shared_expert():
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from grouped_gemm_gating_b200 import workloads as W
    cfg = W.CONFIGS["dsv3"]
    ids = (np.arange(cfg.T * cfg.k, dtype=np.int32) % cfg.E).reshape(cfg.T, cfg.k)
    a = bench.algorithmic(cfg, ids)
    assert a["flops_total"] == a["flops_routed"] + 2 * cfg.T * 3 * cfg.d * cfg.F
    assert a["weight_bytes"] == (cfg.E + 1) * (2 * cfg.F * cfg.d + cfg.d * cfg.F) * 2


def test_roofline_of_a_tensor_bound_kernel_recomputes_against_the_burst_peak():
    """frac = algorithmic FLOPs / per-launch time / burst bf16 peak; the
    sustained fraction beside it; the DRAM traffic ratio from the stored
    ncu figure."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from grouped_gemm_gating_b200 import workloads as W
    cfg = W.CONFIGS["zipf"]
    ids = (np.arange(cfg.T * cfg.k, dtype=np.int32) % 120).reshape(cfg.T, cfg.k)
    alg = bench.algorithmic(cfg, ids)
    peaks = {"hbm_gbs": 6534.8, "bf16_tflops": 1649.5, "bf16_tflops_sustained": 1390.6}
    stages = {"gate_up_gemm": (7.5, 10), "down_gemm": (4.8, 10), "fused_expert": (0.0, 0)}
    r = bench.roofline(cfg, alg, stages, total_ms=13.0, steps=10, launches_per_step=6, rotate=True, peaks=peaks,
                       peak_src="measured")
    fl = alg["gate_up_gemm"][0]
    assert r["bound"] == "tensor" and r["kernel"] == "gate_up_gemm" and r["peak"] == 1649.5
    assert r["per_launch_us"] == pytest.approx(750.0)
    assert r["achieved"] == pytest.approx(fl / 750e-6 / 1e12, rel=1e-4)
    assert r["frac"] == pytest.approx(r["achieved"] / 1649.5, abs=1e-4)
    assert r["frac_of_sustained_peak"] == pytest.approx(r["achieved"] / 1390.6, abs=1e-4)
    assert r["traffic"] == bench.NCU_TRAFFIC[("zipf", "gate_up_gemm")]
    assert r["traffic_vs_algorithmic"] == pytest.approx(r["traffic"] / alg["gate_up_gemm"][1], abs=1e-3)


def test_roofline_of_the_one_kernel_decode_step_is_hbm_bound():
    """The decode step is one kernel: its launch time is the back-to-back
    step time, its numerator the streamed bytes, its denominator the
    measured copy bandwidth (and the nominal 8 TB/s beside it)."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    from grouped_gemm_gating_b200 import workloads as W
    cfg = W.CONFIGS["decode"]
    ids = (np.arange(cfg.T * cfg.k, dtype=np.int32) % 21).reshape(cfg.T, cfg.k)
    alg = bench.algorithmic(cfg, ids)
    peaks = {"hbm_gbs": 6534.8, "bf16_tflops": 1649.5, "bf16_tflops_sustained": 1390.6}
    stages = {"gate_up_gemm": (0.0, 0), "down_gemm": (0.0, 0), "fused_expert": (0.46, 10)}
    r = bench.roofline(cfg, alg, stages, total_ms=0.42, steps=10, launches_per_step=1, rotate=True, peaks=peaks,
                       peak_src="measured")
    assert r["bound"] == "hbm" and r["kernel"] == "fused_expert" and r["peak"] == 6534.8
    assert r["per_launch_us"] == pytest.approx(42.0)
    assert r["achieved"] == pytest.approx(alg["fused_bytes"] / 42e-6 / 1e9, rel=1e-4)
    assert r["frac"] == pytest.approx(r["achieved"] / 6534.8, abs=1e-4)
    assert r["frac_of_nominal_hbm"] == pytest.approx(r["achieved"] / bench.NOMINAL_HBM_GBS, abs=1e-4)
