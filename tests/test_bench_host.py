"""Host logic of bench.py, on the CPU: algorithmic bytes, the derived SFU
ceiling, the traffic-figure staleness rule, the reference arm's rank rule,
and the cross-rank aggregation (world size 2 over gloo)."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from selective_state_space_25_b200.synthetic import WORKLOADS  # noqa: E402


def test_algorithmic_bytes():
    # Mamba-130M-shaped scan: read u, delta, z (bf16), B, C (bf16), A, D,
    # dt_bias (fp32); write y (bf16)
    b, L, d, N = 8, 2048, 1536, 16
    exp = 4 * b * L * d * 2 + 2 * b * L * N * 2 + d * N * 4 + 2 * d * 4
    assert bench.alg_bytes(WORKLOADS["mamba130m-scan"]) == exp == 202485760
    # decode: fp32 state read + write dominates
    assert bench.alg_bytes(WORKLOADS["mamba-decode-step"]) > 2 * 256 * 5120 * 16 * 4
    # the conv decode step adds the bf16 window read + write, weight and bias
    b, d, K = 256, 5120, 4
    assert (bench.alg_bytes(WORKLOADS["mamba-decode-conv-step"])
            - bench.alg_bytes(WORKLOADS["mamba-decode-step"])) == 2 * b * d * K * 2 + d * K * 4 + d * 4


def test_sfu_ceiling():
    # N = 16 with the gate: one exp2 per element, softplus and SiLU per (t, d)
    w = WORKLOADS["mamba1.4b-long-scan"]
    assert bench.sfu_ops_per_element(w) == 1 + 2 / 16
    e = bench.sfu_peak_elems_per_s(w)
    assert e == pytest.approx(16 * 148 * 1.965e9 / 1.125)
    # SS2D (N = 1, no gate): softplus and exp2 per (k, t, d)
    assert bench.sfu_ops_per_element(WORKLOADS["vmamba-ss2d"]) == 2.0
    # the long scan's SFU ceiling is below its HBM roofline: the bound the
    # kernel can reach is about a third of the measured copy bandwidth
    t_sfu = w.elements() / e
    t_hbm = bench.alg_bytes(w) / (bench.FALLBACK_HBM_GBS * 1e9)
    assert 0.25 < t_hbm / t_sfu < 0.4


def test_launches_per_step():
    """The gpu_launches claim: one kernel per step, two for the backward that
    runs the states pass first, three for a scan that takes the split scan;
    the split backward adds the adjoint maps and their carry (and its states
    pass may be the split scan's three passes)."""
    W = WORKLOADS
    assert bench.launches_per_step(W["mamba1.4b-long-scan"]) == 1
    assert bench.launches_per_step(W["mamba1.4b-long-scan"], split=True) == 3
    assert bench.launches_per_step(W["vmamba-ss2d"], split=True) == 1
    assert bench.launches_per_step(W["mamba-decode-step"]) == 1
    assert bench.launches_per_step(W["mamba130m-scan-bwd"]) == 2
    assert bench.launches_per_step(W["mamba130m-scan-bwd-saved"]) == 1
    assert bench.launches_per_step(W["mamba130m-scan-bwd-saved"], bwd_split=True) == 3
    assert bench.launches_per_step(W["mamba130m-scan-bwd"], bwd_split=True) == 4
    assert bench.launches_per_step(W["mamba130m-scan-bwd"], split=True, bwd_split=True) == 6
    assert set(bench.STEP_PARTS) == {"scan", "scan_bwd", "scan_bwd_saved"}


def test_split_flags_from_the_library_queries():
    """The named workloads take no split; the saved-state and self-contained
    backward overridden to few channels over a long sequence do (and the
    latter's states pass takes the split scan), which is what a profiling run
    with --override measures."""
    import dataclasses
    from selective_state_space_25_b200 import ssmscan as S
    for w in WORKLOADS.values():
        assert bench.split_flags(S, w) == (False, False), w.name
    few = dict(b=1, L=16384, d_in=256, N=16)
    saved = dataclasses.replace(WORKLOADS["mamba130m-scan-bwd-saved"], dims=few)
    bwd = dataclasses.replace(WORKLOADS["mamba130m-scan-bwd"], dims=few)
    scan = dataclasses.replace(WORKLOADS["mamba130m-scan"], dims=few)
    assert bench.split_flags(S, saved) == (False, True)
    assert bench.split_flags(S, bwd) == (True, True)
    assert bench.split_flags(S, scan) == (True, False)
    assert bench.launches_per_step(saved, *bench.split_flags(S, saved)) == 3
    assert bench.launches_per_step(bwd, *bench.split_flags(S, bwd)) == 6
    assert bench.launches_per_step(scan, *bench.split_flags(S, scan)) == 3


def test_traffic_is_null_when_kernels_changed(tmp_path, monkeypatch):
    f = tmp_path / "traffic.json"
    f.write_text(json.dumps({"w": {"dram_bytes_per_launch": 123, "source_hash": "stale"}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    assert bench.traffic_for("w") is None
    f.write_text(json.dumps({"w": {"dram_bytes_per_launch": 123,
                                   "source_hash": bench.source_hash()}}))
    assert bench.traffic_for("w") == 123
    # per kernel: a workload's figure is tied to its own kernel's sources
    f.write_text(json.dumps({"w": {"dram_bytes_per_launch": 7,
                                   "source_hash": bench.source_hash("ss2d")}}))
    assert bench.traffic_for("w", "ss2d") == 7
    assert bench.traffic_for("w", "scan") is None
    assert bench.source_hash("scan") != bench.source_hash("ss2d")


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    sys.path.insert(0, ROOT)
    import bench as b
    # rank r processed (r + 1) million elements in (10 + 5 r) ms
    q.put((rank, b.aggregate(1e6 * (rank + 1), 10.0 + 5.0 * rank, world)))
    dist.barrier()
    dist.destroy_process_group()


def test_aggregate_sums_elements_and_takes_max_time_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == (3e6, 15.0)
