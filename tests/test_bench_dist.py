"""Multi-rank host logic of bench.py on CPU with gloo (world size 2).

The head runs as independent replicas (one per GPU, no collective on its data
path); what several ranks share is the timing protocol: a barrier on both
sides of the timed region and the maximum of the ranks' times.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    w, r, _ = bench.dist_setup(None)
    assert (w, r) == (world, rank) and dist.get_backend() == "gloo"
    bench.barrier(w)
    got = bench.max_over_ranks(10.0 + rank, w)
    bench.dist_teardown(w)
    q.put((rank, got))


def test_max_over_ranks_and_barrier_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    results = dict(q.get(timeout=10) for _ in range(2))
    assert results == {0: 11.0, 1: 11.0}


def _run(cmd, env=None):
    e = dict(os.environ)
    e.update(env or {})
    e.pop("CUDA_VISIBLE_DEVICES", None)
    return subprocess.run(cmd, cwd=ROOT, env=e, capture_output=True, text=True, timeout=600)


def test_reference_arm_one_rank_prints_contract_line():
    r = _run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
              "--shape", "64,64,512"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_two_ranks_rank0_only():
    port = _free_port()
    r = _run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
              "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
              "--gpus", "2", "--steps", "1", "--warmup", "0", "--shape", "64,64,512"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2


def _remeasure_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup(None)
    # rank 0 saw a thermal slowdown, rank 1 only the power cap
    clocks = ({"sm_mhz": 900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_thermal_slowdown"]} if r == 0 else
              {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    got = bench.remeasure_needed(clocks, w)
    bench.dist_teardown(w)
    q.put((rank, got))


def test_remeasure_decision_is_the_same_on_every_rank():
    """A timed region rejected on one rank is measured again on all of them."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_remeasure_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    assert got == {0: True, 1: True}


def test_clock_records_rejected_or_kept():
    sys.path.insert(0, ROOT)
    import bench
    keep = [{"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
            {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []},
            {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}]
    reject = [{"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["hw_slowdown"]},
              {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0, "reasons": ["hw_thermal_slowdown", "sw_power_cap"]},
              {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": ["sw_thermal_slowdown"]},
              {"sm_mhz": 1100.0, "sm_max_mhz": 1965.0, "reasons": []}]   # held low with no reason: a clock lock
    assert not any(bench.clocks_rejected(c) for c in keep)
    assert all(bench.clocks_rejected(c) for c in reject)


def test_timeline_summary_spans():
    """bench.timeline_summary on a made-up record: spans by kind, and the
    critical path W copy -> pass 2 -> what follows it."""
    import bench
    tl = [("copy_host_to_device", 0.0, 1.0)] + \
         [("copy_host_to_device", 1.0 + i, 2.0 + i) for i in range(4)] + \
         [("pass1_logits_lse", 2.0 + i, 2.5 + i) for i in range(4)] + \
         [("combine_lse_loss", 5.5, 5.6)] + \
         [("pass2_grad_dw_dx", 6.0 + i, 7.0 + i) for i in range(3)] + \
         [("copy_device_to_host", 7.0 + i, 7.5 + i) for i in range(3)] + \
         [("copy_device_to_host", 9.5, 10.0)]
    s = bench.timeline_summary(tl)
    assert s["x_y_to_device"] == [0.0, 1.0] and s["w_pieces_to_device"] == [1.0, 5.0]
    assert s["pass1_pieces"] == [2.0, 5.5] and s["pass2_sections"] == [6.0, 9.0]
    assert s["dw_sections_to_host"] == [7.0, 9.5] and s["dx_loss_to_host"] == [9.5, 10.0] and s["end"] == 10.0
    assert s["counts"] == {"w_pieces": 4, "pass1_launches": 4, "pass2_launches": 3}
    assert s["critical_path"] == {"w_copy": 5.0, "w_landed_to_pass2": 1.0, "pass2": 3.0, "after_pass2": 1.0}
