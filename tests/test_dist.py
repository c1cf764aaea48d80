"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The verify step has no exchange between GPUs: each rank verifies its own batch
of requests (weak scaling) and the ranks only meet in barriers and in the
max-over-ranks reduction of the timed region.  These tests run that logic on two
CPU processes.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from tree_speculative_decoding_kd_b200 import harness as HN
from tree_speculative_decoding_kd_b200 import workload as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    r, w = HN.init_dist("gloo", timeout_s=60)
    cfg = W.scaled(W.CONFIGS["loop"], seed=HN.rank_seed(W.CONFIGS["loop"].seed, r), B=4, H=1)
    st = W.draw_step(cfg, 0, with_nodes=False)
    elapsed = 0.5 + r                                   # rank 1 is the slow one
    HN.barrier()
    tmax = HN.max_over_ranks(elapsed)
    rate = HN.whole_job_rate(100, w, tmax)
    q.put((r, w, tmax, rate, st.parents.tolist(), HN.dist_env()))
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_timing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, w0, t0, rate0, par0, env0), (r1, w1, t1, rate1, par1, env1) = res
    assert (r0, r1, w0, w1) == (0, 1, 2, 2)
    assert t0 == t1 == 1.5                               # every rank sees the slowest time
    assert rate0 == rate1 == pytest.approx(2 * 100 / 1.5)  # all ranks' steps over the max time
    assert par0 != par1                                  # each rank verifies its own requests
    assert env0 == (0, 2, 0) and env1 == (1, 2, 1)


def _dying_worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import time
    import torch.distributed as dist
    HN.init_dist("gloo", timeout_s=5)
    HN.barrier()                                        # both ranks start the run together
    if rank == 1:
        q.put((1, "left"))                              # rank 1 dies between steps
        q.close()
        q.join_thread()                                 # (the message is sent before the exit)
        os._exit(0)
    t0 = time.monotonic()
    try:
        HN.barrier()                                    # the next step's barrier never completes
        q.put((0, "passed"))
    except Exception as e:                              # the short process-group timeout ends it
        q.put((0, f"error after {time.monotonic() - t0:.1f} s: {type(e).__name__}"))
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_a_rank_that_dies_between_steps_ends_the_others_with_an_error():
    """A rank that leaves between steps (no kernel or collective of it in flight): the
    surviving rank's next barrier ends with an error at the process group's short
    timeout instead of waiting for good."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res[1] == "left"
    assert res[0].startswith("error after"), res[0]
    assert float(res[0].split()[2]) < 60.0


def test_single_process_defaults():
    for k in ["RANK", "WORLD_SIZE", "LOCAL_RANK"]:
        os.environ.pop(k, None)
    assert HN.dist_env() == (0, 1, 0)
    assert HN.max_over_ranks(2.5) == 2.5
    assert HN.whole_job_rate(10, 1, 2.0) == 5.0


def test_algorithmic_work_formulas():
    # chain of 3 nodes, L = 10, H = 2: pairs = n*L + sum(depth+1) = 30 + 6
    assert HN.attn_flops([10], [[0, 1, 2]], 2) == 2.0 * 2 * 1088 * 36
    assert HN.attn_bytes([10], 3, 2) == 13 * 1152 + 3 * 2 * (1152 + 1028)
    c = HN.clocks_rejected
    assert c({"reasons": ["hw_slowdown"], "sm_mhz": 1900, "sm_max_mhz": 1965})
    assert not c({"reasons": ["sw_power_cap"], "sm_mhz": 1400, "sm_max_mhz": 1965})
    assert c({"reasons": [], "sm_mhz": 700, "sm_max_mhz": 1965})


def test_flops_equal_visible_pairs_counted_from_the_masks():
    """The roofline's FLOP count is 2 * H * (576 + 512) per visible (node, key) pair:
    every node sees the L committed keys plus the set bits of its ancestor mask."""
    import bench
    import oracle
    rng = np.random.default_rng(5)
    for name in ["tiny", "kimi_single", "batched", "long", "loop"]:
        cfg = W.CONFIGS[name]
        st = W.draw_step(W.scaled(cfg, B=min(cfg.B, 6), H=1), 0, with_nodes=False)
        lens = rng.integers(0, 5000, size=len(st.parents))
        pairs = 0
        for b, p in enumerate(st.parents):
            bits = sum(bin(int(w)).count("1") for w in oracle.visibility_words(p).ravel())
            pairs += len(p) * int(lens[b]) + bits
        depths = [oracle.depths(p) for p in st.parents]
        assert HN.attn_flops(lens, depths, 64) == 2.0 * 64 * (576 + 512) * pairs
        for p, d in zip(st.parents, depths):                 # the bench's own depth walk
            assert list(bench._depths(list(p))) == list(d)
