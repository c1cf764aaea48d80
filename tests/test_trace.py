"""The trace build (libkdverify_trace.so): the same attention with per-CTA timeline
stamps and wait counters, plus the L2 delivery probes.  Its results must equal the
product build's and its timeline must be ordered."""
import numpy as np
import pytest
import torch

from tree_speculative_decoding_kd_b200 import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def traced(kd):
    from tree_speculative_decoding_kd_b200 import build, trace
    build.build_trace()
    product = kd.lib
    lib, ctas, slots = trace._load()            # rebinds kd.lib to the trace build
    yield trace, lib, product, (ctas, slots)
    kd.lib = product


def test_trace_build_matches_product_and_orders_its_timeline(kd, traced):
    trace, lib, product, dims = traced
    wl = W.make_workload("tiny")
    cfg, st = wl.cfg, wl.step
    args = (kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope), kd.bf16_from_bits(wl.c_kv),
            kd.bf16_from_bits(wl.k_rope), torch.from_numpy(wl.cache_lens.astype(np.int32)).cuda())
    vis, _ = kd.kd_tree_build_mask(torch.from_numpy(st.parents).cuda())
    lib.kd_trace_clear(torch.cuda.current_stream().cuda_stream)
    out_t, lse_t = kd.kd_tree_verify_attn(*args, vis, None, cfg.scale)
    torch.cuda.synchronize()
    tr = np.zeros(dims, np.uint64)
    lib.kd_trace_read(tr.ctypes.data, tr.nbytes)
    kd.lib = product                            # the same call through the product build
    try:
        out_p, lse_p = kd.kd_tree_verify_attn(*args, vis, None, cfg.scale)
        torch.cuda.synchronize()
    finally:
        kd.lib = lib
    assert torch.equal(out_t.view(torch.int16), out_p.view(torch.int16))
    assert torch.equal(lse_t, lse_p)
    qk = tr[0].astype(np.int64)                 # the only cluster's QK CTA
    entry, setup, first_s, last_s, exit_ = qk[0], qk[1], qk[10], qk[11], qk[3]
    assert 0 < entry <= setup <= first_s <= last_s <= exit_
    assert qk[35] == 2 and qk[38] == 1          # tiles and units the QK MMA counted


def test_delivery_probe_runs(kd, traced):
    trace, lib, product, dims = traced
    buf = torch.zeros(1024, 512, dtype=torch.bfloat16, device="cuda")
    cycles = torch.zeros(148, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for pair, box_rows, depth in [(0, 256, 4), (2, 128, 8), (1, 256, 4)]:
        cycles.zero_()
        rc = lib.kd_probe_l2_boxes(buf.data_ptr(), 1024, box_rows, depth, 64, pair, cycles.data_ptr(),
                                   err.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert (cycles.cpu().numpy() > 0).all()


def test_store_probe_covers_each_tile(kd, traced):
    trace, lib, product, dims = traced
    ctas = 4
    cycles = torch.zeros(ctas, dtype=torch.int64, device="cuda")
    for mode in (0, 1, 2):
        buf = torch.ones(ctas, 128, 512, dtype=torch.float32, device="cuda")
        rc = lib.kd_probe_store(buf.data_ptr(), ctas, mode, 2, cycles.data_ptr(),
                                torch.cuda.current_stream().cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert (cycles.cpu().numpy() > 0).all()
        assert int(torch.count_nonzero(buf)) == 0       # every element of every CTA's tile written
    assert lib.kd_probe_store(buf.data_ptr(), 149, 0, 1, cycles.data_ptr(), None) != 0


def test_mma_probe_runs(kd, traced):
    trace, lib, product, dims = traced
    cycles = torch.zeros(148, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for m, n, a_tmem, issuers, wait_every in [(128, 64, 0, 1, 0), (128, 256, 1, 1, 0), (128, 128, 1, 2, 0),
                                              (128, 128, 1, 1, 4), (64, 256, 0, 1, 0)]:
        cycles.zero_()
        rc = lib.kd_probe_mma(m, n, a_tmem, issuers, 64, wait_every, cycles.data_ptr(), err.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert (cycles.cpu().numpy() > 0).all()
    assert lib.kd_probe_mma(128, 96, 0, 1, 64, 0, cycles.data_ptr(), err.data_ptr(), None) != 0
    assert lib.kd_probe_mma(128, 256, 1, 2, 64, 0, cycles.data_ptr(), err.data_ptr(), None) != 0
    assert lib.kd_probe_mma(32, 128, 0, 1, 64, 0, cycles.data_ptr(), err.data_ptr(), None) != 0
    assert lib.kd_probe_mma(64, 128, 1, 1, 64, 0, cycles.data_ptr(), err.data_ptr(), None) != 0
