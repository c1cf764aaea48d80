"""GPU parity of paged KV caches (page size > 1).  The paged attention must give the
same bits as the contiguous kernel on the same logical caches (same splits); the paged
node write and compaction must match the oracle on the whole page pool, unused pages
included."""
import numpy as np
import pytest
import torch

import oracle
from oracle.accept import tree_accept_batch
from oracle.cache import kv_compact_paged, kv_write_nodes_paged
from tests.tolerances import attn_within_tolerance
from tree_speculative_decoding_kd_b200 import workload as W

pytestmark = pytest.mark.gpu


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def masks(st):
    return torch.from_numpy(np.stack([oracle.visibility_words(p) for p in st.parents]).view(np.int32)).cuda()


def attn_pair(kd, wl, P, splits):
    st = wl.step
    qa, qr = kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope)
    lens, vis = dev_i32(wl.cache_lens), masks(st)
    out_c, lse_c = kd.kd_tree_verify_attn(qa, qr, kd.bf16_from_bits(wl.c_kv), kd.bf16_from_bits(wl.k_rope),
                                          lens, vis, None, wl.cfg.scale, kv_splits=splits)
    cp, rp, pt = W.to_paged(wl.c_kv, wl.k_rope, P, seed=P)
    ws = kd.new_workspace(wl.cfg.B, wl.cfg.n, wl.cfg.H, pt.shape[1] * P, splits)
    out_p, lse_p = kd.kd_tree_verify_attn_paged(qa, qr, kd.bf16_from_bits(cp), kd.bf16_from_bits(rp),
                                                dev_i32(pt), P, lens, vis, None, wl.cfg.scale,
                                                workspace=ws, kv_splits=splits)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(ws) == 0
    return (out_c, lse_c), (out_p, lse_p)


@pytest.mark.parametrize("name,B,P,splits", [("kimi_single", None, 64, 1), ("kimi_single", None, 128, 3),
                                             ("kimi_single", None, 256, 1), ("batched", 4, 64, 1),
                                             ("batched", 4, 128, 3), ("tiny", None, 64, 1)])
def test_paged_attention_matches_contiguous_bits(kd, name, B, P, splits):
    cfg = W.CONFIGS[name] if B is None else W.scaled(W.CONFIGS[name], B=B)
    wl = W.make_workload(cfg)
    (oc, lc), (op, lp) = attn_pair(kd, wl, P, splits)
    assert torch.equal(oc.view(torch.int16), op.view(torch.int16))
    assert torch.equal(lc, lp)
    if name == "tiny":                                     # and against the oracle
        ro, rl = oracle.tree_verify_attention(wl.step.q_abs, wl.step.q_rope, wl.c_kv, wl.k_rope,
                                              wl.cache_lens,
                                              np.stack([oracle.visibility_words(p) for p in wl.step.parents]),
                                              wl.cfg.scale)
        o = (kd.bits_from_bf16(op).astype(np.uint32) << 16).view(np.float32)
        ok, e = attn_within_tolerance(o, lp.cpu().numpy(), ro, rl)
        assert ok, e


@pytest.mark.parametrize("name,B,P,splits", [("kimi_single", None, 128, 3), ("batched", 4, 256, 1),
                                             ("batched", 3, 64, 2)])
def test_paged_attention_matches_oracle(kd, name, B, P, splits):
    """The paged attention against the oracle run on the logical view of the page pool
    (not through the contiguous kernel): multi-tile requests, split partitions merged
    in the launch, page sizes below, at and above the 128-key tile."""
    cfg = W.CONFIGS[name] if B is None else W.scaled(W.CONFIGS[name], B=B)
    wl = W.make_workload(cfg)
    st = wl.step
    cp, rp, pt = W.to_paged(wl.c_kv, wl.k_rope, P, seed=P + 1)
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, pt.shape[1] * P, splits)
    out, lse = kd.kd_tree_verify_attn_paged(kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope),
                                            kd.bf16_from_bits(cp), kd.bf16_from_bits(rp), dev_i32(pt), P,
                                            dev_i32(wl.cache_lens), masks(st), None, cfg.scale,
                                            workspace=ws, kv_splits=splits)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(ws) == 0
    vis = np.stack([oracle.visibility_words(p) for p in st.parents])
    ro, rl = oracle.tree_verify_attention(st.q_abs, st.q_rope, oracle.cache.paged_view(cp, pt, P),
                                          oracle.cache.paged_view(rp, pt, P), wl.cache_lens, vis, cfg.scale)
    o = (kd.bits_from_bf16(out).astype(np.uint32) << 16).view(np.float32)
    ok, e = attn_within_tolerance(o, lse.cpu().numpy(), ro, rl)
    assert ok, e


@pytest.mark.parametrize("splits", [1, 2])
def test_paged_attention_bad_page_is_flagged_and_skipped(kd, splits):
    """A page id outside the pool among the pages a request reads: KD_DEV_BAD_PAGE,
    that request's outputs are left as they were, the other request is unaffected."""
    wl = W.make_workload(W.scaled(W.CONFIGS["tiny"], B=2, L_lo=600, L_hi=700))
    st, cfg = wl.step, wl.cfg
    P = 64
    cp, rp, pt = W.to_paged(wl.c_kv, wl.k_rope, P, seed=5)
    bad = pt.copy()
    bad[1, 3] = cp.shape[0] // P + 11                                 # a committed page of request 1
    out = torch.full((cfg.B, cfg.n, cfg.H, 512), 3.0, dtype=torch.bfloat16, device="cuda")
    lse = torch.full((cfg.B, cfg.n, cfg.H), 5.0, dtype=torch.float32, device="cuda")
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, pt.shape[1] * P, splits)
    kd.kd_tree_verify_attn_paged(kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope),
                                 kd.bf16_from_bits(cp), kd.bf16_from_bits(rp), dev_i32(bad), P,
                                 dev_i32(wl.cache_lens), masks(st), None, cfg.scale, out=out, lse=lse,
                                 workspace=ws, kv_splits=splits)
    torch.cuda.synchronize()
    assert "BAD_PAGE" in kd.decode_device_error(kd.kd_read_device_error(ws))
    assert (out[1].float() == 3.0).all() and (lse[1] == 5.0).all()
    vis = np.stack([oracle.visibility_words(p) for p in st.parents])
    ro, rl = oracle.tree_verify_attention(st.q_abs[:1], st.q_rope[:1], wl.c_kv[:1], wl.k_rope[:1],
                                          wl.cache_lens[:1], vis[:1], cfg.scale)
    o = (kd.bits_from_bf16(out[:1]).astype(np.uint32) << 16).view(np.float32)
    ok, e = attn_within_tolerance(o, lse[:1].cpu().numpy(), ro, rl)
    assert ok, e


@pytest.mark.parametrize("P", [1, 16, 64])
def test_paged_write_and_compact_bitexact(kd, P):
    wl = W.make_workload(W.scaled(W.CONFIGS["kimi_single"], B=3, L_lo=100, L_hi=300))
    st, cfg = wl.step, wl.cfg
    rng = np.random.default_rng(P)
    nc = W.to_bf16_bits(rng.standard_normal((cfg.B, cfg.n, 512)).astype(np.float32))
    nr = W.to_bf16_bits(rng.standard_normal((cfg.B, cfg.n, 64)).astype(np.float32))
    cp, rp, pt = W.to_paged(wl.c_kv, wl.k_rope, P, seed=11, spare=5)
    path, ln, _ = tree_accept_batch(st.tokens, st.parents, st.argmax)
    want_c, want_r = kv_write_nodes_paged(cp, rp, pt, P, wl.cache_lens, nc, nr)
    want_c, want_r, want_l = kv_compact_paged(want_c, want_r, pt, P, wl.cache_lens, path, ln)

    gc, gr = kd.bf16_from_bits(cp), kd.bf16_from_bits(rp)
    lens, ptab, err = dev_i32(wl.cache_lens), dev_i32(pt), kd.new_error_word()
    kd.kd_kv_write_nodes_paged(gc, gr, ptab, P, lens, kd.bf16_from_bits(nc), kd.bf16_from_bits(nr), err)
    kd.kd_kv_compact_paged(gc, gr, ptab, P, dev_i32(path), dev_i32(ln), lens, err)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(err) == 0
    assert np.array_equal(kd.bits_from_bf16(gc), want_c)
    assert np.array_equal(kd.bits_from_bf16(gr), want_r)
    assert np.array_equal(lens.cpu().numpy(), want_l)


def test_paged_bad_page_is_flagged_and_skipped(kd):
    wl = W.make_workload(W.scaled(W.CONFIGS["tiny"], B=2))
    cp, rp, pt = W.to_paged(wl.c_kv, wl.k_rope, 64, seed=3)
    bad = pt.copy()
    bad[1, wl.cache_lens[1] // 64] = cp.shape[0] // 64 + 7          # outside the pool
    gc, gr = kd.bf16_from_bits(cp), kd.bf16_from_bits(rp)
    err = kd.new_error_word()
    node = kd.bf16_from_bits(np.zeros((2, wl.cfg.n, 512), np.uint16))
    noder = kd.bf16_from_bits(np.zeros((2, wl.cfg.n, 64), np.uint16))
    kd.kd_kv_write_nodes_paged(gc, gr, dev_i32(bad), 64, dev_i32(wl.cache_lens), node, noder, err)
    torch.cuda.synchronize()
    assert "BAD_PAGE" in kd.decode_device_error(kd.kd_read_device_error(err))
    view_after = oracle.cache.paged_view(kd.bits_from_bf16(gc), pt, 64)
    assert np.array_equal(view_after[1], oracle.cache.paged_view(cp, pt, 64)[1])   # request 1 untouched
