"""GPU parity: every kernel of the verify step against the float64 oracle.

Bit-exact for masks, acceptance, node writes and compaction (whole cache
buffers, untouched slots included); attention within tests/tolerances.py.
Inputs come from the seeded generator; nothing expected comes from the GPU.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from oracle.accept import tree_accept_batch
from tests.tolerances import attn_within_tolerance
from tree_speculative_decoding_kd_b200 import workload as W

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ helpers
def dev_bf16(kd, u16):
    return kd.bf16_from_bits(u16, "cuda")


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def host_u16(kd, t):
    return kd.bits_from_bf16(t)


def vis_for(parents):
    return np.stack([oracle.visibility_words(p) for p in parents])


def run_attn(kd, wl, vis=None, scale=None, kv_splits=0, simt=False, positions=True, c_kv=None,
             k_rope=None):
    st = wl.step
    vis = vis_for(st.parents) if vis is None else vis
    scale = wl.cfg.scale if scale is None else scale
    qa, qr = dev_bf16(kd, st.q_abs), dev_bf16(kd, st.q_rope)
    ck = dev_bf16(kd, wl.c_kv) if c_kv is None else c_kv
    kr = dev_bf16(kd, wl.k_rope) if k_rope is None else k_rope
    lens = dev_i32(wl.cache_lens)
    v = torch.from_numpy(vis.view(np.int32)).cuda()
    pos = None
    if positions:
        depth = np.stack([oracle.depths(p) for p in st.parents])
        pos = dev_i32(wl.cache_lens[:, None] + depth)
    B, n, H = st.q_abs.shape[:3]
    if simt:
        err = kd.new_error_word()
        out, lse = kd.kd_tree_verify_attn_simt(qa, qr, ck, kr, lens, v, pos, scale, dev_error=err)
    else:
        err = kd.new_workspace(B, n, H, wl.cfg.cap if c_kv is None else ck.shape[1], kv_splits)
        out, lse = kd.kd_tree_verify_attn(qa, qr, ck, kr, lens, v, pos, scale, workspace=err,
                                          kv_splits=kv_splits)
    torch.cuda.synchronize()
    bits = kd.kd_read_device_error(err)
    o = kd.bits_from_bf16(out)
    of = (o.astype(np.uint32) << 16).view(np.float32)
    return of, lse.cpu().numpy(), bits


def oracle_attn(wl, vis=None, scale=None, nodes=None):
    st = wl.step
    vis = vis_for(st.parents) if vis is None else vis
    scale = wl.cfg.scale if scale is None else scale
    return oracle.tree_verify_attention(st.q_abs, st.q_rope, wl.c_kv, wl.k_rope, wl.cache_lens,
                                        vis, scale, nodes=nodes)


def assert_attn(out, lse, ref_o, ref_l, tag=""):
    ok, e = attn_within_tolerance(out, lse, ref_o, ref_l)
    assert ok, f"{tag} {e}"
    return e


def small(name, **kw):
    return W.scaled(W.CONFIGS[name], **kw)


# ------------------------------------------------------------------ mask build
@pytest.mark.parametrize("n,rule", [(1, "uniform"), (8, "uniform"), (17, "depth"), (33, "branch"),
                                    (65, "depth"), (128, "uniform"), (128, "chain"), (100, "star")])
def test_build_mask_bitexact(kd, n, rule):
    rng = np.random.default_rng(n)
    parents = np.stack([W.draw_parents(rng, n, rule, 4 if rule == "branch" else 8) for _ in range(6)])
    vis, depth = kd.kd_tree_build_mask(dev_i32(parents))
    torch.cuda.synchronize()
    want = vis_for(parents)
    assert np.array_equal(vis.cpu().numpy().view(np.uint32), want)
    assert np.array_equal(depth.cpu().numpy(), np.stack([oracle.depths(p) for p in parents]))


def test_build_mask_bad_parents(kd):
    parents = np.array([[-1, 0, 1, 2], [-1, 0, 3, 1], [0, -1, 0, 0]], np.int32)
    err = kd.new_error_word()
    vis, _ = kd.kd_tree_build_mask(dev_i32(parents), dev_error=err)
    torch.cuda.synchronize()
    v = vis.cpu().numpy()
    assert np.array_equal(v[0].view(np.uint32), vis_for(parents[:1])[0])
    assert (v[1] == 0).all() and (v[2] == 0).all()
    assert kd.kd_read_device_error(err) & 0x01


# ------------------------------------------------------------------ accept
@pytest.mark.parametrize("name", ["tiny", "kimi_single", "batched", "long", "loop"])
def test_accept_planted_bitexact(kd, name):
    cfg = W.CONFIGS[name]
    st = W.draw_step(W.scaled(cfg, H=1), 0, with_nodes=False)
    path, ln, bonus = kd.kd_tree_accept(dev_i32(st.tokens), dev_i32(st.parents), dev_i32(st.argmax))
    torch.cuda.synchronize()
    rp, rl, rb = tree_accept_batch(st.tokens, st.parents, st.argmax)
    assert np.array_equal(path.cpu().numpy(), rp)
    assert np.array_equal(ln.cpu().numpy(), rl)
    assert np.array_equal(bonus.cpu().numpy(), rb)
    for b in range(cfg.B):
        assert list(rp[b, :rl[b]]) == list(st.planted[b])


def test_accept_small_alphabet_many_matches(kd):
    rng = np.random.default_rng(11)
    B, n = 300, 40
    parents = np.stack([W.draw_parents(rng, n, "branch", 3) for _ in range(B)])
    tokens = np.stack([W.draw_tokens(rng, p, vocab=3) for p in parents])
    argmax = rng.integers(0, 3, size=(B, n)).astype(np.int32)
    path, ln, bonus = kd.kd_tree_accept(dev_i32(tokens), dev_i32(parents), dev_i32(argmax))
    torch.cuda.synchronize()
    rp, rl, rb = tree_accept_batch(tokens, parents, argmax)
    assert np.array_equal(path.cpu().numpy(), rp) and np.array_equal(ln.cpu().numpy(), rl)
    assert np.array_equal(bonus.cpu().numpy(), rb)
    assert rl.max() > 3


def test_accept_duplicate_sibling_tokens(kd):
    """Siblings may carry the same token (a 2-token alphabet, no resampling): the walk
    takes the lowest-index matching child, as the oracle does."""
    rng = np.random.default_rng(13)
    B, n = 200, 70
    parents = np.stack([W.draw_parents(rng, n, "branch", 4) for _ in range(B)])
    tokens = rng.integers(0, 2, size=(B, n)).astype(np.int32)
    argmax = rng.integers(0, 2, size=(B, n)).astype(np.int32)
    path, ln, bonus = kd.kd_tree_accept(dev_i32(tokens), dev_i32(parents), dev_i32(argmax))
    torch.cuda.synchronize()
    rp, rl, rb = tree_accept_batch(tokens, parents, argmax)
    assert np.array_equal(path.cpu().numpy(), rp) and np.array_equal(ln.cpu().numpy(), rl)
    assert np.array_equal(bonus.cpu().numpy(), rb)
    assert rl.max() > 4


def test_accept_budget0_and_max_nodes(kd):
    rng = np.random.default_rng(12)
    for n in [1, 128]:
        parents = np.stack([W.draw_parents(rng, n, "chain", 0) for _ in range(3)])
        tokens = np.stack([W.draw_tokens(rng, p) for p in parents])
        argmax = np.zeros_like(tokens)
        argmax[:, :-1] = tokens[:, 1:]          # every chain fully accepted
        if n > 6:
            argmax[2, 5] = (tokens[2, 6] + 1) % W.VOCAB     # third chain stops after node 5
        path, ln, bonus = kd.kd_tree_accept(dev_i32(tokens), dev_i32(parents), dev_i32(argmax))
        torch.cuda.synchronize()
        rp, rl, rb = tree_accept_batch(tokens, parents, argmax)
        assert np.array_equal(path.cpu().numpy(), rp) and np.array_equal(ln.cpu().numpy(), rl)
        assert np.array_equal(bonus.cpu().numpy(), rb)


# ------------------------------------------------------------------ node write + compaction
def _nan_fill(u16, rows_from):
    """Fill slots from rows_from[b] on with a NaN bit pattern (uninitialised memory)."""
    for b, r in enumerate(rows_from):
        u16[b, r:] = 0x7FC1


def test_write_nodes_and_compact_bitexact(kd):
    cfg = small("loop", B=16, L_lo=0, L_hi=300, steps=1)
    wl = W.make_loop_state(cfg)
    st = wl.step
    _nan_fill(wl.c_kv, wl.cache_lens + cfg.n)
    _nan_fill(wl.k_rope, wl.cache_lens + cfg.n)
    ck, kr = dev_bf16(kd, wl.c_kv), dev_bf16(kd, wl.k_rope)
    lens = dev_i32(wl.cache_lens)
    err = kd.new_error_word()
    kd.kd_kv_write_nodes(ck, kr, lens, dev_bf16(kd, st.node_ckv), dev_bf16(kd, st.node_krope), err)
    rp, rl, _ = tree_accept_batch(st.tokens, st.parents, st.argmax)
    kd.kd_kv_compact(ck, kr, dev_i32(rp), dev_i32(rl), lens, err)
    torch.cuda.synchronize()
    c1, r1 = oracle.kv_write_nodes(wl.c_kv, wl.k_rope, wl.cache_lens, st.node_ckv, st.node_krope)
    c2, r2, l2 = oracle.kv_compact(c1, r1, wl.cache_lens, rp, rl)
    assert kd.kd_read_device_error(err) == 0
    assert np.array_equal(host_u16(kd, ck), c2)
    assert np.array_equal(host_u16(kd, kr), r2)
    assert np.array_equal(lens.cpu().numpy(), l2)


def test_compact_overlapping_path_and_bad_inputs(kd):
    B, n, cap = 4, 8, 40
    rng = np.random.default_rng(13)
    c = rng.integers(0, 0x3F00, size=(B, cap, 512)).astype(np.uint16)
    r = rng.integers(0, 0x3F00, size=(B, cap, 64)).astype(np.uint16)
    L = np.array([4, 10, 31, 0], np.int32)
    path = np.full((B, n), -1, np.int32)
    path[0, :3] = [0, 2, 3]            # overlapping gather
    path[1, :5] = [0, 1, 4, 5, 7]
    path[2, :2] = [0, 9]               # bad entry (>= n)
    path[3, :1] = [0]
    ln = np.array([3, 5, 2, 1], np.int32)
    ck, kr, lens = dev_bf16(kd, c), dev_bf16(kd, r), dev_i32(L)
    err = kd.new_error_word()
    kd.kd_kv_compact(ck, kr, dev_i32(path), dev_i32(ln), lens, err)
    torch.cuda.synchronize()
    keep = [0, 1, 3]
    c2, r2, l2 = oracle.kv_compact(c[keep], r[keep], L[keep], path[keep], ln[keep])
    got_c, got_r, got_l = host_u16(kd, ck), host_u16(kd, kr), lens.cpu().numpy()
    assert np.array_equal(got_c[keep], c2) and np.array_equal(got_r[keep], r2)
    assert np.array_equal(got_l[keep], l2)
    assert np.array_equal(got_c[2], c[2]) and got_l[2] == 31      # bad request untouched
    assert kd.kd_read_device_error(err) & 0x04


def test_cache_overflow_flagged(kd):
    B, n, cap = 2, 8, 20
    c = np.zeros((B, cap, 512), np.uint16)
    r = np.zeros((B, cap, 64), np.uint16)
    ck, kr = dev_bf16(kd, c), dev_bf16(kd, r)
    lens = dev_i32([12, 13])            # 13 + 8 > 20
    nodes_c = dev_bf16(kd, np.full((B, n, 512), 0x3F80, np.uint16))
    nodes_r = dev_bf16(kd, np.full((B, n, 64), 0x3F80, np.uint16))
    err = kd.new_error_word()
    kd.kd_kv_write_nodes(ck, kr, lens, nodes_c, nodes_r, err)
    torch.cuda.synchronize()
    got = host_u16(kd, ck)
    assert (got[0, 12:20] == 0x3F80).all() and (got[1] == 0).all()
    assert kd.kd_read_device_error(err) & 0x02


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("simt", [False, True])
def test_attn_tiny(kd, simt):
    wl = W.make_workload("tiny")
    out, lse, bits = run_attn(kd, wl, simt=simt)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, "tiny")


@pytest.mark.parametrize("simt", [False, True])
def test_attn_kimi_single_full(kd, simt):
    wl = W.make_workload("kimi_single")
    out, lse, bits = run_attn(kd, wl, simt=simt)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, "kimi_single")


def test_attn_batched_recipe_reduced_batch(kd):
    """Config 3's recipe (H 64, n 33, branching <= 4, L ~ U[1024, 8192]) on 4 requests."""
    wl = W.make_workload(small("batched", B=4))
    out, lse, bits = run_attn(kd, wl)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, "batched[4]")


@pytest.mark.parametrize("L_lo,L_hi,n,H", [(0, 0, 8, 16), (1, 1, 1, 16), (127, 129, 17, 64),
                                           (255, 257, 65, 8), (5, 300, 128, 2), (3, 40, 33, 128)])
def test_attn_ragged_and_edge_shapes(kd, L_lo, L_hi, n, H):
    """Tree-only (L = 0), budget 0, tile-boundary lengths, 128 nodes, odd head counts."""
    cfg = W.Config("edge", 3, H, n, L_lo, L_hi, "uniform", 0, 50 + n)
    wl = W.make_workload(cfg)
    out, lse, bits = run_attn(kd, wl)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, f"edge {L_lo}-{L_hi} n{n} H{H}")


def test_a_wait_that_runs_out_reports_and_leaves_the_context_usable(kd):
    """Failure detection without a fault: the first M tile's merge ticket is planted far
    below its partition count, so the CTAs merging that tile wait for partials that never
    complete it.  Their bounded wait gives up after the kernel's 2-second limit, raises
    KD_DEV_TIMEOUT, records where in the control block, and every role leaves; once the
    workspace is cleared, the next call on the same context is correct."""
    cfg = W.Config("timeout", 1, 16, 8, 300, 300, "uniform", 0, 93)   # 308 keys: 2 partitions
    wl = W.make_workload(cfg)
    st = wl.step
    args = (dev_bf16(kd, st.q_abs), dev_bf16(kd, st.q_rope), dev_bf16(kd, wl.c_kv),
            dev_bf16(kd, wl.k_rope), dev_i32(wl.cache_lens))
    vis = torch.from_numpy(vis_for(st.parents).view(np.int32)).cuda()
    ws = kd.new_workspace(1, cfg.n, cfg.H, cfg.cap, 2)
    words = ws.view(torch.int32)
    words[256 // 4] = -1000                     # the first M tile's ticket (after the control block)
    kd.kd_tree_verify_attn(*args, vis, None, cfg.scale, workspace=ws, kv_splits=2)
    torch.cuda.synchronize()
    site = int(words[1].item())
    assert kd.kd_read_device_error(ws) & 0x10, "KD_DEV_TIMEOUT expected"
    assert site & (1 << 31), "the wait that gave up is recorded at byte 4"
    ws.zero_()
    out, lse = kd.kd_tree_verify_attn(*args, vis, None, cfg.scale, workspace=ws, kv_splits=2)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(ws) == 0
    o = kd.bits_from_bf16(out)
    ro, rl = oracle_attn(wl)
    assert_attn((o.astype(np.uint32) << 16).view(np.float32), lse.cpu().numpy(), ro, rl, "after a timeout")


@pytest.mark.parametrize("kv_splits", [0, 2])
def test_attn_more_requests_than_the_longest_first_table(kd, kv_splits):
    """300 requests (more than the kernel's 256-entry longest-first table, so units go in
    request order), each with its own length, some with no committed keys; automatic and
    forced key partitions."""
    cfg = W.Config("many", 300, 2, 2, 0, 300, "uniform", 0, 91)
    wl = W.make_workload(cfg)
    wl.cache_lens[::37] = 0                     # tree-only requests among them
    out, lse, bits = run_attn(kd, wl, kv_splits=kv_splits)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, f"B=300 splits={kv_splits}")


@pytest.mark.parametrize("mul", [16.0, 64.0])
def test_attn_peaked_softmax_with_rescales(kd, mul):
    """Large scale makes the softmax peaked and forces running-max rescales."""
    cfg = W.Config("peaked", 2, 16, 17, 700, 900, "depth", 8, 77)
    wl = W.make_workload(cfg)
    out, lse, bits = run_attn(kd, wl, scale=cfg.scale * mul)
    ro, rl = oracle_attn(wl, scale=cfg.scale * mul)
    assert bits == 0
    assert_attn(out, lse, ro, rl, f"peaked x{mul}")


def test_attn_all_visible_mask(kd):
    cfg = W.Config("dense", 2, 16, 40, 100, 200, "uniform", 0, 78)
    wl = W.make_workload(cfg)
    vis = np.zeros((2, 40, 2), np.uint32)
    vis[:, :, 0] = 0xFFFFFFFF
    vis[:, :, 1] = 0xFF
    out, lse, bits = run_attn(kd, wl, vis=vis, positions=False, scale=cfg.scale * 32)
    ro, rl = oracle_attn(wl, vis=vis, scale=cfg.scale * 32)
    assert_attn(out, lse, ro, rl, "all-visible")


def test_attn_garbage_beyond_tree_is_ignored(kd):
    """Slots past L+n hold NaN bit patterns; the output must not see them."""
    cfg = W.Config("nan", 3, 16, 17, 100, 250, "depth", 8, 79)
    wl = W.make_workload(cfg)
    _nan_fill(wl.c_kv, wl.cache_lens + cfg.n)
    _nan_fill(wl.k_rope, wl.cache_lens + cfg.n)
    out, lse, bits = run_attn(kd, wl)
    ro, rl = oracle_attn(wl)
    assert np.isfinite(out).all()
    assert_attn(out, lse, ro, rl, "nan-beyond")


def test_attn_interleaved_576_layout(kd):
    wl = W.make_workload(small("kimi_single", H=16, L_lo=600, L_hi=600))
    both = np.concatenate([wl.c_kv, wl.k_rope], axis=-1)          # [B][cap][576]
    t = dev_bf16(kd, both)
    out, lse, bits = run_attn(kd, wl, c_kv=t[..., :512], k_rope=t[..., 512:])
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, "interleaved")


@pytest.mark.parametrize("splits", [1, 2, 7, 33])
def test_attn_forced_splits(kd, splits):
    """P9: any split count matches the oracle and the unsplit run."""
    wl = W.make_workload(small("kimi_single", L_lo=4000, L_hi=4000))
    out, lse, bits = run_attn(kd, wl, kv_splits=splits)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, f"splits={splits}")
    o1, l1, _ = run_attn(kd, wl, kv_splits=1)
    np.testing.assert_allclose(lse, l1, rtol=0, atol=2e-5)
    np.testing.assert_allclose(out, o1, rtol=1e-2, atol=1e-5)


def test_attn_error_bits(kd):
    wl = W.make_workload("tiny")
    st = wl.step
    # wrong positions -> BAD_POSITION; output still computed
    depth = oracle.depths(st.parents[0])
    qa, qr = dev_bf16(kd, st.q_abs), dev_bf16(kd, st.q_rope)
    ck, kr = dev_bf16(kd, wl.c_kv), dev_bf16(kd, wl.k_rope)
    v = torch.from_numpy(vis_for(st.parents).view(np.int32)).cuda()
    pos = dev_i32((wl.cache_lens[0] + depth + 1)[None])
    ws = kd.new_workspace(1, 8, 16, wl.cfg.cap)
    kd.kd_tree_verify_attn(qa, qr, ck, kr, dev_i32(wl.cache_lens), v, pos, wl.cfg.scale, workspace=ws)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(ws) & 0x08
    # cache_len + n > cap -> CACHE_FULL, output untouched
    out = torch.full((1, 8, 16, 512), 7.0, dtype=torch.bfloat16, device="cuda")
    lens = dev_i32([wl.cfg.cap - 4])
    kd.kd_tree_verify_attn(qa, qr, ck, kr, lens, v, None, wl.cfg.scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(ws) & 0x02
    assert (out.float() == 7.0).all()


# ------------------------------------------------------------------ the whole step, several times
def test_verify_loop_steps_match_oracle(kd):
    """Config 5's recipe on 8 requests for 4 steps: write nodes, mask, verify,
    accept, compact; caches and lengths bit-exact, attention sampled."""
    cfg = small("loop", B=8, steps=4, L_lo=300, L_hi=1200)
    wl = W.make_loop_state(cfg)
    c_np, r_np, lens_np = wl.c_kv, wl.k_rope, wl.cache_lens.copy()
    ck, kr, lens = dev_bf16(kd, c_np), dev_bf16(kd, r_np), dev_i32(lens_np)
    err = kd.new_error_word()
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cfg.cap)
    for s in range(cfg.steps):
        st = W.draw_step(cfg, s, with_nodes=True)
        kd.kd_kv_write_nodes(ck, kr, lens, dev_bf16(kd, st.node_ckv), dev_bf16(kd, st.node_krope), err)
        vis, depth = kd.kd_tree_build_mask(dev_i32(st.parents), dev_error=err)
        out, lse = kd.kd_tree_verify_attn(dev_bf16(kd, st.q_abs), dev_bf16(kd, st.q_rope), ck, kr,
                                          lens, vis, None, cfg.scale, workspace=ws)
        path, ln, bonus = kd.kd_tree_accept(dev_i32(st.tokens), dev_i32(st.parents),
                                            dev_i32(st.argmax), dev_error=err)
        kd.kd_kv_compact(ck, kr, path, ln, lens, err)
        torch.cuda.synchronize()
        nodes = [(b, i) for b in range(cfg.B) for i in (0, cfg.n - 1)]
        res = oracle.verify_step(c_np, r_np, lens_np, st.parents, st.tokens, st.argmax, st.q_abs,
                                 st.q_rope, cfg.scale, st.node_ckv, st.node_krope, attn_nodes=nodes)
        o = kd.bits_from_bf16(out)
        of = (o.astype(np.uint32) << 16).view(np.float32)
        assert_attn(of, lse.cpu().numpy(), res["out"], res["lse"], f"step {s}")
        assert np.array_equal(path.cpu().numpy(), res["path"])
        assert np.array_equal(bonus.cpu().numpy(), res["bonus"])
        c_np, r_np, lens_np = res["c_kv"], res["k_rope"], res["cache_lens"]
        assert np.array_equal(lens.cpu().numpy(), lens_np)
        assert np.array_equal(host_u16(kd, ck), c_np)
        assert np.array_equal(host_u16(kd, kr), r_np)
    assert kd.kd_read_device_error(err) == 0
    assert kd.kd_read_device_error(ws) == 0


# ------------------------------------------------------------------ full sizes, sampled rows
def _sample_nodes(cfg, rng, per_req=3):
    nodes = []
    for b in range(cfg.B):
        pick = {0, cfg.n - 1, int(rng.integers(1, cfg.n))} if cfg.n > 1 else {0}
        nodes += [(b, i) for i in sorted(pick)][:per_req]
    return nodes


@pytest.mark.parametrize("name", ["batched", "long"])
def test_attn_full_size_sampled(kd, name):
    """Configs 3 and 4 at full size with automatic splitting (the bench's launch
    configuration); the oracle computes three nodes of every request."""
    wl = W.make_workload(name)
    out, lse, bits = run_attn(kd, wl)
    nodes = _sample_nodes(wl.cfg, np.random.default_rng(5))
    ro, rl = oracle_attn(wl, nodes=nodes)
    assert bits == 0
    assert np.isfinite(out).all()
    assert_attn(out, lse, ro, rl, f"{name} full")


def test_causal_extend_chunk_full_size_sampled(kd):
    """Chunked causal extend (a chain tree of 128 nodes) through the verify kernel: 4
    requests over 16384-token caches; the oracle computes three nodes of every request,
    the first and the last included."""
    wl = W.make_workload("extend")
    assert (wl.step.parents[:, 1:] == np.arange(127)).all()
    out, lse, bits = run_attn(kd, wl)
    ro, rl = oracle_attn(wl, nodes=_sample_nodes(wl.cfg, np.random.default_rng(6)))
    assert bits == 0
    assert_attn(out, lse, ro, rl, "extend full")


def test_causal_extend_chunk_small_exact(kd):
    """A ragged 128-token causal chunk over a 300-token cache, every node checked."""
    wl = W.make_workload(small("extend", B=1, H=16, L_lo=300, L_hi=300))
    out, lse, bits = run_attn(kd, wl)
    ro, rl = oracle_attn(wl)
    assert bits == 0
    assert_attn(out, lse, ro, rl, "extend small")


def test_loop_full_size_two_steps(kd):
    """Config 5 exactly (64 requests, cap 18101): two whole steps, caches and
    lengths bit-exact, attention on sampled nodes."""
    cfg = W.CONFIGS["loop"]
    wl = W.make_loop_state(cfg)
    c_np, r_np, lens_np = wl.c_kv, wl.k_rope, wl.cache_lens.copy()
    ck, kr, lens = dev_bf16(kd, c_np), dev_bf16(kd, r_np), dev_i32(lens_np)
    err = kd.new_error_word()
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cfg.cap)
    rng = np.random.default_rng(6)
    for s in range(2):
        st = W.draw_step(cfg, s, with_nodes=True)
        kd.kd_kv_write_nodes(ck, kr, lens, dev_bf16(kd, st.node_ckv), dev_bf16(kd, st.node_krope), err)
        vis, depth = kd.kd_tree_build_mask(dev_i32(st.parents), dev_error=err)
        pos = lens[:, None] + depth
        out, lse = kd.kd_tree_verify_attn(dev_bf16(kd, st.q_abs), dev_bf16(kd, st.q_rope), ck, kr,
                                          lens, vis, pos, cfg.scale, workspace=ws)
        path, ln, bonus = kd.kd_tree_accept(dev_i32(st.tokens), dev_i32(st.parents),
                                            dev_i32(st.argmax), dev_error=err)
        kd.kd_kv_compact(ck, kr, path, ln, lens, err)
        torch.cuda.synchronize()
        res = oracle.verify_step(c_np, r_np, lens_np, st.parents, st.tokens, st.argmax, st.q_abs,
                                 st.q_rope, cfg.scale, st.node_ckv, st.node_krope,
                                 attn_nodes=_sample_nodes(cfg, rng, 2))
        o = kd.bits_from_bf16(out)
        assert_attn((o.astype(np.uint32) << 16).view(np.float32), lse.cpu().numpy(), res["out"],
                    res["lse"], f"loop step {s}")
        assert np.array_equal(path.cpu().numpy(), res["path"])
        assert np.array_equal(ln.cpu().numpy(), res["len"])
        assert np.array_equal(bonus.cpu().numpy(), res["bonus"])
        c_np, r_np, lens_np = res["c_kv"], res["k_rope"], res["cache_lens"]
        assert np.array_equal(lens.cpu().numpy(), lens_np)
        assert np.array_equal(host_u16(kd, ck), c_np)
        assert np.array_equal(host_u16(kd, kr), r_np)
    assert kd.kd_read_device_error(err) == 0 and kd.kd_read_device_error(ws) == 0


@pytest.mark.parametrize("name,kw,splits,mul", [("kimi_single", {}, 0, 1.0), ("batched", {"B": 8}, 0, 1.0),
                                                ("batched", {"B": 3}, 3, 1.0),
                                                ("batched", {"B": 4, "L_lo": 700, "L_hi": 2000}, 2, 32.0)])
def test_attn_repeatable_bits(kd, name, kw, splits, mul):
    """The attention's arithmetic order is fixed (units, tiles, the P hand-over, the
    rescales and the split merge), so repeated calls give the same bits; a race in any
    hand-over between the two CTAs or across clusters would show as a difference."""
    wl = W.make_workload(small(name, **kw) if kw else W.CONFIGS[name])
    scale = wl.cfg.scale * mul
    first = run_attn(kd, wl, kv_splits=splits, scale=scale)
    assert first[2] == 0
    for _ in range(4):
        again = run_attn(kd, wl, kv_splits=splits, scale=scale)
        assert again[2] == 0
        assert np.array_equal(again[0].view(np.uint32), first[0].view(np.uint32))
        assert np.array_equal(again[1].view(np.uint32), first[1].view(np.uint32))
    ro, rl = oracle_attn(wl, scale=scale)
    assert_attn(first[0], first[1], ro, rl, f"{name} x{mul}")
