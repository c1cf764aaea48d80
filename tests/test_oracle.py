"""Pins of the float64 oracle against things other than itself (CPU only).

* attention: torch's scaled_dot_product_attention (float64, CPU) on the special
  cases the tree mask reduces to -- budget 0 (plain decode), chain tree (causal),
  all-visible bitmask (dense), and arbitrary trees given an explicit boolean
  mask built by transitive closure of the parent relation; lse against
  scipy's logsumexp; closed forms (equal scores); softmax invariants.
* accept: brute-force enumeration of root-to-node paths on small trees; the
  planted path the generator knows; budget 0.
* target argmax: an explicit comparison loop over small rows full of ties, signed
  zeros, infinities and NaNs; hand-written special cases; the token the generator
  planted in each row of full-vocabulary logits.
* tree build: brute-force enumeration of every path of small candidate sets (the
  n - 1 best by score); chain (K = 1), star (D = 1) and all-ties (breadth-first)
  special cases; structural invariants (topological parents, scores as exact float32
  sums along the path, tokens of the right candidates).
* compaction: slot-by-slot expectations, including an overlap where copying in
  the wrong order gives a different cache.
* paged caches: the logical view against an explicit per-slot loop over the page
  table; identity page tables reduce to the contiguous functions; writes land only
  in the request's own pages.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from oracle.accept import target_argmax, tree_accept_batch, tree_accept_logits
from tree_speculative_decoding_kd_b200 import workload as W

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- helpers
def rand_bf16(shape, rng, std=1.0 / 24.0):
    return W.to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * np.float32(std))


def dec(u):
    """Independent bf16 decode for the tests: via torch's bfloat16 dtype."""
    t = torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64)


def closure_mask(parents):
    """anc*(i) by boolean transitive closure of (I + child->parent adjacency)."""
    n = len(parents)
    A = np.eye(n, dtype=bool)
    for i in range(1, n):
        A[i, parents[i]] = True
    R = A.copy()
    for _ in range(n):
        R = (R.astype(np.int64) @ A.astype(np.int64)) > 0
    return R  # R[i, k] = k is an ancestor of i or i itself


def words_from_bool(mask_rows):
    n = mask_rows.shape[1]
    out = np.zeros((mask_rows.shape[0], (n + 31) // 32), np.uint32)
    for i, j in zip(*np.nonzero(mask_rows)):
        out[i, j // 32] |= np.uint32(1 << (j % 32))
    return out


def sdpa_tree(q_abs, q_rope, c_kv, k_rope, L, n, tree_mask, scale):
    """Library attention: query = [q_abs | q_rope], key = [c_kv | k_rope], value = c_kv."""
    q = torch.cat([dec(q_abs), dec(q_rope)], -1)           # [n][H][576]
    k = torch.cat([dec(c_kv[:L + n]), dec(k_rope[:L + n])], -1)  # [L+n][576]
    v = dec(c_kv[:L + n])
    m = torch.ones(n, L + n, dtype=torch.bool)
    m[:, L:] = torch.from_numpy(np.asarray(tree_mask, dtype=bool))
    qh = q.permute(1, 0, 2)                                 # [H][n][576]
    o = torch.nn.functional.scaled_dot_product_attention(
        qh, k.expand(qh.shape[0], -1, -1), v.expand(qh.shape[0], -1, -1),
        attn_mask=m, scale=scale)
    s = scale * (qh @ k.T)                                   # [H][n][L+n]
    s = s.masked_fill(~m, -math.inf).numpy()
    lse = scipy.special.logsumexp(s, axis=-1)                # [H][n]
    return o.permute(1, 0, 2).numpy(), lse.T


def make_case(rng, L, n, H, parents, scale=1.0 / math.sqrt(192)):
    cap = L + n + 3
    c_kv = rand_bf16((1, cap, 512), rng)
    k_rope = rand_bf16((1, cap, 64), rng)
    q_abs = rand_bf16((1, n, H, 512), rng)
    q_rope = rand_bf16((1, n, H, 64), rng)
    return c_kv, k_rope, q_abs, q_rope, scale


# ---------------------------------------------------------------- bf16 decode
def test_bf16_decode_closed_forms():
    bits = np.array([0x3F80, 0xC000, 0x3F81, 0x0000, 0x8000, 0x7F7F, 0x0001], np.uint16)
    want = [1.0, -2.0, 1.0 + 2.0 ** -7, 0.0, -0.0, (2 - 2.0 ** -7) * 2.0 ** 127, 2.0 ** -133]
    got = oracle.bf16_to_f64(bits)
    assert [float(x) for x in got] == want


def test_generator_rounding_is_rne():
    # halfway cases round to even, others to nearest
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -8 + 2.0 ** -20], np.float32)
    assert list(W.to_bf16_bits(x)) == [0x3F80, 0x3F82, 0x3F81]


# ---------------------------------------------------------------- tree
def test_tree_hand_example():
    parents = [-1, 0, 0, 1, 1, 2, 5]
    assert oracle.ancestors(parents, 6) == [6, 5, 2, 0]
    assert list(oracle.depths(parents)) == [0, 1, 1, 2, 2, 2, 3]
    v = oracle.visibility_words(parents)[:, 0]
    assert list(v) == [0b1, 0b11, 0b101, 0b1011, 0b10011, 0b100101, 0b1100101]


@pytest.mark.parametrize("n", [1, 2, 31, 32, 33, 65, 128])
def test_visibility_matches_closure_and_recursion(n):
    rng = np.random.default_rng(n)
    for rule in ["uniform", "depth", "chain", "star"]:
        parents = W.draw_parents(rng, n, rule, 5)
        v = oracle.visibility_words(parents)
        assert v.shape == (n, (n + 31) // 32)
        assert np.array_equal(v, words_from_bool(closure_mask(parents)))
        for i in range(1, n):   # vis[i] = vis[parent[i]] | bit(i)
            want = v[parents[i]].copy()
            want[i // 32] |= np.uint32(1 << (i % 32))
            assert np.array_equal(v[i], want)


def test_check_parents_rejects():
    for bad in [[0, 0], [-1, 1], [-1, 0, 2], [-1, -1], []]:
        with pytest.raises(ValueError):
            oracle.check_parents(bad)


# ---------------------------------------------------------------- attention
def _oracle_one(c_kv, k_rope, q_abs, q_rope, L, vis, scale):
    return oracle.tree_verify_attention(q_abs, q_rope, c_kv, k_rope, np.array([L]),
                                        vis[None], scale)


def test_budget0_is_plain_decode():
    """n = 1: one query over L+1 keys with no mask (pages: budget 0 is plain decode)."""
    rng = np.random.default_rng(0)
    for L in [0, 1, 5, 300]:
        c, r, qa, qr, sc = make_case(rng, L, 1, 16, [-1])
        vis = oracle.visibility_words([-1])
        out, lse = _oracle_one(c, r, qa, qr, L, vis, sc)
        o_ref, l_ref = sdpa_tree(qa[0], qr[0], c[0], r[0], L, 1, np.ones((1, 1)), sc)
        np.testing.assert_allclose(out[0], o_ref, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(lse[0], l_ref, rtol=1e-12, atol=1e-13)


def test_chain_tree_is_causal():
    rng = np.random.default_rng(1)
    n, L = 9, 40
    parents = W.draw_parents(rng, n, "chain", 0)
    c, r, qa, qr, sc = make_case(rng, L, n, 8, parents)
    out, lse = _oracle_one(c, r, qa, qr, L, oracle.visibility_words(parents), sc)
    causal = np.tril(np.ones((n, n), dtype=bool))
    o_ref, l_ref = sdpa_tree(qa[0], qr[0], c[0], r[0], L, n, causal, sc)
    np.testing.assert_allclose(out[0], o_ref, rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(lse[0], l_ref, rtol=1e-12, atol=1e-13)


def test_all_visible_bitmask_is_dense():
    rng = np.random.default_rng(2)
    n, L = 40, 17
    parents = W.draw_parents(rng, n, "uniform", 0)
    c, r, qa, qr, sc = make_case(rng, L, n, 4, parents)
    vis = words_from_bool(np.ones((n, n), dtype=bool))
    out, lse = _oracle_one(c, r, qa, qr, L, vis, sc)
    o_ref, l_ref = sdpa_tree(qa[0], qr[0], c[0], r[0], L, n, np.ones((n, n)), sc)
    np.testing.assert_allclose(out[0], o_ref, rtol=1e-11, atol=1e-15)
    np.testing.assert_allclose(lse[0], l_ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("L,n,rule,scale_mul", [(0, 7, "uniform", 1), (33, 33, "depth", 1),
                                                 (5, 65, "branch", 64), (100, 17, "star", 64)])
def test_tree_mask_matches_library_with_explicit_mask(L, n, rule, scale_mul):
    rng = np.random.default_rng(L + n)
    parents = W.draw_parents(rng, n, rule, 3)
    c, r, qa, qr, sc = make_case(rng, L, n, 8, parents)
    sc *= scale_mul
    out, lse = _oracle_one(c, r, qa, qr, L, oracle.visibility_words(parents), sc)
    o_ref, l_ref = sdpa_tree(qa[0], qr[0], c[0], r[0], L, n, closure_mask(parents), sc)
    np.testing.assert_allclose(out[0], o_ref, rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(lse[0], l_ref, rtol=1e-12, atol=1e-12)


def test_equal_scores_closed_form():
    """q = 0: every visible key scores 0, so out is the mean of visible rows and lse = ln|V|."""
    rng = np.random.default_rng(3)
    n, L = 6, 11
    parents = [-1, 0, 1, 1, 0, 4]
    c, r, qa, qr, sc = make_case(rng, L, n, 2, parents)
    qa[:] = 0
    qr[:] = 0
    out, lse = _oracle_one(c, r, qa, qr, L, oracle.visibility_words(parents), sc)
    K = dec(c[0]).numpy()
    for i in range(n):
        anc = oracle.ancestors(parents, i)
        rows = list(range(L)) + [L + k for k in anc]
        np.testing.assert_allclose(out[0, i, 0], K[rows].mean(0), rtol=1e-13, atol=1e-16)
        assert abs(lse[0, i, 0] - math.log(len(rows))) < 1e-13


def test_softmax_invariants():
    rng = np.random.default_rng(4)
    n, L, H = 12, 64, 4
    parents = W.draw_parents(rng, n, "uniform", 0)
    c, r, qa, qr, sc = make_case(rng, L, n, H, parents)
    sc *= 30
    vis = oracle.visibility_words(parents)
    out, lse = _oracle_one(c, r, qa, qr, L, vis, sc)
    K, R = dec(c[0]).numpy(), dec(r[0]).numpy()
    for i in range(n):
        rows = list(range(L)) + [L + k for k in oracle.ancestors(parents, i)]
        q = np.concatenate([dec(qa[0, i]).numpy(), dec(qr[0, i]).numpy()], -1)
        s = sc * q @ np.concatenate([K[rows], R[rows]], -1).T     # [H][|V|]
        p = np.exp(s - lse[0, i][:, None])
        np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-12)
        assert np.all(lse[0, i] >= s.max(-1) - 1e-12)
        assert np.all(lse[0, i] <= s.max(-1) + math.log(len(rows)) + 1e-12)
        lo, hi = K[rows].min(0), K[rows].max(0)
        assert np.all(out[0, i] >= lo - 1e-15) and np.all(out[0, i] <= hi + 1e-15)


def test_flipped_mask_bit_fails_tolerance_on_peaked_case():
    """A planted mask mistake (one bit) must exceed the parity tolerance on the
    peaked-softmax and tree-only cases the GPU tests use."""
    from tests.tolerances import attn_within_tolerance
    rng = np.random.default_rng(5)
    for L, mul in [(0, 1), (64, 64)]:
        n = 17
        parents = W.draw_parents(rng, n, "depth", 8)
        c, r, qa, qr, sc = make_case(rng, L, n, 16, parents)
        vis = oracle.visibility_words(parents)
        out, lse = _oracle_one(c, r, qa, qr, L, vis, sc * mul)
        leaf = int(np.argmax(oracle.depths(parents)))
        anc = oracle.ancestors(parents, leaf)
        bad = vis.copy()
        k = anc[1]                       # hide the leaf's parent from the leaf
        bad[leaf, k // 32] ^= np.uint32(1 << (k % 32))
        out2, lse2 = _oracle_one(c, r, qa, qr, L, bad, sc * mul)
        ok, _ = attn_within_tolerance(out2, lse2, out, lse)
        assert not ok


def test_nodes_subset_equals_full():
    rng = np.random.default_rng(6)
    n, L = 9, 20
    parents = W.draw_parents(rng, n, "uniform", 0)
    c, r, qa, qr, sc = make_case(rng, L, n, 4, parents)
    vis = oracle.visibility_words(parents)
    full, lf = _oracle_one(c, r, qa, qr, L, vis, sc)
    sub, ls = oracle.tree_verify_attention(qa, qr, c, r, np.array([L]), vis[None], sc,
                                           nodes=[(0, 3), (0, 8)])
    assert np.array_equal(sub[0, 3], full[0, 3]) and np.array_equal(ls[0, 8], lf[0, 8])
    assert np.isnan(sub[0, 0]).all()


# ---------------------------------------------------------------- accept
def brute_accept(tokens, parents, argmax):
    """Deepest node whose whole root path matches the target's predictions."""
    n = len(parents)
    best = [0]
    for v in range(n):
        p = oracle.ancestors(parents, v)[::-1]
        if all(argmax[a] == tokens[b] for a, b in zip(p[:-1], p[1:])) and len(p) > len(best):
            best = p
    return best, len(best), int(argmax[best[-1]])


def test_accept_brute_force_small_trees():
    rng = np.random.default_rng(7)
    for trial in range(1500):
        n = int(rng.integers(1, 11))
        parents = W.draw_parents(rng, n, "branch", 3)
        tokens = W.draw_tokens(rng, parents, vocab=3)
        argmax = rng.integers(0, 3, size=n).astype(np.int32)
        assert oracle.tree_accept(tokens, parents, argmax) == brute_accept(tokens, parents, argmax)


def test_accept_exhaustive_n4():
    """All 6 trees on 4 nodes, all distinct-sibling token labelings and argmaxes over {0,1}."""
    for p1, p2, p3 in itertools.product([0], [0, 1], [0, 1, 2]):
        parents = [-1, p1, p2, p3]
        for tokens in itertools.product(range(2), repeat=4):
            sib = {}
            if any(sib.setdefault(parents[c], set()) & {tokens[c]} or sib[parents[c]].add(tokens[c])
                   for c in range(1, 4)):
                continue
            for am in itertools.product(range(2), repeat=4):
                assert oracle.tree_accept(tokens, parents, am) == brute_accept(tokens, parents, am)


def test_accept_budget0_and_planted_paths():
    assert oracle.tree_accept([5], [-1], [9]) == ([0], 1, 9)
    for name in ["tiny", "kimi_single", "batched", "long"]:
        cfg = W.CONFIGS[name]
        st = W.draw_step(W.scaled(cfg, B=min(cfg.B, 8), H=1), 0, with_nodes=False)
        path, ln, bonus = tree_accept_batch(st.tokens, st.parents, st.argmax)
        for b in range(len(st.planted)):
            assert list(path[b, :ln[b]]) == list(st.planted[b])
            assert bonus[b] == st.argmax[b][st.planted[b][-1]]


def test_accept_duplicate_sibling_tokens_take_the_lowest_index():
    """Worked by hand.  Nodes 1 and 2 are both children of the root and both carry
    token 5, the root's prediction; node 3 (token 7) hangs under node 1 and node 4
    (token 9) under node 2, and the target predicts 7 after node 1 and 9 after node 2.
    The lowest-index reading steps to node 1, then node 3: path [0, 1, 3], bonus 4
    (the prediction after node 3).  Stepping to node 2 would give [0, 2, 4]."""
    parents = [-1, 0, 0, 1, 2]
    tokens = [8, 5, 5, 7, 9]
    argmax = [5, 7, 9, 4, 6]
    assert oracle.tree_accept(tokens, parents, argmax) == ([0, 1, 3], 3, 4)


# ---------------------------------------------------------------- compaction
def test_compaction_overlap_order():
    """path [0,2,3]: slot L+1 takes old L+2 and slot L+2 takes old L+3.  Copying
    in reverse order would leave old L+3 in slot L+1 instead."""
    L, cap = 4, 12
    c = np.arange(cap, dtype=np.uint16).repeat(512).reshape(1, cap, 512)
    r = (100 + np.arange(cap, dtype=np.uint16)).repeat(64).reshape(1, cap, 64)
    path = np.array([[0, 2, 3, -1]])
    c2, r2, lens = oracle.kv_compact(c, r, np.array([L]), path, np.array([3]))
    assert list(c2[0, :, 0]) == [0, 1, 2, 3, 4, 6, 7, 7, 8, 9, 10, 11]
    assert list(r2[0, :, 0] - 100) == [0, 1, 2, 3, 4, 6, 7, 7, 8, 9, 10, 11]
    assert list(lens) == [7]
    assert np.array_equal(c, np.arange(cap, dtype=np.uint16).repeat(512).reshape(1, cap, 512))


def test_compaction_accounting_random():
    rng = np.random.default_rng(8)
    B, n, cap = 5, 17, 80
    c = rand_bf16((B, cap, 512), rng)
    r = rand_bf16((B, cap, 64), rng)
    lens0 = rng.integers(0, cap - n, size=B).astype(np.int32)
    st_paths = np.full((B, n), -1, np.int32)
    ln = np.zeros(B, np.int32)
    for b in range(B):
        parents = W.draw_parents(rng, n, "depth", 8)
        leaf = int(rng.integers(0, n))
        p = oracle.ancestors(parents, leaf)[::-1]
        st_paths[b, :len(p)] = p
        ln[b] = len(p)
    c2, r2, lens = oracle.kv_compact(c, r, lens0, st_paths, ln)
    for b in range(B):
        L = lens0[b]
        assert lens[b] == L + ln[b]
        assert np.array_equal(c2[b, :L], c[b, :L])
        assert np.array_equal(c2[b, L + ln[b]:], c[b, L + ln[b]:])
        for j in range(ln[b]):
            assert np.array_equal(c2[b, L + j], c[b, L + st_paths[b, j]])
            assert np.array_equal(r2[b, L + j], r[b, L + st_paths[b, j]])


def test_budget0_compaction_advances_by_one():
    c = np.zeros((1, 4, 512), np.uint16)
    r = np.zeros((1, 4, 64), np.uint16)
    _, _, lens = oracle.kv_compact(c, r, np.array([2]), np.array([[0]]), np.array([1]))
    assert list(lens) == [3]


def test_write_nodes_slots():
    rng = np.random.default_rng(9)
    c = rand_bf16((2, 30, 512), rng)
    r = rand_bf16((2, 30, 64), rng)
    nc = rand_bf16((2, 5, 512), rng)
    nr = rand_bf16((2, 5, 64), rng)
    c2, r2 = oracle.kv_write_nodes(c, r, np.array([3, 25]), nc, nr)
    assert np.array_equal(c2[0, 3:8], nc[0]) and np.array_equal(r2[1, 25:30], nr[1])
    assert np.array_equal(c2[0, :3], c[0, :3]) and np.array_equal(c2[0, 8:], c[0, 8:])
    with pytest.raises(ValueError):
        oracle.kv_write_nodes(c, r, np.array([3, 26]), nc, nr)


# ---------------------------------------------------------------- whole step
def test_verify_step_tiny_consistent_with_planted():
    wl = W.make_workload("tiny")
    st = wl.step
    res = oracle.verify_step(wl.c_kv, wl.k_rope, wl.cache_lens, st.parents, st.tokens,
                             st.argmax, st.q_abs, st.q_rope, wl.cfg.scale)
    assert list(res["path"][0, :res["len"][0]]) == list(st.planted[0])
    assert res["cache_lens"][0] == wl.cache_lens[0] + len(st.planted[0])
    assert np.isfinite(res["out"]).all() and np.isfinite(res["lse"]).all()


def test_verify_step_attends_over_the_written_node_latents():
    """Whole step with node latents, against a closed form built without the oracle's
    cache functions.  With q = 0 every visible key scores 0, so out[b][i][h] is the mean
    of the rows request b's node i sees -- committed slots [0, L) of the input cache and
    the NODE LATENTS of its ancestors-or-self (written at slots L + k before attention:
    "The Architectural Keystone ...", "The Reasoning That Preceded the Header") -- and
    lse = ln |V|.  Slots at and past L hold garbage that must not be seen."""
    rng = np.random.default_rng(21)
    B, n, H = 2, 6, 2
    lens = np.array([7, 3], np.int32)
    parents = np.array([[-1, 0, 1, 0, 3, 4], [-1, 0, 0, 2, 2, 1]], np.int32)
    cap = int(lens.max()) + n + 4
    c_kv = rand_bf16((B, cap, 512), rng, std=1.0)            # garbage past L as well
    k_rope = rand_bf16((B, cap, 64), rng, std=1.0)
    node_c = rand_bf16((B, n, 512), rng, std=1.0)
    node_r = rand_bf16((B, n, 64), rng, std=1.0)
    zq_a = np.zeros((B, n, H, 512), np.uint16)
    zq_r = np.zeros((B, n, H, 64), np.uint16)
    tokens = np.arange(B * n, dtype=np.int32).reshape(B, n)
    argmax = np.full((B, n), -1, np.int32)
    argmax[0, 0], argmax[0, 3] = tokens[0, 3], tokens[0, 4]  # request 0 accepts 0 -> 3 -> 4
    res = oracle.verify_step(c_kv, k_rope, lens, parents, tokens, argmax, zq_a, zq_r,
                             1.0 / math.sqrt(192), node_ckv=node_c, node_krope=node_r)
    C, NC = dec(c_kv).numpy(), dec(node_c).numpy()
    for b in range(B):
        L = int(lens[b])
        for i in range(n):
            anc, k = [], i
            while k >= 0:                                     # ancestors-or-self by walking up
                anc.append(k)
                k = int(parents[b, k])
            rows = np.concatenate([C[b, :L], NC[b, sorted(anc)]])
            for h in range(H):
                np.testing.assert_allclose(res["out"][b, i, h], rows.mean(0), rtol=1e-12, atol=1e-15)
                assert abs(res["lse"][b, i, h] - math.log(L + len(anc))) < 1e-12
        # node k sits at slot L + k after the write; the accepted path is gathered after it
        assert np.array_equal(res["c_kv_pre"][b, L:L + n], node_c[b])
        assert np.array_equal(res["k_rope_pre"][b, L:L + n], node_r[b])
        m = int(res["len"][b])
        assert np.array_equal(res["c_kv"][b, L:L + m], node_c[b, res["path"][b, :m]])
        assert res["cache_lens"][b] == L + m
    assert list(res["path"][0, :res["len"][0]]) == [0, 3, 4] and res["len"][1] == 1


# ---------------------------------------------------------------- regression record
def test_golden_tiny_regression():
    import json
    import os
    from tests.golden.make_golden import compute
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_oracle.json")) as f:
        g = json.load(f)
    now = compute()
    for k in ["parents", "vis_words", "depths", "accept_path", "accept_len", "bonus"]:
        assert now[k] == g[k], k
    np.testing.assert_allclose(now["lse"], g["lse"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(now["out_node_sums"], g["out_node_sums"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(now["out_00_first8"], g["out_00_first8"], rtol=1e-12, atol=1e-16)


# ---------------------------------------------------------------- target argmax
def _argmax_loop(row):
    """The definition spelled out: scan left to right, keep the first maximum, a NaN beats
    every number and the first NaN is kept (Python's > treats -0.0 and +0.0 as equal)."""
    best_i, best = 0, float(row[0])
    for i in range(1, len(row)):
        if math.isnan(best):
            break
        x = float(row[i])
        if math.isnan(x) or x > best:
            best_i, best = i, x
    return best_i


def test_argmax_matches_comparison_loop():
    vals = np.array([-2.0, -1.0, -0.0, 0.0, 1.0, 2.0, np.inf, -np.inf, np.nan], dtype=np.float32)
    rng = np.random.default_rng(77)
    for _ in range(400):
        V = int(rng.integers(1, 24))
        p = rng.random(len(vals))
        p[-1] *= 0.1                     # NaNs are rarer, so many rows have none
        row = rng.choice(vals, size=V, p=p / p.sum()).astype(np.float32)
        assert int(target_argmax(row)) == _argmax_loop(row), row


@pytest.mark.parametrize("row, want", [
    ([-0.0, 0.0], 0), ([0.0, -0.0], 0), ([1.0, np.nan, np.nan], 1), ([-np.inf, -np.inf], 0),
    ([np.inf, np.nan], 1), ([3.0, 5.0, 5.0, 4.0], 1), ([7.0], 0),
    ([np.float32(1e-45), 0.0], 0), ([-1e-45, -0.0], 1),
])
def test_argmax_special_cases(row, want):
    assert int(target_argmax(np.array(row, dtype=np.float32))) == want


def test_accept_logits_recovers_planted_paths():
    wl = W.make_workload("tiny")
    st = wl.step
    lg = W.draw_logits(wl.cfg, st)
    am, path, ln, bonus = tree_accept_logits(st.tokens, st.parents, lg)
    assert (am == st.argmax).all()
    for b in range(wl.cfg.B):
        assert list(path[b, :ln[b]]) == [int(x) for x in st.planted[b]]
    p2, l2, b2 = tree_accept_batch(st.tokens, st.parents, st.argmax)
    assert (path == p2).all() and (ln == l2).all() and (bonus == b2).all()


# ---------------------------------------------------------------- tree build
from oracle.tree_build import tree_build  # noqa: E402


def _draw_cands(rng, D, K, vocab=1000):
    logp = np.sort(np.log(rng.dirichlet(np.ones(K), size=D)).astype(np.float32), axis=1)[:, ::-1]
    toks = np.stack([rng.choice(vocab, K, replace=False) for _ in range(D)]).astype(np.int32)
    return np.ascontiguousarray(logp), toks


def _check_structure(par, tok, dep, sc, logp, toks, root):
    assert par[0] == -1 and tok[0] == root and dep[0] == 0 and sc[0] == 0
    for i in range(1, len(par)):
        p = par[i]
        assert 0 <= p < i and dep[i] == dep[p] + 1
        j = int(np.nonzero(toks[dep[i] - 1] == tok[i])[0][0])
        assert sc[i] == np.float32(sc[p] + logp[dep[i] - 1, j])      # exact float32 sum
        assert sc[i] <= sc[i - 1] or dep[i] > dep[i - 1]              # pop order


def test_tree_build_matches_brute_force_top_paths():
    rng = np.random.default_rng(9)
    for _ in range(60):
        D, K = int(rng.integers(1, 5)), int(rng.integers(1, 4))
        logp, toks = _draw_cands(rng, D, K)
        total = sum(K ** d for d in range(1, D + 1))
        n = int(rng.integers(1, total + 2))
        # every path (j_1..j_d) with its float32 score summed in path order
        paths = []
        for d in range(1, D + 1):
            for js in itertools.product(range(K), repeat=d):
                s = np.float32(0.0)
                for t, j in enumerate(js):
                    s = np.float32(s + logp[t, j])
                paths.append((s, js))
        paths.sort(key=lambda x: (-float(x[0]), len(x[1]), x[1]))
        want = {js for _, js in paths[: n - 1]}
        par, tok, dep, sc = tree_build(logp, toks, 7, n)
        _check_structure(par, tok, dep, sc, logp, toks, 7)
        got = set()
        for i in range(1, n):
            js, k = [], i
            while k > 0:
                js.append(int(np.nonzero(toks[dep[k] - 1] == tok[k])[0][0]))
                k = par[k]
            got.add(tuple(reversed(js)))
        assert got == want


def test_tree_build_chain_star_and_ties():
    rng = np.random.default_rng(3)
    logp, toks = _draw_cands(rng, 6, 1)                     # K = 1: a chain
    par, tok, dep, _ = tree_build(logp, toks, 5, 7)
    assert list(par) == [-1, 0, 1, 2, 3, 4, 5] and list(dep) == list(range(7))
    logp, toks = _draw_cands(rng, 1, 5)                     # D = 1: a star, best first
    par, tok, dep, _ = tree_build(logp, toks, 5, 6)
    assert list(par) == [-1, 0, 0, 0, 0, 0] and list(tok[1:]) == list(toks[0])
    zero = np.zeros((3, 2), np.float32)                     # all ties: breadth first
    toks = np.arange(6, dtype=np.int32).reshape(3, 2)
    par, tok, dep, _ = tree_build(zero, toks, 9, 8)
    assert list(par) == [-1, 0, 0, 1, 1, 2, 2, 3]
    assert list(tok) == [9, 0, 1, 2, 3, 2, 3, 4]
    with pytest.raises(ValueError):                         # too few candidate nodes
        tree_build(zero[:1, :1], toks[:1, :1], 9, 3)


# ---------------------------------------------------------------- paged caches
from oracle.cache import kv_compact_paged, kv_write_nodes_paged, paged_view  # noqa: E402


def test_paged_view_matches_slot_loop():
    rng = np.random.default_rng(21)
    c = rng.integers(0, 1 << 16, size=(3, 70, 8)).astype(np.uint16)
    r = rng.integers(0, 1 << 16, size=(3, 70, 2)).astype(np.uint16)
    for P in (1, 8, 64):
        cp, rp, pt = W.to_paged(c, r, P, seed=P)
        view = paged_view(cp, pt, P)
        for b in range(3):
            for s_ in range(70):
                assert (view[b, s_] == cp[pt[b, s_ // P] * P + s_ % P]).all()
                assert (view[b, s_] == c[b, s_]).all()


def test_paged_updates_reduce_to_contiguous_and_stay_in_their_pages():
    rng = np.random.default_rng(22)
    B, cap, n, P = 2, 64, 5, 16
    c = rng.integers(0, 1 << 16, size=(B, cap, 8)).astype(np.uint16)
    r = rng.integers(0, 1 << 16, size=(B, cap, 2)).astype(np.uint16)
    lens = np.array([10, 40], np.int32)
    nc = rng.integers(0, 1 << 16, size=(B, n, 8)).astype(np.uint16)
    nr = rng.integers(0, 1 << 16, size=(B, n, 2)).astype(np.uint16)
    path = np.array([[0, 2, 3, -1, -1], [0, 1, -1, -1, -1]], np.int32)
    ln = np.array([3, 2], np.int32)
    # identity table: exactly the contiguous functions
    ident = np.arange(B * cap // P, dtype=np.int32).reshape(B, cap // P)
    wc, wr = kv_write_nodes_paged(c.reshape(-1, 8), r.reshape(-1, 2), ident, P, lens, nc, nr)
    ec, er = oracle.kv_write_nodes(c, r, lens, nc, nr)
    assert (wc.reshape(B, cap, 8) == ec).all() and (wr.reshape(B, cap, 2) == er).all()
    cc, cr, cl = kv_compact_paged(wc, wr, ident, P, lens, path, ln)
    ec2, er2, el = oracle.kv_compact(ec, er, lens, path, ln)
    assert (cc.reshape(B, cap, 8) == ec2).all() and (cl == el).all()
    # shuffled pages: same logical result, spare pages untouched
    cp, rp, pt = W.to_paged(c, r, P, seed=5, spare=4)
    wc, wr = kv_write_nodes_paged(cp, rp, pt, P, lens, nc, nr)
    assert (paged_view(wc, pt, P) == ec).all()
    used = np.zeros(cp.shape[0] // P, bool)
    used[pt.ravel()] = True
    for q in np.nonzero(~used)[0]:
        assert (wc[q * P:(q + 1) * P] == cp[q * P:(q + 1) * P]).all()
