"""Planted single mistakes in the oracle, for the pin-strength test (CPU, test
infrastructure only).

Each entry below is one plausible mistake: a dropped term, a wrong index or slot
offset, an off-by-one length, a wrong tie order, a write before a read.  (Compaction
copied in place in ascending order is not among them: a path node at depth j has
index >= j, so no write lands on a row a later copy still reads; the hazard is the
descending or the parallel copy, and the descending one is planted.)  ``apply(name)``
replaces one oracle function, in every ``oracle`` module that holds it, with a copy
that carries that mistake.  ``tests/test_oracle_mutants.py`` then runs the oracle's
pins (``tests/test_oracle.py``) and requires at least one of them to fail.

The copies restate the oracle's definitions with the one change marked ``# MUTANT``;
nothing here is used outside that test.
"""
import math
import sys

import numpy as np

import oracle
import oracle.accept as acc
import oracle.attention as att
import oracle.cache as cache
import oracle.step  # noqa: F401  (holds imported copies that must be replaced too)
import oracle.tree as tree
import oracle.tree_build as tb


def _replace(orig, new):
    """Rebind every name in the loaded oracle modules that refers to ``orig``."""
    for mname, mod in list(sys.modules.items()):
        if mname == "oracle" or mname.startswith("oracle."):
            for k, v in list(vars(mod).items()):
                if v is orig:
                    setattr(mod, k, new)


# ---------------------------------------------------------------- attention
def _attention(bug):
    def fn(q_abs, q_rope, c_kv, k_rope, cache_lens, vis, scale, nodes=None):
        B, n, H, dc = q_abs.shape
        out = np.full((B, n, H, dc), np.nan)
        lse = np.full((B, n, H), np.nan)
        if nodes is None:
            nodes = [(b, i) for b in range(B) for i in range(n)]
        for b, i in nodes:
            L = int(cache_lens[b])
            if L + n > c_kv.shape[1]:
                raise ValueError("cache_len + n exceeds the slot capacity")
            K = att.bf16_to_f64(c_kv[b, :L + n])
            R = att.bf16_to_f64(k_rope[b, :L + n])
            m = np.ones(L + n, dtype=bool)
            for k in range(n):
                bit = k % 32
                if bug == "tree_bits_reversed":
                    bit = 31 - bit                                   # MUTANT
                m[L + k] = bool((int(vis[b, i][k // 32]) >> bit) & 1)
            if bug == "no_self":
                m[L + i] = False                                     # MUTANT
            if bug == "cache_short" and L > 0:
                m[L - 1] = False                                     # MUTANT
            if bug == "tree_ignores_mask":
                m[L:] = True                                         # MUTANT
            Kv, Rv = K[m], R[m]
            qa = att.bf16_to_f64(q_abs[b, i])
            qr = att.bf16_to_f64(q_rope[b, i])
            if bug == "heads_mismatch":
                qr = qr[::-1]                                        # MUTANT
            if bug == "no_rope":
                s = scale * (qa @ Kv.T)                              # MUTANT
            elif bug == "scale_abs_only":
                s = scale * (qa @ Kv.T) + qr @ Rv.T                  # MUTANT
            else:
                s = scale * (qa @ Kv.T + qr @ Rv.T)
            smax = s.max(axis=1, keepdims=True)
            e = np.exp(s - smax)
            l = e.sum(axis=1, keepdims=True)
            out[b, i] = (e @ Kv) if bug == "out_unnormalized" else (e @ Kv) / l   # MUTANT (one arm)
            if bug == "lse_no_max":
                lse[b, i] = np.log(l)[:, 0]                          # MUTANT
            elif bug == "lse_log2":
                lse[b, i] = ((smax + np.log(l)) / math.log(2.0))[:, 0]   # MUTANT
            else:
                lse[b, i] = (smax + np.log(l))[:, 0]
        return out, lse
    return lambda: _replace(att.tree_verify_attention, fn)


def _bf16_as_fp16():
    def fn(u):
        return np.asarray(u, dtype=np.uint16).view(np.float16).astype(np.float64)   # MUTANT
    return _replace(att.bf16_to_f64, fn)


# ---------------------------------------------------------------- tree
def _depth_counts_nodes():
    def fn(parents):
        return np.array([len(tree.ancestors(parents, i)) for i in range(len(parents))],  # MUTANT
                        dtype=np.int32)
    _replace(tree.depths, fn)


def _mask(bug):
    def fn(parents):
        tree.check_parents(parents)
        n = len(parents)
        W = tree.n_words(n)
        out = np.zeros((n, W), dtype=np.uint32)
        for i in range(n):
            ks = tree.ancestors(parents, i)
            if bug == "parent_only":
                ks = ks[:2]                                          # MUTANT
            if bug == "no_self":
                ks = ks[1:]                                          # MUTANT
            for k in ks:
                w = k % W if bug == "word_mod" else k // 32          # MUTANT (one arm)
                out[i, w] |= np.uint32(1) << np.uint32(k % 32)
        return out
    return lambda: _replace(tree.visibility_words, fn)


# ---------------------------------------------------------------- accept
def _accept(bug):
    def fn(node_tokens, parents, target_argmax):
        n = len(parents)
        path = [0]
        cur = 0
        while len(path) < n:
            nxt = -1
            for c in range(n):
                is_child = int(parents[c]) == cur or bug == "any_node"          # MUTANT (one arm)
                want = int(target_argmax[c if bug == "child_index" else cur])   # MUTANT (one arm)
                if c not in path and is_child and int(node_tokens[c]) == want:
                    nxt = c
                    if bug != "last_duplicate":                                 # MUTANT (one arm)
                        break
            if nxt < 0:
                break
            path.append(nxt)
            cur = nxt
        bonus = int(target_argmax[cur])
        if bug == "bonus_parent" and len(path) > 1:
            bonus = int(target_argmax[path[-2]])                     # MUTANT
        if bug == "path_without_root":
            path = path[1:]                                          # MUTANT
        return path, len(path), bonus
    return lambda: _replace(acc.tree_accept, fn)


def _argmax(bug):
    def fn(logits):
        x = np.asarray(logits)
        if bug == "last_tie":
            r = x.shape[-1] - 1 - np.argmax(x[..., ::-1], axis=-1)   # MUTANT
        else:
            r = np.nanargmax(np.where(np.isnan(x), -np.inf, x), axis=-1)   # MUTANT (NaN ignored)
        return np.asarray(r).astype(np.int32)
    return lambda: _replace(acc.target_argmax, fn)


# ---------------------------------------------------------------- caches
def _write_slot_shift():
    def fn(c_kv, k_rope, cache_lens, node_ckv, node_krope):
        c_kv, k_rope = c_kv.copy(), k_rope.copy()
        B, n = node_ckv.shape[:2]
        for b in range(B):
            L = int(cache_lens[b])
            for k in range(n):
                if L + k + 1 < c_kv.shape[1]:
                    c_kv[b, L + k + 1] = node_ckv[b, k]              # MUTANT
                    k_rope[b, L + k + 1] = node_krope[b, k]
        return c_kv, k_rope
    _replace(cache.kv_write_nodes, fn)


def _compact(bug):
    def fn(c_kv, k_rope, cache_lens, path, lens):
        c_kv, k_rope = c_kv.copy(), k_rope.copy()
        new_lens = np.array(cache_lens, dtype=np.int32).copy()
        for b in range(c_kv.shape[0]):
            L, m = int(cache_lens[b]), int(lens[b])
            base = 0 if bug == "src_no_offset" else L                # MUTANT (one arm)
            if bug == "in_place_reversed":
                for j in reversed(range(m)):                         # MUTANT: no staging, last first
                    c_kv[b, L + j] = c_kv[b, base + int(path[b][j])]
                    k_rope[b, L + j] = k_rope[b, base + int(path[b][j])]
            else:
                rc = [c_kv[b, base + int(path[b][j])].copy() for j in range(m)]
                rr = [k_rope[b, base + int(path[b][j])].copy() for j in range(m)]
                for j in range(m):
                    c_kv[b, L + j] = rc[j]
                    k_rope[b, L + j] = rr[j]
            new_lens[b] = L + m - (1 if bug == "len_minus_one" else 0)   # MUTANT (one arm)
        return c_kv, k_rope, new_lens
    return lambda: _replace(cache.kv_compact, fn)


def _paged_no_scale():
    def fn(pages, page_table, page_size):
        pt = np.asarray(page_table, dtype=np.int64)
        B, M = pt.shape
        rows = (pt[:, :, None] + np.arange(page_size)[None, None, :]).reshape(B, M * page_size)  # MUTANT
        return pages[np.minimum(rows, pages.shape[0] - 1)]
    _replace(cache.paged_view, fn)


def _writeback_identity():
    def fn(pages, page_table, page_size, logical):
        out = pages.copy()
        pt = np.asarray(page_table, dtype=np.int64)
        for b in range(pt.shape[0]):
            for q in range(pt.shape[1]):
                dst = b * pt.shape[1] + q                            # MUTANT: table not used
                if (dst + 1) * page_size <= out.shape[0]:
                    out[dst * page_size:(dst + 1) * page_size] = logical[b, q * page_size:(q + 1) * page_size]
        return out
    _replace(cache._write_back, fn)


# ---------------------------------------------------------------- tree build
def _build(bug):
    def fn(logp, cand_tokens, root_token, n):
        logp = np.asarray(logp, dtype=np.float32)
        D, K = logp.shape
        parents, tokens, depth, score = [-1], [int(root_token)], [0], [np.float32(0.0)]
        frontier = []
        if D >= 1 and n > 1:
            frontier.append((np.float32(logp[0, 0]), 1, 0, 0))

        def key(e):
            s, d, p, j = e
            return (float(s), d if bug == "tie_deeper_first" else -d, -p, -j)   # MUTANT (one arm)

        while len(parents) < n and frontier:
            best = max(range(len(frontier)), key=lambda i: key(frontier[i]))
            s, d, p, j = frontier.pop(best)
            me = len(parents)
            parents.append(p)
            tokens.append(int(cand_tokens[d - 1][j]))
            depth.append(d)
            score.append(s)
            if j + 1 < K and bug != "no_sibling":                    # MUTANT (one arm)
                base = s if bug == "sibling_own_score" else score[p]     # MUTANT (one arm)
                frontier.append((np.float32(base + logp[d - 1, j + 1]), d, p, j + 1))
            if d < D:
                row = d - 1 if bug == "child_same_row" else d       # MUTANT (one arm)
                frontier.append((np.float32(s + logp[row, 0]), d + 1, me, 0))
        if len(parents) < n:
            raise ValueError("the candidates hold fewer than n - 1 nodes")
        return (np.array(parents, np.int32), np.array(tokens, np.int32), np.array(depth, np.int32),
                np.array(score, np.float32))
    return lambda: _replace(tb.tree_build, fn)


# ---------------------------------------------------------------- whole step
def _step(bug):
    orig = oracle.step.verify_step

    def fn(c_kv, k_rope, cache_lens, parents, tokens, argmax, q_abs, q_rope, scale,
           node_ckv=None, node_krope=None, attn_nodes=None, with_attention=True):
        c_in, r_in = c_kv, k_rope
        if node_ckv is not None:
            if bug == "write_next_slot":
                c_kv, k_rope = c_kv.copy(), k_rope.copy()
                for b in range(node_ckv.shape[0]):
                    L = int(cache_lens[b])
                    for k in range(node_ckv.shape[1]):
                        c_kv[b, L + k + 1] = node_ckv[b, k]      # MUTANT
                        k_rope[b, L + k + 1] = node_krope[b, k]
            else:
                c_kv, k_rope = cache.kv_write_nodes(c_kv, k_rope, cache_lens, node_ckv, node_krope)
        vis = np.stack([tree.visibility_words(p) for p in parents])
        out = lse = None
        if with_attention:
            src_c, src_r = (c_in, r_in) if bug == "attend_pre_write" else (c_kv, k_rope)  # MUTANT (one arm)
            out, lse = att.tree_verify_attention(q_abs, q_rope, src_c, src_r, cache_lens, vis,
                                                 scale, nodes=attn_nodes)
        path, ln, bonus = acc.tree_accept_batch(tokens, parents, argmax)
        c2, r2, lens2 = cache.kv_compact(c_kv, k_rope, cache_lens, path, ln)
        return dict(out=out, lse=lse, vis=vis, path=path, len=ln, bonus=bonus,
                    c_kv=c2, k_rope=r2, cache_lens=lens2, c_kv_pre=c_kv, k_rope_pre=k_rope)
    return lambda: _replace(orig, fn)


MUTANTS = {
    "attn_no_rope": _attention("no_rope"),
    "attn_scale_abs_only": _attention("scale_abs_only"),
    "attn_no_self": _attention("no_self"),
    "attn_cache_short": _attention("cache_short"),
    "attn_tree_ignores_mask": _attention("tree_ignores_mask"),
    "attn_tree_bits_reversed": _attention("tree_bits_reversed"),
    "attn_heads_mismatch": _attention("heads_mismatch"),
    "attn_out_unnormalized": _attention("out_unnormalized"),
    "attn_lse_no_max": _attention("lse_no_max"),
    "attn_lse_log2": _attention("lse_log2"),
    "bf16_as_fp16": _bf16_as_fp16,
    "depth_counts_nodes": _depth_counts_nodes,
    "mask_parent_only": _mask("parent_only"),
    "mask_no_self": _mask("no_self"),
    "mask_word_mod": _mask("word_mod"),
    "accept_child_index": _accept("child_index"),
    "accept_any_node": _accept("any_node"),
    "accept_last_duplicate": _accept("last_duplicate"),
    "accept_bonus_parent": _accept("bonus_parent"),
    "accept_path_without_root": _accept("path_without_root"),
    "argmax_last_tie": _argmax("last_tie"),
    "argmax_nan_ignored": _argmax("nan_ignored"),
    "write_slot_shift": _write_slot_shift,
    "compact_in_place_reversed": _compact("in_place_reversed"),
    "compact_src_no_offset": _compact("src_no_offset"),
    "compact_len_minus_one": _compact("len_minus_one"),
    "paged_no_scale": _paged_no_scale,
    "paged_writeback_identity": _writeback_identity,
    "build_tie_deeper_first": _build("tie_deeper_first"),
    "build_no_sibling": _build("no_sibling"),
    "build_sibling_own_score": _build("sibling_own_score"),
    "build_child_same_row": _build("child_same_row"),
    "step_attend_pre_write": _step("attend_pre_write"),
    "step_write_next_slot": _step("write_next_slot"),
}


def apply(name):
    if name != "none":
        MUTANTS[name]()
