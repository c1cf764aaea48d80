"""KV-cache updates around a verify step (oracle).

Page size 1: every token owns one contiguous slot ("The Architectural Keystone
...", section "Assumptions Embedded in the Design").  Before verify, the n node
latents occupy slots L..L+n-1 (root first, "The Reasoning That Preceded the
Header").  After acceptance the accepted path's latents, root included, are
gathered into slots L..L+len-1 and the length advances by len (same section).
All kept rows are read before any is written, since source and destination
slots can overlap ("Mistakes and Iterative Refinement").
"""
import numpy as np


def kv_write_nodes(c_kv, k_rope, cache_lens, node_ckv, node_krope):
    """Copies of the caches with node k of request b stored in slot cache_lens[b] + k."""
    c_kv = c_kv.copy()
    k_rope = k_rope.copy()
    B, n = node_ckv.shape[:2]
    for b in range(B):
        L = int(cache_lens[b])
        if L + n > c_kv.shape[1]:
            raise ValueError("cache_len + n exceeds the slot capacity")
        for k in range(n):
            c_kv[b, L + k] = node_ckv[b, k]
            k_rope[b, L + k] = node_krope[b, k]
    return c_kv, k_rope


def kv_compact(c_kv, k_rope, cache_lens, path, lens):
    """Returns new (c_kv, k_rope, cache_lens) after gathering each accepted path.

    path int [B][n] (first lens[b] entries valid), lens int [B].
    """
    c_kv = c_kv.copy()
    k_rope = k_rope.copy()
    new_lens = np.array(cache_lens, dtype=np.int32).copy()
    B = c_kv.shape[0]
    for b in range(B):
        L = int(cache_lens[b])
        m = int(lens[b])
        if L + m > c_kv.shape[1]:
            raise ValueError("cache_len + len exceeds the slot capacity")
        rows_c = [c_kv[b, L + int(path[b][j])].copy() for j in range(m)]   # read all ...
        rows_r = [k_rope[b, L + int(path[b][j])].copy() for j in range(m)]
        for j in range(m):                                                 # ... then write
            c_kv[b, L + j] = rows_c[j]
            k_rope[b, L + j] = rows_r[j]
        new_lens[b] = L + m
    return c_kv, k_rope, new_lens
