"""KV-cache updates around a verify step (oracle).

Page size 1: every token owns one contiguous slot ("The Architectural Keystone
...", section "Assumptions Embedded in the Design").  Before verify, the n node
latents occupy slots L..L+n-1 (root first, "The Reasoning That Preceded the
Header").  After acceptance the accepted path's latents, root included, are
gathered into slots L..L+len-1 and the length advances by len (same section).
All kept rows are read before any is written, since source and destination
slots can overlap ("Mistakes and Iterative Refinement").

Paged caches (page size P > 1, the remedy for the page-size-1 fragmentation the
same section reports): request b's logical slot s lives in physical row
page_table[b][s // P] * P + s % P of a shared pool of pages.  Everything above is
defined on the logical view; the paged forms gather it, apply the definition and
write the request's pages back.
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


def paged_view(pages, page_table, page_size):
    """Logical caches [B][M * P][w] of a paged pool pages [num_pages * P][w] under
    page_table int [B][M] (physical page of each logical page)."""
    pt = np.asarray(page_table, dtype=np.int64)
    B, M = pt.shape
    rows = (pt[:, :, None] * page_size + np.arange(page_size)[None, None, :]).reshape(B, M * page_size)
    return pages[rows]


def _write_back(pages, page_table, page_size, logical):
    out = pages.copy()
    pt = np.asarray(page_table, dtype=np.int64)
    for b in range(pt.shape[0]):
        for q in range(pt.shape[1]):
            out[pt[b, q] * page_size:(pt[b, q] + 1) * page_size] = logical[b, q * page_size:(q + 1) * page_size]
    return out


def kv_write_nodes_paged(c_pages, r_pages, page_table, page_size, cache_lens, node_ckv, node_krope):
    """kv_write_nodes on the logical view of a paged pool; returns the new pools."""
    c, r = kv_write_nodes(paged_view(c_pages, page_table, page_size),
                          paged_view(r_pages, page_table, page_size), cache_lens, node_ckv, node_krope)
    return (_write_back(c_pages, page_table, page_size, c), _write_back(r_pages, page_table, page_size, r))


def kv_compact_paged(c_pages, r_pages, page_table, page_size, cache_lens, path, lens):
    """kv_compact on the logical view of a paged pool; returns (pools, new lengths)."""
    c, r, new_lens = kv_compact(paged_view(c_pages, page_table, page_size),
                                paged_view(r_pages, page_table, page_size), cache_lens, path, lens)
    return (_write_back(c_pages, page_table, page_size, c), _write_back(r_pages, page_table, page_size, r),
            new_lens)
