"""One whole verify step of the DDTree loop (oracle).

Order ("The Architecture of Pragmatic Ambition", section "The Knowledge
Architecture"; "The Architectural Keystone ...", section "The Reasoning That
Preceded the Header"): node latents written at the next free slots, tree
visibility built from the parents, verify attention, greedy accept against the
target argmax, compaction of the accepted path and length advance.
"""
import numpy as np

from .tree import visibility_words
from .attention import tree_verify_attention
from .accept import tree_accept_batch
from .cache import kv_write_nodes, kv_compact


def verify_step(c_kv, k_rope, cache_lens, parents, tokens, argmax, q_abs, q_rope,
                scale, node_ckv=None, node_krope=None, attn_nodes=None,
                with_attention=True):
    """Returns dict(out, lse, vis, path, len, bonus, c_kv, k_rope, cache_lens, c_kv_pre, k_rope_pre).

    ``*_pre`` are the caches after the node write and before compaction.
    """
    if node_ckv is not None:
        c_kv, k_rope = kv_write_nodes(c_kv, k_rope, cache_lens, node_ckv, node_krope)
    vis = np.stack([visibility_words(p) for p in parents])
    out = lse = None
    if with_attention:
        out, lse = tree_verify_attention(q_abs, q_rope, c_kv, k_rope, cache_lens, vis,
                                         scale, nodes=attn_nodes)
    path, ln, bonus = tree_accept_batch(tokens, parents, argmax)
    c2, r2, lens2 = kv_compact(c_kv, k_rope, cache_lens, path, ln)
    return dict(out=out, lse=lse, vis=vis, path=path, len=ln, bonus=bonus,
                c_kv=c2, k_rope=r2, cache_lens=lens2, c_kv_pre=c_kv, k_rope_pre=k_rope)
