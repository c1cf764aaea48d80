"""Tree-verify MLA-absorb attention in float64 (oracle).

Definition followed ("The Architecture of Pragmatic Ambition", sections "The
Thinking Process" and "The Knowledge Architecture"; "The Architectural
Keystone ...", section "The Reasoning That Preceded the Header"):

For request b with committed length L = cache_lens[b], node i, head h:
  visible keys V(i) = {0..L-1} U {L + k : k in anc*(i)}    (node k lives in slot L+k)
  s_j   = scale * (q_abs[i,h] . c_kv[j] + q_rope[i,h] . k_rope[j]),  j in V(i)
  p     = softmax_j(s)
  out[i,h] = sum_j p_j c_kv[j]            (the value is the 512-wide latent itself;
                                           W_UV is applied later, outside this step)
  lse[i,h] = ln sum_j exp(s_j)

Inputs are the same bf16 bit patterns the GPU receives, widened exactly to
float64; nothing else is rounded.  Nodes are processed a few at a time only to
bound memory; each node's scores are formed over its own visible set.
"""
import numpy as np


def bf16_to_f64(u) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    u = np.asarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def _visible(L: int, n: int, words) -> np.ndarray:
    """Boolean mask over key slots 0..L+n-1 for one node."""
    vis = np.ones(L + n, dtype=bool)
    for k in range(n):
        vis[L + k] = bool((int(words[k // 32]) >> (k % 32)) & 1)
    return vis


def tree_verify_attention(q_abs, q_rope, c_kv, k_rope, cache_lens, vis, scale,
                          nodes=None):
    """Returns (out float64 [B][n][H][512], lse float64 [B][n][H]).

    q_abs uint16 [B][n][H][512], q_rope uint16 [B][n][H][64], c_kv uint16
    [B][cap][512], k_rope uint16 [B][cap][64], cache_lens int [B], vis uint32
    [B][n][W].  ``nodes`` optionally restricts the work to a list of (b, i)
    pairs; other rows are left as NaN.
    """
    B, n, H, dc = q_abs.shape
    out = np.full((B, n, H, dc), np.nan)
    lse = np.full((B, n, H), np.nan)
    if nodes is None:
        nodes = [(b, i) for b in range(B) for i in range(n)]
    by_req = {}
    for b, i in nodes:
        by_req.setdefault(int(b), []).append(int(i))
    for b, idx in by_req.items():
        L = int(cache_lens[b])
        if L + n > c_kv.shape[1]:
            raise ValueError("cache_len + n exceeds the slot capacity")
        K = bf16_to_f64(c_kv[b, :L + n])        # [L+n][512]
        R = bf16_to_f64(k_rope[b, :L + n])      # [L+n][64]
        for i in idx:
            m = _visible(L, n, vis[b, i])
            Kv, Rv = K[m], R[m]
            qa = bf16_to_f64(q_abs[b, i])       # [H][512]
            qr = bf16_to_f64(q_rope[b, i])      # [H][64]
            s = scale * (qa @ Kv.T + qr @ Rv.T)  # [H][|V|]
            smax = s.max(axis=1, keepdims=True)
            e = np.exp(s - smax)
            l = e.sum(axis=1, keepdims=True)
            out[b, i] = (e @ Kv) / l
            lse[b, i] = (smax + np.log(l))[:, 0]
    return out, lse
