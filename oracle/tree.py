"""Tree structure: ancestors, depths and per-node visibility bitmasks (oracle).

A verify tree holds budget+1 nodes; node 0 is the root (the last verified
token, re-processed at the next free slot) and every other node is a draft
whose parent precedes it ("The Architectural Keystone ...", section "The
Reasoning That Preceded the Header").  Verify attention lets a node see the
committed cache plus its tree ancestors ("The Architecture of Pragmatic
Ambition", section "The Knowledge Architecture": attention over the tree
"with a visibility mask").  Reading taken: a node also sees itself, which is
what makes a chain-shaped tree equal to causal attention.
"""
import numpy as np


def n_words(n: int) -> int:
    """uint32 words per node mask: one bit per tree node."""
    return (n + 31) // 32


def check_parents(parents) -> None:
    """Raise ValueError unless parent[0] == -1 and 0 <= parent[i] < i for i >= 1."""
    p = [int(x) for x in parents]
    if not p or p[0] != -1:
        raise ValueError("parent[0] must be -1")
    for i in range(1, len(p)):
        if not (0 <= p[i] < i):
            raise ValueError(f"parent[{i}] = {p[i]} is not an earlier node")


def ancestors(parents, i: int) -> list:
    """anc*(i): i and every node on its path to the root, walking parent links."""
    out = [i]
    while parents[out[-1]] != -1:
        out.append(int(parents[out[-1]]))
    return out


def depths(parents) -> np.ndarray:
    """Number of edges from the root, by walking to the root from each node."""
    return np.array([len(ancestors(parents, i)) - 1 for i in range(len(parents))],
                    dtype=np.int32)


def visibility_words(parents) -> np.ndarray:
    """uint32 [n][W] masks: bit k of word k//32 of row i set iff k is in anc*(i)."""
    check_parents(parents)
    n = len(parents)
    out = np.zeros((n, n_words(n)), dtype=np.uint32)
    for i in range(n):
        for k in ancestors(parents, i):
            out[i, k // 32] |= np.uint32(1) << np.uint32(k % 32)
    return out
