"""Greedy tree acceptance (oracle).

"The Architecture of Pragmatic Ambition", section "The Knowledge Architecture":
the accept step walks the verified tree greedily to the longest prefix that
matches the target's predictions.  Written out: start at the root; while some
child c of the current node carries the token the target predicted after the
current node (node_tokens[c] == target_argmax[cur]), step to it (lowest index
first, a reading for duplicate sibling tokens); the bonus token is the target's
prediction after the last accepted node.  The accepted length counts the root
("The Architectural Keystone ...", section "The Reasoning That Preceded the
Header": the cache advances by the accepted count, and budget 0 is plain decode,
i.e. length 1).
"""
import numpy as np


def tree_accept(node_tokens, parents, target_argmax):
    """Per request: returns (path list, length, bonus).  Inputs are 1-D, length n."""
    n = len(parents)
    path = [0]
    cur = 0
    while len(path) < n:          # a root-to-node path has at most n nodes
        nxt = -1
        for c in range(n):
            if int(parents[c]) == cur and int(node_tokens[c]) == int(target_argmax[cur]):
                nxt = c
                break
        if nxt < 0:
            break
        path.append(nxt)
        cur = nxt
    return path, len(path), int(target_argmax[cur])


def tree_accept_batch(node_tokens, parents, target_argmax):
    """[B][n] inputs -> (path int32 [B][n] (-1 padded), len int32 [B], bonus int32 [B])."""
    B, n = np.asarray(parents).shape
    path = np.full((B, n), -1, dtype=np.int32)
    ln = np.zeros(B, dtype=np.int32)
    bonus = np.zeros(B, dtype=np.int32)
    for b in range(B):
        p, l, t = tree_accept(node_tokens[b], parents[b], target_argmax[b])
        path[b, :l] = p
        ln[b] = l
        bonus[b] = t
    return path, ln, bonus


def target_argmax(logits):
    """The target's greedy token after each node: the index of the largest logit in its
    row ("The Architecture of Pragmatic Ambition", section "The Output Knowledge: What
    This Message Creates": argmax is an engine primitive, and the speculative output must
    equal greedy decoding token for token).  Readings for what the pages leave open:
    among equal maxima the lowest index wins, a NaN ranks above every number (the first
    NaN wins), and -0.0 equals +0.0.  numpy's argmax is exactly this definition.
    logits [..., V] -> int32 [...]."""
    return np.argmax(np.asarray(logits), axis=-1).astype(np.int32)


def tree_accept_logits(node_tokens, parents, logits):
    """Greedy acceptance fed by the target argmax of fp32 logits [B][n][V]:
    returns (argmax [B][n], path, len, bonus) as tree_accept_batch."""
    am = target_argmax(logits)
    path, ln, bonus = tree_accept_batch(node_tokens, parents, am)
    return am, path, ln, bonus
