"""Best-first draft-tree construction (oracle; test infrastructure only).

"The Architecture of Pragmatic Ambition", section "The Knowledge Architecture": the
tree builder takes per-depth top-k candidates from a drafter and constructs a
best-first tree, which the verify step then scores.  The pages give no scoring rule;
the reading taken here is the plainest one that the rest supports:

  * the drafter gives, for every depth d = 1..D, K candidate tokens with their
    log-probabilities, sorted from the most to the least likely, independent of
    the path above them (one distribution per draft position);
  * a node at depth d is a path (j_1, ..., j_d) of candidate indices, its token is
    candidate j_d of depth d, and its score is the sum, in float32 and in path
    order, of the log-probabilities along the path;
  * the tree is the root (node 0, depth 0, score 0, the last verified token) plus
    the n - 1 best-scoring nodes, taken one at a time from the frontier of the tree
    built so far, best first; equal scores go to the lower depth, then the lower
    parent index, then the lower candidate index.  Node indices are the pop order,
    which is topological (a child never scores above its parent).

Because each depth's candidates are sorted and log-probabilities are <= 0, a popped
node only needs to offer its next sibling and its first child to the frontier: every
node still outside them scores no better than one of them.  The function below takes
exactly these steps.
"""
import numpy as np


def _key(score, depth, parent, cand):
    # larger is better: higher score, then lower depth, parent, candidate
    return (float(score), -depth, -parent, -cand)


def tree_build(logp, cand_tokens, root_token, n):
    """One request.  logp, cand_tokens: [D][K] (float32, int32), each depth sorted by
    descending logp.  Returns (parents int32 [n], tokens int32 [n], depth int32 [n],
    score float32 [n])."""
    logp = np.asarray(logp, dtype=np.float32)
    D, K = logp.shape
    parents = [-1]
    tokens = [int(root_token)]
    depth = [0]
    score = [np.float32(0.0)]
    frontier = []                     # (score, depth, parent, cand)
    if D >= 1 and n > 1:
        frontier.append((np.float32(logp[0, 0]), 1, 0, 0))
    while len(parents) < n and frontier:
        best = max(range(len(frontier)), key=lambda i: _key(*frontier[i]))
        s, d, p, j = frontier.pop(best)
        me = len(parents)
        parents.append(p)
        tokens.append(int(cand_tokens[d - 1][j]))
        depth.append(d)
        score.append(s)
        if j + 1 < K:                 # next sibling: same parent, next candidate
            frontier.append((np.float32(score[p] + logp[d - 1, j + 1]), d, p, j + 1))
        if d < D:                     # first child
            frontier.append((np.float32(s + logp[d, 0]), d + 1, me, 0))
    if len(parents) < n:
        raise ValueError("the candidates hold fewer than n - 1 nodes")
    return (np.array(parents, np.int32), np.array(tokens, np.int32), np.array(depth, np.int32),
            np.array(score, np.float32))


def tree_build_batch(logp, cand_tokens, root_tokens, n):
    """[B][D][K] inputs -> parents, tokens, depth int32 [B][n], score float32 [B][n]."""
    outs = [tree_build(logp[b], cand_tokens[b], root_tokens[b], n) for b in range(len(root_tokens))]
    return tuple(np.stack([o[i] for o in outs]) for i in range(4))
