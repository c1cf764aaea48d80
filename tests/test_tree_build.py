"""GPU parity of the best-first draft-tree build (kd_tree_build) against the oracle:
parents, tokens, depths and float32 scores all bit-exact."""
import numpy as np
import pytest
import torch

from oracle.tree_build import tree_build_batch
from tree_speculative_decoding_kd_b200 import workload as W

pytestmark = pytest.mark.gpu


def cands(rng, B, D, K, vocab=163840):
    logp = np.sort(np.log(rng.dirichlet(np.ones(K), size=(B, D))).astype(np.float32), axis=2)[:, :, ::-1]
    toks = rng.integers(0, vocab, size=(B, D, K)).astype(np.int32)
    root = rng.integers(0, vocab, size=B).astype(np.int32)
    return logp.copy(), toks, root              # a fresh C-ordered copy (no negative stride)


def check(kd, logp, toks, root, n):
    got = kd.kd_tree_build(torch.from_numpy(logp).cuda(), torch.from_numpy(toks).cuda(),
                           torch.from_numpy(root).cuda(), n)
    torch.cuda.synchronize()
    want = tree_build_batch(logp, toks, root, n)
    for g, w, nm in zip(got, want, ("parents", "tokens", "depth", "score")):
        g = g.cpu().numpy()
        assert np.array_equal(g, w), nm
    return want


@pytest.mark.parametrize("B,D,K,n", [(3, 4, 3, 30), (5, 16, 8, 17), (4, 1, 8, 9), (2, 6, 1, 7),
                                     (2, 127, 2, 128), (2, 2, 255, 128), (33, 8, 4, 64),
                                     (2, 64, 32, 128)])     # the last: a large candidate table
def test_tree_build_random(kd, B, D, K, n):
    rng = np.random.default_rng(D * 1000 + K * 10 + n)
    check(kd, *cands(rng, B, D, K), n)


def test_tree_build_ties_and_infinities(kd):
    rng = np.random.default_rng(11)
    logp, toks, root = cands(rng, 3, 5, 3)
    logp[0] = 0.0                                  # every score ties: breadth first
    logp[1, :, 1:] = -np.inf                       # impossible candidates still rank, last
    logp[2, 2:4] = logp[2, 0:2]                    # equal rows at several depths
    check(kd, logp, toks, root, 40)


def test_tree_build_loop_workload(kd):
    cfg = W.CONFIGS["loop"]
    logp, toks, root = W.draw_candidates(cfg)
    par, tok, dep, sc = check(kd, logp, toks, root, cfg.n)
    assert (par[:, 1:] < np.arange(1, cfg.n)).all()


def test_tree_build_errors(kd):
    rng = np.random.default_rng(2)
    logp, toks, root = cands(rng, 2, 1, 2)
    with pytest.raises(kd.KdError):                # 2 candidate nodes, 3 needed
        check(kd, logp, toks, root, 4)
    with pytest.raises(kd.KdError):                # more than 128 nodes
        check(kd, *cands(rng, 1, 8, 4), 129)
