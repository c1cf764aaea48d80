"""GPU parity of the target argmax fused with greedy acceptance (kd_tree_accept_logits)
against the oracle (numpy argmax feeding the greedy walk).  Everything is bit-exact:
the tokens, the path, its length and the bonus token."""
import numpy as np
import pytest
import torch

from oracle.accept import tree_accept_logits
from tree_speculative_decoding_kd_b200 import workload as W

pytestmark = pytest.mark.gpu

CHUNK = 16384         # logits per CTA in the kernel; ties are planted across this boundary


def dev_i32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()


def run(kd, tokens, parents, logits, **kw):
    am, path, ln, bonus = kd.kd_tree_accept_logits(dev_i32(tokens), dev_i32(parents),
                                                   torch.from_numpy(logits).cuda(), **kw)
    torch.cuda.synchronize()
    return am.cpu().numpy(), path.cpu().numpy(), ln.cpu().numpy(), bonus.cpu().numpy()


def check(kd, tokens, parents, logits):
    got = run(kd, tokens, parents, logits)
    want = tree_accept_logits(tokens, parents, logits)
    for g, w, nm in zip(got, want, ("argmax", "path", "len", "bonus")):
        assert np.array_equal(g, w), nm
    return want


def special_rows(rng, B, n, V, parents, tokens):
    """Logits whose rows exercise the tie, NaN, signed-zero and edge rules; each row's
    winner is, most of the time, the token of one of the node's children, so that the
    greedy walk goes deep."""
    lg = np.clip(rng.standard_normal((B, n, V), dtype=np.float32), -6, 6)
    for b in range(B):
        for i in range(n):
            kids = np.nonzero(parents[b] == i)[0]
            t = int(tokens[b, kids[rng.integers(len(kids))]]) if len(kids) and rng.random() < 0.8 \
                else int(rng.integers(V))
            kind = (b * n + i) % 7
            row = lg[b, i]
            if kind == 0:                                  # unique maximum
                row[t] = 9.0
            elif kind == 1:                                # tie across a chunk boundary
                j = CHUNK if V > CHUNK else V // 2
                row[j - 1] = row[j] = 9.0
            elif kind == 2:                                # tie: the planted token comes first
                row[t] = 9.0
                if t < V - 1:
                    row[t + 1 + int(rng.integers(V - 1 - t))] = 9.0
            elif kind == 3:                                # NaNs: the first one wins
                row[t] = np.nan
                row[V - 1] = np.nan
            elif kind == 4:                                # -0.0 before +0.0, all else negative
                row[:] = -np.abs(row) - 1.0
                a, c = sorted(rng.choice(V, 2, replace=False))
                row[a], row[c] = -0.0, 0.0
            elif kind == 5:                                # every logit -inf
                row[:] = -np.inf
            else:                                          # maximum in the last element
                row[V - 1] = 9.0
    return lg


@pytest.mark.parametrize("B,n,V", [(3, 40, 20000), (2, 8, 8192), (1, 1, 4), (2, 128, 16388)])
def test_accept_logits_rules_and_edges(kd, B, n, V):
    rng = np.random.default_rng(1000 + n)
    parents = np.stack([W.draw_parents(rng, n, "uniform", 0) for _ in range(B)])
    tokens = np.stack([W.draw_tokens(rng, p, vocab=V) for p in parents])
    check(kd, tokens, parents, special_rows(rng, B, n, V, parents, tokens))


def test_accept_logits_recipe_single(kd):
    wl = W.make_workload("kimi_single")
    st = wl.step
    am, path, ln, bonus = check(kd, st.tokens, st.parents, W.draw_logits(wl.cfg, st))
    assert np.array_equal(am, st.argmax)
    assert list(path[0, :ln[0]]) == [int(x) for x in st.planted[0]]


def test_accept_logits_loop_full_size(kd):
    """All 64 requests x 17 nodes x 163840 logits (713 MB) of the loop workload."""
    wl = W.make_workload("loop")
    st = wl.step
    am, path, ln, bonus = check(kd, st.tokens, st.parents, W.draw_logits(wl.cfg, st))
    assert np.array_equal(am, st.argmax)
    for b in range(wl.cfg.B):
        assert list(path[b, :ln[b]]) == [int(x) for x in st.planted[b]]


def test_accept_logits_errors(kd):
    rng = np.random.default_rng(5)
    parents = np.stack([W.draw_parents(rng, 8, "uniform", 0) for _ in range(2)])
    tokens = np.stack([W.draw_tokens(rng, p, vocab=64) for p in parents])
    with pytest.raises(kd.KdError):                        # V not a multiple of 4
        run(kd, tokens, parents, rng.standard_normal((2, 8, 66), dtype=np.float32))
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(kd.KdError):                        # workspace too small
        run(kd, tokens, parents, rng.standard_normal((2, 8, 64), dtype=np.float32), workspace=small)
    bad = parents.copy()
    bad[1, 3] = 5                                          # parent not earlier than the node
    err = kd.new_error_word()
    am, path, ln, bonus = run(kd, tokens, bad, rng.standard_normal((2, 8, 64), dtype=np.float32),
                              dev_error=err)
    bits = kd.kd_read_device_error(err)
    assert "BAD_PARENT" in kd.decode_device_error(bits)
    assert ln[1] == 1 and path[1, 0] == 0 and (path[1, 1:] == -1).all()
