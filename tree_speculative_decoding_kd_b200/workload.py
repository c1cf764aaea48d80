"""Seeded synthetic workloads for the tree-verify step.

This module only draws inputs: random latents, queries, trees, draft tokens,
target argmaxes and target logits that carry them, and drafter candidates.  It computes nothing of the method itself (no attention, no
acceptance walk, no compaction).  Both the CUDA path (through the Python
binding) and the float64 oracle consume what it returns.

Shapes follow the DeepSeek-V3 / Kimi-K2 MLA layout described on the pages
("The Architecture of Pragmatic Ambition", section "The Thinking Process":
score_nope = q_nope . (W_UK c_kv), absorbed into q_nope W_UK so the query meets
the 512-wide compressed latent directly) plus the 64-wide decoupled RoPE part:

  q_abs   bf16 [B][n][H][512]   absorbed no-position query
  q_rope  bf16 [B][n][H][64]    rotated rope query
  c_kv    bf16 [B][cap][512]    compressed latent cache (page size 1)
  k_rope  bf16 [B][cap][64]     rotated rope key cache

bf16 tensors are held as numpy uint16 bit patterns.  Values are fp32
N(0,1)/sqrt(576) rounded to bf16 with round-to-nearest-even.

Tree recipe ("The Architectural Keystone", section "The Reasoning That Preceded
the Header": the verify pass covers budget+1 nodes, the root being the last
verified token re-processed at the next free cache slot): node 0 is the root,
parent[0] = -1 and parent[i] < i (topological order).  Sibling draft tokens are
distinct, as a per-depth top-k drafter would produce.

Draw order is fixed and documented in each function; every large tensor is
drawn in fixed-size chunks, each from its own child seed, so results do not
depend on how many threads fill them.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

D_C = 512          # compressed latent width (kv_lora_rank)
D_R = 64           # decoupled rope width
VOCAB = 163840     # Kimi-K2 vocabulary
CHUNK = 1 << 22    # elements per independently seeded chunk

# --------------------------------------------------------------------------
# configurations
# --------------------------------------------------------------------------


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    n: int                    # budget + 1 nodes
    L_lo: int                 # committed cache length range (inclusive)
    L_hi: int
    tree: str                 # "uniform" | "depth" | "branch"
    tree_arg: int             # max depth (depth rule) or max children (branch rule)
    seed: int
    steps: int = 1            # verify steps (loop workload only)
    scale: float = 1.0 / math.sqrt(192.0)

    @property
    def cap(self) -> int:
        """Slot capacity per request: room for every step's n nodes."""
        return self.L_hi + self.steps * self.n + self.n


CONFIGS = {
    # 1 request, 16 heads, L=256, budget 7, parent[i] uniform in [0, i), seed 0
    "tiny": Config("tiny", 1, 16, 8, 256, 256, "uniform", 0, 0),
    # Kimi-K2-shaped single request: 64 heads, L=4096, budget 16, depth <= 8
    "kimi_single": Config("kimi_single", 1, 64, 17, 4096, 4096, "depth", 8, 1),
    # 32 requests, L ~ U{1024..8192}, budget 32, branching factor <= 4
    "batched": Config("batched", 32, 64, 33, 1024, 8192, "branch", 4, 2),
    # 8 requests, L = 32768, budget 64, depth <= 12 (split-KV required)
    "long": Config("long", 8, 64, 65, 32768, 32768, "depth", 12, 3),
    # 64 requests, L ~ U{2048..16384}, budget 16, 100 verify+accept+compact steps
    "loop": Config("loop", 64, 64, 17, 2048, 16384, "depth", 8, 4, steps=100),
    # chunked causal extend through the same kernel: a chain "tree" (parent[i] = i - 1)
    # makes the visibility mask causal; 4 requests extend a 16384-token cache by 128 tokens
    "extend": Config("extend", 4, 64, 128, 16384, 16384, "chain", 0, 5),
}

# --------------------------------------------------------------------------
# number generation helpers
# --------------------------------------------------------------------------


def _threads() -> int:
    try:
        return max(1, min(16, len(os.sched_getaffinity(0))))
    except AttributeError:  # pragma: no cover
        return max(1, min(16, os.cpu_count() or 1))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def _fill_chunk(out_flat: np.ndarray, start: int, stop: int, ss: np.random.SeedSequence,
                std: float) -> None:
    g = np.random.default_rng(ss)
    v = g.standard_normal(stop - start, dtype=np.float32)
    v /= np.float32(1.0 / std)
    out_flat[start:stop] = to_bf16_bits(v)


def latent_bf16(shape, seed_key, std: float = 1.0 / 24.0, pool=None) -> np.ndarray:
    """bf16 bits of fp32 N(0, 1) * std values, chunk-seeded by ``seed_key``.

    ``seed_key`` is a tuple of non-negative ints; chunk c uses the seed
    sequence (*seed_key, c).  The default std is 1/sqrt(576).
    """
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.uint16)
    starts = list(range(0, total, CHUNK))
    jobs = [(s, min(s + CHUNK, total), np.random.SeedSequence(list(seed_key) + [ci]))
            for ci, s in enumerate(starts)]
    if len(jobs) <= 1:
        for s, e, ss in jobs:
            _fill_chunk(out, s, e, ss, std)
    else:
        ex = pool or ThreadPoolExecutor(_threads())
        try:
            list(ex.map(lambda j: _fill_chunk(out, j[0], j[1], j[2], std), jobs))
        finally:
            if pool is None:
                ex.shutdown()
    return out.reshape(shape)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to fp32 (used by the harness for display only)."""
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# trees, tokens and planted target predictions
# --------------------------------------------------------------------------


def draw_parents(rng: np.random.Generator, n: int, rule: str, arg: int) -> np.ndarray:
    """parent[0] = -1; parent[i] drawn uniformly from the earlier nodes allowed by ``rule``.

    uniform: any earlier node; depth: earlier nodes of depth < arg;
    branch: earlier nodes with fewer than arg children.
    """
    parents = np.full(n, -1, dtype=np.int32)
    depth = np.zeros(n, dtype=np.int32)
    kids = np.zeros(n, dtype=np.int32)
    for i in range(1, n):
        if rule == "uniform":
            allowed = np.arange(i)
        elif rule == "depth":
            allowed = np.nonzero(depth[:i] < arg)[0]
        elif rule == "branch":
            allowed = np.nonzero(kids[:i] < arg)[0]
        elif rule == "chain":
            allowed = np.array([i - 1])
        elif rule == "star":
            allowed = np.array([0])
        else:
            raise ValueError(rule)
        p = int(allowed[rng.integers(0, len(allowed))])
        parents[i] = p
        depth[i] = depth[p] + 1
        kids[p] += 1
    return parents


def node_depths(parents: np.ndarray) -> np.ndarray:
    d = np.zeros(len(parents), dtype=np.int32)
    for i in range(1, len(parents)):
        d[i] = d[parents[i]] + 1
    return d


def draw_tokens(rng: np.random.Generator, parents: np.ndarray, vocab: int = VOCAB) -> np.ndarray:
    """Uniform draft tokens; a node's token is redrawn until it differs from its earlier siblings."""
    n = len(parents)
    tok = np.zeros(n, dtype=np.int32)
    tok[0] = rng.integers(0, vocab)
    seen: dict[int, set] = {}
    for i in range(1, n):
        s = seen.setdefault(int(parents[i]), set())
        t = int(rng.integers(0, vocab))
        while t in s:
            t = int(rng.integers(0, vocab))
        s.add(t)
        tok[i] = t
    return tok


def draw_accept_depth(rng: np.random.Generator, cont: float = 0.7) -> int:
    """K with P(K >= k) = cont**k (number of accepted drafts, before truncation)."""
    k = 0
    while rng.random() < cont:
        k += 1
    return k


def plant_argmax(rng: np.random.Generator, parents: np.ndarray, tokens: np.ndarray,
                 k_target: int, vocab: int = VOCAB):
    """Target argmax with a planted accepted path.

    A node at depth min(k_target, max depth) is picked uniformly; along its
    root path argmax[path[d]] = tokens[path[d+1]]; at its end argmax is a token
    none of its children carries; every other node gets a uniform token.
    Returns (argmax, planted_path).
    """
    n = len(parents)
    depth = node_depths(parents)
    d = min(k_target, int(depth.max()))
    cands = np.nonzero(depth == d)[0]
    end = int(cands[rng.integers(0, len(cands))])
    path = [end]
    while path[-1] != 0:
        path.append(int(parents[path[-1]]))
    path = path[::-1]
    am = rng.integers(0, vocab, size=n).astype(np.int32)
    for a, c in zip(path[:-1], path[1:]):
        am[a] = tokens[c]
    child_toks = {int(tokens[c]) for c in range(n) if parents[c] == end}
    t = int(am[end])
    while t in child_toks:
        t = int(rng.integers(0, vocab))
    am[end] = t
    return am, np.array(path, dtype=np.int32)


# --------------------------------------------------------------------------
# whole workloads
# --------------------------------------------------------------------------


@dataclasses.dataclass
class StepInputs:
    """Per-step tree inputs and queries (and node latents for the loop workload)."""
    parents: np.ndarray      # int32 [B][n]
    tokens: np.ndarray       # int32 [B][n]
    argmax: np.ndarray       # int32 [B][n]
    planted: list            # list of int32 arrays (accepted path per request)
    q_abs: np.ndarray        # uint16 [B][n][H][512]
    q_rope: np.ndarray       # uint16 [B][n][H][64]
    node_ckv: np.ndarray | None = None    # uint16 [B][n][512]
    node_krope: np.ndarray | None = None  # uint16 [B][n][64]


@dataclasses.dataclass
class Workload:
    cfg: Config
    cache_lens: np.ndarray   # int32 [B]
    c_kv: np.ndarray         # uint16 [B][cap][512]
    k_rope: np.ndarray       # uint16 [B][cap][64]
    step: StepInputs


def draw_cache_lens(cfg: Config) -> np.ndarray:
    g = np.random.default_rng([cfg.seed, 0])
    if cfg.L_lo == cfg.L_hi:
        return np.full(cfg.B, cfg.L_lo, dtype=np.int32)
    return g.integers(cfg.L_lo, cfg.L_hi + 1, size=cfg.B).astype(np.int32)


def draw_step(cfg: Config, step: int, with_nodes: bool, vocab: int = VOCAB,
              tree: str | None = None, tree_arg: int | None = None) -> StepInputs:
    """Draw one step's trees and queries.

    Order: per request b: parents, tokens, accept depth, planted argmax (from
    the generator seeded (seed, 1, step)); then q_abs, q_rope, node latents
    from chunk seeds (seed, 2..5, step).
    """
    B, n, H = cfg.B, cfg.n, cfg.H
    rule = tree or cfg.tree
    arg = cfg.tree_arg if tree_arg is None else tree_arg
    g = np.random.default_rng([cfg.seed, 1, step])
    parents = np.zeros((B, n), np.int32)
    tokens = np.zeros((B, n), np.int32)
    argmax = np.zeros((B, n), np.int32)
    planted = []
    for b in range(B):
        parents[b] = draw_parents(g, n, rule, arg)
        tokens[b] = draw_tokens(g, parents[b], vocab)
        k = draw_accept_depth(g)
        argmax[b], path = plant_argmax(g, parents[b], tokens[b], k, vocab)
        planted.append(path)
    with ThreadPoolExecutor(_threads()) as pool:
        q_abs = latent_bf16((B, n, H, D_C), (cfg.seed, 2, step), pool=pool)
        q_rope = latent_bf16((B, n, H, D_R), (cfg.seed, 3, step), pool=pool)
        node_ckv = node_krope = None
        if with_nodes:
            node_ckv = latent_bf16((B, n, D_C), (cfg.seed, 4, step), pool=pool)
            node_krope = latent_bf16((B, n, D_R), (cfg.seed, 5, step), pool=pool)
    return StepInputs(parents, tokens, argmax, planted, q_abs, q_rope, node_ckv, node_krope)


def draw_cache(cfg: Config, cache_lens: np.ndarray, fill: int) -> tuple[np.ndarray, np.ndarray]:
    """Latent caches [B][cap][*]: slots [0, L_b + fill) random, the rest zero.

    Request b's rows come from chunk seeds (seed, 6, b) and (seed, 7, b).
    """
    B, cap = cfg.B, cfg.cap
    c_kv = np.zeros((B, cap, D_C), np.uint16)
    k_rope = np.zeros((B, cap, D_R), np.uint16)
    with ThreadPoolExecutor(_threads()) as pool:
        for b in range(B):
            rows = min(cap, int(cache_lens[b]) + fill)
            c_kv[b, :rows] = latent_bf16((rows, D_C), (cfg.seed, 6, b), pool=pool)
            k_rope[b, :rows] = latent_bf16((rows, D_R), (cfg.seed, 7, b), pool=pool)
    return c_kv, k_rope


def to_paged(c_kv: np.ndarray, k_rope: np.ndarray, page_size: int, seed: int = 0, spare: int = 3):
    """Lay per-request caches [B][cap][w] out as a shared pool of pages of page_size
    slots, in a seeded random physical order with a few unused pages between them
    (each request's capacity rounds up to whole pages; the extra slots are zero).
    Returns (c_pages [N * P][512], r_pages [N * P][64], page_table int32 [B][M])."""
    B, cap = c_kv.shape[:2]
    M = -(-cap // page_size)
    N = B * M + spare
    perm = np.random.default_rng([seed, 7, page_size]).permutation(N)[: B * M].reshape(B, M)
    c_pages = np.zeros((N * page_size, c_kv.shape[2]), dtype=c_kv.dtype)
    r_pages = np.zeros((N * page_size, k_rope.shape[2]), dtype=k_rope.dtype)
    for b in range(B):
        for q in range(M):
            lo, hi = q * page_size, min((q + 1) * page_size, cap)
            dst = perm[b, q] * page_size
            c_pages[dst:dst + hi - lo] = c_kv[b, lo:hi]
            r_pages[dst:dst + hi - lo] = k_rope[b, lo:hi]
    return c_pages, r_pages, perm.astype(np.int32)


def draw_candidates(cfg: Config, step: int = 0, depth: int = 16, k: int = 8, vocab: int = VOCAB):
    """Drafter candidates for the tree builder: per request and depth, k distinct tokens
    with log-probabilities of a Dirichlet(1) draw, sorted from the most likely; and one
    root token per request.  Returns (logp float32 [B][depth][k], tokens int32
    [B][depth][k], root int32 [B])."""
    g = np.random.default_rng([cfg.seed, 6, step])
    p = g.dirichlet(np.ones(k), size=(cfg.B, depth))
    logp = np.sort(np.log(p).astype(np.float32), axis=2)[:, :, ::-1].copy()
    toks = np.stack([np.stack([g.choice(vocab, k, replace=False) for _ in range(depth)])
                     for _ in range(cfg.B)]).astype(np.int32)
    root = g.integers(0, vocab, size=cfg.B).astype(np.int32)
    return logp, toks, root


LOGIT_NOISE_CLIP = 6.0     # noise logits lie in [-6, 6] ...
LOGIT_PLANTED = 7.0        # ... so the planted token is each row's unique maximum


def draw_logits(cfg: Config, st: StepInputs, step: int = 0, vocab: int = VOCAB) -> np.ndarray:
    """Target logits fp32 [B][n][vocab]: clipped N(0,1) noise with the step's planted
    target token (st.argmax) set above the clip, so that the greedy token after each
    node is the planted one."""
    if int(st.argmax.max()) >= vocab:
        raise ValueError("the step's tokens were drawn from a larger vocabulary")
    g = np.random.default_rng([cfg.seed, 5, step])
    B, n = st.parents.shape
    lg = g.standard_normal((B, n, vocab), dtype=np.float32)
    np.clip(lg, -LOGIT_NOISE_CLIP, LOGIT_NOISE_CLIP, out=lg)
    bi, ni = np.meshgrid(np.arange(B), np.arange(n), indexing="ij")
    lg[bi, ni, st.argmax] = LOGIT_PLANTED
    return lg


def make_workload(name_or_cfg, step: int = 0, **tree_override) -> Workload:
    """A single verify step: the cache already holds the n node latents at L_b.. L_b+n-1."""
    cfg = CONFIGS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    lens = draw_cache_lens(cfg)
    c_kv, k_rope = draw_cache(cfg, lens, cfg.n)
    st = draw_step(cfg, step, with_nodes=False, **tree_override)
    return Workload(cfg, lens, c_kv, k_rope, st)


def make_loop_state(name_or_cfg="loop") -> Workload:
    """Initial state of the multi-step loop: committed slots [0, L_b) only; step 0's inputs."""
    cfg = CONFIGS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    lens = draw_cache_lens(cfg)
    c_kv, k_rope = draw_cache(cfg, lens, 0)
    st = draw_step(cfg, 0, with_nodes=True)
    return Workload(cfg, lens, c_kv, k_rope, st)


def scaled(cfg: Config, **changes) -> Config:
    """A copy of ``cfg`` with some fields replaced (smaller parity cases of the same recipe)."""
    return dataclasses.replace(cfg, **changes)
