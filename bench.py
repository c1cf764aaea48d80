#!/usr/bin/env python
"""Tree-verify step benchmark (one B200 per process).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kd|reference]

A step is one pass of the whole verify path over one batch: node-latent write,
mask build, MLA-absorb tree attention (tensor cores), greedy accept and
compaction, for the 64-request loop workload (64 heads, 17 tree nodes, cache
lengths U[2048, 16384]).  Each rank verifies its own 64 requests (weak scaling;
no collective on the data path).  Prints one JSON line on rank 0.

``--impl reference`` times the float64 CPU oracle on a bounded sample of the
same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from tree_speculative_decoding_kd_b200 import harness as HN  # noqa: E402
from tree_speculative_decoding_kd_b200 import workload as W  # noqa: E402

METRIC = "tree-verify MLA attn TFLOP/s + KV HBM GB/s (% roofline); verify steps/s"
N_DISTINCT = 8          # distinct pre-generated step inputs, cycled


def code_sha256_16(path):
    """sha256 (first 16 hex digits) of a CUDA source with its comments and whitespace
    removed, so that it changes exactly when the code does."""
    import hashlib
    import re
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return hashlib.sha256("".join(src.split()).encode()).hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per attention launch from the committed ncu figures
    (profiles/attn_loop_traffic.json), only while the attention kernel's code is the
    one those counters were taken from (else None)."""
    prof = os.path.join(ROOT, "profiles", "attn_loop_traffic.json")
    src = os.path.join(ROOT, "tree_speculative_decoding_kd_b200", "csrc", "kd_attn_tc.cu")
    try:
        with open(prof) as f:
            d = json.load(f)
        if d["kernel_code_sha256_16"] != code_sha256_16(src):
            return None
        return int(d["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kd", "reference"], default="kd")
    ap.add_argument("--no-extras", action="store_true", help="skip the per-config attention lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--attn-only", default=None, choices=["tiny", "kimi_single", "batched", "long", "extend"],
                    help="time only the attention of one single-step configuration")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--gemm-reference", action="store_true",
                    help="with --attn-only batched/long: also time the two plain GEMMs by torch.matmul")
    ap.add_argument("--accept-logits-only", action="store_true",
                    help="time only the fused target argmax + accept on the loop workload's trees")
    ap.add_argument("--requests", type=int, default=0,
                    help="with --accept-logits-only: use the first R requests (0 = all)")
    return ap.parse_args()


def workload_cfg(rank: int, steps_total: int):
    cfg = W.CONFIGS["loop"]
    return W.scaled(cfg, seed=HN.rank_seed(cfg.seed, rank), steps=max(cfg.steps, steps_total))


def config_json(cfg):
    return {"workload": f"loop: {cfg.B} requests x {cfg.H} heads, d_c=512 d_r=64 bf16, "
                        f"{cfg.n} tree nodes (depth<=8), L~U[{cfg.L_lo},{cfg.L_hi}], "
                        "write-nodes+mask+verify+accept+compact per step",
            "requests_per_gpu": cfg.B, "heads": cfg.H, "tree_nodes": cfg.n,
            "cache_len": [cfg.L_lo, cfg.L_hi], "scale": cfg.scale,
            "l2": "inputs larger than L2 (each step reads ~0.8 GB of latent cache)",
            "step_inputs": f"{N_DISTINCT} distinct seeded step inputs cycled"}


# ====================================================================== CPU oracle
def oracle_step_sample(wl_c, wl_r, lens, st, cfg, reqs):
    """Oracle time of one step, measured on `reqs` requests' attention and
    compaction plus every request's accept, extrapolated to all requests."""
    import oracle
    from oracle.accept import tree_accept_batch
    t0 = time.perf_counter()
    vis = np.stack([oracle.visibility_words(p) for p in st.parents])
    path, ln, _ = tree_accept_batch(st.tokens, st.parents, st.argmax)
    t_all = time.perf_counter() - t0
    t1 = time.perf_counter()
    for b in reqs:
        sl = slice(b, b + 1)
        c1, r1 = oracle.kv_write_nodes(wl_c[sl], wl_r[sl], lens[sl], st.node_ckv[sl], st.node_krope[sl])
        oracle.tree_verify_attention(st.q_abs[sl], st.q_rope[sl], c1, r1, lens[sl], vis[sl], cfg.scale)
        oracle.kv_compact(c1, r1, lens[sl], path[sl], ln[sl])
    t_req = (time.perf_counter() - t1) / len(reqs)
    return t_all + t_req * cfg.B


def cpu_baseline(cfg, wl, st, budget_s=12.0):
    """The oracle as it stands, timed on this host's cores on a bounded sample."""
    threads, api = HN.blas_threads()
    reqs, times = [], []
    t_start = time.perf_counter()
    b = 0
    while b < cfg.B and (time.perf_counter() - t_start) < budget_s:
        times.append(oracle_step_sample(wl.c_kv, wl.k_rope, wl.cache_lens, st, cfg, [b]))
        reqs.append(b)
        b += 1
    sec = float(np.median(times))
    return {"value": 1.0 / sec, "unit": "verify steps/s", "cores": threads, "kind": "oracle",
            "sample": f"float64 numpy oracle ({api} BLAS): attention+node write+compaction of "
                      f"{len(reqs)} of {cfg.B} requests of step 0 (one at a time) plus accept of "
                      f"all {cfg.B}, extrapolated to the full 64-request step"}


def run_reference(args):
    rank, world, _ = HN.dist_env()
    if rank != 0:
        return
    cfg = workload_cfg(0, args.steps + args.warmup)
    threads, api = HN.blas_threads()
    wl = W.make_loop_state(cfg)
    lens = wl.cache_lens.copy()
    times, walls = [], []
    for s in range(args.warmup + args.steps):
        st = W.draw_step(cfg, s % N_DISTINCT, with_nodes=True)
        b = s % cfg.B
        w0 = time.perf_counter()
        t = oracle_step_sample(wl.c_kv, wl.k_rope, lens, st, cfg, [b])
        if s >= args.warmup:
            times.append(t)
            walls.append(time.perf_counter() - w0)
    sec = float(np.sum(times))
    value = args.steps / sec
    sample = (f"per step: one request's attention, node write and compaction (rotating) plus all "
              f"{cfg.B} accepts, timed as run ({api} BLAS); value extrapolates the one request to "
              f"{cfg.B}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "verify steps/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * float(np.sum(walls)) / args.steps,
            "extrapolated_ms_per_step": 1e3 * sec / args.steps,
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_json(cfg),
            "parallelism": "one host process (rank 0)",
            "cpu_baseline": {"value": value, "unit": "verify steps/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "verify steps/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ====================================================================== GPU path
class DeviceStep:
    """One step's inputs on the device."""

    def __init__(self, kd, st, torch):
        self.q_abs = kd.bf16_from_bits(st.q_abs)
        self.q_rope = kd.bf16_from_bits(st.q_rope)
        self.node_ckv = kd.bf16_from_bits(st.node_ckv)
        self.node_krope = kd.bf16_from_bits(st.node_krope)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()  # noqa: E731
        self.parents, self.tokens, self.argmax = i32(st.parents), i32(st.tokens), i32(st.argmax)
        self.depth = np.stack([np.asarray(_depths(p)) for p in st.parents])

    def tensors(self):
        return [self.q_abs, self.q_rope, self.node_ckv, self.node_krope, self.parents,
                self.tokens, self.argmax]


def _depths(parents):
    d = [0] * len(parents)
    for i in range(1, len(parents)):
        d[i] = d[parents[i]] + 1
    return d


class Verifier:
    """The five library calls of one verify step on persistent device buffers."""

    def __init__(self, kd, torch, cfg, c_kv, k_rope, lens):
        self.kd, self.torch, self.cfg = kd, torch, cfg
        B, n, H = cfg.B, cfg.n, cfg.H
        self.c_kv, self.k_rope, self.lens = c_kv, k_rope, lens
        dev = c_kv.device
        self.err = kd.new_error_word(dev)
        self.ws = kd.new_workspace(B, n, H, cfg.cap, 0, dev)
        self.vis = torch.empty(B, n, (n + 31) // 32, dtype=torch.int32, device=dev)
        self.depth = torch.empty(B, n, dtype=torch.int32, device=dev)
        self.out = torch.empty(B, n, H, 512, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(B, n, H, dtype=torch.float32, device=dev)
        self.path = torch.empty(B, n, dtype=torch.int32, device=dev)
        self.len = torch.empty(B, dtype=torch.int32, device=dev)
        self.bonus = torch.empty(B, dtype=torch.int32, device=dev)
        # node write, mask, attention (its split-KV merge runs inside the same launch),
        # accept, compaction
        self.launches_per_step = 5

    def step(self, s: DeviceStep, ev=None):
        kd = self.kd
        kd.kd_kv_write_nodes(self.c_kv, self.k_rope, self.lens, s.node_ckv, s.node_krope, self.err)
        kd.kd_tree_build_mask(s.parents, self.vis, self.depth, self.err)
        if ev is not None:
            ev[0].record()
        kd.kd_tree_verify_attn(s.q_abs, s.q_rope, self.c_kv, self.k_rope, self.lens, self.vis,
                               None, self.cfg.scale, self.out, self.lse, self.ws)
        if ev is not None:
            ev[1].record()
        kd.kd_tree_accept(s.tokens, s.parents, s.argmax, self.path, self.len, self.bonus, self.err)
        kd.kd_kv_compact(self.c_kv, self.k_rope, self.path, self.len, self.lens, self.err)


def attn_case(kd, torch, peaks, flush, name, reps=20, warm=3):
    """Attention-only timing of one single-step configuration (L2 flushed per rep)."""
    wl = W.make_workload(name)
    cfg, st = wl.cfg, wl.step
    qa, qr = kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope)
    ck, kr = kd.bf16_from_bits(wl.c_kv), kd.bf16_from_bits(wl.k_rope)
    lens = torch.from_numpy(wl.cache_lens.astype(np.int32)).cuda()
    parents = torch.from_numpy(st.parents).cuda()
    vis, _ = kd.kd_tree_build_mask(parents)
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cfg.cap)
    out = torch.empty(cfg.B, cfg.n, cfg.H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.n, cfg.H, dtype=torch.float32, device="cuda")

    def call():
        kd.kd_tree_verify_attn(qa, qr, ck, kr, lens, vis, None, cfg.scale, out, lse, ws)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    # the call (tensor-map encoding + launch) is captured once and replayed, so the
    # events below measure the kernels, not the Python/ctypes launch path
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    times = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    del graph
    bits = kd.kd_read_device_error(ws)
    t = float(np.median(times))
    depths = [_depths(p) for p in st.parents]
    fl = HN.attn_flops(wl.cache_lens, depths, cfg.H)
    by = HN.attn_bytes(wl.cache_lens, cfg.n, cfg.H)
    t_fl, t_by = fl / (peaks["bf16_tflops"] * 1e12), by / (peaks["hbm_gbs"] * 1e9)
    res = {"us": round(t * 1e6, 2), "us_min": round(min(times) * 1e6, 2),
           "tflops": round(fl / t / 1e12, 1), "hbm_gbs": round(by / t / 1e9, 1),
           "roofline_frac": round(max(t_fl, t_by) / t, 3), "bound": "tensor" if t_fl > t_by else "hbm",
           "splits": "auto", "timing": "CUDA-graph replay of the call, L2 flushed (256 MB write) before each rep",
           "device_errors": bits}
    del qa, qr, ck, kr, ws, out
    torch.cuda.empty_cache()
    return res


def gemm_reference(kd, torch, flush, name, reps=10, warm=2):
    """For scale: the two plain contractions of the attention, S = Q K^T (bf16 out) and
    O = S V per request, by torch.matmul (cuBLAS) on the same inputs: no mask, no softmax,
    S through memory.  Timed like attn_case (CUDA-graph replay after an L2 flush)."""
    wl = W.make_workload(name)
    cfg, st = wl.cfg, wl.step
    B, n, H = cfg.B, cfg.n, cfg.H
    bf = torch.bfloat16
    q = torch.cat([kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope)], dim=-1).reshape(B, n * H, 576)
    # key counts rounded up to 64 (zero rows past the cache), so that every operand row
    # is 16-byte aligned, as cuBLAS's tensor-core kernels want
    cap_pad = (cfg.cap + 63) // 64 * 64
    kv = torch.zeros(B, cap_pad, 576, dtype=bf, device="cuda")
    kv[:, :cfg.cap] = torch.cat([kd.bf16_from_bits(wl.c_kv), kd.bf16_from_bits(wl.k_rope)], dim=-1)
    keys = [(int(wl.cache_lens[b]) + n + 63) // 64 * 64 for b in range(B)]
    S = [torch.empty(n * H, keys[b], dtype=bf, device="cuda") for b in range(B)]
    O = [torch.empty(n * H, 512, dtype=bf, device="cuda") for b in range(B)]

    def call():
        for b in range(B):
            torch.matmul(q[b], kv[b, :keys[b]].t(), out=S[b])
            torch.matmul(S[b], kv[b, :keys[b], :512], out=O[b])

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    times = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    del graph, q, kv, S, O
    torch.cuda.empty_cache()
    t = float(np.median(times))
    flops = sum(2.0 * n * H * k * (576 + 512) for k in keys)
    return {"torch_matmul_qk_then_sv_us": round(t * 1e6, 2), "tflops": round(flops / t / 1e12, 1),
            "what": "S = Q K^T (bf16) then O = S V per request, torch.matmul (cuBLAS), no mask or "
                    "softmax, every key pair computed (keys rounded up to 64)"}


def attn_extras(kd, torch, peaks, flush):
    """Attention-only timings of the single-step configurations (parity cases), with the
    plain two-GEMM time of the large ones for scale."""
    res = {name: attn_case(kd, torch, peaks, flush, name) for name in
           ["tiny", "kimi_single", "batched", "long"]}
    for name in ("batched", "long"):
        res[name]["library_reference"] = gemm_reference(kd, torch, flush, name)
    return res


def accept_logits_case(kd, torch, peaks, name="loop", reps=10, warm=3, requests=0):
    """Target argmax fused with greedy accept (kd_tree_accept_logits) on one step of a
    configuration's trees with full-vocabulary fp32 logits; HBM bound (logits read once,
    larger than L2 at the loop workload's 64 requests, so no flush is needed)."""
    wl = W.make_workload(name)
    st = wl.step
    R = requests or wl.cfg.B
    logits = torch.from_numpy(W.draw_logits(wl.cfg, st)[:R]).cuda()
    tok = torch.from_numpy(st.tokens[:R]).cuda()
    par = torch.from_numpy(st.parents[:R]).cuda()
    B, n, V = logits.shape
    ws = kd.new_accept_workspace(B, n)
    am = torch.empty(B, n, dtype=torch.int32, device="cuda")
    path = torch.empty(B, n, dtype=torch.int32, device="cuda")
    ln = torch.empty(B, dtype=torch.int32, device="cuda")
    bonus = torch.empty(B, dtype=torch.int32, device="cuda")

    def call():
        kd.kd_tree_accept_logits(tok, par, logits, am, path, ln, bonus, ws)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    ok = bool((am.cpu().numpy() == st.argmax[:R]).all())
    t = float(np.median(times))
    nbytes = B * n * V * 4
    # for scale: PyTorch's own row reductions over the same tensor, timed the same way
    # (library kernels, outside every other timed region)
    flat = logits.view(B * n, V)
    ref = {}
    for rname, fn in (("torch_amax", lambda: torch.amax(flat, dim=-1)),
                      ("torch_argmax", lambda: torch.argmax(flat, dim=-1))):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        rt = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            rt.append(e0.elapsed_time(e1) * 1e-3)
        ref[rname + "_us"] = round(float(np.median(rt)) * 1e6, 2)
    del logits, flat
    torch.cuda.empty_cache()
    return {"workload": f"{name}: {B} requests x {n} nodes x {V} fp32 logits", "us": round(t * 1e6, 2),
            "us_min": round(min(times) * 1e6, 2), "hbm_gbs": round(nbytes / t / 1e9, 1),
            "roofline_frac": round(nbytes / t / 1e9 / peaks["hbm_gbs"], 3), "bound": "hbm",
            "bytes": nbytes, "planted_tokens_recovered": ok, "library_reference": ref,
            "timing": "CUDA events around each call; logits larger than L2, so no flush"}


def paged_attn_case(kd, torch, peaks, flush, name="batched", page_size=64, reps=20, warm=3):
    """Attention over a paged cache (the configuration's caches laid out as a shuffled
    pool of page_size-slot pages), timed like attn_case."""
    wl = W.make_workload(name)
    cfg, st = wl.cfg, wl.step
    cp, rp, pt = W.to_paged(wl.c_kv, wl.k_rope, page_size)
    qa, qr = kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope)
    gc, gr = kd.bf16_from_bits(cp), kd.bf16_from_bits(rp)
    ptab = torch.from_numpy(pt).cuda()
    lens = torch.from_numpy(wl.cache_lens.astype(np.int32)).cuda()
    vis, _ = kd.kd_tree_build_mask(torch.from_numpy(st.parents).cuda())
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, pt.shape[1] * page_size)
    out = torch.empty(cfg.B, cfg.n, cfg.H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.n, cfg.H, dtype=torch.float32, device="cuda")

    def call():
        kd.kd_tree_verify_attn_paged(qa, qr, gc, gr, ptab, page_size, lens, vis, None, cfg.scale, out, lse, ws)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    times = []
    for _ in range(reps):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    del graph
    t = float(np.median(times))
    fl = HN.attn_flops(wl.cache_lens, [_depths(p) for p in st.parents], cfg.H)
    res = {"workload": f"{name} over a shuffled pool of {page_size}-slot pages", "us": round(t * 1e6, 2),
           "us_min": round(min(times) * 1e6, 2), "tflops": round(fl / t / 1e12, 1),
           "roofline_frac": round(fl / (peaks["bf16_tflops"] * 1e12) / t, 3), "bound": "tensor",
           "device_errors": kd.kd_read_device_error(ws),
           "timing": "CUDA-graph replay of the call, L2 flushed (256 MB write) before each rep"}
    del gc, gr, ws, out
    torch.cuda.empty_cache()
    return res


def tree_build_case(kd, torch, name="loop", depth=16, k=8, reps=20, warm=3):
    """Best-first draft-tree build for every request of a configuration from drafter
    candidates (depth x k per request); launch-latency sized (one warp per request)."""
    cfg = W.CONFIGS[name]
    logp, toks, root = W.draw_candidates(cfg, depth=depth, k=k)
    lp, tk, rt = (torch.from_numpy(a).cuda() for a in (logp, toks, root))
    outs = kd.kd_tree_build(lp, tk, rt, cfg.n)              # the outputs, reused by every call

    def call():
        kd.kd_tree_build(lp, tk, rt, cfg.n, *outs)

    for _ in range(warm):
        call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    times = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1) * 1e-3)
    del graph
    return {"workload": f"{name}: {cfg.B} requests, {cfg.n} nodes from {depth} depths x {k} candidates",
            "us": round(float(np.median(times)) * 1e6, 2), "us_min": round(min(times) * 1e6, 2),
            "bound": "latency (one warp per request, one pop per node)",
            "timing": "CUDA-graph replay of the call, outputs preallocated (no L2 flush: 64 x 1 KB "
                      "of candidates)"}


def run_accept_logits_only(args):
    """--accept-logits-only: time just kd_tree_accept_logits (profiling aid)."""
    import torch
    torch.cuda.set_device(0)
    from tree_speculative_decoding_kd_b200 import kd
    peaks = HN.load_peaks(ROOT)
    res = accept_logits_case(kd, torch, peaks, reps=args.reps, warm=1, requests=args.requests)
    print(json.dumps({"accept_logits_only": True, **res}), flush=True)


def run_attn_only(args):
    """--attn-only NAME: time just the attention of one configuration (profiling aid)."""
    import torch
    torch.cuda.set_device(0)
    from tree_speculative_decoding_kd_b200 import kd
    peaks = HN.load_peaks(ROOT)
    flush = HN.L2Flush("cuda")
    res = attn_case(kd, torch, peaks, flush, args.attn_only, reps=args.reps, warm=1)
    if args.attn_only in ("batched", "long") and args.gemm_reference:
        res["library_reference"] = gemm_reference(kd, torch, flush, args.attn_only)
    print(json.dumps({"attn_only": args.attn_only, **res}), flush=True)


def run_kd(args):
    import torch

    rank, world, local = HN.dist_env()
    torch.cuda.set_device(local)
    HN.init_dist("nccl" if world > 1 else "gloo")
    from tree_speculative_decoding_kd_b200 import kd

    peaks = HN.load_peaks(ROOT)
    cfg = workload_cfg(rank, args.steps + args.warmup)
    wl = W.make_loop_state(cfg)
    host_steps = [W.draw_step(cfg, s, with_nodes=True) for s in range(N_DISTINCT)]
    dsteps = [DeviceStep(kd, st, torch) for st in host_steps]
    c0 = kd.bf16_from_bits(wl.c_kv)
    r0 = kd.bf16_from_bits(wl.k_rope)
    lens0 = torch.from_numpy(wl.cache_lens.astype(np.int32)).cuda()

    # ---------------- device-resident arm
    c_kv, k_rope, lens = c0.clone(), r0.clone(), lens0.clone()
    V = Verifier(kd, torch, cfg, c_kv, k_rope, lens)
    for s in range(args.warmup):
        V.step(dsteps[s % N_DISTINCT])
    torch.cuda.synchronize()
    # cache lengths each timed step starts from: the generator knows every
    # step's accepted length (its planted path), so no device copy is timed
    lens_np = wl.cache_lens.astype(np.int64).copy()
    step_lens, drafts = [], []
    for s in range(args.warmup + args.steps):
        planted = [len(p) for p in host_steps[s % N_DISTINCT].planted]
        if s >= args.warmup:
            step_lens.append(lens_np.copy())
            drafts += [k - 1 for k in planted]             # accepted drafts (the root excluded)
        lens_np += np.array(planted)
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    HN.barrier(local)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with HN.ClockSampler(local) as clk:
        t0.record()
        for s in range(args.steps):
            V.step(dsteps[(args.warmup + s) % N_DISTINCT], attn_ev[s])
        t1.record()
        torch.cuda.synchronize()
    HN.barrier(local)
    elapsed = t0.elapsed_time(t1) * 1e-3
    elapsed_max = HN.max_over_ranks(elapsed, torch.device("cuda", local))
    attn_times = [a.elapsed_time(b) * 1e-3 for a, b in attn_ev]
    flop_steps, byte_steps = [], []
    for s in range(args.steps):
        depths = dsteps[(args.warmup + s) % N_DISTINCT].depth
        flop_steps.append(HN.attn_flops(step_lens[s], depths, cfg.H))
        byte_steps.append(HN.attn_bytes(step_lens[s], cfg.n, cfg.H))
    assert np.array_equal(V.lens.cpu().numpy(), lens_np), "cache lengths diverged from the planted paths"
    err_bits = kd.kd_read_device_error(V.err) | kd.kd_read_device_error(V.ws)
    attn_avg = float(np.mean(attn_times))
    flop_avg, byte_avg = float(np.mean(flop_steps)), float(np.mean(byte_steps))
    steps_per_s = HN.whole_job_rate(args.steps, world, elapsed_max)

    # ---------------- end-to-end arm: host inputs copied in, results copied out, every step
    c_kv.copy_(c0)
    k_rope.copy_(r0)
    lens.copy_(lens0)
    pinned = []
    for ds in dsteps:
        pinned.append([t.cpu().pin_memory() for t in ds.tensors()])
    # two device stages: step s+1's inputs upload on a copy stream while step s computes
    stages = [DeviceStep.__new__(DeviceStep) for _ in range(2)]
    for sg in stages:
        sg.q_abs, sg.q_rope, sg.node_ckv, sg.node_krope, sg.parents, sg.tokens, \
            sg.argmax = [t.clone() for t in dsteps[0].tensors()]
    res_host = [torch.empty(cfg.B, cfg.n, dtype=torch.int32).pin_memory(),
                torch.empty(cfg.B, dtype=torch.int32).pin_memory(),
                torch.empty(cfg.B, dtype=torch.int32).pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in pinned[0])
    d2h = sum(t.numel() * t.element_size() for t in res_host)
    comp, copy_s = torch.cuda.current_stream(), torch.cuda.Stream()
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]

    def upload(s):
        k = s % 2
        copy_s.wait_event(free[k])                  # the step that last read this stage is done
        with torch.cuda.stream(copy_s):
            for dst, src in zip(stages[k].tensors(), pinned[s % N_DISTINCT]):
                dst.copy_(src, non_blocking=True)
        ready[k].record(copy_s)

    def e2e_run(first, count):
        copy_s.wait_stream(comp)
        upload(first)
        for i in range(count):
            s = first + i
            if i + 1 < count:
                upload(s + 1)
            comp.wait_event(ready[s % 2])
            V.step(stages[s % 2])
            free[s % 2].record(comp)
            for dst, src in zip(res_host, (V.path, V.len, V.bonus)):
                dst.copy_(src, non_blocking=True)

    e2e_run(0, args.warmup)
    torch.cuda.synchronize()
    HN.barrier(local)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    e2e_run(args.warmup, args.steps)
    e1.record()
    torch.cuda.synchronize()
    HN.barrier(local)
    assert np.array_equal(V.lens.cpu().numpy(), lens_np), "end-to-end arm: cache lengths diverged"
    e2e_el = HN.max_over_ranks(e0.elapsed_time(e1) * 1e-3, torch.device("cuda", local))
    e2e_rate = HN.whole_job_rate(args.steps, world, e2e_el)

    extras = None
    next_rows = None
    cpu = None
    if rank == 0 and world == 1:
        if not args.no_extras:
            extras = attn_extras(kd, torch, peaks, HN.L2Flush("cuda"))
            next_rows = {"accept_logits": accept_logits_case(kd, torch, peaks),
                         "causal_extend": attn_case(kd, torch, peaks, HN.L2Flush("cuda"), "extend"),
                         "tree_build": tree_build_case(kd, torch),
                         "paged_kv": paged_attn_case(kd, torch, peaks, HN.L2Flush("cuda"))}
        if not args.no_cpu_baseline:
            cpu = cpu_baseline(cfg, wl, host_steps[0])

    if rank == 0:
        achieved = flop_avg / attn_avg / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": profiled_traffic(),
                "traffic_source": "ncu dram__bytes_read+write of one launch of this workload "
                                  "(profiles/attn_loop_traffic.json); null if the kernel changed "
                                  "since",
                "peak_source": f"{peaks['source']} bf16 burst (cuBLAS)",
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "kernel": "attn_tc_kernel (tree-verify attention)",
                "algorithmic_flops_per_launch": flop_avg,
                "algorithmic_bytes_per_launch": byte_avg,
                "avg_launch_ms": round(attn_avg * 1e3, 4)}
        line = {"metric": METRIC, "value": round(steps_per_s, 3), "unit": "verify steps/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(elapsed_max / args.steps * 1e3, 4), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded N(0,1)/24 latents and queries, random trees, planted accepts)",
                "config": config_json(cfg),
                "parallelism": f"replicas x{world} (requests per rank)",
                "attn_tflops": round(achieved, 2),
                "attn_kv_hbm_gbs": round(byte_avg / attn_avg / 1e9, 1),
                "attn_roofline_frac": round(max(flop_avg / (peaks["bf16_tflops"] * 1e12),
                                                byte_avg / (peaks["hbm_gbs"] * 1e9)) / attn_avg, 4),
                "attn_share_of_step": round(attn_avg / (elapsed / args.steps), 4),
                "roofline": roof,
                "e2e": {"value": round(e2e_rate, 3), "unit": "verify steps/s",
                        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": V.launches_per_step * args.steps,
                "clocks": clk.summary(),
                "device_errors": err_bits,
                "accepted_drafts": {"mean": round(float(np.mean(drafts)), 3),
                                    "histogram": {str(k): int(v) for k, v in
                                                  zip(*np.unique(drafts, return_counts=True))},
                                    "source": "the timed steps' planted paths (per request and step); "
                                              "the device's cache lengths after the run equal their sums"}}
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if extras is not None:
            line["per_config_attention"] = extras
        if next_rows is not None:
            line["next_rows"] = next_rows
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


def main():
    args = parse()
    if args.accept_logits_only:
        run_accept_logits_only(args)
        return
    if args.attn_only:
        run_attn_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_kd(args)


if __name__ == "__main__":
    main()
