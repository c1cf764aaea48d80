"""Timeline and wait counters of attention launches, from the trace build.

    python -m tree_speculative_decoding_kd_b200.build --trace
    python -m tree_speculative_decoding_kd_b200.trace --configs tiny,kimi_single,batched

libkdverify_trace.so is the library with the attention kernel compiled with
-DKD_TRACE: per CTA it records the global timer at fixed points of each role and
cycle counters of the main waits.  For each configuration the call is captured in a
CUDA graph and replayed (warm, and after an L2 flush); this prints, per mode, the
median replay's event time, the kernel's own span, the timeline of the cluster that
finished last, and the per-tile / per-unit wait cycles of the roles.  A replay of a
graph holding one tiny memset gives the event-timing floor (graph launch overhead).

    python -m tree_speculative_decoding_kd_b200.trace --probes

runs the delivery probes of the same library instead: bytes per SM cycle that TMA tile
loads deliver from an L2-resident window with a given number of boxes in flight, for
whole boxes per CTA and for the pair form (two CTAs each loading half of every box,
completing on the even CTA's barrier).
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os

import numpy as np
import torch

from . import harness as HN
from . import kd
from . import workload as W

# timeline slots (global timer, ns) and counter slots (SM cycles), as the kernel fills them
EVENTS = {0: "entry", 1: "setup done (barriers, TMEM, cluster sync)", 2: "teardown sync", 3: "exit (TMEM freed)",
          4: "QK producer: first unit claimed", 5: "QK producer: first Q loads issued",
          6: "QK producer: first unit published", 7: "QK producer: last K load issued",
          8: "QK MMA: first Q in TMEM", 9: "QK MMA: first K chunk landed", 10: "QK MMA: first S committed",
          11: "QK MMA: last S committed", 12: "softmax: first Q copied to TMEM", 13: "softmax: first S loaded",
          14: "softmax: first tile's P emitted", 15: "softmax: last S ready", 16: "softmax: last tile masked",
          17: "softmax: last tile's P emitted", 18: "softmax: last row statistics sent",
          19: "PV producer: first V issued", 20: "PV MMA: first P landed", 21: "PV MMA: last O complete (commit)",
          22: "epilogue: last O and statistics ready", 23: "epilogue: last unit's first O chunk read",
          24: "epilogue: last unit stored", 25: "merge: start", 26: "merge: first ticket complete",
          27: "merge: end"}
QK_COUNTERS = {32: ("QK MMA waits for S to be free", "tile"), 33: ("QK MMA waits for K stages", "tile"),
               34: ("QK MMA issue (fence, MMAs, commits)", "tile"),
               36: ("QK MMA unit start (unit decode to Q ready)", "unit"),
               37: ("QK MMA waits for Q in TMEM", "unit"), 40: ("softmax waits for S", "tile"),
               41: ("softmax emits P (two halves)", "tile"), 42: ("softmax tile total", "tile"),
               47: ("QK MMA fence after S is free (to the first K wait)", "tile"),
               48: ("QK MMA commit of S", "tile"), 49: ("QK MMA role total", "tile"),
               50: ("QK MMA waits for the next unit's schedule slot", "unit"),
               51: ("QK MMA whole tile (S wait to S commit)", "tile"), 52: ("QK MMA tile loops", "tile")}
# The whole-tile counter minus its timed parts is the time the MMA thread spends blocked between
# them, i.e. in the issue of MMAs the tensor pipe is not yet ready to accept.
PV_COUNTERS = {44: ("PV MMA waits for P", "P half-tile"), 45: ("PV MMA waits for V", "P half-tile")}
# split-KV only: the epilogue's partial store (PV CTA, per unit) and the merge (both CTAs, per
# M tile merged; slot 56 counts them)
STORE_COUNTERS = {58: "epilogue: read O, stage and issue the partial's stores",
                  59: "epilogue: wait for the partial's stores to complete, publish the ticket"}
MERGE_COUNTERS = {53: "merge: wait for the tile's ticket", 54: "merge: wait for the partial rows to land",
                  55: "merge: combine rows and store"}


def _load():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libkdverify_trace.so")
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m tree_speculative_decoding_kd_b200.build --trace`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in kd._SIGS.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    lib.kd_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    lib.kd_trace_clear.argtypes = [ctypes.c_void_p]
    lib.kd_trace_dims.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.kd_probe_l2_boxes.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.kd_probe_store.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                   ctypes.c_void_p]
    lib.kd_probe_mma.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    c, s = ctypes.c_int(), ctypes.c_int()
    lib.kd_trace_dims(ctypes.byref(c), ctypes.byref(s))
    kd.lib = lib                       # every kd.* call below runs the trace build
    return lib, c.value, s.value


def _replays(call, flush, flushed, lib, dims, reps=7):
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    runs = []
    for _ in range(reps):
        s = torch.cuda.current_stream()
        lib.kd_trace_clear(s.cuda_stream)
        torch.cuda.synchronize()
        if flushed:
            flush()                    # keeps the GPU busy while the replay is enqueued
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        tr = np.zeros(dims, np.uint64)
        lib.kd_trace_read(tr.ctypes.data, tr.nbytes)
        runs.append((e0.elapsed_time(e1) * 1e3, tr.astype(np.int64)))
    del g
    runs.sort(key=lambda r: r[0])
    return runs[len(runs) // 2]


def _summary(t_ev, tr):
    used = np.nonzero(tr[:, 0])[0]
    tr = tr[: int(used.max()) + 1]
    t0 = tr[:, 0][tr[:, 0] > 0].min()
    res = {"event_us": round(t_ev, 2), "ctas": int(len(tr)),
           "kernel_us (first entry to last exit)": round((tr[:, 3].max() - t0) / 1e3, 2)}
    last = int(np.argmax(tr[1::2, 3])) if len(tr) > 1 else 0
    tl = []
    for cta in (2 * last, 2 * last + 1):
        for i, name in EVENTS.items():
            if cta < len(tr) and tr[cta, i] > 0 and (i > 3 or cta % 2 == 0):
                tl.append((round((tr[cta, i] - t0) / 1e3, 2), ("QK CTA " if cta % 2 == 0 else "PV CTA ") + name
                           if i in (0, 1, 2, 3, 25, 26, 27) else name))
    res["timeline_us (cluster that finished last)"] = dict((n, t) for t, n in sorted(tl))
    qk, pv = tr[0::2], tr[1::2]
    tiles, units, halves = qk[:, 35].sum(), qk[:, 38].sum(), pv[:, 46].sum()
    cyc = {}
    for i, (name, per) in QK_COUNTERS.items():
        den = tiles if per == "tile" else units
        cyc[f"{name} (per {per})"] = round(float(qk[:, i].sum()) / max(den, 1), 1)
    for i, (name, per) in PV_COUNTERS.items():
        cyc[f"{name} (per {per})"] = round(float(pv[:, i].sum()) / max(halves, 1), 1)
    su, mn = pv[:, 60].sum(), tr[:, 56].sum()
    for i, name in STORE_COUNTERS.items():
        if su > 0:
            cyc[f"{name} (per unit)"] = round(float(pv[:, i].sum()) / su, 1)
    for i, name in MERGE_COUNTERS.items():
        if mn > 0:
            cyc[f"{name} (per merged M tile, per CTA)"] = round(float(tr[:, i].sum()) / mn, 1)
    res["tiles"], res["units"] = int(tiles), int(units)
    res["cycles"] = cyc
    return res


def trace_config(name, lib, dims, flush, splits=0):
    wl = W.make_workload(name)
    cfg, st = wl.cfg, wl.step
    qa, qr = kd.bf16_from_bits(st.q_abs), kd.bf16_from_bits(st.q_rope)
    ck, kr = kd.bf16_from_bits(wl.c_kv), kd.bf16_from_bits(wl.k_rope)
    lens = torch.from_numpy(wl.cache_lens.astype(np.int32)).cuda()
    vis, _ = kd.kd_tree_build_mask(torch.from_numpy(st.parents).cuda())
    ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cfg.cap, splits)
    out = torch.empty(cfg.B, cfg.n, cfg.H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(cfg.B, cfg.n, cfg.H, dtype=torch.float32, device="cuda")

    def call():
        kd.kd_tree_verify_attn(qa, qr, ck, kr, lens, vis, None, cfg.scale, out, lse, ws, kv_splits=splits)

    res = []
    for flushed in (False, True):
        t, tr = _replays(call, flush, flushed, lib, dims)
        res.append({"config": name, "splits": splits or "auto", "mode": "flushed" if flushed else "warm",
                    **_summary(t, tr)})
    bits = kd.kd_read_device_error(ws)
    if bits:
        raise RuntimeError(f"{name}: device error bits {bits:#x}")
    return res


def graph_floor(flush):
    """Event time of a replayed graph that holds one 4-byte memset."""
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = []
    for flushed in (False, True):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            z.zero_()
        ts = []
        for _ in range(7):
            torch.cuda.synchronize()
            if flushed:
                flush()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e3)
        out.append({"graph_with_one_memset": "flushed" if flushed else "warm",
                    "event_us": round(float(np.median(ts)), 2)})
        del g
    return out


def probes(lib, iters=3000):
    """Delivery of TMA tile loads from an 8 MB L2-resident window, per SM cycle."""
    rows = 8192
    buf = torch.randn(rows, 512, device="cuda").to(torch.bfloat16)
    cycles = torch.zeros(148, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = []
    # pair: 0 whole boxes (one issuing warp), 1 pair loads, 2 whole boxes from two issuing warps
    cases = [(0, 64, 16), (0, 128, 8), (0, 256, 4), (0, 256, 6),
             (2, 64, 16), (2, 128, 8), (2, 256, 4), (2, 256, 6),
             (1, 64, 24), (1, 128, 16), (1, 256, 8)]
    names = {0: "whole boxes, one issuing thread", 1: "pair: half boxes, even CTA's barrier",
             2: "whole boxes, two issuing warps"}
    for pair, box_rows, depth in cases:
        for _ in range(2):                     # the first run brings the window into L2
            cycles.zero_()
            rc = lib.kd_probe_l2_boxes(buf.data_ptr(), rows, box_rows, depth, iters, pair, cycles.data_ptr(),
                                       err.data_ptr(), torch.cuda.current_stream().cuda_stream)
            if rc != 0:
                raise RuntimeError(f"probe rc {rc}")
            torch.cuda.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError("a probe wait gave up")
        half = 2 if pair == 1 else 1
        per_cta_bytes = iters * box_rows * 128 // half
        bpc = per_cta_bytes / cycles.cpu().numpy().astype(np.float64)
        out.append({"probe": names[pair], "box_rows": box_rows, "bytes_per_load": box_rows * 128 // half,
                    "in_flight_KB_per_SM": depth * box_rows * 128 // half // 1024,
                    "B_per_SM_cycle_median": round(float(np.median(bpc)), 1),
                    "B_per_SM_cycle_min": round(float(bpc.min()), 1)})
    out += store_probes(lib)
    out += mma_probes(lib)
    return out


def mma_probes(lib, count=4096):
    """Dense FLOP per SM cycle of M=128 (or 64) K=16 bf16 MMAs from one or two issuing threads per SM."""
    cycles = torch.zeros(148, dtype=torch.int64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    cases = [(128, n, a, 1, 0) for n in (64, 128, 256) for a in (0, 1)] + \
            [(128, n, 1, 2, 0) for n in (64, 128)] + [(128, n, 1, 1, w) for n in (128, 256) for w in (4, 36)] + \
            [(64, n, 0, 1, 0) for n in (128, 256)]
    out = []
    for m, n, a_tmem, issuers, wait_every in cases:
        for _ in range(2):
            cycles.zero_()
            rc = lib.kd_probe_mma(m, n, a_tmem, issuers, count, wait_every, cycles.data_ptr(), err.data_ptr(),
                                  torch.cuda.current_stream().cuda_stream)
            if rc != 0:
                raise RuntimeError(f"mma probe rc {rc}")
            torch.cuda.synchronize()
        if int(err.item()) != 0:
            raise RuntimeError("an mma probe wait gave up")
        cyc = float(np.median(cycles.cpu().numpy().astype(np.float64)))
        out.append({"probe": "mma", "M": m, "N": n, "A": "tmem" if a_tmem else "smem", "issuers": issuers,
                    "wait_every": wait_every or None,
                    "cycles_per_mma_per_issuer": round(cyc / (count // issuers), 1),
                    "FLOP_per_SM_cycle_median": round(count * 2.0 * m * n * 16 / cyc, 0)})
    return out


def store_probes(lib):
    """Store rate of one 256 KB fp32 tile per CTA in the epilogue's pattern, per SM cycle."""
    kinds = {0: "2 KB TMA box stores (16 fp32 columns x 32 rows), 8 issuing warps",
             1: "4 KB TMA box stores (32 fp32 columns x 32 rows), 8 issuing warps",
             2: "16-byte stores, 512 contiguous bytes per warp instruction"}
    out = []
    for ctas in (54, 148):
        buf = torch.empty(ctas, 128, 512, dtype=torch.float32, device="cuda")
        cycles = torch.zeros(ctas, dtype=torch.int64, device="cuda")
        for mode in (0, 1, 2):
            for reps in (1, 8):
                for _ in range(2):
                    rc = lib.kd_probe_store(buf.data_ptr(), ctas, mode, reps, cycles.data_ptr(),
                                            torch.cuda.current_stream().cuda_stream)
                    if rc != 0:
                        raise RuntimeError(f"store probe rc {rc}")
                    torch.cuda.synchronize()
                bpc = reps * 128 * 512 * 4 / cycles.cpu().numpy().astype(np.float64)
                out.append({"probe": "store: " + kinds[mode], "storing_ctas": ctas, "tiles_per_cta": reps,
                            "cycles_median": int(np.median(cycles.cpu().numpy())),
                            "B_per_SM_cycle_median": round(float(np.median(bpc)), 1)})
        del buf
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--configs", default="tiny,kimi_single,batched")
    ap.add_argument("--probes", action="store_true", help="run the L2 delivery probes instead")
    ap.add_argument("--json", default=None, help="also write the results to this file")
    ap.add_argument("--splits", default="0",
                    help="comma-separated key-partition counts to trace each config at (0: automatic)")
    args = ap.parse_args()
    lib, ctas, slots = _load()
    if args.probes:
        res = probes(lib)
    else:
        flush = HN.L2Flush("cuda")
        res = graph_floor(flush)
        for name in args.configs.split(","):
            for sp in args.splits.split(","):
                res += trace_config(name, lib, (ctas, slots), flush, int(sp))
    for r in res:
        print(json.dumps(r))
    if args.json:
        with open(args.json, "w") as f:
            json.dump(res, f, indent=1)


if __name__ == "__main__":
    main()
