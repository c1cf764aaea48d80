"""Parity tolerances for the tree-verify attention output.

Attention (bf16 inputs, fp32 accumulation, bf16 output): max-abs error 1e-2 and
relative L2 error 5e-3, applied to the whole ``out`` tensor of a call and, as
a stricter reading, to every node's [H][512] block separately (a single wrong
mask bit moves one node's block by about 1/sqrt(visible keys), which a
whole-tensor norm can dilute below 5e-3).  ``lse`` (fp32): max-abs 1e-3.
Accept and compaction are compared bit-exactly.
"""
import numpy as np

OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def attn_errors(out, lse, out_ref, lse_ref):
    out = np.asarray(out, np.float64)
    out_ref = np.asarray(out_ref, np.float64)
    sel = ~np.isnan(out_ref[..., 0, 0])                  # rows the oracle computed
    o, r = out[sel], out_ref[sel]                        # [rows][H][512]
    max_abs = float(np.max(np.abs(o - r))) if o.size else 0.0
    rel = float(np.linalg.norm(o - r) / max(np.linalg.norm(r), 1e-300)) if o.size else 0.0
    d = (o - r).reshape(len(o), -1)
    rn = np.linalg.norm(r.reshape(len(r), -1), axis=1)
    node_rel = float(np.max(np.linalg.norm(d, axis=1) / np.maximum(rn, 1e-300))) if o.size else 0.0
    lsel = np.asarray(lse, np.float64)[sel]
    lref = np.asarray(lse_ref, np.float64)[sel]
    fin = np.isfinite(lref)
    lse_err = float(np.max(np.abs(lsel[fin] - lref[fin]))) if fin.any() else 0.0
    lse_inf_ok = bool(np.all(np.isneginf(lsel[~fin]))) if (~fin).any() else True
    return dict(max_abs=max_abs, rel_l2=rel, node_rel_l2=node_rel, lse_max_abs=lse_err,
                lse_inf_ok=lse_inf_ok, finite=bool(np.isfinite(o).all()))


def attn_within_tolerance(out, lse, out_ref, lse_ref):
    e = attn_errors(out, lse, out_ref, lse_ref)
    ok = (e["finite"] and e["max_abs"] <= OUT_MAX_ABS and e["rel_l2"] <= OUT_REL_L2
          and e["node_rel_l2"] <= OUT_REL_L2 and e["lse_max_abs"] <= LSE_MAX_ABS
          and e["lse_inf_ok"])
    return ok, e
