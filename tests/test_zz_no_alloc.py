"""The allocation-free verify entry point against the regular one.

kd_tree_verify_attn_noalloc serves callers that cannot allocate device memory
when they verify (graph capture, allocator-free serving loops, C hosts without a
device allocator): it runs the same attention with the library's own fixed
workspace.  Two calls in a row, on different inputs, must each match the regular
entry point (which uses a caller-allocated workspace) within the parity
tolerance, so the shared array's leftovers from one call cannot leak into the
next.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from tests.tolerances import attn_within_tolerance
from tree_speculative_decoding_kd_b200 import workload as W

pytestmark = pytest.mark.gpu


def _device_inputs(kd, wl):
    import oracle
    st = wl.step
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()  # noqa: E731
    vis = np.stack([oracle.visibility_words(p) for p in st.parents])
    depth = np.stack([oracle.depths(p) for p in st.parents])
    return dict(q_abs=kd.bf16_from_bits(st.q_abs), q_rope=kd.bf16_from_bits(st.q_rope),
                c_kv=kd.bf16_from_bits(wl.c_kv), k_rope=kd.bf16_from_bits(wl.k_rope),
                cache_lens=i32(wl.cache_lens), vis=torch.from_numpy(vis.view(np.int32)).cuda(),
                positions=i32(wl.cache_lens[:, None] + depth))


def _as_f32(kd, t):
    return (kd.bits_from_bf16(t).astype(np.uint32) << 16).view(np.float32)


def test_noalloc_matches_regular_entry_two_calls(kd):
    # kimi-shaped single request: the automatic policy splits the keys, so the
    # fixed array really carries split-KV partials; then a 3-request batch
    cases = [W.make_workload("kimi_single"),
             W.make_workload(W.scaled(W.CONFIGS["batched"], B=3, seed=9))]
    runs = []
    for wl in cases:                                # regular entry point first
        cfg = wl.cfg
        d = _device_inputs(kd, wl)
        shape = (cfg.B, cfg.n, cfg.H)
        out_ref = torch.empty(*shape, 512, dtype=torch.bfloat16, device="cuda")
        lse_ref = torch.empty(*shape, dtype=torch.float32, device="cuda")
        ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cfg.cap)
        kd.kd_tree_verify_attn(d["q_abs"], d["q_rope"], d["c_kv"], d["k_rope"], d["cache_lens"],
                               d["vis"], d["positions"], cfg.scale, out_ref, lse_ref, ws)
        out = torch.full((*shape, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        runs.append((cfg, d, ws, out_ref, lse_ref, out, lse, kd.new_error_word()))
    torch.cuda.synchronize()
    for cfg, d, ws, out_ref, lse_ref, out, lse, err in runs:   # then two calls in a row
        kd.kd_tree_verify_attn_noalloc(d["q_abs"], d["q_rope"], d["c_kv"], d["k_rope"],
                                       d["cache_lens"], d["vis"], d["positions"], cfg.scale, out,
                                       lse, 0, err)
    torch.cuda.synchronize()
    for cfg, d, ws, out_ref, lse_ref, out, lse, err in runs:
        assert kd.kd_read_device_error(ws) == 0
        assert kd.kd_read_device_error(err) == 0
        ok, e = attn_within_tolerance(_as_f32(kd, out), lse.cpu().numpy(),
                                      _as_f32(kd, out_ref).astype(np.float64),
                                      lse_ref.cpu().numpy().astype(np.float64))
        assert ok, (cfg.name, e)


def test_noalloc_rejects_oversized_split_request(kd):
    cfg = W.CONFIGS["long"]
    need = kd.kd_verify_workspace_bytes(cfg.B, cfg.n, cfg.H, cfg.cap, 64)
    assert need > (32 << 20)
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = kd.lib.kd_tree_verify_attn_noalloc(z.data_ptr(), z.data_ptr(), z.data_ptr(), z.data_ptr(),
                                            512, 64, cfg.cap, z.data_ptr(), z.data_ptr(), None,
                                            cfg.B, cfg.n, cfg.H, 0.1, z.data_ptr(), z.data_ptr(),
                                            64, None, None)
    assert rc == -2                                          # KD_ERANGE, nothing enqueued
    assert b"workspace" in kd.lib.kd_strerror(rc)
