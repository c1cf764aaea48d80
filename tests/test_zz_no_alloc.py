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


def test_noalloc_matches_oracle_and_regular_bits_at_equal_splits(kd):
    """At the same explicit split count both entry points run the same units and the
    same fixed-order merge, so their outputs agree bit for bit; both against the oracle."""
    import oracle
    wl = W.make_workload("kimi_single")
    cfg, st = wl.cfg, wl.step
    d = _device_inputs(kd, wl)
    shape = (cfg.B, cfg.n, cfg.H)
    for splits in (1, 3):
        ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cfg.cap, splits)
        out_r, lse_r = kd.kd_tree_verify_attn(d["q_abs"], d["q_rope"], d["c_kv"], d["k_rope"], d["cache_lens"],
                                              d["vis"], d["positions"], cfg.scale, workspace=ws,
                                              kv_splits=splits)
        out = torch.full((*shape, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        err = kd.new_error_word()
        kd.kd_tree_verify_attn_noalloc(d["q_abs"], d["q_rope"], d["c_kv"], d["k_rope"], d["cache_lens"],
                                       d["vis"], d["positions"], cfg.scale, out, lse, splits, err)
        torch.cuda.synchronize()
        assert kd.kd_read_device_error(ws) == 0 and kd.kd_read_device_error(err) == 0
        assert torch.equal(out.view(torch.int16), out_r.view(torch.int16)), splits
        assert torch.equal(lse, lse_r), splits
        vis = np.stack([oracle.visibility_words(p) for p in st.parents])
        ro, rl = oracle.tree_verify_attention(st.q_abs, st.q_rope, wl.c_kv, wl.k_rope, wl.cache_lens, vis,
                                              cfg.scale)
        ok, e = attn_within_tolerance(_as_f32(kd, out), lse.cpu().numpy(), ro, rl)
        assert ok, (splits, e)


def test_noalloc_captured_in_a_cuda_graph(kd):
    """Captured after one warm-up call, the allocation-free entry replays on new
    inputs copied into the captured buffers, twice, bit-identical each time to the
    regular entry on those inputs at the same split count."""
    cfgs = [W.scaled(W.CONFIGS["batched"], B=3, seed=s, L_lo=1500, L_hi=2500) for s in (21, 22, 23)]
    wls = [W.make_workload(c) for c in cfgs]
    cap = max(c.cap for c in cfgs)

    def padded(wl):
        d = _device_inputs(kd, wl)
        for k in ("c_kv", "k_rope"):
            t = torch.zeros(wl.cfg.B, cap, d[k].shape[2], dtype=d[k].dtype, device="cuda")
            t[:, :d[k].shape[1]] = d[k]
            d[k] = t
        return d

    cfg, splits = cfgs[0], 2
    shape = (cfg.B, cfg.n, cfg.H)
    bufs = padded(wls[0])
    out = torch.zeros(*shape, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(shape, dtype=torch.float32, device="cuda")
    err = kd.new_error_word()
    call = lambda: kd.kd_tree_verify_attn_noalloc(bufs["q_abs"], bufs["q_rope"], bufs["c_kv"],  # noqa: E731
                                                  bufs["k_rope"], bufs["cache_lens"], bufs["vis"],
                                                  bufs["positions"], cfg.scale, out, lse, splits, err)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()                                                    # warm-up: per-device setup
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for wl in wls[1:]:
        new = padded(wl)
        for k, t in new.items():
            bufs[k].copy_(t)
        g.replay()
        ws = kd.new_workspace(cfg.B, cfg.n, cfg.H, cap, splits)
        out_r, lse_r = kd.kd_tree_verify_attn(new["q_abs"], new["q_rope"], new["c_kv"], new["k_rope"],
                                              new["cache_lens"], new["vis"], new["positions"], cfg.scale,
                                              workspace=ws, kv_splits=splits)
        torch.cuda.synchronize()
        assert kd.kd_read_device_error(err) == 0 and kd.kd_read_device_error(ws) == 0
        assert torch.equal(out.view(torch.int16), out_r.view(torch.int16))
        assert torch.equal(lse, lse_r)
    del g


def test_noalloc_lowers_the_automatic_split_to_fit(kd):
    """A shape whose automatic split count needs more scratch than the fixed array:
    with kv_splits = 0 the call lowers the count to the largest that fits (it is not
    refused) and matches the regular entry run at that count bit for bit."""
    B, n, H, L = 40, 8, 16, 32000
    cap = L + n
    lim = 32 << 20
    need = kd.kd_verify_workspace_bytes(B, n, H, cap, 0)
    if need <= lim:
        pytest.skip("automatic split fits the fixed array on this device")
    auto = next(s for s in range(1, 65) if kd.kd_verify_workspace_bytes(B, n, H, cap, s) == need)
    lowered = next(s for s in range(auto, 0, -1) if kd.kd_verify_workspace_bytes(B, n, H, cap, s) <= lim)
    assert 1 < lowered < auto
    g = torch.Generator(device="cuda").manual_seed(5)
    bf = lambda *s: (torch.randn(*s, generator=g, device="cuda") * 0.5).to(torch.bfloat16)  # noqa: E731
    q_abs, q_rope = bf(B, n, H, 512), bf(B, n, H, 64)
    c_kv, k_rope = bf(B, cap, 512), bf(B, cap, 64)
    lens = torch.full((B,), L, dtype=torch.int32, device="cuda")
    parents = torch.tensor([-1] + list(range(n - 1)), dtype=torch.int32, device="cuda").repeat(B, 1)
    vis, _ = kd.kd_tree_build_mask(parents)
    scale = 1.0 / np.sqrt(192.0)
    out = torch.empty(B, n, H, 512, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, n, H, dtype=torch.float32, device="cuda")
    err = kd.new_error_word()
    kd.kd_tree_verify_attn_noalloc(q_abs, q_rope, c_kv, k_rope, lens, vis, None, scale, out, lse, 0, err)
    ws = kd.new_workspace(B, n, H, cap, lowered)
    out_r, lse_r = kd.kd_tree_verify_attn(q_abs, q_rope, c_kv, k_rope, lens, vis, None, scale, workspace=ws,
                                          kv_splits=lowered)
    torch.cuda.synchronize()
    assert kd.kd_read_device_error(err) == 0 and kd.kd_read_device_error(ws) == 0
    assert torch.equal(out.view(torch.int16), out_r.view(torch.int16))
    assert torch.equal(lse, lse_r)
