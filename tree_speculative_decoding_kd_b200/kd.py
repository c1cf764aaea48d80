"""ctypes binding of libkdverify.so (declared in include/kd_verify.h).

Argument marshalling only: shape/dtype checks, ``data_ptr()``s, the current
CUDA stream.  Every step of the verify path runs in the library's kernels.
Importing this module raises if the library has not been built.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkdverify.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python -m tree_speculative_decoding_kd_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_sz = ctypes.c_size_t

_SIGS = {
    "kd_tree_build_mask": (_i, [_p, _i, _i, _p, _p, _p, _p]),
    "kd_verify_workspace_bytes": (_sz, [_i, _i, _i, _i64, _i]),
    "kd_tree_verify_attn": (_i, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i, _f,
                                 _p, _p, _p, _sz, _i, _p]),
    "kd_tree_verify_attn_simt": (_i, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i,
                                      _f, _p, _p, _p, _p]),
    "kd_tree_verify_attn_noalloc": (_i, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p, _i, _i, _i,
                                         _f, _p, _p, _i, _p, _p]),
    "kd_tree_accept": (_i, [_p, _p, _p, _i, _i, _p, _p, _p, _p, _p]),
    "kd_accept_workspace_bytes": (_sz, [_i, _i]),
    "kd_tree_build": (_i, [_p, _p, _p, _i, _i, _i, _i, _p, _p, _p, _p, _p]),
    "kd_tree_verify_attn_paged": (_i, [_p, _p, _p, _p, _i64, _i64, _i, _p, _i64, _i64, _p, _p, _p, _i,
                                       _i, _i, _f, _p, _p, _p, _sz, _i, _p]),
    "kd_kv_write_nodes_paged": (_i, [_p, _p, _i64, _i64, _i, _p, _i64, _i64, _p, _p, _p, _i, _i, _p,
                                     _p]),
    "kd_kv_compact_paged": (_i, [_p, _p, _i64, _i64, _i, _p, _i64, _i64, _p, _p, _p, _i, _i, _p, _p]),
    "kd_tree_accept_logits": (_i, [_p, _p, _p, _i, _i, _i64, _p, _p, _p, _p, _p, _sz, _p, _p]),
    "kd_kv_compact": (_i, [_p, _p, _i64, _i64, _i64, _p, _p, _p, _i, _i, _p, _p]),
    "kd_kv_write_nodes": (_i, [_p, _p, _i64, _i64, _i64, _p, _p, _p, _i, _i, _p, _p]),
    "kd_read_device_error": (_i, [_p, _i, _p]),
    "kd_strerror": (ctypes.c_char_p, [_i]),
}
for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args

D_C, D_R = 512, 64
KD_DEV_BITS = {0x01: "BAD_PARENT", 0x02: "CACHE_FULL", 0x04: "BAD_PATH",
               0x08: "BAD_POSITION", 0x10: "TIMEOUT", 0x20: "BAD_MASK", 0x40: "BAD_PAGE"}


class KdError(RuntimeError):
    pass


def _check(rc: int, what: str) -> None:
    if rc != 0:
        raise KdError(f"{what}: {lib.kd_strerror(rc).decode()} (code {rc})")


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, contiguous=True):
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    dts = dtype if isinstance(dtype, tuple) else (dtype,)
    if t.dtype not in dts:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dts}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _cache_strides(c_kv, k_rope):
    """Row strides (elements) of [B][cap][512] / [B][cap][64] cache views."""
    _need(c_kv, torch.bfloat16, "c_kv", contiguous=False)
    _need(k_rope, torch.bfloat16, "k_rope", contiguous=False)
    B, cap, dc = c_kv.shape
    if dc != D_C or tuple(k_rope.shape) != (B, cap, D_R):
        raise ValueError("c_kv must be [B][cap][512] and k_rope [B][cap][64]")
    for t in (c_kv, k_rope):
        if t.stride(2) != 1 or t.stride(0) != cap * t.stride(1):
            raise ValueError("cache rows must be unit-stride with uniform row pitch")
    return c_kv.stride(1), k_rope.stride(1), cap


def new_error_word(device=None) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def kd_tree_build_mask(parents, vis=None, depth=None, dev_error=None, stream=None):
    _need(parents, torch.int32, "parents")
    B, n = parents.shape
    W = (n + 31) // 32
    if vis is None:
        vis = torch.empty(B, n, W, dtype=torch.int32, device=parents.device)
    if depth is None:
        depth = torch.empty(B, n, dtype=torch.int32, device=parents.device)
    _check(lib.kd_tree_build_mask(_ptr(parents), B, n, _ptr(vis), _ptr(depth), _ptr(dev_error),
                                  _stream(stream)), "kd_tree_build_mask")
    return vis, depth


def kd_verify_workspace_bytes(B, n, H, cap, kv_splits=0) -> int:
    return int(lib.kd_verify_workspace_bytes(B, n, H, cap, kv_splits))


def new_workspace(B, n, H, cap, kv_splits=0, device=None) -> torch.Tensor:
    """Zeroed workspace (its first int32 is the device error word)."""
    nbytes = kd_verify_workspace_bytes(B, n, H, cap, kv_splits)
    if nbytes == 0:
        raise ValueError("invalid shape for the verify workspace")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or "cuda")


def _attn_args(q_abs, q_rope, c_kv, k_rope, cache_lens, vis, positions, out, lse):
    _need(q_abs, torch.bfloat16, "q_abs")
    _need(q_rope, torch.bfloat16, "q_rope")
    _need(cache_lens, torch.int32, "cache_lens")
    _need(vis, (torch.int32, torch.uint32), "vis")
    B, n, H, dc = q_abs.shape
    if dc != D_C or tuple(q_rope.shape) != (B, n, H, D_R):
        raise ValueError("q_abs must be [B][n][H][512] and q_rope [B][n][H][64]")
    if positions is not None:
        _need(positions, torch.int32, "positions")
    sc, sr, cap = _cache_strides(c_kv, k_rope)
    if out is None:
        out = torch.empty(B, n, H, D_C, dtype=torch.bfloat16, device=q_abs.device)
    if lse is None:
        lse = torch.empty(B, n, H, dtype=torch.float32, device=q_abs.device)
    _need(out, torch.bfloat16, "out")
    _need(lse, torch.float32, "lse")
    return B, n, H, sc, sr, cap, out, lse


def kd_tree_verify_attn(q_abs, q_rope, c_kv, k_rope, cache_lens, vis, positions=None,
                        scale=1.0 / math.sqrt(192.0), out=None, lse=None, workspace=None,
                        kv_splits=0, stream=None):
    B, n, H, sc, sr, cap, out, lse = _attn_args(q_abs, q_rope, c_kv, k_rope, cache_lens, vis,
                                                positions, out, lse)
    if workspace is None:
        workspace = new_workspace(B, n, H, cap, kv_splits, q_abs.device)
    _check(lib.kd_tree_verify_attn(_ptr(q_abs), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope), sc, sr,
                                   cap, _ptr(cache_lens), _ptr(vis), _ptr(positions), B, n, H,
                                   float(scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), int(kv_splits),
                                   _stream(stream)), "kd_tree_verify_attn")
    return out, lse


def kd_tree_verify_attn_noalloc(q_abs, q_rope, c_kv, k_rope, cache_lens, vis, positions=None,
                                scale=1.0 / math.sqrt(192.0), out=None, lse=None, kv_splits=0,
                                dev_error=None, stream=None):
    """kd_tree_verify_attn with the library's fixed workspace.

    The C call allocates no device memory.  This wrapper does when `out` or `lse`
    is None (it creates them with torch); under CUDA graph capture or on an
    allocation-free path pass both, and `dev_error`, preallocated.  With
    `dev_error` None the call's device errors are discarded."""
    B, n, H, sc, sr, cap, out, lse = _attn_args(q_abs, q_rope, c_kv, k_rope, cache_lens, vis,
                                                positions, out, lse)
    _check(lib.kd_tree_verify_attn_noalloc(_ptr(q_abs), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope), sc,
                                           sr, cap, _ptr(cache_lens), _ptr(vis), _ptr(positions),
                                           B, n, H, float(scale), _ptr(out), _ptr(lse),
                                           int(kv_splits), _ptr(dev_error), _stream(stream)),
           "kd_tree_verify_attn_noalloc")
    return out, lse


def kd_tree_verify_attn_simt(q_abs, q_rope, c_kv, k_rope, cache_lens, vis, positions=None,
                             scale=1.0 / math.sqrt(192.0), out=None, lse=None, dev_error=None,
                             stream=None):
    B, n, H, sc, sr, cap, out, lse = _attn_args(q_abs, q_rope, c_kv, k_rope, cache_lens, vis,
                                                positions, out, lse)
    _check(lib.kd_tree_verify_attn_simt(_ptr(q_abs), _ptr(q_rope), _ptr(c_kv), _ptr(k_rope), sc,
                                        sr, cap, _ptr(cache_lens), _ptr(vis), _ptr(positions), B,
                                        n, H, float(scale), _ptr(out), _ptr(lse),
                                        _ptr(dev_error), _stream(stream)),
           "kd_tree_verify_attn_simt")
    return out, lse


def kd_tree_build(logp, cand_tokens, root_tokens, n, parents=None, tokens=None, depth=None, score=None,
                  stream=None):
    """Best-first draft trees: logp fp32 [B][D][K] (sorted per depth), cand_tokens int32
    [B][D][K], root_tokens int32 [B] -> (parents, tokens, depth, score), each [B][n]
    (allocated here unless given)."""
    _need(logp, torch.float32, "logp")
    _need(cand_tokens, torch.int32, "cand_tokens")
    _need(root_tokens, torch.int32, "root_tokens")
    B, D, K = logp.shape
    if tuple(cand_tokens.shape) != (B, D, K) or tuple(root_tokens.shape) != (B,):
        raise ValueError("cand_tokens must be [B][D][K] and root_tokens [B]")
    dev = logp.device
    if parents is None:
        parents = torch.empty(B, n, dtype=torch.int32, device=dev)
    if tokens is None:
        tokens = torch.empty(B, n, dtype=torch.int32, device=dev)
    if depth is None:
        depth = torch.empty(B, n, dtype=torch.int32, device=dev)
    if score is None:
        score = torch.empty(B, n, dtype=torch.float32, device=dev)
    for t, dt, name in ((parents, torch.int32, "parents"), (tokens, torch.int32, "tokens"),
                        (depth, torch.int32, "depth"), (score, torch.float32, "score")):
        _need(t, dt, name)
        if tuple(t.shape) != (B, n):
            raise ValueError(f"{name} must be [B][n]")
    _check(lib.kd_tree_build(_ptr(logp), _ptr(cand_tokens), _ptr(root_tokens), B, D, K, n,
                             _ptr(parents), _ptr(tokens), _ptr(depth), _ptr(score), _stream(stream)),
           "kd_tree_build")
    return parents, tokens, depth, score


def new_accept_workspace(B, n, device=None) -> torch.Tensor:
    nbytes = int(lib.kd_accept_workspace_bytes(B, n))
    if nbytes == 0:
        raise KdError("kd_accept_workspace_bytes: invalid shapes")
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


def kd_tree_accept_logits(node_tokens, parents, logits, target_argmax=None, path=None,
                          length=None, bonus=None, workspace=None, dev_error=None, stream=None):
    """Target argmax of fp32 logits [B][n][V] fused with greedy acceptance.
    Returns (target_argmax, path, len, bonus)."""
    for t, nm in ((node_tokens, "node_tokens"), (parents, "parents")):
        _need(t, torch.int32, nm)
    _need(logits, torch.float32, "logits")
    B, n = parents.shape
    if logits.dim() != 3 or tuple(logits.shape[:2]) != (B, n):
        raise ValueError("logits must be [B][n][V]")
    V = logits.shape[2]
    dev = parents.device
    if target_argmax is None:
        target_argmax = torch.empty(B, n, dtype=torch.int32, device=dev)
    path = torch.empty(B, n, dtype=torch.int32, device=dev) if path is None else path
    length = torch.empty(B, dtype=torch.int32, device=dev) if length is None else length
    bonus = torch.empty(B, dtype=torch.int32, device=dev) if bonus is None else bonus
    workspace = new_accept_workspace(B, n, dev) if workspace is None else workspace
    _check(lib.kd_tree_accept_logits(_ptr(node_tokens), _ptr(parents), _ptr(logits), B, n, V,
                                     _ptr(target_argmax), _ptr(path), _ptr(length), _ptr(bonus),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _ptr(dev_error), _stream(stream)), "kd_tree_accept_logits")
    return target_argmax, path, length, bonus


def kd_tree_accept(node_tokens, parents, target_argmax, path=None, length=None, bonus=None,
                   dev_error=None, stream=None):
    for t, nm in ((node_tokens, "node_tokens"), (parents, "parents"), (target_argmax, "target_argmax")):
        _need(t, torch.int32, nm)
    B, n = parents.shape
    dev = parents.device
    path = torch.empty(B, n, dtype=torch.int32, device=dev) if path is None else path
    length = torch.empty(B, dtype=torch.int32, device=dev) if length is None else length
    bonus = torch.empty(B, dtype=torch.int32, device=dev) if bonus is None else bonus
    _check(lib.kd_tree_accept(_ptr(node_tokens), _ptr(parents), _ptr(target_argmax), B, n,
                              _ptr(path), _ptr(length), _ptr(bonus), _ptr(dev_error),
                              _stream(stream)), "kd_tree_accept")
    return path, length, bonus


def kd_kv_compact(c_kv, k_rope, path, length, cache_lens, dev_error=None, stream=None):
    sc, sr, cap = _cache_strides(c_kv, k_rope)
    _need(path, torch.int32, "path")
    _need(length, torch.int32, "len")
    _need(cache_lens, torch.int32, "cache_lens")
    B, n = path.shape
    _check(lib.kd_kv_compact(_ptr(c_kv), _ptr(k_rope), sc, sr, cap, _ptr(path), _ptr(length),
                             _ptr(cache_lens), B, n, _ptr(dev_error), _stream(stream)),
           "kd_kv_compact")


def kd_kv_write_nodes(c_kv, k_rope, cache_lens, node_ckv, node_krope, dev_error=None, stream=None):
    sc, sr, cap = _cache_strides(c_kv, k_rope)
    _need(node_ckv, torch.bfloat16, "node_ckv")
    _need(node_krope, torch.bfloat16, "node_krope")
    _need(cache_lens, torch.int32, "cache_lens")
    B, n, _ = node_ckv.shape
    _check(lib.kd_kv_write_nodes(_ptr(c_kv), _ptr(k_rope), sc, sr, cap, _ptr(cache_lens),
                                 _ptr(node_ckv), _ptr(node_krope), B, n, _ptr(dev_error),
                                 _stream(stream)), "kd_kv_write_nodes")


def _page_args(c_pages, r_pages, page_table, page_size):
    """Strides, pages per request and pool size of a paged cache: pools [rows][512] /
    [rows][64] bf16 (rows = num_pages * page_size), page_table int32 [B][M]."""
    _need(c_pages, torch.bfloat16, "c_pages", contiguous=False)
    _need(r_pages, torch.bfloat16, "r_pages", contiguous=False)
    _need(page_table, torch.int32, "page_table")
    rows = c_pages.shape[0]
    if c_pages.dim() != 2 or c_pages.shape[1] != D_C or tuple(r_pages.shape) != (rows, D_R):
        raise ValueError("c_pages must be [rows][512] and r_pages [rows][64]")
    if rows % page_size:
        raise ValueError("pool rows must be a multiple of page_size")
    for t in (c_pages, r_pages):
        if t.stride(1) != 1:
            raise ValueError("pool rows must be unit-stride")
    return c_pages.stride(0), r_pages.stride(0), page_table.shape[1], rows // page_size


def kd_tree_verify_attn_paged(q_abs, q_rope, c_pages, r_pages, page_table, page_size, cache_lens, vis,
                              positions=None, scale=1.0 / math.sqrt(192.0), out=None, lse=None,
                              workspace=None, kv_splits=0, stream=None):
    sc, sr, M, N = _page_args(c_pages, r_pages, page_table, page_size)
    _need(q_abs, torch.bfloat16, "q_abs")
    _need(q_rope, torch.bfloat16, "q_rope")
    _need(cache_lens, torch.int32, "cache_lens")
    _need(vis, (torch.int32, torch.uint32), "vis")
    B, n, H, _ = q_abs.shape
    if positions is not None:
        _need(positions, torch.int32, "positions")
    out = torch.empty(B, n, H, D_C, dtype=torch.bfloat16, device=q_abs.device) if out is None else out
    lse = torch.empty(B, n, H, dtype=torch.float32, device=q_abs.device) if lse is None else lse
    if workspace is None:
        workspace = new_workspace(B, n, H, M * page_size, kv_splits, q_abs.device)
    _check(lib.kd_tree_verify_attn_paged(_ptr(q_abs), _ptr(q_rope), _ptr(c_pages), _ptr(r_pages), sc, sr,
                                         int(page_size), _ptr(page_table), M, N, _ptr(cache_lens),
                                         _ptr(vis), _ptr(positions), B, n, H, float(scale), _ptr(out),
                                         _ptr(lse), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), int(kv_splits),
                                         _stream(stream)), "kd_tree_verify_attn_paged")
    return out, lse


def kd_kv_write_nodes_paged(c_pages, r_pages, page_table, page_size, cache_lens, node_ckv, node_krope,
                            dev_error=None, stream=None):
    sc, sr, M, N = _page_args(c_pages, r_pages, page_table, page_size)
    _need(node_ckv, torch.bfloat16, "node_ckv")
    _need(node_krope, torch.bfloat16, "node_krope")
    _need(cache_lens, torch.int32, "cache_lens")
    B, n, _ = node_ckv.shape
    _check(lib.kd_kv_write_nodes_paged(_ptr(c_pages), _ptr(r_pages), sc, sr, int(page_size),
                                       _ptr(page_table), M, N, _ptr(cache_lens), _ptr(node_ckv),
                                       _ptr(node_krope), B, n, _ptr(dev_error), _stream(stream)),
           "kd_kv_write_nodes_paged")


def kd_kv_compact_paged(c_pages, r_pages, page_table, page_size, path, length, cache_lens, dev_error=None,
                        stream=None):
    sc, sr, M, N = _page_args(c_pages, r_pages, page_table, page_size)
    _need(path, torch.int32, "path")
    _need(length, torch.int32, "len")
    _need(cache_lens, torch.int32, "cache_lens")
    B, n = path.shape
    _check(lib.kd_kv_compact_paged(_ptr(c_pages), _ptr(r_pages), sc, sr, int(page_size), _ptr(page_table),
                                   M, N, _ptr(path), _ptr(length), _ptr(cache_lens), B, n,
                                   _ptr(dev_error), _stream(stream)), "kd_kv_compact_paged")


def kd_read_device_error(word, clear=True, stream=None) -> int:
    """Device error bits from an error word or a verify workspace (its first int32)."""
    rc = lib.kd_read_device_error(_ptr(word), int(bool(clear)), _stream(stream))
    if rc < 0:
        _check(rc, "kd_read_device_error")
    return rc


def decode_device_error(bits: int) -> list:
    return [name for bit, name in KD_DEV_BITS.items() if bits & bit]


# ------------------------------------------------------------------ host <-> device helpers
def bf16_from_bits(u16, device="cuda") -> torch.Tensor:
    """numpy uint16 bf16 bit patterns -> bf16 tensor on ``device``."""
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(u16).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def bits_from_bf16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (on the host)."""
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
