"""C-ABI boundary checks that need no GPU: the library loads, exports every
function include/kd_verify.h declares, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kd_verify.h")


@pytest.fixture(scope="module")
def lib():
    from tree_speculative_decoding_kd_b200 import build
    build.build()
    from tree_speculative_decoding_kd_b200 import kd
    return kd.lib


def declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kd_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_five_steps():
    names = declared()
    for want in ["kd_tree_build_mask", "kd_tree_verify_attn", "kd_verify_workspace_bytes",
                 "kd_tree_accept", "kd_kv_compact", "kd_kv_write_nodes", "kd_strerror",
                 "kd_read_device_error", "kd_tree_verify_attn_simt"]:
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared():
        assert hasattr(lib, name), name


def test_strerror(lib):
    assert b"invalid" in lib.kd_strerror(-1)
    assert lib.kd_strerror(0) == b"ok"
    assert b"unknown" in lib.kd_strerror(12345)


def test_workspace_bytes(lib):
    from tree_speculative_decoding_kd_b200 import kd
    # no split: control block only
    assert kd.kd_verify_workspace_bytes(1, 8, 16, 300, 1) == 256
    # control block, tickets [B * mtiles][2] int32, partial lse [S][rows], partials [S][rows][512]
    rows, mtiles = 8 * 65 * 64, -(-65 * 64 // 128)
    up = lambda x: -(-x // 256) * 256  # noqa: E731
    want = 256 + up(8 * mtiles * 8) + up(rows * 3 * 4) + rows * 3 * 512 * 4
    assert kd.kd_verify_workspace_bytes(8, 65, 64, 32833, 3) == want
    assert kd.kd_verify_workspace_bytes(8, 65, 64, 32833, 0) >= 256
    for bad in [(0, 8, 16, 300, 0), (1, 0, 16, 300, 0), (1, 129, 16, 300, 0), (1, 8, 0, 300, 0),
                (1, 8, 129, 300, 0), (1, 8, 16, 0, 0), (1, 8, 16, 300, 65), (1, 8, 16, 300, -1)]:
        assert kd.kd_verify_workspace_bytes(*bad) == 0


def test_host_validation_rejects_before_cuda(lib):
    """Null pointers and out-of-range shapes return KD_EINVAL without a device."""
    V = ctypes.c_void_p
    assert lib.kd_tree_build_mask(None, 1, 8, None, None, None, None) == -1
    assert lib.kd_tree_build_mask(V(256), 1, 0, V(512), None, None, None) == -1
    assert lib.kd_tree_build_mask(V(256), 1, 129, V(512), None, None, None) == -1
    assert lib.kd_tree_accept(None, V(16), V(16), 1, 8, V(16), V(16), V(16), None, None) == -1
    assert lib.kd_tree_accept(V(16), V(16), V(16), 0, 8, V(16), V(16), V(16), None, None) == -1
    # misaligned cache pointer, stride below the latent width, odd stride
    assert lib.kd_kv_compact(V(18), V(16), 512, 64, 10, V(16), V(16), V(16), 1, 4, None, None) == -1
    assert lib.kd_kv_compact(V(16), V(16), 500, 64, 10, V(16), V(16), V(16), 1, 4, None, None) == -1
    assert lib.kd_kv_compact(V(16), V(16), 516, 64, 10, V(16), V(16), V(16), 1, 4, None, None) == -1
    assert lib.kd_kv_write_nodes(V(16), V(16), 512, 64, 10, V(16), None, V(16), 1, 4, None, None) == -1
    args = [V(16), V(16), V(16), V(16), 512, 64, 100, V(16), V(16), None, 1, 8, 16, 0.1,
            V(16), V(16), V(256), 4096, 0, None]
    bad = list(args); bad[16] = V(16 + 128)          # workspace not 256-byte aligned
    assert lib.kd_tree_verify_attn(*bad) == -1
    bad = list(args); bad[12] = 129                  # H > 128
    assert lib.kd_tree_verify_attn(*bad) == -1
    bad = list(args); bad[13] = ctypes.c_float(0.0)  # scale must be positive
    assert lib.kd_tree_verify_attn(*bad) == -1
    bad = list(args); bad[18] = 65                   # too many splits
    assert lib.kd_tree_verify_attn(*bad) == -1
    assert lib.kd_read_device_error(None, 0, None) == -1


def test_host_validation_of_the_widened_calls(lib):
    """Fused argmax + accept, tree build and paged caches reject bad arguments on the
    host (KD_EINVAL = -1, KD_ERANGE = -2) without a device."""
    from tree_speculative_decoding_kd_b200 import kd
    V = ctypes.c_void_p
    # accept workspace: 8 B ranks per node, 4 B counters per request (16-byte aligned), tokens
    assert kd.lib.kd_accept_workspace_bytes(2, 17) == 288 + 2 * 17 * 4
    assert kd.lib.kd_accept_workspace_bytes(0, 17) == 0 and kd.lib.kd_accept_workspace_bytes(1, 129) == 0
    ok = [V(16), V(16), V(16), 2, 17, 163840, None, V(16), V(16), V(16), V(256), 4096, None, None]
    bad = list(ok); bad[5] = 163842                  # vocabulary not a multiple of 4
    assert lib.kd_tree_accept_logits(*bad) == -1
    bad = list(ok); bad[2] = V(24)                   # logits not 16-byte aligned
    assert lib.kd_tree_accept_logits(*bad) == -1
    bad = list(ok); bad[10] = None                   # no workspace
    assert lib.kd_tree_accept_logits(*bad) == -1
    bad = list(ok); bad[11] = 100                    # workspace too small
    assert lib.kd_tree_accept_logits(*bad) == -2
    # tree build: shapes, and enough candidate nodes for n
    tb = [V(16), V(16), V(16), 2, 16, 8, 17, V(16), V(16), None, None, None]
    for i, v in ((5, 0), (5, 256), (6, 129), (4, 0), (0, None)):
        bad = list(tb); bad[i] = v
        assert lib.kd_tree_build(*bad) == -1
    bad = list(tb); bad[4], bad[5], bad[6] = 1, 2, 4  # 2 candidate nodes, 3 needed
    assert lib.kd_tree_build(*bad) == -1
    # paged attention: page size, page table, slice limit
    pa = [V(16), V(16), V(16), V(16), 512, 64, 64, V(16), 100, 1000, V(16), V(16), None, 1, 8, 16, 0.1,
          V(16), V(16), V(256), 1 << 20, 0, None]
    for i, v in ((6, 100), (7, None), (8, 2048), (9, 0)):
        bad = list(pa); bad[i] = v
        assert lib.kd_tree_verify_attn_paged(*bad) == -1
    # paged node write / compaction
    pw = [V(16), V(16), 512, 64, 16, V(16), 10, 100, V(16), V(16), V(16), 1, 8, None, None]
    for i, v in ((5, None), (4, 0), (7, 0)):
        bad = list(pw); bad[i] = v
        assert lib.kd_kv_write_nodes_paged(*bad) == -1
    pc = [V(16), V(16), 512, 64, 16, V(16), 10, 100, V(16), V(16), V(16), 1, 8, None, None]
    for i, v in ((5, None), (4, 0), (6, 0)):
        bad = list(pc); bad[i] = v
        assert lib.kd_kv_compact_paged(*bad) == -1
