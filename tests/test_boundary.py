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
    rows = 8 * 65 * 64
    want = 256 + ((rows * 3 * 4 + 255) // 256) * 256 + rows * 3 * 512 * 4
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
