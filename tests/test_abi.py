"""CPU checks of the C ABI: the library loads, exports every entry point that
include/ckv.h declares, and rejects bad arguments on the host before touching
the GPU (these calls launch nothing, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

from semantic_cluster_recall_b200 import build, ckv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ckv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ckv_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return ckv.load()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 15
    assert sorted(ckv.EXPORTS) == names
    for n in names:
        assert hasattr(lib, n), n


def test_no_torch_types_in_header():
    src = open(os.path.join(ROOT, "include", "ckv.h")).read()
    assert "torch" not in src.lower().replace("pytorch", "")
    assert 'extern "C"' in src


def test_status_strings(lib):
    assert lib.ckv_status_string(0) == b"ok"
    assert lib.ckv_status_string(1) == b"invalid argument"
    assert lib.ckv_version() >= 1


def test_workspace_sizes(lib):
    assert ckv.ckv_cluster_workspace_bytes(32, 32688, 400) == 32 * 400 * 16 * 4
    assert ckv.ckv_cluster_workspace_bytes(0, 10, 10) == 0
    # L2 adds the [P][C] fp32 bias, 256-byte aligned; the others need nothing more
    base = ckv.ckv_cluster_workspace_bytes(32, 32688, 400)
    assert ckv.ckv_cluster_ex_workspace_bytes(32, 32688, 400, "cos") == base
    assert ckv.ckv_cluster_ex_workspace_bytes(32, 32688, 400, "ip") == base
    assert ckv.ckv_cluster_ex_workspace_bytes(32, 32688, 400, "l2") == base + 32 * 400 * 4
    assert ckv.load().ckv_cluster_ex_workspace_bytes(32, 32688, 400, 7) == 0
    assert ckv.ckv_select_workspace_bytes(32, 404) % 256 == 0
    assert ckv.ckv_decode_workspace_bytes(32, 1, 128, 1104) > 0
    assert ckv.ckv_decode_workspace_bytes(32, 1, 64, 1104) == 0


def _expect_invalid(status):
    assert status == ckv.CKV_ERR_INVALID, status
    assert ckv.load().ckv_last_error()


def test_validation_rejects_bad_arguments_without_launching(lib):
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: validation fails first
    null = None
    # null keys
    _expect_invalid(lib.ckv_cluster(null, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 0, 0, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None))
    # d != 128
    _expect_invalid(lib.ckv_cluster(fake, 1, 2, 64 * 100, 64, 0, 100, 4, 2, 0, 0, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None))
    # more clusters than tokens
    _expect_invalid(lib.ckv_cluster(fake, 1, 2, 128 * 100, 128, 0, 3, 4, 2, 0, 0, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None))
    # iters < 1
    _expect_invalid(lib.ckv_cluster(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 0, 0, 0, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None))
    # cluster capacity exceeded
    _expect_invalid(lib.ckv_cluster(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 6, 0, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None))
    # perm capacity exceeded
    _expect_invalid(lib.ckv_cluster(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 0, 50, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20, None))
    # workspace too small
    _expect_invalid(lib.ckv_cluster(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 0, 0, 8, 100,
                                    fake, fake, fake, fake, fake, fake, fake, fake, 16, None))
    # clustering with a similarity / in the background: unknown metric, negative
    # SM cap, an L2 workspace without room for the bias, and ckv_cluster's checks
    _expect_invalid(lib.ckv_cluster_ex(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 0, 0, 8, 100,
                                       fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20,
                                       3, 0, None))
    _expect_invalid(lib.ckv_cluster_ex(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 0, 0, 8, 100,
                                       fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20,
                                       0, -1, None))
    ws_cos = ckv.ckv_cluster_workspace_bytes(2, 100, 4)
    _expect_invalid(lib.ckv_cluster_ex(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 2, 0, 0, 8, 100,
                                       fake, fake, fake, fake, fake, fake, fake, fake, ws_cos,
                                       2, 0, None))
    _expect_invalid(lib.ckv_cluster_ex(fake, 1, 2, 128 * 100, 128, 0, 3, 4, 2, 0, 0, 8, 100,
                                       fake, fake, fake, fake, fake, fake, fake, fake, 1 << 20,
                                       1, 16, None))
    # stage calls with a similarity: unknown metric, L2 without a bias array
    _expect_invalid(lib.ckv_init_centroids_ex(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 0, 8,
                                              fake, fake, fake, 5, fake, None))
    _expect_invalid(lib.ckv_init_centroids_ex(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 0, 8,
                                              fake, fake, fake, 2, None, None))
    _expect_invalid(lib.ckv_update_ex(fake, 1, 2, 128 * 100, 128, 0, 100, 4, 0, 8, fake, fake,
                                      100, fake, fake, fake, fake, 2, None, None))
    # timeout self-test: a bound above one second
    _expect_invalid(lib.ckv_selftest_timeout(2_000_000, None))
    # unknown dtype
    _expect_invalid(lib.ckv_assign(fake, 7, 2, 128 * 100, 128, 0, 100, fake, 4, 0, 8, fake, 0,
                                   100, None))
    # negative budget, G out of range
    _expect_invalid(lib.ckv_select(fake, 1, 2, 1, 128, fake, fake, 8, fake, fake, 100, -1, fake,
                                   fake, fake, 1 << 20, None))
    _expect_invalid(lib.ckv_select(fake, 1, 2, 9, 128, fake, fake, 8, fake, fake, 100, 10, fake,
                                   fake, fake, 1 << 20, None))
    # decode: G not a power of two, bad scale, stride too small
    _expect_invalid(lib.ckv_sparse_decode(fake, fake, fake, 1, 2, 3, 128, 128 * 100, 100, 4,
                                          fake, fake, 10, fake, fake, 10, 0.088, fake, fake,
                                          1 << 20, None))
    _expect_invalid(lib.ckv_sparse_decode(fake, fake, fake, 1, 2, 1, 128, 128 * 100, 100, 4,
                                          fake, fake, 10, fake, fake, 10, -1.0, fake, fake,
                                          1 << 20, None))
    _expect_invalid(lib.ckv_sparse_decode(fake, fake, fake, 1, 2, 1, 128, 128 * 10, 100, 4,
                                          fake, fake, 10, fake, fake, 10, 0.088, fake, fake,
                                          1 << 20, None))
    # append: misaligned buffer
    _expect_invalid(lib.ckv_append(ctypes.c_void_p((1 << 20) + 2), fake, 1, 2, 128, 128 * 100,
                                   100, fake, fake, fake, None))


def test_binding_raises_on_invalid(lib):
    import torch
    t = torch.zeros((2, 100, 64), dtype=torch.bfloat16)
    lab = torch.zeros((2, 100), dtype=torch.int32)
    with pytest.raises(ckv.CkvError) as e:
        ckv.ckv_assign(t, t.stride(0), 0, 100, t, 4, 0, 8, lab, 0, 100, d=64)
    assert e.value.status == ckv.CKV_ERR_INVALID
