"""Device timeout reporting, without faulting or hanging the GPU.

Every wait inside the library's kernels is bounded; a wait that gives up
records CKV_DEVERR_TIMEOUT in the device error word, which ckv_device_error
maps to CKV_ERR_TIMEOUT. ckv_selftest_timeout makes one such wait run out (a
device flag that nothing sets, a bound of a few hundred microseconds) so the
reporting path is exercised; the context must stay usable afterwards.
"""
import ctypes

import numpy as np
import pytest
import torch

from semantic_cluster_recall_b200 import ckv

pytestmark = pytest.mark.gpu


def _status_and_flags(clear: int):
    flags = ctypes.c_uint(0)
    st = ckv.load().ckv_device_error(ctypes.byref(flags), clear, None)
    return st, flags.value


def test_bounded_wait_reports_a_timeout_and_the_context_survives(cuda_device):
    ckv.ckv_device_error(clear=True)  # start clean
    for limit_us in (0, 300):
        ckv.ckv_selftest_timeout(limit_us)
        torch.cuda.synchronize()
        st, flags = _status_and_flags(clear=1)
        assert st == ckv.CKV_ERR_TIMEOUT and flags & ckv.CKV_DEVERR_TIMEOUT
        st, flags = _status_and_flags(clear=0)  # cleared by the previous read
        assert st == ckv.CKV_OK and flags == 0
    # the context still runs work: an index of a few labels
    lab = torch.tensor([[2, 0, 1, 2, 0]], dtype=torch.int32, device=cuda_device)
    off = torch.zeros((1, 4), dtype=torch.int32, device=cuda_device)
    perm = torch.zeros((1, 5), dtype=torch.int32, device=cuda_device)
    ws = ckv.workspace(ckv.ckv_index_workspace_bytes(1, 5, 3), cuda_device)
    ckv.ckv_index(lab, 1, 10, 15, 3, 0, 3, 0, 5, off, perm, ws)
    torch.cuda.synchronize()
    assert np.array_equal(off.cpu().numpy()[0], [0, 2, 3, 5])
    assert np.array_equal(perm.cpu().numpy()[0], [11, 14, 12, 10, 13])
    assert ckv.ckv_device_error() == 0
