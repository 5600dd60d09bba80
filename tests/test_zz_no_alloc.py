"""The allocation-free sparse decode entry point (ckv_sparse_decode_noalloc).

Some callers cannot allocate device memory: a plugin or operator hook that a
host framework hands tensors but no allocator (the framework's pool owns the
device memory), or a decode loop that must never call cudaMalloc/cudaFree
because those calls can synchronise the device. For them the library keeps
the split-K partials of sparse decode in a fixed device array of its own, so
the caller passes only inputs and outputs. These tests call that entry point
through the C ABI and check it against ckv_sparse_decode (the caller-workspace
entry point) on two calls in a row, the second with another shape so that the
shared array still holds the first call's contents. This file is named to be
collected last, and passes alone in a fresh process as well as after the rest
of the suite.
"""
import numpy as np
import pytest
import torch

from semantic_cluster_recall_b200 import ckv

pytestmark = pytest.mark.gpu

OUT_MAX_ABS = 2e-3  # the decode tolerance used by the parity tests


def _case(dev, P, G, L, S, budget, tail, seed):
    g = torch.Generator(device="cpu").manual_seed(seed)
    K = (torch.randn((P, L, 128), generator=g) * 0.5).to(torch.bfloat16).to(dev)
    V = torch.randn((P, L, 128), generator=g).to(torch.bfloat16).to(dev)
    q = (torch.randn((P, G, 128), generator=g) * 4).to(torch.bfloat16).to(dev)
    sel = torch.full((P, budget), -1, dtype=torch.int32)
    cnt = torch.zeros(P, dtype=torch.int32)
    for p in range(P):
        n = int(torch.randint(0, budget + 1, (1,), generator=g))
        sel[p, :n] = torch.randperm(L - tail - S, generator=g)[:n].to(torch.int32) + S
        cnt[p] = n
    tb = torch.full((P,), L - tail, dtype=torch.int32)
    te = torch.full((P,), L, dtype=torch.int32)
    return K, V, q, sel.to(dev), cnt.to(dev), tb.to(dev), te.to(dev)


def _both(dev, P, G, L, S, budget, tail, seed):
    K, V, q, sel, cnt, tb, te = _case(dev, P, G, L, S, budget, tail, seed)
    scale = 1 / np.sqrt(128)
    ws = ckv.workspace(ckv.ckv_decode_workspace_bytes(P, G, 128, S + budget + tail), dev)
    ref = torch.empty((P, G, 128), device=dev)
    ckv.ckv_sparse_decode(q, K, V, K.stride(0), L, S, tb, te, tail, sel, cnt, budget, scale,
                          ref, ws)
    got = torch.full((P, G, 128), float("nan"), device=dev)
    ckv.ckv_sparse_decode_noalloc(q, K, V, K.stride(0), L, S, tb, te, tail, sel, cnt, budget,
                                  scale, got)
    torch.cuda.synchronize()
    return ref, got


def test_noalloc_decode_matches_workspace_decode_twice(cuda_device):
    need = ckv.ckv_sparse_decode_noalloc_scratch_bytes(64, 4, 128, 16 + 2048 + 64)
    assert 0 < need <= ckv.NOALLOC_SCRATCH_BYTES
    # first call: GQA, many problems
    ref, got = _both(cuda_device, P=64, G=4, L=6000, S=16, budget=2048, tail=64, seed=1)
    assert torch.isfinite(got).all()
    assert (got - ref).abs().max().item() <= OUT_MAX_ABS
    # second call right after, another shape: the array holds the first call's data
    ref2, got2 = _both(cuda_device, P=7, G=1, L=3000, S=4, budget=300, tail=32, seed=2)
    assert torch.isfinite(got2).all()
    assert (got2 - ref2).abs().max().item() <= OUT_MAX_ABS
    assert ckv.ckv_device_error() == 0


def test_noalloc_decode_rejects_shapes_beyond_its_scratch(cuda_device):
    # 65535 problems x 8 query heads cannot fit: refused on the host, nothing launched
    P, G = 65535, 8
    assert ckv.ckv_sparse_decode_noalloc_scratch_bytes(P, G, 128, 4096) > \
        ckv.NOALLOC_SCRATCH_BYTES
    t = torch.zeros((1, 1, 128), dtype=torch.bfloat16, device=cuda_device)
    i = torch.zeros((P,), dtype=torch.int32, device=cuda_device)
    out = torch.zeros((1, 1, 128), device=cuda_device)
    with pytest.raises(ckv.CkvError) as e:
        ckv.ckv_sparse_decode_noalloc(t, t, t, 128, 1, 0, i, i, 0, i, i, 4096, 0.088, out,
                                      P=P, G=G)
    assert e.value.status == ckv.CKV_ERR_INVALID
    assert "scratch" in str(e.value)
