"""veda_block_scores_noalloc against veda_block_scores, through the C ABI.

The allocation-free entry point exists for callers that cannot give the library a
workspace -- a plugin whose host runtime owns all device memory, or code that must
not call cudaMalloc because it can synchronise the device. It must give the same
scores as the workspace entry point. Two calls in a row (different inputs, then the
first inputs again) check that the shared built-in scratch carries nothing over from
one call to the next. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _inputs(seed, B, H, nT):
    g = torch.Generator().manual_seed(seed)
    pq = torch.randn((B, H, nT, 3, 128), generator=g)
    pk = torch.randn((B, H, nT, 3, 128), generator=g)
    wq = 0.02 * torch.randn((H, 128, 384), generator=g)
    wk = 0.02 * torch.randn((H, 128, 384), generator=g)
    return [t.to(DEV) for t in (pq, pk, wq, wk)]


def _rel_err(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    floor = np.abs(b).mean(axis=(-1, -2), keepdims=True)
    return float((np.abs(a - b) / np.maximum(np.abs(b), floor)).max())


def test_noalloc_matches_workspace_entry_point_twice():
    from block_sparse_attention_max_b200 import build
    build.build()
    from block_sparse_attention_max_b200 import veda as V
    L = V.lib()
    B, H, nT = 1, 8, 200
    stream = torch.cuda.current_stream().cuda_stream
    for seed in (1, 2, 1):
        pq, pk, wq, wk = _inputs(seed, B, H, nT)
        ref = V.block_scores(pq, pk, wq, wk)                      # workspace entry point
        out = torch.full((B, H, nT, nT), float("nan"), device=DEV)
        st = L.veda_block_scores_noalloc(pq.data_ptr(), pk.data_ptr(), wq.data_ptr(), wk.data_ptr(),
                                         out.data_ptr(), B, H, nT, 128, stream)
        assert st == 0, V.lib().veda_last_error()
        V.check_device_status()
        assert torch.isfinite(out).all()
        # same kernels on the same inputs: identical bits, so a scratch that carried
        # anything over from the previous call would show
        assert torch.equal(out, ref), _rel_err(out, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from block_sparse_attention_max_b200 import veda as V
    L = V.lib()
    # 2 * B*H*nT * 128 * 4 bytes > 32 MiB: refused before anything runs
    st = L.veda_block_scores_noalloc(256, 256, 256, 256, 256, 1, 40, 1000, 128, None)
    assert st == 1
    assert b"exceeds" in L.veda_last_error()
