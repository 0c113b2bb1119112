"""instagen_cluster_static: the clustering call for callers that may not
allocate device memory (plug-ins whose host framework owns every device
allocation, deployments that fix their memory budget at start-up, code that
must not let a cudaMalloc synchronise the device).  Its scratch lives in a
fixed device array inside the library, shared by every call.

Checked through the C ABI against instagen_cluster (which takes a
caller-allocated workspace) on two calls in a row with different inputs, so
the second call runs on scratch the first one left behind.  Named to be
collected last: if it fails, a run that stops at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import block_sparse_attention_head_b200 as ig
from block_sparse_attention_head_b200 import workloads

pytestmark = pytest.mark.gpu

IG_ERR_WORKSPACE = 3
STATIC_BYTES = 16 * 1024 * 1024


@pytest.fixture(scope="module")
def lib():
    from block_sparse_attention_head_b200 import build
    build.build()
    return ig.lib()


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _call_static(lib, X, C, iters, p):
    dev = X.device
    cent = torch.full((p.B, p.H, C, p.d), float("nan"), dtype=torch.float32, device=dev)
    assign = torch.full((p.B, p.H, p.N), -7, dtype=torch.int32, device=dev)
    perm = torch.full_like(assign, -7)
    offs = torch.full((p.B, p.H, C + 1), -7, dtype=torch.int32, device=dev)
    rc = lib.instagen_cluster_static(ctypes.c_void_p(X.data_ptr()), C, iters, None, ctypes.byref(p),
                                     ctypes.c_void_p(cent.data_ptr()), ctypes.c_void_p(assign.data_ptr()),
                                     ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(offs.data_ptr()), _stream())
    assert rc == 0, lib.instagen_error_string(rc)
    return cent, assign, perm, offs


@pytest.mark.parametrize("shape", [(2, 1000, 128, 40), (1, 4096, 64, 64)])
def test_static_scratch_matches_workspace_call_twice(lib, shape):
    H, N, d, C = shape
    p = ig.make_params(1, H, N, d, 8, C, iters=4)
    for call in range(2):  # the second call reuses the scratch the first left behind
        Q, K, V = workloads.random_small(100 + call, N, d, n_centres=12, sigma=0.4, H=H)
        X = K.cuda()
        got = _call_static(lib, X, C, 4, p)
        ref = ig.cluster(X, C, 4, p)
        torch.cuda.synchronize()
        for g, r in zip(got[1:], ref[1:]):  # assignments, permutation, offsets
            assert torch.equal(g, r), f"call {call}"
        np.testing.assert_allclose(got[0].cpu().numpy(), ref[0].cpu().numpy(), rtol=0, atol=2e-4)
    ig.device_status()


def test_static_scratch_rejects_oversize(lib):
    # 200 heads x 512 centroids x d=128 needs ~53 MB of scratch: rejected before any launch
    p = ig.make_params(1, 200, 64, 128, 8, 500, iters=1)
    assert ig.cluster_workspace_size(p, 500) > STATIC_BYTES
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.instagen_cluster_static(fake, 500, 1, None, ctypes.byref(p), fake, fake, fake, fake, None)
    assert rc == IG_ERR_WORKSPACE
    ig.device_status()
