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
import os
import re

import numpy as np
import pytest
import torch

import block_sparse_attention_head_b200 as ig
from block_sparse_attention_head_b200 import workloads

pytestmark = pytest.mark.gpu

IG_ERR_WORKSPACE = 3
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _static_bytes():
    """The scratch limit as include/instagen.h states it (the product of the
    factors in INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES)."""
    text = open(os.path.join(ROOT, "include", "instagen.h")).read()
    m = re.search(r"#define\s+INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES\s+\(([^)]*)\)", text)
    assert m, "INSTAGEN_CLUSTER_STATIC_SCRATCH_BYTES not found"
    n = 1
    for f in m.group(1).split("*"):
        n *= int(f.strip().rstrip("uUlL"))
    return n


STATIC_BYTES = _static_bytes()


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


@pytest.mark.parametrize("shapes", [
    # (H, N, d, C) of the first call, then of the second: the second call has
    # fewer heads, clusters and tokens (its norms, partial sums and arrival
    # counters sit at other offsets than the first call left them), or more
    [(4, 3000, 128, 300), (1, 1000, 64, 40)],
    [(1, 4096, 64, 64), (3, 5000, 128, 150)],
])
def test_static_scratch_matches_workspace_call_twice(lib, shapes):
    for call, (H, N, d, C) in enumerate(shapes):
        p = ig.make_params(1, H, N, d, 8, C, iters=4)
        Q, K, V = workloads.random_small(100 + call, N, d, n_centres=12, sigma=0.4, H=H)
        X = K.cuda()
        got = _call_static(lib, X, C, 4, p)
        ref = ig.cluster(X, C, 4, p)
        torch.cuda.synchronize()
        # the same kernels in the same order on the same inputs: equal bit for bit
        for g, r in zip(got, ref):  # centroids, assignments, permutation, offsets
            assert torch.equal(g, r), f"call {call}"
    ig.device_status()


def test_static_scratch_rejects_oversize(lib):
    # 200 heads x 512 centroids x d=128 needs ~53 MB of scratch: rejected before any launch
    p = ig.make_params(1, 200, 64, 128, 8, 500, iters=1)
    assert ig.cluster_workspace_size(p, 500) > STATIC_BYTES
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.instagen_cluster_static(fake, 500, 1, None, ctypes.byref(p), fake, fake, fake, fake, None)
    assert rc == IG_ERR_WORKSPACE
    ig.device_status()
