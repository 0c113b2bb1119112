"""C-ABI checks that need no GPU: the library loads, exports every entry point
include/instagen.h declares, and its host-side logic (budgets, workspace
sizes, argument validation) behaves.  No call here reaches a kernel."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_head_b200 as ig
from block_sparse_attention_head_b200 import build as igbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    igbuild.build()
    return ig.lib()


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "instagen.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(instagen_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert len(declared) >= 12
    for name in declared:
        assert hasattr(lib, name), name
    assert set(declared) == set(ig._SYMBOLS)


def test_params_struct_layout():
    # instagen_params: 7 int32, 3 float, uint64 (8-aligned at 40), uint32, 2 int32, 2 float
    assert ctypes.sizeof(ig.Params) == 72
    assert ig.Params.seed.offset == 40
    assert ig.Params.selection.offset == 56
    assert ig.Params.top_p.offset == 60 and ig.Params.key_floor.offset == 64
    assert ctypes.sizeof(ig.ForwardLayout) == 18 * ctypes.sizeof(ctypes.c_size_t)


def test_budgets_match_oracle(lib, oracle_mod):
    for N, ef, sf in [(4096, 0.08, 0.08), (75600, 0.16, 0.16), (32760, 0.04, 0.32), (3, 0.5, 0.5), (100, 0.0, 0.0)]:
        p = ig.make_params(1, 1, N, 64, 4, 8, exact_frac=ef, sample_frac=sf)
        assert ig.exact_budget(p) == oracle_mod.budget(ef, N)
        assert ig.sample_budget(p) == oracle_mod.budget(sf, N)


def test_workspace_layout(lib):
    # centroid selection: the PQ-voting blocks are empty
    p0 = ig.make_params(1, 40, 75600, 128, 100, 500)
    L0 = ig.forward_layout(p0)
    assert L0.votes == L0.pq_ws == L0.cluster_ws
    p = ig.make_params(1, 40, 75600, 128, 100, 500, selection="pq_vote")
    L = ig.forward_layout(p)
    fields = [f for f, _ in ig.ForwardLayout._fields_ if f != "total"]
    offs = [getattr(L, f) for f in fields]
    assert all(o % 256 == 0 for o in offs)
    assert offs == sorted(offs) and len(set(offs)) == len(offs)
    assert L.total == ig.workspace_size(p)
    assert L.pq_ws - L.votes >= 40 * 100 * 500 * 4
    assert L.total - L0.total == L.cluster_ws - L0.cluster_ws
    BH, N, d, m = 40, 75600, 128, 12096
    assert L.vp - L.kp >= BH * N * d * 2
    assert L.sample_bias - L.sample_pos >= BH * 100 * m * 4
    assert L.total < 16 * 2 ** 30            # fits easily in 180 GB of HBM


@pytest.mark.parametrize("field,value,code", [
    ("d", 96, 2), ("d", 0, 2), ("N", 0, 1), ("B", 0, 1), ("Cq", 0, 1), ("Ck", 5000, 2),
    ("sampling", 7, 1), ("exact_frac", -0.1, 1), ("sample_frac", float("nan"), 1), ("selection", 3, 1),
])
def test_invalid_params_rejected_on_host(lib, field, value, code):
    p = ig.make_params(1, 2, 1000, 64, 8, 16)
    setattr(p, field, value)
    assert lib.instagen_workspace_size(ctypes.byref(p)) == 0
    rc = lib.instagen_forward(None, None, None, None, ctypes.byref(p), None, 0, None)
    assert rc == code


def test_null_pointers_and_workspace_rejected(lib):
    p = ig.make_params(1, 2, 1000, 64, 8, 16)
    assert lib.instagen_forward(None, None, None, None, ctypes.byref(p), None, 0, None) == 1
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any launch
    assert lib.instagen_forward(fake, fake, fake, fake, ctypes.byref(p), fake, 16, None) == 3
    assert lib.instagen_cluster(None, 8, 1, None, ctypes.byref(p), None, None, None, None, None, 0, None) == 1
    assert lib.instagen_cluster(fake, 8, 0, None, ctypes.byref(p), fake, fake, fake, fake, fake, 0, None) == 1
    assert lib.instagen_gather(fake, fake, ctypes.byref(p), fake, 0, None) == 1   # X == Xp
    assert lib.instagen_gather(fake, fake, ctypes.byref(p), ctypes.c_void_p(1 << 21), 2, None) == 1  # bad flag
    assert lib.instagen_select_sample(None, None, None, ctypes.byref(p), None, None, None, None, None) == 1
    big = ig.make_params(1, 2, 1000, 64, 8, 3000)
    assert lib.instagen_attention(fake, fake, fake, fake, fake, fake, fake, fake, fake, fake,
                                  ctypes.byref(big), fake, None) == 2             # Ck > 2048


def test_forward_host_checks_on_host(lib):
    p = ig.make_params(2, 5, 1000, 128, 8, 16)
    L1 = lib.instagen_workspace_size(ctypes.byref(ig.make_params(1, 2, 1000, 128, 8, 16)))
    # three staging slots, each 2 heads x (Q, K, V, O) and one chunk's forward workspace
    assert lib.instagen_forward_host_workspace_size(ctypes.byref(p), 2) >= 3 * (4 * 2 * 1000 * 128 * 2 + L1)
    assert lib.instagen_forward_host_workspace_size(ctypes.byref(p), -1) == 0
    # automatic chunk: all 5 small heads in one chunk
    L5 = lib.instagen_workspace_size(ctypes.byref(ig.make_params(1, 5, 1000, 128, 8, 16)))
    assert lib.instagen_forward_host_workspace_size(ctypes.byref(p), 0) >= L5
    fake = ctypes.c_void_p(1 << 20)  # never dereferenced: rejected before any copy or launch
    assert lib.instagen_forward_host(None, fake, fake, fake, ctypes.byref(p), 2, fake, 1 << 30, None) == 1
    assert lib.instagen_forward_host(fake, fake, fake, fake, ctypes.byref(p), -3, fake, 1 << 30, None) == 1
    assert lib.instagen_forward_host(fake, fake, fake, fake, ctypes.byref(p), 2, fake, 16, None) == 3
    bad = ig.make_params(1, 2, 1000, 96, 8, 16)
    assert lib.instagen_forward_host(fake, fake, fake, fake, ctypes.byref(bad), 1, fake, 1 << 30, None) == 2


def test_error_strings(lib):
    for code in range(6):
        assert lib.instagen_error_string(code)
    assert b"unknown" in lib.instagen_error_string(99)


def test_binding_refuses_cpu_tensors(lib):
    import torch
    p = ig.make_params(1, 1, 16, 64, 2, 2)
    X = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ig.InstaGenError, match="CUDA tensor"):
        ig.forward(X, X, X, p)


def test_pq_vote_selection_checks_on_host(lib):
    """PQ voting keeps votes below 2^20 in the rank key: larger N is refused,
    an unknown selection value is invalid, and the vote scratch is sized."""
    p = ig.make_params(1, 1, 1 << 20, 64, 4, 8, selection="pq_vote")
    assert lib.instagen_workspace_size(ctypes.byref(p)) == 0
    p = ig.make_params(1, 1, (1 << 20) - 1, 64, 4, 8, selection="pq_vote")
    assert lib.instagen_workspace_size(ctypes.byref(p)) > 0
    p.selection = 7
    assert lib.instagen_workspace_size(ctypes.byref(p)) == 0
    p = ig.make_params(1, 40, 75600, 128, 100, 500, selection="pq_vote")
    # codebooks [40][2][16][16][8] fp32 + key-group codes [40][500][16]
    assert lib.instagen_pq_votes_workspace_size(ctypes.byref(p)) == 40 * 2 * 16 * 16 * 8 * 4 + 40 * 500 * 16


@pytest.mark.parametrize("kw,code", [
    (dict(top_p=1.5), 1), (dict(top_p=-0.1), 1), (dict(key_floor=2.0), 1), (dict(top_p=float("nan")), 1),
    (dict(sample_frac=0.01), 1), (dict(N=1 << 20), 2),
])
def test_top_p_params_rejected_on_host(lib, kw, code):
    args = dict(N=1000, top_p=0.9, key_floor=0.1, sample_frac=0.0)
    args.update(kw)
    N = args.pop("N")
    p = ig.make_params(1, 2, N, 64, 8, 16, selection="top_p", **args)
    assert lib.instagen_workspace_size(ctypes.byref(p)) == 0
    rc = lib.instagen_forward(None, None, None, None, ctypes.byref(p), None, 0, None)
    assert rc == code


def test_top_p_params_accepted(lib):
    p = ig.make_params(1, 2, 75600, 128, 100, 500, selection="top_p", top_p=0.95, key_floor=0.1, sample_frac=0.0)
    assert ig.workspace_size(p) > 0
