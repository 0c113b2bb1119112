"""GPU parity of the top-p comparator (the SVG2-style selection of the
thelatestinai.com paper page, Figure 2 caption: top-p 0.5 to 0.95, key floor
0.1; no sample).

Inputs flow one way: seeded generator -> oracle (clustering, permutation, and
its top-p selection) -> the CUDA stage under test.  The kept groups and counts
are integer decisions and must agree bit for bit; the attention over them is
held to the same bars as the main path (max-abs 1e-2, mean relative 2e-3 of
the fp64 oracle)."""
import numpy as np
import pytest
import torch

import block_sparse_attention_head_b200 as ig
from block_sparse_attention_head_b200 import workloads

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_REL = 2e-3

CASES = {
    # name: (H, N, d, Cq, Ck, iters, top_p, key_floor, seed)
    "tiny_p09": (1, 4096, 64, 16, 64, 10, 0.9, 0.1, 0),
    "ragged_p05": (2, 1000, 128, 7, 40, 4, 0.5, 0.1, 3),
    "floor_dominant": (1, 2048, 128, 9, 33, 3, 0.05, 0.4, 7),
    "p1_dense": (1, 640, 64, 4, 10, 3, 1.0, 0.0, 11),
    "p0_top_group": (1, 900, 64, 5, 30, 3, 0.0, 0.0, 13),
    "many_groups": (1, 3000, 64, 6, 700, 3, 0.75, 0.1, 17),
}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_head_b200 import build
    build.build()
    ig.lib()
    yield
    ig.device_status()


def np_(t):
    return t.detach().cpu().numpy()


def cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _inputs(case):
    H, N, d, Cq, Ck, iters, tp, kf, seed = CASES[case]
    if case == "tiny_p09":
        Q, K, V = workloads.make_inputs(workloads.TINY)
    else:
        Q, K, V = workloads.random_small(seed, N, d, n_centres=12, sigma=0.4, H=H)
    p = ig.make_params(1, H, N, d, Cq, Ck, iters=iters, exact_frac=0.0, sample_frac=0.0, seed=seed,
                       selection="top_p", top_p=tp, key_floor=kf)
    return p, Q, K, V


@pytest.fixture(scope="module")
def runs(oracle_mod):
    out = {}
    for case in CASES:
        p, Q, K, V = _inputs(case)
        heads = []
        for h in range(p.H):
            f = lambda t: np_(t[0, h].float())
            heads.append(oracle_mod.forward_head(f(Q), f(K), f(V), Cq=p.Cq, Ck=p.Ck, iters=p.kmeans_iters,
                                                 exact_frac=0.0, sample_frac=0.0, scale=p.softmax_scale,
                                                 selection="top_p", top_p=p.top_p, key_floor=p.key_floor))
        out[case] = (p, Q, K, V, heads)
    return out


def _stack(heads, attr, dtype=None):
    return cuda(np.stack([getattr(h, attr) for h in heads])[None], dtype)


@pytest.mark.parametrize("case", list(CASES))
def test_top_p_lists_bit_exact(runs, case):
    p, Q, K, V, heads = runs[case]
    eg, cnt, sp, sb = ig.select_sample(_stack(heads, "cq"), _stack(heads, "ck"), _stack(heads, "k_offsets"), p)
    eg, cnt = np_(eg)[0], np_(cnt)[0]
    for h, hr in enumerate(heads):
        assert np.array_equal(cnt[h], hr.counts), f"head {h} counts"
        assert np.array_equal(eg[h], hr.exact_groups), f"head {h} kept groups"
        assert np.all(cnt[h][:, 2] == 0)
    if case == "p1_dense":
        nonempty = (np.diff(heads[0].k_offsets) > 0).sum()
        assert np.all(cnt[0][:, 0] == nonempty)
    if case == "p0_top_group":
        assert np.all(cnt[0][:, 0] == 1)
    ig.device_status()


@pytest.mark.parametrize("case", ["tiny_p09", "ragged_p05", "floor_dominant", "p1_dense"])
def test_top_p_attention_matches_oracle(runs, case):
    p, Q, K, V, heads = runs[case]
    kperm = _stack(heads, "k_perm")
    Kp = ig.gather(K.cuda(), kperm, p)
    Vp = ig.gather(V.cuda(), kperm, p, to_f16=True)
    empty_i = torch.empty((1, p.H, p.Cq, 0), dtype=torch.int32, device="cuda")
    empty_f = torch.empty((1, p.H, p.Cq, 0), dtype=torch.float32, device="cuda")
    O = ig.attention(Q.cuda(), Kp, Vp, _stack(heads, "q_perm"), _stack(heads, "q_offsets"),
                     _stack(heads, "k_offsets"), _stack(heads, "exact_groups"), _stack(heads, "counts"),
                     empty_i, empty_f, p)
    O = np_(O.float())[0].astype(np.float64)
    for h, hr in enumerate(heads):
        diff = np.abs(O[h] - hr.out)
        mean_rel = diff.sum() / np.abs(hr.out).sum()
        assert diff.max() <= MAX_ABS and mean_rel <= MEAN_REL, (case, h, diff.max(), mean_rel)
    ig.device_status()


def test_top_p_forward_equals_staged_and_is_deterministic():
    p, Q, K, V = _inputs("ragged_p05")
    Qc, Kc, Vc = Q.cuda(), K.cuda(), V.cuda()
    ws = torch.empty(ig.workspace_size(p), dtype=torch.uint8, device="cuda")
    O1 = ig.forward(Qc, Kc, Vc, p, workspace=ws)
    assert torch.equal(O1, ig.forward(Qc, Kc, Vc, p))
    cq, qa, qp, qo = ig.cluster(Qc, p.Cq, p.kmeans_iters, p)
    ck, ka, kp, ko = ig.cluster(Kc, p.Ck, p.kmeans_iters, p)
    eg, cnt, sp, sb = ig.select_sample(cq, ck, ko, p)
    inter = ig.forward_intermediates(ws, p)
    assert torch.equal(inter["exact_groups"], eg) and torch.equal(inter["counts"], cnt)
    O3 = ig.attention(Qc, ig.gather(Kc, kp, p), ig.gather(Vc, kp, p, to_f16=True), qp, qo, ko, eg, cnt, sp, sb, p)
    assert torch.equal(O1, O3)
    ig.device_status()
