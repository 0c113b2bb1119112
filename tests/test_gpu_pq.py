"""GPU parity of the product-quantised per-query voting selection (the
abstract's rule; readings in the oracle and the C header): votes and the
vote-ranked exact sets bit-exact against the oracle on the oracle's own
centroids and permutations, attention over the resulting lists within the
attention tolerances, and the fused call in this mode equal to its stages."""
import numpy as np
import pytest
import torch

import block_sparse_attention_head_b200 as ig
from block_sparse_attention_head_b200 import workloads

pytestmark = pytest.mark.gpu

MAX_ABS = 1e-2
MEAN_REL = 2e-3

CASES = {
    # name: (H, N, d, Cq, Ck, iters, exact, sample, seed)  -- Ck spans every
    # keys-per-lane instantiation of the vote kernel (<= 128, 256, 512, 1024, 2048)
    "tiny_d64": (1, 4096, 64, 16, 64, 4, 0.08, 0.08, 0),
    "ragged_d128": (2, 1000, 128, 7, 40, 3, 0.2, 0.1, 3),
    "cq1": (1, 777, 64, 1, 13, 3, 0.3, 0.05, 5),
    "ck300": (1, 6000, 64, 12, 300, 3, 0.12, 0.1, 17),
    "ck1000": (1, 9000, 64, 20, 1000, 2, 0.1, 0.05, 19),
    "ck2048": (1, 12000, 128, 9, 2048, 2, 0.15, 0.05, 23),
    "exact_zero": (1, 900, 64, 5, 30, 3, 0.0, 0.15, 13),
    "exact_all": (1, 640, 128, 4, 10, 3, 1.0, 0.1, 11),
}


def np_(t):
    return t.detach().cpu().numpy()


def cuda(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def _inputs(case):
    H, N, d, Cq, Ck, iters, ef, sf, seed = CASES[case]
    if case == "tiny_d64":
        Q, K, V = workloads.make_inputs(workloads.TINY)
    else:
        Q, K, V = workloads.random_small(seed, N, d, n_centres=12, sigma=0.4, H=H)
    p = ig.make_params(1, H, N, d, Cq, Ck, iters=iters, exact_frac=ef, sample_frac=sf, seed=99 + seed, layer=seed,
                       selection="pq_vote")
    return p, Q, K, V


@pytest.fixture(scope="module")
def runs(oracle_mod):
    out = {}
    for case in CASES:
        p, Q, K, V = _inputs(case)
        heads, votes = [], []
        for h in range(p.H):
            f = lambda t: np_(t[0, h].float())
            hr = oracle_mod.forward_head(f(Q), f(K), f(V), Cq=p.Cq, Ck=p.Ck, iters=p.kmeans_iters,
                                         exact_frac=p.exact_frac, sample_frac=p.sample_frac, scale=p.softmax_scale,
                                         seed=p.seed, layer=p.layer, bh=h, selection="pq_vote")
            heads.append(hr)
            votes.append(oracle_mod.pq_votes(f(Q), hr.cq, hr.ck, hr.q_perm, hr.q_offsets, hr.k_offsets,
                                             oracle_mod.budget(p.exact_frac, p.N)))
        out[case] = (p, Q, K, V, heads, np.stack(votes))
    return out


def _stack(heads, attr, dtype=None):
    return cuda(np.stack([getattr(h, attr) for h in heads])[None], dtype)


@pytest.mark.parametrize("case", list(CASES))
def test_votes_bit_exact(runs, case):
    p, Q, K, V, heads, votes = runs[case]
    got = ig.pq_votes(Q.cuda(), _stack(heads, "cq"), _stack(heads, "ck"), _stack(heads, "q_perm"),
                      _stack(heads, "q_offsets"), _stack(heads, "k_offsets"), p)
    assert np.array_equal(np_(got)[0], votes), case
    ig.device_status()


@pytest.mark.parametrize("case", list(CASES))
def test_vote_ranked_selection_bit_exact(runs, case):
    p, Q, K, V, heads, votes = runs[case]
    eg, cnt, sp, sb = ig.select_sample(_stack(heads, "cq"), _stack(heads, "ck"), _stack(heads, "k_offsets"), p,
                                       votes=cuda(votes[None]))
    m = ig.sample_budget(p)
    for h, hr in enumerate(heads):
        assert np.array_equal(np_(cnt)[0, h], hr.counts)
        assert np.array_equal(np_(eg)[0, h], hr.exact_groups)
        for i in range(p.Cq):
            ns = hr.counts[i, 2]
            assert np.array_equal(np_(sp)[0, h, i, :ns], hr.sample_pos[i, :ns])
            np.testing.assert_allclose(np_(sb)[0, h, i, :ns], hr.sample_bias[i, :ns], rtol=0, atol=1e-4)
        if m:
            assert (np_(sp)[0, h, :, :][np.arange(m)[None] >= hr.counts[:, 2:3]] == -1).all()
    ig.device_status()


@pytest.mark.parametrize("case", ["tiny_d64", "ragged_d128", "ck300", "ck2048"])
def test_attention_over_vote_selection(runs, case):
    p, Q, K, V, heads, votes = runs[case]
    Kp = cuda(np.stack([np_(K[0, h].float())[hr.k_perm] for h, hr in enumerate(heads)])[None], torch.bfloat16)
    Vp = cuda(np.stack([np_(V[0, h].float())[hr.k_perm] for h, hr in enumerate(heads)])[None], torch.float16)
    O = ig.attention(Q.cuda(), Kp, Vp, _stack(heads, "q_perm"), _stack(heads, "q_offsets"),
                     _stack(heads, "k_offsets"), _stack(heads, "exact_groups"), _stack(heads, "counts"),
                     _stack(heads, "sample_pos"), _stack(heads, "sample_bias", torch.float32), p)
    for h, hr in enumerate(heads):
        got = np_(O[0, h].float()).astype(np.float64)
        diff = np.abs(got - hr.out)
        assert diff.max() <= MAX_ABS, (case, h, diff.max())
        assert diff.sum() / np.abs(hr.out).sum() <= MEAN_REL, (case, h)
    ig.device_status()


@pytest.mark.parametrize("case", ["tiny_d64", "ragged_d128", "ck300"])
def test_forward_pq_vote_equals_its_stages(case):
    p, Q, K, V = _inputs(case)
    Qc, Kc, Vc = Q.cuda(), K.cuda(), V.cuda()
    ws = torch.empty(ig.workspace_size(p), dtype=torch.uint8, device="cuda")
    O1 = ig.forward(Qc, Kc, Vc, p, workspace=ws)
    it = {k: v.clone() for k, v in ig.forward_intermediates(ws, p).items()}
    assert "votes" in it
    assert torch.equal(O1, ig.forward(Qc, Kc, Vc, p))  # deterministic
    votes = ig.pq_votes(Qc, it["cq"], it["ck"], it["q_perm"], it["q_offsets"], it["k_offsets"], p)
    assert torch.equal(votes, it["votes"])
    eg, cnt, sp, sb = ig.select_sample(it["cq"], it["ck"], it["k_offsets"], p, votes=votes)
    assert torch.equal(eg, it["exact_groups"]) and torch.equal(cnt, it["counts"])
    assert torch.equal(sp, it["sample_pos"]) and torch.equal(sb, it["sample_bias"])
    O3 = ig.attention(Qc, it["kp"], it["vp"], it["q_perm"], it["q_offsets"], it["k_offsets"], eg, cnt, sp, sb, p)
    assert torch.equal(O1, O3)
    # the centroid ranking on the same call differs only in the selection
    pc = ig.make_params(p.B, p.H, p.N, p.d, p.Cq, p.Ck, iters=p.kmeans_iters, exact_frac=p.exact_frac,
                        sample_frac=p.sample_frac, seed=p.seed, layer=p.layer)
    wc = torch.empty(ig.workspace_size(pc), dtype=torch.uint8, device="cuda")
    ig.forward(Qc, Kc, Vc, pc, workspace=wc)
    ic = ig.forward_intermediates(wc, pc)
    assert torch.equal(ic["cq"], it["cq"]) and torch.equal(ic["k_offsets"], it["k_offsets"])
    ig.device_status()


def test_full_size_heads_votes_bit_exact(oracle_mod):
    """Wan2.1-14B 720p shape (N=75600, d=128, Cq=100, Ck=500, 16%+16%), heads 0
    and 39: votes and vote-ranked selections from the oracle's (one-iteration)
    centroids and permutations, bit-exact."""
    w = workloads.WAN14B_720P
    heads = [0, w.H - 1]
    Q, K, V = workloads.make_inputs(w, heads=heads)
    p = ig.make_params(1, len(heads), w.N, w.d, w.Cq, w.Ck, iters=1, exact_frac=w.exact_frac,
                       sample_frac=w.sample_frac, seed=77, layer=0, selection="pq_vote")
    E = oracle_mod.budget(w.exact_frac, w.N)
    hr, votes = [], []
    for h in range(len(heads)):
        f = lambda t: np_(t[0, h].float())
        r = oracle_mod.forward_head(f(Q), f(K), f(V), Cq=w.Cq, Ck=w.Ck, iters=1, exact_frac=w.exact_frac,
                                    sample_frac=w.sample_frac, scale=p.softmax_scale, seed=p.seed, layer=0, bh=h,
                                    rows=[], selection="pq_vote")
        hr.append(r)
        votes.append(oracle_mod.pq_votes(f(Q), r.cq, r.ck, r.q_perm, r.q_offsets, r.k_offsets, E))
    votes = np.stack(votes)
    got = ig.pq_votes(Q.cuda(), _stack(hr, "cq"), _stack(hr, "ck"), _stack(hr, "q_perm"), _stack(hr, "q_offsets"),
                      _stack(hr, "k_offsets"), p)
    assert np.array_equal(np_(got)[0], votes)
    eg, cnt, sp, sb = ig.select_sample(_stack(hr, "cq"), _stack(hr, "ck"), _stack(hr, "k_offsets"), p, votes=got)
    for h in range(len(heads)):
        assert np.array_equal(np_(cnt)[0, h], hr[h].counts)
        assert np.array_equal(np_(eg)[0, h], hr[h].exact_groups)
        assert np.array_equal(np_(sp)[0, h], hr[h].sample_pos)
    ig.device_status()
