"""Pins for the CPU oracle: each check ties an oracle function to something
other than itself (a library routine, brute force, a closed form, a special
case that reduces to textbook attention, or PyTorch's open-source Philox
engine), chosen so that a dropped term, wrong sign/index or transposed operand
fails at least one of them.

Method statements come from the InstaGen pages (arXiv 2611.08610 abstract;
thelatestinai.com paper page, Figure 3 (a)-(d); acceptodds.com ICLR listing).
"""
import math
import os
import subprocess
import tempfile
from fractions import Fraction

import numpy as np
import pytest
import torch

from block_sparse_attention_head_b200 import workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# --------------------------------------------------------------------- helpers
def _f32_round(x: Fraction) -> Fraction:
    """Exact rational -> nearest fp32 (ties to even), as a Fraction (normal range)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    # fix e so that 2^e <= a < 2^(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 23)
    n = a / ulp
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def _dense_attention(Q, K, V, scale):
    """Textbook softmax attention in fp64 via torch library ops."""
    q = torch.from_numpy(np.asarray(Q, np.float64))
    k = torch.from_numpy(np.asarray(K, np.float64))
    v = torch.from_numpy(np.asarray(V, np.float64))
    return (torch.softmax(scale * q @ k.T, dim=-1) @ v).numpy()


def _head(w, N=None, bh=0):
    Q, K, V = workloads.make_inputs(w, N=N, heads=[bh])
    return Q[0, 0].float().numpy(), K[0, 0].float().numpy(), V[0, 0].float().numpy()


# ----------------------------------------------------------------- Philox (P7)
def test_philox_matches_pytorch_engine(oracle_mod):
    inc = os.path.join(os.path.dirname(torch.__file__), "include")
    with tempfile.TemporaryDirectory() as td:
        exe = os.path.join(td, "probe")
        subprocess.run(["g++", "-std=c++17", "-O2", "-I" + inc,
                        os.path.join(ROOT, "tests", "torch_philox_probe.cpp"), "-o", exe], check=True)
        rng = np.random.default_rng(1234)
        n = 1_000_000
        rec = rng.integers(0, 2 ** 32, size=(n, 6), dtype=np.uint64).astype(np.uint32)
        # include structured counters like the ones the sampler uses
        rec[:1000, 0] = np.arange(1000)
        rec[:1000, 1:4] = [3, 7, 0]
        rec[:1000, 4:6] = [0, 0]
        res = subprocess.run([exe], input=rec.tobytes(), stdout=subprocess.PIPE, check=True)
        ref = np.frombuffer(res.stdout, dtype=np.uint32).reshape(n, 4)
    got = oracle_mod.philox4x32_10(rec[:, :4], rec[:, 4:6])
    assert np.array_equal(got, ref)


# --------------------------------------------------------------------- budgets
def test_budget_rounding(oracle_mod):
    assert oracle_mod.budget(0.08, 4096) == 328          # 327.68
    assert oracle_mod.budget(0.16, 75600) == 12096       # 12096.0000...
    assert oracle_mod.budget(0.5, 3) == 2                # 1.5 -> away from zero
    assert oracle_mod.budget(0.0, 1000) == 0
    assert oracle_mod.budget(1.0, 75600) == 75600


# -------------------------------------------------------------- k-means (P5)
def test_kmeans_assign_is_library_argmin(oracle_mod):
    from scipy.spatial.distance import cdist
    Q, K, _ = _head(workloads.TINY, N=1500)
    cent = oracle_mod.kmeans_init(K, 37)
    a, inertia = oracle_mod.kmeans_assign(K, cent)
    D = cdist(K.astype(np.float64), cent.astype(np.float64), "sqeuclidean")
    assert np.array_equal(a, D.argmin(axis=1))
    assert inertia == pytest.approx(D.min(axis=1).sum(), rel=1e-12)


def test_kmeans_init_and_ties(oracle_mod):
    X = np.random.default_rng(0).standard_normal((10, 4)).astype(np.float32)
    cent = oracle_mod.kmeans_init(X, 4)
    assert np.array_equal(cent, X[[0, 2, 5, 7]])          # floor(j*10/4)
    # duplicated centroids: the lowest index wins every tie
    dup = np.stack([cent[1], cent[0], cent[1], cent[0]])
    a, _ = oracle_mod.kmeans_assign(X, dup)
    assert set(np.unique(a)) <= {0, 1}


def test_kmeans_update_means_and_empty(oracle_mod):
    rng = np.random.default_rng(1)
    X = rng.standard_normal((200, 8)).astype(np.float32)
    a = rng.integers(0, 5, 200).astype(np.int32)
    a[a == 3] = 2                                         # cluster 3 empty
    old = rng.standard_normal((5, 8)).astype(np.float32)
    new = oracle_mod.kmeans_update(X, a, old)
    for j in range(5):
        if j == 3:
            assert np.array_equal(new[j], old[j])
        else:
            ref = np.mean(X[a == j].astype(np.float64), axis=0).astype(np.float32)
            np.testing.assert_array_max_ulp(new[j], ref, maxulp=1)


def test_kmeans_matches_sklearn_lloyd(oracle_mod):
    from sklearn.cluster import KMeans
    w = workloads.TINY
    _, K, _ = _head(w, N=2048)
    C, T = 16, 60
    init = oracle_mod.kmeans_init(K, C)
    cent, a, hist = oracle_mod.kmeans(K, C, T)
    km = KMeans(n_clusters=C, init=init.astype(np.float64), n_init=1, max_iter=T, tol=0.0,
                algorithm="lloyd").fit(K.astype(np.float64))
    assert km.n_iter_ < T, "reference run did not converge; pick a larger T"
    np.testing.assert_allclose(cent, km.cluster_centers_, rtol=0, atol=1e-5)
    assert np.array_equal(a, km.labels_)
    assert np.all(np.diff(hist) <= 1e-9 * hist[0])     # Lloyd never increases inertia


def test_kmeans_recovers_planted_mixture(oracle_mod):
    w = workloads.TINY
    Q, K, V, ql, kl = workloads.make_labelled_head(w)
    K = K.float().numpy()
    cent, a, hist = oracle_mod.kmeans(K, 64, 10)
    kl = kl.numpy()
    # purity: share of tokens whose cluster's majority planted label is theirs.
    # Data-point init covers only part of the 64 planted centres, so Lloyd ends
    # in a local optimum; it must still clearly improve on the initial split.
    def purity(assign):
        return sum(np.bincount(kl[assign == j]).max() for j in range(64) if np.any(assign == j)) / len(assign)
    a0, _ = oracle_mod.kmeans_assign(K, oracle_mod.kmeans_init(K, 64))
    assert purity(a) > 0.75 and purity(a) > purity(a0) + 0.1
    assert np.all(np.diff(hist) <= 1e-9 * hist[0])
    # final centroids are the means of the final clusters
    for j in range(64):
        if np.any(a == j):
            np.testing.assert_allclose(cent[j], K[a == j].astype(np.float64).mean(0), rtol=0, atol=1e-6)


# ---------------------------------------------------------- permutation (P6)
def test_permutation_is_stable_sort(oracle_mod):
    rng = np.random.default_rng(2)
    a = rng.integers(0, 11, 5000).astype(np.int32)
    a[a == 4] = 5                                         # an empty cluster
    perm, off = oracle_mod.permutation(a, 11)
    assert np.array_equal(perm, np.argsort(a, kind="stable"))
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(a, minlength=11))]))
    assert np.array_equal(np.sort(perm), np.arange(5000))
    perm1, off1 = oracle_mod.permutation(np.zeros(77, np.int32), 1)
    assert np.array_equal(perm1, np.arange(77)) and list(off1) == [0, 77]


# -------------------------------------------------------------- scores (3b)
def test_scores_fmaf_chain_exact(oracle_mod):
    rng = np.random.default_rng(3)
    cq = rng.standard_normal((3, 16)).astype(np.float32)
    ck = rng.standard_normal((4, 16)).astype(np.float32)
    scale = np.float32(0.125)
    S = oracle_mod.scores(cq, ck, scale)
    for i in range(3):
        for j in range(4):
            acc = Fraction(0)
            for k in range(16):
                acc = _f32_round(Fraction(float(cq[i, k])) * Fraction(float(ck[j, k])) + acc)
            ref = _f32_round(acc * Fraction(float(scale)))
            assert Fraction(float(S[i, j])) == ref
    # and it is the scaled dot product, not its transpose
    np.testing.assert_allclose(S, scale * (cq.astype(np.float64) @ ck.T.astype(np.float64)), atol=1e-5)


# ------------------------------------------------------------- weights pi (3b,c)
def test_taylor_coefficients_are_exp2_series(oracle_mod):
    from decimal import Decimal, getcontext
    getcontext().prec = 60
    ln2 = Decimal(2).ln()
    c = oracle_mod.taylor_coefficients()
    for k in range(7):
        exact = ln2 ** k / math.factorial(k)
        assert c[k] == np.float32(float(exact))


def test_group_weight_tracks_exp(oracle_mod):
    for y in np.linspace(-23.99, 0.0, 4001):
        s = np.float32(y / np.float32(1.4426950408889634))
        q = oracle_mod.group_weight(float(s), 0.0)
        yy = float(np.float32(np.float32(s - np.float32(0.0)) * np.float32(1.4426950408889634)))
        assert 1 <= q <= 2 ** 24
        ref = 2.0 ** (24 + yy)
        assert abs(q - ref) <= 1.0 + 1e-4 * ref          # floor (<= 1) + series truncation
    assert oracle_mod.group_weight(3.0, 3.0) == 2 ** 24
    assert oracle_mod.group_weight(-100.0, 0.0) == 1
    assert oracle_mod.group_weight(-16.7, 0.0) == 1       # y < -24


# ------------------------------------------------------------ exact set (3c, P4)
def test_exact_set_prefix_rule_hand_example(oracle_mod):
    S = np.array([0.5, 2.0, 1.0, 2.0, -1.0, 3.0], np.float32)
    counts = [3, 5, 2, 4, 0, 10]
    koff = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    r = oracle_mod.select_sample_group(S, koff, 0, E=12, m=0)
    assert list(r["exact_groups"]) == [5]                 # 10 fits, 10+5 does not: stop there
    r = oracle_mod.select_sample_group(S, koff, 0, E=15, m=0)
    assert list(r["exact_groups"]) == [5, 1]              # tie 2.0: lower j (1) before 3
    r = oracle_mod.select_sample_group(S, koff, 0, E=19, m=0)
    assert list(r["exact_groups"]) == [5, 1, 3]
    r = oracle_mod.select_sample_group(S, koff, 0, E=0, m=4)
    assert list(r["exact_groups"]) == [5]                 # top group always kept (Figure 3c)
    assert r["exact_keys"] == 10 and r["n_sample"] == 4
    r = oracle_mod.select_sample_group(S, koff, 0, E=24, m=4)
    assert sorted(r["exact_groups"]) == [0, 1, 2, 3, 5] and r["n_sample"] == 0  # nothing skipped


@pytest.mark.parametrize("exact_frac", [0.0, 0.02, 0.16, 0.5])
def test_top_group_always_kept(oracle_mod, exact_frac):
    w = workloads.TINY
    Q, K, V = _head(w, N=1024)
    hr = oracle_mod.forward_head(Q, K, V, Cq=8, Ck=32, iters=3, exact_frac=exact_frac, sample_frac=0.05,
                                 scale=w.softmax_scale, rows=[])
    S = oracle_mod.scores(hr.cq, hr.ck, w.softmax_scale)
    nonempty = np.diff(hr.k_offsets) > 0
    for i in range(8):
        top = max(np.flatnonzero(nonempty), key=lambda j: (S[i, j], -j))
        assert hr.exact_groups[i, 0] == top
        assert hr.counts[i, 1] <= max(oracle_mod.budget(exact_frac, 1024),
                                      hr.k_offsets[top + 1] - hr.k_offsets[top])


# ------------------------------------------------------- sampling law (P3)
def _tiny_case(oracle_mod, mode):
    w = workloads.Workload("pin", 1, 1, 256, 16, 6, "uniform", (0.6, 0.6), 4, 8, 5, 0.10, 0.05, seed=9)
    Q, K, V = _head(w)
    hr = oracle_mod.forward_head(Q, K, V, Cq=4, Ck=8, iters=5, exact_frac=0.10, sample_frac=0.05,
                                 scale=w.softmax_scale, mode=mode, rows=[])
    return w, Q, K, V, hr


@pytest.mark.parametrize("mode", [0, 1])
def test_sampling_probabilities_closed_form(oracle_mod, mode):
    w, Q, K, V, hr = _tiny_case(oracle_mod, mode)
    S = oracle_mod.scores(hr.cq, hr.ck, w.softmax_scale)
    m = oracle_mod.budget(0.05, 256)
    for i in range(4):
        r = oracle_mod.select_sample_group(S[i], hr.k_offsets, i, oracle_mod.budget(0.10, 256), m,
                                           seed=5, mode=mode)
        cnt = np.diff(hr.k_offsets)
        skipped = [j for j in range(8) if cnt[j] > 0 and j not in set(r["exact_groups"])]
        assert r["total"] == sum(int(cnt[j]) * int(r["q"][j]) for j in skipped)   # p sums to 1
        if mode == 1:
            assert all(r["q"][j] == 1 for j in skipped)
        for t, p in enumerate(r["sample_pos"]):
            j = int(np.searchsorted(hr.k_offsets, p, side="right") - 1)
            assert j in skipped                                  # samples only from the skipped region
            prob = r["q"][j] / r["total"]
            assert math.exp(r["sample_bias"][t]) * prob * m == pytest.approx(1.0, rel=1e-12)


@pytest.mark.parametrize("mode", [0, 1])
def test_sample_frequencies_chi_square(oracle_mod, mode):
    from scipy.stats import chisquare
    w, Q, K, V, hr = _tiny_case(oracle_mod, mode)
    S = oracle_mod.scores(hr.cq, hr.ck, w.softmax_scale)
    i = int(np.argmax(np.diff(hr.q_offsets)))
    r = oracle_mod.select_sample_group(S[i], hr.k_offsets, i, 0, 200_000, seed=77, mode=mode)
    cnt = np.diff(hr.k_offsets)
    keys = [p for j in range(8) if cnt[j] > 0 and j not in set(r["exact_groups"])
            for p in range(hr.k_offsets[j], hr.k_offsets[j + 1])]
    probs = np.array([r["q"][np.searchsorted(hr.k_offsets, p, side="right") - 1] for p in keys],
                     np.float64) / r["total"]
    obs = np.array([np.count_nonzero(r["sample_pos"] == p) for p in keys])
    keep = probs * len(r["sample_pos"]) >= 5
    stat, pval = chisquare(obs[keep], probs[keep] / probs[keep].sum() * obs[keep].sum())
    assert pval > 1e-4


@pytest.mark.parametrize("mode", [0, 1])
def test_reweighted_sample_is_unbiased(oracle_mod, mode):
    """Monte-Carlo over seeds: the reweighted sampled numerator and
    denominator converge to the dense sums over the skipped keys."""
    w, Q, K, V, hr = _tiny_case(oracle_mod, mode)
    S = oracle_mod.scores(hr.cq, hr.ck, w.softmax_scale)
    E, m = oracle_mod.budget(0.10, 256), oracle_mod.budget(0.05, 256)
    i = int(np.argmax(np.diff(hr.q_offsets)))
    q_tok = int(hr.q_perm[hr.q_offsets[i]])
    r0 = oracle_mod.select_sample_group(S[i], hr.k_offsets, i, E, m, seed=0, mode=mode)
    skipped = [p for j in range(8) if np.diff(hr.k_offsets)[j] > 0 and j not in set(r0["exact_groups"])
               for p in range(hr.k_offsets[j], hr.k_offsets[j + 1])]
    Kp, Vp = K[hr.k_perm].astype(np.float64), V[hr.k_perm].astype(np.float64)
    logit = w.softmax_scale * (Kp @ Q[q_tok].astype(np.float64))
    den_true = np.exp(logit[skipped]).sum()
    num_true = (np.exp(logit[skipped])[:, None] * Vp[skipped]).sum(0)
    n_seeds = 20000
    den = np.empty(n_seeds)
    num = np.empty((n_seeds, Q.shape[1]))
    for s in range(n_seeds):
        r = oracle_mod.select_sample_group(S[i], hr.k_offsets, i, E, m, seed=s, mode=mode)
        wts = np.exp(logit[r["sample_pos"]] + r["sample_bias"])
        den[s] = wts.sum()
        num[s] = (wts[:, None] * Vp[r["sample_pos"]]).sum(0)
    se = den.std() / math.sqrt(n_seeds)
    assert abs(den.mean() - den_true) < 5 * se + 1e-12 * den_true
    se_n = num.std(0) / math.sqrt(n_seeds)
    assert np.all(np.abs(num.mean(0) - num_true) < 5 * se_n + 1e-9 * np.abs(num_true).max())


# --------------------------------------------------------- dense limits (P1, P2)
def test_dense_limit_exact_everything(oracle_mod):
    w = workloads.TINY
    Q, K, V = _head(w, N=512)
    hr = oracle_mod.forward_head(Q, K, V, Cq=5, Ck=12, iters=4, exact_frac=1.0, sample_frac=0.08,
                                 scale=w.softmax_scale)
    assert np.all(hr.counts[:, 2] == 0) and np.all(hr.counts[:, 1] == 512)
    ref = _dense_attention(Q, K, V, w.softmax_scale)
    np.testing.assert_allclose(hr.out, ref, rtol=1e-12, atol=1e-13)


def test_uniform_enumeration_is_dense(oracle_mod):
    """Uniform pi with the sample = every skipped key once: the log-weight is
    ln(R) - ln(1) - ln(R) = 0 and the call equals dense attention."""
    w = workloads.TINY
    Q, K, V = _head(w, N=384)
    hr = oracle_mod.forward_head(Q, K, V, Cq=4, Ck=10, iters=4, exact_frac=0.2, sample_frac=0.0,
                                 scale=w.softmax_scale, mode=1, rows=[])
    S = oracle_mod.scores(hr.cq, hr.ck, w.softmax_scale)
    E = oracle_mod.budget(0.2, 384)
    R_max = 384
    pos = np.full((4, R_max), -1, np.int32)
    bias = np.zeros((4, R_max))
    counts = hr.counts.copy()
    for i in range(4):
        r = oracle_mod.select_sample_group(S[i], hr.k_offsets, i, E, 1, mode=1)
        skipped = [p for j in range(10) if np.diff(hr.k_offsets)[j] > 0 and j not in set(r["exact_groups"])
                   for p in range(hr.k_offsets[j], hr.k_offsets[j + 1])]
        R = len(skipped)
        assert r["total"] == R
        pos[i, :R] = skipped
        bias[i, :R] = math.log(r["total"]) - math.log(1) - math.log(R)
        counts[i, 2] = R
    out = oracle_mod.attention_rows(Q, K, V, w.softmax_scale, hr.q_assign, hr.k_perm, hr.k_offsets,
                                    hr.exact_groups, counts, pos, bias, np.arange(384))
    np.testing.assert_allclose(out, _dense_attention(Q, K, V, w.softmax_scale), rtol=1e-12, atol=1e-13)


def test_singleton_groups_give_topk_attention(oracle_mod):
    """Cq = Ck = N and no sample: every token is its own group, the exact set is
    the top-E keys per query and the call is textbook top-k attention."""
    rng = np.random.default_rng(11)
    N, d, E = 48, 16, 9
    Q = torch.from_numpy(rng.standard_normal((N, d))).to(torch.bfloat16).float().numpy()
    K = torch.from_numpy(rng.standard_normal((N, d))).to(torch.bfloat16).float().numpy()
    V = torch.from_numpy(rng.standard_normal((N, d))).to(torch.bfloat16).float().numpy()
    scale = 0.25
    hr = oracle_mod.forward_head(Q, K, V, Cq=N, Ck=N, iters=2, exact_frac=E / N, sample_frac=0.0, scale=scale)
    assert np.array_equal(hr.q_assign, np.arange(N)) and np.array_equal(hr.k_assign, np.arange(N))
    logits = scale * (Q.astype(np.float64) @ K.T.astype(np.float64))
    checked = 0
    for qi in range(N):
        srt = np.sort(logits[qi])[::-1]
        if srt[E - 1] - srt[E] < 1e-4:
            continue                                       # near-tie at the boundary: skip
        top = np.argsort(-logits[qi])[:E]
        assert set(hr.exact_groups[qi, :hr.counts[qi, 0]]) == set(top)
        ref = torch.softmax(torch.from_numpy(logits[qi, top]), 0).numpy() @ V[top].astype(np.float64)
        np.testing.assert_allclose(hr.out[qi], ref, rtol=1e-12, atol=1e-13)
        checked += 1
    assert checked > N // 2


def test_attention_rows_counts_duplicates(oracle_mod):
    """A key drawn twice enters the softmax twice, with its log-weight."""
    rng = np.random.default_rng(5)
    N, d = 20, 8
    Q, K, V = (rng.standard_normal((N, d)).astype(np.float32) for _ in range(3))
    q_assign = np.zeros(N, np.int32)
    k_perm = np.arange(N, dtype=np.int32)
    k_off = np.array([0, 6, 20], np.int32)
    ex = np.array([[0, -1]], np.int32)
    cnt = np.array([[1, 6, 3]], np.int32)
    pos = np.array([[7, 7, 15]], np.int32)
    bias = np.array([[0.3, 0.3, -0.2]])
    out = oracle_mod.attention_rows(Q, K, V, 0.5, q_assign, k_perm, k_off, ex, cnt, pos, bias, [4])
    keys = [0, 1, 2, 3, 4, 5, 7, 7, 15]
    b = np.array([0, 0, 0, 0, 0, 0, 0.3, 0.3, -0.2])
    lg = 0.5 * (K[keys].astype(np.float64) @ Q[4].astype(np.float64)) + b
    ref = torch.softmax(torch.from_numpy(lg), 0).numpy() @ V[keys].astype(np.float64)
    np.testing.assert_allclose(out[0], ref, rtol=1e-13)


def test_error_falls_with_sample_size(oracle_mod):
    """The tiny configuration (N=4096, d=64, Cq=16, Ck=64, exact 8%) runs in
    seconds; its error against dense attention falls as the sample grows
    (ICLR listing: the reconstruction error shrinks as the sample grows;
    an i.i.d. estimator's error shrinks like 1/sqrt(m)), and importance
    sampling beats uniform at every size (Figure 4 caption)."""
    w = workloads.TINY
    Q, K, V = _head(w)
    rows = np.arange(0, 4096, 7)
    dense = _dense_attention(Q[rows], K, V, w.softmax_scale)
    err = {}
    for mode in (0, 1):
        for sf in (0.08, 0.32, 1.28):
            hr = oracle_mod.forward_head(Q, K, V, Cq=w.Cq, Ck=w.Ck, iters=w.iters, exact_frac=w.exact_frac,
                                         sample_frac=sf, scale=w.softmax_scale, rows=rows, mode=mode)
            if sf == 0.08:
                assert np.all(hr.counts[:, 2][np.diff(hr.q_offsets) > 0] == 328)
            err[mode, sf] = np.linalg.norm(hr.out - dense) / np.linalg.norm(dense)
    for mode in (0, 1):
        assert err[mode, 0.32] < 0.75 * err[mode, 0.08]
        assert err[mode, 1.28] < 0.75 * err[mode, 0.32]
    for sf in (0.08, 0.32, 1.28):
        assert err[0, sf] < err[1, sf]
