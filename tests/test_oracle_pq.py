"""Pins of the oracle's product-quantised voting selection (the abstract's
selection rule; its parameters are readings: 8-dimension subspaces, 16
codewords, 5 Lloyd iterations on the group centroids, per-query budget
prefix, votes then centroid score).  Each check is against something other
than the oracle's own formula: the identity codebook of <= 16 points, cluster
means of separated data, brute-force nearest codewords in fp64, brute-force
per-query rankings by the exact dot product, and the centroid-ranked
selection the vote ranking reduces to."""
import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def test_codebook_of_at_most_16_points_is_the_points():
    P = _rng(1).standard_normal((11, 32)).astype(np.float32)
    cb, codes, kc = oracle.pq_codebook(P)
    assert kc == 11
    for m in range(4):
        np.testing.assert_array_equal(cb[m, :11], P[:, 8 * m:8 * m + 8])
        np.testing.assert_array_equal(codes[:, m], np.arange(11))


def test_codebook_of_separated_clusters_is_their_means():
    """16 tight, far-apart clusters per subspace, the first 16 points one per
    cluster: Lloyd settles on the cluster means after one step."""
    rng = _rng(2)
    C, d = 160, 16
    centres = rng.standard_normal((16, d)) * 50.0
    lab = np.concatenate([np.arange(16), rng.integers(0, 16, C - 16)])
    P = (centres[lab] + 0.01 * rng.standard_normal((C, d))).astype(np.float32)
    cb, codes, kc = oracle.pq_codebook(P)
    assert kc == 16
    for m in range(d // 8):
        np.testing.assert_array_equal(codes[:, m], lab)
        for c in range(16):
            mean = P[lab == c, 8 * m:8 * m + 8].astype(np.float64).mean(0)
            np.testing.assert_allclose(cb[m, c], mean, rtol=0, atol=1e-4)


def test_encode_is_the_nearest_codeword():
    rng = _rng(3)
    cb = rng.standard_normal((4, 16, 8)).astype(np.float32)
    X = rng.standard_normal((500, 32)).astype(np.float32)
    codes = oracle.pq_encode(X, cb, 16)
    for m in range(4):
        dist = ((X[:, None, 8 * m:8 * m + 8].astype(np.float64) - cb[m][None].astype(np.float64)) ** 2).sum(-1)
        srt = np.sort(dist, 1)
        clear = srt[:, 1] - srt[:, 0] > 1e-4 * srt[:, 1]
        assert clear.mean() > 0.95
        np.testing.assert_array_equal(codes[clear, m], dist.argmin(1)[clear])


def _prefix(scores, sizes, E):
    """Brute force: non-empty groups by score desc (ties: lowest j), rank 0
    always, then while the running key count stays <= E."""
    order = sorted((j for j in range(len(sizes)) if sizes[j] > 0), key=lambda j: (-scores[j], j))
    out, keys = [], 0
    for r, j in enumerate(order):
        if r > 0 and keys + sizes[j] > E:
            break
        out.append(j)
        keys += sizes[j]
    return out


def test_votes_equal_exact_dot_rankings_when_the_codebooks_are_exact():
    """Cq, Ck <= 16: both codebooks are the centroids themselves; queries that
    equal their group centroid then score every key group by the exact dot
    product <cq_i, ck_j>, so their votes follow a brute-force ranking."""
    rng = _rng(4)
    Cq, Ck, d = 5, 12, 32
    cq = rng.standard_normal((Cq, d)).astype(np.float32)
    ck = rng.standard_normal((Ck, d)).astype(np.float32)
    n_i = np.array([3, 1, 4, 2, 5])
    Q = np.repeat(cq, n_i, axis=0)
    q_perm = np.arange(Q.shape[0], dtype=np.int32)
    q_offsets = np.concatenate([[0], np.cumsum(n_i)]).astype(np.int32)
    sizes = rng.integers(1, 40, Ck)
    sizes[7] = 0  # an empty key group never gets a vote
    k_offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    E = int(sizes.sum() * 0.4)
    votes = oracle.pq_votes(Q, cq, ck, q_perm, q_offsets, k_offsets, E)
    dots = cq.astype(np.float64) @ ck.astype(np.float64).T
    for i in range(Cq):
        srt = np.sort(dots[i])
        assert np.min(np.diff(srt)) > 1e-4  # no near-ties in this draw
        want = np.zeros(Ck, np.int32)
        want[_prefix(dots[i], sizes, E)] = n_i[i]
        np.testing.assert_array_equal(votes[i], want)


def test_vote_totals():
    """Every query votes for its own budget prefix: a group's votes sum to the
    sum of its queries' prefix lengths, each at most the group's size, and
    every group's top-scored key group of each query counts."""
    rng = _rng(5)
    N, d, Cq, Ck = 600, 32, 6, 40
    Q = rng.standard_normal((N, d)).astype(np.float32)
    cq = rng.standard_normal((Cq, d)).astype(np.float32)
    ck = rng.standard_normal((Ck, d)).astype(np.float32)
    qa = rng.integers(0, Cq, N)
    q_perm = np.argsort(qa, kind="stable").astype(np.int32)
    q_offsets = np.concatenate([[0], np.cumsum(np.bincount(qa, minlength=Cq))]).astype(np.int32)
    sizes = rng.integers(0, 30, Ck)
    k_offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    E = int(sizes.sum() * 0.25)
    votes = oracle.pq_votes(Q, cq, ck, q_perm, q_offsets, k_offsets, E)
    n_i = np.diff(q_offsets)
    assert (votes >= 0).all() and (votes <= n_i[:, None]).all()
    assert (votes[:, sizes == 0] == 0).all()
    assert (votes.sum(1) >= n_i).all()  # at least the rank-0 group per query
    # budget: a query's prefix holds at most E keys unless it is one group
    per_query_keys_max = E + sizes.max()
    assert (votes * sizes[None]).sum(1).max() <= n_i.max() * per_query_keys_max


def test_vote_ranking_reduces_to_centroid_ranking_for_equal_votes():
    rng = _rng(6)
    Cq, Ck, d = 4, 30, 32
    cq = rng.standard_normal((Cq, d)).astype(np.float32)
    ck = rng.standard_normal((Ck, d)).astype(np.float32)
    sizes = rng.integers(1, 50, Ck)
    ko = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    E, m = int(sizes.sum() * 0.3), 64
    base = oracle.select_sample(cq, ck, ko, 0.125, E, m, seed=9)
    flat = oracle.select_sample(cq, ck, ko, 0.125, E, m, seed=9, votes=np.full((Cq, Ck), 3, np.int32))
    for a, b in zip(base, flat):
        np.testing.assert_array_equal(a, b)


def test_vote_ranking_takes_votes_first():
    """Hand case: three key groups of 10 keys, E = 20: the two most-voted
    groups form the exact set whatever their centroid scores, a vote tie is
    broken by the higher score."""
    S_row = np.array([3.0, 2.0, 1.0], np.float32)
    ko = np.array([0, 10, 20, 30], np.int32)
    r = oracle.select_sample_group(S_row, ko, 0, E=20, m=0, votes=np.array([1, 5, 5], np.int32))
    np.testing.assert_array_equal(r["exact_groups"], [1, 2])
    r = oracle.select_sample_group(S_row, ko, 0, E=20, m=0, votes=np.array([0, 0, 7], np.int32))
    np.testing.assert_array_equal(r["exact_groups"], [2, 0])


def test_forward_head_pq_vote_runs_and_differs_only_in_the_exact_sets():
    rng = _rng(7)
    N, d = 512, 32
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = rng.standard_normal((N, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    kw = dict(Cq=8, Ck=24, iters=3, exact_frac=0.2, sample_frac=0.1, scale=d ** -0.5, seed=3, rows=np.arange(16))
    a = oracle.forward_head(Q, K, V, **kw)
    b = oracle.forward_head(Q, K, V, selection="pq_vote", **kw)
    np.testing.assert_array_equal(a.q_perm, b.q_perm)
    np.testing.assert_array_equal(a.k_offsets, b.k_offsets)
    assert b.out.shape == (16, d) and np.isfinite(b.out).all()
    # the exact-key budget rule holds for both rankings
    for r in (a, b):
        sizes = np.diff(r.k_offsets)
        for i in range(8):
            ne = r.counts[i, 0]
            keys = sizes[r.exact_groups[i, :ne]].sum()
            assert keys == r.counts[i, 1]
            assert ne == 1 or keys <= oracle.budget(0.2, N)
