"""Pins for the oracle's top-p key-group selection (the comparator the pages
run InstaGen against: thelatestinai.com paper page, Figure 2 caption, SVG2 at
top-p 0.5 / 0.75 / 0.9 / 0.95 with key floor 0.1; ICLR listing abstract: top-p
keeps the best blocks and varies their number to reach a target share of the
attention mass, skipping the rest).

Each check ties the selection to something other than its own code: a hand
example, the fp64 nucleus rule computed here from exp(S), the dense limit
against textbook softmax attention, and structural properties (prefix of one
ranking, monotone in p and in the floor, the top group always kept)."""
import numpy as np
import pytest
import torch


def _random_row(rng, Ck, n_max=60, spread=3.0, empty_frac=0.2):
    S = (rng.standard_normal(Ck) * spread).astype(np.float32)
    sizes = rng.integers(1, n_max, Ck)
    sizes[rng.random(Ck) < empty_frac] = 0
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    return S, offs


def test_hand_example_mass_order_share_and_floor(oracle_mod):
    # sizes 10, 20, 5, 65; scores 1.0, 0.5, 2.0, 0.1 -> masses proportional to
    # size * exp(S - 2): 3.68, 4.46, 5.00, 9.72 (total 22.86), so the nucleus
    # order is 3, 2, 1, 0 with cumulative shares 0.425, 0.644, 0.839, 1
    S = np.array([1.0, 0.5, 2.0, 0.1], np.float32)
    offs = np.array([0, 10, 30, 35, 100], np.int32)
    sel = lambda p, F: list(oracle_mod.select_top_p_group(S, offs, p, F)["exact_groups"])
    assert sel(0.3, 0) == [3]
    assert sel(0.5, 0) == [3, 2]
    assert sel(0.7, 0) == [3, 2, 1]
    assert sel(0.9, 0) == [3, 2, 1, 0]
    # the key floor keeps adding groups until the kept keys reach it
    assert sel(0.5, 70) == [3, 2]          # 65 + 5 = 70 keys: the floor is met exactly
    assert sel(0.5, 80) == [3, 2, 1]       # 90 keys
    assert sel(0.5, 95) == [3, 2, 1, 0]    # 100 keys
    assert sel(0.0, 0) == [3]              # the first-ranked group is always kept
    r = oracle_mod.select_top_p_group(S, offs, 0.5, 80)
    assert r["exact_keys"] == 90 and r["n_sample"] == 0


def test_equal_masses_tie_to_lower_group(oracle_mod):
    S = np.zeros(5, np.float32)
    offs = np.array([0, 4, 8, 12, 16, 20], np.int32)
    r = oracle_mod.select_top_p_group(S, offs, 0.5, 0)
    assert list(r["exact_groups"]) == [0, 1, 2]   # 3/5 of the mass is the first prefix >= 1/2


def test_matches_fp64_nucleus_rule(oracle_mod):
    """Away from near-ties, the kept set is the shortest prefix of the groups
    sorted by |K_j| exp(S_j) (fp64) whose share of the total reaches p."""
    rng = np.random.default_rng(3)
    checked = 0
    for trial in range(300):
        Ck = int(rng.integers(3, 40))
        S, offs = _random_row(rng, Ck)
        size = np.diff(offs).astype(np.float64)
        if (size > 0).sum() < 2:
            continue
        mass = np.where(size > 0, size * np.exp(S.astype(np.float64) - S[size > 0].max()), 0.0)
        nz = np.nonzero(size > 0)[0]
        order = nz[np.lexsort((nz, -mass[nz]))]
        m_sorted = mass[order]
        if np.any(np.abs(np.diff(m_sorted)) <= 1e-3 * m_sorted[1:]):
            continue  # near-tie: the integer weights may order it either way
        share = np.cumsum(m_sorted) / m_sorted.sum()
        for p in (0.1, 0.33, 0.5, 0.75, 0.9, 0.95, 0.99):
            if np.any(np.abs(share - p) < 1e-3):
                continue  # p on a prefix boundary within the weights' precision
            k = int(np.searchsorted(share, p) + 1)
            r = oracle_mod.select_top_p_group(S, offs, p, 0)
            assert list(r["exact_groups"]) == list(order[:k]), (trial, p)
            checked += 1
    assert checked > 300


def test_prefix_of_one_ranking_and_monotone(oracle_mod):
    rng = np.random.default_rng(7)
    for _ in range(60):
        Ck = int(rng.integers(2, 64))
        S, offs = _random_row(rng, Ck)
        if offs[-1] == 0:
            continue
        N = int(offs[-1])
        prev = []
        for p in np.linspace(0.0, 1.0, 21):
            ex = list(oracle_mod.select_top_p_group(S, offs, float(p), 0)["exact_groups"])
            assert ex[:len(prev)] == prev and len(ex) >= len(prev)
            prev = ex
        prev = []
        for F in np.linspace(0, N, 11).astype(int):
            ex = list(oracle_mod.select_top_p_group(S, offs, 0.3, int(F))["exact_groups"])
            assert ex[:len(prev)] == prev and len(ex) >= len(prev)
            assert np.diff(offs)[ex].sum() >= F
            prev = ex


def test_p_one_keeps_every_group_and_equals_dense_attention(oracle_mod):
    """p = 1 needs the whole mass: every non-empty group is kept, and the
    attention over them is textbook softmax attention."""
    rng = np.random.default_rng(11)
    N, d, Cq, Ck = 384, 32, 4, 16
    Q = rng.standard_normal((N, d)).astype(np.float32)
    K = rng.standard_normal((N, d)).astype(np.float32)
    V = rng.standard_normal((N, d)).astype(np.float32)
    scale = float(np.float32(1.0 / np.sqrt(d)))  # the oracle takes the scale in fp32
    res = oracle_mod.forward_head(Q, K, V, Cq=Cq, Ck=Ck, iters=3, exact_frac=0.0, sample_frac=0.0,
                                  scale=scale, selection="top_p", top_p=1.0, key_floor=0.0)
    nonempty = int((np.diff(res.k_offsets) > 0).sum())
    assert np.all(res.counts[:, 0] == nonempty) and np.all(res.counts[:, 1] == N) and np.all(res.counts[:, 2] == 0)
    q = torch.from_numpy(Q.astype(np.float64))
    k = torch.from_numpy(K.astype(np.float64))
    v = torch.from_numpy(V.astype(np.float64))
    dense = (torch.softmax(scale * q @ k.T, dim=-1) @ v).numpy()
    np.testing.assert_allclose(res.out, dense, rtol=1e-12, atol=1e-12)


def test_floor_of_all_keys_is_dense(oracle_mod):
    rng = np.random.default_rng(5)
    S, offs = _random_row(rng, 30)
    r = oracle_mod.select_top_p_group(S, offs, 0.0, int(offs[-1]))
    assert r["exact_keys"] == int(offs[-1])
