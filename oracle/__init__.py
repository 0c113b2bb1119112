"""CPU oracle for InstaGen group-shared importance-sampled permuted block-sparse
attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg
may import this package.  The product path (``block_sparse_attention_head_b200``)
never does and shares no code with it.  The arithmetic lives in
``instagen_oracle.c`` (plain C, fp64 except where an integer decision needs a
reproducible fp32 rule); this module only builds that file with gcc, marshals
numpy arrays through ctypes and strings the per-stage functions together in
the pages' order: cluster (Figure 3a) -> permute -> score (3b) -> exact set and
sample (3c) -> attention over exact keys plus the weighted sample (3d).

Every function is pinned by ``tests/test_oracle_pins.py`` against something
other than itself (closed forms, brute force, library routines, PyTorch's
open-source Philox engine).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "instagen_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (OpenMP, no FMA contraction)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-D_GNU_SOURCE", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _SelectCfg(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int64), ("m", ctypes.c_int64), ("seed", ctypes.c_uint64),
                ("layer", ctypes.c_uint32), ("bh", ctypes.c_uint32), ("mode", ctypes.c_int)]


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    i64, i32, u32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_uint32, ctypes.c_float
    lib.orc_philox_batch.argtypes = [i64, P, P, P]
    lib.orc_budget.argtypes = [f32, i64]
    lib.orc_budget.restype = i64
    lib.orc_kmeans_init.argtypes = [P, i64, i32, i32, P]
    lib.orc_kmeans_assign.argtypes = [P, i64, i32, P, i32, P, P]
    lib.orc_kmeans_update.argtypes = [P, i64, i32, P, i32, P]
    lib.orc_kmeans_update.restype = i32
    lib.orc_kmeans.argtypes = [P, i64, i32, i32, i32, P, P, P, P]
    lib.orc_kmeans.restype = i32
    lib.orc_permutation.argtypes = [P, i64, i32, P, P]
    lib.orc_permutation.restype = i32
    lib.orc_scores.argtypes = [P, i32, P, i32, i32, f32, P]
    lib.orc_taylor_coefficients.argtypes = [P]
    lib.orc_group_weight.argtypes = [f32, f32]
    lib.orc_group_weight.restype = u32
    lib.orc_select_sample_group.argtypes = [P, P, i32, i32, ctypes.POINTER(_SelectCfg), P,
                                            P, P, P, P, P, P]
    lib.orc_select_sample_group.restype = i32
    lib.orc_select_sample.argtypes = [P, i32, P, i32, i32, f32, P, ctypes.POINTER(_SelectCfg), P,
                                      P, P, P, P]
    lib.orc_select_top_p_group.argtypes = [P, P, i32, f32, i64, P, P, P, P]
    lib.orc_select_top_p_group.restype = i32
    lib.orc_select_top_p.argtypes = [P, i32, P, i32, i32, f32, P, f32, i64, P, P]
    lib.orc_select_top_p.restype = i32
    lib.orc_pq_codebook.argtypes = [P, i32, i32, P, P]
    lib.orc_pq_codebook.restype = i32
    lib.orc_pq_encode.argtypes = [P, i64, i32, P, i32, P]
    lib.orc_pq_votes.argtypes = [P, i64, i32, P, P, i32, P, i32, P, i32, P, P, i32, i64, P]
    lib.orc_pq_votes.restype = i32
    lib.orc_select_sample.restype = i32
    lib.orc_attention_rows.argtypes = [P, P, P, i64, i32, f32, P, P, P, i32, P, P, P, P, i64,
                                       P, i64, P]
    lib.orc_attention_rows.restype = i32
    lib.orc_num_threads.restype = i32
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use."""
    return int(_load().orc_num_threads())


# --------------------------------------------------------------------------- RNG
def philox4x32_10(counters: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """Philox4x32-10 on rows of counters [n,4] and keys [n,2] (uint32)."""
    lib = _load()
    c = np.ascontiguousarray(counters, dtype=np.uint32).reshape(-1, 4)
    k = np.ascontiguousarray(keys, dtype=np.uint32).reshape(-1, 2)
    assert c.shape[0] == k.shape[0]
    out = np.empty_like(c)
    lib.orc_philox_batch(c.shape[0], _ptr(c), _ptr(k), _ptr(out))
    return out


def budget(frac: float, n: int) -> int:
    """Keys for a share of N (nearest, halves away from zero)."""
    return int(_load().orc_budget(float(np.float32(frac)), int(n)))


# ----------------------------------------------------------------------- k-means
def kmeans_init(X: np.ndarray, C: int) -> np.ndarray:
    lib = _load()
    X = _f32(X)
    N, d = X.shape
    cent = np.empty((C, d), np.float32)
    lib.orc_kmeans_init(_ptr(X), N, d, C, _ptr(cent))
    return cent


def kmeans_assign(X: np.ndarray, cent: np.ndarray):
    """(assign, inertia): nearest centroid in fp64, lowest index on ties."""
    lib = _load()
    X, cent = _f32(X), _f32(cent)
    N, d = X.shape
    a = np.empty(N, np.int32)
    inertia = ctypes.c_double(0.0)
    lib.orc_kmeans_assign(_ptr(X), N, d, _ptr(cent), cent.shape[0], _ptr(a), ctypes.byref(inertia))
    return a, inertia.value


def kmeans_update(X: np.ndarray, assign: np.ndarray, cent: np.ndarray) -> np.ndarray:
    lib = _load()
    X, a = _f32(X), _i32(assign)
    out = _f32(cent).copy()
    _check(lib.orc_kmeans_update(_ptr(X), X.shape[0], X.shape[1], _ptr(a), out.shape[0], _ptr(out)),
           "kmeans_update")
    return out


def kmeans(X: np.ndarray, C: int, iters: int, init: Optional[np.ndarray] = None):
    """(centroids [C,d] fp32, assign [N] int32, inertia per iteration)."""
    lib = _load()
    X = _f32(X)
    N, d = X.shape
    cent = np.empty((C, d), np.float32)
    a = np.empty(N, np.int32)
    hist = np.empty(iters, np.float64)
    keep = _f32(init) if init is not None else None
    init_p = _ptr(keep) if keep is not None else None
    _check(lib.orc_kmeans(_ptr(X), N, d, C, iters, init_p, _ptr(cent), _ptr(a), _ptr(hist)), "kmeans")
    return cent, a, hist


def permutation(assign: np.ndarray, C: int):
    """(perm [N], offsets [C+1]) of the stable counting sort by cluster."""
    lib = _load()
    a = _i32(assign)
    perm = np.empty(a.shape[0], np.int32)
    off = np.empty(C + 1, np.int32)
    _check(lib.orc_permutation(_ptr(a), a.shape[0], C, _ptr(perm), _ptr(off)), "permutation")
    return perm, off


# ------------------------------------------------------------- scores / selection
def scores(cq: np.ndarray, ck: np.ndarray, scale: float) -> np.ndarray:
    lib = _load()
    cq, ck = _f32(cq), _f32(ck)
    S = np.empty((cq.shape[0], ck.shape[0]), np.float32)
    lib.orc_scores(_ptr(cq), cq.shape[0], _ptr(ck), ck.shape[0], cq.shape[1], float(np.float32(scale)),
                   _ptr(S))
    return S


def taylor_coefficients() -> np.ndarray:
    out = np.empty(7, np.float32)
    _load().orc_taylor_coefficients(_ptr(out))
    return out


def group_weight(s: float, smax: float) -> int:
    return int(_load().orc_group_weight(float(np.float32(s)), float(np.float32(smax))))


IMPORTANCE, UNIFORM = 0, 1


def _cfg(E, m, seed, layer, bh, mode):
    return _SelectCfg(int(E), int(m), int(seed) & 0xFFFFFFFFFFFFFFFF, int(layer), int(bh), int(mode))


def select_sample_group(S_row, k_offsets, i, E, m, seed=0, layer=0, bh=0, mode=IMPORTANCE, votes=None):
    """One query group: dict with exact groups, counts, sample positions and
    log-weights, the integer weights q_j (0 off the skipped set) and T.
    ``votes`` ([Ck] int32): rank the exact set by votes first (PQ voting)."""
    lib = _load()
    vrow = None if votes is None else _i32(votes)
    S_row = _f32(S_row)
    koff = _i32(k_offsets)
    Ck = S_row.shape[0]
    ex = np.empty(Ck, np.int32)
    cnt = np.empty(3, np.int32)
    pos = np.full(max(m, 1), -1, np.int32)
    bias = np.zeros(max(m, 1), np.float64)
    qw = np.zeros(Ck, np.uint32)
    tot = ctypes.c_uint64(0)
    cfg = _cfg(E, m, seed, layer, bh, mode)
    _check(lib.orc_select_sample_group(_ptr(S_row), _ptr(koff), Ck, i, ctypes.byref(cfg),
                                       None if vrow is None else _ptr(vrow), _ptr(ex),
                                       _ptr(cnt), _ptr(pos), _ptr(bias), _ptr(qw), ctypes.byref(tot)),
           "select_sample_group")
    ne, _, ns = (int(v) for v in cnt)
    return dict(exact_groups=ex[:ne].copy(), n_exact=ne, exact_keys=int(cnt[1]), n_sample=ns,
                sample_pos=pos[:ns].copy(), sample_bias=bias[:ns].copy(), q=qw, total=int(tot.value))


def select_sample(cq, ck, k_offsets, scale, E, m, seed=0, layer=0, bh=0, mode=IMPORTANCE, votes=None):
    """Whole head: (exact_groups [Cq,Ck], counts [Cq,3], sample_pos [Cq,m],
    sample_bias [Cq,m] fp64).  ``votes`` [Cq,Ck]: PQ-voting ranking."""
    lib = _load()
    vv = None if votes is None else _i32(votes)
    cq, ck, koff = _f32(cq), _f32(ck), _i32(k_offsets)
    Cq, d = cq.shape
    Ck = ck.shape[0]
    ex = np.empty((Cq, Ck), np.int32)
    cnt = np.empty((Cq, 3), np.int32)
    pos = np.empty((Cq, max(m, 1)), np.int32)
    bias = np.empty((Cq, max(m, 1)), np.float64)
    cfg = _cfg(E, m, seed, layer, bh, mode)
    _check(lib.orc_select_sample(_ptr(cq), Cq, _ptr(ck), Ck, d, float(np.float32(scale)), _ptr(koff),
                                 ctypes.byref(cfg), None if vv is None else _ptr(vv), _ptr(ex), _ptr(cnt),
                                 _ptr(pos), _ptr(bias)),
           "select_sample")
    return ex, cnt, pos[:, :m], bias[:, :m]


def select_top_p_group(S_row, k_offsets, top_p, floor_keys):
    """Top-p selection for one query group: dict with the kept groups (rank
    order), kept keys, the masses W_j and their total T (no draws)."""
    lib = _load()
    S_row, koff = _f32(S_row), _i32(k_offsets)
    Ck = S_row.shape[0]
    ex = np.empty(Ck, np.int32)
    cnt = np.empty(3, np.int32)
    W = np.zeros(Ck, np.uint64)
    tot = ctypes.c_uint64(0)
    _check(lib.orc_select_top_p_group(_ptr(S_row), _ptr(koff), Ck, float(np.float32(top_p)), int(floor_keys),
                                      _ptr(ex), _ptr(cnt), _ptr(W), ctypes.byref(tot)), "select_top_p_group")
    ne = int(cnt[0])
    return dict(exact_groups=ex[:ne].copy(), n_exact=ne, exact_keys=int(cnt[1]), n_sample=int(cnt[2]), W=W,
                total=int(tot.value))


def select_top_p(cq, ck, k_offsets, scale, top_p, floor_keys):
    """Whole head, top-p selection: (exact_groups [Cq,Ck], counts [Cq,3],
    sample_pos [Cq,0], sample_bias [Cq,0])."""
    lib = _load()
    cq, ck, koff = _f32(cq), _f32(ck), _i32(k_offsets)
    Cq, d = cq.shape
    Ck = ck.shape[0]
    ex = np.empty((Cq, Ck), np.int32)
    cnt = np.empty((Cq, 3), np.int32)
    _check(lib.orc_select_top_p(_ptr(cq), Cq, _ptr(ck), Ck, d, float(np.float32(scale)), _ptr(koff),
                                float(np.float32(top_p)), int(floor_keys), _ptr(ex), _ptr(cnt)), "select_top_p")
    return ex, cnt, np.zeros((Cq, 0), np.int32), np.zeros((Cq, 0), np.float64)


# ------------------------------------------------------------ PQ voting (readings
# in the C source: 8-dimension subspaces, 16 codewords, 5 Lloyd iterations on
# the group centroids, per-query budget prefix, votes then centroid score)
PQ_SUB, PQ_KC, PQ_ITERS = 8, 16, 5


def pq_codebook(P):
    """Codebook of the points P [C,d]: (cb [M,16,8] fp32, codes [C,M] uint8,
    codewords in use)."""
    lib = _load()
    P = _f32(P)
    C, d = P.shape
    M = d // PQ_SUB
    cb = np.zeros((M, PQ_KC, PQ_SUB), np.float32)
    codes = np.zeros((C, M), np.uint8)
    kc = lib.orc_pq_codebook(_ptr(P), C, d, _ptr(cb), _ptr(codes))
    if kc < 1:
        raise ValueError("pq_codebook: bad shape")
    return cb, codes, int(kc)


def pq_encode(X, cb, kc):
    """codes [n,M] of the rows X [n,d] against cb (kc codewords in use)."""
    lib = _load()
    X = _f32(X)
    n, d = X.shape
    codes = np.zeros((n, d // PQ_SUB), np.uint8)
    lib.orc_pq_encode(_ptr(X), n, d, _ptr(np.ascontiguousarray(cb, np.float32)), int(kc), _ptr(codes))
    return codes


def pq_votes(Q, cq, ck, q_perm, q_offsets, k_offsets, E):
    """Votes [Cq,Ck] of one head: codebooks from the centroids, key groups
    encoded by their centroids, each query voting for its budget prefix."""
    lib = _load()
    Q = _f32(Q)
    N, d = Q.shape
    cbq, _, kcq = pq_codebook(cq)
    cbk, kcodes, kck = pq_codebook(ck)
    qp, qo, ko = _i32(q_perm), _i32(q_offsets), _i32(k_offsets)
    Cq, Ck = qo.shape[0] - 1, ko.shape[0] - 1
    votes = np.zeros((Cq, Ck), np.int32)
    _check(lib.orc_pq_votes(_ptr(Q), N, d, _ptr(qp), _ptr(qo), Cq, _ptr(cbq), kcq, _ptr(cbk), kck,
                            _ptr(np.ascontiguousarray(kcodes)), _ptr(ko), Ck, int(E), _ptr(votes)), "pq_votes")
    return votes


# ---------------------------------------------------------------------- attention
def attention_rows(Q, K, V, scale, q_assign, k_perm, k_offsets, exact_groups, counts, sample_pos,
                   sample_bias, rows) -> np.ndarray:
    """fp64 output rows (original query indices ``rows``) of the sparse call."""
    lib = _load()
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    N, d = Q.shape
    qa, kp, ko = _i32(q_assign), _i32(k_perm), _i32(k_offsets)
    ex, cnt = _i32(exact_groups), _i32(counts)
    m = sample_pos.shape[1] if sample_pos.ndim == 2 else 0
    sp = _i32(sample_pos if m > 0 else np.full((ex.shape[0], 1), -1))
    sb = np.ascontiguousarray(np.asarray(sample_bias if m > 0 else np.zeros((ex.shape[0], 1)),
                                         dtype=np.float64))
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    out = np.empty((r.shape[0], d), np.float64)
    _check(lib.orc_attention_rows(_ptr(Q), _ptr(K), _ptr(V), N, d, float(np.float32(scale)), _ptr(qa),
                                  _ptr(kp), _ptr(ko), ex.shape[1], _ptr(ex), _ptr(cnt), _ptr(sp), _ptr(sb),
                                  sp.shape[1], _ptr(r), r.shape[0], _ptr(out)),
           "attention_rows")
    return out


# ---------------------------------------------------------------- whole head call
@dataclass
class HeadResult:
    cq: np.ndarray
    ck: np.ndarray
    q_assign: np.ndarray
    k_assign: np.ndarray
    q_perm: np.ndarray
    q_offsets: np.ndarray
    k_perm: np.ndarray
    k_offsets: np.ndarray
    exact_groups: np.ndarray
    counts: np.ndarray
    sample_pos: np.ndarray
    sample_bias: np.ndarray
    out: Optional[np.ndarray]


def forward_head(Q, K, V, *, Cq, Ck, iters, exact_frac, sample_frac, scale, seed=0, layer=0, bh=0,
                 mode=IMPORTANCE, rows=None, cq_init=None, ck_init=None, selection="centroid",
                 top_p=0.9, key_floor=0.1) -> HeadResult:
    """All stages for one head, in the pages' order.  ``rows`` limits the
    attention stage to those original query indices (all when None).
    ``selection``: "centroid" (Figure 3), "pq_vote" (the abstract's
    product-quantised per-query voting) or "top_p" (the SVG2-style comparator:
    the groups holding the share ``top_p`` of the estimated mass, at least
    ``key_floor`` of the keys, no sample; exact_frac and sample_frac unused)."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    N = Q.shape[0]
    cq, qa, _ = kmeans(Q, Cq, iters, cq_init)
    ck, ka, _ = kmeans(K, Ck, iters, ck_init)
    qp, qo = permutation(qa, Cq)
    kp, ko = permutation(ka, Ck)
    E, m = budget(exact_frac, N), budget(sample_frac, N)
    if selection == "top_p":
        ex, cnt, sp, sb = select_top_p(cq, ck, ko, scale, top_p, budget(key_floor, N))
    else:
        votes = pq_votes(Q, cq, ck, qp, qo, ko, E) if selection == "pq_vote" else None
        ex, cnt, sp, sb = select_sample(cq, ck, ko, scale, E, m, seed, layer, bh, mode, votes)
    if rows is None:
        rows = np.arange(N)
    out = attention_rows(Q, K, V, scale, qa, kp, ko, ex, cnt, sp, sb, rows) if len(rows) else None
    return HeadResult(cq, ck, qa, ka, qp, qo, kp, ko, ex, cnt, sp, sb, out)
