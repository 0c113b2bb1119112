"""B200-native InstaGen group-shared importance-sampled permuted block-sparse
attention (one DiT self-attention call, per head).

Thin Python binding of ``libinstagen.so`` (C ABI in ``include/instagen.h``):
argument marshalling only.  PyTorch supplies device memory and the current
CUDA stream; every step of the computation runs in the library's sm_100a
kernels.  There is no fallback: if the library is missing or a call fails the
binding raises.

Entry points (same names as the C ABI, without the ``instagen_`` prefix):
``cluster``, ``permutation``, ``gather``, ``select_sample``, ``attention``,
``forward``, ``forward_host`` plus ``make_params``, ``exact_budget``, ``sample_budget``,
``workspace_size``, ``forward_layout`` and ``device_status``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libinstagen.so")

IMPORTANCE, UNIFORM = 0, 1
CENTROID, PQ_VOTE, TOP_P = 0, 1, 2  # instagen_selection


class InstaGenError(RuntimeError):
    pass


class Params(ctypes.Structure):
    """Mirror of ``instagen_params``."""
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
                ("Cq", ctypes.c_int32), ("Ck", ctypes.c_int32), ("kmeans_iters", ctypes.c_int32),
                ("exact_frac", ctypes.c_float), ("sample_frac", ctypes.c_float),
                ("softmax_scale", ctypes.c_float), ("seed", ctypes.c_uint64), ("layer", ctypes.c_uint32),
                ("sampling", ctypes.c_int32), ("selection", ctypes.c_int32), ("top_p", ctypes.c_float),
                ("key_floor", ctypes.c_float)]


class ForwardLayout(ctypes.Structure):
    """Mirror of ``instagen_forward_layout`` (byte offsets into the workspace)."""
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "cq", "ck", "q_assign", "k_assign", "q_perm", "k_perm", "q_offsets", "k_offsets", "kp", "vp",
        "exact_groups", "counts", "sample_pos", "sample_bias", "votes", "pq_ws", "cluster_ws", "total")]


_lib = None
_SYMBOLS = ("instagen_exact_budget", "instagen_sample_budget", "instagen_workspace_size",
            "instagen_cluster_workspace_size", "instagen_error_string", "instagen_device_status",
            "instagen_cluster", "instagen_permutation", "instagen_gather", "instagen_select_sample",
            "instagen_attention", "instagen_forward", "instagen_forward_layout_get",
            "instagen_cluster_static", "instagen_forward_host_workspace_size", "instagen_forward_host",
            "instagen_forward_init", "instagen_pq_votes_workspace_size", "instagen_pq_votes",
            "instagen_select_sample_votes")


def lib():
    """The loaded ``libinstagen.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise InstaGenError(f"{LIB_PATH} is missing: build it with block_sparse_attention_head_b200.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, PP, vp = ctypes.POINTER(Params), ctypes.c_void_p, ctypes.c_void_p
    i32, i64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "instagen_exact_budget": (i64, [P]),
        "instagen_sample_budget": (i64, [P]),
        "instagen_workspace_size": (sz, [P]),
        "instagen_cluster_workspace_size": (sz, [P, i32]),
        "instagen_error_string": (ctypes.c_char_p, [ctypes.c_int]),
        "instagen_device_status": (ctypes.c_int, [vp]),
        "instagen_cluster": (ctypes.c_int, [PP, i32, i32, PP, P, PP, PP, PP, PP, PP, sz, vp]),
        "instagen_permutation": (ctypes.c_int, [PP, i32, P, PP, PP, vp]),
        "instagen_gather": (ctypes.c_int, [PP, PP, P, PP, i32, vp]),
        "instagen_select_sample": (ctypes.c_int, [PP, PP, PP, P, PP, PP, PP, PP, vp]),
        "instagen_attention": (ctypes.c_int, [PP, PP, PP, PP, PP, PP, PP, PP, PP, PP, P, PP, vp]),
        "instagen_forward": (ctypes.c_int, [PP, PP, PP, PP, P, PP, sz, vp]),
        "instagen_forward_layout_get": (ctypes.c_int, [P, ctypes.POINTER(ForwardLayout)]),
        "instagen_cluster_static": (ctypes.c_int, [PP, i32, i32, PP, P, PP, PP, PP, PP, vp]),
        "instagen_forward_host_workspace_size": (sz, [P, i32]),
        "instagen_forward_host": (ctypes.c_int, [PP, PP, PP, PP, P, i32, PP, sz, vp]),
        "instagen_forward_init": (ctypes.c_int, [PP, PP, PP, PP, P, PP, PP, PP, sz, vp]),
        "instagen_pq_votes_workspace_size": (sz, [P]),
        "instagen_pq_votes": (ctypes.c_int, [PP, PP, PP, PP, PP, PP, P, PP, PP, sz, vp]),
        "instagen_select_sample_votes": (ctypes.c_int, [PP, PP, PP, PP, P, PP, PP, PP, PP, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != 0:
        msg = lib().instagen_error_string(rc).decode()
        raise InstaGenError(f"{what}: {msg} (status {rc})")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise InstaGenError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def make_params(B: int, H: int, N: int, d: int, Cq: int, Ck: int, *, iters: int = 10, exact_frac: float = 0.16,
                sample_frac: float = 0.16, softmax_scale: Optional[float] = None, seed: int = 0, layer: int = 0,
                sampling: int | str = IMPORTANCE, selection: int | str = CENTROID, top_p: float = 0.9,
                key_floor: float = 0.1) -> Params:
    """``selection``: "centroid" (default), "pq_vote", or "top_p" (the comparator:
    keep the key groups holding the share ``top_p`` of the estimated mass and at
    least ``key_floor`` of the keys; no sample, so sample_frac must be 0)."""
    if isinstance(sampling, str):
        sampling = {"importance": IMPORTANCE, "uniform": UNIFORM}[sampling]
    if isinstance(selection, str):
        selection = {"centroid": CENTROID, "pq_vote": PQ_VOTE, "top_p": TOP_P}[selection]
    scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    return Params(B, H, N, d, Cq, Ck, iters, exact_frac, sample_frac, scale, seed & (2 ** 64 - 1), layer, sampling,
                  selection, top_p, key_floor)


def exact_budget(p: Params) -> int:
    return int(lib().instagen_exact_budget(ctypes.byref(p)))


def sample_budget(p: Params) -> int:
    return int(lib().instagen_sample_budget(ctypes.byref(p)))


def workspace_size(p: Params) -> int:
    n = int(lib().instagen_workspace_size(ctypes.byref(p)))
    if n == 0:
        raise InstaGenError("invalid parameters for instagen_workspace_size")
    return n


def cluster_workspace_size(p: Params, C: int) -> int:
    return int(lib().instagen_cluster_workspace_size(ctypes.byref(p), C))


def forward_layout(p: Params) -> ForwardLayout:
    L = ForwardLayout()
    _check(lib().instagen_forward_layout_get(ctypes.byref(p), ctypes.byref(L)), "instagen_forward_layout_get")
    return L


def device_status():
    """Synchronise the current stream; raise if a kernel recorded an
    out-of-range index or a wait timeout."""
    _check(lib().instagen_device_status(_stream()), "device check")


def _bhnd(p: Params):
    return (p.B, p.H, p.N, p.d)


def cluster(X: torch.Tensor, C: int, iters: int, p: Params, init: Optional[torch.Tensor] = None):
    """k-means of X [B,H,N,d] bf16 into C clusters + stable permutation.
    Returns (centroids fp32 [B,H,C,d], assign, perm [B,H,N] int32, offsets [B,H,C+1])."""
    _need(X, "X", torch.bfloat16, _bhnd(p))
    dev = X.device
    if init is not None:
        _need(init, "init", torch.float32, (p.B, p.H, C, p.d))
    cent = torch.empty((p.B, p.H, C, p.d), dtype=torch.float32, device=dev)
    assign = torch.empty((p.B, p.H, p.N), dtype=torch.int32, device=dev)
    perm = torch.empty_like(assign)
    offs = torch.empty((p.B, p.H, C + 1), dtype=torch.int32, device=dev)
    nws = cluster_workspace_size(p, C)
    if nws == 0:
        raise InstaGenError("invalid parameters for instagen_cluster")
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)
    _check(lib().instagen_cluster(_ptr(X), C, iters, _ptr(init), ctypes.byref(p), _ptr(cent), _ptr(assign),
                                  _ptr(perm), _ptr(offs), _ptr(ws), nws, _stream()), "instagen_cluster")
    return cent, assign, perm, offs


def cluster_static(X: torch.Tensor, C: int, iters: int, p: Params, init: Optional[torch.Tensor] = None):
    """``cluster`` without a workspace: the scratch lives in a fixed device
    array inside the library, for callers that may not allocate device
    memory.  Only the outputs (allocated here by torch for convenience) are
    passed; see ``instagen_cluster_static`` in include/instagen.h."""
    _need(X, "X", torch.bfloat16, _bhnd(p))
    dev = X.device
    if init is not None:
        _need(init, "init", torch.float32, (p.B, p.H, C, p.d))
    cent = torch.empty((p.B, p.H, C, p.d), dtype=torch.float32, device=dev)
    assign = torch.empty((p.B, p.H, p.N), dtype=torch.int32, device=dev)
    perm = torch.empty_like(assign)
    offs = torch.empty((p.B, p.H, C + 1), dtype=torch.int32, device=dev)
    _check(lib().instagen_cluster_static(_ptr(X), C, iters, _ptr(init), ctypes.byref(p), _ptr(cent), _ptr(assign),
                                         _ptr(perm), _ptr(offs), _stream()), "instagen_cluster_static")
    return cent, assign, perm, offs


def permutation(assign: torch.Tensor, C: int, p: Params):
    _need(assign, "assign", torch.int32, (p.B, p.H, p.N))
    perm = torch.empty_like(assign)
    offs = torch.empty((p.B, p.H, C + 1), dtype=torch.int32, device=assign.device)
    _check(lib().instagen_permutation(_ptr(assign), C, ctypes.byref(p), _ptr(perm), _ptr(offs), _stream()),
           "instagen_permutation")
    return perm, offs


def gather(X: torch.Tensor, perm: torch.Tensor, p: Params, to_f16: bool = False) -> torch.Tensor:
    """Rows of X [B,H,N,d] bf16 in permuted order; fp16 output when to_f16
    (the layout instagen_attention expects for V)."""
    _need(X, "X", torch.bfloat16, _bhnd(p))
    _need(perm, "perm", torch.int32, (p.B, p.H, p.N))
    Xp = torch.empty(X.shape, dtype=torch.float16 if to_f16 else torch.bfloat16, device=X.device)
    _check(lib().instagen_gather(_ptr(X), _ptr(perm), ctypes.byref(p), _ptr(Xp), 1 if to_f16 else 0, _stream()),
           "instagen_gather")
    return Xp


def pq_votes(Q: torch.Tensor, cq: torch.Tensor, ck: torch.Tensor, q_perm: torch.Tensor, q_offsets: torch.Tensor,
             k_offsets: torch.Tensor, p: Params) -> torch.Tensor:
    """Product-quantised per-query votes [B,H,Cq,Ck] int32 (instagen_pq_votes)."""
    _need(Q, "Q", torch.bfloat16, (p.B, p.H, p.N, p.d))
    _need(cq, "cq", torch.float32, (p.B, p.H, p.Cq, p.d))
    _need(ck, "ck", torch.float32, (p.B, p.H, p.Ck, p.d))
    _need(q_perm, "q_perm", torch.int32, (p.B, p.H, p.N))
    _need(q_offsets, "q_offsets", torch.int32, (p.B, p.H, p.Cq + 1))
    _need(k_offsets, "k_offsets", torch.int32, (p.B, p.H, p.Ck + 1))
    votes = torch.empty((p.B, p.H, p.Cq, p.Ck), dtype=torch.int32, device=Q.device)
    nws = int(lib().instagen_pq_votes_workspace_size(ctypes.byref(p)))
    ws = torch.empty(max(nws, 256), dtype=torch.uint8, device=Q.device)
    _check(lib().instagen_pq_votes(_ptr(Q), _ptr(cq), _ptr(ck), _ptr(q_perm), _ptr(q_offsets), _ptr(k_offsets),
                                   ctypes.byref(p), _ptr(votes), _ptr(ws), ws.numel(), _stream()),
           "instagen_pq_votes")
    return votes


def select_sample(cq: torch.Tensor, ck: torch.Tensor, k_offsets: torch.Tensor, p: Params,
                  votes: Optional[torch.Tensor] = None):
    """Returns (exact_groups [B,H,Cq,Ck], counts [B,H,Cq,3], sample_pos [B,H,Cq,m] int32,
    sample_bias [B,H,Cq,m] fp32).  With ``votes`` [B,H,Cq,Ck] int32 the exact
    set is ranked by votes first (instagen_select_sample_votes)."""
    _need(cq, "cq", torch.float32, (p.B, p.H, p.Cq, p.d))
    _need(ck, "ck", torch.float32, (p.B, p.H, p.Ck, p.d))
    _need(k_offsets, "k_offsets", torch.int32, (p.B, p.H, p.Ck + 1))
    m = sample_budget(p)
    dev = cq.device
    eg = torch.empty((p.B, p.H, p.Cq, p.Ck), dtype=torch.int32, device=dev)
    cnt = torch.empty((p.B, p.H, p.Cq, 3), dtype=torch.int32, device=dev)
    sp = torch.empty((p.B, p.H, p.Cq, m), dtype=torch.int32, device=dev)
    sb = torch.empty((p.B, p.H, p.Cq, m), dtype=torch.float32, device=dev)
    if votes is not None:
        _need(votes, "votes", torch.int32, (p.B, p.H, p.Cq, p.Ck))
        _check(lib().instagen_select_sample_votes(_ptr(cq), _ptr(ck), _ptr(k_offsets), _ptr(votes), ctypes.byref(p),
                                                  _ptr(eg), _ptr(cnt), _ptr(sp) if m else None,
                                                  _ptr(sb) if m else None, _stream()),
               "instagen_select_sample_votes")
        return eg, cnt, sp, sb
    _check(lib().instagen_select_sample(_ptr(cq), _ptr(ck), _ptr(k_offsets), ctypes.byref(p), _ptr(eg), _ptr(cnt),
                                        _ptr(sp) if m else None, _ptr(sb) if m else None, _stream()),
           "instagen_select_sample")
    return eg, cnt, sp, sb


def attention(Q, Kp, Vp, q_perm, q_offsets, k_offsets, exact_groups, counts, sample_pos, sample_bias,
              p: Params, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Q bf16 original order; Kp bf16 and Vp fp16 in key-cluster order (``gather``);
    returns O [B,H,N,d] bf16 (original order)."""
    _need(Q, "Q", torch.bfloat16, _bhnd(p))
    _need(Kp, "Kp", torch.bfloat16, _bhnd(p))
    _need(Vp, "Vp", torch.float16, _bhnd(p))
    m = sample_budget(p)
    _need(q_perm, "q_perm", torch.int32, (p.B, p.H, p.N))
    _need(q_offsets, "q_offsets", torch.int32, (p.B, p.H, p.Cq + 1))
    _need(k_offsets, "k_offsets", torch.int32, (p.B, p.H, p.Ck + 1))
    _need(exact_groups, "exact_groups", torch.int32, (p.B, p.H, p.Cq, p.Ck))
    _need(counts, "counts", torch.int32, (p.B, p.H, p.Cq, 3))
    _need(sample_pos, "sample_pos", torch.int32, (p.B, p.H, p.Cq, m))
    _need(sample_bias, "sample_bias", torch.float32, (p.B, p.H, p.Cq, m))
    O = torch.empty_like(Q) if out is None else out
    _need(O, "O", torch.bfloat16, _bhnd(p))
    _check(lib().instagen_attention(_ptr(Q), _ptr(Kp), _ptr(Vp), _ptr(q_perm), _ptr(q_offsets), _ptr(k_offsets),
                                    _ptr(exact_groups), _ptr(counts), _ptr(sample_pos) if m else None,
                                    _ptr(sample_bias) if m else None, ctypes.byref(p), _ptr(O), _stream()),
           "instagen_attention")
    return O


def forward(Q, K, V, p: Params, workspace: Optional[torch.Tensor] = None,
            out: Optional[torch.Tensor] = None, cq_init: Optional[torch.Tensor] = None,
            ck_init: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The whole InstaGen attention call; O [B,H,N,d] bf16 in original order.
    cq_init / ck_init (fp32 [B,H,C,d] on the device): warm-start centroids
    (instagen_forward_init), e.g. the previous call's ``forward_intermediates``."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _need(t, n, torch.bfloat16, _bhnd(p))
    nws = workspace_size(p)
    ws = torch.empty(nws, dtype=torch.uint8, device=Q.device) if workspace is None else workspace
    if ws.numel() * ws.element_size() < nws:
        raise InstaGenError(f"workspace too small: {ws.numel() * ws.element_size()} < {nws}")
    O = torch.empty_like(Q) if out is None else out
    _need(O, "O", torch.bfloat16, _bhnd(p))
    if cq_init is None and ck_init is None:
        _check(lib().instagen_forward(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), ctypes.byref(p), _ptr(ws),
                                      ws.numel() * ws.element_size(), _stream()), "instagen_forward")
        return O
    if cq_init is not None:
        _need(cq_init, "cq_init", torch.float32, (p.B, p.H, p.Cq, p.d))
    if ck_init is not None:
        _need(ck_init, "ck_init", torch.float32, (p.B, p.H, p.Ck, p.d))
    _check(lib().instagen_forward_init(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), ctypes.byref(p), _ptr(cq_init),
                                       _ptr(ck_init), _ptr(ws), ws.numel() * ws.element_size(), _stream()),
           "instagen_forward_init")
    return O


def forward_host_workspace_size(p: Params, heads_per_chunk: int = 0) -> int:
    return int(lib().instagen_forward_host_workspace_size(ctypes.byref(p), heads_per_chunk))


def forward_host(Q, K, V, p: Params, out: Optional[torch.Tensor] = None, heads_per_chunk: int = 0,
                 workspace: Optional[torch.Tensor] = None, device=None) -> torch.Tensor:
    """The whole call on HOST tensors (CPU, contiguous bf16 [B,H,N,d];
    page-locked for overlapped copies): head chunks are copied in, computed
    and copied out in a pipeline on the current CUDA stream.  Returns the host
    output O (synchronise the stream before reading it)."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        if not isinstance(t, torch.Tensor) or t.is_cuda:
            raise InstaGenError(f"{n} must be a host (CPU) tensor")
        if t.dtype != torch.bfloat16 or not t.is_contiguous() or tuple(t.shape) != _bhnd(p):
            raise ValueError(f"{n} must be contiguous bf16 {_bhnd(p)}")
    O = torch.empty(Q.shape, dtype=Q.dtype, pin_memory=Q.is_pinned()) if out is None else out
    if O.is_cuda or O.dtype != torch.bfloat16 or not O.is_contiguous() or tuple(O.shape) != _bhnd(p):
        raise ValueError(f"out must be a contiguous host bf16 tensor {_bhnd(p)}")
    nws = forward_host_workspace_size(p, heads_per_chunk)
    if nws == 0:
        raise InstaGenError("invalid parameters for instagen_forward_host")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    ws = torch.empty(nws, dtype=torch.uint8, device=dev) if workspace is None else workspace
    if ws.numel() * ws.element_size() < nws:
        raise InstaGenError(f"workspace too small: {ws.numel() * ws.element_size()} < {nws}")
    _check(lib().instagen_forward_host(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), ctypes.byref(p), heads_per_chunk,
                                       _ptr(ws), ws.numel() * ws.element_size(), _stream()), "instagen_forward_host")
    return O


def forward_intermediates(workspace: torch.Tensor, p: Params) -> dict:
    """Views of instagen_forward's intermediates inside its workspace."""
    L = forward_layout(p)
    m = sample_budget(p)
    B, H, N, d, Cq, Ck = p.B, p.H, p.N, p.d, p.Cq, p.Ck

    def view(off, n_elem, dtype, shape):
        nbytes = n_elem * torch.empty((), dtype=dtype).element_size()
        return workspace[off:off + nbytes].view(dtype).reshape(shape)

    return dict(
        cq=view(L.cq, B * H * Cq * d, torch.float32, (B, H, Cq, d)),
        ck=view(L.ck, B * H * Ck * d, torch.float32, (B, H, Ck, d)),
        q_assign=view(L.q_assign, B * H * N, torch.int32, (B, H, N)),
        k_assign=view(L.k_assign, B * H * N, torch.int32, (B, H, N)),
        q_perm=view(L.q_perm, B * H * N, torch.int32, (B, H, N)),
        k_perm=view(L.k_perm, B * H * N, torch.int32, (B, H, N)),
        q_offsets=view(L.q_offsets, B * H * (Cq + 1), torch.int32, (B, H, Cq + 1)),
        k_offsets=view(L.k_offsets, B * H * (Ck + 1), torch.int32, (B, H, Ck + 1)),
        kp=view(L.kp, B * H * N * d, torch.bfloat16, (B, H, N, d)),
        vp=view(L.vp, B * H * N * d, torch.float16, (B, H, N, d)),
        exact_groups=view(L.exact_groups, B * H * Cq * Ck, torch.int32, (B, H, Cq, Ck)),
        counts=view(L.counts, B * H * Cq * 3, torch.int32, (B, H, Cq, 3)),
        sample_pos=view(L.sample_pos, B * H * Cq * m, torch.int32, (B, H, Cq, m)),
        sample_bias=view(L.sample_bias, B * H * Cq * m, torch.float32, (B, H, Cq, m)),
        **({"votes": view(L.votes, B * H * Cq * Ck, torch.int32, (B, H, Cq, Ck))} if p.selection == PQ_VOTE else {}),
    )
