"""Seeded synthetic inputs for the InstaGen attention call.

This module only draws random numbers: it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle may consume what it makes.

The pages measure on Wan2.1-T2V-1.3B / 14B activations (thelatestinai.com
paper page, Figures 1-6 and Table 1: 720p, 81 frames -> 21 latent frames of
45x80 tokens; the 1.3B model at 480p gives 21x30x52).  Those activations need
model weights that are not available, so clustered Gaussian mixtures with the
same shapes stand in for them:

  * per head, ``n_centres`` centres c_r ~ N(0, I_d) (scale 1);
  * query and key labels drawn independently from the same centre set, either
    uniformly or with Zipf(s) weights p_r ~ r^-s (uneven cluster sizes);
  * Q_i = c_label + sigma * eps, K_j likewise, V ~ N(0, 1);
  * tokens come out in random order (labels are i.i.d. per token);
  * fp32 draws rounded to bf16 (round to nearest even).

Every tensor is [B, H, N, d] bf16, contiguous.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    """One attention-call configuration (shape, mixture and budgets)."""
    name: str
    B: int
    H: int
    N: int
    d: int
    n_centres: int
    labels: str            # "uniform" or "zipf"
    sigma: Tuple[float, float]  # per-head noise sigma, linearly spaced from [0] to [1] over heads
    Cq: int
    Ck: int
    iters: int
    exact_frac: float
    sample_frac: float
    seed: int = 0
    zipf_s: float = 1.1
    layers: int = 1
    sweep: Tuple[Tuple[float, float], ...] = field(default_factory=tuple)

    @property
    def softmax_scale(self) -> float:
        return 1.0 / (self.d ** 0.5)


# Wan2.1 latent token counts: 21 frames x (30x52) at 480p, x (45x80) at 720p.
TINY = Workload("tiny_n4096_d64", 1, 1, 4096, 64, 64, "uniform", (0.3, 0.3), 16, 64, 10, 0.08, 0.08, seed=0)
WAN13B_480P = Workload("wan2.1-1.3b_480p", 1, 12, 32760, 128, 256, "zipf", (0.3, 0.3), 100, 500, 10,
                       0.16, 0.16, seed=1)
WAN13B_720P = Workload("wan2.1-1.3b_720p", 1, 12, 75600, 128, 256, "zipf", (0.3, 0.3), 100, 500, 10,
                       0.16, 0.16, seed=2,
                       sweep=((0.04, 0.04), (0.08, 0.08), (0.16, 0.16), (0.32, 0.32)))
WAN14B_720P = Workload("wan2.1-14b_720p", 1, 40, 75600, 128, 512, "zipf", (0.2, 0.6), 100, 500, 10,
                       0.16, 0.16, seed=3)
WAN14B_STACK = Workload("wan2.1-14b_720p_stack", 1, 40, 75600, 128, 512, "zipf", (0.2, 0.6), 100, 500, 10,
                        0.08, 0.16, seed=4, layers=40,
                        sweep=((0.08, 0.02), (0.08, 0.04), (0.08, 0.08), (0.08, 0.16), (0.08, 0.32)))

WORKLOADS = {w.name: w for w in (TINY, WAN13B_480P, WAN13B_720P, WAN14B_720P, WAN14B_STACK)}


def head_sigmas(w: Workload) -> List[float]:
    lo, hi = w.sigma
    if w.H == 1:
        return [lo]
    return [lo + (hi - lo) * h / (w.H - 1) for h in range(w.H)]


def _label_probs(w: Workload, device) -> torch.Tensor:
    if w.labels == "uniform":
        return torch.full((w.n_centres,), 1.0 / w.n_centres, dtype=torch.float64, device=device)
    r = torch.arange(1, w.n_centres + 1, dtype=torch.float64, device=device)
    p = r.pow(-w.zipf_s)
    return p / p.sum()


def make_inputs(w: Workload, *, layer: int = 0, device: str | torch.device = "cpu",
                N: Optional[int] = None, heads: Optional[Sequence[int]] = None):
    """(Q, K, V) bf16 [B, H, N, d] for layer ``layer`` of workload ``w``.

    Each (layer, b, h) head has its own generator seeded from (w.seed, layer,
    b*H+h), so a subset of heads (``heads``) reproduces exactly the same
    tensors as the full call.  ``N`` overrides the token count (same recipe).
    """
    n_tok = w.N if N is None else N
    head_ids = list(range(w.B * w.H)) if heads is None else list(heads)
    sig = head_sigmas(w)
    dev = torch.device(device)
    probs = _label_probs(w, dev)
    out_q, out_k, out_v = [], [], []
    for bh in head_ids:
        g = torch.Generator(device=dev)
        g.manual_seed(int(w.seed) * 1_000_003 + int(layer) * 10_007 + int(bh) + 17)
        centres = torch.randn(w.n_centres, w.d, generator=g, device=dev, dtype=torch.float32)
        ql = torch.multinomial(probs, n_tok, replacement=True, generator=g)
        kl = torch.multinomial(probs, n_tok, replacement=True, generator=g)
        s = sig[bh % w.H]
        q = centres[ql] + s * torch.randn(n_tok, w.d, generator=g, device=dev, dtype=torch.float32)
        k = centres[kl] + s * torch.randn(n_tok, w.d, generator=g, device=dev, dtype=torch.float32)
        v = torch.randn(n_tok, w.d, generator=g, device=dev, dtype=torch.float32)
        out_q.append(q.to(torch.bfloat16))
        out_k.append(k.to(torch.bfloat16))
        out_v.append(v.to(torch.bfloat16))
    shape = (1, len(head_ids), n_tok, w.d) if heads is not None else (w.B, w.H, n_tok, w.d)
    Q = torch.stack(out_q).reshape(shape).contiguous()
    K = torch.stack(out_k).reshape(shape).contiguous()
    V = torch.stack(out_v).reshape(shape).contiguous()
    return Q, K, V


def make_labelled_head(w: Workload, *, bh: int = 0, layer: int = 0, N: Optional[int] = None):
    """(Q, K, V, q_labels, k_labels) for one head, with the planted labels
    (used to check that clustering recovers the mixture)."""
    n_tok = w.N if N is None else N
    probs = _label_probs(w, torch.device("cpu"))
    g = torch.Generator()
    g.manual_seed(int(w.seed) * 1_000_003 + int(layer) * 10_007 + int(bh) + 17)
    centres = torch.randn(w.n_centres, w.d, generator=g, dtype=torch.float32)
    ql = torch.multinomial(probs, n_tok, replacement=True, generator=g)
    kl = torch.multinomial(probs, n_tok, replacement=True, generator=g)
    s = head_sigmas(w)[bh % w.H]
    q = centres[ql] + s * torch.randn(n_tok, w.d, generator=g, dtype=torch.float32)
    k = centres[kl] + s * torch.randn(n_tok, w.d, generator=g, dtype=torch.float32)
    v = torch.randn(n_tok, w.d, generator=g, dtype=torch.float32)
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16), ql, kl)


def random_small(seed: int, N: int, d: int, n_centres: int = 8, sigma: float = 0.5,
                 H: int = 1, device: str = "cpu"):
    """Small mixed-scale inputs for edge-case tests: [1, H, N, d] bf16."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    qs, ks, vs = [], [], []
    for _ in range(H):
        centres = torch.randn(n_centres, d, generator=g, device=device)
        ql = torch.randint(0, n_centres, (N,), generator=g, device=device)
        kl = torch.randint(0, n_centres, (N,), generator=g, device=device)
        qs.append((centres[ql] + sigma * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16))
        ks.append((centres[kl] + sigma * torch.randn(N, d, generator=g, device=device)).to(torch.bfloat16))
        vs.append(torch.randn(N, d, generator=g, device=device).to(torch.bfloat16))
    return (torch.stack(qs)[None].contiguous(), torch.stack(ks)[None].contiguous(),
            torch.stack(vs)[None].contiguous())
