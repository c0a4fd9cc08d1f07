"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This module draws random numbers and nothing else: none of the method's
arithmetic lives here.  Both the CUDA path and the CPU oracle receive the
same host arrays it produces.

Recipe (the workloads are video-DiT attention layers; no model weights or
datasets are used):

* ``g = torch.Generator().manual_seed(seed)``;
* ``eq, ek, ev = randn(B, T, H, W, Hh, D)`` drawn in that order (fp32);
* if ``alpha > 0`` a shared rank-8 smooth spatiotemporal component is added
  to Q and K: random Fourier features of a Gaussian kernel with a length
  scale of sigma = 2 tiles (a tile is P x P tokens in space, one frame in
  time), ``Omega = randn(8, 3) / sigma``, ``phase = 2*pi*rand(8)``,
  ``phi(x) = sqrt(2/8) * cos(Omega x + phase)`` at ``x = (t, h/P, w/P)``,
  ``U = randn(Hh, 8, D)``, ``pos = phi . U`` (per-element variance ~ 1),
  ``Q = eq + alpha*pos``, ``K = ek + alpha*pos``, ``V = ev``;
* rounded to bf16 (round to nearest even), grid order, BSHD layout
  ``[B, S = T*H*W, Hh, D]``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hh: int
    D: int
    T: int
    H: int
    W: int
    alpha: float
    thr: float
    sta: tuple = (0, 0, 0)
    seed: int = 0
    P: int = 8
    # "nabla": the adaptive mask (OR the sliding-tile window when sta is set,
    # OR the radial window when radial > 0); "sta" / "radial": that static
    # window alone (thr unused)
    mask: str = "nabla"
    radial: int = 0  # radial window half-width at temporal distance 0 (0: off)

    @property
    def S(self) -> int:
        return self.T * self.H * self.W

    @property
    def Nb(self) -> int:
        return self.S // (self.P * self.P)

    @property
    def nbh(self) -> int:
        return self.H // self.P

    @property
    def nbw(self) -> int:
        return self.W // self.P

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The five layer configurations the method is measured on.
TINY = Workload("tiny: B1 Hh2 D64 grid 4x16x16, thr 0.9, no STA", 1, 2, 64, 4, 16, 16, 0.0, 0.9, seed=0)
WAN13B = Workload("Wan-1.3B-like: B1 Hh12 D128 grid 16x48x80, thr 0.7, no STA", 1, 12, 128, 16, 48, 80, 1.0, 0.7, seed=2)
HUNYUAN = Workload("HunyuanVideo-like: B1 Hh24 D128 grid 32x48x80, thr 0.9 OR STA 3x3x3", 1, 24, 128, 32, 48, 80, 1.0, 0.9,
                   sta=(3, 3, 3), seed=3)
# The same layer under the static window alone: the pure-STA configuration
# the method is compared with.
HUNYUAN_STA = Workload("HunyuanVideo-like, static STA 3x3x3 only: B1 Hh24 D128 grid 32x48x80", 1, 24, 128, 32, 48,
                       80, 1.0, 1.0, sta=(3, 3, 3), seed=3, mask="sta")
# The HunyuanVideo-like layer with the radial decay window (half-width 2
# patches at temporal distance 0, halving per doubling of the distance) as
# the OR-term, and the long-video layer under that window alone.
HUNYUAN_RADIAL = Workload("HunyuanVideo-like: B1 Hh24 D128 grid 32x48x80, thr 0.9 OR radial window r0=2", 1, 24, 128,
                          32, 48, 80, 1.0, 0.9, seed=3, radial=2)
LONG_RADIAL = Workload("long video, static radial window r0=2 only: B1 Hh24 D128 grid 64x48x80", 1, 24, 128, 64, 48,
                       80, 1.0, 1.0, seed=5, mask="radial", radial=2)
LONG = Workload("long video: B1 Hh24 D128 grid 64x48x80, thr 0.9 OR STA 3x3x3", 1, 24, 128, 64, 48, 80, 1.0, 0.9,
                sta=(3, 3, 3), seed=5)
# The long-video layer with 4 of its 24 heads: the same 3,840 blocks per row
# and per-head structure at a size a full hardware-counter capture can hold
# (~2 GB on the device), for profiling the kernels of the long layer.
LONG_4H = Workload("long video, 4 heads: B1 Hh4 D128 grid 64x48x80, thr 0.9 OR STA 3x3x3", 1, 4, 128, 64, 48, 80,
                   1.0, 0.9, sta=(3, 3, 3), seed=5)


def sweep_points():
    """Sparsity sweep on the Wan-1.3B-like shape: 3 amplitudes x 5 thresholds."""
    pts = []
    for alpha in (0.0, 0.5, 1.0):
        for thr in (0.5, 0.7, 0.9, 0.95, 1.0):
            pts.append(Workload(f"sweep: Wan-1.3B-like shape, alpha {alpha}, thr {thr}", 1, 12, 128, 16, 48, 80,
                                alpha, thr, seed=4))
    return pts


def make_qkv(w: Workload):
    """Return (q, k, v) bf16 CPU tensors [B, S, Hh, D] in grid order."""
    g = torch.Generator().manual_seed(w.seed)
    shape = (w.B, w.T, w.H, w.W, w.Hh, w.D)
    q = torch.randn(shape, generator=g)
    k = torch.randn(shape, generator=g)
    v = torch.randn(shape, generator=g)
    if w.alpha > 0:
        sigma = 2.0
        omega = torch.randn(8, 3, generator=g) / sigma
        phase = 2.0 * math.pi * torch.rand(8, generator=g)
        U = torch.randn(w.Hh, 8, w.D, generator=g)
        t = torch.arange(w.T, dtype=torch.float32).view(w.T, 1, 1).expand(w.T, w.H, w.W)
        h = (torch.arange(w.H, dtype=torch.float32) / w.P).view(1, w.H, 1).expand(w.T, w.H, w.W)
        x = (torch.arange(w.W, dtype=torch.float32) / w.P).view(1, 1, w.W).expand(w.T, w.H, w.W)
        coords = torch.stack([t, h, x], dim=-1)  # [T, H, W, 3]
        phi = math.sqrt(2.0 / 8.0) * torch.cos(coords @ omega.T + phase)  # [T, H, W, 8]
        pos = torch.einsum("thwr,nrd->thwnd", phi, U)  # [T, H, W, Hh, D]
        q.add_(pos.unsqueeze(0), alpha=w.alpha)
        k.add_(pos.unsqueeze(0), alpha=w.alpha)
        del pos
    out = []
    for x_ in (q, k, v):
        out.append(x_.to(torch.bfloat16).reshape(w.B, w.S, w.Hh, w.D).contiguous())
    return tuple(out)


def sample_query_blocks(Nb: int, n: int = 64, seed: int = 1234):
    """Seeded subset of query blocks (without replacement), ascending."""
    g = torch.Generator().manual_seed(seed)
    n = min(n, Nb)
    idx = torch.randperm(Nb, generator=g)[:n]
    return torch.sort(idx).values.to(torch.int32).numpy()


def randn_bf16(shape, seed: int):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


# ------------------------------------------------------------- AB-Attention
@dataclass(frozen=True)
class ABWorkload:
    """A layer under the AB-Attention scheme: the Q, K, V recipe of
    `base` (grid order, not permuted), 128-token query blocks, 8 clusters,
    4-token key blocks, `kmeans_iters` Lloyd iterations, and an expected
    sample of `budget_frac` of the key blocks per query block."""
    name: str
    base: Workload
    budget_frac: float
    kmeans_iters: int = 4
    seed_u: int = 77

    @property
    def nqb(self) -> int:
        return self.base.S // 128

    @property
    def nkb(self) -> int:
        return self.base.S // 4

    @property
    def budget(self) -> float:
        return float(math.ceil(self.budget_frac * self.nkb))


def ab_uniforms(w: ABWorkload) -> torch.Tensor:
    """The sampling's uniform random numbers in [0, 1), one per (batch, head,
    query block, key block): fp32 [B, Hh, NQB, NKB], seeded."""
    g = torch.Generator().manual_seed(w.seed_u)
    return torch.rand((w.base.B, w.base.Hh, w.nqb, w.nkb), generator=g)


# The AB-Attention workloads: the Wan-1.3B-like layer with 10% of the key
# blocks sampled in expectation (the page reports 89-92% of the attention
# skipped), and a small one the oracle finishes in seconds.
AB_TINY = ABWorkload("AB tiny: B1 Hh2 D64 grid 4x16x32 (2048 tokens), 10% sampled",
                     Workload("ab-tiny", 1, 2, 64, 4, 16, 32, 1.0, 1.0, seed=61), 0.10)
AB_WAN13B = ABWorkload("AB Wan-1.3B-like: B1 Hh12 D128 grid 16x48x80, 10% sampled",
                       Workload("ab-wan", 1, 12, 128, 16, 48, 80, 1.0, 1.0, seed=2), 0.10)
