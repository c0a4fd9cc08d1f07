"""Helpers shared by the GPU parity tests: run the CUDA path through the C
ABI binding and compare it with the CPU oracle on the same seeded inputs.

Comparison rules (fixed by the method's acceptance criteria):
* flattening and the block lists are bit-exact, except blocks whose oracle
  cumulative mass lies within 1e-5 of 1 - thr ("band" blocks), which are
  counted and reported;
* attention outputs (bf16 out, fp32 accumulation) are within max-abs 2e-2
  and mean-abs 2e-3 of the fp64 oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
LSE_ABS = 2e-3


def flat_order(T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    """g[f] = grid row (t*H + h)*W + w of flattened row f: 8 x 8 patches of
    each frame, patch-row-major, pixels row-major inside a patch."""
    t, bh, bw, ph, pw = np.meshgrid(np.arange(T), np.arange(H // P), np.arange(W // P), np.arange(P), np.arange(P),
                                    indexing="ij")
    return ((t * H + bh * P + ph) * W + bw * P + pw).reshape(-1)


def grid_to_flat_rows(x: torch.Tensor, T: int, H: int, W: int, dim: int) -> torch.Tensor:
    """Rows of x along `dim` taken from grid order to flattened order."""
    idx = torch.as_tensor(flat_order(T, H, W), device=x.device)
    return x.index_select(dim, idx)


def flat_to_grid_rows(x: torch.Tensor, T: int, H: int, W: int, dim: int) -> torch.Tensor:
    """Rows of x along `dim` taken from flattened order to grid order."""
    idx = torch.as_tensor(flat_order(T, H, W), device=x.device)
    return torch.empty_like(x).index_copy_(dim, idx, x)


class Case:
    """One workload on the device, flattened, with its mask and attention."""

    def __init__(self, w: inputs.Workload, q=None, k=None, v=None):
        self.w = w
        if q is None:
            q, k, v = inputs.make_qkv(w)
        self.q, self.k, self.v = q, k, v  # host bf16, grid order
        dev = torch.device("cuda")
        self.qd = q.to(dev)
        self.kd = k.to(dev)
        self.vd = v.to(dev)
        self.qf = nabla.flatten(self.qd, w.T, w.H, w.W)
        self.kf = nabla.flatten(self.kd, w.T, w.H, w.W)
        self.vf = nabla.flatten(self.vd, w.T, w.H, w.W)
        self.kv_count, self.kv_idx, self.ws = nabla.build_mask(self.qf, self.kf, w.T, w.H, w.W, w.thr, w.sta,
                                                               radial=w.radial)
        torch.cuda.synchronize()
        assert nabla.get_status() == 0

    def attention(self, grid: bool = True):
        """grid=True calls the grid entry point (the one bench.py times) on the
        grid-order tensors; its out and lse, in grid order, are returned
        permuted back to flattened order, so both paths compare against the
        oracle alike.  grid=False calls the plain entry point on the
        flattened tensors."""
        w = self.w
        if grid:  # grid-order inputs and outputs
            out, lse = nabla.sparse_attn_fwd(self.qd, self.kd, self.vd, self.kv_count, self.kv_idx,
                                             grid=(w.T, w.H, w.W))
            out, lse = grid_to_flat_rows(out, w.T, w.H, w.W, 1), grid_to_flat_rows(lse, w.T, w.H, w.W, 2)
        else:
            out, lse = nabla.sparse_attn_fwd(self.qf, self.kf, self.vf, self.kv_count, self.kv_idx)
        torch.cuda.synchronize()
        assert nabla.get_status() == 0
        return out, lse

    def host_flat(self):
        """The oracle's own flattening of the host inputs (uint16 bf16 bits),
        computed once: oracle inputs never come from the CUDA path."""
        if not hasattr(self, "_host_flat"):
            w = self.w
            self._host_flat = tuple(oracle.flatten(x, w.T, w.H, w.W).reshape(x.shape)
                                    for x in (self.q, self.k, self.v))
        return self._host_flat

    def assert_flatten_matches_oracle(self):
        """The GPU's flattened Q, K, V equal the oracle's bit for bit."""
        for xf, ref in zip((self.qf, self.kf, self.vf), self.host_flat()):
            assert np.array_equal(xf.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def keep_matrix_gpu(kv_count: torch.Tensor, kv_idx: torch.Tensor) -> torch.Tensor:
    """Dense [B,Hh,Nb,Nb] bool keep matrix from block lists (on the device)."""
    B, Hh, Nb = kv_count.shape
    e = torch.arange(Nb, device=kv_count.device, dtype=torch.int32).view(1, 1, 1, Nb)
    valid = e < kv_count.unsqueeze(-1)
    cols = torch.where(valid, kv_idx, torch.full_like(kv_idx, Nb)).long()
    keep = torch.zeros((B, Hh, Nb, Nb + 1), dtype=torch.bool, device=kv_count.device)
    keep.scatter_(3, cols, True)
    return keep[..., :Nb]


def compare_masks(case: Case, status: np.ndarray):
    """Returns (mismatches outside the band, mismatches inside the band,
    number of band blocks).  status is the oracle's per-block byte: bit 0
    kept, bit 1 band (cumulative mass within 1e-5 of 1 - thr, the one class
    the acceptance rule excuses)."""
    st = torch.from_numpy(status).to(case.kv_count.device)
    kept_o = (st & 1).bool()
    band = (st & 2).bool()
    keep_g = keep_matrix_gpu(case.kv_count, case.kv_idx)
    mism = keep_g != kept_o
    bad = int((mism & ~band).sum().item())
    in_band = int((mism & band).sum().item())
    nband = int(band.sum().item())
    # the lists themselves: ascending, in range, count consistent
    assert nabla.validate_mask(case.kv_count, case.kv_idx) == 0
    return bad, in_band, nband


def oracle_masks(case: Case, qf_host, kf_host):
    w = case.w
    qbar = oracle.pool(qf_host)
    kbar = oracle.pool(kf_host)
    cnt, idx, status, _ = oracle.build_mask(qbar, kbar, w.thr, w.scale, w.nbh, w.nbw, sta_window=w.sta,
                                            radial_r0=w.radial)
    return qbar, kbar, cnt, idx, status


def gpu_lists_for(case: Case, qblocks):
    sel = torch.as_tensor(np.asarray(qblocks), dtype=torch.long, device=case.kv_count.device)
    cnt = case.kv_count.index_select(2, sel).cpu().numpy()
    idx = case.kv_idx.index_select(2, sel).cpu().numpy()
    return cnt, idx


def attention_rows(x: torch.Tensor, qblocks) -> np.ndarray:
    """Rows of the listed query blocks from a [B,S,Hh,D] tensor, as fp64."""
    rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qblocks])
    return x[:, torch.as_tensor(rows, device=x.device)].double().cpu().numpy()


def lse_rows(lse: torch.Tensor, qblocks) -> np.ndarray:
    rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qblocks])
    return lse[:, :, torch.as_tensor(rows, device=lse.device)].double().cpu().numpy()


def check_attention(case: Case, out: torch.Tensor, lse: torch.Tensor, qblocks, host_flat=None):
    """Compare GPU attention on the listed query blocks with the oracle run on
    the GPU's own block lists.  Returns (max_abs, mean_abs, lse_max_abs)."""
    qf, kf, vf = host_flat if host_flat is not None else case.host_flat()
    cnt, idx = gpu_lists_for(case, qblocks)
    ref, ref_lse = oracle.attention(qf, kf, vf, cnt, idx, case.w.scale, qblocks=qblocks)
    got = attention_rows(out, qblocks)
    err = np.abs(got - ref)
    got_lse = lse_rows(lse, qblocks)
    finite = np.isfinite(ref_lse)
    assert np.array_equal(finite, np.isfinite(got_lse))
    lse_err = float(np.abs(got_lse[finite] - ref_lse[finite]).max()) if finite.any() else 0.0
    return float(err.max()), float(err.mean()), lse_err


def block_rows(blocks) -> np.ndarray:
    """Flattened token rows of the listed blocks, in list order."""
    return np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in blocks])


def sampled_gradient_errors(dq, dk, dv, ref, qblocks, kblocks):
    """Relative errors of flattened-order gradients [B,S,Hh,D] (torch, any
    device) against the oracle's sampled gradient (dq of qblocks, dk and dv
    of kblocks): per tensor (max|err| / max|ref|, mean|err| / mean|ref|)."""
    out = []
    for got, r, blocks in ((dq, ref[0], qblocks), (dk, ref[1], kblocks), (dv, ref[2], kblocks)):
        rows = torch.as_tensor(block_rows(blocks), device=got.device)
        g = got.index_select(1, rows).double().cpu().numpy()
        err = np.abs(g - r)
        out.append((err.max() / max(np.abs(r).max(), 1e-30), err.mean() / max(np.abs(r).mean(), 1e-30)))
    return out
