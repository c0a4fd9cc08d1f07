"""CPU oracle for NABLA block-sparse attention -- test infrastructure only.

This package wraps ``oracle.c`` (plain scalar C, OpenMP over independent
rows) with ctypes.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product path (``block_sparse_attention_flatten_b200``) never imports it
and shares no code with it.

Every function restates one step of the method as described on the page
"Resumo Tecnico: NABLA - Atencao de Bloco Adaptativa de Vizinhanca para
Geracao de Video Eficiente" (section "Metodologia: NABLA"); the C source
names the item each one follows.

Parity unpinned: the STA window geometry beyond "a static local window"
(centred, truncated at the border, temporal tile = one frame) is a reading
of the pages, checked only against its own closed-form count.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

BLOCK = 64  # N = P * P tokens per block (P = 8)
BAND = 1e-5  # |c - (1 - thr)| below this marks a band block


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no fused multiply-add)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
               "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        P = ctypes.c_void_p
        i, i64, f, d = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        lib.oracle_flatten.argtypes = [P, P, i, i, i, i, i, i64]
        lib.oracle_unflatten.argtypes = [P, P, i, i, i, i, i, i64]
        lib.oracle_pool.argtypes = [P, P, i, i, i, i]
        lib.oracle_mask.argtypes = [P, P, i, i, i, i, f, f, i, i, i, i, i, i, d, P, P, P, P]
        lib.oracle_attention.argtypes = [P, P, P, P, P, i, i, i, i, d, P, i, P, P]
        lib.oracle_block_probs_row.argtypes = [P, P, i, i, f, i, P]
        lib.oracle_block_numerators_row.argtypes = [P, P, i, i, f, i, P]
        lib.oracle_cdf_keep.argtypes = [P, i, f, P, P, P, d]
        lib.oracle_cdf_keep.restype = i
        lib.oracle_sta.argtypes = [i, i, i, i, i, i, i]
        lib.oracle_sta.restype = i
        lib.oracle_sta_lists.argtypes = [i, i, i, i, i, i, P, P]
        lib.oracle_radial_lists.argtypes = [i, i, i, i, P, P]
        lib.oracle_radial.argtypes = [i, i, i, i, i]
        lib.oracle_radial.restype = i
        lib.oracle_attention_bwd.argtypes = [P, P, P, P, P, P, i, i, i, i, d, P, P, P]
        lib.oracle_attention_bwd_sampled.argtypes = [P, P, P, P, P, P, i, i, i, i, d, P, i, P, i, P, P, P]
        lib.oracle_num_threads.restype = i
        lib.oracle_set_num_threads.argtypes = [i]
        lib.oracle_ab_key_means.argtypes = [P, i, i, i, i, P]
        lib.oracle_ab_kmeans.argtypes = [P, i, i, i, i, i, P, P, P]
        lib.oracle_ab_scores.argtypes = [P, P, P, i, i, i, i, i, f, P]
        lib.oracle_ab_inclusion.argtypes = [P, i, d, P]
        lib.oracle_ab_inclusion.restype = d
        lib.oracle_ab_inclusion_all.argtypes = [P, i64, i, d, P]
        lib.oracle_ab_attention.argtypes = [P, P, P, P, P, P, i, i, i, i, d, P, i, P, P]
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    """Threads of the oracle's OpenMP loops (results do not depend on it)."""
    _load().oracle_set_num_threads(int(n))


def _bits(x: np.ndarray) -> np.ndarray:
    """bf16 data as raw uint16 bits (accepts a uint16 array or a torch bf16 tensor)."""
    if hasattr(x, "view") and not isinstance(x, np.ndarray):  # torch tensor
        import torch
        x = x.contiguous().view(torch.int16).numpy().view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


def flatten(x, T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    """Fractal flattening of a grid-order [B, S, row] bf16 array (uint16 bits)."""
    x = _bits(x)
    B = x.shape[0]
    row = int(np.prod(x.shape[2:]))
    out = np.empty_like(x)
    _load().oracle_flatten(_ptr(x), _ptr(out), B, T, H, W, P, row)
    return out


def unflatten(x, T: int, H: int, W: int, P: int = 8) -> np.ndarray:
    """Inverse of :func:`flatten`."""
    x = _bits(x)
    B = x.shape[0]
    row = int(np.prod(x.shape[2:]))
    out = np.empty_like(x)
    _load().oracle_unflatten(_ptr(x), _ptr(out), B, T, H, W, P, row)
    return out


def pool(xf) -> np.ndarray:
    """Block means of a flattened [B, S, Hh, D] bf16 array -> fp32 [B, Hh, Nb, D]."""
    xf = _bits(xf)
    B, S, Hh, D = xf.shape
    out = np.empty((B, Hh, S // BLOCK, D), dtype=np.float32)
    _load().oracle_pool(_ptr(xf), _ptr(out), B, S, Hh, D)
    return out


def block_probs_row(qbar_bh: np.ndarray, kbar_bh: np.ndarray, i: int, scale: float) -> np.ndarray:
    """Reduced-attention probabilities of query block i for one (b, head)."""
    qbar_bh = np.ascontiguousarray(qbar_bh, dtype=np.float32)
    kbar_bh = np.ascontiguousarray(kbar_bh, dtype=np.float32)
    Nb, D = kbar_bh.shape
    p = np.empty(Nb, dtype=np.float32)
    _load().oracle_block_probs_row(_ptr(qbar_bh), _ptr(kbar_bh), Nb, D, scale, i, _ptr(p))
    return p


def block_numerators_row(qbar_bh: np.ndarray, kbar_bh: np.ndarray, i: int, scale: float) -> np.ndarray:
    """Softmax numerators e = exp(s - max s) (fp32) of query block i for one
    (b, head): the weights the CDF rule orders and accumulates."""
    qbar_bh = np.ascontiguousarray(qbar_bh, dtype=np.float32)
    kbar_bh = np.ascontiguousarray(kbar_bh, dtype=np.float32)
    Nb, D = kbar_bh.shape
    e = np.empty(Nb, dtype=np.float32)
    _load().oracle_block_numerators_row(_ptr(qbar_bh), _ptr(kbar_bh), Nb, D, scale, i, _ptr(e))
    return e


def cdf_keep(p: np.ndarray, thr: float, band: float = BAND):
    """CDF keep flags, per-block cumulative mass, band flags and the arg-max
    for one row of weights (probabilities, or the softmax numerators: the
    rule normalises them by their sum)."""
    p = np.ascontiguousarray(p, dtype=np.float32)
    keep = np.empty(p.shape[0], dtype=np.uint8)
    cum = np.empty(p.shape[0], dtype=np.float64)
    bandf = np.empty(p.shape[0], dtype=np.uint8)
    argmax = _load().oracle_cdf_keep(_ptr(p), p.shape[0], thr, _ptr(keep), _ptr(cum), _ptr(bandf), band)
    return keep.astype(bool), cum, bandf.astype(bool), argmax


def sta(i: int, j: int, nbh: int, nbw: int, window=(3, 3, 3)) -> bool:
    return bool(_load().oracle_sta(i, j, nbh, nbw, *window))


def sta_lists(nbt: int, nbh: int, nbw: int, window=(3, 3, 3)):
    """The static window alone as block lists for one (b, head):
    kv_count int32 [Nb], kv_idx int32 [Nb, Nb] (ascending, -1 past the count)."""
    Nb = nbt * nbh * nbw
    kv_count = np.zeros(Nb, dtype=np.int32)
    kv_idx = np.full((Nb, Nb), -1, dtype=np.int32)
    _load().oracle_sta_lists(Nb, nbh, nbw, int(window[0]), int(window[1]), int(window[2]),
                             _ptr(kv_count), _ptr(kv_idx))
    return kv_count, kv_idx


def radial(i: int, j: int, nbh: int, nbw: int, r0: int) -> bool:
    return bool(_load().oracle_radial(i, j, nbh, nbw, r0))


def radial_lists(nbt: int, nbh: int, nbw: int, r0: int):
    """The radial window alone as block lists for one (b, head): kv_count
    int32 [Nb], kv_idx int32 [Nb, Nb] (ascending, -1 past the count)."""
    Nb = nbt * nbh * nbw
    kv_count = np.zeros(Nb, dtype=np.int32)
    kv_idx = np.full((Nb, Nb), -1, dtype=np.int32)
    _load().oracle_radial_lists(Nb, nbh, nbw, int(r0), _ptr(kv_count), _ptr(kv_idx))
    return kv_count, kv_idx


def build_mask(qbar: np.ndarray, kbar: np.ndarray, thr: float, scale: float, nbh: int, nbw: int,
               sta_window=(0, 0, 0), band: float = BAND, want_status: bool = True,
               want_probs: bool = False, radial_r0: int = 0):
    """Masks for every row, the adaptive mask OR-ed with the sliding-tile
    window (sta_window) and the radial window (radial_r0 > 0).  Returns
    (kv_count, kv_idx, status, probs).

    kv_count int32 [B,Hh,Nb]; kv_idx int32 [B,Hh,Nb,Nb] (ascending, padded
    with -1 past the count); status uint8 [B,Hh,Nb,Nb] (bit0 kept, bit1 band)
    or None; probs fp32 [B,Hh,Nb,Nb] or None.
    """
    qbar = np.ascontiguousarray(qbar, dtype=np.float32)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, Hh, Nb, D = qbar.shape
    kv_count = np.zeros((B, Hh, Nb), dtype=np.int32)
    kv_idx = np.full((B, Hh, Nb, Nb), -1, dtype=np.int32)
    status = np.zeros((B, Hh, Nb, Nb), dtype=np.uint8) if want_status else None
    probs = np.zeros((B, Hh, Nb, Nb), dtype=np.float32) if want_probs else None
    _load().oracle_mask(_ptr(qbar), _ptr(kbar), B, Hh, Nb, D, scale, thr, nbh, nbw,
                        int(sta_window[0]), int(sta_window[1]), int(sta_window[2]), int(radial_r0), band,
                        _ptr(kv_count), _ptr(kv_idx),
                        _ptr(status) if status is not None else None,
                        _ptr(probs) if probs is not None else None)
    return kv_count, kv_idx, status, probs


def attention(qf, kf, vf, kv_count: np.ndarray, kv_idx: np.ndarray, scale: float, qblocks=None):
    """Masked attention (fp64) for the listed query blocks (all heads).

    kv_count/kv_idx are the full lists [B,Hh,Nb] / [B,Hh,Nb,Nb] or, when
    qblocks is given, may already be restricted to those blocks
    ([B,Hh,nq] / [B,Hh,nq,Nb]).
    Returns (out fp64 [B, nq*64, Hh, D], lse fp64 [B, Hh, nq*64]).
    """
    qf, kf, vf = _bits(qf), _bits(kf), _bits(vf)
    B, S, Hh, D = qf.shape
    Nb = S // BLOCK
    if qblocks is None:
        qblocks = np.arange(Nb, dtype=np.int32)
    qblocks = np.ascontiguousarray(qblocks, dtype=np.int32)
    nq = qblocks.shape[0]
    kv_count = np.asarray(kv_count)
    kv_idx = np.asarray(kv_idx)
    if kv_count.shape[-1] != nq:
        kv_count = kv_count[:, :, qblocks]
        kv_idx = kv_idx[:, :, qblocks]
    kv_count = np.ascontiguousarray(kv_count, dtype=np.int32)
    kv_idx = np.ascontiguousarray(kv_idx, dtype=np.int32)
    assert kv_count.shape == (B, Hh, nq) and kv_idx.shape == (B, Hh, nq, Nb)
    out = np.zeros((B, nq * BLOCK, Hh, D), dtype=np.float64)
    lse = np.zeros((B, Hh, nq * BLOCK), dtype=np.float64)
    _load().oracle_attention(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(kv_count), _ptr(kv_idx), B, S, Hh, D,
                             scale, _ptr(qblocks), nq, _ptr(out), _ptr(lse))
    return out, lse


def attention_bwd(qf, kf, vf, dof, kv_count: np.ndarray, kv_idx: np.ndarray, scale: float):
    """Gradients (dq, dk, dv), fp64 [B, S, Hh, D], of sum(dO * O) for the
    attention on the kept tiles (flattened order; full lists)."""
    qf, kf, vf, dof = _bits(qf), _bits(kf), _bits(vf), _bits(dof)
    B, S, Hh, D = qf.shape
    kv_count = np.ascontiguousarray(kv_count, dtype=np.int32)
    kv_idx = np.ascontiguousarray(kv_idx, dtype=np.int32)
    assert kv_count.shape == (B, Hh, S // BLOCK) and kv_idx.shape == (B, Hh, S // BLOCK, S // BLOCK)
    dq = np.empty((B, S, Hh, D), dtype=np.float64)
    dk = np.empty_like(dq)
    dv = np.empty_like(dq)
    _load().oracle_attention_bwd(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(dof), _ptr(kv_count), _ptr(kv_idx),
                                 B, S, Hh, D, scale, _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


def attention_bwd_sampled(qf, kf, vf, dof, kv_count: np.ndarray, kv_idx: np.ndarray, scale: float,
                          qblocks, kblocks):
    """:func:`attention_bwd` restricted to listed blocks: dq fp64 [B, nq*64,
    Hh, D] for the query blocks qblocks, dk and dv fp64 [B, nk*64, Hh, D] for
    the key blocks kblocks (each list ascending or not, no repeats)."""
    qf, kf, vf, dof = _bits(qf), _bits(kf), _bits(vf), _bits(dof)
    B, S, Hh, D = qf.shape
    kv_count = np.ascontiguousarray(kv_count, dtype=np.int32)
    kv_idx = np.ascontiguousarray(kv_idx, dtype=np.int32)
    qblocks = np.ascontiguousarray(qblocks, dtype=np.int32)
    kblocks = np.ascontiguousarray(kblocks, dtype=np.int32)
    nq, nk = qblocks.shape[0], kblocks.shape[0]
    dq = np.empty((B, nq * BLOCK, Hh, D), dtype=np.float64)
    dk = np.empty((B, nk * BLOCK, Hh, D), dtype=np.float64)
    dv = np.empty_like(dk)
    _load().oracle_attention_bwd_sampled(_ptr(qf), _ptr(kf), _ptr(vf), _ptr(dof), _ptr(kv_count), _ptr(kv_idx),
                                         B, S, Hh, D, scale, _ptr(qblocks), nq, _ptr(kblocks), nk,
                                         _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv


# ---------------------------------------------------------------- AB-Attention
AB_QBLOCK = 128
AB_CLUSTERS = 8
AB_KBLOCK = 4


def ab_key_means(k) -> np.ndarray:
    """Mean key of every 4-token block (grid order): fp32 [B, Hh, S/4, D]."""
    k = _bits(k)
    B, S, Hh, D = k.shape
    out = np.empty((B, Hh, S // AB_KBLOCK, D), dtype=np.float32)
    _load().oracle_ab_key_means(_ptr(k), B, S, Hh, D, _ptr(out))
    return out


def ab_kmeans(q, iters: int = 4):
    """IBCS clustering of every 128-query block: (centroids fp32 [B, Hh, NQB,
    8, D], counts int32 [B, Hh, NQB, 8], assignment int32 [B, Hh, S])."""
    q = _bits(q)
    B, S, Hh, D = q.shape
    nqb = S // AB_QBLOCK
    cent = np.empty((B, Hh, nqb, AB_CLUSTERS, D), dtype=np.float32)
    counts = np.empty((B, Hh, nqb, AB_CLUSTERS), dtype=np.int32)
    assign = np.empty((B, Hh, S), dtype=np.int32)
    _load().oracle_ab_kmeans(_ptr(q), B, S, Hh, D, iters, _ptr(cent), _ptr(counts), _ptr(assign))
    return cent, counts, assign


def ab_scores(cent: np.ndarray, counts: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """IBCS block scores, fp64 [B, Hh, NQB, NKB]."""
    cent = np.ascontiguousarray(cent, dtype=np.float32)
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    kbar = np.ascontiguousarray(kbar, dtype=np.float32)
    B, Hh, nqb, _, D = cent.shape
    nkb = kbar.shape[2]
    out = np.empty((B, Hh, nqb, nkb), dtype=np.float64)
    _load().oracle_ab_scores(_ptr(cent), _ptr(counts), _ptr(kbar), B, Hh, nqb, nkb, D, scale, _ptr(out))
    return out


def ab_inclusion(score: np.ndarray, budget: float) -> np.ndarray:
    """SIP inclusion probabilities (fp64) for every row of scores (last axis)."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    pi = np.empty_like(score)
    n = score.shape[-1]
    _load().oracle_ab_inclusion_all(_ptr(score), score.size // n, n, float(budget), _ptr(pi))
    return pi


def ab_inclusion_row(score: np.ndarray, budget: float):
    """(pi, lambda) for one row."""
    score = np.ascontiguousarray(score, dtype=np.float64)
    pi = np.empty_like(score)
    lam = _load().oracle_ab_inclusion(_ptr(score), score.shape[0], float(budget), _ptr(pi))
    return pi, lam


def ab_sample(pi: np.ndarray, u: np.ndarray):
    """Poisson sampling: block J of a row is in the sample iff u_J < pi_J.
    Returns (count int32 [...], idx int32 [..., NKB] ascending and -1 past the
    count, shift fp64 [..., NKB] = -log(pi) of each listed block)."""
    inc = u.astype(np.float64) < pi
    n = pi.shape[-1]
    count = inc.sum(axis=-1).astype(np.int32)
    idx = np.full(pi.shape, -1, dtype=np.int32)
    shift = np.zeros(pi.shape, dtype=np.float64)
    flat_inc = inc.reshape(-1, n)
    flat_pi = pi.reshape(-1, n)
    fi, fs = idx.reshape(-1, n), shift.reshape(-1, n)
    for r in range(flat_inc.shape[0]):
        js = np.nonzero(flat_inc[r])[0]
        fi[r, :js.size] = js
        fs[r, :js.size] = -np.log(flat_pi[r, js])
    return count, idx, shift


def ab_attention(q, k, v, kcount, kidx, shift, scale: float, qblocks=None):
    """Attention of the listed 128-token query blocks over their sampled
    4-token key blocks with the Horvitz-Thompson logit shifts (fp64).
    kcount/kidx/shift either cover every query block or, when qblocks is
    given, may already be restricted to them.  Returns (out fp64 [B,
    nq*128, Hh, D], lse fp64 [B, Hh, nq*128])."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, S, Hh, D = q.shape
    nqb, nkb = S // AB_QBLOCK, S // AB_KBLOCK
    if qblocks is None:
        qblocks = np.arange(nqb, dtype=np.int32)
    qblocks = np.ascontiguousarray(qblocks, dtype=np.int32)
    nq = qblocks.shape[0]
    kcount, kidx, shift = np.asarray(kcount), np.asarray(kidx), np.asarray(shift)
    if kcount.shape[-1] != nq:
        kcount, kidx, shift = kcount[:, :, qblocks], kidx[:, :, qblocks], shift[:, :, qblocks]
    kcount = np.ascontiguousarray(kcount, dtype=np.int32)
    kidx = np.ascontiguousarray(kidx, dtype=np.int32)
    shift = np.ascontiguousarray(shift, dtype=np.float64)
    assert kidx.shape == (B, Hh, nq, nkb) and shift.shape == (B, Hh, nq, nkb)
    out = np.zeros((B, nq * AB_QBLOCK, Hh, D), dtype=np.float64)
    lse = np.zeros((B, Hh, nq * AB_QBLOCK), dtype=np.float64)
    _load().oracle_ab_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(kcount), _ptr(kidx), _ptr(shift), B, S, Hh, D,
                                scale, _ptr(qblocks), nq, _ptr(out), _ptr(lse))
    return out, lse
