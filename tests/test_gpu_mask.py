"""GPU mask selection on hand-built pooled vectors, against the oracle.

The selection never sorts a row: it finds the boundary of the ascending
order of the softmax numerators with mass histograms, then recomputes the
correctly rounded numerator wherever CUDA's expf (within 2 ulp) could order
two blocks differently.  These cases aim at exactly those paths:

* every score equal (all numerators 1: more than 32 equal values, the
  boundary is an index among them, ties kept from the highest index);
* scores clustered within a few ulp (hundreds of blocks inside the
  exactness window: the whole row is recomputed exactly);
* exact duplicates among the key vectors (ties broken by block index);
* random rows at the shapes of the measured layers' heads, an odd block
  count and a single block.

The pooled vectors are written straight into the mask workspace, so the
scores are fixed by construction; the block lists of nabla_build_mask_pooled
must equal the oracle's everywhere outside the 1e-5 band.  The same kinds of
rows also go through the in-shared-memory kernel (the no-allocation entry
point) from bf16 inputs built to pool to them.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from _parity import keep_matrix_gpu
from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    oracle.build()


def run_pooled(qbar: np.ndarray, kbar: np.ndarray, T, H, W, thr, sta=(0, 0, 0)):
    """GPU lists from given pooled vectors (fp32 [B,Hh,Nb,D]) and the oracle's
    status for the same vectors; returns (bad, in_band, band, kv_count)."""
    B, Hh, Nb, D = qbar.shape
    prm = nabla.params(thr, sta)
    ws = torch.empty(nabla.mask_workspace_bytes(B, Hh, D, T, H, W, prm), dtype=torch.uint8, device="cuda")
    qv, kv = nabla.pooled_from_workspace(ws, B, Hh, Nb, D)
    qv.copy_(torch.from_numpy(qbar))
    kv.copy_(torch.from_numpy(kbar))
    cnt, idx = nabla.build_mask_pooled(ws, B, Hh, D, T, H, W, thr, sta)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    assert nabla.validate_mask(cnt, idx) == 0
    scale = 1.0 / np.sqrt(D)
    _, _, status, _ = oracle.build_mask(qbar, kbar, thr, scale, H // 8, W // 8, sta_window=sta)
    return compare(cnt, idx, status) + (cnt,)


def compare(cnt, idx, status):
    st = torch.from_numpy(status).cuda()
    kept_o = (st & 1).bool()
    band = (st & 2).bool()
    mism = keep_matrix_gpu(cnt, idx) != kept_o
    return int((mism & ~band).sum()), int((mism & band).sum()), int(band.sum())


def rng_vectors(seed, shape, scale=1.0):
    g = np.random.default_rng(seed)
    return (g.standard_normal(shape) * scale).astype(np.float32)


GRID_960 = (16, 48, 80)  # 960 blocks, 6 x 10 per frame
GRID_3840 = (64, 48, 80)  # 3,840 blocks


@pytest.mark.parametrize("thr", [0.0, 0.37, 0.5, 0.9, 1.0])
def test_all_scores_equal(thr):
    """q = 0: every score is 0, every numerator exactly 1; the kept blocks are
    the highest indices whose count the threshold fixes (ceil(thr * Nb) of
    them, strictly: cumulative (k+1)/Nb > 1 - thr)."""
    T, H, W = GRID_960
    Nb = 960
    qbar = np.zeros((1, 2, Nb, 128), np.float32)
    kbar = rng_vectors(1, (1, 2, Nb, 128))
    bad, in_band, band, cnt = run_pooled(qbar, kbar, T, H, W, thr)
    assert bad == 0, (bad, in_band, band)


@pytest.mark.parametrize("thr", [0.5, 0.9])
@pytest.mark.parametrize("spread", [1e-7, 1e-6, 3e-6])
def test_scores_clustered_within_a_few_ulp(thr, spread):
    """Key vectors equal up to a relative perturbation of `spread`: the
    numerators of a row lie within a few ulp of each other, so hundreds of
    blocks fall in the window where expf's error could reorder them."""
    T, H, W = GRID_960
    Nb = 960
    base = rng_vectors(2, (1, 2, 1, 128))
    kbar = (base * (1.0 + spread * rng_vectors(3, (1, 2, Nb, 128)))).astype(np.float32)
    qbar = rng_vectors(4, (1, 2, Nb, 128), 0.3)
    bad, in_band, band, cnt = run_pooled(qbar, kbar, T, H, W, thr)
    assert bad == 0, (bad, in_band, band)


@pytest.mark.parametrize("thr", [0.3, 0.7, 0.95])
def test_exact_duplicate_keys(thr):
    """Key vectors drawn from five distinct ones: exact ties in every row,
    ordered by block index."""
    T, H, W = GRID_960
    Nb = 960
    pool = rng_vectors(5, (5, 128))
    pick = np.random.default_rng(6).integers(0, 5, size=Nb)
    kbar = np.broadcast_to(pool[pick], (1, 1, Nb, 128)).astype(np.float32).copy()
    kbar = np.concatenate([kbar, kbar[:, :, ::-1]], axis=1).copy()
    qbar = rng_vectors(7, (1, 2, Nb, 128))
    bad, in_band, band, cnt = run_pooled(qbar, kbar, T, H, W, thr)
    assert bad == 0, (bad, in_band, band)


@pytest.mark.parametrize("shape,thr,sta", [
    (GRID_960, 0.7, (0, 0, 0)),
    (GRID_960, 0.9, (3, 3, 3)),
    (GRID_3840, 0.9, (3, 3, 3)),
    ((37, 8, 8), 0.8, (0, 0, 0)),   # odd block count (Nb = 37, padded to 40)
    ((1, 8, 8), 0.5, (0, 0, 0)),    # a single block
    ((5, 24, 24), 0.6, (3, 3, 3)),  # Nb = 45, D 64 below
])
def test_random_rows(shape, thr, sta):
    T, H, W = shape
    Nb = T * (H // 8) * (W // 8)
    D = 64 if Nb == 45 else 128
    Hh = 1 if Nb == 3840 else 3
    # pooled vectors of the locality-structured inputs have a common
    # component; mimic it so the rows are peaked like the layers'
    common = rng_vectors(8, (1, Hh, 1, D))
    qbar = (common + 0.5 * rng_vectors(9, (1, Hh, Nb, D))).astype(np.float32)
    kbar = (common + 0.5 * rng_vectors(10, (1, Hh, Nb, D))).astype(np.float32)
    bad, in_band, band, cnt = run_pooled(qbar, kbar, T, H, W, thr, sta)
    print(f"\nNb {Nb}: kept {float(cnt.double().mean()) / Nb:.3f}, band blocks {band}, in-band mismatches {in_band}")
    assert bad == 0, (bad, in_band, band)


def _noalloc(qf, kf, T, H, W, thr, sta):
    B, S, Hh, D = qf.shape
    Nb = S // 64
    prm = nabla.params(thr, sta)
    cnt = torch.empty((B, Hh, Nb), dtype=torch.int32, device="cuda")
    idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device="cuda")
    rc = nabla.lib().nabla_build_mask_noalloc(
        ctypes.c_void_p(qf.data_ptr()), ctypes.c_void_p(kf.data_ptr()), B, Hh, D, T, H, W, ctypes.byref(prm),
        ctypes.c_void_p(cnt.data_ptr()), ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == nabla.NABLA_OK, nabla.strerror(rc)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    return cnt, idx


@pytest.mark.parametrize("kind", ["zero queries", "duplicate key blocks"])
@pytest.mark.parametrize("thr", [0.5, 0.9])
def test_in_shared_memory_kernel_on_tied_rows(kind, thr):
    """The single-kernel path (scores in shared memory, no scratch) on inputs
    whose pooled vectors tie: Q = 0 (every score 0), or K made of copies of
    a few 64-token blocks (exactly equal key vectors)."""
    w = inputs.Workload("tied", 1, 2, 128, 4, 48, 80, 1.0, thr, seed=12)
    q, k, _ = inputs.make_qkv(w)
    if kind == "zero queries":
        q = torch.zeros_like(q)
    else:
        kf_host = torch.from_numpy(oracle.flatten(k, w.T, w.H, w.W).reshape(k.shape).view(np.int16)).view(torch.bfloat16)
        src = np.random.default_rng(13).integers(0, 4, size=w.Nb)
        kf_host = kf_host.view(w.B, w.Nb, 64, w.Hh, w.D)[:, src].reshape(k.shape).contiguous()
        k = torch.from_numpy(oracle.unflatten(kf_host, w.T, w.H, w.W).reshape(k.shape).view(np.int16)).view(torch.bfloat16)
    qf = nabla.flatten(q.cuda(), w.T, w.H, w.W)
    kf = nabla.flatten(k.cuda(), w.T, w.H, w.W)
    cnt, idx = _noalloc(qf, kf, w.T, w.H, w.W, thr, (0, 0, 0))
    qf_h = oracle.flatten(q, w.T, w.H, w.W).reshape(q.shape)
    kf_h = oracle.flatten(k, w.T, w.H, w.W).reshape(k.shape)
    _, _, status, _ = oracle.build_mask(oracle.pool(qf_h), oracle.pool(kf_h), thr, w.scale, w.nbh, w.nbw)
    bad, in_band, band = compare(cnt, idx, status)
    assert bad == 0, (bad, in_band, band)
    # and the scratch path agrees with it exactly
    cnt2, idx2, _ = nabla.build_mask(qf, kf, w.T, w.H, w.W, thr)
    assert torch.equal(keep_matrix_gpu(cnt, idx), keep_matrix_gpu(cnt2, idx2))
