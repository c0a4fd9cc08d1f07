"""nabla_build_mask_noalloc: the mask entry point for callers that cannot
allocate device memory (a plug-in host or serving runtime that owns all
device memory and exposes no allocator, or a latency-critical path that
cannot afford cudaMalloc's device-wide synchronisation).

It keeps the pooled queries and keys in the library's own static 16 MiB
device buffer instead of a caller-provided workspace.  Its block lists must
equal those of nabla_build_mask, the allocating entry point, exactly (they
are integers; the existing tests hold masks to bit-exactness), on two calls
in a row that reuse the shared buffer with different shapes.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process, where its first call performs the per-device set-up.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu


def _noalloc_call(qf, kf, w, kv_count, kv_idx):
    """Call the C entry point directly through the C ABI."""
    B, S, Hh, D = qf.shape
    prm = nabla.params(w.thr, w.sta)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return nabla.lib().nabla_build_mask_noalloc(
        ctypes.c_void_p(qf.data_ptr()), ctypes.c_void_p(kf.data_ptr()), B, Hh, D, w.T, w.H, w.W,
        ctypes.byref(prm), ctypes.c_void_p(kv_count.data_ptr()), ctypes.c_void_p(kv_idx.data_ptr()), stream)


def _lists_equal(cnt_a, idx_a, cnt_b, idx_b):
    if not torch.equal(cnt_a, cnt_b):
        return False
    Nb = cnt_a.shape[-1]
    valid = torch.arange(Nb, device=cnt_a.device).view(1, 1, 1, Nb) < cnt_a.unsqueeze(-1)
    return torch.equal(torch.where(valid, idx_a, -1), torch.where(valid, idx_b, -1))


def test_noalloc_mask_matches_build_mask_on_two_calls():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    workloads = [
        inputs.WAN13B,  # workspace 11.8 MB of the 16 MiB buffer
        inputs.Workload("STA layer", 2, 4, 64, 5, 24, 24, 1.0, 0.8, sta=(3, 3, 3), seed=71),
    ]
    for w in workloads:
        q, k, _ = inputs.make_qkv(w)
        qf = nabla.flatten(q.cuda(), w.T, w.H, w.W)
        kf = nabla.flatten(k.cuda(), w.T, w.H, w.W)
        ref_cnt, ref_idx, _ = nabla.build_mask(qf, kf, w.T, w.H, w.W, w.thr, w.sta)
        cnt = torch.full_like(ref_cnt, -7)
        idx = torch.full_like(ref_idx, -7)
        rc = _noalloc_call(qf, kf, w, cnt, idx)
        assert rc == nabla.NABLA_OK, nabla.strerror(rc)
        torch.cuda.synchronize()
        assert nabla.get_status() == nabla.NABLA_OK
        assert _lists_equal(cnt, idx, ref_cnt, ref_idx), w.name


def test_noalloc_rejects_problems_larger_than_its_buffer():
    w = inputs.HUNYUAN  # needs 2 * 24 * 1920 * 128 * 4 = 47 MB of pooled vectors
    prm = nabla.params(w.thr, w.sta)
    assert nabla.mask_workspace_bytes(w.B, w.Hh, w.D, w.T, w.H, w.W, prm) > nabla.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(0x1000)
    rc = nabla.lib().nabla_build_mask_noalloc(fake, fake, w.B, w.Hh, w.D, w.T, w.H, w.W, ctypes.byref(prm), fake,
                                              fake, ctypes.c_void_p(0))
    assert rc == nabla.NABLA_ERR_TOO_LARGE
    assert "scratch" in nabla.strerror(rc)
