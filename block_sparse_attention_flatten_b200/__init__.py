"""NABLA adaptive block-sparse attention for one NVIDIA B200 (sm_100a).

The compute path is libnabla.so (hand-written CUDA, C ABI in
include/nabla.h); this package is its thin Python binding.  PyTorch only
provides device memory and streams.

Grid-order tensors (token (t, h, w) at row (t*H + h)*W + w), no flattened
copies -- the fractal flattening happens inside the kernels:

    from block_sparse_attention_flatten_b200 import nabla
    kv_count, kv_idx, _ = nabla.build_mask_grid(q, k, T, H, W, thr=0.9, sta=(3, 3, 3))
    o, lse = nabla.sparse_attn_fwd(q, k, v, kv_count, kv_idx, grid=(T, H, W))

Backward pass over the same lists (training), grid order as well:

    dq, dk, dv = nabla.sparse_attn_bwd(q, k, v, o, do, lse, kv_count, kv_idx, grid=(T, H, W))

The static sliding-tile window alone, without reading Q or K:

    kv_count, kv_idx = nabla.build_mask_sta(B, Hh, T, H, W, (3, 3, 3))

A radial decay window, alone or OR-ed into the adaptive mask:

    kv_count, kv_idx = nabla.build_mask_radial(B, Hh, T, H, W, r0=2)
    kv_count, kv_idx, _ = nabla.build_mask_grid(q, k, T, H, W, thr=0.9, radial=2)

AB-Attention on the same grid-order tensors (u: uniforms [B, Hh, S/128, S/4]):

    kcount, kidx, kshift, _ = nabla.ab_plan(q, k, u, budget=0.1 * S / 4)
    o, lse = nabla.ab_attn_fwd(q, k, v, kcount, kidx, kshift)

Flattened tensors (e.g. flattened once per sequence):

    qf = nabla.flatten(q, T, H, W)                       # per tensor
    kv_count, kv_idx, _ = nabla.build_mask(qf, kf, T, H, W, thr=0.9, sta=(3, 3, 3))
    of, lse = nabla.sparse_attn_fwd(qf, kf, vf, kv_count, kv_idx)
    o = nabla.unflatten(of, T, H, W)
"""
from . import _lib as nabla  # noqa: F401

__all__ = ["nabla"]
