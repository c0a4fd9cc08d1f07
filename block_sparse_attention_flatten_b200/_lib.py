"""ctypes binding of libnabla.so: argument marshalling only.

Every function here checks that its tensors are CUDA tensors of the right
dtype and layout, allocates missing outputs with torch (the library itself
allocates no device memory), and passes raw device pointers, sizes and the
current CUDA stream to the C entry point of the same name (include/nabla.h).
There is no CPU fallback: a missing library or a non-CUDA tensor raises.

To capture calls in a CUDA graph, pass every output and workspace
preallocated (then nothing here allocates, and the calls launch only on the
capturing stream); get_status and validate_mask synchronise and stay
outside a capture.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnabla.so")
BLOCK = 64

NABLA_OK = 0
NABLA_ERR_INVALID = 1
NABLA_ERR_ALIGN = 2
NABLA_ERR_CUDA = 3
NABLA_ERR_DEVICE_TIMEOUT = 4
NABLA_ERR_DEVICE_BOUNDS = 5
NABLA_ERR_UNSUPPORTED = 6
NABLA_ERR_TOO_LARGE = 7
NOALLOC_SCRATCH_BYTES = 16 << 20

EXPORTS = (
    "nabla_flatten",
    "nabla_unflatten",
    "nabla_mask_workspace_bytes",
    "nabla_build_mask",
    "nabla_build_mask_noalloc",
    "nabla_flatten_pool_qk",
    "nabla_build_mask_pooled",
    "nabla_build_mask_grid",
    "nabla_build_mask_sta",
    "nabla_build_mask_radial",
    "nabla_sparse_attn_fwd",
    "nabla_sparse_attn_fwd_grid",
    "nabla_sparse_attn_fwd_grid_split",
    "nabla_attn_split_workspace_bytes",
    "nabla_transpose_lists",
    "nabla_sparse_attn_bwd",
    "nabla_sparse_attn_bwd_grid",
    "nabla_ab_workspace_bytes",
    "nabla_ab_plan",
    "nabla_ab_attn_fwd",
    "nabla_get_status",
    "nabla_validate_mask",
    "nabla_selftest_wait_timeout",
    "nabla_strerror",
)


class NablaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (code {code})")


class NablaParams(ctypes.Structure):
    _fields_ = [
        ("P", ctypes.c_int),
        ("thr", ctypes.c_float),
        ("sta_t", ctypes.c_int),
        ("sta_h", ctypes.c_int),
        ("sta_w", ctypes.c_int),
        ("scale", ctypes.c_float),
        ("flags", ctypes.c_uint),
        ("radial", ctypes.c_int),
    ]


_lib = None


def lib():
    """Load libnabla.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libnabla.so is missing at {LIB_PATH}; build it with "
                               "`python -m block_sparse_attention_flatten_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        pp = ctypes.POINTER(NablaParams)
        L.nabla_flatten.argtypes = [vp, vp, i, i, i, i, i, i, vp]
        L.nabla_unflatten.argtypes = [vp, vp, i, i, i, i, i, i, vp]
        L.nabla_mask_workspace_bytes.argtypes = [i, i, i, i, i, i, pp]
        L.nabla_mask_workspace_bytes.restype = sz
        L.nabla_build_mask.argtypes = [vp, vp, i, i, i, i, i, i, pp, vp, vp, vp, vp]
        L.nabla_build_mask_noalloc.argtypes = [vp, vp, i, i, i, i, i, i, pp, vp, vp, vp]
        L.nabla_flatten_pool_qk.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, pp, vp, vp]
        L.nabla_build_mask_pooled.argtypes = [vp, i, i, i, i, i, i, pp, vp, vp, vp]
        L.nabla_build_mask_grid.argtypes = [vp, vp, i, i, i, i, i, i, pp, vp, vp, vp, vp]
        L.nabla_build_mask_sta.argtypes = [i, i, i, i, i, i, i, i, i, vp, vp, vp]
        L.nabla_build_mask_radial.argtypes = [i, i, i, i, i, i, i, vp, vp, vp]
        L.nabla_sparse_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, vp, vp, vp]
        L.nabla_sparse_attn_fwd_grid.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, vp, vp]
        L.nabla_sparse_attn_fwd_grid_split.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp, vp]
        L.nabla_attn_split_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        L.nabla_attn_split_workspace_bytes.restype = sz
        L.nabla_transpose_lists.argtypes = [vp, vp, i, i, i, vp, vp, vp]
        L.nabla_sparse_attn_bwd.argtypes = [vp] * 10 + [i, i, i, i, f, vp, vp, vp, vp, vp]
        L.nabla_sparse_attn_bwd_grid.argtypes = [vp] * 10 + [i, i, i, i, i, i, f, vp, vp, vp, vp, vp]
        L.nabla_ab_workspace_bytes.argtypes = [i, i, i, i]
        L.nabla_ab_workspace_bytes.restype = sz
        L.nabla_ab_plan.argtypes = [vp, vp, vp, i, i, i, i, i, ctypes.c_double, f, vp, vp, vp, vp, vp]
        L.nabla_ab_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, f, vp, vp, vp]
        L.nabla_get_status.argtypes = [vp]
        L.nabla_validate_mask.argtypes = [vp, vp, i, i, i, vp, vp]
        L.nabla_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
        L.nabla_strerror.argtypes = [i]
        L.nabla_strerror.restype = ctypes.c_char_p
        for name in EXPORTS:
            if name not in ("nabla_mask_workspace_bytes", "nabla_ab_workspace_bytes", "nabla_attn_split_workspace_bytes",
                            "nabla_strerror"):
                getattr(L, name).restype = i
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().nabla_strerror(int(code)).decode()


def _check(rc: int, where: str):
    if rc != NABLA_OK:
        raise NablaError(rc, where)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def params(thr: float, sta=(0, 0, 0), scale: float = 0.0, P: int = 8, radial: int = 0) -> NablaParams:
    return NablaParams(P, float(thr), int(sta[0]), int(sta[1]), int(sta[2]), float(scale), 0, int(radial))


def _permute(fn, x: torch.Tensor, T: int, H: int, W: int, out, stream, P: int):
    if out is None:
        out = torch.empty_like(x)
    B = x.shape[0]
    row = x[0, 0].numel() if x.dim() > 2 else 1
    _check(fn(_dev(x, torch.bfloat16, "x"), _dev(out, torch.bfloat16, "out"), B, T, H, W, P, row, _stream(stream)),
           "nabla_flatten" if fn is lib().nabla_flatten else "nabla_unflatten")
    return out


def flatten(x: torch.Tensor, T: int, H: int, W: int, out=None, stream=None, P: int = 8) -> torch.Tensor:
    """Fractal flattening of a grid-order [B, S, ...] bf16 CUDA tensor."""
    return _permute(lib().nabla_flatten, x, T, H, W, out, stream, P)


def unflatten(x: torch.Tensor, T: int, H: int, W: int, out=None, stream=None, P: int = 8) -> torch.Tensor:
    """Inverse of :func:`flatten`."""
    return _permute(lib().nabla_unflatten, x, T, H, W, out, stream, P)


def mask_workspace_bytes(B: int, Hh: int, D: int, T: int, H: int, W: int, prm: NablaParams) -> int:
    return int(lib().nabla_mask_workspace_bytes(B, Hh, D, T, H, W, ctypes.byref(prm)))


def build_mask(qf: torch.Tensor, kf: torch.Tensor, T: int, H: int, W: int, thr: float, sta=(0, 0, 0),
               scale: float = 0.0, kv_count=None, kv_idx=None, workspace=None, stream=None, P: int = 8,
               radial: int = 0):
    """Adaptive block mask from flattened Q, K [B, S, Hh, D] (bf16, CUDA).

    Returns (kv_count int32 [B,Hh,Nb], kv_idx int32 [B,Hh,Nb,Nb], workspace
    uint8 holding the pooled qbar^T and kbar^T [B,Hh,D,Nbp] (fp32, see
    :func:`pooled_from_workspace`) and the score scratch).
    """
    B, S, Hh, D = qf.shape
    Nb = S // BLOCK
    prm = params(thr, sta, scale, P, radial)
    dev = qf.device
    if kv_count is None:
        kv_count = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
    if kv_idx is None:
        kv_idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
    if workspace is None:
        nbytes = mask_workspace_bytes(B, Hh, D, T, H, W, prm)
        if nbytes == 0:
            raise NablaError(NABLA_ERR_INVALID, "nabla_mask_workspace_bytes")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib().nabla_build_mask(_dev(qf, torch.bfloat16, "qf"), _dev(kf, torch.bfloat16, "kf"), B, Hh, D, T, H, W,
                                  ctypes.byref(prm), _dev(kv_count, torch.int32, "kv_count"),
                                  _dev(kv_idx, torch.int32, "kv_idx"), _dev(workspace, torch.uint8, "workspace"),
                                  _stream(stream)), "nabla_build_mask")
    return kv_count, kv_idx, workspace


def flatten_pool_qk(q: torch.Tensor, k: torch.Tensor, T: int, H: int, W: int, qf=None, kf=None, workspace=None,
                    thr: float = 0.0, sta=(0, 0, 0), stream=None, P: int = 8, write_flat: bool = True):
    """Flatten Q and K (grid order [B, T*H*W, Hh, D], bf16, CUDA) and pool
    them into a mask workspace in one pass (nabla_flatten_pool_qk); with
    write_flat=False only the pooled vectors are written.
    Returns (qf, kf, workspace) (qf, kf None without write_flat); finish the
    mask with :func:`build_mask_pooled`."""
    B, S, Hh, D = q.shape
    prm = params(thr, sta, 0.0, P)
    if write_flat and qf is None:
        qf = torch.empty_like(q)
    if write_flat and kf is None:
        kf = torch.empty_like(k)
    if workspace is None:
        nbytes = mask_workspace_bytes(B, Hh, D, T, H, W, prm)
        if nbytes == 0:
            raise NablaError(NABLA_ERR_INVALID, "nabla_mask_workspace_bytes")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    qf_p = _dev(qf, torch.bfloat16, "qf") if write_flat else None
    kf_p = _dev(kf, torch.bfloat16, "kf") if write_flat else None
    _check(lib().nabla_flatten_pool_qk(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"), qf_p, kf_p, B, Hh,
                                       D, T, H, W, ctypes.byref(prm), _dev(workspace, torch.uint8, "workspace"),
                                       _stream(stream)), "nabla_flatten_pool_qk")
    return qf, kf, workspace


def build_mask_grid(q: torch.Tensor, k: torch.Tensor, T: int, H: int, W: int, thr: float, sta=(0, 0, 0),
                    scale: float = 0.0, kv_count=None, kv_idx=None, workspace=None, stream=None, P: int = 8,
                    radial: int = 0):
    """:func:`build_mask` on Q, K in grid order [B, T*H*W, Hh, D] (no
    flattened copies; nabla_build_mask_grid).  Returns (kv_count, kv_idx,
    workspace)."""
    B, S, Hh, D = q.shape
    Nb = S // BLOCK
    prm = params(thr, sta, scale, P, radial)
    dev = q.device
    if kv_count is None:
        kv_count = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
    if kv_idx is None:
        kv_idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
    if workspace is None:
        nbytes = mask_workspace_bytes(B, Hh, D, T, H, W, prm)
        if nbytes == 0:
            raise NablaError(NABLA_ERR_INVALID, "nabla_mask_workspace_bytes")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib().nabla_build_mask_grid(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"), B, Hh, D, T, H, W,
                                       ctypes.byref(prm), _dev(kv_count, torch.int32, "kv_count"),
                                       _dev(kv_idx, torch.int32, "kv_idx"), _dev(workspace, torch.uint8, "workspace"),
                                       _stream(stream)), "nabla_build_mask_grid")
    return kv_count, kv_idx, workspace


def build_mask_pooled(workspace: torch.Tensor, B: int, Hh: int, D: int, T: int, H: int, W: int, thr: float,
                      sta=(0, 0, 0), scale: float = 0.0, kv_count=None, kv_idx=None, stream=None, P: int = 8,
                      radial: int = 0):
    """The mask from a workspace that already holds the pooled Q and K
    (nabla_build_mask_pooled).  Returns (kv_count, kv_idx)."""
    Nb = T * H * W // BLOCK
    prm = params(thr, sta, scale, P, radial)
    dev = workspace.device
    if kv_count is None:
        kv_count = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
    if kv_idx is None:
        kv_idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
    _check(lib().nabla_build_mask_pooled(_dev(workspace, torch.uint8, "workspace"), B, Hh, D, T, H, W,
                                         ctypes.byref(prm), _dev(kv_count, torch.int32, "kv_count"),
                                         _dev(kv_idx, torch.int32, "kv_idx"), _stream(stream)),
           "nabla_build_mask_pooled")
    return kv_count, kv_idx


def build_mask_sta(B: int, Hh: int, T: int, H: int, W: int, sta=(3, 3, 3), kv_count=None, kv_idx=None,
                   device=None, stream=None, P: int = 8):
    """The static sliding-tile window alone as block lists (nabla_build_mask_sta;
    reads no Q or K).  Returns (kv_count int32 [B,Hh,Nb], kv_idx int32
    [B,Hh,Nb,Nb])."""
    Nb = T * H * W // BLOCK
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    if kv_count is None:
        kv_count = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
    if kv_idx is None:
        kv_idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
    _check(lib().nabla_build_mask_sta(B, Hh, T, H, W, P, int(sta[0]), int(sta[1]), int(sta[2]),
                                      _dev(kv_count, torch.int32, "kv_count"), _dev(kv_idx, torch.int32, "kv_idx"),
                                      _stream(stream)), "nabla_build_mask_sta")
    return kv_count, kv_idx


def build_mask_radial(B: int, Hh: int, T: int, H: int, W: int, r0: int, kv_count=None, kv_idx=None, device=None,
                      stream=None, P: int = 8):
    """The radial decay window alone as block lists (nabla_build_mask_radial;
    reads no Q or K).  Returns (kv_count int32 [B,Hh,Nb], kv_idx int32
    [B,Hh,Nb,Nb])."""
    Nb = T * H * W // BLOCK
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    if kv_count is None:
        kv_count = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
    if kv_idx is None:
        kv_idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
    _check(lib().nabla_build_mask_radial(B, Hh, T, H, W, P, int(r0), _dev(kv_count, torch.int32, "kv_count"),
                                         _dev(kv_idx, torch.int32, "kv_idx"), _stream(stream)),
           "nabla_build_mask_radial")
    return kv_count, kv_idx


def build_mask_noalloc(qf: torch.Tensor, kf: torch.Tensor, T: int, H: int, W: int, thr: float, sta=(0, 0, 0),
                       scale: float = 0.0, kv_count=None, kv_idx=None, stream=None, P: int = 8, radial: int = 0):
    """The mask of :func:`build_mask` through nabla_build_mask_noalloc: the
    library keeps the pooled vectors in its own static device buffer (16 MiB)
    and allocates nothing (the scores stay in shared memory); calls sharing
    that buffer must not overlap on the GPU.  Returns (kv_count, kv_idx)."""
    B, S, Hh, D = qf.shape
    Nb = S // BLOCK
    prm = params(thr, sta, scale, P, radial)
    dev = qf.device
    if kv_count is None:
        kv_count = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
    if kv_idx is None:
        kv_idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
    _check(lib().nabla_build_mask_noalloc(_dev(qf, torch.bfloat16, "qf"), _dev(kf, torch.bfloat16, "kf"), B, Hh, D,
                                          T, H, W, ctypes.byref(prm), _dev(kv_count, torch.int32, "kv_count"),
                                          _dev(kv_idx, torch.int32, "kv_idx"), _stream(stream)),
           "nabla_build_mask_noalloc")
    return kv_count, kv_idx


def pooled_from_workspace(workspace: torch.Tensor, B: int, Hh: int, Nb: int, D: int):
    """qbar [B,Hh,Nb,D] and kbar [B,Hh,Nb,D] from a mask workspace.  Both are
    stored transposed, [B,Hh,D,Nbp] with Nbp = Nb rounded up to 4; the
    returned tensors are strided views of their first Nb columns."""
    f = workspace.view(torch.float32)
    nbp = (Nb + 3) // 4 * 4
    n = B * Hh * D * nbp
    qt = f[:n].view(B, Hh, D, nbp)
    kt = f[n:2 * n].view(B, Hh, D, nbp)
    return qt[..., :Nb].transpose(2, 3), kt[..., :Nb].transpose(2, 3)


def sparse_attn_fwd(qf: torch.Tensor, kf: torch.Tensor, vf: torch.Tensor, kv_count: torch.Tensor,
                    kv_idx: torch.Tensor, scale: float = 0.0, out=None, lse=None, want_lse: bool = True,
                    stream=None, grid=None, split: int = 1, workspace=None):
    """Block-sparse attention on the kept tiles; returns (out, lse or None).

    grid = None: qf, kf, vf are flattened; nabla_sparse_attn_fwd (pairs 2p,
    2p+1; out and lse in flattened order).
    grid = (T, H, W): the three tensors are in GRID order (token (t, h, w) at
    row (t*H + h)*W + w); nabla_sparse_attn_fwd_grid reads the blocks through
    5-D TMA boxes, pairs query blocks by their lists' overlap and returns out
    and lse in grid order.  split > 1 (grid order only): each head's walk
    split into that many key ranges (nabla_sparse_attn_fwd_grid_split); the
    workspace (uint8 CUDA tensor of at least attn_split_workspace_bytes) is
    allocated when not given."""
    B, S, Hh, D = qf.shape
    if out is None:
        out = torch.empty_like(qf)
    if lse is None and want_lse:
        lse = torch.empty((B, Hh, S), dtype=torch.float32, device=qf.device)
    lse_p = _dev(lse, torch.float32, "lse") if lse is not None else None
    ptrs = (_dev(qf, torch.bfloat16, "qf"), _dev(kf, torch.bfloat16, "kf"), _dev(vf, torch.bfloat16, "vf"),
            _dev(kv_count, torch.int32, "kv_count"), _dev(kv_idx, torch.int32, "kv_idx"))
    o_p = _dev(out, torch.bfloat16, "out")
    if grid is None:
        _check(lib().nabla_sparse_attn_fwd(*ptrs, B, S, Hh, D, float(scale), o_p, lse_p, _stream(stream)),
               "nabla_sparse_attn_fwd")
    else:
        T, H, W = (int(x) for x in grid)
        if T * H * W != S:
            raise ValueError(f"grid {grid} does not hold {S} tokens")
        if split > 1:
            if workspace is None:
                workspace = torch.empty(attn_split_workspace_bytes(B, Hh, D, T, H, W, split), dtype=torch.uint8,
                                        device=qf.device)
            _check(lib().nabla_sparse_attn_fwd_grid_split(*ptrs, B, Hh, D, T, H, W, float(scale), int(split),
                                                          _dev(workspace, torch.uint8, "workspace"), o_p, lse_p,
                                                          _stream(stream)),
                   "nabla_sparse_attn_fwd_grid_split")
        else:
            _check(lib().nabla_sparse_attn_fwd_grid(*ptrs, B, Hh, D, T, H, W, float(scale), o_p, lse_p,
                                                    _stream(stream)),
                   "nabla_sparse_attn_fwd_grid")
    return out, lse


def attn_split_workspace_bytes(B: int, Hh: int, D: int, T: int, H: int, W: int, split: int) -> int:
    n = int(lib().nabla_attn_split_workspace_bytes(B, Hh, D, T, H, W, int(split)))
    if n == 0:
        raise ValueError("invalid arguments for the key-range split")
    return n


def transpose_lists(kv_count: torch.Tensor, kv_idx: torch.Tensor, q_count=None, q_idx=None, stream=None):
    """Column lists of the block lists (nabla_transpose_lists): for every key
    block the query blocks that keep it, ascending.  Returns (q_count,
    q_idx), shaped like (kv_count, kv_idx)."""
    B, Hh, Nb = kv_count.shape
    if q_count is None:
        q_count = torch.empty_like(kv_count)
    if q_idx is None:
        q_idx = torch.empty_like(kv_idx)
    _check(lib().nabla_transpose_lists(_dev(kv_count, torch.int32, "kv_count"), _dev(kv_idx, torch.int32, "kv_idx"),
                                       B, Hh, Nb, _dev(q_count, torch.int32, "q_count"),
                                       _dev(q_idx, torch.int32, "q_idx"), _stream(stream)), "nabla_transpose_lists")
    return q_count, q_idx


def sparse_attn_bwd(qf: torch.Tensor, kf: torch.Tensor, vf: torch.Tensor, out: torch.Tensor, dout: torch.Tensor,
                    lse: torch.Tensor, kv_count: torch.Tensor, kv_idx: torch.Tensor, q_lists=None,
                    scale: float = 0.0, dq=None, dk=None, dv=None, delta=None, stream=None, grid=None):
    """Gradients (dq, dk, dv) of sum(dout * out) for the attention on the kept
    tiles.  q_lists = (q_count, q_idx) from :func:`transpose_lists` (computed
    here when None).  grid = None: flattened tensors (nabla_sparse_attn_bwd);
    grid = (T, H, W): grid-order tensors, LSE and outputs as
    :func:`sparse_attn_fwd` with a grid (nabla_sparse_attn_bwd_grid)."""
    B, S, Hh, D = qf.shape
    if q_lists is None:
        q_lists = transpose_lists(kv_count, kv_idx, stream=stream)
    q_count, q_idx = q_lists
    dq = torch.empty_like(qf) if dq is None else dq
    dk = torch.empty_like(kf) if dk is None else dk
    dv = torch.empty_like(vf) if dv is None else dv
    if delta is None:
        delta = torch.empty((B, Hh, S), dtype=torch.float32, device=qf.device)
    ptrs = [_dev(x, torch.bfloat16, n) for x, n in ((qf, "q"), (kf, "k"), (vf, "v"), (out, "out"), (dout, "dout"))]
    ptrs += [_dev(lse, torch.float32, "lse"), _dev(kv_count, torch.int32, "kv_count"), _dev(kv_idx, torch.int32, "kv_idx"),
             _dev(q_count, torch.int32, "q_count"), _dev(q_idx, torch.int32, "q_idx")]
    outs = [_dev(dq, torch.bfloat16, "dq"), _dev(dk, torch.bfloat16, "dk"), _dev(dv, torch.bfloat16, "dv"),
            _dev(delta, torch.float32, "delta"), _stream(stream)]
    if grid is None:
        _check(lib().nabla_sparse_attn_bwd(*ptrs, B, S, Hh, D, float(scale), *outs), "nabla_sparse_attn_bwd")
    else:
        T, H, W = (int(x) for x in grid)
        if T * H * W != S:
            raise ValueError(f"grid {grid} does not hold {S} tokens")
        _check(lib().nabla_sparse_attn_bwd_grid(*ptrs, B, Hh, D, T, H, W, float(scale), *outs),
               "nabla_sparse_attn_bwd_grid")
    return dq, dk, dv


# ---------------------------------------------------------------- AB-Attention
AB_QBLOCK = 128
AB_KBLOCK = 4
AB_CLUSTERS = 8


def ab_workspace_bytes(B: int, S: int, Hh: int, D: int) -> int:
    return int(lib().nabla_ab_workspace_bytes(B, S, Hh, D))


def ab_plan(q: torch.Tensor, k: torch.Tensor, u: torch.Tensor, budget: float, kmeans_iters: int = 4,
            scale: float = 0.0, kcount=None, kidx=None, kshift=None, workspace=None, stream=None):
    """The AB-Attention sampling plan (nabla_ab_plan) for Q, K [B, S, Hh, D]
    in grid order and uniforms u fp32 [B, Hh, S/128, S/4].  Returns (kcount
    int32 [B,Hh,NQB], kidx int32 [B,Hh,NQB,NKB], kshift fp32 [B,Hh,NQB,NKB],
    workspace; see :func:`ab_views`)."""
    B, S, Hh, D = q.shape
    nqb, nkb = S // AB_QBLOCK, S // AB_KBLOCK
    dev = q.device
    kcount = torch.empty((B, Hh, nqb), dtype=torch.int32, device=dev) if kcount is None else kcount
    kidx = torch.empty((B, Hh, nqb, nkb), dtype=torch.int32, device=dev) if kidx is None else kidx
    kshift = torch.empty((B, Hh, nqb, nkb), dtype=torch.float32, device=dev) if kshift is None else kshift
    if workspace is None:
        nbytes = ab_workspace_bytes(B, S, Hh, D)
        if nbytes == 0:
            raise NablaError(NABLA_ERR_INVALID, "nabla_ab_workspace_bytes")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(lib().nabla_ab_plan(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"), _dev(u, torch.float32, "u"),
                               B, S, Hh, D, int(kmeans_iters), float(budget), float(scale),
                               _dev(kcount, torch.int32, "kcount"), _dev(kidx, torch.int32, "kidx"),
                               _dev(kshift, torch.float32, "kshift"), _dev(workspace, torch.uint8, "workspace"),
                               _stream(stream)), "nabla_ab_plan")
    return kcount, kidx, kshift, workspace


def ab_views(workspace: torch.Tensor, B: int, S: int, Hh: int, D: int):
    """Views into an AB plan workspace: (kbar [B,Hh,NKB,D], cent [B,Hh,NQB,8,D]
    (both strided views of the transposed storage), counts int32
    [B,Hh,NQB,8], logits fp32 [B,Hh,NQB*8,NKB])."""
    up = lambda x: (x + 255) // 256 * 256  # noqa: E731
    nkb, nqb = S // AB_KBLOCK, S // AB_QBLOCK
    R = nqb * AB_CLUSTERS
    bh = B * Hh
    o_cent = up(bh * D * nkb * 4)
    o_counts = o_cent + up(bh * D * R * 4)
    o_logits = o_counts + up(bh * nqb * AB_CLUSTERS * 4)
    kt = workspace[:bh * D * nkb * 4].view(torch.float32).view(B, Hh, D, nkb)
    ct = workspace[o_cent:o_cent + bh * D * R * 4].view(torch.float32).view(B, Hh, D, nqb, AB_CLUSTERS)
    counts = workspace[o_counts:o_counts + bh * nqb * AB_CLUSTERS * 4].view(torch.int32).view(B, Hh, nqb, AB_CLUSTERS)
    logits = workspace[o_logits:o_logits + bh * R * nkb * 4].view(torch.float32).view(B, Hh, R, nkb)
    return kt.transpose(2, 3), ct.permute(0, 1, 3, 4, 2), counts, logits


def ab_attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, kcount: torch.Tensor, kidx: torch.Tensor,
                kshift: torch.Tensor, scale: float = 0.0, out=None, lse=None, want_lse: bool = True, stream=None):
    """AB-Attention forward on the sampled 4-token key blocks with their
    logit shifts (nabla_ab_attn_fwd); grid-order tensors in and out.
    Returns (out, lse or None)."""
    B, S, Hh, D = q.shape
    out = torch.empty_like(q) if out is None else out
    if lse is None and want_lse:
        lse = torch.empty((B, Hh, S), dtype=torch.float32, device=q.device)
    lse_p = _dev(lse, torch.float32, "lse") if lse is not None else None
    _check(lib().nabla_ab_attn_fwd(_dev(q, torch.bfloat16, "q"), _dev(k, torch.bfloat16, "k"),
                                   _dev(v, torch.bfloat16, "v"), _dev(kcount, torch.int32, "kcount"),
                                   _dev(kidx, torch.int32, "kidx"), _dev(kshift, torch.float32, "kshift"), B, S, Hh,
                                   D, float(scale), _dev(out, torch.bfloat16, "out"), lse_p, _stream(stream)),
           "nabla_ab_attn_fwd")
    return out, lse


def get_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device status word."""
    return int(lib().nabla_get_status(_stream(stream)))


def validate_mask(kv_count: torch.Tensor, kv_idx: torch.Tensor, stream=None) -> int:
    """Number of malformed block-list rows (synchronises)."""
    B, Hh, Nb = kv_count.shape
    bad = torch.zeros(1, dtype=torch.int32, device=kv_count.device)
    _check(lib().nabla_validate_mask(_dev(kv_count, torch.int32, "kv_count"), _dev(kv_idx, torch.int32, "kv_idx"),
                                     B, Hh, Nb, _dev(bad, torch.int32, "bad_rows"), _stream(stream)),
           "nabla_validate_mask")
    return int(bad.item())


def selftest_wait_timeout(limit_cycles: int = 2_000_000, stream=None) -> int:
    """Run the bounded-wait self-test and return the status it leaves
    (synchronises; NABLA_ERR_DEVICE_TIMEOUT when the wait gave up)."""
    _check(lib().nabla_selftest_wait_timeout(int(limit_cycles), _stream(stream)), "nabla_selftest_wait_timeout")
    return get_status(stream)


def default_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
