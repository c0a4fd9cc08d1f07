"""The layer's calls captured in one CUDA graph and replayed.

A serving loop or a training step that replays a CUDA graph per layer needs
every call it captures to allocate nothing, never synchronise and launch only
on the caller's stream.  The entry points are written that way.  Captured
here once on static buffers: the grid-order hot path (pooling, mask on the
pooled workspace, attention with one key range and with two plus their
merge, column lists, backward), and in a second graph the other paths (the
materialised flattening, the mask and attention on flattened tensors, the
unflattening and the flattened backward, the one-call grid-order mask, the
static sliding-tile and radial windows, the AB-Attention plan and
attention).  Every replay on new inputs must give the same bits as the same
calls run eagerly on those inputs (the kernels are deterministic: no
atomics, fixed summation orders).  nabla_get_status synchronises and stays
outside the graphs."""
import numpy as np
import pytest
import torch

from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    yield
    torch.cuda.synchronize()


class _Layer:
    """Static device buffers of one layer and the calls of one step on them."""

    def __init__(self, B, Hh, D, grid, thr, sta, split):
        T, H, W = grid
        self.B, self.Hh, self.D, self.grid, self.thr, self.sta, self.split = B, Hh, D, grid, thr, sta, split
        S, Nb = T * H * W, T * H * W // 64
        dev = torch.device("cuda")
        self.q, self.k, self.v, self.do = (torch.empty((B, S, Hh, D), dtype=torch.bfloat16, device=dev)
                                           for _ in range(4))
        prm = nabla.params(thr, sta)
        self.ws = torch.empty(nabla.mask_workspace_bytes(B, Hh, D, T, H, W, prm), dtype=torch.uint8, device=dev)
        self.split_ws = (torch.empty(nabla.attn_split_workspace_bytes(B, Hh, D, T, H, W, split), dtype=torch.uint8,
                                     device=dev) if split > 1 else None)
        self.cnt = torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev)
        self.idx = torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)
        self.qc, self.qi = torch.empty_like(self.cnt), torch.empty_like(self.idx)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty((B, Hh, S), dtype=torch.float32, device=dev)
        self.delta = torch.empty_like(self.lse)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)

    def load(self, tensors):
        for dst, src in zip((self.q, self.k, self.v, self.do), tensors):
            dst.copy_(src)

    def step(self):
        B, Hh, D, (T, H, W) = self.B, self.Hh, self.D, self.grid
        nabla.flatten_pool_qk(self.q, self.k, T, H, W, workspace=self.ws, thr=self.thr, sta=self.sta,
                              write_flat=False)
        nabla.build_mask_pooled(self.ws, B, Hh, D, T, H, W, self.thr, self.sta, kv_count=self.cnt, kv_idx=self.idx)
        nabla.sparse_attn_fwd(self.q, self.k, self.v, self.cnt, self.idx, out=self.o, lse=self.lse, grid=self.grid,
                              split=self.split, workspace=self.split_ws)
        nabla.transpose_lists(self.cnt, self.idx, q_count=self.qc, q_idx=self.qi)
        nabla.sparse_attn_bwd(self.q, self.k, self.v, self.o, self.do, self.lse, self.cnt, self.idx,
                              q_lists=(self.qc, self.qi), dq=self.dq, dk=self.dk, dv=self.dv, delta=self.delta,
                              grid=self.grid)

    def results(self):
        """Host copies of every output; list entries past a row's count are
        never written, so they are cleared here before comparing."""
        cnt, idx = self.cnt.cpu().numpy(), self.idx.cpu().numpy().copy()
        qc, qi = self.qc.cpu().numpy(), self.qi.cpu().numpy().copy()
        Nb = cnt.shape[-1]
        idx[np.arange(Nb)[None, None, None, :] >= cnt[..., None]] = -1
        qi[np.arange(Nb)[None, None, None, :] >= qc[..., None]] = -1
        out = {"kv_count": cnt, "kv_idx": idx, "q_count": qc, "q_idx": qi}
        for name in ("o", "lse", "dq", "dk", "dv"):
            t = getattr(self, name)
            out[name] = (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).cpu().numpy()
        return out


def _inputs(B, Hh, D, grid, seed):
    S = grid[0] * grid[1] * grid[2]
    g = torch.Generator().manual_seed(seed)
    # Q and K with a shared component, so the masks keep a mix of blocks
    base = torch.randn(B, S, Hh, D, generator=g)
    q = (torch.randn(B, S, Hh, D, generator=g) + base).to(torch.bfloat16)
    k = (torch.randn(B, S, Hh, D, generator=g) + base).to(torch.bfloat16)
    v, do = (torch.randn(B, S, Hh, D, generator=g).to(torch.bfloat16) for _ in range(2))
    return [x.cuda() for x in (q, k, v, do)]


def _same(a, b, what):
    for key in a:
        assert np.array_equal(a[key], b[key]), f"{what}: {key} differs"


@pytest.mark.parametrize("B,Hh,D,grid,thr,sta,split", [
    (1, 2, 128, (4, 32, 64), 0.9, (3, 3, 3), 2),   # 128 blocks, two key ranges and their merge
    (1, 2, 128, (4, 32, 64), 0.7, (0, 0, 0), 1),
    (2, 3, 64, (2, 16, 32), 0.9, (3, 3, 3), 1),    # batch 2, D = 64, odd head count
])
def test_graph_replay_equals_eager(B, Hh, D, grid, thr, sta, split):
    layer = _Layer(B, Hh, D, grid, thr, sta, split)
    sets = [_inputs(B, Hh, D, grid, seed) for seed in (301, 302)]
    eager = []
    for tensors in sets:
        layer.load(tensors)
        layer.step()
        torch.cuda.synchronize()
        assert nabla.get_status() == 0
        eager.append(layer.results())
    # the two input sets give different masks and outputs, so a replay that
    # reused the captured inputs' results would fail the comparison
    assert not np.array_equal(eager[0]["o"], eager[1]["o"])

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        layer.step()
    torch.cuda.synchronize()
    for rep in range(2):
        for s in (1, 0):
            layer.load(sets[s])
            graph.replay()
            torch.cuda.synchronize()
            assert nabla.get_status() == 0
            _same(layer.results(), eager[s], f"replay {rep} on input set {s}")
    del graph


def _masked(cnt, idx):
    """Host copies of block lists with the entries past each count cleared."""
    c, x = cnt.cpu().numpy(), idx.cpu().numpy().copy()
    x[np.arange(x.shape[-1])[None, None, None, :] >= c[..., None]] = -1
    return c, x


def _bits(t):
    return (t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)).cpu().numpy()


def test_graph_replay_other_paths():
    B, Hh, D, grid, thr, sta, r0 = 1, 2, 128, (4, 32, 64), 0.9, (3, 3, 3), 2
    T, H, W = grid
    S, Nb = T * H * W, T * H * W // 64
    ab = inputs.ABWorkload("graph AB", inputs.Workload("graph-ab", B, Hh, D, T, H, W, 1.0, 1.0, seed=71), 0.1)
    dev = torch.device("cuda")
    q, k, v, do = (torch.empty((B, S, Hh, D), dtype=torch.bfloat16, device=dev) for _ in range(4))
    u = torch.empty((B, Hh, ab.nqb, ab.nkb), dtype=torch.float32, device=dev)
    qf, kf, vf, of, og, dq, dk, dv = (torch.empty_like(q) for _ in range(8))
    lse, delta = (torch.empty((B, Hh, S), dtype=torch.float32, device=dev) for _ in range(2))
    ws = torch.empty(nabla.mask_workspace_bytes(B, Hh, D, T, H, W, nabla.params(thr, sta)), dtype=torch.uint8,
                     device=dev)
    lists = {n: (torch.empty((B, Hh, Nb), dtype=torch.int32, device=dev),
                 torch.empty((B, Hh, Nb, Nb), dtype=torch.int32, device=dev)) for n in ("flat", "grid", "sta", "rad", "t")}
    ab_ws = torch.empty(nabla.ab_workspace_bytes(B, S, Hh, D), dtype=torch.uint8, device=dev)
    kcount = torch.empty((B, Hh, ab.nqb), dtype=torch.int32, device=dev)
    kidx = torch.empty((B, Hh, ab.nqb, ab.nkb), dtype=torch.int32, device=dev)
    kshift = torch.empty((B, Hh, ab.nqb, ab.nkb), dtype=torch.float32, device=dev)
    oab, lse_ab = torch.empty_like(q), torch.empty((B, Hh, S), dtype=torch.float32, device=dev)

    def step():
        for src, dst in ((q, qf), (k, kf), (v, vf)):
            nabla.flatten(src, T, H, W, out=dst)
        cf, xf = lists["flat"]
        nabla.build_mask(qf, kf, T, H, W, thr, sta, kv_count=cf, kv_idx=xf, workspace=ws)
        nabla.sparse_attn_fwd(qf, kf, vf, cf, xf, out=of, lse=lse)
        nabla.unflatten(of, T, H, W, out=og)
        ct, xt = lists["t"]
        nabla.transpose_lists(cf, xf, q_count=ct, q_idx=xt)
        nabla.sparse_attn_bwd(qf, kf, vf, of, do, lse, cf, xf, q_lists=(ct, xt), dq=dq, dk=dk, dv=dv, delta=delta)
        cg, xg = lists["grid"]
        nabla.build_mask_grid(q, k, T, H, W, thr, sta, kv_count=cg, kv_idx=xg, workspace=ws)
        nabla.build_mask_sta(B, Hh, T, H, W, sta, kv_count=lists["sta"][0], kv_idx=lists["sta"][1])
        nabla.build_mask_radial(B, Hh, T, H, W, r0, kv_count=lists["rad"][0], kv_idx=lists["rad"][1])
        nabla.ab_plan(q, k, u, ab.budget, ab.kmeans_iters, kcount=kcount, kidx=kidx, kshift=kshift, workspace=ab_ws)
        nabla.ab_attn_fwd(q, k, v, kcount, kidx, kshift, out=oab, lse=lse_ab)

    def results():
        out = {}
        for n, (c, x) in lists.items():
            out[n + "_count"], out[n + "_idx"] = _masked(c, x)
        kc, ki = _masked(kcount, kidx)
        ks = kshift.cpu().numpy().copy()
        ks[np.arange(ab.nkb)[None, None, None, :] >= kc[..., None]] = 0.0
        out.update(kcount=kc, kidx=ki, kshift=ks.view(np.int32))
        for name, t in (("of", of), ("og", og), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv), ("oab", oab),
                        ("lse_ab", lse_ab)):
            out[name] = _bits(t)
        return out

    sets = []
    for seed in (401, 402):
        tensors = _inputs(B, Hh, D, grid, seed)
        g = torch.Generator().manual_seed(seed + 50)
        tensors.append(torch.rand((B, Hh, ab.nqb, ab.nkb), generator=g).cuda())
        sets.append(tensors)

    def load(tensors):
        for dst, src in zip((q, k, v, do, u), tensors):
            dst.copy_(src)

    eager = []
    for tensors in sets:
        load(tensors)
        step()
        torch.cuda.synchronize()
        assert nabla.get_status() == 0
        eager.append(results())
    assert not np.array_equal(eager[0]["oab"], eager[1]["oab"])
    assert not np.array_equal(eager[0]["of"], eager[1]["of"])

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    torch.cuda.synchronize()
    for rep in range(2):
        for s in (1, 0):
            load(sets[s])
            graph.replay()
            torch.cuda.synchronize()
            assert nabla.get_status() == 0
            _same(results(), eager[s], f"replay {rep} on input set {s}")
    del graph
