"""AB-Attention on the GPU against the oracle (news page "AB-Attention
acelera a geracao de video em ate 2,23x e pula 92% da atencao", section
"Os tres recursos do AB-Attention").

* key-block means, cluster centroids and counts: bit-exact (the same fp32
  operations in the same order);
* the sampling decisions (u < pi): equal to the oracle's except where
  |u - pi| < 1e-5 (the GPU's pi uses expf and its own summation order; such
  blocks are counted), shifts within 1e-5 of -log(pi);
* attention on the GPU's sample, against the oracle's fp64 attention on the
  same blocks with its own shifts: max-abs 2e-2, mean-abs 2e-3, LSE 2e-3;
* edge cases: a budget above the number of key blocks (every block with
  pi = 1, i.e. dense attention), a tiny budget (mostly one or two blocks),
  D = 64, batch 2, a list entry out of range (skipped and reported).
"""

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_flatten_b200 import inputs
from block_sparse_attention_flatten_b200 import nabla

pytestmark = pytest.mark.gpu

BAND = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    from block_sparse_attention_flatten_b200 import build
    build.build()
    assert torch.cuda.is_available()
    oracle.build()


def run(w: inputs.ABWorkload, budget=None, qblocks=None):
    base = w.base
    q, k, v = inputs.make_qkv(base)
    u = inputs.ab_uniforms(w)
    budget = w.budget if budget is None else budget
    qd, kd, vd, ud = q.cuda(), k.cuda(), v.cuda(), u.cuda()
    kcount, kidx, kshift, ws = nabla.ab_plan(qd, kd, ud, budget, w.kmeans_iters)
    out, lse = nabla.ab_attn_fwd(qd, kd, vd, kcount, kidx, kshift)
    torch.cuda.synchronize()
    assert nabla.get_status() == 0
    # plan stages against the oracle
    kbar_g, cent_g, counts_g, _ = nabla.ab_views(ws, base.B, base.S, base.Hh, base.D)
    kbar_o = oracle.ab_key_means(k)
    cent_o, counts_o, _ = oracle.ab_kmeans(q, iters=w.kmeans_iters)
    assert np.array_equal(kbar_g.cpu().numpy(), kbar_o)
    assert np.array_equal(counts_g.cpu().numpy(), counts_o)
    assert np.array_equal(cent_g.cpu().numpy(), cent_o)
    score = oracle.ab_scores(cent_o, counts_o, kbar_o, base.scale)
    pi = oracle.ab_inclusion(score, budget)
    un = u.numpy().astype(np.float64)
    inc_o = un < pi
    cnt_g, idx_g, sh_g = kcount.cpu().numpy(), kidx.cpu().numpy(), kshift.cpu().numpy()
    inc_g = np.zeros_like(inc_o)
    nkb = w.nkb
    for b in range(base.B):
        for h in range(base.Hh):
            for I in range(w.nqb):
                c = cnt_g[b, h, I]
                js = idx_g[b, h, I, :c]
                assert np.all(np.diff(js) > 0) and (c == 0 or (js[0] >= 0 and js[-1] < nkb))
                inc_g[b, h, I, js] = True
                np.testing.assert_allclose(sh_g[b, h, I, :c], -np.log(pi[b, h, I, js]), atol=1e-5)
    band = np.abs(un - pi) < BAND
    bad = int(np.sum((inc_g != inc_o) & ~band))
    in_band = int(np.sum((inc_g != inc_o) & band))
    # attention on the GPU's sample with the oracle's shifts for those blocks
    if qblocks is None:
        qblocks = inputs.sample_query_blocks(w.nqb, min(w.nqb, 16), seed=1234)
    shift_o = np.zeros_like(sh_g, dtype=np.float64)
    for b in range(base.B):
        for h in range(base.Hh):
            for I in qblocks:
                c = cnt_g[b, h, I]
                shift_o[b, h, I, :c] = -np.log(pi[b, h, I, idx_g[b, h, I, :c]])
    ref, ref_lse = oracle.ab_attention(q, k, v, cnt_g, idx_g, shift_o, base.scale, qblocks=qblocks)
    rows = np.concatenate([np.arange(I * 128, (I + 1) * 128) for I in qblocks])
    got = out[:, torch.as_tensor(rows, device="cuda")].double().cpu().numpy()
    got_lse = lse[:, :, torch.as_tensor(rows, device="cuda")].double().cpu().numpy()
    err = np.abs(got - ref)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(fin, np.isfinite(got_lse))
    lse_err = float(np.abs(got_lse[fin] - ref_lse[fin]).max()) if fin.any() else 0.0
    frac = float(cnt_g.mean()) / nkb
    print(f"\n{w.name}: sampled fraction {frac:.4f} (budget {budget / nkb:.4f}), decisions outside band "
          f"{bad}, inside {in_band}; attention max {err.max():.2e} mean {err.mean():.2e} lse {lse_err:.2e}")
    return bad, float(err.max()), float(err.mean()), lse_err, cnt_g


CASES = [
    inputs.AB_TINY,
    inputs.ABWorkload("AB D128 B2 4x16x32", inputs.Workload("ab-b2", 2, 3, 128, 4, 16, 32, 1.0, 1.0, seed=62), 0.2),
    inputs.ABWorkload("AB D64 odd Nq 3x16x16 (6 query blocks)", inputs.Workload("ab-d64", 1, 2, 64, 3, 16, 16, 0.5,
                                                                                  1.0, seed=63), 0.05),
    inputs.ABWorkload("AB 4 Lloyd iterations -> 1", inputs.Workload("ab-it1", 1, 2, 128, 4, 16, 32, 1.0, 1.0, seed=64),
                      0.1, kmeans_iters=1),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_ab_plan_and_attention(w):
    bad, mx, mean, lse_err, _ = run(w)
    assert bad == 0
    assert mx <= 2e-2 and mean <= 2e-3 and lse_err <= 2e-3


def test_ab_budget_above_block_count_is_dense_attention():
    w = inputs.ABWorkload("AB dense", inputs.Workload("ab-dense", 1, 2, 64, 2, 16, 16, 1.0, 1.0, seed=65), 1.0)
    bad, mx, mean, lse_err, cnt = run(w, budget=w.nkb * 2.0)
    assert bad == 0 and np.all(cnt == w.nkb)
    assert mx <= 2e-2 and mean <= 2e-3 and lse_err <= 2e-3


def test_ab_tiny_budget():
    w = inputs.ABWorkload("AB budget 1", inputs.Workload("ab-b1", 1, 2, 128, 2, 16, 32, 1.0, 1.0, seed=66), 0.0)
    bad, mx, mean, lse_err, cnt = run(w, budget=1.0)
    assert bad == 0
    assert mx <= 2e-2 and mean <= 2e-3 and lse_err <= 2e-3


@pytest.mark.slow
def test_ab_wan_layer():
    w = inputs.AB_WAN13B
    bad, mx, mean, lse_err, cnt = run(w, qblocks=inputs.sample_query_blocks(w.nqb, 8, seed=1234))
    assert bad == 0
    assert mx <= 2e-2 and mean <= 2e-3 and lse_err <= 2e-3


def test_ab_out_of_range_entry_is_skipped_and_reported():
    w = inputs.AB_TINY
    base = w.base
    q, k, v = (x.cuda() for x in inputs.make_qkv(base))
    kcount = torch.full((base.B, base.Hh, w.nqb), 3, dtype=torch.int32, device="cuda")
    kidx = torch.zeros((base.B, base.Hh, w.nqb, w.nkb), dtype=torch.int32, device="cuda")
    kidx[..., 1] = 5
    kidx[..., 2] = w.nkb + 7  # out of range
    kshift = torch.zeros((base.B, base.Hh, w.nqb, w.nkb), dtype=torch.float32, device="cuda")
    out, lse = nabla.ab_attn_fwd(q, k, v, kcount, kidx, kshift)
    assert nabla.get_status() == nabla.NABLA_ERR_DEVICE_BOUNDS
    assert nabla.get_status() == 0
    # the valid blocks 0 and 5 are attended as if the bad entry were absent
    kcount2 = torch.full_like(kcount, 2)
    out2, _ = nabla.ab_attn_fwd(q, k, v, kcount2, kidx, kshift)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)
