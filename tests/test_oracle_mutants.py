"""Planted mistakes in the CPU oracle must be caught by its pins.

Each case copies oracle.c, plants one plausible mistake by a text edit (a
transposed index, a wrong divisor, a dropped term, a flipped sign or
comparison, a reversed tie order), builds the copy into a temporary library
and runs the pins that should notice against it: at least one of them must
fail.  The oracle's own source is never modified.  A control run of the
same pins on an unmodified copy must pass, so a failure is the mistake's.
"""
import importlib.util
import os

import numpy as np
import pytest

import test_oracle as pins
import test_oracle_ab as ab_pins
from block_sparse_attention_flatten_b200 import inputs

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")


def tiny_flat(mod):
    w = inputs.TINY
    q, k, v = inputs.make_qkv(w)
    qf = mod.flatten(q, w.T, w.H, w.W).reshape(q.shape)
    kf = mod.flatten(k, w.T, w.H, w.W).reshape(k.shape)
    vf = mod.flatten(v, w.T, w.H, w.W).reshape(v.shape)
    return w, (q, k, v), (qf, kf, vf)


def ab_tiny(mod):
    w = inputs.AB_TINY
    q, k, v = inputs.make_qkv(w.base)
    return w, q, k, v


# pin name -> call with an oracle module
PINS = {
    "flatten_reshape": lambda m: [pins.test_flatten_matches_reshape_formulation(m, *a)
                                  for a in [(4, 16, 16, 8), (3, 8, 24, 8), (5, 16, 8, 24)]],
    "flatten_first_patch": lambda m: pins.test_flatten_first_patch_listing(m),
    "pool_mean": lambda m: pins.test_pool_is_block_mean(m, tiny_flat(m)),
    "block_probs": lambda m: pins.test_block_probs_is_softmax_of_scaled_tile_means(m, tiny_flat(m)),
    "uniform_golden": lambda m: [pins.test_uniform_worked_case(m, thr, kept) for thr, kept in pins.read_uniform_cases()],
    "top_p": lambda m: [pins.test_cdf_rule_equals_exact_top_p(m, thr) for thr in (0.5, 0.9)],
    "thr_extremes": lambda m: pins.test_thr_one_keeps_all_and_thr_zero_keeps_argmax(m, tiny_flat(m)),
    "sta_counts": lambda m: [pins.test_sta_closed_form_counts(m, *r) for r in pins.read_sta_counts()],
    "sta_lists": lambda m: (pins.test_sta_lists_degenerate_windows(m),
                            [pins.test_sta_lists_other_windows(m, wnd) for wnd in [(1, 3, 5), (7, 7, 7)]]),
    "radial_lists": lambda m: [pins.test_radial_lists_equal_enumeration_and_closed_form(m, *g)
                               for g in pins.RADIAL_GRIDS[:3]],
    "radial_union": lambda m: pins.test_radial_union_is_superset(m),
    "ab_key_means": lambda m: ab_pins.test_key_means_are_block_means(m, ab_tiny(m)),
    "ab_kmeans": lambda m: (ab_pins.test_kmeans_recovers_separated_clusters(m),
                            ab_pins.test_kmeans_centroids_assignment_and_descent(m, ab_tiny(m))),
    "ab_scores": lambda m: ab_pins.test_scores_restated_in_fp64(m, ab_tiny(m)),
    "ab_inclusion": lambda m: [ab_pins.test_inclusion_probabilities(m, *a)
                               for a in [(1, 40, 4.0), (2, 64, 10.0), (5, 50, 1.0)]],
    "ab_unbiased": lambda m: ab_pins.test_horvitz_thompson_unbiased_by_enumeration(m),
    "ab_dense": lambda m: ab_pins.test_full_sample_equals_dense_attention(m, ab_tiny(m)),
    "dense_attention": lambda m: pins.test_thr_one_equals_dense_attention(m, tiny_flat(m)),
    "attention_special": lambda m: pins.test_attention_special_cases(m),
    "bwd_autograd": lambda m: [pins.test_attention_bwd_equals_autograd(m, *a) for a in [(64, 0.5, ()), (128, 0.3, (2,))]],
    "bwd_invariants": lambda m: pins.test_attention_bwd_invariants(m),
    "bwd_sampled": lambda m: pins.test_attention_bwd_sampled_equals_autograd_on_listed_blocks(m),
}

# (name, text in oracle.c, planted replacement, pins expected to catch it)
MUTANTS = [
    ("within-patch index transposed", "(h % P) * P + (w % P)", "(w % P) * P + (h % P)",
     ["flatten_reshape", "flatten_first_patch"]),
    ("patches in column-major order", "(int64_t)(bh * nbw + bw) * P * P", "(int64_t)(bw * (H / P) + bh) * P * P",
     ["flatten_reshape"]),
    ("pooling divides by 63", "acc * (1.0f / 64.0f)", "acc * (1.0f / 63.0f)", ["pool_mean"]),
    ("score scale dropped", "float s = dot * scale;", "float s = dot;", ["block_probs"]),
    ("softmax not normalised", "p[j] = (float)((double)p[j] / Z);", "p[j] = (float)((double)p[j]);",
     ["block_probs"]),
    ("CDF keeps c >= 1 - thr", "(c > tau)", "(c >= tau)", ["uniform_golden"]),
    ("tie order reversed", "return (x->j > y->j) - (x->j < y->j);", "return (x->j < y->j) - (x->j > y->j);",
     ["uniform_golden"]),
    ("CDF accumulates descending", "run += (double)scratch[k].w;", "run += (double)scratch[Nb - 1 - k].w;",
     ["uniform_golden", "top_p"]),
    ("CDF not normalised", "double c = run / Z;", "double c = run;", ["uniform_golden", "top_p"]),
    ("CDF orders blocks by index only", "if (x->w < y->w) return -1;\n  if (x->w > y->w) return 1;\n", "",
     ["top_p", "uniform_golden"]),
    ("arg-max not forced", " || (k == Nb - 1));", ");", ["thr_extremes"]),
    ("STA window exclusive", "abs(ti - tj) <= st / 2", "abs(ti - tj) < st / 2", ["sta_counts"]),
    ("STA lists skip the query block",
     "if (sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w)) kv_idx",
     "if (j != i && sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w)) kv_idx", ["sta_lists"]),
    ("radial bands one frame late", "while ((dt + 1) >> (r + 1)) ++r;", "while (dt >> (r + 1)) ++r;",
     ["radial_lists"]),
    ("radial window never shrinks", "int rho = r0 >> radial_band(abs(ti - tj));", "int rho = r0;", ["radial_lists"]),
    ("radial window left out of the union",
     "sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w) || radial_keep(i, j, nbh, nbw, radial_r0);",
     "sta_keep(i, j, nbh, nbw, sta_t, sta_h, sta_w);", ["radial_union"]),
    ("AB key means over 3 tokens", "kbar[(((int64_t)b * Hh + hd) * nkb + J) * D + d] = acc * 0.25f;",
     "kbar[(((int64_t)b * Hh + hd) * nkb + J) * D + d] = acc * (1.0f / 3.0f);", ["ab_key_means"]),
    ("AB centroid divides by count + 1", "mu[c * D + d] = acc[d] / (float)n;", "mu[c * D + d] = acc[d] / (float)(n + 1);",
     ["ab_kmeans"]),
    ("AB clusters weighted equally", "double w = (double)n / (double)AB_QBLOCK;", "double w = 1.0 / AB_CLUSTERS;",
     ["ab_scores"]),
    ("AB inclusion never capped", "if (lambda * v[m].s < 1.0) break;", "break;", ["ab_inclusion"]),
    ("AB Horvitz-Thompson shift sign flipped", "logit[n] = dot * scale + sh[e];", "logit[n] = dot * scale - sh[e];",
     ["ab_unbiased"]),
    ("AB attention scale dropped", "logit[n] = dot * scale + sh[e];", "logit[n] = dot + sh[e];", ["ab_dense"]),
    ("attention scale dropped", "double l = dot * scale;", "double l = dot;", ["dense_attention"]),
    ("attention normaliser dropped", "o[d] = cnt > 0 ? acc[d] / den : 0.0;", "o[d] = cnt > 0 ? acc[d] : 0.0;",
     ["attention_special", "dense_attention"]),
    ("gradient: softmax Jacobian sign", "double ds = pr[n] * (dp[n] - pdp);", "double ds = pr[n] * (dp[n] + pdp);",
     ["bwd_autograd", "bwd_invariants"]),
    ("gradient: dK without the scale", "dkc[d] += scale * ds *", "dkc[d] += ds *", ["bwd_autograd"]),
    ("gradient: dV from dS instead of P", "dvc[d] += pr[n] *", "dvc[d] += ds *", ["bwd_autograd", "bwd_invariants"]),
    ("gradient: dQ from q instead of k",
     "dqa[d] += scale * ds * (double)bf16_bits_to_f32(k[d]);",
     "dqa[d] += scale * ds * (double)bf16_bits_to_f32(q[d]);", ["bwd_autograd"]),
    ("sampled gradient: row term over the sampled block only", "              pdp += pr[n] * dot;\n              ++n;\n            }\n          double* dqa = qpos",
     "              if (kpos[lst[e]] >= 0) pdp += pr[n] * dot;\n              ++n;\n            }\n          double* dqa = qpos",
     ["bwd_sampled"]),
    ("sampled gradient: dK, dV rows limited to sampled query blocks", "int needed = qpos[i] >= 0;\n        for (int e = 0; e < cnt && !needed; ++e) needed = kpos[lst[e]] >= 0;",
     "int needed = qpos[i] >= 0;", ["bwd_sampled"]),
]


def build_variant(tmp_path, tag, old=None, new=None):
    with open(os.path.join(ORACLE_DIR, "oracle.c")) as fh:
        src = fh.read()
    if old is not None:
        # every occurrence is planted (the gradient's formulas appear in both
        # the full and the sampled function)
        assert src.count(old) >= 1, f"mutation target missing: {old!r}"
        src = src.replace(old, new)
    d = tmp_path / tag
    d.mkdir()
    (d / "oracle.c").write_text(src)
    spec = importlib.util.spec_from_file_location(f"oracle_variant_{tag}", os.path.join(ORACLE_DIR, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(d / "oracle.c")
    mod._LIB_PATH = str(d / "liboracle.so")
    mod._lib = None
    mod.build(force=True)
    return mod


def test_control_copy_passes_every_pin(tmp_path):
    mod = build_variant(tmp_path, "control")
    for name, run in PINS.items():
        run(mod)


@pytest.mark.parametrize("name,old,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, catchers):
    mod = build_variant(tmp_path, "mutant", old, new)
    caught = []
    with np.errstate(all="ignore"):
        for pin in catchers:
            try:
                PINS[pin](mod)
            except AssertionError:
                caught.append(pin)
    assert caught, f"planted mistake '{name}' passed the pins {catchers}"
