"""Plant plausible mistakes into copies of the oracle and check that the pins catch every one.

Each mutant is the oracle source with one small textual change (a dropped term, a wrong divisor,
a swapped index, a reversed tie-break, ...). It is compiled into a temporary library and the pin
suite (tests/test_oracle_pins.py) runs against it in a subprocess; the suite must fail. The
mistakes are planted on the CPU only, in throw-away copies; the committed oracle is untouched.
"""
import concurrent.futures as cf
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "s3r_oracle.c")

MUTANTS = {
    "pool_divides_by_block_size": (
        "double mean = sum / (double)n;", "double mean = sum / (double)p->block;"),
    "pool_skips_bf16_rounding": (
        "p->exact_pool ? mean : s3r_ref_round_bf16(mean)", "mean"),
    "lse_drops_the_max": (
        "const double lse = m + log(l);", "const double lse = log(l);"),
    "lse_skips_the_tail_block": (
        "for (int64_t j = 0; j < nb; ++j) l += exp(s[j] - m);",
        "for (int64_t j = 0; j < nb - 1; ++j) l += exp(s[j] - m);"),
    "scores_sum_unnormalised_weights": (
        "if (score_row) score_row[j] += pj;", "if (score_row) score_row[j] += exp(s[j] - m);"),
    "cmp_reads_head_zero_keys": (
        "const double* krow = c->kc + j * HD + h * d;", "const double* krow = c->kc + j * HD;"),
    "scores_transposed_layout": (
        "double* score_row = c->scores ? c->scores + (h * rm->nq + i) * nb : NULL;",
        "double* score_row = c->scores ? c->scores + (i * p->H + h) * nb : NULL;"),
    "cmp_ignores_scale": ("s[j] = p->scale * dot;", "s[j] = dot;"),
    "topk_ties_to_higher_index": (
        "return (x->index > y->index) - (x->index < y->index);",
        "return (x->index < y->index) - (x->index > y->index);"),
    "topk_gap_from_the_top": (
        "a[c->k - 1].score - a[c->k].score", "a[0].score - a[c->k].score"),
    "sel_ignores_scale": (" s[a] = p->scale * dot;", " s[a] = dot;"),
    "sel_uses_first_query_row": (
        "const int64_t t_q = rm->first[i] + r;", "const int64_t t_q = rm->first[i];"),
    "sel_keys_from_values": (
        "const uint16_t* krow = c->k + tokens[a] * HD + h * d;",
        "const uint16_t* krow = c->v + tokens[a] * HD + h * d;"),
    "combine_swaps_gates": (
        "const double g_cmp = sigmoid((double)gates[(r * H + h) * 2 + 0]);",
        "const double g_cmp = sigmoid((double)gates[(r * H + h) * 2 + 1]);"),
    "round_bf16_truncates": ("double r = nearbyint(scaled);", "double r = trunc(scaled);"),
    "topk_forced_offset_dropped": (
        "a[j].index = c->forced + j;", "a[j].index = j;"),
    "topk_forced_blocks_compete": (
        "a[j].score = c->scores[r * c->n + c->forced + j];",
        "a[j].score = c->scores[r * c->n + j];"),
    "topk_forced_list_not_opened": (
        "for (int32_t f = 0; f < c->forced; ++f) out[f] = f;",
        "for (int32_t f = 0; f < c->forced; ++f) out[f] = c->forced;"),
    "window_spills_past_grid_edge": (
        "c < (wc + 1) * win_w && c < p->grid_w; ++c)", "c < (wc + 1) * win_w; ++c)"),
    "window_forgets_special_offset": (
        "out[n++] = first + p->special + r * p->grid_w + c;", "out[n++] = first + r * p->grid_w + c;"),
    "window_index_ignores_special_block": ("    m -= 1;\n", "\n"),
    "window_rows_use_grid_width": (
        "const int64_t wr = m / cols, wc = m % cols;", "const int64_t wr = m / p->grid_w, wc = m % cols;"),
    "sel_list_skips_forced_blocks": (
        "const int32_t n_list = p->forced + p->topk; /* always-kept",
        "const int32_t n_list = p->topk; /* always-kept"),
    "bwd_sel_drops_softmax_centering": (
        "const double dsa = ss[a] * (dp - ds);", "const double dsa = ss[a] * dp;"),
    "bwd_cmp_centres_with_the_other_branch": (
        "const double dsj = sc[j] * (dp - dc);", "const double dsj = sc[j] * (dp - ds);"),
    "bwd_pool_spread_without_divisor": (
        "c->dk[tokens[a] * HD + h * d + e] += dkc[j * d + e] / (double)n;",
        "c->dk[tokens[a] * HD + h * d + e] += dkc[j * d + e];"),
    "bwd_gate_derivative_drops_one_minus": (
        "c->dgates[(o * H + h) * 2 + 0] = g0 * (1.0 - g0) * yc;",
        "c->dgates[(o * H + h) * 2 + 0] = g0 * yc;"),
    "bwd_sel_value_grad_ignores_gate": (
        "c->dv[t * HD + h * d + e] += ss[a] * dos[e];",
        "c->dv[t * HD + h * d + e] += ss[a] * dy[e];"),
    "bwd_rows_use_the_first_query_row": (
        "const int64_t r = rm->first[i] + rr, o = rm->offset[i] + rr;",
        "const int64_t r = rm->first[i], o = rm->offset[i] + rr;"),
    "bwd_cmp_key_grad_misses_scale": (
        "dkc[j * d + e] += p->scale * dsj * qv[e];", "dkc[j * d + e] += dsj * qv[e];"),
    "bwd_keys_pool_spread_without_divisor": (
        "dk[(a * p->block + u) * d + e] += sk / (double)n;",
        "dk[(a * p->block + u) * d + e] += sk;"),
    "bwd_keys_sel_drops_softmax_centering": (
        "const double dst = ss[t] * (dp - ds);", "const double dst = ss[t] * dp;"),
    "bwd_keys_cmp_value_grad_ignores_gate": (
        "dvc[a * d + e] += pr[j] * doc[e];",
        "dvc[a * d + e] += pr[j] * c->dout[r * HD + h * d + e];"),
    "bwd_sel_dq_from_values": (
        "dqr[e] += p->scale * dsa * bf16_value(c->k[t * HD + h * d + e]);",
        "dqr[e] += p->scale * dsa * bf16_value(c->v[t * HD + h * d + e]);"),
}


def _run_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, f"{name}: anchor not found exactly once"
    d = os.path.join(tmp, name)
    os.makedirs(d)
    with open(os.path.join(d, "s3r_oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    lib = os.path.join(d, "libmutant.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-D_GNU_SOURCE", "-fPIC", "-shared", "-pthread",
                    "-I", os.path.join(ROOT, "oracle"), "-o", lib,
                    os.path.join(d, "s3r_oracle.c"), "-lm"], check=True)
    env = dict(os.environ, S3R_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode, r.stdout[-400:]


def test_every_planted_mistake_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with cf.ThreadPoolExecutor(max_workers=4) as ex:
            futs = [ex.submit(_run_mutant, n, o, w, tmp) for n, (o, w) in MUTANTS.items()]
            results = [f.result() for f in futs]
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"pins did not catch: {survivors}"
