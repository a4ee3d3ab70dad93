"""Planted mistakes in the oracle must be caught by its pins.

Each mutant is a copy of ``oracle/oracle.c`` with one plausible mistake (a dropped term,
a wrong sign, index or operand order, a swapped nibble).  It is compiled into a temporary
directory and the pins of ``pins.py`` run against it in a child process; the test
passes when at least one pin fails.  Nothing here touches the committed oracle.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))

MUTANTS = {
    "int4_nibble_order": ("int n = (k & 1) ? (int)(b >> 4) : (int)(b & 15);",
                          "int n = (k & 1) ? (int)(b & 15) : (int)(b >> 4);"),
    "int4_unsigned": ("return n >= 8 ? n - 16 : n;", "return n;"),
    "int4_offset_binary": ("return n >= 8 ? n - 16 : n;", "return n - 8;"),
    "half_exponent": ("v = ldexp((double)(1024 + m), e - 25);", "v = ldexp((double)(1024 + m), e - 24);"),
    "half_subnormal": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "e2m1_bias": ("ldexp(1.0 + 0.5 * m, e - 1);", "ldexp(1.0 + 0.5 * m, e);"),
    "e2m1_subnormal": ("0.5 * m :", "1.0 * m :"),
    "e4m3_bias": ("ldexp(1.0 + m / 8.0, e - 7);", "ldexp(1.0 + m / 8.0, e - 8);"),
    "e4m3_subnormal": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "nvfp4_block_index": ("(size_t)(k / 16)];", "(size_t)((k / 16 + 1) % (M->K / 16))];"),
    "nvfp4_no_tensor_scale": ("* (double)M->tensor_scale;", ";"),
    "nvfp4_nibble_order": ("unsigned c = (k & 1) ? (b >> 4) : (b & 15);",
                           "unsigned c = (k & 1) ? (b & 15) : (b >> 4);"),
    "router_transposed": ("acc += (double)Wr[(size_t)e * H + h]", "acc += (double)Wr[(size_t)h * E + e]"),
    "router_no_fp32_round": ("logits[(size_t)t * E + e] = (float)acc;",
                             "logits[(size_t)t * E + e] = (float)(acc * (1.0 + 1e-6));"),
    "sigmoid_sign": ("return (float)(1.0 / (1.0 + exp(-(double)logit)));",
                     "return (float)(1.0 / (1.0 + exp((double)logit)));"),
    "bias_sign": ("sel[e] = s[e] + bias[e];", "sel[e] = s[e] - bias[e];"),
    "bias_dropped": ("sel[e] = s[e] + bias[e];", "sel[e] = s[e];"),
    "topk_tie_high": ("(best < 0 || sel[e] > sel[best])", "(best < 0 || sel[e] >= sel[best])"),
    "weights_from_sel": ("(float)(scaling * ((double)s[topk_idx[(size_t)t * k + j]] / sum));",
                         "(float)(scaling * ((double)sel[topk_idx[(size_t)t * k + j]] / sum));"),
    "weights_no_scaling": ("(float)(scaling * ((double)s[", "(float)(1.0 * ((double)s["),
    "weights_no_norm": ("((double)s[topk_idx[(size_t)t * k + j]] / sum));",
                        "((double)s[topk_idx[(size_t)t * k + j]] / 1.0));"),
    "group_unique_all": ("if (counts[e] > 0) unique[u++] = e;", "if (counts[e] >= 0) unique[u++] = e;"),
    "group_count_dropped": ("for (int a = 0; a < n; a++)\n        if (topk_idx[a] >= 0) counts[topk_idx[a]]++;",
                            "for (int a = 1; a < n; a++)\n        if (topk_idx[a] >= 0) counts[topk_idx[a]]++;"),
    "group_perm_reverse": ("for (int a = 0; a < n; a++) {                      /* ascending a: stable */",
                           "for (int a = n - 1; a >= 0; a--) {"),
    "silu_gate_up_swapped": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = u / (1.0 + exp(-u)) * g;"),
    "silu_sign": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = g / (1.0 + exp(g)) * u;"),
    "silu_dropped": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = g * u;"),
    "down_row_col": ("acc += wq(Wd, m, n) * h[n];", "acc += wq(Wd, m % Wd->K, n % Wd->N) * h[n];"),
    "combine_no_shared": ("double acc = L->n_shared ? y_shared[(size_t)t * H + m] : 0.0;", "double acc = 0.0;"),
    "combine_wrong_j": ("acc += (double)topk_w[(size_t)t * k + j] * y_assign",
                        "acc += (double)topk_w[(size_t)t * k + (k - 1 - j)] * y_assign"),
    "batched_token_index": ("int a = R->perm[p], t = a / k;", "int a = R->perm[p], t = a % T;"),
    "gap_wrong": ("gap = (float)((double)last - (double)next);", "gap = (float)((double)last);"),
    # int8 / int2 codes and the quantiser
    "int8_unsigned": ("return n >= 128 ? n - 256 : n;", "return n;"),
    "int8_row_stride": ("return format == ORC_INT8 ? (size_t)K :", "return format == ORC_INT8 ? (size_t)(K / 2) :"),
    "int2_bit_order": ("int n = (int)((b >> (2 * (k & 3))) & 3u);", "int n = (int)((b >> (6 - 2 * (k & 3))) & 3u);"),
    "int2_unsigned": ("return n >= 2 ? n - 4 : n;", "return n;"),
    "quant_levels": ("float sc = (float)(amax / qmax);", "float sc = (float)(amax / (qmax + 1));"),
    "quant_truncate": ("double v = rint((double)w[(size_t)n * K + k] / (double)sc);",
                       "double v = trunc((double)w[(size_t)n * K + k] / (double)sc);"),
    "quant_int2_pack": ("row[k >> 2] |= (uint8_t)((u & 3u) << (2 * (k & 3)));",
                        "row[k >> 2] |= (uint8_t)((u & 3u) << (2 * (3 - (k & 3))));"),
    "quant_int4_pack": ("row[k >> 1] |= (uint8_t)((u & 15u) << (4 * (k & 1)));",
                        "row[k >> 1] |= (uint8_t)((u & 15u) << (4 * (1 - (k & 1))));"),
    # adaptive expert top-p
    "topp_le": ("keep[at[r]] = before < top_p * S;", "keep[at[r]] = before <= top_p * S;"),
    "topp_rank_ascending": ("if (si > sj || (si == sj && idx[i] < idx[j])) r++;",
                            "if (si < sj || (si == sj && idx[i] < idx[j])) r++;"),
    "topp_tie_high": ("if (si > sj || (si == sj && idx[i] < idx[j])) r++;",
                      "if (si > sj || (si == sj && idx[i] > idx[j])) r++;"),
    "topp_no_renorm": ("w[m] = (float)(scaling * ((double)s[old[j]] / S2));",
                       "w[m] = (float)(scaling * ((double)s[old[j]] / S));"),
    "topp_score_order_out": ("idx[m] = old[j];", "idx[m] = old[at[m]];"),
    "topp_margin_missing": ("if (m < (double)gap) gap = (float)m;", ";"),
    "topp_kept_not_skipped": ("if (e >= 0) perm[offsets[e] + fill[e]++] = a;",
                              "if (e >= 0) perm[offsets[e] + fill[e]++] = a; else perm[0] = a;"),
}


def _build_mutant(name, tmp):
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) >= 1, f"mutant {name}: pattern not found in oracle.c"
    d = os.path.join(tmp, name)
    os.makedirs(d, exist_ok=True)
    path = os.path.join(d, "oracle.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new, 1))
    so = os.path.join(d, "liboracle.so")
    oracle.compile_oracle(path, so, os.path.dirname(oracle.SRC))
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, os.path.join(HERE, "pins.py"), so], capture_output=True,
                       text=True, timeout=300, env=env)
    return r


@pytest.fixture(scope="module")
def mutant_results(tmp_path_factory):
    tmp = str(tmp_path_factory.mktemp("mutants"))
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        futs = {n: ex.submit(_build_mutant, n, tmp) for n in MUTANTS}
        return {n: f.result() for n, f in futs.items()}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(mutant_results, name):
    r = mutant_results[name]
    # a crash of the child counts as caught; otherwise at least one pin must fail
    failed = r.stdout.strip().splitlines()[-1] if r.returncode == 0 and r.stdout.strip() else ""
    assert r.returncode != 0 or failed, f"mutant {name} passed every pin\n{r.stderr[-2000:]}"
