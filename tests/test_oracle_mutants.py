"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of oracle/kivi_oracle.c (on the CPU,
in a temporary directory), compiles it, and runs the oracle pin suite against
the broken build: at least one pin must fail.  The committed oracle itself
passes the same suite (the other test files).
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle_quantize.py", "tests/test_oracle_cache.py",
             "tests/test_oracle_attention.py", "tests/test_oracle_sparse_cache.py"]

# (name, exact text in kivi_oracle.c, replacement)
MUTANTS = [
    ("range_sign", "range = mx - mn;", "range = mx + mn;"),
    ("levels_off_by_one", "L = (float)((1u << bits) - 1u);", "L = (float)(1u << bits);"),
    ("round_half_up", "float c = nearbyintf(t);", "float c = floorf(t + 0.5f);"),
    ("round_truncate", "float c = nearbyintf(t);", "float c = truncf(t);"),
    ("reciprocal_multiply", "float t = (x[i * stride] - z) / s;",
     "float t = (x[i * stride] - z) * (1.0f / s);"),
    ("binary64_quotient", "float t = (x[i * stride] - z) / s;\n      float c = nearbyintf(t);",
     "double t = ((double)x[i * stride] - (double)z) / (double)s;\n"
     "      float c = (float)nearbyint(t);"),
    ("zero_is_max", "  z = mn;\n", "  z = mx;\n"),
    ("min_keeps_last_tie", "if (v < mn) mn = v;", "if (v <= mn) mn = v;"),
    ("pack_msb_first", "w |= ((uint32_t)codes[i] & mask) << (bits * i);",
     "w |= ((uint32_t)codes[i] & mask) << (bits * (E - 1 - i));"),
    ("keys_grouped_per_token", "kivi_oracle_quantize_group_meta(&K[(g * G) * D + d], G, D, bits,",
     "kivi_oracle_quantize_group_meta(&K[(g * G) * D + d], G, 1, bits,"),
    ("value_pack_transposed", "for (i = 0; i < E; ++i) tmp[i] = cv[(t * E + i) * D + d];",
     "for (i = 0; i < E; ++i) tmp[i] = cv[(t * E) * D + (d / E) * E + i];"),
    ("residual_length", "r = (T == 0) ? 0 : ((T - 1) % u->R) + 1;", "r = T % u->R;"),
    ("flush_position", "rc = quantize_block(u, u->k_res, u->v_res, u->n_q, u->R);",
     "rc = quantize_block(u, u->k_res, u->v_res, 0, u->R);"),
    ("dequant_sign", "return (double)c * (double)scale + (double)zero;",
     "return (double)c * (double)scale - (double)zero;"),
    ("value_unpack_index", "uint32_t c = unpack_block(blk, (int)(t % E), u->bits);",
     "uint32_t c = unpack_block(blk, (int)(d % E), u->bits);"),
    ("residual_key_index", "out[(u->n_q + t) * D + d] = (double)u->k_res[t * D + d];",
     "out[(u->n_q + t) * D + d] = (double)u->k_res[d];"),
    ("scores_use_values", "for (d = 0; d < u->D; ++d) acc += (double)qh[d] * Kh[t * u->D + d];",
     "for (d = 0; d < u->D; ++d) acc += (double)qh[d] * Vh[t * u->D + d];"),
    ("sigma_dropped", "p[t] = sigma * acc;", "p[t] = acc;"),
    ("unnormalised", "out[(long long)h * u->D + d] = o / l;", "out[(long long)h * u->D + d] = o;"),
    # binary16-metadata variant
    ("codes_against_unrounded_scale",
     "    s = kivi_oracle_round_half(s);\n    z = kivi_oracle_round_half(mn);\n  }\n  *scale = s;",
     "    z = kivi_oracle_round_half(mn);\n  }\n  *scale = meta_f16 ? kivi_oracle_round_half(s) : s;"),
    ("half_ties_away", "r = nearbyint(a / q) * q;", "r = round(a / q) * q;"),
    ("half_no_subnormal_quantum", "if (e < -24) e = -24;", ""),
    ("half_overflow_kept", "if (r > 65504.0) r = INFINITY;", ""),
    ("planes_bit_order_swapped", "    for (i = 0; i < 32; ++i) w |= (uint32_t)((codes[i] >> b) & 1u) << i;",
     "    for (i = 0; i < 32; ++i) w |= (uint32_t)((codes[i] >> (2 - b)) & 1u) << i;"),
    ("planes_unpack_plane_dropped",
     "    return ((w[0] >> pos) & 1u) | (((w[1] >> pos) & 1u) << 1) | (((w[2] >> pos) & 1u) << 2);",
     "    return ((w[0] >> pos) & 1u) | (((w[1] >> pos) & 1u) << 1);"),
    ("sparse_takes_smallest",
     "if (best < 0 || fabsf(x[i * stride]) > fabsf(x[best * stride])) best = i;",
     "if (best < 0 || fabsf(x[i * stride]) < fabsf(x[best * stride])) best = i;"),
    ("sparse_tie_takes_last",
     "if (best < 0 || fabsf(x[i * stride]) > fabsf(x[best * stride])) best = i;",
     "if (best < 0 || fabsf(x[i * stride]) >= fabsf(x[best * stride])) best = i;"),
    ("sparse_outliers_kept_in_range", "    if (!is_out[i]) rest[m++] = x[i * stride];",
     "    rest[m++] = x[i * stride];"),
    ("sparse_key_outliers_not_restored",
     "        out[(t * u->G + u->k_out_idx[e]) * D + d] = (double)u->k_out_val[e];", ""),
    ("sparse_value_outlier_group_offset_dropped",
     "        out[t * D + j * u->Gv + u->v_out_idx[e]] = (double)u->v_out_val[e];",
     "        out[t * D + u->v_out_idx[e]] = (double)u->v_out_val[e];"),
]


def _run_mutant(tmp, name, old, new):
    src = open(os.path.join(ROOT, "oracle", "kivi_oracle.c")).read()
    assert src.count(old) == 1, f"{name}: anchor text not found exactly once"
    d = os.path.join(tmp, name)
    os.makedirs(d)
    with open(os.path.join(d, "kivi_oracle.c"), "w") as f:
        f.write(src.replace(old, new))
    with open(os.path.join(d, "kivi_oracle.h"), "w") as f:
        f.write(open(os.path.join(ROOT, "oracle", "kivi_oracle.h")).read())
    so = os.path.join(d, "libmutant.so")
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", so, os.path.join(d, "kivi_oracle.c"), "-lm"],
                   check=True)
    env = dict(os.environ, KIVI_ORACLE_LIB=so)
    p = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        *PIN_FILES], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    return name, p.returncode, p.stdout[-400:]


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
            results = list(ex.map(lambda m: _run_mutant(tmp, *m), MUTANTS))
    survivors = [(n, out) for n, rc, out in results if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
    for n, rc, out in results:
        assert rc == 1, f"{n}: pin run did not fail cleanly (rc={rc}): {out}"
