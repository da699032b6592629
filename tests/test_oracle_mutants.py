"""Plausible mistakes planted in copies of the oracle (on the CPU) must each
fail at least one pin: evidence that the pins can catch a dropped term, a
wrong sign or index, or a transposed operand."""
import os
import shutil

import pytest

import oracle
from oracle_pins import FAST_PINS

# (name, text in na_oracle.c, replacement)
MUTANTS = [
    ("leader_at_group_start", "int c = g * s + s / 2;", "int c = g * s;"),
    ("window_off_by_one", "int start = c - w / 2;", "int start = c - w / 2 + 1;"),
    ("window_not_centred", "int start = c - w / 2;", "int start = c - w;"),
    ("no_upper_clamp", "if (start > L - w) start = L - w;", ""),
    ("dropped_scale", "z[cnt] = J->scale * dot;", "z[cnt] = dot;"),
    ("key_index_is_query", "load_in(J->k, J->dtype, koff + c)", "load_in(J->k, J->dtype, qoff + c)"),
    ("value_of_query", "(size_t)N + (size_t)idx[e]) * (size_t)d;", "(size_t)N + (size_t)t) * (size_t)d;"),
    ("lse_without_max", "J->lse[r] = m + log(l);", "J->lse[r] = log(l);"),
    ("lse_log2", "J->lse[r] = m + log(l);", "J->lse[r] = m + log2(l);"),
    ("unnormalised", "double p = exp(z[e] - m) / l;", "double p = exp(z[e] - m);"),
    ("sign_flip_exp", "double p = exp(z[e] - m) / l;", "double p = exp(m - z[e]) / l;"),
    ("column_major_tokens", "for (int a = ndim - 1; a >= 0; --a) {\n        coord[a]",
     "for (int a = 0; a < ndim; ++a) {\n        coord[a]"),
    ("mask_upper_inclusive", "u >= hi[a]) in = 0;", "u > hi[a]) in = 0;"),
    ("full_partial_swapped", "m == ra * cb ? 2 : 1", "m == ra * cb ? 1 : 2"),
    ("causal_excludes_self", "a = (g + 1) * s - w;", "a = g * s - w;"),
    ("causal_looks_ahead", "a = (g + 1) * s - w;", "a = g * s;"),
    ("truncated_not_centred", "a = g * s + s / 2 - w / 2;", "a = g * s - w / 2;"),
    ("truncated_as_clamped", "if (mode == WIN_CLAMPED) {", "if (mode != WIN_CAUSAL) {"),
    ("cut_upper_short", "*hi = a + w > L ? L : a + w;", "*hi = a + w > L ? L - 1 : a + w;"),
    ("mode_ignored_in_mask", "mode ? mode[a] : WIN_CLAMPED", "WIN_CLAMPED"),
    ("f16_exponent_bias", "ldexp((double)(1024 + f), e - 25)", "ldexp((double)(1024 + f), e - 24)"),
    ("f16_subnormal_as_normal", "v = ldexp((double)f, -24);", "v = ldexp((double)(1024 + f), -25);"),
    ("f16_read_as_bf16", "if (dtype == IN_F16) return", "if (dtype == -1) return"),
    ("bwd_no_delta", "const double dz = p * (dp - Di);", "const double dz = p * dp;"),
    ("bwd_dk_from_k", "J->dk[koff + c] += J->scale * dz * load_in(J->q, J->dtype, qoff + c);",
     "J->dk[koff + c] += J->scale * dz * load_in(J->k, J->dtype, koff + c);"),
    ("bwd_dv_without_p", "J->dv[koff + c] += p * load_in(J->dout, J->dtype, qoff + c);",
     "J->dv[koff + c] += load_in(J->dout, J->dtype, qoff + c);"),
    ("bwd_dq_unscaled", "g[c] += J->scale * dz * load_in(J->k, J->dtype, koff + (size_t)c);",
     "g[c] += dz * load_in(J->k, J->dtype, koff + (size_t)c);"),
    ("dilation_floor_length", "const int Lr = (L - res + dil - 1) / dil;",
     "const int Lr = L / dil;"),
    ("dilation_residue_ignored", "if (kj[a] % step[a] != res[a]) in = 0;", ""),
    ("dilation_position_undivided", "na_oracle_window(Lr, w, s, mode, i / dil, lo, hi)",
     "na_oracle_window(Lr, w, s, mode, i / dil / dil, lo, hi)"),
    ("dilation_step_one", "const int u = kj[a] / step[a];", "const int u = kj[a];"),
    ("bwd_dilation_ignored", "J->mode, J->dil, t, mask);\n            const size_t qoff",
     "J->mode, NULL, t, mask);\n            const size_t qoff"),
    ("bwd_delta_from_v", "Di += load_in(J->dout, J->dtype, qoff + c) * o[c];",
     "Di += load_in(J->dout, J->dtype, qoff + c) * load_in(J->v, J->dtype, qoff + c);"),
    ("e4m3_exponent_bias", "v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 9);"),
    ("e4m3_subnormal_as_normal", "v = ldexp((double)m, -9);", "v = ldexp((double)(8 + m), -10);"),
    ("e4m3_read_as_f16_byte", "if (dtype == IN_E4M3) return", "if (dtype == -1) return"),
    # the sampled backward forgets the queries that only its key rows read
    ("sampled_stats_miss_key_queries",
     "if (window_holds(ndim, L, w, s, mode, qi, kj)) needed[t] = 1;", ""),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new, tmp_path):
    src = open(oracle.SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mpath = tmp_path / f"mut_{name}.c"
    mpath.write_text(src.replace(old, new))
    lib_path = str(tmp_path / f"libmut_{name}.so")
    oracle.compile_lib(str(mpath), lib_path)
    lib = oracle.OracleLib(lib_path)
    pins = list(FAST_PINS)
    if name == "full_partial_swapped":
        from oracle_pins import pin_block_counts_closed_forms
        pins = [pin_block_counts_closed_forms]
    caught = []
    for pin in pins:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, ValueError):
            caught.append(pin.__name__)
            break
    assert caught, f"mutant {name} passed every pin"
