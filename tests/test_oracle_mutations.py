"""Plant plausible mistakes in copies of the oracle (on the CPU) and check
that at least one pin catches each of them."""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "blasst_oracle.c")

MUTATIONS = [
    ("dropped_rescale_of_O",
     "for (int64_t x = 0; x < d; ++x) acc[r * d + x] *= alpha;", ""),
    ("wrong_sign_in_exp", "double p = exp(sv - ref_new);", "double p = exp(ref_new - sv);"),
    ("causal_off_by_one", "(c0 + j) <= (r0 + r) + off", "(c0 + j) < (r0 + r) + off"),
    ("running_max_starts_at_zero", "    m[r] = -INFINITY;\n    mref[r] = -INFINITY;",
     "    m[r] = 0.0;\n    mref[r] = -INFINITY;"),
    ("skipped_block_still_adds_to_l", "    if (skip) continue; /* no V",
     "    if (skip) { for (int64_t r = 0; r < nr; ++r) for (int64_t j = 0; j < nc; ++j)"
     " if (s[r * Bc + j] > -INFINITY && mref[r] > -INFINITY) l[r] += exp(s[r * Bc + j] - mref[r]);"
     " continue; } /* no V"),
    ("vote_on_any_row_instead_of_all", "      if (dr > mu) mu = dr;", "      if (dr < mu || mu == -INFINITY) mu = dr;"),
    ("gqa_modulo_mapping", "hk = hq / g;\n  const int64_t r0", "hk = hq % a->Hkv;\n  const int64_t r0"),
    ("lse_without_log", "a->lse[slot * Br + r] = mref[r] + log(l[r]);", "a->lse[slot * Br + r] = mref[r] + l[r];"),
    ("non_strict_threshold", "(mu < log_lambda);\n    visited_before", "(mu <= log_lambda);\n    visited_before"),
    ("vote_without_scale", "        if (sv > mb[r]) mb[r] = sv;",
     "        if (sv / a->scale > mb[r]) mb[r] = sv / a->scale;"),
    ("blocks_right_to_left", "for (int64_t kt = 0; kt < nKt; ++kt) {", "for (int64_t kt = nKt - 1; kt >= 0; --kt) {"),
    ("decode_split_drops_a_key", "const int64_t k1 = k0 + Ls < a->Lkv ? k0 + Ls : a->Lkv;",
     "const int64_t k1 = (k0 + Ls < a->Lkv ? k0 + Ls : a->Lkv) - 1;"),
    ("merge_weight_sign", "double w = (ls == -INFINITY) ? 0.0 : exp(ls - M);",
     "double w = (ls == -INFINITY) ? 0.0 : exp(M - ls);"),
    ("static_mask_ignored", "if (kt > kt_last || (smask && smask[kt])) {", "if (kt > kt_last) {"),
    ("static_masked_block_still_raises_max",
     "    if (kt > kt_last || (smask && smask[kt])) {\n      if (mask) mask[kt] = MASK_NOT_VISITED;",
     "    if (smask && smask[kt] && kt <= kt_last) {\n      for (int64_t r = 0; r < nr; ++r) {\n"
     "        for (int64_t j = 0; j < Bc && kt * Bc + j < a->Lkv; ++j) {\n"
     "          double dot = 0.0;\n"
     "          for (int64_t x = 0; x < d; ++x) dot += qrow[r * d + x] * widen(a->k, a->dtype, kvbase + (kt * Bc + j) * d + x);\n"
     "          if (a->scale * dot > m[r]) m[r] = a->scale * dot;\n        }\n      }\n    }\n"
     "    if (kt > kt_last || (smask && smask[kt])) {\n      if (mask) mask[kt] = MASK_NOT_VISITED;"),
    ("backward_drops_D", "const double dsj = p[j] * (ds[j] - D);", "const double dsj = p[j] * ds[j];"),
    ("backward_dk_from_k", "dkj[x] += a->scale * dsj * qi[x];",
     "dkj[x] += a->scale * dsj * widen(a->k, a->dtype, kvbase + j * d + x);"),
    ("backward_dv_without_p", "dvj[x] += p[j] * doi[x];", "dvj[x] += doi[x];"),
    ("backward_ignores_tile_mask", "if (kept && a->tile_mask)", "if (0 && kept && a->tile_mask)"),
    ("select_background_includes_first", "for (int64_t j = 1; j < jl; ++j) bg += row[j];",
     "for (int64_t j = 0; j < jl; ++j) bg += row[j];"),
    ("select_background_not_strict", "if (row[j] > bg) m[j] = 0;", "if (row[j] >= bg) m[j] = 0;"),
    ("select_theta_strict", "if (row[j] >= theta) m[j] = 0;", "if (row[j] > theta) m[j] = 0;"),
    ("select_cstruct_without_window", "cs += row[0] + (jl > 0 ? row[jl] : 0.0);", "cs += row[0];"),
    ("select_route_inverted", "const int structured = cs >= a->tau;", "const int structured = cs < a->tau;"),
    ("select_ragged_block_mean", "kbar[j * d + x] = acc / (double)(c1 - c0);",
     "kbar[j * d + x] = acc / (double)a->Bc;"),
    ("select_last_block_off_by_one", "int64_t jl = (r1 - 1 + (a->Lkv - a->Lq)) / a->Bc;",
     "int64_t jl = (r1 + (a->Lkv - a->Lq)) / a->Bc;"),
    ("decode_skipped_block_still_used", "    if (skip) continue;\n    for (int64_t j = 0; j < nc; ++j)\n      for (int64_t x = 0; x < d; ++x)\n        kv_v",
     "    for (int64_t j = 0; j < nc; ++j)\n      for (int64_t x = 0; x < d; ++x)\n        kv_v"),
]


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/not found"
    mutated = src.replace(old, new)
    c_path = tmp_path / "mut.c"
    so_path = tmp_path / "libmut.so"
    c_path.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so_path),
                           str(c_path), "-lm", "-lpthread"])
    orc = oracle.Oracle(str(so_path))
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
            break
    assert caught, f"no pin caught the planted mistake {name!r}"
