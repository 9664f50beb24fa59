"""Planted mistakes in the CPU oracle must each break at least one pin.

Each mutant is a copy of ``oracle/hkv_oracle.c`` with one plausible mistake
(a dropped term, a wrong sign, index or comparison), compiled on the CPU into a
temporary library. The pins of ``tests/pins.py`` run against it; at least one
must fail, which shows the pins constrain that part of the oracle.
"""
import os
import shutil

import pytest

import oracle
from oracle import build as obuild
from tests import pins

MUTANTS = {
    "gqa_group_mapping": ("h * G + g, sp, h, j)", "g * d->Hkv + h, sp, h, j)"),
    "score_scale_dropped": ("double s = d->scale * dot_qk(d, q, b, h * G + g, sp, h, j);",
                            "double s = dot_qk(d, q, b, h * G + g, sp, h, j);"),
    "pool_min_not_max": ("if (s > best)\n                    best = s;",
                         "if (s < best || best == -INFINITY)\n                    best = s;"),
    "bf16_widen_shift": ("(uint32_t)bits << 16", "(uint32_t)bits << 15"),
    "calib_beta_dropped": ("return exp(beta * ((double)zj - (double)m));",
                           "return exp(((double)zj - (double)m));"),
    "calib_sign": ("return exp(beta * ((double)zj - (double)m));",
                   "return exp(beta * ((double)m - (double)zj));"),
    "calib_not_normalised": ("(float)(calib_weight(zu[j], mu, bu) / Z)",
                             "(float)(calib_weight(zu[j], mu, bu))"),
    "tie_higher_index_first": ("return (x->j > y->j) - (x->j < y->j);",
                               "return (x->j < y->j) - (x->j > y->j);"),
    "order_ascending": ("if (x->z > y->z)\n        return -1;\n    if (x->z < y->z)\n        return 1;",
                        "if (x->z > y->z)\n        return 1;\n    if (x->z < y->z)\n        return -1;"),
    "mass_strictly_above_p": ("if (C >= (double)p) {", "if (C > (double)p) {"),
    "kstar_off_by_one": ("kstar = i + 1;", "kstar = i;"),
    "no_cap_at_n": ("if (k > n)\n        k = n;", "if (k > n + 1000000)\n        k = n;"),
    "bmin_ignored": ("if (k < bmin)\n        k = bmin;", "if (k < 0)\n        k = bmin;"),
    "bmax_ignored": ("int32_t k = kstar < bmax ? kstar : bmax;", "int32_t k = kstar;"),
    "rows_not_index_sorted": ("qsort(row, (size_t)k, sizeof(int32_t), by_index);", ";"),
    "flat_offsets_not_scanned": ("offsets[u + 1] = offsets[u] + sel_len[u];",
                                 "offsets[u + 1] = sel_len[u];"),
    "condensed_tier_dropped": [("int32_t T = W + k + C;", "int32_t T = W + k;"),
                               ("for (int32_t j = 0; j < C; ++j)\n            toks[t++] = (token_ref){condensed, j};",
                                "for (int32_t j = 0; j < 0; ++j)\n            toks[t++] = (token_ref){condensed, j};")],
    "lse_missing_max": ("(float)(M + log(L))", "(float)(log(L))"),
    "attention_v_from_k": ("elem(toks[i].t->v, d->dtype, vo + x)", "elem(toks[i].t->k, d->dtype, vo + x)"),
}


@pytest.fixture(scope="module")
def src_text():
    with open(obuild.SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, src_text, tmp_path, monkeypatch):
    edits = MUTANTS[name]
    if isinstance(edits, tuple):
        edits = [edits]
    mutated = src_text
    for old, new in edits:
        assert mutated.count(old) >= 1, f"mutation site for {name} not found"
        mutated = mutated.replace(old, new)
    src = tmp_path / "hkv_oracle.c"
    src.write_text(mutated)
    shutil.copy(os.path.join(obuild.HERE, "hkv_oracle.h"), tmp_path / "hkv_oracle.h")
    so = str(tmp_path / f"libhkv_oracle_{name}.so")
    obuild.build(force=True, src=str(src), out=so, extra=("-I", str(tmp_path)))
    monkeypatch.setattr(oracle, "_lib", oracle.lib(so))
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin()
        except (AssertionError, ValueError) as e:  # a pin failed or the oracle refused
            caught.append((pin.__name__, type(e).__name__))
            break
    assert caught, f"mutant {name} passed every pin"


# ---- the numpy append (TS 2.A pipeline step 1): planted mistakes in copies of it ----

APPEND_MUTANTS = {
    "head_not_advanced": ("hd[u] = (hd[u] + 1) % wcap", "hd[u] = hd[u] % wcap"),
    "newest_ages_out": ("old_k, old_v = dk[b, h, hd[u]].copy(), dv[b, h, hd[u]].copy()",
                        "old_k, old_v = k_new[b, h], v_new[b, h]"),
    "sparse_full_one_early": ("if slen[u] < ncap:", "if slen[u] < ncap - 1:"),
    "window_never_fills": ("if dlen[u] < wcap:", "if dlen[u] < wcap - 1:"),
}


@pytest.mark.parametrize("name", sorted(APPEND_MUTANTS))
def test_append_mutant_is_caught(name, monkeypatch):
    import inspect
    import textwrap

    import oracle
    from tests import pins

    src = textwrap.dedent(inspect.getsource(oracle.append))
    old, new = APPEND_MUTANTS[name]
    assert old in src, name
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, "append", ns["append"])
    failed = False
    for pin in (pins.pin_append_matches_list_model, pins.pin_append_without_window_goes_to_sparse):
        try:
            pin()
        except Exception:
            failed = True
    assert failed, f"mutant {name} passed every append pin"


# ---- the numpy fitted temperature (TS 2.B, TS 3): planted mistakes in copies of it ----

FIT_MUTANTS = {
    "entropy_in_bits": ("softmax_entropy", "np.log(P[nz])", "np.log2(P[nz])"),
    "entropy_sign": ("softmax_entropy", "-(P[nz] * np.log(P[nz])).sum()", "(P[nz] * np.log(P[nz])).sum()"),
    "softmax_without_max": ("softmax_entropy", "w = np.exp(x - x.max())", "w = np.exp(x - x.min())"),
    "max_over_heads": ("attention_entropy", "np.mean([softmax_entropy", "np.max([softmax_entropy"),
    "wrong_group": ("attention_entropy", "qf[b, h * G:(h + 1) * G]", "qf[b, h:h + G]"),
    "scale_dropped": ("attention_entropy", "logits = scale * (", "logits = ("),
    "bisection_flipped": ("fit_temperature", "> t:\n                lo = mid", "< t:\n                lo = mid"),
    "temperature_not_inverse": ("fit_temperature", "softmax_entropy(mid * zu)", "softmax_entropy(zu / mid)"),
    "lower_bound_missing": ("fit_temperature", "if t >= np.log(n):", "if t > np.log(n) + 1.0:"),
}


@pytest.mark.filterwarnings("ignore::RuntimeWarning")  # a mutant may overflow; that is how it fails
@pytest.mark.parametrize("name", sorted(FIT_MUTANTS))
def test_fit_mutant_is_caught(name, monkeypatch):
    import inspect
    import textwrap

    import oracle
    from tests import pins

    fn, old, new = FIT_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(getattr(oracle, fn)))
    assert old in src, name
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    failed = False
    for pin in (pins.pin_attention_entropy_matches_scipy, pins.pin_attention_entropy_of_equal_keys_is_log_n,
                pins.pin_fit_identical_heads_gives_one, pins.pin_fit_two_tokens_closed_form,
                pins.pin_fit_matches_brentq, pins.pin_fit_boundaries_and_order):
        try:
            pin()
        except Exception:
            failed = True
    assert failed, f"mutant {name} passed every fitted-temperature pin"


# ---- the numpy condensed-tier formation (TS 2.A Tier 3, pipeline step 4) ----

CONDENSE_MUTANTS = {
    "newest_block_condensed": ("condense", "rows_k, rows_v = _f64(sk[b, h, :block]), _f64(sv[b, h, :block])",
                               "rows_k, rows_v = _f64(sk[b, h, n - block:n]), _f64(sv[b, h, n - block:n])"),
    "full_tier_not_shifted": ("condense", "ck[b, h, 1:ccap - 1] = ck[b, h, 2:ccap].copy()",
                              "ck[b, h, 1:ccap - 1] = ck[b, h, 1:ccap - 1].copy()"),
    "evict_least_important": ("condense", "jstar = int(np.argmax(zz))", "jstar = int(np.argmin(zz))"),
    "evict_drops_newest_slot": ("condense", "ck[b, h, 0:ccap - 1] = ck[b, h, 1:ccap].copy()",
                                "ck[b, h, 0:ccap - 1] = ck[b, h, 0:ccap - 1].copy()"),
    "sparse_not_moved_down": ("condense", "sk[b, h, :n - block] = sk[b, h, block:n].copy()",
                              "sk[b, h, :n - block] = sk[b, h, :n - block].copy()"),
    "trigger_ignored": ("condense", "if n < max(trigger, block, 1):", "if n < max(block, 1):"),
    "mass_not_kept": ("condense", "w[u, C] = np.float32(_seq_sum(a))", "w[u, C] = np.float32(1.0)"),
    "beta_ignored": ("condense", "a = np.exp(be * (zz", "a = np.exp(1.0 * (zz"),
    "unweighted_mean": ("_weighted_mean", "num = num + a[j] * rows[j]", "num = num + rows[j] * (den * 0 + 1)"),
    "bf16_round_half_up": ("round_to_bf16", "r = np.rint(np.ldexp(x, -sh))", "r = np.floor(np.ldexp(x, -sh) + 0.5)"),
    "bf16_through_float32": ("round_to_bf16", "f, e = np.frexp(x)",
                             "x = x.astype(np.float32).astype(np.float64)\n    f, e = np.frexp(x)"),
}


@pytest.mark.filterwarnings("ignore::RuntimeWarning")
@pytest.mark.parametrize("name", sorted(CONDENSE_MUTANTS))
def test_condense_mutant_is_caught(name, monkeypatch):
    import inspect
    import textwrap

    import oracle
    from tests import pins

    fn, old, new = CONDENSE_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(getattr(oracle, fn)))
    assert old in src, name
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    # the module's other functions look helpers up in the module namespace
    failed = False
    for pin in (pins.pin_round_to_bf16_is_nearest_even, pins.pin_condense_merge_is_weighted_average,
                pins.pin_condense_matches_list_model, pins.pin_condense_noop_drop_and_single_slot,
                pins.pin_condense_bf16_merge_exact):
        try:
            pin()
        except Exception:
            failed = True
    assert failed, f"mutant {name} passed every condensation pin"


# ---- the numpy Rewrite Cache / Sparse Loading trigger (TS 2.C Trade-off Management) ----

MTI_MUTANTS = {
    "trigger_inverted": ("mti_trigger", "if k > L_upper:\n        return MODE_REWRITE",
                         "if k > L_upper:\n        return MODE_SPARSE"),
    "no_hysteresis": ("mti_trigger", "    return mode", "    return MODE_SPARSE"),
    "horizon_floor_missing": ("mti_horizon", "max(1, mti_cap // k)", "max(1, -(-mti_cap // k))"),
    "reuse_not_counted_down": ("step_mti", 'st["left"][u] -= 1', 'st["left"][u] -= 0'),
    "horizon_counts_the_rewrite_step_twice": ("step_mti", "mti_horizon(ku, mti_cap) - 1", "mti_horizon(ku, mti_cap)"),
    "rewrite_of_the_wrong_rows": ("step_mti", "rows = idf[u, :ku]", "rows = idf[u, :ku] * 0"),
    "reuse_attends_plain_step": ("step_mti", "out[b, h * G:(h + 1) * G] = r_out[b, h * G:(h + 1) * G]",
                                 "out[b, h * G:(h + 1) * G] = plain['out'][b, h * G:(h + 1) * G]"),
}


@pytest.mark.parametrize("name", sorted(MTI_MUTANTS))
def test_mti_mutant_is_caught(name, monkeypatch):
    import inspect
    import textwrap

    import oracle
    from tests import pins

    fn, old, new = MTI_MUTANTS[name]
    src = textwrap.dedent(inspect.getsource(getattr(oracle, fn)))
    assert old in src, name
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    monkeypatch.setattr(oracle, fn, ns[fn])
    failed = False
    for pin in (pins.pin_mti_trigger_and_horizon, pins.pin_mti_reuse_attends_the_rewritten_rows,
                pins.pin_mti_rewrite_copies_the_top_rows, pins.pin_mti_state_matches_model):
        try:
            pin()
        except Exception:
            failed = True
    assert failed, f"mutant {name} passed every trigger pin"
