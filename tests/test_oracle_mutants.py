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
