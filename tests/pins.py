"""Pins of the CPU oracle to things other than itself.

Each ``pin_*`` function raises ``AssertionError`` when the oracle disagrees with
a library routine (numpy/scipy/torch), a brute-force search, a closed form or
an invariant fixed by the pages. They are run as tests (``test_oracle_pins``)
and against deliberately broken builds of the oracle (``test_oracle_mutants``),
which must each fail at least one pin.

Sources named below: the arXiv abstract on the mlsanity.com page "HARD-KV:
Head-Adaptive Regularization for Decoding-time KV Compression" ("Abstract") and
the gist.science Technical Summary of that paper ("TS", with its section).
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import scipy.special as sps
import torch
import torch.nn.functional as F

import oracle
from tests.helpers import as_f64, bf16_bits, order_desc, rand_q, rand_tier

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _ulp_close(a, b, ulps=1):
    a = np.asarray(a, np.float32)
    b = np.asarray(b, np.float32)
    tol = ulps * np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float32))
    assert np.all(np.abs(a.astype(np.float64) - b.astype(np.float64)) <= tol), (
        f"max diff {np.max(np.abs(a.astype(np.float64) - b.astype(np.float64)))}")


# --------------------------------------------------------------------------- S1


def pin_score_single_head_is_matmul():
    """G = 1: z = fl32(scale * q K^T), numpy's float64 matmul (TS 2.B attention scores)."""
    rng = np.random.default_rng(11)
    B, H, n, D = 2, 3, 57, 64
    q = rand_q(rng, B, H, D)
    k, v, ln = rand_tier(rng, B, H, n, D)
    scale = 1 / math.sqrt(D)
    z = oracle.score(q, oracle.Tier(k, v, ln), scale)
    ref = np.einsum("bhd,bhnd->bhn", q.astype(np.float64), k.astype(np.float64)) * scale
    _ulp_close(z.reshape(B, H, n), ref.astype(np.float32))


def pin_score_gqa_maxpool_bf16_strided():
    """GQA groups and max pooling vs torch repeat_interleave + amax; bf16; odd strides."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, n, D = 2, 8, 2, 45, 128
    G = Hq // Hkv
    q = rand_q(rng, B, Hq, D, "bf16")
    k, v, ln = rand_tier(rng, B, Hkv, n, D, "bf16")
    scale = 0.37
    # store heads-outer, batch-inner, rows padded to D + 8 elements
    big_k = np.zeros((Hkv, B, n, D + 8), np.uint16)
    big_v = np.zeros((Hkv, B, n, D + 8), np.uint16)
    big_k[..., :D] = k.transpose(1, 0, 2, 3)
    big_v[..., :D] = v.transpose(1, 0, 2, 3)
    ks = big_k.transpose(1, 0, 2, 3)[..., :D]
    vs = big_v.transpose(1, 0, 2, 3)[..., :D]
    z = oracle.score(q, oracle.Tier(ks, vs, ln), scale)
    qt = torch.from_numpy(as_f64(q))
    kt = torch.repeat_interleave(torch.from_numpy(as_f64(k)), G, dim=1)
    logits = torch.einsum("bhd,bhnd->bhn", qt, kt) * scale
    ref = logits.view(B, Hkv, G, n).amax(dim=2).float().numpy()
    _ulp_close(z.reshape(B, Hkv, n), ref)


def pin_score_ragged_lengths():
    """Only the first len[u] scores of a unit are written."""
    rng = np.random.default_rng(13)
    B, H, n, D = 1, 3, 40, 64
    q = rand_q(rng, B, H, D)
    ln = np.array([0, 17, 40], np.int32)
    k, v, _ = rand_tier(rng, B, H, n, D)
    z = oracle.score(q, oracle.Tier(k, v, ln), 0.125)
    ref = np.einsum("bhd,bhnd->bhn", q.astype(np.float64), k.astype(np.float64)) * 0.125
    for u in range(H):
        _ulp_close(z[u, : ln[u]], ref[0, u, : ln[u]].astype(np.float32))
        assert np.all(z[u, ln[u]:] == 0)


# --------------------------------------------------------------------------- S2


def pin_calibration_is_softmax():
    """P = softmax(beta z) (scipy), sums to 1, logZ = logsumexp(beta (z - m)) (TS 2.B)."""
    rng = np.random.default_rng(21)
    units, n = 6, 300
    z = (rng.standard_normal((units, n)) * 2).astype(np.float32)
    ln = np.array([300, 299, 1, 150, 300, 7], np.int32)
    beta = np.array([1.0, 0.5, 3.0, 1.7, 0.25, 1.0], np.float32)
    P, m, lz = oracle.calibrate(z, ln, beta)
    for u in range(units):
        zz = z[u, : ln[u]].astype(np.float64)
        ref = sps.softmax(float(beta[u]) * zz)
        assert np.allclose(P[u, : ln[u]], ref, rtol=1e-6, atol=0)
        assert abs(np.sum(P[u, : ln[u]].astype(np.float64)) - 1.0) < 1e-6
        assert m[u] == z[u, : ln[u]].max()
        assert abs(lz[u] - sps.logsumexp(float(beta[u]) * (zz - zz.max()))) < 1e-6


def pin_calibration_special_cases():
    """beta = 0 gives the uniform distribution; -inf scores get no mass."""
    z = np.array([[3.0, -1.0, 0.5, 2.0], [1.0, -np.inf, 0.0, -np.inf]], np.float32)
    ln = np.array([4, 4], np.int32)
    P, m, lz = oracle.calibrate(z, ln, np.array([0.0, 1.0], np.float32))
    assert np.allclose(P[0], 0.25, rtol=0, atol=1e-7)
    assert P[1, 1] == 0 and P[1, 3] == 0
    assert np.allclose(P[1, [0, 2]], sps.softmax([1.0, 0.0]), rtol=1e-6)


def pin_calibration_order_invariant():
    """Calibration keeps the order of the scores (TS 2.B order-invariance)."""
    rng = np.random.default_rng(22)
    z = np.sort(rng.choice(np.arange(-400, 400), 200, replace=False))[::-1].astype(np.float32) / 50
    rng.shuffle(z)
    z = z[None, :]
    for beta in (0.5, 1.0, 3.0):
        P, _, _ = oracle.calibrate(z, np.array([200], np.int32), np.array([beta], np.float32))
        assert np.array_equal(np.argsort(-P[0], kind="stable"), np.argsort(-z[0], kind="stable"))


def pin_calibration_golden():
    """Hand-derived closed form: z = ln w gives P = w / sum(w) (tests/golden)."""
    with open(os.path.join(GOLDEN, "calibration_closed_form.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        z = np.array([case["z"]], np.float32)
        P, m, lz = oracle.calibrate(z, np.array([z.shape[1]], np.int32),
                                    np.array([case["beta"]], np.float32))
        assert np.allclose(P[0], case["P"], rtol=1e-6, atol=0), (P, case)
        assert abs(lz[0] - case["logZ"]) < 1e-6


# --------------------------------------------------------------------------- S3/S4


def _brute_force_selection(z, p, bmin, bmax, beta):
    """Minimum-cardinality subset with mass >= p, clamped, best by (z desc, idx asc)."""
    n = len(z)
    P = sps.softmax(beta * z.astype(np.float64))
    if p >= 1:
        kstar = n
    elif p <= 0:
        kstar = 0
    else:
        kstar = n
        for size in range(1, n + 1):
            best = max(sum(P[list(c)]) for c in itertools.combinations(range(n), size))
            if abs(best - p) < 1e-9:
                return None  # too close to call in any summation order
            if best >= p:
                kstar = size
                break
    k = min(n, max(bmin, min(kstar, bmax)))

    def rank_key(c):
        return sorted(((float(z[j]) + 0.0, -j) for j in c), reverse=True)

    best_set = max(itertools.combinations(range(n), k), key=rank_key) if k else ()
    return k, sorted(best_set)


def pin_topp_brute_force():
    """Top-p budget and set vs exhaustive search over all subsets (Abstract; TS 2.A)."""
    rng = np.random.default_rng(31)
    checked = 0
    for trial in range(160):
        n = int(rng.integers(1, 10))
        if trial % 3 == 0:
            z = (rng.integers(-3, 4, n) / 2).astype(np.float32)  # many ties
        else:
            z = (rng.standard_normal(n) * rng.uniform(0.2, 3)).astype(np.float32)
        p = float(np.float32(rng.choice([rng.uniform(0.05, 0.99), 1.0, 0.0])))
        bmin = int(rng.integers(0, 4))
        bmax = int(rng.integers(bmin, 12))
        beta = float(rng.choice([1.0, 0.5, 2.0]))
        ref = _brute_force_selection(z, p, bmin, bmax, beta)
        if ref is None:
            continue
        k_ref, set_ref = ref
        zz = z[None, :]
        ln = np.array([n], np.int32)
        be = np.array([beta], np.float32)
        r = oracle.topp(zz, ln, p, bmin, bmax, be)
        assert r["k"][0] == k_ref, (z, p, bmin, bmax, beta, r, k_ref)
        idx = oracle.compact(zz, ln, r["k"], max(bmax, 1))
        assert list(idx[0, :k_ref]) == set_ref
        assert np.all(idx[0, k_ref:] == -1)
        checked += 1
    assert checked > 100


def pin_topp_minimal_prefix():
    """C_{k*-1} < p <= C_{k*} with masses from numpy sort + cumsum (large n)."""
    rng = np.random.default_rng(32)
    units, n = 5, 3000
    z = (rng.standard_normal((units, n)) * np.array([[0.3], [1], [2], [4], [0.05]])).astype(np.float32)
    ln = np.full(units, n, np.int32)
    for p in (0.5, 0.8, 0.9, 0.95, 0.99):
        r = oracle.topp(z, ln, p, 0, n)
        for u in range(units):
            P = np.sort(sps.softmax(z[u].astype(np.float64)))[::-1]
            c = np.cumsum(P)
            ks = r["kstar"][u]
            assert c[ks - 1] >= p - 1e-12
            assert ks == 1 or c[ks - 2] < p + 1e-12
            assert r["k"][u] == ks


def pin_topp_clamps_and_extremes():
    """p = 1 keeps everything up to bmax; p = 0 keeps bmin; clamps cap at n."""
    rng = np.random.default_rng(33)
    z = rng.standard_normal((3, 50)).astype(np.float32)
    ln = np.array([50, 10, 0], np.int32)
    r = oracle.topp(z, ln, 1.0, 0, 64)
    assert list(r["k"]) == [50, 10, 0]
    r = oracle.topp(z, ln, 1.0, 0, 20)
    assert list(r["k"]) == [20, 10, 0]
    r = oracle.topp(z, ln, 0.0, 5, 20)
    assert list(r["k"]) == [5, 5, 0]
    r = oracle.topp(z, ln, 0.5, 12, 20)
    assert r["k"][1] == 10


def pin_topk_when_clamped_to_k():
    """bmin = bmax = k gives torch.topk's set, whatever beta (order-invariance, TS 2.B)."""
    rng = np.random.default_rng(34)
    n, k = 500, 37
    z = (rng.permutation(n) / 17.0 - 10).astype(np.float32)[None, :]
    ln = np.array([n], np.int32)
    want = sorted(torch.topk(torch.from_numpy(z[0]), k).indices.tolist())
    for beta in (0.1, 1.0, 5.0):
        for p in (0.3, 0.9):
            r = oracle.topp(z, ln, p, k, k, np.array([beta], np.float32))
            idx = oracle.compact(z, ln, r["k"], k)
            assert list(idx[0]) == want


def pin_ties_lower_index_first():
    """Equal scores (including -0 and +0) are taken in ascending token order."""
    z = np.array([[1.0, -0.0, 0.0, 1.0, 0.0, -0.0, 2.0, 0.0]], np.float32)
    ln = np.array([8], np.int32)
    idx = oracle.compact(z, ln, np.array([5], np.int32), 8)
    # 2.0 (6), 1.0 (0, 3), then zeros by index: 1, 2
    assert list(idx[0]) == [0, 1, 2, 3, 6, -1, -1, -1]


def pin_topp_golden():
    """Hand-derived budgets and sets (tests/golden/topp_closed_form.json)."""
    with open(os.path.join(GOLDEN, "topp_closed_form.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        z = np.array([case["z"]], np.float32)
        ln = np.array([z.shape[1]], np.int32)
        r = oracle.topp(z, ln, case["p"], case["bmin"], case["bmax"])
        assert r["k"][0] == case["k"], (case, r)
        idx = oracle.compact(z, ln, r["k"], case["bmax"])
        assert list(idx[0, : case["k"]]) == case["idx"], (case, idx)


def pin_compact_is_nonzero_gather():
    """Rows equal np.nonzero of the selection mask; FLAT_SUM = cumsum offsets (TS 2.C)."""
    rng = np.random.default_rng(41)
    units, n, bmax = 7, 200, 64
    z = rng.standard_normal((units, n)).astype(np.float32)
    ln = np.array([200, 0, 5, 199, 64, 100, 33], np.int32)
    k = np.array([64, 0, 5, 10, 64, 1, 33], np.int32)
    idx = oracle.compact(z, ln, k, bmax)
    flat, off = oracle.compact(z, ln, k, bmax, oracle.FLAT_SUM)
    assert list(off) == [0] + list(np.cumsum(k))
    for u in range(units):
        mask = np.zeros(n, bool)
        mask[order_desc(z[u, : ln[u]])[: k[u]]] = True
        want = np.nonzero(mask)[0]
        assert np.array_equal(idx[u, : k[u]], want)
        assert np.all(idx[u, k[u]:] == -1)
        assert np.array_equal(flat[off[u]: off[u + 1]], want)


def pin_gather_bit_copies():
    """Rewrite Cache rows are bit copies of K[idx], V[idx] (numpy fancy indexing)."""
    rng = np.random.default_rng(42)
    B, H, n, D, bmax = 2, 2, 90, 64, 16
    k, v, _ = rand_tier(rng, B, H, n, D, "bf16")
    ln = np.array([90, 80, 3, 90], np.int32)
    z = rng.standard_normal((B * H, n)).astype(np.float32)
    sel = np.array([16, 9, 3, 0], np.int32)
    idx = oracle.compact(z, ln, sel, bmax)
    kc, vc = oracle.gather(oracle.Tier(k, v, ln), idx, sel, bmax)
    kk = k.reshape(B * H, n, D)
    vv = v.reshape(B * H, n, D)
    for u in range(B * H):
        assert np.array_equal(kc[u, : sel[u]], kk[u, idx[u, : sel[u]]])
        assert np.array_equal(vc[u, : sel[u]], vv[u, idx[u, : sel[u]]])


# --------------------------------------------------------------------------- S5


def _sdpa(q, k, v, scale):
    """torch scaled_dot_product_attention in float64 with its own GQA mapping."""
    qt = torch.from_numpy(as_f64(q))[:, :, None, :]
    kt = torch.from_numpy(as_f64(k))
    vt = torch.from_numpy(as_f64(v))
    o = F.scaled_dot_product_attention(qt, kt, vt, scale=scale, enable_gqa=True)
    return o[:, :, 0, :].numpy()


def _lse(q, k, scale):
    G = q.shape[1] // k.shape[1]
    kt = torch.repeat_interleave(torch.from_numpy(as_f64(k)), G, dim=1)
    s = torch.einsum("bhd,bhnd->bhn", torch.from_numpy(as_f64(q)), kt) * scale
    return torch.logsumexp(s, dim=-1).numpy()


def pin_attention_dense_only_is_sdpa():
    """Dense-only step equals plain softmax attention (torch SDPA, float64)."""
    rng = np.random.default_rng(51)
    for dtype in ("f32", "bf16"):
        B, Hq, Hkv, W, D = 2, 8, 2, 70, 64
        q = rand_q(rng, B, Hq, D, dtype)
        k, v, ln = rand_tier(rng, B, Hkv, W, D, dtype)
        out, lse = oracle.attend(q, oracle.Tier(k, v, ln), None, None, None, 0, None, 0.125)
        assert np.allclose(out, _sdpa(q, k, v, 0.125), rtol=1e-6, atol=1e-7)
        assert np.allclose(lse, _lse(q, k, 0.125), rtol=1e-6, atol=1e-6)


def pin_step_p1_is_full_attention():
    """p = 1 with bmax >= n keeps every token and reproduces full attention."""
    rng = np.random.default_rng(52)
    B, Hq, Hkv, D = 1, 4, 2, 64
    W, n, Cn = 16, 100, 8
    q = rand_q(rng, B, Hq, D, "bf16")
    dk, dv, dl = rand_tier(rng, B, Hkv, W, D, "bf16")
    sk, sv, sl = rand_tier(rng, B, Hkv, n, D, "bf16")
    ck, cv, cl = rand_tier(rng, B, Hkv, Cn, D, "bf16")
    r = oracle.step(q, oracle.Tier(dk, dv, dl), oracle.Tier(sk, sv, sl), oracle.Tier(ck, cv, cl),
                    1 / 8, 1.0, 0, 128)
    assert list(r["k"]) == [n, n]
    kk = np.concatenate([dk, sk, ck], axis=2)
    vv = np.concatenate([dv, sv, cv], axis=2)
    assert np.allclose(r["out"], _sdpa(q, kk, vv, 1 / 8), rtol=1e-6, atol=1e-7)
    assert np.allclose(r["lse"], _lse(q, kk, 1 / 8), rtol=1e-6, atol=1e-6)


def pin_step_topk_set_attention():
    """bmin = bmax = k: attention over dense + torch.topk(z) tokens + condensed."""
    rng = np.random.default_rng(53)
    B, Hq, Hkv, D = 1, 4, 1, 64
    W, n, Cn, kk = 5, 300, 3, 20
    q = rand_q(rng, B, Hq, D)
    dk, dv, dl = rand_tier(rng, B, Hkv, W, D)
    sk, sv, sl = rand_tier(rng, B, Hkv, n, D)
    ck, cv, cl = rand_tier(rng, B, Hkv, Cn, D)
    r = oracle.step(q, oracle.Tier(dk, dv, dl), oracle.Tier(sk, sv, sl), oracle.Tier(ck, cv, cl),
                    0.125, 0.7, kk, kk)
    zmax = (np.einsum("bhd,bnd->bhn", q.astype(np.float64), sk[:, 0].astype(np.float64)) * 0.125).max(1)
    top = torch.topk(torch.from_numpy(zmax[0]), kk).indices.sort().values.numpy()
    assert np.array_equal(r["idx"][0, :kk], top)
    keys = np.concatenate([dk[:, :, :], sk[:, :, top], ck], axis=2)
    vals = np.concatenate([dv[:, :, :], sv[:, :, top], cv], axis=2)
    assert np.allclose(r["out"], _sdpa(q, keys, vals, 0.125), rtol=1e-6, atol=1e-7)


def pin_attention_tier_concatenation():
    """The output depends on the token multiset, not on which tier holds a token."""
    rng = np.random.default_rng(54)
    B, Hq, Hkv, D = 2, 4, 2, 64
    q = rand_q(rng, B, Hq, D)
    k, v, _ = rand_tier(rng, B, Hkv, 30, D)
    a = oracle.Tier(k[:, :, :10].copy(), v[:, :, :10].copy(), np.full(4, 10, np.int32))
    c = oracle.Tier(k[:, :, 10:].copy(), v[:, :, 10:].copy(), np.full(4, 20, np.int32))
    full = oracle.Tier(k, v, np.full(4, 30, np.int32))
    o1, l1 = oracle.attend(q, a, None, None, None, 0, c, 0.1)
    o2, l2 = oracle.attend(q, None, None, None, None, 0, full, 0.1, Hkv=Hkv)
    o3, l3 = oracle.attend(q, c, None, None, None, 0, a, 0.1)
    for o, lz in ((o2, l2), (o3, l3)):
        assert np.allclose(o1, o, rtol=1e-6, atol=1e-7)
        assert np.allclose(l1, lz, rtol=1e-6, atol=1e-6)


def pin_attention_empty_and_golden():
    """Empty token list -> out 0, lse -inf; hand-derived two-token case (tests/golden)."""
    q = np.ones((1, 2, 4), np.float32)
    k = np.zeros((1, 1, 3, 4), np.float32)
    t = oracle.Tier(k, k, np.zeros(1, np.int32))
    out, lse = oracle.attend(q, t, None, None, None, 0, None, 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    with open(os.path.join(GOLDEN, "attention_closed_form.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        q = np.array(case["q"], np.float32)[None, None, :]
        k = np.array(case["k"], np.float32)[None, None]
        v = np.array(case["v"], np.float32)[None, None]
        t = oracle.Tier(k, v, np.array([k.shape[2]], np.int32))
        out, lse = oracle.attend(q, t, None, None, None, 0, None, case["scale"])
        assert np.allclose(out[0, 0], case["out"], rtol=1e-6, atol=1e-6), (out, case)
        assert abs(lse[0, 0] - case["lse"]) < 1e-6


# ---- KV append (TS 2.A pipeline step 1) -----------------------------------------------


def pin_append_matches_list_model():
    """A run of appends against a plain Python model: per unit, a list of the
    window's tokens in arrival order (a token leaving the window goes to the
    end of the sparse list), compared as multisets of rows for the window
    (its slot order is the ring's) and in order for the sparse tier."""
    rng = np.random.default_rng(11)
    B, H, D, wcap, ncap = 2, 3, 8, 4, 6
    dense = oracle.Tier(np.zeros((B, H, wcap, D), np.float32), np.zeros((B, H, wcap, D), np.float32),
                        np.array([0, 2, 4, 4, 1, 3], np.int32))
    sparse = oracle.Tier(np.zeros((B, H, ncap, D), np.float32), np.zeros((B, H, ncap, D), np.float32),
                         np.array([0, 5, 0, 6, 2, 1], np.int32))
    # give the pre-filled slots distinct contents
    dense.k[...] = rng.standard_normal(dense.k.shape).astype(np.float32)
    dense.v[...] = rng.standard_normal(dense.v.shape).astype(np.float32)
    sparse.k[...] = rng.standard_normal(sparse.k.shape).astype(np.float32)
    sparse.v[...] = rng.standard_normal(sparse.v.shape).astype(np.float32)
    head = np.zeros(B * H, np.int32)
    # the model: window list (oldest first) and sparse list
    win = [[(dense.k[u // H, u % H, i].copy(), dense.v[u // H, u % H, i].copy()) for i in range(dense.len[u])]
           for u in range(B * H)]
    sp = [[(sparse.k[u // H, u % H, i].copy(), sparse.v[u // H, u % H, i].copy()) for i in range(sparse.len[u])]
          for u in range(B * H)]
    drops = 0
    for step in range(9):
        kn = rng.standard_normal((B, H, D)).astype(np.float32)
        vn = rng.standard_normal((B, H, D)).astype(np.float32)
        dense, head, sparse, dropped = oracle.append(kn, vn, dense, head, sparse)
        for u in range(B * H):
            win[u].append((kn[u // H, u % H], vn[u // H, u % H]))
            dropped_now = 0
            if len(win[u]) > wcap:
                old = win[u].pop(0)
                if len(sp[u]) < ncap:
                    sp[u].append(old)
                else:
                    dropped_now = 1
            drops += dropped_now
            assert dropped[u] == dropped_now, (step, u)
            assert dense.len[u] == len(win[u]) and sparse.len[u] == len(sp[u])
            rows = sorted(tuple(dense.k[u // H, u % H, i]) for i in range(dense.len[u]))
            assert rows == sorted(tuple(k) for k, _ in win[u]), (step, u)
            vrows = sorted(tuple(dense.v[u // H, u % H, i]) for i in range(dense.len[u]))
            assert vrows == sorted(tuple(v) for _, v in win[u]), (step, u)
            # the ring's head slot holds the oldest token once the window is full
            if dense.len[u] == wcap:
                assert np.array_equal(dense.k[u // H, u % H, head[u]], win[u][0][0])
            for i, (k, v) in enumerate(sp[u]):
                assert np.array_equal(sparse.k[u // H, u % H, i], k) and np.array_equal(sparse.v[u // H, u % H, i], v)
    assert drops > 0  # the run reaches full sparse tiers


def pin_append_without_window_goes_to_sparse():
    """W_cap = 0: every new token goes straight to the end of the sparse tier."""
    B, H, D = 1, 2, 4
    dense = oracle.Tier(np.zeros((B, H, 0, D), np.float32), np.zeros((B, H, 0, D), np.float32),
                        np.zeros(B * H, np.int32))
    sparse = oracle.Tier(np.zeros((B, H, 3, D), np.float32), np.zeros((B, H, 3, D), np.float32),
                         np.array([1, 3], np.int32))
    kn = np.arange(B * H * D, dtype=np.float32).reshape(B, H, D)
    d2, hd, s2, dropped = oracle.append(kn, -kn, dense, np.zeros(B * H, np.int32), sparse)
    assert list(s2.len) == [2, 3] and list(dropped) == [0, 1]
    assert np.array_equal(s2.k[0, 0, 1], kn[0, 0]) and np.array_equal(s2.v[0, 0, 1], -kn[0, 0])


# ---- Fitted temperature (TS 2.B, TS 3, TS 2.A Tier 2 "attention entropy") ----------------


def _entropy_ref(x):
    """Entropy of softmax(x) by library routines (scipy), not the oracle's code."""
    import scipy.special as sps
    import scipy.stats as sst

    return float(sst.entropy(sps.softmax(np.asarray(x, np.float64))))


def pin_attention_entropy_matches_scipy():
    """Group-averaged raw-attention entropy against torch float64 logits and
    scipy's softmax and entropy, on bf16 (exact widening by torch) and fp32
    inputs with GQA groups and ragged lengths."""
    import torch

    rng = np.random.default_rng(21)
    # the last case has logits spread over hundreds (exp overflows without the max shift)
    for dt, spread in ((torch.bfloat16, 2.0), (torch.float32, 2.0), (torch.float32, 400.0)):
        B, Hkv, G, D, cap = 2, 2, 4, 16, 40
        q = torch.as_tensor(rng.standard_normal((B, Hkv * G, D)), dtype=torch.float32).to(dt)
        k = torch.as_tensor(rng.standard_normal((B, Hkv, cap, D)) * spread, dtype=torch.float32).to(dt)
        ln = np.array([40, 17, 1, 0], np.int32)
        scale = 0.3
        def host(x):
            return x.view(torch.int16).numpy().view(np.uint16) if x.dtype == torch.bfloat16 else x.numpy()

        t = oracle.Tier(host(k), host(k), ln)
        got = oracle.attention_entropy(host(q), t, scale)
        qd, kd = q.double(), k.double()
        for u in range(B * Hkv):
            b, h = divmod(u, Hkv)
            n = int(ln[u])
            if n == 0:
                assert got[u] == 0.0
                continue
            lg = scale * torch.einsum("gd,nd->gn", qd[b, h * G:(h + 1) * G], kd[b, h, :n]).numpy()
            want = np.mean([_entropy_ref(lg[g]) for g in range(G)])
            assert abs(got[u] - want) <= 1e-12 * max(1.0, want), (dt, u, got[u], want)


def pin_attention_entropy_of_equal_keys_is_log_n():
    """Keys all equal: every head attends uniformly, so the entropy is ln n."""
    B, Hkv, G, D, n = 1, 1, 2, 8, 37
    q = np.random.default_rng(3).standard_normal((B, Hkv * G, D)).astype(np.float32)
    k = np.tile(np.linspace(-1, 1, D, dtype=np.float32), (B, Hkv, n, 1))
    got = oracle.attention_entropy(q, oracle.Tier(k, k, np.array([n], np.int32)), 1.0)
    assert abs(got[0] - np.log(n)) < 1e-12


def pin_fit_identical_heads_gives_one():
    """A group of identical query heads: the max-pooled logits are each head's
    raw logits, so the temperature that matches their entropy is 1."""
    rng = np.random.default_rng(5)
    B, Hkv, G, D, cap = 1, 2, 4, 32, 300
    q1 = rng.standard_normal((B, Hkv, 1, D)).astype(np.float32)
    q = np.repeat(q1, G, axis=2).reshape(B, Hkv * G, D)
    k = (rng.standard_normal((B, Hkv, cap, D)) * 1.5).astype(np.float32)
    ln = np.array([300, 123], np.int32)
    t = oracle.Tier(k, k, ln)
    scale = 1.0 / np.sqrt(D)
    z = np.einsum("bhd,bhnd->bhn", q1[:, :, 0].astype(np.float64), k.astype(np.float64)).reshape(B * Hkv, cap)
    beta = oracle.fit_temperature(scale * z, ln, oracle.attention_entropy(q, t, scale))
    assert np.all(np.abs(beta - 1.0) < 1e-9), beta


def pin_fit_two_tokens_closed_form():
    """Two tokens a gap d apart: softmax(beta z) is Bernoulli(1/(1+e^(-beta d))),
    whose entropy is the binary entropy; the fit inverts it."""
    for d, b0 in ((1.0, 0.5), (3.0, 2.25), (0.2, 9.0), (5.0, 0.01)):
        pr = 1.0 / (1.0 + np.exp(-b0 * d))
        h = -(pr * np.log(pr) + (1 - pr) * np.log(1 - pr))
        beta = oracle.fit_temperature(np.array([[0.0, d]]), np.array([2]), np.array([h]))
        assert abs(beta[0] - b0) < 1e-9 * max(1.0, b0), (d, b0, beta)


def pin_fit_matches_brentq():
    """Random metrics and reachable targets: the same root as scipy's brentq on
    scipy's entropy of scipy's softmax."""
    from scipy.optimize import brentq

    rng = np.random.default_rng(9)
    units, cap = 6, 500
    z = (rng.standard_normal((units, cap)) * rng.uniform(0.2, 3.0, (units, 1))).astype(np.float32)
    ln = np.array([500, 2, 77, 300, 499, 10], np.int32)
    tgt = np.array([rng.uniform(0.05, 0.95) * np.log(n) for n in ln])
    beta = oracle.fit_temperature(z, ln, tgt)
    for u in range(units):
        zu = z[u, :ln[u]].astype(np.float64)
        f = lambda b: _entropy_ref(b * zu) - tgt[u]
        if f(oracle.FIT_BETA_MAX) > 0:
            assert beta[u] == oracle.FIT_BETA_MAX
            continue
        want = brentq(f, 0.0, oracle.FIT_BETA_MAX, xtol=1e-14, rtol=1e-14)
        assert abs(beta[u] - want) < 1e-9 * max(1.0, want), (u, beta[u], want)


def pin_fit_boundaries_and_order():
    """Targets at or above ln n give 0; below the entropy at the largest beta
    give that beta; n <= 1 and constant metrics give 1; a larger target never
    gives a larger beta."""
    z = np.array([[0.0, 1.0, 3.0, 3.0, -2.0], [1.0, 1.0, 1.0, 1.0, 1.0], [4.0, 0, 0, 0, 0]])
    n = np.array([5, 5, 1])
    b = oracle.fit_temperature(z, n, np.array([np.log(5) + 1e-3, 0.3, 0.0]))
    assert list(b) == [0.0, 1.0, 1.0]
    b = oracle.fit_temperature(z[:1], n[:1], np.array([1e-30]))
    assert b[0] == oracle.FIT_BETA_MAX
    ts = np.linspace(0.75, 1.55, 9)
    bs = [oracle.fit_temperature(z[:1], n[:1], np.array([t]))[0] for t in ts]
    assert all(x > y for x, y in zip(bs, bs[1:])), bs
    # ties at the top: the entropy falls to ln 2, not 0, so a lower target is out of reach
    assert oracle.fit_temperature(z[:1], n[:1], np.array([np.log(2) - 1e-6]))[0] == oracle.FIT_BETA_MAX


# ---- Condensed-tier formation (TS 2.A Tier 3 and pipeline step 4) -----------------------


def _nearest_bf16_exact(x: float) -> float:
    """The bf16 value nearest x (ties to an even last mantissa bit), by exact
    rational arithmetic over the neighbouring representable values."""
    from fractions import Fraction

    fx = Fraction(x)
    if fx == 0:
        return 0.0
    sign = -1 if fx < 0 else 1
    a = abs(fx)
    e = math.floor(math.log2(a))
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    step = Fraction(2) ** max(e - 7, -133)  # 8 significant bits; fixed spacing below 2^-126
    lo = (a // step) * step
    hi = lo + step
    if a - lo < hi - a:
        r = lo
    elif hi - a < a - lo:
        r = hi
    else:
        r = lo if (lo / step) % 2 == 0 else hi
    return sign * float(r)


def pin_round_to_bf16_is_nearest_even():
    """Rounding a double to bf16 gives the nearest bf16 value, ties to even,
    by exact rational arithmetic; this includes doubles that a detour through
    float32 would round to a tie and then the wrong way."""
    rng = np.random.default_rng(31)
    xs = list(rng.standard_normal(300) * np.exp(rng.uniform(-20, 20, 300)))
    xs += [1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, 1 + 2.0 ** -8 + 2.0 ** -40, 1 + 2.0 ** -8 - 2.0 ** -40,
           -(1 + 2.0 ** -8 + 2.0 ** -40), 2.0 ** -130 * 1.37, 3.0e38, 0.0]
    got = oracle.round_to_bf16(np.array(xs))
    want = bf16_bits(np.array([_nearest_bf16_exact(x) for x in xs], np.float32))
    assert np.array_equal(got, want), [(x, g, w) for x, g, w in zip(xs, got, want) if g != w][:3]


def _calibrated(z, beta):
    """m, logZ and the calibrated probabilities of scores z (scipy)."""
    z64 = z.astype(np.float64)
    m = np.float32(z64.max())
    lz = sps.logsumexp(beta * (z64 - np.float64(m)))
    return m, np.float32(lz), sps.softmax(beta * z64)


def _cond_state(rng, B, H, ncap, ccap, D, n, C, dtype="f32"):
    k, v, _ = rand_tier(rng, B, H, ncap, D, dtype)
    ck, cv, _ = rand_tier(rng, B, H, ccap, D, dtype)
    sp = oracle.Tier(k, v, np.asarray(n, np.int32))
    co = oracle.Tier(ck, cv, np.asarray(C, np.int32))
    w = rng.uniform(0.0, 1.0, (B * H, ccap)).astype(np.float32)
    return sp, co, w


def pin_condense_merge_is_weighted_average():
    """MERGE: the new condensed slot is numpy's weighted average of the oldest
    block's rows, weighted by the calibrated probabilities (scipy softmax);
    its weight is the block's mass."""
    rng = np.random.default_rng(32)
    B, H, ncap, ccap, D, block = 1, 3, 40, 5, 16, 7
    sp, co, w = _cond_state(rng, B, H, ncap, ccap, D, [40, 33, 7], [0, 2, 4])
    z = rng.standard_normal((B * H, ncap)).astype(np.float32) * 3
    beta = np.array([1.0, 0.5, 2.0], np.float32)
    m = np.zeros(B * H, np.float32)
    lz = np.zeros(B * H, np.float32)
    P = []
    for u in range(B * H):
        m[u], lz[u], Pu = _calibrated(z[u, :sp.len[u]], float(beta[u]))
        P.append(Pu)
    s2, c2, w2, done = oracle.condense(sp, co, w, z, m, lz, beta, block, block, oracle.CONDENSE_MERGE)
    assert list(done) == [1, 1, 1]
    for u in range(B * H):
        C = int(co.len[u])
        a = P[u][:block]
        for t_in, t_out in ((sp.k, c2.k), (sp.v, c2.v)):
            ref = np.average(t_in[0, u, :block].astype(np.float64), axis=0, weights=a).astype(np.float32)
            _ulp_close(t_out[0, u, C], ref)
        assert abs(float(w2[u, C]) - a.sum()) <= 1e-6 * a.sum()
        assert c2.len[u] == C + 1
        # earlier slots untouched
        assert np.array_equal(c2.k[0, u, :C], co.k[0, u, :C]) and np.array_equal(w2[u, :C], w[u, :C])


def pin_condense_matches_list_model():
    """A run of condensations against a plain Python model: per unit the sparse
    tier as a list of rows in age order and the condensed tier as a list of
    (row, weight); blocks leave from the old end; a full condensed tier first
    merges its two oldest slots (MERGE, numpy weighted average) or drops its
    oldest (EVICT); EVICT keeps the block's first highest-scoring token."""
    rng = np.random.default_rng(33)
    for policy in (oracle.CONDENSE_MERGE, oracle.CONDENSE_EVICT):
        B, H, ncap, ccap, D, block, trig = 1, 2, 30, 3, 8, 4, 10
        sp, co, w = _cond_state(rng, B, H, ncap, ccap, D, [30, 12], [1, 3])
        model_s = [[(sp.k[0, u, i].copy(), sp.v[0, u, i].copy()) for i in range(sp.len[u])] for u in range(2)]
        model_c = [[(co.k[0, u, i].copy(), co.v[0, u, i].copy(), np.float64(w[u, i])) for i in range(co.len[u])]
                   for u in range(2)]
        for rnd in range(7):
            z = np.round(rng.standard_normal((2, ncap)) * 2).astype(np.float32)  # ties happen
            m = np.zeros(2, np.float32)
            lz = np.zeros(2, np.float32)
            Ps = []
            for u in range(2):
                n = int(sp.len[u])
                if n:
                    m[u], lz[u], Pu = _calibrated(z[u, :n], 1.0)
                else:
                    Pu = np.zeros(0)
                Ps.append(Pu)
            sp, co, w, done = oracle.condense(sp, co, w, z, m, lz, None, block, trig, policy)
            for u in range(2):
                if len(model_s[u]) >= max(trig, block):
                    assert done[u] == 1
                    blk = model_s[u][:block]
                    model_s[u] = model_s[u][block:]
                    a = Ps[u][:block]
                    if policy == oracle.CONDENSE_MERGE:
                        if len(model_c[u]) == ccap:
                            (k0, v0, w0), (k1, v1, w1) = model_c[u][0], model_c[u][1]
                            ww = np.array([w0, w1])
                            mk = np.average(np.stack([k0, k1]).astype(np.float64), axis=0, weights=ww)
                            mv = np.average(np.stack([v0, v1]).astype(np.float64), axis=0, weights=ww)
                            model_c[u] = [(mk.astype(np.float32), mv.astype(np.float32), w0 + w1)] + model_c[u][2:]
                        nk = np.average(np.stack([r[0] for r in blk]).astype(np.float64), axis=0, weights=a)
                        nv = np.average(np.stack([r[1] for r in blk]).astype(np.float64), axis=0, weights=a)
                        model_c[u].append((nk.astype(np.float32), nv.astype(np.float32), a.sum()))
                    else:
                        if len(model_c[u]) == ccap:
                            model_c[u] = model_c[u][1:]
                        j = int(np.flatnonzero(z[u, :block] == z[u, :block].max())[0])
                        model_c[u].append((blk[j][0], blk[j][1], a[j]))
                else:
                    assert done[u] == 0
                assert sp.len[u] == len(model_s[u]) and co.len[u] == len(model_c[u]), (policy, rnd, u)
                for i, (kk, vv) in enumerate(model_s[u]):
                    assert np.array_equal(sp.k[0, u, i], kk) and np.array_equal(sp.v[0, u, i], vv)
                for i, (kk, vv, ww) in enumerate(model_c[u]):
                    # weights are known to about 1e-7 relative (the model keeps
                    # float64 masses, the tier float32 ones), and a mean moves
                    # by at most that times the spread of its rows
                    for got, want in ((co.k[0, u, i], kk), (co.v[0, u, i], vv)):
                        err = np.abs(got.astype(np.float64) - np.asarray(want, np.float64))
                        assert np.all(err <= 1e-6 * (1 + np.abs(want))), (policy, rnd, u, i, err.max())
                    assert abs(float(w[u, i]) - ww) <= 1e-5 * max(ww, 1e-30), (policy, rnd, u, i)


def pin_condense_noop_drop_and_single_slot():
    """Below the trigger nothing changes; a condensed tier of capacity 0 drops
    the block; with one slot, MERGE folds the block into it (numpy weighted
    average of the slot, weighted by its weight, and the block's rows)."""
    rng = np.random.default_rng(34)
    sp, co, w = _cond_state(rng, 1, 2, 20, 1, 8, [9, 20], [1, 1])
    z = rng.standard_normal((2, 20)).astype(np.float32)
    m = np.array([z[0, :9].max(), z[1].max()], np.float32)
    lz = np.array([sps.logsumexp(z[0, :9] - m[0]), sps.logsumexp(z[1] - m[1])], np.float32)
    s2, c2, w2, done = oracle.condense(sp, co, w, z, m, lz, None, 5, 10, oracle.CONDENSE_MERGE)
    assert list(done) == [0, 1] and list(s2.len) == [9, 15] and list(c2.len) == [1, 1]
    assert np.array_equal(s2.k[0, 0], sp.k[0, 0]) and np.array_equal(c2.k[0, 0], co.k[0, 0])
    a = np.concatenate([[np.float64(w[1, 0])], np.exp(z[1, :5].astype(np.float64) - m[1] - np.float64(lz[1]))])
    rows = np.concatenate([co.k[0, 1, :1], sp.k[0, 1, :5]]).astype(np.float64)
    _ulp_close(c2.k[0, 1, 0], np.average(rows, axis=0, weights=a).astype(np.float32))
    assert np.array_equal(s2.k[0, 1, :15], sp.k[0, 1, 5:20])
    empty = oracle.Tier(np.zeros((1, 2, 0, 8), np.float32), np.zeros((1, 2, 0, 8), np.float32),
                        np.zeros(2, np.int32))
    s3, c3, w3, done = oracle.condense(sp, empty, np.zeros((2, 0), np.float32), z, m, lz, None, 5, 5,
                                       oracle.CONDENSE_EVICT)
    assert list(done) == [1, 1] and list(s3.len) == [4, 15] and list(c3.len) == [0, 0]
    assert np.array_equal(s3.v[0, 0, :4], sp.v[0, 0, 5:9])


def pin_condense_bf16_merge_exact():
    """bf16 tiers: each merged element is the nearest bf16 value (ties to even,
    exact rational arithmetic) to the exact weighted mean of the block, when
    the mean is not within 1e-12 of a rounding tie."""
    from fractions import Fraction

    rng = np.random.default_rng(35)
    sp, co, w = _cond_state(rng, 1, 1, 12, 4, 16, [12], [0], "bf16")
    z = rng.standard_normal((1, 12)).astype(np.float32)
    m = np.array([z[0].max()], np.float32)
    lz = np.array([sps.logsumexp(z[0] - m[0])], np.float32)
    s2, c2, w2, _ = oracle.condense(sp, co, w, z, m, lz, None, 6, 6, oracle.CONDENSE_MERGE)
    a = np.exp(z[0, :6].astype(np.float64) - np.float64(m[0]) - np.float64(lz[0]))
    for t_in, t_out in ((sp.k, c2.k), (sp.v, c2.v)):
        rows = as_f64(t_in[0, 0, :6])
        for d in range(16):
            exact = sum(Fraction(float(a[j])) * Fraction(float(rows[j, d])) for j in range(6)) / \
                sum(Fraction(float(x)) for x in a)
            want = _nearest_bf16_exact(float(exact))
            got = as_f64(t_out[0, 0, 0:1])[0, d]
            if got != want:
                # the float64 sums may only move a value that sits at a tie
                spacing = abs(want) * 2.0 ** -8
                assert abs(abs(float(exact) - want) - spacing / 2) <= 1e-12 * abs(want), (d, got, want)


# ---- Rewrite Cache vs Sparse Loading (TS 2.C Trade-off Management) ------------------------


def pin_mti_trigger_and_horizon():
    """The trigger is a hysteresis on the budget: above L_upper rewrite, below
    L_lower sparse loading, in between the previous mode; a rewrite of k rows
    serves the largest H >= 1 with k H within the memory-time allowance
    (brute force)."""
    R, S = oracle.MODE_REWRITE, oracle.MODE_SPARSE
    table = [(5, S, 10, 20, S), (5, R, 10, 20, S), (10, R, 10, 20, R), (10, S, 10, 20, S), (15, R, 10, 20, R),
             (20, S, 10, 20, S), (21, S, 10, 20, R), (21, R, 10, 20, R), (0, R, 0, 0, R), (1, S, 0, 0, R)]
    for k, mode, lo, hi, want in table:
        assert oracle.mti_trigger(k, mode, lo, hi) == want, (k, mode, lo, hi)
    for k in range(1, 70):
        for cap in (0, 1, 63, 64, 65, 1000, 4096):
            best = max([h for h in range(1, 5000) if k * h <= cap] or [1])
            assert oracle.mti_horizon(k, cap) == best, (k, cap)
    assert oracle.mti_horizon(0, 100) == 1


def _mti_case(seed, dtype="f32"):
    rng = np.random.default_rng(seed)
    B, Hkv, G, D, n, W, C = 1, 3, 2, 16, 40, 5, 3
    q = rand_q(rng, B, Hkv * G, D, dtype)
    tiers = [oracle.Tier(*rand_tier(rng, B, Hkv, cap, D, dtype)) for cap in (W, n, C)]
    return rng, q, tiers


def pin_mti_reuse_attends_the_rewritten_rows():
    """A unit whose rewrite still serves attends over dense ++ its rewritten
    rows ++ condensed (torch SDPA over the concatenation), reports those rows'
    indices, and counts one step down; the others run the plain step."""
    rng, q, (dense, sparse, cond) = _mti_case(41)
    B, Hkv, D, bmax = 1, 3, 16, 12
    scale = 1 / math.sqrt(D)
    st = oracle.mti_state(3, bmax, B, Hkv, D, sparse.k)
    st["left"][:] = [2, 0, 1]
    st["rw_len"][:] = [7, 0, 12]
    st["rw_k"][...] = rng.standard_normal(st["rw_k"].shape).astype(np.float32)
    st["rw_v"][...] = rng.standard_normal(st["rw_v"].shape).astype(np.float32)
    st["rw_idx"][:] = rng.integers(0, 40, (3, bmax))
    res, st2 = oracle.step_mti(q, dense, sparse, cond, scale, 0.9, 2, bmax, st, 4, 8, 100)
    assert list(res["fresh"]) == [0, 1, 0] and list(st2["left"][[0, 2]]) == [1, 0]
    for u in (0, 2):
        n = int(st["rw_len"][u])
        k = np.concatenate([dense.k[0, u], st["rw_k"][0, u, :n], cond.k[0, u]]).astype(np.float64)
        v = np.concatenate([dense.v[0, u], st["rw_v"][0, u, :n], cond.v[0, u]]).astype(np.float64)
        qq = torch.from_numpy(q[0, 2 * u:2 * u + 2].astype(np.float64))
        ref = F.scaled_dot_product_attention(qq[None, :, None, :], torch.from_numpy(k)[None, None].expand(1, 2, -1, -1),
                                             torch.from_numpy(v)[None, None].expand(1, 2, -1, -1), scale=scale)
        assert np.allclose(res["out"][0, 2 * u:2 * u + 2], ref[0, :, 0].numpy(), atol=1e-6)
        assert res["k"][u] == n and np.array_equal(res["idx"][u, :n], st["rw_idx"][u, :n])
        assert np.all(res["idx"][u, n:] == -1)
    plain = oracle.step(q, dense, sparse, cond, scale, 0.9, 2, bmax)
    assert np.array_equal(res["out"][0, 2:4], plain["out"][0, 2:4]) and res["k"][1] == plain["k"][1]


def pin_mti_rewrite_copies_the_top_rows():
    """A fresh unit whose budget crosses L_upper copies its selected rows: the
    rows of the top-k tokens by (score desc, index asc) from numpy's own sort,
    in token order (numpy fancy indexing); one whose budget falls below L_lower
    drops its rewrite."""
    rng, q, (dense, sparse, cond) = _mti_case(42)
    B, Hkv, D, bmax = 1, 3, 16, 6
    scale = 1 / math.sqrt(D)
    st = oracle.mti_state(3, bmax, B, Hkv, D, sparse.k)
    st["mode"][:] = [0, 1, 1]
    st["rw_len"][:] = [0, 3, 3]
    # budgets: bmin = bmax = 6 makes every fresh budget 6
    res, st2 = oracle.step_mti(q, dense, sparse, cond, scale, 0.5, bmax, bmax, st, 4, 5, 60)
    assert list(st2["mode"]) == [1, 1, 1] and list(st2["rw_len"]) == [6, 6, 6] and list(st2["left"]) == [9, 9, 9]
    qf = q.astype(np.float64).reshape(1, 3, 2, 16)
    for u in range(3):
        z = (np.einsum("gd,nd->gn", qf[0, u], sparse.k[0, u].astype(np.float64)) * scale).max(axis=0)
        top = np.sort(order_desc(z.astype(np.float32))[:6])
        assert np.array_equal(st2["rw_idx"][u, :6], top)
        assert np.array_equal(st2["rw_k"][0, u, :6], sparse.k[0, u][top])
        assert np.array_equal(st2["rw_v"][0, u, :6], sparse.v[0, u][top])
    res3, st3 = oracle.step_mti(q, dense, sparse, cond, scale, 1e-4, 1, bmax,
                                st2 | {"left": np.zeros(3, np.int32)}, 4, 5, 60)
    assert np.all(res3["k"] < 4)
    assert list(st3["mode"]) == [0, 0, 0] and list(st3["rw_len"]) == [0, 0, 0] and list(st3["left"]) == [0, 0, 0]


def pin_mti_state_matches_model():
    """Many steps with scripted budgets against a plain model of the trigger:
    per unit a mode and a count of steps left, a rewrite served H(k) steps."""
    rng, q, (dense, sparse, cond) = _mti_case(43)
    B, Hkv, D, bmax = 1, 3, 16, 30
    scale = 1 / math.sqrt(D)
    lo, hi, cap = 8, 20, 90
    st = oracle.mti_state(3, bmax, B, Hkv, D, sparse.k)
    model = [[0, 0, 0] for _ in range(3)]  # mode, left, rows
    for step_i in range(40):
        kf = rng.integers(0, 31, 3).astype(np.int32)
        idf = np.stack([np.sort(rng.choice(40, bmax, replace=False)).astype(np.int32) for _ in range(3)])
        res, st = oracle.step_mti(q, dense, sparse, cond, scale, 0.9, 1, bmax, st, lo, hi, cap, kf, idf)
        for u in range(3):
            mode, left, rows = model[u]
            if left > 0:
                assert res["fresh"][u] == 0 and res["k"][u] == rows
                model[u] = [mode, left - 1, rows]
            else:
                assert res["fresh"][u] == 1
                k = int(kf[u])
                mode = 1 if k > hi else (0 if k < lo else mode)
                model[u] = [mode, (max(1, cap // k) - 1) if (mode and k) else 0, k if mode else 0]
                if mode:
                    assert np.array_equal(st["rw_idx"][u, :k], idf[u, :k])
            assert [int(st["mode"][u]), int(st["left"][u]), int(st["rw_len"][u])] == model[u], (step_i, u)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
