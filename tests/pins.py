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


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_") and callable(v)]
