"""CPU oracle of one HARD-KV Cascade Cache decode step (numpy in, numpy out).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package. The CUDA library and its
Python binding never import it; the two implementations share no code.

The arithmetic of S1-S5 lives in ``hkv_oracle.c`` (plain C, IEEE double) and
this module only marshals arrays for it; the KV append and the fitted
temperature, further down, are plain numpy (float64 for the arithmetic).
bf16 tensors travel as their raw 16-bit patterns (``numpy.uint16``); fp32
tensors as ``numpy.float32``.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import build as _build

BF16, F32 = 0, 1
PAD_MAX, FLAT_SUM = 0, 1

_lib = None


def lib(path: Optional[str] = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if path is not None:
        return _bind(C.CDLL(path))
    if _lib is None:
        _lib = _bind(C.CDLL(_build.build()))
    return _lib


class _Tier(C.Structure):
    _fields_ = [
        ("k", C.c_void_p), ("v", C.c_void_p),
        ("sb", C.c_int64), ("sh", C.c_int64), ("st", C.c_int64),
        ("cap", C.c_int32), ("len", C.c_void_p),
    ]


class _Dims(C.Structure):
    _fields_ = [
        ("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("D", C.c_int32),
        ("dtype", C.c_int32), ("scale", C.c_double),
    ]


def _bind(L):
    P = C.c_void_p
    i32 = C.c_int32
    L.hkvo_score.argtypes = [P, P, P, P, i32]
    L.hkvo_calibrate.argtypes = [i32, P, i32, P, P, P, P, P]
    L.hkvo_topp.argtypes = [i32, P, i32, P, P, C.c_float, P, i32, i32, P, P, P, P]
    L.hkvo_compact.argtypes = [i32, P, i32, P, P, i32, i32, P, P]
    L.hkvo_gather.argtypes = [P, P, P, P, i32, P, P]
    L.hkvo_attend.argtypes = [P, P, P, P, P, P, i32, P, P, P]
    L.hkvo_step.argtypes = [P, P, P, P, P, P, C.c_float, P, i32, i32, P, P, P, P, P]
    for f in ("hkvo_score", "hkvo_calibrate", "hkvo_topp", "hkvo_compact", "hkvo_gather",
              "hkvo_attend", "hkvo_step", "hkvo_num_threads"):
        getattr(L, f).restype = C.c_int
    return L


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle takes uint16 (bf16 bits) or float32, got {a.dtype}")


@dataclass
class Tier:
    """One cache tier: K, V of shape [B, Hkv, cap, D] (D contiguous) and len[B*Hkv]."""

    k: np.ndarray
    v: np.ndarray
    len: np.ndarray

    def c(self, keep: list) -> _Tier:
        k, v = self.k, self.v
        ln = np.ascontiguousarray(self.len, dtype=np.int32)
        if k.size == 0:  # an empty tier (numpy gives empty arrays arbitrary strides)
            keep += [k, ln]
            B, H, _, D = k.shape
            return _Tier(k.ctypes.data, k.ctypes.data, H * D, D, D, 0, ln.ctypes.data)
        assert k.shape == v.shape and k.strides == v.strides and k.ndim == 4
        assert k.strides[3] == k.itemsize, "D must be contiguous"
        keep += [k, v, ln]
        es = k.itemsize
        return _Tier(k.ctypes.data, v.ctypes.data, k.strides[0] // es, k.strides[1] // es,
                     k.strides[2] // es, k.shape[2], ln.ctypes.data)


def _dims(q: np.ndarray, Hkv: int, scale: float) -> _Dims:
    B, Hq, D = q.shape
    return _Dims(B, Hq, Hkv, D, _dtype_code(q), float(scale))


def _ck(r: int, what: str):
    if r != 0:
        raise ValueError(f"oracle {what} failed with code {r}")


def score(q: np.ndarray, sparse: Tier, scale: float) -> np.ndarray:
    """S1: z[B*Hkv, cap] (entries past len are left at 0)."""
    keep: list = []
    q = np.ascontiguousarray(q)
    t = sparse.c(keep)
    d = _dims(q, sparse.k.shape[1], scale)
    z = np.zeros((d.B * d.Hkv, t.cap), np.float32)
    _ck(lib().hkvo_score(C.byref(d), _ptr(q), C.byref(t), _ptr(z), t.cap), "score")
    return z


def calibrate(z: np.ndarray, length: np.ndarray, beta: Optional[np.ndarray] = None,
              want_P: bool = True):
    """S2: (P or None, m, logZ) per unit."""
    z = np.ascontiguousarray(z, np.float32)
    ln = np.ascontiguousarray(length, np.int32)
    units, zcap = z.shape
    be = None if beta is None else np.ascontiguousarray(beta, np.float32)
    P = np.zeros_like(z) if want_P else None
    m = np.zeros(units, np.float32)
    lz = np.zeros(units, np.float32)
    _ck(lib().hkvo_calibrate(units, _ptr(z), zcap, _ptr(ln), _ptr(be), _ptr(P), _ptr(m),
                             _ptr(lz)), "calibrate")
    return P, m, lz


def topp(z: np.ndarray, length: np.ndarray, p: float, bmin: int, bmax: int,
         beta: Optional[np.ndarray] = None, p_unit: Optional[np.ndarray] = None) -> dict:
    """S3: dict(k, kstar, c_before, c_at) per unit."""
    z = np.ascontiguousarray(z, np.float32)
    ln = np.ascontiguousarray(length, np.int32)
    units, zcap = z.shape
    be = None if beta is None else np.ascontiguousarray(beta, np.float32)
    pu = None if p_unit is None else np.ascontiguousarray(p_unit, np.float32)
    k = np.zeros(units, np.int32)
    ks = np.zeros(units, np.int32)
    cb = np.zeros(units, np.float64)
    ca = np.zeros(units, np.float64)
    _ck(lib().hkvo_topp(units, _ptr(z), zcap, _ptr(ln), _ptr(be), float(p), _ptr(pu), int(bmin),
                        int(bmax), _ptr(k), _ptr(ks), _ptr(cb), _ptr(ca)), "topp")
    return {"k": k, "kstar": ks, "c_before": cb, "c_at": ca}


def compact(z: np.ndarray, length: np.ndarray, sel_len: np.ndarray, bmax: int,
            layout: int = PAD_MAX):
    """S4: PAD_MAX -> idx[units, bmax]; FLAT_SUM -> (flat idx, offsets[units+1])."""
    z = np.ascontiguousarray(z, np.float32)
    ln = np.ascontiguousarray(length, np.int32)
    k = np.ascontiguousarray(sel_len, np.int32)
    units, zcap = z.shape
    if layout == PAD_MAX:
        idx = np.zeros((units, bmax), np.int32)
        off = None
    else:
        idx = np.full(max(int(k.sum()), 1), -7, np.int32)
        off = np.zeros(units + 1, np.int32)
    _ck(lib().hkvo_compact(units, _ptr(z), zcap, _ptr(ln), _ptr(k), int(bmax), int(layout),
                           _ptr(idx), _ptr(off)), "compact")
    if layout == PAD_MAX:
        return idx
    return idx[: int(off[-1])], off


def gather(sparse: Tier, idx: np.ndarray, sel_len: np.ndarray, bmax: int, Hq: int = 1):
    """S4 Rewrite Cache: (Kc, Vc) of shape [units, bmax, D] (rows past sel_len are 0)."""
    keep: list = []
    t = sparse.c(keep)
    B, Hkv, _, D = sparse.k.shape
    d = _Dims(B, Hkv * Hq, Hkv, D, _dtype_code(sparse.k), 1.0)
    idx = np.ascontiguousarray(idx, np.int32)
    k = np.ascontiguousarray(sel_len, np.int32)
    kc = np.zeros((B * Hkv, bmax, D), sparse.k.dtype)
    vc = np.zeros((B * Hkv, bmax, D), sparse.k.dtype)
    _ck(lib().hkvo_gather(C.byref(d), C.byref(t), _ptr(idx), _ptr(k), int(bmax), _ptr(kc),
                          _ptr(vc)), "gather")
    return kc, vc


def attend(q: np.ndarray, dense: Optional[Tier], sparse: Optional[Tier],
           idx: Optional[np.ndarray], sel_len: Optional[np.ndarray], bmax: int,
           condensed: Optional[Tier], scale: float, Hkv: Optional[int] = None):
    """S5: (out[B, Hq, D] fp32, lse[B, Hq] fp32)."""
    keep: list = []
    q = np.ascontiguousarray(q)
    tiers = [t for t in (dense, sparse, condensed) if t is not None]
    if Hkv is None:
        Hkv = tiers[0].k.shape[1]
    d = _dims(q, Hkv, scale)
    ct = [None if t is None else t.c(keep) for t in (dense, sparse, condensed)]
    idx = None if idx is None else np.ascontiguousarray(idx, np.int32)
    k = None if sel_len is None else np.ascontiguousarray(sel_len, np.int32)
    out = np.zeros(q.shape, np.float32)
    lse = np.zeros(q.shape[:2], np.float32)
    refs = [None if t is None else C.byref(t) for t in ct]
    _ck(lib().hkvo_attend(C.byref(d), _ptr(q), refs[0], refs[1], _ptr(idx), _ptr(k), int(bmax),
                          refs[2], _ptr(out), _ptr(lse)), "attend")
    return out, lse


def step(q: np.ndarray, dense: Optional[Tier], sparse: Tier, condensed: Optional[Tier],
         scale: float, p: float, bmin: int, bmax: int, beta: Optional[np.ndarray] = None,
         p_unit: Optional[np.ndarray] = None) -> dict:
    """S1..S5: dict(z, k, idx, out, lse)."""
    keep: list = []
    q = np.ascontiguousarray(q)
    d = _dims(q, sparse.k.shape[1], scale)
    ct = [None if t is None else t.c(keep) for t in (dense, sparse, condensed)]
    units = d.B * d.Hkv
    z = np.zeros((units, ct[1].cap), np.float32)
    k = np.zeros(units, np.int32)
    idx = np.zeros((units, bmax), np.int32)
    out = np.zeros(q.shape, np.float32)
    lse = np.zeros(q.shape[:2], np.float32)
    be = None if beta is None else np.ascontiguousarray(beta, np.float32)
    pu = None if p_unit is None else np.ascontiguousarray(p_unit, np.float32)
    refs = [None if t is None else C.byref(t) for t in ct]
    _ck(lib().hkvo_step(C.byref(d), _ptr(q), refs[0], refs[1], refs[2], _ptr(be), float(p),
                        _ptr(pu), int(bmin), int(bmax), _ptr(z), _ptr(k), _ptr(idx), _ptr(out),
                        _ptr(lse)), "step")
    return {"z": z, "k": k, "idx": idx, "out": out, "lse": lse}


def num_threads() -> int:
    return int(lib().hkvo_num_threads())


# ---- KV append with the dense-window roll ----------------------------------------------
#
# [TS 2.A] Cascade Cache Hierarchy, pipeline step (1): the new token enters the
# dense window of recent tokens; once the window is full, its oldest token
# ages out into the sparse tier. Reading taken: the window is a ring of W_cap
# slots per unit (attention does not depend on the order of its tokens), its
# oldest slot is head[u]; an aged-out token is appended at the end of the
# sparse tier (so sparse order is age order); when the sparse tier is full
# the aged-out token is dropped and reported (forming condensed slots is not
# part of this step).


def append(k_new: np.ndarray, v_new: np.ndarray, dense: Tier, head: np.ndarray, sparse: Tier):
    """One append per unit, in place on copies: returns (dense, head, sparse,
    dropped) with dropped[u] = 1 where an aged-out token found the sparse tier
    full. k_new, v_new: [B, Hkv, D]. All arrays keep their dtypes."""
    B, H, D = k_new.shape
    dk, dv = dense.k.copy(), dense.v.copy()
    sk, sv = sparse.k.copy(), sparse.v.copy()
    dlen = np.array(dense.len, dtype=np.int32).copy()
    slen = np.array(sparse.len, dtype=np.int32).copy()
    hd = np.array(head, dtype=np.int32).copy()
    wcap, ncap = dk.shape[2], sk.shape[2]
    dropped = np.zeros(B * H, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            u = b * H + h
            if dlen[u] < wcap:  # the window still has room
                dk[b, h, dlen[u]] = k_new[b, h]
                dv[b, h, dlen[u]] = v_new[b, h]
                dlen[u] += 1
                continue
            # full window (or none): the oldest token ages out first
            if wcap > 0:
                old_k, old_v = dk[b, h, hd[u]].copy(), dv[b, h, hd[u]].copy()
            else:
                old_k, old_v = k_new[b, h], v_new[b, h]
            if slen[u] < ncap:
                sk[b, h, slen[u]] = old_k
                sv[b, h, slen[u]] = old_v
                slen[u] += 1
            else:
                dropped[u] = 1
            if wcap > 0:
                dk[b, h, hd[u]] = k_new[b, h]
                dv[b, h, hd[u]] = v_new[b, h]
                hd[u] = (hd[u] + 1) % wcap
    return Tier(dk, dv, dlen), hd, Tier(sk, sv, slen), dropped


# ---- Fitted temperature: group-averaged raw-attention entropy and the beta that meets it ----
#
# [TS 2.B] Logits Calibration maps an importance metric onto a softmax
# distribution "by adjusting the temperature"; [TS 3] says the mapping goes
# onto the raw attention distribution; [TS 2.A] Tier 2 sets each head's budget
# from its attention entropy. Reading taken: the target of unit u is the mean,
# over the G query heads of its group, of the entropy (natural log) of each
# head's raw attention softmax(scale q_g . k_j) over the unit's sparse tokens;
# the fitted inverse temperature is the beta in [0, FIT_BETA_MAX] at which the
# calibrated distribution softmax(beta z) of the unit's metric z has that
# entropy. The entropy of softmax(beta z) does not increase with beta (its
# derivative is -beta Var(z)), so the root is unique wherever z is not
# constant. Degenerate units (n <= 1, or every score equal) get beta = 1.

FIT_BETA_MAX = 64.0


def _f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 values of bf16 bit patterns (uint16) or float32 arrays."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def softmax_entropy(x: np.ndarray) -> float:
    """Entropy (nats) of softmax(x) for a 1-D float64 array, 0 log 0 = 0."""
    x = np.asarray(x, np.float64)
    if x.size == 0:
        return 0.0
    w = np.exp(x - x.max())
    P = w / w.sum()
    nz = P > 0
    return float(-(P[nz] * np.log(P[nz])).sum())


def attention_entropy(q: np.ndarray, sparse: Tier, scale: float) -> np.ndarray:
    """Per unit: mean over the group's query heads of the entropy of their raw
    attention over the sparse tier. q: [B, Hq, D]. Returns float64 [B*Hkv]
    (0 for an empty unit)."""
    B, Hq, D = q.shape
    Hkv = sparse.k.shape[1]
    G = Hq // Hkv
    qf = _f64(q)
    kf = _f64(sparse.k)
    out = np.zeros(B * Hkv, np.float64)
    for b in range(B):
        for h in range(Hkv):
            u = b * Hkv + h
            n = int(sparse.len[u])
            if n == 0:
                continue
            logits = scale * (qf[b, h * G:(h + 1) * G] @ kf[b, h, :n].T)  # [G, n]
            out[u] = np.mean([softmax_entropy(logits[g]) for g in range(G)])
    return out


def fit_temperature(z: np.ndarray, length: np.ndarray, h_target: np.ndarray,
                    beta_max: float = FIT_BETA_MAX) -> np.ndarray:
    """Per unit the beta in [0, beta_max] with entropy(softmax(beta z)) equal
    to h_target[u], by bisection in float64 on the monotone entropy. A target
    at or above ln n gives 0; one below the entropy at beta_max gives beta_max.
    z: [units, >= n] scores. Returns float64 [units]."""
    units = len(length)
    beta = np.ones(units, np.float64)
    for u in range(units):
        n = int(length[u])
        zu = _f64(np.asarray(z[u, :n]))
        if n <= 1 or zu.max() == zu.min():
            continue
        t = float(h_target[u])
        if t >= np.log(n):
            beta[u] = 0.0
            continue
        if softmax_entropy(beta_max * zu) >= t:
            beta[u] = beta_max
            continue
        lo, hi = 0.0, beta_max  # entropy(lo) > t > entropy(hi)
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if mid <= lo or mid >= hi:
                break
            if softmax_entropy(mid * zu) > t:
                lo = mid
            else:
                hi = mid
        beta[u] = 0.5 * (lo + hi)
    return beta


# ---- Condensed-tier formation ([TS 2.A] Tier 3 and pipeline step 4) ----------------
#
# Tier 3 keeps the oldest context in storage of constant size: "the oldest
# blocks are further compressed into constant-sized storage via eviction or
# weighted merging", and the pipeline's fourth step is the "eviction or
# merging of the oldest blocks". Reading taken: a unit whose sparse tier holds
# at least `trigger` tokens (and at least `block`) gives up its oldest `block`
# tokens (sparse slots 0 .. block-1, the tier being in age order); they become
# ONE condensed slot, appended after the existing ones:
#   MERGE: the slot's K and V are the weighted means of the block's rows, the
#          weights a_j being the tokens' calibrated probabilities under the
#          step's scores, a_j = exp(beta (z_j - m) - logZ); the slot keeps the
#          block's mass sum_j a_j as its weight. When the condensed tier is
#          full, its two oldest slots first merge the same way (weights w_0,
#          w_1; the merged slot weighs w_0 + w_1) and the later slots move down.
#   EVICT: the slot is a copy of the block's most important token (largest z,
#          the older one on ties) with weight a_j; the rest of the block is
#          dropped. When the condensed tier is full its oldest slot is dropped
#          first and the later slots move down.
# Weights that sum to zero (or no scores given) mean equal weights. Means are
# float64 sums in slot order, rounded once to the tier's element type (nearest,
# ties to even). The sparse tier then moves down by `block` rows, keeping its
# age order. A condensed tier of capacity 0 just drops the block.

CONDENSE_MERGE, CONDENSE_EVICT = 0, 1


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (8 significant bits; nearest, ties to even)
    straight from the double, and return their bit patterns (uint16)."""
    x = np.asarray(x, np.float64)
    f, e = np.frexp(x)  # x = f 2^e, 0.5 <= |f| < 1
    # spacing of bf16 values near x: 2^(e - 8) for normal values, 2^-133 below 2^-126
    sh = np.where(e - 8 < -133, -133, e - 8)
    r = np.rint(np.ldexp(x, -sh))  # exact scaling, then round half to even
    y = np.ldexp(r, sh).astype(np.float32)  # exactly representable in bf16 (hence fp32)
    return (y.view(np.uint32) >> 16).astype(np.uint16)


def _round_to(x: np.ndarray, like: np.ndarray) -> np.ndarray:
    """float64 -> the element type of `like` (bf16 bits or float32), nearest-even."""
    if like.dtype == np.uint16:
        return round_to_bf16(x)
    return np.asarray(x, np.float64).astype(np.float32)


def _seq_sum(a) -> float:
    """float64 sum in index order (no pairwise summation)."""
    t = 0.0
    for x in a:
        t = t + float(x)
    return t


def _weighted_mean(rows: np.ndarray, a: np.ndarray) -> np.ndarray:
    """sum_j a_j rows_j / sum_j a_j in float64, summed in row order; equal
    weights when the a_j sum to zero. rows: [b, D] float64."""
    if not _seq_sum(a) > 0.0:
        a = np.ones(len(a), np.float64)
    num = np.zeros(rows.shape[1], np.float64)
    den = 0.0
    for j in range(len(a)):
        num = num + a[j] * rows[j]
        den = den + a[j]
    return num / den


def condense(sparse: Tier, condensed: Tier, cond_w: np.ndarray, z: Optional[np.ndarray],
             m: Optional[np.ndarray], logZ: Optional[np.ndarray], beta: Optional[np.ndarray],
             block: int, trigger: int, policy: int = CONDENSE_MERGE):
    """One condensation pass over every unit, on copies. Returns (sparse,
    condensed, cond_w, done) with done[u] = 1 where unit u gave up a block.
    z: the step's scores [units, >= sparse cap] (None: equal weights); m, logZ:
    the step's per-unit max and log normaliser; beta: per-unit inverse
    temperature (None = 1); cond_w: per-slot weights [units, condensed cap].
    A condensed tier of one slot under MERGE takes the block into that slot
    (the old slot weighing its weight)."""
    B, H, ncap, D = sparse.k.shape
    ccap = condensed.k.shape[2]
    sk, sv = sparse.k.copy(), sparse.v.copy()
    ck, cv = condensed.k.copy(), condensed.v.copy()
    slen = np.array(sparse.len, np.int32).copy()
    clen = np.array(condensed.len, np.int32).copy()
    w = np.array(cond_w, np.float32).copy().reshape(B * H, ccap)
    done = np.zeros(B * H, np.int32)
    for b in range(B):
        for h in range(H):
            u = b * H + h
            n, C = int(slen[u]), int(clen[u])
            if n < max(trigger, block, 1):
                continue
            done[u] = 1
            if z is not None:
                be = 1.0 if beta is None else float(beta[u])
                zz = np.asarray(z[u, :block], np.float32).astype(np.float64)
                a = np.exp(be * (zz - np.float64(m[u])) - np.float64(logZ[u]))
            else:
                zz = np.zeros(block, np.float64)
                a = np.ones(block, np.float64)
            if ccap > 0 and policy == CONDENSE_MERGE:
                rows_k, rows_v = _f64(sk[b, h, :block]), _f64(sv[b, h, :block])
                if C >= ccap and ccap >= 2:  # the two oldest slots merge into slot 0
                    wp = np.array([w[u, 0], w[u, 1]], np.float64)
                    ck[b, h, 0] = _round_to(_weighted_mean(_f64(ck[b, h, 0:2]), wp), ck)
                    cv[b, h, 0] = _round_to(_weighted_mean(_f64(cv[b, h, 0:2]), wp), cv)
                    w[u, 0] = np.float32(_seq_sum(wp))
                    ck[b, h, 1:ccap - 1] = ck[b, h, 2:ccap].copy()
                    cv[b, h, 1:ccap - 1] = cv[b, h, 2:ccap].copy()
                    w[u, 1:ccap - 1] = w[u, 2:ccap].copy()
                    C = ccap - 1
                elif C >= ccap:  # one slot: the block merges into it
                    rows_k = np.concatenate([_f64(ck[b, h, 0:1]), rows_k])
                    rows_v = np.concatenate([_f64(cv[b, h, 0:1]), rows_v])
                    a = np.concatenate([[np.float64(w[u, 0])], a])
                    C = 0
                ck[b, h, C] = _round_to(_weighted_mean(rows_k, a), ck)
                cv[b, h, C] = _round_to(_weighted_mean(rows_v, a), cv)
                w[u, C] = np.float32(_seq_sum(a))
                clen[u] = C + 1
            elif ccap > 0:  # EVICT
                if C >= ccap:  # the oldest slot goes
                    ck[b, h, 0:ccap - 1] = ck[b, h, 1:ccap].copy()
                    cv[b, h, 0:ccap - 1] = cv[b, h, 1:ccap].copy()
                    w[u, 0:ccap - 1] = w[u, 1:ccap].copy()
                    C = ccap - 1
                jstar = int(np.argmax(zz))  # the first maximum: the older token
                ck[b, h, C] = sk[b, h, jstar]
                cv[b, h, C] = sv[b, h, jstar]
                w[u, C] = np.float32(a[jstar])
                clen[u] = C + 1
            # the sparse tier moves down by one block, in age order
            sk[b, h, :n - block] = sk[b, h, block:n].copy()
            sv[b, h, :n - block] = sv[b, h, block:n].copy()
            slen[u] = n - block
    return Tier(sk, sv, slen), Tier(ck, cv, clen), w, done


# ---- Rewrite Cache vs Sparse Loading ([TS 2.C] Trade-off Management) ------------------
#
# The pages: a Memory-Time Integral (MTI) weighs the upfront cost of rewriting
# against the per-step decoding gains, and budget thresholds L_lower and
# L_upper trigger sparse loading or full rewriting; the rewrite overhead is
# amortized within a few decoding steps ([TS 4]). Reading taken, per unit:
#   - a unit whose rewrite still serves (left > 0) is not scored or selected
#     this step: it attends over dense ++ its rewritten rows ++ condensed, and
#     left drops by one;
#   - any other unit runs the plain step (Sparse Loading of the fresh
#     selection, budget k); then its mode becomes Rewrite Cache when k > L_upper,
#     Sparse Loading when k < L_lower, and stays as it was in between; under
#     Rewrite Cache its k selected rows are copied, in token order, into its
#     rewrite buffer, which serves H(k) = max(1, floor(mti_cap / k)) steps in
#     all (this one included), so that the rewrite's memory-time integral
#     k H stays within mti_cap.

MODE_SPARSE, MODE_REWRITE = 0, 1


def mti_trigger(k: int, mode: int, L_lower: int, L_upper: int) -> int:
    """The mode after a fresh step whose budget is k."""
    if k > L_upper:
        return MODE_REWRITE
    if k < L_lower:
        return MODE_SPARSE
    return mode


def mti_horizon(k: int, mti_cap: int) -> int:
    """Steps a rewrite of k rows serves, the step that made it included."""
    return max(1, mti_cap // k) if k > 0 else 1


def mti_state(units: int, bmax: int, B: int, Hkv: int, D: int, like: np.ndarray) -> dict:
    """The all-Sparse-Loading starting state (the rewrite buffer of `like`'s dtype)."""
    return {"mode": np.zeros(units, np.int32), "left": np.zeros(units, np.int32),
            "rw_k": np.zeros((B, Hkv, bmax, D), like.dtype), "rw_v": np.zeros((B, Hkv, bmax, D), like.dtype),
            "rw_len": np.zeros(units, np.int32), "rw_idx": np.zeros((units, bmax), np.int32)}


def step_mti(q: np.ndarray, dense: Optional[Tier], sparse: Tier, condensed: Optional[Tier], scale: float,
             p: float, bmin: int, bmax: int, state: dict, L_lower: int, L_upper: int, mti_cap: int,
             k_fresh: Optional[np.ndarray] = None, idx_fresh: Optional[np.ndarray] = None,
             p_unit: Optional[np.ndarray] = None):
    """One decode step under the trigger. Returns (result, new state): result
    holds k, idx [units, bmax], out, lse and fresh (1 where the unit ran the
    plain step). k_fresh / idx_fresh: optional budgets and index rows of the
    fresh units to take the trigger and the rewrite with (another
    implementation's, where its budget may differ at an ambiguous cut); by
    default the step's own."""
    B, Hq, D = q.shape
    Hkv = sparse.k.shape[1]
    G = Hq // Hkv
    U = B * Hkv
    st = {key: np.array(v, copy=True) for key, v in state.items()}
    plain = step(q, dense, sparse, condensed, scale, p, bmin, bmax, p_unit=p_unit)
    kf = plain["k"] if k_fresh is None else np.asarray(k_fresh, np.int32)
    idf = plain["idx"] if idx_fresh is None else np.asarray(idx_fresh, np.int32).reshape(U, bmax)
    # the reusing units' attention: the rewrite buffer as the selected tokens
    rw = Tier(state["rw_k"], state["rw_v"], state["rw_len"])
    rw_cap = state["rw_k"].shape[2]
    ident = np.tile(np.arange(rw_cap, dtype=np.int32), (U, 1))
    r_out, r_lse = attend(q, dense, rw, ident, state["rw_len"], rw_cap, condensed, scale, Hkv=Hkv)
    out, lse = plain["out"].copy(), plain["lse"].copy()
    k = plain["k"].copy()
    idx = plain["idx"].copy()
    fresh = np.ones(U, np.int32)
    for u in range(U):
        b, h = divmod(u, Hkv)
        if state["left"][u] > 0:
            fresh[u] = 0
            out[b, h * G:(h + 1) * G] = r_out[b, h * G:(h + 1) * G]
            lse[b, h * G:(h + 1) * G] = r_lse[b, h * G:(h + 1) * G]
            n = int(state["rw_len"][u])
            k[u] = n
            idx[u, :] = -1
            idx[u, :n] = state["rw_idx"][u, :n]
            st["left"][u] -= 1
            continue
        ku = int(kf[u])
        st["mode"][u] = mti_trigger(ku, int(state["mode"][u]), L_lower, L_upper)
        if st["mode"][u] == MODE_REWRITE:
            rows = idf[u, :ku]
            st["rw_k"][b, h, :ku] = sparse.k[b, h, rows]
            st["rw_v"][b, h, :ku] = sparse.v[b, h, rows]
            st["rw_idx"][u, :ku] = rows
            st["rw_len"][u] = ku
            st["left"][u] = mti_horizon(ku, mti_cap) - 1
        else:
            st["rw_len"][u] = 0
            st["left"][u] = 0
    return {"k": k, "idx": idx, "out": out, "lse": lse, "fresh": fresh}, st
