"""Condensed-tier formation (hkv_condense) against the oracle, and a decode
loop of append + step + condense that runs far past the sparse capacity.

Given the same scores, both sides compute the same float64 sums in the same
order and round once, so every row, length and weight is compared bit for bit.
The one allowance: a mean that lies within 1e-12 of a rounding tie between two
neighbouring values may round either way (the two exp implementations can differ
in the last bit of a weight)."""
import numpy as np
import pytest
import scipy.special as sps
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, make_inputs, to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_step import check_step

pytestmark = pytest.mark.gpu


def _values(bits_or_f32):
    a = np.asarray(bits_or_f32)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def assert_rows_match(got, want, exact_mean=None, what=""):
    """Bit equality; a differing element is accepted only when `exact_mean`
    (float64 reference means, same shape) sits at the midpoint of the two
    neighbouring values got and want, to 1e-12 relative."""
    got, want = np.asarray(got), np.asarray(want)
    diff = got != want
    if not diff.any():
        return
    assert exact_mean is not None, (what, int(diff.sum()))
    g, w, x = _values(got[diff]), _values(want[diff]), np.asarray(exact_mean)[diff]
    mid = 0.5 * (g + w)
    assert np.all(np.abs(x - mid) <= 1e-12 * np.abs(mid)), (what, g[:3], w[:3], x[:3])


def make_state(dtype, D, ncap, ccap, n, C, seed, G=2):
    B, Hkv = 2, len(n) // 2
    gen = torch.Generator(device=H.dev()).manual_seed(seed)
    dev = H.dev()

    def tier(cap, ln):
        k = torch.randn(B, Hkv, cap, D, generator=gen, device=dev).to(dtype)
        v = torch.randn(B, Hkv, cap, D, generator=gen, device=dev).to(dtype)
        return k, v, torch.tensor(ln, dtype=torch.int32, device=dev)

    sp, co = tier(ncap, n), tier(ccap, C)
    rng = np.random.default_rng(seed)
    w = rng.uniform(0.0, 1.0, (B * Hkv, ccap)).astype(np.float32)
    z = np.round(rng.standard_normal((B * Hkv, ncap)).astype(np.float32) * 6) / 2  # with ties
    m = np.array([z[u, :max(n[u], 1)].max() for u in range(B * Hkv)], np.float32)
    lz = np.array([sps.logsumexp(z[u, :n[u]].astype(np.float64) - m[u]) if n[u] else 0.0
                   for u in range(B * Hkv)], np.float32)
    return sp, co, w, z, m, lz


def exact_means(sp_k, co_k, w, a, u, C0, ccap, block, policy):
    """float64 reference of the new slot's mean (numpy average), for the tie rule."""
    B, Hkv = sp_k.shape[:2]
    b, h = divmod(u, Hkv)
    rows = _values(sp_k[b, h, :block])
    if ccap == 1 and C0 >= 1 and policy == oracle.CONDENSE_MERGE:
        rows = np.concatenate([_values(co_k[b, h, :1]), rows])
        a = np.concatenate([[float(w[u, 0])], a])
    if not a.sum() > 0:
        a = np.ones_like(a)
    return np.average(rows, axis=0, weights=a)


CASES = [
    # dtype, D, ncap, ccap, n per unit, C per unit, block, trigger, policy, scores, beta
    (torch.bfloat16, 128, 300, 5, [300, 100, 64, 30], [5, 0, 3, 5], 32, 64, oracle.CONDENSE_MERGE, True, False),
    (torch.bfloat16, 128, 300, 5, [300, 100, 64, 30], [5, 0, 3, 5], 32, 64, oracle.CONDENSE_EVICT, True, False),
    (torch.bfloat16, 128, 300, 1, [300, 290, 64, 10], [1, 0, 1, 1], 40, 50, oracle.CONDENSE_MERGE, True, True),
    (torch.bfloat16, 64, 520, 0, [520, 17, 16, 15], [0, 0, 0, 0], 16, 0, oracle.CONDENSE_MERGE, True, False),
    (torch.float32, 64, 257, 4, [257, 200, 129, 128], [4, 4, 0, 2], 129, 129, oracle.CONDENSE_MERGE, True, True),
    (torch.float32, 128, 257, 4, [257, 200, 129, 128], [4, 4, 0, 2], 100, 129, oracle.CONDENSE_EVICT, False, False),
    (torch.bfloat16, 128, 2048, 3, [2048, 2047, 1500, 9], [3, 3, 2, 0], 1024, 1024, oracle.CONDENSE_MERGE, False, False),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_condense_matches_oracle(case):
    dtype, D, ncap, ccap, n, C, block, trig, policy, scores, use_beta = CASES[case]
    sp, co, w, z, m, lz = make_state(dtype, D, ncap, ccap, n, C, seed=100 + case)
    U = len(n)
    beta = np.linspace(0.5, 2.0, U).astype(np.float32) if use_beta else None
    prob = hkv.Problem(2, 2 * U // 2, U // 2, D, dtype, 0.9, 1, 8,
                       inv_temp=None if beta is None else torch.from_numpy(beta).to(H.dev()))
    s_t, c_t = hkv.Tier(*sp), hkv.Tier(*co)
    host_s = oracle.Tier(to_host_bits(sp[0]), to_host_bits(sp[1]), np.array(n, np.int32))
    host_c = oracle.Tier(to_host_bits(co[0]), to_host_bits(co[1]), np.array(C, np.int32))
    ws = hkv.Workspace(prob, None, s_t, c_t)
    wt = torch.from_numpy(w).to(H.dev())
    done = torch.full((U,), -1, dtype=torch.int32, device=H.dev())
    zt, mt, lzt = (torch.from_numpy(x).to(H.dev()) for x in (z, m, lz))
    hkv.condense(prob, s_t, c_t if ccap else None, wt if ccap else None, ws, block, trig, policy,
                 z=zt if scores else None, m=mt if scores else None, logZ=lzt if scores else None, done=done)
    torch.cuda.synchronize()
    assert ws.status() == 0
    s2, c2, w2, d2 = oracle.condense(host_s, host_c, w, z if scores else None, m if scores else None,
                                     lz if scores else None, beta, block, trig, policy)
    assert np.array_equal(done.cpu().numpy(), d2)
    assert np.array_equal(sp[2].cpu().numpy(), s2.len)
    gk, gv = to_host_bits(sp[0]), to_host_bits(sp[1])
    for u in range(U):
        b, h = divmod(u, U // 2)
        k = s2.len[u]
        assert np.array_equal(gk[b, h, :k], s2.k[b, h, :k]) and np.array_equal(gv[b, h, :k], s2.v[b, h, :k]), u
    if ccap == 0:
        return
    assert np.array_equal(co[2].cpu().numpy(), c2.len)
    ck, cv, gw = to_host_bits(co[0]), to_host_bits(co[1]), wt.cpu().numpy()
    for u in range(U):
        b, h = divmod(u, U // 2)
        Cn = c2.len[u]
        new = Cn - 1 if d2[u] else -1
        for i in range(Cn):
            exact_k = exact_v = None
            if i == new and policy == oracle.CONDENSE_MERGE:
                be = 1.0 if beta is None else float(beta[u])
                a = (np.exp(be * (z[u, :block].astype(np.float64) - np.float64(m[u])) - np.float64(lz[u]))
                     if scores else np.ones(block))
                exact_k = exact_means(host_s.k, host_c.k, w, a, u, C[u], ccap, block, policy)
                exact_v = exact_means(host_s.v, host_c.v, w, a, u, C[u], ccap, block, policy)
            assert_rows_match(ck[b, h, i], c2.k[b, h, i], exact_k, ("k", case, u, i))
            assert_rows_match(cv[b, h, i], c2.v[b, h, i], exact_v, ("v", case, u, i))
            assert np.array_equal(gw[u, i], w2[u, i]) or abs(gw[u, i] - w2[u, i]) <= np.spacing(w2[u, i]), \
                (case, u, i, gw[u, i], w2[u, i])


def _loop_wl():
    return WORKLOADS[2].with_(B=2, Hq=8, Hkv=2, n_cap=256, w_cap=16, c_cap=4, bmin=4, bmax=64, p=0.9)


def _loop_state(wl):
    x = make_inputs(wl, H.dev(), 3)
    x.sparse.len.fill_(250)
    x.condensed.len.copy_(torch.tensor([3, 4, 1, 0], dtype=torch.int32))
    return x


STEPS, BLOCK = 40, 16


def _new_tokens(wl):
    g = torch.Generator(device=H.dev()).manual_seed(77)
    return [torch.randn(STEPS, wl.B, wl.Hkv, wl.D, generator=g, device=H.dev()).to(wl.dtype) for _ in range(2)]


def test_decode_loop_runs_past_sparse_capacity():
    """append -> step -> condense, 40 times, with the sparse tier starting six
    tokens short of full: the tier is condensed whenever it fills, no token is
    ever dropped, and after every step the tiers and weights equal the oracle's
    (append, then condense fed with the step's own scores) bit for bit; the
    step's outputs on the final tiers match the oracle. Then the whole loop, captured in one CUDA graph from the same start,
    leaves exactly the same state."""
    wl = _loop_wl()
    U = wl.units
    kn, vn = _new_tokens(wl)

    def run(x):
        prob = H.problem_of(wl)
        tiers = H.tiers_of(x)
        ws = hkv.Workspace(prob, *tiers)
        out = hkv.StepOutputs.allocate(prob, tiers[1], H.dev(), with_z=True, with_stats=True)
        head = torch.zeros(U, dtype=torch.int32, device=H.dev())
        w = torch.zeros(U, wl.c_cap, device=H.dev())
        dropped = torch.zeros(U, dtype=torch.int32, device=H.dev())
        done = torch.zeros(U, dtype=torch.int32, device=H.dev())

        def one(i):
            hkv.append(prob, kn[i], vn[i], tiers[0], head, tiers[1], ws, dropped=dropped)
            hkv.step(prob, x.q, *tiers, out, ws)
            hkv.condense(prob, tiers[1], tiers[2], w, ws, BLOCK, wl.n_cap, hkv.CONDENSE_MERGE,
                         z=out.z, m=out.m, logZ=out.logZ, done=done)
        return prob, ws, out, head, w, dropped, done, one

    x = _loop_state(wl)
    prob, ws, out, head, w, dropped, done, one = run(x)
    ot = lambda t: oracle.Tier(to_host_bits(t.k), to_host_bits(t.v), t.len.cpu().numpy())
    hd, hs, hc = ot(x.dense), ot(x.sparse), ot(x.condensed)
    hh = np.zeros(U, np.int32)
    hw = np.zeros((U, wl.c_cap), np.float32)
    condensations = 0
    for i in range(STEPS):
        one(i)
        torch.cuda.synchronize()
        assert ws.status() == 0, i
        assert int(dropped.sum()) == 0, i
        hd, hh, hs, dr = oracle.append(to_host_bits(kn[i]), to_host_bits(vn[i]), hd, hh, hs)
        hs, hc, hw, dn = oracle.condense(hs, hc, hw, out.z.cpu().numpy(), out.m.cpu().numpy(),
                                         out.logZ.cpu().numpy(), None, BLOCK, wl.n_cap, oracle.CONDENSE_MERGE)
        condensations += int(dn.sum())
        assert np.array_equal(done.cpu().numpy(), dn), i
        for got, want in ((ot(x.dense), hd), (ot(x.sparse), hs), (ot(x.condensed), hc)):
            assert np.array_equal(got.len, want.len), i
            for a, b in ((got.k, want.k), (got.v, want.v)):
                for u in range(U):
                    bb, h = divmod(u, wl.Hkv)
                    assert np.array_equal(a[bb, h, :want.len[u]], b[bb, h, :want.len[u]]), (i, u)
        assert np.array_equal(head.cpu().numpy(), hh), i
        gw = w.cpu().numpy()
        for u in range(U):
            c = hc.len[u]
            assert np.array_equal(gw[u, :c], hw[u, :c]), (i, u)
    assert condensations >= 2 * U
    assert int(x.condensed.len.max()) == wl.c_cap  # full condensed tiers were merged into
    # the step's outputs on the final tiers
    prob2, out2, ws2 = H.run_step(wl, x)
    check_step(wl, x, out2, wl.p, wl.bmin, wl.bmax, tag="after the loop")

    # the same loop as one CUDA graph, from the same start
    y = _loop_state(wl)
    prob, ws, out, head, w, dropped, done, one = run(y)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(STEPS):
                one(i)
    g.replay()
    torch.cuda.synchronize()
    assert ws.status() == 0
    for a, b in ((x.dense, y.dense), (x.sparse, y.sparse), (x.condensed, y.condensed)):
        assert torch.equal(a.len, b.len)
        assert torch.equal(a.k, b.k) and torch.equal(a.v, b.v)
