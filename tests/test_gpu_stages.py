"""Per-step parity of the CUDA library (through the C ABI) against the CPU oracle."""
import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, to_host_bits
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

# Small cases that still span several score tiles (1024 bf16 rows / 1024 fp32
# rows of 64), several attention tiles and ragged tails.
CASES = {
    "tiny_fp32": WORKLOADS[1],
    "bf16_b2_n3000": WORKLOADS[2].with_(B=2, n_cap=3000, bmin=64, bmax=512),
    "bf16_ragged": WORKLOADS[3].with_(B=4, n_cap=5000, ctx_range=(320, 5320), bmin=32, bmax=700),
    "bf16_hetero": WORKLOADS[4].with_(B=2, n_cap=4000, bmax=1000),
    "fp32_d128_g8": WORKLOADS[2].with_(B=1, Hq=16, Hkv=2, D=128, dtype=torch.float32, n_cap=2100,
                                       w_cap=40, c_cap=8, bmin=3, bmax=300),
    "bf16_d64_g1": WORKLOADS[2].with_(B=2, Hq=4, Hkv=4, D=64, n_cap=2500, w_cap=32, c_cap=0, bmin=1,
                                      bmax=2500, p=0.5),
}


@pytest.fixture(scope="module", params=sorted(CASES))
def case(request):
    wl = CASES[request.param]
    x = H.inputs(wl)
    return request.param, wl, x


def _ws(prob, x):
    return hkv.Workspace(prob, *H.tiers_of(x))


def test_score(case):
    name, wl, x = case
    prob = H.problem_of(wl)
    sp = H.tiers_of(x)[1]
    z = torch.full((wl.units, sp.cap + 3), float("nan"), device=H.dev())
    hkv.score(prob, x.q, sp, z, _ws(prob, x))
    torch.cuda.synchronize()
    zg = z.cpu().numpy()
    q = to_host_bits(x.q)
    zr = oracle.score(q, H.host_tier(x.sparse), H.scale_of(wl))
    ln = x.sparse.len.cpu().numpy()
    bound = H.score_bound(q, to_host_bits(x.sparse.k), ln, wl.G, H.scale_of(wl))
    for u in range(wl.units):
        n = ln[u]
        err = np.abs(zg[u, :n].astype(np.float64) - zr[u, :n])
        assert np.all(err <= bound[u, :n]), (name, u, err.max())
        assert np.all(np.isnan(zg[u, n:])), "wrote past the unit's length"


def _oracle_z(wl, x):
    return oracle.score(to_host_bits(x.q), H.host_tier(x.sparse), H.scale_of(wl))


def test_calibrate(case):
    name, wl, x = case
    zr = _oracle_z(wl, x)
    ln = x.sparse.len.cpu().numpy()
    beta = np.linspace(0.0, 2.0, wl.units).astype(np.float32)
    prob = H.problem_of(wl, inv_temp=torch.from_numpy(beta).to(H.dev()))
    zt = torch.from_numpy(zr).to(H.dev())
    Pg = torch.zeros_like(zt)
    m = torch.zeros(wl.units, device=H.dev())
    lz = torch.zeros(wl.units, device=H.dev())
    hkv.calibrate(prob, zt, H.tiers_of(x)[1], m, lz, _ws(prob, x), P=Pg)
    Pr, mr, lzr = oracle.calibrate(zr, ln, beta)
    Pg = Pg.cpu().numpy()
    assert np.array_equal(m.cpu().numpy(), mr)
    assert np.allclose(lz.cpu().numpy(), lzr, rtol=0, atol=2e-6)
    # P = w / Z in fp32. The weight is within 2^-22 + 3 2^-24 ln2 x_j relative
    # (x_j = beta log2e (m - z_j); see gpu_helpers.window), Z (the exact sum of
    # such weights floored to 40-bit fixed point) within 2^-22 + 3 2^-24 ln2
    # E_P[x] + n 2^-40, and the rounding of 1/Z to fp32 and of the product add
    # 2^-23; 1.5 times that, for results in the normal fp32 range.
    c = 3 * 2.0 ** -24 * np.log(2)
    for u in range(wl.units):
        n = ln[u]
        x = beta[u] * np.log2(np.e) * (np.float64(mr[u]) - zr[u, :n].astype(np.float64))
        ex = float(np.sum(Pr[u, :n].astype(np.float64) * x))
        rel = 2 * 2.0 ** -22 + c * (x + ex) + 2.0 ** -23 + n * 2.0 ** -40
        tol = 1.5 * rel * Pr[u, :n] + 2e-38
        err = np.abs(Pg[u, :n] - Pr[u, :n])
        assert np.all(err <= tol), (name, u, float(np.max(err / np.maximum(Pr[u, :n], 1e-300))))


@pytest.mark.parametrize("p", [0.0, 0.3, 0.8, 0.95, 1.0])
def test_topp_and_compact_identical_scores(case, p):
    """Given identical fp32 scores: budgets bit-exact (except ambiguous cuts) and
    the compacted rows bit-exact for the budget chosen."""
    name, wl, x = case
    zr = _oracle_z(wl, x)
    ln = x.sparse.len.cpu().numpy()
    U = wl.units
    zt = torch.from_numpy(zr).to(H.dev())
    for layout in (hkv.PAD_MAX, hkv.FLAT_SUM):
        prob = H.problem_of(wl, p=p, layout=layout)
        ws = _ws(prob, x)
        sel = torch.zeros(U, dtype=torch.int32, device=H.dev())
        cut = torch.zeros(U, 4, dtype=torch.int32, device=H.dev())
        hkv.topp_select(prob, zt, H.tiers_of(x)[1], sel, cut, ws)
        idx = torch.full((U * wl.bmax,), -7, dtype=torch.int32, device=H.dev())
        off = torch.zeros(U + 1, dtype=torch.int32, device=H.dev()) if layout == hkv.FLAT_SUM else None
        hkv.compact(prob, zt, H.tiers_of(x)[1], sel, cut, idx, ws, offsets=off)
        torch.cuda.synchronize()
        assert ws.status() == 0
        kg = sel.cpu().numpy()
        r = oracle.topp(zr, ln, p, wl.bmin, wl.bmax)
        ok, bad = H.budgets_match(kg, r, p, zr, ln)
        assert ok, (name, p, bad)
        ct = cut.cpu().numpy()
        assert np.array_equal(ct[:, 1] + ct[:, 2], kg)
        want = oracle.compact(zr, ln, kg, wl.bmax, layout)
        got = idx.cpu().numpy()
        if layout == hkv.PAD_MAX:
            assert np.array_equal(got.reshape(U, wl.bmax), want)
        else:
            flat, offs = want
            assert np.array_equal(off.cpu().numpy(), offs)
            assert np.array_equal(got[: offs[-1]], flat)


def test_rewrite_cache_bit_exact(case):
    name, wl, x = case
    zr = _oracle_z(wl, x)
    ln = x.sparse.len.cpu().numpy()
    U = wl.units
    prob = H.problem_of(wl)
    ws = _ws(prob, x)
    zt = torch.from_numpy(zr).to(H.dev())
    sel = torch.zeros(U, dtype=torch.int32, device=H.dev())
    cut = torch.zeros(U, 4, dtype=torch.int32, device=H.dev())
    hkv.topp_select(prob, zt, H.tiers_of(x)[1], sel, cut, ws)
    idx = torch.zeros(U * wl.bmax, dtype=torch.int32, device=H.dev())
    kc = torch.zeros(U * wl.bmax, wl.D, dtype=wl.dtype, device=H.dev())
    vc = torch.zeros_like(kc)
    hkv.compact(prob, zt, H.tiers_of(x)[1], sel, cut, idx, ws, k_out=kc, v_out=vc)
    torch.cuda.synchronize()
    kg = sel.cpu().numpy()
    ir = oracle.compact(zr, ln, kg, wl.bmax)
    kr, vr = oracle.gather(H.host_tier(x.sparse), ir, kg, wl.bmax)
    kcg = to_host_bits(kc).reshape(U, wl.bmax, wl.D)
    vcg = to_host_bits(vc).reshape(U, wl.bmax, wl.D)
    for u in range(U):
        assert np.array_equal(kcg[u, : kg[u]], kr[u, : kg[u]])
        assert np.array_equal(vcg[u, : kg[u]], vr[u, : kg[u]])


def test_cascade_decode(case):
    name, wl, x = case
    zr = _oracle_z(wl, x)
    ln = x.sparse.len.cpu().numpy()
    U = wl.units
    r = oracle.topp(zr, ln, wl.p, wl.bmin, wl.bmax)
    ir = oracle.compact(zr, ln, r["k"], wl.bmax)
    for layout in (hkv.PAD_MAX, hkv.FLAT_SUM):
        prob = H.problem_of(wl, layout=layout)
        if layout == hkv.PAD_MAX:
            idx = torch.from_numpy(ir.reshape(-1)).to(H.dev())
            off = None
        else:
            flat, offs = oracle.compact(zr, ln, r["k"], wl.bmax, hkv.FLAT_SUM)
            idx = torch.from_numpy(np.concatenate([flat, np.zeros(1, np.int32)])).to(H.dev())
            off = torch.from_numpy(offs).to(H.dev())
        sel = torch.from_numpy(r["k"]).to(H.dev())
        out = torch.zeros(wl.B, wl.Hq, wl.D, device=H.dev())
        lse = torch.zeros(wl.B, wl.Hq, device=H.dev())
        dense, sparse, cond = H.tiers_of(x)
        ws = _ws(prob, x)
        hkv.cascade_decode(prob, x.q, dense, sparse, idx, sel, cond, out, ws, lse=lse, offsets=off)
        torch.cuda.synchronize()
        assert ws.status() == 0
        o_ref, l_ref = oracle.attend(to_host_bits(x.q), H.host_tier(x.dense), H.host_tier(x.sparse), ir,
                                     r["k"], wl.bmax, H.host_tier(x.condensed), H.scale_of(wl))
        ok, err = H.attn_close(out.cpu().numpy(), o_ref)
        assert ok, (name, err)
        ok, err = H.attn_close(lse.cpu().numpy(), l_ref)
        assert ok, (name, err)
