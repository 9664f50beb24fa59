"""End-to-end parity of the fused decode step (hkv_step) against the CPU oracle,
on small cases and on the full-size workloads."""
import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, make_inputs, to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_stages import CASES

pytestmark = pytest.mark.gpu


def check_step(wl, x, out, p, bmin, bmax, b_sel=None, beta=None, tag=""):
    """z within the fp32 bound, selection by the end-to-end rule, attention over
    the GPU's selection within tolerance. b_sel: sequences to check (all)."""
    bs = range(wl.B) if b_sel is None else b_sel
    scale = H.scale_of(wl)
    z_all = out.z.cpu().numpy() if out.z is not None else None
    k_all = out.sel_len.cpu().numpy()
    row = max(1, wl.bmax if bmax is None else bmax)  # a bmax of 0 still allocates one slot per unit
    idx_all = out.idx.cpu().numpy()[: wl.units * row].reshape(wl.units, row)
    o_all = out.out.cpu().numpy()
    l_all = out.lse.cpu().numpy()
    for b in bs:
        sl = slice(b, b + 1)
        q = to_host_bits(x.q[sl])
        sp = H.host_tier(x.sparse, sl)
        zr = oracle.score(q, sp, scale)
        ln = sp.len
        units = range(b * wl.Hkv, (b + 1) * wl.Hkv)
        if z_all is not None:
            bound = H.score_bound(q, sp.k, ln, wl.G, scale)
            for i, u in enumerate(units):
                n = ln[i]
                err = np.abs(z_all[u, :n].astype(np.float64) - zr[i, :n])
                assert np.all(err <= bound[i, :n]), (tag, b, u, err.max())
        for i, u in enumerate(units):
            be = 1.0 if beta is None else float(beta[u])
            ok, why = H.selection_ok(zr[i], int(ln[i]), int(k_all[u]), idx_all[u], p, bmin, bmax, be)
            assert ok, (tag, b, u, why)
        bm = idx_all.shape[1]
        o_ref, l_ref = oracle.attend(q, H.host_tier(x.dense, sl), sp, idx_all[list(units)],
                                     k_all[list(units)], bm, H.host_tier(x.condensed, sl), scale)
        ok, err = H.attn_close(o_all[sl], o_ref)
        assert ok, (tag, b, "out", err)
        ok, err = H.attn_close(l_all[sl], l_ref)
        assert ok, (tag, b, "lse", err)


@pytest.mark.parametrize("name", sorted(CASES))
def test_step_small(name):
    wl = CASES[name]
    x = H.inputs(wl)
    for p in (wl.p, 0.5, 1.0):
        prob, out, ws = H.run_step(wl, x, p=p)
        assert ws.status() == 0
        check_step(wl, x, out, p, wl.bmin, wl.bmax, tag=f"{name} p={p}")


@pytest.mark.parametrize("name", sorted(CASES))
def test_step_equals_stage_chain(name):
    """hkv_step and the five separate calls give bit-identical scores,
    selections, index rows, m and logZ. The attention outputs agree to a few
    ulp: hkv_step reuses the scorer's per-head logits for the selected tokens,
    while hkv_cascade_decode recomputes them from K."""
    wl = CASES[name]
    x = H.inputs(wl)
    prob, out, ws = H.run_step(wl, x)
    U = wl.units
    dense, sparse, cond = H.tiers_of(x)
    z = torch.zeros(U, sparse.cap, device=H.dev())
    hkv.score(prob, x.q, sparse, z, ws)
    sel = torch.zeros(U, dtype=torch.int32, device=H.dev())
    cut = torch.zeros(U, 4, dtype=torch.int32, device=H.dev())
    hkv.topp_select(prob, z, sparse, sel, cut, ws)
    idx = torch.zeros(U * wl.bmax, dtype=torch.int32, device=H.dev())
    hkv.compact(prob, z, sparse, sel, cut, idx, ws)
    o = torch.zeros(wl.B, wl.Hq, wl.D, device=H.dev())
    lse = torch.zeros(wl.B, wl.Hq, device=H.dev())
    hkv.cascade_decode(prob, x.q, dense, sparse, idx, sel, cond, o, ws, lse=lse)
    m = torch.zeros(U, device=H.dev())
    lz = torch.zeros(U, device=H.dev())
    hkv.calibrate(prob, z, sparse, m, lz, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ln = x.sparse.len.cpu().numpy()
    zs, zf = z.cpu().numpy(), out.z.cpu().numpy()
    for u in range(U):
        assert np.array_equal(zs[u, : ln[u]], zf[u, : ln[u]])
    assert torch.equal(sel, out.sel_len)
    assert torch.equal(cut, out.cut)
    assert torch.equal(idx, out.idx)
    torch.testing.assert_close(o, out.out, atol=1e-5, rtol=1e-5)
    torch.testing.assert_close(lse, out.lse, atol=1e-5, rtol=1e-5)
    assert torch.equal(m, out.m)
    assert torch.equal(lz, out.logZ)


@pytest.mark.parametrize("name", ["bf16_b2_n3000", "bf16_ragged"])
def test_step_flat_sum_and_rewrite(name):
    wl = CASES[name]
    x = H.inputs(wl)
    _, pad, _ = H.run_step(wl, x, rewrite=True)
    _, flat, ws = H.run_step(wl, x, layout=hkv.FLAT_SUM, rewrite=True)
    assert ws.status() == 0
    U = wl.units
    k = pad.sel_len.cpu().numpy()
    assert np.array_equal(k, flat.sel_len.cpu().numpy())
    offs = flat.offsets.cpu().numpy()
    assert list(offs) == [0] + list(np.cumsum(k))
    rows = pad.idx.cpu().numpy().reshape(U, wl.bmax)
    fl = flat.idx.cpu().numpy()
    kp = to_host_bits(pad.k_out).reshape(U, wl.bmax, wl.D)
    kf = to_host_bits(flat.k_out)
    vp = to_host_bits(pad.v_out).reshape(U, wl.bmax, wl.D)
    vf = to_host_bits(flat.v_out)
    ks = to_host_bits(x.sparse.k).reshape(U, -1, wl.D)
    vs = to_host_bits(x.sparse.v).reshape(U, -1, wl.D)
    for u in range(U):
        r = rows[u, : k[u]]
        assert np.array_equal(fl[offs[u]: offs[u + 1]], r)
        assert np.all(rows[u, k[u]:] == -1)
        assert np.array_equal(kp[u, : k[u]], ks[u, r]) and np.array_equal(vp[u, : k[u]], vs[u, r])
        assert np.array_equal(kf[offs[u]: offs[u + 1]], ks[u, r])
        assert np.array_equal(vf[offs[u]: offs[u + 1]], vs[u, r])
    assert torch.equal(pad.out, flat.out)


def test_step_per_unit_p_and_temperature():
    wl = CASES["bf16_hetero"]
    x = H.inputs(wl)
    U = wl.units
    beta = np.linspace(0.25, 3.0, U).astype(np.float32)
    pu = np.linspace(0.6, 0.99, U).astype(np.float32)
    prob, out, ws = H.run_step(wl, x, inv_temp=torch.from_numpy(beta).to(H.dev()),
                               p_unit=torch.from_numpy(pu).to(H.dev()))
    assert ws.status() == 0
    k = out.sel_len.cpu().numpy()
    idx = out.idx.cpu().numpy().reshape(U, wl.bmax)
    z = out.z.cpu().numpy()
    ln = x.sparse.len.cpu().numpy()
    r = oracle.topp(z, ln, 0.0, wl.bmin, wl.bmax, beta, pu)
    ok, bad = H.budgets_match(k, r, pu, z, ln, beta)
    assert ok, bad
    want = oracle.compact(z, ln, k, wl.bmax)
    assert np.array_equal(idx, want)


# ---- full-size workloads -----------------------------------------------------------


@pytest.mark.slow
def test_workload1_full():
    wl = WORKLOADS[1]
    x = H.inputs(wl)
    prob, out, ws = H.run_step(wl, x)
    assert ws.status() == 0
    check_step(wl, x, out, wl.p, wl.bmin, wl.bmax, tag="w1")


@pytest.mark.slow
def test_workload2_full():
    wl = WORKLOADS[2]
    x = H.inputs(wl)
    prob, out, ws = H.run_step(wl, x)
    assert ws.status() == 0
    check_step(wl, x, out, wl.p, wl.bmin, wl.bmax, tag="w2")


@pytest.mark.slow
def test_workload3_full():
    """Every sequence of the ragged 64-sequence workload."""
    wl = WORKLOADS[3]
    x = H.inputs(wl)
    prob, out, ws = H.run_step(wl, x)
    assert ws.status() == 0
    check_step(wl, x, out, wl.p, wl.bmin, wl.bmax, tag="w3")
    k = out.sel_len.cpu().numpy()
    assert k.min() >= wl.bmin and k.max() <= wl.bmax


@pytest.mark.slow
def test_workload4_full_p_sweep():
    """Every sequence of the heterogeneous-head workload at every p of its sweep."""
    wl = WORKLOADS[4]
    x = H.inputs(wl)
    for p in wl.p_sweep:
        prob, out, ws = H.run_step(wl, x, p=p)
        assert ws.status() == 0
        check_step(wl, x, out, p, wl.bmin, wl.bmax, tag=f"w4 p={p}")


def _step_outputs(prob, sparse, n):
    return [hkv.StepOutputs.allocate(prob, sparse, H.dev(), with_z=True) for _ in range(n)]


@pytest.mark.slow
def test_workload5_36_layers_back_to_back_and_as_one_graph():
    """The 36-layer decode step: all layers issued back to back on one stream
    (one workspace), every layer and sequence checked against the oracle; then
    the same 36 steps captured in one CUDA graph and replayed, bit for bit equal
    to the eager run."""
    wl = WORKLOADS[5]
    L = wl.layers
    xs = [make_inputs(wl, H.dev(), layer) for layer in range(L)]
    prob = H.problem_of(wl)
    tiers = [H.tiers_of(x) for x in xs]
    ws = hkv.Workspace(prob, *tiers[0])
    outs = _step_outputs(prob, tiers[0][1], L)
    for layer in range(L):
        hkv.step(prob, xs[layer].q, *tiers[layer], outs[layer], ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    # the same 36 steps as one captured graph, into fresh outputs
    outs2 = _step_outputs(prob, tiers[0][1], L)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for layer in range(L):
            hkv.step(prob, xs[layer].q, *tiers[layer], outs2[layer], ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert ws.status() == 0
    for layer in range(L):
        a, b = outs[layer], outs2[layer]
        for name in ("sel_len", "idx", "out", "lse", "z"):
            assert torch.equal(getattr(a, name), getattr(b, name)), (layer, name)
    del g, outs2
    for layer in range(L):
        check_step(wl, xs[layer], outs[layer], wl.p, wl.bmin, wl.bmax, tag=f"w5 layer {layer}")
