"""The decode step under the Rewrite Cache / Sparse Loading trigger
(hkv_step_mti) against the oracle, over several steps with a new query each.

The oracle takes the trigger and the rewrite with the GPU's own fresh budgets
and index rows (which may differ from its own only at an ambiguous cut, checked
separately by the end-to-end selection rule), so the states -- modes, steps
left, rewritten rows and their indices -- must agree bit for bit, and every
output is compared with the oracle's attention over what the GPU attended."""
import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, make_inputs, to_host_bits
from tests import gpu_helpers as H

pytestmark = pytest.mark.gpu

STEPS = 8


def _case(long=False):
    # long: units beyond what one CTA stages, so the selection runs split over
    # clusters of CTAs, and reusing units leave their clusters idle
    wl = WORKLOADS[2].with_(B=2, Hq=8, Hkv=4, n_cap=30000 if long else 3000, w_cap=32, c_cap=8, bmin=16,
                            bmax=16384 if long else 1024, p=0.95)
    x = make_inputs(wl, H.dev(), 5)
    g = torch.Generator(device=H.dev()).manual_seed(9)
    qs = [torch.randn(x.q.shape, generator=g, device=H.dev()).to(wl.dtype) for _ in range(STEPS)]
    # budgets spread over the units, below the clamp
    pu = np.linspace(0.005, 0.3, wl.units) if long else np.linspace(0.3, 0.99, wl.units)
    pu = pu.astype(np.float32)
    return wl, x, qs, pu


def _thresholds(wl, x, pu):
    """Thresholds between the units' budgets, so that some units rewrite and
    some load sparsely, with horizons of a few steps."""
    prob, out, ws = H.run_step(wl, x, p_unit=torch.from_numpy(pu).to(H.dev()))
    k = np.sort(out.sel_len.cpu().numpy())
    lo, hi = int(k[len(k) // 4]), int(k[len(k) // 2])
    return lo, hi, int(3 * k[-1])


def _host_state(st: hkv.MtiState):
    return {"mode": st.mode.cpu().numpy(), "left": st.left.cpu().numpy(), "rw_k": to_host_bits(st.rewrite.k),
            "rw_v": to_host_bits(st.rewrite.v), "rw_len": st.rewrite.len.cpu().numpy(),
            "rw_idx": st.rw_idx.cpu().numpy().reshape(len(st.mode), -1)}


@pytest.mark.parametrize("long", [False, True])
def test_step_mti_matches_oracle_over_steps_and_in_a_graph(long):
    wl, x, qs, pu = _case(long)
    lo, hi, cap = _thresholds(wl, x, pu)
    prob = H.problem_of(wl, p_unit=torch.from_numpy(pu).to(H.dev()))
    tiers = H.tiers_of(x)
    ws = hkv.Workspace(prob, *tiers)
    st = hkv.MtiState.allocate(prob, H.dev(), lo, hi, cap)
    out = hkv.StepOutputs.allocate(prob, tiers[1], H.dev(), with_z=True)
    U, bmax, scale = wl.units, wl.bmax, H.scale_of(wl)
    ot = lambda t: oracle.Tier(to_host_bits(t.k), to_host_bits(t.v), t.len.cpu().numpy())
    hd, hs, hc = ot(x.dense), ot(x.sparse), ot(x.condensed)
    ref_state = _host_state(st)
    seen_reuse = seen_rewrite = seen_sparse = 0
    for i in range(STEPS):
        x.q.copy_(qs[i])
        hkv.step_mti(prob, x.q, *tiers, st, out, ws)
        torch.cuda.synchronize()
        assert ws.status() == 0, i
        q = to_host_bits(x.q)
        k = out.sel_len.cpu().numpy()
        idx = out.idx.cpu().numpy().reshape(U, bmax)
        res, ref_state = oracle.step_mti(q, hd, hs, hc, scale, wl.p, wl.bmin, bmax, ref_state, lo, hi, cap,
                                         k_fresh=k, idx_fresh=idx, p_unit=pu)
        got = _host_state(st)
        for key in ("mode", "left", "rw_len"):
            assert np.array_equal(got[key], ref_state[key]), (i, key, got[key], ref_state[key])
        zr = oracle.score(q, hs, scale)
        for u in range(U):
            b, h = divmod(u, wl.Hkv)
            n = int(ref_state["rw_len"][u])
            assert np.array_equal(got["rw_idx"][u, :n], ref_state["rw_idx"][u, :n]), (i, u)
            assert np.array_equal(got["rw_k"][b, h, :n], ref_state["rw_k"][b, h, :n]), (i, u)
            assert np.array_equal(got["rw_v"][b, h, :n], ref_state["rw_v"][b, h, :n]), (i, u)
            if res["fresh"][u]:
                ok, why = H.selection_ok(zr[u], int(hs.len[u]), int(k[u]), idx[u], float(pu[u]), wl.bmin, bmax)
                assert ok, (i, u, why)
                seen_rewrite += int(ref_state["mode"][u] == 1)
                seen_sparse += int(ref_state["mode"][u] == 0)
            else:
                seen_reuse += 1
                assert k[u] == res["k"][u] and np.array_equal(idx[u], res["idx"][u]), (i, u)
        # the attention: fresh units over the GPU's selection, reusing units over their rewrite
        o_ref, l_ref = oracle.attend(q, hd, hs, idx, k, bmax, hc, scale)
        fresh = res["fresh"].astype(bool).repeat(wl.G).reshape(wl.B, wl.Hq)
        o_ref = np.where(fresh[..., None], o_ref, res["out"])
        l_ref = np.where(fresh, l_ref, res["lse"])
        ok, err = H.attn_close(out.out.cpu().numpy(), o_ref)
        assert ok, (i, "out", err)
        ok, err = H.attn_close(out.lse.cpu().numpy(), l_ref)
        assert ok, (i, "lse", err)
    assert seen_reuse > 0 and seen_rewrite > 0 and seen_sparse > 0, (seen_reuse, seen_rewrite, seen_sparse)

    # the same steps as one CUDA graph, from the same start, end in the same state
    final = {key: v.copy() for key, v in _host_state(st).items()}
    out_final = out.out.clone()
    st2 = hkv.MtiState.allocate(prob, H.dev(), lo, hi, cap)
    out2 = hkv.StepOutputs.allocate(prob, tiers[1], H.dev(), with_z=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(STEPS):
            x.q.copy_(qs[i])
            hkv.step_mti(prob, x.q, *tiers, st2, out2, ws, stream=s)
    g.replay()
    torch.cuda.synchronize()
    assert ws.status() == 0
    got = _host_state(st2)
    for key in final:
        assert np.array_equal(got[key], final[key]), key
    assert torch.equal(out2.out, out_final)


def test_step_mti_with_no_rewrites_is_the_plain_step():
    """Thresholds no budget crosses: every step is fresh and equals hkv_step bit for bit."""
    wl, x, qs, pu = _case()
    prob = H.problem_of(wl, p_unit=torch.from_numpy(pu).to(H.dev()))
    tiers = H.tiers_of(x)
    ws = hkv.Workspace(prob, *tiers)
    st = hkv.MtiState.allocate(prob, H.dev(), 1 << 20, 1 << 20, 1 << 30)
    a = hkv.StepOutputs.allocate(prob, tiers[1], H.dev(), with_z=True, with_cut=True, with_stats=True)
    b = hkv.StepOutputs.allocate(prob, tiers[1], H.dev(), with_z=True, with_cut=True, with_stats=True)
    for i in range(3):
        x.q.copy_(qs[i])
        hkv.step_mti(prob, x.q, *tiers, st, a, ws)
        hkv.step(prob, x.q, *tiers, b, ws)
        torch.cuda.synchronize()
        for name in ("sel_len", "idx", "out", "lse", "z", "cut", "m", "logZ"):
            assert torch.equal(getattr(a, name), getattr(b, name)), (i, name)
        assert int(st.left.abs().sum()) == 0 and int(st.mode.abs().sum()) == 0
