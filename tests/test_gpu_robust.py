"""Edge cases, CUDA-graph replay with device-side lengths, device status flags
and a bounded-wait timeout injected from the host (no GPU fault is provoked:
out-of-range lengths are clamped in bounds and the withheld flag makes waits
end by their time limit)."""
import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_step import check_step

pytestmark = pytest.mark.gpu

WL = WORKLOADS[2].with_(B=3, n_cap=2300, w_cap=16, c_cap=8, bmin=5, bmax=400)


def test_empty_and_ragged_units():
    x = H.inputs(WL)
    U = WL.units
    sp = np.full(U, WL.n_cap, np.int32)
    sp[[0, 5, 9]] = [0, 1, 1100]
    de = np.full(U, WL.w_cap, np.int32)
    de[[0, 2]] = 0
    co = np.full(U, WL.c_cap, np.int32)
    co[[0, 3]] = 0
    x.sparse.len.copy_(torch.from_numpy(sp))
    x.dense.len.copy_(torch.from_numpy(de))
    x.condensed.len.copy_(torch.from_numpy(co))
    prob, out, ws = H.run_step(WL, x)
    assert ws.status() == 0
    o = out.out.cpu().numpy()
    lse = out.lse.cpu().numpy()
    # unit 0 has no token at all: out = 0, lse = -inf for its query heads
    assert np.all(o[0, : WL.G] == 0) and np.all(np.isneginf(lse[0, : WL.G]))
    assert out.sel_len.cpu().numpy()[0] == 0
    check_step(WL, x, out, WL.p, WL.bmin, WL.bmax, tag="ragged")


def test_all_scores_tied():
    x = H.inputs(WL)
    x.sparse.k[:] = x.sparse.k[:, :, :1, :]  # every sparse key equal -> every score equal
    for p in (0.1, 0.5, 0.99):
        prob, out, ws = H.run_step(WL, x, p=p)
        k = out.sel_len.cpu().numpy()
        idx = out.idx.cpu().numpy().reshape(WL.units, WL.bmax)
        n = WL.n_cap
        for u in range(WL.units):
            kk = min(n, max(WL.bmin, min(int(np.ceil(p * n - 1e-6 * n)), WL.bmax)))
            assert abs(int(k[u]) - kk) <= 1
            assert np.array_equal(idx[u, : k[u]], np.arange(k[u]))  # ties: lowest indices first
        check_step(WL, x, out, p, WL.bmin, WL.bmax, tag=f"ties p={p}")


def test_extreme_budgets():
    x = H.inputs(WL)
    for bmin, bmax in ((0, 0), (0, 1), (2300, 2300), (400, 5000)):
        wl = WL.with_(bmin=bmin, bmax=bmax)
        prob, out, ws = H.run_step(wl, x, bmin=bmin, bmax=bmax)
        assert ws.status() == 0
        check_step(wl, x, out, wl.p, bmin, bmax, tag=f"clamp {bmin},{bmax}")


def test_cuda_graph_replay_with_device_lengths():
    """One captured hkv_step replayed with new device-side lengths, p_unit and
    queries equals eager calls bit for bit."""
    x = H.inputs(WL)
    U = WL.units
    pu = torch.full((U,), 0.9, device=H.dev())
    prob = H.problem_of(WL, p_unit=pu)
    tiers = H.tiers_of(x)
    ws = hkv.Workspace(prob, *tiers)
    out = hkv.StepOutputs.allocate(prob, tiers[1], H.dev(), with_z=True)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        hkv.step(prob, x.q, *tiers, out, ws, stream=s)  # warm-up outside capture
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        hkv.step(prob, x.q, *tiers, out, ws)
    rng = np.random.default_rng(5)
    for trial in range(4):
        x.sparse.len.copy_(torch.from_numpy(rng.integers(0, WL.n_cap + 1, U).astype(np.int32)))
        x.dense.len.copy_(torch.from_numpy(rng.integers(0, WL.w_cap + 1, U).astype(np.int32)))
        pu.copy_(torch.from_numpy(rng.uniform(0.5, 1.0, U).astype(np.float32)))
        x.q.copy_(torch.randn_like(x.q, dtype=torch.float32).to(x.q.dtype))
        g.replay()
        torch.cuda.synchronize()
        replay = {k: getattr(out, k).clone() for k in ("sel_len", "idx", "out", "lse")}
        hkv.step(prob, x.q, *tiers, out, ws)
        torch.cuda.synchronize()
        for k, v in replay.items():
            assert torch.equal(v, getattr(out, k)), (trial, k)
    assert ws.status() == 0
    del g


def test_length_above_capacity_is_flagged_and_clamped():
    x = H.inputs(WL)
    x.sparse.len[1] = WL.n_cap + 50
    prob, out, ws = H.run_step(WL, x)
    flags = ws.status()
    assert flags & 0x1, flags
    assert ws.status() == 0  # reading cleared the word


def test_negative_temperature_is_flagged():
    x = H.inputs(WL)
    beta = torch.ones(WL.units, device=H.dev())
    beta[2] = -1.0
    prob, out, ws = H.run_step(WL, x, inv_temp=beta)
    assert ws.status() & 0x4


def test_withheld_publish_times_out_and_context_survives():
    """Attention tiles wait for a selection that is never published: each wait
    ends at its limit, the status word reports HKV_DEV_TIMEOUT, and the next
    normal step on the same context is correct."""
    x = H.inputs(WL)
    hkv.set_wait_limit_ns(20_000_000)
    hkv.debug_withhold_publish(True)
    try:
        prob, out, ws = H.run_step(WL, x)
        flags = ws.status()
        assert flags & 0x2, flags
    finally:
        hkv.debug_withhold_publish(False)
        hkv.set_wait_limit_ns(1_000_000_000)
    # the workspace of the failed call is re-zeroed; a fresh call is correct
    prob, out, ws2 = H.run_step(WL, x)
    assert ws2.status() == 0
    check_step(WL, x, out, WL.p, WL.bmin, WL.bmax, tag="after timeout")


def test_candidates_crowded_into_one_warp_segment():
    """A unit whose best 2000 scores are its first 2000 tokens: the warps that
    list the candidates each take a contiguous segment of the unit, so the
    first two segments hold far more candidates than a warp's region, the
    one-sweep list gives up, and the two-sweep list (in another order) with
    the bitmap row takes over. Budgets, cuts, rows and outputs still match the
    oracle; the other units take the one-sweep path in the same launch."""
    wl = WORKLOADS[2].with_(B=1, Hq=8, Hkv=2, n_cap=16000, bmin=1, bmax=2048)
    x = H.inputs(wl)
    g = torch.Generator(device="cpu").manual_seed(7)
    k = x.sparse.k[0, 0]
    # keys along the unit's first query head, longer than the others: the top scores
    q0 = x.q[0, 0].float().cpu()
    scale_k = float(k.float().norm(dim=1).mean())
    noise = 0.05 * torch.randn(2000, wl.D, generator=g)
    k[:2000] = (q0 / q0.norm() * (1.5 * scale_k) + noise).to(k.dtype).to(k.device)
    for p in (0.5, 0.95, 1.0):
        prob, out, ws = H.run_step(wl, x, p=p)
        assert ws.status() == 0
        check_step(wl, x, out, p, wl.bmin, wl.bmax, tag=f"crowded p={p}")
