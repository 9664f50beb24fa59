"""KV append with the dense-window roll (hkv_append) against the oracle: the
tiers' K, V and lengths, the window heads and the dropped flags must match bit
for bit after every call, and a decode loop of append + step captured in one
CUDA graph must decode each step over the tiers the oracle's appends produce."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import TierTensors, to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_stages import CASES

pytestmark = pytest.mark.gpu

PAD = 8  # extra elements per token row: tiers with stride_t = D + PAD


def _rows(g, shape, dtype):
    return torch.randn(*shape, generator=g).to(dtype)


def _padded_tier(g, B, Hkv, cap, D, dtype, lens):
    """A tier whose rows are D + PAD elements apart; the padding is random too
    and must come through every append untouched."""
    k = _rows(g, (B, Hkv, cap, D + PAD), dtype).to(H.dev())
    v = _rows(g, (B, Hkv, cap, D + PAD), dtype).to(H.dev())
    ln = torch.as_tensor(lens, dtype=torch.int32, device=H.dev())
    return SimpleNamespace(kst=k, vst=v, tier=hkv.Tier(k[..., :D], v[..., :D], ln))


def _host(t):
    return oracle.Tier(to_host_bits(t.tier.k), to_host_bits(t.tier.v), t.tier.len.cpu().numpy())


def _empty_host(B, Hkv, D, dtype):
    z = np.zeros((B, Hkv, 0, D), np.uint16 if dtype == torch.bfloat16 else np.float32)
    return oracle.Tier(z, z.copy(), np.zeros(B * Hkv, np.int32))


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


# per-unit starting states (B = 2, Hkv = 3, window 4, sparse 6): an empty
# window, a half-full one, a full one over an empty sparse tier, a full one over
# a full sparse tier (head mid-ring), a full one with head at the last slot, a
# nearly full window over a nearly full sparse tier
W_CAP, N_CAP = 4, 6
DLENS = [0, 2, 4, 4, 4, 3]
SLENS = [0, 5, 0, 6, 3, 5]
HEADS = [0, 0, 0, 2, 3, 0]


@pytest.mark.parametrize("dtype,D", [(torch.bfloat16, 128), (torch.bfloat16, 64), (torch.float32, 128),
                                     (torch.float32, 64)])
def test_append_matches_oracle_bit_for_bit(dtype, D):
    B, Hkv, steps = 2, 3, 11
    g = torch.Generator().manual_seed(4100 + D)
    dense = _padded_tier(g, B, Hkv, W_CAP, D, dtype, DLENS)
    sparse = _padded_tier(g, B, Hkv, N_CAP, D, dtype, SLENS)
    head = torch.as_tensor(HEADS, dtype=torch.int32, device=H.dev())
    dropped = torch.full((B * Hkv,), -1, dtype=torch.int32, device=H.dev())
    prob = hkv.Problem(B, 4 * Hkv, Hkv, D, dtype, 0.9, 1, 8)
    ws = hkv.Workspace(prob, dense.tier, sparse.tier, None)
    pads = [_bits(t[..., D:]).clone() for t in (dense.kst, dense.vst, sparse.kst, sparse.vst)]
    hd, hh, hs = _host(dense), np.array(HEADS, np.int32), _host(sparse)
    total_drops = 0
    for t in range(steps):
        kn, vn = _rows(g, (B, Hkv, D), dtype).to(H.dev()), _rows(g, (B, Hkv, D), dtype).to(H.dev())
        hkv.append(prob, kn, vn, dense.tier, head, sparse.tier, ws, dropped=dropped)
        hd, hh, hs, hdrop = oracle.append(to_host_bits(kn), to_host_bits(vn), hd, hh, hs)
        torch.cuda.synchronize()
        for name, gpu, ref in (("dense k", dense.tier.k, hd.k), ("dense v", dense.tier.v, hd.v),
                               ("sparse k", sparse.tier.k, hs.k), ("sparse v", sparse.tier.v, hs.v)):
            assert np.array_equal(to_host_bits(gpu), ref), (t, name)
        assert np.array_equal(dense.tier.len.cpu().numpy(), hd.len), t
        assert np.array_equal(sparse.tier.len.cpu().numpy(), hs.len), t
        assert np.array_equal(head.cpu().numpy(), hh), t
        assert np.array_equal(dropped.cpu().numpy(), hdrop), t
        st = ws.status()
        assert st == (hkv.DEV_SPARSE_FULL if hdrop.any() else 0), (t, st)
        total_drops += int(hdrop.sum())
    assert total_drops > 0  # the full sparse tiers were reached
    for before, t in zip(pads, (dense.kst, dense.vst, sparse.kst, sparse.vst)):
        assert torch.equal(before, _bits(t[..., D:])), "row padding was written"


@pytest.mark.parametrize("which", ["no_window", "no_sparse"])
def test_append_with_an_empty_tier(which):
    B, Hkv, D, dtype = 1, 2, 128, torch.bfloat16
    g = torch.Generator().manual_seed(4200)
    prob = hkv.Problem(B, 2 * Hkv, Hkv, D, dtype, 0.9, 1, 8)
    dropped = torch.full((B * Hkv,), -1, dtype=torch.int32, device=H.dev())
    if which == "no_window":
        sparse = _padded_tier(g, B, Hkv, 3, D, dtype, [0, 2])
        dense, head, hd = None, None, _empty_host(B, Hkv, D, dtype)
        hs = _host(sparse)
    else:
        dense = _padded_tier(g, B, Hkv, 2, D, dtype, [1, 2])
        head = torch.zeros(B * Hkv, dtype=torch.int32, device=H.dev())
        sparse, hd, hs = None, _host(dense), _empty_host(B, Hkv, D, dtype)
    ws = hkv.Workspace(prob, dense and dense.tier, sparse and sparse.tier, None, device=H.dev())
    hh = np.zeros(B * Hkv, np.int32)
    for t in range(4):
        kn, vn = _rows(g, (B, Hkv, D), dtype).to(H.dev()), _rows(g, (B, Hkv, D), dtype).to(H.dev())
        hkv.append(prob, kn, vn, dense and dense.tier, head, sparse and sparse.tier, ws, dropped=dropped)
        hd, hh, hs, hdrop = oracle.append(to_host_bits(kn), to_host_bits(vn), hd, hh, hs)
        torch.cuda.synchronize()
        live = dense if which == "no_sparse" else sparse
        ref = hd if which == "no_sparse" else hs
        assert np.array_equal(to_host_bits(live.tier.k), ref.k), t
        assert np.array_equal(to_host_bits(live.tier.v), ref.v), t
        assert np.array_equal(live.tier.len.cpu().numpy(), ref.len), t
        if head is not None:
            assert np.array_equal(head.cpu().numpy(), hh), t
        assert np.array_equal(dropped.cpu().numpy(), hdrop), t
        assert ws.status() == (hkv.DEV_SPARSE_FULL if hdrop.any() else 0)


def test_append_leaves_a_corrupt_unit_untouched():
    """A length above its capacity or a head outside the ring: the unit is not
    written and the status word says why; the other units append as usual."""
    B, Hkv, D, dtype = 1, 3, 64, torch.float32
    g = torch.Generator().manual_seed(4300)
    dense = _padded_tier(g, B, Hkv, 4, D, dtype, [4, 5, 4])
    sparse = _padded_tier(g, B, Hkv, 4, D, dtype, [1, 1, 1])
    head = torch.as_tensor([1, 0, 4], dtype=torch.int32, device=H.dev())
    prob = hkv.Problem(B, Hkv, Hkv, D, dtype, 0.9, 1, 8)
    ws = hkv.Workspace(prob, dense.tier, sparse.tier, None)
    before = [t.clone() for t in (dense.kst, dense.vst, sparse.kst, sparse.vst)]
    kn, vn = _rows(g, (B, Hkv, D), dtype).to(H.dev()), _rows(g, (B, Hkv, D), dtype).to(H.dev())
    dropped = torch.full((B * Hkv,), -1, dtype=torch.int32, device=H.dev())
    hkv.append(prob, kn, vn, dense.tier, head, sparse.tier, ws, dropped=dropped)
    torch.cuda.synchronize()
    assert ws.status() == hkv.DEV_LEN_CLAMPED | hkv.DEV_BAD_INDEX
    after = [dense.kst, dense.vst, sparse.kst, sparse.vst]
    for a, b in zip(before, after):
        assert torch.equal(_bits(a[0, 1:]), _bits(b[0, 1:]))  # units 1 and 2 untouched
    assert dense.tier.len.tolist() == [4, 5, 4] and sparse.tier.len.tolist() == [2, 1, 1]
    assert head.tolist() == [2, 0, 4] and dropped.tolist() == [0, 0, 0]
    assert torch.equal(_bits(dense.tier.k[0, 0, 1]), _bits(kn[0, 0]))
    assert torch.equal(_bits(sparse.tier.v[0, 0, 1]), _bits(before[1][0, 0, 1, :D]))


def _check_decode(wl, q, dense_h, sparse_h, cond_h, out, tag):
    """One step's selection by the end-to-end rule and its attention within
    tolerance, both against the oracle over the given host tiers."""
    scale = H.scale_of(wl)
    qh = to_host_bits(q)
    zr = oracle.score(qh, sparse_h, scale).reshape(wl.units, -1)
    k_all = out.sel_len.cpu().numpy()
    idx_all = out.idx.cpu().numpy()[: wl.units * wl.bmax].reshape(wl.units, wl.bmax)
    for u in range(wl.units):
        ok, why = H.selection_ok(zr[u], int(sparse_h.len[u]), int(k_all[u]), idx_all[u], wl.p, wl.bmin,
                                 wl.bmax)
        assert ok, (tag, u, why)
    o_ref, l_ref = oracle.attend(qh, dense_h, sparse_h, idx_all, k_all, wl.bmax, cond_h, scale)
    ok, err = H.attn_close(out.out.cpu().numpy(), o_ref)
    assert ok, (tag, "out", err)
    ok, err = H.attn_close(out.lse.cpu().numpy(), l_ref)
    assert ok, (tag, "lse", err)


def test_decode_loop_in_one_cuda_graph():
    """Four decode steps, each an append of the step's new token followed by
    hkv_step over the updated tiers, captured as one CUDA graph and replayed
    once: every step decodes over the tiers the oracle's appends give."""
    wl = CASES["bf16_ragged"]
    x = H.inputs(wl)
    T = 4
    dense, sparse, cond = H.tiers_of(x)
    prob = H.problem_of(wl)
    ws = hkv.Workspace(prob, dense, sparse, cond)
    head = torch.zeros(wl.units, dtype=torch.int32, device=H.dev())
    dropped = torch.zeros(T, wl.units, dtype=torch.int32, device=H.dev())
    g = torch.Generator().manual_seed(4400)
    kn = _rows(g, (T, wl.B, wl.Hkv, wl.D), wl.dtype).to(H.dev())
    vn = _rows(g, (T, wl.B, wl.Hkv, wl.D), wl.dtype).to(H.dev())
    qs = _rows(g, (T, wl.B, wl.Hq, wl.D), wl.dtype).to(H.dev())
    qs[0] = x.q  # the workload's query, whose group direction the heavy keys follow
    outs = [hkv.StepOutputs.allocate(prob, sparse, H.dev(), with_stats=True) for _ in range(T)]
    # host copies of the starting state, then a warm-up of both calls on
    # scratch copies (kernel attributes are set outside the capture)
    hd, hs, hc = H.host_tier(x.dense), H.host_tier(x.sparse), H.host_tier(x.condensed)
    scratch = [TierTensors(t.k.clone(), t.v.clone(), t.len.clone()) for t in (x.dense, x.sparse)]
    sd, ss = (hkv.Tier(t.k, t.v, t.len) for t in scratch)
    hkv.append(prob, kn[0], vn[0], sd, head.clone(), ss, ws)
    hkv.step(prob, qs[0], sd, ss, cond, outs[0], ws)
    torch.cuda.synchronize()
    assert ws.status() in (0, hkv.DEV_SPARSE_FULL)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for t in range(T):
            hkv.append(prob, kn[t], vn[t], dense, head, sparse, ws, dropped=dropped[t])
            hkv.step(prob, qs[t], dense, sparse, cond, outs[t], ws)
    graph.replay()
    torch.cuda.synchronize()
    st = ws.status()
    hh = np.zeros(wl.units, np.int32)
    for t in range(T):
        hd, hh, hs, hdrop = oracle.append(to_host_bits(kn[t]), to_host_bits(vn[t]), hd, hh, hs)
        assert np.array_equal(dropped[t].cpu().numpy(), hdrop), t
        _check_decode(wl, qs[t], hd, hs, hc, outs[t], f"step {t}")
    assert st == (hkv.DEV_SPARSE_FULL if dropped.any() else 0)
    for gpu, ref in ((x.dense.k, hd.k), (x.dense.v, hd.v), (x.sparse.k, hs.k), (x.sparse.v, hs.v)):
        assert np.array_equal(to_host_bits(gpu), ref)
    assert np.array_equal(x.sparse.len.cpu().numpy(), hs.len)
    assert np.array_equal(head.cpu().numpy(), hh)
    del graph
