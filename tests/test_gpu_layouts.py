"""The attention reads the selected tokens' rows by four-row TMA gathers when
the sparse tier is laid out plainly (rows of D contiguous elements, units
back to back) and by per-row copies otherwise. The same tokens in both
layouts must give the same results bit for bit: the copies differ, the
arithmetic and its order do not. Both are also checked against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_step import check_step

pytestmark = pytest.mark.gpu

PAD = 8  # extra elements per row of the padded copy: stride_t = D + PAD

CASES = {
    "bf16_d128_g4": WORKLOADS[2].with_(B=2, n_cap=3000, bmin=4, bmax=700),
    "bf16_d64_g8": WORKLOADS[2].with_(B=2, Hq=16, Hkv=2, D=64, n_cap=2500, bmin=1, bmax=600),
    "fp32_d128_g2": WORKLOADS[2].with_(B=1, Hq=8, Hkv=4, dtype=torch.float32, n_cap=2000, bmin=8, bmax=500),
}


def _padded(t: torch.Tensor) -> torch.Tensor:
    """The same [B, Hkv, cap, D] values with rows D + PAD elements apart."""
    B, Hkv, cap, D = t.shape
    buf = torch.zeros((B, Hkv, cap, D + PAD), dtype=t.dtype, device=t.device)
    buf[..., :D] = t
    return buf[..., :D]


def _padded_sparse(x) -> hkv.Tier:
    return hkv.Tier(_padded(x.sparse.k), _padded(x.sparse.v), x.sparse.len)


@pytest.mark.parametrize("name", sorted(CASES))
def test_step_same_bits_in_both_layouts(name):
    wl = CASES[name]
    x = H.inputs(wl)
    prob, plain, ws = H.run_step(wl, x)
    assert ws.status() == 0
    check_step(wl, x, plain, wl.p, wl.bmin, wl.bmax, tag=f"{name} plain")
    dense, _, cond = H.tiers_of(x)
    sparse = _padded_sparse(x)
    ws2 = hkv.Workspace(prob, dense, sparse, cond)
    padded = hkv.StepOutputs.allocate(prob, sparse, H.dev(), with_z=True, with_cut=True, with_stats=True)
    hkv.step(prob, x.q, dense, sparse, cond, padded, ws2)
    torch.cuda.synchronize()
    assert ws2.status() == 0
    assert torch.equal(plain.sel_len, padded.sel_len)
    assert torch.equal(plain.idx, padded.idx)
    assert torch.equal(plain.out, padded.out)
    assert torch.equal(plain.lse, padded.lse)


@pytest.mark.parametrize("name", sorted(CASES))
def test_cascade_decode_same_bits_in_both_layouts(name):
    wl = CASES[name]
    x = H.inputs(wl)
    prob, st, _ = H.run_step(wl, x)
    idx, sel = st.idx, st.sel_len
    dense, sparse, cond = H.tiers_of(x)
    results = []
    for sp in (sparse, _padded_sparse(x)):
        ws = hkv.Workspace(prob, dense, sp, cond)
        out = torch.zeros(wl.B, wl.Hq, wl.D, device=H.dev())
        lse = torch.zeros(wl.B, wl.Hq, device=H.dev())
        hkv.cascade_decode(prob, x.q, dense, sp, idx, sel, cond, out, ws, lse=lse)
        torch.cuda.synchronize()
        assert ws.status() == 0
        results.append((out, lse))
    assert torch.equal(results[0][0], results[1][0])
    assert torch.equal(results[0][1], results[1][1])
    k = sel.cpu().numpy()
    o_ref, l_ref = oracle.attend(to_host_bits(x.q), H.host_tier(x.dense), H.host_tier(x.sparse),
                                 idx.cpu().numpy().reshape(wl.units, wl.bmax), k, wl.bmax,
                                 H.host_tier(x.condensed), H.scale_of(wl))
    ok, err = H.attn_close(results[0][0].cpu().numpy(), o_ref)
    assert ok, (name, err)
    ok, err = H.attn_close(results[0][1].cpu().numpy(), l_ref)
    assert ok, (name, err)
