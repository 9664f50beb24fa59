"""Bins too large to sort: the exact radix descent of the selection.

The selection drops scores into linear bins over each unit's range and resolves
the bin where the cut falls by sorting its tokens; a bin of more than 6144
tokens is resolved instead by a radix descent over its score keys, by mass
(the Top-p cut) or by count (a clamp). These cases put over 10000 tokens into
one bin, on a unit whose scores are staged in shared memory (n <= 24576) and on
one that is not (n > 24576), and compare budgets, cuts and index rows with the
oracle: given identical fp32 scores, bit for bit except at an ambiguous cut."""
import math

import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, make_inputs
from tests import gpu_helpers as H
from tests.test_gpu_step import check_step

pytestmark = pytest.mark.gpu

N_STAGED, N_GLOBAL = 12000, 30000


def one_big_bin(n, seed):
    """One score at 5, one at -5, the other n - 2 in [0.001, 0.0035]: with 2048
    linear bins over [-5, 5] they all fall into bin 1023."""
    rng = np.random.default_rng(seed)
    z = rng.uniform(0.001, 0.0035, n).astype(np.float32)
    hi, lo = rng.choice(n, 2, replace=False)
    z[hi], z[lo] = 5.0, -5.0
    bins = np.floor((np.float32(5.0) - z.astype(np.float64)) * (2048 / 10.0))
    assert np.sum(bins == 1023) == n - 2 > 6144
    return z


@pytest.mark.parametrize("p,bmin,bmax", [
    (0.5, 1, N_GLOBAL),      # the mass decides, inside the big bin
    (0.5, 1, 3000),          # a mass descent, then the clamp at bmax (count descent)
    (0.2, 7000, N_GLOBAL),   # the clamp at bmin above k* (count descent)
    (0.999, 1, N_GLOBAL),    # a cut near the end of the bin
])
def test_big_bin_radix_descent(p, bmin, bmax):
    U = 2
    z = np.zeros((U, N_GLOBAL), np.float32)
    z[0, :N_STAGED] = one_big_bin(N_STAGED, 1)
    z[1] = one_big_bin(N_GLOBAL, 2)
    ln = np.array([N_STAGED, N_GLOBAL], np.int32)
    wl = WORKLOADS[2].with_(B=1, Hq=2, Hkv=2, n_cap=N_GLOBAL, bmin=bmin, bmax=bmax)
    prob = H.problem_of(wl, p=p, bmin=bmin, bmax=bmax)
    dev = H.dev()
    k_dummy = torch.zeros(1, U, N_GLOBAL, wl.D, dtype=torch.bfloat16, device=dev)
    sparse = hkv.Tier(k_dummy, None, torch.from_numpy(ln).to(dev))
    ws = hkv.Workspace(prob, None, sparse, None)
    zt = torch.from_numpy(z).to(dev)
    sel = torch.zeros(U, dtype=torch.int32, device=dev)
    cut = torch.zeros(U, 4, dtype=torch.int32, device=dev)
    hkv.topp_select(prob, zt, sparse, sel, cut, ws)
    idx = torch.full((U * bmax,), -7, dtype=torch.int32, device=dev)
    hkv.compact(prob, zt, sparse, sel, cut, idx, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    kg = sel.cpu().numpy()
    r = oracle.topp(z, ln, p, bmin, bmax)
    ok, bad = H.budgets_match(kg, r, p, z, ln)
    assert ok, bad
    # the mass (first two cases) or the clamp decided inside the big bin
    assert np.all(kg > 2)
    ct = cut.cpu().numpy()
    assert np.array_equal(ct[:, 1] + ct[:, 2], kg)
    ks = ct[:, 3]
    for u in range(U):
        if r["kstar"][u] <= bmax and p < 1:
            assert ks[u] == r["kstar"][u] or abs(int(ks[u]) - int(r["kstar"][u])) <= 1
    want = oracle.compact(z, ln, kg, bmax)
    assert np.array_equal(idx.cpu().numpy().reshape(U, bmax), want)


def tied_bulk_inputs(wl):
    """A decode state whose sparse keys are all one row except two outliers,
    so that every other score ties in one bin of more than 6144 tokens."""
    x = make_inputs(wl, H.dev(), 0)
    q = x.q.float().view(wl.B, wl.Hkv, wl.G, wl.D)
    qbar = q.mean(dim=2)
    direction = qbar * (math.sqrt(wl.D) / qbar.pow(2).sum(-1, keepdim=True))  # logit ~1 per unit
    for b in range(wl.B):
        for h in range(wl.Hkv):
            d = direction[b, h]
            x.sparse.k[b, h, :] = (0.1 * d).to(wl.dtype)
            x.sparse.k[b, h, 17] = (2.0 * d).to(wl.dtype)
            x.sparse.k[b, h, 4242] = (-2.0 * d).to(wl.dtype)
    return x


@pytest.mark.parametrize("p,bmin,bmax", [(0.5, 1, 30000), (0.95, 64, 3000), (0.3, 9000, 30000)])
def test_step_with_one_huge_tied_bin(p, bmin, bmax):
    """Through hkv_step: a unit of 12000 tokens (its scores staged; the fused
    path gives way to the general one) and one of 30000 (not staged)."""
    wl = WORKLOADS[2].with_(B=1, Hq=8, Hkv=2, n_cap=N_GLOBAL, w_cap=64, c_cap=16, bmin=bmin, bmax=bmax)
    x = tied_bulk_inputs(wl)
    x.sparse.len.copy_(torch.tensor([N_STAGED, N_GLOBAL], dtype=torch.int32))
    prob, out, ws = H.run_step(wl, x, p=p, bmin=bmin, bmax=bmax)
    assert ws.status() == 0
    check_step(wl, x, out, p, bmin, bmax, tag=f"tied p={p} [{bmin},{bmax}]")
