"""Fitted temperature on the GPU against the oracle: the group-averaged
raw-attention entropy (hkv_attention_entropy), the inverse temperature that
meets a target (hkv_fit_temperature), and the decode step that fits it before
selecting (hkv_step with beta_fit).

Tolerances. The GPU's per-head logits carry fp32 dot-product rounding and its
exponentials come from the SFU (relative error below 2^-22), so its entropies
differ from the oracle's float64 ones by far less than H_ATOL + H_RTOL * H.
A fitted beta is accepted when the oracle's own float64 entropy at that beta is
within FIT_TOL * max(1, target) of the target (the root is what is unique; its
position moves with the slope of the entropy), and, where that slope is not
small, when beta is within BETA_RTOL of the oracle's root."""
import math

import numpy as np
import pytest
import torch

import oracle
from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_stages import CASES

pytestmark = pytest.mark.gpu

H_ATOL, H_RTOL = 2e-4, 1e-5
FIT_TOL = 1e-5
BETA_RTOL = 1e-3


def _entropy64(z, beta):
    return oracle.softmax_entropy(beta * np.asarray(z, np.float64))


def _check_fit(z_host, lens, target, beta_gpu, tag):
    """beta_gpu against the oracle for metric rows z_host and targets."""
    ref = oracle.fit_temperature(z_host, lens, target)
    for u in range(len(lens)):
        n = int(lens[u])
        b, r, t = float(beta_gpu[u]), float(ref[u]), float(target[u])
        zu = np.asarray(z_host[u, :n], np.float64)
        if n <= 1 or zu.max() == zu.min():
            assert b == 1.0, (tag, u, b)
            continue
        if r in (0.0, oracle.FIT_BETA_MAX):
            assert b == r, (tag, u, b, r)
            continue
        err = abs(_entropy64(zu, b) - t)
        assert err <= FIT_TOL * max(1.0, t), (tag, u, b, r, err)
        P = np.exp(r * (zu - zu.max()))
        P /= P.sum()
        slope = r * (np.sum(P * zu * zu) - np.sum(P * zu) ** 2)
        if slope > 1e-2:
            assert abs(b - r) <= BETA_RTOL * max(1.0, r), (tag, u, b, r, slope)


@pytest.mark.parametrize("name", sorted(CASES))
def test_attention_entropy_matches_oracle(name):
    wl = CASES[name]
    x = H.inputs(wl)
    prob = H.problem_of(wl)
    dense, sparse, cond = H.tiers_of(x)
    ws = hkv.Workspace(prob, dense, sparse, cond)
    h = torch.full((wl.units,), float("nan"), device=H.dev())
    hkv.attention_entropy(prob, x.q, sparse, h, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    ref = oracle.attention_entropy(to_host_bits(x.q), H.host_tier(x.sparse), H.scale_of(wl))
    got = h.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= H_ATOL + H_RTOL * np.abs(ref)), (name, float(err.max()))


@pytest.mark.parametrize("name", sorted(CASES))
def test_fit_temperature_matches_oracle(name):
    """Targets spread over the reachable range of each unit, fitted on the
    GPU's own scores (the same z on both sides)."""
    wl = CASES[name]
    x = H.inputs(wl)
    prob = H.problem_of(wl)
    dense, sparse, cond = H.tiers_of(x)
    ws = hkv.Workspace(prob, dense, sparse, cond)
    z = torch.zeros(wl.units, sparse.cap, device=H.dev())
    hkv.score(prob, x.q, sparse, z, ws)
    lens = x.sparse.len.cpu().numpy()
    rng = np.random.default_rng(31)
    frac = rng.uniform(0.05, 0.98, wl.units)
    target = np.array([f * math.log(max(int(n), 2)) for f, n in zip(frac, lens)], np.float32)
    beta = torch.full((wl.units,), float("nan"), device=H.dev())
    hkv.fit_temperature(prob, z, sparse, torch.as_tensor(target, device=H.dev()), beta, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    _check_fit(z.cpu().numpy(), lens, target.astype(np.float64), beta.cpu().numpy(), name)


def test_fit_temperature_edge_cases():
    """Empty and one-token units, constant scores, a target at ln n, one out of
    reach, a staged and an unstaged (longer than shared memory) unit, and a NaN
    target (1 and a status bit)."""
    B, Hkv, D, cap = 1, 8, 64, 30000
    prob = hkv.Problem(B, Hkv, Hkv, D, torch.float32, 0.9, 1, 8)
    lens = np.array([0, 1, 50, 50, 50, 30000, 4000, 50], np.int32)
    rng = np.random.default_rng(41)
    z = rng.standard_normal((B * Hkv, cap)).astype(np.float32)
    z[2] = 0.75                              # constant scores
    z[4, :2] = 10.0                          # two tied maxima: the entropy never falls below ln 2
    tgt = np.array([1.0, 0.5, 1.0, math.log(50) + 1e-3, 0.1, 0.6 * math.log(30000), 0.3 * math.log(4000),
                    float("nan")], np.float32)
    kk = torch.zeros(B, Hkv, cap, D, device=H.dev())
    sparse = hkv.Tier(kk, kk, torch.as_tensor(lens, device=H.dev()))
    ws = hkv.Workspace(prob, None, sparse, None)
    zt = torch.as_tensor(z, device=H.dev())
    beta = torch.full((B * Hkv,), float("nan"), device=H.dev())
    hkv.fit_temperature(prob, zt, sparse, torch.as_tensor(tgt, device=H.dev()), beta, ws)
    torch.cuda.synchronize()
    assert ws.status() == hkv.DEV_BAD_TEMP
    b = beta.cpu().numpy()
    assert b[0] == 1.0 and b[1] == 1.0 and b[2] == 1.0 and b[7] == 1.0
    assert b[3] == 0.0
    assert b[4] == oracle.FIT_BETA_MAX
    _check_fit(z[5:7], lens[5:7], tgt[5:7].astype(np.float64), b[5:7], "long units")


@pytest.mark.parametrize("name", ["bf16_b2_n3000", "fp32_d128_g8", "bf16_hetero"])
def test_step_with_fitted_temperature(name):
    """hkv_step with beta_fit: the targets and betas equal the standalone calls
    bit for bit, the betas meet the oracle's targets, and the selection and the
    attention follow the oracle at the fitted beta."""
    wl = CASES[name]
    x = H.inputs(wl)
    prob = H.problem_of(wl)
    dense, sparse, cond = H.tiers_of(x)
    ws = hkv.Workspace(prob, dense, sparse, cond)
    out = hkv.StepOutputs.allocate(prob, sparse, H.dev(), with_z=True, with_stats=True)
    out.beta_fit = torch.full((wl.units,), float("nan"), device=H.dev())
    out.h_attn = torch.full((wl.units,), float("nan"), device=H.dev())
    hkv.step(prob, x.q, dense, sparse, cond, out, ws)
    torch.cuda.synchronize()
    assert ws.status() == 0
    # the standalone chain gives the same bits
    h2 = torch.zeros(wl.units, device=H.dev())
    hkv.attention_entropy(prob, x.q, sparse, h2, ws)
    b2 = torch.zeros(wl.units, device=H.dev())
    hkv.fit_temperature(prob, out.z, sparse, h2, b2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out.h_attn, h2) and torch.equal(out.beta_fit, b2)
    # against the oracle
    lens = x.sparse.len.cpu().numpy()
    qh, sp = to_host_bits(x.q), H.host_tier(x.sparse)
    scale = H.scale_of(wl)
    h_ref = oracle.attention_entropy(qh, sp, scale)
    h_gpu = out.h_attn.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(h_gpu - h_ref) <= H_ATOL + H_RTOL * np.abs(h_ref)), name
    z_ref = oracle.score(qh, sp, scale).reshape(wl.units, -1)
    beta = out.beta_fit.cpu().numpy()
    _check_fit(out.z.cpu().numpy(), lens, h_gpu, beta, name)
    k_all = out.sel_len.cpu().numpy()
    idx_all = out.idx.cpu().numpy()[: wl.units * wl.bmax].reshape(wl.units, wl.bmax)
    for u in range(wl.units):
        ok, why = H.selection_ok(z_ref[u], int(lens[u]), int(k_all[u]), idx_all[u], wl.p, wl.bmin, wl.bmax,
                                 float(beta[u]))
        assert ok, (name, u, why)
    o_ref, l_ref = oracle.attend(qh, H.host_tier(x.dense), sp, idx_all, k_all, wl.bmax, H.host_tier(x.condensed),
                                 scale)
    ok, err = H.attn_close(out.out.cpu().numpy(), o_ref)
    assert ok, (name, "out", err)
