"""Seeded synthetic decode workloads for the Cascade Cache step.

This module only makes inputs: it holds none of the step's arithmetic. Both the
CUDA path and the CPU oracle are fed from it (the tests copy device tensors to
the host for the oracle).

The paper measures on math-reasoning generation with Qwen3 models (AIME24,
AIME25, U-Math; 10k+ token contexts -- gist.science Technical Summary of
"HARD-KV: Head-Adaptive Regularization for Decoding-time KV Compression",
section 4 Experimental Results). Neither datasets nor weights are used here:
seeded Gaussian keys/values with planted heavy hitters stand in for the
long-context decode states those runs produce.

Layout of every tier: K and V are ``[B, Hkv, cap, D]`` tensors (D contiguous),
lengths are int32 ``[B*Hkv]``. q is ``[B, Hq, D]``. bf16 values are rounded from
fp32 draws.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np
import torch

# Zipf boost gain of the heterogeneous-head workload: tuned once with the
# oracle so that the spiky heads' median budget at p = 0.8 is about ten tokens.
HETERO_GAMMA = 0.31


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: torch.dtype
    w_cap: int          # dense tier capacity (= its length)
    c_cap: int          # condensed tier capacity (= its length)
    n_cap: int          # sparse tier capacity
    p: float
    bmin: int
    bmax: int
    layers: int = 1
    seed: int = 0
    keys: str = "heavy"              # "normal" | "heavy" | "hetero"
    ctx_range: Optional[tuple] = None  # ragged: total context drawn uniformly in this range
    p_sweep: tuple = ()
    note: str = ""

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def units(self) -> int:
        return self.B * self.Hkv

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five decode workloads (sizes of the tiers follow the dense / sparse /
# condensed split of the Cascade Cache, section 2.A of the Technical Summary).
WORKLOADS: Dict[int, Workload] = {
    1: Workload("tiny_fp32_b1_ctx512", B=1, Hq=4, Hkv=2, D=64, dtype=torch.float32,
                w_cap=64, c_cap=16, n_cap=432, p=0.9, bmin=8, bmax=256, seed=1000,
                keys="normal"),
    2: Workload("bf16_b8_ctx16k", B=8, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16,
                w_cap=256, c_cap=64, n_cap=16064, p=0.95, bmin=64, bmax=2048, seed=2000,
                keys="heavy"),
    3: Workload("bf16_ragged_b64_ctx4k_32k", B=64, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16,
                w_cap=256, c_cap=64, n_cap=32768 - 320, p=0.9, bmin=32, bmax=4096, seed=3000,
                keys="heavy", ctx_range=(4096, 32768)),
    4: Workload("bf16_hetero_b16_ctx16k", B=16, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16,
                w_cap=256, c_cap=64, n_cap=16064, p=0.8, bmin=1, bmax=4096, seed=4000,
                keys="hetero", p_sweep=(0.8, 0.9, 0.95, 0.99)),
    5: Workload("bf16_36layer_b4_ctx64k", B=4, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16,
                w_cap=512, c_cap=128, n_cap=65536 - 640, p=0.95, bmin=128, bmax=8192,
                layers=36, seed=5000, keys="heavy"),
}


@dataclass
class TierTensors:
    k: torch.Tensor
    v: torch.Tensor
    len: torch.Tensor  # int32 [B*Hkv]

    @property
    def cap(self) -> int:
        return self.k.shape[2]


@dataclass
class StepInputs:
    wl: Workload
    q: torch.Tensor
    dense: TierTensors
    sparse: TierTensors
    condensed: TierTensors
    layer: int = 0
    extra: dict = field(default_factory=dict)


def _gen(device: torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _randn(shape, gen, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return x.mul_(std) if std != 1.0 else x


def sparse_lengths(wl: Workload, seed: int) -> np.ndarray:
    """Per-unit sparse lengths; ragged workloads draw a context per sequence."""
    if wl.ctx_range is None:
        return np.full(wl.units, wl.n_cap, np.int32)
    rng = np.random.Generator(np.random.PCG64(seed))
    lo, hi = wl.ctx_range
    ctx = rng.integers(lo, hi + 1, size=wl.B)
    n = np.minimum(ctx - wl.w_cap - wl.c_cap, wl.n_cap).astype(np.int32)
    return np.repeat(n, wl.Hkv).astype(np.int32)


def _group_direction(q32: torch.Tensor, wl: Workload) -> torch.Tensor:
    """sqrt(D) * qbar / |qbar|^2 per unit, qbar = mean of the group's queries.

    A key displaced by a multiple ``a`` of this vector gains a scaled logit of
    about ``a`` against the group's queries.
    """
    qbar = q32.view(wl.B, wl.Hkv, wl.G, wl.D).mean(dim=2)
    return qbar * (math.sqrt(wl.D) / qbar.pow(2).sum(-1, keepdim=True))


def make_inputs(wl: Workload, device="cpu", layer: int = 0,
                n_override: Optional[np.ndarray] = None) -> StepInputs:
    """Draw one layer's decode state for workload ``wl`` (seed = wl.seed + layer)."""
    device = torch.device(device)
    seed = wl.seed + layer
    gen = _gen(device, seed)
    B, Hkv, D = wl.B, wl.Hkv, wl.D
    q32 = _randn((B, wl.Hq, D), gen, device)
    q = q32.to(wl.dtype)
    q32 = q.float()

    lens = sparse_lengths(wl, seed) if n_override is None else np.asarray(n_override, np.int32)

    def tier(cap: int, length: np.ndarray, keys: str) -> TierTensors:
        k = torch.empty((B, Hkv, cap, D), dtype=wl.dtype, device=device)
        v = torch.empty((B, Hkv, cap, D), dtype=wl.dtype, device=device)
        for b in range(B):  # per sequence, to bound fp32 temporaries
            k[b] = _randn((Hkv, cap, D), gen, device, 0.1 if keys == "hetero_flat" else 1.0).to(wl.dtype)
            v[b] = _randn((Hkv, cap, D), gen, device).to(wl.dtype)
        return TierTensors(k, v, torch.as_tensor(length, dtype=torch.int32, device=device))

    dense = tier(wl.w_cap, np.full(wl.units, wl.w_cap, np.int32), "normal")
    condensed = tier(wl.c_cap, np.full(wl.units, wl.c_cap, np.int32), "normal")
    sparse = tier(wl.n_cap, lens, "hetero_flat" if wl.keys == "hetero" else "normal")

    if wl.keys in ("heavy", "hetero"):
        direction = _group_direction(q32, wl)  # [B, Hkv, D]
        hv = np.random.Generator(np.random.PCG64(seed + 7919))
        for u in range(wl.units):
            b, h = divmod(u, Hkv)
            n = int(lens[u])
            if n == 0:
                continue
            if wl.keys == "heavy":
                # 1% of the sparse positions, a per-head boost a ~ U[0, 4].
                m = int(math.ceil(0.01 * n))
                pos = hv.choice(n, size=m, replace=False)
                a = np.full(m, hv.uniform(0.0, 4.0), np.float32)
            else:
                if h < Hkv // 2:
                    continue  # near-flat heads
                # every position gets gamma * ln(s), s ~ Zipf(1.2)
                pos = np.arange(n)
                s = hv.zipf(1.2, size=n).astype(np.float64)
                a = (HETERO_GAMMA * np.log(s)).astype(np.float32)
            pos_t = torch.as_tensor(pos, dtype=torch.long, device=device)
            a_t = torch.as_tensor(a, device=device)
            rows = sparse.k[b, h, pos_t].float() + a_t[:, None] * direction[b, h][None, :]
            sparse.k[b, h, pos_t] = rows.to(wl.dtype)

    return StepInputs(wl, q, dense, sparse, condensed, layer)


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of ``wl`` with some sizes changed (for small parity cases)."""
    return wl.with_(**kw)


def to_host_bits(t: torch.Tensor) -> np.ndarray:
    """A tensor as a host numpy array: bf16 as raw uint16 bits, fp32 as float32."""
    t = t.detach().to("cpu")
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float32:
        return t.contiguous().numpy()
    if t.dtype == torch.int32:
        return t.contiguous().numpy()
    raise TypeError(t.dtype)


def lens_list(t: torch.Tensor) -> List[int]:
    return [int(x) for x in t.cpu().tolist()]
