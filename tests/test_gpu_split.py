"""Units too long for one CTA to stage (more than 24576 sparse tokens), split
over a cluster of CTAs inside hkv_step: four per unit when the clusters all fit
the SMs at once, else two.

Each CTA of the cluster counts and lists its part of the unit; the parts meet
in distributed shared memory, one CTA finds the cut, and every CTA writes its
part of the index row. These cases run that path on long units (uniform and
ragged lengths, flat and spiky heads, bf16 and fp32, short units in the same
launch) and on a unit whose cut falls in a block of identical keys, which no
part can list and which therefore goes back to the one-CTA general path. Each
is checked end to end against the oracle, as the other step tests are."""
import numpy as np
import pytest
import torch

from head_adaptive_kv_b200 import hkv
from head_adaptive_kv_b200.workloads import WORKLOADS, to_host_bits
from tests import gpu_helpers as H
from tests.test_gpu_step import check_step

pytestmark = pytest.mark.gpu

SPLIT_CASES = {
    # 16 units of 40000 tokens: budgets from the mass cut up to the 12000 clamp
    "bf16_long": WORKLOADS[2].with_(B=2, n_cap=40000, bmin=16, bmax=12000),
    # lengths from a few hundred to 60000: short units stay on one CTA
    "bf16_long_ragged": WORKLOADS[3].with_(B=2, n_cap=60000, ctx_range=(320, 60320), bmin=8, bmax=6000),
    # flat and Zipf-spiky heads side by side
    "bf16_hetero_long": WORKLOADS[4].with_(B=1, n_cap=50000, bmax=9000),
    # fp32 keys, D 64, four query heads per KV head
    "fp32_long_d64": WORKLOADS[2].with_(B=1, Hq=8, Hkv=2, D=64, dtype=torch.float32, n_cap=30000, bmin=1,
                                        bmax=3000),
    # 40 units: too many for clusters of four on the SMs at once, so pairs
    "bf16_ragged_pairs": WORKLOADS[3].with_(B=5, n_cap=30000, ctx_range=(320, 30320), bmin=8, bmax=4000),
}


@pytest.mark.parametrize("name", sorted(SPLIT_CASES))
def test_split_step(name):
    wl = SPLIT_CASES[name]
    x = H.inputs(wl)
    for p in (wl.p, 0.5, 0.99, 1.0):
        prob, out, ws = H.run_step(wl, x, p=p)
        assert ws.status() == 0
        check_step(wl, x, out, p, wl.bmin, wl.bmax, tag=f"{name} p={p}")


def test_split_step_with_a_block_of_identical_keys():
    """30000 identical keys in one unit: their scores tie, the bin that holds
    them is far beyond what a part can list, and the unit is redone on the
    one-CTA general path (radix descent); the other unit stays split."""
    wl = WORKLOADS[2].with_(B=1, Hq=8, Hkv=2, n_cap=36000, bmin=1, bmax=20000)
    x = H.inputs(wl)
    x.sparse.k[0, 0, 100:30100] = x.sparse.k[0, 0, 50]
    for p in (0.3, 0.9, 0.999):
        prob, out, ws = H.run_step(wl, x, p=p)
        assert ws.status() == 0
        check_step(wl, x, out, p, wl.bmin, wl.bmax, tag=f"tied p={p}")


def test_split_step_flat_sum_and_rewrite():
    """The split path's rows through the FLAT_SUM layout and the Rewrite Cache
    copy: the same budgets and rows as PAD_MAX, offsets the scan of the
    budgets, and the copied K/V rows bit for bit."""
    wl = SPLIT_CASES["bf16_long_ragged"]
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
    kf = to_host_bits(flat.k_out)
    vf = to_host_bits(flat.v_out)
    ks = to_host_bits(x.sparse.k).reshape(U, -1, wl.D)
    vs = to_host_bits(x.sparse.v).reshape(U, -1, wl.D)
    for u in range(U):
        r = rows[u, : k[u]]
        assert np.array_equal(fl[offs[u]: offs[u + 1]], r)
        assert np.array_equal(kf[offs[u]: offs[u + 1]], ks[u, r])
        assert np.array_equal(vf[offs[u]: offs[u + 1]], vs[u, r])
    assert torch.equal(pad.out, flat.out)
