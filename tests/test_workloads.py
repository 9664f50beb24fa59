"""The seeded input generators (CPU): the same seed gives the same bits, each
layer gets its own state, shapes and lengths follow the workload table, and the
ragged workload's lengths follow its context range."""
import numpy as np
import torch

from head_adaptive_kv_b200.workloads import WORKLOADS, make_inputs, sparse_lengths


def _small(i, **kw):
    """Workload i with fewer sequences and a shorter sparse tier (CPU sizes)."""
    wl = WORKLOADS[i]
    d = dict(B=min(wl.B, 2), n_cap=min(wl.n_cap, 600))
    if wl.ctx_range is not None:
        d["ctx_range"] = (wl.w_cap + wl.c_cap + 1, wl.w_cap + wl.c_cap + 600)
    d.update(kw)
    return wl.with_(**d)


def test_same_seed_same_bits_and_layers_differ():
    wl = _small(2)
    a, b, c = make_inputs(wl), make_inputs(wl), make_inputs(wl, layer=1)
    for x, y in ((a.q, b.q), (a.sparse.k, b.sparse.k), (a.dense.v, b.dense.v), (a.condensed.k, b.condensed.k)):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))
    assert not torch.equal(a.q, c.q) and not torch.equal(a.sparse.k, c.sparse.k)


def test_shapes_dtypes_and_lengths_follow_the_table():
    for i in sorted(WORKLOADS):
        wl = _small(i)
        x = make_inputs(wl)
        U = wl.B * wl.Hkv
        assert x.q.shape == (wl.B, wl.Hq, wl.D) and x.q.dtype == wl.dtype
        for t, cap in ((x.dense, wl.w_cap), (x.sparse, wl.n_cap), (x.condensed, wl.c_cap)):
            assert t.k.shape == (wl.B, wl.Hkv, cap, wl.D) and t.v.shape == t.k.shape
            assert t.k.dtype == wl.dtype and t.k.stride(3) == 1
            assert t.len.dtype == torch.int32 and t.len.shape == (U,)
            assert int(t.len.min()) >= 0 and int(t.len.max()) <= cap
        assert torch.all(x.dense.len == wl.w_cap) and torch.all(x.condensed.len == wl.c_cap)
        if wl.ctx_range is None:
            assert torch.all(x.sparse.len == wl.n_cap)


def test_ragged_lengths_follow_the_context_range():
    wl = WORKLOADS[3]
    n = sparse_lengths(wl, wl.seed)
    lo, hi = wl.ctx_range
    assert n.shape == (wl.units,)
    assert np.all(n >= lo - wl.w_cap - wl.c_cap) and np.all(n <= min(hi - wl.w_cap - wl.c_cap, wl.n_cap))
    per_seq = n.reshape(wl.B, wl.Hkv)
    assert np.all(per_seq == per_seq[:, :1])        # one context per sequence, shared by its heads
    assert len(np.unique(per_seq[:, 0])) > wl.B // 2  # and the contexts differ between sequences
