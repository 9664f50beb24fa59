"""hkv_cascade_decode_noalloc: the cascade decode for callers that cannot
allocate device memory where they decode (an engine that hands nearly all HBM
to its KV pool at start-up, a plugin hook with no workspace to give). Its
scratch is a fixed array inside the library instead of a caller workspace, so
these tests check that it gives what the workspace entry point gives, call
after call, and that a problem too large for the array is refused up front.

This file is named to be collected last: the array keeps whatever the previous
call left in it, and the tests must pass both alone in a fresh process and
after every other test of the suite."""
import ctypes as C

import pytest
import torch

from head_adaptive_kv_b200 import hkv
from tests import gpu_helpers as H
from tests.test_gpu_stages import CASES


def _reference_and_inputs(name, layout=hkv.PAD_MAX):
    """Selection from hkv_step (index rows in `layout`), then the workspace
    cascade decode over it."""
    wl = CASES[name]
    x = H.inputs(wl)
    prob, step_out, ws = H.run_step(wl, x, layout=layout)
    dense, sparse, cond = H.tiers_of(x)
    ref = torch.zeros(wl.B, wl.Hq, wl.D, device=H.dev())
    ref_lse = torch.zeros(wl.B, wl.Hq, device=H.dev())
    hkv.cascade_decode(prob, x.q, dense, sparse, step_out.idx, step_out.sel_len, cond, ref, ws, lse=ref_lse,
                       offsets=step_out.offsets)
    torch.cuda.synchronize()
    assert ws.status() == 0
    return wl, x, prob, step_out, (dense, sparse, cond), ref, ref_lse


@pytest.mark.gpu
def test_noalloc_decode_matches_workspace_decode_on_consecutive_calls():
    # calls in a row on different problems and layouts, the first problem
    # again, and calls without lse or status: each must match the workspace
    # entry point whatever the array last held
    cases = [("bf16_b2_n3000", hkv.PAD_MAX, True), ("fp32_d128_g8", hkv.PAD_MAX, True),
             ("bf16_ragged", hkv.FLAT_SUM, True), ("bf16_b2_n3000", hkv.PAD_MAX, True),
             ("bf16_hetero", hkv.FLAT_SUM, False), ("bf16_b2_n3000", hkv.PAD_MAX, False)]
    for call, (name, layout, extras) in enumerate(cases):
        wl, x, prob, so, (dense, sparse, cond), ref, ref_lse = _reference_and_inputs(name, layout)
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan")) if extras else None
        status = torch.full((1,), -1, dtype=torch.int32, device=H.dev()) if extras else None
        hkv.cascade_decode_noalloc(prob, x.q, dense, sparse, so.idx, so.sel_len, cond, out, lse=lse,
                                   offsets=so.offsets, status=status)
        torch.cuda.synchronize()
        if status is not None:
            assert int(status.item()) == 0, (call, name, int(status.item()))
        ok, err = H.attn_close(out.cpu().numpy(), ref.cpu().numpy())
        assert ok, (call, name, "out", err)
        if lse is not None:
            ok, err = H.attn_close(lse.cpu().numpy(), ref_lse.cpu().numpy())
            assert ok, (call, name, "lse", err)


def test_noalloc_refuses_problems_beyond_its_array():
    """Refused on the host before anything touches a device (runs without a GPU)."""
    prob = hkv.Problem(B=512, Hq=32, Hkv=8, D=128, dtype=torch.bfloat16, p=0.9, bmin=32, bmax=256)
    cap = 4096

    def tier(cap_, addr):
        return hkv._Tier(addr, addr + 0x1000000, 8 * 128 * cap_, 128 * cap_, 128, cap_, 0x2000)

    dense, sparse, cond = tier(256, 0x10000), tier(cap, 0x20000000), tier(64, 0x40000000)
    st = hkv.lib.hkv_cascade_decode_noalloc(C.byref(prob.c()), C.c_void_p(0x100000), C.byref(dense),
                                            C.byref(sparse), C.c_void_p(0x200000), None, C.c_void_p(0x300000),
                                            C.byref(cond), C.c_void_p(0x400000), None, None, None)
    assert hkv.STATUS[st] == "HKV_ERR_WORKSPACE"
    # the same problem fits the workspace entry point, whose size is the caller's
    n = C.c_size_t(0)
    assert hkv.lib.hkv_workspace_size(C.byref(prob.c()), C.byref(dense), C.byref(sparse), C.byref(cond),
                                      C.byref(n)) == 0
    assert n.value > 4 << 20
