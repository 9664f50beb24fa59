"""Python binding of ``libhkv.so`` (the C ABI declared in ``include/hkv.h``).

Argument marshalling only: every step of the decode path runs in the CUDA
library. torch supplies device memory and the current stream. There is no CPU
fallback: importing this module fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes as C
import os
from dataclasses import dataclass, field
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("HKV_LIBRARY") or os.path.join(_HERE, "libhkv.so")

HKV_BF16, HKV_F32 = 0, 1
PAD_MAX, FLAT_SUM = 0, 1
STATUS = {0: "HKV_OK", 1: "HKV_ERR_INVALID_ARG", 2: "HKV_ERR_UNSUPPORTED", 3: "HKV_ERR_CUDA",
          4: "HKV_ERR_TIMEOUT", 5: "HKV_ERR_DEVICE", 6: "HKV_ERR_WORKSPACE"}
DEV_LEN_CLAMPED, DEV_TIMEOUT, DEV_BAD_TEMP, DEV_BAD_INDEX, DEV_BAD_P = 0x1, 0x2, 0x4, 0x8, 0x10
DEV_SPARSE_FULL = 0x20
CONDENSE_MERGE, CONDENSE_EVICT = 0, 1
CONDENSE_MAX_BLOCK = 8192


class HkvError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class _Tier(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("stride_b", C.c_int64), ("stride_h", C.c_int64),
                ("stride_t", C.c_int64), ("cap", C.c_int32), ("len", C.c_void_p)]


class _Problem(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("D", C.c_int32),
                ("dtype", C.c_int), ("scale", C.c_float), ("p", C.c_float), ("bmin", C.c_int32),
                ("bmax", C.c_int32), ("layout", C.c_int), ("inv_temp", C.c_void_p),
                ("p_unit", C.c_void_p)]


class Cut(C.Structure):
    """Mirror of ``hkv_cut`` (16 bytes per unit)."""
    _fields_ = [("z_cut", C.c_float), ("n_above", C.c_int32), ("n_tie", C.c_int32),
                ("kstar", C.c_int32)]


class _StepOut(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("sel_len", "idx", "offsets", "out", "lse", "z", "cut", "m", "logZ", "k_out", "v_out",
                 "beta_fit", "h_attn")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libhkv.so not built at {LIB_PATH}; run head_adaptive_kv_b200/build.py")
    L = C.CDLL(LIB_PATH)
    P, i32, i64, sz = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t
    sig = {
        "hkv_workspace_size": [P, P, P, P, C.POINTER(C.c_size_t)],
        "hkv_workspace_init": [P, sz, P],
        "hkv_score": [P, P, P, P, i64, P, sz, P],
        "hkv_calibrate": [P, P, i64, P, P, P, P, P, sz, P],
        "hkv_topp_select": [P, P, i64, P, P, P, P, sz, P],
        "hkv_compact": [P, P, i64, P, P, P, P, P, P, P, P, sz, P],
        "hkv_cascade_decode": [P, P, P, P, P, P, P, P, P, P, P, sz, P],
        "hkv_step": [P, P, P, P, P, P, P, sz, P],
        "hkv_step_mti": [P, P, P, P, P, P, P, P, sz, P],
        "hkv_cascade_decode_noalloc": [P, P, P, P, P, P, P, P, P, P, P, P],
        "hkv_append": [P, P, P, P, P, P, P, P, sz, P],
        "hkv_condense": [P, P, P, P, P, i64, P, P, i32, i32, i32, P, P, sz, P],
        "hkv_attention_entropy": [P, P, P, P, P, sz, P],
        "hkv_fit_temperature": [P, P, i64, P, P, P, P, sz, P],
        "hkv_get_status": [P, C.POINTER(C.c_uint32), P],
        "hkv_set_wait_limit_ns": [C.c_uint64],
        "hkv_debug_withhold_publish": [i32],
        "hkv_set_timeline": [i32],
        "hkv_read_timeline": [P, C.POINTER(C.c_uint64), P],
        "hkv_launch_count": [],
        "hkv_status_string": [i32],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = C.c_int
    L.hkv_launch_count.restype = C.c_uint64
    L.hkv_status_string.restype = C.c_char_p
    return L


lib = _load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _check(code: int, what: str):
    if code != 0:
        raise HkvError(code, what)


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return HKV_BF16
    if dt == torch.float32:
        return HKV_F32
    raise TypeError(f"unsupported dtype {dt}")


@dataclass
class Tier:
    """K, V of shape [B, Hkv, cap, D] (D contiguous, any other strides) and len[B*Hkv] int32."""

    k: torch.Tensor
    v: Optional[torch.Tensor]
    len: torch.Tensor

    def c(self) -> _Tier:
        k = self.k
        if k.dim() != 4 or k.stride(3) != 1:
            raise ValueError("tier tensors must be [B, Hkv, cap, D] with D contiguous")
        if self.v is not None and (self.v.shape != k.shape or self.v.stride() != k.stride()):
            raise ValueError("K and V must share shape and strides")
        if self.len.dtype != torch.int32:
            raise TypeError("lengths must be int32")
        return _Tier(k.data_ptr(), None if self.v is None else self.v.data_ptr(), k.stride(0), k.stride(1),
                     k.stride(2), k.shape[2], self.len.data_ptr())

    @property
    def cap(self) -> int:
        return self.k.shape[2]


@dataclass
class Problem:
    B: int
    Hq: int
    Hkv: int
    D: int
    dtype: torch.dtype
    p: float
    bmin: int
    bmax: int
    scale: float = 0.0
    layout: int = PAD_MAX
    inv_temp: Optional[torch.Tensor] = None
    p_unit: Optional[torch.Tensor] = None

    def c(self) -> _Problem:
        return _Problem(self.B, self.Hq, self.Hkv, self.D, _dtype_code(self.dtype), float(self.scale),
                        float(self.p), int(self.bmin), int(self.bmax), int(self.layout),
                        None if self.inv_temp is None else self.inv_temp.data_ptr(),
                        None if self.p_unit is None else self.p_unit.data_ptr())

    @property
    def units(self) -> int:
        return self.B * self.Hkv


def _tref(t: Optional[Tier]):
    return None if t is None else C.byref(t.c())


class Workspace:
    """Device workspace of ``hkv_workspace_size`` bytes, zeroed once on creation."""

    def __init__(self, prob: Problem, dense: Optional[Tier], sparse: Optional[Tier],
                 condensed: Optional[Tier], device=None):
        n = C.c_size_t(0)
        _check(lib.hkv_workspace_size(C.byref(prob.c()), _tref(dense), _tref(sparse), _tref(condensed),
                                      C.byref(n)), "hkv_workspace_size")
        self.nbytes = int(n.value)
        dev = device if device is not None else (sparse or dense).k.device
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=dev)
        off = (-self.buf.data_ptr()) % 256
        self.tensor = self.buf[off: off + self.nbytes]
        _check(lib.hkv_workspace_init(_ptr(self.tensor), self.nbytes, _stream()), "hkv_workspace_init")

    @property
    def ptr(self):
        return _ptr(self.tensor)

    def status(self, stream=None) -> int:
        """Read and clear the device status word; returns the HKV_DEV_* bits."""
        flags = C.c_uint32(0)
        code = lib.hkv_get_status(self.ptr, C.byref(flags), _stream(stream))
        if code not in (0, 4, 5):
            _check(code, "hkv_get_status")
        return int(flags.value)


def score(prob: Problem, q: torch.Tensor, sparse: Tier, z: torch.Tensor, ws: Workspace, stream=None):
    _check(lib.hkv_score(C.byref(prob.c()), _ptr(q), C.byref(sparse.c()), _ptr(z), z.stride(0), ws.ptr,
                         ws.nbytes, _stream(stream)), "hkv_score")


def calibrate(prob: Problem, z: torch.Tensor, sparse: Tier, m: torch.Tensor, logZ: torch.Tensor,
              ws: Workspace, P: Optional[torch.Tensor] = None, stream=None):
    if P is not None and P.stride(0) != z.stride(0):
        raise ValueError("P must share z's row stride")
    _check(lib.hkv_calibrate(C.byref(prob.c()), _ptr(z), z.stride(0), C.byref(sparse.c()), _ptr(P), _ptr(m),
                             _ptr(logZ), ws.ptr, ws.nbytes, _stream(stream)), "hkv_calibrate")


def topp_select(prob: Problem, z: torch.Tensor, sparse: Tier, sel_len: torch.Tensor, cut: torch.Tensor,
                ws: Workspace, stream=None):
    """cut: int32 tensor of shape [units, 4] holding hkv_cut records."""
    _check(lib.hkv_topp_select(C.byref(prob.c()), _ptr(z), z.stride(0), C.byref(sparse.c()), _ptr(sel_len),
                               _ptr(cut), ws.ptr, ws.nbytes, _stream(stream)), "hkv_topp_select")


def compact(prob: Problem, z: torch.Tensor, sparse: Tier, sel_len: torch.Tensor, cut: torch.Tensor,
            idx: torch.Tensor, ws: Workspace, offsets: Optional[torch.Tensor] = None,
            k_out: Optional[torch.Tensor] = None, v_out: Optional[torch.Tensor] = None, stream=None):
    _check(lib.hkv_compact(C.byref(prob.c()), _ptr(z), z.stride(0), C.byref(sparse.c()), _ptr(sel_len),
                           _ptr(cut), _ptr(idx), _ptr(offsets), _ptr(k_out), _ptr(v_out), ws.ptr, ws.nbytes,
                           _stream(stream)), "hkv_compact")


def cascade_decode(prob: Problem, q: torch.Tensor, dense: Optional[Tier], sparse: Optional[Tier],
                   idx: Optional[torch.Tensor], sel_len: Optional[torch.Tensor], condensed: Optional[Tier],
                   out: torch.Tensor, ws: Workspace, lse: Optional[torch.Tensor] = None,
                   offsets: Optional[torch.Tensor] = None, stream=None):
    _check(lib.hkv_cascade_decode(C.byref(prob.c()), _ptr(q), _tref(dense), _tref(sparse), _ptr(idx),
                                  _ptr(offsets), _ptr(sel_len), _tref(condensed), _ptr(out), _ptr(lse), ws.ptr,
                                  ws.nbytes, _stream(stream)), "hkv_cascade_decode")


@dataclass
class StepOutputs:
    sel_len: torch.Tensor
    idx: torch.Tensor
    out: torch.Tensor
    lse: Optional[torch.Tensor] = None
    offsets: Optional[torch.Tensor] = None
    z: Optional[torch.Tensor] = None
    cut: Optional[torch.Tensor] = None
    m: Optional[torch.Tensor] = None
    logZ: Optional[torch.Tensor] = None
    k_out: Optional[torch.Tensor] = None
    v_out: Optional[torch.Tensor] = None
    beta_fit: Optional[torch.Tensor] = None
    h_attn: Optional[torch.Tensor] = None

    def c(self) -> _StepOut:
        return _StepOut(*[None if t is None else t.data_ptr() for t in
                          (self.sel_len, self.idx, self.offsets, self.out, self.lse, self.z, self.cut,
                           self.m, self.logZ, self.k_out, self.v_out, self.beta_fit, self.h_attn)])

    @staticmethod
    def allocate(prob: Problem, sparse: Tier, device, with_z=False, with_cut=False, with_stats=False,
                 rewrite=False) -> "StepOutputs":
        U = prob.units
        dev = torch.device(device)
        o = StepOutputs(
            sel_len=torch.zeros(U, dtype=torch.int32, device=dev),
            idx=torch.zeros(U * max(prob.bmax, 1), dtype=torch.int32, device=dev),
            out=torch.zeros(prob.B, prob.Hq, prob.D, dtype=torch.float32, device=dev),
            lse=torch.zeros(prob.B, prob.Hq, dtype=torch.float32, device=dev),
        )
        if prob.layout == FLAT_SUM:
            o.offsets = torch.zeros(U + 1, dtype=torch.int32, device=dev)
        if with_z:
            o.z = torch.zeros(U, sparse.cap, dtype=torch.float32, device=dev)
        if with_cut:
            o.cut = torch.zeros(U, 4, dtype=torch.int32, device=dev)
        if with_stats:
            o.m = torch.zeros(U, dtype=torch.float32, device=dev)
            o.logZ = torch.zeros(U, dtype=torch.float32, device=dev)
        if rewrite:
            o.k_out = torch.zeros(U * max(prob.bmax, 1), prob.D, dtype=prob.dtype, device=dev)
            o.v_out = torch.zeros_like(o.k_out)
        return o


def step(prob: Problem, q: torch.Tensor, dense: Optional[Tier], sparse: Tier, condensed: Optional[Tier],
         out: StepOutputs, ws: Workspace, stream=None):
    _check(lib.hkv_step(C.byref(prob.c()), _ptr(q), _tref(dense), C.byref(sparse.c()), _tref(condensed),
                        C.byref(out.c()), ws.ptr, ws.nbytes, _stream(stream)), "hkv_step")


class _Mti(C.Structure):
    _fields_ = [("L_lower", C.c_int32), ("L_upper", C.c_int32), ("mti_cap", C.c_int64), ("mode", C.c_void_p),
                ("left", C.c_void_p), ("rewrite", _Tier), ("rw_idx", C.c_void_p)]


@dataclass
class MtiState:
    """Rewrite Cache / Sparse Loading trigger: thresholds, memory-time allowance
    and the per-unit state (mode, left), the rewrite buffer (a Tier of capacity
    >= bmax whose len holds the rows each unit's rewrite keeps) and the token
    indices of those rows (rw_idx, int32 [B*Hkv*bmax])."""

    L_lower: int
    L_upper: int
    mti_cap: int
    mode: torch.Tensor
    left: torch.Tensor
    rewrite: Tier
    rw_idx: torch.Tensor

    def c(self) -> _Mti:
        for t in (self.mode, self.left, self.rw_idx):
            if t.dtype != torch.int32 or not t.is_contiguous():
                raise TypeError("mode, left and rw_idx must be contiguous int32")
        return _Mti(int(self.L_lower), int(self.L_upper), int(self.mti_cap), self.mode.data_ptr(),
                    self.left.data_ptr(), self.rewrite.c(), self.rw_idx.data_ptr())

    @staticmethod
    def allocate(prob: "Problem", device, L_lower: int, L_upper: int, mti_cap: int) -> "MtiState":
        U, dev = prob.units, torch.device(device)
        z = lambda: torch.zeros(U, dtype=torch.int32, device=dev)
        buf = lambda: torch.zeros(prob.B, prob.Hkv, max(prob.bmax, 1), prob.D, dtype=prob.dtype, device=dev)
        return MtiState(L_lower, L_upper, mti_cap, z(), z(), Tier(buf(), buf(), z()),
                        torch.zeros(U * max(prob.bmax, 1), dtype=torch.int32, device=dev))


def step_mti(prob: "Problem", q: torch.Tensor, dense: Optional[Tier], sparse: Tier, condensed: Optional[Tier],
             mti: MtiState, out: "StepOutputs", ws: "Workspace", stream=None):
    """hkv_step under the Rewrite Cache / Sparse Loading trigger (see hkv_step_mti)."""
    _check(lib.hkv_step_mti(C.byref(prob.c()), _ptr(q), _tref(dense), C.byref(sparse.c()), _tref(condensed),
                            C.byref(mti.c()), C.byref(out.c()), ws.ptr, ws.nbytes, _stream(stream)),
           "hkv_step_mti")


def cascade_decode_noalloc(prob: Problem, q: torch.Tensor, dense: Optional[Tier], sparse: Optional[Tier],
                           idx: Optional[torch.Tensor], sel_len: Optional[torch.Tensor],
                           condensed: Optional[Tier], out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                           offsets: Optional[torch.Tensor] = None, status: Optional[torch.Tensor] = None,
                           stream=None):
    """cascade_decode for callers that cannot allocate device memory: no
    workspace argument; the library's fixed scratch array is used instead
    (see hkv_cascade_decode_noalloc in include/hkv.h for its limit and for why
    overlapping calls must be serialised). status: optional device int32/uint32
    tensor of one element that receives the call's device status bits."""
    _check(lib.hkv_cascade_decode_noalloc(C.byref(prob.c()), _ptr(q), _tref(dense), _tref(sparse), _ptr(idx),
                                          _ptr(offsets), _ptr(sel_len), _tref(condensed), _ptr(out), _ptr(lse),
                                          _ptr(status), _stream(stream)), "hkv_cascade_decode_noalloc")


def append(prob: Problem, k_new: torch.Tensor, v_new: torch.Tensor, dense: Optional[Tier],
           head: Optional[torch.Tensor], sparse: Optional[Tier], ws: Workspace,
           dropped: Optional[torch.Tensor] = None, stream=None):
    """KV append with the dense-window roll, in place on the tiers' K, V and
    lengths and on head (int32 [B*Hkv]). k_new, v_new: [B, Hkv, D] contiguous.
    dropped: optional int32 [B*Hkv], 1 where a token left the window while the
    sparse tier was full."""
    for t in (k_new, v_new):
        if not t.is_contiguous() or t.dtype != prob.dtype:
            raise ValueError("k_new and v_new must be contiguous [B, Hkv, D] of the problem's dtype")
    if head is not None and head.dtype != torch.int32:
        raise TypeError("head must be int32")
    _check(lib.hkv_append(C.byref(prob.c()), _ptr(k_new), _ptr(v_new), _tref(dense), _ptr(head),
                          _tref(sparse), _ptr(dropped), ws.ptr, ws.nbytes, _stream(stream)), "hkv_append")


def condense(prob: Problem, sparse: Tier, condensed: Optional[Tier], cond_w: Optional[torch.Tensor],
             ws: Workspace, block: int, trigger: int, policy: int = CONDENSE_MERGE,
             z: Optional[torch.Tensor] = None, m: Optional[torch.Tensor] = None,
             logZ: Optional[torch.Tensor] = None, done: Optional[torch.Tensor] = None, stream=None):
    """Condensed-tier formation, in place on the tiers' K, V and lengths and on
    cond_w (fp32 [B*Hkv, condensed cap]): units whose sparse tier holds at
    least max(trigger, block) tokens turn their oldest `block` tokens into one
    condensed slot (MERGE: weighted mean; EVICT: the most important token),
    weighted by the calibrated probabilities of the step's scores z (with its
    m and logZ; all three or none). done: optional int32 [B*Hkv]."""
    if cond_w is not None and (cond_w.dtype != torch.float32 or not cond_w.is_contiguous()):
        raise ValueError("cond_w must be a contiguous fp32 tensor [B*Hkv, condensed cap]")
    if z is not None and (z.dtype != torch.float32 or z.dim() != 2 or z.stride(1) != 1):
        raise ValueError("z must be fp32 [B*Hkv, >= sparse cap] with contiguous rows")
    _check(lib.hkv_condense(C.byref(prob.c()), C.byref(sparse.c()), _tref(condensed), _ptr(cond_w), _ptr(z),
                            0 if z is None else z.stride(0), _ptr(m), _ptr(logZ), int(block), int(trigger),
                            int(policy), _ptr(done), ws.ptr, ws.nbytes, _stream(stream)), "hkv_condense")


def _f32_vector(t: torch.Tensor, n: int, what: str):
    if t.dtype != torch.float32 or t.dim() != 1 or t.stride(0) != 1 or t.numel() < n:
        raise ValueError(f"{what} must be a contiguous fp32 vector of at least {n} elements")


def attention_entropy(prob: Problem, q: torch.Tensor, sparse: Tier, h: torch.Tensor, ws: Workspace, stream=None):
    """Per unit the group-averaged entropy of the raw attention over the sparse tier (h: fp32 [B*Hkv])."""
    _f32_vector(h, prob.units, "h")
    _check(lib.hkv_attention_entropy(C.byref(prob.c()), _ptr(q), C.byref(sparse.c()), _ptr(h), ws.ptr,
                                     ws.nbytes, _stream(stream)), "hkv_attention_entropy")


def fit_temperature(prob: Problem, z: torch.Tensor, sparse: Tier, h_target: torch.Tensor, beta: torch.Tensor,
                    ws: Workspace, stream=None):
    """Per unit the inverse temperature at which softmax(beta z) has entropy
    h_target (z: fp32 [B*Hkv, >= cap]; h_target, beta: fp32 [B*Hkv])."""
    if z.dtype != torch.float32 or z.dim() != 2 or z.stride(1) != 1 or z.shape[1] < sparse.cap:
        raise ValueError("z must be fp32 [B*Hkv, >= cap] with contiguous rows")
    _f32_vector(h_target, prob.units, "h_target")
    _f32_vector(beta, prob.units, "beta")
    _check(lib.hkv_fit_temperature(C.byref(prob.c()), _ptr(z), z.stride(0), C.byref(sparse.c()), _ptr(h_target),
                                   _ptr(beta), ws.ptr, ws.nbytes, _stream(stream)), "hkv_fit_temperature")


def set_wait_limit_ns(ns: int):
    _check(lib.hkv_set_wait_limit_ns(int(ns)), "hkv_set_wait_limit_ns")


TL_KINDS = ("score", "select", "attention", "merge", "layout", "fit", "trigger")


def set_timeline(on: bool):
    """Record the step kernels' start and end times in their workspace (see hkv_set_timeline)."""
    _check(lib.hkv_set_timeline(1 if on else 0), "hkv_set_timeline")


def read_timeline(ws: Workspace, stream=None) -> dict:
    """Read and clear a workspace's kernel timeline: {kind: (start_ns, end_ns)}
    for the kinds that ran since the last read."""
    buf = (C.c_uint64 * (2 * len(TL_KINDS)))()
    _check(lib.hkv_read_timeline(ws.ptr, buf, _stream(stream)), "hkv_read_timeline")
    return {k: (int(buf[2 * i]), int(buf[2 * i + 1])) for i, k in enumerate(TL_KINDS) if buf[2 * i + 1]}


def debug_withhold_publish(on: bool):
    _check(lib.hkv_debug_withhold_publish(1 if on else 0), "hkv_debug_withhold_publish")


def launch_count() -> int:
    return int(lib.hkv_launch_count())


def status_string(code: int) -> str:
    return lib.hkv_status_string(int(code)).decode()
