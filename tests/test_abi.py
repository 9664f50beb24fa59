"""The C ABI library loads, exports every entry point of include/hkv.h and
validates arguments on the host (these calls launch nothing, so no GPU is used)."""
import ctypes as C
import os
import re

import pytest
import torch

from head_adaptive_kv_b200 import build as hbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def hk():
    hbuild.build()
    from head_adaptive_kv_b200 import hkv

    return hkv


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "hkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hkv_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(hk):
    names = declared_symbols()
    assert len(names) == 21, names
    for n in names:
        assert hasattr(hk.lib, n), n
    nm = os.popen(f"nm -D --defined-only {hk.LIB_PATH}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", nm), f"{n} not exported"


def _prob(hk, **kw):
    d = dict(B=2, Hq=8, Hkv=2, D=128, dtype=torch.bfloat16, p=0.9, bmin=4, bmax=64)
    d.update(kw)
    return hk.Problem(**d)


def _tier(hk, cap, addr=0x10000):
    t = hk._Tier(addr, addr + 0x100000, 2 * 128 * cap, 128 * cap, 128, cap, 0x2000)
    return t


def _ws_size(hk, prob, dense, sparse, cond):
    n = C.c_size_t(0)
    code = hk.lib.hkv_workspace_size(C.byref(prob.c()), dense and C.byref(dense), C.byref(sparse),
                                     cond and C.byref(cond), C.byref(n))
    return code, n.value


def test_workspace_size_and_validation(hk):
    d, s, c = _tier(hk, 64), _tier(hk, 1000), _tier(hk, 16)
    code, n = _ws_size(hk, _prob(hk), d, s, c)
    assert code == 0 and n > 0 and n % 256 == 0
    # the workspace depends on capacities only and grows with them
    code2, n2 = _ws_size(hk, _prob(hk), d, _tier(hk, 4000), c)
    assert code2 == 0 and n2 > n
    cases = {
        "bmin > bmax": (_prob(hk, bmin=10, bmax=5), 1),
        "Hq % Hkv": (_prob(hk, Hq=7), 1),
        "D 96": (_prob(hk, D=96), 2),
        "G 3": (_prob(hk, Hq=6), 2),
        "p NaN": (_prob(hk, p=float("nan")), 1),
        "negative scale": (_prob(hk, scale=-1.0), 1),
    }
    for what, (prob, want) in cases.items():
        assert _ws_size(hk, prob, d, s, c)[0] == want, what
    assert hk.lib.hkv_workspace_size(None, None, None, None, None) == 1
    bad = _tier(hk, 64, addr=0x10008)  # misaligned base
    assert _ws_size(hk, _prob(hk), bad, s, c)[0] == 1
    odd = hk._Tier(0x10000, 0x20000, 1, 1, 130, 64, 0x2000)  # stride_t not a 16-byte multiple
    assert _ws_size(hk, _prob(hk), odd, s, c)[0] == 1


def test_compute_calls_reject_bad_workspace_without_launching(hk):
    prob = _prob(hk)
    s = _tier(hk, 1000)
    before = hk.launch_count()
    z = 0x40000
    # workspace missing / misaligned / too small -> HKV_ERR_WORKSPACE
    assert hk.lib.hkv_score(C.byref(prob.c()), 0x1000, C.byref(s), z, 1000, None, 0, None) == 6
    assert hk.lib.hkv_score(C.byref(prob.c()), 0x1000, C.byref(s), z, 1000, 0x100010, 1 << 30, None) == 6
    assert hk.lib.hkv_score(C.byref(prob.c()), 0x1000, C.byref(s), z, 1000, 0x100000, 256, None) == 6
    # z row stride below capacity -> invalid
    assert hk.lib.hkv_score(C.byref(prob.c()), 0x1000, C.byref(s), z, 999, 0x100000, 1 << 30, None) == 1
    # misaligned q
    assert hk.lib.hkv_score(C.byref(prob.c()), 0x1008, C.byref(s), z, 1000, 0x100000, 1 << 30, None) == 1
    assert hk.launch_count() == before


def test_status_strings(hk):
    assert hk.status_string(0) == "HKV_OK"
    assert hk.status_string(4) == "HKV_ERR_TIMEOUT"
    assert hk.status_string(99) == "HKV_ERR_UNKNOWN"


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_call_without_gpu_fails_cleanly(hk):
    prob = _prob(hk)
    s = _tier(hk, 1000)
    code = hk.lib.hkv_score(C.byref(prob.c()), 0x1000, C.byref(s), 0x40000, 1000, 0x100000, 1 << 30, None)
    assert code == 3  # HKV_ERR_CUDA, not a crash


def test_append_validates_on_the_host(hk):
    """hkv_append refuses bad arguments before launching anything."""
    prob = _prob(hk)
    d, s = _tier(hk, 64), _tier(hk, 1000, addr=0x40000000)
    ws, kn, vn, head = C.c_void_p(0x500000), C.c_void_p(0x600000), C.c_void_p(0x700000), C.c_void_p(0x800000)

    def call(kn=kn, vn=vn, dense=d, head=head, sparse=s, ws=ws, ws_bytes=256):
        return hk.STATUS[hk.lib.hkv_append(C.byref(prob.c()), kn, vn, dense and C.byref(dense), head,
                                           sparse and C.byref(sparse), None, ws, ws_bytes, None)]

    assert call(head=None) == "HKV_ERR_INVALID_ARG"            # a window needs its head
    assert call(kn=C.c_void_p(0x600008)) == "HKV_ERR_INVALID_ARG"  # new rows 16-byte aligned
    assert call(vn=None) == "HKV_ERR_INVALID_ARG"
    assert call(ws_bytes=128) == "HKV_ERR_WORKSPACE"
    assert call(ws=C.c_void_p(0x500010)) == "HKV_ERR_WORKSPACE"
    assert call(ws=None) == "HKV_ERR_WORKSPACE"
    bad = _tier(hk, 64)
    bad.stride_t = 100                                         # 200-byte rows: not 16-byte multiples
    assert call(dense=bad) == "HKV_ERR_INVALID_ARG"
    assert hk.STATUS[hk.lib.hkv_append(C.byref(_prob(hk, D=96).c()), kn, vn, C.byref(d), head, C.byref(s),
                                       None, ws, 256, None)] == "HKV_ERR_UNSUPPORTED"


def test_condense_validates_on_the_host(hk):
    """hkv_condense refuses bad arguments before launching anything."""
    prob = _prob(hk)
    s, c = _tier(hk, 1000, addr=0x40000000), _tier(hk, 16)
    ws, w, z, m, lz = (C.c_void_p(a) for a in (0x500000, 0x600000, 0x700000, 0x800000, 0x900000))

    def call(sparse=s, cond=c, w=w, z=z, zs=1000, m=m, lz=lz, block=16, trig=1000, pol=0, ws=ws, wsb=256):
        return hk.STATUS[hk.lib.hkv_condense(C.byref(prob.c()), sparse and C.byref(sparse), cond and C.byref(cond),
                                             w, z, zs, m, lz, block, trig, pol, None, ws, wsb, None)]

    assert call(sparse=None) == "HKV_ERR_INVALID_ARG"
    assert call(block=0) == "HKV_ERR_INVALID_ARG"
    assert call(block=1001) == "HKV_ERR_INVALID_ARG"          # more than the sparse capacity
    assert call(block=hk.CONDENSE_MAX_BLOCK + 1) == "HKV_ERR_INVALID_ARG"
    assert call(trig=-1) == "HKV_ERR_INVALID_ARG"
    assert call(pol=2) == "HKV_ERR_INVALID_ARG"
    assert call(w=None) == "HKV_ERR_INVALID_ARG"              # slots need their weights
    assert call(m=None) == "HKV_ERR_INVALID_ARG"              # scores: all three or none
    assert call(zs=999) == "HKV_ERR_INVALID_ARG"
    assert call(wsb=128) == "HKV_ERR_WORKSPACE"
    assert call(ws=None) == "HKV_ERR_WORKSPACE"


def test_step_mti_validates_on_the_host(hk):
    """hkv_step_mti refuses bad thresholds, state or outputs before launching anything."""
    prob = _prob(hk)
    d, s, c = _tier(hk, 64), _tier(hk, 1000, addr=0x40000000), _tier(hk, 16)
    code, n = _ws_size(hk, prob, d, s, c)
    assert code == 0
    ws = C.c_void_p(0x7000000)

    def mti(**kw):
        f = dict(L_lower=10, L_upper=20, mti_cap=1000, mode=0x500000, left=0x510000,
                 rewrite=_tier(hk, 64, addr=0x60000000), rw_idx=0x520000)
        f.update(kw)
        return hk._Mti(**f)

    def call(m, **out):
        o = dict(sel_len=0x800000, idx=0x810000, out=0x820000)
        o.update(out)
        so = hk._StepOut(**o)
        return hk.STATUS[hk.lib.hkv_step_mti(C.byref(prob.c()), C.c_void_p(0x100000), C.byref(d), C.byref(s),
                                             C.byref(c), m and C.byref(m), C.byref(so), ws, n, None)]

    assert call(None) == "HKV_ERR_INVALID_ARG"
    assert call(mti(L_lower=30)) == "HKV_ERR_INVALID_ARG"          # L_lower above L_upper
    assert call(mti(L_lower=-1)) == "HKV_ERR_INVALID_ARG"
    assert call(mti(mti_cap=-5)) == "HKV_ERR_INVALID_ARG"
    assert call(mti(left=None)) == "HKV_ERR_INVALID_ARG"
    assert call(mti(rw_idx=0x520002)) == "HKV_ERR_INVALID_ARG"     # misaligned
    assert call(mti(rewrite=_tier(hk, 63, addr=0x60000000))) == "HKV_ERR_INVALID_ARG"  # buffer below bmax
    assert call(mti(), k_out=0x900000, v_out=0x910000) == "HKV_ERR_INVALID_ARG"     # no Rewrite Cache outputs
    assert call(mti(), beta_fit=0x920000) == "HKV_ERR_INVALID_ARG"                 # no fitted temperature
    big = _prob(hk, B=600, Hkv=2)
    code, nb = _ws_size(hk, big, d, s, c)
    so = hk._StepOut(sel_len=0x800000, idx=0x810000, out=0x820000)
    assert hk.STATUS[hk.lib.hkv_step_mti(C.byref(big.c()), C.c_void_p(0x100000), C.byref(d), C.byref(s), C.byref(c),
                                         C.byref(mti()), C.byref(so), ws, nb, None)] == "HKV_ERR_UNSUPPORTED"


def test_fit_entry_points_validate_on_the_host(hk):
    """hkv_attention_entropy, hkv_fit_temperature and the step's fitted-temperature
    outputs refuse bad arguments before launching anything."""
    prob = _prob(hk)
    s = _tier(hk, 1000, addr=0x40000000)
    code, n = _ws_size(hk, prob, None, s, None)
    assert code == 0
    ws, q, z, h, b = (C.c_void_p(a) for a in (0x1000000, 0x600000, 0x700000, 0x800000, 0x900000))

    def ent(q=q, h=h):
        return hk.STATUS[hk.lib.hkv_attention_entropy(C.byref(prob.c()), q, C.byref(s), h, ws, n, None)]

    def fit(z=z, zs=1000, h=h, b=b, nbytes=n):
        return hk.STATUS[hk.lib.hkv_fit_temperature(C.byref(prob.c()), z, zs, C.byref(s), h, b, ws, nbytes, None)]

    assert ent(h=None) == "HKV_ERR_INVALID_ARG"
    assert ent(q=C.c_void_p(0x600004)) == "HKV_ERR_INVALID_ARG"
    assert fit(h=None) == "HKV_ERR_INVALID_ARG"
    assert fit(b=None) == "HKV_ERR_INVALID_ARG"
    assert fit(zs=999) == "HKV_ERR_INVALID_ARG"        # z rows shorter than the tier's capacity
    assert fit(z=None) == "HKV_ERR_INVALID_ARG"
    assert fit(nbytes=n - 256) == "HKV_ERR_WORKSPACE"
    # the step: h_attn without beta_fit is refused
    o = hk._StepOut(sel_len=0x110000, idx=0x120000, out=0x130000, h_attn=0x140000)
    st = hk.lib.hkv_step(C.byref(prob.c()), q, None, C.byref(s), None, C.byref(o), ws, n, None)
    assert hk.STATUS[st] == "HKV_ERR_INVALID_ARG"


def test_struct_layouts_match_the_header(hk, tmp_path):
    """The ctypes mirrors of the header's structs have the C compiler's field
    names, order, offsets and sizes (gcc compiles a probe of the header)."""
    import subprocess

    mirrors = {"hkv_tier": hk._Tier, "hkv_problem": hk._Problem, "hkv_cut": hk.Cut, "hkv_step_out": hk._StepOut}
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "hkv.h")).read(), flags=re.S)
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "hkv.h"', "int main(void) {"]
    for cname, mirror in mirrors.items():
        body = re.search(r"typedef struct \{([^{}]*)\}\s*" + cname + ";", text).group(1)
        names = []
        for decl in body.split(";"):
            decl = decl.strip()
            if decl:
                names += [n.strip().lstrip("*") for n in re.sub(r"^[\w\s]+?(?=\*?\w+\s*(,|$))", "", decl).split(",")]
        assert names == [f[0] for f in mirror._fields_], (cname, names)
        lines.append(f'printf("{cname} size %zu\\n", sizeof({cname}));')
        for n in names:
            lines.append(f'printf("{cname} {n} %zu\\n", offsetof({cname}, {n}));')
    lines += ["return 0; }"]
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines))
    exe = tmp_path / "probe"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split("\n")
    for line in filter(None, out):
        cname, field, value = line.split()
        mirror = mirrors[cname]
        got = C.sizeof(mirror) if field == "size" else getattr(mirror, field).offset
        assert got == int(value), (cname, field, got, value)


def test_binding_checks_fit_arguments_before_the_library(hk):
    """The Python binding refuses ill-shaped fitted-temperature arguments
    itself (CPU tensors suffice: nothing reaches the library)."""
    prob = _prob(hk)
    k = torch.zeros(2, 2, 16, 128, dtype=torch.bfloat16)
    sparse = hk.Tier(k, k, torch.zeros(4, dtype=torch.int32))
    ws = object()
    good = torch.zeros(4, dtype=torch.float32)
    with pytest.raises(ValueError):
        hk.fit_temperature(prob, torch.zeros(4, 16, dtype=torch.float64), sparse, good, good, ws)
    with pytest.raises(ValueError):
        hk.fit_temperature(prob, torch.zeros(16, 4).t(), sparse, good, good, ws)   # rows not contiguous
    with pytest.raises(ValueError):
        hk.fit_temperature(prob, torch.zeros(4, 8), sparse, good, good, ws)        # rows shorter than cap
    with pytest.raises(ValueError):
        hk.fit_temperature(prob, torch.zeros(4, 16), sparse, good[:3], good, ws)   # too few targets
    with pytest.raises(ValueError):
        hk.attention_entropy(prob, torch.zeros(2, 8, 128), sparse, torch.zeros(4, dtype=torch.int32), ws)
