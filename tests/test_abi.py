"""CPU-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import re
import subprocess
from pathlib import Path

import pytest

import lut_clustered_weight_b200 as cq

ROOT = Path(__file__).resolve().parent.parent


def test_header_declarations_are_exported():
    hdr = (ROOT / "include" / "cq.h").read_text()
    declared = set(re.findall(r"CQ_API\s+[\w\s\*]+?\b(cq_\w+)\s*\(", hdr))
    assert declared == set(cq.EXPORTS)
    nm = subprocess.run(["nm", "-D", "--defined-only", str(cq.LIB_PATH)], capture_output=True,
                        text=True, check=True).stdout
    exported = {l.split()[-1] for l in nm.splitlines() if " T " in l}
    assert declared <= exported
    for name in declared:
        assert hasattr(cq.lib, name)


def test_status_strings_and_version():
    assert cq.status_string(cq.CQ_OK) == "CQ_OK"
    assert cq.status_string(cq.CQ_ERR_WORKSPACE) == "CQ_ERR_WORKSPACE"
    assert "sm_100a" in cq.version()


FAKE = 1 << 20  # a 16-byte aligned address that is never dereferenced


def test_rotate_quantize_argument_checks():
    f = cq.lib.cq_rotate_quantize
    ok = dict(x=FAKE, M=2, K=64, b=16, bits=4, q=FAKE, s=FAKE)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["x"], a["M"], a["K"], a["b"], a["bits"], a["q"], a["s"], None)

    assert call(bits=5) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(b=12) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(b=128) == cq.CQ_ERR_INVALID_ARGUMENT          # K % b
    assert call(x=0) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(x=FAKE + 2) == cq.CQ_ERR_INVALID_ARGUMENT     # misaligned
    assert call(M=-1) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(K=12, b=4) == cq.CQ_ERR_UNSUPPORTED           # K % 8
    assert call(K=32768, b=16) == cq.CQ_ERR_UNSUPPORTED       # K > 16384
    assert call(K=16384, b=16384) == cq.CQ_ERR_UNSUPPORTED    # b > 8192
    assert call(M=0) == cq.CQ_OK                              # no-op, nothing launched


def test_lut_gemm_argument_checks():
    f = cq.lib.cq_lut_gemm
    base = dict(q=FAKE, s=FAKE, M=4, K=256, bits=4, w=FAKE, cb=FAKE, N=128, y=FAKE, S=None,
                ws=None, wsb=0)

    def call(**kw):
        a = {**base, **kw}
        return f(a["q"], a["s"], a["M"], a["K"], a["bits"], a["w"], a["cb"], a["N"], a["y"],
                 a["S"], a["ws"], a["wsb"], None)

    assert call(bits=2) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(w=None) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(K=255) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(K=240) == cq.CQ_ERR_UNSUPPORTED      # K % 32
    assert call(N=96) == cq.CQ_ERR_UNSUPPORTED       # N % 64
    assert call(cb=FAKE + 8) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(M=0) == cq.CQ_OK
    need = cq.cq_lut_gemm_workspace_size(4, 128, 9728, 4)
    assert need > 0       # K = 9728 splits over several CTAs per row tile
    assert call(K=9728, ws=None, wsb=0) == cq.CQ_ERR_WORKSPACE
    assert call(K=9728, ws=FAKE, wsb=need - 1) == cq.CQ_ERR_WORKSPACE


def _desc(**kw):
    d = dict(H=256, I=128, E=8, top_k=2, n_shared=0, I_shared=0, act_bits=4, had_block_h=256,
             had_block_i=128, had_block_i_shared=128, renormalize=1)
    d.update(kw)
    return cq.MoEDesc(*[d[n] for n, _ in cq.MoEDesc._fields_])


def _moe_call(d, T=4, logits=FAKE, ws=FAKE, wsb=1 << 30, weights=None):
    w = weights or cq.MoEWeights(*([FAKE] * 12))
    return cq.lib.cq_moe_ffn(ctypes.byref(d), FAKE, logits, T, ctypes.byref(w), ws, wsb, FAKE,
                             None, None)


def test_moe_argument_checks():
    assert _moe_call(_desc(act_bits=3)) == cq.CQ_ERR_INVALID_ARGUMENT
    assert _moe_call(_desc(top_k=9)) == cq.CQ_ERR_INVALID_ARGUMENT          # k > E
    assert _moe_call(_desc(E=0, top_k=0, n_shared=0)) == cq.CQ_ERR_INVALID_ARGUMENT
    assert _moe_call(_desc(had_block_h=96)) == cq.CQ_ERR_INVALID_ARGUMENT
    assert _moe_call(_desc(E=512, top_k=2)) == cq.CQ_ERR_UNSUPPORTED
    assert _moe_call(_desc(I=96, had_block_i=32)) == cq.CQ_ERR_UNSUPPORTED  # I % 64
    assert _moe_call(_desc(), logits=None) == cq.CQ_ERR_INVALID_ARGUMENT    # E > 0 needs logits
    assert _moe_call(_desc(E=0, top_k=0, n_shared=1, I_shared=128), logits=FAKE) \
        == cq.CQ_ERR_INVALID_ARGUMENT
    need = cq.lib.cq_moe_ffn_workspace_size(ctypes.byref(_desc()), 4)
    assert need > 0
    assert _moe_call(_desc(), ws=FAKE, wsb=need - 1) == cq.CQ_ERR_WORKSPACE
    w = cq.MoEWeights(*([FAKE] * 12))
    w.down_cb = None
    assert _moe_call(_desc(), weights=w) == cq.CQ_ERR_INVALID_ARGUMENT
    assert _moe_call(_desc(), T=0) == cq.CQ_OK


def test_workspace_sizes_grow_with_tokens():
    c = cq.MoEConfig(2048, 768, 128, 8, 0, 0, 4, 2048, 256, 256)
    assert cq.cq_moe_ffn_workspace_size(c, 64) < cq.cq_moe_ffn_workspace_size(c, 4096)
    assert cq.cq_moe_ffn_workspace_size(c, 64) == cq.cq_moe_ffn_workspace_size(c, 64)


def test_timing_record_argument_checks():
    f = cq.lib.cq_timing_read_launches
    n = ctypes.c_int64(-1)
    # empty record: nothing recorded, no CUDA call made
    assert f(None, None, 0, ctypes.byref(n)) == cq.CQ_OK and n.value == 0
    assert f(None, None, 0, None) == cq.CQ_ERR_INVALID_ARGUMENT
    assert f(None, None, -1, ctypes.byref(n)) == cq.CQ_ERR_INVALID_ARGUMENT
    assert f(None, None, 4, ctypes.byref(n)) == cq.CQ_ERR_INVALID_ARGUMENT
    assert cq.cq_timing_read_launches() == []


def test_rotate_quantize_ex_argument_checks():
    f = cq.lib.cq_rotate_quantize_ex
    ok = dict(x=FAKE, M=2, K=64, b=16, bits=4, scale=FAKE, perm=FAKE, q=FAKE, s=FAKE)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["x"], a["M"], a["K"], a["b"], a["bits"], a["scale"], a["perm"], a["q"],
                 a["s"], None)

    assert call(bits=5) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(b=12) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(scale=FAKE + 2) == cq.CQ_ERR_INVALID_ARGUMENT   # misaligned scale
    assert call(perm=FAKE + 4) == cq.CQ_ERR_INVALID_ARGUMENT    # misaligned perm
    assert call(q=None) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(K=12, b=4) == cq.CQ_ERR_UNSUPPORTED             # K % 8
    assert call(M=0) == cq.CQ_OK
    assert call(M=0, scale=None, perm=None) == cq.CQ_OK         # both optional


def test_lut_gemm_ex_argument_checks():
    f = cq.lib.cq_lut_gemm_ex
    base = dict(q=FAKE, s=FAKE, M=4, K=256, bits=4, w=FAKE, ib=3, cb=FAKE, N=128, y=FAKE,
                ws=None, wsb=0)

    def call(**kw):
        a = {**base, **kw}
        return f(a["q"], a["s"], a["M"], a["K"], a["bits"], a["w"], a["ib"], a["cb"], a["N"],
                 a["y"], a["ws"], a["wsb"], None)

    for ib in (0, 2, 6, 8):
        assert call(ib=ib) == cq.CQ_ERR_UNSUPPORTED
        assert cq.lib.cq_lut_gemm_ex_workspace_size(4, 128, 256, 4, ib) == 0
    for ib in (3, 5):
        assert call(ib=ib, bits=2) == cq.CQ_ERR_INVALID_ARGUMENT
        assert call(ib=ib, w=None) == cq.CQ_ERR_INVALID_ARGUMENT
        assert call(ib=ib, cb=FAKE + 8) == cq.CQ_ERR_INVALID_ARGUMENT
        assert call(ib=ib, K=240) == cq.CQ_ERR_UNSUPPORTED      # K % 32
        assert call(ib=ib, N=96) == cq.CQ_ERR_UNSUPPORTED       # N % 64
        assert call(ib=ib, M=0) == cq.CQ_OK
        need = cq.lib.cq_lut_gemm_ex_workspace_size(4, 128, 256, 4, ib)
        assert need > 0 and need % 256 == 0                      # split-K partial sums
        assert call(ib=ib) == cq.CQ_ERR_WORKSPACE
        assert call(ib=ib, ws=FAKE, wsb=need - 1) == cq.CQ_ERR_WORKSPACE
    # 4-bit indices are cq_lut_gemm exactly, checks included
    assert cq.lib.cq_lut_gemm_ex_workspace_size(4, 128, 9728, 4, 4) == \
        cq.cq_lut_gemm_workspace_size(4, 128, 9728, 4)
    assert call(ib=4, K=255) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(ib=4, K=240) == cq.CQ_ERR_UNSUPPORTED
    assert call(ib=4, M=0) == cq.CQ_OK


def test_lut_gemm_noalloc_argument_checks():
    f = cq.lib.cq_lut_gemm_noalloc
    base = dict(q=FAKE, s=FAKE, M=4, K=256, bits=4, w=FAKE, cb=FAKE, N=128, y=FAKE)

    def call(**kw):
        a = {**base, **kw}
        return f(a["q"], a["s"], a["M"], a["K"], a["bits"], a["w"], a["cb"], a["N"], a["y"],
                 None)

    assert call(bits=2) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(y=None) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(q=FAKE + 1) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(K=255) == cq.CQ_ERR_INVALID_ARGUMENT
    assert call(K=240) == cq.CQ_ERR_UNSUPPORTED
    assert call(N=96) == cq.CQ_ERR_UNSUPPORTED
    assert call(M=0) == cq.CQ_OK
    # a problem whose scratch exceeds the fixed array is refused before any launch
    M, N, K = 16, 65536, 16384
    need = cq.cq_lut_gemm_workspace_size(M, N, K, 4)
    assert need > cq.NOALLOC_SCRATCH_BYTES
    assert call(M=M, N=N, K=K) == cq.CQ_ERR_UNSUPPORTED
