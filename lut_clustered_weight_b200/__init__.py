"""Python binding of the B200 CodeQuant LUT MoE linear layer (libcq_b200.so).

Argument marshalling only: every step runs in the CUDA library behind the C
ABI declared in include/cq.h.  torch supplies device memory and streams.
There is no CPU fallback: importing this package fails if the library has not
been built (``python lut_clustered_weight_b200/build.py``).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass
from pathlib import Path

import torch

from .packing import outlier_grouping_perm, permute_weight_columns  # noqa: F401

_PKG = Path(__file__).resolve().parent
LIB_PATH = _PKG / "libcq_b200.so"

# symbols declared in include/cq.h
EXPORTS = ("cq_status_string", "cq_version", "cq_rotate_quantize", "cq_lut_gemm_workspace_size",
           "cq_lut_gemm", "cq_moe_ffn_workspace_size", "cq_moe_ffn", "cq_launch_count",
           "cq_timing_enable", "cq_timing_read", "cq_lut_gemm_noalloc", "cq_device_error",
           "cq_timing_read_launches", "cq_selftest_wait_timeout", "cq_rotate_quantize_ex",
           "cq_lut_gemm_ex_workspace_size", "cq_lut_gemm_ex")

CQ_OK, CQ_ERR_INVALID_ARGUMENT, CQ_ERR_UNSUPPORTED, CQ_ERR_WORKSPACE, CQ_ERR_CUDA = range(5)


class CQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


if not LIB_PATH.exists():
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python lut_clustered_weight_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(str(LIB_PATH))

_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t


class MoEDesc(ctypes.Structure):
    _fields_ = [("H", _I64), ("I", _I64), ("E", _I64), ("top_k", _I64), ("n_shared", _I64),
                ("I_shared", _I64), ("act_bits", _I32), ("had_block_h", _I32),
                ("had_block_i", _I32), ("had_block_i_shared", _I32), ("renormalize", _I32)]


class MoEWeights(ctypes.Structure):
    _fields_ = [(n, _P) for n in ("gate_idx", "up_idx", "down_idx", "gate_cb", "up_cb", "down_cb",
                                  "sh_gate_idx", "sh_up_idx", "sh_down_idx", "sh_gate_cb",
                                  "sh_up_cb", "sh_down_cb", "x_scale", "x_perm")]


MOE_DEBUG_FIELDS = ("topk_ids", "topk_w", "counts", "offsets", "perm", "x_codes", "x_scales",
                    "h", "h_codes", "h_scales", "y_rows")


class MoEDebug(ctypes.Structure):
    _fields_ = [(n, _P) for n in MOE_DEBUG_FIELDS]


lib.cq_status_string.argtypes = [ctypes.c_int]
lib.cq_status_string.restype = ctypes.c_char_p
lib.cq_version.argtypes = []
lib.cq_version.restype = ctypes.c_char_p
lib.cq_rotate_quantize.argtypes = [_P, _I64, _I64, _I32, _I32, _P, _P, _P]
lib.cq_rotate_quantize.restype = ctypes.c_int
lib.cq_rotate_quantize_ex.argtypes = [_P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _P]
lib.cq_rotate_quantize_ex.restype = ctypes.c_int
lib.cq_lut_gemm_workspace_size.argtypes = [_I64, _I64, _I64, _I32]
lib.cq_lut_gemm_workspace_size.restype = _SZ
lib.cq_lut_gemm.argtypes = [_P, _P, _I64, _I64, _I32, _P, _P, _I64, _P, _P, _P, _SZ, _P]
lib.cq_lut_gemm.restype = ctypes.c_int
lib.cq_lut_gemm_ex_workspace_size.argtypes = [_I64, _I64, _I64, _I32, _I32]
lib.cq_lut_gemm_ex_workspace_size.restype = _SZ
lib.cq_lut_gemm_ex.argtypes = [_P, _P, _I64, _I64, _I32, _P, _I32, _P, _I64, _P, _P, _SZ, _P]
lib.cq_lut_gemm_ex.restype = ctypes.c_int
lib.cq_moe_ffn_workspace_size.argtypes = [ctypes.POINTER(MoEDesc), _I64]
lib.cq_moe_ffn_workspace_size.restype = _SZ
lib.cq_moe_ffn.argtypes = [ctypes.POINTER(MoEDesc), _P, _P, _I64, ctypes.POINTER(MoEWeights), _P,
                           _SZ, _P, ctypes.POINTER(MoEDebug), _P]
lib.cq_moe_ffn.restype = ctypes.c_int
lib.cq_lut_gemm_noalloc.argtypes = [_P, _P, _I64, _I64, _I32, _P, _P, _I64, _P, _P]
lib.cq_lut_gemm_noalloc.restype = ctypes.c_int
lib.cq_device_error.argtypes = []
lib.cq_device_error.restype = _I32
lib.cq_launch_count.argtypes = []
lib.cq_launch_count.restype = _I64
lib.cq_timing_enable.argtypes = [_I32]
lib.cq_timing_enable.restype = ctypes.c_int
lib.cq_timing_read.argtypes = [ctypes.POINTER(_I64), ctypes.POINTER(ctypes.c_double)]
lib.cq_timing_read.restype = ctypes.c_int
lib.cq_selftest_wait_timeout.argtypes = [_P]
lib.cq_selftest_wait_timeout.restype = ctypes.c_int
lib.cq_timing_read_launches.argtypes = [_P, _P, _I64, ctypes.POINTER(_I64)]
lib.cq_timing_read_launches.restype = ctypes.c_int


def cq_launch_count() -> int:
    """Kernels launched by the library since it was loaded."""
    return int(lib.cq_launch_count())


def cq_device_error() -> int:
    """Device error word (0 = none); synchronizes and clears it."""
    return int(lib.cq_device_error())


def cq_timing_enable(on: bool | int = True, every_kernel: bool = False) -> None:
    """Time LUT GEMM launches (on), or every launch of the library
    (every_kernel as well); on = False stops recording."""
    _check(lib.cq_timing_enable((2 if every_kernel else 1) if on else 0), "cq_timing_enable")


def cq_timing_read() -> tuple[int, float]:
    """(timed LUT GEMM launches, their total device time in ms); clears the record."""
    n = _I64(0)
    ms = ctypes.c_double(0.0)
    _check(lib.cq_timing_read(ctypes.byref(n), ctypes.byref(ms)), "cq_timing_read")
    return int(n.value), float(ms.value)


def cq_selftest_wait_timeout(stream=None) -> None:
    """Launch the kernel whose bounded wait always runs out (about 1 s); it sets
    the device error word read by cq_device_error()."""
    _check(lib.cq_selftest_wait_timeout(_stream(stream)), "cq_selftest_wait_timeout")


KERNEL_KINDS = {0: "k_lut_mma", 1: "k_lut_tc", 2: "k_lut_ts", 3: "k_lut_vb",   # cq_kernel_kind
                4: "rotate_quantize", 5: "codes_to_f16", 6: "route", 7: "combine", 8: "reduce",
                9: "centroid_sums"}
LUT_KERNELS = frozenset(v for v in KERNEL_KINDS.values() if v.startswith("k_lut"))


def cq_timing_read_launches(cap: int = 1 << 16) -> list[tuple[str, float]]:
    """[(kernel, device ms)] of every timed launch, in launch order; clears
    the record."""
    kinds = (ctypes.c_int32 * cap)()
    ms = (ctypes.c_float * cap)()
    n = _I64(0)
    _check(lib.cq_timing_read_launches(kinds, ms, cap, ctypes.byref(n)), "cq_timing_read_launches")
    if n.value > cap:
        raise CQError(CQ_ERR_INVALID_ARGUMENT, f"cq_timing_read_launches: {n.value} > cap {cap}")
    return [(KERNEL_KINDS[int(kinds[i])], float(ms[i])) for i in range(int(n.value))]


def status_string(s: int) -> str:
    return lib.cq_status_string(int(s)).decode()


def version() -> str:
    return lib.cq_version().decode()


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(rc: int, where: str):
    if rc != CQ_OK:
        raise CQError(rc, where)


def code_bytes(K: int, bits: int) -> int:
    return K // 2 if bits == 4 else K


def _empty_codes(M, K, bits, device):
    return torch.empty((M, code_bytes(K, bits)),
                       dtype=torch.uint8 if bits == 4 else torch.int8, device=device)


# ---------------------------------------------------------------------------


def cq_rotate_quantize(x: torch.Tensor, had_block: int, act_bits: int, q_out=None, s_out=None,
                       stream=None, scale=None, perm=None):
    """x fp16 [M, K] (CUDA) -> (codes, scales fp32 [M]); see include/cq.h.
    scale (fp16 [K]) / perm (int32 [K]): the online smoothing scale and
    channel order (cq_rotate_quantize_ex)."""
    M, K = x.shape
    if q_out is None:
        q_out = _empty_codes(M, K, act_bits, x.device)
    if s_out is None:
        s_out = torch.empty((M,), dtype=torch.float32, device=x.device)
    if scale is None and perm is None:
        _check(lib.cq_rotate_quantize(_ptr(x), M, K, had_block, act_bits, _ptr(q_out),
                                      _ptr(s_out), _stream(stream)), "cq_rotate_quantize")
    else:
        _check(lib.cq_rotate_quantize_ex(_ptr(x), M, K, had_block, act_bits, _ptr(scale),
                                         _ptr(perm), _ptr(q_out), _ptr(s_out), _stream(stream)),
               "cq_rotate_quantize_ex")
    return q_out, s_out


def cq_lut_gemm_workspace_size(M: int, N: int, K: int, act_bits: int) -> int:
    return int(lib.cq_lut_gemm_workspace_size(M, N, K, act_bits))


def cq_lut_gemm(q: torch.Tensor, s_x: torch.Tensor, K: int, act_bits: int, w_idx: torch.Tensor,
                codebook: torch.Tensor, y=None, centroid_sums=None, workspace=None, stream=None):
    """y fp32 [M, N] = s_x * sum_k C[n, I[n,k]] q[m,k]; see include/cq.h.

    centroid_sums: None, True (allocate int32 [M, N, 16]) or a tensor.
    Returns y, or (y, centroid_sums) when they were requested."""
    M = s_x.shape[0]
    N = w_idx.shape[0]
    dev = w_idx.device
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
    want_S = centroid_sums is not None and centroid_sums is not False
    if centroid_sums is True:
        centroid_sums = torch.empty((M, N, 16), dtype=torch.int32, device=dev)
    ws_bytes = cq_lut_gemm_workspace_size(M, N, K, act_bits)
    if workspace is None and ws_bytes:
        workspace = torch.empty((ws_bytes,), dtype=torch.uint8, device=dev)
    wb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.cq_lut_gemm(_ptr(q), _ptr(s_x), M, K, act_bits, _ptr(w_idx), _ptr(codebook), N,
                           _ptr(y), _ptr(centroid_sums if want_S else None), _ptr(workspace), wb,
                           _stream(stream)), "cq_lut_gemm")
    return (y, centroid_sums) if want_S else y


def cq_lut_gemm_ex_workspace_size(M: int, N: int, K: int, act_bits: int, idx_bits: int) -> int:
    return int(lib.cq_lut_gemm_ex_workspace_size(M, N, K, act_bits, idx_bits))


def cq_lut_gemm_ex(q: torch.Tensor, s_x: torch.Tensor, K: int, act_bits: int, w_idx: torch.Tensor,
                   idx_bits: int, codebook: torch.Tensor, y=None, workspace=None, stream=None):
    """cq_lut_gemm with 2^idx_bits centroids per row (idx_bits 3, 4, 5); w_idx
    uint8 [N, K*idx_bits/8], codebook fp16 [N, 2^idx_bits]; see include/cq.h."""
    M = s_x.shape[0]
    N = w_idx.shape[0]
    dev = w_idx.device
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=dev)
    nb = int(lib.cq_lut_gemm_ex_workspace_size(M, N, K, act_bits, idx_bits))
    if workspace is None and nb:
        workspace = torch.empty((nb,), dtype=torch.uint8, device=dev)
    wb = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib.cq_lut_gemm_ex(_ptr(q), _ptr(s_x), M, K, act_bits, _ptr(w_idx), idx_bits,
                              _ptr(codebook), N, _ptr(y), _ptr(workspace), wb, _stream(stream)),
           "cq_lut_gemm_ex")
    return y


NOALLOC_SCRATCH_BYTES = 4 << 20


def cq_lut_gemm_noalloc(q: torch.Tensor, s_x: torch.Tensor, K: int, act_bits: int,
                        w_idx: torch.Tensor, codebook: torch.Tensor, y=None, stream=None):
    """cq_lut_gemm without a workspace argument, for callers that cannot
    allocate device memory: the split-K partial sums live in a fixed 4 MiB
    array inside the library (shared by all calls; overlapping calls race).
    Raises CQError(CQ_ERR_UNSUPPORTED) for problems whose partials exceed it."""
    M = s_x.shape[0]
    N = w_idx.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.float32, device=w_idx.device)
    _check(lib.cq_lut_gemm_noalloc(_ptr(q), _ptr(s_x), M, K, act_bits, _ptr(w_idx),
                                   _ptr(codebook), N, _ptr(y), _stream(stream)),
           "cq_lut_gemm_noalloc")
    return y


@dataclass
class MoEConfig:
    H: int
    I: int
    E: int
    top_k: int
    n_shared: int
    I_shared: int
    act_bits: int
    had_block_h: int
    had_block_i: int
    had_block_i_shared: int
    renormalize: int = 1

    def desc(self) -> MoEDesc:
        return MoEDesc(self.H, self.I, self.E, self.top_k, self.n_shared, self.I_shared,
                       self.act_bits, self.had_block_h, self.had_block_i,
                       self.had_block_i_shared, self.renormalize)


def cq_moe_ffn_workspace_size(cfg: MoEConfig, T: int) -> int:
    d = cfg.desc()
    return int(lib.cq_moe_ffn_workspace_size(ctypes.byref(d), T))


def cq_moe_ffn(cfg: MoEConfig, x: torch.Tensor, router_logits, weights: dict, out=None,
               workspace=None, debug: dict | None = None, stream=None):
    """MoE / dense SwiGLU FFN layer; see include/cq.h.  ``weights`` maps the
    cq_moe_weights field names to CUDA tensors; ``debug`` maps cq_moe_debug
    field names to preallocated CUDA tensors."""
    T = x.shape[0]
    d = cfg.desc()
    if out is None:
        out = torch.empty((T, cfg.H), dtype=torch.float32, device=x.device)
    ws_bytes = int(lib.cq_moe_ffn_workspace_size(ctypes.byref(d), T))
    if workspace is None:
        workspace = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=x.device)
    wb = workspace.numel() * workspace.element_size()
    w = MoEWeights(*[_ptr(weights.get(n)) for n, _ in MoEWeights._fields_])
    dbg = None
    if debug:
        dbg = MoEDebug(*[_ptr(debug.get(n)) for n in MOE_DEBUG_FIELDS])
    _check(lib.cq_moe_ffn(ctypes.byref(d), _ptr(x), _ptr(router_logits), T, ctypes.byref(w),
                          _ptr(workspace), wb, _ptr(out),
                          ctypes.byref(dbg) if dbg is not None else None, _stream(stream)),
           "cq_moe_ffn")
    return out


class MoELayer:
    """A prepared cq_moe_ffn call: the descriptor, the weight pointers and the
    workspace are marshalled once, so each call only passes the activation,
    logits and output pointers (serving loops, CUDA-graph capture).  The
    caller keeps the weight tensors alive."""

    def __init__(self, cfg: MoEConfig, T: int, weights: dict, device, workspace=None):
        self.cfg = cfg
        self.T = T
        self._desc = cfg.desc()
        self._w = MoEWeights(*[_ptr(weights.get(n)) for n, _ in MoEWeights._fields_])
        self._weights = weights
        nbytes = int(lib.cq_moe_ffn_workspace_size(ctypes.byref(self._desc), T))
        self.workspace = workspace if workspace is not None else torch.empty(
            (max(nbytes, 1),), dtype=torch.uint8, device=device)
        self._wsb = self.workspace.numel() * self.workspace.element_size()
        self._fn = lib.cq_moe_ffn

    def __call__(self, x: torch.Tensor, router_logits, out: torch.Tensor, debug=None,
                 stream=None):
        dbg = MoEDebug(*[_ptr(debug.get(n)) for n in MOE_DEBUG_FIELDS]) if debug else None
        _check(self._fn(ctypes.byref(self._desc), x.data_ptr(), _ptr(router_logits), self.T,
                        ctypes.byref(self._w), self.workspace.data_ptr(), self._wsb,
                        out.data_ptr(), ctypes.byref(dbg) if dbg is not None else None,
                        _stream(stream)), "cq_moe_ffn")
        return out
