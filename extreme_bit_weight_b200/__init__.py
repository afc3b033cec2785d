"""Python binding of libccq (CCQ WINT2 W2A16 matmul and MoE FFN on B200, sm_100a).

Argument marshalling only: every step of the computation runs in libccq's CUDA kernels (or, for
the offline encoders, its host C++ code).  PyTorch supplies device memory and streams.  The
functions carry the C ABI's names (include/ccq.h); `CcqError` is raised for any non-OK status.
If libccq.so has not been built, importing this package raises ImportError: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libccq.so")

CCQ_OK = 0
CCQ_ERR_INVALID_ARG = 1
CCQ_ERR_UNSUPPORTED = 2
CCQ_ERR_CUDA = 3
CCQ_ERR_DEVICE_CHECK = 4
CCQ_ERR_TIMEOUT = 5

CCQ_FMT_W2_CCQ_G64 = 1
CCQ_FMT_W4_PER_CHANNEL = 2
CCQ_FMT_W2_CCQ_G64_Q4SCALE = 3
CCQ_FMT_W2_STD_G64 = 4
CCQ_FMT_W275_432 = 5
CCQ_FMT_W25_HYBRID = 6
EMB_GROUP_BYTES = {CCQ_FMT_W275_432: 22, CCQ_FMT_W25_HYBRID: 20}
CCQ_ENC_LITERAL_EQ1 = 1
CCQ_ENC_REFIT_SCALE = 2

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libccq.so not built at {LIB_PATH}; run `python extreme_bit_weight_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)


class CcqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.ccq_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})")


class ccq_weight(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32),
        ("n", ctypes.c_int32),
        ("k", ctypes.c_int32),
        ("group", ctypes.c_int32),
        ("codes", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p),
        ("beta", ctypes.c_void_p),
        ("scale_q4", ctypes.c_void_p),
        ("super_scale", ctypes.c_void_p),
    ]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_lib.ccq_status_string.argtypes = [ctypes.c_int]
_lib.ccq_status_string.restype = ctypes.c_char_p
_lib.ccq_build_info.restype = ctypes.c_char_p
_lib.ccq_encode_host.argtypes = [_P, _I, _I, _I, ctypes.c_uint32, _I, _P, _P, _P, _P, _P]
_lib.ccq_quantize_w4_host.argtypes = [_P, _I, _I, _I, _P, _P]
_lib.ccq_encode_device_workspace_size.argtypes = [_I, _I]
_lib.ccq_encode_device_workspace_size.restype = ctypes.c_size_t
_lib.ccq_encode_device.argtypes = [_P, _I, _I, _I, ctypes.c_uint32, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.ccq_encode_host_q4.argtypes = [_P, _I, _I, _I, ctypes.c_uint32, _I, _P, _P, _P, _P, _P, _P]
_lib.ccq_quantize_std_device.argtypes = [_P, _I, _I, _P, _P, _P]
_lib.ccq_encode_emb_device.argtypes = [_I, _P, _I, _I, _P, _P, _P]
_lib.ccq_dequant_bf16.argtypes = [ctypes.POINTER(ccq_weight), _I, _P, _P]
_lib.ccq_gemm_workspace_size.argtypes = [ctypes.POINTER(ccq_weight), _I]
_lib.ccq_gemm_workspace_size.restype = ctypes.c_size_t
_lib.ccq_w2a16_gemm.argtypes = [ctypes.POINTER(ccq_weight), _P, _I, _P, _P, ctypes.c_size_t, _P]
_lib.ccq_moe_workspace_size.argtypes = [_I, _I, _I, _I, _I]
_lib.ccq_moe_workspace_size.restype = ctypes.c_size_t
_lib.ccq_moe_w2a16_forward.argtypes = [ctypes.POINTER(ccq_weight), ctypes.POINTER(ccq_weight), _I, _P, _I, _P,
                                       _P, _I, _P, _P, ctypes.c_size_t, _P]
_lib.ccq_moe_w2a16_forward_traced.argtypes = [ctypes.POINTER(ccq_weight), ctypes.POINTER(ccq_weight), _I, _P, _I,
                                              _P, _P, _I, _P, _P, ctypes.c_size_t, _P, _P]
_lib.ccq_check_device_error.argtypes = [_P, _P]
_lib.ccq_selftest_bounded_wait.argtypes = [_P, _I, _I, _P]
_lib.ccq_w2a16_gemm_noalloc.argtypes = [ctypes.POINTER(ccq_weight), _P, _I, _P, _P]
_lib.ccq_w2a16_gemm_noalloc_max_scratch.restype = ctypes.c_size_t
CCQ_MOE_TRACE_POINTS = 7


def _check(status: int, where: str):
    if status != CCQ_OK:
        raise CcqError(status, where)


def _np_ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _dptr(t):
    """Device address of a tensor (None and raw integer addresses pass through).  A host tensor is
    refused here: every pointer the library's compute entry points take is device memory, and the
    C ABI cannot tell a host address from a device one without a driver query per call."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise CcqError(CCQ_ERR_INVALID_ARG, "host tensor passed where device memory is required")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def ccq_status_string(status: int) -> str:
    return _lib.ccq_status_string(status).decode()


def ccq_build_info() -> str:
    return _lib.ccq_build_info().decode()


# ------------------------------------------------------------------------------------------------
# host encoders
# ------------------------------------------------------------------------------------------------
def ccq_encode_host(w: np.ndarray, group: int = 64, flags: int = 0, threads: int = 0):
    """CCQ (6,4,3) code-cluster encode of fp32 w [n][k] -> (codes, scales, alpha, beta, sq_err)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 4), np.uint8)
    scales = np.zeros((n, k // group), np.float32)
    alpha = np.zeros(n, np.float32)
    beta = np.zeros(n, np.float32)
    err = ctypes.c_double(0.0)
    _check(_lib.ccq_encode_host(_np_ptr(w), n, k, group, flags, threads, _np_ptr(codes), _np_ptr(scales),
                                _np_ptr(alpha), _np_ptr(beta), ctypes.byref(err)), "ccq_encode_host")
    return codes, scales, alpha, beta, err.value


def ccq_encode_host_q4(w: np.ndarray, group: int = 64, flags: int = 0, threads: int = 0):
    """CCQ encode with 4-bit group scales (CCQ_FMT_W2_CCQ_G64_Q4SCALE) of fp32 w [n][k]
    -> (codes, scale_q4 [n][k/128], super_scale [n], alpha, beta, sq_err)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 4), np.uint8)
    sq = np.zeros((n, k // (2 * group)), np.uint8)
    sup = np.zeros(n, np.float32)
    alpha = np.zeros(n, np.float32)
    beta = np.zeros(n, np.float32)
    err = ctypes.c_double(0.0)
    _check(_lib.ccq_encode_host_q4(_np_ptr(w), n, k, group, flags, threads, _np_ptr(codes), _np_ptr(sq),
                                   _np_ptr(sup), _np_ptr(alpha), _np_ptr(beta), ctypes.byref(err)),
           "ccq_encode_host_q4")
    return codes, sq, sup, alpha, beta, err.value


def ccq_encode_device(w: torch.Tensor, group: int = 64, flags: int = 0, ws: torch.Tensor = None, stream=None):
    """CCQ (6,4,3) code-cluster encode of fp32 w [n][k] on the GPU (the same bytes as
    ccq_encode_host) -> device tensors (codes, scales, alpha, beta)."""
    w = w.contiguous()
    n, k = w.shape
    dev = w.device
    codes = torch.empty((n, k // 4), dtype=torch.uint8, device=dev)
    scales = torch.empty((n, k // group), dtype=torch.float32, device=dev)
    alpha = torch.empty(n, dtype=torch.float32, device=dev)
    beta = torch.empty(n, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(max(int(_lib.ccq_encode_device_workspace_size(n, k)), 256), dev)
    _check(_lib.ccq_encode_device(_dptr(w), n, k, group, flags, _dptr(codes), _dptr(scales), _dptr(alpha),
                                  _dptr(beta), _dptr(ws), ws.numel(), _stream(stream)), "ccq_encode_device")
    return codes, scales, alpha, beta


def ccq_quantize_std_device(w: torch.Tensor, stream=None):
    """WINT2-Standard round-to-nearest of fp32 w [n][k] on the GPU -> device tensors
    (codes [n][k/4], scales [n][k/64])."""
    w = w.contiguous()
    n, k = w.shape
    codes = torch.empty((n, k // 4), dtype=torch.uint8, device=w.device)
    scales = torch.empty((n, k // 64), dtype=torch.float32, device=w.device)
    _check(_lib.ccq_quantize_std_device(_dptr(w), n, k, _dptr(codes), _dptr(scales), _stream(stream)),
           "ccq_quantize_std_device")
    return codes, scales


def ccq_encode_emb_device(fmt: int, w: torch.Tensor, stream=None):
    """Encode fp32 w [n][k] on the GPU into CCQ_FMT_W275_432 or CCQ_FMT_W25_HYBRID -> device tensors
    (codes [n][k/64 * 22 or 20] uint8, super_scale [n])."""
    w = w.contiguous()
    n, k = w.shape
    codes = torch.empty((n, k // 64 * EMB_GROUP_BYTES[fmt]), dtype=torch.uint8, device=w.device)
    sup = torch.empty(n, dtype=torch.float32, device=w.device)
    _check(_lib.ccq_encode_emb_device(fmt, _dptr(w), n, k, _dptr(codes), _dptr(sup), _stream(stream)),
           "ccq_encode_emb_device")
    return codes, sup


def ccq_quantize_w4_host(w: np.ndarray, threads: int = 0):
    """W4 per-channel RTN of fp32 w [n][k] -> (codes [n][k/2], scales [n])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    codes = np.zeros((n, k // 2), np.uint8)
    scales = np.zeros(n, np.float32)
    _check(_lib.ccq_quantize_w4_host(_np_ptr(w), n, k, threads, _np_ptr(codes), _np_ptr(scales)),
           "ccq_quantize_w4_host")
    return codes, scales


# ------------------------------------------------------------------------------------------------
# device weights
# ------------------------------------------------------------------------------------------------
class CcqWeight:
    """Device copy of one (or E stacked) quantized weight(s) [E][n][k] and its ccq_weight view.
    The tensors are fixed at construction: the ccq_weight view is built once and reused."""

    def __init__(self, fmt: int, n: int, k: int, codes, scales, alpha=None, beta=None, experts: int = 1,
                 device="cuda", scale_q4=None, super_scale=None):
        self.fmt, self.n, self.k, self.experts = int(fmt), int(n), int(k), int(experts)

        def dev(a, dtype):
            if a is None:
                return None
            if isinstance(a, torch.Tensor):
                return a.to(device=device, dtype=dtype).contiguous()
            return torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dtype).contiguous()

        self.codes = dev(codes, torch.uint8)
        self.scales = dev(scales, torch.float32)
        self.alpha = dev(alpha, torch.float32)
        self.beta = dev(beta, torch.float32)
        self.scale_q4 = dev(scale_q4, torch.uint8)
        self.super_scale = dev(super_scale, torch.float32)
        self._struct = ccq_weight(self.fmt, self.n, self.k, 0 if self.fmt == CCQ_FMT_W4_PER_CHANNEL else 64,
                                  _dptr(self.codes), _dptr(self.scales), _dptr(self.alpha), _dptr(self.beta),
                                  _dptr(self.scale_q4), _dptr(self.super_scale))
        self._ref = ctypes.byref(self._struct)

    def struct(self) -> ccq_weight:
        return self._struct

    @property
    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size()
                   for t in (self.codes, self.scales, self.alpha, self.beta, self.scale_q4, self.super_scale)
                   if t is not None)


def ccq_dequant_bf16(w: CcqWeight, out: torch.Tensor = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((w.experts, w.n, w.k), dtype=torch.bfloat16, device=w.codes.device)
    s = w.struct()
    _check(_lib.ccq_dequant_bf16(ctypes.byref(s), w.experts, _dptr(out), _stream(stream)), "ccq_dequant_bf16")
    return out


def ccq_gemm_workspace_size(w: CcqWeight, m: int) -> int:
    s = w.struct()
    return int(_lib.ccq_gemm_workspace_size(ctypes.byref(s), int(m)))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A device workspace buffer (256-byte aligned allocation from PyTorch's allocator)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def ccq_w2a16_gemm(w: CcqWeight, x: torch.Tensor, y: torch.Tensor = None, ws: torch.Tensor = None,
                   stream=None) -> torch.Tensor:
    """y = x W^T (x BF16 [m][k] on the device)."""
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, w.n), dtype=torch.bfloat16, device=x.device)
    if ws is None:  # (a caller's workspace is size-checked by the library)
        ws = workspace(ccq_gemm_workspace_size(w, m), x.device)
    _check(_lib.ccq_w2a16_gemm(w._ref, _dptr(x), m, _dptr(y), _dptr(ws), ws.numel(), _stream(stream)),
           "ccq_w2a16_gemm")
    return y


def ccq_w2a16_gemm_noalloc(w: CcqWeight, x: torch.Tensor, y: torch.Tensor, stream=None) -> torch.Tensor:
    """y = x W^T without a caller workspace: for code that cannot allocate device memory, the
    library uses its own fixed per-device scratch array (see ccq_w2a16_gemm_noalloc in ccq.h).
    `y` must be supplied by the caller; nothing here allocates."""
    s = w.struct()
    _check(_lib.ccq_w2a16_gemm_noalloc(ctypes.byref(s), _dptr(x), x.shape[0], _dptr(y), _stream(stream)),
           "ccq_w2a16_gemm_noalloc")
    return y


def ccq_w2a16_gemm_noalloc_max_scratch() -> int:
    return int(_lib.ccq_w2a16_gemm_noalloc_max_scratch())


def ccq_moe_workspace_size(T: int, topk: int, H: int, I: int, num_experts: int) -> int:
    return int(_lib.ccq_moe_workspace_size(T, topk, H, I, num_experts))


def ccq_moe_w2a16_forward(w13: CcqWeight, w2: CcqWeight, x: torch.Tensor, expert_ids: torch.Tensor,
                          routing_w: torch.Tensor, y: torch.Tensor = None, ws: torch.Tensor = None,
                          stream=None) -> torch.Tensor:
    """One MoE FFN layer: y[t] = sum_j r_tj * (SiLU(x Wg^T) * (x Wu^T)) Wd^T over the routed experts."""
    T, H = x.shape
    topk = expert_ids.shape[1]
    E = w13.experts
    I = w13.n // 2
    if y is None:
        y = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = workspace(ccq_moe_workspace_size(T, topk, H, I, E), x.device)
    a, b = w13.struct(), w2.struct()
    _check(_lib.ccq_moe_w2a16_forward(ctypes.byref(a), ctypes.byref(b), E, _dptr(x), T, _dptr(expert_ids),
                                      _dptr(routing_w), topk, _dptr(y), _dptr(ws), ws.numel(), _stream(stream)),
           "ccq_moe_w2a16_forward")
    return y


def ccq_moe_w2a16_forward_traced(w13: CcqWeight, w2: CcqWeight, x: torch.Tensor, expert_ids: torch.Tensor,
                                 routing_w: torch.Tensor, y: torch.Tensor, ws: torch.Tensor, events,
                                 stream=None) -> torch.Tensor:
    """ccq_moe_w2a16_forward recording CCQ_MOE_TRACE_POINTS torch.cuda.Event objects between its steps."""
    T, H = x.shape
    topk = expert_ids.shape[1]
    arr = (ctypes.c_void_p * CCQ_MOE_TRACE_POINTS)(*[ev.cuda_event for ev in events])
    a, b = w13.struct(), w2.struct()
    _check(_lib.ccq_moe_w2a16_forward_traced(ctypes.byref(a), ctypes.byref(b), w13.experts, _dptr(x), T,
                                             _dptr(expert_ids), _dptr(routing_w), topk, _dptr(y), _dptr(ws),
                                             ws.numel(), _stream(stream), arr), "ccq_moe_w2a16_forward_traced")
    return y


def ccq_check_device_error(ws: torch.Tensor, stream=None) -> int:
    """Status of the device-side checks recorded in an MoE workspace (waits for the stream)."""
    return int(_lib.ccq_check_device_error(_dptr(ws), _stream(stream)))


def exported_symbols():
    """Names of the C entry points declared in include/ccq.h."""
    import re

    hdr = os.path.join(_HERE, "..", "include", "ccq.h")
    with open(hdr) as f:
        txt = f.read()
    return sorted(set(re.findall(r"\b(ccq_[a-z0-9_]+)\s*\(", txt)))


def ccq_selftest_bounded_wait(ws: torch.Tensor, kind: int, limit_us: int = 20000, stream=None) -> None:
    """Failure-detection self-test: a kernel whose bounded wait cannot be satisfied (kind 0: an
    mbarrier phase, 1: a global counter) gives up after limit_us and records a timeout in ws's error
    word; read it with ccq_check_device_error."""
    _check(_lib.ccq_selftest_bounded_wait(_dptr(ws), kind, limit_us, _stream(stream)), "ccq_selftest_bounded_wait")
