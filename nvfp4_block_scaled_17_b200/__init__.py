"""NVFP4 W4A4 linear for B200 (sm_100a): a thin Python binding over the C ABI.

    y = dequant(Q(x.H)) . dequant(Q(W.H))^T + b

Every function here marshals arguments and calls the same-named entry point of
``libnvfp4_b200.so`` (declared in ``include/nvfp4.h``); all arithmetic runs in
that library's CUDA kernels.  PyTorch only provides device memory and the current
stream.  There is no CPU fallback: if the library is missing or the device is not
a B200, the calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4_b200.so")

STATUS = {0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_SHAPE", 3: "NVFP4_ERR_ALIGN",
          4: "NVFP4_ERR_WORKSPACE", 5: "NVFP4_ERR_DEVICE", 6: "NVFP4_ERR_CUDA",
          7: "NVFP4_ERR_TIMEOUT"}
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_WORKSPACE, ERR_DEVICE, ERR_CUDA, ERR_TIMEOUT = range(8)

# name -> (restype, argtypes); the full exported surface of include/nvfp4.h
_vp, _i64, _sz, _int, _u32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint32
SIGNATURES = {
    "nvfp4_status_string": (ctypes.c_char_p, [_int]),
    "nvfp4_abi_version": (_int, []),
    "nvfp4_scale_bytes": (_sz, [_i64, _i64]),
    "nvfp4_packed_bytes": (_sz, [_i64, _i64]),
    "hadamard_rotate": (_int, [_vp, _vp, _i64, _i64, _int, _vp]),
    "nvfp4_quantize_workspace_bytes": (_sz, []),
    "nvfp4_quantize": (_int, [_vp, _i64, _i64, _int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                              _vp]),
    "nvfp4_gemm": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "nvfp4_gemm_prepared": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "nvfp4_prepared_scale_bytes": (_sz, [_i64, _i64]),
    "nvfp4_prepare_weight_scales": (_int, [_vp, _i64, _i64, _vp, _vp]),
    "nvfp4_dequantize": (_int, [_vp, _vp, _vp, _i64, _i64, _vp, _vp]),
    "int8_quantize_rows": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "int8_gemm": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp]),
    "int8_linear_workspace_bytes": (_sz, [_i64, _i64]),
    "int8_linear": (_int, [_vp, _i64, _i64, _vp, _vp, _i64, _vp, _vp, _sz, _vp, _vp]),
    "nvfp4_gemm_quantize_out": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64,
                                       _i64, _vp]),
    "nvfp4_linear_workspace_bytes": (_sz, [_i64, _i64]),
    "nvfp4_linear": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _int, _vp, _sz, _vp,
                            _vp]),
    "nvfp4_linear_prepared": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _int, _vp,
                                     _sz, _vp, _vp]),
    "nvfp4_linear_fixed_scratch": (_int, [_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _int,
                                          _vp, _vp]),
    "nvfp4_last_device_status": (_int, [_vp, ctypes.POINTER(_int)]),
    "nvfp4_debug_cvt_sweep": (_int, [_u32, _i64, _vp, _vp, _vp, _vp]),
    "nvfp4_debug_wait_timeout": (_int, [_i64, _vp]),
    "nvfp4_debug_gemm_f32": (_int, [_vp, _vp, _vp, _vp, _int, _vp, _vp, _vp, _i64, _i64, _i64,
                                    _vp]),
}

_lib = None


class NVFP4Error(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it first "
                               "(python -c 'import __graft_entry__ as g; g.build()')")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, st: int):
    if st != OK:
        raise NVFP4Error(fn, st)


def _bf16_2d(x: torch.Tensor, name: str) -> torch.Tensor:
    if x.dtype != torch.bfloat16 or not x.is_cuda:
        raise TypeError(f"{name} must be a CUDA bf16 tensor")
    if x.dim() != 2 or not x.is_contiguous():
        raise ValueError(f"{name} must be a contiguous 2-D tensor")
    return x


def _scalar(t, device, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        t = torch.tensor(float(t), dtype=torch.float32, device=device)
    if t.dtype != torch.float32 or t.numel() != 1 or not t.is_cuda:
        raise TypeError(f"{name} must be a one-element CUDA float32 tensor")
    return t


# ---------------------------------------------------------------------------
# sizes
# ---------------------------------------------------------------------------

def nvfp4_scale_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_scale_bytes(rows, K))


def nvfp4_packed_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_packed_bytes(rows, K))


def nvfp4_quantize_workspace_bytes() -> int:
    return int(lib().nvfp4_quantize_workspace_bytes())


def nvfp4_linear_workspace_bytes(M: int, K: int) -> int:
    return int(lib().nvfp4_linear_workspace_bytes(M, K))


# ---------------------------------------------------------------------------
# the path
# ---------------------------------------------------------------------------

def hadamard_rotate(x: torch.Tensor, group: int, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """bf16 [rows, K] -> bf16 [rows, K], each group of `group` values times H/sqrt(g)."""
    _bf16_2d(x, "x")
    y = torch.empty_like(x) if out is None else out
    _check("hadamard_rotate", lib().hadamard_rotate(_ptr(x), _ptr(y), x.shape[0], x.shape[1],
                                                    int(group), _stream(stream)))
    return y


def nvfp4_quantize(x: torch.Tensor, rotate_group: int = 0, gsf: torch.Tensor | float | None = None,
                   out: tuple | None = None, workspace: torch.Tensor | None = None,
                   gsf_w: torch.Tensor | None = None, alpha_out: torch.Tensor | None = None,
                   stream=None):
    """bf16 [rows, K] -> (packed uint8 [rows, K/2], scales uint8 [scale_bytes], gsf fp32 [1]).

    gsf=None computes the dynamic global scale 2688/amax over the whole tensor.  With
    gsf_w and alpha_out the kernel also writes alpha = 1/(gsf * gsf_w) for nvfp4_gemm."""
    _bf16_2d(x, "x")
    R, K = x.shape
    gsf_in = _scalar(gsf, x.device, "gsf")
    if out is None:
        packed = torch.empty(R, K // 2, dtype=torch.uint8, device=x.device)
        sf = torch.empty(max(nvfp4_scale_bytes(R, K), 1), dtype=torch.uint8, device=x.device)
        gsf_out = torch.empty(1, dtype=torch.float32, device=x.device)
    else:
        packed, sf, gsf_out = out
    ws = workspace
    if gsf_in is None and ws is None:
        ws = torch.empty(nvfp4_quantize_workspace_bytes(), dtype=torch.uint8, device=x.device)
    _check("nvfp4_quantize", lib().nvfp4_quantize(
        _ptr(x), R, K, int(rotate_group), _ptr(gsf_in), _ptr(gsf_out), _ptr(packed), _ptr(sf),
        _ptr(gsf_w), _ptr(alpha_out), _ptr(ws), 0 if ws is None else ws.numel(), _stream(stream)))
    return packed, sf, gsf_out


def nvfp4_gemm(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
               alpha: torch.Tensor, bias: torch.Tensor | None, M: int, N: int, K: int,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y bf16 [M, N] = bf16(alpha * deq(a) deq(b)^T + bias)."""
    alpha = _scalar(alpha, a.device, "alpha")
    y = torch.empty(M, N, dtype=torch.bfloat16, device=a.device) if out is None else out
    _check("nvfp4_gemm", lib().nvfp4_gemm(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(alpha),
                                          _ptr(bias), _ptr(y), M, N, K, _stream(stream)))
    return y


def nvfp4_debug_gemm_f32(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                         alpha: torch.Tensor, bias: torch.Tensor | None, M: int, N: int, K: int,
                         prepared: bool = False, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """The GEMM with its unrounded output: y fp32 [M, N] = fp32(alpha * acc) + bias (the
    value nvfp4_gemm / nvfp4_gemm_prepared round once to bf16)."""
    alpha = _scalar(alpha, a.device, "alpha")
    y = torch.empty(M, N, dtype=torch.float32, device=a.device) if out is None else out
    _check("nvfp4_debug_gemm_f32", lib().nvfp4_debug_gemm_f32(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), 1 if prepared else 0, _ptr(alpha), _ptr(bias),
        _ptr(y), M, N, K, _stream(stream)))
    return y


def nvfp4_prepared_scale_bytes(N: int, K: int) -> int:
    return lib().nvfp4_prepared_scale_bytes(N, K)


def prepare_weight_scales(sf: torch.Tensor, N: int, K: int, out: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """A weight's 128x4 scales in the order nvfp4_gemm_prepared / nvfp4_linear_prepared
    read (one 4 KiB block per 256-row block and 256-value K stage)."""
    if out is None:
        out = torch.empty(max(nvfp4_prepared_scale_bytes(N, K), 1), dtype=torch.uint8,
                          device=sf.device)
    _check("nvfp4_prepare_weight_scales",
           lib().nvfp4_prepare_weight_scales(_ptr(sf), N, K, _ptr(out), _stream(stream)))
    return out


def nvfp4_gemm_prepared(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                        sfb_prepared: torch.Tensor, alpha: torch.Tensor,
                        bias: torch.Tensor | None, M: int, N: int, K: int,
                        out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """nvfp4_gemm with the weight scales from prepare_weight_scales."""
    alpha = _scalar(alpha, a.device, "alpha")
    y = torch.empty(M, N, dtype=torch.bfloat16, device=a.device) if out is None else out
    _check("nvfp4_gemm_prepared", lib().nvfp4_gemm_prepared(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb_prepared), _ptr(alpha), _ptr(bias), _ptr(y), M, N,
        K, _stream(stream)))
    return y


def nvfp4_linear(x: torch.Tensor, w_packed: torch.Tensor, w_sf: torch.Tensor,
                 gsf_w: torch.Tensor, N: int, bias: torch.Tensor | None = None,
                 gsf_x: torch.Tensor | float | None = None, rotate_group: int = 0,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 stream=None, prepared: bool = False) -> torch.Tensor:
    """The whole W4A4 linear: bf16 x [M, K] with a packed weight [N, K/2] -> bf16 [M, N].
    With prepared=True, w_sf is the output of prepare_weight_scales."""
    _bf16_2d(x, "x")
    M, K = x.shape
    gsf_x = _scalar(gsf_x, x.device, "gsf_x")
    gsf_w = _scalar(gsf_w, x.device, "gsf_w")
    if workspace is None:
        workspace = torch.empty(nvfp4_linear_workspace_bytes(M, K), dtype=torch.uint8,
                                device=x.device)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
    name = "nvfp4_linear_prepared" if prepared else "nvfp4_linear"
    _check(name, getattr(lib(), name)(
        _ptr(x), M, K, _ptr(w_packed), _ptr(w_sf), _ptr(gsf_w), N, _ptr(bias), _ptr(gsf_x),
        int(rotate_group), _ptr(workspace), workspace.numel(), _ptr(y), _stream(stream)))
    return y


def nvfp4_gemm_quantize_out(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                            sfb: torch.Tensor, alpha: torch.Tensor, M: int, N: int, K: int,
                            gsf_out: torch.Tensor, bias: torch.Tensor | None = None,
                            out: tuple | None = None, stream=None):
    """GEMM with the next linear's NVFP4 input as output: (packed uint8 [M, N/2], 128x4
    scales) of bf16(alpha * A B^T + bias) under the static global scale gsf_out."""
    alpha = _scalar(alpha, a.device, "alpha")
    gsf_out = _scalar(gsf_out, a.device, "gsf_out")
    if out is None:
        packed = torch.empty(M, N // 2, dtype=torch.uint8, device=a.device)
        sf = torch.empty(max(nvfp4_scale_bytes(M, N), 1), dtype=torch.uint8, device=a.device)
    else:
        packed, sf = out
    _check("nvfp4_gemm_quantize_out", lib().nvfp4_gemm_quantize_out(
        _ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(alpha), _ptr(bias), _ptr(gsf_out),
        _ptr(packed), _ptr(sf), M, N, K, _stream(stream)))
    return packed, sf


# ---------------------------------------------------------------------------
# int8 per-row W8A8 linear
# ---------------------------------------------------------------------------

def int8_quantize_rows(x: torch.Tensor, out: tuple | None = None, stream=None):
    """bf16 [rows, K] -> (int8 codes [rows, K], fp32 row scales [rows])."""
    _bf16_2d(x, "x")
    R, K = x.shape
    if out is None:
        q = torch.empty(R, K, dtype=torch.int8, device=x.device)
        s = torch.empty(max(R, 1), dtype=torch.float32, device=x.device)
    else:
        q, s = out
    _check("int8_quantize_rows", lib().int8_quantize_rows(_ptr(x), R, K, _ptr(q), _ptr(s),
                                                          _stream(stream)))
    return q, s


def int8_gemm(a: torch.Tensor, sa: torch.Tensor, b: torch.Tensor, sb: torch.Tensor,
              bias: torch.Tensor | None = None, out: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """y bf16 [M, N] = bf16((fp32(a b^T) * sa[m]) * sb[n] + bias)."""
    M, K = a.shape
    N = b.shape[0]
    y = torch.empty(M, N, dtype=torch.bfloat16, device=a.device) if out is None else out
    _check("int8_gemm", lib().int8_gemm(_ptr(a), _ptr(sa), _ptr(b), _ptr(sb), _ptr(bias), _ptr(y),
                                        M, N, K, _stream(stream)))
    return y


def int8_linear(x: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                bias: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The int8 per-row linear: bf16 x [M, K] with stored int8 codes wq [N, K] and scales
    sw [N] -> bf16 [M, N]."""
    _bf16_2d(x, "x")
    M, K = x.shape
    N = wq.shape[0]
    if workspace is None:
        workspace = torch.empty(max(int(lib().int8_linear_workspace_bytes(M, K)), 1),
                                dtype=torch.uint8, device=x.device)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if out is None else out
    _check("int8_linear", lib().int8_linear(_ptr(x), M, K, _ptr(wq), _ptr(sw), N, _ptr(bias),
                                            _ptr(workspace), workspace.numel(), _ptr(y),
                                            _stream(stream)))
    return y


def nvfp4_dequantize(packed: torch.Tensor, sf: torch.Tensor, gsf: torch.Tensor, K: int,
                     out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """NVFP4 -> bf16: packed uint8 [rows, K/2] + 128x4 scales + device gsf -> bf16 [rows, K]."""
    rows = packed.shape[0]
    gsf = _scalar(gsf, packed.device, "gsf")
    y = torch.empty(rows, K, dtype=torch.bfloat16, device=packed.device) if out is None else out
    _check("nvfp4_dequantize", lib().nvfp4_dequantize(_ptr(packed), _ptr(sf), _ptr(gsf), rows, K,
                                                      _ptr(y), _stream(stream)))
    return y


FIXED_SCRATCH_BYTES = 8 << 20


def nvfp4_linear_fixed_scratch(x: torch.Tensor, w_packed: torch.Tensor, w_sf: torch.Tensor,
                               gsf_w: torch.Tensor, N: int, out: torch.Tensor,
                               bias: torch.Tensor | None = None,
                               gsf_x: torch.Tensor | None = None, rotate_group: int = 0,
                               stream=None) -> torch.Tensor:
    """nvfp4_linear for callers that cannot hand over a workspace: the library's
    own fixed device scratch (FIXED_SCRATCH_BYTES per device) holds the packed
    activation.  Nothing is allocated here either, so `out` and the device
    scalars are required as tensors.  Calls on one device that can overlap race
    on the shared scratch; make the first call on a device before any stream
    capture."""
    _bf16_2d(x, "x")
    M, K = x.shape
    for t, name in ((gsf_w, "gsf_w"), (gsf_x, "gsf_x")):
        if t is not None and not isinstance(t, torch.Tensor):
            raise TypeError(f"{name} must be a one-element CUDA float32 tensor")
    gsf_x = _scalar(gsf_x, x.device, "gsf_x")
    gsf_w = _scalar(gsf_w, x.device, "gsf_w")
    _check("nvfp4_linear_fixed_scratch", lib().nvfp4_linear_fixed_scratch(
        _ptr(x), M, K, _ptr(w_packed), _ptr(w_sf), _ptr(gsf_w), N, _ptr(bias), _ptr(gsf_x),
        int(rotate_group), _ptr(out), _stream(stream)))
    return out


def pack_weight(w: torch.Tensor, rotate_group: int = 0, stream=None):
    """Offline weight packing: [rotate] then quantize with the weight's own dynamic
    global scale -> (packed, scales, gsf_w)."""
    if rotate_group:
        w = hadamard_rotate(w, rotate_group, stream=stream)
    return nvfp4_quantize(w, 0, None, stream=stream)


def last_device_status(stream=None) -> int:
    """Synchronises the stream; returns and clears the device's asynchronous status."""
    v = ctypes.c_int(0)
    _check("nvfp4_last_device_status", lib().nvfp4_last_device_status(_stream(stream),
                                                                      ctypes.byref(v)))
    return v.value
