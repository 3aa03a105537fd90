"""ctypes binding of libqlora (the C ABI in include/qlora.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream; outputs and
workspaces that the caller does not pass are allocated here with torch (the
library itself never allocates).  There is no CPU fallback: if the shared
library is missing or a call fails, a ``QLoRAError`` is raised.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqlora.so")

QLORA_OK = 0
QLORA_ERR_NULL = -1
QLORA_ERR_SHAPE = -2
QLORA_ERR_ALIGN = -3
QLORA_ERR_WORKSPACE = -4
QLORA_ERR_CUDA = -5
QLORA_ERR_DEVICE = -6
QLORA_ERR_CODEBOOK = -7
QLORA_ERR_FORMAT = -8

# 4-bit codebooks (the weight's `codebook`): NF4 and the FP4 / INT4 baselines.
QLORA_CODEBOOK_NF4 = 0
QLORA_CODEBOOK_FP4 = 1
QLORA_CODEBOOK_INT4 = 2
CODEBOOKS = {"nf4": QLORA_CODEBOOK_NF4, "fp4": QLORA_CODEBOOK_FP4, "int4": QLORA_CODEBOOK_INT4}

# Storage formats of the double-quantized absmax (the weight's `dq_format`):
# unsigned linear 8-bit codes, or E4M3 offsets from the tensor mean.
QLORA_DQ_LINEAR8 = 0
QLORA_DQ_FP8_MEAN = 1
DQ_FORMATS = {"linear8": QLORA_DQ_LINEAR8, "fp8_mean": QLORA_DQ_FP8_MEAN}

# Bits of the device error word (qlora_poll_device_error).
QLORA_DEVERR_OPERANDS = 1 << 0
QLORA_DEVERR_WEIGHT_TILE = 1 << 1
QLORA_DEVERR_FREE_STAGE = 1 << 2
QLORA_DEVERR_ACCUMULATOR = 1 << 3
QLORA_DEVERR_DRAIN = 1 << 4
QLORA_DEVERR_SELFTEST = 1 << 5

QLORA_OP_FWD = 0
QLORA_OP_BWD_DX = 1
QLORA_OP_LORA_BWD = 2

BLOCK = 64
GROUP = 256


class QLoRAError(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        self.cuda_error = cuda_error
        msg = lib().qlora_status_string(status).decode()
        if status == QLORA_ERR_CUDA:
            msg += f" (cudaError {cuda_error})"
        super().__init__(f"{fn}: {msg}")


class NF4WeightC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("absmax_q", ctypes.c_void_p),
                ("group_scale", ctypes.c_void_p), ("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("block", ctypes.c_int32), ("group", ctypes.c_int32), ("codebook", ctypes.c_int32),
                ("dq_format", ctypes.c_int32)]


_LIB = None

_SIGNATURES = {
    "qlora_quantize_nf4_dq": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_quantize_4bit_dq": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p]),
    "qlora_quantize_4bit_dq_format": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                     ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                     ctypes.c_void_p]),
    "qlora_codebook_levels": (ctypes.c_int, [ctypes.c_int32, ctypes.POINTER(ctypes.c_float)]),
    "qlora_dequant": (ctypes.c_int, [ctypes.POINTER(NF4WeightC), ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_merge_adapter": (ctypes.c_int, [ctypes.POINTER(NF4WeightC), ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_int32, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.c_void_p]),
    "qlora_linear_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(NF4WeightC),
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear_bwd_dx": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(NF4WeightC),
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_lora_bwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                      ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                ctypes.c_int32]),
    "qlora_last_cuda_error": (ctypes.c_int, []),
    "qlora_poll_device_error": (ctypes.c_int, [ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint)]),
    "qlora_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "qlora_nf4_levels": (None, [ctypes.POINTER(ctypes.c_float)]),
    "qlora_version": (ctypes.c_int, []),
    "qlora_set_profile_events": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_launch_count": (ctypes.c_uint64, []),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(NF4WeightC),
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                                                ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_linear_bwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.POINTER(NF4WeightC), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                        ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_lora_dropout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_float,
                                          ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_linear_fwd_dropout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(NF4WeightC),
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                                                ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                                ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_linear_bwd_dx_dropout": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(NF4WeightC),
                                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float,
                                                   ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "qlora_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_uint64, ctypes.c_void_p, ctypes.c_void_p]),
    "qlora_selftest_div255": (ctypes.c_int, [ctypes.c_uint32, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p]),
}


def lib() -> ctypes.CDLL:
    """Load libqlora.so from the package directory (built in-tree)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m bit_nf4_quantized_qlora_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def _check(fn: str, status: int) -> None:
    if status != QLORA_OK:
        raise QLoRAError(fn, status, lib().qlora_last_cuda_error() if status == QLORA_ERR_CUDA else 0)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _need_cuda(*ts: Optional[torch.Tensor]) -> None:
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


@dataclass
class NF4Weight:
    """A quantized weight: packed codes, absmax codes and group scales (all on
    the device) plus its shape [n x k]."""
    codes: torch.Tensor          # uint8 [n*k/2]
    absmax_q: torch.Tensor       # uint8 [n*k/64]
    group_scale: torch.Tensor    # float32 [ceil(n*k/64/256)] (+ the mean, QLORA_DQ_FP8_MEAN)
    n: int
    k: int
    codebook: int = QLORA_CODEBOOK_NF4
    dq_format: int = QLORA_DQ_LINEAR8

    def c_struct(self) -> NF4WeightC:
        return NF4WeightC(self.codes.data_ptr(), self.absmax_q.data_ptr(), self.group_scale.data_ptr(),
                          self.n, self.k, BLOCK, GROUP, self.codebook, self.dq_format)

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + self.absmax_q.numel() + 4 * self.group_scale.numel()


def n_groups(numel: int) -> int:
    return (numel // BLOCK + GROUP - 1) // GROUP


def qlora_workspace_bytes(op: int, m: int, n: int, k: int, r: int) -> int:
    return int(lib().qlora_workspace_bytes(op, m, n, k, r))


def qlora_nf4_levels() -> list:
    buf = (ctypes.c_float * 16)()
    lib().qlora_nf4_levels(buf)
    return [float(v) for v in buf]


def qlora_codebook_levels(codebook: int) -> list:
    buf = (ctypes.c_float * 16)()
    _check("qlora_codebook_levels", lib().qlora_codebook_levels(codebook, buf))
    return [float(v) for v in buf]


def qlora_set_profile_events(start: Optional[torch.cuda.Event], stop: Optional[torch.cuda.Event]) -> None:
    """Record `start`/`stop` around the main kernel of the following linear
    calls on this thread (None, None clears)."""
    a = None if start is None else start.cuda_event
    b = None if stop is None else stop.cuda_event
    _check("qlora_set_profile_events", lib().qlora_set_profile_events(a, b))


def qlora_launch_count() -> int:
    return int(lib().qlora_launch_count())


def qlora_poll_device_error(stream=None) -> int:
    flags = ctypes.c_uint(0)
    _check("qlora_poll_device_error", lib().qlora_poll_device_error(_stream(stream), ctypes.byref(flags)))
    return int(flags.value)


def qlora_quantize_nf4_dq(W: torch.Tensor, absmax_fp32: Optional[torch.Tensor] = None,
                          out: Optional[NF4Weight] = None, stream=None) -> NF4Weight:
    """fp32 W [n x k] on the device -> NF4Weight."""
    return qlora_quantize_4bit_dq(W, QLORA_CODEBOOK_NF4, absmax_fp32, out, stream)


def qlora_quantize_4bit_dq(W: torch.Tensor, codebook: int, absmax_fp32: Optional[torch.Tensor] = None,
                           out: Optional[NF4Weight] = None, stream=None,
                           dq_format: int = QLORA_DQ_LINEAR8) -> NF4Weight:
    """fp32 W [n x k] on the device -> NF4Weight in `codebook` (QLORA_CODEBOOK_*)
    with its absmax stored in `dq_format` (QLORA_DQ_*)."""
    _need_cuda(W, absmax_fp32)
    if W.dtype != torch.float32 or W.dim() != 2:
        raise ValueError("W must be a 2-D float32 tensor")
    n, k = W.shape
    numel = n * k
    n_scales = max(n_groups(numel), 1) + (1 if dq_format == QLORA_DQ_FP8_MEAN else 0)
    if out is None:
        dev = W.device
        out = NF4Weight(torch.empty(numel // 2, dtype=torch.uint8, device=dev),
                        torch.empty(numel // BLOCK, dtype=torch.uint8, device=dev),
                        torch.empty(n_scales, dtype=torch.float32, device=dev), n, k, codebook, dq_format)
    else:
        if out.group_scale.numel() < n_scales:
            raise ValueError(f"out.group_scale holds {out.group_scale.numel()} entries, {n_scales} needed")
        out.codebook = codebook
        out.dq_format = dq_format
    _check("qlora_quantize_4bit_dq_format",
           lib().qlora_quantize_4bit_dq_format(W.data_ptr(), n, k, codebook, dq_format, out.codes.data_ptr(),
                                               out.absmax_q.data_ptr(), out.group_scale.data_ptr(),
                                               _ptr(absmax_fp32), _stream(stream)))
    return out


def qlora_dequant(w: NF4Weight, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """NF4Weight -> bf16 W^ [n x k]."""
    if out is None:
        out = torch.empty(w.n, w.k, dtype=torch.bfloat16, device=w.codes.device)
    _need_cuda(out)
    ws = w.c_struct()
    _check("qlora_dequant", lib().qlora_dequant(ctypes.byref(ws), out.data_ptr(), _stream(stream)))
    return out


def qlora_merge_adapter(w: NF4Weight, A: Optional[torch.Tensor], B: Optional[torch.Tensor], r: int,
                        scale: float, out_bf16: Optional[torch.Tensor] = None, out_f32: Optional[torch.Tensor] = None,
                        want_bf16: bool = True, want_f32: bool = False, stream=None):
    """W' = W^ + scale . B . A [n x k]; returns (bf16 or None, fp32 or None)."""
    A, B, r = _lora_args(A, B, r)
    dev = w.codes.device
    if out_bf16 is None and want_bf16:
        out_bf16 = torch.empty(w.n, w.k, dtype=torch.bfloat16, device=dev)
    if out_f32 is None and want_f32:
        out_f32 = torch.empty(w.n, w.k, dtype=torch.float32, device=dev)
    _need_cuda(A, B, out_bf16, out_f32)
    ws = w.c_struct()
    _check("qlora_merge_adapter",
           lib().qlora_merge_adapter(ctypes.byref(ws), _ptr(A), _ptr(B), r, float(scale), _ptr(out_bf16),
                                     _ptr(out_f32), _stream(stream)))
    return out_bf16, out_f32


def _lora_args(A, B, r):
    if A is None or B is None or r == 0:
        return None, None, 0
    return A, B, r


def _workspace(op, m, n, k, r, ws, device):
    need = qlora_workspace_bytes(op, m, n, k, r)
    if ws is None and need > 0:
        ws = torch.empty(need, dtype=torch.uint8, device=device)
    return ws, (ws.numel() * ws.element_size() if ws is not None else 0)


def qlora_linear_fwd(X: torch.Tensor, w: NF4Weight, A: Optional[torch.Tensor] = None,
                     B: Optional[torch.Tensor] = None, r: int = 0, scale: float = 0.0,
                     out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """Y = bf16(X . W^T + bf16(s X A^T) . B^T); X bf16 [m x k]."""
    A, B, r = _lora_args(A, B, r)
    _need_cuda(X, A, B, out, ws)
    m = X.shape[0]
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.bfloat16, device=X.device)
    ws, ws_bytes = _workspace(QLORA_OP_FWD, m, w.n, w.k, r, ws, X.device)
    ws_c = w.c_struct()
    _check("qlora_linear_fwd",
           lib().qlora_linear_fwd(X.data_ptr(), m, ctypes.byref(ws_c), _ptr(A), _ptr(B), r, float(scale),
                                  out.data_ptr(), _ptr(ws), ws_bytes, _stream(stream)))
    return out


def qlora_linear_bwd_dx(dY: torch.Tensor, w: NF4Weight, A: Optional[torch.Tensor] = None,
                        B: Optional[torch.Tensor] = None, r: int = 0, scale: float = 0.0,
                        out: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                        stream=None) -> torch.Tensor:
    """dX = bf16(dY . W^ + bf16(s dY B) . A); dY bf16 [m x n]."""
    A, B, r = _lora_args(A, B, r)
    _need_cuda(dY, A, B, out, ws)
    m = dY.shape[0]
    if out is None:
        out = torch.empty(m, w.k, dtype=torch.bfloat16, device=dY.device)
    ws, ws_bytes = _workspace(QLORA_OP_BWD_DX, m, w.n, w.k, r, ws, dY.device)
    ws_c = w.c_struct()
    _check("qlora_linear_bwd_dx",
           lib().qlora_linear_bwd_dx(dY.data_ptr(), m, ctypes.byref(ws_c), _ptr(A), _ptr(B), r, float(scale),
                                     out.data_ptr(), _ptr(ws), ws_bytes, _stream(stream)))
    return out


def qlora_lora_bwd(X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor, r: int, scale: float,
                   dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                   ws: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(dA, dB) = (bf16(U^T X), bf16(dY^T T)) with U = bf16(s dY B), T = bf16(s X A^T)."""
    _need_cuda(X, dY, A, B, dA, dB, ws)
    m, k = X.shape
    n = dY.shape[1]
    if dA is None:
        dA = torch.empty(r, k, dtype=torch.bfloat16, device=X.device)
    if dB is None:
        dB = torch.empty(n, r, dtype=torch.bfloat16, device=X.device)
    ws, ws_bytes = _workspace(QLORA_OP_LORA_BWD, m, n, k, r, ws, X.device)
    _check("qlora_lora_bwd",
           lib().qlora_lora_bwd(X.data_ptr(), dY.data_ptr(), m, n, k, A.data_ptr(), B.data_ptr(), r, float(scale),
                                dA.data_ptr(), dB.data_ptr(), _ptr(ws), ws_bytes, _stream(stream)))
    return dA, dB


def qlora_linear_bwd(dY: torch.Tensor, X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor, r: int,
                     scale: float, T: Optional[torch.Tensor] = None, dX: Optional[torch.Tensor] = None,
                     dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None, want_dx: bool = True,
                     ws: Optional[torch.Tensor] = None, stream=None):
    """(dX or None, dA, dB) of the layer in one call; T = the forward's
    bf16(s X A^T) (the first m*r*2 bytes of its workspace) or None."""
    _need_cuda(dY, X, A, B, T, dX, dA, dB, ws)
    m, k = X.shape
    n = dY.shape[1]
    if dX is None and want_dx:
        dX = torch.empty(m, k, dtype=torch.bfloat16, device=X.device)
    if dA is None:
        dA = torch.empty(r, k, dtype=torch.bfloat16, device=X.device)
    if dB is None:
        dB = torch.empty(n, r, dtype=torch.bfloat16, device=X.device)
    ws, ws_bytes = _workspace(QLORA_OP_LORA_BWD, m, n, k, r, ws, X.device)
    ws_c = w.c_struct()
    _check("qlora_linear_bwd",
           lib().qlora_linear_bwd(dY.data_ptr(), X.data_ptr(), _ptr(T), m, ctypes.byref(ws_c), A.data_ptr(),
                                  B.data_ptr(), r, float(scale), _ptr(dX), dA.data_ptr(), dB.data_ptr(), _ptr(ws),
                                  ws_bytes, _stream(stream)))
    return dX, dA, dB


def qlora_lora_dropout(X: torch.Tensor, p: float, seed: int, offset: int, out: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """Xd = bf16(D . X . fp32(1 / fp32(1 - p))) with the counter-based keep
    mask of (seed, offset); X bf16 [m x k]."""
    _need_cuda(X, out)
    m, k = X.shape
    if out is None:
        out = torch.empty_like(X)
    _check("qlora_lora_dropout", lib().qlora_lora_dropout(X.data_ptr(), m, k, float(p), int(seed), int(offset),
                                                          out.data_ptr(), _stream(stream)))
    return out


def qlora_linear_fwd_dropout(X: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor, r: int, scale: float,
                             p: float, seed: int, offset: int, out: Optional[torch.Tensor] = None,
                             Xd: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None,
                             stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """(Y, Xd): Y = bf16(X . W^T + bf16(s Xd A^T) . B^T) with Xd the dropout of X."""
    _need_cuda(X, A, B, out, Xd, ws)
    m = X.shape[0]
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.bfloat16, device=X.device)
    if Xd is None:
        Xd = torch.empty_like(X)
    ws, ws_bytes = _workspace(QLORA_OP_FWD, m, w.n, w.k, r, ws, X.device)
    ws_c = w.c_struct()
    _check("qlora_linear_fwd_dropout",
           lib().qlora_linear_fwd_dropout(X.data_ptr(), m, ctypes.byref(ws_c), _ptr(A), _ptr(B), r, float(scale),
                                          float(p), int(seed), int(offset), Xd.data_ptr(), out.data_ptr(), _ptr(ws),
                                          ws_bytes, _stream(stream)))
    return out, Xd


def qlora_linear_bwd_dx_dropout(dY: torch.Tensor, w: NF4Weight, A: torch.Tensor, B: torch.Tensor, r: int,
                                scale: float, p: float, seed: int, offset: int, out: Optional[torch.Tensor] = None,
                                ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """dX = bf16(bf16(dY . W^) + D . (U . A) . fp32(1 / fp32(1 - p))), U = bf16(s dY B)."""
    _need_cuda(dY, A, B, out, ws)
    m = dY.shape[0]
    if out is None:
        out = torch.empty(m, w.k, dtype=torch.bfloat16, device=dY.device)
    ws, ws_bytes = _workspace(QLORA_OP_BWD_DX, m, w.n, w.k, r, ws, dY.device)
    ws_c = w.c_struct()
    _check("qlora_linear_bwd_dx_dropout",
           lib().qlora_linear_bwd_dx_dropout(dY.data_ptr(), m, ctypes.byref(ws_c), _ptr(A), _ptr(B), r, float(scale),
                                             float(p), int(seed), int(offset), out.data_ptr(), _ptr(ws), ws_bytes,
                                             _stream(stream)))
    return out


def qlora_linear_fwd_noalloc(X: torch.Tensor, w: NF4Weight, A: Optional[torch.Tensor] = None,
                             B: Optional[torch.Tensor] = None, r: int = 0, scale: float = 0.0,
                             out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Forward without a workspace: the library's built-in device scratch
    (QLORA_NOALLOC_SCRATCH_BYTES) holds T.  For callers that cannot allocate;
    `out` must then be passed in."""
    A, B, r = _lora_args(A, B, r)
    _need_cuda(X, A, B, out)
    m = X.shape[0]
    if out is None:
        out = torch.empty(m, w.n, dtype=torch.bfloat16, device=X.device)
    ws_c = w.c_struct()
    _check("qlora_linear_fwd_noalloc",
           lib().qlora_linear_fwd_noalloc(X.data_ptr(), m, ctypes.byref(ws_c), _ptr(A), _ptr(B), r, float(scale),
                                          out.data_ptr(), _stream(stream)))
    return out


def qlora_selftest_bounded_wait(limit_ns: int, expired: Optional[torch.Tensor] = None, stream=None) -> None:
    """Launch the bounded-wait self-test (a wait on a barrier nothing arrives
    at, given up after limit_ns); `expired` is an int32 [1] device tensor that
    receives 1 when the wait ran out."""
    _need_cuda(expired)
    _check("qlora_selftest_bounded_wait",
           lib().qlora_selftest_bounded_wait(int(limit_ns), _ptr(expired), _stream(stream)))


def qlora_selftest_div255(first_bits: int, count: int, mismatches: torch.Tensor, stream=None) -> None:
    """Add to the int64 [1] device tensor `mismatches` the number of fp32 bit
    patterns in [first_bits, first_bits + count) whose library fp32(s / 255)
    differs from IEEE division."""
    _need_cuda(mismatches)
    _check("qlora_selftest_div255",
           lib().qlora_selftest_div255(int(first_bits), int(count), mismatches.data_ptr(), _stream(stream)))
