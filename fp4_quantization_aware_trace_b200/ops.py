"""Thin ctypes binding of libtrace_fp4.so (C ABI in include/trace_fp4.h).

Argument marshalling only: every step of the path runs in the library's
CUDA kernels.  Tensors must be CUDA tensors; bf16 data is passed by pointer
as raw 16-bit words.  Calls are asynchronous on the given stream (default:
torch's current stream).  If the library is missing or fails to load, the
first call raises -- there is no fallback of any kind.

Method: rcap.io post "TRACE: Rollout-Guided Quantization-Aware Training for
FP4" -- rollout capture of the compact cache (1 mantissa bit + scales), the
guided QAT fake-quant forward and its straight-through backward.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtrace_fp4.so")
_lock = threading.Lock()
_lib = None

TRACE_OK = 0
TRACE_ERR_TIMEOUT = 6


class TraceError(RuntimeError):
    pass


def library() -> ctypes.CDLL:
    """Load libtrace_fp4.so (raises if it is missing: build it with
    ``python -c 'import __graft_entry__ as g; g.build()'``)."""
    global _lib
    lib = _lib
    if lib is not None:  # loaded: no lock on the per-call path
        return lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise TraceError(f"{LIB_PATH} is missing: the CUDA library has not been built")
        lib = ctypes.CDLL(LIB_PATH)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        lib.trace_strerror.argtypes = [ctypes.c_int]
        lib.trace_strerror.restype = ctypes.c_char_p
        lib.trace_abi_version.argtypes = []
        lib.trace_abi_version.restype = ctypes.c_int
        lib.trace_capture_workspace_bytes.argtypes = [i64, i64, i32]
        lib.trace_capture_workspace_bytes.restype = sz
        lib.trace_capture.argtypes = [P, i64, i64, i32, P, P, P, P, P, P, sz, P]
        lib.trace_capture.restype = ctypes.c_int
        lib.trace_guided_fq_fwd.argtypes = [P, i64, i64, i32, P, P, P, P, P, P, P]
        lib.trace_guided_fq_fwd.restype = ctypes.c_int
        lib.trace_fq_bwd.argtypes = [P, P, i64, P, P]
        lib.trace_fq_bwd.restype = ctypes.c_int
        lib.trace_rtn_fq_fwd.argtypes = [P, i64, i64, i32, P, P, P, P, P, P]
        lib.trace_rtn_fq_fwd.restype = ctypes.c_int
        lib.trace_copy_bf16.argtypes = [P, P, i64, P]
        lib.trace_copy_bf16.restype = ctypes.c_int
        lib.trace_copy_bf16_staged.argtypes = [P, P, i64, P, P]
        lib.trace_copy_bf16_staged.restype = ctypes.c_int
        lib.trace_full_guided_fq_fwd.argtypes = [P, i64, i64, i32, P, P, P, P, P, P, P]
        lib.trace_full_guided_fq_fwd.restype = ctypes.c_int
        lib.trace_capture_static_ws.argtypes = [P, i64, i64, i32, P, P, P, P, P, P]
        lib.trace_capture_static_ws.restype = ctypes.c_int
        lib.trace_mismatch_histogram.argtypes = [P, i64, i64, i32, P, P, P, P, P, P]
        lib.trace_mismatch_histogram.restype = ctypes.c_int
        lib.trace_mx_mismatch_histogram.argtypes = [P, i64, i64, P, P, P, P]
        lib.trace_mx_mismatch_histogram.restype = ctypes.c_int
        lib.trace_cache_record_bytes.argtypes = [i64, i64, i32, P, P, P]
        lib.trace_cache_record_bytes.restype = sz
        lib.trace_mx_capture.argtypes = [P, i64, i64, P, P, P, P]
        lib.trace_mx_capture.restype = ctypes.c_int
        lib.trace_mx_guided_fq_fwd.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.trace_mx_guided_fq_fwd.restype = ctypes.c_int
        lib.trace_mx_full_guided_fq_fwd.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.trace_mx_full_guided_fq_fwd.restype = ctypes.c_int
        lib.trace_mx_rtn_fq_fwd.argtypes = [P, i64, i64, P, P, P, P]
        lib.trace_mx_rtn_fq_fwd.restype = ctypes.c_int
        lib.trace_scale_bytes.argtypes = [i64, i64, i32, i32]
        lib.trace_scale_bytes.restype = sz
        lib.trace_capture_ex.argtypes = [P, i64, i64, i32, P, P, P, P, P, P, sz, i32, P]
        lib.trace_capture_ex.restype = ctypes.c_int
        lib.trace_fq_fwd_ex.argtypes = [i32, P, i64, i64, i32, P, P, P, P, P, P, P, i32, P]
        lib.trace_fq_fwd_ex.restype = ctypes.c_int
        lib.trace_mx_capture_ex.argtypes = [P, i64, i64, P, P, P, i32, P]
        lib.trace_mx_capture_ex.restype = ctypes.c_int
        lib.trace_mx_fq_fwd_ex.argtypes = [i32, P, i64, i64, P, P, P, P, P, i32, P]
        lib.trace_mx_fq_fwd_ex.restype = ctypes.c_int
        lib.trace_capture_amax.argtypes = [P, i64, i64, i32, P, P, P]
        lib.trace_capture_amax.restype = ctypes.c_int
        lib.trace_mx8_capture.argtypes = [P, i64, i64, P, P, P, P]
        lib.trace_mx8_capture.restype = ctypes.c_int
        lib.trace_mx8_guided_fq_fwd.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.trace_mx8_guided_fq_fwd.restype = ctypes.c_int
        lib.trace_mx8_full_guided_fq_fwd.argtypes = [P, i64, i64, P, P, P, P, P]
        lib.trace_mx8_full_guided_fq_fwd.restype = ctypes.c_int
        lib.trace_mx8_rtn_fq_fwd.argtypes = [P, i64, i64, P, P, P, P]
        lib.trace_mx8_rtn_fq_fwd.restype = ctypes.c_int
        lib.trace_validate_offsets.argtypes = [P, i32, i64, P, P]
        lib.trace_validate_offsets.restype = ctypes.c_int
        lib.trace_selftest_e4m3_sweep.argtypes = [ctypes.c_uint32, ctypes.c_uint32, P, P]
        lib.trace_selftest_e4m3_sweep.restype = ctypes.c_int
        lib.trace_mx8_capture_ex.argtypes = [P, i64, i64, P, P, P, i32, P]
        lib.trace_mx8_capture_ex.restype = ctypes.c_int
        lib.trace_mx8_fq_fwd_ex.argtypes = [i32, P, i64, i64, P, P, P, P, P, i32, P]
        lib.trace_mx8_fq_fwd_ex.restype = ctypes.c_int
        lib.trace_capture_amax_accumulate.argtypes = [P, i64, i64, i32, P, P, P]
        lib.trace_capture_amax_accumulate.restype = ctypes.c_int
        lib.trace_capture_with_amax.argtypes = [P, i64, i64, i32, P, P, P, P, P, P, i32, P]
        lib.trace_capture_with_amax.restype = ctypes.c_int
        lib.trace_capture_status.argtypes = [P, P]
        lib.trace_capture_status.restype = ctypes.c_int
        _lib = lib
        return lib


def _check(status: int, what: str) -> None:
    if status != TRACE_OK:
        msg = library().trace_strerror(status).decode()
        raise TraceError(f"{what}: status {status} ({msg})")


def _p(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise TraceError("tensors passed to libtrace_fp4 must be CUDA tensors")
    if not t.is_contiguous():
        raise TraceError("tensors passed to libtrace_fp4 must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


DEBUG = os.environ.get("TRACE_DEBUG", "0") not in ("", "0")


def validate_offsets(offsets: torch.Tensor, rows: int, stream=None) -> int:
    """0 when the device offsets are valid for `rows` rows, else 1 + the
    first offending index (synchronises the stream)."""
    flag = torch.empty(1, dtype=torch.int32, device=offsets.device)
    _check(library().trace_validate_offsets(_p(offsets), int(offsets.numel()) - 1, rows, _p(flag),
                                            _stream(stream)), "trace_validate_offsets")
    return int(flag.item())


def _groups(offsets: torch.Tensor | None, rows: int | None = None) -> int:
    if offsets is None:
        return 1
    if offsets.dtype != torch.int64:
        raise TraceError("group offsets must be int64")
    if DEBUG and rows is not None:   # TRACE_DEBUG=1: check the device offsets first
        bad = validate_offsets(offsets, rows)
        if bad:
            raise TraceError(f"group offsets invalid at entry {bad - 1}")
    return int(offsets.numel()) - 1


# ---------------------------------------------------------------------------
# Raw C-ABI calls, same names and argument order as include/trace_fp4.h
# ---------------------------------------------------------------------------

def trace_capture_workspace_bytes(rows: int, cols: int, num_groups: int) -> int:
    return int(library().trace_capture_workspace_bytes(rows, cols, num_groups))


def trace_cache_record_bytes(rows: int, cols: int, num_groups: int) -> tuple[int, int, int, int]:
    """(record bytes, mbits offset, scales offset, gscale offset); record
    bytes is 0 for an invalid shape."""
    om, os_, og = ctypes.c_size_t(0), ctypes.c_size_t(0), ctypes.c_size_t(0)
    nb = library().trace_cache_record_bytes(rows, cols, num_groups, ctypes.byref(om),
                                            ctypes.byref(os_), ctypes.byref(og))
    return int(nb), om.value, os_.value, og.value


def trace_capture(x, rows, cols, num_groups, offsets, codes, mbits, scales, gscale,
                  workspace, workspace_bytes, stream=None) -> None:
    _check(library().trace_capture(_p(x), rows, cols, num_groups, _p(offsets), _p(codes),
                                   _p(mbits), _p(scales), _p(gscale), _p(workspace),
                                   workspace_bytes, _stream(stream)), "trace_capture")


def trace_guided_fq_fwd(x_train, rows, cols, num_groups, offsets, mbits, scales, gscale,
                        out, ste_mask, stream=None) -> None:
    _check(library().trace_guided_fq_fwd(_p(x_train), rows, cols, num_groups, _p(offsets),
                                         _p(mbits), _p(scales), _p(gscale), _p(out),
                                         _p(ste_mask), _stream(stream)), "trace_guided_fq_fwd")


def trace_full_guided_fq_fwd(x_train, rows, cols, num_groups, offsets, codes, scales, gscale,
                             out, ste_mask, stream=None) -> None:
    _check(library().trace_full_guided_fq_fwd(_p(x_train), rows, cols, num_groups, _p(offsets),
                                              _p(codes), _p(scales), _p(gscale), _p(out),
                                              _p(ste_mask), _stream(stream)),
           "trace_full_guided_fq_fwd")


def trace_fq_bwd(grad_out, ste_mask, numel, grad_in, stream=None) -> None:
    _check(library().trace_fq_bwd(_p(grad_out), _p(ste_mask), numel, _p(grad_in),
                                  _stream(stream)), "trace_fq_bwd")


def trace_rtn_fq_fwd(x, rows, cols, num_groups, offsets, scales, gscale, out, ste_mask,
                     stream=None) -> None:
    _check(library().trace_rtn_fq_fwd(_p(x), rows, cols, num_groups, _p(offsets), _p(scales),
                                      _p(gscale), _p(out), _p(ste_mask), _stream(stream)),
           "trace_rtn_fq_fwd")


def trace_capture_static_ws(x, rows, cols, num_groups, offsets, codes, mbits, scales, gscale,
                            stream=None) -> None:
    """trace_capture for callers that cannot supply a workspace: the library
    keeps the scratch in a fixed per-GPU array (at most
    TRACE_STATIC_MAX_GROUPS groups; calls must not overlap on the GPU)."""
    _check(library().trace_capture_static_ws(_p(x), rows, cols, num_groups, _p(offsets),
                                             _p(codes), _p(mbits), _p(scales), _p(gscale),
                                             _stream(stream)), "trace_capture_static_ws")


TRACE_STATIC_MAX_GROUPS = 4096


def trace_mismatch_histogram(x_train, rows, cols, num_groups, offsets, codes, scales, gscale,
                             hist, stream=None) -> None:
    _check(library().trace_mismatch_histogram(_p(x_train), rows, cols, num_groups, _p(offsets),
                                              _p(codes), _p(scales), _p(gscale), _p(hist),
                                              _stream(stream)), "trace_mismatch_histogram")


def trace_selftest_e4m3_sweep(first_bits: int, count: int, out, stream=None) -> None:
    _check(library().trace_selftest_e4m3_sweep(first_bits, count, _p(out), _stream(stream)),
           "trace_selftest_e4m3_sweep")


def trace_copy_bf16(src, dst, numel, stream=None) -> None:
    _check(library().trace_copy_bf16(_p(src), _p(dst), numel, _stream(stream)), "trace_copy_bf16")


def trace_copy_bf16_staged(src, dst, numel, err, stream=None) -> None:
    _check(library().trace_copy_bf16_staged(_p(src), _p(dst), numel, _p(err), _stream(stream)),
           "trace_copy_bf16_staged")


# ---------------------------------------------------------------------------
# Convenience wrappers that allocate their outputs (still no arithmetic here)
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class Capture:
    """What one capture site records: the rollout's full FP4 codes (for its
    own FP4 GEMM) and the compact cache (mbits + scales + gscale)."""
    codes: torch.Tensor    # uint8 [N/2]
    mbits: torch.Tensor    # int32 words [N/32] (bit patterns; uint32 ABI)
    scales: torch.Tensor   # uint8 [rows, cols/16] E4M3
    gscale: torch.Tensor   # float32 [G]
    offsets: torch.Tensor | None = None

    def cache_nbytes(self) -> int:
        """Bytes of the compact cache (mantissa bits + block and global scales)."""
        return self.mbits.numel() * 4 + self.scales.numel() + self.gscale.numel() * 4


def _bf16_2d(x: torch.Tensor) -> tuple[int, int]:
    if x.dtype != torch.bfloat16:
        raise TraceError("activations must be bf16")
    if x.dim() != 2:
        raise TraceError("activations must be 2-D [rows, cols]")
    return int(x.shape[0]), int(x.shape[1])


def alloc_capture(rows: int, cols: int, num_groups: int = 1, device="cuda",
                  offsets: torch.Tensor | None = None) -> tuple[Capture, torch.Tensor]:
    """Allocate capture outputs and the workspace (torch device memory)."""
    n = rows * cols
    cap = Capture(codes=torch.empty(n // 2, dtype=torch.uint8, device=device),
                  mbits=torch.empty(n // 32, dtype=torch.int32, device=device),
                  scales=torch.empty(rows, cols // 16, dtype=torch.uint8, device=device),
                  gscale=torch.empty(num_groups, dtype=torch.float32, device=device),
                  offsets=offsets)
    # zeros before its first use; every capture leaves it zeroed again
    ws = torch.zeros(max(trace_capture_workspace_bytes(rows, cols, num_groups), 256),
                     dtype=torch.uint8, device=device)
    return cap, ws


def capture(x: torch.Tensor, offsets: torch.Tensor | None = None, out: Capture | None = None,
            workspace: torch.Tensor | None = None, stream=None) -> Capture:
    """Rollout capture of one site (x bf16 [rows, cols]; offsets int64 [G+1])."""
    rows, cols = _bf16_2d(x)
    G = _groups(offsets, rows)
    if out is None or workspace is None:
        out, workspace = alloc_capture(rows, cols, G, x.device, offsets)
    trace_capture(x, rows, cols, G, offsets, out.codes, out.mbits, out.scales, out.gscale,
                  workspace, workspace.numel(), stream)
    return out


def capture_status(workspace: torch.Tensor, stream=None) -> bool:
    """True when no capture that used `workspace` has given up waiting at
    its grid barrier since the last check (trace_capture_status: waits for
    the stream, reads and clears the workspace's error word)."""
    st = library().trace_capture_status(_p(workspace), _stream(stream))
    if st == TRACE_ERR_TIMEOUT:
        return False
    _check(st, "trace_capture_status")
    return True

def guided_fq_fwd(x_train: torch.Tensor, cache: Capture, out: torch.Tensor | None = None,
                  mask: torch.Tensor | None = None, stream=None):
    """Guided fake-quant forward with a rollout cache.  Returns (out, mask)."""
    rows, cols = _bf16_2d(x_train)
    out = torch.empty_like(x_train) if out is None else out
    mask = torch.empty(rows * cols // 32, dtype=torch.int32, device=x_train.device) if mask is None else mask
    trace_guided_fq_fwd(x_train, rows, cols, _groups(cache.offsets), cache.offsets, cache.mbits,
                        cache.scales, cache.gscale, out, mask, stream)
    return out, mask


def full_guided_fq_fwd(x_train: torch.Tensor, cache: Capture, out: torch.Tensor | None = None,
                       mask: torch.Tensor | None = None, stream=None):
    """Full-information guided forward (the cache keeps the rollout's whole
    codes).  Returns (out, mask)."""
    rows, cols = _bf16_2d(x_train)
    out = torch.empty_like(x_train) if out is None else out
    mask = torch.empty(rows * cols // 32, dtype=torch.int32, device=x_train.device) if mask is None else mask
    trace_full_guided_fq_fwd(x_train, rows, cols, _groups(cache.offsets), cache.offsets, cache.codes,
                             cache.scales, cache.gscale, out, mask, stream)
    return out, mask


def rtn_fq_fwd(x: torch.Tensor, scales: torch.Tensor, gscale: torch.Tensor,
               offsets: torch.Tensor | None = None, out: torch.Tensor | None = None,
               mask: torch.Tensor | None = None, stream=None):
    """Round-to-nearest fake-quant with given scales.  Returns (out, mask)."""
    rows, cols = _bf16_2d(x)
    out = torch.empty_like(x) if out is None else out
    mask = torch.empty(rows * cols // 32, dtype=torch.int32, device=x.device) if mask is None else mask
    trace_rtn_fq_fwd(x, rows, cols, _groups(offsets), offsets, scales, gscale, out, mask, stream)
    return out, mask


def fq_bwd(grad_out: torch.Tensor, mask: torch.Tensor, out: torch.Tensor | None = None,
           stream=None) -> torch.Tensor:
    """Masked straight-through backward."""
    if grad_out.dtype != torch.bfloat16:
        raise TraceError("gradients must be bf16")
    out = torch.empty_like(grad_out) if out is None else out
    trace_fq_bwd(grad_out, mask, grad_out.numel(), out, stream)
    return out


def trace_mx_capture(x, rows, cols, codes, mbits, scales, stream=None) -> None:
    _check(library().trace_mx_capture(_p(x), rows, cols, _p(codes), _p(mbits), _p(scales),
                                      _stream(stream)), "trace_mx_capture")


def trace_mx_guided_fq_fwd(x_train, rows, cols, mbits, scales, out, ste_mask, stream=None) -> None:
    _check(library().trace_mx_guided_fq_fwd(_p(x_train), rows, cols, _p(mbits), _p(scales),
                                            _p(out), _p(ste_mask), _stream(stream)),
           "trace_mx_guided_fq_fwd")


def trace_mx_full_guided_fq_fwd(x_train, rows, cols, codes, scales, out, ste_mask,
                                stream=None) -> None:
    _check(library().trace_mx_full_guided_fq_fwd(_p(x_train), rows, cols, _p(codes), _p(scales),
                                                 _p(out), _p(ste_mask), _stream(stream)),
           "trace_mx_full_guided_fq_fwd")


def trace_mx_rtn_fq_fwd(x, rows, cols, scales, out, ste_mask, stream=None) -> None:
    _check(library().trace_mx_rtn_fq_fwd(_p(x), rows, cols, _p(scales), _p(out), _p(ste_mask),
                                         _stream(stream)), "trace_mx_rtn_fq_fwd")


@dataclasses.dataclass
class MxCapture:
    """One MXFP4 capture site: full codes plus the compact cache (mantissa
    bits + E8M0 block scales, 1.25 bits per element)."""
    codes: torch.Tensor    # uint8 [N/2]
    mbits: torch.Tensor    # int32 words [N/32]
    scales: torch.Tensor   # uint8 [rows, cols/32] E8M0

    def cache_nbytes(self) -> int:
        return self.mbits.numel() * 4 + self.scales.numel()


def mx_capture(x: torch.Tensor, out: MxCapture | None = None, stream=None) -> MxCapture:
    """MXFP4 rollout capture of one site (x bf16 [rows, cols])."""
    rows, cols = _bf16_2d(x)
    n = rows * cols
    if out is None:
        out = MxCapture(codes=torch.empty(n // 2, dtype=torch.uint8, device=x.device),
                        mbits=torch.empty(n // 32, dtype=torch.int32, device=x.device),
                        scales=torch.empty(rows, cols // 32, dtype=torch.uint8, device=x.device))
    trace_mx_capture(x, rows, cols, out.codes, out.mbits, out.scales, stream)
    return out


def _fq_outputs(x, out, mask):
    rows, cols = _bf16_2d(x)
    out = torch.empty_like(x) if out is None else out
    mask = torch.empty(rows * cols // 32, dtype=torch.int32, device=x.device) if mask is None else mask
    return rows, cols, out, mask


def mx_guided_fq_fwd(x_train: torch.Tensor, cache: MxCapture, out=None, mask=None, stream=None):
    """MXFP4 1-bit guided forward.  Returns (out, mask)."""
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    trace_mx_guided_fq_fwd(x_train, rows, cols, cache.mbits, cache.scales, out, mask, stream)
    return out, mask


def mx_full_guided_fq_fwd(x_train: torch.Tensor, cache: MxCapture, out=None, mask=None,
                          stream=None):
    """MXFP4 full-information guided forward.  Returns (out, mask)."""
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    trace_mx_full_guided_fq_fwd(x_train, rows, cols, cache.codes, cache.scales, out, mask, stream)
    return out, mask


def mx_rtn_fq_fwd(x: torch.Tensor, scales: torch.Tensor, out=None, mask=None, stream=None):
    """MXFP4 round-to-nearest fake-quant with given E8M0 scales."""
    rows, cols, out, mask = _fq_outputs(x, out, mask)
    trace_mx_rtn_fq_fwd(x, rows, cols, scales, out, mask, stream)
    return out, mask


def trace_mx8_capture(x, rows, cols, codes, mbits, scales, stream=None) -> None:
    _check(library().trace_mx8_capture(_p(x), rows, cols, _p(codes), _p(mbits), _p(scales),
                                       _stream(stream)), "trace_mx8_capture")


def trace_mx8_guided_fq_fwd(x_train, rows, cols, mbits, scales, out, ste_mask, stream=None) -> None:
    _check(library().trace_mx8_guided_fq_fwd(_p(x_train), rows, cols, _p(mbits), _p(scales),
                                             _p(out), _p(ste_mask), _stream(stream)),
           "trace_mx8_guided_fq_fwd")


def trace_mx8_full_guided_fq_fwd(x_train, rows, cols, codes, scales, out, ste_mask,
                                 stream=None) -> None:
    _check(library().trace_mx8_full_guided_fq_fwd(_p(x_train), rows, cols, _p(codes), _p(scales),
                                                  _p(out), _p(ste_mask), _stream(stream)),
           "trace_mx8_full_guided_fq_fwd")


def trace_mx8_rtn_fq_fwd(x, rows, cols, scales, out, ste_mask, stream=None) -> None:
    _check(library().trace_mx8_rtn_fq_fwd(_p(x), rows, cols, _p(scales), _p(out), _p(ste_mask),
                                          _stream(stream)), "trace_mx8_rtn_fq_fwd")


def mx8_capture(x: torch.Tensor, out: MxCapture | None = None, stream=None) -> MxCapture:
    """W4A8 rollout capture (E4M3 activations, MX scales): codes are one
    byte per element."""
    rows, cols = _bf16_2d(x)
    n = rows * cols
    if out is None:
        out = MxCapture(codes=torch.empty(n, dtype=torch.uint8, device=x.device),
                        mbits=torch.empty(n // 32, dtype=torch.int32, device=x.device),
                        scales=torch.empty(rows, cols // 32, dtype=torch.uint8, device=x.device))
    trace_mx8_capture(x, rows, cols, out.codes, out.mbits, out.scales, stream)
    return out


def mx8_guided_fq_fwd(x_train: torch.Tensor, cache: MxCapture, out=None, mask=None, stream=None):
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    trace_mx8_guided_fq_fwd(x_train, rows, cols, cache.mbits, cache.scales, out, mask, stream)
    return out, mask


def mx8_full_guided_fq_fwd(x_train: torch.Tensor, cache: MxCapture, out=None, mask=None,
                           stream=None):
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    trace_mx8_full_guided_fq_fwd(x_train, rows, cols, cache.codes, cache.scales, out, mask, stream)
    return out, mask


def mx8_rtn_fq_fwd(x: torch.Tensor, scales: torch.Tensor, out=None, mask=None, stream=None):
    rows, cols, out, mask = _fq_outputs(x, out, mask)
    trace_mx8_rtn_fq_fwd(x, rows, cols, scales, out, mask, stream)
    return out, mask


# scale layouts and rounding rules of the _ex calls
TRACE_SCALES_ROW_MAJOR, TRACE_SCALES_TILED_128x4 = 0, 1
TRACE_RULE_RTN, TRACE_RULE_GUIDED, TRACE_RULE_FULL = 0, 1, 2


def trace_scale_bytes(rows: int, cols: int, block_size: int, scale_layout: int) -> int:
    return int(library().trace_scale_bytes(rows, cols, block_size, scale_layout))


def trace_capture_ex(x, rows, cols, num_groups, offsets, codes, mbits, scales, gscale, workspace,
                     workspace_bytes, scale_layout, stream=None) -> None:
    _check(library().trace_capture_ex(_p(x), rows, cols, num_groups, _p(offsets), _p(codes),
                                      _p(mbits), _p(scales), _p(gscale), _p(workspace),
                                      workspace_bytes, scale_layout, _stream(stream)),
           "trace_capture_ex")


def trace_fq_fwd_ex(rule, x_train, rows, cols, num_groups, offsets, mbits, codes, scales, gscale,
                    out, ste_mask, scale_layout, stream=None) -> None:
    _check(library().trace_fq_fwd_ex(rule, _p(x_train), rows, cols, num_groups, _p(offsets),
                                     _p(mbits), _p(codes), _p(scales), _p(gscale), _p(out),
                                     _p(ste_mask), scale_layout, _stream(stream)), "trace_fq_fwd_ex")


def trace_mx_capture_ex(x, rows, cols, codes, mbits, scales, scale_layout, stream=None) -> None:
    _check(library().trace_mx_capture_ex(_p(x), rows, cols, _p(codes), _p(mbits), _p(scales),
                                         scale_layout, _stream(stream)), "trace_mx_capture_ex")


def trace_mx_fq_fwd_ex(rule, x_train, rows, cols, mbits, codes, scales, out, ste_mask,
                       scale_layout, stream=None) -> None:
    _check(library().trace_mx_fq_fwd_ex(rule, _p(x_train), rows, cols, _p(mbits), _p(codes),
                                        _p(scales), _p(out), _p(ste_mask), scale_layout,
                                        _stream(stream)), "trace_mx_fq_fwd_ex")


def capture_tiled(x: torch.Tensor, offsets: torch.Tensor | None = None, stream=None) -> Capture:
    """NVFP4 capture with the scales in the 128 x 4 tiled layout of a
    block-scaled FP4 GEMM (Capture.scales is then a flat uint8 tensor of
    trace_scale_bytes(...) bytes, padding zeroed)."""
    rows, cols = _bf16_2d(x)
    G = _groups(offsets)
    cap, ws = alloc_capture(rows, cols, G, x.device, offsets)
    cap.scales = torch.zeros(trace_scale_bytes(rows, cols, 16, TRACE_SCALES_TILED_128x4),
                             dtype=torch.uint8, device=x.device)
    trace_capture_ex(x, rows, cols, G, offsets, cap.codes, cap.mbits, cap.scales, cap.gscale, ws,
                     ws.numel(), TRACE_SCALES_TILED_128x4, stream)
    return cap


def fq_fwd_tiled(rule: int, x_train: torch.Tensor, cache: Capture, out=None, mask=None,
                 stream=None):
    """NVFP4 forward (rule TRACE_RULE_*) reading tiled scales.  Returns (out, mask)."""
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    trace_fq_fwd_ex(rule, x_train, rows, cols, _groups(cache.offsets), cache.offsets, cache.mbits,
                    cache.codes, cache.scales, cache.gscale, out, mask, TRACE_SCALES_TILED_128x4,
                    stream)
    return out, mask


def mx_capture_tiled(x: torch.Tensor, stream=None) -> MxCapture:
    """MXFP4 capture with the E8M0 scales in the 128 x 4 tiled layout."""
    rows, cols = _bf16_2d(x)
    n = rows * cols
    cap = MxCapture(codes=torch.empty(n // 2, dtype=torch.uint8, device=x.device),
                    mbits=torch.empty(n // 32, dtype=torch.int32, device=x.device),
                    scales=torch.zeros(trace_scale_bytes(rows, cols, 32, TRACE_SCALES_TILED_128x4),
                                       dtype=torch.uint8, device=x.device))
    trace_mx_capture_ex(x, rows, cols, cap.codes, cap.mbits, cap.scales, TRACE_SCALES_TILED_128x4,
                        stream)
    return cap


def mx_fq_fwd_tiled(rule: int, x_train: torch.Tensor, cache: MxCapture, out=None, mask=None,
                    stream=None):
    """MXFP4 forward (rule TRACE_RULE_*) reading tiled scales."""
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    trace_mx_fq_fwd_ex(rule, x_train, rows, cols, cache.mbits, cache.codes, cache.scales, out,
                       mask, TRACE_SCALES_TILED_128x4, stream)
    return out, mask


def trace_capture_amax(x, rows, cols, num_groups, offsets, amax, stream=None) -> None:
    _check(library().trace_capture_amax(_p(x), rows, cols, num_groups, _p(offsets), _p(amax),
                                        _stream(stream)), "trace_capture_amax")


def trace_capture_amax_accumulate(x, rows, cols, num_groups, offsets, amax, stream=None) -> None:
    _check(library().trace_capture_amax_accumulate(_p(x), rows, cols, num_groups, _p(offsets),
                                                   _p(amax), _stream(stream)),
           "trace_capture_amax_accumulate")


def trace_capture_with_amax(x, rows, cols, num_groups, offsets, amax, codes, mbits, scales,
                            gscale, scale_layout=0, stream=None) -> None:
    _check(library().trace_capture_with_amax(_p(x), rows, cols, num_groups, _p(offsets), _p(amax),
                                             _p(codes), _p(mbits), _p(scales), _p(gscale),
                                             scale_layout, _stream(stream)),
           "trace_capture_with_amax")


def capture_sharded(x: torch.Tensor, offsets: torch.Tensor | None = None, group=None,
                    stream=None) -> Capture:
    """Capture of this rank's row shard of a tensor whose rows are spread
    over the ranks of `group` (torch.distributed; None = no reduction): the
    per-group amax is all-reduced (MAX) between the two passes, so every
    rank ends with the global scales of the whole tensor.  The one
    collective moves 4 bytes per group."""
    rows, cols = _bf16_2d(x)
    G = _groups(offsets)
    cap, _ = alloc_capture(rows, cols, G, x.device, offsets)
    amax = torch.empty(G, dtype=torch.int32, device=x.device)
    trace_capture_amax(x, rows, cols, G, offsets, amax, stream)
    if group is not None:
        import torch.distributed as dist
        s = torch.cuda.current_stream(x.device) if stream is None else stream
        with torch.cuda.stream(s):
            dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    trace_capture_with_amax(x, rows, cols, G, offsets, amax, cap.codes, cap.mbits, cap.scales,
                            cap.gscale, TRACE_SCALES_ROW_MAJOR, stream)
    return cap


def mx8_capture_tiled(x: torch.Tensor, stream=None) -> MxCapture:
    """W4A8 capture with the E8M0 scales in the 128 x 4 tiled layout."""
    rows, cols = _bf16_2d(x)
    n = rows * cols
    cap = MxCapture(codes=torch.empty(n, dtype=torch.uint8, device=x.device),
                    mbits=torch.empty(n // 32, dtype=torch.int32, device=x.device),
                    scales=torch.zeros(trace_scale_bytes(rows, cols, 32, TRACE_SCALES_TILED_128x4),
                                       dtype=torch.uint8, device=x.device))
    _check(library().trace_mx8_capture_ex(_p(x), rows, cols, _p(cap.codes), _p(cap.mbits),
                                          _p(cap.scales), TRACE_SCALES_TILED_128x4,
                                          _stream(stream)), "trace_mx8_capture_ex")
    return cap


def mx8_fq_fwd_tiled(rule: int, x_train: torch.Tensor, cache: MxCapture, out=None, mask=None,
                     stream=None):
    """W4A8 forward (rule TRACE_RULE_*) reading tiled scales."""
    rows, cols, out, mask = _fq_outputs(x_train, out, mask)
    _check(library().trace_mx8_fq_fwd_ex(rule, _p(x_train), rows, cols, _p(cache.mbits),
                                         _p(cache.codes), _p(cache.scales), _p(out), _p(mask),
                                         TRACE_SCALES_TILED_128x4, _stream(stream)),
           "trace_mx8_fq_fwd_ex")
    return out, mask


MISMATCH_RULES = ("rtn", "guided_1bit", "full_guided")
MISMATCH_BINS = 15


def mismatch_histogram(x_train: torch.Tensor, cache: Capture, hist: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """Add the ladder-distance counts of x_train against the rollout cache
    into hist (int64 [3, 15], the uint64 counts' bits; zeros if None).  Row k
    is the rule MISMATCH_RULES[k]; column d counts the elements d codewords
    from the rollout's code."""
    rows, cols = _bf16_2d(x_train)
    if hist is None:
        hist = torch.zeros(len(MISMATCH_RULES), MISMATCH_BINS, dtype=torch.int64,
                           device=x_train.device)
    trace_mismatch_histogram(x_train, rows, cols, _groups(cache.offsets), cache.offsets,
                             cache.codes, cache.scales, cache.gscale, hist, stream)
    return hist


_FORWARDS = {
    ("nvfp4", "guided"): lambda x, c: guided_fq_fwd(x, c),
    ("nvfp4", "full"): lambda x, c: full_guided_fq_fwd(x, c),
    ("nvfp4", "rtn"): lambda x, c: rtn_fq_fwd(x, c.scales, c.gscale, c.offsets),
    ("mxfp4", "guided"): lambda x, c: mx_guided_fq_fwd(x, c),
    ("mxfp4", "full"): lambda x, c: mx_full_guided_fq_fwd(x, c),
    ("mxfp4", "rtn"): lambda x, c: mx_rtn_fq_fwd(x, c.scales),
    ("w4a8", "guided"): lambda x, c: mx8_guided_fq_fwd(x, c),
    ("w4a8", "full"): lambda x, c: mx8_full_guided_fq_fwd(x, c),
    ("w4a8", "rtn"): lambda x, c: mx8_rtn_fq_fwd(x, c.scales),
}


def mx_mismatch_histogram(x_train: torch.Tensor, cache: MxCapture,
                          hist: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """mismatch_histogram for the MXFP4 variant (E8M0 scales)."""
    rows, cols = _bf16_2d(x_train)
    if hist is None:
        hist = torch.zeros(len(MISMATCH_RULES), MISMATCH_BINS, dtype=torch.int64,
                           device=x_train.device)
    _check(library().trace_mx_mismatch_histogram(_p(x_train), rows, cols, _p(cache.codes),
                                                 _p(cache.scales), _p(hist), _stream(stream)),
           "trace_mx_mismatch_histogram")
    return hist


class TraceFakeQuant(torch.autograd.Function):
    """Autograd wrapper: forward = the fake-quant forward of `fmt` ("nvfp4",
    "mxfp4", "w4a8") with `rule` ("guided": the 1-bit cache, "full": the
    whole rollout codes, "rtn": round to nearest with the rollout's scales)
    against a rollout capture of that format; backward = the masked
    straight-through estimator.  Both run in the library."""

    @staticmethod
    def forward(ctx, x_train, cache, fmt="nvfp4", rule="guided"):
        fwd = _FORWARDS.get((fmt, rule))
        if fwd is None:
            raise TraceError(f"unknown format / rule {fmt!r} / {rule!r}")
        out, mask = fwd(x_train, cache)
        ctx.save_for_backward(mask)
        return out

    @staticmethod
    def backward(ctx, grad):
        (mask,) = ctx.saved_tensors
        return fq_bwd(grad.contiguous(), mask), None, None, None


def trace_fake_quant(x_train: torch.Tensor, cache, fmt: str = "nvfp4", rule: str = "guided"):
    """Differentiable fake-quant of x_train guided by a rollout capture."""
    return TraceFakeQuant.apply(x_train, cache, fmt, rule)


class GuidedFakeQuant(torch.autograd.Function):
    """NVFP4 1-bit guided forward with the masked straight-through backward
    (the common case of TraceFakeQuant)."""

    @staticmethod
    def forward(ctx, x_train, cache: Capture):
        out, mask = guided_fq_fwd(x_train, cache)
        ctx.save_for_backward(mask)
        return out

    @staticmethod
    def backward(ctx, grad):
        (mask,) = ctx.saved_tensors
        return fq_bwd(grad.contiguous(), mask), None
