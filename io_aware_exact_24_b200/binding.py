"""ctypes binding for ``libfa_b200.so`` -- argument marshalling only.

Every function here has the name of the C entry point it wraps (declared in
``include/fa.h``) and does nothing but convert Python arguments (torch
tensors, ints, streams) into the plain pointers and sizes the C ABI takes.
All computation happens in the library's CUDA kernels.  If the library is
missing the first call raises; nothing falls back to another implementation.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

FA_OK = 0
FA_ERR_INVALID_ARG = -1
FA_ERR_UNSUPPORTED = -2
FA_ERR_MISALIGNED = -3
FA_ERR_CUDA = -4
FA_ERR_NO_DEVICE = -5
FA_ERR_DEVICE_TIMEOUT = -6

_LIB_NAME = "libfa_b200.so"
_lock = threading.Lock()
_lib = None


class FaError(RuntimeError):
    """A non-zero status returned by the C library."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        detail = fa_last_error() if status == FA_ERR_CUDA else ""
        super().__init__(f"{where}: {fa_status_string(status)} (status {status})"
                         + (f": {detail}" if detail else ""))


def library_path() -> str:
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), _LIB_NAME)


def load_library() -> ctypes.CDLL:
    """Load the compiled library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            path = library_path()
            if not os.path.exists(path):
                raise ImportError(
                    f"{path} is missing: build it with `python -m io_aware_exact_24_b200.build` "
                    "(there is no fallback implementation)")
            lib = ctypes.CDLL(path)
            vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32,
                                   vp, vp]
            lib.fa_fwd.restype = i32
            lib.fa_fwd_window.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32,
                                          vp, i32, vp]
            lib.fa_fwd_window.restype = i32
            lib.fa_fwd_bias.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32,
                                        vp, vp, i32, vp]
            lib.fa_fwd_bias.restype = i32
            lib.fa_fwd_bias_table.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                              i32, vp, vp, i32, i32, vp]
            lib.fa_fwd_bias_table.restype = i32
            lib.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, f32,
                                       f32, i32, vp, vp]
            lib.fa_fwd_fp8.restype = i32
            lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                   i32, vp, vp, sz, vp]
            lib.fa_bwd.restype = i32
            lib.fa_bwd_workspace_size.argtypes = [i32, i32, i32, i32]
            lib.fa_bwd_workspace_size.restype = sz
            lib.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                          f32, i32, vp]
            lib.fa_fwd_varlen.restype = i32
            lib.fa_fwd_host_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
            lib.fa_fwd_host_workspace_size.restype = sz
            lib.fa_fwd_host.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                        i32, vp, vp, sz, vp]
            lib.fa_fwd_host.restype = i32
            lib.fa_splitkv_num_splits.argtypes = [i32, i32, i32, i32]
            lib.fa_splitkv_num_splits.restype = i32
            lib.fa_fwd_splitkv_workspace_size.argtypes = [i32, i32, i32, i32, i32]
            lib.fa_fwd_splitkv_workspace_size.restype = sz
            lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32,
                                           i32, vp, i32, vp, sz, vp]
            lib.fa_fwd_splitkv.restype = i32
            lib.fa_fwd_splitkv_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                   f32, i32, vp, i32, vp]
            lib.fa_fwd_splitkv_noalloc.restype = i32
            lib.fa_status_string.argtypes = [i32]
            lib.fa_status_string.restype = ctypes.c_char_p
            lib.fa_get_device_status.argtypes = [vp]
            lib.fa_get_device_status.restype = i32
            lib.fa_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, vp]
            lib.fa_selftest_wait_timeout.restype = i32
            lib.fa_selftest_fwd_timeout.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32,
                                                    f32, i32, ctypes.c_ulonglong, vp]
            lib.fa_selftest_fwd_timeout.restype = i32
            lib.fa_selftest_bwd_timeout.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32,
                                                    i32, i32, f32, i32, vp, sz, ctypes.c_ulonglong, vp]
            lib.fa_selftest_bwd_timeout.restype = i32
            lib.fa_last_error.argtypes = []
            lib.fa_last_error.restype = ctypes.c_char_p
            lib.fa_version.argtypes = []
            lib.fa_version.restype = i32
            _lib = lib
    return _lib


def _addr(x) -> int | None:
    """Raw address of a torch tensor / numpy array / int / None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return int(x.data_ptr())
    if hasattr(x, "ctypes"):
        return int(x.ctypes.data)
    raise TypeError(f"cannot take the address of {type(x)!r}")


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def fa_status_string(status: int) -> str:
    return load_library().fa_status_string(int(status)).decode()


def fa_last_error() -> str:
    return load_library().fa_last_error().decode()


def fa_version() -> int:
    return int(load_library().fa_version())


def fa_fwd(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal=False, key_lens=None,
           stream=None, check=True) -> int:
    """``fa_fwd`` of include/fa.h.  Pointers are device tensors (or raw ints)."""
    st = load_library().fa_fwd(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                               int(B), int(H), int(N_q), int(N_k), int(d), float(scale),
                               int(bool(causal)), _addr(key_lens), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd")
    return st


def fa_fwd_window(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens, window_left,
                  stream=None, check=True) -> int:
    """``fa_fwd_window`` of include/fa.h: forward with a sliding window of window_left keys."""
    st = load_library().fa_fwd_window(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                      int(B), int(H), int(N_q), int(N_k), int(d), float(scale),
                                      int(bool(causal)), _addr(key_lens), int(window_left),
                                      _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_window")
    return st


def fa_fwd_bias(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens, slopes,
                window_left=-1, stream=None, check=True) -> int:
    """``fa_fwd_bias`` of include/fa.h: forward with the additive positional bias."""
    st = load_library().fa_fwd_bias(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                    int(B), int(H), int(N_q), int(N_k), int(d), float(scale),
                                    int(bool(causal)), _addr(key_lens), _addr(slopes),
                                    int(window_left), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_bias")
    return st


def fa_fwd_bias_table(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens, table, radius,
                      window_left=-1, stream=None, check=True) -> int:
    """``fa_fwd_bias_table`` of include/fa.h: forward with a custom positional bias table."""
    st = load_library().fa_fwd_bias_table(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                          int(B), int(H), int(N_q), int(N_k), int(d), float(scale),
                                          int(bool(causal)), _addr(key_lens), _addr(table),
                                          int(radius), int(window_left), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_bias_table")
    return st


def fa_fwd_fp8(q8, k8, v8, o, lse, B, H, N_q, N_k, d, scale, q_descale, k_descale, v_descale,
               causal, key_lens, stream=None, check=True) -> int:
    """``fa_fwd_fp8`` of include/fa.h: forward on E4M3 inputs with per-tensor descales."""
    st = load_library().fa_fwd_fp8(_addr(q8), _addr(k8), _addr(v8), _addr(o), _addr(lse),
                                   int(B), int(H), int(N_q), int(N_k), int(d), float(scale),
                                   float(q_descale), float(k_descale), float(v_descale),
                                   int(bool(causal)), _addr(key_lens), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_fp8")
    return st


def fa_bwd_workspace_size(B, H, N_q, d) -> int:
    return int(load_library().fa_bwd_workspace_size(int(B), int(H), int(N_q), int(d)))


def fa_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, H, N_q, N_k, d, scale, causal, key_lens,
           workspace, workspace_bytes, stream=None, check=True) -> int:
    """``fa_bwd`` of include/fa.h: gradients of the forward given dO (device workspace given)."""
    st = load_library().fa_bwd(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), _addr(dout),
                               _addr(dq), _addr(dk), _addr(dv), int(B), int(H), int(N_q), int(N_k),
                               int(d), float(scale), int(bool(causal)), _addr(key_lens),
                               _addr(workspace), int(workspace_bytes), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_bwd")
    return st


def fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, total_q, total_k,
                  max_seqlen_q, d, scale, causal=False, stream=None, check=True) -> int:
    """``fa_fwd_varlen`` of include/fa.h: packed variable-length batches."""
    st = load_library().fa_fwd_varlen(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                      _addr(cu_seqlens_q), _addr(cu_seqlens_k), int(B), int(H),
                                      int(total_q), int(total_k), int(max_seqlen_q), int(d),
                                      float(scale), int(bool(causal)), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_varlen")
    return st


def fa_splitkv_num_splits(B, H, N_q, N_k) -> int:
    return int(load_library().fa_splitkv_num_splits(int(B), int(H), int(N_q), int(N_k)))


def fa_fwd_splitkv_workspace_size(B, H, N_q, d, num_splits) -> int:
    return int(load_library().fa_fwd_splitkv_workspace_size(int(B), int(H), int(N_q), int(d),
                                                             int(num_splits)))


def fa_fwd_splitkv(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens, num_splits,
                   workspace, workspace_bytes, stream=None, check=True) -> int:
    """``fa_fwd_splitkv`` of include/fa.h: split-KV forward, device workspace given."""
    st = load_library().fa_fwd_splitkv(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                       int(B), int(H), int(N_q), int(N_k), int(d),
                                       float(scale), int(bool(causal)), _addr(key_lens),
                                       int(num_splits), _addr(workspace), int(workspace_bytes),
                                       _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv")
    return st


def fa_fwd_splitkv_noalloc(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens,
                           num_splits, stream=None, check=True) -> int:
    """``fa_fwd_splitkv_noalloc`` of include/fa.h: split-KV forward on the library's own scratch."""
    st = load_library().fa_fwd_splitkv_noalloc(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                               int(B), int(H), int(N_q), int(N_k), int(d),
                                               float(scale), int(bool(causal)), _addr(key_lens),
                                               int(num_splits), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_splitkv_noalloc")
    return st


def fa_fwd_host_workspace_size(B, H, N_q, N_k, d, has_key_lens) -> int:
    return int(load_library().fa_fwd_host_workspace_size(
        int(B), int(H), int(N_q), int(N_k), int(d), int(bool(has_key_lens))))


def fa_fwd_host(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens, workspace,
                workspace_bytes, stream=None, check=True) -> int:
    """``fa_fwd_host`` of include/fa.h: host buffers in and out, device workspace given."""
    st = load_library().fa_fwd_host(_addr(q), _addr(k), _addr(v), _addr(o), _addr(lse),
                                    int(B), int(H), int(N_q), int(N_k), int(d),
                                    float(scale), int(bool(causal)), _addr(key_lens),
                                    _addr(workspace), int(workspace_bytes), _stream(stream))
    if check and st != FA_OK:
        raise FaError(st, "fa_fwd_host")
    return st


def fa_get_device_status(stream=None) -> int:
    return int(load_library().fa_get_device_status(_stream(stream)))


def fa_selftest_wait_timeout(limit_cycles: int, stream=None) -> int:
    """``fa_selftest_wait_timeout`` of include/fa.h (bounded-wait self test)."""
    return int(load_library().fa_selftest_wait_timeout(int(limit_cycles), _stream(stream)))


def fa_selftest_fwd_timeout(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, limit_cycles,
                            stream=None) -> int:
    """``fa_selftest_fwd_timeout`` of include/fa.h: the forward kernel with a short wait limit."""
    return int(load_library().fa_selftest_fwd_timeout(
        _addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), int(B), int(H), int(N_q), int(N_k),
        int(d), float(scale), int(bool(causal)), int(limit_cycles), _stream(stream)))


def fa_selftest_bwd_timeout(q, k, v, o, lse, dout, dq, dk, dv, B, H, N_q, N_k, d, scale, causal,
                            workspace, workspace_bytes, limit_cycles, stream=None) -> int:
    """``fa_selftest_bwd_timeout`` of include/fa.h: the backward kernel with a short wait limit."""
    return int(load_library().fa_selftest_bwd_timeout(
        _addr(q), _addr(k), _addr(v), _addr(o), _addr(lse), _addr(dout), _addr(dq), _addr(dk),
        _addr(dv), int(B), int(H), int(N_q), int(N_k), int(d), float(scale), int(bool(causal)),
        _addr(workspace), int(workspace_bytes), int(limit_cycles), _stream(stream)))


def attention(q, k, v, causal=False, key_lens=None, scale=None, stream=None):
    """Convenience wrapper: allocate O and LSE with torch and call ``fa_fwd``.

    q: bf16 [B,H,N_q,d]; k, v: bf16 [B,H,N_k,d]; all contiguous on one CUDA
    device.  key_lens: int32 [B] on the same device, or None.  Returns
    (O bf16 [B,H,N_q,d], LSE fp32 [B,H,N_q]).
    """
    import torch
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor [B,H,N,d]")
    B, H, N_q, d = q.shape
    N_k = k.shape[2]
    if tuple(k.shape) != (B, H, N_k, d) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("shape mismatch between q, k and v")
    if key_lens is not None:
        if key_lens.dtype != torch.int32 or key_lens.device != q.device or key_lens.numel() != B:
            raise ValueError("key_lens must be int32 [B] on q's device")
        key_lens = key_lens.contiguous()
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, o, lse, B, H, N_q, N_k, d, scale, causal, key_lens, stream)
    return o, lse
