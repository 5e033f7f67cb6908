"""fp64 CPU oracle for the exact attention forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg (and its ``--impl reference`` arm) may import this package.  The product
path (``io_aware_exact_24_b200``) never does, and this package never imports
the product.

Two independent C formulations are wrapped here:

* ``attn_ref``    (attn_ref.c): the plain definition, S and P materialised per
  row -- "FlashAttention 与边缘设备上的注意力内存瓶颈", section 2, and
  "FlashAttention：把注意力从公式写成数据流", opening paragraph.
* ``attn_online`` (attn_online.c): the block-wise online-softmax recurrence --
  "FlashAttention：把注意力从公式写成数据流", section "分块与在线 softmax".

Inputs are bf16 *bit patterns* (``numpy.uint16``) so that the oracle sees
exactly the bytes the GPU sees; outputs are fp64 and never rounded.

Pins (what ties this oracle to something other than itself) live in
``tests/test_oracle_pins.py`` and ``tests/test_golden.py``.  The GPU-internal
rounding of P to bf16 has no counterpart here: "parity unpinned" for that
detail, bounded only by the stated output tolerances.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SOURCES = ("attn_ref.c", "attn_online.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, OpenMP)."""
    srcs = [os.path.join(_HERE, s) for s in _SOURCES]
    if not force and os.path.exists(_LIB_PATH):
        lib_mtime = os.path.getmtime(_LIB_PATH)
        if all(os.path.getmtime(s) <= lib_mtime for s in srcs):
            return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-Wall",
           "-o", tmp, *srcs, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            i64, i32, f32 = ctypes.c_int64, ctypes.c_int, ctypes.c_float
            f64 = ctypes.c_double
            vp = ctypes.c_void_p
            lib.attn_ref_fp64.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                          f64, i32, vp, vp, vp]
            lib.attn_ref_fp64.restype = i32
            lib.attn_ref_fp64_window.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                                 f64, i32, i64, vp, vp, vp]
            lib.attn_ref_fp64_window.restype = i32
            lib.attn_ref_fp64_bias.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                               f64, i32, i64, vp, vp, vp, vp]
            lib.attn_ref_fp64_bias.restype = i32
            lib.attn_ref_fp64_bias_table.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                                     f64, i32, i64, vp, i64, vp, vp, vp]
            lib.attn_ref_fp64_bias_table.restype = i32
            lib.attn_ref_fp64_rows.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64,
                                               i64, f64, i32, vp, i64, vp, vp]
            lib.attn_ref_fp64_rows.restype = i32
            lib.attn_online_fp64.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64,
                                             i64, f32, i32, i64, vp, vp]
            lib.attn_online_fp64.restype = i32
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = i32
            lib.oracle_set_num_threads.argtypes = [i32]
            lib.oracle_set_num_threads.restype = None
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (set OMP_NUM_THREADS, or set_num_threads, to change)."""
    return int(_load().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Use n OpenMP threads in the following oracle calls (n >= 1)."""
    _load().oracle_set_num_threads(int(n))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(q, k, v, key_lens):
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B,H,N,d] bf16 bit arrays")
    B, H, Nq, d = q.shape
    if k.shape[:2] != (B, H) or k.shape[3] != d or v.shape != k.shape:
        raise ValueError("shape mismatch between q, k, v")
    if key_lens is not None:
        key_lens = np.ascontiguousarray(key_lens, dtype=np.int32)
        if key_lens.shape != (B,):
            raise ValueError("key_lens must be int32 [B]")
    return q, k, v, key_lens, B, H, Nq, k.shape[2], d


def attn_ref(q, k, v, scale, causal=False, key_lens=None, return_p=False):
    """Plain definition.  Returns (O fp64 [B,H,Nq,d], LSE fp64 [B,H,Nq][, P]).
    ``scale`` is rounded to fp32 first: it is the fp32 value the library receives."""
    return _attn_ref_f64scale(q, k, v, float(np.float32(scale)), causal, key_lens, return_p)


def _attn_ref_f64scale(q, k, v, scale, causal=False, key_lens=None, return_p=False):
    """attn_ref with ``scale`` taken as the fp64 value given (no rounding)."""
    q, k, v, key_lens, B, H, Nq, Nk, d = _check(q, k, v, key_lens)
    o = np.empty((B, H, Nq, d), np.float64)
    lse = np.empty((B, H, Nq), np.float64)
    p = np.empty((B, H, Nq, Nk), np.float64) if return_p else None
    rc = _load().attn_ref_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(key_lens), B, H,
                               Nq, Nk, d, float(scale), int(bool(causal)),
                               _ptr(o), _ptr(lse), _ptr(p))
    if rc != 0:
        raise RuntimeError(f"attn_ref_fp64 failed ({rc})")
    return (o, lse, p) if return_p else (o, lse)


def attn_ref_window(q, k, v, scale, window_left, causal=False, key_lens=None):
    """Plain definition with a sliding window of window_left keys before each
    row's diagonal position.  Returns (O fp64 [B,H,Nq,d], LSE fp64 [B,H,Nq])."""
    q, k, v, key_lens, B, H, Nq, Nk, d = _check(q, k, v, key_lens)
    o = np.empty((B, H, Nq, d), np.float64)
    lse = np.empty((B, H, Nq), np.float64)
    rc = _load().attn_ref_fp64_window(_ptr(q), _ptr(k), _ptr(v), _ptr(key_lens), B, H,
                                      Nq, Nk, d, float(np.float32(scale)), int(bool(causal)),
                                      int(window_left), _ptr(o), _ptr(lse), None)
    if rc != 0:
        raise RuntimeError(f"attn_ref_fp64_window failed ({rc})")
    return o, lse


def attn_ref_bias(q, k, v, scale, slopes, causal=False, key_lens=None, window_left=-1):
    """Plain definition with the additive positional bias -slopes[h]*|i + Nk - Nq - j|
    (slopes: fp32 [H]) and optionally a sliding window.  Returns (O, LSE) in fp64."""
    q, k, v, key_lens, B, H, Nq, Nk, d = _check(q, k, v, key_lens)
    sl = np.ascontiguousarray(slopes, dtype=np.float32)
    if sl.shape != (H,):
        raise ValueError("slopes must be fp32 [H]")
    o = np.empty((B, H, Nq, d), np.float64)
    lse = np.empty((B, H, Nq), np.float64)
    rc = _load().attn_ref_fp64_bias(_ptr(q), _ptr(k), _ptr(v), _ptr(key_lens), B, H, Nq, Nk,
                                    d, float(np.float32(scale)), int(bool(causal)),
                                    int(window_left), _ptr(sl), _ptr(o), _ptr(lse), None)
    if rc != 0:
        raise RuntimeError(f"attn_ref_fp64_bias failed ({rc})")
    return o, lse


def attn_ref_bias_table(q, k, v, scale, table, causal=False, key_lens=None, window_left=-1):
    """Plain definition with a custom positional bias: table fp32 [H, 2R+1] adds
    table[h, clamp(j - (i + Nk - Nq), -R, R) + R] to the score of query i and key j
    (natural-log units, after the scale), optionally with a sliding window.
    Returns (O fp64 [B,H,Nq,d], LSE fp64 [B,H,Nq])."""
    q, k, v, key_lens, B, H, Nq, Nk, d = _check(q, k, v, key_lens)
    tb = np.ascontiguousarray(table, dtype=np.float32)
    if tb.ndim != 2 or tb.shape[0] != H or tb.shape[1] % 2 != 1:
        raise ValueError("table must be fp32 [H, 2R+1]")
    R = (tb.shape[1] - 1) // 2
    o = np.empty((B, H, Nq, d), np.float64)
    lse = np.empty((B, H, Nq), np.float64)
    rc = _load().attn_ref_fp64_bias_table(_ptr(q), _ptr(k), _ptr(v), _ptr(key_lens), B, H, Nq,
                                          Nk, d, float(np.float32(scale)), int(bool(causal)),
                                          int(window_left), _ptr(tb), R, _ptr(o), _ptr(lse), None)
    if rc != 0:
        raise RuntimeError(f"attn_ref_fp64_bias_table failed ({rc})")
    return o, lse


def attn_ref_varlen(q, k, v, cu_q, cu_k, scale, causal=False):
    """Packed variable-length batches: q [Tq,H,d], k/v [Tk,H,d] bf16 bits, cu_q/cu_k
    int [B+1].  Each sequence is an independent problem, evaluated with attn_ref on
    its own slice.  Returns (O fp64 [Tq,H,d], LSE fp64 [Tq,H])."""
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k = np.ascontiguousarray(k, dtype=np.uint16)
    v = np.ascontiguousarray(v, dtype=np.uint16)
    Tq, H, d = q.shape
    o = np.zeros((Tq, H, d), np.float64)
    lse = np.full((Tq, H), -np.inf, np.float64)
    for b in range(len(cu_q) - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 <= q0:
            continue
        qb = q[q0:q1].transpose(1, 0, 2)[None]
        kb = k[k0:k1].transpose(1, 0, 2)[None]
        vb = v[k0:k1].transpose(1, 0, 2)[None]
        ob, lb = attn_ref(qb, kb, vb, scale, causal, None)
        o[q0:q1] = ob[0].transpose(1, 0, 2)
        lse[q0:q1] = lb[0].T
    return o, lse


def attn_ref_rows(q, k, v, scale, row_ids, causal=False, key_lens=None):
    """Definition on selected flat rows r=(b*H+h)*Nq+i.  Returns (O [n,d], LSE [n]).
    ``scale`` is rounded to fp32 first, as in attn_ref."""
    return _attn_ref_rows_f64scale(q, k, v, float(np.float32(scale)), row_ids, causal, key_lens)


def _attn_ref_rows_f64scale(q, k, v, scale, row_ids, causal=False, key_lens=None):
    """attn_ref_rows with ``scale`` taken as the fp64 value given."""
    q, k, v, key_lens, B, H, Nq, Nk, d = _check(q, k, v, key_lens)
    rows = np.ascontiguousarray(row_ids, dtype=np.int64)
    o = np.empty((rows.size, d), np.float64)
    lse = np.empty((rows.size,), np.float64)
    rc = _load().attn_ref_fp64_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(key_lens), B, H,
                                    Nq, Nk, d, float(scale),
                                    int(bool(causal)), _ptr(rows), rows.size,
                                    _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"attn_ref_fp64_rows failed ({rc})")
    return o, lse


def attn_online(q, k, v, scale, causal=False, key_lens=None, block=7):
    """Online-softmax formulation.  Returns (O fp64, LSE fp64)."""
    q, k, v, key_lens, B, H, Nq, Nk, d = _check(q, k, v, key_lens)
    o = np.empty((B, H, Nq, d), np.float64)
    lse = np.empty((B, H, Nq), np.float64)
    rc = _load().attn_online_fp64(_ptr(q), _ptr(k), _ptr(v), _ptr(key_lens), B, H,
                                  Nq, Nk, d, float(np.float32(scale)),
                                  int(bool(causal)), int(block), _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError(f"attn_online_fp64 failed ({rc})")
    return o, lse


# --------------------------------------------------------------------------------------
# FP8 (e4m3) inputs with per-tensor scales: "FlashAttention：把注意力从公式写成数据流",
# section "FA2 与 FA3" (the Hopper kernel brings low-precision arithmetic in) and
# section "用实验验证而不是背诵结论" (FP8 saves HBM bytes but needs scaling; report
# its error against a 16-bit baseline).  What is computed is the attention of the
# dequantised inputs: Q = q_descale * Q8, K = k_descale * K8, V = v_descale * V8.

def e4m3_to_f64(codes) -> np.ndarray:
    """Decode 8-bit E4M3 codes (the OCP 8-bit floating point format, 'fn' flavour):
    sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 holds
    the subnormals m * 2^-9; no infinities; 0x7F and 0xFF are NaN (largest finite
    value 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    val = sign * mag
    return np.where((e == 15) & (m == 7), np.nan, val)


def e4m3_to_bf16_bits(codes) -> np.ndarray:
    """The bf16 bit pattern of each E4M3 value (exact: 4 significant bits and
    exponents -9..8 fit in bf16)."""
    f = e4m3_to_f64(codes).astype(np.float32)
    u = f.view(np.uint32)
    finite = np.isfinite(f)
    if np.any((u[finite] & np.uint32(0xFFFF)) != 0):
        raise AssertionError("e4m3 value not exact in bf16")
    return (u >> np.uint32(16)).astype(np.uint16)


def _e4m3_scale(scale, q_descale, k_descale):
    # The scores of the dequantised inputs are scale * (qd Q8)(kd K8)^T =
    # (scale * qd * kd) * Q8 K8^T: the product of the three fp32 factors, taken
    # exactly (in fp64, where the product of three 24-bit significands is off by
    # at most one rounding of 2^-53), not folded into one fp32 number.
    return float(np.float64(np.float32(scale)) * np.float64(np.float32(q_descale))
                 * np.float64(np.float32(k_descale)))


def attn_ref_e4m3(q8, k8, v8, scale, q_descale, k_descale, v_descale, causal=False, key_lens=None):
    """Plain definition on dequantised e4m3 inputs (uint8 codes [B,H,N,d]):
    softmax(scale * (qd Q8)(kd K8)^T) (vd V8) = vd * attn(Q8, K8, V8; scale*qd*kd).
    Returns (O fp64 [B,H,Nq,d], LSE fp64 [B,H,Nq])."""
    o, lse = _attn_ref_f64scale(e4m3_to_bf16_bits(q8), e4m3_to_bf16_bits(k8),
                                e4m3_to_bf16_bits(v8), _e4m3_scale(scale, q_descale, k_descale),
                                causal, key_lens)
    return o * np.float64(np.float32(v_descale)), lse


def attn_ref_rows_e4m3(q8, k8, v8, scale, q_descale, k_descale, v_descale, row_ids, causal=False,
                       key_lens=None):
    """attn_ref_e4m3 on selected flat rows r=(b*H+h)*Nq+i.  Returns (O [n,d], LSE [n])."""
    o, lse = _attn_ref_rows_f64scale(e4m3_to_bf16_bits(q8), e4m3_to_bf16_bits(k8),
                                     e4m3_to_bf16_bits(v8), _e4m3_scale(scale, q_descale, k_descale),
                                     row_ids, causal, key_lens)
    return o * np.float64(np.float32(v_descale)), lse


# Backward pass (gradients of the plain definition): numpy, in its own module.
from .attn_bwd import attn_bwd_ref  # noqa: E402,F401
