"""Seeded synthetic inputs for the attention forward (shared by tests, bench, oracle checks).

This module only draws numbers and rounds them to bf16 (or quantises them to
8-bit E4M3 with a per-tensor scale); it contains none of
the attention arithmetic, so both the CUDA path and the CPU oracle can consume
its output without sharing any of the method's code.

Recipe (stated once, used everywhere):

* generator: numpy's ``Philox`` bit generator (Philox4x64-10, Salmon et al.,
  "Parallel random numbers: as easy as 1, 2, 3", SC'11), one independent stream
  per tensor, keyed by ``seed * 16 + tensor_id`` with tensor_id Q=0, K=1, V=2,
  key_lens=3, dO=4 (the backward pass's upstream gradient);
* values: ``standard_normal`` in float32 times sigma (sigma = 1 or 0.5, both
  exact in float32), rounded to bf16 with round-to-nearest-even;
* key lengths: integers uniform on [lo, hi] inclusive, one per sequence,
  shared by all heads.

The workload shapes stand in for the pages' benchmarks (GPT-2 at 1K, a
BERT-large encoder with padding, Long-Range-Arena-like long sequences); their
datasets and weights are not used -- only the shapes, mask kinds and value
distributions.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

TENSOR_Q, TENSOR_K, TENSOR_V, TENSOR_KEYLEN = 0, 1, 2, 3
TENSOR_DO = 4   # upstream gradient dL/dO for the backward pass
TENSOR_BIAS_TABLE = 5   # custom positional bias table


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-forward problem: shapes, mask kind, value distribution, seed."""

    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    scale: float
    sigma: float = 1.0
    key_len_range: tuple[int, int] | None = None  # inclusive; None = no padding
    seed: int = 0
    window_left: int = -1                          # sliding window (fa_fwd_window); -1 = none
    alibi: bool = False                            # additive positional bias with alibi_slopes(H)
    bias_table_radius: int = -1                    # custom bias table of 2R+1 entries per head; -1 = none

    @property
    def flop(self) -> float:
        """4*B*H*Nq*Nk*d, causal counted as exactly half; with a sliding window,
        4*B*H*d times the exact number of visible (query, key) pairs."""
        if self.window_left >= 0:
            i = np.arange(self.Nq, dtype=np.int64)
            diag = i + (self.Nk - self.Nq)
            hi = np.minimum(diag + 1, self.Nk) if self.causal else np.full_like(i, self.Nk)
            lo = np.maximum(diag - self.window_left, 0)
            pairs = int(np.maximum(hi - lo, 0).sum())
            return 4.0 * self.B * self.H * self.d * pairs
        f = 4.0 * self.B * self.H * self.Nq * self.Nk * self.d
        return f / 2.0 if self.causal else f

    @property
    def algorithmic_bytes(self) -> int:
        """Every operand moved once: Q,K,V read and O written as bf16, LSE as fp32."""
        return (2 * self.B * self.H * self.d * (2 * self.Nq + 2 * self.Nk)
                + 4 * self.B * self.H * self.Nq)

    def describe(self) -> str:
        mask = "causal" if self.causal else "none"
        if self.key_len_range:
            mask = f"key_len~U{{{self.key_len_range[0]}..{self.key_len_range[1]}}}"
        return (f"B{self.B} H{self.H} Nq{self.Nq} Nk{self.Nk} d{self.d} mask={mask} "
                f"sigma={self.sigma} scale={self.scale:.6g} seed={self.seed}")


# The five problems the library is measured and checked on.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 128, 128, 64, False, 1 / 8, 1.0, None, 1),
    "gpt2_causal_1k": Workload("gpt2_causal_1k", 8, 12, 1024, 1024, 64, True, 1 / 8,
                               1.0, None, 2),
    "bert_padded_512": Workload("bert_padded_512", 16, 16, 512, 512, 64, False, 1 / 8,
                                1.0, (128, 512), 3),
    "long_16k_d64": Workload("long_16k_d64", 1, 16, 16384, 16384, 64, False, 1 / 8,
                             1.0, None, 4),
    "causal_8000_d128": Workload("causal_8000_d128", 2, 32, 8000, 8000, 128, True,
                                 float(np.float32(1 / math.sqrt(128))), 0.5, None, 5),
}
WORKLOAD_ORDER = ["tiny", "gpt2_causal_1k", "bert_padded_512", "long_16k_d64",
                  "causal_8000_d128"]

# Decode-shaped problems for the split-KV forward: one query row per (b, h)
# against a long key sequence (the inference case FlashAttention's long-sequence
# discussion leads to).  K and V (1.07 GB) are far larger than L2, so these
# measure the HBM stream.
DECODE_WORKLOADS = {
    "decode_16k_d128": Workload("decode_16k_d128", 4, 32, 1, 16384, 128, False,
                                float(np.float32(1 / math.sqrt(128))), 1.0, None, 6),
    # few heads: 8 query blocks cannot fill the GPU without splitting the keys
    "decode_64k_h8_d128": Workload("decode_64k_h8_d128", 1, 8, 1, 65536, 128, False,
                                   float(np.float32(1 / math.sqrt(128))), 1.0, None, 7),
}


def _rng(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=int(seed) * 16 + int(tensor_id)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    x = np.asarray(x, dtype=np.float32)
    u = np.ascontiguousarray(x).reshape(-1).view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16).reshape(x.shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).reshape(b.shape)


def normal_bf16(shape, seed: int, tensor_id: int, sigma: float = 1.0) -> np.ndarray:
    """N(0, sigma^2) samples rounded to bf16, as uint16 bit patterns."""
    x = _rng(seed, tensor_id).standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    return f32_to_bf16_bits(x)


def key_lengths(B: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """Per-sequence key lengths, uniform on the integers [lo, hi]."""
    return _rng(seed, TENSOR_KEYLEN).integers(lo, hi + 1, size=B, dtype=np.int64).astype(np.int32)


def make_inputs(w: Workload):
    """Return dict(q, k, v: uint16 bf16 bits [B,H,N,d]; key_lens: int32 [B] or None)."""
    q = normal_bf16((w.B, w.H, w.Nq, w.d), w.seed, TENSOR_Q, w.sigma)
    k = normal_bf16((w.B, w.H, w.Nk, w.d), w.seed, TENSOR_K, w.sigma)
    v = normal_bf16((w.B, w.H, w.Nk, w.d), w.seed, TENSOR_V, w.sigma)
    kl = None
    if w.key_len_range is not None:
        kl = key_lengths(w.B, w.key_len_range[0], w.key_len_range[1], w.seed)
    return {"q": q, "k": k, "v": v, "key_lens": kl}

def normal_e4m3(shape, seed: int, tensor_id: int, sigma: float = 1.0):
    """The same N(0, sigma^2) float32 samples as normal_bf16, stored as 8-bit E4M3
    codes with one fp32 scale per tensor: scale = max|x| / 448 (448 is the largest
    finite E4M3 value), codes = E4M3(x / scale) rounded to nearest even (torch's
    float8_e4m3fn conversion).  Returns (uint8 codes, descale = scale as float)."""
    import torch

    x = _rng(seed, tensor_id).standard_normal(size=shape, dtype=np.float32)
    if sigma != 1.0:
        x *= np.float32(sigma)
    amax = float(np.abs(x).max()) if x.size else 0.0
    scale = np.float32(amax / 448.0) if amax > 0 else np.float32(1.0)
    y = torch.from_numpy(np.ascontiguousarray(x / scale, dtype=np.float32))
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    return codes, float(scale)


def make_inputs_fp8(w: Workload):
    """E4M3 inputs of workload w (the tensors make_inputs rounds to bf16, quantised
    per tensor instead): dict(q8, k8, v8: uint8 [B,H,N,d]; q_descale, k_descale,
    v_descale: float; key_lens: int32 [B] or None)."""
    q8, qs = normal_e4m3((w.B, w.H, w.Nq, w.d), w.seed, TENSOR_Q, w.sigma)
    k8, ks = normal_e4m3((w.B, w.H, w.Nk, w.d), w.seed, TENSOR_K, w.sigma)
    v8, vs = normal_e4m3((w.B, w.H, w.Nk, w.d), w.seed, TENSOR_V, w.sigma)
    kl = None
    if w.key_len_range is not None:
        kl = key_lengths(w.B, w.key_len_range[0], w.key_len_range[1], w.seed)
    return {"q8": q8, "k8": k8, "v8": v8, "q_descale": qs, "k_descale": ks, "v_descale": vs,
            "key_lens": kl}


def alibi_slopes(H: int) -> np.ndarray:
    """The usual geometric per-head bias slopes 2^(-8(h+1)/H), fp32 [H]."""
    return (2.0 ** (-8.0 * (np.arange(H) + 1) / H)).astype(np.float32)


def bias_table(H: int, R: int, seed: int) -> np.ndarray:
    """A custom positional bias table for fa_fwd_bias_table: fp32 [H, 2R+1] of
    N(0, 1) samples (stream seed*16 + 5), one value per head and clamped relative
    position."""
    return _rng(seed, TENSOR_BIAS_TABLE).standard_normal(size=(H, 2 * R + 1), dtype=np.float32)


# Mask variants: sliding-window (local) causal attention for fa_fwd_window, each
# query seeing the 2048 keys before its position and itself; and the
# causal_8000_d128 shape with the additive positional bias (fa_fwd_bias).
WINDOW_WORKLOADS = {
    "window_16k_w2k_d128": Workload("window_16k_w2k_d128", 1, 16, 16384, 16384, 128, True,
                                    float(np.float32(1 / math.sqrt(128))), 1.0, None, 8,
                                    window_left=2048),
    "alibi_causal_8000_d128": Workload("alibi_causal_8000_d128", 2, 32, 8000, 8000, 128, True,
                                       float(np.float32(1 / math.sqrt(128))), 0.5, None, 5,
                                       alibi=True),
    # the same shape with a custom positional bias table of 2*1024+1 entries per head
    # (relative positions beyond +-1024 clamped)
    "table_causal_8000_d128": Workload("table_causal_8000_d128", 2, 32, 8000, 8000, 128, True,
                                       float(np.float32(1 / math.sqrt(128))), 0.5, None, 5,
                                       bias_table_radius=1024),
}
