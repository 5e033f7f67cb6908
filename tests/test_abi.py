"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from io_aware_exact_24_b200 import binding
from io_aware_exact_24_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.load_library()


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        names += re.findall(r"^FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text, flags=re.M)
    return names


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("fa_fwd", "fa_fwd_host", "fa_fwd_host_workspace_size", "fa_status_string",
                 "fa_get_device_status", "fa_version", "fa_selftest_wait_timeout",
                 "fa_selftest_fwd_timeout", "fa_selftest_bwd_timeout"):
        assert must in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings_and_version(lib):
    assert binding.fa_status_string(0) == "FA_OK"
    for code in range(-6, 0):
        assert binding.fa_status_string(code).startswith("FA_ERR_")
    assert binding.fa_status_string(12345) == "unknown status"
    assert binding.fa_version() == 10000


# A fake, suitably aligned "device" address: validation must fail before it is used.
P = 1 << 20


def call(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Nq=8, Nk=8, d=64, scale=0.125, causal=0,
         key_lens=None):
    return binding.fa_fwd(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, key_lens,
                          stream=0, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(d=32), binding.FA_ERR_UNSUPPORTED),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(d=256), binding.FA_ERR_UNSUPPORTED),
    (dict(B=-1), binding.FA_ERR_INVALID_ARG),
    (dict(H=-2), binding.FA_ERR_INVALID_ARG),
    (dict(Nq=-1), binding.FA_ERR_INVALID_ARG),
    (dict(Nk=-1), binding.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(scale=-0.5), binding.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.FA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), binding.FA_ERR_INVALID_ARG),
    (dict(scale=1e-46), binding.FA_ERR_INVALID_ARG),   # 0 once rounded to fp32
    (dict(q=None), binding.FA_ERR_INVALID_ARG),
    (dict(o=None), binding.FA_ERR_INVALID_ARG),
    (dict(lse=None), binding.FA_ERR_INVALID_ARG),
    (dict(k=None), binding.FA_ERR_INVALID_ARG),
    (dict(v=None), binding.FA_ERR_INVALID_ARG),
    (dict(q=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(k=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(v=P + 4), binding.FA_ERR_MISALIGNED),
    (dict(o=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(lse=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(key_lens=P + 1), binding.FA_ERR_MISALIGNED),
    (dict(B=70000), binding.FA_ERR_UNSUPPORTED),
    (dict(H=65536), binding.FA_ERR_UNSUPPORTED),
])
def test_argument_errors_are_reported_before_any_cuda_call(lib, kw, code):
    assert call(**kw) == code


@pytest.mark.parametrize("kw", [dict(B=0), dict(H=0), dict(Nq=0),
                                dict(B=0, q=None, k=None, v=None, o=None, lse=None)])
def test_empty_problems_are_noops(lib, kw):
    assert call(**kw) == binding.FA_OK


def test_no_keys_allows_null_k_v_until_the_device_check(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("would launch on fake addresses; covered by the GPU tests")
    assert call(Nk=0, k=None, v=None) == binding.FA_ERR_NO_DEVICE


def test_host_entry_validates_workspace(lib):
    need = binding.fa_fwd_host_workspace_size(2, 3, 100, 50, 64, True)
    assert need >= 2 * 3 * (100 + 2 * 50 + 100) * 64 * 2 + 2 * 3 * 100 * 4 + 8
    assert need % 256 == 0
    assert binding.fa_fwd_host_workspace_size(1, 1, 8, 8, 96, False) == 0
    st = binding.fa_fwd_host(P, P, P, P, P, 1, 1, 8, 8, 64, 0.125, 0, None, P, 16,
                             stream=0, check=False)
    assert st == binding.FA_ERR_INVALID_ARG
    need = binding.fa_fwd_host_workspace_size(1, 1, 8, 8, 64, False)
    st = binding.fa_fwd_host(P, P, P, P, P, 1, 1, 8, 8, 64, 0.125, 0, None, P + 16, need,
                             stream=0, check=False)
    assert st == binding.FA_ERR_MISALIGNED


def test_without_a_gpu_valid_calls_report_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call() == binding.FA_ERR_NO_DEVICE
    assert binding.fa_get_device_status(0) == binding.FA_ERR_NO_DEVICE


# ---------------------------------------------------------------- split-KV entry points

def test_splitkv_workspace_size_formula(lib):
    for B, H, Nq, d, S in ((1, 1, 1, 64, 1), (2, 3, 5, 128, 7), (4, 32, 1, 128, 16)):
        rows = S * B * H * Nq
        need = binding.fa_fwd_splitkv_workspace_size(B, H, Nq, d, S)
        o_bytes = -(-rows * d * 4 // 256) * 256
        blocks = -(-Nq // 128) * B * H          # one 64-bit arrival word per query block
        assert need == o_bytes + -(-rows * 4 // 256) * 256 + -(-blocks * 8 // 256) * 256
    assert binding.fa_fwd_splitkv_workspace_size(1, 1, 1, 96, 2) == 0
    assert binding.fa_fwd_splitkv_workspace_size(1, 1, 1, 64, 0) == 0
    assert binding.fa_fwd_splitkv_workspace_size(1, 1, 1, 64, 257) == 0
    assert binding.fa_fwd_splitkv_workspace_size(-1, 1, 1, 64, 2) == 0


def test_splitkv_num_splits_heuristic(lib):
    # few query blocks and many key tiles: spread over the SMs, >= 2 tiles per range
    assert binding.fa_splitkv_num_splits(1, 1, 1, 1 << 20) == 148
    assert binding.fa_splitkv_num_splits(1, 8, 1, 16384) == 18      # 144 CTAs: one wave
    assert binding.fa_splitkv_num_splits(1, 8, 1, 1024) == 4        # 8 tiles -> ranges of >= 2
    assert binding.fa_splitkv_num_splits(1, 1, 1, 300) == 1         # 3 tiles -> ranges of >= 2
    assert binding.fa_splitkv_num_splits(1, 70, 1, 8192) == 2
    assert binding.fa_splitkv_num_splits(1, 100, 1, 8192) == 1
    assert binding.fa_splitkv_num_splits(4, 32, 1, 16384) == 1      # 128 CTAs fill the GPU
    assert binding.fa_splitkv_num_splits(8, 32, 128, 8192) == 1
    assert binding.fa_splitkv_num_splits(0, 1, 1, 100) == 1


def splitkv_call(num_splits=4, ws=P, ws_bytes=1 << 30, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Nq=8, Nk=8, d=64, scale=0.125, causal=0,
             key_lens=None)
    a.update(kw)
    return binding.fa_fwd_splitkv(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                                  a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"],
                                  a["key_lens"], num_splits, ws, ws_bytes, stream=0, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(num_splits=0), binding.FA_ERR_INVALID_ARG),
    (dict(num_splits=257), binding.FA_ERR_INVALID_ARG),
    (dict(ws=None), binding.FA_ERR_INVALID_ARG),
    (dict(ws_bytes=16), binding.FA_ERR_INVALID_ARG),
    (dict(ws=P + 128), binding.FA_ERR_MISALIGNED),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(scale=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(q=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(num_splits=0, B=0), binding.FA_ERR_INVALID_ARG),
    (dict(B=0, ws=None), binding.FA_OK),
])
def test_splitkv_argument_errors_before_any_cuda_call(lib, kw, code):
    assert splitkv_call(**kw) == code


def test_splitkv_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert splitkv_call() == binding.FA_ERR_NO_DEVICE


# ---------------------------------------------------------------- sliding window entry point

def window_call(window_left=16, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=1, Nq=8, Nk=8, d=64, scale=0.125, causal=1,
             key_lens=None)
    a.update(kw)
    return binding.fa_fwd_window(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                                 a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"],
                                 a["key_lens"], window_left, stream=0, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(window_left=-1), binding.FA_ERR_INVALID_ARG),
    (dict(window_left=-100, B=0), binding.FA_ERR_INVALID_ARG),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(o=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(Nq=0), binding.FA_OK),
])
def test_window_argument_errors_before_any_cuda_call(lib, kw, code):
    assert window_call(**kw) == code


def test_window_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert window_call(window_left=0) == binding.FA_ERR_NO_DEVICE


# ---------------------------------------------------------------- additive bias entry point

def bias_call(slopes=P, window_left=-1, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=2, Nq=8, Nk=8, d=64, scale=0.125, causal=1,
             key_lens=None)
    a.update(kw)
    return binding.fa_fwd_bias(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                               a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"], a["key_lens"],
                               slopes, window_left, stream=0, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(slopes=None), binding.FA_ERR_INVALID_ARG),
    (dict(slopes=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(scale=-1.0), binding.FA_ERR_INVALID_ARG),
    (dict(B=0, slopes=None), binding.FA_OK),
])
def test_bias_argument_errors_before_any_cuda_call(lib, kw, code):
    assert bias_call(**kw) == code


def test_bias_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert bias_call() == binding.FA_ERR_NO_DEVICE


# ---------------------------------------------------------------- bias table entry point

def table_call(table=P, radius=4, window_left=-1, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=2, Nq=8, Nk=8, d=64, scale=0.125, causal=1,
             key_lens=None)
    a.update(kw)
    return binding.fa_fwd_bias_table(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"],
                                     a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"],
                                     a["key_lens"], table, radius, window_left, stream=0,
                                     check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(table=None), binding.FA_ERR_INVALID_ARG),
    (dict(table=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(radius=-1), binding.FA_ERR_INVALID_ARG),
    (dict(radius=(1 << 30) + 1), binding.FA_ERR_INVALID_ARG),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), binding.FA_ERR_INVALID_ARG),
    (dict(B=0, table=None), binding.FA_OK),
])
def test_bias_table_argument_errors_before_any_cuda_call(lib, kw, code):
    assert table_call(**kw) == code


def test_bias_table_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert table_call() == binding.FA_ERR_NO_DEVICE
    assert table_call(radius=0) == binding.FA_ERR_NO_DEVICE


def test_selftest_fwd_timeout_argument_errors(lib):
    f = lambda **kw: binding.fa_selftest_fwd_timeout(
        P, P, P, P, P, kw.get("B", 1), 2, kw.get("Nq", 8), kw.get("Nk", 8), 64, 0.125, 1,
        kw.get("limit", 2), stream=0)
    assert f(limit=0) == binding.FA_ERR_INVALID_ARG
    assert f(limit=(1 << 32) + 1) == binding.FA_ERR_INVALID_ARG
    assert f(Nk=0) == binding.FA_ERR_INVALID_ARG
    assert f(B=0) == binding.FA_ERR_INVALID_ARG


def test_selftest_bwd_timeout_argument_errors(lib):
    f = lambda **kw: binding.fa_selftest_bwd_timeout(
        P, P, P, P, P, P, P, P, P, kw.get("B", 1), 2, kw.get("Nq", 8), kw.get("Nk", 8), 64, 0.125, 1,
        P, 1 << 20, kw.get("limit", 2), stream=0)
    assert f(limit=0) == binding.FA_ERR_INVALID_ARG
    assert f(limit=(1 << 32) + 1) == binding.FA_ERR_INVALID_ARG
    assert f(Nk=0) == binding.FA_ERR_INVALID_ARG
    assert f(Nq=0) == binding.FA_ERR_INVALID_ARG
    assert f(B=0) == binding.FA_ERR_INVALID_ARG


# ---------------------------------------------------------------- packed variable-length entry point

def varlen_call(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, cu_q=P, cu_k=P, B=2, H=2, Tq=100, Tk=100, maxq=64, d=64,
             scale=0.125, causal=1)
    a.update(kw)
    return binding.fa_fwd_varlen(a["q"], a["k"], a["v"], a["o"], a["lse"], a["cu_q"], a["cu_k"],
                                 a["B"], a["H"], a["Tq"], a["Tk"], a["maxq"], a["d"], a["scale"],
                                 a["causal"], stream=0, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(cu_q=None), binding.FA_ERR_INVALID_ARG),
    (dict(cu_k=None), binding.FA_ERR_INVALID_ARG),
    (dict(cu_q=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(q=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(Tq=-1), binding.FA_ERR_INVALID_ARG),
    (dict(maxq=-1), binding.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(k=None), binding.FA_ERR_INVALID_ARG),
    (dict(Tq=0), binding.FA_OK),
    (dict(maxq=0), binding.FA_OK),
    (dict(B=0, q=None, cu_q=None), binding.FA_OK),
])
def test_varlen_argument_errors_before_any_cuda_call(lib, kw, code):
    assert varlen_call(**kw) == code


def test_varlen_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert varlen_call() == binding.FA_ERR_NO_DEVICE


# ---------------------------------------------------------------- E4M3 entry point

def fp8_call(**kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, B=1, H=2, Nq=8, Nk=8, d=128, scale=0.088, qd=0.01,
             kd=0.02, vd=0.005, causal=1, key_lens=None)
    a.update(kw)
    return binding.fa_fwd_fp8(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["Nq"],
                              a["Nk"], a["d"], a["scale"], a["qd"], a["kd"], a["vd"], a["causal"],
                              a["key_lens"], stream=0, check=False)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(d=32), binding.FA_ERR_UNSUPPORTED),
    (dict(qd=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(kd=-1.0), binding.FA_ERR_INVALID_ARG),
    (dict(vd=float("nan")), binding.FA_ERR_INVALID_ARG),
    (dict(vd=float("inf")), binding.FA_ERR_INVALID_ARG),
    (dict(qd=1e-30, kd=1e-30), binding.FA_ERR_INVALID_ARG),   # scale * qd * kd is 0 in fp32
    (dict(qd=1e30, kd=1e30), binding.FA_ERR_INVALID_ARG),     # ... or inf
    (dict(scale=-1.0), binding.FA_ERR_INVALID_ARG),
    (dict(q=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(v=P + 4), binding.FA_ERR_MISALIGNED),
    (dict(o=None), binding.FA_ERR_INVALID_ARG),
    (dict(B=0), binding.FA_OK),
    (dict(Nq=0, d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(Nq=0, d=64), binding.FA_OK),
])
def test_fp8_argument_errors_before_any_cuda_call(lib, kw, code):
    assert fp8_call(**kw) == code


def test_fp8_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert fp8_call() == binding.FA_ERR_NO_DEVICE
    assert fp8_call(d=64) == binding.FA_ERR_NO_DEVICE


# ---------------------------------------------------------------- backward entry point

def bwd_call(ws_bytes=None, **kw):
    a = dict(q=P, k=P, v=P, o=P, lse=P, do=P, dq=P, dk=P, dv=P, B=1, H=2, Nq=8, Nk=8, d=64,
             scale=0.125, causal=1, key_lens=None, ws=P)
    a.update(kw)
    need = binding.fa_bwd_workspace_size(a["B"], a["H"], a["Nq"], a["d"])
    return binding.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["do"], a["dq"], a["dk"], a["dv"],
                          a["B"], a["H"], a["Nq"], a["Nk"], a["d"], a["scale"], a["causal"],
                          a["key_lens"], a["ws"], need if ws_bytes is None else ws_bytes, stream=0,
                          check=False)


def test_bwd_workspace_size(lib):
    # D [B,H,N_q] fp32 then the fp32 dQ accumulator, each rounded up to 256 bytes
    assert binding.fa_bwd_workspace_size(2, 3, 100, 64) == 2560 + 153600
    assert binding.fa_bwd_workspace_size(1, 1, 1, 128) == 256 + 512
    assert binding.fa_bwd_workspace_size(1, 1, 1, 96) == 0
    assert binding.fa_bwd_workspace_size(-1, 1, 1, 64) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), binding.FA_ERR_UNSUPPORTED),
    (dict(scale=0.0), binding.FA_ERR_INVALID_ARG),
    (dict(B=-1), binding.FA_ERR_INVALID_ARG),
    (dict(do=None), binding.FA_ERR_INVALID_ARG),
    (dict(dq=None), binding.FA_ERR_INVALID_ARG),
    (dict(dk=None), binding.FA_ERR_INVALID_ARG),
    (dict(dv=None), binding.FA_ERR_INVALID_ARG),
    (dict(ws=None), binding.FA_ERR_INVALID_ARG),
    (dict(ws_bytes=16), binding.FA_ERR_INVALID_ARG),
    (dict(ws=P + 128), binding.FA_ERR_MISALIGNED),
    (dict(do=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(dk=P + 2), binding.FA_ERR_MISALIGNED),
    (dict(q=P + 8), binding.FA_ERR_MISALIGNED),
    (dict(B=0, q=None, do=None), binding.FA_OK),
    (dict(Nq=0, q=None, o=None, lse=None, do=None, dq=None, dk=None), binding.FA_ERR_INVALID_ARG),
])
def test_bwd_argument_errors_before_any_cuda_call(lib, kw, code):
    assert bwd_call(**kw) == code


def test_bwd_without_a_gpu_reports_no_device(lib):
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert bwd_call() == binding.FA_ERR_NO_DEVICE
