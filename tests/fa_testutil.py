"""Helpers shared by the GPU tests: upload seeded bf16 bits, run the library, compare with the oracle."""
import numpy as np

from io_aware_exact_24_b200.inputs import bf16_bits_to_f32

# The parity bar for bf16 outputs against the fp64 oracle.
TOL_MAX_ABS_O = 1.5e-2
TOL_REL_FROB_O = 4e-3
TOL_ABS_LSE = 1e-3


def to_device_bf16(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(device).view(torch.bfloat16)


def to_host_f64(t):
    import torch
    bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return bf16_bits_to_f32(bits).astype(np.float64)


def run_fa(q, k, v, scale, causal=False, key_lens=None, *, o_guard=0, out=None):
    """Run fa_fwd on bf16 bit arrays.  Returns (O f64, LSE f32 as f64) as numpy arrays.

    With o_guard > 0, O and LSE are carved out of larger buffers whose guard
    regions hold a sentinel; the returned dict-free tuple is extended with a
    flag telling whether every guard survived.
    """
    import torch
    from io_aware_exact_24_b200 import fa_fwd
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    tq, tk, tv = to_device_bf16(q), to_device_bf16(k), to_device_bf16(v)
    tkl = None if key_lens is None else torch.from_numpy(np.asarray(key_lens, np.int32)).cuda()
    n_o, n_l = B * H * Nq * d, B * H * Nq
    g = int(o_guard)
    o_buf = torch.full((n_o + 2 * g,), -12345.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 2 * g,), -777.0, dtype=torch.float32, device="cuda")
    o = o_buf[g:g + n_o].view(B, H, Nq, d)
    lse = l_buf[g:g + n_l].view(B, H, Nq)
    fa_fwd(tq, tk if Nk else None, tv if Nk else None, o, lse, B, H, Nq, Nk, d, scale, causal,
           tkl)
    torch.cuda.synchronize()
    guards_ok = True
    if g:
        guards_ok = bool((o_buf[:g] == -12345.0).all() and (o_buf[g + n_o:] == -12345.0).all()
                         and (l_buf[:g] == -777.0).all() and (l_buf[g + n_l:] == -777.0).all())
    res = (to_host_f64(o), lse.cpu().numpy().astype(np.float64))
    if out is not None:
        out["o_bits"] = o.view(torch.int16).cpu().numpy()
        out["lse_raw"] = lse.cpu().numpy()
        out["guards_ok"] = guards_ok
    return res


def compare(o, lse, o_ref, lse_ref, what=""):
    """Assert the parity bar; returns the three error figures."""
    assert not np.isnan(o).any(), f"{what}: NaN in O"
    assert not np.isnan(lse).any(), f"{what}: NaN in LSE"
    masked = np.isneginf(lse_ref)
    # fully masked rows: exactly O = +0.0 and LSE = -inf
    assert np.all(np.isneginf(lse[masked])), f"{what}: masked rows must give LSE=-inf"
    om = o[masked]
    assert np.all(om == 0) and not np.signbit(om).any(), f"{what}: masked rows must give O=+0"
    assert np.all(np.isfinite(lse[~masked])), f"{what}: unexpected non-finite LSE"
    err = np.abs(o - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o - o_ref) / denom) if denom > 0 else float(np.linalg.norm(o))
    lse_err = float(np.abs(lse[~masked] - lse_ref[~masked]).max()) if (~masked).any() else 0.0
    assert max_abs <= TOL_MAX_ABS_O, f"{what}: max|dO| {max_abs:.3e}"
    assert rel <= TOL_REL_FROB_O, f"{what}: rel Frobenius {rel:.3e}"
    assert lse_err <= TOL_ABS_LSE, f"{what}: max|dLSE| {lse_err:.3e}"
    return max_abs, rel, lse_err
