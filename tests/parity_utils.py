"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerance for attention outputs (bf16) against the fp64 oracle: max-abs error
<= 1e-2 and relative Frobenius error <= 2e-3 (the bound stated for the
benchmark workloads, whose near-uniform softmax gives |out| ~ 0.02). Derivation: rounding the output
to bf16 alone gives a relative error of about 2^-8/sqrt(12) / E|m| ~ 1.5e-3
(m the mantissa); the fp16 probabilities add about 1e-4; query values survive
their power-of-two-scaled fp16 conversion exactly and the dequantised keys are
exact in fp16; fp32 accumulation of 2048 terms adds ~1e-6. Indices and scores
of integer-valued indexer inputs are exact, so they must match bit for bit.
"""
import numpy as np
import torch

ATTN_MAX_ABS = 1e-2
ATTN_REL_FROB = 2e-3
LSE_ABS = 2e-3


def dev(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def bf16_dev(bits, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def host(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def row_vmax(values, idx):
    """Largest |v| over the entries each (b, t) row selected: values [B][N][D]
    (dequantised, e.g. by the oracle), idx [B][Tq][K] with -1 padding ->
    [B][Tq][1][1] (0 for a row with nothing selected)."""
    B, Tq, _ = idx.shape
    vmax = np.zeros((B, Tq, 1, 1), np.float64)
    amax = np.abs(np.asarray(values, np.float64)).max(axis=2)          # [B][N]
    for b in range(B):
        for t in range(Tq):
            sel = idx[b, t][idx[b, t] >= 0]
            vmax[b, t] = amax[b, sel].max() if sel.size else 0.0
    return vmax


def assert_attn_close(got, want, what="", sharp=False, vmax=None):
    """Benchmark tolerance, or with sharp=True an element-wise bound derived
    from the arithmetic, for softmax scales far above the workloads' and value
    magnitudes like the pages' (|out| of several units, where rounding to bf16
    alone exceeds 1e-2). The returned value is the bf16 rounding of an fp32
    result x' of the exact x: |rn(x') - x| <= ulp(|x| + e) / 2 + e, where e
    bounds |x' - x|. With vmax the largest |v| of the row's selected entries:
    the probabilities enter P V rounded to fp16 (relative 2^-11 each, moving
    sum_k p_k v_k / sum_k p_k by at most 2^-11 vmax); split partials merged
    inside a cluster are rounded to fp16 (at most 2^-11 vmax more); fp32
    accumulation and the hardware exp2 (relative 2^-22) add less than
    2^-16 vmax. So e = 2^-9 vmax leaves a factor of almost two. The relative
    Frobenius bound is kept."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), what
    err = got - want
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / den if den > 0 else float(np.linalg.norm(err))
    if sharp:
        assert vmax is not None, "the sharp bound needs the rows' largest |v|"
        e = 2.0 ** -9 * np.broadcast_to(np.asarray(vmax, np.float64), want.shape)
        bound = 0.5 * bf16_ulp(np.abs(want) + e) + e
        worst = float(np.max(np.abs(err) - bound)) if err.size else -1.0
        assert worst <= 0.0, "%s exceeds the derived bound by %.3e (max-abs %.3e)" % (
            what, worst, max_abs)
    else:
        assert max_abs <= ATTN_MAX_ABS, "%s max-abs %.3e" % (what, max_abs)
    assert rel <= ATTN_REL_FROB, "%s rel-Frobenius %.3e" % (what, rel)
    return max_abs, rel


def assert_lse_close(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    inf = np.isinf(want)
    assert np.array_equal(np.isinf(got), inf), what
    if np.any(~inf):
        np.testing.assert_allclose(got[~inf], want[~inf], rtol=0, atol=LSE_ABS, err_msg=what)
