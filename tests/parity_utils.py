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


def assert_attn_close(got, want, what="", sharp=False):
    """Benchmark tolerance. With sharp=True (softmax scales far above the
    workloads', where outputs reach |out| of several units and rounding to bf16
    alone can exceed 1e-2) every element must instead lie within one bf16 ulp
    of the fp64 reference, plus 1e-3; the relative Frobenius bound is kept."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), what
    err = got - want
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / den if den > 0 else float(np.linalg.norm(err))
    if sharp:
        bound = bf16_ulp(want) + 1e-3
        worst = float(np.max(np.abs(err) - bound)) if err.size else -1.0
        assert worst <= 0.0, "%s exceeds one bf16 ulp by %.3e (max-abs %.3e)" % (what, worst, max_abs)
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
