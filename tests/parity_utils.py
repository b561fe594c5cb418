"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerance for attention outputs (bf16) against the fp64 oracle: max-abs error
<= 1e-2 and relative Frobenius error <= 2e-3. Derivation: rounding the output
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


def assert_attn_close(got, want, what=""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), what
    err = got - want
    max_abs = float(np.max(np.abs(err))) if err.size else 0.0
    den = float(np.linalg.norm(want))
    rel = float(np.linalg.norm(err)) / den if den > 0 else float(np.linalg.norm(err))
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
