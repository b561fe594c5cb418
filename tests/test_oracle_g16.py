"""Pins for the oracle's FP4 layout with one E4M3 scale per 16 channels of an
entry (no GPU). The 16-channel grouping and the absence of a global scale are
the pages' ("FP4 Main KV Cache To Halve Storage Again"; the mengman.github.io
interpretation, 3.5); the scale rule max|x|/6 and the row layout (codes, then
scales) are the readings shared with the block layout. Each test checks the
oracle against something other than itself: torch's float8_e4m3fn cast and a
brute-force nearest-grid search, closed forms, the format's error bound, the
row independence the layout implies, the already-pinned block layout on data
where both layouts must agree, and numpy softmax attention."""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")
GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _e4m3_bytes(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def _e4m3_values(b):
    return torch.from_numpy(np.asarray(b, np.uint8)).view(torch.float8_e4m3fn).to(
        torch.float64).numpy()


def _split(rows, D):
    codes = rows[..., :D // 2]
    scales = rows[..., D // 2:]
    return codes, scales


def test_group_size_is_the_pages(oracle_lib):
    with open(GOLDEN) as f:
        facts = json.load(f)
    assert oracle.GROUP_CHANNELS == facts["scale_group_channels"]["value"]
    assert oracle.g16_row_bytes(512) == 288          # 256 code bytes + 32 scale bytes


def test_pack_matches_torch_scales_and_brute_force_codes(oracle_lib):
    rng = np.random.default_rng(21)
    B, N, D = 2, 5, 64
    kv = (rng.standard_normal((B, N, D)) * 3.0).astype(np.float32)
    kv[0, 1, 16:32] = 0.0                        # an all-zero group
    kv[1, 2, 0:16] *= np.float32(1e-4)           # a tiny group: scale near E4M3's bottom
    kv[1, 4, 48:64] *= np.float32(500.0)         # a huge group: the scale saturates
    rows = oracle.fp4_kv_pack_g16(kv)
    codes, scales = _split(rows, D)
    amax = np.abs(kv.reshape(B, N, D // 16, 16)).max(axis=-1)
    # torch's cast turns values above 448 into NaN; the format reading saturates
    assert np.array_equal(scales, _e4m3_bytes(np.minimum(amax / np.float32(6.0), 448.0)))
    s = np.repeat(_e4m3_values(scales), 16, axis=-1)
    want = np.zeros((B, N, D), np.uint8)
    for idx in np.ndindex(B, N, D):
        a = abs(float(kv[idx]))
        if s[idx] == 0.0:
            continue
        d = np.abs(a - GRID * s[idx])
        best = np.flatnonzero(d == d.min())
        c = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        want[idx] = c | (8 if math.copysign(1.0, float(kv[idx])) < 0 else 0)
    assert np.array_equal(codes, (want[..., 0::2] | (want[..., 1::2] << 4)).astype(np.uint8))


def test_scale_closed_forms(oracle_lib):
    D = 64
    kv = np.zeros((1, 1, D), np.float32)
    kv[0, 0, 0:16] = np.linspace(-6.0, 6.0, 16)  # max 6 -> scale 1.0 (E4M3 0x38)
    kv[0, 0, 32:48] = 1e6                        # max 1e6 -> scale saturates at 448 (0x7E)
    kv[0, 0, 48] = 0.5625                        # max 0.5625 -> scale 0.09375 = 1.5 * 2^-4 (0x1C)
    rows = oracle.fp4_kv_pack_g16(kv)
    _, scales = _split(rows, D)
    assert list(scales[0, 0]) == [0x38, 0x00, 0x7E, 0x1C]
    back = oracle.fp4_kv_unpack_g16(rows, D)
    assert back[0, 0, 0] == -6.0 and back[0, 0, 15] == 6.0
    assert np.all(back[0, 0, 16:32] == 0.0)      # zero group: zero scale, zero codes
    assert np.all(back[0, 0, 32:48] == 6.0 * 448.0)   # saturated codes and scale
    assert back[0, 0, 48] == 6.0 * 0.09375


def test_grid_values_round_trip_exactly(oracle_lib):
    rng = np.random.default_rng(22)
    B, N, D = 2, 7, 128
    s_choice = _e4m3_values(np.array([0x20, 0x2C, 0x38, 0x41, 0x55], np.uint8))
    s = s_choice[rng.integers(0, len(s_choice), (B, N, D // 16))]
    vals = GRID[rng.integers(0, 8, (B, N, D))] * np.where(rng.random((B, N, D)) < 0.5, -1, 1)
    vals = vals.reshape(B, N, D // 16, 16)
    vals[..., 3] = 6.0                           # every group's maximum is 6 s
    kv = (vals * s[..., None]).reshape(B, N, D).astype(np.float32)
    rows = oracle.fp4_kv_pack_g16(kv)
    assert np.array_equal(oracle.fp4_kv_unpack_g16(rows, D), kv.astype(np.float64))


def test_error_within_one_scale_step(oracle_lib):
    rng = np.random.default_rng(23)
    B, N, D = 3, 16, 512
    kv = rng.standard_normal((B, N, D)).astype(np.float32)
    rows = oracle.fp4_kv_pack_g16(kv)
    back = oracle.fp4_kv_unpack_g16(rows, D)
    _, scales = _split(rows, D)
    s = np.repeat(_e4m3_values(scales), 16, axis=-1)
    err = np.abs(back - kv.astype(np.float64))
    # nearest point of a grid whose widest step is 2 (between 4 and 6), and a
    # group maximum that may sit up to 6.4 s after the scale is rounded down
    assert np.all(err <= s + 1e-12)
    small = np.abs(kv) < 0.25 * s
    assert np.all(back[small] == 0.0)
    assert np.all(np.sign(back[back != 0]) == np.sign(kv[back != 0]))


def test_append_equals_pack_and_touches_only_its_rows(oracle_lib):
    rng = np.random.default_rng(24)
    B, N, D, T = 2, 40, 64, 3
    kv = rng.standard_normal((B, N, D)).astype(np.float32)
    full = oracle.fp4_kv_pack_g16(kv)
    pos = np.array([[0, 17, 39], [5, 6, 38]], np.int32)
    base = kv.copy()
    for b in range(B):
        base[b, pos[b]] = 0.0
    cache = oracle.fp4_kv_pack_g16(base)
    new = np.stack([kv[b, pos[b]] for b in range(B)])
    appended = oracle.fp4_kv_append_g16(cache, new, pos)
    assert np.array_equal(appended, full)
    untouched = np.ones((B, N), bool)
    for b in range(B):
        untouched[b, pos[b]] = False
    assert np.array_equal(appended[untouched], cache[untouched])
    with pytest.raises(oracle.OracleError):
        oracle.fp4_kv_append_g16(cache, new, np.array([[0, 1, N], [0, 1, 2]], np.int32))


def test_nonfinite_is_an_error(oracle_lib):
    kv = np.zeros((1, 2, 32), np.float32)
    kv[0, 1, 20] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.fp4_kv_pack_g16(kv)


def _agreeing_cache(seed, B, N, D, s_code=0x30):
    """Values on the E2M1 grid times one scale s, with +-6 s placed so that every
    16-channel group of every entry and every 64-entry block of every channel
    holds it: both layouts then store the scale s everywhere and the same codes."""
    rng = np.random.default_rng(seed)
    s = float(_e4m3_values(np.array([s_code], np.uint8))[0])
    vals = GRID[rng.integers(0, 8, (B, N, D))] * np.where(rng.random((B, N, D)) < 0.5, -1, 1)
    n = np.arange(N)[:, None]
    c = np.arange(D)[None, :]
    vals[:, (n + c) % 16 == 0] = 6.0
    return (vals * s).astype(np.float32)


def test_agrees_with_block_layout_where_scales_agree(oracle_lib):
    B, Tq, Hq, N, D, K = 2, 1, 3, 128, 64, 40
    kv = _agreeing_cache(25, B, N, D)
    rows = oracle.fp4_kv_pack_g16(kv)
    packed, sc = oracle.fp4_kv_pack(kv)
    codes, scales = _split(rows, D)
    assert np.array_equal(codes, packed)
    assert np.all(scales == 0x30) and np.all(sc == 0x30)
    assert np.array_equal(oracle.fp4_kv_unpack_g16(rows, D), oracle.fp4_kv_unpack(packed, sc))
    rng = np.random.default_rng(26)
    q = torch.from_numpy(rng.standard_normal((B, Tq, Hq, D)).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    idx = np.full((B, Tq, K), -1, np.int32)
    idx[0, 0, :30] = np.sort(rng.choice(N, 30, replace=False))
    idx[1, 0, :] = rng.choice(N, K, replace=False)
    for scale in (0.125, 1.0):
        a, la = oracle.sparse_attn_g16(q, rows, idx, scale)
        b, lb = oracle.sparse_attn(q, packed, sc, idx, scale)
        assert np.array_equal(a, b) and np.array_equal(la, lb)


@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 1.0])
def test_full_selection_matches_numpy_softmax(oracle_lib, scale):
    rng = np.random.default_rng(27)
    B, Tq, Hq, N, D = 2, 2, 3, 48, 64
    kv = rng.standard_normal((B, N, D)).astype(np.float32)
    rows = oracle.fp4_kv_pack_g16(kv)
    V = oracle.fp4_kv_unpack_g16(rows, D)
    qf32 = (rng.standard_normal((B, Tq, Hq, D)) / math.sqrt(512.0)).astype(np.float32)
    qb = torch.from_numpy(qf32).to(torch.bfloat16)
    qbits = qb.view(torch.int16).numpy().view(np.uint16)
    qf = qb.to(torch.float64).numpy()
    idx = np.full((B, Tq, N + 5), -1, np.int32)
    idx[:, :, :N] = rng.permutation(N)
    out, lse = oracle.sparse_attn_g16(qbits, rows, idx, scale)
    for b in range(B):
        for t in range(Tq):
            logits = scale * qf[b, t] @ V[b].T
            np.testing.assert_allclose(out[b, t], scipy.special.softmax(logits, -1) @ V[b],
                                       rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(lse[b, t], scipy.special.logsumexp(logits, -1),
                                       rtol=1e-13)
    idx[0, 0, :] = -1                            # nothing selected: zeros, lse -inf
    out, lse = oracle.sparse_attn_g16(qbits, rows, idx, scale)
    assert np.all(out[0, 0] == 0.0) and np.all(np.isneginf(lse[0, 0]))
