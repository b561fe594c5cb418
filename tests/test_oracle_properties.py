"""Property-based pins for the oracle (no GPU): hypothesis draws shapes,
values and tie patterns, and each property is checked against a brute force
written here (nearest grid point by exhaustive search, block ranking by
Python's sort) or against torch's own float8 cast."""
import math

import numpy as np
import torch
from hypothesis import given, settings, strategies as st

import oracle

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _e4m3_value(b):
    return float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)[0])


@settings(max_examples=40, deadline=None)
@given(groups=st.integers(1, 4), seed=st.integers(0, 2**31 - 1),
       spread=st.sampled_from([1e-3, 1.0, 30.0, 5000.0]))
def test_g16_row_is_the_nearest_grid_point_at_the_torch_scale(oracle_lib, groups, seed, spread):
    D = 16 * groups * 2                          # an even number of groups keeps D/2 whole
    rng = np.random.default_rng(seed)
    kv = (rng.standard_normal((1, 1, D)) * spread).astype(np.float32)
    rows = oracle.fp4_kv_pack_g16(kv)
    for g in range(D // 16):
        x = kv[0, 0, 16 * g:16 * g + 16].astype(np.float64)
        sc = rows[0, 0, D // 2 + g]
        want_sc = torch.tensor([min(np.abs(x).max() / 6.0, 448.0)], dtype=torch.float32).to(
            torch.float8_e4m3fn).view(torch.uint8).item()
        assert sc == want_sc
        s = _e4m3_value(sc)
        for i, xv in enumerate(x):
            c = 16 * g + i
            nib = (rows[0, 0, c // 2] >> (4 * (c % 2))) & 0xF
            if s == 0.0:
                assert nib == 0
                continue
            d = np.abs(abs(xv) - GRID * s)
            best = [k for k in range(8) if d[k] == d.min()]
            code = best[0] if len(best) == 1 else [k for k in best if k % 2 == 0][0]
            assert nib & 7 == code
            if code:
                assert (nib >> 3) == (1 if math.copysign(1.0, xv) < 0 else 0)


@settings(max_examples=60, deadline=None)
@given(ld=st.integers(1, 90), block=st.integers(1, 9), nblocks=st.integers(1, 12),
       levels=st.integers(1, 5), seed=st.integers(0, 2**31 - 1), data=st.data())
def test_block_pool_is_the_brute_force_ranking(oracle_lib, ld, block, nblocks, levels, seed, data):
    rng = np.random.default_rng(seed)
    scores = rng.integers(0, levels, ld).astype(np.float64)   # few levels: many ties
    nv = data.draw(st.integers(0, ld))
    got = oracle.block_pool(scores[None, :], np.array([nv], np.int32), block, nblocks)[0]
    nb = -(-nv // block)
    bmax = [max(scores[j] for j in range(b * block, min(b * block + block, nv))) for b in range(nb)]
    kept = sorted(sorted(range(nb), key=lambda b: (-bmax[b], b))[:nblocks])
    want = [j for b in kept for j in range(b * block, min(b * block + block, nv))]
    want += [-1] * (nblocks * block - len(want))
    assert list(got) == want


@settings(max_examples=30, deadline=None)
@given(n=st.integers(0, 40), W=st.integers(0, 50), seed=st.integers(0, 2**31 - 1))
def test_swa_window_bounds(oracle_lib, n, W, seed):
    """The union with an empty selection attends exactly the tokens
    [max(0, n - W), n): checked by moving every other token far away."""
    rng = np.random.default_rng(seed)
    D, Tw = 32, 40
    packed, sc = oracle.fp4_kv_pack(rng.standard_normal((1, 64, D)).astype(np.float32))
    q = torch.from_numpy(rng.standard_normal((1, 1, 1, D)).astype(np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    win = np.zeros((1, Tw, D), np.float32)
    win[0, :, 0] = np.arange(Tw)                  # value channel 0 = the token's position
    wbytes = torch.from_numpy(win).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    idx = np.full((1, 1, 4), -1, np.int32)
    out, lse = oracle.swa_sparse_attn(q, packed, sc, idx, wbytes, np.array([[n]], np.int32),
                                      0.0, W=W)   # scale 0: the mean of the attended tokens
    lo = max(0, n - W)
    if n - lo == 0:
        assert out[0, 0, 0, 0] == 0.0 and np.isneginf(lse[0, 0, 0])
    else:
        pos = torch.from_numpy(np.arange(lo, n, dtype=np.float32)).to(torch.float8_e4m3fn).to(
            torch.float64).numpy()
        assert abs(out[0, 0, 0, 0] - pos.mean()) < 1e-9
        assert abs(lse[0, 0, 0] - math.log(n - lo)) < 1e-12
