"""Pins for the CPU oracle (no GPU). Each test checks the oracle against
something other than itself: a value the pages print, a library routine that
implements the same format (torch's float8_e4m3fn), a closed form, brute
force on tiny inputs, or an invariant the method fixes (mode semantics,
sparse = dense at K = N)."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from fp4_kv_cache_step_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


@pytest.fixture(scope="module")
def facts():
    with open(GOLDEN) as f:
        return json.load(f)


# ----------------------------------------------------------------- formats
def test_e2m1_grid_matches_mx_table(oracle_lib, facts):
    grid = facts["e2m1_grid"]["value"]
    for code in range(8):
        assert oracle.e2m1_value(code) == grid[code]
        neg = oracle.e2m1_value(code | 8)
        assert neg == -grid[code] and math.copysign(1.0, neg) == -1.0


@pytest.mark.parametrize("scale_code", [0x01, 0x08, 0x30, 0x38, 0x3F, 0x55, 0x7E])
def test_e2m1_grid_round_trips_exactly(oracle_lib, scale_code):
    s = oracle.e4m3_value(scale_code)
    for code in range(16):
        x = oracle.e2m1_value(code) * s
        assert oracle.e2m1_code(x, s) == code


def test_e2m1_midpoints_go_to_even_code(oracle_lib, facts):
    grid = facts["e2m1_grid"]["value"]
    s = oracle.e4m3_value(0x3A)  # 1.25
    for c in range(7):
        mid = 0.5 * (grid[c] + grid[c + 1]) * s
        even = c if c % 2 == 0 else c + 1
        assert oracle.e2m1_code(mid, s) == even
        assert oracle.e2m1_code(-mid, s) == (even | 8)
        # just either side of the midpoint picks the nearer code
        assert oracle.e2m1_code(np.nextafter(mid, 0.0), s) == c
        assert oracle.e2m1_code(np.nextafter(mid, np.inf), s) == c + 1


def test_e2m1_saturates_at_six(oracle_lib):
    s = 2.0
    assert oracle.e2m1_code(6 * s * 1.5, s) == 7
    assert oracle.e2m1_code(-1e30, s) == 15
    assert oracle.e2m1_code(5.0 * s, s) == 6      # midpoint of 4 and 6 -> even (4)
    assert oracle.e2m1_code(5.0 * s + 1e-9, s) == 7


def test_e4m3_decode_matches_torch_float8(oracle_lib):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan_ref = np.isnan(ref)
    assert np.array_equal(nan_ref, np.isnan(mine))
    assert set(np.flatnonzero(nan_ref)) == {0x7F, 0xFF}
    assert np.array_equal(ref[~nan_ref], mine[~nan_ref])
    # signed zero survives
    assert math.copysign(1.0, oracle.e4m3_value(0x80)) == -1.0


def test_e4m3_encode_matches_torch_round_to_nearest_even(oracle_lib, facts):
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])   # 0 .. 448
    assert vals[-1] == facts["e4m3_max"]["value"]
    mids = 0.5 * (vals[:-1] + vals[1:])
    rng = np.random.default_rng(7)
    sweep = np.concatenate([
        vals, mids, np.nextafter(mids, 0), np.nextafter(mids, np.inf),
        rng.uniform(0, 448, 4000), np.exp(rng.uniform(-14, 6, 4000)),
    ]).astype(np.float32)
    sweep = np.concatenate([sweep, -sweep])
    ref = torch.from_numpy(sweep).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_from_double(float(x)) for x in sweep], np.uint8)
    assert np.array_equal(ref, mine)


def test_e4m3_encode_saturates(oracle_lib, facts):
    top = 0x7E
    for x in (448.0, 449.0, 464.0, 470.0, 1e6, float("inf")):
        assert oracle.e4m3_from_double(x) == top
        assert oracle.e4m3_from_double(-x) == (top | 0x80)
    # the largest main-KV value the format can hold ("thousands")
    assert oracle.e2m1_value(7) * oracle.e4m3_value(top) == facts["fp4_max_representable"]["value"]


def test_bf16_decode(oracle_lib):
    x = np.float32([0.0, -0.0, 1.0, -2.5, 3.140625, 1e-30, 6.5e4])
    bits = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    for b, r in zip(bits, ref):
        assert oracle.bf16_value(int(b)) == r


# ----------------------------------------------------------------- FP4 pack
def _brute_codes(x, s):
    """Nearest E2M1 grid point of |x|/s by exhaustive distance, ties to even."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    out = np.zeros(x.shape, np.uint8)
    for idx in np.ndindex(x.shape):
        a = abs(float(x[idx]))
        if s[idx] == 0.0:
            out[idx] = 0
            continue
        d = np.abs(a - grid * s[idx])
        best = np.flatnonzero(d == d.min())
        code = best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]
        out[idx] = code | (8 if math.copysign(1.0, float(x[idx])) < 0 else 0)
    return out


def test_pack_matches_brute_force_on_small_blocks(oracle_lib):
    rng = np.random.default_rng(3)
    B, N, D = 2, 128, 16
    kv = rng.standard_normal((B, N, D)).astype(np.float32) * np.float32(3.0)
    kv[0, :64, 3] = 0.0                          # an all-zero channel block
    kv[1, 64:, 5] *= np.float32(1e-4)            # tiny block: scale near E4M3's bottom
    packed, scale = oracle.fp4_kv_pack(kv)
    # scales = RNE_e4m3(blockmax / 6), computed with torch's own cast
    amax = np.abs(kv.reshape(B, N // 64, 64, D)).max(axis=2)
    ref_scale = torch.from_numpy((amax / np.float32(6.0)).astype(np.float32)).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(scale, ref_scale)
    s = np.repeat(torch.from_numpy(ref_scale).view(torch.float8_e4m3fn).to(torch.float64).numpy(),
                  64, axis=1)
    codes = _brute_codes(kv, s)
    ref_packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    assert np.array_equal(packed, ref_packed)


def test_pack_grid_values_round_trip(oracle_lib):
    rng = np.random.default_rng(4)
    B, N, D = 1, 64, 32
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    s = np.float32(0.375)                        # exactly E4M3 (0x2C... any E4M3 value)
    vals = grid[rng.integers(0, 8, (B, N, D))] * np.where(rng.random((B, N, D)) < 0.5, -1, 1)
    vals[0, 0, :] = 6.0                          # amax = 6 s in every channel
    kv = (vals * s).astype(np.float32)
    packed, scale = oracle.fp4_kv_pack(kv)
    assert np.all(scale == torch.tensor([0.375]).to(torch.float8_e4m3fn).view(torch.uint8).item())
    back = oracle.fp4_kv_unpack(packed, scale)
    assert np.array_equal(back, kv.astype(np.float64))


def test_pack_nonfinite_is_an_error(oracle_lib):
    kv = np.zeros((1, 64, 4), np.float32)
    kv[0, 5, 2] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.fp4_kv_pack(kv)


def test_unpack_layout_low_nibble_is_even_channel(oracle_lib):
    packed = np.zeros((1, 64, 2), np.uint8)
    scale = np.zeros((1, 1, 4), np.uint8)
    scale[0, 0, :] = 0x38                        # 1.0
    packed[0, 0, 0] = 0x2 | (0x7 << 4)           # ch0 = 1.0, ch1 = 6.0
    packed[0, 1, 1] = 0xB | (0x1 << 4)           # ch2 = -1.5, ch3 = 0.5
    out = oracle.fp4_kv_unpack(packed, scale)
    assert list(out[0, 0]) == [1.0, 6.0, 0.0, 0.0]
    assert list(out[0, 1]) == [0.0, 0.0, -1.5, 0.5]


# ----------------------------------------------------------------- indexer
def _e4m3(ints):
    return torch.from_numpy(np.asarray(ints, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def test_score_one_hot_queries_closed_form(oracle_lib):
    """q_h = 4 * e_{c_h}: the score is sum_h w_h * max(0, 4 * k[c_h])."""
    rng = np.random.default_rng(5)
    B, Tq, N, Hi, Di = 2, 2, 64, 4, 16
    chan = np.array([[[3, 0, 9, 15], [1, 1, 2, 7]], [[0, 5, 5, 12], [8, 4, 11, 2]]])
    qi = np.zeros((B, Tq, Hi, Di), np.float32)
    for b, t, h in itertools.product(range(B), range(Tq), range(Hi)):
        qi[b, t, h, chan[b, t, h]] = 4.0
    ki = rng.integers(-4, 5, (B, N, Di)).astype(np.float32)
    w = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    nv = np.array([[64, 40], [17, 64]], np.int32)
    got = oracle.index_score(_e4m3(qi), w, _e4m3(ki), nvalid=nv)
    for b, t in itertools.product(range(B), range(Tq)):
        for j in range(N):
            if j >= nv[b, t]:
                assert got[b, t, j] == -np.inf
                continue
            want = sum(w[b, t, h] * max(0.0, 4.0 * ki[b, j, chan[b, t, h]]) for h in range(Hi))
            assert got[b, t, j] == want


def test_score_exact_integer_and_head_symmetries(oracle_lib):
    rng = np.random.default_rng(6)
    B, Tq, N, Hi, Di = 1, 3, 128, 8, 32
    qi = rng.integers(-4, 5, (B, Tq, Hi, Di)).astype(np.float32)
    ki = rng.integers(-4, 5, (B, N, Di)).astype(np.float32)
    w = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    nv = np.full((B, Tq), N, np.int32)
    s = oracle.index_score(_e4m3(qi), w, _e4m3(ki), nvalid=nv)
    assert np.all(s == np.round(s)) and s.max() < 2 ** 24      # exact in fp32 too
    # permuting heads (queries and weights together) leaves scores unchanged
    perm = rng.permutation(Hi)
    s2 = oracle.index_score(_e4m3(qi[:, :, perm]), w[:, :, perm].copy(), _e4m3(ki), nvalid=nv)
    assert np.array_equal(s, s2)
    # doubling the weights doubles the scores; negating every query turns each
    # head's ReLU onto the other half-line: s(q) + s(-q) = sum_h w_h |q_h . k|
    s3 = oracle.index_score(_e4m3(qi), 2 * w, _e4m3(ki), nvalid=nv)
    assert np.array_equal(s3, 2 * s)
    s4 = oracle.index_score(_e4m3(-qi), w, _e4m3(ki), nvalid=nv)
    dots = np.einsum("bthc,bjc->bthj", qi.astype(np.int64), ki.astype(np.int64))
    absum = np.einsum("bth,bthj->btj", w.astype(np.int64), np.abs(dots))
    assert np.array_equal(s + s4, absum.astype(np.float64))


def test_score_pool_matches_full_scan(oracle_lib):
    rng = np.random.default_rng(8)
    B, Tq, N, Hi, Di, C = 2, 1, 256, 4, 32, 40
    qb = _e4m3(rng.integers(-4, 5, (B, Tq, Hi, Di)))
    kb = _e4m3(rng.integers(-4, 5, (B, N, Di)))
    w = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    full = oracle.index_score(qb, w, kb, nvalid=np.full((B, Tq), N, np.int32))
    cand = np.full((B, Tq, C), -1, np.int32)
    for b in range(B):
        ids = np.sort(rng.choice(N, 33, replace=False))
        cand[b, 0, :33] = ids
    pooled = oracle.index_score(qb, w, kb, cand=cand)
    for b in range(B):
        assert np.array_equal(pooled[b, 0, :33], full[b, 0, cand[b, 0, :33]])
        assert np.all(pooled[b, 0, 33:] == -np.inf)


# ----------------------------------------------------------------- top-K
def _brute_topk(scores, ids, K):
    order = sorted(range(len(ids)), key=lambda i: (-scores[i], ids[i]))
    sel = sorted(ids[i] for i in order[:K])
    return sel + [-1] * (K - len(sel))


def test_topk_equals_full_sort(oracle_lib):
    rng = np.random.default_rng(9)
    rows, N = 6, 3000
    scores = rng.integers(0, 400, (rows, N)).astype(np.float64)   # many ties
    nv = np.array([3000, 2999, 100, 64, 1, 0], np.int32)
    for K in (1, 7, 64, 256, 2999, 3000, 3100):
        got = oracle.topk(scores, K, nvalid=nv)
        for r in range(rows):
            assert list(got[r]) == _brute_topk(scores[r, :nv[r]], list(range(nv[r])), K)


def test_topk_exhaustive_ties_small(oracle_lib):
    for n in range(1, 7):
        for vals in itertools.product([0.0, 1.0, 2.0], repeat=n):
            sc = np.array([vals], np.float64)
            for K in range(1, n + 2):
                got = oracle.topk(sc, K, nvalid=np.array([n], np.int32))
                assert list(got[0]) == _brute_topk(list(vals), list(range(n)), K)


def test_topk_negative_zero_ties_with_zero(oracle_lib):
    sc = np.array([[0.0, -0.0, 0.0, -1.0]])
    got = oracle.topk(sc, 2, nvalid=np.array([4], np.int32))
    assert list(got[0]) == [0, 1]


def test_topk_is_prefix_of_topc_and_pool_reselects(oracle_lib):
    rng = np.random.default_rng(10)
    rows, N, K, C = 4, 5000, 100, 700
    scores = rng.integers(0, 800, (rows, N)).astype(np.float64)
    nv = np.full(rows, N, np.int32)
    tk = oracle.topk(scores, K, nvalid=nv)
    tc = oracle.topk(scores, C, nvalid=nv)
    for r in range(rows):
        assert set(tk[r]) <= set(tc[r])
        assert np.all(np.diff(tk[r]) > 0) and np.all(np.diff(tc[r]) > 0)
    # re-ranking the pool's own scores gives the same top-K
    pooled_scores = np.take_along_axis(scores, tc.astype(np.int64), axis=1)
    again = oracle.topk(pooled_scores, K, cand=tc)
    assert np.array_equal(again, tk)


def test_topk_nan_is_an_error(oracle_lib):
    sc = np.array([[1.0, np.nan, 2.0]])
    with pytest.raises(oracle.OracleError):
        oracle.topk(sc, 1, nvalid=np.array([3], np.int32))


# ----------------------------------------------------------------- attention
def _small_kv(seed, B, N, D):
    rng = np.random.default_rng(seed)
    kv = rng.standard_normal((B, N, D)).astype(np.float32)
    return oracle.fp4_kv_pack(kv)


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _bf16_f64(bits):
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 1.0])
def test_dense_and_full_sparse_match_numpy_softmax(oracle_lib, scale):
    B, Tq, Hq, N, D = 2, 2, 3, 128, 64
    packed, sc = _small_kv(11, B, N, D)
    rng = np.random.default_rng(12)
    qb = _bf16(rng.standard_normal((B, Tq, Hq, D)) / math.sqrt(512.0))
    V = oracle.fp4_kv_unpack(packed, sc)
    nv = np.array([[128, 77], [1, 128]], np.int32)
    dense, dlse = oracle.dense_attn(qb, packed, sc, nv, scale)
    idx = np.full((B, Tq, N), -1, np.int32)
    for b, t in itertools.product(range(B), range(Tq)):
        idx[b, t, :nv[b, t]] = np.arange(nv[b, t])
    sparse, slse = oracle.sparse_attn(qb, packed, sc, idx, scale)
    qf = _bf16_f64(qb)
    for b, t in itertools.product(range(B), range(Tq)):
        Vb = V[b, :nv[b, t]]
        logits = scale * qf[b, t] @ Vb.T
        ref = scipy.special.softmax(logits, axis=-1) @ Vb
        ref_lse = scipy.special.logsumexp(logits, axis=-1)
        np.testing.assert_allclose(dense[b, t], ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(sparse[b, t], ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(dlse[b, t], ref_lse, rtol=1e-13)
        np.testing.assert_allclose(slse[b, t], ref_lse, rtol=1e-13)


def test_attention_special_cases(oracle_lib):
    B, Tq, Hq, N, D = 1, 1, 4, 256, 32
    packed, sc = _small_kv(13, B, N, D)
    V = oracle.fp4_kv_unpack(packed, sc)
    rng = np.random.default_rng(14)
    qb = _bf16(rng.standard_normal((B, Tq, Hq, D)))
    # K = 1: the output is the selected row exactly, lse = its logit
    idx = np.array([[[37]]], np.int32)
    out, lse = oracle.sparse_attn(qb, packed, sc, idx, 0.3)
    for h in range(Hq):
        assert np.array_equal(out[0, 0, h], V[0, 37])
        assert lse[0, 0, h] == pytest.approx(0.3 * _bf16_f64(qb)[0, 0, h] @ V[0, 37], rel=1e-14)
    # scale 0: the mean of the selected rows, lse = log(count)
    sel = np.array([3, 9, 200, 201, 255], np.int32)
    idx = np.concatenate([sel, [-1, -1, -1]]).astype(np.int32)[None, None]
    out, lse = oracle.sparse_attn(qb, packed, sc, idx, 0.0)
    np.testing.assert_allclose(out[0, 0, 0], V[0, sel].mean(axis=0), rtol=1e-13, atol=1e-15)
    assert lse[0, 0, 0] == pytest.approx(math.log(5.0), rel=1e-14)
    # the order of the index list does not matter; -1 entries are skipped
    idx2 = np.array([[[255, -1, 3, 201, -1, 9, 200, -1]]], np.int32)
    out2, lse2 = oracle.sparse_attn(qb, packed, sc, idx2, 0.0)
    np.testing.assert_allclose(out2, out, rtol=1e-13, atol=1e-15)
    # nothing selected: zeros and lse = -inf
    out3, lse3 = oracle.sparse_attn(qb, packed, sc, np.full((1, 1, 4), -1, np.int32), 1.0)
    assert np.all(out3 == 0) and np.all(lse3 == -np.inf)
    # an index past N is an error
    with pytest.raises(oracle.OracleError):
        oracle.sparse_attn(qb, packed, sc, np.array([[[256]]], np.int32), 1.0)


# ----------------------------------------------------------------- modes
def _tiny_workload():
    return wl.small(B=2, Tq=2, N=512, Hq=4, Hi=4, Di=32, K=24, D=64, C=64)


def _inputs(w, layer=0):
    return dict(q=wl.q(w, layer), idx_q=wl.idx_q(w, layer), idx_w=wl.idx_w(w, layer))


def test_reuse_of_full_indices_reproduces_full(oracle_lib):
    w = _tiny_workload()
    packed, sc = oracle.fp4_kv_pack(wl.kv(w))
    ik, nv = wl.idx_k(w), wl.nvalid(w)
    nv[1, 0] = 300
    x = _inputs(w)
    topk = np.zeros((w.B, w.Tq, w.K), np.int32)
    cand = np.zeros((w.B, w.Tq, w.C), np.int32)
    o_full, l_full = oracle.layer_step(oracle.MODE_FULL, x["q"], x["idx_q"], x["idx_w"], ik,
                                       packed, sc, nv, w.K, 1.0, topk, cand, C=w.C)
    assert np.all(topk[1, 0][topk[1, 0] >= 0] < 300)
    o_reuse, l_reuse = oracle.layer_step(oracle.MODE_REUSE, x["q"], None, None, None, packed, sc,
                                         nv, w.K, 1.0, topk.copy())
    assert np.array_equal(o_full, o_reuse) and np.array_equal(l_full, l_reuse)
    # REINDEX with FULL's own indexer inputs over FULL's top-C pool gives FULL's top-K
    t2 = np.zeros_like(topk)
    oracle.layer_step(oracle.MODE_REINDEX, x["q"], x["idx_q"], x["idx_w"], ik, packed, sc, nv,
                      w.K, 1.0, t2, cand, C=w.C, use_pool=True)
    assert np.array_equal(t2, topk)


def test_pool_of_all_entries_equals_unrestricted_reindex(oracle_lib):
    w = _tiny_workload().replace(C=512)
    packed, sc = oracle.fp4_kv_pack(wl.kv(w))
    ik, nv = wl.idx_k(w), wl.nvalid(w)
    x = _inputs(w, layer=1)
    t_plain = np.zeros((w.B, w.Tq, w.K), np.int32)
    o1, _ = oracle.layer_step(oracle.MODE_REINDEX, x["q"], x["idx_q"], x["idx_w"], ik, packed, sc,
                              nv, w.K, 1.0, t_plain)
    cand = np.broadcast_to(np.arange(512, dtype=np.int32), (w.B, w.Tq, 512)).copy()
    t_pool = np.zeros_like(t_plain)
    o2, _ = oracle.layer_step(oracle.MODE_REINDEX, x["q"], x["idx_q"], x["idx_w"], ik, packed, sc,
                              nv, w.K, 1.0, t_pool, cand, C=512, use_pool=True)
    assert np.array_equal(t_plain, t_pool) and np.array_equal(o1, o2)


def test_layer_step_full_matches_composed_calls(oracle_lib):
    w = _tiny_workload()
    packed, sc = oracle.fp4_kv_pack(wl.kv(w))
    ik, nv = wl.idx_k(w), wl.nvalid(w)
    x = _inputs(w)
    s = oracle.index_score(x["idx_q"], x["idx_w"], ik, nvalid=nv)
    tk = oracle.topk(s, w.K, nvalid=nv)
    o, l = oracle.sparse_attn(x["q"], packed, sc, tk, 0.5)
    t2 = np.zeros_like(tk)
    o2, l2 = oracle.layer_step(oracle.MODE_FULL, x["q"], x["idx_q"], x["idx_w"], ik, packed, sc,
                               nv, w.K, 0.5, t2)
    assert np.array_equal(tk, t2) and np.array_equal(o, o2) and np.array_equal(l, l2)
    # the top-K indices really are the K best scores (brute force)
    for b, t in itertools.product(range(w.B), range(w.Tq)):
        assert list(tk[b, t]) == _brute_topk(list(s[b, t, :nv[b, t]]), list(range(nv[b, t])), w.K)


# ----------------------------------------------------------------- workloads
def test_workloads_are_seeded_and_shaped(facts):
    w = wl.PREFILL_CHUNK
    nv = wl.nvalid(w)
    assert nv.shape == (1, 4096) and nv.min() == 65536 - 1024 and nv.max() == 65536
    assert nv[0, 0] == 64512 and nv[0, 3] == 64513 and nv[0, 4095] == 65536
    w1 = wl.DECODE_128K
    n1 = wl.nvalid(w1)
    assert n1.shape == (32, 1) and n1.min() >= 16384 and n1.max() <= 32768
    assert np.array_equal(n1, wl.nvalid(w1))
    w0 = wl.TINY_DECODE
    a, b = wl.idx_q(w0), wl.idx_q(w0)
    assert np.array_equal(a, b) and a.shape == (1, 1, 4, 64)
    vals = torch.from_numpy(a).view(torch.float8_e4m3fn).float().numpy()
    assert set(np.unique(vals)) <= set(range(-4, 5))
    ww = wl.idx_w(w0)
    assert set(np.unique(ww)) <= {1.0, 2.0, 3.0, 4.0}
    assert facts["hierarchical_pool"]["blocks"] * facts["hierarchical_pool"]["block_size"] == \
        facts["hierarchical_pool"]["positions"]
