"""GPU parity of every C-ABI call against the CPU oracle, on seeded inputs
small enough for the oracle to finish in seconds but spanning several tiles and
ragged tails. Indices, packed bytes and integer-valued scores must match bit
for bit; attention outputs within the tolerance in parity_utils."""
import math

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2
from fp4_kv_cache_step_b200 import workloads as wl
from fp4_kv_cache_step_b200.runner import DeviceWorkload
from tests.parity_utils import (assert_attn_close, assert_lse_close, bf16_dev, dev, host,
                                row_vmax)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    libbuild.build()
    csa2.load()
    oracle.build()
    yield
    csa2.check_device_errors()


def _e4m3(ints):
    return torch.from_numpy(np.asarray(ints, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


# ------------------------------------------------------------------ FP4 pack
@pytest.mark.parametrize("B,N,D,mult", [(2, 192, 512, 1.0), (1, 64, 64, 7.5), (3, 128, 96, 1e-3)])
def test_pack_unpack_bit_exact(B, N, D, mult):
    rng = np.random.default_rng(B * 1000 + N + D)
    kv = (rng.standard_normal((B, N, D)) * mult).astype(np.float32)
    kv[0, :64, 1] = 0.0                                  # zero block
    kv[-1, -64:, 2] = np.float32(1e-30)                  # block whose scale rounds to 0
    # exact grid points and midpoints at a known scale
    s = np.float32(0.5)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)
    col = np.concatenate([grid, mids, -grid, -mids])
    kv[0, :len(col), 4] = col * s
    kv[0, len(col):64, 4] = 0.0
    kv[0, 0, 4] = 6 * s
    want_p, want_s = oracle.fp4_kv_pack(kv)
    p, sc = csa2.fp4_kv_pack(dev(kv))
    assert np.array_equal(host(p), want_p)
    assert np.array_equal(host(sc), want_s)
    back = host(csa2.fp4_kv_unpack(p, sc)).astype(np.float64)
    assert np.array_equal(back, oracle.fp4_kv_unpack(want_p, want_s))
    csa2.check_device_errors()


def test_pack_saturates_and_flags_nonfinite():
    kv = np.zeros((1, 64, 32), np.float32)
    kv[0, 3, 0] = 1e6                                    # scale saturates at 448
    kv[0, 4, 0] = -5e3
    p, sc = csa2.fp4_kv_pack(dev(kv))
    want_p, want_s = oracle.fp4_kv_pack(kv)
    assert np.array_equal(host(p), want_p) and np.array_equal(host(sc), want_s)
    kv[0, 9, 5] = np.nan
    csa2.fp4_kv_pack(dev(kv))
    with pytest.raises(csa2.Csa2Error) as ei:
        csa2.check_device_errors()
    assert ei.value.status == 5
    csa2.check_device_errors()                           # cleared


# ------------------------------------------------------------------ indexer
# (3, 2, 1024, 64, 128), (1, 5, 2048, 64, 128) and (2, 3, 1024, 128, 128) take
# the tensor-core scorer's multi-query path (groups of 4 and 2 queries, the
# last group partial; 128 heads in two 64-column chunks per query)
@pytest.mark.parametrize("B,Tq,N,Hi,Di", [(1, 1, 4096, 4, 64), (3, 2, 1000 // 64 * 64 + 64, 64, 128),
                                          (2, 3, 640, 16, 32), (1, 5, 2048, 64, 128),
                                          (2, 3, 1024, 128, 128)])
def test_index_score_exact(B, Tq, N, Hi, Di):
    rng = np.random.default_rng(N + Hi)
    qb = _e4m3(rng.integers(-4, 5, (B, Tq, Hi, Di)))
    kb = _e4m3(rng.integers(-4, 5, (B, N, Di)))
    w = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    nv = rng.integers(0, N + 1, (B, Tq)).astype(np.int32)
    nv[0, 0] = N
    if B * Tq > 1:
        nv.flat[1] = 1
    want = oracle.index_score(qb, w, kb, nvalid=nv)
    got = host(csa2.csa2_index_score(dev(qb), dev(w), dev(kb), nvalid=dev(nv)))
    for b in range(B):
        for t in range(Tq):
            n = nv[b, t]
            assert np.array_equal(got[b, t, :n].astype(np.float64), want[b, t, :n]), (b, t)


def test_index_score_pool_exact():
    rng = np.random.default_rng(21)
    B, Tq, N, Hi, Di, C = 2, 2, 2048, 64, 128, 300
    qb = _e4m3(rng.integers(-4, 5, (B, Tq, Hi, Di)))
    kb = _e4m3(rng.integers(-4, 5, (B, N, Di)))
    w = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    cand = np.full((B, Tq, C), -1, np.int32)
    for b in range(B):
        for t in range(Tq):
            m = [C, 257, 1, 0][b * Tq + t]
            cand[b, t, :m] = np.sort(rng.choice(N, m, replace=False))
    want = oracle.index_score(qb, w, kb, cand=cand)
    got = host(csa2.csa2_index_score(dev(qb), dev(w), dev(kb), cand=dev(cand)))
    assert np.array_equal(got.astype(np.float64), want)


# ------------------------------------------------------------------ top-K
def _scores(rng, shape, kind):
    if kind == "ties":
        return rng.integers(0, 50, shape).astype(np.float32)
    if kind == "signed":
        x = rng.integers(-30, 30, shape).astype(np.float32)
        x[x == 0] = np.where(rng.random(np.count_nonzero(x == 0)) < 0.5, -0.0, 0.0)
        return x
    if kind == "wide":
        return (rng.standard_normal(shape) * 1e4).astype(np.float32)
    if kind == "const":
        return np.full(shape, 7.0, np.float32)
    if kind == "twovals":
        return np.where(rng.random(shape) < 0.5, 3.0, -2.0).astype(np.float32)
    if kind == "gauss_int":       # like the indexer scores: integers ~ N(4800, 1000)
        return np.round(rng.normal(4800, 1000, shape)).astype(np.float32)
    raise ValueError(kind)


@pytest.mark.parametrize("ld,K", [(3000, 64), (3000, 1), (4096, 256), (32768, 2048), (70000, 2048),
                                  (100, 200)])
@pytest.mark.parametrize("kind", ["ties", "signed", "wide", "const", "twovals", "gauss_int"])
def test_topk_bit_exact(ld, K, kind):
    rng = np.random.default_rng(ld + K)
    rows = 6
    sc = _scores(rng, (2, rows // 2, ld), kind)
    sc[0, 0, 5] = -np.inf
    nv = rng.integers(0, ld + 1, (2, rows // 2)).astype(np.int32)
    nv[0, 0] = ld
    nv[0, 1] = min(ld, K)
    nv[0, 2] = 0
    nv[1, 0] = min(ld, K + 1)
    want = oracle.topk(sc.astype(np.float64), K, nvalid=nv)
    got = host(csa2.csa2_topk(dev(sc), K, nvalid=dev(nv)))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("ld,K,Cout", [(16384, 2048, 8192), (262144 // 16, 256, 1024), (5000, 64, 64)])
def test_topk_with_pool_output(ld, K, Cout):
    rng = np.random.default_rng(ld + Cout)
    sc = _scores(rng, (2, 1, ld), "ties")
    nv = np.array([[ld], [ld - 17]], np.int32)
    tk, cd = csa2.csa2_topk(dev(sc), K, nvalid=dev(nv), Cout=Cout)
    assert np.array_equal(host(tk), oracle.topk(sc.astype(np.float64), K, nvalid=nv))
    assert np.array_equal(host(cd), oracle.topk(sc.astype(np.float64), Cout, nvalid=nv))


def test_topk_inside_pool():
    rng = np.random.default_rng(31)
    B, Tq, C, K = 2, 2, 8192, 2048
    cand = np.full((B, Tq, C), -1, np.int32)
    for i, m in enumerate([C, 5000, 2048, 10]):
        cand.reshape(-1, C)[i, :m] = np.sort(rng.choice(10 ** 6, m, replace=False))
    sc = _scores(rng, (B, Tq, C), "ties")
    got = host(csa2.csa2_topk(dev(sc), K, cand=dev(cand)))
    assert np.array_equal(got, oracle.topk(sc.astype(np.float64), K, cand=cand))


def test_topk_unsorted_pool_is_flagged():
    cand = np.array([[[5, 3, 9, -1]]], np.int32)
    sc = np.array([[[1.0, 2.0, 3.0, 0.0]]], np.float32)
    csa2.csa2_topk(dev(sc), 2, cand=dev(cand))
    with pytest.raises(csa2.Csa2Error) as ei:
        csa2.check_device_errors()
    assert ei.value.status == 4


# ------------------------------------------------------------------ attention
def _attn_case(seed, B, Tq, Hq, N, K, pad_frac=0.1, max_valid=None):
    rng = np.random.default_rng(seed)
    kv = rng.standard_normal((B, N, 512)).astype(np.float32)
    packed, scale = oracle.fp4_kv_pack(kv)
    q = wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / math.sqrt(512))
    idx = np.full((B, Tq, K), -1, np.int32)
    for b in range(B):
        for t in range(Tq):
            m = K if rng.random() > pad_frac else int(rng.integers(0, K))
            m = min(m, N)
            idx[b, t, :m] = np.sort(rng.choice(N if max_valid is None else max_valid, m,
                                               replace=False))
    return packed, scale, q, idx


@pytest.mark.parametrize("B,Tq,Hq,N,K", [(2, 1, 64, 4096, 256), (1, 1, 16, 4096, 256),
                                         (1, 2, 128, 2048, 200), (3, 1, 64, 16384, 2048),
                                         (40, 1, 64, 4096, 100), (1, 3, 48, 1024, 64)])
@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 1.0, 24.0])
def test_sparse_attn_within_tolerance(B, Tq, Hq, N, K, scale):
    packed, sc, q, idx = _attn_case(B * 7 + K, B, Tq, Hq, N, K)
    idx[0, 0, :] = -1                                   # a row with nothing selected
    want, want_lse = oracle.sparse_attn(q, packed, sc, idx, scale)
    out, lse = csa2.csa2_sparse_attn(bf16_dev(q), dev(packed), dev(sc), dev(idx), scale)
    assert_attn_close(host(out), want, "out", sharp=scale > 4.0,
                      vmax=row_vmax(oracle.fp4_kv_unpack(packed, sc), idx))
    assert_lse_close(host(lse), want_lse, "lse")
    assert np.all(host(out)[0, 0] == 0.0)


def _block_case(seed, B, N, K, magnitude):
    """Block-layout caches at the value ranges the pages report and below:
    'pages' scales every (64-entry block, channel) to a maximum between 10 and
    22 ('Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words', section
    'FP4 Main KV Cache To Halve Storage Again': observed maxima of about 10 to
    22, so no global scale is needed); 'subnormal' makes every block maximum below
    0.075, so scale = max / 6 rounds to a nonzero E4M3 subnormal (1 to 7
    times 2^-9)."""
    rng = np.random.default_rng(seed)
    kv = rng.standard_normal((B, N, 512)).astype(np.float32)
    blk = kv.reshape(B, N // 64, 64, 512)
    amax = np.abs(blk).max(axis=2, keepdims=True)
    if magnitude == "pages":
        target = rng.uniform(10.0, 22.0, amax.shape).astype(np.float32)
    else:
        target = rng.uniform(0.012, 0.075, amax.shape).astype(np.float32)
    kv = (blk / amax * target).reshape(B, N, 512).astype(np.float32)
    packed, scale = oracle.fp4_kv_pack(kv)
    if magnitude == "subnormal":
        assert np.all((scale & 0x78) == 0) and np.all(scale != 0), "nonzero subnormal scales"
    idx = np.stack([np.sort(rng.choice(N, K, replace=False)) for _ in range(B)])[:, None, :]
    return packed, scale, idx.astype(np.int32)


# the in-cluster merge (2 rows, 4 splits) and the combine kernel (3 rows, 32 splits)
@pytest.mark.parametrize("B,N,K", [(2, 4096, 256), (3, 16384, 2048)])
@pytest.mark.parametrize("magnitude", ["pages", "subnormal"])
@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 1.0])
def test_sparse_attn_block_layout_value_ranges(B, N, K, magnitude, scale):
    packed, sc, idx = _block_case(B * 31 + K, B, N, K, magnitude)
    rng = np.random.default_rng(B + K)
    q = wl._to_bf16_bits(rng.standard_normal((B, 1, 64, 512)).astype(np.float32) / math.sqrt(512))
    want, want_lse = oracle.sparse_attn(q, packed, sc, idx, scale)
    out, lse = csa2.csa2_sparse_attn(bf16_dev(q), dev(packed), dev(sc), dev(idx), scale)
    csa2.check_device_errors()
    assert_attn_close(host(out), want, "out %s" % magnitude, sharp=True,
                      vmax=row_vmax(oracle.fp4_kv_unpack(packed, sc), idx))
    assert_lse_close(host(lse), want_lse, "lse %s" % magnitude)


def test_sparse_attn_rising_max_across_tiles():
    """Logits that grow tile after tile force the running max to be raised and
    the accumulated output to be rescaled many times."""
    B, Tq, Hq, N, K = 2, 1, 64, 4096, 1024
    packed, sc, q, idx = _attn_case(77, B, Tq, Hq, N, K, pad_frac=0.0)
    V = oracle.fp4_kv_unpack(packed, sc)
    qf = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double().numpy()
    for b in range(B):
        logits = qf[b, 0] @ V[b].T                     # [Hq][N]
        order = np.argsort(logits[0])                  # head 0: ascending logit
        idx[b, 0] = np.sort(order[-K:]).astype(np.int32)
        idx[b, 0] = order[-K:].astype(np.int32)        # unsorted: rising logits along the list
    vmax = row_vmax(V, idx)
    for scale in (8.0, 40.0):
        want, want_lse = oracle.sparse_attn(q, packed, sc, idx, scale)
        out, lse = csa2.csa2_sparse_attn(bf16_dev(q), dev(packed), dev(sc), dev(idx), scale)
        assert_attn_close(host(out), want, "out scale=%g" % scale, sharp=True, vmax=vmax)
        assert_lse_close(host(lse), want_lse, "lse scale=%g" % scale)


def test_sparse_attn_bad_index_is_flagged_and_skipped():
    packed, sc, q, idx = _attn_case(5, 1, 1, 64, 1024, 64)
    idx[0, 0, 3] = 1024
    out, lse = csa2.csa2_sparse_attn(bf16_dev(q), dev(packed), dev(sc), dev(idx), 1.0)
    with pytest.raises(csa2.Csa2Error) as ei:
        csa2.check_device_errors()
    assert ei.value.status == 4
    idx2 = idx.copy()
    idx2[0, 0, 3] = -1
    want, _ = oracle.sparse_attn(q, packed, sc, idx2, 1.0)
    assert_attn_close(host(out), want, "out")


# ------------------------------------------------------------------ layer steps
def _oracle_stack(w, rows=None):
    """Oracle run of the workload's mode schedule for the given batch rows."""
    rows = list(range(w.B)) if rows is None else list(rows)
    res = {}
    nv_all = wl.nvalid(w)
    for b in rows:
        packed, sc = oracle.fp4_kv_pack(wl.kv(w, rows=[b]))
        ik = wl.idx_k(w, rows=[b])
        nv = nv_all[b:b + 1]
        topk = np.full((1, w.Tq, w.K), -1, np.int32)
        cand = np.full((1, w.Tq, w.C), -1, np.int32) if w.C else None
        layers = []
        for layer, mode in enumerate(w.modes):
            m = {wl.FULL: oracle.MODE_FULL, wl.REINDEX: oracle.MODE_REINDEX,
                 wl.REUSE: oracle.MODE_REUSE}[mode]
            qb = wl.q(w, layer, rows=[b])
            iq = wl.idx_q(w, layer, rows=[b]) if mode != wl.REUSE else None
            iw = wl.idx_w(w, layer, rows=[b]) if mode != wl.REUSE else None
            out, lse = oracle.layer_step(m, qb, iq, iw, ik, packed, sc, nv, w.K, w.softmax_scale,
                                         topk, cand, C=w.C, use_pool=(mode == wl.REINDEX and w.C > 0))
            layers.append((topk.copy(), None if cand is None else cand.copy(), out, lse))
        res[b] = dict(packed=packed, scale=sc, layers=layers)
    return res


def _check_stack(w, dw, want, rows):
    for b in rows:
        assert np.array_equal(host(dw.kv_packed[b]), want[b]["packed"][0]), b
        assert np.array_equal(host(dw.kv_scale[b]), want[b]["scale"][0]), b
        for layer, (tk, cd, out, lse) in enumerate(want[b]["layers"]):
            assert np.array_equal(host(dw.topk_per_layer[layer][b]), tk[0]), (b, layer)
            assert_attn_close(host(dw.out[layer][b]), out[0], "out b=%d layer=%d" % (b, layer))
            assert_lse_close(host(dw.lse[layer][b]), lse[0], "lse b=%d layer=%d" % (b, layer))
            if cd is not None and w.modes[layer] == wl.FULL:
                assert np.array_equal(host(dw.cand[b]), cd[0]), b


def test_layer_step_config0_full():
    w = wl.TINY_DECODE
    dw = DeviceWorkload(w)
    dw.step(snapshot_topk=True)
    csa2.check_device_errors()
    _check_stack(w, dw, _oracle_stack(w), range(w.B))


@pytest.mark.parametrize("softmax_scale", [1.0 / math.sqrt(512.0), 1.0])
def test_mode_stack_small(softmax_scale):
    w = wl.small(name="stack_small", seed=41, B=3, N=2048, Hq=64, Hi=64, Di=128, K=256,
                 modes=(wl.FULL, wl.REINDEX, wl.REUSE, wl.REUSE), lengths="uniform",
                 len_lo=100, len_hi=2048, softmax_scale=softmax_scale)
    dw = DeviceWorkload(w)
    dw.step(snapshot_topk=True)
    csa2.check_device_errors()
    _check_stack(w, dw, _oracle_stack(w), range(w.B))
    # REUSE over FULL's own indices reproduces FULL's output bit for bit
    dw.step(layers=[0], snapshot_topk=True)
    full_out = dw.out[0].clone()
    args = csa2.layer_args(dw.q[0], dw.nvalid, dw.out[2], w.K, w.softmax_scale, lse=dw.lse[2], N=w.N)
    csa2.csa2_layer_step("REUSE", args, dw.shared, dw.workspace)
    assert torch.equal(dw.out[2], full_out)


def test_hierarchical_pool_small():
    w = wl.small(name="hier_small", seed=43, B=2, N=16384, Hq=64, Hi=64, Di=128, K=256, C=1024,
                 modes=(wl.FULL, wl.REINDEX))
    dw = DeviceWorkload(w)
    dw.step(snapshot_topk=True)
    csa2.check_device_errors()
    _check_stack(w, dw, _oracle_stack(w), range(w.B))


def test_prefill_chunk_small():
    w = wl.small(name="prefill_small", seed=44, B=1, Tq=64, N=2048, Hq=64, Hi=64, Di=128, K=128,
                 lengths="chunk_end")
    dw = DeviceWorkload(w)
    dw.step(snapshot_topk=True)
    csa2.check_device_errors()
    _check_stack(w, dw, _oracle_stack(w), range(w.B))
