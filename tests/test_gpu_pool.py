"""GPU parity of the blockwise candidate pool of the hierarchical indexer
(blocks of 8 positions scored by their best position, the best blocks kept;
"Hierarchical Sparse Indexer In Simple Terms", mengman.github.io 3.4): the
pool is compared with the oracle's bit for bit, alone and inside a FULL
(emitting the pool) -> REINDEX (scoring only the pool) layer pair."""
import math

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2
from fp4_kv_cache_step_b200 import workloads as wl
from tests.parity_utils import (assert_attn_close, assert_lse_close, bf16_dev, dev, host)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    libbuild.build()
    csa2.load()
    oracle.build()
    csa2.check_device_errors()
    yield
    csa2.check_device_errors()


@pytest.mark.parametrize("ld,block,nblocks", [(5000, 8, 5), (5000, 8, 64), (5000, 8, 2048),
                                              (777, 1, 100), (777, 3, 40), (8, 8, 1)])
def test_block_pool_bit_exact_with_ties(ld, block, nblocks):
    rng = np.random.default_rng(ld + block * 10 + nblocks)
    B, Tq = 3, 2
    scores = rng.integers(0, 5, (B, Tq, ld)).astype(np.float32)      # many equal block maxima
    nv = np.array([[ld, ld - 1], [1, 0], [ld // 2 + 3, min(ld, 17)]], np.int32)
    want = oracle.block_pool(scores.astype(np.float64), nv, block, nblocks)
    got = csa2.csa2_block_pool(dev(scores), dev(nv), nblocks, block)
    assert np.array_equal(host(got), want)


def test_block_pool_at_the_pages_size():
    """2048 blocks of 8 (16384 candidates) over a 1M-token decoder history
    (262144 entries), Gaussian scores."""
    rng = np.random.default_rng(5)
    B, Tq, N = 2, 1, 262144
    scores = rng.standard_normal((B, Tq, N)).astype(np.float32)
    nv = np.array([[N], [200003]], np.int32)
    want = oracle.block_pool(scores.astype(np.float64), nv, 8, 2048)
    got = csa2.csa2_block_pool(dev(scores), dev(nv), 2048)
    assert np.array_equal(host(got), want)


def test_block_pool_flags_nan():
    scores = np.zeros((1, 1, 100), np.float32)
    scores[0, 0, 42] = np.nan
    csa2.csa2_block_pool(dev(scores), dev(np.array([[100]], np.int32)), 4)
    with pytest.raises(csa2.Csa2Error) as ei:
        csa2.check_device_errors()
    assert ei.value.status == 5


def test_full_emits_blockwise_pool_and_reindex_scores_inside_it():
    B, Tq, N, Hq, Hi, Di, K, nblocks = 2, 1, 20480, 16, 8, 128, 256, 512
    C = 8 * nblocks
    rng = np.random.default_rng(11)
    kv = rng.standard_normal((B, N, 512), dtype=np.float32)
    packed, sc = oracle.fp4_kv_pack(kv)
    e4m3 = lambda x: torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()
    idx_k = e4m3(rng.integers(-4, 5, (B, N, Di)))
    iq = [e4m3(rng.integers(-4, 5, (B, Tq, Hi, Di))) for _ in range(2)]
    iw = [rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32) for _ in range(2)]
    q = [wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / 22.6)
         for _ in range(2)]
    nvalid = np.array([[N], [19999]], np.int32)                      # a partial last block
    scale = 1.0 / math.sqrt(512.0)

    s_full = oracle.index_score(iq[0], iw[0], idx_k, nvalid)
    want_top = oracle.topk(s_full, K, nvalid)
    want_pool = oracle.block_pool(s_full, nvalid, 8, nblocks)
    s_re = oracle.index_score(iq[1], iw[1], idx_k, cand=want_pool)
    want_top2 = oracle.topk(s_re, K, cand=want_pool)

    topk = torch.full((B, Tq, K), -1, dtype=torch.int32, device="cuda")
    cand = torch.full((B, Tq, C), -7, dtype=torch.int32, device="cuda")
    shared = csa2.Csa2Shared(dev(packed), dev(sc), dev(idx_k), topk, cand)
    nv = dev(nvalid)
    for layer, (mode, emit, use) in enumerate((("FULL", 2, False), ("REINDEX", 0, True))):
        out = torch.empty((B, Tq, Hq, 512), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device="cuda")
        args = csa2.layer_args(bf16_dev(q[layer]), nv, out, K, scale, idx_q=dev(iq[layer]),
                               idx_w=dev(iw[layer]), lse=lse, N=N, emit_pool=emit, use_pool=use)
        csa2.csa2_layer_step(mode, args, shared)
        top = want_top if layer == 0 else want_top2
        assert np.array_equal(host(topk), top), mode
        assert np.array_equal(host(cand), want_pool), mode
        want, want_lse = oracle.sparse_attn(q[layer], packed, sc, top, scale)
        assert_attn_close(host(out), want, "out %s" % mode)
        assert_lse_close(host(lse), want_lse, "lse %s" % mode)
    # the FULL layer's own top-K lies inside the pool it emitted
    for b in range(B):
        assert set(want_top[b, 0]) <= set(want_pool[b, 0][want_pool[b, 0] >= 0])
