"""Pins for the oracle's blockwise candidate pool (no GPU): positions grouped
in blocks of 8, a block scored by its best valid position, the best 2048
blocks kept ("Hierarchical Sparse Indexer In Simple Terms"; mengman.github.io
3.4). Checked against the pinned per-entry selection (block size 1), a brute
force written here, the pages' pool size, and what the method relies on: the
FULL layer's own top-K lies inside its pool, so a REINDEX layer scoring only
the pool with the same query finds the same top-K."""
import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _brute(scores, nv, block, nblocks):
    nb = -(-nv // block)
    bmax = [max(scores[j] for j in range(b * block, min((b + 1) * block, nv))) for b in range(nb)]
    order = sorted(range(nb), key=lambda b: (-bmax[b], b))[:nblocks]
    pos = sorted(j for b in order for j in range(b * block, min((b + 1) * block, nv)))
    return pos + [-1] * (nblocks * block - len(pos))


def test_block_size_one_is_the_per_entry_selection(oracle_lib):
    rng = np.random.default_rng(41)
    scores = rng.integers(-5, 6, (4, 300)).astype(np.float64)
    nv = np.array([300, 1, 0, 173], np.int32)
    assert np.array_equal(oracle.block_pool(scores, nv, 1, 64), oracle.topk(scores, 64, nv))


@pytest.mark.parametrize("block,nblocks", [(8, 5), (8, 64), (3, 4), (4, 1)])
def test_matches_brute_force_with_ties(oracle_lib, block, nblocks):
    rng = np.random.default_rng(block * 100 + nblocks)
    rows, ld = 6, 97
    scores = rng.integers(0, 4, (rows, ld)).astype(np.float64)   # many equal block maxima
    nv = np.array([97, 96, 9, 8, 1, 0], np.int32)
    got = oracle.block_pool(scores, nv, block, nblocks)
    for r in range(rows):
        assert list(got[r]) == _brute(list(scores[r]), int(nv[r]), block, nblocks), r


def test_pool_is_everything_when_all_blocks_fit(oracle_lib):
    rng = np.random.default_rng(42)
    scores = rng.standard_normal((3, 50))
    nv = np.array([50, 43, 7], np.int32)
    got = oracle.block_pool(scores, nv, 8, 7)                   # 7 blocks cover 56 >= 50
    for r in range(3):
        want = list(range(nv[r])) + [-1] * (56 - nv[r])
        assert list(got[r]) == want


def test_the_pages_pool_size(oracle_lib):
    with open(GOLDEN) as f:
        hp = json.load(f)["hierarchical_pool"]
    rng = np.random.default_rng(43)
    N = 40000
    scores = rng.standard_normal((2, N))
    nv = np.array([N, 30005], np.int32)
    got = oracle.block_pool(scores, nv, hp["block_size"], hp["blocks"])
    assert got.shape[-1] == hp["positions"]
    for r in range(2):
        valid = got[r][got[r] >= 0]
        assert np.all(np.diff(valid) > 0) and valid.max() < nv[r]
        blocks = np.unique(valid // hp["block_size"])
        assert blocks.size == hp["blocks"]
        # every kept block's score is at least every dropped block's
        bmax = np.array([scores[r, b * 8:min(b * 8 + 8, nv[r])].max()
                         for b in range(-(-int(nv[r]) // 8))])
        dropped = np.setdiff1d(np.arange(bmax.size), blocks)
        assert bmax[blocks].min() >= bmax[dropped].max()


@pytest.mark.parametrize("K,nblocks", [(16, 16), (16, 40), (64, 64)])
def test_full_topk_lies_inside_the_pool(oracle_lib, K, nblocks):
    rng = np.random.default_rng(K + nblocks)
    rows, ld = 20, 2000
    scores = rng.integers(0, 6, (rows, ld)).astype(np.float64)  # heavy ties
    nv = rng.integers(1, ld + 1, rows).astype(np.int32)
    top = oracle.topk(scores, K, nv)
    pool = oracle.block_pool(scores, nv, 8, nblocks)
    for r in range(rows):
        assert set(top[r][top[r] >= 0]) <= set(pool[r][pool[r] >= 0]), r


def test_reindex_in_the_pool_with_the_same_query_finds_the_same_topk(oracle_lib):
    rng = np.random.default_rng(44)
    B, Tq, N, Hi, Di, K = 2, 1, 3000, 4, 32, 64
    e4m3 = lambda x: torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()
    iq = e4m3(rng.integers(-4, 5, (B, Tq, Hi, Di)))
    ik = e4m3(rng.integers(-4, 5, (B, N, Di)))
    iw = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    nv = np.array([[3000], [2222]], np.int32)
    scores = oracle.index_score(iq, iw, ik, nv)
    full = oracle.topk(scores, K, nv)
    pool = oracle.block_pool(scores, nv, 8, 128)
    pooled = oracle.topk(oracle.index_score(iq, iw, ik, cand=pool), K, cand=pool)
    assert np.array_equal(pooled, full)


def test_nan_is_an_error(oracle_lib):
    scores = np.zeros((1, 20))
    scores[0, 13] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.block_pool(scores, np.array([20], np.int32), 8, 2)
