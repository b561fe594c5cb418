"""The sequence split of one long context over ranks, as host logic on CPU
with gloo at world size 2 (no GPU; unmeasured on hardware). The N entries
(indexer keys, main KV and its 64-entry scale blocks) are cut into contiguous
shards, one per rank. Then:
  1. each rank scores its shard and keeps a local top-K of (score, global id);
  2. one all-gather of those K pairs per query; every rank merges them with
     the same ranking (score descending, lower id first) into the global top-K;
  3. each rank attends over the selected entries it owns: a partial (out, lse);
  4. an all-gather of the partials and a log-sum-exp weighted combine.
The merged top-K must equal the one-rank top-K bit for bit (every entry of the
global top-K is in its own shard's local top-K, since the ranking is a total
order), and the combined attention must equal the one-rank attention up to
fp64 rounding: with m = max_r lse_r, softmax over the union gives
out = sum_r e^(lse_r - m) out_r / sum_r e^(lse_r - m), lse = m + log sum_r e^(lse_r - m).
The per-shard steps are the oracle's (the rule of "Hierarchical Sparse Indexer
In Simple Terms" and "Compressed Sparse Attention 2 Or CSA2 In Simple Terms"
in "Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words": score, keep
the top-K, attend over them)."""
import datetime
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from fp4_kv_cache_step_b200 import workloads as wl

W = wl.small("seq_split", seed=77, B=1, Tq=3, N=2048, Hq=16, Hi=4, Di=64, K=256)
NVALID = np.array([[2048, 1500, 700]], np.int32)     # the last query sees rank 0's shard only


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs():
    kv = wl.kv(W)
    return (wl.idx_q(W), wl.idx_w(W), wl.idx_k(W), wl.q(W), kv)


def lse_combine(outs, lses):
    """Partials out_r [..][D] and lse_r [..] (lse = -inf for an empty part)
    merged into the softmax over the union of the parts."""
    lses = np.stack(lses)
    outs = np.stack(outs)
    m = lses.max(axis=0)
    m = np.where(np.isfinite(m), m, 0.0)
    wts = np.exp(lses - m)                              # 0 for an empty part
    z = wts.sum(axis=0)
    safe = np.where(z > 0, z, 1.0)
    out = np.where(z[..., None] > 0, (wts[..., None] * outs).sum(axis=0) / safe[..., None], 0.0)
    lse = np.where(z > 0, m + np.log(safe), -np.inf)
    return out, lse


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        oracle.build()
        iq, iw, ik, qb, kv = _inputs()
        shard = W.N // world
        lo = rank * shard
        # 1. the shard's scores and local top-K, as (score, global id) pairs
        nv_local = np.clip(NVALID - lo, 0, shard).astype(np.int32)
        s_local = oracle.index_score(iq, iw, ik[:, lo:lo + shard], nv_local)
        t_local = oracle.topk(s_local, W.K, nv_local)
        ids = np.where(t_local >= 0, t_local + lo, -1).astype(np.int32)
        sc = np.take_along_axis(s_local, np.maximum(t_local, 0), axis=-1)
        sc = np.where(t_local >= 0, sc, -np.inf)
        # 2. one all-gather of the pairs, merged with the same ranking
        g_sc = [torch.empty(sc.shape, dtype=torch.float64) for _ in range(world)]
        g_id = [torch.empty(ids.shape, dtype=torch.int32) for _ in range(world)]
        dist.all_gather(g_sc, torch.from_numpy(sc))
        dist.all_gather(g_id, torch.from_numpy(ids))
        all_sc = np.concatenate([t.numpy() for t in g_sc], axis=-1)
        all_id = np.concatenate([t.numpy() for t in g_id], axis=-1)
        merged = oracle.topk(all_sc, W.K, cand=all_id)
        # 3. attention over the selected entries this rank owns
        packed, scale = oracle.fp4_kv_pack(kv[:, lo:lo + shard])
        own = np.where((merged >= lo) & (merged < lo + shard), merged - lo, -1).astype(np.int32)
        out_r, lse_r = oracle.sparse_attn(qb, packed, scale, own, W.softmax_scale)
        # 4. the partials gathered and combined by their log-sum-exps
        g_o = [torch.empty(out_r.shape, dtype=torch.float64) for _ in range(world)]
        g_l = [torch.empty(lse_r.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(g_o, torch.from_numpy(out_r))
        dist.all_gather(g_l, torch.from_numpy(lse_r))
        out, lse = lse_combine([t.numpy() for t in g_o], [t.numpy() for t in g_l])
        q.put((rank, merged, out, lse))
    finally:
        dist.destroy_process_group()


def test_sequence_split_over_two_ranks_equals_one_rank():
    oracle.build()
    world = 2
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, merged, out, lse = qu.get(timeout=240)
        res[rank] = (merged, out, lse)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0

    iq, iw, ik, qb, kv = _inputs()
    want_idx = oracle.topk(oracle.index_score(iq, iw, ik, NVALID), W.K, NVALID)
    packed, scale = oracle.fp4_kv_pack(kv)
    want_out, want_lse = oracle.sparse_attn(qb, packed, scale, want_idx, W.softmax_scale)
    # the integer-valued indexer gives many equal scores: the tie-break decides
    s = oracle.index_score(iq, iw, ik, NVALID)
    assert len(np.unique(s[0, 0])) < W.N // 4
    for rank in range(world):
        merged, out, lse = res[rank]
        assert np.array_equal(merged, want_idx), rank          # every rank, the same top-K
        np.testing.assert_allclose(out, want_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, want_lse, rtol=0, atol=1e-12)
    # the last query's selection lies in rank 0's shard: rank 1's part was empty
    assert want_idx[0, 2].max() < W.N // 2


def test_lse_combine_special_cases():
    """An empty part (lse = -inf) drops out; all parts empty give 0 and -inf;
    equal parts give the same output and lse + log(parts)."""
    rng = np.random.default_rng(3)
    o = rng.standard_normal((4, 8))
    l = rng.standard_normal(4)
    out, lse = lse_combine([o, np.zeros_like(o)], [l, np.full(4, -np.inf)])
    np.testing.assert_array_equal(out, o)
    np.testing.assert_array_equal(lse, l)
    out, lse = lse_combine([o, o], [np.full(4, -np.inf)] * 2)
    assert np.all(out == 0) and np.all(np.isneginf(lse))
    out, lse = lse_combine([o, o, o], [l, l, l])
    np.testing.assert_allclose(out, o, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, l + math.log(3.0), rtol=0, atol=1e-15)
