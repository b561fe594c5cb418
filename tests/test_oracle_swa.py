"""Pins for the oracle's sliding-window branch (no GPU): every CSA2 layer also
attends the last 128 tokens, kept at 8 bits ("Detailed Notes On DeepSeek V4
Point 1 Flash In Simple Words", "Compressed Sparse Attention 2 Or CSA2 In
Simple Terms", "Model Setup Numbers Without Jargon"; mengman.github.io 3.3,
3.5). The combination with the sparse set is the reading taken here: one
softmax over both. Checked against the pinned sparse attention (empty
window), numpy softmax attention over torch-decoded E4M3 values (empty
selection, window clipping), and the identity that one softmax over a union
equals the two softmaxes merged by their log-sum-exps."""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def _bf16(x):
    t = torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16), t.to(torch.float64).numpy()


def _e4m3(x):
    t = torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy(), t.to(torch.float64).numpy()


def _case(seed, B=2, Tq=2, Hq=3, N=256, D=64, K=40, Tw=160):
    rng = np.random.default_rng(seed)
    packed, sc = oracle.fp4_kv_pack(rng.standard_normal((B, N, D)).astype(np.float32))
    qbits, qf = _bf16(rng.standard_normal((B, Tq, Hq, D)) / math.sqrt(512.0))
    idx = np.full((B, Tq, K), -1, np.int32)
    for b in range(B):
        for t in range(Tq):
            m = int(rng.integers(1, K + 1))
            idx[b, t, :m] = np.sort(rng.choice(N, m, replace=False))
    wbytes, wf = _e4m3(rng.standard_normal((B, Tw, D)))
    return packed, sc, qbits, qf, idx, wbytes, wf


def _np_attn(qf, V, scale):
    logits = scale * qf @ V.T
    return scipy.special.softmax(logits, axis=-1) @ V, scipy.special.logsumexp(logits, axis=-1)


def test_window_size_is_the_pages():
    with open(GOLDEN) as f:
        assert oracle.SWA_WINDOW == json.load(f)["swa_window"]["value"]


def test_empty_window_is_the_sparse_attention(oracle_lib):
    packed, sc, q, qf, idx, w, wf = _case(1)
    swa_n = np.zeros(idx.shape[:2], np.int32)
    a, la = oracle.swa_sparse_attn(q, packed, sc, idx, w, swa_n, 0.7)
    b, lb = oracle.sparse_attn(q, packed, sc, idx, 0.7)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


@pytest.mark.parametrize("W,hi", [(128, 128), (128, 160), (128, 50), (16, 100)])
def test_empty_selection_is_window_attention(oracle_lib, W, hi):
    packed, sc, q, qf, idx, w, wf = _case(2)
    idx[:] = -1
    swa_n = np.full(idx.shape[:2], hi, np.int32)
    out, lse = oracle.swa_sparse_attn(q, packed, sc, idx, w, swa_n, 0.9, W=W)
    lo = max(0, hi - W)
    for b in range(q.shape[0]):
        for t in range(q.shape[1]):
            ref, ref_lse = _np_attn(qf[b, t], wf[b, lo:hi], 0.9)
            np.testing.assert_allclose(out[b, t], ref, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(lse[b, t], ref_lse, rtol=1e-13)


@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 1.0, 8.0])
def test_union_is_the_lse_merge_of_the_two_branches(oracle_lib, scale):
    packed, sc, q, qf, idx, w, wf = _case(3)
    B, Tq = idx.shape[:2]
    swa_n = np.array([[128, 77], [160, 3]], np.int32)
    out, lse = oracle.swa_sparse_attn(q, packed, sc, idx, w, swa_n, scale)
    s_out, s_lse = oracle.sparse_attn(q, packed, sc, idx, scale)
    for b in range(B):
        for t in range(Tq):
            lo, hi = max(0, swa_n[b, t] - 128), swa_n[b, t]
            w_out, w_lse = _np_attn(qf[b, t], wf[b, lo:hi], scale)
            tot = np.logaddexp(s_lse[b, t], w_lse)
            merged = (np.exp(s_lse[b, t] - tot)[:, None] * s_out[b, t] +
                      np.exp(w_lse - tot)[:, None] * w_out)
            np.testing.assert_allclose(out[b, t], merged, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(lse[b, t], tot, rtol=1e-12)


def test_nothing_at_all_gives_zeros(oracle_lib):
    packed, sc, q, qf, idx, w, wf = _case(4)
    idx[:] = -1
    out, lse = oracle.swa_sparse_attn(q, packed, sc, idx, w, np.zeros(idx.shape[:2], np.int32), 1.0)
    assert np.all(out == 0.0) and np.all(np.isneginf(lse))


def test_window_beyond_its_memory_is_an_error(oracle_lib):
    packed, sc, q, qf, idx, w, wf = _case(5)
    swa_n = np.full(idx.shape[:2], w.shape[1] + 1, np.int32)
    with pytest.raises(oracle.OracleError):
        oracle.swa_sparse_attn(q, packed, sc, idx, w, swa_n, 1.0)
