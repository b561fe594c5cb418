"""GPU parity of the sliding-window branch (csa2_sparse_attn_swa and the
window fields of csa2_layer_step) against the oracle's or_swa_sparse_attn:
one softmax over the selected main-KV rows and the last W tokens of each
row's E4M3 window memory ("Detailed Notes On DeepSeek V4 Point 1 Flash In
Simple Words", sections "The Three Modes Full Reindex And Reuse" and "Model
Setup Numbers Without Jargon": window of 128 tokens; section "FP4 Main KV
Cache To Halve Storage Again" and mengman.github.io 3.5: the window's cache
stays at 8 bits). Covers full, partial (shorter than W, from token 0),
clipped (ending at the memory's last token) and empty windows, empty
selections, both layouts of the main cache, the three attention paths (one
split per row, splits merged inside a cluster, splits merged by the combine
kernel), three softmax scales, and the device-side error records."""
import math

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2
from fp4_kv_cache_step_b200 import workloads as wl
from tests.parity_utils import (assert_attn_close, assert_lse_close, bf16_dev, dev, host,
                                row_vmax)

pytestmark = pytest.mark.gpu

W = oracle.SWA_WINDOW


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


def _swa_case(seed, B, Tq, Hq, N, K, Tw, g16=False):
    """Main cache, queries, selections (some padded, row 0 empty) and window
    memory; the windows' ends cycle through full-from-0, clipped at the end of
    the memory, partial and empty."""
    rng = np.random.default_rng(seed)
    kv = rng.standard_normal((B, N, 512)).astype(np.float32)
    if g16:
        packed, sc = oracle.fp4_kv_pack_g16(kv), None
    else:
        packed, sc = oracle.fp4_kv_pack(kv)
    q = wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / math.sqrt(512))
    idx = np.full((B, Tq, K), -1, np.int32)
    for b in range(B):
        for t in range(Tq):
            m = K if rng.random() > 0.1 else int(rng.integers(0, K))
            m = min(m, N)
            idx[b, t, :m] = np.sort(rng.choice(N, m, replace=False))
    idx[0, 0, :] = -1                                  # a row with nothing selected
    swa = wl._to_e4m3_bytes(rng.standard_normal((B, Tw, 512)).astype(np.float32))
    ends = [min(W, Tw), Tw, min(Tw, 37), 0]
    swa_n = np.array([[ends[(b * Tq + t) % 4] for t in range(Tq)] for b in range(B)], np.int32)
    return packed, sc, q, idx, swa, swa_n


def _values(packed, sc):
    return oracle.fp4_kv_unpack_g16(packed, 512) if sc is None else oracle.fp4_kv_unpack(packed, sc)


def _vmax(packed, sc, idx, swa, swa_n):
    """Largest |v| over each row's selected rows and window tokens."""
    vm = row_vmax(_values(packed, sc), idx)
    wv = np.abs(torch.from_numpy(swa).view(torch.float8_e4m3fn).to(torch.float64).numpy())
    for b in range(idx.shape[0]):
        for t in range(idx.shape[1]):
            hi = swa_n[b, t]
            lo = max(0, hi - W)
            if hi > lo:
                vm[b, t] = max(vm[b, t], wv[b, lo:hi].max())
    return vm


def _run(q, packed, sc, idx, swa, swa_n, scale):
    out, lse = csa2.csa2_sparse_attn_swa(bf16_dev(q), dev(packed),
                                         None if sc is None else dev(sc), dev(idx), dev(swa),
                                         dev(swa_n), scale)
    csa2.check_device_errors()
    return host(out), host(lse)


# (B, Tq, Hq, N, K, Tw): 2 rows -> 6 splits merged in a cluster; 3 rows of
# 2048 + 128 entries -> 34 splits through the combine kernel; 40 rows -> 3
# splits per row; 2 query tokens per row with 128 heads (2 head blocks)
SHAPES = [(2, 1, 64, 4096, 256, 300), (3, 1, 64, 16384, 2048, 256), (40, 1, 64, 4096, 100, 128),
          (1, 2, 128, 2048, 200, 129)]


@pytest.mark.parametrize("B,Tq,Hq,N,K,Tw", SHAPES)
@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 1.0, 24.0])
def test_swa_sparse_attn_matches_oracle(B, Tq, Hq, N, K, Tw, scale):
    packed, sc, q, idx, swa, swa_n = _swa_case(B * 13 + K, B, Tq, Hq, N, K, Tw)
    want, want_lse = oracle.swa_sparse_attn(q, packed, sc, idx, swa, swa_n, scale)
    out, lse = _run(q, packed, sc, idx, swa, swa_n, scale)
    assert_attn_close(out, want, "out", sharp=scale > 4.0,
                      vmax=_vmax(packed, sc, idx, swa, swa_n))
    assert_lse_close(lse, want_lse, "lse")
    # row 0 selects nothing; when its window is empty too the output is 0
    if swa_n[0, 0] == 0:
        assert np.all(out[0, 0] == 0.0) and np.all(np.isneginf(lse[0, 0]))


@pytest.mark.parametrize("ends", ["empty", "full", "clipped"])
def test_window_alone_and_empty_everything(ends):
    """Every selection empty: the window alone decides, and with an empty
    window too the output is 0 and lse is -inf."""
    B, Tq, Hq, N, K, Tw = 4, 1, 64, 1024, 64, 200
    packed, sc, q, _, swa, _ = _swa_case(7, B, Tq, Hq, N, K, Tw)
    idx = np.full((B, Tq, K), -1, np.int32)
    n = {"empty": 0, "full": W, "clipped": Tw}[ends]
    swa_n = np.full((B, Tq), n, np.int32)
    want, want_lse = oracle.swa_sparse_attn(q, packed, sc, idx, swa, swa_n, 1.0)
    out, lse = _run(q, packed, sc, idx, swa, swa_n, 1.0)
    if ends == "empty":
        assert np.all(out == 0.0) and np.all(np.isneginf(lse))
    else:
        assert_attn_close(out, want, "window only", sharp=True,
                          vmax=_vmax(packed, sc, idx, swa, swa_n))
        assert_lse_close(lse, want_lse, "lse")


def test_swa_over_the_16_channel_layout():
    """The 16-channel cache: the oracle's union softmax is formed from its
    two parts (the selection alone and the window alone, each pinned) merged
    by their log-sum-exps, an identity the oracle's own pins establish."""
    B, Tq, Hq, N, K, Tw = 2, 1, 64, 4096, 256, 300
    packed, _, q, idx, swa, swa_n = _swa_case(21, B, Tq, Hq, N, K, Tw, g16=True)
    scale = 1.0
    o1, l1 = oracle.sparse_attn_g16(q, packed, idx, scale)
    # the window alone: an empty selection in a one-block dummy cache
    dummy_p, dummy_s = oracle.fp4_kv_pack(np.zeros((B, 64, 512), np.float32))
    none = np.full((B, Tq, 1), -1, np.int32)
    o2, l2 = oracle.swa_sparse_attn(q, dummy_p, dummy_s, none, swa, swa_n, scale)
    m = np.maximum(l1, l2)
    m = np.where(np.isfinite(m), m, 0.0)
    a1, a2 = np.exp(l1 - m), np.exp(l2 - m)
    z = a1 + a2
    want = np.where(z[..., None] > 0, (a1[..., None] * o1 + a2[..., None] * o2) /
                    np.where(z > 0, z, 1.0)[..., None], 0.0)
    want_lse = np.where(z > 0, m + np.log(np.where(z > 0, z, 1.0)), -np.inf)
    out, lse = _run(q, packed, None, idx, swa, swa_n, scale)
    assert_attn_close(out, want, "g16 + window", sharp=True,
                      vmax=_vmax(packed, None, idx, swa, swa_n))
    assert_lse_close(lse, want_lse, "lse")


def test_window_of_zero_is_the_sparse_attention_bit_for_bit():
    B, Tq, Hq, N, K, Tw = 3, 1, 64, 16384, 2048, 128
    packed, sc, q, idx, swa, swa_n = _swa_case(5, B, Tq, Hq, N, K, Tw)
    args = (bf16_dev(q), dev(packed), dev(sc), dev(idx))
    o1, l1 = csa2.csa2_sparse_attn(*args, 1.0)
    o2, l2 = csa2.csa2_sparse_attn_swa(*args, dev(swa), dev(swa_n), 1.0, W=0)
    csa2.check_device_errors()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_shorter_window_length():
    B, Tq, Hq, N, K, Tw = 2, 2, 64, 2048, 128, 160
    packed, sc, q, idx, swa, swa_n = _swa_case(9, B, Tq, Hq, N, K, Tw)
    want, want_lse = oracle.swa_sparse_attn(q, packed, sc, idx, swa, swa_n, 1.0, W=64)
    out, lse = csa2.csa2_sparse_attn_swa(bf16_dev(q), dev(packed), dev(sc), dev(idx), dev(swa),
                                         dev(swa_n), 1.0, W=64)
    csa2.check_device_errors()
    assert_attn_close(host(out), want, "W=64")
    assert_lse_close(host(lse), want_lse, "lse")


def test_layer_step_with_window_in_every_mode():
    """csa2_layer_step with the window fields: FULL (own top-K) then REUSE,
    each against the oracle's top-K and window attention."""
    w = wl.small(B=2, Tq=1, N=2048, Hq=64, Hi=4, Di=64, K=128)
    nv = wl.nvalid(w)
    kv = wl.kv(w)
    packed, sc = oracle.fp4_kv_pack(kv)
    ik = wl.idx_k(w)
    swa = wl.swa_kv(w)
    swa_n = wl.swa_n(w)
    d_packed, d_sc, d_ik = dev(packed), dev(sc), dev(ik)
    topk = torch.empty((w.B, w.Tq, w.K), dtype=torch.int32, device="cuda")
    shared = csa2.Csa2Shared(d_packed, d_sc, d_ik, topk)
    d_swa, d_n, d_nv = dev(swa), dev(swa_n), dev(nv)
    for layer, mode in enumerate((wl.FULL, wl.REUSE)):
        q = wl.q(w, layer)
        iq, iw = wl.idx_q(w, layer), wl.idx_w(w, layer)
        d_q, d_iq, d_iw = bf16_dev(q), dev(iq), dev(iw)
        out = torch.empty_like(d_q)
        lse = torch.empty((w.B, w.Tq, w.Hq), dtype=torch.float32, device="cuda")
        args = csa2.layer_args(d_q, d_nv, out, w.K, w.softmax_scale, idx_q=d_iq, idx_w=d_iw,
                               lse=lse, N=w.N, swa_kv=d_swa, swa_n=d_n)
        csa2.csa2_layer_step(mode, args, shared)
        csa2.check_device_errors()
        if mode == wl.FULL:
            want_idx = oracle.topk(oracle.index_score(iq, iw, ik, nv), w.K, nv)
            assert np.array_equal(host(topk), want_idx)
        want, want_lse = oracle.swa_sparse_attn(q, packed, sc, host(topk), swa, swa_n,
                                                w.softmax_scale)
        assert_attn_close(host(out), want, "layer %d %s" % (layer, mode))
        assert_lse_close(host(lse), want_lse, "lse layer %d" % layer)


def test_window_end_outside_the_memory_is_recorded_and_empties_that_window():
    B, Tq, Hq, N, K, Tw = 2, 1, 64, 1024, 64, 150
    packed, sc, q, idx, swa, _ = _swa_case(11, B, Tq, Hq, N, K, Tw)
    bad = np.array([[Tw + 1], [W]], np.int32)
    out, lse = csa2.csa2_sparse_attn_swa(bf16_dev(q), dev(packed), dev(sc), dev(idx), dev(swa),
                                         dev(bad), 1.0)
    with pytest.raises(csa2.Csa2Error) as e:
        csa2.check_device_errors()
    assert csa2.STATUS[e.value.status] == "DEVICE_INDEX"
    good = np.array([[0], [W]], np.int32)
    want, want_lse = oracle.swa_sparse_attn(q, packed, sc, idx, swa, good, 1.0)
    assert_attn_close(host(out), want, "emptied window")
    assert_lse_close(host(lse), want_lse, "lse")


def test_nan_byte_in_a_window_row_is_recorded():
    B, Tq, Hq, N, K, Tw = 1, 1, 16, 1024, 64, 128
    packed, sc, q, idx, swa, _ = _swa_case(13, B, Tq, Hq, N, K, Tw)
    swa = swa.copy()
    swa[0, 100, 7] = 0x7F                              # E4M3 NaN
    swa_n = np.full((B, Tq), Tw, np.int32)
    csa2.csa2_sparse_attn_swa(bf16_dev(q), dev(packed), dev(sc), dev(idx), dev(swa), dev(swa_n),
                              1.0)
    with pytest.raises(csa2.Csa2Error) as e:
        csa2.check_device_errors()
    assert csa2.STATUS[e.value.status] == "NONFINITE"
