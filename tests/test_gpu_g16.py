"""GPU parity of the 16-channel-scale FP4 layout (the pages' own: one E4M3
scale per 16 channels of an entry, no global scale; "FP4 Main KV Cache To
Halve Storage Again", mengman.github.io 3.5) against the oracle: pack, unpack
and append bit-exact, sparse attention within the attention tolerance, and
bit-equal to the block layout's kernel where both layouts hold the same values."""
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

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


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


def _kv(seed, B, N, D):
    rng = np.random.default_rng(seed)
    kv = rng.standard_normal((B, N, D)).astype(np.float32)
    kv[0, 0, 16:32] = 0.0                        # an all-zero group
    if N > 1:
        kv[0, 1, 0:16] *= np.float32(1e-4)      # a tiny group
    kv[-1, -1, -16:] *= np.float32(800.0)       # a group whose scale saturates
    return kv


@pytest.mark.parametrize("B,N,D", [(2, 100, 512), (1, 3, 128), (3, 64, 256)])
def test_pack_g16_bit_exact(B, N, D):
    kv = _kv(B * 1000 + N, B, N, D)
    want = oracle.fp4_kv_pack_g16(kv)
    rows = csa2.fp4_kv_pack_g16(dev(kv))
    assert np.array_equal(host(rows), want)
    back = csa2.fp4_kv_unpack_g16(rows, D)
    assert np.array_equal(host(back).astype(np.float64), oracle.fp4_kv_unpack_g16(want, D))


def test_append_g16_bit_exact_and_flags_bad_positions():
    B, N, D, T = 2, 96, 512, 4
    kv = _kv(5, B, N, D)
    rng = np.random.default_rng(6)
    pos = np.stack([rng.choice(N, T, replace=False) for _ in range(B)]).astype(np.int32)
    base = kv.copy()
    for b in range(B):
        base[b, pos[b]] = 0.0
    new = np.stack([kv[b, pos[b]] for b in range(B)])
    rows = csa2.fp4_kv_pack_g16(dev(base))
    csa2.fp4_kv_append_g16(rows, dev(new), dev(pos))
    want = oracle.fp4_kv_append_g16(oracle.fp4_kv_pack_g16(base), new, pos)
    assert np.array_equal(host(rows), want)
    assert np.array_equal(host(rows), oracle.fp4_kv_pack_g16(kv))
    bad = pos.copy()
    bad[1, 2] = N
    before = host(rows).copy()
    csa2.fp4_kv_append_g16(rows, dev(new), dev(bad))
    with pytest.raises(csa2.Csa2Error) as ei:
        csa2.check_device_errors()
    assert ei.value.status == 4
    assert np.array_equal(host(rows), before)   # the same values again; the bad one skipped


def test_pack_g16_flags_nonfinite():
    kv = np.zeros((1, 4, 128), np.float32)
    kv[0, 2, 77] = np.nan
    csa2.fp4_kv_pack_g16(dev(kv))
    with pytest.raises(csa2.Csa2Error) as ei:
        csa2.check_device_errors()
    assert ei.value.status == 5


def _case(seed, B, Tq, Hq, N, K, pad_frac=0.1):
    rng = np.random.default_rng(seed)
    kv = rng.standard_normal((B, N, 512)).astype(np.float32)
    rows = oracle.fp4_kv_pack_g16(kv)
    q = wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / math.sqrt(512))
    idx = np.full((B, Tq, K), -1, np.int32)
    for b in range(B):
        for t in range(Tq):
            m = K if rng.random() > pad_frac else int(rng.integers(0, K))
            m = min(m, N)
            idx[b, t, :m] = np.sort(rng.choice(N, m, replace=False))
    return rows, q, idx


# one CTA per row (Tq = 3 rows, nothing to split), splits merged in a cluster
# (2 rows, 4 splits; 40 rows, ragged), splits merged by the combine kernel
# (3 rows, 32 splits), 48 heads (a partial head block)
@pytest.mark.parametrize("B,Tq,Hq,N,K", [(1, 3, 48, 1000, 64), (2, 1, 64, 4096, 256),
                                         (40, 1, 64, 4100, 100), (3, 1, 64, 16384, 2048)])
@pytest.mark.parametrize("scale", [1.0 / math.sqrt(512.0), 24.0])
def test_sparse_attn_g16_within_tolerance(B, Tq, Hq, N, K, scale):
    rows, q, idx = _case(B * 13 + K, B, Tq, Hq, N, K)
    idx[0, 0, :] = -1                            # a row with nothing selected
    want, want_lse = oracle.sparse_attn_g16(q, rows, idx, scale)
    out, lse = csa2.csa2_sparse_attn_g16(bf16_dev(q), dev(rows), dev(idx), scale)
    assert_attn_close(host(out), want, "out", sharp=scale > 4.0,
                      vmax=row_vmax(oracle.fp4_kv_unpack_g16(rows, 512), idx))
    assert_lse_close(host(lse), want_lse, "lse")
    assert np.all(host(out)[0, 0] == 0.0)


def test_sparse_attn_g16_decode_128k_sampled_rows():
    """The 128K decode shape (32 rows, N = 32768, K = 2048, 64 heads; four
    splits merged in a cluster): every row on the GPU, rows 0, 17, 31 against
    the oracle."""
    B, Hq, N, K = 32, 64, 32768, 2048
    rng = np.random.default_rng(99)
    kv = rng.standard_normal((B, N, 512), dtype=np.float32)
    rows_d = csa2.fp4_kv_pack_g16(dev(kv))
    q = wl._to_bf16_bits(rng.standard_normal((B, 1, Hq, 512)).astype(np.float32) / math.sqrt(512))
    idx = np.stack([np.sort(rng.choice(N, K, replace=False)) for _ in range(B)])[:, None, :]
    idx = idx.astype(np.int32)
    out, lse = csa2.csa2_sparse_attn_g16(bf16_dev(q), rows_d, dev(idx), 1.0 / math.sqrt(512.0))
    out_h, lse_h = host(out), host(lse)
    rows_h = host(rows_d)
    for b in (0, 17, 31):
        want, want_lse = oracle.sparse_attn_g16(q[b:b + 1], rows_h[b:b + 1], idx[b:b + 1],
                                                1.0 / math.sqrt(512.0))
        assert_attn_close(out_h[b:b + 1], want, "out b=%d" % b)
        assert_lse_close(lse_h[b:b + 1], want_lse, "lse b=%d" % b)


def test_sparse_attn_g16_equals_block_layout_where_values_agree():
    """Grid values times one scale, with +-6 s in every 16-channel group of
    every entry and every 64-entry block of every channel: both layouts store
    the same codes and scales, so the two kernels see the same dequantised
    values and must give the same bits."""
    B, Tq, Hq, N, K = 4, 1, 64, 1024, 512
    rng = np.random.default_rng(7)
    vals = GRID[rng.integers(0, 8, (B, N, 512))] * np.where(rng.random((B, N, 512)) < 0.5, -1, 1)
    n = np.arange(N)[:, None]
    c = np.arange(512)[None, :]
    vals[:, (n + c) % 16 == 0] = 6.0
    kv = (vals * 0.5).astype(np.float32)
    rows = csa2.fp4_kv_pack_g16(dev(kv))
    packed, sc = csa2.fp4_kv_pack(dev(kv))
    q = wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / math.sqrt(512))
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(B)])[:, None, :].astype(np.int32)
    for scale in (1.0 / math.sqrt(512.0), 8.0):
        a, la = csa2.csa2_sparse_attn_g16(bf16_dev(q), rows, dev(idx), scale)
        b, lb = csa2.csa2_sparse_attn(bf16_dev(q), packed, sc, dev(idx), scale)
        assert torch.equal(a, b) and torch.equal(la, lb)


def test_layer_step_modes_over_g16_cache():
    """FULL then REUSE through csa2_layer_step with the cache in the 16-channel
    layout (a NULL block-scale pointer selects it): the top-K matches the
    oracle's bit for bit and the outputs match the oracle's attention over the
    same rows."""
    B, Tq, N, Hq, Hi, Di, K = 2, 1, 4096, 16, 4, 64, 256
    rng = np.random.default_rng(31)
    kv = rng.standard_normal((B, N, 512), dtype=np.float32)
    rows_h = oracle.fp4_kv_pack_g16(kv)
    e4m3 = lambda x: torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()
    idx_q = e4m3(rng.integers(-4, 5, (B, Tq, Hi, Di)))
    idx_k = e4m3(rng.integers(-4, 5, (B, N, Di)))
    idx_w = rng.integers(1, 5, (B, Tq, Hi)).astype(np.float32)
    nvalid = np.array([[N], [3000]], np.int32)
    scale = 1.0 / math.sqrt(512.0)
    q_full = wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / 22.6)
    q_reuse = wl._to_bf16_bits(rng.standard_normal((B, Tq, Hq, 512)).astype(np.float32) / 22.6)
    want_idx = oracle.topk(oracle.index_score(idx_q, idx_w, idx_k, nvalid), K, nvalid)

    rows = dev(rows_h)
    topk = torch.full((B, Tq, K), -1, dtype=torch.int32, device="cuda")
    shared = csa2.Csa2Shared(rows, None, dev(idx_k), topk)
    nv = dev(nvalid)
    for mode, qb in (("FULL", q_full), ("REUSE", q_reuse)):
        out = torch.empty((B, Tq, Hq, 512), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device="cuda")
        q_d = bf16_dev(qb)
        args = csa2.layer_args(q_d, nv, out, K, scale, idx_q=dev(idx_q) if mode == "FULL" else None,
                               idx_w=dev(idx_w) if mode == "FULL" else None, lse=lse, N=N)
        csa2.csa2_layer_step(mode, args, shared)
        assert np.array_equal(host(topk), want_idx)
        want, want_lse = oracle.sparse_attn_g16(qb, rows_h, want_idx, scale)
        assert_attn_close(host(out), want, "out %s" % mode)
        assert_lse_close(host(lse), want_lse, "lse %s" % mode)
