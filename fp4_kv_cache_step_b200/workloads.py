"""Seeded synthetic inputs for the CSA2 step (shared by the tests, the smoke
check and the benchmark; used by both the CUDA path and the CPU oracle).

This module holds no arithmetic of the method: it draws random numbers with
numpy's PCG64 generator and converts them to the storage formats with torch's
own dtype casts (float32 -> bfloat16, small integers -> float8_e4m3fn). Every
tensor has its own stream keyed by (seed, tensor tag, layer, batch row), so a
test can regenerate one batch row of a large workload without the rest.

Workloads (sizes and value distributions the benchmark and the parity tests
use), by name in WORKLOADS:

TINY_DECODE    tiny decode, FULL: B=1, N=4096, 16 query heads, indexer 4 x 64,
               top-256
DECODE_128K    decode at 128K tokens, FULL: B=32, N=32768, 64 heads, indexer
               64 x 128, top-2048, lengths uniform in [16384, 32768]
STACK_4        4-layer stack FULL, REINDEX, REUSE, REUSE: B=16, N=16384
HIER_1M        1M tokens, FULL emitting a top-8192 pool, then REINDEX inside
               the pool: B=4, N=262144
PREFILL_CHUNK  prefill chunk, FULL: 4096 query tokens at the end of N=65536
               entries at 4:1 compression, each query sees entries whose 4
               tokens are all at or before its own position

The model's own shapes ("Model Setup Numbers Without Jargon" in "Detailed
Notes On DeepSeek V4 Point 1 Flash In Simple Words"; mengman.github.io 3.3,
3.4) as a layer stack, `production_stack(T, B)`: of the 40 layers the first 2
use only the sliding window (no CSA2 step); 18 encoder layers at 2 tokens per
entry form three groups [FULL + 5 REUSE], each FULL building its own main KV
and indexer keys; 20 decoder layers at 1 token per entry form [FULL + 3 REUSE]
and four [REINDEX + 3 REUSE] over the decoder FULL's cache, that FULL emitting
the blockwise pool (2048 blocks of 8) which the REINDEX layers score; top-512,
indexer 32 heads x 128, 64 query heads of 512.

Values: main KV ~ N(0, 1) (quantised by the library), queries ~ N(0, 1)/sqrt(512)
rounded to bf16, indexer queries and keys integers uniform in [-4, 4] stored
as E4M3, head weights integers uniform in [1, 4].

The sliding-window branch every CSA2 layer has beside the sparse set (window
of 128 tokens, its cache kept at 8 bits): each layer's window memory holds
the W - 1 tokens before the query block and the block's own Tq tokens, values
~ N(0, 1) rounded to E4M3; query t of a row sees the W tokens ending at its
own (which sits at W - 1 + t): window memory [t, t + W), so swa_n = W + t.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np
import torch

TAG_KV, TAG_IDXK, TAG_Q, TAG_IDXQ, TAG_W, TAG_LEN, TAG_SWA = 1, 2, 3, 4, 5, 6, 7
SWA_WINDOW = 128

FULL, REINDEX, REUSE = "FULL", "REINDEX", "REUSE"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    B: int
    Tq: int
    N: int
    Hq: int
    Hi: int
    Di: int
    K: int
    D: int = 512
    C: int = 0                      # candidate pool size emitted by FULL (0 = none)
    pool_block: int = 1             # 1: the top-C entries; 8: the blockwise pool, C/8 blocks
    modes: Tuple[str, ...] = (FULL,)
    lengths: str = "all"            # "all" | "uniform" | "chunk_end"
    len_lo: int = 0
    len_hi: int = 0
    softmax_scale: float = 1.0 / math.sqrt(512.0)

    @property
    def rows(self) -> int:
        return self.B * self.Tq

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


TINY_DECODE = Workload("tiny_decode_full", 0, B=1, Tq=1, N=4096, Hq=16, Hi=4, Di=64, K=256)
DECODE_128K = Workload("decode_128k_full", 1, B=32, Tq=1, N=32768, Hq=64, Hi=64, Di=128, K=2048,
                       lengths="uniform", len_lo=16384, len_hi=32768)
STACK_4 = Workload("stack_full_reindex_reuse_reuse", 2, B=16, Tq=1, N=16384, Hq=64, Hi=64,
                   Di=128, K=2048, modes=(FULL, REINDEX, REUSE, REUSE))
HIER_1M = Workload("hier_1m_full_pool_reindex", 3, B=4, Tq=1, N=262144, Hq=64, Hi=64, Di=128,
                   K=2048, C=8192, modes=(FULL, REINDEX))
PREFILL_CHUNK = Workload("prefill_chunk_4096_full", 4, B=1, Tq=4096, N=65536, Hq=64, Hi=64,
                         Di=128, K=2048, lengths="chunk_end")
WORKLOADS = {w.name: w for w in (TINY_DECODE, DECODE_128K, STACK_4, HIER_1M, PREFILL_CHUNK)}


def _rng(seed: int, *key: int) -> np.random.Generator:
    return np.random.default_rng([int(seed)] + [int(k) for k in key])


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


# ------------------------------------------------------------ per-row draws
def kv_row(w: Workload, b: int) -> np.ndarray:
    """Unquantised main KV of batch row b: float32 [N][D] ~ N(0, 1)."""
    out = np.empty((w.N, w.D), np.float32)
    _rng(w.seed, TAG_KV, b).standard_normal(out=out, dtype=np.float32)
    return out


def idx_k_row(w: Workload, b: int) -> np.ndarray:
    """Shared indexer keys of batch row b: E4M3 bytes [N][Di], integers in [-4, 4]."""
    ints = _rng(w.seed, TAG_IDXK, b).integers(-4, 5, size=(w.N, w.Di), dtype=np.int8)
    return _to_e4m3_bytes(ints.astype(np.float32))


def q_row(w: Workload, layer: int, b: int) -> np.ndarray:
    """Attention queries: bf16 bits [Tq][Hq][D], N(0, 1)/sqrt(512)."""
    x = _rng(w.seed, TAG_Q, layer, b).standard_normal((w.Tq, w.Hq, w.D), dtype=np.float32)
    x *= np.float32(1.0 / math.sqrt(512.0))
    return _to_bf16_bits(x)


def idx_q_row(w: Workload, layer: int, b: int) -> np.ndarray:
    """Indexer queries: E4M3 bytes [Tq][Hi][Di], integers in [-4, 4]."""
    ints = _rng(w.seed, TAG_IDXQ, layer, b).integers(-4, 5, size=(w.Tq, w.Hi, w.Di), dtype=np.int8)
    return _to_e4m3_bytes(ints.astype(np.float32))


def idx_w_row(w: Workload, layer: int, b: int) -> np.ndarray:
    """Indexer head weights: float32 [Tq][Hi], integers in [1, 4]."""
    return _rng(w.seed, TAG_W, layer, b).integers(1, 5, size=(w.Tq, w.Hi)).astype(np.float32)


def nvalid(w: Workload) -> np.ndarray:
    """Visible entry count per (b, t): int32 [B][Tq]."""
    if w.lengths == "all":
        return np.full((w.B, w.Tq), w.N, np.int32)
    if w.lengths == "uniform":
        lens = _rng(w.seed, TAG_LEN).integers(w.len_lo, w.len_hi + 1, size=w.B)
        return np.repeat(lens[:, None], w.Tq, axis=1).astype(np.int32)
    if w.lengths == "chunk_end":
        # query i sits at token 4N - Tq + i; entry j holds tokens 4j..4j+3 and
        # is visible once all four are at or before the query's token
        i = np.arange(w.Tq, dtype=np.int64)
        tok = 4 * w.N - w.Tq + i
        nv = (tok + 1) // 4
        return np.broadcast_to(nv.astype(np.int32), (w.B, w.Tq)).copy()
    raise ValueError(w.lengths)


def swa_tokens(w: Workload) -> int:
    """Tokens in each row's window memory: the W - 1 before the query block
    and the block's Tq."""
    return w.Tq + SWA_WINDOW - 1


def swa_kv_row(w: Workload, layer: int, b: int) -> np.ndarray:
    """Window memory of batch row b at a layer: E4M3 bytes [Tw][D], N(0, 1)."""
    x = _rng(w.seed, TAG_SWA, layer, b).standard_normal((swa_tokens(w), w.D), dtype=np.float32)
    return _to_e4m3_bytes(x)


def swa_n(w: Workload) -> np.ndarray:
    """End of each query's window in the window memory: int32 [B][Tq], W + t."""
    t = np.arange(w.Tq, dtype=np.int32) + SWA_WINDOW
    return np.broadcast_to(t, (w.B, w.Tq)).copy()


# ------------------------------------------------------------ whole tensors
def _stack(fn, rows, *args):
    first = fn(*args, rows[0])
    out = np.empty((len(rows),) + first.shape, first.dtype)
    out[0] = first
    for i, b in enumerate(rows[1:], 1):
        out[i] = fn(*args, b)
    return out


def kv(w: Workload, rows=None) -> np.ndarray:
    return _stack(lambda b: kv_row(w, b), list(range(w.B)) if rows is None else list(rows))


def idx_k(w: Workload, rows=None) -> np.ndarray:
    return _stack(lambda b: idx_k_row(w, b), list(range(w.B)) if rows is None else list(rows))


def q(w: Workload, layer: int = 0, rows=None) -> np.ndarray:
    return _stack(lambda b: q_row(w, layer, b), list(range(w.B)) if rows is None else list(rows))


def idx_q(w: Workload, layer: int = 0, rows=None) -> np.ndarray:
    return _stack(lambda b: idx_q_row(w, layer, b), list(range(w.B)) if rows is None else list(rows))


def idx_w(w: Workload, layer: int = 0, rows=None) -> np.ndarray:
    return _stack(lambda b: idx_w_row(w, layer, b), list(range(w.B)) if rows is None else list(rows))


def swa_kv(w: Workload, layer: int = 0, rows=None) -> np.ndarray:
    return _stack(lambda b: swa_kv_row(w, layer, b), list(range(w.B)) if rows is None else list(rows))


# ------------------------------------------------------------ the model's stack
PROD_HQ, PROD_HI, PROD_DI, PROD_K = 64, 32, 128, 512
PROD_POOL_BLOCKS, PROD_POOL_BLOCK = 2048, 8
PROD_SWA_ONLY_LAYERS = 2
PROD_ENCODER_GROUPS = 3                             # [FULL + 5 REUSE] each, 2 tokens per entry
PROD_DECODER_GROUPS = 5                             # [FULL|REINDEX + 3 REUSE], 1 token per entry


@dataclasses.dataclass(frozen=True)
class Stack:
    """The CSA2 layers of the model's 40 in order, as segments that each share
    one main KV and indexer-key cache: `segments[i]` is a Workload whose
    `modes` are its layers; `layers` lists (segment, layer in segment) in
    model order; `swa_only` counts the leading layers with no CSA2 step."""
    segments: Tuple[Workload, ...]
    layers: Tuple[Tuple[int, int], ...]
    swa_only: int


def production_stack(T: int, B: int, seed: int = 50, Hq: int = PROD_HQ, Hi: int = PROD_HI,
                     Di: int = PROD_DI, K: int = PROD_K,
                     pool_blocks: int = PROD_POOL_BLOCKS) -> Stack:
    """The model's layer schedule for one decode step at context T tokens
    (T even, T/2 a multiple of 64): encoder caches of T/2 entries (2 tokens
    per entry, all visible to the newest query), a decoder cache of T entries."""
    if T % 128 != 0:
        raise ValueError("T must be a multiple of 128")
    segs = []
    for g in range(PROD_ENCODER_GROUPS):
        segs.append(Workload("prod_encoder_group%d" % g, seed + g, B=B, Tq=1, N=T // 2, Hq=Hq,
                             Hi=Hi, Di=Di, K=K, modes=(FULL,) + (REUSE,) * 5))
    dec_modes = (FULL, REUSE, REUSE, REUSE) + (REINDEX, REUSE, REUSE, REUSE) * (
        PROD_DECODER_GROUPS - 1)
    segs.append(Workload("prod_decoder", seed + PROD_ENCODER_GROUPS, B=B, Tq=1, N=T, Hq=Hq, Hi=Hi,
                         Di=Di, K=K, C=pool_blocks * PROD_POOL_BLOCK,
                         pool_block=PROD_POOL_BLOCK, modes=dec_modes))
    layers = tuple((i, l) for i, w in enumerate(segs) for l in range(len(w.modes)))
    return Stack(tuple(segs), layers, PROD_SWA_ONLY_LAYERS)


def small(name="small", seed=100, B=2, Tq=1, N=1024, Hq=8, Hi=4, Di=64, K=64, D=512, C=0,
          modes=(FULL,), lengths="all", len_lo=0, len_hi=0,
          softmax_scale: Optional[float] = None) -> Workload:
    """A reduced workload with the same value distributions, for parity tests."""
    return Workload(name, seed, B=B, Tq=Tq, N=N, Hq=Hq, Hi=Hi, Di=Di, K=K, D=D, C=C,
                    modes=tuple(modes), lengths=lengths, len_lo=len_lo, len_hi=len_hi,
                    softmax_scale=(1.0 / math.sqrt(512.0)) if softmax_scale is None
                    else float(softmax_scale))
