"""CPU oracle for the CSA2 step over an FP4 main KV cache (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It wraps the plain C oracle in
``csa2_oracle.c`` (double precision, no blocking or fusion) with numpy
marshalling, and shares nothing with the CUDA library. Its definitions follow
"Detailed Notes On DeepSeek V4 Point 1 Flash In Simple Words" (sections on
CSA2, the three modes, the hierarchical indexer and the FP4 main KV cache) and
the mengman.github.io interpretation of the report, sections 3.3-3.5.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa2_oracle.c")
_LIB = os.path.join(_HERE, "libcsa2_oracle.so")

MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2
BLOCK_ENTRIES = 64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into an in-tree shared library."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "csa2_oracle.h"))
    ):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
             "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        L.or_e4m3_value.restype = D
        L.or_e4m3_value.argtypes = [ctypes.c_uint8]
        L.or_e4m3_from_double.restype = ctypes.c_uint8
        L.or_e4m3_from_double.argtypes = [D]
        L.or_e2m1_value.restype = D
        L.or_e2m1_value.argtypes = [ctypes.c_uint8]
        L.or_e2m1_code.restype = ctypes.c_uint8
        L.or_e2m1_code.argtypes = [D, D]
        L.or_bf16_value.restype = D
        L.or_bf16_value.argtypes = [ctypes.c_uint16]
        L.or_fp4_kv_pack.argtypes = [P, I, I, I, P, P]
        L.or_fp4_kv_unpack.argtypes = [P, P, I, I, I, P]
        L.or_fp4_kv_pack_g16.argtypes = [P, I, I, I, P]
        L.or_fp4_kv_unpack_g16.argtypes = [P, I, I, I, P]
        L.or_fp4_kv_append_g16.argtypes = [P, P, I, I, I, I, P]
        L.or_sparse_attn_g16.argtypes = [P, P, P, I, I, I, I, I, I, D, P, P]
        L.or_block_pool.argtypes = [P, I, I, P, I, I, P]
        L.or_swa_sparse_attn.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, D, P, P]
        L.or_index_score.argtypes = [P, P, P, I, I, I, I, I, P, P, I, P]
        L.or_topk.argtypes = [P, I, I, P, P, I, P]
        L.or_sparse_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, D, P, P]
        L.or_dense_attn.argtypes = [P, P, P, P, I, I, I, I, I, D, P, P]
        L.or_layer_step.argtypes = [I, P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, D,
                                    P, P, P, P]
        for f in (L.or_fp4_kv_pack, L.or_fp4_kv_unpack, L.or_index_score, L.or_topk,
                  L.or_sparse_attn, L.or_dense_attn, L.or_layer_step, L.or_fp4_kv_pack_g16,
                  L.or_fp4_kv_unpack_g16, L.or_fp4_kv_append_g16, L.or_sparse_attn_g16,
                  L.or_block_pool, L.or_swa_sparse_attn):
            f.restype = I
        _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _check(rc, what):
    if rc != 0:
        raise OracleError("%s failed with code %d" % (what, rc))


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats
def e4m3_value(code: int) -> float:
    return lib().or_e4m3_value(int(code))


def e4m3_from_double(x: float) -> int:
    return int(lib().or_e4m3_from_double(float(x)))


def e2m1_value(code: int) -> float:
    return lib().or_e2m1_value(int(code))


def e2m1_code(x: float, s: float) -> int:
    return int(lib().or_e2m1_code(float(x), float(s)))


def bf16_value(bits: int) -> float:
    return lib().or_bf16_value(int(bits))


# ---------------------------------------------------------------- FP4 KV
def fp4_kv_pack(kv: np.ndarray):
    """kv float32 [B][N][D] -> (packed u8 [B][N][D/2], scale u8 [B][N/64][D])."""
    kv = _c(kv, np.float32)
    B, N, D = kv.shape
    packed = np.zeros((B, N, D // 2), np.uint8)
    scale = np.zeros((B, N // BLOCK_ENTRIES, D), np.uint8)
    _check(lib().or_fp4_kv_pack(_ptr(kv), B, N, D, _ptr(packed), _ptr(scale)), "or_fp4_kv_pack")
    return packed, scale


def fp4_kv_unpack(packed: np.ndarray, scale: np.ndarray) -> np.ndarray:
    packed = _c(packed, np.uint8)
    scale = _c(scale, np.uint8)
    B, N, Dh = packed.shape
    D = 2 * Dh
    out = np.zeros((B, N, D), np.float64)
    _check(lib().or_fp4_kv_unpack(_ptr(packed), _ptr(scale), B, N, D, _ptr(out)),
           "or_fp4_kv_unpack")
    return out


# ---------------------------------------------------------------- FP4 KV, 16-channel scales
GROUP_CHANNELS = 16


def g16_row_bytes(D: int) -> int:
    """Bytes of one entry in the pages' layout: D/2 code bytes, then D/16 scales."""
    return D // 2 + D // GROUP_CHANNELS


def fp4_kv_pack_g16(kv: np.ndarray) -> np.ndarray:
    """kv float32 [B][N][D] -> rows u8 [B][N][D/2 + D/16] (one E4M3 scale per 16
    channels of an entry, after its codes)."""
    kv = _c(kv, np.float32)
    B, N, D = kv.shape
    rows = np.zeros((B, N, g16_row_bytes(D)), np.uint8)
    _check(lib().or_fp4_kv_pack_g16(_ptr(kv), B, N, D, _ptr(rows)), "or_fp4_kv_pack_g16")
    return rows


def fp4_kv_unpack_g16(rows: np.ndarray, D: int) -> np.ndarray:
    rows = _c(rows, np.uint8)
    B, N, rb = rows.shape
    assert rb == g16_row_bytes(D)
    out = np.zeros((B, N, D), np.float64)
    _check(lib().or_fp4_kv_unpack_g16(_ptr(rows), B, N, D, _ptr(out)), "or_fp4_kv_unpack_g16")
    return out


def fp4_kv_append_g16(rows: np.ndarray, kv_new: np.ndarray, pos: np.ndarray) -> np.ndarray:
    """A copy of `rows` with kv_new[b][t] (float32 [B][T][D]) quantised into
    row pos[b][t]."""
    out = np.array(rows, dtype=np.uint8, copy=True, order="C")
    kv_new = _c(kv_new, np.float32)
    pos = _c(pos, np.int32)
    B, T, D = kv_new.shape
    N = out.shape[1]
    _check(lib().or_fp4_kv_append_g16(_ptr(kv_new), _ptr(pos), B, T, N, D, _ptr(out)),
           "or_fp4_kv_append_g16")
    return out


def sparse_attn_g16(q_bf16, rows, idx, softmax_scale):
    """Sparse attention over a cache in the 16-channel layout; as sparse_attn."""
    q_bf16 = _c(q_bf16, np.uint16)
    rows = _c(rows, np.uint8)
    idx = _c(idx, np.int32)
    B, Tq, Hq, D = q_bf16.shape
    N = rows.shape[1]
    K = idx.shape[2]
    out = np.zeros((B, Tq, Hq, D), np.float64)
    lse = np.zeros((B, Tq, Hq), np.float64)
    _check(lib().or_sparse_attn_g16(_ptr(q_bf16), _ptr(rows), _ptr(idx), B, Tq, Hq, D, N, K,
                                    float(softmax_scale), _ptr(out), _ptr(lse)),
           "or_sparse_attn_g16")
    return out, lse


# ---------------------------------------------------------------- indexer
def index_score(idx_q, idx_w, idx_k, nvalid=None, cand=None) -> np.ndarray:
    """idx_q u8 [B][Tq][Hi][Di], idx_w f32 [B][Tq][Hi], idx_k u8 [B][N][Di] ->
    float64 [B][Tq][N] (or [B][Tq][C] with a candidate pool)."""
    idx_q = _c(idx_q, np.uint8)
    idx_w = _c(idx_w, np.float32)
    idx_k = _c(idx_k, np.uint8)
    B, Tq, Hi, Di = idx_q.shape
    N = idx_k.shape[1]
    nv = None if nvalid is None else _c(nvalid, np.int32)
    cd = None if cand is None else _c(cand, np.int32)
    C = 0 if cd is None else cd.shape[-1]
    out = np.zeros((B, Tq, C if cd is not None else N), np.float64)
    _check(lib().or_index_score(_ptr(idx_q), _ptr(idx_w), _ptr(idx_k), B, Tq, N, Hi, Di,
                                _ptr(nv), _ptr(cd), C, _ptr(out)), "or_index_score")
    return out


def topk(scores, K, nvalid=None, cand=None) -> np.ndarray:
    """scores [..., ld] (float64) -> int32 [..., K], ascending ids, -1 padded."""
    scores = _c(scores, np.float64)
    lead = scores.shape[:-1]
    ld = scores.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    nv = None if nvalid is None else _c(nvalid, np.int32)
    cd = None if cand is None else _c(cand, np.int32)
    out = np.zeros(lead + (K,), np.int32)
    _check(lib().or_topk(_ptr(scores), rows, ld, _ptr(nv), _ptr(cd), K, _ptr(out)), "or_topk")
    return out


def block_pool(scores, nvalid, block: int, nblocks: int) -> np.ndarray:
    """scores [..., ld] (float64), nvalid [...] -> int32 [..., nblocks*block]:
    the valid positions of the best `nblocks` blocks of `block` positions
    (block score = max over its valid positions), ascending, -1 padded."""
    scores = _c(scores, np.float64)
    lead = scores.shape[:-1]
    ld = scores.shape[-1]
    rows = int(np.prod(lead)) if lead else 1
    nv = _c(nvalid, np.int32)
    out = np.zeros(lead + (nblocks * block,), np.int32)
    _check(lib().or_block_pool(_ptr(scores), rows, ld, _ptr(nv), int(block), int(nblocks),
                               _ptr(out)), "or_block_pool")
    return out


# ---------------------------------------------------------------- attention
def sparse_attn(q_bf16, packed, scale, idx, softmax_scale):
    """q bf16 bits u16 [B][Tq][Hq][D], idx i32 [B][Tq][K] -> (out f64, lse f64)."""
    q_bf16 = _c(q_bf16, np.uint16)
    packed = _c(packed, np.uint8)
    scale = _c(scale, np.uint8)
    idx = _c(idx, np.int32)
    B, Tq, Hq, D = q_bf16.shape
    N = packed.shape[1]
    K = idx.shape[-1]
    out = np.zeros((B, Tq, Hq, D), np.float64)
    lse = np.zeros((B, Tq, Hq), np.float64)
    _check(lib().or_sparse_attn(_ptr(q_bf16), _ptr(packed), _ptr(scale), _ptr(idx), B, Tq, Hq,
                                D, N, K, float(softmax_scale), _ptr(out), _ptr(lse)),
           "or_sparse_attn")
    return out, lse


SWA_WINDOW = 128


def swa_sparse_attn(q_bf16, packed, scale, idx, swa_kv, swa_n, softmax_scale, W=SWA_WINDOW):
    """Sparse attention plus the sliding-window branch, one softmax over both:
    swa_kv u8 (E4M3) [B][Tw][D], swa_n i32 [B][Tq] (query sees window tokens
    [max(0, swa_n - W), swa_n))."""
    q_bf16 = _c(q_bf16, np.uint16)
    packed = _c(packed, np.uint8)
    scale = _c(scale, np.uint8)
    idx = _c(idx, np.int32)
    swa_kv = _c(swa_kv, np.uint8)
    swa_n = _c(swa_n, np.int32)
    B, Tq, Hq, D = q_bf16.shape
    N = packed.shape[1]
    K = idx.shape[-1]
    Tw = swa_kv.shape[1]
    out = np.zeros((B, Tq, Hq, D), np.float64)
    lse = np.zeros((B, Tq, Hq), np.float64)
    _check(lib().or_swa_sparse_attn(_ptr(q_bf16), _ptr(packed), _ptr(scale), _ptr(idx),
                                    _ptr(swa_kv), _ptr(swa_n), B, Tq, Hq, D, N, K, Tw, int(W),
                                    float(softmax_scale), _ptr(out), _ptr(lse)),
           "or_swa_sparse_attn")
    return out, lse


def dense_attn(q_bf16, packed, scale, nvalid, softmax_scale):
    q_bf16 = _c(q_bf16, np.uint16)
    packed = _c(packed, np.uint8)
    scale = _c(scale, np.uint8)
    nvalid = _c(nvalid, np.int32)
    B, Tq, Hq, D = q_bf16.shape
    N = packed.shape[1]
    out = np.zeros((B, Tq, Hq, D), np.float64)
    lse = np.zeros((B, Tq, Hq), np.float64)
    _check(lib().or_dense_attn(_ptr(q_bf16), _ptr(packed), _ptr(scale), _ptr(nvalid), B, Tq,
                               Hq, D, N, float(softmax_scale), _ptr(out), _ptr(lse)),
           "or_dense_attn")
    return out, lse


def layer_step(mode, q_bf16, idx_q, idx_w, idx_k, packed, scale, nvalid, K,
               softmax_scale, topk_io, cand_io=None, C=0, use_pool=False):
    """One CSA2 layer. ``topk_io`` (int32 [B][Tq][K]) is written by FULL and
    REINDEX and read by REUSE; ``cand_io`` ([B][Tq][C]) is written by FULL when
    C > 0 and read by a pooled REINDEX. Returns (out f64, lse f64)."""
    q_bf16 = _c(q_bf16, np.uint16)
    B, Tq, Hq, D = q_bf16.shape
    N = packed.shape[1]
    packed = _c(packed, np.uint8)
    scale = _c(scale, np.uint8)
    if mode == MODE_REUSE:
        Hi = Di = 1
        idx_q = np.zeros(1, np.uint8)
        idx_w = np.zeros(1, np.float32)
        idx_k = np.zeros(1, np.uint8) if idx_k is None else _c(idx_k, np.uint8)
    else:
        idx_q = _c(idx_q, np.uint8)
        idx_w = _c(idx_w, np.float32)
        idx_k = _c(idx_k, np.uint8)
        Hi, Di = idx_q.shape[2], idx_q.shape[3]
    nvalid = _c(nvalid, np.int32)
    assert topk_io.dtype == np.int32 and topk_io.flags["C_CONTIGUOUS"]
    if cand_io is not None:
        assert cand_io.dtype == np.int32 and cand_io.flags["C_CONTIGUOUS"]
    out = np.zeros((B, Tq, Hq, D), np.float64)
    lse = np.zeros((B, Tq, Hq), np.float64)
    _check(lib().or_layer_step(int(mode), _ptr(q_bf16), _ptr(idx_q), _ptr(idx_w), _ptr(idx_k),
                               _ptr(packed), _ptr(scale), _ptr(nvalid), B, Tq, N, D, Hq, Hi, Di,
                               K, int(C), int(bool(use_pool)), float(softmax_scale),
                               _ptr(topk_io), _ptr(cand_io), _ptr(out), _ptr(lse)),
           "or_layer_step")
    return out, lse
