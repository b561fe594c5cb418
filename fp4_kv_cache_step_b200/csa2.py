"""Thin Python binding of libcsa2_fp4 (include/csa2.h).

Argument marshalling only: the functions below take torch CUDA tensors, check
their dtype/shape/contiguity, allocate outputs and workspace with torch, and
call the C ABI of the same name on the current torch stream. Every step of the
computation runs in the library's CUDA kernels; there is no fallback. If the
shared library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2_fp4.so")

MODE_FULL, MODE_REINDEX, MODE_REUSE = 0, 1, 2
_MODES = {"FULL": MODE_FULL, "REINDEX": MODE_REINDEX, "REUSE": MODE_REUSE}
STATUS = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "DEVICE_INDEX",
          5: "NONFINITE", 6: "TIMEOUT", 7: "WORKSPACE"}


class Csa2Error(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__("%s (%s)" % (msg, STATUS.get(status, status)))
        self.status = status


class SharedState(ctypes.Structure):
    _fields_ = [("kv_packed", ctypes.c_void_p), ("kv_scale", ctypes.c_void_p),
                ("idx_k", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p),
                ("cand_idx", ctypes.c_void_p), ("C", ctypes.c_int)]


class LayerArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Tq", ctypes.c_int), ("N", ctypes.c_int),
                ("D", ctypes.c_int), ("Hq", ctypes.c_int), ("Hi", ctypes.c_int),
                ("Di", ctypes.c_int), ("K", ctypes.c_int), ("nvalid", ctypes.c_void_p),
                ("q", ctypes.c_void_p), ("idx_q", ctypes.c_void_p), ("idx_w", ctypes.c_void_p),
                ("softmax_scale", ctypes.c_float), ("out", ctypes.c_void_p),
                ("lse", ctypes.c_void_p), ("emit_pool", ctypes.c_int),
                ("use_pool", ctypes.c_int), ("swa_kv", ctypes.c_void_p),
                ("swa_n", ctypes.c_void_p), ("Tw", ctypes.c_int), ("W", ctypes.c_int)]


EXPORTS = ("fp4_kv_pack", "fp4_kv_unpack", "csa2_index_score", "csa2_topk",
           "csa2_sparse_attn_workspace_bytes", "csa2_sparse_attn",
           "csa2_layer_step_workspace_bytes", "csa2_layer_step", "csa2_check_device_errors",
           "csa2_last_error", "csa2_sparse_attn_noalloc", "fp4_kv_pack_g16", "fp4_kv_unpack_g16",
           "fp4_kv_append_g16", "csa2_sparse_attn_g16", "csa2_block_pool_workspace_bytes",
           "csa2_block_pool", "csa2_sparse_attn_swa")

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError("libcsa2_fp4.so not found at %s: build it with "
                           "`python -m fp4_kv_cache_step_b200.build`" % path)
    L = ctypes.CDLL(path)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.fp4_kv_pack.argtypes = [P, I, I, I, P, P, P]
    L.fp4_kv_unpack.argtypes = [P, P, I, I, I, P, P]
    L.csa2_index_score.argtypes = [P, P, P, I, I, I, I, I, P, P, I, P, P]
    L.csa2_topk.argtypes = [P, I, P, P, I, I, I, P, I, P, P]
    L.csa2_sparse_attn_workspace_bytes.argtypes = [I, I, I, I, I]
    L.csa2_sparse_attn_workspace_bytes.restype = Z
    L.csa2_sparse_attn.argtypes = [P, P, P, P, I, I, I, I, I, I, F, P, P, P, Z, P]
    L.csa2_sparse_attn_noalloc.argtypes = [P, P, P, P, I, I, I, I, I, I, F, P, P, P]
    L.fp4_kv_pack_g16.argtypes = [P, I, I, I, P, P]
    L.fp4_kv_unpack_g16.argtypes = [P, I, I, I, P, P]
    L.fp4_kv_append_g16.argtypes = [P, P, I, I, I, I, P, P]
    L.csa2_sparse_attn_g16.argtypes = [P, P, P, I, I, I, I, I, I, F, P, P, P, Z, P]
    L.csa2_sparse_attn_swa.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, P, P, P, Z,
                                       P]
    L.csa2_block_pool_workspace_bytes.argtypes = [I, I, I, I, I]
    L.csa2_block_pool_workspace_bytes.restype = Z
    L.csa2_block_pool.argtypes = [P, I, P, I, I, I, I, P, P, Z, P]
    L.csa2_layer_step_workspace_bytes.argtypes = [ctypes.POINTER(LayerArgs), I,
                                                  ctypes.POINTER(SharedState)]
    L.csa2_layer_step_workspace_bytes.restype = Z
    L.csa2_layer_step.argtypes = [ctypes.POINTER(LayerArgs), I, ctypes.POINTER(SharedState), P, Z, P]
    L.csa2_check_device_errors.argtypes = [P]
    L.csa2_last_error.argtypes = []
    L.csa2_last_error.restype = ctypes.c_char_p
    for f in ("fp4_kv_pack", "fp4_kv_unpack", "csa2_index_score", "csa2_topk", "csa2_sparse_attn",
              "csa2_layer_step", "csa2_check_device_errors", "csa2_sparse_attn_noalloc",
              "fp4_kv_pack_g16", "fp4_kv_unpack_g16", "fp4_kv_append_g16", "csa2_sparse_attn_g16",
              "csa2_block_pool", "csa2_sparse_attn_swa"):
        getattr(L, f).restype = I
    _lib = L
    return L


def _check(rc: int, what: str):
    if rc != 0:
        msg = load().csa2_last_error().decode(errors="replace")
        raise Csa2Error(rc, "%s: %s" % (what, msg))


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _want(t, dtype, name, ndim=None):
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if ndim is not None and t.dim() != ndim:
        raise ValueError("%s must have %d dims, got shape %s" % (name, ndim, tuple(t.shape)))


def check_device_errors():
    """Synchronise the current stream and raise if a kernel recorded a data error."""
    _check(load().csa2_check_device_errors(_stream()), "csa2_check_device_errors")


# ------------------------------------------------------------------- FP4 KV
def fp4_kv_pack(kv: torch.Tensor, packed: Optional[torch.Tensor] = None,
                scale: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """kv float32 [B][N][D] -> (packed uint8 [B][N][D/2], scale uint8 [B][N/64][D])."""
    _want(kv, torch.float32, "kv", 3)
    B, N, D = kv.shape
    if packed is None:
        packed = torch.empty((B, N, D // 2), dtype=torch.uint8, device=kv.device)
    if scale is None:
        scale = torch.empty((B, N // 64, D), dtype=torch.uint8, device=kv.device)
    _check(load().fp4_kv_pack(_p(kv), B, N, D, _p(packed), _p(scale), _stream(kv.device)),
           "fp4_kv_pack")
    return packed, scale


def fp4_kv_unpack(packed: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    _want(packed, torch.uint8, "packed", 3)
    _want(scale, torch.uint8, "scale", 3)
    B, N, Dh = packed.shape
    out = torch.empty((B, N, 2 * Dh), dtype=torch.float32, device=packed.device)
    _check(load().fp4_kv_unpack(_p(packed), _p(scale), B, N, 2 * Dh, _p(out),
                                _stream(packed.device)), "fp4_kv_unpack")
    return out


# ------------------------------------------------------------------- FP4 KV, 16-channel scales
def g16_row_bytes(D: int) -> int:
    """Bytes of one entry in the 16-channel layout: D/2 codes, then D/16 scales."""
    return D // 2 + D // 16


def fp4_kv_pack_g16(kv: torch.Tensor, rows: Optional[torch.Tensor] = None) -> torch.Tensor:
    """kv float32 [B][N][D] -> rows uint8 [B][N][D/2 + D/16]."""
    _want(kv, torch.float32, "kv", 3)
    B, N, D = kv.shape
    if rows is None:
        rows = torch.empty((B, N, g16_row_bytes(D)), dtype=torch.uint8, device=kv.device)
    _check(load().fp4_kv_pack_g16(_p(kv), B, N, D, _p(rows), _stream(kv.device)),
           "fp4_kv_pack_g16")
    return rows


def fp4_kv_unpack_g16(rows: torch.Tensor, D: int) -> torch.Tensor:
    _want(rows, torch.uint8, "rows", 3)
    B, N, rb = rows.shape
    if rb != g16_row_bytes(D):
        raise ValueError("rows of %d bytes do not hold D=%d" % (rb, D))
    out = torch.empty((B, N, D), dtype=torch.float32, device=rows.device)
    _check(load().fp4_kv_unpack_g16(_p(rows), B, N, D, _p(out), _stream(rows.device)),
           "fp4_kv_unpack_g16")
    return out


def fp4_kv_append_g16(rows: torch.Tensor, kv_new: torch.Tensor, pos: torch.Tensor) -> torch.Tensor:
    """Quantise kv_new float32 [B][T][D] into rows[b][pos[b][t]] in place."""
    _want(rows, torch.uint8, "rows", 3)
    _want(kv_new, torch.float32, "kv_new", 3)
    _want(pos, torch.int32, "pos", 2)
    B, T, D = kv_new.shape
    N = rows.shape[1]
    _check(load().fp4_kv_append_g16(_p(kv_new), _p(pos), B, T, N, D, _p(rows),
                                    _stream(rows.device)), "fp4_kv_append_g16")
    return rows


# ------------------------------------------------------------------- indexer
def csa2_index_score(idx_q: torch.Tensor, idx_w: torch.Tensor, idx_k: torch.Tensor,
                     nvalid: Optional[torch.Tensor] = None, cand: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """idx_q uint8 (E4M3) [B][Tq][Hi][Di], idx_w float32 [B][Tq][Hi], idx_k uint8 [B][N][Di]
    -> scores float32 [B][Tq][N] (or [B][Tq][C] with a candidate pool)."""
    _want(idx_q, torch.uint8, "idx_q", 4)
    _want(idx_w, torch.float32, "idx_w", 3)
    _want(idx_k, torch.uint8, "idx_k", 3)
    B, Tq, Hi, Di = idx_q.shape
    N = idx_k.shape[1]
    C = 0
    if cand is not None:
        _want(cand, torch.int32, "cand", 3)
        C = cand.shape[-1]
    elif nvalid is not None:
        _want(nvalid, torch.int32, "nvalid", 2)
    if out is None:
        out = torch.empty((B, Tq, C if cand is not None else N), dtype=torch.float32,
                          device=idx_q.device)
    _check(load().csa2_index_score(_p(idx_q), _p(idx_w), _p(idx_k), B, Tq, N, Hi, Di, _p(nvalid),
                                   _p(cand), C, _p(out), _stream(idx_q.device)), "csa2_index_score")
    return out


def csa2_topk(scores: torch.Tensor, K: int, nvalid: Optional[torch.Tensor] = None,
              cand: Optional[torch.Tensor] = None, Cout: int = 0,
              out: Optional[torch.Tensor] = None, cand_out: Optional[torch.Tensor] = None):
    """scores float32 [B][Tq][ld] -> topk int32 [B][Tq][K] (and the top-Cout pool)."""
    _want(scores, torch.float32, "scores", 3)
    B, Tq, ld = scores.shape
    if out is None:
        out = torch.empty((B, Tq, K), dtype=torch.int32, device=scores.device)
    if Cout and cand_out is None:
        cand_out = torch.empty((B, Tq, Cout), dtype=torch.int32, device=scores.device)
    _check(load().csa2_topk(_p(scores), ld, _p(nvalid), _p(cand), B, Tq, K, _p(out), int(Cout),
                            _p(cand_out), _stream(scores.device)), "csa2_topk")
    return (out, cand_out) if Cout else out


def csa2_block_pool(scores: torch.Tensor, nvalid: torch.Tensor, nblocks: int, block: int = 8,
                    out: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None) -> torch.Tensor:
    """scores float32 [B][Tq][ld] -> the blockwise pool int32 [B][Tq][nblocks * block]."""
    _want(scores, torch.float32, "scores", 3)
    _want(nvalid, torch.int32, "nvalid", 2)
    B, Tq, ld = scores.shape
    L = load()
    if out is None:
        out = torch.empty((B, Tq, nblocks * block), dtype=torch.int32, device=scores.device)
    need = L.csa2_block_pool_workspace_bytes(B, Tq, ld, block, nblocks)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=scores.device)
    _check(L.csa2_block_pool(_p(scores), ld, _p(nvalid), B, Tq, int(block), int(nblocks), _p(out),
                             _p(workspace) if need else None, need, _stream(scores.device)),
           "csa2_block_pool")
    return out


# ------------------------------------------------------------------- attention
def csa2_sparse_attn(q: torch.Tensor, kv_packed: torch.Tensor, kv_scale: torch.Tensor,
                     topk_idx: torch.Tensor, softmax_scale: float, want_lse: bool = True,
                     out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None):
    """q bf16 [B][Tq][Hq][D] -> (out bf16 [B][Tq][Hq][D], lse float32 [B][Tq][Hq] or None)."""
    _want(q, torch.bfloat16, "q", 4)
    _want(topk_idx, torch.int32, "topk_idx", 3)
    B, Tq, Hq, D = q.shape
    N = kv_packed.shape[1]
    K = topk_idx.shape[-1]
    L = load()
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    need = L.csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(L.csa2_sparse_attn(_p(q), _p(kv_packed), _p(kv_scale), _p(topk_idx), B, Tq, Hq, D, N, K,
                              float(softmax_scale), _p(out), _p(lse if want_lse else None),
                              _p(workspace) if need else None, need, _stream(q.device)),
           "csa2_sparse_attn")
    return out, (lse if want_lse else None)


def csa2_sparse_attn_g16(q: torch.Tensor, kv_rows: torch.Tensor, topk_idx: torch.Tensor,
                         softmax_scale: float, want_lse: bool = True,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None):
    """csa2_sparse_attn over a cache in the 16-channel layout (fp4_kv_pack_g16)."""
    _want(q, torch.bfloat16, "q", 4)
    _want(kv_rows, torch.uint8, "kv_rows", 3)
    _want(topk_idx, torch.int32, "topk_idx", 3)
    B, Tq, Hq, D = q.shape
    N = kv_rows.shape[1]
    K = topk_idx.shape[-1]
    L = load()
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    need = L.csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K)
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(L.csa2_sparse_attn_g16(_p(q), _p(kv_rows), _p(topk_idx), B, Tq, Hq, D, N, K,
                                  float(softmax_scale), _p(out), _p(lse if want_lse else None),
                                  _p(workspace) if need else None, need, _stream(q.device)),
           "csa2_sparse_attn_g16")
    return out, (lse if want_lse else None)


SWA_WINDOW = 128   # tokens in the sliding window of every CSA2 layer


def csa2_sparse_attn_swa(q: torch.Tensor, kv_packed: torch.Tensor,
                         kv_scale: Optional[torch.Tensor], topk_idx: torch.Tensor,
                         swa_kv: torch.Tensor, swa_n: torch.Tensor, softmax_scale: float,
                         W: int = SWA_WINDOW, want_lse: bool = True,
                         out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None):
    """csa2_sparse_attn plus the sliding-window branch: one softmax over the
    selected rows and the tokens [max(0, n - W), n) of each row's E4M3 window
    memory swa_kv uint8 [B][Tw][D], n = swa_n int32 [B][Tq]. kv_scale None:
    kv_packed is in the 16-channel layout."""
    _want(q, torch.bfloat16, "q", 4)
    _want(topk_idx, torch.int32, "topk_idx", 3)
    _want(swa_kv, torch.uint8, "swa_kv", 3)
    _want(swa_n, torch.int32, "swa_n", 2)
    B, Tq, Hq, D = q.shape
    N = kv_packed.shape[1]
    K = topk_idx.shape[-1]
    Tw = swa_kv.shape[1]
    L = load()
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    need = L.csa2_sparse_attn_workspace_bytes(B, Tq, Hq, D, K + int(W))
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check(L.csa2_sparse_attn_swa(_p(q), _p(kv_packed), _p(kv_scale), _p(topk_idx), _p(swa_kv),
                                  _p(swa_n), B, Tq, Hq, D, N, K, Tw, int(W),
                                  float(softmax_scale), _p(out), _p(lse if want_lse else None),
                                  _p(workspace) if need else None, need, _stream(q.device)),
           "csa2_sparse_attn_swa")
    return out, (lse if want_lse else None)


def csa2_sparse_attn_noalloc(q: torch.Tensor, kv_packed: torch.Tensor, kv_scale: torch.Tensor,
                             topk_idx: torch.Tensor, softmax_scale: float, want_lse: bool = True,
                             out: Optional[torch.Tensor] = None,
                             lse: Optional[torch.Tensor] = None):
    """csa2_sparse_attn for callers that cannot allocate device memory: the
    library's built-in scratch array stands in for the workspace (outputs are
    still the caller's). Calls that overlap on the GPU must be avoided."""
    _want(q, torch.bfloat16, "q", 4)
    _want(topk_idx, torch.int32, "topk_idx", 3)
    B, Tq, Hq, D = q.shape
    N = kv_packed.shape[1]
    K = topk_idx.shape[-1]
    if out is None:
        out = torch.empty_like(q)
    if want_lse and lse is None:
        lse = torch.empty((B, Tq, Hq), dtype=torch.float32, device=q.device)
    _check(load().csa2_sparse_attn_noalloc(_p(q), _p(kv_packed), _p(kv_scale), _p(topk_idx), B, Tq,
                                           Hq, D, N, K, float(softmax_scale), _p(out),
                                           _p(lse if want_lse else None), _stream(q.device)),
           "csa2_sparse_attn_noalloc")
    return out, (lse if want_lse else None)


class Csa2Shared:
    """Buffers one stack of CSA2 layers shares: the FP4 main KV and indexer keys
    a FULL layer built, and the latest top-K (and candidate pool)."""

    def __init__(self, kv_packed, kv_scale, idx_k, topk_idx, cand_idx=None):
        self.kv_packed, self.kv_scale, self.idx_k = kv_packed, kv_scale, idx_k
        self.topk_idx, self.cand_idx = topk_idx, cand_idx

    def c_struct(self) -> SharedState:
        return SharedState(_p(self.kv_packed), _p(self.kv_scale), _p(self.idx_k),
                           _p(self.topk_idx), _p(self.cand_idx),
                           0 if self.cand_idx is None else int(self.cand_idx.shape[-1]))


def layer_args(q, nvalid, out, K, softmax_scale, idx_q=None, idx_w=None, lse=None, N=None,
               emit_pool=False, use_pool=False, swa_kv=None, swa_n=None,
               W=SWA_WINDOW) -> LayerArgs:
    """emit_pool: False/0 none, True/1 the top-C entries, 2 the blockwise pool.
    swa_kv / swa_n: the sliding-window branch (as in csa2_sparse_attn_swa)."""
    B, Tq, Hq, D = q.shape
    Hi = Di = 0
    if idx_q is not None:
        Hi, Di = idx_q.shape[2], idx_q.shape[3]
    Tw = 0 if swa_kv is None else int(swa_kv.shape[1])
    return LayerArgs(B, Tq, int(N), D, Hq, Hi, Di, int(K), _p(nvalid), _p(q), _p(idx_q),
                     _p(idx_w), float(softmax_scale), _p(out), _p(lse), int(emit_pool),
                     int(bool(use_pool)), _p(swa_kv), _p(swa_n), Tw,
                     int(W) if swa_kv is not None else 0)


def csa2_layer_step(mode, args: LayerArgs, shared: Csa2Shared,
                    workspace: Optional[torch.Tensor] = None, device=None) -> torch.Tensor:
    """Run one CSA2 layer in `mode` ("FULL" | "REINDEX" | "REUSE" or 0/1/2)."""
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    L = load()
    st = shared.c_struct()
    need = L.csa2_layer_step_workspace_bytes(ctypes.byref(args), m, ctypes.byref(st))
    if need and (workspace is None or workspace.numel() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=shared.kv_packed.device)
    _check(L.csa2_layer_step(ctypes.byref(args), m, ctypes.byref(st),
                             _p(workspace) if need else None, need,
                             _stream(shared.kv_packed.device)), "csa2_layer_step")
    return workspace


def layer_step_workspace_bytes(mode, args: LayerArgs, shared: Csa2Shared) -> int:
    m = _MODES[mode] if isinstance(mode, str) else int(mode)
    st = shared.c_struct()
    return int(load().csa2_layer_step_workspace_bytes(ctypes.byref(args), m, ctypes.byref(st)))
