"""GPU parity of the model's own CSA2 layer stack at reduced context: the 38
CSA2 layers of workloads.production_stack (three encoder groups [FULL + 5
REUSE] at 2 tokens per entry, the decoder's [FULL + 3 REUSE] + 4 x [REINDEX +
3 REUSE] at 1 token per entry with the blockwise pool), top-512 and 32 x 128
indexer heads, run through csa2_layer_step and compared layer by layer with
the oracle's composition of the pinned steps (score, top-K, blockwise pool,
attention)."""
import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2
from fp4_kv_cache_step_b200 import workloads as wl
from fp4_kv_cache_step_b200.runner import DeviceStack
from tests.parity_utils import assert_attn_close, assert_lse_close, host

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


def _oracle_segment(w, b):
    """(topk, pool, out, lse) per layer of one segment, batch row b."""
    packed, sc = oracle.fp4_kv_pack(wl.kv(w, rows=[b]))
    ik = wl.idx_k(w, rows=[b])
    nv = wl.nvalid(w)[b:b + 1]
    topk = pool = None
    res = []
    for layer, mode in enumerate(w.modes):
        if mode in (wl.FULL, wl.REINDEX):
            iq, iw = wl.idx_q(w, layer, rows=[b]), wl.idx_w(w, layer, rows=[b])
            if mode == wl.REINDEX and pool is not None:
                topk = oracle.topk(oracle.index_score(iq, iw, ik, cand=pool), w.K, cand=pool)
            else:
                s = oracle.index_score(iq, iw, ik, nv)
                topk = oracle.topk(s, w.K, nv)
                if mode == wl.FULL and w.C:
                    pool = oracle.block_pool(s, nv, w.pool_block, w.C // w.pool_block)
        out, lse = oracle.sparse_attn(wl.q(w, layer, rows=[b]), packed, sc, topk, w.softmax_scale)
        res.append((topk, pool, out, lse))
    return res


def test_production_stack_reduced_context():
    # 16384 tokens: encoder caches of 8192 entries, a decoder cache of 16384
    # with a pool of 512 blocks of 8 (a quarter of it), batch 2
    st = wl.production_stack(16384, 2, pool_blocks=512)
    ds = DeviceStack(st)
    ds.step(snapshot_topk=True)
    torch.cuda.synchronize()
    csa2.check_device_errors()
    for si, w in enumerate(st.segments):
        dw = ds.segments[si]
        for b in range(w.B):
            want = _oracle_segment(w, b)
            for layer, (topk, pool, out, lse) in enumerate(want):
                what = "%s layer %d (%s) b=%d" % (w.name, layer, w.modes[layer], b)
                assert np.array_equal(host(dw.topk_per_layer[layer][b]), topk[0]), what
                assert_attn_close(host(dw.out[layer][b]), out[0], "out " + what)
                assert_lse_close(host(dw.lse[layer][b]), lse[0], "lse " + what)
            if w.C:
                assert np.array_equal(host(dw.cand[b]), want[-1][1][0]), w.name
