"""Parity at the benchmark workloads' full sizes, in the launch configuration
the benchmark times (the whole batch through csa2_layer_step), checked on
sampled batch rows / query tokens that the oracle computes one by one: packed
bytes and top-K indices bit for bit, outputs within tolerance."""
import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2
from fp4_kv_cache_step_b200 import workloads as wl
from fp4_kv_cache_step_b200.runner import DeviceWorkload
from tests.parity_utils import assert_attn_close, assert_lse_close, host
from tests.test_gpu_parity import _check_stack, _oracle_stack

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    libbuild.build()
    csa2.load()
    oracle.build()


def _run(w):
    dw = DeviceWorkload(w)
    dw.step(snapshot_topk=True)
    csa2.check_device_errors()
    return dw


@pytest.mark.parametrize("name,rows", [("decode_128k_full", [0, 13, 31]),
                                       ("stack_full_reindex_reuse_reuse", [0, 15]),
                                       ("hier_1m_full_pool_reindex", [2])])
def test_full_size_workload(name, rows):
    w = wl.WORKLOADS[name]
    dw = _run(w)
    _check_stack(w, dw, _oracle_stack(w, rows), rows)
    # every row's indices are valid: ascending, inside [0, nvalid), -1 only as padding
    nv = wl.nvalid(w)
    for layer in range(len(w.modes)):
        tk = host(dw.topk_per_layer[layer]).reshape(-1, w.K)
        for r in range(tk.shape[0]):
            v = tk[r][tk[r] >= 0]
            assert np.all(np.diff(v) > 0) and v.size == min(w.K, nv.reshape(-1)[r])
            assert v.size == 0 or v[-1] < nv.reshape(-1)[r]
    del dw
    torch.cuda.empty_cache()


def test_full_size_prefill_chunk_sampled_queries():
    w = wl.PREFILL_CHUNK
    dw = _run(w)
    tsel = [0, 1, 3, 4, 2047, 4095]
    packed, sc = oracle.fp4_kv_pack(wl.kv(w, rows=[0]))
    assert np.array_equal(host(dw.kv_packed[0]), packed[0])
    assert np.array_equal(host(dw.kv_scale[0]), sc[0])
    ik = wl.idx_k(w, rows=[0])
    q = wl.q(w, 0, rows=[0])[:, tsel]
    iq = wl.idx_q(w, 0, rows=[0])[:, tsel]
    iw = wl.idx_w(w, 0, rows=[0])[:, tsel]
    nv = wl.nvalid(w)[:, tsel]
    topk = np.full((1, len(tsel), w.K), -1, np.int32)
    out, lse = oracle.layer_step(oracle.MODE_FULL, q, iq, iw, ik, packed, sc, nv, w.K,
                                 w.softmax_scale, topk)
    got_tk = host(dw.topk)[0, tsel]
    assert np.array_equal(got_tk, topk[0])
    assert_attn_close(host(dw.out[0])[0, tsel], out[0], "prefill out")
    assert_lse_close(host(dw.lse[0])[0, tsel], lse[0], "prefill lse")
    # causal mask: every selected entry is visible to its query
    tk_all = host(dw.topk)[0]
    nv_all = wl.nvalid(w)[0]
    assert np.all(tk_all.max(axis=1) < nv_all)
    del dw
    torch.cuda.empty_cache()
