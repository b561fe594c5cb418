"""csa2_sparse_attn_noalloc, the attention entry point that allocates nothing,
against csa2_sparse_attn (the entry point with a caller workspace).

The file name sorts last so that pytest collects it after every other test:
the shared scratch array then holds whatever earlier calls left in it, and the
test must still pass (it must also pass alone in a fresh process)."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2
from tests.parity_utils import assert_attn_close, assert_lse_close, bf16_dev, dev, host
from tests.test_gpu_parity import _attn_case

NOALLOC_CAP = 32 << 20          # CSA2_NOALLOC_SCRATCH_BYTES in include/csa2.h


def test_noalloc_checks_arguments_and_its_scratch_covers_the_decode_workload():
    """Host-side: bad arguments are reported before any launch (no GPU needed),
    and the split scratch of the 128K decode workload fits the built-in array."""
    libbuild.build()
    L = csa2.load()
    a = ctypes.c_void_p(256)
    rc = L.csa2_sparse_attn_noalloc(a, a, a, a, 1, 1, 16, 256, 64, 8, ctypes.c_float(1.0), a,
                                    None, None)
    assert csa2.STATUS[rc] == "UNSUPPORTED"
    rc = L.csa2_sparse_attn_noalloc(None, a, a, a, 1, 1, 16, 512, 64, 8, ctypes.c_float(1.0), a,
                                    None, None)
    assert csa2.STATUS[rc] == "INVALID_ARG"
    assert 0 < L.csa2_sparse_attn_workspace_bytes(32, 1, 64, 512, 2048) <= NOALLOC_CAP


@pytest.mark.gpu
@pytest.mark.parametrize("B,Tq,Hq,N,K", [(3, 1, 64, 16384, 2048), (2, 2, 128, 4096, 1000),
                                         (32, 1, 64, 4096, 2048)])
def test_noalloc_matches_workspace_entry_point_twice(B, Tq, Hq, N, K):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    libbuild.build()
    L = csa2.load()
    need = L.csa2_sparse_attn_workspace_bytes(B, Tq, Hq, 512, K)
    assert 0 < need <= NOALLOC_CAP            # these shapes split the index list
    scale = 1.0 / math.sqrt(512.0)
    for call in range(2):                     # two calls in a row, different inputs
        packed, sc, q, idx = _attn_case(1000 * call + B + K, B, Tq, Hq, N, K)
        args = (bf16_dev(q), dev(packed), dev(sc), dev(idx), scale)
        out_ws, lse_ws = csa2.csa2_sparse_attn(*args)
        out_na, lse_na = csa2.csa2_sparse_attn_noalloc(*args)
        torch.cuda.synchronize()
        csa2.check_device_errors()
        assert_attn_close(host(out_na), host(out_ws), "noalloc vs workspace, call %d" % call)
        assert_lse_close(host(lse_na), host(lse_ws), "lse, call %d" % call)
    # the last call also agrees with the oracle
    oracle.build()
    want, want_lse = oracle.sparse_attn(q, packed, sc, idx, scale)
    assert_attn_close(host(out_na), want, "noalloc vs oracle")
    assert_lse_close(host(lse_na), want_lse, "noalloc lse vs oracle")
