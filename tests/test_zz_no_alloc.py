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


def test_noalloc_scratch_bound_holds_for_every_shape():
    """The CSA2_ERR_WORKSPACE rejection cannot be reached on a 148-SM B200: the
    split plan gives each SM at most one (row, head block, split) slot of
    64 heads x (512 fp32 partial outputs + an fp32 (max, sum) pair) bytes, and
    148 such slots are 19.5 MB, under the 32 MiB array. The host computes the
    plan for 148 SMs when no GPU is present; this sweeps the shapes around the
    splitting threshold and checks the bound and that the array is never short."""
    libbuild.build()
    L = csa2.load()
    slot = 64 * (512 * 4 + 8)
    worst = 0
    for rows in (1, 2, 3, 4, 5, 7, 8, 9, 16, 18, 19, 37, 73, 74, 75, 147, 148, 149, 300):
        for Tq in (1, 2, 4):
            if rows % Tq:
                continue
            for Hq in (16, 64, 65, 128, 192, 1024):
                for K in (1, 64, 65, 512, 1000, 2048, 8192, 1 << 17):
                    need = L.csa2_sparse_attn_workspace_bytes(rows // Tq, Tq, Hq, 512, K)
                    assert need <= 148 * slot + 256, (rows, Tq, Hq, K, need)
                    worst = max(worst, need)
    assert 0 < worst <= NOALLOC_CAP


# Which cases touch the built-in scratch follows from the split plan for 148
# SMs: a list is split when the (row, head block) pairs are fewer than the SMs,
# and up to 8 splits merge inside a thread-block cluster without scratch.
NOALLOC_CASES = [
    # 3 rows: 49 splits, cut to 32 by the 64-entry tiles -> scratch + combine
    (3, 1, 64, 16384, 2048, True),
    # 4 rows x 2 head blocks: 18 splits, cut to 16 by the tiles -> scratch
    (2, 2, 128, 4096, 1000, True),
    # 32 rows: 4 splits merged in the cluster -> a control that uses no scratch
    (32, 1, 64, 4096, 2048, False),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,Tq,Hq,N,K,uses_scratch", NOALLOC_CASES)
def test_noalloc_matches_workspace_entry_point_twice(B, Tq, Hq, N, K, uses_scratch):
    """Same kernels and split plan as the workspace entry point, so the two
    must agree bit for bit, whether or not the plan goes through scratch."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    libbuild.build()
    L = csa2.load()
    need = L.csa2_sparse_attn_workspace_bytes(B, Tq, Hq, 512, K)
    assert 0 < need <= NOALLOC_CAP            # these shapes split the index list
    slots_over_8 = 9 * B * Tq * ((Hq + 63) // 64)   # slots with more splits than a cluster
    assert (need >= slots_over_8 * 64 * (512 * 4 + 8)) == uses_scratch
    scale = 1.0 / math.sqrt(512.0)
    for call in range(2):                     # two calls in a row, different inputs
        packed, sc, q, idx = _attn_case(1000 * call + B + K, B, Tq, Hq, N, K)
        args = (bf16_dev(q), dev(packed), dev(sc), dev(idx), scale)
        out_ws, lse_ws = csa2.csa2_sparse_attn(*args)
        out_na, lse_na = csa2.csa2_sparse_attn_noalloc(*args)
        torch.cuda.synchronize()
        csa2.check_device_errors()
        assert torch.equal(out_na, out_ws), "noalloc vs workspace output, call %d" % call
        assert torch.equal(lse_na, lse_ws), "noalloc vs workspace lse, call %d" % call
    # the last call also agrees with the oracle
    oracle.build()
    want, want_lse = oracle.sparse_attn(q, packed, sc, idx, scale)
    assert_attn_close(host(out_na), want, "noalloc vs oracle")
    assert_lse_close(host(lse_na), want_lse, "noalloc lse vs oracle")
