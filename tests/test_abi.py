"""Host-side checks of the C ABI (no GPU): the library builds for sm_100a,
loads, exports every function include/csa2.h declares, and rejects bad
arguments with a status code before launching anything."""
import ctypes
import os
import re

import pytest

from fp4_kv_cache_step_b200 import build as libbuild
from fp4_kv_cache_step_b200 import csa2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa2.h")


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return csa2.load()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^CSA2_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for required in ("fp4_kv_pack", "fp4_kv_unpack", "csa2_index_score", "csa2_topk",
                     "csa2_sparse_attn", "csa2_layer_step", "csa2_check_device_errors",
                     "csa2_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_binding_covers_every_declared_symbol():
    assert set(declared_functions()) <= set(csa2.EXPORTS)


def _status(rc):
    return csa2.STATUS[rc]


def test_null_and_misaligned_pointers_are_rejected(lib):
    P = ctypes.c_void_p
    rc = lib.fp4_kv_pack(None, 1, 64, 512, P(16), P(32), None)
    assert _status(rc) == "INVALID_ARG"
    assert b"kv" in lib.csa2_last_error()
    rc = lib.fp4_kv_pack(P(16), 1, 64, 512, P(17), P(32), None)
    assert _status(rc) == "INVALID_ARG"
    rc = lib.fp4_kv_pack(P(16), 1, 65, 512, P(16), P(32), None)      # N not a multiple of 64
    assert _status(rc) == "INVALID_ARG"
    rc = lib.fp4_kv_unpack(P(16), P(16), 1, 64, 20, P(16), None)     # D not a multiple of 32
    assert _status(rc) == "INVALID_ARG"


def test_shape_limits_are_rejected(lib):
    P = ctypes.c_void_p
    a = P(256)
    # indexer dimension must be a multiple of 16 and at most 256
    rc = lib.csa2_index_score(a, a, a, 1, 1, 64, 4, 24, a, None, 0, a, None)
    assert _status(rc) == "INVALID_ARG"
    rc = lib.csa2_index_score(a, a, a, 1, 1, 64, 129, 64, a, None, 0, a, None)
    assert _status(rc) == "INVALID_ARG"
    # a pool needs C >= 1
    rc = lib.csa2_index_score(a, a, a, 1, 1, 64, 4, 64, None, a, 0, a, None)
    assert _status(rc) == "INVALID_ARG"
    # top-K bounds
    rc = lib.csa2_topk(a, 64, a, None, 1, 1, 0, a, 0, None, None)
    assert _status(rc) == "INVALID_ARG"
    rc = lib.csa2_topk(a, 64, None, None, 1, 1, 8, a, 0, None, None)
    assert _status(rc) == "INVALID_ARG"
    # attention is built for D = 512
    rc = lib.csa2_sparse_attn(a, a, a, a, 1, 1, 16, 256, 64, 8, ctypes.c_float(1.0), a, None, None,
                              0, None)
    assert _status(rc) == "UNSUPPORTED"


def test_workspace_is_checked_before_launch(lib):
    P = ctypes.c_void_p
    a = P(256)
    need = lib.csa2_sparse_attn_workspace_bytes(2, 1, 64, 512, 2048)
    assert need > 0 and need % 256 == 0
    rc = lib.csa2_sparse_attn(a, a, a, a, 2, 1, 64, 512, 4096, 2048, ctypes.c_float(1.0), a, None,
                              None, 0, None)
    assert _status(rc) == "WORKSPACE"
    # enough rows to give every SM a CTA: no split, whatever K
    assert lib.csa2_sparse_attn_workspace_bytes(4096, 1, 64, 512, 512) == 0
    assert lib.csa2_sparse_attn_workspace_bytes(4096, 1, 64, 512, 2048) == 0
    # 32 rows on 148 SMs: the 2048 entries are split four ways, partial outputs
    # plus (max, sum) per head
    assert lib.csa2_sparse_attn_workspace_bytes(32, 1, 64, 512, 2048) >= 32 * 4 * 64 * 512 * 4


def test_swa_arguments_are_checked(lib):
    P, F = ctypes.c_void_p, ctypes.c_float(1.0)
    a = P(256)
    # no window memory, a negative window, a misaligned window end array
    rc = lib.csa2_sparse_attn_swa(a, a, a, a, None, a, 1, 1, 16, 512, 64, 8, 128, 128, F, a,
                                  None, None, 0, None)
    assert _status(rc) == "INVALID_ARG" and b"swa_kv" in lib.csa2_last_error()
    rc = lib.csa2_sparse_attn_swa(a, a, a, a, a, a, 1, 1, 16, 512, 64, 8, 128, -1, F, a, None,
                                  None, 0, None)
    assert _status(rc) == "INVALID_ARG"
    rc = lib.csa2_sparse_attn_swa(a, a, a, a, a, P(258), 1, 1, 16, 512, 64, 8, 128, 128, F, a,
                                  None, None, 0, None)
    assert _status(rc) == "INVALID_ARG"
    # the window's slots follow the K selected entries: 2 rows of 256 + 128
    # entries split 6 ways where 256 alone split 4 ways
    ws_k = lib.csa2_sparse_attn_workspace_bytes(2, 1, 64, 512, 256)
    ws_kw = lib.csa2_sparse_attn_workspace_bytes(2, 1, 64, 512, 256 + 128)
    assert ws_kw > ws_k > 0
    rc = lib.csa2_sparse_attn_swa(a, a, a, a, a, a, 2, 1, 64, 512, 4096, 256, 300, 128, F, a,
                                  None, a, ws_k, None)
    assert _status(rc) == "WORKSPACE"


def test_layer_args_struct_matches_the_header():
    """The binding's ctypes mirror of csa2_layer_args has the C layout (size
    and the offsets of the window fields), checked by compiling the header."""
    import subprocess
    import tempfile
    src = r"""
#include <stddef.h>
#include <stdio.h>
#include "csa2.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu\n", sizeof(csa2_layer_args), offsetof(csa2_layer_args, swa_kv),
         offsetof(csa2_layer_args, swa_n), offsetof(csa2_layer_args, Tw),
         offsetof(csa2_layer_args, W));
  return 0;
}
"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "layout.c")
        exe = os.path.join(d, "layout")
        with open(c, "w") as f:
            f.write(src)
        subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I",
                        "/usr/local/cuda/include", c, "-o", exe], check=True)
        got = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                               check=True).stdout.split()]
    L = csa2.LayerArgs
    assert got == [ctypes.sizeof(L), L.swa_kv.offset, L.swa_n.offset, L.Tw.offset, L.W.offset]


def test_layer_step_rejects_bad_mode_and_pool(lib):
    sh = csa2.SharedState(256, 256, 256, 256, None, 0)
    args = csa2.LayerArgs(1, 1, 4096, 512, 16, 4, 64, 256, 256, 256, 256, 256, 1.0, 256, None, 1, 0)
    rc = lib.csa2_layer_step(ctypes.byref(args), 7, ctypes.byref(sh), None, 0, None)
    assert _status(rc) == "INVALID_ARG"
    # FULL asked to emit a pool without a pool buffer
    rc = lib.csa2_layer_step(ctypes.byref(args), 0, ctypes.byref(sh), None, 0, None)
    assert _status(rc) == "INVALID_ARG"
    # REUSE needs no indexer inputs but still checks the attention arguments
    args2 = csa2.LayerArgs(1, 1, 4096, 512, 16, 0, 0, 256, 256, 256, None, None, 1.0, 256, None, 0, 0)
    sh2 = csa2.SharedState(256, 256, None, None, None, 0)
    rc = lib.csa2_layer_step(ctypes.byref(args2), 2, ctypes.byref(sh2), None, 0, None)
    assert _status(rc) == "INVALID_ARG" and b"topk_idx" in lib.csa2_last_error()


def test_workspace_query_for_layer_modes(lib):
    sh = csa2.SharedState(256, 256, 256, 256, 256, 8192)
    full = csa2.LayerArgs(4, 1, 262144, 512, 64, 64, 128, 2048, 256, 256, 256, 256, 1.0, 256, None,
                          1, 0)
    b_full = lib.csa2_layer_step_workspace_bytes(ctypes.byref(full), 0, ctypes.byref(sh))
    assert b_full >= 4 * 262144 * 4
    pooled = csa2.LayerArgs(4, 1, 262144, 512, 64, 64, 128, 2048, 256, 256, 256, 256, 1.0, 256,
                            None, 0, 1)
    b_pool = lib.csa2_layer_step_workspace_bytes(ctypes.byref(pooled), 1, ctypes.byref(sh))
    assert 4 * 8192 * 4 <= b_pool < b_full
    b_reuse = lib.csa2_layer_step_workspace_bytes(ctypes.byref(pooled), 2, ctypes.byref(sh))
    assert b_reuse < b_pool


def test_g16_layout_arguments_are_checked(lib):
    P = ctypes.c_void_p
    a = P(256)
    # rows of the 16-channel layout need D % 128 == 0 (8-byte aligned rows)
    assert _status(lib.fp4_kv_pack_g16(a, 1, 64, 96, a, None)) == "INVALID_ARG"
    assert _status(lib.fp4_kv_pack_g16(a, 1, 64, 512, None, None)) == "INVALID_ARG"
    assert _status(lib.fp4_kv_unpack_g16(a, 1, 64, 512, P(8), None)) == "INVALID_ARG"
    assert _status(lib.fp4_kv_append_g16(a, a, 1, -1, 64, 512, a, None)) == "INVALID_ARG"
    assert _status(lib.fp4_kv_append_g16(a, None, 1, 2, 64, 512, a, None)) == "INVALID_ARG"
    # attention over the layout is built for D = 512, like the block layout
    rc = lib.csa2_sparse_attn_g16(a, a, a, 1, 1, 16, 256, 64, 8, ctypes.c_float(1.0), a, None,
                                  None, 0, None)
    assert _status(rc) == "UNSUPPORTED"
    rc = lib.csa2_sparse_attn_g16(a, a, a, 2, 1, 64, 512, 100, 2048, ctypes.c_float(1.0), a, None,
                                  None, 0, None)
    assert _status(rc) == "WORKSPACE"


def test_block_pool_arguments_are_checked(lib):
    P = ctypes.c_void_p
    a = P(256)
    assert _status(lib.csa2_block_pool(a, 100, a, 1, 1, 8, 0, a, a, 1 << 20, None)) == "INVALID_ARG"
    assert _status(lib.csa2_block_pool(a, 100, a, 1, 1, 0, 4, a, a, 1 << 20, None)) == "INVALID_ARG"
    assert _status(lib.csa2_block_pool(a, 100, None, 1, 1, 8, 4, a, a, 1 << 20, None)) == "INVALID_ARG"
    need = lib.csa2_block_pool_workspace_bytes(2, 1, 262144, 8, 2048)
    assert need >= 2 * (32768 * 4 + 2048 * 4)
    assert _status(lib.csa2_block_pool(a, 262144, a, 2, 1, 8, 2048, a, a, need - 256, None)) == \
        "WORKSPACE"


def test_layer_step_blockwise_pool_needs_a_multiple_of_eight(lib):
    sh = csa2.SharedState(256, 256, 256, 256, 256, 8190)
    args = csa2.LayerArgs(1, 1, 4096, 512, 16, 4, 64, 256, 256, 256, 256, 256, 1.0, 256, None, 2, 0)
    rc = lib.csa2_layer_step(ctypes.byref(args), 0, ctypes.byref(sh), None, 0, None)
    assert _status(rc) == "INVALID_ARG" and b"multiple of 8" in lib.csa2_last_error()
    args.emit_pool = 3
    rc = lib.csa2_layer_step(ctypes.byref(args), 0, ctypes.byref(sh), None, 0, None)
    assert _status(rc) == "INVALID_ARG"


def test_header_compiles_as_plain_c(tmp_path):
    """A C caller needs nothing but the header: it compiles as strict C99 with
    no CUDA headers, and every declared call can be referenced."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    names = declared_functions()
    src = tmp_path / "use_header.c"
    src.write_text(
        '#include "csa2.h"\n'
        "typedef void (*any_fn)(void);\n"
        "any_fn table[] = {\n" + "".join("  (any_fn)%s,\n" % n for n in names) + "};\n"
        "int main(void) { return table[0] == 0; }\n")
    rc = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                         "-c", str(src), "-I", os.path.dirname(HEADER),
                         "-o", str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert rc.returncode == 0, rc.stderr
