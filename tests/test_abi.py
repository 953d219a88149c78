"""C-ABI library: loads, exports every declared symbol, host-side logic.

No compute call is made here (these run without a GPU): only size helpers and
argument checks that fail before any CUDA call.
"""
import ctypes
import os
import re

import pytest

import oracle as O
from block_sparse_attention_stats_b200 import _lib as L
from block_sparse_attention_stats_b200.build import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "pisa.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return L.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pisa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
        assert n in L.SIGNATURES, f"binding lacks a prototype for {n}"


def test_num_blocks_and_selected_match_oracle(lib):
    for L_, b in ((1, 64), (64, 64), (65, 64), (75600, 64), (119056, 64)):
        assert lib.pisa_num_blocks(L_, b) == O.block_partition(L_, b)[0]
    for N in (1, 2, 7, 16, 72, 1182, 1861):
        for dens in (0.01, 0.05, 0.1, 0.125, 0.15, 0.25, 0.5, 1.0):
            assert lib.pisa_num_selected(N, dens) == O.num_selected(N, dens)
    assert lib.pisa_num_selected(10, 0.0) == -1
    assert lib.pisa_num_selected(10, 1.01) == -1
    assert lib.pisa_num_blocks(0, 64) == -1


def test_selection_workspace_holds_the_score_matrix(lib):
    """The selection scratch holds the float32 score matrix of the two-pass path."""
    for BH, N in ((40, 1182), (24, 1861), (24, 72), (1, 4205), (3, 600)):
        need = lib.pisa_select_workspace_bytes(1, BH, N)
        assert need >= BH * N * N * 4
        assert need % 256 == 0


def test_workspace_sizes(lib):
    w = lib.pisa_workspace_bytes(1, 40, 75600, 128, 64, 0.125, L.PISA_BF16, 0)
    assert w > 0 and w % 256 == 0
    # covariance and f32 inputs need more scratch
    assert lib.pisa_workspace_bytes(1, 24, 4608, 128, 64, 0.15, L.PISA_BF16, 1) > \
        lib.pisa_workspace_bytes(1, 24, 4608, 128, 64, 0.15, L.PISA_BF16, 0)
    assert lib.pisa_workspace_bytes(1, 2, 1024, 64, 64, 0.25, L.PISA_F32, 0) > \
        lib.pisa_workspace_bytes(1, 2, 1024, 64, 64, 0.25, L.PISA_BF16, 0)
    # unsupported shapes report 0
    assert lib.pisa_workspace_bytes(1, 1, 1024, 96, 64, 0.25, L.PISA_BF16, 0) == 0
    assert lib.pisa_workspace_bytes(1, 1, 1024, 128, 32, 0.25, L.PISA_BF16, 0) == 0
    assert lib.pisa_workspace_bytes(1, 1, 1024, 128, 128, 0.25, L.PISA_BF16, 0) > 0
    assert lib.pisa_sparse_attention_bwd_workspace_bytes(1, 1, 1024, 128, 128, 4) > 0
    assert lib.pisa_sparse_attention_bwd_workspace_bytes(1, 1, 1024, 128, 128, 9) == 0
    assert lib.pisa_sparse_attention_bwd_workspace_bytes(1, 1, 1024, 128, 64, 4) > 0
    assert lib.pisa_sparse_attention_bwd_workspace_bytes(1, 1, 1024, 128, 64, 17) == 0


def _attn(lib, q=0x1000, k=0x2000, v=0x3000, out=0x4000, B=1, H=1, Ln=128, d=128, bs=64,
          dens=0.5, sink=L.PISA_SINK_NONE, mode=L.PISA_MODE_HYD, opts=None):
    return lib.pisa_attention_ex(q, k, v, out, B, H, Ln, d, bs, dens, sink, mode,
                                 ctypes.byref(opts) if opts else None, None)


def test_argument_checks_fail_before_any_launch(lib):
    assert _attn(lib, q=None) == L.PISA_ERR_INVALID_ARG
    assert _attn(lib, q=0x1001) == L.PISA_ERR_INVALID_ARG          # misaligned
    assert _attn(lib, out=0x1000) == L.PISA_ERR_INVALID_ARG        # out aliases q
    assert _attn(lib, d=96) == L.PISA_ERR_UNSUPPORTED
    assert _attn(lib, bs=96) == L.PISA_ERR_UNSUPPORTED
    # size limits, refused before any launch: more than 65535 (batch, head) pairs,
    # more than 2^24 tokens, a selection row that no longer fits on chip
    assert _attn(lib, B=2, H=40000) == L.PISA_ERR_UNSUPPORTED
    assert _attn(lib, Ln=(1 << 24) + 1) == L.PISA_ERR_UNSUPPORTED
    assert _attn(lib, Ln=64 * 60000) == L.PISA_ERR_UNSUPPORTED
    assert _attn(lib, Ln=64 * 40000, dens=0.01) == L.PISA_ERR_UNSUPPORTED   # fused kernel
    # block_size 128 is supported, but not by the block-wise first-order mode
    assert _attn(lib, bs=128, mode=L.PISA_MODE_1ST) == L.PISA_ERR_UNSUPPORTED
    assert _attn(lib, Ln=0) == L.PISA_ERR_INVALID_ARG
    assert _attn(lib, dens=0.0) == L.PISA_ERR_INVALID_ARG
    assert _attn(lib, dens=1.5) == L.PISA_ERR_INVALID_ARG
    assert _attn(lib, sink=3) == L.PISA_ERR_INVALID_ARG
    assert _attn(lib, mode=7) == L.PISA_ERR_INVALID_ARG
    o = L.PisaOptions()
    o.workspace = 0x10000
    o.ws_bytes = 16
    assert _attn(lib, opts=o) == L.PISA_ERR_WORKSPACE
    o = L.PisaOptions()
    o.scale = float("nan")
    assert _attn(lib, opts=o) == L.PISA_ERR_INVALID_ARG
    # selection inside the fused kernel needs 128-token blocks; idx_out 4-byte aligned
    o = L.PisaOptions()
    o.fuse_select = 1
    assert _attn(lib, opts=o) == L.PISA_ERR_UNSUPPORTED
    o = L.PisaOptions()
    o.idx_out = 0x5002
    assert _attn(lib, bs=128, opts=o) == L.PISA_ERR_INVALID_ARG
    assert lib.pisa_select(None, None, None, 0.0, 0.1, 1, 1, 4, 64, 0.5, 0, None, None, 0,
                           None) == L.PISA_ERR_INVALID_ARG
    assert lib.pisa_status_string(L.PISA_ERR_TIMEOUT).decode().startswith("device-side")


def test_float32_output_argument_checks(lib):
    """The optional float32 output of the training forward, and its use by the
    backward, are refused before any launch when misaligned or aliased."""
    q, k, v, out, lse = 0x100000, 0x200000, 0x300000, 0x400000, 0x500000
    kbar, vsum, hbar, idx, ws = 0x600000, 0x700000, 0x800000, 0x900000, 0xA00000

    def fwd(o32):
        return lib.pisa_sparse_attention_fwd(q, k, v, L.PISA_BF16, kbar, vsum, hbar, idx, 1, 1,
                                             1, 128, 128, 64, 0.0, L.PISA_MODE_0TH, out, lse,
                                             o32, ws, 1 << 40, None)

    assert fwd(0x400004) == L.PISA_ERR_INVALID_ARG      # misaligned
    assert fwd(out) == L.PISA_ERR_INVALID_ARG           # aliases the output
    assert fwd(q) == L.PISA_ERR_INVALID_ARG             # aliases an input
    dq, dk, dv, g = 0xB00000, 0xC00000, 0xD00000, 0xE00000

    def bwd(o32):
        return lib.pisa_sparse_attention_bwd(q, k, v, g, lse, o32, kbar, vsum, idx, 1, 1, 1, 128,
                                             128, 64, 0.0, dq, dk, dv, ws, 1 << 40, None)

    assert bwd(0x400004) == L.PISA_ERR_INVALID_ARG      # misaligned
    assert bwd(dq) == L.PISA_ERR_INVALID_ARG            # a gradient would overwrite it


def test_binding_checks_tensor_arguments():
    """The Python binding refuses, before any pointer is taken, tensors the
    library would misread: non-contiguous q/k/v, a non-bf16 backward, and
    side outputs of the wrong dtype or shape."""
    import torch
    import block_sparse_attention_stats_b200 as P
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    t = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16).transpose(1, 2)   # [1,2,128,64], strided
    lse = torch.zeros(1, 2, 128)
    with pytest.raises(ValueError, match="contiguous"):
        P.pisa_sparse_attention(t, q, q, None, None, None, torch.zeros(1, 2, 2, 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="bf16"):
        P.pisa_sparse_attention_bwd(q.float(), q.float(), q.float(), q.float(), lse, None, None,
                                    torch.zeros(1, 2, 2, 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="dout"):
        P.pisa_sparse_attention_bwd(q, q, q, q[:, :1], lse, None, None,
                                    torch.zeros(1, 2, 2, 1, dtype=torch.int32))
    with pytest.raises(ValueError, match="out_f32"):
        P.pisa_sparse_attention_bwd(q, q, q, q, lse, None, None,
                                    torch.zeros(1, 2, 2, 1, dtype=torch.int32), out_f32=q)
    with pytest.raises(ValueError, match="lse"):
        P.pisa_sparse_attention_fwd(q, q, q, None, None, None,
                                    torch.zeros(1, 2, 2, 1, dtype=torch.int32), lse=lse[:, :1])
    with pytest.raises(ValueError, match="bf16"):
        P.piecewise_sparse_attention_0th(q.float(), q.float(), q.float())


def test_plain_c_program_links_and_calls_the_abi(lib, tmp_path):
    """The boundary is a C ABI: a C99 program that includes only include/pisa.h
    compiles with -pedantic, links against libpisa.so and makes host-side calls
    (no GPU needed for these)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_pisa.c"
    src.write_text(
        '#include <stdio.h>\n#include "pisa.h"\n'
        "int main(void) {\n"
        "  printf(\"%d %d %s\\n\", pisa_num_blocks(75600, 64), pisa_num_selected(1182, 0.125),\n"
        "         pisa_status_string(PISA_ERR_UNSUPPORTED));\n"
        "  return 0;\n}\n")
    libdir = os.path.dirname(L.LIB_PATH)
    exe = tmp_path / "use_pisa"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I",
                    os.path.dirname(HEADER), str(src), "-o", str(exe), libdir + "/libpisa.so",
                    "-Wl,-rpath," + libdir], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[:2] == ["1182", "147"]
    assert len(" ".join(out[2:])) > 0
