"""The C-ABI library on the CPU: it loads, exports every entry point include/*.h declares,
its host-side codebook equals the oracle's bit for bit, and its argument validation answers
before any device work (no GPU needed: these paths return before the first CUDA call)."""

import ctypes
import glob
import os
import re

import numpy as np
import pytest

from nf4_base_lora_blockwise_b200 import abi
from oracle import nf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(abi.LIB_PATH):
        from nf4_base_lora_blockwise_b200 import build
        build.build()
    return abi._lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        txt = open(h).read()
        names |= set(re.findall(r"QLORA_API\s+[\w\s\*]+?\b(qlora_\w+)\s*\(", txt))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared()
    assert declared, "no declarations found"
    assert declared == set(abi.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(8):
        assert lib.qlora_status_str(code)


def test_codebook_matches_oracle_bit_exact(lib):
    """Two independent derivations of the NF4 levels (C++ bisection on erfc in the library,
    scipy's ndtri in the oracle) agree on every fp32 bit."""
    got = np.array(abi.qlora_nf4_codebook(), dtype=np.float32)
    assert np.array_equal(got.view(np.uint32), nf4.codebook_f32().view(np.uint32))


FAKE = 1 << 20          # an aligned, non-null address: never dereferenced on these paths


def _w(N=128, K=256, dq=0, q=FAKE, absmax=FAKE):
    return abi.Nf4Weight(q, absmax if not dq else None, FAKE if dq else None,
                         FAKE if dq else None, N, K, dq)


def _fwd(lib, X=FAKE, W=None, M=64, r=16, H=FAKE, ws=FAKE, ws_bytes=1 << 30):
    W = W or _w()
    return lib.qlora_linear_fwd(X, ctypes.byref(W), FAKE, FAKE, M, r, 32.0, H, FAKE, ws,
                                ws_bytes, None)


def test_validation_codes(lib):
    assert _fwd(lib, X=None) == 1                      # NULL
    assert _fwd(lib, W=_w(q=None)) == 1
    assert _fwd(lib, W=_w(K=100)) == 2                 # K % 64
    assert _fwd(lib, W=_w(N=96)) == 2                  # N % 64
    assert _fwd(lib, M=0) == 2
    assert _fwd(lib, r=0) == 2                         # r out of [1, 128]
    assert _fwd(lib, r=136) == 2
    assert _fwd(lib, r=12, ws_bytes=16) == 5           # r = 12 (padded copies): workspace
    assert _fwd(lib, r=12, X=FAKE + 8) == 3            # ... and alignment, before any work
    assert _fwd(lib, X=FAKE + 8) == 3                  # misaligned
    assert _fwd(lib, ws_bytes=16) == 5                 # workspace too small
    assert _fwd(lib, ws=None) == 5
    assert lib.qlora_nf4_pack(FAKE, 64, 100, 0, FAKE, FAKE, None, None, None) == 2
    assert lib.qlora_nf4_pack(FAKE, 64, 128, 1, FAKE, FAKE, None, None, None) == 1


def test_workspace_bytes(lib):
    assert lib.qlora_workspace_bytes(0, 128, 128, 16) == 0
    assert lib.qlora_workspace_bytes(64, 128, 128, 129) == 0
    assert lib.qlora_workspace_bytes(64, 128, 128, 0) == 0
    # r = 12 runs at 16 on padded copies: more than the rank-16 workspace
    assert lib.qlora_workspace_bytes(64, 128, 128, 12) > lib.qlora_workspace_bytes(64, 128, 128, 16)
    small = lib.qlora_workspace_bytes(64, 512, 256, 8)
    big = lib.qlora_workspace_bytes(4096, 4096, 4096, 16)
    # 4096^3 runs whole tiles and the rank-r products reduce inside their clusters, so the
    # workspace is the two bf16 rank-r activations plus one 256-byte-aligned block of per-token-
    # tile counters (4 bytes per 128 tokens, + 2) for the down-projection fused into the GEMM;
    # 64 tokens on a 512 x 256 weight run stream-K and add the GEMM's partial-sum slots.
    flags = (4 * (4096 // 128 + 2) + 255) // 256 * 256
    assert big == 2 * 4096 * 16 * 2 + flags
    assert small > 2 * 64 * 8 * 2


def _gfwd(lib, rows, N=None, r=16, ws_bytes=1 << 30):
    N = sum(rows) if N is None else N
    W = _w(N=N)
    arr = (ctypes.c_int * max(len(rows), 1))(*rows)
    return lib.qlora_grouped_fwd(FAKE, ctypes.byref(W), FAKE, FAKE, arr if rows else None,
                                 len(rows), 64, r, 32.0, FAKE, FAKE, FAKE, ws_bytes, None)


def test_grouped_validation_codes(lib):
    """Packed adapters: 1..8 adapters, each a multiple of 128 rows (of 64 for one adapter),
    summing to W's rows, with n r a valid rank."""
    assert _gfwd(lib, [], N=256) == 1                   # no group array
    assert _gfwd(lib, [128] * 9) == 2                   # more than 8 adapters
    assert _gfwd(lib, [256, 192]) == 2                  # 192 rows: not a multiple of 128
    assert _gfwd(lib, [256, 128], N=512) == 2           # rows do not sum to N
    assert _gfwd(lib, [128, 128], r=72) == 2            # n r = 144 > 128
    assert _gfwd(lib, [128, 128], r=12) == 2
    assert _gfwd(lib, [256, 128], ws_bytes=16) == 5     # valid groups, workspace too small
    assert _gfwd(lib, [192], ws_bytes=16) == 5          # one adapter: multiples of 64 suffice
    W = _w(N=384)
    arr = (ctypes.c_int * 2)(256, 128)
    assert lib.qlora_grouped_bwd(FAKE, FAKE, ctypes.byref(W), FAKE, FAKE, FAKE, arr, 2, 64, 16,
                                 32.0, FAKE, FAKE, None, FAKE, 1 << 30, None) == 1  # dB NULL
    assert lib.qlora_grouped_workspace_bytes(64, 384, 256, 16, 9) == 0
    assert lib.qlora_grouped_workspace_bytes(64, 384, 256, 72, 2) == 0
    # The packed rank sizes the workspace: n adapters of rank r need what rank n r needs.
    assert (lib.qlora_grouped_workspace_bytes(4096, 6144, 4096, 16, 3)
            == lib.qlora_workspace_bytes(4096, 6144, 4096, 48))
    assert (lib.qlora_grouped_workspace_bytes(64, 512, 256, 16, 1)
            == lib.qlora_workspace_bytes(64, 512, 256, 16))


def test_xa_saved_may_be_null(lib):
    """Recompute instead of store: a NULL XA_saved passes validation in the forward, the
    backward and the packed entry points (the workspace check answers next)."""
    W = _w()
    assert lib.qlora_linear_fwd(FAKE, ctypes.byref(W), FAKE, FAKE, 64, 16, 32.0, FAKE, None,
                                FAKE, 16, None) == 5
    assert lib.qlora_linear_bwd(FAKE, FAKE, ctypes.byref(W), FAKE, FAKE, None, 64, 16, 32.0,
                                FAKE, FAKE, FAKE, FAKE, 16, None) == 5
    arr = (ctypes.c_int * 1)(128)
    assert lib.qlora_grouped_bwd(FAKE, FAKE, ctypes.byref(W), FAKE, FAKE, None, arr, 1, 64, 16,
                                 32.0, FAKE, FAKE, FAKE, FAKE, 16, None) == 5
    assert lib.qlora_linear_fwd(FAKE, ctypes.byref(W), FAKE, FAKE, 64, 16, 32.0, FAKE, FAKE + 8,
                                FAKE, 1 << 30, None) == 3


def test_lm_head_and_plain_gemm_validation(lib):
    """LM head + cross-entropy and the GEMM without extension: argument checks answer before
    any device work."""
    head = _w(N=1024, K=256)
    args = lambda W=head, X=FAKE, labels=FAKE, loss=FAKE, ws_bytes=1 << 34: (
        X, ctypes.byref(W), labels, 64, 16, loss, None, FAKE, FAKE, ws_bytes, None)
    assert lib.qlora_lm_head_ce(*args(X=None)) == 1
    assert lib.qlora_lm_head_ce(*args(labels=None)) == 1
    assert lib.qlora_lm_head_ce(*args(loss=None)) == 1
    assert lib.qlora_lm_head_ce(*args(W=_w(N=1024, K=64))) == 2      # K < 128
    assert lib.qlora_lm_head_ce(*args(W=_w(N=1000, K=256))) == 2     # V % 64
    assert lib.qlora_lm_head_ce(*args(W=_w(N=64, K=256))) == 2       # V < 128 (dX: one step)
    assert lib.qlora_lm_head_ce_workspace_bytes(64, 64, 256, 16) == 0
    assert lib.qlora_lm_head_ce(*args(ws_bytes=16)) == 5
    need = lib.qlora_lm_head_ce_workspace_bytes(64, 1024, 256, 16)
    assert need >= 16 * 1024 * 2 + 64 * 4                          # one chunk of logits + losses
    assert lib.qlora_lm_head_ce_workspace_bytes(64, 1024, 256, 0) >= 64 * 1024 * 2
    assert lib.qlora_lm_head_ce_workspace_bytes(64, 1024, 64, 16) == 0
    # r = 0: no extension operands needed, but the reduction must be >= 128 and unsplit.
    W = _w(N=128, K=64)
    assert lib.qlora_nf4_gemm(FAKE, ctypes.byref(W), 0, None, None, 64, 0, None, 0, FAKE, FAKE,
                              1 << 30, None) == 2                  # K = 64: one step per tile
    W = _w(N=128, K=256)
    arr = (ctypes.c_int * 1)(128)
    assert lib.qlora_nf4_gemm(FAKE, ctypes.byref(W), 0, None, None, 64, 0, arr, 1, FAKE, FAKE,
                              1 << 30, None) == 2                  # no adapter split without r
    assert lib.qlora_nf4_gemm(FAKE, ctypes.byref(W), 0, None, None, 64, 8, None, 0, FAKE, FAKE,
                              1 << 30, None) == 1                  # r > 0 needs its operands
    assert lib.qlora_cross_entropy_rows(FAKE, 4, 100, FAKE, FAKE, FAKE, 1, None) == 2  # V % 8
    assert lib.qlora_cross_entropy_count(None, 4, 128, FAKE, None) == 1


def test_header_is_plain_c(tmp_path):
    """include/qlora_nf4.h is a C header: a C11 translation unit that includes it and calls
    every entry point compiles with gcc (syntax and types only)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    src = tmp_path / "use_header.c"
    src.write_text('#include "qlora_nf4.h"\n'
                   "int main(void) {\n"
                   "  qlora_nf4_weight w = {0};\n"
                   "  size_t n = qlora_workspace_bytes(64, 128, 128, 16);\n"
                   "  n += qlora_grouped_workspace_bytes(64, 256, 128, 16, 2);\n"
                   "  n += qlora_lm_head_ce_workspace_bytes(64, 1024, 256, 16);\n"
                   "  (void)qlora_linear_fwd(0, &w, 0, 0, 64, 16, 32.0f, 0, 0, 0, n, 0);\n"
                   "  (void)qlora_status_str(QLORA_OK);\n"
                   "  return 0;\n"
                   "}\n")
    r = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-fsyntax-only",
                        "-I" + os.path.join(ROOT, "include"), str(src)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
