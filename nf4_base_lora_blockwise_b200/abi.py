"""ctypes binding of libqlora_nf4.so -- argument marshalling only.

Every function here mirrors one entry point of ``include/qlora_nf4.h`` with the same name and
takes raw integers (device addresses, sizes, a cudaStream_t handle).  Nothing is computed in
Python.  The library is loaded on first use; if it is missing the call raises -- there is no
fallback path.
"""

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libqlora_nf4.so")

# Exported entry points of include/qlora_nf4.h (kept in sync by tests/test_abi.py).
EXPORTS = (
    "qlora_status_str",
    "qlora_nf4_codebook",
    "qlora_nf4_pack",
    "qlora_nf4_dequant",
    "qlora_workspace_bytes",
    "qlora_linear_fwd",
    "qlora_linear_bwd",
    "qlora_swiglu_fwd",
    "qlora_swiglu_bwd",
    "qlora_lora_down",
    "qlora_nf4_gemm",
    "qlora_lora_grad",
    "qlora_launch_counter",
    "qlora_linear_fwd_noalloc",
    "qlora_noalloc_scratch_bytes",
    "qlora_device_error",
    "qlora_grouped_workspace_bytes",
    "qlora_grouped_fwd",
    "qlora_grouped_fwd_swiglu",
    "qlora_grouped_bwd",
    "qlora_swiglu_packed_fwd",
    "qlora_swiglu_packed_bwd",
    "qlora_lm_head_ce_workspace_bytes",
    "qlora_lm_head_ce",
    "qlora_cross_entropy_count",
    "qlora_cross_entropy_rows",
    "qlora_cross_entropy_mean",
    "qlora_gemm_plan",
    "qlora_gemm_rank_fusable",
    "qlora_set_rank_fusion",
    "qlora_set_side_overlap",
    "qlora_backward_side_sms",
    "qlora_selftest_bounded_wait",
)

STATUS = {
    0: "QLORA_OK", 1: "QLORA_ERR_NULL", 2: "QLORA_ERR_SHAPE", 3: "QLORA_ERR_ALIGN",
    4: "QLORA_ERR_ARCH", 5: "QLORA_ERR_WORKSPACE", 6: "QLORA_ERR_CUDA", 7: "QLORA_ERR_TIMEOUT",
}


class QLoraError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({_lib().qlora_status_str(code).decode()})")


class Nf4Weight(ctypes.Structure):
    """Mirror of ``qlora_nf4_weight``."""
    _fields_ = [
        ("q", ctypes.c_void_p),
        ("absmax", ctypes.c_void_p),
        ("absmax_q8", ctypes.c_void_p),
        ("absmax_scale", ctypes.c_void_p),
        ("N", ctypes.c_int),
        ("K", ctypes.c_int),
        ("double_quant", ctypes.c_int),
    ]


_LIB = None
_VP = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t
_I64 = ctypes.c_int64


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m nf4_base_lora_blockwise_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        sig = {
            "qlora_status_str": (ctypes.c_char_p, [_I]),
            "qlora_nf4_codebook": (_I, [ctypes.POINTER(ctypes.c_float)]),
            "qlora_nf4_pack": (_I, [_VP, _I, _I, _I, _VP, _VP, _VP, _VP, _VP]),
            "qlora_nf4_dequant": (_I, [ctypes.POINTER(Nf4Weight), _VP, _VP]),
            "qlora_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
            "qlora_linear_fwd": (_I, [_VP, ctypes.POINTER(Nf4Weight), _VP, _VP, _I, _I, _F, _VP,
                                      _VP, _VP, _SZ, _VP]),
            "qlora_linear_bwd": (_I, [_VP, _VP, ctypes.POINTER(Nf4Weight), _VP, _VP, _VP, _I, _I,
                                      _F, _VP, _VP, _VP, _VP, _SZ, _VP]),
            "qlora_swiglu_fwd": (_I, [_VP, _VP, _VP, _I64, _VP]),
            "qlora_swiglu_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I64, _VP]),
            "qlora_lora_down": (_I, [_VP, _I, _I, _VP, _I, _I, ctypes.POINTER(_I), _I, _F, _VP,
                                     _VP, _VP, _SZ, _VP]),
            "qlora_nf4_gemm": (_I, [_VP, ctypes.POINTER(Nf4Weight), _I, _VP, _VP, _I, _I,
                                    ctypes.POINTER(_I), _I, _VP, _VP, _SZ, _VP]),
            "qlora_lora_grad": (_I, [_VP, _I, _I, _VP, _I, ctypes.POINTER(_I), _I, _F, _VP, _I,
                                     _VP, _SZ, _VP]),
            "qlora_launch_counter": (ctypes.c_uint64, []),
            "qlora_linear_fwd_noalloc": (_I, [_VP, ctypes.POINTER(Nf4Weight), _VP, _VP, _I, _I,
                                              _F, _VP, _VP, _VP]),
            "qlora_noalloc_scratch_bytes": (_SZ, []),
            "qlora_device_error": (_I, [ctypes.POINTER(ctypes.c_int)]),
            "qlora_selftest_bounded_wait": (_I, [_VP]),
            "qlora_grouped_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
            "qlora_swiglu_packed_fwd": (_I, [_VP, _VP, _I64, _I, _VP]),
            "qlora_swiglu_packed_bwd": (_I, [_VP, _VP, _VP, _I64, _I, _VP]),
            "qlora_lm_head_ce_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
            "qlora_lm_head_ce": (_I, [_VP, ctypes.POINTER(Nf4Weight), _VP, _I, _I, _VP, _VP, _VP,
                                      _VP, _SZ, _VP]),
            "qlora_cross_entropy_count": (_I, [_VP, _I, _I, _VP, _VP]),
            "qlora_cross_entropy_rows": (_I, [_VP, _I, _I, _VP, _VP, _VP, _I, _VP]),
            "qlora_cross_entropy_mean": (_I, [_VP, _I, _VP, _VP, _VP]),
            "qlora_gemm_plan": (_I, [_I, _I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I),
                                     ctypes.POINTER(_I), ctypes.POINTER(_I),
                                     ctypes.POINTER(_SZ)]),
            "qlora_gemm_rank_fusable": (_I, [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_I)]),
            "qlora_set_rank_fusion": (_I, [_I]),
            "qlora_set_side_overlap": (_I, [_I]),
            "qlora_backward_side_sms": (_I, [_I, _I, _I, _I, _I, _I]),
            "qlora_grouped_fwd": (_I, [_VP, ctypes.POINTER(Nf4Weight), _VP, _VP,
                                       ctypes.POINTER(_I), _I, _I, _I, _F, _VP, _VP, _VP, _SZ,
                                       _VP]),
            "qlora_grouped_fwd_swiglu": (_I, [_VP, ctypes.POINTER(Nf4Weight), _VP, _VP, _I, _I,
                                              _F, _VP, _VP, _VP, _VP, _SZ, _VP]),
            "qlora_grouped_bwd": (_I, [_VP, _VP, ctypes.POINTER(Nf4Weight), _VP, _VP, _VP,
                                       ctypes.POINTER(_I), _I, _I, _I, _F, _VP, _VP, _VP, _VP,
                                       _SZ, _VP]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _LIB = lib
    return _LIB


def _check(fn, code):
    if code != 0:
        raise QLoraError(fn, code)


def loaded_path():
    """Path of the loaded shared library (loads it)."""
    _lib()
    return LIB_PATH


def qlora_nf4_codebook():
    buf = (ctypes.c_float * 16)()
    _check("qlora_nf4_codebook", _lib().qlora_nf4_codebook(buf))
    return [buf[i] for i in range(16)]


def qlora_nf4_pack(W, N, K, double_quant, q, absmax, absmax_q8, absmax_scale, stream):
    _check("qlora_nf4_pack", _lib().qlora_nf4_pack(W, N, K, int(double_quant), q, absmax,
                                                   absmax_q8, absmax_scale, stream))


def qlora_nf4_dequant(weight, Wd, stream):
    _check("qlora_nf4_dequant", _lib().qlora_nf4_dequant(ctypes.byref(weight), Wd, stream))


def qlora_workspace_bytes(M, N, K, r):
    return int(_lib().qlora_workspace_bytes(M, N, K, r))


def qlora_linear_fwd(X, weight, A, B, M, r, alpha, H, XA_saved, ws, ws_bytes, stream):
    _check("qlora_linear_fwd", _lib().qlora_linear_fwd(X, ctypes.byref(weight), A, B, M, r,
                                                       float(alpha), H, XA_saved, ws, ws_bytes,
                                                       stream))


def qlora_linear_bwd(dY, X, weight, A, B, XA_saved, M, r, alpha, dX, dA, dB, ws, ws_bytes,
                     stream):
    _check("qlora_linear_bwd", _lib().qlora_linear_bwd(dY, X, ctypes.byref(weight), A, B,
                                                       XA_saved, M, r, float(alpha), dX, dA, dB,
                                                       ws, ws_bytes, stream))


def _int_array(values):
    values = [int(v) for v in values]
    return (_I * max(len(values), 1))(*values), len(values)


def qlora_grouped_workspace_bytes(M, N, K, r, n_groups):
    return int(_lib().qlora_grouped_workspace_bytes(M, N, K, r, n_groups))


def qlora_grouped_fwd(X, weight, A, B, group_rows, M, r, alpha, H, XA_saved, ws, ws_bytes,
                      stream):
    rows, n = _int_array(group_rows)
    _check("qlora_grouped_fwd", _lib().qlora_grouped_fwd(X, ctypes.byref(weight), A, B, rows, n,
                                                         M, r, float(alpha), H, XA_saved, ws,
                                                         ws_bytes, stream))


def qlora_grouped_fwd_swiglu(X, weight, A, B, M, r, alpha, GU, XA_saved, act, ws, ws_bytes,
                             stream):
    _check("qlora_grouped_fwd_swiglu",
           _lib().qlora_grouped_fwd_swiglu(X, ctypes.byref(weight), A, B, M, r, float(alpha), GU,
                                           XA_saved, act, ws, ws_bytes, stream))


def qlora_grouped_bwd(dY, X, weight, A, B, XA_saved, group_rows, M, r, alpha, dX, dA, dB, ws,
                      ws_bytes, stream):
    rows, n = _int_array(group_rows)
    _check("qlora_grouped_bwd", _lib().qlora_grouped_bwd(dY, X, ctypes.byref(weight), A, B,
                                                         XA_saved, rows, n, M, r, float(alpha),
                                                         dX, dA, dB, ws, ws_bytes, stream))


def qlora_swiglu_packed_fwd(gu, a, M, I, stream):
    _check("qlora_swiglu_packed_fwd", _lib().qlora_swiglu_packed_fwd(gu, a, M, I, stream))


def qlora_swiglu_packed_bwd(gu, da, dgu, M, I, stream):
    _check("qlora_swiglu_packed_bwd", _lib().qlora_swiglu_packed_bwd(gu, da, dgu, M, I, stream))


def qlora_lm_head_ce_workspace_bytes(M, V, K, chunk):
    return int(_lib().qlora_lm_head_ce_workspace_bytes(M, V, K, chunk))


def qlora_lm_head_ce(X, weight, labels, M, chunk, loss, token_loss, dX, ws, ws_bytes, stream):
    _check("qlora_lm_head_ce", _lib().qlora_lm_head_ce(X, ctypes.byref(weight), labels, M, chunk,
                                                       loss, token_loss, dX, ws, ws_bytes,
                                                       stream))


def qlora_cross_entropy_count(labels, M, V, count_out, stream):
    _check("qlora_cross_entropy_count", _lib().qlora_cross_entropy_count(labels, M, V, count_out,
                                                                         stream))


def qlora_cross_entropy_rows(z, rows, V, labels, count_in, token_loss, write_grad, stream):
    _check("qlora_cross_entropy_rows", _lib().qlora_cross_entropy_rows(
        z, rows, V, labels, count_in, token_loss, int(write_grad), stream))


def qlora_cross_entropy_mean(token_loss, M, count_in, loss, stream):
    _check("qlora_cross_entropy_mean", _lib().qlora_cross_entropy_mean(token_loss, M, count_in,
                                                                       loss, stream))


def qlora_swiglu_fwd(g, u, a, n, stream):
    _check("qlora_swiglu_fwd", _lib().qlora_swiglu_fwd(g, u, a, n, stream))


def qlora_swiglu_bwd(g, u, da, dg, du, n, stream):
    _check("qlora_swiglu_bwd", _lib().qlora_swiglu_bwd(g, u, da, dg, du, n, stream))


def _groups(group_rows):
    """(int array or None, n) for an optional list of adapter row counts."""
    if group_rows is None:
        return None, 0
    return _int_array(group_rows)


def qlora_lora_down(inp, M, C, w, w_is_r_by_c, r, group_rows, scale, saved, scaled, ws, ws_bytes,
                    stream):
    rows, n = _groups(group_rows)
    _check("qlora_lora_down", _lib().qlora_lora_down(inp, M, C, w, int(w_is_r_by_c), r, rows, n,
                                                     float(scale), saved, scaled, ws, ws_bytes,
                                                     stream))


def qlora_nf4_gemm(act, weight, transpose_w, ext_w, ext_act, M, r, group_rows, out, ws, ws_bytes,
                   stream):
    rows, n = _groups(group_rows)
    _check("qlora_nf4_gemm", _lib().qlora_nf4_gemm(act, ctypes.byref(weight), int(transpose_w),
                                                   ext_w, ext_act, M, r, rows, n, out, ws,
                                                   ws_bytes, stream))


def qlora_lora_grad(big, M, C, small, r, group_rows, scale, out, out_r_by_c, ws, ws_bytes,
                    stream):
    rows, n = _groups(group_rows)
    _check("qlora_lora_grad", _lib().qlora_lora_grad(big, M, C, small, r, rows, n, float(scale),
                                                     out, int(out_r_by_c), ws, ws_bytes, stream))


def qlora_gemm_plan(M, rows_w, steps_per_tile, sm_count):
    """dict(bt, nh, streamk, grid, partial_bytes) of the dequant GEMM's launch plan."""
    v = [_I() for _ in range(4)]
    pb = _SZ()
    _check("qlora_gemm_plan", _lib().qlora_gemm_plan(M, rows_w, steps_per_tile, sm_count,
                                                     *[ctypes.byref(x) for x in v],
                                                     ctypes.byref(pb)))
    return {"bt": v[0].value, "nh": v[1].value, "streamk": v[2].value, "grid": v[3].value,
            "partial_bytes": pb.value}


def qlora_gemm_rank_fusable(M, rows_w, steps_per_tile, sm_count, rank_cols, r, transpose_w):
    """Tokens per half tile of the GEMM launch that computes the rank-r down-projection itself,
    or 0 when that launch does not."""
    bt = _I()
    ok = _lib().qlora_gemm_rank_fusable(M, rows_w, steps_per_tile, sm_count, rank_cols, r,
                                        int(transpose_w), ctypes.byref(bt))
    return bt.value if ok else 0


def qlora_set_rank_fusion(enable):
    """Fuse the rank-r down-projections into the GEMM launches (process-wide); returns the
    previous setting."""
    return bool(_lib().qlora_set_rank_fusion(int(bool(enable))))


def qlora_set_side_overlap(mode):
    """Where dB and dA of the backward run (process-wide): 0 after the dX GEMM, 1 beside it on
    SMs taken from it when the schedule model expects that to pay (default), 2 beside it
    whenever the GEMM runs whole tiles.  Returns the previous mode."""
    return int(_lib().qlora_set_side_overlap(int(mode)))


def qlora_backward_side_sms(M, N, K, R, sm_count, mode=-1):
    """SMs the backward gives to dB / dA beside the dX GEMM for M tokens, W0 [N, K] and R packed
    rank columns under side-overlap mode `mode` (-1: the current setting); 0: after the GEMM."""
    return int(_lib().qlora_backward_side_sms(M, N, K, R, sm_count, int(mode)))


def qlora_launch_counter():
    return int(_lib().qlora_launch_counter())


def qlora_linear_fwd_noalloc(X, weight, A, B, M, r, alpha, H, XA_saved, stream):
    _check("qlora_linear_fwd_noalloc",
           _lib().qlora_linear_fwd_noalloc(X, ctypes.byref(weight), A, B, M, r, float(alpha), H,
                                           XA_saved, stream))


def qlora_noalloc_scratch_bytes():
    return int(_lib().qlora_noalloc_scratch_bytes())


def qlora_selftest_bounded_wait(stream):
    _check("qlora_selftest_bounded_wait", _lib().qlora_selftest_bounded_wait(stream))


def qlora_device_error():
    code = ctypes.c_int(0)
    st = _lib().qlora_device_error(ctypes.byref(code))
    if st not in (0, 7):
        _check("qlora_device_error", st)
    return code.value
