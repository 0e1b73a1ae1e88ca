"""KronQ per-layer quantization pass on NVIDIA B200 (sm_100a).

Python binding of libkronq.so: one wrapper per C entry point, same names,
argument marshalling only (torch tensors -> device pointers, the current CUDA
stream).  Every step of the pass runs in the library's CUDA kernels; PyTorch
supplies device memory and streams.  See ``include/kronq.h`` for the
contract of each call.
"""
from __future__ import annotations

import ctypes

from ._lib import (BF16, BIIP_MODES, F32, ORDERED_FP32, R_FORM, U_GIVEN, WRITE_E, KronqError,
                   QuantParams, check, lib)

__all__ = [
    "KronqError", "QuantParams", "U_GIVEN", "ORDERED_FP32", "WRITE_E", "R_FORM",
    "kronq_accumulate_factors", "kronq_sensitivity", "kronq_trace_tokens",
    "kronq_sensitivity_from_traces", "kronq_allocate_bits",
    "kronq_allocate_topn_types", "kronq_biip_workspace_bytes", "kronq_biip_forward",
    "kronq_biip_inverse", "kronq_quantize_workspace_bytes", "kronq_quantize_layer",
    "kronq_quantize_layer_static", "kronq_quantize_act_order_workspace_bytes",
    "kronq_quantize_layer_act_order", "kronq_quantize_two_sided_workspace_bytes", "kronq_quantize_two_sided",
    "kronq_pack", "kronq_unpack", "kronq_device_status", "kronq_wait_selftest",
    "kronq_kfac_loss_workspace_bytes",
    "kronq_kfac_loss", "kronq_launch_count", "kronq_last_error", "kronq_version", "workspace", "words_per_row",
    "EST_INPUT", "EST_MARGINAL", "EST_FROBENIUS", "EST_FLIPFLOP",
    "kronq_kron_factors_workspace_bytes", "kronq_kron_factors",
    "kronq_decode_matvec_workspace_bytes", "kronq_decode_matvec",
]

# kronq_estimator (Table 1 rows of the "WaterKron and FlipFlop Hessian" page)
EST_INPUT, EST_MARGINAL, EST_FROBENIUS, EST_FLIPFLOP = 0, 1, 2, 3


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _rowmajor(t, name):
    """The C ABI takes dense row-major arrays; refuse anything else loudly."""
    if t is not None and not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous row-major tensor")
    if t is not None and not t.is_cuda:
        raise ValueError(f"{name} must live in device memory")
    return t


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def workspace(nbytes: int, device="cuda"):
    """A device byte buffer for the calls that take a workspace (256-byte aligned)."""
    import torch
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def words_per_row(n: int, bits: int) -> int:
    return (n * bits + 31) // 32


def kronq_version() -> str:
    return lib.kronq_version().decode()


def kronq_launch_count() -> int:
    return int(lib.kronq_launch_count())


def kronq_last_error() -> str:
    return lib.kronq_last_error().decode(errors="replace")


def kronq_accumulate_factors(A, H, zero_first: bool = False, lda: int | None = None, stream=None):
    """H (d x d float32) += A^T A for A (T x d, bf16 or float32, row stride lda)."""
    T, d = A.shape
    if A.stride(1) != 1:
        raise ValueError("A must have unit stride along d (row-major token rows)")
    _rowmajor(H, "H")
    lda = A.stride(0) if lda is None else lda
    check(lib.kronq_accumulate_factors(_ptr(A), _dtype_code(A), T, d, lda, _ptr(H),
                                       1 if zero_first else 0, _stream(stream)))


def kronq_sensitivity(HX, HG, ws=None, stream=None):
    """(tr(H_X), tr(H_G), tr(H_G) * tr(H_X)) as Python floats (synchronises)."""
    _rowmajor(HX, "HX"), _rowmajor(HG, "HG")
    out = (ctypes.c_double * 3)()
    ws = workspace(256, HX.device) if ws is None else ws
    check(lib.kronq_sensitivity(_ptr(HX), HX.shape[0], _ptr(HG), HG.shape[0], out, _ptr(ws),
                                ws.numel(), _stream(stream)))
    return out[0], out[1], out[2]


def kronq_trace_tokens(A, trace, zero_first: bool = True, ws=None, stream=None):
    """trace (one device float64) (+)= sum_t |a_t|^2 = tr(A^T A) for tokens A (T x d)."""
    T, d = A.shape
    if A.stride(1) != 1:
        raise ValueError("A must have unit stride along d (row-major token rows)")
    _rowmajor(trace, "trace")
    ws = workspace(int(lib.kronq_trace_tokens_workspace_bytes()), A.device) if ws is None else ws
    check(lib.kronq_trace_tokens(_ptr(A), _dtype_code(A), T, d, A.stride(0), _ptr(trace),
                                 1 if zero_first else 0, _ptr(ws), ws.numel(), _stream(stream)))


def kronq_sensitivity_from_traces(traces, stream=None):
    """(tr(H_X), tr(H_G), tr(H_G) * tr(H_X)) from two device float64 traces (synchronises)."""
    _rowmajor(traces, "traces")
    out = (ctypes.c_double * 3)()
    check(lib.kronq_sensitivity_from_traces(_ptr(traces), out, _stream(stream)))
    return out[0], out[1], out[2]


def kronq_allocate_bits(sens, sizes, avg_bits: float = 2.5, bmin: int = 2, bmax: int = 4):
    L = len(sens)
    s = (ctypes.c_double * L)(*[float(v) for v in sens])
    z = (ctypes.c_int64 * L)(*[int(v) for v in sizes])
    out = (ctypes.c_int * L)()
    check(lib.kronq_allocate_bits(s, z, L, float(avg_bits), bmin, bmax, out))
    return list(out)


def kronq_allocate_topn_types(sens, type_ids, n_types: int, base_bits: int, N: int):
    L = len(sens)
    s = (ctypes.c_double * L)(*[float(v) for v in sens])
    t = (ctypes.c_int * L)(*[int(v) for v in type_ids])
    out = (ctypes.c_int * L)()
    check(lib.kronq_allocate_topn_types(s, t, L, n_types, base_bits, N, out))
    return list(out)


def kronq_biip_workspace_bytes(m: int, n: int) -> int:
    return int(lib.kronq_biip_workspace_bytes(m, n))


def kronq_biip_forward(W, Wt, HX, HG, seed: int, alpha: float, mode: str, d_in, d_out, ws=None,
                       stream=None):
    m, n = W.shape
    for t, name in ((W, "W"), (Wt, "Wt"), (HX, "HX"), (HG, "HG"), (d_in, "d_in"), (d_out, "d_out")):
        _rowmajor(t, name)
    ws = workspace(kronq_biip_workspace_bytes(m, n), W.device) if ws is None else ws
    check(lib.kronq_biip_forward(_ptr(W), _dtype_code(W), _ptr(Wt), m, n, _ptr(HX), _ptr(HG),
                                 int(seed), float(alpha), BIIP_MODES[mode], _ptr(d_in), _ptr(d_out),
                                 _ptr(ws), ws.numel(), _stream(stream)))


def kronq_biip_inverse(W, seed: int, mode: str, d_in, d_out, ws=None, stream=None):
    m, n = W.shape
    _rowmajor(W, "W")
    ws = workspace(kronq_biip_workspace_bytes(m, n), W.device) if ws is None else ws
    check(lib.kronq_biip_inverse(_ptr(W), m, n, int(seed), BIIP_MODES[mode], _ptr(d_in),
                                 _ptr(d_out), _ptr(ws), ws.numel(), _stream(stream)))


def kronq_quantize_workspace_bytes(m: int, n: int, params: QuantParams) -> int:
    return int(lib.kronq_quantize_workspace_bytes(m, n, ctypes.byref(params)))


def kronq_quantize_layer(Wt, HX, params: QuantParams, codes, scales, zeros, info, E=None, ws=None,
                         stream=None):
    m, n = Wt.shape
    for t, name in ((Wt, "Wt"), (HX, "HX"), (codes, "codes"), (scales, "scales"), (zeros, "zeros"),
                    (info, "info"), (E, "E")):
        _rowmajor(t, name)
    ws = workspace(kronq_quantize_workspace_bytes(m, n, params), Wt.device) if ws is None else ws
    check(lib.kronq_quantize_layer(_ptr(Wt), _ptr(HX), m, n, ctypes.byref(params), _ptr(codes),
                                   _ptr(scales), _ptr(zeros), _ptr(E), _ptr(info), _ptr(ws),
                                   ws.numel(), _stream(stream)))


def kronq_quantize_layer_static(Wt, HX, params: QuantParams, codes, scales, zeros, info, E=None,
                                stream=None):
    """kronq_quantize_layer without a workspace, for callers that cannot
    allocate device memory: the scratch is the library's 64 MiB static device
    array (shared by all calls on a device; overlapping calls race)."""
    m, n = Wt.shape
    for t, name in ((Wt, "Wt"), (HX, "HX"), (codes, "codes"), (scales, "scales"), (zeros, "zeros"),
                    (info, "info"), (E, "E")):
        _rowmajor(t, name)
    check(lib.kronq_quantize_layer_static(_ptr(Wt), _ptr(HX), m, n, ctypes.byref(params),
                                          _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(E),
                                          _ptr(info), _stream(stream)))


def kronq_quantize_act_order_workspace_bytes(m: int, n: int, params: QuantParams) -> int:
    return int(lib.kronq_quantize_act_order_workspace_bytes(m, n, ctypes.byref(params)))


def kronq_quantize_layer_act_order(Wt, HX, params: QuantParams, codes, scales, zeros, g_idx, info,
                                   E=None, perm=None, ws=None, stream=None):
    """kronq_quantize_layer with the act-order sweep order; outputs in the
    original column order, scales/zeros per sweep-order group, g_idx (n int32)."""
    m, n = Wt.shape
    for t, name in ((Wt, "Wt"), (HX, "HX"), (codes, "codes"), (scales, "scales"), (zeros, "zeros"),
                    (g_idx, "g_idx"), (info, "info"), (E, "E"), (perm, "perm")):
        _rowmajor(t, name)
    if ws is None:
        ws = workspace(kronq_quantize_act_order_workspace_bytes(m, n, params), Wt.device)
    check(lib.kronq_quantize_layer_act_order(_ptr(Wt), _ptr(HX), m, n, ctypes.byref(params), _ptr(codes),
                                             _ptr(scales), _ptr(zeros), _ptr(E), _ptr(g_idx), _ptr(perm),
                                             _ptr(info), _ptr(ws), ws.numel(), _stream(stream)))


def kronq_quantize_two_sided_workspace_bytes(m: int, n: int, params: QuantParams) -> int:
    return int(lib.kronq_quantize_two_sided_workspace_bytes(m, n, ctypes.byref(params)))


def kronq_quantize_two_sided(Wt, HX, HG, params: QuantParams, codes, scales, zeros, info, E=None, ws=None,
                             stream=None):
    """Two-sided rounding under H_X (x) H_G; info holds two int32 (H_X, H_G)."""
    m, n = Wt.shape
    for t, name in ((Wt, "Wt"), (HX, "HX"), (HG, "HG"), (codes, "codes"), (scales, "scales"),
                    (zeros, "zeros"), (info, "info"), (E, "E")):
        _rowmajor(t, name)
    if info.numel() < 2:
        raise ValueError("info: two int32 (H_X, H_G)")
    if ws is None:
        ws = workspace(kronq_quantize_two_sided_workspace_bytes(m, n, params), Wt.device)
    check(lib.kronq_quantize_two_sided(_ptr(Wt), _ptr(HX), _ptr(HG), m, n, ctypes.byref(params), _ptr(codes),
                                       _ptr(scales), _ptr(zeros), _ptr(E), _ptr(info), _ptr(ws), ws.numel(),
                                       _stream(stream)))


def kronq_pack(codes, bits: int, out, stream=None):
    m, n = codes.shape
    _rowmajor(codes, "codes"), _rowmajor(out, "out")
    check(lib.kronq_pack(_ptr(codes), m, n, bits, _ptr(out), _stream(stream)))


def kronq_unpack(words, m: int, n: int, bits: int, codes, stream=None):
    check(lib.kronq_unpack(_ptr(words), m, n, bits, _ptr(codes), _stream(stream)))


def kronq_device_status(stream=None) -> int:
    v = ctypes.c_int(0)
    check(lib.kronq_device_status(ctypes.byref(v), _stream(stream)))
    return v.value


def kronq_wait_selftest(which: int, limit_ns: int, ws, stream=None):
    """One CTA whose bounded wait (0: mbarrier, 1: cross-CTA counter) is never
    satisfied gives up after limit_ns; read the result with kronq_device_status."""
    check(lib.kronq_wait_selftest(int(which), int(limit_ns), _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)))


def kronq_kron_factors_workspace_bytes(T: int, n: int, m: int) -> int:
    return int(lib.kronq_kron_factors_workspace_bytes(T, n, m))


def kronq_kron_factors(X, G, est: int, iters: int, A, B, info, ws=None, stream=None):
    """Kronecker factors (A n x n, B m x m, fp32 out) of E[x x^T (x) g g^T]
    from bf16 tokens X (T x n) and G (T x m); info (device int) 0 on success."""
    import torch
    T, n = X.shape
    m = G.shape[1]
    if X.dtype != torch.bfloat16 or G.dtype != torch.bfloat16:
        raise ValueError("X and G must be bfloat16")
    for t, name in ((X, "X"), (G, "G"), (A, "A"), (B, "B"), (info, "info")):
        _rowmajor(t, name)
    ws = workspace(kronq_kron_factors_workspace_bytes(T, n, m), X.device) if ws is None else ws
    check(lib.kronq_kron_factors(_ptr(X), _ptr(G), T, n, m, int(est), int(iters), _ptr(A), _ptr(B),
                                 _ptr(info), _ptr(ws), ws.numel(), _stream(stream)))


def kronq_decode_matvec_workspace_bytes(m: int, n: int) -> int:
    return int(lib.kronq_decode_matvec_workspace_bytes(m, n))


def kronq_decode_matvec(packed, scales, zeros, n: int, bits: int, group: int, seed: int, mode: str,
                        d_in, d_out, x, y, ws=None, stream=None):
    """y (m, float32) = D_o^-1 U^T Q V D_i^-1 x from packed codes (int32 words)."""
    m = packed.shape[0]
    for t, name in ((packed, "packed"), (scales, "scales"), (zeros, "zeros"), (d_in, "d_in"),
                    (d_out, "d_out"), (x, "x"), (y, "y")):
        _rowmajor(t, name)
    ws = workspace(kronq_decode_matvec_workspace_bytes(m, n), x.device) if ws is None else ws
    check(lib.kronq_decode_matvec(_ptr(packed), _ptr(scales), _ptr(zeros), m, n, bits, group, seed,
                                  BIIP_MODES[mode], _ptr(d_in), _ptr(d_out), _ptr(x), _dtype_code(x),
                                  _ptr(y), _ptr(ws), ws.numel(), _stream(stream)))


def kronq_kfac_loss_workspace_bytes(m: int, n: int) -> int:
    return int(lib.kronq_kfac_loss_workspace_bytes(m, n))


def kronq_kfac_loss(E, HG, ws=None, stream=None) -> float:
    m, n = E.shape
    _rowmajor(E, "E"), _rowmajor(HG, "HG")
    ws = workspace(kronq_kfac_loss_workspace_bytes(m, n), E.device) if ws is None else ws
    out = ctypes.c_double(0.0)
    check(lib.kronq_kfac_loss(_ptr(E), _ptr(HG), m, n, ctypes.byref(out), _ptr(ws), ws.numel(),
                              _stream(stream)))
    return out.value
