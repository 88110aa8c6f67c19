"""Thin ctypes binding of the C ABI in ``include/gdn.h``.

Argument marshalling only: every step of the mixer runs in the CUDA library.
torch tensors are accepted for convenience (their device pointers and the
current CUDA stream are passed through); plain integer device pointers work
too.  The library is loaded from this package directory; if it is missing
the import of the binding fails loudly -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgdn_b200.so")

GDN_OK = 0
GDN_ERR_NULL = -1
GDN_ERR_DIMS = -2
GDN_ERR_ALIGN = -3
GDN_ERR_UNSUPPORTED = -4
GDN_ERR_CUDA = -5
GDN_ERR_WORKSPACE = -6
GDN_ERR_ALIAS = -7
GDN_ERR_TIMEOUT = -8

GDN_F32 = 0
GDN_BF16 = 1
GDN_F16 = 2

GDN_IMPL_AUTO = 0
GDN_IMPL_SIMT = 1
GDN_IMPL_TC = 2
GDN_IMPL_TC_SPLIT = 3
GDN_IMPL_TC_FUSED = 4

EXPORTED = ["gdn_prefill_workspace_size", "gdn_prefill_workspace_size_n", "gdn_prefill",
            "gdn_prefill_auto_segments", "gdn_prefill_resolve_impl", "gdn_prefill_noalloc", "gdn_prefill_state_map",
            "gdn_state_fold", "gdn_decode", "gdn_chunk_core", "gdn_core_workspace_size",
            "gdn_core_workspace_size_split",
            "gdn_linear", "gdn_layer_activation_bytes", "gdn_layer_workspace_size", "gdn_layer_prefill",
            "gdn_device_error", "gdn_selftest_bounded_wait", "gdn_status_string", "gdn_version"]

# Size of the library's own scratch used by gdn_prefill_noalloc (gdn.h).
GDN_NOALLOC_SCRATCH_BYTES = 64 << 20


class gdn_dims(ctypes.Structure):
    _fields_ = [("Hk", ctypes.c_int), ("Hv", ctypes.c_int), ("dk", ctypes.c_int),
                ("dv", ctypes.c_int), ("conv_k", ctypes.c_int), ("scale", ctypes.c_float),
                ("eps_l2", ctypes.c_float), ("eps_norm", ctypes.c_float)]


_vp = ctypes.c_void_p


class gdn_prefill_args(ctypes.Structure):
    _fields_ = [("mixed_qkv", _vp), ("conv_w", _vp), ("a", _vp), ("b", _vp), ("A_log", _vp),
                ("dt_bias", _vp), ("z", _vp), ("norm_w", _vp), ("cu_seqlens", _vp),
                ("N", ctypes.c_int), ("T_tot", ctypes.c_int), ("chunk", ctypes.c_int),
                ("dtype", ctypes.c_int), ("impl", ctypes.c_int),
                ("initial_state", _vp), ("final_state", _vp), ("conv_state_in", _vp),
                ("conv_state_out", _vp), ("out", _vp), ("workspace", _vp),
                ("workspace_bytes", ctypes.c_size_t), ("core_event_begin", _vp),
                ("core_event_end", _vp), ("segments", ctypes.c_int), ("reuse_workspace", ctypes.c_int)]


class gdn_decode_args(ctypes.Structure):
    _fields_ = [("mixed_qkv", _vp), ("conv_w", _vp), ("a", _vp), ("b", _vp), ("A_log", _vp),
                ("dt_bias", _vp), ("z", _vp), ("norm_w", _vp), ("state", _vp),
                ("conv_state", _vp), ("out", _vp), ("B", ctypes.c_int), ("dtype", ctypes.c_int),
                ("state_dtype", ctypes.c_int), ("T", ctypes.c_int)]


class gdn_core_args(ctypes.Structure):
    _fields_ = [("q", _vp), ("k", _vp), ("v", _vp), ("g", _vp), ("beta", _vp),
                ("cu_seqlens", _vp), ("N", ctypes.c_int), ("T_tot", ctypes.c_int),
                ("chunk", ctypes.c_int), ("dtype", ctypes.c_int), ("impl", ctypes.c_int),
                ("initial_state", _vp), ("final_state", _vp), ("o", _vp), ("workspace", _vp),
                ("workspace_bytes", ctypes.c_size_t)]


class gdn_linear_args(ctypes.Structure):
    _fields_ = [("x", _vp), ("w", _vp), ("M", ctypes.c_int), ("N", ctypes.c_int), ("K", ctypes.c_int),
                ("ldx", ctypes.c_int), ("ldw", ctypes.c_int), ("n_outputs", ctypes.c_int),
                ("out", _vp * 4), ("out_cols", ctypes.c_int * 4), ("out_ld", ctypes.c_int * 4)]


class gdn_layer_args(ctypes.Structure):
    _fields_ = [("hidden", _vp), ("w_in", _vp), ("w_out", _vp), ("y", _vp), ("d_model", ctypes.c_int),
                ("conv_w", _vp), ("A_log", _vp), ("dt_bias", _vp), ("norm_w", _vp), ("cu_seqlens", _vp),
                ("N", ctypes.c_int), ("T_tot", ctypes.c_int), ("chunk", ctypes.c_int), ("impl", ctypes.c_int),
                ("initial_state", _vp), ("final_state", _vp), ("conv_state_in", _vp),
                ("conv_state_out", _vp), ("workspace", _vp), ("workspace_bytes", ctypes.c_size_t)]


_lib = None


def lib():
    """Load libgdn_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libgdn_b200.so is missing; build it with "
                "`python -m hybrid_linear_attention_05_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.gdn_prefill_workspace_size.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int]
        L.gdn_prefill_workspace_size.restype = ctypes.c_size_t
        L.gdn_prefill_workspace_size_n.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int]
        L.gdn_prefill_workspace_size_n.restype = ctypes.c_size_t
        L.gdn_prefill_auto_segments.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int]
        L.gdn_prefill_auto_segments.restype = ctypes.c_int
        L.gdn_prefill_resolve_impl.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_size_t]
        L.gdn_prefill_resolve_impl.restype = ctypes.c_int
        L.gdn_prefill.argtypes = [ctypes.POINTER(gdn_dims), ctypes.POINTER(gdn_prefill_args), _vp]
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_prefill_noalloc.argtypes = [ctypes.POINTER(gdn_dims), ctypes.POINTER(gdn_prefill_args),
                                          _vp]
        L.gdn_prefill_noalloc.restype = ctypes.c_int
        L.gdn_prefill_state_map.argtypes = [ctypes.POINTER(gdn_dims), ctypes.POINTER(gdn_prefill_args),
                                            _vp, _vp]
        L.gdn_prefill_state_map.restype = ctypes.c_int
        L.gdn_state_fold.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp]
        L.gdn_state_fold.restype = ctypes.c_int
        L.gdn_decode.argtypes = [ctypes.POINTER(gdn_dims), ctypes.POINTER(gdn_decode_args), _vp]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_chunk_core.argtypes = [ctypes.POINTER(gdn_dims), ctypes.POINTER(gdn_core_args), _vp]
        L.gdn_chunk_core.restype = ctypes.c_int
        L.gdn_core_workspace_size.argtypes = [ctypes.c_int]
        L.gdn_core_workspace_size.restype = ctypes.c_size_t
        L.gdn_core_workspace_size_split.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int]
        L.gdn_core_workspace_size_split.restype = ctypes.c_size_t
        L.gdn_linear.argtypes = [ctypes.POINTER(gdn_linear_args), _vp]
        L.gdn_linear.restype = ctypes.c_int
        L.gdn_layer_activation_bytes.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int]
        L.gdn_layer_activation_bytes.restype = ctypes.c_size_t
        L.gdn_layer_workspace_size.argtypes = [ctypes.POINTER(gdn_dims), ctypes.c_int, ctypes.c_int,
                                               ctypes.c_int]
        L.gdn_layer_workspace_size.restype = ctypes.c_size_t
        L.gdn_layer_prefill.argtypes = [ctypes.POINTER(gdn_dims), ctypes.POINTER(gdn_layer_args), _vp]
        L.gdn_layer_prefill.restype = ctypes.c_int
        L.gdn_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
        L.gdn_device_error.restype = ctypes.c_int
        L.gdn_selftest_bounded_wait.argtypes = [ctypes.c_int, _vp]
        L.gdn_selftest_bounded_wait.restype = ctypes.c_int
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_version.argtypes = []
        L.gdn_version.restype = ctypes.c_char_p
        _lib = L
    return _lib


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (%d)" % (where, status_string(status), status))


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()


def make_dims(Hk, Hv, dk, dv=None, scale=None, eps_l2=1e-6, eps_norm=1e-6, conv_k=4) -> gdn_dims:
    dv = dk if dv is None else dv
    return gdn_dims(int(Hk), int(Hv), int(dk), int(dv), int(conv_k),
                    float(dk ** -0.5 if scale is None else scale), float(eps_l2), float(eps_norm))


def ptr(x) -> Optional[int]:
    """Device pointer of a tensor (or pass-through int / None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.float16:
        return GDN_F16
    raise TypeError("unsupported dtype %s" % t.dtype)


def current_stream_handle() -> int:
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(status, where, raise_on_error):
    if raise_on_error and status != GDN_OK:
        raise GdnError(status, where)
    return status


def gdn_prefill_workspace_size(dims: gdn_dims, T_tot: int, dtype: int) -> int:
    return int(lib().gdn_prefill_workspace_size(ctypes.byref(dims), int(T_tot), int(dtype)))


def gdn_prefill_workspace_size_n(dims: gdn_dims, N: int, T_tot: int, dtype: int) -> int:
    return int(lib().gdn_prefill_workspace_size_n(ctypes.byref(dims), int(N), int(T_tot), int(dtype)))


def gdn_prefill_auto_segments(dims: gdn_dims, N: int, T_tot: int) -> int:
    """Segments per sequence the two-kernel path picks by itself (gdn.h)."""
    return int(lib().gdn_prefill_auto_segments(ctypes.byref(dims), int(N), int(T_tot)))


def gdn_prefill_resolve_impl(dims: gdn_dims, N: int, T_tot: int, chunk: int, dtype: int,
                             impl: int = GDN_IMPL_AUTO, workspace_bytes: int = 0) -> int:
    """The implementation gdn_prefill runs for these sizes and workspace (gdn.h)."""
    return int(lib().gdn_prefill_resolve_impl(ctypes.byref(dims), int(N), int(T_tot), int(chunk),
                                              int(dtype), int(impl), int(workspace_bytes)))


def gdn_prefill(dims: gdn_dims, *, mixed_qkv, conv_w, a, b, A_log, dt_bias, z, norm_w,
                cu_seqlens, N, T_tot, chunk, dtype, out, workspace, workspace_bytes,
                initial_state=None, final_state=None, conv_state_in=None, conv_state_out=None,
                impl=GDN_IMPL_AUTO, core_event_begin=None, core_event_end=None, segments=0,
                reuse_workspace=0, stream=None, raise_on_error=True) -> int:
    args = gdn_prefill_args(
        ptr(mixed_qkv), ptr(conv_w), ptr(a), ptr(b), ptr(A_log), ptr(dt_bias), ptr(z),
        ptr(norm_w), ptr(cu_seqlens), int(N), int(T_tot), int(chunk), int(dtype), int(impl),
        ptr(initial_state), ptr(final_state), ptr(conv_state_in), ptr(conv_state_out), ptr(out),
        ptr(workspace), int(workspace_bytes), core_event_begin, core_event_end, int(segments),
        int(reuse_workspace))
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_prefill(ctypes.byref(dims), ctypes.byref(args), s), "gdn_prefill",
                  raise_on_error)


def gdn_prefill_noalloc(dims: gdn_dims, *, mixed_qkv, conv_w, a, b, A_log, dt_bias, z, norm_w,
                        cu_seqlens, N, T_tot, chunk, dtype, out, initial_state=None,
                        final_state=None, conv_state_in=None, conv_state_out=None,
                        impl=GDN_IMPL_AUTO, reuse_workspace=0, stream=None, raise_on_error=True) -> int:
    """gdn_prefill on the library's own scratch: for callers that have no way
    to allocate a workspace (see gdn.h).  Calls that overlap on the GPU race
    on the shared scratch."""
    args = gdn_prefill_args(
        ptr(mixed_qkv), ptr(conv_w), ptr(a), ptr(b), ptr(A_log), ptr(dt_bias), ptr(z),
        ptr(norm_w), ptr(cu_seqlens), int(N), int(T_tot), int(chunk), int(dtype), int(impl),
        ptr(initial_state), ptr(final_state), ptr(conv_state_in), ptr(conv_state_out), ptr(out),
        None, 0, None, None, 0, int(reuse_workspace))
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_prefill_noalloc(ctypes.byref(dims), ctypes.byref(args), s),
                  "gdn_prefill_noalloc", raise_on_error)


def gdn_prefill_state_map(dims: gdn_dims, *, mixed_qkv, conv_w, a, b, A_log, dt_bias, cu_seqlens, N,
                          T_tot, chunk, dtype, map_out, workspace, workspace_bytes, conv_state_in=None,
                          conv_state_out=None, z=None, norm_w=None, segments=0, stream=None,
                          raise_on_error=True) -> int:
    """(M, R) of every sequence: final state = initial state @ M + R (gdn.h)."""
    args = gdn_prefill_args(
        ptr(mixed_qkv), ptr(conv_w), ptr(a), ptr(b), ptr(A_log), ptr(dt_bias), ptr(z), ptr(norm_w),
        ptr(cu_seqlens), int(N), int(T_tot), int(chunk), int(dtype), int(GDN_IMPL_TC_SPLIT), None,
        None, ptr(conv_state_in), ptr(conv_state_out), None, ptr(workspace), int(workspace_bytes),
        None, None, int(segments))
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_prefill_state_map(ctypes.byref(dims), ctypes.byref(args), ptr(map_out), s),
                  "gdn_prefill_state_map", raise_on_error)


def gdn_state_fold(dims: gdn_dims, *, N, count, maps, S_out, S_first=None, stream=None,
                   raise_on_error=True) -> int:
    """S_out = fold of `count` consecutive maps [count, N, Hv, 2, d, d] from S_first."""
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_state_fold(ctypes.byref(dims), int(N), int(count), ptr(maps), ptr(S_first),
                                       ptr(S_out), s), "gdn_state_fold", raise_on_error)


def gdn_decode(dims: gdn_dims, *, mixed_qkv, conv_w, a, b, A_log, dt_bias, z, norm_w, state,
               conv_state, out, B, dtype, state_dtype=GDN_F32, T=1, stream=None,
               raise_on_error=True) -> int:
    args = gdn_decode_args(ptr(mixed_qkv), ptr(conv_w), ptr(a), ptr(b), ptr(A_log),
                           ptr(dt_bias), ptr(z), ptr(norm_w), ptr(state), ptr(conv_state),
                           ptr(out), int(B), int(dtype), int(state_dtype), int(T))
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_decode(ctypes.byref(dims), ctypes.byref(args), s), "gdn_decode",
                  raise_on_error)


def gdn_core_workspace_size(N: int) -> int:
    return int(lib().gdn_core_workspace_size(int(N)))


def gdn_core_workspace_size_split(dims: gdn_dims, N: int, T_tot: int) -> int:
    return int(lib().gdn_core_workspace_size_split(ctypes.byref(dims), int(N), int(T_tot)))


def gdn_chunk_core(dims: gdn_dims, *, q, k, v, g, beta, cu_seqlens, N, T_tot, chunk, dtype, o,
                   initial_state=None, final_state=None, impl=GDN_IMPL_AUTO, workspace=None,
                   workspace_bytes=0, stream=None, raise_on_error=True) -> int:
    args = gdn_core_args(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(cu_seqlens), int(N),
                         int(T_tot), int(chunk), int(dtype), int(impl), ptr(initial_state),
                         ptr(final_state), ptr(o), ptr(workspace), int(workspace_bytes))
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_chunk_core(ctypes.byref(dims), ctypes.byref(args), s),
                  "gdn_chunk_core", raise_on_error)


def gdn_linear(*, x, w, M, N, K, outs, ldx=None, ldw=None, stream=None, raise_on_error=True) -> int:
    """Y = x w^T (bf16); `outs` lists (tensor or pointer, columns, row stride) for
    the consecutive column ranges of Y (gdn.h)."""
    args = gdn_linear_args()
    args.x, args.w = ptr(x), ptr(w)
    args.M, args.N, args.K = int(M), int(N), int(K)
    args.ldx = int(K if ldx is None else ldx)
    args.ldw = int(K if ldw is None else ldw)
    args.n_outputs = len(outs)
    for i, (o, cols, ld) in enumerate(outs[:4]):  # more than four: the library rejects n_outputs
        args.out[i] = ptr(o)
        args.out_cols[i] = int(cols)
        args.out_ld[i] = int(ld)
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_linear(ctypes.byref(args), s), "gdn_linear", raise_on_error)


def gdn_layer_activation_bytes(dims: gdn_dims, d_model: int, T_tot: int) -> int:
    return int(lib().gdn_layer_activation_bytes(ctypes.byref(dims), int(d_model), int(T_tot)))


def gdn_layer_workspace_size(dims: gdn_dims, d_model: int, N: int, T_tot: int) -> int:
    return int(lib().gdn_layer_workspace_size(ctypes.byref(dims), int(d_model), int(N), int(T_tot)))


def gdn_layer_prefill(dims: gdn_dims, *, hidden, w_in, w_out, y, d_model, conv_w, A_log, dt_bias, norm_w,
                      cu_seqlens, N, T_tot, chunk, workspace, workspace_bytes, initial_state=None,
                      final_state=None, conv_state_in=None, conv_state_out=None, impl=GDN_IMPL_AUTO,
                      stream=None, raise_on_error=True) -> int:
    args = gdn_layer_args(ptr(hidden), ptr(w_in), ptr(w_out), ptr(y), int(d_model), ptr(conv_w), ptr(A_log),
                          ptr(dt_bias), ptr(norm_w), ptr(cu_seqlens), int(N), int(T_tot), int(chunk), int(impl),
                          ptr(initial_state), ptr(final_state), ptr(conv_state_in), ptr(conv_state_out),
                          ptr(workspace), int(workspace_bytes))
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_layer_prefill(ctypes.byref(dims), ctypes.byref(args), s), "gdn_layer_prefill",
                  raise_on_error)


def gdn_device_error(clear: bool = True) -> int:
    """Synchronise the device and return (and clear) the kernels' error word."""
    code = ctypes.c_int(0)
    _check(lib().gdn_device_error(ctypes.byref(code), int(clear)), "gdn_device_error", True)
    return code.value


def gdn_selftest_bounded_wait(limit_us: int, stream=None, raise_on_error=True) -> int:
    """Launch the failure-path test kernel (gdn.h): a bounded wait that gives up."""
    s = current_stream_handle() if stream is None else stream
    return _check(lib().gdn_selftest_bounded_wait(int(limit_us), s), "gdn_selftest_bounded_wait",
                  raise_on_error)


def gdn_version() -> str:
    return lib().gdn_version().decode()
