"""ctypes wrapper around the fp64 CPU oracle (``gdn_oracle.cpp``).

TEST INFRASTRUCTURE ONLY.  This module is imported by the tests, by the
smoke check and by the CPU-baseline leg of the benchmark -- never by the
product path.  It shares no code with the CUDA library.

All arrays cross the boundary as C-contiguous float64 (and int64 for
``cu_seqlens``); the functions return new numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.cpp")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libgdn_oracle.so`` with g++."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        cmd = ["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread",
               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        lp = ctypes.POINTER(ctypes.c_int64)
        i, d = ctypes.c_int, ctypes.c_double
        _lib.gdn_oracle_prefill.argtypes = [i, i, i, i, d, d, d, i, lp] + [dp] * 10 + [dp] * 3 + [dp] * 7 + [i]
        _lib.gdn_oracle_prefill.restype = i
        _lib.gdn_oracle_decode.argtypes = [i, i, i, i, d, d, d, i] + [dp] * 8 + [dp] * 3 + [i]
        _lib.gdn_oracle_decode.restype = i
        _lib.gdn_oracle_core.argtypes = [i, i, i, i, i, lp] + [dp] * 6 + [dp, dp, i, i]
        _lib.gdn_oracle_core.restype = i
        _lib.gdn_oracle_silu.argtypes = [i, dp, dp]
        _lib.gdn_oracle_silu.restype = None
        _lib.gdn_oracle_gated_rmsnorm.argtypes = [i, i, d, dp, dp, dp, dp]
        _lib.gdn_oracle_gated_rmsnorm.restype = None
    return _lib


def _d(x):
    """float64 C-contiguous copy/view, or None."""
    if x is None:
        return None
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


@dataclass
class PrefillResult:
    out: np.ndarray            # [T, Hv, dv]
    final_state: np.ndarray    # [N, Hv, dv, dk]
    conv_state_out: np.ndarray  # [N, Cc, 3]
    y_pre: np.ndarray          # [T, Cc] conv output before SiLU
    q: np.ndarray              # [T, Hk, dk] normalised, scaled
    k: np.ndarray              # [T, Hk, dk] normalised
    v: np.ndarray              # [T, Hv, dv]
    g: np.ndarray              # [T, Hv] log decay
    beta: np.ndarray           # [T, Hv]
    o: np.ndarray              # [T, Hv, dv] core output before the gated norm


def prefill(Hk, Hv, dk, dv, cu_seqlens, mixed_qkv, conv_w, a, b, A_log, dt_bias, z, norm_w,
            initial_state=None, conv_state_in=None, scale=None, eps_l2=1e-6, eps_norm=1e-6,
            nthreads=None) -> PrefillResult:
    """Whole mixer over packed sequences (recurrent core)."""
    lib = _load()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    T = int(cu[-1])
    Cc = 2 * Hk * dk + Hv * dv
    if scale is None:
        scale = dk ** -0.5
    x = _d(mixed_qkv).reshape(T, Cc)
    w = _d(conv_w).reshape(Cc, 4)
    a_, b_ = _d(a).reshape(T, Hv), _d(b).reshape(T, Hv)
    Al, dt = _d(A_log).reshape(Hv), _d(dt_bias).reshape(Hv)
    z_ = _d(z).reshape(T, Hv * dv)
    nw = _d(norm_w).reshape(dv)
    S0 = None if initial_state is None else _d(initial_state).reshape(N, Hv, dv, dk)
    cs = None if conv_state_in is None else _d(conv_state_in).reshape(N, Cc, 3)
    res = PrefillResult(
        out=np.zeros((T, Hv, dv)), final_state=np.zeros((N, Hv, dv, dk)),
        conv_state_out=np.zeros((N, Cc, 3)), y_pre=np.zeros((T, Cc)),
        q=np.zeros((T, Hk, dk)), k=np.zeros((T, Hk, dk)), v=np.zeros((T, Hv, dv)),
        g=np.zeros((T, Hv)), beta=np.zeros((T, Hv)), o=np.zeros((T, Hv, dv)))
    rc = lib.gdn_oracle_prefill(
        Hk, Hv, dk, dv, float(scale), float(eps_l2), float(eps_norm), N,
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(x), _ptr(w), _ptr(a_), _ptr(b_), _ptr(Al), _ptr(dt), _ptr(z_), _ptr(nw),
        _ptr(S0), _ptr(cs),
        _ptr(res.out), _ptr(res.final_state), _ptr(res.conv_state_out),
        _ptr(res.y_pre), _ptr(res.q), _ptr(res.k), _ptr(res.v), _ptr(res.g), _ptr(res.beta),
        _ptr(res.o), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions")
    return res


def state_map(Hk, Hv, dk, dv, mixed_qkv, conv_w, a, b, A_log, dt_bias, conv_state_in=None, scale=None,
              eps_l2=1e-6, nthreads=None):
    """The affine state map of one sequence: final state = S0 @ M + R.

    The delta rule S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
    ("Qwen (text & vision-language)", Architecture notes) is linear in S, so
      M = prod over t, in token order, of alpha_t (I - beta_t k_t k_t^T)  [Hv, dk, dk]
      R = the final state from S0 = 0                                     [Hv, dv, dk]
    k, alpha, beta are the prepared values of ``prefill`` (conv from
    conv_state_in, L2 norm, gates); M is accumulated token by token here.
    """
    Cc = 2 * Hk * dk + Hv * dv
    x = _d(mixed_qkv).reshape(-1, Cc)
    T = x.shape[0]
    res = prefill(Hk, Hv, dk, dv, [0, T], x, conv_w, a, b, A_log, dt_bias,
                  np.zeros((T, Hv * dv)), np.ones(dv), initial_state=None,
                  conv_state_in=conv_state_in, scale=scale, eps_l2=eps_l2, nthreads=nthreads)
    G = Hv // Hk
    M = np.zeros((Hv, dk, dk))
    for h in range(Hv):
        Mh = np.eye(dk)
        for t in range(T):
            k = res.k[t, h // G]
            Mh = np.exp(res.g[t, h]) * (Mh - res.beta[t, h] * np.outer(Mh @ k, k))
        M[h] = Mh
    return M, res.final_state[0].copy()


def decode(Hk, Hv, dk, dv, mixed_qkv, conv_w, a, b, A_log, dt_bias, z, norm_w, state,
           conv_state, scale=None, eps_l2=1e-6, eps_norm=1e-6, nthreads=None):
    """One recurrent step for B sequences.  Returns (out, new_state, new_conv_state)."""
    lib = _load()
    Cc = 2 * Hk * dk + Hv * dv
    x = _d(mixed_qkv).reshape(-1, Cc)
    B = x.shape[0]
    if scale is None:
        scale = dk ** -0.5
    S = _d(state).reshape(B, Hv, dv, dk).copy()
    cs = _d(conv_state).reshape(B, Cc, 3).copy()
    out = np.zeros((B, Hv, dv))
    rc = lib.gdn_oracle_decode(
        Hk, Hv, dk, dv, float(scale), float(eps_l2), float(eps_norm), B,
        _ptr(x), _ptr(_d(conv_w).reshape(Cc, 4)), _ptr(_d(a).reshape(B, Hv)),
        _ptr(_d(b).reshape(B, Hv)), _ptr(_d(A_log).reshape(Hv)), _ptr(_d(dt_bias).reshape(Hv)),
        _ptr(_d(z).reshape(B, Hv * dv)), _ptr(_d(norm_w).reshape(dv)), _ptr(S), _ptr(cs),
        _ptr(out), int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions")
    return out, S, cs


def core(Hk, Hv, dk, dv, cu_seqlens, q, k, v, g, beta, initial_state=None, chunk=0,
         nthreads=None):
    """The delta-rule core alone.  chunk <= 0: recurrent form; chunk > 0: chunked form.

    q, k [T, Hk, dk]; v [T, Hv, dv]; g (log decay), beta [T, Hv].
    Returns (o [T, Hv, dv], final_state [N, Hv, dv, dk]).
    """
    lib = _load()
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))
    N = cu.shape[0] - 1
    T = int(cu[-1])
    o = np.zeros((T, Hv, dv))
    S = np.zeros((N, Hv, dv, dk))
    S0 = None if initial_state is None else _d(initial_state).reshape(N, Hv, dv, dk)
    rc = lib.gdn_oracle_core(
        Hk, Hv, dk, dv, N, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
        _ptr(_d(q).reshape(T, Hk, dk)), _ptr(_d(k).reshape(T, Hk, dk)),
        _ptr(_d(v).reshape(T, Hv, dv)), _ptr(_d(g).reshape(T, Hv)),
        _ptr(_d(beta).reshape(T, Hv)), _ptr(S0), _ptr(o), _ptr(S), int(chunk),
        int(nthreads or default_threads()))
    if rc != 0:
        raise ValueError("oracle rejected the dimensions")
    return o, S


def silu(x):
    """The oracle's SiLU (step 2 of the mixer), element-wise."""
    lib = _load()
    x = _d(x)
    y = np.zeros_like(x)
    lib.gdn_oracle_silu(int(x.size), _ptr(x), _ptr(y))
    return y


def gated_rmsnorm(o, z, w, eps=1e-6):
    """The oracle's gated RMSNorm (step 6) over the last axis of o and z, with
    the one weight vector w shared by every row."""
    lib = _load()
    o, z, w = _d(o), _d(z), _d(w)
    dv = int(o.shape[-1])
    assert z.shape == o.shape and w.shape == (dv,)
    out = np.zeros_like(o)
    lib.gdn_oracle_gated_rmsnorm(int(o.size // max(dv, 1)), dv, float(eps), _ptr(o), _ptr(z), _ptr(w),
                                 _ptr(out))
    return out


def bf16(x):
    """x rounded to the nearest bf16 (ties to even), through its fp32 value;
    returned as float64."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = f.view(np.uint32).copy()
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    u &= np.uint32(0xFFFF0000)
    return u.view(np.float32).astype(np.float64)


@dataclass
class LayerResult:
    y: np.ndarray          # [T, d_model] layer output (out_proj of the mixer output)
    mixed_qkv: np.ndarray  # [T, Cc] in_proj_qkv output, as the mixer consumed it
    z: np.ndarray          # [T, Hv*dv]
    a: np.ndarray          # [T, Hv]
    b: np.ndarray          # [T, Hv]
    mixer: PrefillResult


def layer(Hk, Hv, dk, dv, cu_seqlens, hidden, W_qkv, W_z, W_a, W_b, W_out, conv_w, A_log, dt_bias,
          norm_w, initial_state=None, conv_state_in=None, scale=None, activations_bf16=True,
          nthreads=None) -> LayerResult:
    """The linear-attention layer around the mixer ("Qwen/Qwen3.5-9B", module
    tree of a Gated DeltaNet block: in_proj_qkv, in_proj_z, in_proj_b,
    in_proj_a, the mixer, out_proj): the four input projections of the hidden
    states (x W^T with W in [out, in] layout), the mixer, and the output
    projection of its gated-norm output.

    With activations_bf16 the tensors that pass between the projections and
    the mixer -- the projections' outputs and the mixer output -- are rounded
    to bf16, the layer's activation type; every product is fp64."""
    hid = _d(hidden)
    T, d_model = hid.shape
    Cc = 2 * Hk * dk + Hv * dv
    W_qkv, W_z, W_a, W_b, W_out = (_d(w) for w in (W_qkv, W_z, W_a, W_b, W_out))
    assert W_qkv.shape == (Cc, d_model) and W_z.shape == (Hv * dv, d_model)
    assert W_a.shape == (Hv, d_model) and W_b.shape == (Hv, d_model)
    assert W_out.shape == (d_model, Hv * dv)
    act = bf16 if activations_bf16 else (lambda v: v)
    mixed = act(hid @ W_qkv.T)
    z = act(hid @ W_z.T)
    a = act(hid @ W_a.T)
    b = act(hid @ W_b.T)
    r = prefill(Hk, Hv, dk, dv, cu_seqlens, mixed, conv_w, a, b, A_log, dt_bias, z, norm_w,
                initial_state, conv_state_in, scale=scale, nthreads=nthreads)
    out = act(r.out.reshape(T, Hv * dv))
    return LayerResult(y=out @ W_out.T, mixed_qkv=mixed, z=z, a=a, b=b, mixer=r)
