"""Helpers shared by the test files: oracle runs on seeded workloads,
per-(sequence, head) sub-problems, error metrics and guarded buffers."""
from __future__ import annotations

import numpy as np

import oracle
from hybrid_linear_attention_05_b200.workloads import PrefillInputs

# max|gpu - ref| / max|ref| bars
PREFILL_TOL = 5e-3      # bf16-operand tensor-core prefill (and the fp32 CUDA-core one)
DECODE_TOL = 1e-4       # fp32 decode step
BF16_HALF_ULP = 2.0 ** -8  # relative rounding bound of a bf16 output


def relerr(gpu, ref) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), "non-finite GPU output"
    m = float(np.max(np.abs(ref))) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(gpu - ref))) / max(m, 1e-30)


def relerr_beyond_bf16(gpu, ref) -> float:
    """Error left after allowing the output's own bf16 rounding (half an ulp
    of the reference value), relative to max|ref|."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(gpu))
    excess = np.maximum(np.abs(gpu - ref) - BF16_HALF_ULP * np.abs(ref), 0.0)
    return float(np.max(excess)) / max(float(np.max(np.abs(ref))), 1e-30) if ref.size else 0.0


def oracle_prefill(inp: PrefillInputs, nthreads=None):
    w = inp.w
    return oracle.prefill(w.Hk, w.Hv, w.d, w.d, inp.cu_seqlens, inp.mixed_qkv, inp.conv_w, inp.a,
                          inp.b, inp.A_log, inp.dt_bias, inp.z, inp.norm_w, inp.initial_state,
                          inp.conv_state_in, scale=w.scale, nthreads=nthreads)


def head_columns(w, h):
    """Channels of the mixed projection that value head h reads."""
    d, G = w.d, w.Hv // w.Hk
    kh = h // G
    q = np.arange(kh * d, (kh + 1) * d)
    k = w.Hk * d + q
    v = 2 * w.Hk * d + np.arange(h * d, (h + 1) * d)
    return np.concatenate([q, k, v])


def oracle_subproblem(inp: PrefillInputs, n: int, h: int, nthreads=1):
    """Oracle on sequence n, value head h alone (a 1-key-head, 1-value-head
    layer on the channels that head reads).  The mixer is separable over
    (sequence, value head), so this equals the full problem's rows."""
    w = inp.w
    cu = inp.cu_seqlens
    s = slice(int(cu[n]), int(cu[n + 1]))
    cols = head_columns(w, h)
    d = w.d
    res = oracle.prefill(
        1, 1, d, d, [0, s.stop - s.start], inp.mixed_qkv[s][:, cols], inp.conv_w[cols],
        inp.a[s][:, h:h + 1], inp.b[s][:, h:h + 1], inp.A_log[h:h + 1], inp.dt_bias[h:h + 1],
        inp.z[s][:, h * d:(h + 1) * d], inp.norm_w,
        None if inp.initial_state is None else inp.initial_state[n:n + 1, h:h + 1],
        None if inp.conv_state_in is None else inp.conv_state_in[n:n + 1, cols],
        scale=w.scale, nthreads=nthreads)
    return res, s, cols
