"""Seeded synthetic inputs for the Gated DeltaNet mixer.

This module only draws random numbers and rounds them to bf16; it holds none
of the mixer's arithmetic.  Both the CUDA path (through the tests and the
benchmark) and the CPU oracle consume exactly the arrays produced here.

Value distributions (N(mu, s) means mean mu and *standard deviation* s):
  mixed q|k|v projection    N(0, 1)
  conv weight  [Cc, 4]      N(0, 0.25)
  a, b         [T, Hv]      N(0, 1)
  A_log        [Hv]         U(0, ln 16)   -> exp(A_log) in [1, 16]
                            (tests also draw U(-7, -5): a slow decay that
                            carries the state across many chunks)
  dt_bias      [Hv]         N(0, 0.1)
  z            [T, Hv*dv]   N(0, 1)
  norm weight  [dv]         1 + N(0, 0.1)
  initial state             0, or N(0, 0.02) per sequence
  decode conv cache         N(0, 1)
Shapes follow the Qwen3.5 family pages: 0.8B (16 key / 16 value heads, head
width 128, conv kernel 4), 9B (16 key / 32 value heads, 8192 conv channels)
and 397B-A17B (16 key / 64 value heads).

All floating inputs are drawn in fp32 with numpy's PCG64 and, for bf16
workloads, rounded to bf16 once here (round to nearest even); A_log, dt_bias
and the states stay fp32.  The returned arrays are float32 holding exactly
the values the GPU consumes.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

LN16 = float(np.log(16.0))


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str                 # "prefill" | "decode"
    Hk: int
    Hv: int
    d: int                    # dk = dv
    dtype: str                # "bf16" | "f32"
    seed: int
    seqlens: tuple = ()       # prefill: per-sequence lengths
    batch: int = 0            # decode: number of sequences
    chunk: int = 64
    s0_std: float = 0.0       # 0 -> zero initial state
    varlen_total: int = 0     # >0: lengths drawn at random summing to this
    varlen_n: int = 0
    q_scale: Optional[float] = None  # factor on the normalised q; None -> d ** -0.5
    A_log_range: tuple = (0.0, LN16)  # A_log ~ U(lo, hi)

    @property
    def Cc(self) -> int:
        return 2 * self.Hk * self.d + self.Hv * self.d

    @property
    def scale(self) -> float:
        return self.d ** -0.5 if self.q_scale is None else float(self.q_scale)


WORKLOADS = {
    w.name: w for w in [
        Workload("prefill_T64_Hk2_Hv2_d32_c16_f32", "prefill", Hk=2, Hv=2, d=32, dtype="f32",
                 seed=0, seqlens=(64,), chunk=16),
        Workload("prefill_T4096_Hk16_Hv16_d128", "prefill", Hk=16, Hv=16, d=128, dtype="bf16",
                 seed=1, seqlens=(4096,)),
        Workload("prefill_4x8192_Hk16_Hv32_d128", "prefill", Hk=16, Hv=32, d=128, dtype="bf16",
                 seed=2, seqlens=(8192,) * 4, s0_std=0.02),
        Workload("decode_B256_Hk16_Hv32_d128", "decode", Hk=16, Hv=32, d=128, dtype="bf16",
                 seed=3, batch=256, s0_std=0.02),
        Workload("prefill_varlen8_T65536_Hk16_Hv64_d128", "prefill", Hk=16, Hv=64, d=128,
                 dtype="bf16", seed=4, s0_std=0.02, varlen_total=65536, varlen_n=8),
    ]
}


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); float32 out."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).copy()
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    u &= np.uint32(0xFFFF0000)
    return u.view(np.float32)


def varlen_lengths(total: int, n: int, rng: np.random.Generator) -> tuple:
    """n lengths >= 1 summing to `total`: n-1 distinct cut points drawn
    uniformly from [1, total-1], sorted."""
    cuts = np.sort(rng.choice(np.arange(1, total), size=n - 1, replace=False))
    edges = np.concatenate([[0], cuts, [total]])
    lens = np.diff(edges)
    assert lens.min() >= 1 and lens.sum() == total
    return tuple(int(x) for x in lens)


@dataclass
class PrefillInputs:
    w: Workload
    cu_seqlens: np.ndarray     # [N+1] int32
    mixed_qkv: np.ndarray      # [T, Cc]
    conv_w: np.ndarray         # [Cc, 4]
    a: np.ndarray              # [T, Hv]
    b: np.ndarray              # [T, Hv]
    A_log: np.ndarray          # [Hv] fp32
    dt_bias: np.ndarray        # [Hv] fp32
    z: np.ndarray              # [T, Hv*dv]
    norm_w: np.ndarray         # [dv]
    initial_state: Optional[np.ndarray]  # [N, Hv, dv, dk] fp32 or None
    conv_state_in: Optional[np.ndarray]  # [N, Cc, 3] or None

    @property
    def N(self) -> int:
        return self.cu_seqlens.shape[0] - 1

    @property
    def T(self) -> int:
        return int(self.cu_seqlens[-1])


@dataclass
class DecodeInputs:
    w: Workload
    mixed_qkv: np.ndarray      # [B, Cc]
    conv_w: np.ndarray
    a: np.ndarray              # [B, Hv]
    b: np.ndarray
    A_log: np.ndarray
    dt_bias: np.ndarray
    z: np.ndarray              # [B, Hv*dv]
    norm_w: np.ndarray
    state: np.ndarray          # [B, Hv, dv, dk] fp32
    conv_state: np.ndarray     # [B, Cc, 3]


def _normal(rng, shape, std=1.0, mean=0.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def _cast(x: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_round(x) if dtype == "bf16" else np.ascontiguousarray(x, dtype=np.float32)


def _weights(w: Workload, rng):
    conv_w = _cast(_normal(rng, (w.Cc, 4), 0.25), w.dtype)
    A_log = rng.uniform(w.A_log_range[0], w.A_log_range[1], size=(w.Hv,)).astype(np.float32)
    dt_bias = _normal(rng, (w.Hv,), 0.1)
    norm_w = _cast(_normal(rng, (w.d,), 0.1, 1.0), w.dtype)
    return conv_w, A_log, dt_bias, norm_w


def make_prefill(w: Workload, seqlens: Optional[tuple] = None, with_conv_state: bool = False
                 ) -> PrefillInputs:
    """Draw one prefill batch.  `seqlens` overrides the workload's lengths
    (smaller parity cases with the same distributions)."""
    assert w.kind == "prefill"
    rng = np.random.Generator(np.random.PCG64(w.seed))
    if seqlens is None:
        seqlens = varlen_lengths(w.varlen_total, w.varlen_n, rng) if w.varlen_total else w.seqlens
    seqlens = tuple(int(s) for s in seqlens)
    N = len(seqlens)
    cu = np.zeros(N + 1, dtype=np.int32)
    cu[1:] = np.cumsum(seqlens)
    T = int(cu[-1])
    conv_w, A_log, dt_bias, norm_w = _weights(w, rng)
    x = _cast(_normal(rng, (T, w.Cc)), w.dtype)
    a = _cast(_normal(rng, (T, w.Hv)), w.dtype)
    b = _cast(_normal(rng, (T, w.Hv)), w.dtype)
    z = _cast(_normal(rng, (T, w.Hv * w.d)), w.dtype)
    S0 = _normal(rng, (N, w.Hv, w.d, w.d), w.s0_std) if w.s0_std > 0 else None
    cs = _cast(_normal(rng, (N, w.Cc, 3)), w.dtype) if with_conv_state else None
    return PrefillInputs(w, cu, x, conv_w, a, b, A_log, dt_bias, z, norm_w, S0, cs)


def make_decode(w: Workload, batch: Optional[int] = None) -> DecodeInputs:
    assert w.kind == "decode"
    rng = np.random.Generator(np.random.PCG64(w.seed))
    B = int(batch or w.batch)
    conv_w, A_log, dt_bias, norm_w = _weights(w, rng)
    x = _cast(_normal(rng, (B, w.Cc)), w.dtype)
    a = _cast(_normal(rng, (B, w.Hv)), w.dtype)
    b = _cast(_normal(rng, (B, w.Hv)), w.dtype)
    z = _cast(_normal(rng, (B, w.Hv * w.d)), w.dtype)
    state = _normal(rng, (B, w.Hv, w.d, w.d), w.s0_std)
    cs = _cast(_normal(rng, (B, w.Cc, 3)), w.dtype)
    return DecodeInputs(w, x, conv_w, a, b, A_log, dt_bias, z, norm_w, state, cs)


def resized(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (same distributions)."""
    return replace(w, **kw)


@dataclass
class LayerInputs:
    """The layer around the mixer: hidden states and the projection weights
    (in the [out, in] layout), drawn after the mixer's own inputs."""
    mixer: PrefillInputs
    d_model: int
    hidden: np.ndarray         # [T, d_model]
    w_in: np.ndarray           # [Cc + Hv*dv + 2*Hv, d_model]: in_proj_qkv; in_proj_z; in_proj_b; in_proj_a
    w_out: np.ndarray          # [d_model, Hv*dv]


def make_layer(w: Workload, d_model: int, seqlens: Optional[tuple] = None,
               with_conv_state: bool = False) -> LayerInputs:
    """Hidden states ~ N(0, 1) and weights ~ N(0, 1/fan_in) -- so that the
    projections come out near unit scale, as the mixer workloads draw them --
    rounded to bf16 for bf16 workloads; the mixer's parameters, states and
    lengths are those of make_prefill (its projection outputs are replaced)."""
    mix = make_prefill(w, seqlens=seqlens, with_conv_state=with_conv_state)
    rng = np.random.Generator(np.random.PCG64(w.seed + 1000))
    n_in = w.Cc + w.Hv * w.d + 2 * w.Hv
    hidden = _cast(_normal(rng, (mix.T, d_model)), w.dtype)
    w_in = _cast(_normal(rng, (n_in, d_model), d_model ** -0.5), w.dtype)
    w_out = _cast(_normal(rng, (d_model, w.Hv * w.d), (w.Hv * w.d) ** -0.5), w.dtype)
    return LayerInputs(mix, d_model, hidden, w_in, w_out)
