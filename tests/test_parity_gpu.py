"""GPU parity: the CUDA library (through the C ABI) against the fp64 oracle
on the same seeded inputs.

Bars (max|gpu - ref| / max|ref|): 5e-3 for prefill (bf16 inputs, fp16
tensor-core operands, fp32 accumulation; the CUDA-core kernel is held to the
same bar), 1e-4 for the fp32 decode step (state exactly; bf16 outputs after
allowing their own rounding).
"""
import dataclasses

import numpy as np
import pytest

from gdn_testlib import (DECODE_TOL, PREFILL_TOL, oracle_prefill, oracle_subproblem, relerr,
                         relerr_beyond_bf16)
import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_05_b200 import api, build, gdn  # noqa: E402
from hybrid_linear_attention_05_b200.workloads import (WORKLOADS, make_decode, make_prefill,  # noqa: E402
                                                       resized)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gdn.lib()


TINY = WORKLOADS["prefill_T64_Hk2_Hv2_d32_c16_f32"]
P08 = WORKLOADS["prefill_T4096_Hk16_Hv16_d128"]
P9B = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]
D9B = WORKLOADS["decode_B256_Hk16_Hv32_d128"]
P397 = WORKLOADS["prefill_varlen8_T65536_Hk16_Hv64_d128"]

IMPLS = {"simt": (gdn.GDN_IMPL_SIMT, 32), "tc": (gdn.GDN_IMPL_TC, 64),
         "split": (gdn.GDN_IMPL_TC_SPLIT, 64), "fused": (gdn.GDN_IMPL_TC_FUSED, 64)}
# A_log range of a slow decay (alpha ~ 0.995-0.9995 per token): the workloads'
# own U(0, ln 16) decays the state by e^-45 or more per 64-token chunk, so only
# slow-decay cases show whether the state is carried right across chunks
SLOW_DECAY = (-7.0, -5.0)


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_prefill(inp, impl, chunk, guard=True, segments=0):
    dp = api.to_device(inp, chunk=chunk)
    bufs = api.PrefillBuffers(dp)
    if guard:  # canaries on both sides of every output
        for name in ("out", "final_state", "conv_state_out"):
            t = getattr(bufs, name)
            big = torch.full((t.numel() + 2 * 64,), float("nan"), dtype=t.dtype, device=t.device)
            setattr(bufs, name, big[64:64 + t.numel()].view(t.shape))
            setattr(bufs, name + "_guard", big)
    status = gdn.gdn_prefill(
        bufs.dims, mixed_qkv=dp.mixed_qkv, conv_w=dp.conv_w, a=dp.a, b=dp.b, A_log=dp.A_log,
        dt_bias=dp.dt_bias, z=dp.z, norm_w=dp.norm_w, cu_seqlens=dp.cu_seqlens, N=dp.N,
        T_tot=dp.T, chunk=dp.chunk, dtype=bufs.dtype_code, out=bufs.out, workspace=bufs.workspace,
        workspace_bytes=bufs.ws_bytes, initial_state=dp.initial_state,
        final_state=bufs.final_state, conv_state_in=dp.conv_state_in,
        conv_state_out=bufs.conv_state_out, impl=impl, segments=segments, raise_on_error=False)
    if status == gdn.GDN_ERR_UNSUPPORTED:
        pytest.skip("implementation not available for this shape")
    assert status == gdn.GDN_OK, gdn.status_string(status)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0, "a bounded wait inside a kernel gave up"
    if guard:
        for name in ("out", "final_state", "conv_state_out"):
            big = getattr(bufs, name + "_guard")
            n = getattr(bufs, name).numel()
            assert torch.isnan(big[:64].float()).all() and torch.isnan(big[64 + n:].float()).all(), \
                "write outside " + name
    return bufs


def check_full(inp, bufs, tol=PREFILL_TOL):
    ref = oracle_prefill(inp)
    e_out = relerr(np64(bufs.out), ref.out)
    e_S = relerr(np64(bufs.final_state), ref.final_state)
    assert e_out <= tol, e_out
    assert e_S <= tol, e_S
    # the conv tail is a copy of raw inputs: exact
    np.testing.assert_array_equal(np64(bufs.conv_state_out), ref.conv_state_out)
    return e_out, e_S


# ------------------------------------------------------------------ prefill


def test_tiny_fp32_workload():
    """The tiny fp32 workload (T=64, 2/2 heads of width 32, chunk 16) in full."""
    inp = make_prefill(TINY)
    bufs = run_prefill(inp, gdn.GDN_IMPL_AUTO, 16)
    e_out, e_S = check_full(inp, bufs)
    assert e_out < 1e-4 and e_S < 1e-4  # fp32 CUDA-core path: far inside the bar


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("d", [32, 64])
def test_simt_small_heads(chunk, d):
    w = resized(TINY, Hk=2, Hv=4, d=d, dtype="bf16", s0_std=0.02, seed=21)
    inp = make_prefill(w, seqlens=(chunk * 3 + 7, 1, 2, chunk - 1, 0, chunk), with_conv_state=True)
    bufs = run_prefill(inp, gdn.GDN_IMPL_SIMT, chunk)
    check_full(inp, bufs)


@pytest.mark.parametrize("impl", ["simt", "tc", "split", "fused"])
def test_qwen08b_shapes_ragged(impl):
    """16/16 heads of width 128 over several chunks with a ragged tail."""
    code, chunk = IMPLS[impl]
    inp = make_prefill(P08, seqlens=(333,))
    bufs = run_prefill(inp, code, chunk)
    check_full(inp, bufs)


@pytest.mark.parametrize("impl", ["simt", "tc", "split", "fused"])
def test_9b_shapes_gqa_varlen(impl):
    """16 key / 32 value heads, nonzero initial states, conv history,
    sequences of lengths 1, 2, 3, 64 and one spanning several chunks."""
    code, chunk = IMPLS[impl]
    inp = make_prefill(P9B, seqlens=(200, 1, 2, 3, 64, 0, 129), with_conv_state=True)
    bufs = run_prefill(inp, code, chunk)
    check_full(inp, bufs)


@pytest.mark.parametrize("seqlens", [(200, 0), (3, 190), (64, 129)])
def test_split_value_pairs_varlen(seqlens):
    """Two-kernel path with few (value head, sequence) chains, where each chain
    runs as a pair of CTAs over half the value columns: GQA, initial states,
    conv history, an empty sequence, one shorter than the conv window, and
    sequences ending on and off a chunk boundary."""
    inp = make_prefill(P9B, seqlens=seqlens, with_conv_state=True)
    bufs = run_prefill(inp, gdn.GDN_IMPL_TC_SPLIT, 64)
    check_full(inp, bufs)


@pytest.mark.parametrize("segments,seqlens,decay", [
    (3, (64 * 11 + 5, 130, 0, 64 * 3, 1), "slow"),
    (5, (64 * 5, 64 * 9 + 63, 2), "slow"),
    (8, (64 * 11 + 5, 130, 0, 64 * 3, 1), "slow"),
    (8, (64 * 8, 64 * 16 + 1), "workload"),
])
def test_split_segmented_chain_varlen(segments, seqlens, decay):
    """Segmented state chains: each sequence's chunks cut into `segments`
    pieces whose affine maps and start states are formed first.  Covers
    segments with several chunks and with none (a sequence of fewer chunks
    than segments), an empty sequence, GQA, nonzero initial states and conv
    history, with half-width CTA pairs (3, 5) and whole-row CTAs (8)."""
    w = resized(P9B, Hk=2, Hv=4, seed=70 + segments)
    if decay == "slow":
        w = resized(w, A_log_range=SLOW_DECAY)
    inp = make_prefill(w, seqlens=seqlens, with_conv_state=True)
    bufs = run_prefill(inp, gdn.GDN_IMPL_TC_SPLIT, 64, segments=segments)
    check_full(inp, bufs)


def test_split_segments_agree_with_serial_chain():
    """The same call with one serial chain and with 4 and 8 segments: the
    results agree with each other within the parity bar and each matches
    the oracle."""
    w = resized(P08, Hk=4, Hv=4, seed=77, A_log_range=SLOW_DECAY)
    inp = make_prefill(w, seqlens=(64 * 24 + 17,))
    ref = oracle_prefill(inp)
    outs = []
    for seg in (1, 4, 8):
        bufs = run_prefill(inp, gdn.GDN_IMPL_TC_SPLIT, 64, segments=seg)
        outs.append((np64(bufs.out), np64(bufs.final_state)))
        assert relerr(outs[-1][0], ref.out) <= PREFILL_TOL
        assert relerr(outs[-1][1], ref.final_state) <= PREFILL_TOL
    for o, S in outs[1:]:
        assert relerr(o, outs[0][0]) <= PREFILL_TOL
        assert relerr(S, outs[0][1]) <= PREFILL_TOL


@pytest.mark.parametrize("impl,segments", [("tc", 0), ("split", 1), ("split", 4), ("split", 8),
                                           ("fused", 0)])
def test_slow_decay_state_carry(impl, segments):
    """Slow decay (exp(A_log) ~ 1e-3, alpha near 1) so that the state written
    in early chunks still shapes the outputs and the final state many chunks
    later -- the regime where the chunk-to-chunk carry, and for segmented
    chains the segment maps and the scan, are actually exercised.  Nonzero
    initial states, GQA, two sequences of 17 and 9 chunks."""
    w = resized(P9B, Hk=2, Hv=4, seed=79, A_log_range=SLOW_DECAY)
    inp = make_prefill(w, seqlens=(64 * 16 + 40, 64 * 9))
    code, chunk = IMPLS[impl]
    bufs = run_prefill(inp, code, chunk, segments=segments)
    check_full(inp, bufs)


def test_split_segments_in_place_state():
    """final_state the same buffer as initial_state with segmented chains: the
    state is read (by the scan) before any chain writes it back."""
    w = resized(P9B, Hk=2, Hv=4, seed=78, A_log_range=SLOW_DECAY)
    inp = make_prefill(w, seqlens=(64 * 9 + 3, 64 * 4))
    dp = api.to_device(inp, chunk=64)
    bufs = api.PrefillBuffers(dp)
    S = dp.initial_state.clone()
    gdn.gdn_prefill(bufs.dims, mixed_qkv=dp.mixed_qkv, conv_w=dp.conv_w, a=dp.a, b=dp.b,
                    A_log=dp.A_log, dt_bias=dp.dt_bias, z=dp.z, norm_w=dp.norm_w,
                    cu_seqlens=dp.cu_seqlens, N=dp.N, T_tot=dp.T, chunk=64,
                    dtype=bufs.dtype_code, out=bufs.out, workspace=bufs.workspace,
                    workspace_bytes=bufs.ws_bytes, initial_state=S, final_state=S,
                    impl=gdn.GDN_IMPL_TC_SPLIT, segments=4)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    ref = oracle_prefill(inp)
    assert relerr(np64(S), ref.final_state) <= PREFILL_TOL
    assert relerr(np64(bufs.out), ref.out) <= PREFILL_TOL


@pytest.mark.parametrize("impl", ["simt", "tc", "split", "fused"])
def test_397b_shapes_varlen(impl):
    code, chunk = IMPLS[impl]
    inp = make_prefill(P397, seqlens=(65, 130, 7, 64))
    bufs = run_prefill(inp, code, chunk)
    check_full(inp, bufs)


def test_in_place_state_update():
    """final_state may be the initial_state buffer itself."""
    w = resized(P9B, Hk=2, Hv=4, seed=31)
    inp = make_prefill(w, seqlens=(70, 5))
    dp = api.to_device(inp, chunk=32)
    bufs = api.PrefillBuffers(dp)
    S = dp.initial_state.clone()
    gdn.gdn_prefill(bufs.dims, mixed_qkv=dp.mixed_qkv, conv_w=dp.conv_w, a=dp.a, b=dp.b,
                    A_log=dp.A_log, dt_bias=dp.dt_bias, z=dp.z, norm_w=dp.norm_w,
                    cu_seqlens=dp.cu_seqlens, N=dp.N, T_tot=dp.T, chunk=32,
                    dtype=bufs.dtype_code, out=bufs.out, workspace=bufs.workspace,
                    workspace_bytes=bufs.ws_bytes, initial_state=S, final_state=S,
                    impl=gdn.GDN_IMPL_AUTO)
    torch.cuda.synchronize()
    ref = oracle_prefill(inp)
    assert relerr(np64(S), ref.final_state) <= PREFILL_TOL
    assert relerr(np64(bufs.out), ref.out) <= PREFILL_TOL


# ------------------------------------------------------- full-size workloads

_INPUTS = {}


def workload_inputs(name):
    """The full workload, drawn once per test session (cfg 4 takes ~20 s)."""
    if name not in _INPUTS:
        _INPUTS[name] = make_prefill(WORKLOADS[name])
    return _INPUTS[name]


def sampled_check(inp, bufs, pairs):
    worst = 0.0
    for n, h in pairs:
        ref, s, cols = oracle_subproblem(inp, n, h)
        e1 = relerr(np64(bufs.out[s, h]), ref.out[:, 0])
        e2 = relerr(np64(bufs.final_state[n, h]), ref.final_state[0, 0])
        np.testing.assert_array_equal(np64(bufs.conv_state_out[n][cols]), ref.conv_state_out[0])
        assert e1 <= PREFILL_TOL and e2 <= PREFILL_TOL, (n, h, e1, e2)
        worst = max(worst, e1, e2)
    return worst


# Value heads checked at full size: the first and the last head of four GQA
# groups (key heads 0, 7, 8 and 15), in every sequence.
SAMPLED_HEADS = {
    "prefill_4x8192_Hk16_Hv32_d128": [0, 1, 14, 15, 16, 17, 30, 31],
    "prefill_varlen8_T65536_Hk16_Hv64_d128": [0, 3, 28, 31, 32, 35, 60, 63],
}


def heads_check(inp, bufs, heads):
    """Every sequence, the given value heads: one multithreaded oracle run on
    the sub-layer made of those heads and the key heads they read (the mixer
    is separable over value heads, so its rows equal the full problem's)."""
    w = inp.w
    G, d = w.Hv // w.Hk, w.d
    kheads = sorted({h // G for h in heads})
    assert all(heads[2 * i] // G == heads[2 * i + 1] // G == kheads[i] for i in range(len(kheads)))
    q_cols = np.concatenate([np.arange(kh * d, (kh + 1) * d) for kh in kheads])
    v_cols = np.concatenate([2 * w.Hk * d + np.arange(h * d, (h + 1) * d) for h in heads])
    cols = np.concatenate([q_cols, w.Hk * d + q_cols, v_cols])
    zc = np.concatenate([np.arange(h * d, (h + 1) * d) for h in heads])
    ref = oracle.prefill(
        len(kheads), len(heads), d, d, inp.cu_seqlens, inp.mixed_qkv[:, cols], inp.conv_w[cols],
        inp.a[:, heads], inp.b[:, heads], inp.A_log[heads], inp.dt_bias[heads], inp.z[:, zc],
        inp.norm_w, None if inp.initial_state is None else inp.initial_state[:, heads],
        None if inp.conv_state_in is None else inp.conv_state_in[:, cols], scale=w.scale)
    e_out = relerr(np64(bufs.out[:, heads]), ref.out)
    e_S = relerr(np64(bufs.final_state[:, heads]), ref.final_state)
    np.testing.assert_array_equal(np64(bufs.conv_state_out[:, cols]), ref.conv_state_out)
    assert e_out <= PREFILL_TOL and e_S <= PREFILL_TOL, (e_out, e_S)
    return e_out, e_S


@pytest.mark.parametrize("impl", ["auto", "tc", "fused"])
def test_full_size_08b_every_head(impl):
    """The 0.8B-shaped workload (4096 tokens, 16/16 heads) at full size in the
    benchmark's launch configuration (AUTO) and on the single-kernel path:
    every output, the final state and the conv tail against the oracle."""
    inp = workload_inputs("prefill_T4096_Hk16_Hv16_d128")
    code = gdn.GDN_IMPL_AUTO if impl == "auto" else IMPLS[impl][0]
    bufs = run_prefill(inp, code, 64, guard=False)
    check_full(inp, bufs)


@pytest.mark.parametrize("name", list(SAMPLED_HEADS))
@pytest.mark.parametrize("impl", ["auto", "tc", "split", "fused"])
def test_full_size_sampled(name, impl):
    """The 9B- and 397B-shaped workloads at full size in the benchmark's
    launch configuration (AUTO), and on the single-kernel path: every
    sequence, eight value heads (first and last of four GQA groups)."""
    inp = workload_inputs(name)
    code = gdn.GDN_IMPL_AUTO if impl == "auto" else IMPLS[impl][0]
    bufs = run_prefill(inp, code, 64, guard=False)
    heads_check(inp, bufs, SAMPLED_HEADS[name])
    assert torch.isfinite(bufs.out.float()).all()


# The statement of the method writes o_t = S_t q_t with no factor on q: these
# cases run the whole mixer at q scale 1, where the gated RMSNorm passes the
# relative error of every token's o straight to its output (at dk^-1/2 the
# norm's eps damps it for the smallest outputs).
@pytest.mark.parametrize("impl", ["simt", "tc", "split", "fused"])
@pytest.mark.parametrize("name,seqlens", [
    ("prefill_T4096_Hk16_Hv16_d128", (1024,)),
    ("prefill_4x8192_Hk16_Hv32_d128", (700, 333, 1, 64)),
    ("prefill_varlen8_T65536_Hk16_Hv64_d128", (400, 90, 257)),
])
def test_unit_q_scale(impl, name, seqlens):
    w = resized(WORKLOADS[name], q_scale=1.0)
    inp = make_prefill(w, seqlens=seqlens, with_conv_state=True)
    code, chunk = IMPLS[impl]
    bufs = run_prefill(inp, code, chunk)
    check_full(inp, bufs)


def test_unit_q_scale_08b_full_size():
    """The full 0.8B-shaped workload at q scale 1 in the benchmark's launch
    configuration: every output against the oracle."""
    base = workload_inputs("prefill_T4096_Hk16_Hv16_d128")
    inp = dataclasses.replace(base, w=resized(base.w, q_scale=1.0))  # same draws, scale 1
    bufs = run_prefill(inp, gdn.GDN_IMPL_AUTO, 64, guard=False)
    check_full(inp, bufs)


@pytest.mark.parametrize("name", list(SAMPLED_HEADS))
def test_unit_q_scale_full_size_sampled(name):
    """The 9B- and 397B-shaped workloads at q scale 1, full size, AUTO:
    every sequence, eight value heads."""
    base = workload_inputs(name)
    inp = dataclasses.replace(base, w=resized(base.w, q_scale=1.0))  # same draws, scale 1
    bufs = run_prefill(inp, gdn.GDN_IMPL_AUTO, 64, guard=False)
    heads_check(inp, bufs, SAMPLED_HEADS[name])


# ------------------------------------------------------------------- decode


def run_decode(inp):
    dd = api.decode_to_device(inp)
    out = api.decode(dd)
    torch.cuda.synchronize()
    return dd, out


def oracle_decode(inp):
    w = inp.w
    return oracle.decode(w.Hk, w.Hv, w.d, w.d, inp.mixed_qkv, inp.conv_w, inp.a, inp.b, inp.A_log,
                         inp.dt_bias, inp.z, inp.norm_w, inp.state, inp.conv_state, scale=w.scale)


def test_decode_full_batch():
    """The full decode workload: batch 256, 16/32 heads, 512 MiB fp32 state."""
    inp = make_decode(D9B)
    dd, out = run_decode(inp)
    ref_out, ref_S, ref_cs = oracle_decode(inp)
    assert relerr(np64(dd.state), ref_S) <= DECODE_TOL
    assert relerr_beyond_bf16(np64(out), ref_out) <= DECODE_TOL
    np.testing.assert_array_equal(np64(dd.conv_state), ref_cs)


@pytest.mark.parametrize("d,Hk,Hv", [(32, 2, 2), (64, 2, 8), (128, 4, 16)])
def test_decode_fp32(d, Hk, Hv):
    w = resized(D9B, Hk=Hk, Hv=Hv, d=d, dtype="f32", seed=40 + d)
    inp = make_decode(w, batch=5)
    dd, out = run_decode(inp)
    ref_out, ref_S, ref_cs = oracle_decode(inp)
    assert relerr(np64(dd.state), ref_S) <= DECODE_TOL
    assert relerr(np64(out), ref_out) <= DECODE_TOL
    np.testing.assert_array_equal(np64(dd.conv_state), ref_cs)


def test_decode_bf16_state_full_batch():
    """The decode workload with its recurrent state held in bf16 (256 MiB):
    the step widens the state to fp32, updates it and rounds it back.  The
    oracle runs in fp64 from the same bf16 values; the new state and out
    must match beyond their own bf16 rounding."""
    import dataclasses
    from hybrid_linear_attention_05_b200.workloads import bf16_round
    inp = make_decode(D9B)
    inp = dataclasses.replace(inp, state=bf16_round(inp.state))
    dd = api.decode_to_device(inp, state_dtype=torch.bfloat16)
    out = api.decode(dd)
    torch.cuda.synchronize()
    ref_out, ref_S, ref_cs = oracle_decode(inp)
    assert relerr_beyond_bf16(np64(dd.state), ref_S) <= DECODE_TOL
    assert relerr_beyond_bf16(np64(out), ref_out) <= DECODE_TOL
    np.testing.assert_array_equal(np64(dd.conv_state), ref_cs)


@pytest.mark.parametrize("d,Hk,Hv,dtype", [(32, 2, 2, "f32"), (64, 2, 8, "bf16"), (128, 4, 16, "f32")])
def test_decode_bf16_state_shapes(d, Hk, Hv, dtype):
    """bf16 state at every head width, with fp32 and bf16 token inputs, over
    three steps in a row (each step reads the state the previous one rounded)."""
    import dataclasses
    from hybrid_linear_attention_05_b200.workloads import bf16_round
    w = resized(D9B, Hk=Hk, Hv=Hv, d=d, dtype=dtype, seed=90 + d)
    inp = make_decode(w, batch=5)
    inp = dataclasses.replace(inp, state=bf16_round(inp.state))
    dd = api.decode_to_device(inp, state_dtype=torch.bfloat16)
    state, conv = inp.state, inp.conv_state
    for step in range(3):
        out = api.decode(dd)
        torch.cuda.synchronize()
        cur = dataclasses.replace(inp, state=state, conv_state=conv)
        ref_out, ref_S, ref_cs = oracle_decode(cur)
        got_S = np64(dd.state)
        assert relerr_beyond_bf16(got_S, ref_S) <= DECODE_TOL, step
        if dtype == "f32":
            assert relerr(np64(out), ref_out) <= DECODE_TOL, step
        else:
            assert relerr_beyond_bf16(np64(out), ref_out) <= DECODE_TOL, step
        np.testing.assert_array_equal(np64(dd.conv_state), ref_cs)
        state, conv = got_S.astype(np.float32), ref_cs.astype(np.float32)


@pytest.mark.parametrize("T,state_dtype,d,Hk,Hv", [
    (2, "f32", 128, 16, 32), (3, "f32", 32, 2, 2), (4, "f32", 64, 2, 8), (8, "bf16", 128, 4, 16)])
def test_decode_multi_token(T, state_dtype, d, Hk, Hv):
    """Short multi-token decode: one gdn_decode step of T tokens per sequence
    equals the fp64 oracle's prefill of those T tokens from the same state and
    conv history (out, final state, conv cache)."""
    from hybrid_linear_attention_05_b200.workloads import bf16_round
    w = resized(D9B, Hk=Hk, Hv=Hv, d=d, seed=100 + T)
    B = 6
    tok = make_decode(w, batch=B * T)  # row b * T + t: token t of sequence b
    state = tok.state[:B].copy()
    if state_dtype == "bf16":
        state = bf16_round(state)
    cs = tok.conv_state[:B].copy()
    t = lambda x, dt=torch.bfloat16: torch.from_numpy(np.ascontiguousarray(x)).cuda().to(dt)  # noqa: E731
    dd = api.DeviceDecode(
        Hk=w.Hk, Hv=w.Hv, d=w.d, scale=w.scale, B=B, mixed_qkv=t(tok.mixed_qkv), conv_w=t(tok.conv_w),
        a=t(tok.a), b=t(tok.b), A_log=t(tok.A_log, torch.float32), dt_bias=t(tok.dt_bias, torch.float32),
        z=t(tok.z), norm_w=t(tok.norm_w),
        state=t(state, torch.float32 if state_dtype == "f32" else torch.bfloat16), conv_state=t(cs))
    out = api.decode(dd, T=T)
    torch.cuda.synchronize()
    cu = np.arange(B + 1, dtype=np.int32) * T
    ref = oracle.prefill(w.Hk, w.Hv, w.d, w.d, cu, tok.mixed_qkv, tok.conv_w, tok.a, tok.b, tok.A_log,
                         tok.dt_bias, tok.z, tok.norm_w, state, cs, scale=w.scale)
    assert relerr_beyond_bf16(np64(out).reshape(B * T, w.Hv, w.d), ref.out) <= DECODE_TOL
    if state_dtype == "f32":
        assert relerr(np64(dd.state), ref.final_state) <= DECODE_TOL
    else:
        assert relerr_beyond_bf16(np64(dd.state), ref.final_state) <= DECODE_TOL
    np.testing.assert_array_equal(np64(dd.conv_state), ref.conv_state_out)


def test_prefill_then_decode_composition():
    """prefill of T tokens followed by a decode of token T+1 equals the
    oracle's prefill of T+1 tokens (state and last output)."""
    w = resized(P9B, Hk=2, Hv=4, seed=50)
    T = 70
    inp = make_prefill(w, seqlens=(T + 1, T + 1), with_conv_state=True)
    cu = inp.cu_seqlens
    first = np.concatenate([np.arange(cu[n], cu[n] + T) for n in range(2)])
    last = cu[1:] - 1
    import dataclasses
    pre = dataclasses.replace(inp, cu_seqlens=np.array([0, T, 2 * T], np.int32),
                              mixed_qkv=inp.mixed_qkv[first], a=inp.a[first], b=inp.b[first],
                              z=inp.z[first])
    bufs = run_prefill(pre, gdn.GDN_IMPL_AUTO, 32, guard=False)
    dd = api.DeviceDecode(
        Hk=w.Hk, Hv=w.Hv, d=w.d, scale=w.scale, B=2,
        mixed_qkv=torch.from_numpy(inp.mixed_qkv[last]).cuda().bfloat16(),
        conv_w=torch.from_numpy(inp.conv_w).cuda().bfloat16(),
        a=torch.from_numpy(inp.a[last]).cuda().bfloat16(), b=torch.from_numpy(inp.b[last]).cuda().bfloat16(),
        A_log=torch.from_numpy(inp.A_log).cuda(), dt_bias=torch.from_numpy(inp.dt_bias).cuda(),
        z=torch.from_numpy(inp.z[last]).cuda().bfloat16(),
        norm_w=torch.from_numpy(inp.norm_w).cuda().bfloat16(),
        state=bufs.final_state.clone(), conv_state=bufs.conv_state_out.clone())
    out = api.decode(dd)
    torch.cuda.synchronize()
    ref = oracle_prefill(inp)
    assert relerr(np64(dd.state), ref.final_state) <= PREFILL_TOL
    assert relerr(np64(out), ref.out[last]) <= PREFILL_TOL
    np.testing.assert_array_equal(np64(dd.conv_state), ref.conv_state_out)


# ------------------------------------------------------------- core only


def rounded(x, dtype):
    """x as float64 holding exactly the values of its `dtype` copy."""
    if dtype == torch.float32:
        return x.astype(np.float32).astype(np.float64)
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dtype).double().numpy()


def run_core(q, k, v, g, beta, cu, Hk, Hv, d, chunk, impl, S0=None, dtype=torch.float32):
    dev = "cuda"
    T = q.shape[0]
    N = len(cu) - 1
    t = lambda x, dt=dtype: torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(dev, dt)
    o = torch.empty((T, Hv, d), dtype=torch.float32, device=dev)
    S = torch.empty((N, Hv, d, d), dtype=torch.float32, device=dev)
    # room for every path: the fused kernel's queue, the two-kernel path's records
    ws = torch.empty(gdn.gdn_core_workspace_size_split(gdn.make_dims(Hk, Hv, d), N, T), dtype=torch.uint8,
                     device=dev)
    status = gdn.gdn_chunk_core(
        gdn.make_dims(Hk, Hv, d, scale=1.0), q=t(q), k=t(k), v=t(v),
        g=t(np.ascontiguousarray(g.T), torch.float32), beta=t(np.ascontiguousarray(beta.T), torch.float32),
        cu_seqlens=torch.tensor(cu, dtype=torch.int32, device=dev), N=N, T_tot=T, chunk=chunk,
        dtype=gdn.dtype_code(t(q)), o=o, initial_state=None if S0 is None else t(S0, torch.float32),
        final_state=S, impl=impl, workspace=ws, workspace_bytes=ws.numel(), raise_on_error=False)
    if status == gdn.GDN_ERR_UNSUPPORTED:
        pytest.skip("implementation not available for this shape")
    assert status == gdn.GDN_OK
    torch.cuda.synchronize()
    return np64(o), np64(S)


@pytest.mark.parametrize("impl,d,chunk,dtype", [
    ("simt", 32, 16, torch.float32), ("simt", 128, 32, torch.float32),
    ("tc", 128, 64, torch.float16), ("split", 128, 64, torch.float16), ("fused", 128, 64, torch.float16)])
def test_core_orthonormal_overwrite(impl, d, chunk, dtype):
    """alpha = 1, beta = 1, orthonormal keys: S k_i = v_i after writing, and
    a rewritten key returns its new value (exact in real arithmetic)."""
    code = IMPLS[impl][0]
    rng = np.random.default_rng(60)
    m = min(d, 40)
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm[:, :m].T
    if dtype != torch.float32:  # keys exactly representable: use signed unit vectors
        keys = np.eye(d)[rng.permutation(d)[:m]] * rng.choice([-1.0, 1.0], size=(m, 1))
    vals = rng.standard_normal((m, d))
    order = np.concatenate([np.arange(m), [0, 1]])
    newv = rng.standard_normal((2, d))
    kseq = keys[order]
    vseq = np.concatenate([vals, newv])
    vseq = rounded(vseq, dtype)
    T = len(order)
    k = kseq[:, None, :]
    o, S = run_core(k, k, vseq[:, None, :], np.zeros((T, 1)), np.ones((T, 1)), [0, T], 1, 1, d,
                    chunk, code, dtype=dtype)
    tol = 1e-4 if dtype == torch.float32 else PREFILL_TOL
    exp_vals = vseq[:m].copy()
    exp_vals[0], exp_vals[1] = vseq[m], vseq[m + 1]
    got = S[0, 0] @ keys.T  # column i = S k_i
    assert relerr(got.T, exp_vals) <= tol
    assert relerr(o[:m, 0], vseq[:m]) <= tol  # read-back right after each write


@pytest.mark.parametrize("impl,d,chunk,dtype", [
    ("simt", 64, 32, torch.float32), ("tc", 128, 64, torch.float16),
    ("split", 128, 64, torch.float16), ("fused", 128, 64, torch.float16)])
def test_core_beta_zero_only_decays(impl, d, chunk, dtype):
    code = IMPLS[impl][0]
    rng = np.random.default_rng(61)
    T, Hv = 150, 2
    q = rng.standard_normal((T, 1, d)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k = rng.standard_normal((T, 1, d)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, Hv, d))
    g = -rng.uniform(0, 0.05, (T, Hv))
    S0 = rng.standard_normal((1, Hv, d, d)) * 0.1
    q, k, v = [rounded(x, dtype) for x in (q, k, v)]
    o, S = run_core(q, k, v, g, np.zeros((T, Hv)), [0, T], 1, Hv, d, chunk, code, S0=S0, dtype=dtype)
    cum = np.exp(np.cumsum(g, axis=0))
    tol = 1e-4 if dtype == torch.float32 else PREFILL_TOL
    for h in range(Hv):
        assert relerr(S[0, h], cum[-1, h] * S0[0, h]) <= tol
        assert relerr(o[:, h], cum[:, h:h + 1] * (q[:, 0] @ S0[0, h].T)) <= tol


@pytest.mark.parametrize("impl,d,chunk,dtype", [
    ("simt", 32, 16, torch.float32), ("simt", 128, 32, torch.bfloat16),
    ("simt", 64, 64, torch.float16), ("tc", 128, 64, torch.float16),
    ("split", 128, 64, torch.float16), ("fused", 128, 64, torch.float16)])
def test_core_matches_oracle(impl, d, chunk, dtype):
    code = IMPLS[impl][0]
    rng = np.random.default_rng(62)
    Hk, Hv = 2, 4
    lens = [3 * chunk + 11, 1, chunk]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    q = rng.standard_normal((T, Hk, d)); q /= np.linalg.norm(q, axis=-1, keepdims=True) * np.sqrt(d)
    k = rng.standard_normal((T, Hk, d)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, Hv, d))
    g = -np.exp(rng.uniform(0, np.log(16), Hv))[None] * np.log1p(np.exp(rng.standard_normal((T, Hv))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, Hv))))
    S0 = rng.standard_normal((3, Hv, d, d)) * 0.02
    q, k, v = [rounded(x, dtype) for x in (q, k, v)]
    g = g.astype(np.float32).astype(np.float64)
    beta = beta.astype(np.float32).astype(np.float64)
    o, S = run_core(q, k, v, g, beta, cu, Hk, Hv, d, chunk, code, S0=S0, dtype=dtype)
    o_ref, S_ref = oracle.core(Hk, Hv, d, d, cu, q, k, v, g, beta, S0.astype(np.float32))
    tol = 1e-4 if dtype == torch.float32 else PREFILL_TOL
    assert relerr(o, o_ref) <= tol
    assert relerr(S, S_ref) <= tol


def test_no_device_error_recorded():
    """Every bounded wait inside the tensor-core kernel completed."""
    assert gdn.gdn_device_error(clear=True) == 0
