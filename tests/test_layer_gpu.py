"""GPU parity of the projections around the mixer (gdn_linear) and of the
whole layer (gdn_layer_prefill: in_proj, mixer, out_proj) against the fp64
oracle ("Qwen/Qwen3.5-9B", module tree of a Gated DeltaNet block).

Bars: each projection output within its own bf16 rounding plus 1e-4 of
max|ref| (fp32 accumulation of bf16 products); the layer output within the
mixer's 5e-3 (relative to max|ref|)."""
import numpy as np
import pytest

from gdn_testlib import PREFILL_TOL, relerr, relerr_beyond_bf16
import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_05_b200 import api, build, gdn  # noqa: E402
from hybrid_linear_attention_05_b200.workloads import WORKLOADS, bf16_round, make_layer  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gdn.lib()


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).cuda().bfloat16()


@pytest.mark.parametrize("M,splits,K", [
    (333, [64, 128, 8, 8], 128),          # ragged rows, four ranges, one K tile pair
    (1000, [512], 4096),
    (129, [8192, 4096, 32, 32], 4096),    # the 9B in_proj columns (qkv | z | b | a)
    (256, [4096], 4096),                  # the 9B out_proj
    (1, [256], 64),                       # one row, one K tile
    (7, [24, 8], 192),                    # a few rows, ranges inside one column tile
])
def test_linear_matches_fp64_product(M, splits, K):
    rng = np.random.default_rng(M + K)
    N = sum(splits)
    x = bf16_round(rng.standard_normal((M, K)).astype(np.float32))
    w = bf16_round((rng.standard_normal((N, K)) * K ** -0.5).astype(np.float32))
    outs = api.linear(bf(x), bf(w), splits)
    outs = outs if isinstance(outs, list) else [outs]
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    ref = x.astype(np.float64) @ w.astype(np.float64).T
    c = 0
    for o, n in zip(outs, splits):
        assert relerr_beyond_bf16(np64(o), ref[:, c:c + n]) <= 1e-4, (c, n)
        c += n


def test_linear_full_9b_in_proj_sampled_rows():
    """The 9B in_proj at the 9B-shaped workload's size (32768 rows, 12352
    columns, K = 4096): sampled rows against their fp64 products."""
    rng = np.random.default_rng(5)
    M, K = 32768, 4096
    splits = [8192, 4096, 32, 32]
    N = sum(splits)
    x = bf16_round(rng.standard_normal((M, K)).astype(np.float32))
    w = bf16_round((rng.standard_normal((N, K)) * K ** -0.5).astype(np.float32))
    outs = api.linear(bf(x), bf(w), splits)
    torch.cuda.synchronize()
    y = torch.cat(outs, dim=1)
    rows = np.array([0, 1, 127, 128, 4095, 16384, 32639, 32767])
    ref = x[rows].astype(np.float64) @ w.astype(np.float64).T
    assert relerr_beyond_bf16(np64(y[torch.from_numpy(rows).cuda()]), ref) <= 1e-4


@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_TC_FUSED, gdn.GDN_IMPL_TC_SPLIT])
def test_layer_matches_oracle_9b(impl):
    """The whole layer at the 9B shapes (d_model 4096, 16 key / 32 value heads
    of width 128): several sequences, one shorter than the conv window, conv
    history and initial states."""
    w = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]
    li = make_layer(w, 4096, seqlens=(300, 1, 65), with_conv_state=True)
    dl = api.layer_to_device(li)
    bufs = api.layer_prefill(dl, impl=impl)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    m = li.mixer
    Cc, HVd = w.Cc, w.Hv * w.d
    ref = oracle.layer(w.Hk, w.Hv, w.d, w.d, m.cu_seqlens, li.hidden, li.w_in[:Cc], li.w_in[Cc:Cc + HVd],
                       li.w_in[Cc + HVd + w.Hv:], li.w_in[Cc + HVd:Cc + HVd + w.Hv], li.w_out, m.conv_w, m.A_log,
                       m.dt_bias, m.norm_w, m.initial_state, m.conv_state_in, scale=w.scale)
    assert relerr(np64(bufs.y), ref.y) <= PREFILL_TOL
    assert relerr(np64(bufs.final_state), ref.mixer.final_state) <= PREFILL_TOL
    # conv_state_out carries projected values verbatim: fp32 accumulation can put
    # one on the other side of a bf16 rounding midpoint than the fp64 product, so
    # allow one bf16 ulp of each value (plus accumulation error near zero)
    cs, ref_cs = np64(bufs.conv_state_out), ref.mixer.conv_state_out
    assert np.all(np.abs(cs - ref_cs) <= 2.0 ** -7 * np.abs(ref_cs) + 1e-5 * np.abs(ref_cs).max())


def test_layer_unit_q_scale_and_no_records():
    """The layer at q scale 1 with only the base workspace (the mixer then
    runs without records)."""
    from hybrid_linear_attention_05_b200.workloads import resized
    w = resized(WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"], q_scale=1.0, Hk=4, Hv=8, seed=44)
    li = make_layer(w, 1024, seqlens=(200, 90))
    dl = api.layer_to_device(li)
    bufs = api.LayerBuffers(dl, records=False)
    api.layer_prefill(dl, bufs=bufs)
    torch.cuda.synchronize()
    m = li.mixer
    Cc, HVd = w.Cc, w.Hv * w.d
    ref = oracle.layer(w.Hk, w.Hv, w.d, w.d, m.cu_seqlens, li.hidden, li.w_in[:Cc], li.w_in[Cc:Cc + HVd],
                       li.w_in[Cc + HVd + w.Hv:], li.w_in[Cc + HVd:Cc + HVd + w.Hv], li.w_out, m.conv_w, m.A_log,
                       m.dt_bias, m.norm_w, m.initial_state, m.conv_state_in, scale=w.scale)
    assert relerr(np64(bufs.y), ref.y) <= PREFILL_TOL


def test_linear_strided_rows():
    """X and W with row strides larger than K (a column slice of wider
    tensors), and an output range with a row stride larger than its columns."""
    rng = np.random.default_rng(9)
    M, N, K = 300, 136, 256
    xw = bf16_round(rng.standard_normal((M, K + 64)).astype(np.float32))
    ww = bf16_round((rng.standard_normal((N, K + 128)) * K ** -0.5).astype(np.float32))
    x_t, w_t = bf(xw), bf(ww)
    y = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    gdn.gdn_linear(x=x_t, w=w_t, M=M, N=N, K=K, ldx=K + 64, ldw=K + 128, outs=[(y, N, N + 8)])
    torch.cuda.synchronize()
    ref = xw[:, :K].astype(np.float64) @ ww[:, :K].astype(np.float64).T
    got = np64(y)
    assert relerr_beyond_bf16(got[:, :N], ref) <= 1e-4
    assert np.all(got[:, N:] == 0)  # the columns past the range are not written


def test_layer_matches_oracle_397b():
    """The whole layer at the 397B shapes (16 key / 64 value heads, d_model
    4096): in_proj of 20 608 columns, two sequences with initial states."""
    w = WORKLOADS["prefill_varlen8_T65536_Hk16_Hv64_d128"]
    li = make_layer(w, 4096, seqlens=(130, 77))
    dl = api.layer_to_device(li)
    bufs = api.layer_prefill(dl)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    m = li.mixer
    Cc, HVd = w.Cc, w.Hv * w.d
    ref = oracle.layer(w.Hk, w.Hv, w.d, w.d, m.cu_seqlens, li.hidden, li.w_in[:Cc], li.w_in[Cc:Cc + HVd],
                       li.w_in[Cc + HVd + w.Hv:], li.w_in[Cc + HVd:Cc + HVd + w.Hv], li.w_out, m.conv_w, m.A_log,
                       m.dt_bias, m.norm_w, m.initial_state, m.conv_state_in, scale=w.scale)
    assert relerr(np64(bufs.y), ref.y) <= PREFILL_TOL
    assert relerr(np64(bufs.final_state), ref.mixer.final_state) <= PREFILL_TOL


def test_layer_full_size_window_tails():
    """The whole layer at the 9B workload's full size (4 x 8192 tokens, d_model
    4096) in the launch the bench times.  The last 128 tokens of every
    sequence are checked against the oracle's layer run on that sequence's
    last 1024 tokens alone, from a zero state, with the projected inputs of
    the three tokens before them as the conv history: the workloads' gates
    decay the state by e^-45 or more per 64-token chunk, so the state at the
    window's start cannot matter."""
    w = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]
    li = make_layer(w, 4096)
    dl = api.layer_to_device(li)
    bufs = api.layer_prefill(dl)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    m = li.mixer
    Cc, HVd = w.Cc, w.Hv * w.d
    W_qkv = li.w_in[:Cc]
    y = bufs.y
    for n in range(m.N):
        end = int(m.cu_seqlens[n + 1])
        lo = end - 1024
        hist = oracle.bf16(li.hidden[lo - 3:lo].astype(np.float64) @ W_qkv.astype(np.float64).T).T[None]
        ref = oracle.layer(w.Hk, w.Hv, w.d, w.d, [0, 1024], li.hidden[lo:end], W_qkv, li.w_in[Cc:Cc + HVd],
                           li.w_in[Cc + HVd + w.Hv:], li.w_in[Cc + HVd:Cc + HVd + w.Hv], li.w_out, m.conv_w,
                           m.A_log, m.dt_bias, m.norm_w, None, hist, scale=w.scale)
        assert relerr(np64(y[end - 128:end]), ref.y[-128:]) <= PREFILL_TOL, n
