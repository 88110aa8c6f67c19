"""GPU parity of the context-parallel pieces through the C ABI:
``gdn_prefill_state_map`` against the oracle's (M, R), ``gdn_state_fold``
against an fp64 fold, and a whole context-parallel prefill, its parts run one
after another on one device, against the oracle's prefill of the sequence.

Bars: 5e-3 of max|ref| for the maps and the prefill (the prefill bar: bf16
inputs, fp16 tensor-core operands, fp32 accumulation); 2e-5 for the fold
(fp32 products of length 128 on the CUDA cores).
"""
import numpy as np
import pytest

from gdn_testlib import PREFILL_TOL, oracle_prefill, relerr
import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_05_b200 import api, build, gdn  # noqa: E402
from hybrid_linear_attention_05_b200 import context_parallel as cp  # noqa: E402
from hybrid_linear_attention_05_b200.workloads import WORKLOADS, make_prefill, resized  # noqa: E402

P9B = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]
SLOW_DECAY = (-7.0, -5.0)  # alpha near 1: M stays far from 0 over many chunks
FOLD_TOL = 2e-5


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gdn.lib()


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_maps(inp):
    w, cu = inp.w, inp.cu_seqlens
    res = []
    for n in range(len(cu) - 1):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        hist = None if inp.conv_state_in is None else inp.conv_state_in[n:n + 1]
        res.append(oracle.state_map(w.Hk, w.Hv, w.d, w.d, inp.mixed_qkv[sl], inp.conv_w, inp.a[sl],
                                    inp.b[sl], inp.A_log, inp.dt_bias, conv_state_in=hist, scale=w.scale))
    return res


@pytest.mark.parametrize("segments,seqlens", [
    (1, (64 * 5 + 7,)),
    (3, (64 * 7 + 13, 130, 0)),
    (7, (64 * 3, 1)),            # more segments than chunks: empty segments are identity maps
    (0, (64 * 9 + 1, 64 * 2)),
])
def test_state_map_matches_oracle(segments, seqlens):
    """M and R of every sequence (GQA, conv history, ragged and empty
    sequences), with one chain and with segments composed in fp32; the conv
    tail written beside them is exact."""
    w = resized(P9B, Hk=2, Hv=4, seed=90 + segments, A_log_range=SLOW_DECAY)
    inp = make_prefill(w, seqlens=seqlens, with_conv_state=True)
    dp = api.to_device(inp, chunk=64)
    bufs = api.PrefillBuffers(dp)
    cs_out = torch.full_like(bufs.conv_state_out, float("nan"))
    maps = api.state_map(dp, bufs, segments=segments, conv_state_out=cs_out)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    for n, (M, R) in enumerate(oracle_maps(inp)):
        assert np.max(np.abs(M)) > 0.05
        assert relerr(np64(maps[n, :, 0]), M) <= PREFILL_TOL
        if np.max(np.abs(R)) > 0:
            assert relerr(np64(maps[n, :, 1]), R) <= PREFILL_TOL
        else:
            assert np.max(np.abs(np64(maps[n, :, 1]))) == 0.0
    np.testing.assert_array_equal(np64(cs_out), oracle_prefill(inp).conv_state_out)


def test_state_map_many_chains():
    """17 sequences x 4 value heads (68 chains, past the segment buffers): one
    serial chain per (sequence, head) writes its maps straight into the
    caller's array."""
    w = resized(P9B, Hk=2, Hv=4, seed=96, A_log_range=SLOW_DECAY)
    rng = np.random.default_rng(96)
    seqlens = tuple(int(x) for x in rng.integers(1, 200, 17))
    inp = make_prefill(w, seqlens=seqlens, with_conv_state=True)
    dp = api.to_device(inp, chunk=64)
    maps = api.state_map(dp)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    for n, (M, R) in enumerate(oracle_maps(inp)):
        assert relerr(np64(maps[n, :, 0]), M) <= PREFILL_TOL
        assert relerr(np64(maps[n, :, 1]), R) <= PREFILL_TOL


@pytest.mark.parametrize("count,with_first,in_place", [(0, True, False), (0, False, False), (1, False, False),
                                                        (3, True, False), (5, True, True)])
def test_state_fold_matches_fp64(count, with_first, in_place):
    """S <- S M_s + R_s over `count` maps of two sequences and three heads."""
    rng = np.random.default_rng(100 + count)
    N, Hv, d = 2, 3, 128
    M = np.eye(d) * 0.8 + rng.standard_normal((count, N, Hv, d, d)) * (0.3 / np.sqrt(d))
    R = rng.standard_normal((count, N, Hv, d, d)) * 0.1
    maps = np.stack([M, R], axis=3).astype(np.float32)
    S0 = rng.standard_normal((N, Hv, d, d)).astype(np.float32) * 0.2 if with_first else None
    ref = np.zeros((N, Hv, d, d)) if S0 is None else S0.astype(np.float64)
    for s in range(count):
        ref = ref @ maps[s, :, :, 0].astype(np.float64) + maps[s, :, :, 1]
    dev_maps = torch.from_numpy(maps).cuda()
    first = None if S0 is None else torch.from_numpy(S0).cuda()
    out = first if in_place else None
    got = api.state_fold(dev_maps, first, Hk=1, Hv=Hv, d=d, out=out)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    if count == 0:
        np.testing.assert_array_equal(np64(got), 0.0 if S0 is None else S0)
    else:
        assert relerr(np64(got), ref) <= FOLD_TOL


@pytest.mark.parametrize("lens", [(2, 64 * 5 + 3, 0, 1, 64 * 6 + 30), (64 * 4, 64 * 4, 64 * 4 + 17)])
def test_context_parallel_parts_on_one_device(lens):
    """One sequence cut into parts (parts of 0, 1 and 2 tokens among them):
    every part's map, the fold of the earlier ones from the sequence's own
    initial state and conv history, the part's prefill from there.  The
    concatenated outputs and the final state match the oracle's prefill of
    the whole sequence, and the library's own single call."""
    T = sum(lens)
    w = resized(P9B, Hk=2, Hv=4, seed=97 + len(lens), A_log_range=SLOW_DECAY, s0_std=0.02)
    inp = make_prefill(w, seqlens=(T,), with_conv_state=True)
    dp = api.to_device(inp, chunk=64)
    parts = cp.split_sequence(dp, lens)
    res = cp.prefill_parts_local(parts, initial_state=dp.initial_state, conv_state_in=dp.conv_state_in)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    out = torch.cat([r.out for r in res])
    ref = oracle_prefill(inp)
    assert relerr(np64(out), ref.out) <= PREFILL_TOL
    assert relerr(np64(res[-1].final_state), ref.final_state) <= PREFILL_TOL
    whole = api.prefill(dp)
    assert relerr(np64(out), np64(whole.out)) <= PREFILL_TOL
    assert relerr(np64(res[-1].final_state), np64(whole.final_state)) <= PREFILL_TOL


def test_prefill_on_a_state_maps_workspace_is_the_full_prefill():
    """gdn_prefill with reuse_workspace after gdn_prefill_state_map on the same
    inputs skips the conv and key-side kernels and gives exactly the result
    of the full call (same records, same chains)."""
    w = resized(P9B, Hk=2, Hv=4, seed=98, A_log_range=SLOW_DECAY, s0_std=0.02)
    inp = make_prefill(w, seqlens=(64 * 7 + 5, 64 * 2), with_conv_state=True)
    dp = api.to_device(inp, chunk=64)
    full = api.prefill(dp)
    out, S = full.out.clone(), full.final_state.clone()
    bufs = api.PrefillBuffers(dp)
    api.state_map(dp, bufs)
    r = api.prefill(dp, bufs=bufs, reuse_workspace=True)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(True) == 0
    assert torch.equal(r.out, out)
    assert torch.equal(r.final_state, S)
