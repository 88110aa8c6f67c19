"""gdn_prefill_noalloc, checked against gdn_prefill.

Some callers of this library cannot allocate device memory for gdn_prefill's
workspace: an operator plugin handed only its input and output tensors, with
no allocator for temporaries, or a serving runtime that has divided up all
device memory in advance and allows no allocation while it runs.
gdn_prefill_noalloc serves them from a fixed scratch array held inside the
library.  These tests call it through the C ABI, twice in a row (the scratch
keeps the previous call's contents), and compare with gdn_prefill on the same
inputs.  The file name sorts last so that a run that stops at the first
failure has already run every other test; it also passes on its own in a
fresh process, where its first call is the one that sets the scratch up.
"""
import numpy as np
import pytest

from gdn_testlib import PREFILL_TOL, oracle_prefill, relerr

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_05_b200 import api, build, gdn  # noqa: E402
from hybrid_linear_attention_05_b200.workloads import WORKLOADS, make_prefill, resized  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gdn.lib()


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_SIMT])
def test_noalloc_matches_prefill_on_two_calls(impl):
    w = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]
    inp = make_prefill(w, seqlens=(700, 1, 129, 64), with_conv_state=True)
    chunk = 64 if impl == gdn.GDN_IMPL_AUTO else 32
    dp = api.to_device(inp, chunk=chunk)
    ref = api.prefill(dp, impl=impl)
    ref_out, ref_S, ref_cs = ref.out.clone(), ref.final_state.clone(), ref.conv_state_out.clone()
    torch.cuda.synchronize()
    dims = gdn.make_dims(dp.Hk, dp.Hv, dp.d, scale=dp.scale)
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        S = torch.full_like(ref_S, float("nan"))
        cs = torch.full_like(ref_cs, float("nan"))
        gdn.gdn_prefill_noalloc(
            dims, mixed_qkv=dp.mixed_qkv, conv_w=dp.conv_w, a=dp.a, b=dp.b, A_log=dp.A_log,
            dt_bias=dp.dt_bias, z=dp.z, norm_w=dp.norm_w, cu_seqlens=dp.cu_seqlens, N=dp.N,
            T_tot=dp.T, chunk=dp.chunk, dtype=gdn.dtype_code(dp.mixed_qkv), out=out,
            initial_state=dp.initial_state, final_state=S, conv_state_in=dp.conv_state_in,
            conv_state_out=cs, impl=impl)
        torch.cuda.synchronize()
        assert relerr(np64(out), np64(ref_out)) <= PREFILL_TOL
        assert relerr(np64(S), np64(ref_S)) <= PREFILL_TOL
        np.testing.assert_array_equal(np64(cs), np64(ref_cs))
    # and the second call's results against the fp64 oracle itself
    oref = oracle_prefill(inp)
    assert relerr(np64(out), oref.out) <= PREFILL_TOL
    assert relerr(np64(S), oref.final_state) <= PREFILL_TOL
    np.testing.assert_array_equal(np64(cs), oref.conv_state_out)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A batch whose workspace exceeds the built-in scratch is refused with
    GDN_ERR_WORKSPACE before anything is launched."""
    dims = gdn.make_dims(16, 16, 128)
    fake = 1 << 20  # never dereferenced: the size check comes first
    T_ok = 3000
    T_big = 3500
    assert gdn.gdn_prefill_workspace_size(dims, T_ok, gdn.GDN_BF16) <= gdn.GDN_NOALLOC_SCRATCH_BYTES
    assert gdn.gdn_prefill_workspace_size(dims, T_big, gdn.GDN_BF16) > gdn.GDN_NOALLOC_SCRATCH_BYTES
    status = gdn.gdn_prefill_noalloc(
        dims, mixed_qkv=fake, conv_w=fake, a=fake, b=fake, A_log=fake, dt_bias=fake, z=fake,
        norm_w=fake, cu_seqlens=fake, N=1, T_tot=T_big, chunk=64, dtype=gdn.GDN_BF16, out=fake,
        raise_on_error=False)
    assert status == gdn.GDN_ERR_WORKSPACE
