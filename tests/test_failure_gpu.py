"""The failure path of the kernels' bounded waits, exercised on the GPU
without a fault: a test kernel waits on an mbarrier that nothing arrives at,
gives up after 1 ms and records the timeout in the library's error word.  The
test checks that the kernel returns, that gdn_device_error reports
GDN_ERR_TIMEOUT and clears it, and that the library is usable afterwards (a
prefill on the same context matches the oracle)."""
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


def test_bounded_wait_gives_up_and_reports():
    assert gdn.gdn_device_error(clear=True) == 0  # nothing recorded before
    gdn.gdn_selftest_bounded_wait(1000)
    torch.cuda.synchronize()  # the kernel returned by itself
    assert gdn.gdn_device_error(clear=True) == gdn.GDN_ERR_TIMEOUT
    assert gdn.gdn_device_error(clear=True) == 0  # cleared


@pytest.mark.parametrize("impl", [gdn.GDN_IMPL_AUTO, gdn.GDN_IMPL_TC_FUSED])
def test_library_usable_after_a_timeout(impl):
    gdn.gdn_selftest_bounded_wait(1000)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(clear=True) == gdn.GDN_ERR_TIMEOUT
    w = resized(WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"], Hk=4, Hv=8, seed=90)
    inp = make_prefill(w, seqlens=(150, 70))
    res = api.prefill(api.to_device(inp), impl=impl)
    torch.cuda.synchronize()
    assert gdn.gdn_device_error(clear=True) == 0
    ref = oracle_prefill(inp)
    assert relerr(res.out.float().cpu().numpy(), ref.out) <= PREFILL_TOL
    assert relerr(res.final_state.cpu().numpy(), ref.final_state) <= PREFILL_TOL
