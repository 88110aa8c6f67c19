"""The prefill at the model's maximum context: one sequence of 262 144 tokens
("Qwen/Qwen3.5-9B", config: max_position_embeddings 262144) at the 9B mixer
shapes (16 key / 32 value heads of width 128, bf16), in the launch the
library picks (the two-kernel path with a segmented state chain).

The oracle cannot run the whole sequence in a test, so the checks use a
property that holds at any length: with the workloads' gates (A_log ~ U(0,
ln 16)) every 64-token chunk decays the state by e^-45 or more, so the outputs
of the last tokens of a window, and the state at its end, do not depend on the
state at the window's start.  The oracle runs windows of 1024 tokens from a
zero state, with the three raw inputs before each window as its conv history,
and the GPU's outputs there (and its final state) must match to the prefill
bar.  The first tokens are checked against the oracle from the sequence's
true start.  Inputs are drawn on the device from a seeded generator, with the
workloads' distributions.
"""
import numpy as np
import pytest

from gdn_testlib import PREFILL_TOL, relerr
import oracle

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from hybrid_linear_attention_05_b200 import api, build, gdn  # noqa: E402

T = 262144
HK, HV, D = 16, 32, 128
CC = 2 * HK * D + HV * D
WINDOW = 1024
CHECK = 128  # tokens compared at the end of each window


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    gdn.lib()


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def device_normal(gen, shape, std=1.0, rows_per_slice=16384):
    """bf16 draws of N(0, std) made on the device in row slices (bounded fp32 scratch)."""
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, shape[0], rows_per_slice):
        r1 = min(shape[0], r0 + rows_per_slice)
        out[r0:r1] = (torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen, device="cuda") * std).bfloat16()
    return out


@pytest.fixture(scope="module")
def run():
    rng = np.random.Generator(np.random.PCG64(262144))
    bf = lambda x: torch.from_numpy(np.ascontiguousarray(x, np.float32)).bfloat16()  # noqa: E731
    conv_w = bf(rng.standard_normal((CC, 4)) * 0.25)
    A_log = rng.uniform(0.0, np.log(16.0), HV).astype(np.float32)
    dt_bias = (rng.standard_normal(HV) * 0.1).astype(np.float32)
    norm_w = bf(1.0 + rng.standard_normal(D) * 0.1)
    S0 = (rng.standard_normal((1, HV, D, D)) * 0.02).astype(np.float32)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(262144)
    mixed = device_normal(gen, (T, CC))
    a = device_normal(gen, (T, HV))
    b = device_normal(gen, (T, HV))
    z = device_normal(gen, (T, HV * D))
    dev = lambda x, dt=None: x.to("cuda") if isinstance(x, torch.Tensor) else torch.from_numpy(x).to("cuda")  # noqa: E731
    dp = api.DevicePrefill(Hk=HK, Hv=HV, d=D, chunk=64, scale=D ** -0.5, N=1, T=T,
                           cu_seqlens=torch.tensor([0, T], dtype=torch.int32, device="cuda"), mixed_qkv=mixed,
                           conv_w=dev(conv_w), a=a, b=b, A_log=dev(A_log), dt_bias=dev(dt_bias), z=z,
                           norm_w=dev(norm_w), initial_state=dev(S0), conv_state_in=None)
    res = api.prefill(dp)
    torch.cuda.synchronize()
    host = dict(conv_w=conv_w.float().numpy(), A_log=A_log, dt_bias=dt_bias, norm_w=norm_w.float().numpy(), S0=S0)
    return dp, res, host


def window_oracle(dp, host, end, S0=None, start_hist=True):
    """The oracle on tokens [end - WINDOW, end) from a zero state (or S0), with
    the three raw inputs before the window as its conv history."""
    lo = end - WINDOW
    sl = lambda t: np64(t[lo:end])  # noqa: E731
    hist = None
    if start_hist and lo >= 3:
        hist = np64(dp.mixed_qkv[lo - 3:lo]).T[None]  # [1, Cc, 3], oldest first
    return oracle.prefill(HK, HV, D, D, [0, WINDOW], sl(dp.mixed_qkv), host["conv_w"], sl(dp.a), sl(dp.b),
                          host["A_log"], host["dt_bias"], sl(dp.z), host["norm_w"], S0, hist, scale=D ** -0.5)


def test_max_context_runs_clean(run):
    dp, res, _ = run
    assert gdn.gdn_device_error(True) == 0
    assert bool(torch.isfinite(res.out.float()).all())
    assert bool(torch.isfinite(res.final_state).all())


def test_max_context_first_tokens(run):
    """The first window from the sequence's true start (initial state, no history)."""
    dp, res, host = run
    ref = window_oracle(dp, host, WINDOW, S0=host["S0"], start_hist=False)
    assert relerr(np64(res.out[:WINDOW]), ref.out.reshape(WINDOW, HV, D)) <= PREFILL_TOL


@pytest.mark.parametrize("end", [T // 2 + 4096 + 37 * 64, T])
def test_max_context_window_ends(run, end):
    """The last tokens of a window in the middle and at the very end, against
    the oracle from a zero state at the window's start."""
    dp, res, host = run
    ref = window_oracle(dp, host, end)
    got = np64(res.out[end - CHECK:end])
    assert relerr(got, ref.out.reshape(WINDOW, HV, D)[-CHECK:]) <= PREFILL_TOL
    if end == T:
        assert relerr(np64(res.final_state), ref.final_state) <= PREFILL_TOL
        # the conv tail is the sequence's last three raw inputs
        np.testing.assert_array_equal(np64(res.conv_state_out)[0], np64(dp.mixed_qkv[T - 3:T]).T)
