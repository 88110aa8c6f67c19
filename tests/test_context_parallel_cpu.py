"""Context-parallel prefill, host side, on CPU.

The rank logic of ``context_parallel.prefill_context_parallel`` (conv
histories that reach back over short parts, the gather of the parts' maps,
the fold order, the final state from the last rank) runs here on gloo ranks,
with the three compute calls answered by the fp64 oracle instead of the CUDA
library.  The result must be the oracle's own prefill of the whole sequence.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from hybrid_linear_attention_05_b200 import api  # noqa: E402
from hybrid_linear_attention_05_b200 import context_parallel as cp  # noqa: E402

HK, HV, D = 2, 4, 8


def _inputs(T, seed):
    rng = np.random.default_rng(seed)
    Cc = 2 * HK * D + HV * D
    return dict(
        mixed_qkv=rng.standard_normal((T, Cc)), conv_w=rng.standard_normal((Cc, 4)) * 0.5,
        a=rng.standard_normal((T, HV)), b=rng.standard_normal((T, HV)),
        A_log=rng.uniform(-7.0, -5.0, HV), dt_bias=rng.standard_normal(HV) * 0.1,
        z=rng.standard_normal((T, HV * D)), norm_w=1 + 0.1 * rng.standard_normal(D),
        S0=rng.standard_normal((1, HV, D, D)) * 0.1, hist=rng.standard_normal((1, Cc, 3)))


def _device_prefill(inp, lo, hi):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))  # noqa: E731
    L = hi - lo
    return api.DevicePrefill(
        Hk=HK, Hv=HV, d=D, chunk=64, scale=D ** -0.5, N=1, T=L,
        cu_seqlens=torch.tensor([0, L], dtype=torch.int32), mixed_qkv=t(inp["mixed_qkv"][lo:hi]),
        conv_w=t(inp["conv_w"]), a=t(inp["a"][lo:hi]), b=t(inp["b"][lo:hi]), A_log=t(inp["A_log"]),
        dt_bias=t(inp["dt_bias"]), z=t(inp["z"][lo:hi]), norm_w=t(inp["norm_w"]), initial_state=None,
        conv_state_in=None)


class OracleCompute:
    """The three compute calls of the context-parallel path on the fp64 oracle."""

    def _args(self, part):
        n = lambda x: x.numpy()  # noqa: E731
        return dict(mixed_qkv=n(part.mixed_qkv), conv_w=n(part.conv_w), a=n(part.a), b=n(part.b),
                    A_log=n(part.A_log), dt_bias=n(part.dt_bias))

    def state_map(self, part):
        import oracle
        M, R = oracle.state_map(part.Hk, part.Hv, part.d, part.d, **self._args(part),
                                conv_state_in=part.conv_state_in.numpy(), scale=part.scale)
        return torch.from_numpy(np.stack([M, R], axis=1)[None])

    def fold(self, maps, S_first, part):
        S = (np.zeros((1, part.Hv, part.d, part.d)) if S_first is None else S_first.numpy().copy())
        for s in range(maps.shape[0]):
            m = maps[s, 0].numpy()
            S[0] = S[0] @ m[:, 0] + m[:, 1]
        return torch.from_numpy(S)

    def prefill(self, part):
        import oracle
        r = oracle.prefill(part.Hk, part.Hv, part.d, part.d, [0, part.T], **self._args(part),
                           z=part.z.numpy(), norm_w=part.norm_w.numpy(),
                           initial_state=part.initial_state.numpy(),
                           conv_state_in=part.conv_state_in.numpy(), scale=part.scale)
        return torch.from_numpy(r.out), torch.from_numpy(r.final_state)


def _whole(inp):
    import oracle
    T = inp["mixed_qkv"].shape[0]
    return oracle.prefill(HK, HV, D, D, [0, T], inp["mixed_qkv"], inp["conv_w"], inp["a"], inp["b"],
                          inp["A_log"], inp["dt_bias"], inp["z"], inp["norm_w"], initial_state=inp["S0"],
                          conv_state_in=inp["hist"])


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def test_conv_history_reaches_over_short_parts():
    """The history before part r is the last three raw rows of [h0; parts
    0..r-1], whatever the part lengths (0, 1, 2 and longer)."""
    rng = np.random.default_rng(5)
    Cc = 7
    lens = [2, 0, 1, 5, 1, 0, 3]
    x = rng.standard_normal((sum(lens), Cc))
    h0 = rng.standard_normal((Cc, 3))
    raw = np.concatenate([h0.T, x], axis=0)
    tails, t0 = [], 0
    for L in lens:
        tails.append(cp._tail(torch.from_numpy(x[t0:t0 + L])))
        t0 += L
    tails = torch.stack(tails)
    t0 = 0
    for r, L in enumerate(lens):
        got = cp.conv_history(torch.from_numpy(h0), tails, lens, r).numpy()
        np.testing.assert_array_equal(got, raw[t0:t0 + 3].T)
        t0 += L


def test_parts_local_match_whole_sequence():
    """All parts in one process (the one-device form of the same logic)."""
    lens = [2, 40, 0, 1, 29]
    inp = _inputs(sum(lens), 31)
    parts, t0 = [], 0
    for L in lens:
        parts.append(_device_prefill(inp, t0, t0 + L))
        t0 += L
    res = cp.prefill_parts_local(parts, compute=OracleCompute(), initial_state=torch.from_numpy(inp["S0"]),
                                 conv_state_in=torch.from_numpy(inp["hist"]))
    whole = _whole(inp)
    assert rel(np.concatenate([r.out.numpy() for r in res]), whole.out) < 1e-12
    for r in res:
        assert rel(r.final_state.numpy(), whole.final_state) < 1e-12


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, lens, seed, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = _inputs(sum(lens), seed)
        lo = sum(lens[:rank])
        part = _device_prefill(inp, lo, lo + lens[rank])
        r = cp.prefill_context_parallel(part, compute=OracleCompute(),
                                        initial_state=torch.from_numpy(inp["S0"]),
                                        conv_state_in=torch.from_numpy(inp["hist"]))
        q.put((rank, r.out.numpy(), r.final_state.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [(33, 31), (1, 2, 45)])
def test_context_parallel_gloo_ranks(lens):
    """2 and 3 gloo ranks, one part each (the 3-rank case with parts of 1 and
    2 tokens, so rank 2's conv history spans both earlier ranks)."""
    world, port, seed = len(lens), _free_port(), 41
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, list(lens), seed, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=180) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    whole = _whole(_inputs(sum(lens), seed))
    assert rel(np.concatenate([g[1] for g in got]), whole.out) < 1e-12
    for g in got:  # every rank holds the sequence's final state
        assert rel(g[2], whole.final_state) < 1e-12


def test_split_sequence_and_tails():
    """Parts are consecutive slices with their own cu_seqlens; a part's tail
    is its last min(3, T) rows, right-aligned in zeros."""
    inp = _inputs(10, 7)
    dp = _device_prefill(inp, 0, 10)
    parts = cp.split_sequence(dp, [4, 0, 1, 5])
    assert [p.T for p in parts] == [4, 0, 1, 5]
    got = torch.cat([p.mixed_qkv for p in parts]).numpy()
    np.testing.assert_array_equal(got, inp["mixed_qkv"])
    for p in parts:
        assert p.cu_seqlens.tolist() == [0, p.T] and p.N == 1
        assert p.initial_state is None and p.conv_state_in is None
        t = cp._tail(p.mixed_qkv).numpy()
        take = min(3, p.T)
        np.testing.assert_array_equal(t[:3 - take], 0.0)
        np.testing.assert_array_equal(t[3 - take:], p.mixed_qkv.numpy()[p.T - take:])
    with pytest.raises(AssertionError):
        cp.split_sequence(dp, [4, 5])  # lengths must cover the sequence
