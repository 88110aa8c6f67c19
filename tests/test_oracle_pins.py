"""Pins for the fp64 CPU oracle.

Each test checks the oracle against something other than itself: brute-force
dense matrix products on tiny inputs, closed forms, invariants of the gated
delta rule, the chunked form (a different algorithm), structural identities
(GQA sharing, sequence packing, prefill/decode composition) and values
printed on the pages or worked out by hand (``tests/golden``).
"""
import math
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def rand_core(rng, T, Hk, Hv, dk, dv, g_scale=1.0, N=1, s0=True):
    q = rng.standard_normal((T, Hk, dk))
    k = rng.standard_normal((T, Hk, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((T, Hv, dv))
    g = -g_scale * rng.uniform(0.0, 1.0, (T, Hv))
    beta = rng.uniform(0.0, 1.0, (T, Hv))
    S0 = rng.standard_normal((N, Hv, dv, dk)) * 0.3 if s0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- recurrence


def brute_force(q, k, v, g, beta, S0, Hk, Hv):
    """Literal dense form: S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T."""
    T, _, dk = k.shape
    dv = v.shape[-1]
    G = Hv // Hk
    o = np.zeros((T, Hv, dv))
    Sf = np.zeros((Hv, dv, dk))
    for h in range(Hv):
        S = S0[h].copy() if S0 is not None else np.zeros((dv, dk))
        for t in range(T):
            kt, qt, vt = k[t, h // G], q[t, h // G], v[t, h]
            M = np.eye(dk) - beta[t, h] * np.outer(kt, kt)
            S = math.exp(g[t, h]) * (S @ M) + beta[t, h] * np.outer(vt, kt)
            o[t, h] = S @ qt
        Sf[h] = S
    return o, Sf


@pytest.mark.parametrize("Hk,Hv", [(1, 1), (1, 2), (2, 4)])
@pytest.mark.parametrize("chunk", [0, 3, 8])
def test_core_matches_brute_force(oracle_mod, Hk, Hv, chunk):
    rng = np.random.default_rng(11 + Hk * 7 + Hv + chunk)
    T, dk, dv = 8, 4, 4
    q, k, v, g, beta, S0 = rand_core(rng, T, Hk, Hv, dk, dv)
    o_ref, S_ref = brute_force(q, k, v, g, beta, S0[0], Hk, Hv)
    o, S = oracle_mod.core(Hk, Hv, dk, dv, [0, T], q, k, v, g, beta, S0, chunk=chunk)
    assert rel(o, o_ref) < 1e-13
    assert rel(S[0], S_ref) < 1e-13


def test_length_one_closed_form(oracle_mod):
    rng = np.random.default_rng(3)
    dk = dv = 5
    q, k, v, g, beta, S0 = rand_core(rng, 1, 1, 1, dk, dv)
    al, bt = math.exp(g[0, 0]), beta[0, 0]
    kk, qq, vv, s0 = k[0, 0], q[0, 0], v[0, 0], S0[0, 0]
    # zero initial state: o = beta (k . q) v
    o, S = oracle_mod.core(1, 1, dk, dv, [0, 1], q, k, v, g, beta, None)
    np.testing.assert_allclose(o[0, 0], bt * np.dot(kk, qq) * vv, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S[0, 0], bt * np.outer(vv, kk), rtol=1e-13, atol=1e-15)
    # nonzero initial state: S1 = a S0 - a b (S0 k) k^T + b v k^T
    o, S = oracle_mod.core(1, 1, dk, dv, [0, 1], q, k, v, g, beta, S0)
    S1 = al * s0 - al * bt * np.outer(s0 @ kk, kk) + bt * np.outer(vv, kk)
    np.testing.assert_allclose(S[0, 0], S1, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(o[0, 0], S1 @ qq, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("chunk", [0, 4])
def test_beta_zero_only_decays(oracle_mod, chunk):
    rng = np.random.default_rng(5)
    T, dk, dv = 9, 6, 3
    q, k, v, g, beta, S0 = rand_core(rng, T, 1, 2, dk, dv, g_scale=0.5)
    beta[:] = 0.0
    o, S = oracle_mod.core(1, 2, dk, dv, [0, T], q, k, v, g, beta, S0, chunk=chunk)
    cum = np.exp(np.cumsum(g, axis=0))  # [T, Hv]
    for h in range(2):
        np.testing.assert_allclose(S[0, h], cum[-1, h] * S0[0, h], rtol=1e-12)
        for t in range(T):
            np.testing.assert_allclose(o[t, h], cum[t, h] * (S0[0, h] @ q[t, 0]), rtol=1e-11,
                                       atol=1e-14)
    # with a zero initial state nothing is ever written
    o, S = oracle_mod.core(1, 2, dk, dv, [0, T], q, k, v, g, beta, None, chunk=chunk)
    assert np.all(o == 0.0) and np.all(S == 0.0)


@pytest.mark.parametrize("chunk", [0, 2, 16])
def test_orthonormal_write_and_overwrite(oracle_mod, chunk):
    """alpha = 1, beta = 1, orthonormal keys: the state becomes an exact
    associative memory -- S k_i = v_i, and rewriting a key replaces its value."""
    rng = np.random.default_rng(7)
    dk, dv, m = 8, 5, 5
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm[:, :m].T  # m orthonormal keys
    vals = rng.standard_normal((m, dv))
    new_v0 = rng.standard_normal(dv)
    # tokens: write k_0..k_{m-1}, then overwrite k_0 with new_v0
    kseq = np.concatenate([keys, keys[:1]])
    vseq = np.concatenate([vals, new_v0[None]])
    T = m + 1
    k = kseq[:, None, :]
    v = vseq[:, None, :]
    q = kseq[:, None, :].copy()  # query token t with its own key
    g = np.zeros((T, 1))
    beta = np.ones((T, 1))
    o, S = oracle_mod.core(1, 1, dk, dv, [0, T], q, k, v, g, beta, None, chunk=chunk)
    for i in range(m):
        np.testing.assert_allclose(o[i, 0], vals[i], atol=1e-12)  # read-back right after write
    np.testing.assert_allclose(S[0, 0] @ keys[0], new_v0, atol=1e-12)
    for i in range(1, m):
        np.testing.assert_allclose(S[0, 0] @ keys[i], vals[i], atol=1e-12)


@pytest.mark.parametrize("chunk", [16, 64])
def test_chunked_equals_recurrent(oracle_mod, chunk):
    """Chunked (WY/UT) and recurrent forms agree to fp64 rounding, over
    several chunks, a ragged last chunk, packed sequences, GQA and the strong
    decay of the benchmark gates (exp(A_log) up to 16)."""
    rng = np.random.default_rng(chunk)
    Hk, Hv, dk, dv = 2, 4, 16, 8
    lens = [chunk * 2 + 5, 1, chunk - 1, 3 * chunk]
    cu = np.concatenate([[0], np.cumsum(lens)])
    T = int(cu[-1])
    q, k, v, g, beta, _ = rand_core(rng, T, Hk, Hv, dk, dv, g_scale=20.0)
    S0 = rng.standard_normal((len(lens), Hv, dv, dk)) * 0.1
    o_r, S_r = oracle_mod.core(Hk, Hv, dk, dv, cu, q, k, v, g, beta, S0, chunk=0)
    o_c, S_c = oracle_mod.core(Hk, Hv, dk, dv, cu, q, k, v, g, beta, S0, chunk=chunk)
    assert rel(o_c, o_r) < 1e-12
    assert rel(S_c, S_r) < 1e-12
    # weak decay too (long memory)
    g2 = g / 200.0
    o_r, S_r = oracle_mod.core(Hk, Hv, dk, dv, cu, q, k, v, g2, beta, S0, chunk=0)
    o_c, S_c = oracle_mod.core(Hk, Hv, dk, dv, cu, q, k, v, g2, beta, S0, chunk=chunk)
    assert rel(o_c, o_r) < 1e-12
    assert rel(S_c, S_r) < 1e-12


# ----------------------------------------------------------- the whole mixer


def mixer_inputs(rng, N_lens, Hk, Hv, d, with_hist=True, with_s0=True):
    cu = np.concatenate([[0], np.cumsum(N_lens)]).astype(np.int64)
    T = int(cu[-1])
    Cc = 2 * Hk * d + Hv * d
    N = len(N_lens)
    return dict(
        cu_seqlens=cu,
        mixed_qkv=rng.standard_normal((T, Cc)),
        conv_w=rng.standard_normal((Cc, 4)) * 0.5,
        a=rng.standard_normal((T, Hv)),
        b=rng.standard_normal((T, Hv)),
        A_log=rng.uniform(0, math.log(16), Hv),
        dt_bias=rng.standard_normal(Hv) * 0.1,
        z=rng.standard_normal((T, Hv * d)),
        norm_w=1 + 0.1 * rng.standard_normal(d),
        initial_state=rng.standard_normal((N, Hv, d, d)) * 0.05 if with_s0 else None,
        conv_state_in=rng.standard_normal((N, Cc, 3)) if with_hist else None,
    )


def call_prefill(oracle_mod, Hk, Hv, d, inp, **kw):
    return oracle_mod.prefill(Hk, Hv, d, d, **inp, **kw)


def test_golden_gates(oracle_mod):
    rows = []
    with open(os.path.join(GOLDEN, "gates.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([float(x) for x in line.split()])
    rows = np.array(rows)
    Hv = rows.shape[0]
    d = 4
    inp = dict(
        cu_seqlens=[0, 1], mixed_qkv=np.ones((1, 2 * d + Hv * d)), conv_w=np.ones((2 * d + Hv * d, 4)),
        a=rows[None, :, 1], b=rows[None, :, 3], A_log=rows[:, 0], dt_bias=rows[:, 2],
        z=np.ones((1, Hv * d)), norm_w=np.ones(d))
    r = oracle_mod.prefill(1, Hv, d, d, **inp)
    np.testing.assert_allclose(r.g[0], rows[:, 4], rtol=1e-12, atol=0)
    np.testing.assert_allclose(r.beta[0], rows[:, 5], rtol=1e-12, atol=0)


def _golden_rows(name, tag):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line.startswith(tag + " "):
                rows.append([float(x) for x in line.split()[1:]])
    return np.array(rows)


def test_golden_silu(oracle_mod):
    """SiLU at hand-evaluated points (tests/golden/silu_norm.txt): a dropped
    factor x, a sign slip in the sigmoid or a swapped argument fails a row."""
    rows = _golden_rows("silu_norm.txt", "silu")
    assert rows.shape == (6, 2)
    y = oracle_mod.silu(rows[:, 0])
    np.testing.assert_allclose(y, rows[:, 1], rtol=2e-15, atol=0)


def test_golden_gated_rmsnorm(oracle_mod):
    """The gated RMSNorm at hand-evaluated rows (tests/golden/silu_norm.txt):
    eps near, above and below mean(o^2), per-channel weights and gates, a
    mean (not a sum) over the row, and eps = 0."""
    rows = _golden_rows("silu_norm.txt", "norm")
    assert rows.shape == (5, 17)
    for r in rows:
        eps, o, z, w, expect = r[0], r[1:5], r[5:9], r[9:13], r[13:17]
        out = oracle_mod.gated_rmsnorm(o[None], z[None], w, eps=eps)[0]
        np.testing.assert_allclose(out, expect, rtol=2e-15, atol=1e-300)


def test_mixer_uses_the_pinned_silu_and_norm(oracle_mod):
    """The whole mixer applies exactly the pinned pieces: v is silu of the conv
    output, and out is the gated RMSNorm of the core output o."""
    rng = np.random.default_rng(21)
    Hk, Hv, d = 1, 2, 8
    inp = mixer_inputs(rng, [5, 3], Hk, Hv, d)
    r = oracle_mod.prefill(Hk, Hv, d, d, **inp)
    T = r.o.shape[0]
    np.testing.assert_array_equal(r.v.reshape(T, Hv * d), oracle_mod.silu(r.y_pre[:, 2 * Hk * d:]))
    out = oracle_mod.gated_rmsnorm(r.o, inp["z"].reshape(T, Hv, d), inp["norm_w"], eps=1e-6)
    np.testing.assert_array_equal(r.out, out)


def test_conv_impulse_and_history(oracle_mod):
    """Single-tap conv weights reproduce the input shifted by (3 - tap); the
    positions before the sequence start come from the conv history, oldest
    first, or are zero without one."""
    rng = np.random.default_rng(9)
    Hk, Hv, d = 1, 1, 4
    T = 6
    inp = mixer_inputs(rng, [T], Hk, Hv, d)
    x, hist = inp["mixed_qkv"], inp["conv_state_in"][0]
    full = np.concatenate([hist.T, x], axis=0)  # history rows then tokens, [3+T, Cc]
    for tap in range(4):
        w = np.zeros_like(inp["conv_w"])
        w[:, tap] = 1.0
        r = oracle_mod.prefill(Hk, Hv, d, d, **{**inp, "conv_w": w})
        # y[t] = x[t - 3 + tap]; in `full` token t sits at row t + 3
        np.testing.assert_array_equal(r.y_pre, full[tap:tap + T])
        r0 = oracle_mod.prefill(Hk, Hv, d, d, **{**inp, "conv_w": w, "conv_state_in": None})
        shifted = np.concatenate([np.zeros((3, x.shape[1])), x])[tap:tap + T]
        np.testing.assert_array_equal(r0.y_pre, shifted)


def test_conv_tail(oracle_mod):
    rng = np.random.default_rng(10)
    Hk, Hv, d = 1, 2, 4
    inp = mixer_inputs(rng, [5, 2, 1], Hk, Hv, d)
    r = oracle_mod.prefill(Hk, Hv, d, d, **inp)
    cu, x, hist = inp["cu_seqlens"], inp["mixed_qkv"], inp["conv_state_in"]
    for n in range(3):
        seq = np.concatenate([hist[n].T, x[cu[n]:cu[n + 1]]])  # oldest first
        np.testing.assert_array_equal(r.conv_state_out[n], seq[-3:].T)
    r0 = oracle_mod.prefill(Hk, Hv, d, d, **{**inp, "conv_state_in": None})
    np.testing.assert_array_equal(r0.conv_state_out[2][:, :2], 0.0)   # length-1 sequence
    np.testing.assert_array_equal(r0.conv_state_out[2][:, 2], x[cu[2]])


def test_l2_norm_and_scale(oracle_mod):
    rng = np.random.default_rng(12)
    Hk, Hv, d = 2, 2, 8
    inp = mixer_inputs(rng, [7], Hk, Hv, d)
    scale = 0.37
    r = oracle_mod.prefill(Hk, Hv, d, d, **inp, scale=scale, eps_l2=0.0)
    np.testing.assert_allclose(np.linalg.norm(r.k, axis=-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(np.linalg.norm(r.q, axis=-1), scale, rtol=1e-14)
    # direction = SiLU of the conv output
    y = r.y_pre / (1 + np.exp(-r.y_pre))
    yq = y[:, :Hk * d].reshape(-1, Hk, d)
    cos = np.sum(yq * r.q, -1) / (np.linalg.norm(yq, axis=-1) * scale)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-13)
    # v is the SiLU output itself
    np.testing.assert_allclose(r.v.reshape(-1, Hv * d), y[:, 2 * Hk * d:], rtol=1e-14)


def test_length_one_full_mixer_closed_form(oracle_mod):
    """One token, no history, zero state: o = beta (k.q) v, so the gated norm
    gives sign(k.q) v / sqrt(mean(v^2) + eps/(beta k.q)^2) * w * silu(z)."""
    rng = np.random.default_rng(13)
    Hk, Hv, d = 1, 2, 8
    inp = mixer_inputs(rng, [1], Hk, Hv, d, with_hist=False, with_s0=False)
    eps = 1e-6
    r = oracle_mod.prefill(Hk, Hv, d, d, **inp, eps_norm=eps)
    z = inp["z"].reshape(Hv, d)
    for h in range(Hv):
        c = r.beta[0, h] * np.dot(r.k[0, 0], r.q[0, 0])
        vv = r.v[0, h]
        np.testing.assert_allclose(r.o[0, h], c * vv, rtol=1e-13)
        expect = c * vv / np.sqrt(np.mean((c * vv) ** 2) + eps) * inp["norm_w"] * z[h] / (1 + np.exp(-z[h]))
        np.testing.assert_allclose(r.out[0, h], expect, rtol=1e-12)
    # z = 0 gates everything off
    r = oracle_mod.prefill(Hk, Hv, d, d, **{**inp, "z": np.zeros_like(inp["z"])})
    assert np.all(r.out == 0.0)


def test_gqa_equals_duplicated_key_heads(oracle_mod):
    """Value heads 2i and 2i+1 reading key head i == a G=1 layer whose key
    heads are the originals duplicated."""
    rng = np.random.default_rng(14)
    Hk, Hv, d = 2, 4, 4
    inp = mixer_inputs(rng, [6, 3], Hk, Hv, d)
    r = oracle_mod.prefill(Hk, Hv, d, d, **inp)

    def dup_cols(x):  # duplicate every q / k head block along the channel axis
        qb = x[..., :Hk * d].reshape(*x.shape[:-1], Hk, d)
        kb = x[..., Hk * d:2 * Hk * d].reshape(*x.shape[:-1], Hk, d)
        vb = x[..., 2 * Hk * d:]
        q2 = np.repeat(qb, 2, axis=-2).reshape(*x.shape[:-1], Hv * d)
        k2 = np.repeat(kb, 2, axis=-2).reshape(*x.shape[:-1], Hv * d)
        return np.concatenate([q2, k2, vb], axis=-1)

    inp2 = dict(inp)
    inp2["mixed_qkv"] = dup_cols(inp["mixed_qkv"])
    inp2["conv_w"] = dup_cols(inp["conv_w"].T).T
    inp2["conv_state_in"] = np.swapaxes(dup_cols(np.swapaxes(inp["conv_state_in"], 1, 2)), 1, 2)
    r2 = oracle_mod.prefill(Hv, Hv, d, d, **inp2)
    assert rel(r2.out, r.out) < 1e-14
    assert rel(r2.final_state, r.final_state) < 1e-14


def test_packed_equals_separate(oracle_mod):
    rng = np.random.default_rng(15)
    Hk, Hv, d = 1, 2, 4
    lens = [5, 1, 9]
    inp = mixer_inputs(rng, lens, Hk, Hv, d)
    r = oracle_mod.prefill(Hk, Hv, d, d, **inp)
    cu = inp["cu_seqlens"]
    for n in range(len(lens)):
        s = slice(cu[n], cu[n + 1])
        one = dict(inp)
        one.update(cu_seqlens=[0, lens[n]], mixed_qkv=inp["mixed_qkv"][s], a=inp["a"][s],
                   b=inp["b"][s], z=inp["z"][s], initial_state=inp["initial_state"][n:n + 1],
                   conv_state_in=inp["conv_state_in"][n:n + 1])
        r1 = oracle_mod.prefill(Hk, Hv, d, d, **one)
        np.testing.assert_array_equal(r1.out, r.out[s])
        np.testing.assert_array_equal(r1.final_state[0], r.final_state[n])
        np.testing.assert_array_equal(r1.conv_state_out[0], r.conv_state_out[n])


def test_prefill_then_decode_equals_longer_prefill(oracle_mod):
    rng = np.random.default_rng(16)
    Hk, Hv, d = 2, 4, 8
    B, T = 3, 6
    inp = mixer_inputs(rng, [T + 1] * B, Hk, Hv, d)
    full = oracle_mod.prefill(Hk, Hv, d, d, **inp)
    cu = inp["cu_seqlens"]
    first = np.concatenate([np.arange(cu[n], cu[n] + T) for n in range(B)])
    last = cu[1:] - 1
    pre = dict(inp)
    pre.update(cu_seqlens=np.arange(B + 1) * T, mixed_qkv=inp["mixed_qkv"][first],
               a=inp["a"][first], b=inp["b"][first], z=inp["z"][first])
    rp = oracle_mod.prefill(Hk, Hv, d, d, **pre)
    out, S, cs = oracle_mod.decode(Hk, Hv, d, d, inp["mixed_qkv"][last], inp["conv_w"],
                                   inp["a"][last], inp["b"][last], inp["A_log"], inp["dt_bias"],
                                   inp["z"][last], inp["norm_w"], rp.final_state,
                                   rp.conv_state_out)
    assert rel(out, full.out[last]) < 1e-13
    assert rel(S, full.final_state) < 1e-13
    np.testing.assert_array_equal(cs, full.conv_state_out)


# ------------------------------------------------- shapes printed on the pages


def _golden_counts():
    vals = {}
    with open(os.path.join(GOLDEN, "qwen35_param_counts.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                parts = line.split()
                vals[parts[0]] = parts[1]
    return vals


def _fmt(n):
    """Abbreviate the way the module tree prints counts (one decimal, K / M)."""
    if n >= 1e6:
        return "%.1fM" % (n / 1e6)
    if n >= 1e3:
        return "%.1fK" % (n / 1e3)
    return str(n)


def test_9b_gdn_parameter_counts():
    """The mixer shapes read for the 9B layer (16 key heads, 32 value heads,
    head width 128, conv kernel 4 without bias, a dv-wide norm weight, one
    A_log and one dt_bias per value head) reproduce every count printed in
    the module tree."""
    from hybrid_linear_attention_05_b200.workloads import WORKLOADS
    w = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]
    d_model, Hk, Hv, d = 4096, w.Hk, w.Hv, w.d
    Cc = 2 * Hk * d + Hv * d
    counts = dict(
        conv1d=Cc * 4, norm=d, out_proj=Hv * d * d_model, in_proj_qkv=Cc * d_model,
        in_proj_z=Hv * d * d_model, in_proj_b=Hv * d_model, in_proj_a=Hv * d_model)
    counts["linear_attn"] = sum(counts.values()) + 2 * Hv
    gold = _golden_counts()
    for k, n in counts.items():
        assert _fmt(n) == gold[k], (k, n, gold[k])
    assert Cc == w.Cc == 8192


def test_397b_state_size():
    """KV cache + recurrent state at 262144 tokens, bf16, is 7.59 GiB only if
    the state is Hv * dk * dv per layer (one matrix per *value* head)."""
    gold = _golden_counts()
    full_layers, gdn_layers, kv_heads, head_dim = 15, 45, 2, 256
    Hk, Hv, d, ctx = 16, 64, 128, 262144
    kv_tok = full_layers * 2 * kv_heads * head_dim * 2
    assert "%dKiB" % (kv_tok // 1024) == gold["kv_cache_per_token_bf16"]
    conv = gdn_layers * (2 * Hk * d + Hv * d) * 3 * 2
    per_value_head = kv_tok * ctx + gdn_layers * Hv * d * d * 2 + conv
    per_key_head = kv_tok * ctx + gdn_layers * Hk * d * d * 2 + conv
    assert "%.2fGiB" % (per_value_head / 2 ** 30) == gold["kv_cache_plus_state_256k_bf16"]
    assert "%.2fGiB" % (per_key_head / 2 ** 30) != gold["kv_cache_plus_state_256k_bf16"]


# ----------------------------------------- affine state maps (context parallel)
# The delta rule is linear in the state, so over a stretch of tokens the state
# after it is S0 @ M + R ("Qwen (text & vision-language)", Architecture notes:
# S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T).


def _map(oracle_mod, Hk, Hv, d, inp, sl=slice(None), hist=None):
    return oracle_mod.state_map(Hk, Hv, d, d, inp["mixed_qkv"][sl], inp["conv_w"], inp["a"][sl],
                                inp["b"][sl], inp["A_log"], inp["dt_bias"], conv_state_in=hist)


def test_state_map_affine_in_start_state(oracle_mod):
    """The final state from any S0 equals S0 @ M + R: the C++ recurrence of
    ``prefill`` against the map that ``state_map`` accumulates token by token
    in numpy.  Slow decay, so that S0 @ M is not negligible."""
    rng = np.random.default_rng(21)
    Hk, Hv, d = 2, 4, 8
    inp = mixer_inputs(rng, [37], Hk, Hv, d)
    inp["A_log"] = rng.uniform(-7.0, -5.0, Hv)
    M, R = _map(oracle_mod, Hk, Hv, d, inp, hist=inp["conv_state_in"])
    assert np.max(np.abs(M)) > 0.1
    for _ in range(3):
        S0 = rng.standard_normal((1, Hv, d, d))
        r = oracle_mod.prefill(Hk, Hv, d, d, **dict(inp, initial_state=S0))
        assert rel(r.final_state[0], S0[0] @ M + R) < 1e-12


def test_state_map_one_token_closed_form(oracle_mod):
    """One token: M = alpha (I - beta k k^T) and R = beta v k^T, from the
    prepared k, v, g, beta of ``prefill``."""
    rng = np.random.default_rng(23)
    Hk, Hv, d = 1, 2, 6
    inp = mixer_inputs(rng, [1], Hk, Hv, d)
    r = oracle_mod.prefill(Hk, Hv, d, d, **dict(inp, initial_state=None))
    M, R = _map(oracle_mod, Hk, Hv, d, inp, hist=inp["conv_state_in"])
    for h in range(Hv):
        k, v = r.k[0, h // (Hv // Hk)], r.v[0, h]
        al, be = math.exp(r.g[0, h]), r.beta[0, h]
        assert rel(M[h], al * (np.eye(d) - be * np.outer(k, k))) < 1e-13
        assert rel(R[h], be * np.outer(v, k)) < 1e-13


def test_state_map_empty_is_identity(oracle_mod):
    rng = np.random.default_rng(24)
    Hk, Hv, d = 1, 2, 4
    inp = mixer_inputs(rng, [5], Hk, Hv, d)
    M, R = _map(oracle_mod, Hk, Hv, d, inp, sl=slice(0, 0), hist=inp["conv_state_in"])
    np.testing.assert_array_equal(M, np.broadcast_to(np.eye(d), (Hv, d, d)))
    np.testing.assert_array_equal(R, 0.0)


def test_parts_fold_to_the_whole_sequence(oracle_mod):
    """A sequence cut into consecutive parts, some shorter than the conv
    window and one empty.  Each part's conv history is the three raw inputs
    before it, its start state the fold of the earlier parts' maps from S0;
    run from there, the parts give the whole sequence's outputs, and the
    fold of all maps its final state."""
    rng = np.random.default_rng(22)
    Hk, Hv, d = 2, 4, 8
    lens = [2, 17, 0, 1, 25]
    T = sum(lens)
    inp = mixer_inputs(rng, [T], Hk, Hv, d)
    inp["A_log"] = rng.uniform(-7.0, -5.0, Hv)
    whole = oracle_mod.prefill(Hk, Hv, d, d, **inp)
    raw = np.concatenate([inp["conv_state_in"][0].T, inp["mixed_qkv"]], axis=0)  # row j = token j - 3
    S = inp["initial_state"][0]
    outs, t0 = [], 0
    for L in lens:
        sl = slice(t0, t0 + L)
        hist = raw[t0:t0 + 3].T[None]
        part = dict(inp, cu_seqlens=[0, L], mixed_qkv=inp["mixed_qkv"][sl], a=inp["a"][sl],
                    b=inp["b"][sl], z=inp["z"][sl], conv_state_in=hist, initial_state=S[None])
        r = oracle_mod.prefill(Hk, Hv, d, d, **part)
        outs.append(r.out)
        M, R = _map(oracle_mod, Hk, Hv, d, inp, sl=sl, hist=hist)
        S_next = S @ M + R
        assert rel(S_next, r.final_state[0]) < 1e-12
        S = S_next
        t0 += L
    assert rel(np.concatenate(outs), whole.out) < 1e-12
    assert rel(S, whole.final_state[0]) < 1e-12


# ------------------------------------------------------- layer projections


def _loop_matmul_t(x, w):
    """x w^T by explicit loops (x [m, k], w [n, k])."""
    m, k = x.shape
    n = w.shape[0]
    y = np.zeros((m, n))
    for i in range(m):
        for j in range(n):
            acc = 0.0
            for t in range(k):
                acc += x[i, t] * w[j, t]
            y[i, j] = acc
    return y


def _layer_inputs(rng, lens, Hk, Hv, d, d_model):
    inp = mixer_inputs(rng, lens, Hk, Hv, d)
    Cc = 2 * Hk * d + Hv * d
    T = int(np.sum(lens))
    hidden = rng.standard_normal((T, d_model))
    Ws = dict(W_qkv=rng.standard_normal((Cc, d_model)) * 0.3, W_z=rng.standard_normal((Hv * d, d_model)) * 0.3,
              W_a=rng.standard_normal((Hv, d_model)) * 0.3, W_b=rng.standard_normal((Hv, d_model)) * 0.3,
              W_out=rng.standard_normal((d_model, Hv * d)) * 0.3)
    for k in ("mixed_qkv", "a", "b", "z"):
        inp.pop(k)
    return hidden, Ws, inp


@pytest.mark.parametrize("act", [False, True])
def test_layer_projections_brute_force(oracle_mod, act):
    """The layer's four input projections and out_proj against explicit loops
    (x W^T, weights in [out, in] layout), around the oracle's own mixer; with
    activations_bf16 the projections' outputs and the mixer output are the
    bf16 roundings of those products."""
    rng = np.random.default_rng(31)
    Hk, Hv, d, d_model = 1, 2, 4, 6
    hidden, Ws, inp = _layer_inputs(rng, [3, 2], Hk, Hv, d, d_model)
    r = oracle_mod.layer(Hk, Hv, d, d, hidden=hidden, **Ws, **inp, activations_bf16=act)
    rnd = oracle_mod.bf16 if act else (lambda v: v)
    np.testing.assert_allclose(r.mixed_qkv, rnd(_loop_matmul_t(hidden, Ws["W_qkv"])), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r.z, rnd(_loop_matmul_t(hidden, Ws["W_z"])), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r.a, rnd(_loop_matmul_t(hidden, Ws["W_a"])), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r.b, rnd(_loop_matmul_t(hidden, Ws["W_b"])), rtol=1e-13, atol=1e-14)
    out = rnd(r.mixer.out.reshape(5, Hv * d))
    np.testing.assert_allclose(r.y, _loop_matmul_t(out, Ws["W_out"]), rtol=1e-12, atol=1e-14)


def test_layer_linear_in_out_proj(oracle_mod):
    """y is linear in W_out (zero weight -> zero output, twice the weight ->
    twice the output), and the mixer inside sees exactly the projections."""
    rng = np.random.default_rng(32)
    Hk, Hv, d, d_model = 1, 2, 4, 8
    hidden, Ws, inp = _layer_inputs(rng, [4], Hk, Hv, d, d_model)
    r = oracle_mod.layer(Hk, Hv, d, d, hidden=hidden, **Ws, **inp, activations_bf16=False)
    r0 = oracle_mod.layer(Hk, Hv, d, d, hidden=hidden, **{**Ws, "W_out": 0 * Ws["W_out"]}, **inp,
                          activations_bf16=False)
    r2 = oracle_mod.layer(Hk, Hv, d, d, hidden=hidden, **{**Ws, "W_out": 2 * Ws["W_out"]}, **inp,
                          activations_bf16=False)
    assert np.all(r0.y == 0.0)
    np.testing.assert_allclose(r2.y, 2 * r.y, rtol=1e-14, atol=0)
    m = oracle_mod.prefill(Hk, Hv, d, d, inp["cu_seqlens"], r.mixed_qkv, inp["conv_w"], r.a, r.b,
                           inp["A_log"], inp["dt_bias"], r.z, inp["norm_w"], inp["initial_state"],
                           inp["conv_state_in"])
    np.testing.assert_array_equal(m.out, r.mixer.out)


def test_bf16_rounding_points(oracle_mod):
    """The oracle's bf16 rounding at hand-checked values: exact bf16 numbers
    stay, halfway cases go to the even significand, 1 + 2^-9 rounds to 1."""
    x = np.array([1.0, 1.0 + 2 ** -7, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38])
    got = oracle_mod.bf16(x)
    expect = np.array([1.0, 1.0 + 2 ** -7, 1.0, 1.0 + 2 ** -6, 1.0, -2.5, 2.9993510e38])
    np.testing.assert_allclose(got[:6], expect[:6], rtol=0, atol=0)
    assert abs(got[6] - 3.0e38) / 3.0e38 < 2 ** -8


def test_9b_layer_weight_shapes_accepted(oracle_mod):
    """The layer function takes the 9B module tree's weight shapes (in_proj_qkv
    8192x4096, in_proj_z 4096x4096, in_proj_a/b 32x4096, out_proj 4096x4096):
    shape checks only, on a one-token call with small random values."""
    rng = np.random.default_rng(33)
    Hk, Hv, d, d_model = 16, 32, 128, 4096
    Cc = 2 * Hk * d + Hv * d
    assert (Cc, Hv * d) == (8192, 4096)
    hidden = rng.standard_normal((1, d_model)) * 0.01
    Ws = dict(W_qkv=np.zeros((Cc, d_model)), W_z=np.zeros((Hv * d, d_model)), W_a=np.zeros((Hv, d_model)),
              W_b=np.zeros((Hv, d_model)), W_out=np.zeros((d_model, Hv * d)))
    r = oracle_mod.layer(Hk, Hv, d, d, [0, 1], hidden, **Ws, conv_w=np.zeros((Cc, 4)), A_log=np.zeros(Hv),
                         dt_bias=np.zeros(Hv), norm_w=np.ones(d))
    assert r.y.shape == (1, d_model) and np.all(r.y == 0.0)
