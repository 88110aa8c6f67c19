"""CPU checks of the seeded input recipe and of the bench's work counts: the
shapes and dtypes the workloads promise, the layer inputs' scales, and the
algorithmic FLOPs and bytes the bench divides by."""
import os
import sys

import numpy as np

from hybrid_linear_attention_05_b200.workloads import WORKLOADS, make_layer, make_prefill, resized

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

P9B = WORKLOADS["prefill_4x8192_Hk16_Hv32_d128"]


def is_bf16(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return bool(np.all((u & 0xFFFF) == 0))


def test_layer_inputs_shapes_scales_and_rounding():
    w = resized(P9B, Hk=4, Hv=8)
    li = make_layer(w, 512, seqlens=(300, 212))
    T, Cc, HVd = 512, w.Cc, w.Hv * w.d
    assert li.hidden.shape == (T, 512)
    assert li.w_in.shape == (Cc + HVd + 2 * w.Hv, 512)  # in_proj_qkv; in_proj_z; in_proj_b; in_proj_a
    assert li.w_out.shape == (512, HVd)
    for x in (li.hidden, li.w_in, li.w_out):
        assert is_bf16(x)
    # weights ~ N(0, 1/fan_in): projections come out near unit scale
    assert abs(np.std(li.hidden) - 1.0) < 0.02
    assert abs(np.std(li.w_in) * np.sqrt(512) - 1.0) < 0.02
    assert abs(np.std(li.w_out) * np.sqrt(HVd) - 1.0) < 0.05
    proj = li.hidden.astype(np.float64) @ li.w_in.astype(np.float64).T
    assert 0.9 < np.std(proj) < 1.1


def test_layer_inputs_are_seeded():
    w = resized(P9B, Hk=2, Hv=4)
    a = make_layer(w, 256, seqlens=(64,))
    b = make_layer(w, 256, seqlens=(64,))
    assert np.array_equal(a.hidden, b.hidden) and np.array_equal(a.w_in, b.w_in)
    # the mixer's own draws are those of make_prefill (the layer's come after them)
    m = make_prefill(w, seqlens=(64,))
    assert np.array_equal(a.mixer.conv_w, m.conv_w) and np.array_equal(a.mixer.A_log, m.A_log)


def test_layer_counts_match_the_products():
    w = resized(P9B, Hk=2, Hv=4)
    inp = make_prefill(w, seqlens=(100, 28))
    T, Cc, HVd, dm = 128, w.Cc, w.Hv * w.d, 1024
    n_in = Cc + HVd + 2 * w.Hv
    c = bench.layer_counts(inp, dm)
    assert c["in_flops"] == 2 * T * n_in * dm
    assert c["out_flops"] == 2 * T * dm * HVd
    assert c["in_bytes"] == 2 * (T * dm + n_in * dm + T * n_in)      # X, W, Y in bf16
    assert c["out_bytes"] == 2 * (T * HVd + dm * HVd + T * dm)


def test_prefill_counts_follow_the_stated_formula():
    """Core FLOPs 10 C d + 6 d^2 per value-head token; core bytes per token
    q, k (Hk heads), v, z and out (Hv heads) in bf16 plus g and beta."""
    w = P9B
    inp = make_prefill(resized(w, Hk=16, Hv=32), seqlens=(64, 64))
    c = bench.prefill_counts(inp, 64)
    T, d = 128, 128
    assert c["core_flops"] == T * 32 * (10 * 64 * d + 6 * d * d)
    per_token = 2 * 16 * d * 2 + 3 * 32 * d * 2 + 32 * 8
    states = 2 * 2 * 32 * d * d * 4  # initial (the workload has one) and final
    assert c["core_bytes"] == T * per_token + states
