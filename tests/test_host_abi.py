"""CPU-side checks of the C ABI: the library builds for sm_100a, loads
without a GPU, exports every function gdn.h declares, sizes its workspace
and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from hybrid_linear_attention_05_b200 import build, gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return gdn.lib()


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(gdn_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "gdn_prefill" in names and "gdn_decode" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(gdn.EXPORTED) <= set(names)


def test_version_and_status_strings(L):
    assert gdn.gdn_version().startswith("gdn-b200")
    for code in range(-8, 1):
        assert gdn.status_string(code) not in ("", "unknown status")
    assert gdn.status_string(-99) == "unknown status"


def test_workspace_size():
    dims = gdn.make_dims(16, 32, 128)
    T = 1000
    n = gdn.gdn_prefill_workspace_size(dims, T, gdn.GDN_BF16)
    # fp16 q, k, v, the fp32 gates, the fp16 rounding residuals of q and k, and
    # the chain queue of the fused path (a counter and the order of up to 1024
    # sequences)
    raw = T * (2 * 16 * 128 * 2 + 32 * 128 * 2 + 2 * 32 * 4 + 2 * 16 * 128 * 2) + 4 * 1025
    assert raw <= n <= raw + 8 * 256
    assert gdn.gdn_prefill_workspace_size(dims, T, gdn.GDN_F32) > n
    assert gdn.gdn_prefill_workspace_size(gdn.make_dims(3, 4, 128), T, gdn.GDN_BF16) == 0
    assert gdn.gdn_prefill_workspace_size(dims, -1, gdn.GDN_BF16) == 0


FAKE = 1 << 20  # a 16-byte aligned, never dereferenced "device" address


def prefill_kwargs(**over):
    kw = dict(mixed_qkv=FAKE, conv_w=FAKE, a=FAKE, b=FAKE, A_log=FAKE, dt_bias=FAKE, z=FAKE,
              norm_w=FAKE, cu_seqlens=FAKE, N=1, T_tot=16, chunk=32, dtype=gdn.GDN_BF16,
              out=FAKE, workspace=FAKE, workspace_bytes=1 << 30, impl=gdn.GDN_IMPL_SIMT,
              stream=0, raise_on_error=False)
    kw.update(over)
    return kw


@pytest.mark.parametrize("dims,status", [
    (gdn.make_dims(3, 4, 128), gdn.GDN_ERR_DIMS),        # Hv % Hk != 0
    (gdn.make_dims(0, 4, 128), gdn.GDN_ERR_DIMS),
    (gdn.make_dims(2, 4, 128, dv=64), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 96), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 128, conv_k=3), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 128, eps_norm=-1.0), gdn.GDN_ERR_DIMS),
])
def test_prefill_rejects_bad_dims(L, dims, status):
    assert gdn.gdn_prefill(dims, **prefill_kwargs()) == status


@pytest.mark.parametrize("over,status", [
    (dict(mixed_qkv=None), gdn.GDN_ERR_NULL),
    (dict(cu_seqlens=None), gdn.GDN_ERR_NULL),
    (dict(workspace=None), gdn.GDN_ERR_NULL),
    (dict(out=None), gdn.GDN_ERR_NULL),
    (dict(z=FAKE + 8), gdn.GDN_ERR_ALIGN),
    (dict(final_state=FAKE + 4), gdn.GDN_ERR_ALIGN),
    (dict(workspace_bytes=1000), gdn.GDN_ERR_WORKSPACE),
    (dict(chunk=48), gdn.GDN_ERR_UNSUPPORTED),
    (dict(N=-1), gdn.GDN_ERR_DIMS),
    (dict(T_tot=-5), gdn.GDN_ERR_DIMS),
    (dict(N=0, T_tot=3), gdn.GDN_ERR_DIMS),
    (dict(dtype=7), gdn.GDN_ERR_DIMS),
    (dict(chunk=64, impl=gdn.GDN_IMPL_SIMT), gdn.GDN_ERR_UNSUPPORTED),  # d=128 needs chunk <= 32 on CUDA cores
    (dict(conv_state_in=FAKE, conv_state_out=FAKE + 1024), gdn.GDN_ERR_ALIAS),
    (dict(initial_state=FAKE, final_state=FAKE + 4096), gdn.GDN_ERR_ALIAS),
    (dict(chunk=16, impl=gdn.GDN_IMPL_TC), gdn.GDN_ERR_UNSUPPORTED),
    (dict(segments=-1), gdn.GDN_ERR_UNSUPPORTED),
    (dict(segments=9), gdn.GDN_ERR_UNSUPPORTED),
    (dict(segments=2, N=17, T_tot=17), gdn.GDN_ERR_UNSUPPORTED),  # 17 x 4 chains > 64
])
def test_prefill_rejects_bad_args(L, over, status):
    dims = gdn.make_dims(2, 4, 128)
    assert gdn.gdn_prefill(dims, **prefill_kwargs(**over)) == status


def test_workspace_size_with_segments():
    """The two-kernel workspace adds the records and, for at most 64 chains,
    room for 8-segment chains: 7 maps (M, R) and 8 start states of d x d fp32
    per (sequence, value head)."""
    dims = gdn.make_dims(2, 4, 128)
    base = gdn.gdn_prefill_workspace_size(dims, 1000, gdn.GDN_BF16)
    rec = (1000 // 64 + 3 + 1) * 4 * 82432
    seg = 3 * 4 * (2 * 7 + 8) * 128 * 128 * 4
    n = gdn.gdn_prefill_workspace_size_n(dims, 3, 1000, gdn.GDN_BF16)
    assert base + rec + seg <= n <= base + rec + seg + 2 * 256
    # 17 sequences x 4 value heads = 68 chains: no segment buffers
    n17 = gdn.gdn_prefill_workspace_size_n(dims, 17, 1000, gdn.GDN_BF16)
    rec17 = (1000 // 64 + 17 + 1) * 4 * 82432
    assert base + rec17 <= n17 <= base + rec17 + 2 * 256


def test_prefill_empty_batch_is_noop(L):
    dims = gdn.make_dims(2, 4, 128)
    assert gdn.gdn_prefill(dims, **prefill_kwargs(N=0, T_tot=0)) == gdn.GDN_OK


def test_null_struct_pointers(L):
    assert L.gdn_prefill(None, None, None) == gdn.GDN_ERR_NULL
    dims = gdn.make_dims(2, 4, 128)
    assert L.gdn_prefill(ctypes.byref(dims), None, None) == gdn.GDN_ERR_NULL
    assert L.gdn_decode(ctypes.byref(dims), None, None) == gdn.GDN_ERR_NULL
    assert L.gdn_chunk_core(ctypes.byref(dims), None, None) == gdn.GDN_ERR_NULL


def decode_kwargs(**over):
    kw = dict(mixed_qkv=FAKE, conv_w=FAKE, a=FAKE, b=FAKE, A_log=FAKE, dt_bias=FAKE, z=FAKE,
              norm_w=FAKE, state=FAKE, conv_state=FAKE, out=FAKE, B=4, dtype=gdn.GDN_BF16,
              stream=0, raise_on_error=False)
    kw.update(over)
    return kw


@pytest.mark.parametrize("over,status", [
    (dict(state=None), gdn.GDN_ERR_NULL),
    (dict(conv_state=None), gdn.GDN_ERR_NULL),
    (dict(out=FAKE + 2), gdn.GDN_ERR_ALIGN),
    (dict(B=-1), gdn.GDN_ERR_DIMS),
    (dict(B=0), gdn.GDN_OK),
    (dict(state_dtype=7), gdn.GDN_ERR_DIMS),
    (dict(state_dtype=gdn.GDN_F16), gdn.GDN_ERR_DIMS),
    (dict(T=-1), gdn.GDN_ERR_DIMS),
    (dict(T=9), gdn.GDN_ERR_UNSUPPORTED),
])
def test_decode_rejects_bad_args(L, over, status):
    assert gdn.gdn_decode(gdn.make_dims(2, 4, 128), **decode_kwargs(**over)) == status


def test_core_rejects_bad_args(L):
    dims = gdn.make_dims(1, 1, 32)
    kw = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu_seqlens=FAKE, N=1, T_tot=8, chunk=16,
              dtype=gdn.GDN_F32, o=FAKE, stream=0, raise_on_error=False)
    assert gdn.gdn_chunk_core(dims, **{**kw, "o": None}) == gdn.GDN_ERR_NULL
    assert gdn.gdn_chunk_core(dims, **{**kw, "beta": FAKE + 4}) == gdn.GDN_ERR_ALIGN
    assert gdn.gdn_chunk_core(dims, **{**kw, "chunk": 8}) == gdn.GDN_ERR_UNSUPPORTED


def test_core_split_needs_its_record_workspace(L):
    """The two-kernel core takes one 82 432-byte record per (chunk slot, value
    head); with less workspace it is refused before anything is launched."""
    dims = gdn.make_dims(2, 4, 128)
    N, T = 3, 1000
    need = gdn.gdn_core_workspace_size_split(dims, N, T)
    slots = T // 64 + N + 1
    assert need >= slots * 4 * 82432 and need < slots * 4 * 82432 + 4096
    assert need >= gdn.gdn_core_workspace_size(N)
    assert gdn.gdn_core_workspace_size_split(dims, -1, T) == 0
    kw = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, cu_seqlens=FAKE, N=N, T_tot=T, chunk=64,
              dtype=gdn.GDN_F16, o=FAKE, impl=gdn.GDN_IMPL_TC_SPLIT, stream=0, raise_on_error=False)
    assert gdn.gdn_chunk_core(dims, workspace=FAKE, workspace_bytes=need - 256, **kw) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_core(dims, workspace=None, workspace_bytes=0, **kw) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_chunk_core(dims, workspace=FAKE, workspace_bytes=need, **{**kw, "chunk": 32}) == \
        gdn.GDN_ERR_UNSUPPORTED  # the tensor-core paths take chunks of 64


def map_kwargs(**over):
    kw = dict(mixed_qkv=FAKE, conv_w=FAKE, a=FAKE, b=FAKE, A_log=FAKE, dt_bias=FAKE, cu_seqlens=FAKE,
              N=1, T_tot=16, chunk=64, dtype=gdn.GDN_BF16, map_out=FAKE + (1 << 30),
              workspace=FAKE, workspace_bytes=1 << 29, stream=0, raise_on_error=False)
    kw.update(over)
    return kw


@pytest.mark.parametrize("dims,over,status", [
    (gdn.make_dims(2, 4, 64), {}, gdn.GDN_ERR_UNSUPPORTED),          # the tensor-core width only
    (gdn.make_dims(2, 4, 128), dict(chunk=32), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 128), dict(dtype=gdn.GDN_F32), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 128), dict(map_out=None), gdn.GDN_ERR_NULL),
    (gdn.make_dims(2, 4, 128), dict(map_out=FAKE + (1 << 30) + 8), gdn.GDN_ERR_ALIGN),
    (gdn.make_dims(2, 4, 128), dict(map_out=FAKE + 4096), gdn.GDN_ERR_ALIAS),  # inside the workspace
    (gdn.make_dims(2, 4, 128), dict(workspace_bytes=1 << 20), gdn.GDN_ERR_WORKSPACE),
    (gdn.make_dims(2, 4, 128), dict(workspace=None), gdn.GDN_ERR_WORKSPACE),
    (gdn.make_dims(2, 4, 128), dict(segments=8), gdn.GDN_ERR_UNSUPPORTED),   # at most 7 in map mode
    (gdn.make_dims(2, 4, 128), dict(segments=2, N=17, T_tot=17), gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 128), dict(mixed_qkv=None), gdn.GDN_ERR_NULL),
    (gdn.make_dims(2, 4, 128), dict(N=0, T_tot=0), gdn.GDN_OK),
])
def test_state_map_rejects_bad_args(L, dims, over, status):
    assert gdn.gdn_prefill_state_map(dims, **map_kwargs(**over)) == status


@pytest.mark.parametrize("dims,over,status", [
    (gdn.make_dims(2, 4, 64), {}, gdn.GDN_ERR_UNSUPPORTED),
    (gdn.make_dims(2, 4, 128), dict(S_out=None), gdn.GDN_ERR_NULL),
    (gdn.make_dims(2, 4, 128), dict(maps=None), gdn.GDN_ERR_NULL),
    (gdn.make_dims(2, 4, 128), dict(count=0, maps=None, N=0), gdn.GDN_OK),
    (gdn.make_dims(2, 4, 128), dict(S_out=FAKE + 8), gdn.GDN_ERR_ALIGN),
    (gdn.make_dims(2, 4, 128), dict(S_out=FAKE + 4096), gdn.GDN_ERR_ALIAS),   # overlaps the maps
    (gdn.make_dims(2, 4, 128), dict(S_first=FAKE + (1 << 28) + 4096), gdn.GDN_ERR_ALIAS),
    (gdn.make_dims(2, 4, 128), dict(count=-1), gdn.GDN_ERR_DIMS),
])
def test_state_fold_rejects_bad_args(L, dims, over, status):
    kw = dict(N=1, count=3, maps=FAKE, S_out=FAKE + (1 << 28), S_first=None, stream=0, raise_on_error=False)
    kw.update(over)
    assert gdn.gdn_state_fold(dims, **kw) == status


@pytest.mark.parametrize("over", [dict(reuse_workspace=1, impl=gdn.GDN_IMPL_SIMT),
                                  dict(reuse_workspace=1, impl=gdn.GDN_IMPL_TC, chunk=64),
                                  dict(reuse_workspace=2, impl=gdn.GDN_IMPL_TC_SPLIT, chunk=64)])
def test_reuse_workspace_only_on_the_two_kernel_path(L, over):
    dims = gdn.make_dims(2, 4, 128)
    assert gdn.gdn_prefill(dims, **prefill_kwargs(**over)) == gdn.GDN_ERR_UNSUPPORTED


def test_reuse_workspace_rejected_without_workspace(L):
    dims = gdn.make_dims(2, 4, 128)
    assert gdn.gdn_prefill_noalloc(dims, mixed_qkv=FAKE, conv_w=FAKE, a=FAKE, b=FAKE, A_log=FAKE,
                                   dt_bias=FAKE, z=FAKE, norm_w=FAKE, cu_seqlens=FAKE, N=1, T_tot=16,
                                   chunk=64, dtype=gdn.GDN_BF16, out=FAKE, reuse_workspace=1, stream=0,
                                   raise_on_error=False) == gdn.GDN_ERR_UNSUPPORTED


def test_state_map_gate_inputs_both_or_neither(L):
    dims = gdn.make_dims(2, 4, 128)
    assert gdn.gdn_prefill_state_map(dims, **map_kwargs(z=FAKE)) == gdn.GDN_ERR_NULL
    assert gdn.gdn_prefill_state_map(dims, **map_kwargs(norm_w=FAKE)) == gdn.GDN_ERR_NULL


def test_selftest_rejects_limits_before_launching(L):
    """The failure-path test kernel checks its limit on the host (no GPU
    needed): outside 1 .. 1e6 microseconds nothing is launched."""
    for bad in (0, -5, 1000001):
        assert gdn.gdn_selftest_bounded_wait(bad, stream=0, raise_on_error=False) == gdn.GDN_ERR_DIMS


def lin(**over):
    kw = dict(x=FAKE, w=FAKE, M=300, N=208, K=128, outs=[(FAKE, 64, 64), (FAKE, 128, 128), (FAKE, 8, 8),
                                                         (FAKE, 8, 8)], stream=0, raise_on_error=False)
    kw.update(over)
    return gdn.gdn_linear(**kw)


@pytest.mark.parametrize("over,status", [
    (dict(K=96), gdn.GDN_ERR_UNSUPPORTED),                      # K a multiple of 64
    (dict(K=0), gdn.GDN_ERR_DIMS),
    (dict(N=216), gdn.GDN_ERR_DIMS),                            # ranges do not add up to N
    (dict(outs=[(FAKE, 204, 204), (FAKE, 4, 8)]), gdn.GDN_ERR_UNSUPPORTED),  # ranges of 8 columns
    (dict(outs=[(FAKE, 200, 200), (FAKE, 8, 4)]), gdn.GDN_ERR_DIMS),         # row stride below the range
    (dict(outs=[(FAKE, 208, 212)]), gdn.GDN_ERR_DIMS),          # row stride of whole 16-byte units
    (dict(outs=[(FAKE, 8, 8)] * 5, N=40), gdn.GDN_ERR_DIMS),    # at most four ranges
    (dict(ldx=100), gdn.GDN_ERR_DIMS),                          # row stride below K
    (dict(x=None), gdn.GDN_ERR_NULL),
    (dict(outs=[(FAKE + 2, 208, 208)]), gdn.GDN_ERR_ALIGN),
])
def test_linear_rejects_bad_args(L, over, status):
    assert lin(**over) == status


def test_linear_empty_is_noop(L):
    assert lin(M=0, x=None, w=None) == gdn.GDN_OK


def test_layer_sizes_and_checks(L):
    """Activation bytes: mixed_qkv, z, b, a and the mixer output in bf16, each
    rounded up to 256 bytes; the full workspace adds the mixer's own."""
    dims = gdn.make_dims(16, 32, 128)
    T = 1000
    Cc, HVd = 2 * 16 * 128 + 32 * 128, 32 * 128
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    act = up(T * Cc * 2) + 2 * up(T * HVd * 2) + 2 * up(T * 32 * 2)
    assert gdn.gdn_layer_activation_bytes(dims, 4096, T) == act
    assert gdn.gdn_layer_workspace_size(dims, 4096, 3, T) == \
        act + gdn.gdn_prefill_workspace_size_n(dims, 3, T, gdn.GDN_BF16)
    assert gdn.gdn_layer_activation_bytes(dims, 4000, T) == 0     # d_model a multiple of 64
    kw = dict(hidden=FAKE, w_in=FAKE, w_out=FAKE, y=FAKE, d_model=4096, conv_w=FAKE, A_log=FAKE,
              dt_bias=FAKE, norm_w=FAKE, cu_seqlens=FAKE, N=1, T_tot=T, chunk=64, workspace=FAKE,
              stream=0, raise_on_error=False)
    assert gdn.gdn_layer_prefill(dims, workspace_bytes=act - 256, **kw) == gdn.GDN_ERR_WORKSPACE
    assert gdn.gdn_layer_prefill(dims, workspace_bytes=act, **dict(kw, d_model=100)) == gdn.GDN_ERR_UNSUPPORTED
    assert gdn.gdn_layer_prefill(dims, workspace_bytes=act, **dict(kw, hidden=None)) == gdn.GDN_ERR_NULL
    assert gdn.gdn_layer_prefill(dims, workspace_bytes=0, **dict(kw, N=0, T_tot=0)) == gdn.GDN_OK
