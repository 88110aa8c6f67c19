// C ABI of the library: host-side validation, workspace carving and kernel
// dispatch.  See include/gdn.h for the contract of every entry point.
#include <stdint.h>
#include <string.h>

#include "gdn_internal.h"

using namespace gdn;

namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
size_t esize(gdn_dtype dt) { return dt == GDN_BF16 ? 2 : 4; }
bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

gdn_status check_dims(const gdn_dims* d) {
  if (!d) return GDN_ERR_NULL;
  if (d->Hk < 1 || d->Hv < 1 || d->Hv % d->Hk != 0 || d->dk < 1 || d->dv < 1 || d->conv_k < 1)
    return GDN_ERR_DIMS;
  if (!(d->eps_l2 >= 0.f) || !(d->eps_norm >= 0.f) || !(d->scale == d->scale)) return GDN_ERR_DIMS;
  if (d->dk != d->dv || d->conv_k != 4) return GDN_ERR_UNSUPPORTED;
  if (d->dk != 32 && d->dk != 64 && d->dk != 128) return GDN_ERR_UNSUPPORTED;
  // keep every packed row index below 2^31 elements
  if ((int64_t)(2 * d->Hk + d->Hv) * d->dk > (1 << 24)) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

bool dtype_ok(gdn_dtype dt) { return dt == GDN_F32 || dt == GDN_BF16; }
bool core_dtype_ok(gdn_dtype dt) { return dt == GDN_F32 || dt == GDN_BF16 || dt == GDN_F16; }
// Type of the normalised q, k and v between the kernels of gdn_prefill.
gdn_dtype mid_dtype(gdn_dtype in) { return in == GDN_BF16 ? GDN_F16 : GDN_F32; }

struct Workspace {
  void* q; void* k; void* v; float* g; float* beta;
  void* q_lo; void* k_lo;  // fp16 intermediates: rounding residuals of q and k (else null)
  int* sched;              // chain queue of the fused tensor-core path
  uint8_t* rec;  // operand records of the two-kernel tensor-core path (or null)
  float* seg_mr;     // segment maps and start states of its segmented chain (or null)
  float* seg_start;
  size_t bytes;
};

// Workspace layout; with N >= 0 it also holds the two-kernel path's records.
Workspace carve(const gdn_dims* d, int T, gdn_dtype dt, void* base, int N = -1) {
  Workspace w{};
  const size_t e = esize(dt);
  const size_t nq = align_up((size_t)T * d->Hk * d->dk * e, 256);
  const size_t nv = align_up((size_t)T * d->Hv * d->dv * e, 256);
  const size_t ng = align_up((size_t)T * d->Hv * sizeof(float), 256);
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.q = p ? p + off : nullptr; off += nq;
  w.k = p ? p + off : nullptr; off += nq;
  w.v = p ? p + off : nullptr; off += nv;
  w.g = p ? reinterpret_cast<float*>(p + off) : nullptr; off += ng;
  w.beta = p ? reinterpret_cast<float*>(p + off) : nullptr; off += ng;
  w.q_lo = w.k_lo = nullptr;
  if (mid_dtype(dt) == GDN_F16) {
    w.q_lo = p ? p + off : nullptr; off += nq;
    w.k_lo = p ? p + off : nullptr; off += nq;
  }
  w.sched = p ? reinterpret_cast<int*>(p + off) : nullptr;
  off += align_up(kFusedSchedBytes, 256);
  w.rec = nullptr;
  w.seg_mr = w.seg_start = nullptr;
  if (N >= 0) {
    w.rec = p ? reinterpret_cast<uint8_t*>(p + off) : nullptr;
    off += align_up(chunk_tc_split_record_bytes(N, T, d->Hv), 256);
    const size_t sb = chunk_tc_split_seg_bytes(N, d->Hv);
    if (sb > 0 && p) {
      w.seg_mr = reinterpret_cast<float*>(p + off);
      w.seg_start = w.seg_mr + (size_t)N * d->Hv * 2 * (kSegMax - 1) * d->dk * d->dk;
    }
    off += align_up(sb, 256);
  }
  w.bytes = off;
  return w;
}

enum class Path { None, Simt, Tc, TcSplit, TcFused };

// `records` tells whether the workspace can hold the two-kernel path's records.
Path pick_path(gdn_impl impl, int d, int chunk, gdn_dtype dt_mid, bool records, int N = 0, int Hv = 0) {
  const bool tc = chunk_tc_supported(d, chunk, dt_mid);
  const bool simt = chunk_simt_supported(d, chunk);
  (void)N; (void)Hv;
  switch (impl) {
    case GDN_IMPL_TC: return tc ? Path::Tc : Path::None;
    case GDN_IMPL_TC_SPLIT: return tc ? Path::TcSplit : Path::None;
    case GDN_IMPL_TC_FUSED: return tc ? Path::TcFused : Path::None;
    case GDN_IMPL_SIMT: return simt ? Path::Simt : Path::None;
    case GDN_IMPL_AUTO:
      // two kernels when the workspace holds their records; otherwise the fused
      // kernel, which needs no more than the base workspace
      return tc ? (records ? Path::TcSplit : Path::TcFused) : (simt ? Path::Simt : Path::None);
  }
  return Path::None;
}

gdn_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA; }

}  // namespace

extern "C" {

size_t gdn_prefill_workspace_size(const gdn_dims* dims, int T_tot, gdn_dtype dtype) {
  if (check_dims(dims) != GDN_OK || T_tot < 0 || !dtype_ok(dtype)) return 0;
  return carve(dims, T_tot, dtype, nullptr).bytes;
}

size_t gdn_prefill_workspace_size_n(const gdn_dims* dims, int N, int T_tot, gdn_dtype dtype) {
  if (check_dims(dims) != GDN_OK || T_tot < 0 || N < 0 || !dtype_ok(dtype)) return 0;
  return carve(dims, T_tot, dtype, nullptr, N).bytes;
}

int gdn_prefill_resolve_impl(const gdn_dims* dims, int N, int T_tot, int chunk, gdn_dtype dtype,
                             gdn_impl impl, size_t workspace_bytes) {
  const gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (N < 1 || T_tot < 0 || !dtype_ok(dtype)) return GDN_ERR_DIMS;
  if (chunk != 16 && chunk != 32 && chunk != 64) return GDN_ERR_UNSUPPORTED;
  const size_t full = carve(dims, T_tot, dtype, nullptr, N).bytes;
  const Path path = pick_path(impl, dims->dk, chunk, mid_dtype(dtype), workspace_bytes >= full, N, dims->Hv);
  switch (path) {
    case Path::Simt: return GDN_IMPL_SIMT;
    case Path::Tc: return GDN_IMPL_TC;
    case Path::TcSplit: return workspace_bytes >= full ? (int)GDN_IMPL_TC_SPLIT : (int)GDN_ERR_WORKSPACE;
    case Path::TcFused: return GDN_IMPL_TC_FUSED;
    case Path::None: break;
  }
  return GDN_ERR_UNSUPPORTED;
}

int gdn_prefill_auto_segments(const gdn_dims* dims, int N, int T_tot) {
  if (check_dims(dims) != GDN_OK || N < 1 || T_tot < 0) return 0;
  return chunk_tc_split_auto_segments(N, T_tot, dims->Hv);
}

gdn_status gdn_prefill(const gdn_dims* dims, const gdn_prefill_args* a, void* stream) {
  gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (!a) return GDN_ERR_NULL;
  if (a->N < 0 || a->T_tot < 0) return GDN_ERR_DIMS;
  if (!dtype_ok(a->dtype)) return GDN_ERR_DIMS;
  if (a->chunk != 16 && a->chunk != 32 && a->chunk != 64) return GDN_ERR_UNSUPPORTED;
  if (a->segments < 0 || a->segments > kSegMax) return GDN_ERR_UNSUPPORTED;
  if (a->segments > 1 && (long)a->N * dims->Hv > kSegMaxChains) return GDN_ERR_UNSUPPORTED;
  if (a->N == 0) return a->T_tot == 0 ? GDN_OK : GDN_ERR_DIMS;
  const int d = dims->dk;
  const int Cc = 2 * dims->Hk * d + dims->Hv * d;
  const size_t full = carve(dims, a->T_tot, a->dtype, nullptr, a->N).bytes;
  const bool records = a->workspace && a->workspace_bytes >= full;
  const Path path = pick_path(a->impl, d, a->chunk, mid_dtype(a->dtype), records, a->N, dims->Hv);
  if (path == Path::None) return GDN_ERR_UNSUPPORTED;
  if (path == Path::TcSplit && !records) return GDN_ERR_WORKSPACE;
  if (a->reuse_workspace != 0 && (a->reuse_workspace != 1 || path != Path::TcSplit)) return GDN_ERR_UNSUPPORTED;
  if (!a->cu_seqlens || !a->conv_w || !a->A_log || !a->dt_bias || !a->norm_w) return GDN_ERR_NULL;
  if (a->T_tot > 0 && (!a->mixed_qkv || !a->a || !a->b || !a->z || !a->out || !a->workspace))
    return GDN_ERR_NULL;
  const void* ptrs[] = {a->mixed_qkv, a->conv_w, a->a, a->b, a->A_log, a->dt_bias, a->z,
                        a->norm_w, a->cu_seqlens, a->initial_state, a->final_state,
                        a->conv_state_in, a->conv_state_out, a->out, a->workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const Workspace need = carve(dims, a->T_tot, a->dtype, nullptr);
  if (a->T_tot > 0 && a->workspace_bytes < need.bytes) return GDN_ERR_WORKSPACE;
  const size_t cs_bytes = (size_t)a->N * Cc * 3 * esize(a->dtype);
  if (overlap(a->conv_state_in, cs_bytes, a->conv_state_out, cs_bytes)) return GDN_ERR_ALIAS;
  const size_t st_bytes = (size_t)a->N * dims->Hv * d * d * sizeof(float);
  if (a->initial_state != a->final_state && overlap(a->initial_state, st_bytes, a->final_state, st_bytes))
    return GDN_ERR_ALIAS;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Workspace ws = carve(dims, a->T_tot, a->dtype, a->workspace, path == Path::TcSplit ? a->N : -1);

  ConvPrepParams cp{};
  cp.x = a->mixed_qkv; cp.conv_w = a->conv_w; cp.a = a->a; cp.b = a->b;
  cp.A_log = a->A_log; cp.dt_bias = a->dt_bias; cp.cu_seqlens = a->cu_seqlens;
  cp.conv_state_in = a->conv_state_in; cp.conv_state_out = a->conv_state_out;
  cp.q = ws.q; cp.k = ws.k; cp.v = ws.v; cp.g = ws.g; cp.beta = ws.beta;
  cp.q_lo = ws.q_lo; cp.k_lo = ws.k_lo;
  cp.T = a->T_tot; cp.N = a->N; cp.Hk = dims->Hk; cp.Hv = dims->Hv; cp.Cc = Cc;
  cp.scale = dims->scale; cp.eps_l2 = dims->eps_l2;
  if (path == Path::TcFused) {  // the chain queue (reads only cu_seqlens), ahead of the conv
    ChunkParams q{};
    q.cu_seqlens = a->cu_seqlens; q.N = a->N; q.T = a->T_tot;
    s = from_cuda(launch_chunk_fused_order(q, ws.sched, st));
    if (s != GDN_OK) return s;
  }
  if (!a->reuse_workspace) {
    s = from_cuda(launch_conv_prep(cp, d, a->dtype, st));
    if (s != GDN_OK) return s;
  }

  ChunkParams ch{};
  ch.q = ws.q; ch.k = ws.k; ch.v = ws.v; ch.g = ws.g; ch.beta = ws.beta;
  ch.q_lo = ws.q_lo; ch.k_lo = ws.k_lo;
  ch.cu_seqlens = a->cu_seqlens; ch.S0 = a->initial_state; ch.S_out = a->final_state;
  ch.z = a->z; ch.norm_w = a->norm_w; ch.out = a->out; ch.o_raw = nullptr;
  ch.reuse_records = a->reuse_workspace;
  ch.T = a->T_tot; ch.N = a->N; ch.Hk = dims->Hk; ch.Hv = dims->Hv; ch.chunk = a->chunk;
  ch.eps_norm = dims->eps_norm;
  ch.rec = ws.rec;
  ch.nseg = 1;
  if (path == Path::TcSplit && ws.seg_mr) {
    ch.nseg = a->segments > 0 ? a->segments : chunk_tc_split_auto_segments(a->N, a->T_tot, dims->Hv);
    ch.seg_mr = ws.seg_mr;
    ch.seg_start = ws.seg_start;
  }
  if (a->core_event_begin && cudaEventRecord(static_cast<cudaEvent_t>(a->core_event_begin), st) != cudaSuccess)
    return GDN_ERR_CUDA;
  s = from_cuda(path == Path::TcSplit ? launch_chunk_tc_split(ch, st)
                : path == Path::TcFused ? launch_chunk_fused(ch, ws.sched, st)
                : path == Path::Tc    ? launch_chunk_tc(ch, st)
                                      : launch_chunk_simt(ch, d, a->dtype, mid_dtype(a->dtype), st));
  if (s != GDN_OK) return s;
  if (a->core_event_end && cudaEventRecord(static_cast<cudaEvent_t>(a->core_event_end), st) != cudaSuccess)
    return GDN_ERR_CUDA;
  return GDN_OK;
}

gdn_status gdn_prefill_state_map(const gdn_dims* dims, const gdn_prefill_args* a, float* map, void* stream) {
  gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (!a || !map) return GDN_ERR_NULL;
  if (a->N < 0 || a->T_tot < 0) return GDN_ERR_DIMS;
  if (!dtype_ok(a->dtype)) return GDN_ERR_DIMS;
  if (a->chunk != 16 && a->chunk != 32 && a->chunk != 64) return GDN_ERR_UNSUPPORTED;
  if (a->segments < 0 || a->segments > kSegMax - 1) return GDN_ERR_UNSUPPORTED;
  if (a->segments > 1 && (long)a->N * dims->Hv > kSegMaxChains) return GDN_ERR_UNSUPPORTED;
  if (a->N == 0) return a->T_tot == 0 ? GDN_OK : GDN_ERR_DIMS;
  const int d = dims->dk;
  if (!chunk_tc_supported(d, a->chunk, mid_dtype(a->dtype)) || dims->dv != d) return GDN_ERR_UNSUPPORTED;
  const int Cc = 2 * dims->Hk * d + dims->Hv * d;
  const size_t full = carve(dims, a->T_tot, a->dtype, nullptr, a->N).bytes;
  if (!a->workspace || a->workspace_bytes < full) return GDN_ERR_WORKSPACE;
  if (!a->cu_seqlens || !a->conv_w || !a->A_log || !a->dt_bias) return GDN_ERR_NULL;
  if (a->T_tot > 0 && (!a->mixed_qkv || !a->a || !a->b)) return GDN_ERR_NULL;
  if (a->T_tot > 0 && (a->z == nullptr) != (a->norm_w == nullptr)) return GDN_ERR_NULL;
  const void* ptrs[] = {a->mixed_qkv, a->conv_w, a->a, a->b, a->A_log, a->dt_bias, a->cu_seqlens,
                        a->conv_state_in, a->conv_state_out, a->workspace, map, a->z, a->norm_w};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const size_t cs_bytes = (size_t)a->N * Cc * 3 * esize(a->dtype);
  if (overlap(a->conv_state_in, cs_bytes, a->conv_state_out, cs_bytes)) return GDN_ERR_ALIAS;
  const size_t map_bytes = (size_t)a->N * dims->Hv * 2 * d * d * sizeof(float);
  if (overlap(map, map_bytes, a->workspace, a->workspace_bytes)) return GDN_ERR_ALIAS;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Workspace ws = carve(dims, a->T_tot, a->dtype, a->workspace, a->N);
  ConvPrepParams cp{};
  cp.x = a->mixed_qkv; cp.conv_w = a->conv_w; cp.a = a->a; cp.b = a->b;
  cp.A_log = a->A_log; cp.dt_bias = a->dt_bias; cp.cu_seqlens = a->cu_seqlens;
  cp.conv_state_in = a->conv_state_in; cp.conv_state_out = a->conv_state_out;
  cp.q = ws.q; cp.k = ws.k; cp.v = ws.v; cp.g = ws.g; cp.beta = ws.beta;
  cp.q_lo = ws.q_lo; cp.k_lo = ws.k_lo;
  cp.T = a->T_tot; cp.N = a->N; cp.Hk = dims->Hk; cp.Hv = dims->Hv; cp.Cc = Cc;
  cp.scale = dims->scale; cp.eps_l2 = dims->eps_l2;
  s = from_cuda(launch_conv_prep(cp, d, a->dtype, st));
  if (s != GDN_OK) return s;

  ChunkParams ch{};
  ch.q = ws.q; ch.k = ws.k; ch.v = ws.v; ch.g = ws.g; ch.beta = ws.beta;
  ch.q_lo = ws.q_lo; ch.k_lo = ws.k_lo;
  ch.cu_seqlens = a->cu_seqlens; ch.S0 = nullptr; ch.S_out = nullptr;
  ch.z = a->T_tot > 0 ? a->z : nullptr; ch.norm_w = a->norm_w; ch.out = nullptr; ch.o_raw = nullptr;
  ch.T = a->T_tot; ch.N = a->N; ch.Hk = dims->Hk; ch.Hv = dims->Hv; ch.chunk = a->chunk;
  ch.eps_norm = dims->eps_norm;
  ch.rec = ws.rec;
  ch.map_out = map;
  ch.nseg = ws.seg_mr ? (a->segments > 0 ? a->segments : chunk_tc_split_map_segments(a->N, dims->Hv)) : 1;
  ch.seg_mr = ch.nseg > 1 ? ws.seg_mr : map;
  ch.seg_start = nullptr;
  return from_cuda(launch_chunk_tc_split(ch, st));
}

gdn_status gdn_state_fold(const gdn_dims* dims, int N, int count, const float* maps, const float* S_first,
                          float* S_out, void* stream) {
  gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (N < 0 || count < 0) return GDN_ERR_DIMS;
  if (dims->dk != 128 || dims->dv != 128) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!S_out || (count > 0 && !maps)) return GDN_ERR_NULL;
  if (!aligned16(maps) || !aligned16(S_first) || !aligned16(S_out)) return GDN_ERR_ALIGN;
  const size_t dd = (size_t)dims->dk * dims->dk;
  const size_t st_bytes = (size_t)N * dims->Hv * dd * sizeof(float);
  const size_t map_bytes = (size_t)count * N * dims->Hv * 2 * dd * sizeof(float);
  if (overlap(maps, map_bytes, S_out, st_bytes)) return GDN_ERR_ALIAS;
  if (S_first != S_out && overlap(S_first, st_bytes, S_out, st_bytes)) return GDN_ERR_ALIAS;
  FoldParams f{};
  f.x0 = S_first;
  f.x0_n = (size_t)dims->Hv * dd;
  f.x0_h = dd;
  f.maps = maps;
  f.map_s = (size_t)N * dims->Hv * 2 * dd;
  f.map_n = (size_t)dims->Hv * 2 * dd;
  f.nmaps = count;
  f.rows = dims->dk;
  f.r_add = 0;
  f.out = S_out;
  f.N = N;
  f.Hv = dims->Hv;
  return from_cuda(launch_state_fold(f, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_decode(const gdn_dims* dims, const gdn_decode_args* a, void* stream) {
  gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (!a) return GDN_ERR_NULL;
  if (a->B < 0 || !dtype_ok(a->dtype) || !dtype_ok(a->state_dtype)) return GDN_ERR_DIMS;
  if (a->T < 0) return GDN_ERR_DIMS;
  if (a->T > 8) return GDN_ERR_UNSUPPORTED;
  if (a->B == 0) return GDN_OK;
  if (!a->mixed_qkv || !a->conv_w || !a->a || !a->b || !a->A_log || !a->dt_bias || !a->z ||
      !a->norm_w || !a->state || !a->conv_state || !a->out)
    return GDN_ERR_NULL;
  const void* ptrs[] = {a->mixed_qkv, a->conv_w, a->a, a->b, a->A_log, a->dt_bias, a->z,
                        a->norm_w, a->state, a->conv_state, a->out};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const int d = dims->dk;
  DecodeParams p{};
  p.x = a->mixed_qkv; p.conv_w = a->conv_w; p.a = a->a; p.b = a->b;
  p.A_log = a->A_log; p.dt_bias = a->dt_bias; p.z = a->z; p.norm_w = a->norm_w;
  p.state = a->state; p.conv_state = a->conv_state; p.out = a->out;
  p.B = a->B; p.Hk = dims->Hk; p.Hv = dims->Hv; p.Cc = 2 * dims->Hk * d + dims->Hv * d;
  p.scale = dims->scale; p.eps_l2 = dims->eps_l2; p.eps_norm = dims->eps_norm;
  p.state_bf16 = a->state_dtype == GDN_BF16;
  p.T = a->T > 0 ? a->T : 1;
  return from_cuda(launch_decode(p, d, a->dtype, static_cast<cudaStream_t>(stream)));
}

gdn_status gdn_chunk_core(const gdn_dims* dims, const gdn_core_args* a, void* stream) {
  gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (!a) return GDN_ERR_NULL;
  if (a->N < 0 || a->T_tot < 0 || !core_dtype_ok(a->dtype)) return GDN_ERR_DIMS;
  if (a->chunk != 16 && a->chunk != 32 && a->chunk != 64) return GDN_ERR_UNSUPPORTED;
  if (a->N == 0) return a->T_tot == 0 ? GDN_OK : GDN_ERR_DIMS;
  const int d = dims->dk;
  // AUTO takes the fused kernel only when given its chain-queue workspace; the
  // two-kernel path runs when asked for and given room for its records
  Path path = pick_path(a->impl, d, a->chunk, a->dtype, false);
  if (a->impl == GDN_IMPL_AUTO && path == Path::TcFused &&
      (!a->workspace || a->workspace_bytes < kFusedSchedBytes))
    path = Path::Tc;
  if (path == Path::None) return GDN_ERR_UNSUPPORTED;
  if (path == Path::TcFused && (!a->workspace || a->workspace_bytes < kFusedSchedBytes)) return GDN_ERR_WORKSPACE;
  if (path == Path::TcSplit &&
      (!a->workspace || a->workspace_bytes < chunk_tc_split_record_bytes(a->N, a->T_tot, dims->Hv)))
    return GDN_ERR_WORKSPACE;
  if (!aligned16(a->workspace)) return GDN_ERR_ALIGN;
  if (!a->cu_seqlens) return GDN_ERR_NULL;
  if (a->T_tot > 0 && (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->o)) return GDN_ERR_NULL;
  const void* ptrs[] = {a->q, a->k, a->v, a->g, a->beta, a->cu_seqlens, a->initial_state,
                        a->final_state, a->o};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const size_t st_bytes = (size_t)a->N * dims->Hv * d * d * sizeof(float);
  if (a->initial_state != a->final_state && overlap(a->initial_state, st_bytes, a->final_state, st_bytes))
    return GDN_ERR_ALIAS;
  ChunkParams ch{};
  ch.q = a->q; ch.k = a->k; ch.v = a->v; ch.g = a->g; ch.beta = a->beta;
  ch.cu_seqlens = a->cu_seqlens; ch.S0 = a->initial_state; ch.S_out = a->final_state;
  ch.z = nullptr; ch.norm_w = nullptr; ch.out = nullptr; ch.o_raw = a->o;
  ch.T = a->T_tot; ch.N = a->N; ch.Hk = dims->Hk; ch.Hv = dims->Hv; ch.chunk = a->chunk;
  ch.eps_norm = dims->eps_norm;
  ch.nseg = 1;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (path == Path::TcSplit) {
    ch.rec = static_cast<uint8_t*>(a->workspace);
    return from_cuda(launch_chunk_tc_split(ch, st));
  }
  if (path == Path::TcFused) {
    int* sched = static_cast<int*>(a->workspace);
    s = from_cuda(launch_chunk_fused_order(ch, sched, st));
    if (s != GDN_OK) return s;
    return from_cuda(launch_chunk_fused(ch, sched, st));
  }
  return from_cuda(path == Path::Tc ? launch_chunk_tc(ch, st)
                                    : launch_chunk_simt(ch, d, GDN_F32, a->dtype, st));
}

size_t gdn_core_workspace_size(int N) { return N < 0 ? 0 : kFusedSchedBytes; }

size_t gdn_core_workspace_size_split(const gdn_dims* dims, int N, int T_tot) {
  if (check_dims(dims) != GDN_OK || N < 0 || T_tot < 0) return 0;
  const size_t rec = chunk_tc_split_record_bytes(N, T_tot, dims->Hv);
  return rec > kFusedSchedBytes ? rec : kFusedSchedBytes;
}

gdn_status gdn_linear(const gdn_linear_args* a, void* stream) {
  if (!a) return GDN_ERR_NULL;
  if (a->M < 0 || a->N < 1 || a->K < 1 || a->n_outputs < 1 || a->n_outputs > 4) return GDN_ERR_DIMS;
  if (a->K % 64 != 0) return GDN_ERR_UNSUPPORTED;
  if (a->ldx < a->K || a->ldw < a->K || a->ldx % 8 != 0 || a->ldw % 8 != 0) return GDN_ERR_DIMS;
  long cols = 0;
  for (int i = 0; i < a->n_outputs; ++i) {
    if (a->out_cols[i] < 8 || a->out_cols[i] % 8 != 0) return GDN_ERR_UNSUPPORTED;
    if (a->out_ld[i] < a->out_cols[i] || a->out_ld[i] % 8 != 0) return GDN_ERR_DIMS;
    cols += a->out_cols[i];
  }
  if (cols != a->N) return GDN_ERR_DIMS;
  if (a->M == 0) return GDN_OK;
  if (!a->x || !a->w) return GDN_ERR_NULL;
  if (!aligned16(a->x) || !aligned16(a->w)) return GDN_ERR_ALIGN;
  for (int i = 0; i < a->n_outputs; ++i) {
    if (!a->out[i]) return GDN_ERR_NULL;
    if (!aligned16(a->out[i])) return GDN_ERR_ALIGN;
  }
  LinearParams p{};
  p.M = a->M; p.N = a->N; p.K = a->K; p.n_out = a->n_outputs;
  for (int i = 0; i < a->n_outputs; ++i) {
    p.out[i] = a->out[i];
    p.out_cols[i] = a->out_cols[i];
    p.out_ld[i] = a->out_ld[i];
  }
  return from_cuda(launch_linear_tc(p, a->x, a->ldx, a->w, a->ldw, static_cast<cudaStream_t>(stream)));
}

namespace {
// Activations of the layer in its workspace: mixed_qkv, z, b, a, and the mixer output.
struct LayerWs {
  void* mixed; void* z; void* b; void* a; void* out;
  size_t bytes;
};
LayerWs carve_layer(const gdn_dims* d, int T, void* base) {
  LayerWs w{};
  const int Cc = 2 * d->Hk * d->dk + d->Hv * d->dv;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t n) { void* r = p ? p + off : nullptr; off += align_up(n, 256); return r; };
  w.mixed = take((size_t)T * Cc * 2);
  w.z = take((size_t)T * d->Hv * d->dv * 2);
  w.b = take((size_t)T * d->Hv * 2);
  w.a = take((size_t)T * d->Hv * 2);
  w.out = take((size_t)T * d->Hv * d->dv * 2);
  w.bytes = off;
  return w;
}
bool layer_dims_ok(const gdn_dims* d, int d_model) {
  return d_model > 0 && d_model % 64 == 0 && (d->Hv * d->dv) % 64 == 0;
}
}  // namespace

size_t gdn_layer_activation_bytes(const gdn_dims* dims, int d_model, int T_tot) {
  if (check_dims(dims) != GDN_OK || T_tot < 0 || !layer_dims_ok(dims, d_model)) return 0;
  return carve_layer(dims, T_tot, nullptr).bytes;
}

size_t gdn_layer_workspace_size(const gdn_dims* dims, int d_model, int N, int T_tot) {
  if (check_dims(dims) != GDN_OK || T_tot < 0 || N < 0 || !layer_dims_ok(dims, d_model)) return 0;
  return carve_layer(dims, T_tot, nullptr).bytes + carve(dims, T_tot, GDN_BF16, nullptr, N).bytes;
}

gdn_status gdn_layer_prefill(const gdn_dims* dims, const gdn_layer_args* a, void* stream) {
  gdn_status s = check_dims(dims);
  if (s != GDN_OK) return s;
  if (!a) return GDN_ERR_NULL;
  if (a->N < 0 || a->T_tot < 0) return GDN_ERR_DIMS;
  if (!layer_dims_ok(dims, a->d_model)) return GDN_ERR_UNSUPPORTED;
  if (a->N == 0) return a->T_tot == 0 ? GDN_OK : GDN_ERR_DIMS;
  const int Cc = 2 * dims->Hk * dims->dk + dims->Hv * dims->dv;
  const int HVd = dims->Hv * dims->dv;
  const LayerWs need = carve_layer(dims, a->T_tot, nullptr);
  if (a->T_tot > 0 && (!a->hidden || !a->w_in || !a->w_out || !a->y)) return GDN_ERR_NULL;
  if (!a->workspace || a->workspace_bytes < need.bytes) return GDN_ERR_WORKSPACE;
  const void* ptrs[] = {a->hidden, a->w_in, a->w_out, a->y, a->workspace};
  for (const void* p : ptrs)
    if (!aligned16(p)) return GDN_ERR_ALIGN;
  const LayerWs w = carve_layer(dims, a->T_tot, a->workspace);
  // in_proj: [mixed_qkv | z | b | a] = hidden w_in^T
  gdn_linear_args li{};
  li.x = a->hidden; li.w = a->w_in; li.M = a->T_tot; li.N = Cc + HVd + 2 * dims->Hv; li.K = a->d_model;
  li.ldx = a->d_model; li.ldw = a->d_model; li.n_outputs = 4;
  li.out[0] = w.mixed; li.out_cols[0] = Cc; li.out_ld[0] = Cc;
  li.out[1] = w.z; li.out_cols[1] = HVd; li.out_ld[1] = HVd;
  li.out[2] = w.b; li.out_cols[2] = dims->Hv; li.out_ld[2] = dims->Hv;
  li.out[3] = w.a; li.out_cols[3] = dims->Hv; li.out_ld[3] = dims->Hv;
  if (a->T_tot > 0) {
    s = gdn_linear(&li, stream);
    if (s != GDN_OK) return s;
  }
  // the mixer on the rest of the workspace
  gdn_prefill_args pa{};
  pa.mixed_qkv = w.mixed; pa.conv_w = a->conv_w; pa.a = w.a; pa.b = w.b; pa.A_log = a->A_log;
  pa.dt_bias = a->dt_bias; pa.z = w.z; pa.norm_w = a->norm_w; pa.cu_seqlens = a->cu_seqlens;
  pa.N = a->N; pa.T_tot = a->T_tot; pa.chunk = a->chunk; pa.dtype = GDN_BF16; pa.impl = a->impl;
  pa.initial_state = a->initial_state; pa.final_state = a->final_state;
  pa.conv_state_in = a->conv_state_in; pa.conv_state_out = a->conv_state_out; pa.out = w.out;
  pa.workspace = static_cast<char*>(a->workspace) + need.bytes;
  pa.workspace_bytes = a->workspace_bytes - need.bytes;
  s = gdn_prefill(dims, &pa, stream);
  if (s != GDN_OK || a->T_tot == 0) return s;
  // out_proj: y = out w_out^T
  gdn_linear_args lo{};
  lo.x = w.out; lo.w = a->w_out; lo.M = a->T_tot; lo.N = a->d_model; lo.K = HVd;
  lo.ldx = HVd; lo.ldw = HVd; lo.n_outputs = 1;
  lo.out[0] = a->y; lo.out_cols[0] = a->d_model; lo.out_ld[0] = a->d_model;
  return gdn_linear(&lo, stream);
}

const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "ok";
    case GDN_ERR_NULL: return "a required pointer is NULL";
    case GDN_ERR_DIMS: return "inconsistent or out-of-range sizes";
    case GDN_ERR_ALIGN: return "a pointer is not 16-byte aligned";
    case GDN_ERR_UNSUPPORTED: return "shape or option not supported by the library";
    case GDN_ERR_CUDA: return "a CUDA call failed";
    case GDN_ERR_WORKSPACE: return "workspace missing or too small";
    case GDN_ERR_ALIAS: return "buffers that must not overlap overlap";
    case GDN_ERR_TIMEOUT: return "a bounded wait inside a kernel gave up";
  }
  return "unknown status";
}

const char* gdn_version(void) { return "gdn-b200 0.1"; }

}  // extern "C"
