// C ABI of libdma: argument checks, workspace carving and the launch sequence
// of each entry point.  See include/dma.h for the contract of every call.
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/dma.h"
#include "dma_internal.h"

namespace dma {

namespace {

thread_local int g_last_cuda_error = 0;
thread_local void* const* g_stage_events = nullptr;

// Records caller-provided stage event i on stream s (no-op unless set).
cudaError_t stage_mark(int i, cudaStream_t s) {
  if (!g_stage_events) return cudaSuccess;
  return cudaEventRecord(static_cast<cudaEvent_t>(g_stage_events[i]), s);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool hkv_ok(int Hkv) { return Hkv == 1 || Hkv == 2 || Hkv == 4 || Hkv == 8 || Hkv == 16; }

}  // namespace

dma_status_t cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return DMA_ERR_CUDA;
}

// sm_100 check, cached per device.
dma_status_t device_ok() {
  static std::mutex mu;
  static int cached[64];   // 0 unknown, 1 ok, 2 not ok
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return DMA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0) {
    int major = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    cached[dev] = major == 10 ? 1 : 2;
  }
  return cached[dev] == 1 ? DMA_OK : DMA_ERR_UNSUPPORTED;
}

namespace {

// Shape checks shared by every entry point (Lk is the key axis).
dma_status_t check_shape(int B, int Lk, int Hq, int Hkv, int d, int w) {
  if (B < 1 || Lk < 1 || Hq < 1 || Hkv < 1 || d < 1 || w < 1) return DMA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return DMA_ERR_INVALID_ARG;
  if (!hkv_ok(Hkv) || (d != 64 && d != 128) || Hq / Hkv > 8) return DMA_ERR_UNSUPPORTED;
  if (Lk > kMaxLen) return DMA_ERR_UNSUPPORTED;
  if (Lk > w && w > kMaxKeep) return DMA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * Lk * (Hq > Hkv ? Hq : Hkv) >= (1LL << 31)) return DMA_ERR_UNSUPPORTED;
  return DMA_OK;
}

int prefill_cap(int L, int w) {
  const int lim = L > w ? (w + kRowTile - 1 < L ? w + kRowTile - 1 : L) : L;
  return static_cast<int>(align_up(static_cast<size_t>(lim), kKeyTile));
}

int decode_cap(int Lk, int w) {
  const int lim = w < Lk ? w : Lk;
  return static_cast<int>(align_up(static_cast<size_t>(lim), kDecodeChunk));
}

}  // namespace

int sm_count() {
  static std::mutex mu;
  static int cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cached[dev] == 0 && cudaDeviceGetAttribute(&cached[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    cached[dev] = 0;
  return cached[dev];
}

cudaError_t ensure_dyn_smem(const void* func, int bytes) {
  struct Entry {
    const void* func;
    int dev, bytes;
  };
  static std::mutex mu;
  static Entry table[64];
  static int n = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int slot = -1;
  for (int i = 0; i < n; ++i)
    if (table[i].func == func && table[i].dev == dev) slot = i;
  if (slot >= 0 && table[slot].bytes >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  if (slot < 0 && n < 64) slot = n++;
  if (slot >= 0) table[slot] = Entry{func, dev, bytes};
  return cudaSuccess;
}

size_t prefill_plan_bytes(const Geometry& g) {
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  const size_t nrt = (g.Lk + kRowTile - 1) / kRowTile;
  const size_t tiles = bg * nrt;
  const size_t cap = prefill_cap(g.Lk, g.w);
  size_t off = kHeaderBytes;
  off = align_up(off + bg * g.Lk * 4, 256);         // dt
  off = align_up(off + bg * g.Lk * 8, 256);         // tau
  off = align_up(off + tiles * cap * 4, 256);       // idx
  off = align_up(off + tiles * cap * 4, 256);       // bias
  off = align_up(off + tiles * cap * 4, 256);       // span
  off = align_up(off + tiles * 8, 256);             // counts
  off = align_up(off + tiles * (cap / kKeyTile) * 4, 256);   // kbase
  return off;
}

PrefillPlan carve_prefill_plan(void* ws, const Geometry& g) {
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  const int nrt = (g.Lk + kRowTile - 1) / kRowTile;
  const size_t tiles = bg * nrt;
  const int cap = prefill_cap(g.Lk, g.w);
  char* base = static_cast<char*>(ws);
  PrefillPlan p;
  p.dt_src = nullptr;
  p.lengths = nullptr;
  p.no_topk = 0;
  size_t off = kHeaderBytes;
  p.dt = reinterpret_cast<float*>(base + off);
  off = align_up(off + bg * g.Lk * 4, 256);
  p.tau = reinterpret_cast<uint64_t*>(base + off);
  off = align_up(off + bg * g.Lk * 8, 256);
  p.idx = reinterpret_cast<int32_t*>(base + off);
  off = align_up(off + tiles * cap * 4, 256);
  p.bias = reinterpret_cast<float*>(base + off);
  off = align_up(off + tiles * cap * 4, 256);
  p.span = reinterpret_cast<uint32_t*>(base + off);
  off = align_up(off + tiles * cap * 4, 256);
  p.counts = reinterpret_cast<int2*>(base + off);
  off = align_up(off + tiles * 8, 256);
  p.kbase = reinterpret_cast<int32_t*>(base + off);
  p.cap = cap;
  p.n_row_tiles = nrt;
  return p;
}

size_t decode_plan_bytes(const Geometry& g) {
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  const size_t cap = decode_cap(g.Lk, g.w);
  const size_t nsplit = cap / kDecodeChunk;
  size_t off = kHeaderBytes;
  off = align_up(off + bg * g.Lk * 4, 256);                                  // dt
  off = align_up(off + bg * 8, 256);                                         // tau
  off = align_up(off + bg * cap * 4, 256);                                   // idx
  off = align_up(off + bg * cap * 4, 256);                                   // bias
  off = align_up(off + bg * 4, 256);                                         // count
  off = align_up(off + static_cast<size_t>(g.B) * g.Hq * nsplit * (g.d + 2) * 4, 256);   // partials
  return off;
}

DecodePlan carve_decode_plan(void* ws, const Geometry& g) {
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  const int cap = decode_cap(g.Lk, g.w);
  char* base = static_cast<char*>(ws);
  DecodePlan p;
  size_t off = kHeaderBytes;
  p.dt = reinterpret_cast<float*>(base + off);
  off = align_up(off + bg * g.Lk * 4, 256);
  p.tau = reinterpret_cast<uint64_t*>(base + off);
  off = align_up(off + bg * 8, 256);
  p.idx = reinterpret_cast<int32_t*>(base + off);
  off = align_up(off + bg * cap * 4, 256);
  p.bias = reinterpret_cast<float*>(base + off);
  off = align_up(off + bg * cap * 4, 256);
  p.count = reinterpret_cast<int32_t*>(base + off);
  off = align_up(off + bg * 4, 256);
  p.part = reinterpret_cast<float*>(base + off);
  p.cap = cap;
  p.n_split = cap / kDecodeChunk;
  return p;
}

}  // namespace dma

using namespace dma;

// ---- incremental decode with cached dt -----------------------------------------

namespace dma {
// decode state = a decode plan (kept across steps) + per (b, g) the number of
// tokens taken in and the list position of the worst kept key
struct DecodeState {
  DecodePlan plan;
  int32_t* done;
  int32_t* worst;
};
size_t state_extra_off(const Geometry& g) { return align_up(decode_plan_bytes(g), 256); }
size_t state_bytes_for(const Geometry& g) {
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  return state_extra_off(g) + 2 * align_up(bg * 4, 256);
}
DecodeState carve_state(void* st, const Geometry& g) {
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  DecodeState s;
  s.plan = carve_decode_plan(st, g);
  s.done = reinterpret_cast<int32_t*>(static_cast<char*>(st) + state_extra_off(g));
  s.worst = s.done + align_up(bg * 4, 256) / 4;
  return s;
}
}  // namespace dma

extern "C" {

size_t dma_workspace_size(int B, int Lq, int Lk, int Hq, int Hkv, int d, int keep_window_size) {
  if (check_shape(B, Lk, Hq, Hkv, d, keep_window_size) != DMA_OK) return 0;
  const Geometry g{B, Lq, Lk, Hq, Hkv, d, keep_window_size};
  size_t need = 0;
  if (Lq == Lk) need = prefill_plan_bytes(g);
  if (Lq == 1) {
    const size_t dn = decode_plan_bytes(g);
    need = dn > need ? dn : need;
  }
  return need;
}

dma_status_t dma_dt_scores(const void* v, const float* W_dt, const float* A, int B, int L, int Hkv, int d,
                           float* dt_out, dma_stream_t stream) {
  if (!v || !W_dt || !A || !dt_out) return DMA_ERR_INVALID_ARG;
  if (!aligned16(v) || !aligned16(W_dt) || !aligned16(A) || !aligned16(dt_out)) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, L, Hkv, Hkv, d, 1);
  if (st != DMA_OK) return st;
  if ((st = device_ok()) != DMA_OK) return st;
  cudaError_t e = launch_dt_scores(v, W_dt, A, B, L, Hkv, d, dt_out, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DMA_OK : cuda_fail(e);
}

dma_status_t dma_build_mask(const float* dt, const int32_t* lengths, int B, int Hkv, int Lq, int Lk,
                            int keep_window_size, uint64_t* tau_out, uint32_t* bitmask_out, void* workspace,
                            size_t ws_bytes, dma_stream_t stream) {
  if (!dt || !workspace) return DMA_ERR_INVALID_ARG;
  if (!aligned16(dt) || !aligned16(workspace) || (lengths && !aligned16(lengths)) ||
      (tau_out && !aligned16(tau_out)) || (bitmask_out && !aligned16(bitmask_out)))
    return DMA_ERR_INVALID_ARG;
  if (Lq != Lk && Lq != 1) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, Lk, Hkv, Hkv, 64, keep_window_size);
  if (st != DMA_OK) return st;
  if ((st = device_ok()) != DMA_OK) return st;
  const Geometry g{B, Lq, Lk, Hkv, Hkv, 64, keep_window_size};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(workspace);
  cudaError_t e;
  if (Lq == Lk) {
    if (ws_bytes < prefill_plan_bytes(g)) return DMA_ERR_WORKSPACE;
    const PrefillPlan plan = carve_prefill_plan(workspace, g);
    if ((e = launch_select_prefill(dt, lengths, g, plan, err, s)) != cudaSuccess) return cuda_fail(e);
    if (tau_out &&
        (e = cudaMemcpyAsync(tau_out, plan.tau, static_cast<size_t>(B) * Hkv * Lk * 8, cudaMemcpyDeviceToDevice,
                             s)) != cudaSuccess)
      return cuda_fail(e);
    if (bitmask_out) {
      const size_t words = (static_cast<size_t>(Lk) + 31) / 32;
      if ((e = cudaMemsetAsync(bitmask_out, 0, static_cast<size_t>(B) * Hkv * Lq * words * 4, s)) != cudaSuccess)
        return cuda_fail(e);
      if ((e = launch_prefill_bitmask(plan, g, bitmask_out, s)) != cudaSuccess) return cuda_fail(e);
    }
  } else {
    if (ws_bytes < decode_plan_bytes(g)) return DMA_ERR_WORKSPACE;
    const DecodePlan plan = carve_decode_plan(workspace, g);
    if ((e = launch_select_decode(dt, lengths, g, plan, err, s)) != cudaSuccess) return cuda_fail(e);
    if (tau_out && (e = cudaMemcpyAsync(tau_out, plan.tau, static_cast<size_t>(B) * Hkv * 8,
                                        cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
      return cuda_fail(e);
    if (bitmask_out) {
      const size_t words = (static_cast<size_t>(Lk) + 31) / 32;
      if ((e = cudaMemsetAsync(bitmask_out, 0, static_cast<size_t>(B) * Hkv * words * 4, s)) != cudaSuccess)
        return cuda_fail(e);
      if ((e = launch_decode_bitmask(plan, g, bitmask_out, s)) != cudaSuccess) return cuda_fail(e);
    }
  }
  return DMA_OK;
}

dma_status_t dma_forward_prefill(const void* q, const void* k, const void* v, const float* W_dt, const float* A,
                                 const int32_t* lengths, int B, int L, int Hq, int Hkv, int d, int keep_window_size,
                                 float scale, const float* dt_in, void* out, void* workspace, size_t ws_bytes,
                                 dma_stream_t stream) {
  return dma_forward_prefill_lse(q, k, v, W_dt, A, lengths, B, L, Hq, Hkv, d, keep_window_size, scale, dt_in, out,
                                 nullptr, workspace, ws_bytes, stream);
}

dma_status_t dma_forward_prefill_lse(const void* q, const void* k, const void* v, const float* W_dt, const float* A,
                                     const int32_t* lengths, int B, int L, int Hq, int Hkv, int d,
                                     int keep_window_size, float scale, const float* dt_in, void* out, float* lse_out,
                                     void* workspace, size_t ws_bytes, dma_stream_t stream) {
  if (!q || !k || !v || !out || !workspace) return DMA_ERR_INVALID_ARG;
  if (lse_out && !aligned16(lse_out)) return DMA_ERR_INVALID_ARG;
  if (!dt_in && (!W_dt || !A)) return DMA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace) ||
      (W_dt && !aligned16(W_dt)) || (A && !aligned16(A)) || (dt_in && !aligned16(dt_in)) ||
      (lengths && !aligned16(lengths)))
    return DMA_ERR_INVALID_ARG;
  // the attention kernel carries the dt bias through the tensor core as dt / scale
  if (!(scale >= 1.0e-20f && scale <= 1.0e20f)) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, L, Hq, Hkv, d, keep_window_size);
  if (st != DMA_OK) return st;
  if ((st = device_ok()) != DMA_OK) return st;
  const Geometry g{B, L, L, Hq, Hkv, d, keep_window_size};
  if (ws_bytes < prefill_plan_bytes(g)) return DMA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(workspace);
  PrefillPlan plan = carve_prefill_plan(workspace, g);
  cudaError_t e;
  const float* dt = dt_in;
  if ((e = stage_mark(0, s)) != cudaSuccess) return cuda_fail(e);
  if (!dt) {
    if ((e = launch_dt_scores(v, W_dt, A, B, L, Hkv, d, plan.dt, err, s)) != cudaSuccess) return cuda_fail(e);
    dt = plan.dt;
  }
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e);
  plan.dt_src = dt;
  plan.lengths = lengths;
  plan.no_topk = L <= keep_window_size;
  // with no top-k there is nothing to select: the attention kernel derives
  // each tile's key list (causal and padding bounds) itself
  if (!plan.no_topk && (e = launch_select_prefill(dt, lengths, g, plan, err, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_attn_prefill(q, k, v, g, scale, plan, out, lse_out, err, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e);
  return DMA_OK;
}

}  // extern "C"

namespace dma {
dma_status_t check_decode_args(const void* q, const void* k_cache, const void* v_cache, const float* W_dt,
                               const float* A, const int32_t* lengths, int B, int Lk, int Hq, int Hkv, int d,
                               int keep_window_size, float scale, const float* dt_in, const void* out,
                               const void* workspace) {
  if (!q || !k_cache || !v_cache || !out || !workspace) return DMA_ERR_INVALID_ARG;
  if (!dt_in && (!W_dt || !A)) return DMA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(workspace) ||
      (W_dt && !aligned16(W_dt)) || (A && !aligned16(A)) || (dt_in && !aligned16(dt_in)) ||
      (lengths && !aligned16(lengths)))
    return DMA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, Lk, Hq, Hkv, d, keep_window_size);
  if (st != DMA_OK) return st;
  return device_ok();
}
}  // namespace dma

extern "C" {

dma_status_t dma_decode_step(const void* q, const void* k_cache, const void* v_cache, const float* W_dt,
                             const float* A, const int32_t* lengths, int B, int Lk, int Hq, int Hkv, int d,
                             int keep_window_size, float scale, const float* dt_in, void* out, void* workspace,
                             size_t ws_bytes, dma_stream_t stream) {
  const dma_status_t st = check_decode_args(q, k_cache, v_cache, W_dt, A, lengths, B, Lk, Hq, Hkv, d,
                                            keep_window_size, scale, dt_in, out, workspace);
  if (st != DMA_OK) return st;
  const Geometry g{B, 1, Lk, Hq, Hkv, d, keep_window_size};
  if (ws_bytes < decode_plan_bytes(g)) return DMA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(workspace);
  const DecodePlan plan = carve_decode_plan(workspace, g);
  cudaError_t e;
  const float* dt = dt_in;
  if ((e = stage_mark(0, s)) != cudaSuccess) return cuda_fail(e);
  if (!dt) {
    if ((e = launch_dt_scores(v_cache, W_dt, A, B, Lk, Hkv, d, plan.dt, err, s)) != cudaSuccess) return cuda_fail(e);
    dt = plan.dt;
  }
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_select_decode(dt, lengths, g, plan, err, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_attn_decode(q, k_cache, v_cache, g, scale, plan, out, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e);
  return DMA_OK;
}


size_t dma_decode_state_size(int B, int Lk, int Hq, int Hkv, int d, int keep_window_size) {
  if (check_shape(B, Lk, Hq, Hkv, d, keep_window_size) != DMA_OK) return 0;
  return dma::state_bytes_for(Geometry{B, 1, Lk, Hq, Hkv, d, keep_window_size});
}

dma_status_t dma_decode_state_init(const void* v_cache, const float* W_dt, const float* A, const int32_t* lengths,
                                   int B, int Lk, int Hq, int Hkv, int d, int keep_window_size, void* state,
                                   size_t state_bytes, dma_stream_t stream) {
  if (!v_cache || !W_dt || !A || !state) return DMA_ERR_INVALID_ARG;
  if (!aligned16(v_cache) || !aligned16(W_dt) || !aligned16(A) || !aligned16(state) ||
      (lengths && !aligned16(lengths)))
    return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, Lk, Hq, Hkv, d, keep_window_size);
  if (st != DMA_OK) return st;
  if ((st = device_ok()) != DMA_OK) return st;
  const Geometry g{B, 1, Lk, Hq, Hkv, d, keep_window_size};
  if (state_bytes < dma::state_bytes_for(g)) return DMA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(state);
  const dma::DecodeState ds = dma::carve_state(state, g);
  cudaError_t e;
  if ((e = cudaMemsetAsync(state, 0, kHeaderBytes, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_dt_scores(v_cache, W_dt, A, B, Lk, Hkv, d, ds.plan.dt, err, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_select_decode(ds.plan.dt, lengths, g, ds.plan, err, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_decode_state_finish(lengths, g, ds.plan, ds.done, ds.worst, s)) != cudaSuccess) return cuda_fail(e);
  return DMA_OK;
}

dma_status_t dma_decode_step_cached(const void* q, const void* k_cache, const void* v_cache, const float* W_dt,
                                    const float* A, const int32_t* lengths, int B, int Lk, int Hq, int Hkv, int d,
                                    int keep_window_size, float scale, void* out, void* state, size_t state_bytes,
                                    dma_stream_t stream) {
  if (!q || !k_cache || !v_cache || !W_dt || !A || !out || !state) return DMA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(state) ||
      !aligned16(W_dt) || !aligned16(A) || (lengths && !aligned16(lengths)))
    return DMA_ERR_INVALID_ARG;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, Lk, Hq, Hkv, d, keep_window_size);
  if (st != DMA_OK) return st;
  if ((st = device_ok()) != DMA_OK) return st;
  const Geometry g{B, 1, Lk, Hq, Hkv, d, keep_window_size};
  if (state_bytes < dma::state_bytes_for(g)) return DMA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(state);
  const dma::DecodeState ds = dma::carve_state(state, g);
  cudaError_t e;
  if ((e = stage_mark(0, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_decode_update(v_cache, W_dt, A, lengths, g, ds.plan, ds.done, ds.worst, err, s)) != cudaSuccess)
    return cuda_fail(e);
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_attn_decode(q, k_cache, v_cache, g, scale, ds.plan, out, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e);
  return DMA_OK;
}

dma_status_t dma_prologue(const void* q, const void* k, const void* v, const float* q_norm_w,
                          const float* k_norm_w, float eps, float rope_theta, const int32_t* positions, int B, int L,
                          int Lmax, int Hq, int Hkv, int d, void* q_out, void* k_cache, void* v_cache,
                          void* workspace, size_t ws_bytes, dma_stream_t stream) {
  if (!q || !k || !v || !q_norm_w || !k_norm_w || !positions || !q_out || !k_cache || !v_cache || !workspace)
    return DMA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q_norm_w) || !aligned16(k_norm_w) ||
      !aligned16(positions) || !aligned16(q_out) || !aligned16(k_cache) || !aligned16(v_cache) ||
      !aligned16(workspace))
    return DMA_ERR_INVALID_ARG;
  if (ws_bytes < kHeaderBytes) return DMA_ERR_WORKSPACE;
  if (!(eps >= 0.0f && eps <= 1.0f) || !(rope_theta > 1.0f && rope_theta < 3.0e38f)) return DMA_ERR_INVALID_ARG;
  if (L < 1 || Lmax < 1 || L > Lmax) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, Lmax, Hq, Hkv, d, 1);
  if (st != DMA_OK) return st;
  if (static_cast<long long>(B) * L * Hq >= (1LL << 31)) return DMA_ERR_UNSUPPORTED;
  if ((st = device_ok()) != DMA_OK) return st;
  const cudaError_t e = launch_prologue(q, k, v, q_norm_w, k_norm_w, eps, rope_theta, positions, B, L, Lmax, Hq, Hkv,
                                        d, q_out, k_cache, v_cache, static_cast<uint32_t*>(workspace),
                                        reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DMA_OK : cuda_fail(e);
}

// backward workspace: the prefill plan, then float32 dK, dV [B, L, Hkv, d],
// d_dt [B, Hkv, L] and dx [B, L, Hkv]
static size_t bwd_extra_off(const Geometry& g) { return align_up(prefill_plan_bytes(g), 256); }
static size_t bwd_bytes(const Geometry& g) {
  const size_t kv = static_cast<size_t>(g.B) * g.Lk * g.Hkv * g.d * 4;
  const size_t per_key = static_cast<size_t>(g.B) * g.Hkv * g.Lk * 4;
  return bwd_extra_off(g) + 2 * align_up(kv, 256) + 2 * align_up(per_key, 256);
}

size_t dma_backward_workspace_size(int B, int L, int Hq, int Hkv, int d, int keep_window_size) {
  if (check_shape(B, L, Hq, Hkv, d, keep_window_size) != DMA_OK) return 0;
  return bwd_bytes(Geometry{B, L, L, Hq, Hkv, d, keep_window_size});
}

dma_status_t dma_backward_prefill(const void* q, const void* k, const void* v, const float* W_dt, const float* A,
                                  const int32_t* lengths, int B, int L, int Hq, int Hkv, int d, int keep_window_size,
                                  float scale, const float* dt_in, const void* out, const void* dout,
                                  const float* lse_in, void* dq, void* dk, void* dv, float* d_dt, float* dW_dt,
                                  float* dA, void* workspace, size_t ws_bytes, dma_stream_t stream) {
  if (!q || !k || !v || !W_dt || !A || !out || !dout || !dq || !dk || !dv || !dW_dt || !dA || !workspace)
    return DMA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(W_dt) || !aligned16(A) || !aligned16(out) ||
      !aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dW_dt) ||
      !aligned16(dA) || !aligned16(workspace) || (dt_in && !aligned16(dt_in)) || (d_dt && !aligned16(d_dt)) ||
      (lengths && !aligned16(lengths)) || (lse_in && !aligned16(lse_in)))
    return DMA_ERR_INVALID_ARG;
  if (!(scale >= 1.0e-20f && scale <= 1.0e20f)) return DMA_ERR_INVALID_ARG;
  dma_status_t st = check_shape(B, L, Hq, Hkv, d, keep_window_size);
  if (st != DMA_OK) return st;
  if ((st = device_ok()) != DMA_OK) return st;
  const Geometry g{B, L, L, Hq, Hkv, d, keep_window_size};
  if (ws_bytes < bwd_bytes(g)) return DMA_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(workspace);
  const PrefillPlan plan = carve_prefill_plan(workspace, g);
  char* base = static_cast<char*>(workspace) + bwd_extra_off(g);
  const size_t kv = align_up(static_cast<size_t>(B) * L * Hkv * d * 4, 256);
  const size_t per_key = align_up(static_cast<size_t>(B) * Hkv * L * 4, 256);
  float* dk32 = reinterpret_cast<float*>(base);
  float* dv32 = reinterpret_cast<float*>(base + kv);
  float* ddt32 = reinterpret_cast<float*>(base + 2 * kv);
  float* dx = reinterpret_cast<float*>(base + 2 * kv + per_key);
  cudaError_t e;
  const float* dt = dt_in;
  if ((e = stage_mark(0, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaMemsetAsync(base, 0, 2 * kv + per_key, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaMemsetAsync(dW_dt, 0, static_cast<size_t>(Hkv) * d * Hkv * 4, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = cudaMemsetAsync(dA, 0, static_cast<size_t>(Hkv) * 4, s)) != cudaSuccess) return cuda_fail(e);
  if (!dt) {
    if ((e = launch_dt_scores(v, W_dt, A, B, L, Hkv, d, plan.dt, err, s)) != cudaSuccess) return cuda_fail(e);
    dt = plan.dt;
  }
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e);
  // the kept-key lists of every row tile (the forward's plan), built even when
  // keep_window_size >= L (the lists then hold every visible key)
  if ((e = launch_select_prefill(dt, lengths, g, plan, err, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_attn_backward(q, k, v, out, dout, lse_in, g, scale, plan, dq, dk32, dv32, ddt32, err, s)) !=
      cudaSuccess)
    return cuda_fail(e);
  if ((e = launch_dt_backward(v, W_dt, A, ddt32, dk32, dv32, B, L, Hkv, d, dx, dW_dt, dA, dk, dv, s)) != cudaSuccess)
    return cuda_fail(e);
  if (d_dt && (e = cudaMemcpyAsync(d_dt, ddt32, static_cast<size_t>(B) * Hkv * L * 4, cudaMemcpyDeviceToDevice, s)) !=
                  cudaSuccess)
    return cuda_fail(e);
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e);
  return DMA_OK;
}

static int cdmoe_keys(int num_experts) {
  for (int K = 16; K <= 128; K *= 2)
    if (K * K == num_experts) return K;
  return 0;
}

size_t dma_cdmoe_workspace_size(int T, int num_experts) {
  const int K = cdmoe_keys(num_experts);
  if (T < 1 || K == 0) return 0;
  return kHeaderBytes + align_up(static_cast<size_t>(T) * 2 * K * 4, 256);
}

dma_status_t dma_cdmoe_forward(const void* h, const void* W_router, const void* down_embed, const void* up_embed,
                               int T, int hidden, int num_experts, int top_k, const float* logits_in, void* out,
                               int32_t* experts_out, float* scores_out, void* workspace, size_t ws_bytes,
                               dma_stream_t stream) {
  if (!h || !down_embed || !up_embed || !out || !workspace || (!logits_in && !W_router)) return DMA_ERR_INVALID_ARG;
  if ((experts_out == nullptr) != (scores_out == nullptr)) return DMA_ERR_INVALID_ARG;
  if (!aligned16(h) || !aligned16(down_embed) || !aligned16(up_embed) || !aligned16(out) || !aligned16(workspace) ||
      (W_router && !aligned16(W_router)) || (logits_in && !aligned16(logits_in)) ||
      (experts_out && !aligned16(experts_out)) || (scores_out && !aligned16(scores_out)))
    return DMA_ERR_INVALID_ARG;
  if (T < 1 || hidden < 1 || top_k < 1) return DMA_ERR_INVALID_ARG;
  const int K = cdmoe_keys(num_experts);
  if (K == 0 || hidden % 64 != 0 || hidden > 8192 || top_k > K || top_k > 64) return DMA_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * hidden >= (1LL << 31)) return DMA_ERR_UNSUPPORTED;
  if (ws_bytes < dma_cdmoe_workspace_size(T, num_experts)) return DMA_ERR_WORKSPACE;
  dma_status_t st = device_ok();
  if (st != DMA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* err = static_cast<uint32_t*>(workspace);
  const float* logits = logits_in;
  cudaError_t e;
  if ((e = stage_mark(0, s)) != cudaSuccess) return cuda_fail(e);
  if (!logits) {
    float* lg = reinterpret_cast<float*>(static_cast<char*>(workspace) + kHeaderBytes);
    if ((e = launch_cdmoe_logits(h, W_router, T, hidden, K, lg, err, s)) != cudaSuccess) return cuda_fail(e);
    logits = lg;
  }
  if ((e = stage_mark(1, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = stage_mark(2, s)) != cudaSuccess) return cuda_fail(e);
  if ((e = launch_cdmoe_route_experts(h, logits, down_embed, up_embed, T, hidden, K, top_k, out, experts_out,
                                      scores_out, s)) != cudaSuccess)
    return cuda_fail(e);
  if ((e = stage_mark(3, s)) != cudaSuccess) return cuda_fail(e);
  return DMA_OK;
}

dma_status_t dma_check(void* workspace, int clear, dma_stream_t stream) {
  if (!workspace) return DMA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e);
  uint32_t word = 0;
  if ((e = cudaMemcpy(&word, workspace, 4, cudaMemcpyDeviceToHost)) != cudaSuccess) return cuda_fail(e);
  if (clear && word != 0 && (e = cudaMemset(workspace, 0, 4)) != cudaSuccess) return cuda_fail(e);
  if (word == kDevErrNone) return DMA_OK;
  if (word == kDevErrBadLength) return DMA_ERR_BAD_LENGTH;
  if (word == kDevErrBadPosition) return DMA_ERR_BAD_POSITION;
  return DMA_ERR_TIMEOUT;
}

dma_status_t dma_set_stage_events(void* const* events, int n) {
  if (events && n < 4) return DMA_ERR_INVALID_ARG;
  g_stage_events = events;
  return DMA_OK;
}

const char* dma_status_string(dma_status_t status) {
  switch (status) {
    case DMA_OK: return "DMA_OK";
    case DMA_ERR_INVALID_ARG: return "DMA_ERR_INVALID_ARG";
    case DMA_ERR_UNSUPPORTED: return "DMA_ERR_UNSUPPORTED";
    case DMA_ERR_WORKSPACE: return "DMA_ERR_WORKSPACE";
    case DMA_ERR_CUDA: return "DMA_ERR_CUDA";
    case DMA_ERR_TIMEOUT: return "DMA_ERR_TIMEOUT";
    case DMA_ERR_BAD_LENGTH: return "DMA_ERR_BAD_LENGTH";
    case DMA_ERR_BAD_POSITION: return "DMA_ERR_BAD_POSITION";
  }
  return "DMA_ERR_UNKNOWN";
}

int dma_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
