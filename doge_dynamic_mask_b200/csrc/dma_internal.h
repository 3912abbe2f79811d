// Internal constants, workspace plan layouts and kernel launchers of libdma.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/dma.h"

namespace dma {

// Query rows per prefill row tile and keys per attention key tile.
constexpr int kRowTile = 128;
constexpr int kKeyTile = 128;
// Keys per split of the decode attention.
constexpr int kDecodeChunk = 128;
// Largest keep_window_size the selectors accept when the top-k is active.
constexpr int kMaxKeep = 8192;
// Longest key axis (key indices live in 16..31 bits of the composite key and
// the selectors count in 32-bit words).
constexpr int kMaxLen = 1 << 20;
// Bounded waits give up after this many SM clock cycles (about one second).
constexpr long long kWaitLimitCycles = 2000000000LL;

// Device-side error codes recorded in the workspace's status word.
enum DeviceError : uint32_t {
  kDevErrNone = 0,
  kDevErrBadLength = 6,      // a lengths[b] outside [1, Lk]
  kDevErrBadPosition = 7,    // a prologue token whose cache row is outside [0, Lmax)
  kDevErrTimeoutBase = 100,  // 100 + site: a bounded wait gave up
};

// Workspace header: status word at offset 0; the prefill attention's
// work-item counter and finished-CTA counter at words kHdrItemWord and
// kHdrDoneWord (the last CTA of each launch returns both to zero); the rest of
// the first 256 bytes is reserved.
constexpr size_t kHeaderBytes = 256;
constexpr int kHdrItemWord = 16;
constexpr int kHdrDoneWord = 17;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Per-(batch, kv head, row tile) compacted key list produced by the prefill
// selector and consumed by the prefill attention kernel.
//   idx [tiles][cap]  int32   key index j
//   bias[tiles][cap]  float   dt[b, g, j]
//   span[tiles][cap]  uint32  lo | hi << 16: the key is kept on tile rows [lo, hi)
//   counts[tiles]     int2    (n_full, n_total); entries [0, n_full) are kept by
//                             every row of the tile; entries past n_total up to
//                             the next multiple of kKeyTile are padding (span 0).
//   kbase[tiles][cap / kKeyTile] int32  j0 when the key tile's listed keys are
//                             exactly j0, j0+1, ... (in list order), else -1
// tiles are ordered ((b * Hkv + g) * n_row_tiles + t).
struct PrefillPlan {
  float* dt;        // [B, Hkv, L]
  uint64_t* tau;    // [B, Hkv, L] row thresholds
  int32_t* idx;
  float* bias;
  uint32_t* span;
  int2* counts;
  int32_t* kbase;
  int cap;          // entries per tile (multiple of kKeyTile)
  int n_row_tiles;
  // Set by the caller before the attention launch.  no_topk (Lk <= w): every
  // row keeps every key it sees, so no list was built and the attention kernel
  // derives each tile's list itself: keys 0 .. q in order (q the tile's last
  // visible key, from lengths), bias dt_src[(b, g), j], key j > r0 kept from
  // tile row j - r0 on.
  const float* dt_src;
  const int32_t* lengths;
  int no_topk;
};

// Decode plan: per (batch, kv head) the kept keys in ascending index order.
struct DecodePlan {
  float* dt;        // [B, Hkv, Lk]
  uint64_t* tau;    // [B, Hkv]
  int32_t* idx;     // [B, Hkv, cap]
  float* bias;      // [B, Hkv, cap]
  int32_t* count;   // [B, Hkv]
  float* part;      // [B, Hq, n_split, d + 2]  (o[d], m, l)
  int cap;          // multiple of kDecodeChunk
  int n_split;
};

struct Geometry {
  int B, Lq, Lk, Hq, Hkv, d, w;
};

size_t prefill_plan_bytes(const Geometry& g);
size_t decode_plan_bytes(const Geometry& g);
PrefillPlan carve_prefill_plan(void* ws, const Geometry& g);
DecodePlan carve_decode_plan(void* ws, const Geometry& g);

// cuTensorMapEncodeTiled from the driver (through the runtime's entry-point
// query, so the library links no driver stub); nullptr when unavailable.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_fn();

// Launch-path host queries, cached per device: the SM count (0 on error), and
// the dynamic shared-memory limit of a kernel, set once per (kernel, device).
int sm_count();
cudaError_t ensure_dyn_smem(const void* func, int bytes);

// Launches kern(args...) with programmatic stream serialization: it may start
// while the stream's previous kernel finishes, and calls pdl_wait() before it
// reads anything that kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_after(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Entry-point helpers shared by the C ABI's translation units: record a CUDA
// error for dma_last_cuda_error() and return DMA_ERR_CUDA; the sm_100 device
// check; and the argument checks of dma_decode_step (everything it verifies
// before it enqueues work, workspace size aside).
dma_status_t cuda_fail(cudaError_t e);
dma_status_t device_ok();
dma_status_t check_decode_args(const void* q, const void* k_cache, const void* v_cache, const float* W_dt,
                               const float* A, const int32_t* lengths, int B, int Lk, int Hq, int Hkv, int d,
                               int keep_window_size, float scale, const float* dt_in, const void* out,
                               const void* workspace);

// launchers (return cudaGetLastError() after the launch); err: device status word or nullptr
cudaError_t launch_dt_scores(const void* v, const float* W, const float* A, int B, int L, int Hkv, int d,
                             float* dt, uint32_t* err, cudaStream_t s);
cudaError_t launch_select_prefill(const float* dt, const int32_t* lengths, const Geometry& g,
                                  const PrefillPlan& plan, uint32_t* err, cudaStream_t s);
cudaError_t launch_select_decode(const float* dt, const int32_t* lengths, const Geometry& g,
                                 const DecodePlan& plan, uint32_t* err, cudaStream_t s);
cudaError_t launch_prefill_bitmask(const PrefillPlan& plan, const Geometry& g, uint32_t* bitmask, cudaStream_t s);
cudaError_t launch_decode_bitmask(const DecodePlan& plan, const Geometry& g, uint32_t* bitmask, cudaStream_t s);
// lse_out (may be null): float32 [B, Hq, L], each row's log-sum-exp in log2 units
cudaError_t launch_attn_prefill(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                                const PrefillPlan& plan, void* out, float* lse_out, uint32_t* err, cudaStream_t s);
cudaError_t launch_attn_decode(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                               const DecodePlan& plan, void* out, cudaStream_t s);
// incremental decode: take in the tokens cached since the last step / finish a freshly selected state
cudaError_t launch_decode_update(const void* v_cache, const float* W, const float* A, const int32_t* lengths,
                                 const Geometry& g, const DecodePlan& plan, int32_t* done, int32_t* worst,
                                 uint32_t* err, cudaStream_t s);
cudaError_t launch_prologue(const void* q, const void* k, const void* v, const float* q_w, const float* k_w,
                            float eps, float theta, const int32_t* positions, int B, int L, int Lmax, int Hq, int Hkv,
                            int d, void* q_out, void* k_cache, void* v_cache, uint32_t* err, cudaStream_t s);
// CDMoE routing: router logits on the tensor cores (2K in {32, 64, 128, 256},
// hidden a multiple of 64), then routing and experts (one CTA per token).
cudaError_t launch_cdmoe_logits(const void* h, const void* W_router, int T, int hidden, int K, float* logits,
                                uint32_t* err, cudaStream_t s);
cudaError_t launch_cdmoe_route_experts(const void* h, const float* logits, const void* down_embed,
                                       const void* up_embed, int T, int hidden, int K, int k, void* out,
                                       int32_t* experts_out, float* scores_out, cudaStream_t s);
// backward: attention with the selection held fixed (float32 dK / dV / d_dt
// accumulators, zeroed by the caller), then the dt chain (dk / dv to bf16, dW, dA)
// lse_in (may be null): the forward's row log-sum-exp [B, Hq, L] (log2 units);
// when given, the backward skips recomputing the row statistics
cudaError_t launch_attn_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                                 const float* lse_in, const Geometry& g, float scale, const PrefillPlan& plan,
                                 void* dq, float* dk32, float* dv32, float* ddt32, uint32_t* err, cudaStream_t s);
cudaError_t launch_dt_backward(const void* v, const float* W, const float* A, const float* ddt32, const float* dk32,
                               const float* dv32, int B, int L, int Hkv, int d, float* dx, float* dW, float* dA,
                               void* dk, void* dv, cudaStream_t s);
cudaError_t launch_decode_state_finish(const int32_t* lengths, const Geometry& g, const DecodePlan& plan,
                                       int32_t* done, int32_t* worst, cudaStream_t s);

}  // namespace dma
