// Incremental decode with cached dt: a persistent decode state per (batch, kv
// head) that each step extends by the newly cached tokens only.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 3: dt is dt_proj of
// the cached value states, one linear projection per token, followed by
// exp(A * softplus(.)); the decode query keeps the keep_window_size best
// cached keys.  A token's dt therefore depends on that token's value states
// alone and never changes once it is cached (the page's introduction calls
// the mask a zero-order hold over cached value states): recomputing dt over
// the whole cache every step, as dma_decode_step does, gives the same values
// as computing it once per token.
//
// State (the layout of a decode plan, kept across steps): dt of every cached
// key [B, Hkv, Lk]; per (b, g) the kept list (key index, dt) with its count;
// the composite key of the worst kept key (tau) and its list position; and the
// number of cached tokens already taken in.  Top-k over a growing prefix only
// ever inserts the newest key and evicts the current worst: a key evicted once
// can never return, since later keys only add competition.  So each new token
// j of sequence b is taken in by
//   - computing dt[b, g, j] (a dot product over the Hkv*d value channels),
//   - appending it while the list holds fewer than keep_window_size keys,
//   - else replacing the worst kept key when j's composite key is larger,
//     and finding the new worst (a block-wide arg-min over the list).
// The kept set after the step is exactly the top-keep_window_size of the
// len_b cached keys (ties: lower index), as a full selection would give.
#include "common.cuh"

namespace dma {
namespace {

constexpr int kUpdThreads = 256;

// Block-wide arg-min of the composite keys of list entries [0, n): returns the
// position (ties cannot occur: composite keys are distinct).
__device__ __forceinline__ int list_argmin(const int32_t* __restrict__ idx, const float* __restrict__ bias, int n,
                                           uint64_t* red_key, int* red_pos, uint64_t* out_key) {
  uint64_t best = ~0ull;
  int pos = 0;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const uint64_t ck = composite_key(__float_as_uint(bias[e]), static_cast<uint32_t>(idx[e]));
    if (ck < best) {
      best = ck;
      pos = e;
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t ok = __shfl_xor_sync(0xFFFFFFFFu, best, o);
    const int op = __shfl_xor_sync(0xFFFFFFFFu, pos, o);
    if (ok < best) {
      best = ok;
      pos = op;
    }
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) {
    red_key[warp] = best;
    red_pos[warp] = pos;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t b = ~0ull;
    int p = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w)
      if (red_key[w] < b) {
        b = red_key[w];
        p = red_pos[w];
      }
    red_key[32] = b;
    red_pos[32] = p;
  }
  __syncthreads();
  *out_key = red_key[32];
  const int r = red_pos[32];
  __syncthreads();
  return r;
}

__device__ __forceinline__ float softplus_dc(float x) { return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x))); }

// One CTA per (kv head g, batch b): takes the tokens cached since the last step.
__global__ void __launch_bounds__(kUpdThreads) decode_update_kernel(const uint16_t* __restrict__ vc,
                                                                     const float* __restrict__ W,
                                                                     const float* __restrict__ A,
                                                                     const int32_t* __restrict__ lengths, int Lk,
                                                                     int Hkv, int d, int w, DecodePlan plan,
                                                                     int32_t* __restrict__ done,
                                                                     int32_t* __restrict__ worst, uint32_t* err) {
  __shared__ uint64_t red_key[33];
  __shared__ int red_pos[33];
  __shared__ float red_x[kUpdThreads / 32];
  pdl_trigger();   // the decode attention may be scheduled
  const int g = blockIdx.x, b = blockIdx.y;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const int C = Hkv * d;
  int len = lengths ? lengths[b] : Lk;
  const int start = done[bg];
  if (len < 1 || len > Lk || len < start) {
    // a length outside [1, Lk] or one that went backwards: reported, state kept
    if (threadIdx.x == 0) raise_error(err, kDevErrBadLength);
    return;
  }
  int32_t* idx = plan.idx + bg * plan.cap;
  float* bias = plan.bias + bg * plan.cap;
  float* dtrow = plan.dt + bg * Lk;
  int count = plan.count[bg];
  int wpos = worst[bg];
  uint64_t tau = plan.tau[bg];
  const float a = A[g];
  for (int j = start; j < len; ++j) {
    // dt of key j: x = sum_c V[b, j, c] * W[c, g]
    const uint16_t* vrow = vc + (static_cast<size_t>(b) * Lk + j) * C;
    float x = 0.0f;
    for (int c = threadIdx.x; c < C; c += blockDim.x)
      x = fmaf(__uint_as_float(static_cast<uint32_t>(vrow[c]) << 16), W[static_cast<size_t>(c) * Hkv + g], x);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
    if ((threadIdx.x & 31) == 0) red_x[threadIdx.x >> 5] = x;
    __syncthreads();
    float xs = 0.0f;
    for (int k = 0; k < static_cast<int>(blockDim.x >> 5); ++k) xs += red_x[k];
    __syncthreads();
    const float dtj = expf(a * softplus_dc(xs));
    if (threadIdx.x == 0) dtrow[j] = dtj;
    const uint64_t ck = composite_key(__float_as_uint(dtj), static_cast<uint32_t>(j));
    if (count < w) {
      if (threadIdx.x == 0) {
        idx[count] = j;
        bias[count] = dtj;
      }
      ++count;
      if (count == w) {
        __syncthreads();   // the appended entry is visible to every thread
        wpos = list_argmin(idx, bias, count, red_key, red_pos, &tau);
      }
    } else if (ck > tau) {
      // j displaces the worst kept key
      if (threadIdx.x == 0) {
        idx[wpos] = j;
        bias[wpos] = dtj;
      }
      __syncthreads();
      wpos = list_argmin(idx, bias, count, red_key, red_pos, &tau);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    plan.count[bg] = count;
    plan.tau[bg] = count < w ? 0ull : tau;
    worst[bg] = wpos;
    done[bg] = len;
  }
}

// After a full selection (dt kernel + decode selector) over the cache: record
// how many tokens the state holds and the position of the worst kept key.
__global__ void __launch_bounds__(kUpdThreads) decode_state_finish_kernel(const int32_t* __restrict__ lengths,
                                                                           int Lk, int Hkv, int w, DecodePlan plan,
                                                                           int32_t* __restrict__ done,
                                                                           int32_t* __restrict__ worst) {
  __shared__ uint64_t red_key[33];
  __shared__ int red_pos[33];
  const int g = blockIdx.x, b = blockIdx.y;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  int len = lengths ? lengths[b] : Lk;
  len = len < 1 ? 1 : (len > Lk ? Lk : len);   // the selector reported a bad length already
  const int count = plan.count[bg];
  uint64_t tau = 0ull;
  int wpos = 0;
  if (count >= w) wpos = list_argmin(plan.idx + bg * plan.cap, plan.bias + bg * plan.cap, count, red_key, red_pos, &tau);
  if (threadIdx.x == 0) {
    worst[bg] = wpos;
    done[bg] = len;
    if (count >= w) plan.tau[bg] = tau;
  }
}

}  // namespace

cudaError_t launch_decode_update(const void* v_cache, const float* W, const float* A, const int32_t* lengths,
                                 const Geometry& g, const DecodePlan& plan, int32_t* done, int32_t* worst,
                                 uint32_t* err, cudaStream_t s) {
  dim3 grid(g.Hkv, g.B);
  decode_update_kernel<<<grid, kUpdThreads, 0, s>>>(static_cast<const uint16_t*>(v_cache), W, A, lengths, g.Lk,
                                                    g.Hkv, g.d, g.w, plan, done, worst, err);
  return cudaGetLastError();
}

cudaError_t launch_decode_state_finish(const int32_t* lengths, const Geometry& g, const DecodePlan& plan,
                                       int32_t* done, int32_t* worst, cudaStream_t s) {
  dim3 grid(g.Hkv, g.B);
  decode_state_finish_kernel<<<grid, kUpdThreads, 0, s>>>(lengths, g.Lk, g.Hkv, g.w, plan, done, worst);
  return cudaGetLastError();
}

}  // namespace dma
