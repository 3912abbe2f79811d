// S1: per-key score dt = exp(A * softplus(dt_proj(value_states))), float32.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", forward chain step 3
// (dt_proj projects the value states to num_key_value_heads outputs; A is one
// scalar per kv head).  No bias: attention_bias=False in section
// "DogeConfig 全参数详解".
//
// Design.  The projection is a skinny GEMV: every token row of Hkv*d bf16
// values meets the same [Hkv*d, Hkv] weight, so the kernel is bound by the one
// read of V from HBM.  Each thread owns one 16-byte chunk (8 channels) of the
// token row for the whole kernel and keeps those 8 x Hkv weights in
// registers; it streams many tokens, accumulating Hkv partial sums per token
// with packed f32x2 FMAs.  The R = Hkv*d/8 threads sharing a token combine
// their partials with a butterfly reduce-scatter inside the warp (Hkv values
// shrink to one per lane in log2(Hkv) shuffle stages) and, when a row spans
// several warps, a tiny shared-memory sum.  The epilogue applies softplus, the
// A multiply and exp in float32 and writes dt [B, Hkv, L] coalesced.
#include "common.cuh"

namespace dma {
namespace {

constexpr int kDtThreads = 256;

__device__ __forceinline__ void bf16x2_to_f32(uint32_t u, float& lo, float& hi) {
  lo = __uint_as_float(u << 16);
  hi = __uint_as_float(u & 0xFFFF0000u);
}

__device__ __forceinline__ unsigned long long pack_f32x2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack_f32x2(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// acc = a * b + acc on both float32 halves (round-to-nearest, like fmaf).
__device__ __forceinline__ void fma_f32x2(unsigned long long& acc, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}

__device__ __forceinline__ float softplus_f32(float x) {
  // log(1 + e^x) in the overflow-free form max(x, 0) + log1p(e^-|x|).
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

// HKV outputs per token; R = HKV*D/8 threads share one token row.
template <int HKV, int D, int UNROLL>
__global__ void __launch_bounds__(kDtThreads) dt_scores_kernel(const uint4* __restrict__ v,
                                                                const float* __restrict__ W,
                                                                const float* __restrict__ A, long long ntok,
                                                                int L, float* __restrict__ dt) {
  constexpr int R = HKV * D / 8;                   // chunks (threads) per token row
  constexpr int TS = kDtThreads / R;               // tokens per step (>= 1)
  constexpr int TB = TS * UNROLL;                  // tokens per block iteration
  constexpr int RW = R < 32 ? R : 32;              // lanes of one warp sharing a token
  constexpr int NPART = R > 32 ? R / 32 : 1;       // warps sharing a token
  static_assert(kDtThreads % R == 0, "row must tile the block");

  __shared__ float part[NPART][TB][HKV];

  const int tid = threadIdx.x;
  const int c = tid % R;                            // chunk of the row owned by this thread
  const int slot = tid / R;                         // token slot within a step
  const int lane = tid & 31;

  // weights of this thread's 8 channels, packed in f32x2 pairs over outputs
  constexpr int HP = HKV >= 2 ? HKV / 2 : 1;
  unsigned long long w2[8][HP];
#pragma unroll
  for (int e = 0; e < 8; ++e)
#pragma unroll
    for (int i = 0; i < HP; ++i)
      w2[e][i] = HKV >= 2 ? pack_f32x2(W[(c * 8 + e) * HKV + 2 * i], W[(c * 8 + e) * HKV + 2 * i + 1])
                          : pack_f32x2(W[c * 8 + e], 0.0f);

  const long long n_iter = (ntok + TB - 1) / TB;
  for (long long it = blockIdx.x; it < n_iter; it += gridDim.x) {
    const long long tok0 = it * TB;
    uint4 buf[UNROLL];
#pragma unroll
    for (int s = 0; s < UNROLL; ++s) {
      const long long t = tok0 + slot + s * TS;
      buf[s] = t < ntok ? v[t * R + c] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int s = 0; s < UNROLL; ++s) {
      float x[8];
      bf16x2_to_f32(buf[s].x, x[0], x[1]);
      bf16x2_to_f32(buf[s].y, x[2], x[3]);
      bf16x2_to_f32(buf[s].z, x[4], x[5]);
      bf16x2_to_f32(buf[s].w, x[6], x[7]);
      unsigned long long acc2[HP];
#pragma unroll
      for (int i = 0; i < HP; ++i) acc2[i] = 0ull;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const unsigned long long xx = pack_f32x2(x[e], x[e]);
#pragma unroll
        for (int i = 0; i < HP; ++i) fma_f32x2(acc2[i], xx, w2[e][i]);
      }
      float acc[HKV];
#pragma unroll
      for (int i = 0; i < HP; ++i) {
        float lo, hi;
        unpack_f32x2(acc2[i], lo, hi);
        acc[2 * i < HKV ? 2 * i : 0] = lo;
        if (2 * i + 1 < HKV) acc[2 * i + 1] = hi;
      }

      // butterfly reduce-scatter over the RW lanes sharing this token: each
      // split stage halves the outputs a lane holds (kLogH stages), then plain
      // xor stages sum over the remaining lanes.
      constexpr int kLogH = HKV >= 16 ? 4 : HKV >= 8 ? 3 : HKV >= 4 ? 2 : HKV >= 2 ? 1 : 0;
      static_assert((1 << kLogH) == HKV && HKV <= RW, "outputs must fit the lanes of a row");
      int gbase = 0;
#pragma unroll
      for (int st = 0; st < kLogH; ++st) {
        const int o = RW >> (st + 1);
        const int half = HKV >> (st + 1);
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < half; ++i) {
          const float send = upper ? acc[i] : acc[i + half];
          const float keep = upper ? acc[i + half] : acc[i];
          acc[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
        }
        if (upper) gbase += half;
      }
#pragma unroll
      for (int o = RW >> (kLogH + 1); o >= 1; o >>= 1) acc[0] += __shfl_xor_sync(0xFFFFFFFFu, acc[0], o);
      // one lane per output (low plain-stage lane bits clear) writes the warp's partial
      constexpr int kPlainMask = (RW >> kLogH) - 1;
      if ((lane & kPlainMask) == 0) {
        const int p = NPART > 1 ? (tid / 32) % NPART : 0;
        part[p][slot + s * TS][gbase] = acc[0];
      }
    }
    __syncthreads();
    for (int i = tid; i < TB * HKV; i += kDtThreads) {
      const int g = i / TB;
      const int tl = i % TB;
      const long long t = tok0 + tl;
      if (t < ntok) {
        float x = 0.0f;
#pragma unroll
        for (int p = 0; p < NPART; ++p) x += part[p][tl][g];
        const float y = expf(A[g] * softplus_f32(x));
        const long long b = t / L;
        const long long l = t - b * L;
        dt[(b * HKV + g) * L + l] = y;
      }
    }
    __syncthreads();
  }
}

template <int HKV, int D>
cudaError_t launch_t(const void* v, const float* W, const float* A, int B, int L, float* dt, cudaStream_t s) {
  constexpr int R = HKV * D / 8;
  constexpr int UNROLL = 8;
  constexpr int TB = (kDtThreads / R) * UNROLL;
  const long long ntok = static_cast<long long>(B) * L;
  const long long n_iter = (ntok + TB - 1) / TB;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = n_iter < 4LL * nsm ? n_iter : 4LL * nsm;
  dt_scores_kernel<HKV, D, UNROLL><<<static_cast<int>(grid), kDtThreads, 0, s>>>(
      static_cast<const uint4*>(v), W, A, ntok, L, dt);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dt_scores(const void* v, const float* W, const float* A, int B, int L, int Hkv, int d,
                             float* dt, cudaStream_t s) {
#define DMA_DT_CASE(H, DD) \
  if (Hkv == H && d == DD) return launch_t<H, DD>(v, W, A, B, L, dt, s);
  DMA_DT_CASE(1, 64) DMA_DT_CASE(2, 64) DMA_DT_CASE(4, 64) DMA_DT_CASE(8, 64) DMA_DT_CASE(16, 64)
  DMA_DT_CASE(1, 128) DMA_DT_CASE(2, 128) DMA_DT_CASE(4, 128) DMA_DT_CASE(8, 128) DMA_DT_CASE(16, 128)
#undef DMA_DT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dma
