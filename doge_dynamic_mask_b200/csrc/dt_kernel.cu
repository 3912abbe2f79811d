// S1: per-key score dt = exp(A * softplus(dt_proj(value_states))), float32.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", forward chain step 3
// (dt_proj projects the value states to num_key_value_heads outputs; A is one
// scalar per kv head).  No bias: attention_bias=False in section
// "DogeConfig 全参数详解".
//
// Design.  The projection is a skinny GEMV: every token row of C = Hkv*d bf16
// values meets the same [C, Hkv] weight, so the kernel is bound by the one read
// of V from HBM.  Each lane owns whole tokens (K of them): it streams its rows
// in 32-byte chunks (16 channels, one full sector per 256-bit load), keeps
// DEPTH chunks per token in flight in registers, and accumulates all Hkv dot products itself, so there is no
// cross-lane reduction and no block barrier in the main loop.  The weight is
// staged once per block in shared memory as channel pairs
// (W[2p][g], W[2p+1][g]); all lanes of a warp read the same chunk's weights at
// the same time (broadcast), and each pair feeds one packed fma.rn.f32x2 with
// the matching pair of value channels.  The epilogue adds the two halves,
// applies softplus, the A multiply and exp in float32 and writes dt
// [B, Hkv, L] coalesced across lanes.
#include "common.cuh"

namespace dma {
namespace {

constexpr int kDtThreads = 256;

__device__ __forceinline__ unsigned long long pack_f32x2(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void unpack_f32x2(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// acc = a * b + acc on both float32 halves (round-to-nearest, like fmaf).
__device__ __forceinline__ void fma_acc_f32x2(unsigned long long& acc, unsigned long long a, unsigned long long b) {
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(a), "l"(b));
}
// Two bf16 (low half first) as a float32 pair.
__device__ __forceinline__ unsigned long long bf16x2_to_f32x2(uint32_t u) {
  return pack_f32x2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__device__ __forceinline__ float softplus_f32(float x) {
  // log(1 + e^x) in the overflow-free form max(x, 0) + log1p(e^-|x|).
  return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x)));
}

__device__ __forceinline__ uint32_t word(const uint4& u, int i) {
  return i == 0 ? u.x : i == 1 ? u.y : i == 2 ? u.z : u.w;
}

// 32 bytes (16 bf16 channels) of one token row.  WIDE: one 256-bit load (the
// base pointer is 32-byte aligned); else two 128-bit loads.
struct Chunk32 {
  uint32_t w[8];
};

template <bool WIDE>
__device__ __forceinline__ Chunk32 load_chunk(const uint4* __restrict__ v, long long idx16) {
  Chunk32 c;
  if constexpr (WIDE) {
    asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(c.w[0]), "=r"(c.w[1]), "=r"(c.w[2]), "=r"(c.w[3]), "=r"(c.w[4]), "=r"(c.w[5]),
                   "=r"(c.w[6]), "=r"(c.w[7])
                 : "l"(v + idx16));
  } else {
    const uint4 a = __ldcs(v + idx16), b = __ldcs(v + idx16 + 1);
    c.w[0] = a.x; c.w[1] = a.y; c.w[2] = a.z; c.w[3] = a.w;
    c.w[4] = b.x; c.w[5] = b.y; c.w[6] = b.z; c.w[7] = b.w;
  }
  return c;
}

// HKV outputs per token, D head dims, K tokens per lane, DEPTH 32-byte chunks
// per token in flight.
template <int HKV, int D, int K, int DEPTH, bool WIDE>
__global__ void __launch_bounds__(kDtThreads) dt_scores_kernel(const uint4* __restrict__ v,
                                                                const float* __restrict__ W,
                                                                const float* __restrict__ A, long long ntok,
                                                                int L, float* __restrict__ dt) {
  constexpr int C = HKV * D;          // channels per token
  constexpr int N16 = C / 8;          // 16-byte pieces per token
  constexpr int NCH = C / 16;         // 32-byte chunks per token
  static_assert(NCH % DEPTH == 0, "chunk ring must tile the row");
  extern __shared__ unsigned long long w2s[];   // [C/2][HKV] channel pairs

  for (int i = threadIdx.x; i < (C / 2) * HKV; i += kDtThreads) {
    const int p = i / HKV, g = i % HKV;
    w2s[i] = pack_f32x2(W[(2 * p) * HKV + g], W[(2 * p + 1) * HKV + g]);
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const long long warp_global = static_cast<long long>(blockIdx.x) * (kDtThreads / 32) + (threadIdx.x >> 5);
  const long long nwarps = static_cast<long long>(gridDim.x) * (kDtThreads / 32);
  const long long per_warp = 32LL * K;
  for (long long base = warp_global * per_warp; base < ntok; base += nwarps * per_warp) {
    long long tok[K];
    bool live[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
      tok[k] = base + k * 32 + lane;
      live[k] = tok[k] < ntok;
    }
    unsigned long long acc[K][HKV];
#pragma unroll
    for (int k = 0; k < K; ++k)
#pragma unroll
      for (int g = 0; g < HKV; ++g) acc[k][g] = 0ull;

    Chunk32 ring[DEPTH][K];
#pragma unroll
    for (int s = 0; s < DEPTH; ++s)
#pragma unroll
      for (int k = 0; k < K; ++k)
        if (live[k]) ring[s][k] = load_chunk<WIDE>(v, tok[k] * N16 + 2 * s);

#pragma unroll 1
    for (int ch0 = 0; ch0 < NCH; ch0 += DEPTH) {
#pragma unroll
      for (int s = 0; s < DEPTH; ++s) {
        const int ch = ch0 + s;
        Chunk32 cur[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
          cur[k] = ring[s][k];
          const int nx = ch + DEPTH;
          if (live[k] && nx < NCH) ring[s][k] = load_chunk<WIDE>(v, tok[k] * N16 + 2 * nx);
        }
        const unsigned long long* wc = w2s + static_cast<size_t>(ch) * 8 * HKV;   // this chunk's 8 pairs
#pragma unroll
        for (int pp = 0; pp < 8; ++pp) {
          unsigned long long wp[HKV];
#pragma unroll
          for (int g = 0; g < HKV; ++g) wp[g] = wc[pp * HKV + g];
#pragma unroll
          for (int k = 0; k < K; ++k) {
            const unsigned long long xp = bf16x2_to_f32x2(cur[k].w[pp]);
#pragma unroll
            for (int g = 0; g < HKV; ++g) fma_acc_f32x2(acc[k][g], xp, wp[g]);
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
      if (!live[k]) continue;
      const long long b = tok[k] / L;
      const long long l = tok[k] - b * L;
#pragma unroll
      for (int g = 0; g < HKV; ++g) {
        float lo, hi;
        unpack_f32x2(acc[k][g], lo, hi);
        dt[(b * HKV + g) * L + l] = expf(A[g] * softplus_f32(lo + hi));
      }
    }
  }
}

template <int HKV, int D, int K, bool WIDE>
cudaError_t launch_k(const void* v, const float* W, const float* A, long long ntok, int L, float* dt, int nsm,
                     cudaStream_t s) {
  constexpr int DEPTH = 2;
  const size_t smem = static_cast<size_t>(HKV) * D / 2 * HKV * sizeof(unsigned long long);
  auto kern = dt_scores_kernel<HKV, D, K, DEPTH, WIDE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long warps_needed = (ntok + 32LL * K - 1) / (32LL * K);
  long long blocks = (warps_needed + kDtThreads / 32 - 1) / (kDtThreads / 32);
  const long long cap = 4LL * nsm;
  if (blocks > cap) blocks = cap;
  kern<<<static_cast<int>(blocks), kDtThreads, smem, s>>>(static_cast<const uint4*>(v), W, A, ntok, L, dt);
  return cudaGetLastError();
}

template <int HKV, int D>
cudaError_t launch_t(const void* v, const float* W, const float* A, int B, int L, float* dt, cudaStream_t s) {
  constexpr int KBIG = HKV >= 8 ? 2 : 4;
  const long long ntok = static_cast<long long>(B) * L;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const bool wide = (reinterpret_cast<uintptr_t>(v) & 31u) == 0;
  // short inputs: one token per lane so that every SM gets warps
  if (ntok < 32LL * KBIG * 8 * 2 * nsm)
    return wide ? launch_k<HKV, D, 1, true>(v, W, A, ntok, L, dt, nsm, s)
                : launch_k<HKV, D, 1, false>(v, W, A, ntok, L, dt, nsm, s);
  return wide ? launch_k<HKV, D, KBIG, true>(v, W, A, ntok, L, dt, nsm, s)
              : launch_k<HKV, D, KBIG, false>(v, W, A, ntok, L, dt, nsm, s);
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
