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
//
// Tensor-core path (Hkv <= 8, d in {64, 128}).  The same projection as a
// [tokens x C] x [C x N] product on tcgen05 tensor cores, so the kernel is
// bound by streaming V from HBM rather than by float32 FMA issue: a persistent
// CTA per SM streams 128-token tiles of V through an 8-stage ring of 16 KB
// shared-memory stages (TMA, 128-byte swizzle, 64 channels per stage); one
// thread issues M=128, K=16 MMAs into a double-buffered TMEM accumulator; four
// epilogue warps finish the tiles.  B holds the float32 weight split exactly
// into three bf16 terms, W = W_hi + W_mid + W_lo (each the bf16 rounding of
// what the previous terms leave), as column groups [W_hi | W_mid | W_lo]:
// products of bf16 values are exact and the tensor core accumulates in
// float32, so the three column sums add up to the float32 projection.
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
  pdl_trigger();   // the next kernel (selection or attention) may be scheduled

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
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
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
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const bool wide = (reinterpret_cast<uintptr_t>(v) & 31u) == 0;
  // short inputs: one token per lane so that every SM gets warps
  if (ntok < 32LL * KBIG * 8 * 2 * nsm)
    return wide ? launch_k<HKV, D, 1, true>(v, W, A, ntok, L, dt, nsm, s)
                : launch_k<HKV, D, 1, false>(v, W, A, ntok, L, dt, nsm, s);
  return wide ? launch_k<HKV, D, KBIG, true>(v, W, A, ntok, L, dt, nsm, s)
              : launch_k<HKV, D, KBIG, false>(v, W, A, ntok, L, dt, nsm, s);
}


// ---- tensor-core path ---------------------------------------------------------

__device__ __forceinline__ bool aborted_flag(volatile int* flag) { return *flag != 0; }

constexpr int kDtTcThreads = 192;   // warp 0: TMA producer; warp 1: MMA issuer, TMEM owner; warps 2-5: epilogue
constexpr int kDtTile = 128;        // tokens per tile (MMA M)
constexpr int kDtStages = 8;
constexpr int kDtChunk = 64;        // channels per stage: one 128-byte swizzled row per token

template <int HKV, int D>
struct DtTc {
  static constexpr int C = HKV * D;
  static constexpr int kChunks = C / kDtChunk;
  static constexpr int N = (3 * HKV + 15) / 16 * 16;     // three bf16 terms per head, padded for the MMA
  static constexpr int kStageBytes = kDtTile * 128;      // 16 KB
  static constexpr int kBChunkBytes = N * 128;           // B rows (N) x 64 channels
  static constexpr int kOffA = kChunks * kBChunkBytes;
  static constexpr int kOffBar = kOffA + kDtStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;   // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * N <= 32 ? 32 : (2 * N <= 64 ? 64 : 128);
  static_assert(kBChunkBytes % 1024 == 0, "swizzle atoms need 1024-byte aligned chunks");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// byte offset of element (row n, channel c) of B in the K-major 128-byte-swizzled layout
template <int N>
__device__ __forceinline__ uint32_t b_offset(int n, int c) {
  const int kc = c / kDtChunk, cc = c % kDtChunk;
  return static_cast<uint32_t>(kc * N * 128 + n * 128 + (((cc >> 3) ^ (n & 7)) << 4) + (cc & 7) * 2);
}

template <int HKV, int D>
__global__ void __launch_bounds__(kDtTcThreads, 1)
    dt_tc_kernel(const __grid_constant__ CUtensorMap tmap_v, const float* __restrict__ W,
                 const float* __restrict__ A, int ntok, int L, float* __restrict__ dt, uint32_t* err) {
  using T = DtTc<HKV, D>;
  extern __shared__ unsigned char smem_raw[];
  pdl_trigger();   // the next kernel (selection or attention) may be scheduled
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  unsigned char* sB = smem;
  unsigned char* sA = smem + T::kOffA;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + T::kOffBar);
  uint64_t* empty = full + kDtStages;
  uint64_t* acc_full = empty + kDtStages;    // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* fin = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (ntok + kDtTile - 1) / kDtTile;

  // the producer (thread 0) sets up the barriers and issues the first
  // kDtStages copies at once, so the weight split below overlaps their latency
  int pt = blockIdx.x, pkc = 0, pgs = 0;   // producer cursor: tile, chunk, copies issued
  auto issue = [&]() {
    const int s = pgs % kDtStages;
    mbar_arrive_expect_tx(full + s, T::kStageBytes);
    tma_load_2d(sA + s * T::kStageBytes, &tmap_v, full + s, pkc * kDtChunk, pt * kDtTile);
    ++pgs;
    if (++pkc == T::kChunks) {
      pkc = 0;
      pt += gridDim.x;
    }
  };
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDtStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, 4);   // one arrival per epilogue warp
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_v);
    while (pgs < kDtStages && pt < n_tiles) issue();
  }

  // B = [W_hi | W_mid | W_lo | 0], row n = term * HKV + g, K-major over the
  // channels; each thread loads sixteen weights at a time, so their latencies
  // overlap instead of adding up
  constexpr int kWBatch = 16;
  for (int i0 = 0; i0 < T::C * HKV; i0 += kWBatch * kDtTcThreads) {
    float wv[kWBatch];
#pragma unroll
    for (int r = 0; r < kWBatch; ++r) {
      const int i = i0 + r * kDtTcThreads + static_cast<int>(threadIdx.x);
      wv[r] = i < T::C * HKV ? __ldg(W + i) : 0.0f;
    }
#pragma unroll
    for (int r = 0; r < kWBatch; ++r) {
      const int i = i0 + r * kDtTcThreads + static_cast<int>(threadIdx.x);
      if (i < T::C * HKV) {
        const int c = i / HKV, g = i % HKV;
        const float w = wv[r];
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
        *reinterpret_cast<__nv_bfloat16*>(sB + b_offset<T::N>(g, c)) = hi;
        *reinterpret_cast<__nv_bfloat16*>(sB + b_offset<T::N>(HKV + g, c)) = mid;
        *reinterpret_cast<__nv_bfloat16*>(sB + b_offset<T::N>(2 * HKV + g, c)) = lo;
      }
    }
  }
  for (int i = threadIdx.x; i < (T::N - 3 * HKV) * T::C; i += blockDim.x) {
    const int n = 3 * HKV + i / T::C, c = i % T::C;
    *reinterpret_cast<uint16_t*>(sB + b_offset<T::N>(n, c)) = 0;
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(tmem_slot, T::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      while (ok && pt < n_tiles) {
        const int s = pgs % kDtStages;
        if (!mbar_wait(empty + s, ((pgs / kDtStages) - 1) & 1, err, kDevErrTimeoutBase + 20)) {
          ok = false;
          *abort_flag = 1;
          break;
        }
        if (aborted_flag(abort_flag)) {
          ok = false;
          break;
        }
        issue();
      }
      // every copy issued must land before the CTA leaves
      for (int j = pgs - kDtStages < 0 ? 0 : pgs - kDtStages; j < pgs; ++j)
        mbar_wait(full + j % kDtStages, (j / kDtStages) & 1, err, kDevErrTimeoutBase + 21);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(kDtTile, T::N, false, false);
      const uint32_t a_lo = desc_lo(smem_u32(sA), 16), b_lo = desc_lo(smem_u32(sB), 16);
      int gs = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++it) {
        const int buf = it & 1;
        if (it >= 2 && !mbar_wait_hot(acc_empty + buf, ((it - 2) >> 1) & 1, err, kDevErrTimeoutBase + 22)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(buf * T::N);
        for (int kc = 0; kc < T::kChunks; ++kc, ++gs) {
          const int s = gs % kDtStages;
          if (!mbar_wait_hot(full + s, (gs / kDtStages) & 1, err, kDevErrTimeoutBase + 23)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = a_lo + static_cast<uint32_t>(s * (T::kStageBytes >> 4));
          const uint32_t b = b_lo + static_cast<uint32_t>(kc * (T::kBChunkBytes >> 4));
          if (kc == 0) umma_ss_w<0, kDescHiSw128, kDescHiSw128>(d, a, b, idesc);
          else umma_ss_w<1, kDescHiSw128, kDescHiSw128>(d, a, b, idesc);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk)
            umma_ss_w<1, kDescHiSw128, kDescHiSw128>(d, a + 2 * kk, b + 2 * kk, idesc);
          umma_commit(empty + s);
        }
        if (!ok) break;
        umma_commit(acc_full + buf);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(fin);
      mbar_wait_hot(fin, 0, err, kDevErrTimeoutBase + 24);
    }
    __syncwarp();
  } else {
    // epilogue: thread = token of the tile (TMEM lane)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    float a[HKV];
#pragma unroll
    for (int g = 0; g < HKV; ++g) a[g] = A[g];
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
      const int buf = it & 1;
      const bool ok = mbar_wait(acc_full + buf, (it >> 1) & 1, err, kDevErrTimeoutBase + 25) && !aborted_flag(abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      uint32_t r[T::N];
      const uint32_t taddr = tmem + lane_base + static_cast<uint32_t>(buf * T::N);
      if constexpr (T::N == 16) {
        DMA_TMEM_LD16(taddr, r);
      } else if constexpr (T::N == 32) {
        DMA_TMEM_LD32(taddr, r);
      } else {
        DMA_TMEM_LD32(taddr, r);
        DMA_TMEM_LD16(taddr + 32, (r + 32));
      }
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive_warp(acc_empty + buf);
      const long long tok = static_cast<long long>(t) * kDtTile + row;
      if (tok < ntok) {
        const long long b = tok / L;
        const long long l = tok - b * L;
#pragma unroll
        for (int g = 0; g < HKV; ++g) {
          const float z = (__uint_as_float(r[g]) + __uint_as_float(r[HKV + g])) + __uint_as_float(r[2 * HKV + g]);
          dt[(b * HKV + g) * L + l] = expf(a[g] * softplus_f32(z));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, T::kTmemCols);
}

template <int HKV, int D>
cudaError_t launch_tc(const void* v, const float* W, const float* A, long long ntok, int L, float* dt,
                      uint32_t* err, cudaStream_t s) {
  using T = DtTc<HKV, D>;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tm;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(T::C), static_cast<cuuint64_t>(ntok)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(T::C) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kDtChunk), static_cast<cuuint32_t>(kDtTile)};
  cuuint32_t es[2] = {1, 1};
  if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(v), dims, strides, box, es,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(dt_tc_kernel<HKV, D>), T::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const long long n_tiles = (ntok + kDtTile - 1) / kDtTile;
  const int grid = static_cast<int>(n_tiles < nsm ? n_tiles : nsm);
  dt_tc_kernel<HKV, D><<<grid, kDtTcThreads, T::kSmemBytes, s>>>(tm, W, A, static_cast<int>(ntok), L, dt, err);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_dt_scores(const void* v, const float* W, const float* A, int B, int L, int Hkv, int d,
                             float* dt, uint32_t* err, cudaStream_t s) {
  const long long ntok = static_cast<long long>(B) * L;
  // tensor-core path: TMA needs a 16-byte aligned V and fewer than 2^31 tokens
  if ((reinterpret_cast<uintptr_t>(v) & 15u) == 0 && ntok < (1LL << 31) && get_encode_fn()) {
#define DMA_DT_TC(H, DD) \
  if (Hkv == H && d == DD) return launch_tc<H, DD>(v, W, A, ntok, L, dt, err, s);
    DMA_DT_TC(1, 64) DMA_DT_TC(2, 64) DMA_DT_TC(4, 64) DMA_DT_TC(8, 64)
    DMA_DT_TC(1, 128) DMA_DT_TC(2, 128) DMA_DT_TC(4, 128) DMA_DT_TC(8, 128)
#undef DMA_DT_TC
  }
#define DMA_DT_CASE(H, DD) \
  if (Hkv == H && d == DD) return launch_t<H, DD>(v, W, A, B, L, dt, s);
  DMA_DT_CASE(1, 64) DMA_DT_CASE(2, 64) DMA_DT_CASE(4, 64) DMA_DT_CASE(8, 64) DMA_DT_CASE(16, 64)
  DMA_DT_CASE(1, 128) DMA_DT_CASE(2, 128) DMA_DT_CASE(4, 128) DMA_DT_CASE(8, 128) DMA_DT_CASE(16, 128)
#undef DMA_DT_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dma
