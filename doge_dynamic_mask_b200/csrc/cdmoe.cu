// CDMoE routing: router logits, per-domain top-k, the k best of their
// Cartesian product, and the embedding-table experts.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "跨域 MoE（CDMoE）：在稠密 checkpoint 上“叠加”稀疏专家": router_gate maps the
// hidden state to num_keys * 2 logits, a top-k runs along each of the two
// domains x and y (num_keys = floor(sqrt(num_experts))), and their Cartesian
// product names the experts, rows of two embedding tables (down_embed,
// up_embed) that are looked up and applied to the hidden state as
// down-projection -> activation -> up-projection.  num_experts_per_tok (the
// top-k) and hidden_act = silu come from "DogeConfig 全参数详解".
//
// Readings: logits columns [0, K) are domain x and [K, 2K) domain y; each
// domain keeps its k best keys (ties: lower key index); pair (a, b) scores
// s_x[a] + s_y[b] in float32 and names expert a * K + b; a token keeps the k
// best pairs (ties: lower expert index); routing weights are the softmax of
// the k kept scores; expert e adds w_e * silu(h . down_embed[e]) * up_embed[e].
//
// Design.
//   * cdmoe_logits_kernel: the router is a real GEMM, [T x hidden] x
//     [hidden x 2K], so it runs on the tcgen05 tensor cores: persistent CTAs
//     over 128-token tiles, TMA streams 64-channel chunks of h and of the
//     router weight (K-major, 128-byte swizzle) through a 4-stage ring, one
//     thread issues M=128, N=2K, K=16 MMAs into a TMEM accumulator, and four
//     epilogue warps write the float32 logits.
//   * cdmoe_route_experts_kernel: one CTA per token.  Each selection is a
//     radix select over 64-bit composite keys (order-preserving float bits
//     above, 0xFFFFFFFF - index below, so every key is distinct and the k-th
//     largest is unique): the k best keys of each domain, then the k best of
//     the k*k pair keys.  The expert part is a gather bound by the two
//     embedding rows per expert (2 * hidden * 2 bytes each): each warp reduces
//     whole down rows against h, then every thread owns hidden/blockDim
//     channels and accumulates the weighted up rows; there is nothing to tile
//     for the tensor cores, since every token has its own experts.
#include <cuda.h>

#include "select_common.cuh"

namespace dma {
namespace {

// ---- router logits on the tensor cores ------------------------------------------

constexpr int kRtThreads = 192;   // warp 0: TMA producer; warp 1: MMA issuer, TMEM owner; warps 2-5: epilogue
constexpr int kRtTile = 128;      // tokens per tile (MMA M)
constexpr int kRtStages = 4;
constexpr int kRtChunk = 64;      // channels per stage

template <int N>
struct RtCfg {
  static constexpr int kABytes = kRtTile * 128;              // 16 KB
  static constexpr int kBBytes = N * 128;                     // N rows x 64 channels
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kOffBar = kRtStages * kStageBytes;
  static constexpr int kSmemBytes = kOffBar + 256 + 1024;     // + alignment slack
  static constexpr uint32_t kTmemCols = N <= 32 ? 32 : (N <= 64 ? 64 : (N <= 128 ? 128 : 256));
  static_assert(kBBytes % 1024 == 0, "swizzle atoms need 1024-byte aligned chunks");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

template <int N>
__global__ void __launch_bounds__(kRtThreads, 1)
    cdmoe_logits_kernel(const __grid_constant__ CUtensorMap tmap_h, const __grid_constant__ CUtensorMap tmap_w,
                        int T, int hidden, float* __restrict__ logits, uint32_t* err) {
  using C = RtCfg<N>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* empty = full + kRtStages;
  uint64_t* acc_full = empty + kRtStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* fin = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (T + kRtTile - 1) / kRtTile;
  const int n_chunks = hidden / kRtChunk;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRtStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 4);   // one arrival per epilogue warp
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_h);
    prefetch_tmap(&tmap_w);
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int gs = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        for (int kc = 0; kc < n_chunks; ++kc, ++gs) {
          const int s = gs % kRtStages;
          if (gs >= kRtStages && !mbar_wait(empty + s, ((gs / kRtStages) - 1) & 1, err, kDevErrTimeoutBase + 30)) {
            ok = false;
            *abort_flag = 1;
            break;
          }
          if (*abort_flag) {
            ok = false;
            break;
          }
          unsigned char* st = smem + s * C::kStageBytes;
          mbar_arrive_expect_tx(full + s, C::kStageBytes);
          tma_load_2d(st, &tmap_h, full + s, kc * kRtChunk, t * kRtTile);
          tma_load_2d(st + C::kABytes, &tmap_w, full + s, kc * kRtChunk, 0);
        }
      }
      for (int j = gs - kRtStages < 0 ? 0 : gs - kRtStages; j < gs; ++j)
        mbar_wait(full + j % kRtStages, (j / kRtStages) & 1, err, kDevErrTimeoutBase + 31);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(kRtTile, N, false, false);
      const uint32_t base_lo = desc_lo(smem_u32(smem), 16);
      int gs = 0, it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++it) {
        if (it >= 1 && !mbar_wait_hot(acc_empty, (it - 1) & 1, err, kDevErrTimeoutBase + 32)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kc = 0; kc < n_chunks; ++kc, ++gs) {
          const int s = gs % kRtStages;
          if (!mbar_wait_hot(full + s, (gs / kRtStages) & 1, err, kDevErrTimeoutBase + 33)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = base_lo + static_cast<uint32_t>((s * C::kStageBytes) >> 4);
          const uint32_t b = a + static_cast<uint32_t>(C::kABytes >> 4);
          if (kc == 0) umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem, a, b, idesc);
          else umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem, a, b, idesc);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk) umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem, a + 2 * kk, b + 2 * kk, idesc);
          umma_commit(empty + s);
        }
        if (!ok) break;
        umma_commit(acc_full);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(fin);
      mbar_wait_hot(fin, 0, err, kDevErrTimeoutBase + 34);
    }
    __syncwarp();
  } else {
    // epilogue: thread = token of the tile (TMEM lane)
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    int it = 0;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++it) {
      const bool ok = mbar_wait(acc_full, it & 1, err, kDevErrTimeoutBase + 35) && !*abort_flag;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const long long tok = static_cast<long long>(t) * kRtTile + row;
      float* dst = logits + tok * N;
#pragma unroll
      for (int c0 = 0; c0 < N; c0 += 32) {
        uint32_t r[32];
        DMA_TMEM_LD32(tmem + lane_base + c0, r);
        tmem_wait_ld();
        if (tok < T) {
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<uint4*>(dst + c0 + c) = make_uint4(r[c], r[c + 1], r[c + 2], r[c + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive_warp(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

// ---- routing and experts, one CTA per token -----------------------------------------

constexpr int kRouteThreads = 256;
constexpr int kMaxTopK = 64;         // k = num_experts_per_tok

// float32 bits -> uint32 with the same order (finite values)
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct RouteSmem {
  uint32_t hist[kBins];
  uint32_t red[64];
  uint64_t vars[8];
  uint64_t keys[kMaxTopK * kMaxTopK];   // candidate keys (domain keys first, then pair keys)
  float sx[kMaxTopK], sy[kMaxTopK];     // kept domain scores
  int ix[kMaxTopK], iy[kMaxTopK];       // kept domain key indices
  uint64_t fin[kMaxTopK];               // kept pair keys
  float wt[kMaxTopK];                   // routing weight * silu(h . down) per kept expert
  int ex[kMaxTopK];                     // kept experts, best first
  float sc[kMaxTopK];
  int coff[kMaxTopK + 1];               // first candidate pair of each x key
  float mout;                           // best pair score outside the candidate region
};

// two bf16 channels (one 32-bit word, low channel first) as packed float32
__device__ __forceinline__ unsigned long long widen_bf16x2(uint32_t w) {
  return f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Keeps the k best of the domain's K <= blockDim keys, best first: thread j
// ranks key j by counting the keys above it (composite keys are distinct) and
// writes its score and index at that rank when the rank is below k.  Every
// thread must call it.
__device__ __forceinline__ void domain_topk(const float* __restrict__ lg, int K, int k, RouteSmem& sm,
                                            float* s_out, int* i_out) {
  uint64_t mine = 0ull;
  if (static_cast<int>(threadIdx.x) < K) {
    mine = (static_cast<uint64_t>(ordered_bits(lg[threadIdx.x])) << 32) | (0xFFFFFFFFu - threadIdx.x);
    sm.keys[threadIdx.x] = mine;
  }
  __syncthreads();
  if (static_cast<int>(threadIdx.x) < K) {
    int rank = 0;
#pragma unroll 8
    for (int q = 0; q < K; ++q) rank += sm.keys[q] > mine;
    if (rank < k) {
      s_out[rank] = lg[threadIdx.x];
      i_out[rank] = static_cast<int>(threadIdx.x);
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kRouteThreads)
    cdmoe_route_experts_kernel(const uint16_t* __restrict__ h, const float* __restrict__ logits,
                               const uint16_t* __restrict__ down_embed, const uint16_t* __restrict__ up_embed,
                               int hidden, int K, int k, uint16_t* __restrict__ out, int32_t* __restrict__ experts_out,
                               float* __restrict__ scores_out) {
  __shared__ RouteSmem sm;
  pdl_wait();   // the logits come from the previous kernel
  const SelScratch sc{sm.hist, nullptr, sm.red, sm.vars};
  const int t = blockIdx.x;
  const float* lg = logits + static_cast<size_t>(t) * 2 * K;

  // 1. the k best keys of each domain, best first
  domain_topk(lg, K, k, sm, sm.sx, sm.ix);
  domain_topk(lg + K, K, k, sm, sm.sy, sm.iy);
  // 2. the k best pairs.  With both domains sorted, pair (a, b) is beaten by
  // the (a+1)(b+1) pairs (a' <= a, b' <= b) at least as good, so the k best
  // lie among the pairs with (a+1)(b+1) <= k (about k ln k of them): rank those
  // by counting.  That is exact when the k-th of them scores strictly above
  // every pair outside the region, whose best is sx[a] + sy[floor(k/(a+1))]
  // for some a; otherwise (ties at the boundary) all k*k pairs are selected.
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int a = 0; a < k; ++a) {
      sm.coff[a] = acc;
      const int nb = k / (a + 1);
      acc += nb < k ? nb : k;
    }
    sm.coff[k] = acc;
  }
  __syncthreads();
  const int nc = sm.coff[k];
  auto pair_key = [&](int a, int b) {
    const float s = sm.sx[a] + sm.sy[b];
    const uint32_t e = static_cast<uint32_t>(sm.ix[a] * K + sm.iy[b]);
    return (static_cast<uint64_t>(ordered_bits(s)) << 32) | (0xFFFFFFFFu - e);
  };
  for (int c = threadIdx.x; c < nc; c += blockDim.x) {
    int a = 0;
    while (sm.coff[a + 1] <= c) ++a;
    sm.keys[c] = pair_key(a, c - sm.coff[a]);
  }
  if (threadIdx.x < 32) {
    // best score outside the region
    float m = -INFINITY;
    for (int a = threadIdx.x; a < k; a += 32) {
      const int b = k / (a + 1);
      if (b < k) m = fmaxf(m, sm.sx[a] + sm.sy[b]);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0) sm.mout = m;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < nc; c += blockDim.x) {
    const uint64_t mine = sm.keys[c];
    int rank = 0;
#pragma unroll 8
    for (int q = 0; q < nc; ++q) rank += sm.keys[q] > mine;
    if (rank < k) {
      sm.fin[rank] = mine;
      if (rank == k - 1) sm.vars[0] = mine;
    }
  }
  __syncthreads();
  const uint32_t ob_k = static_cast<uint32_t>(sm.vars[0] >> 32);
  const bool exact = __uint_as_float((ob_k & 0x80000000u) ? (ob_k & 0x7FFFFFFFu) : ~ob_k) > sm.mout;
  __syncthreads();
  if (!exact) {
    const int n = k * k;
    for (int p = threadIdx.x; p < n; p += blockDim.x) sm.keys[p] = pair_key(p / k, p % k);
    __syncthreads();
    const uint64_t tau = select_kth_smem(sm.keys, n, static_cast<uint32_t>(k), sc);
    ordered_compact(n, [&](int p) { return sm.keys[p] >= tau; }, [&](int pos, int p) { sm.fin[pos] = sm.keys[p]; },
                    sc);
    // best first: rank of each kept key among the k (all distinct)
    uint64_t mine = 0ull;
    if (threadIdx.x < k) mine = sm.fin[threadIdx.x];
    int rank = 0;
    if (threadIdx.x < k)
      for (int q = 0; q < k; ++q) rank += sm.fin[q] > mine;
    __syncthreads();
    if (threadIdx.x < k) sm.fin[rank] = mine;
    __syncthreads();
  }
  // h of the token in float32, once, for the 64 down-row products: in the
  // candidate-key buffer (free now) after the up-projection's partial sums
  // (groups * hidden <= 8192 floats: hidden <= 8192, and groups * hidden =
  // 8 * blockDim when a row has fewer pieces than the block has threads)
  const int n16 = hidden / 8;   // 16-byte pieces per row
  const int groups = n16 >= static_cast<int>(blockDim.x) ? 1 : static_cast<int>(blockDim.x) / n16;
  float* hf = reinterpret_cast<float*>(sm.keys) + (groups - 1) * hidden;
  {
    const uint4* h4 = reinterpret_cast<const uint4*>(h + static_cast<size_t>(t) * hidden);
    for (int c = threadIdx.x; c < n16; c += blockDim.x) {
      const uint4 u = __ldg(h4 + c);
      const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        hf[8 * c + 2 * i] = __uint_as_float(x[i] << 16);
        hf[8 * c + 2 * i + 1] = __uint_as_float(x[i] & 0xFFFF0000u);
      }
    }
  }
  // 3. the kept experts and their scores, best first
  if (threadIdx.x < k) {
    const uint64_t mine = sm.fin[threadIdx.x];
    const int e = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(mine & 0xFFFFFFFFull));
    // recover the float32 score from its ordered bits
    const uint32_t ob = static_cast<uint32_t>(mine >> 32);
    sm.ex[threadIdx.x] = e;
    sm.sc[threadIdx.x] = __uint_as_float((ob & 0x80000000u) ? (ob & 0x7FFFFFFFu) : ~ob);
  }
  __syncthreads();
  if (experts_out && threadIdx.x < k) {
    experts_out[static_cast<size_t>(t) * k + threadIdx.x] = sm.ex[threadIdx.x];
    scores_out[static_cast<size_t>(t) * k + threadIdx.x] = sm.sc[threadIdx.x];
  }
  // 4. down-projection: one warp per expert row, h . down_embed[e] (packed
  // float32 pairs against h in shared memory)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const float4* hf4 = reinterpret_cast<const float4*>(hf);
  for (int q = warp; q < k; q += nwarps) {
    const uint4* d4 = reinterpret_cast<const uint4*>(down_embed + static_cast<size_t>(sm.ex[q]) * hidden);
    unsigned long long acc2 = 0ull;
    for (int c = lane; c < n16; c += 32) {
      const uint4 dv = __ldg(d4 + c);
      const float4 ha = hf4[2 * c], hb = hf4[2 * c + 1];
      acc2 = fma_f32x2(widen_bf16x2(dv.x), f32x2(ha.x, ha.y), acc2);
      acc2 = fma_f32x2(widen_bf16x2(dv.y), f32x2(ha.z, ha.w), acc2);
      acc2 = fma_f32x2(widen_bf16x2(dv.z), f32x2(hb.x, hb.y), acc2);
      acc2 = fma_f32x2(widen_bf16x2(dv.w), f32x2(hb.z, hb.w), acc2);
    }
    float a0, a1;
    f32x2_split(acc2, a0, a1);
    float acc = a0 + a1;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (lane == 0) sm.wt[q] = acc / (1.0f + expf(-acc));   // silu
  }
  __syncthreads();
  // routing weights: softmax of the kept scores (best first, so sc[0] is the max)
  if (threadIdx.x < 32) {
    float z = 0.0f;
    for (int q = lane; q < k; q += 32) z += expf(sm.sc[q] - sm.sc[0]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
    const float inv = 1.0f / z;
    for (int q = lane; q < k; q += 32) sm.wt[q] *= expf(sm.sc[q] - sm.sc[0]) * inv;
  }
  __syncthreads();
  // 5. up-projection: every thread owns one 8-channel piece of the row and a
  // share of the kept experts (groups of threads split the experts when the
  // row has fewer pieces than the block has threads); the groups' partial
  // sums meet in shared memory (the candidate-key buffer, free by now)
  float* part = reinterpret_cast<float*>(sm.keys);   // [groups - 1][hidden]
  for (int c0 = 0; c0 < n16; c0 += static_cast<int>(blockDim.x) / groups) {
    const int c = c0 + static_cast<int>(threadIdx.x) % (static_cast<int>(blockDim.x) / groups);
    const int grp = static_cast<int>(threadIdx.x) / (static_cast<int>(blockDim.x) / groups);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (c < n16 && grp < groups) {
      unsigned long long acc2[4] = {0ull, 0ull, 0ull, 0ull};   // packed channel pairs
#pragma unroll 4
      for (int q = grp; q < k; q += groups) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(up_embed + static_cast<size_t>(sm.ex[q]) * hidden) + c);
        const float wq = sm.wt[q];
        const unsigned long long w2 = f32x2(wq, wq);
        const uint32_t x[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) acc2[i] = fma_f32x2(widen_bf16x2(x[i]), w2, acc2[i]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) f32x2_split(acc2[i], acc[2 * i], acc[2 * i + 1]);
      if (grp > 0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) part[(grp - 1) * hidden + 8 * c + i] = acc[i];
      }
    }
    __syncthreads();
    if (c < n16 && grp == 0) {
      for (int g2 = 1; g2 < groups; ++g2) {
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += part[(g2 - 1) * hidden + 8 * c + i];
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(out + static_cast<size_t>(t) * hidden)[c] = o;
    }
    __syncthreads();
  }
}

template <int N>
cudaError_t launch_logits_n(const void* h, const void* W, int T, int hidden, float* logits, uint32_t* err,
                            cudaStream_t s) {
  using C = RtCfg<N>;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap th, tw;
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(T)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(hidden) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kRtChunk), static_cast<cuuint32_t>(kRtTile)};
    cuuint32_t es[2] = {1, 1};
    if (enc(&th, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(h), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(hidden), static_cast<cuuint64_t>(N)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(hidden) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kRtChunk), static_cast<cuuint32_t>(N)};
    cuuint32_t es[2] = {1, 1};
    if (enc(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(W), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(cdmoe_logits_kernel<N>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const int n_tiles = (T + kRtTile - 1) / kRtTile;
  const int grid = n_tiles < nsm ? n_tiles : nsm;
  cdmoe_logits_kernel<N><<<grid, kRtThreads, C::kSmemBytes, s>>>(th, tw, T, hidden, logits, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_cdmoe_logits(const void* h, const void* W_router, int T, int hidden, int K, float* logits,
                                uint32_t* err, cudaStream_t s) {
  switch (2 * K) {
    case 32: return launch_logits_n<32>(h, W_router, T, hidden, logits, err, s);
    case 64: return launch_logits_n<64>(h, W_router, T, hidden, logits, err, s);
    case 128: return launch_logits_n<128>(h, W_router, T, hidden, logits, err, s);
    case 256: return launch_logits_n<256>(h, W_router, T, hidden, logits, err, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_cdmoe_route_experts(const void* h, const float* logits, const void* down_embed,
                                       const void* up_embed, int T, int hidden, int K, int k, void* out,
                                       int32_t* experts_out, float* scores_out, cudaStream_t s) {
  return launch_after(cdmoe_route_experts_kernel, dim3(static_cast<unsigned>(T)), dim3(kRouteThreads), 0, s,
                      static_cast<const uint16_t*>(h), logits, static_cast<const uint16_t*>(down_embed),
                      static_cast<const uint16_t*>(up_embed), hidden, K, k, static_cast<uint16_t*>(out), experts_out,
                      scores_out);
}

}  // namespace dma
