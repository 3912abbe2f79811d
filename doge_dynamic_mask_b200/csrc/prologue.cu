// Prologue of the attention forward: q_norm / k_norm, rotary embedding, KV-cache append.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", forward-chain steps 1 and 2:
// after the projections, Q and K pass an RMSNorm over head_dim (q_norm / k_norm,
// the Llama RMSNorm the section "从源码理解两大核心模块" says Doge reuses), then
// the rotary position embedding (Llama's apply_rotary_pos_emb); K and V are then
// appended to the KV cache.  rms_norm_eps comes from "DogeConfig 全参数详解".
//
//   y_c   = w_c * x_c / sqrt(mean_c(x^2) + eps)                  (per head row of d channels)
//   out_i = y_i cos(a_i) - y_{i+d/2} sin(a_i),  out_{i+d/2} = y_{i+d/2} cos(a_i) + y_i sin(a_i)
//   a_i   = pos * theta^(-2i/d),  i < d/2,  pos = positions[b] + t
//
// Design.  Memory-bound: every projected row is read once and written once.
// One CTA per token: the d/2 angles of its position are formed in double
// precision (a position of 10^5 times a frequency near 1 would lose about
// 2^-7 rad of its angle in float32, the size of a bf16 rounding) as turns
// (pos times theta^(-2i/d) / (2 pi), the factors formed once per call by the
// launcher), reduced to their fractional part, and their cosines and sines
// taken in float32 (sincospi) and kept in shared memory; then each group of d/8 lanes owns
// one head row as sixteen-byte vectors (eight bf16 channels per lane): the
// mean square is a group shuffle reduction, and channel i's rotation partner
// i + d/2 sits in the lane d/16 positions away, one shuffle.  A lane's
// channels are the same for every row it handles, so its norm weights,
// cosines and sines live in registers (shared memory and L1 then carry only
// the rows).  Each lane keeps two row pieces in flight (the first two are
// requested before the angles are formed, and each piece's successor as soon
// as it is taken).  Arithmetic is float32 with one rounding to bf16 at the
// end; V rows are copied bit for bit.
#include <cuda_runtime.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kPrologueThreads = 128;

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// One row-group step: this lane's 16-byte piece of head row r (q, k or v).
struct RowPiece {
  uint4 u;
  int r;
};

// theta^(-2i/d) / (2 pi) for i < d/2: each angle in turns is pos times one of
// these, formed once per call in double precision by the launcher
struct RopeTurns {
  double t[64];
};

template <int D>
__global__ void __launch_bounds__(kPrologueThreads)
    prologue_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
                    const float* __restrict__ q_w, const float* __restrict__ k_w, float eps,
                    const __grid_constant__ RopeTurns turns,
                    const int32_t* __restrict__ positions, int L, int Lmax, int Hq, int Hkv,
                    uint4* __restrict__ q_out, uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                    uint32_t* err) {
  constexpr int kLanesPerRow = D / 8;               // 16-byte vectors per head row
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  constexpr int kHalf = kLanesPerRow / 2;           // lane distance of channel i's partner i + d/2
  constexpr int kStride = (kPrologueThreads / 32) * kRowsPerWarp;   // rows per block step
  constexpr int kBatch = 2;                         // block steps whose loads are in flight together
  __shared__ float s_cos[D / 2], s_sin[D / 2];

  const int token = blockIdx.x;                     // b * L + t
  const int b = token / L, t = token - b * L;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % kLanesPerRow;              // this lane's 8 channels: [8 sub, 8 sub + 8)
  const int rows = Hq + 2 * Hkv;                    // q heads, then k heads, then v heads
  const size_t qrow0 = static_cast<size_t>(token) * Hq;
  const size_t krow0 = static_cast<size_t>(token) * Hkv;
  const int row_in_step = warp * kRowsPerWarp + lane / kLanesPerRow;

  auto load = [&](int r) -> uint4 {
    if (r >= rows) return make_uint4(0u, 0u, 0u, 0u);
    if (r < Hq) return __ldcs(q + (qrow0 + r) * kLanesPerRow + sub);
    if (r < Hq + Hkv) return __ldcs(k + (krow0 + (r - Hq)) * kLanesPerRow + sub);
    return __ldcs(v + (krow0 + (r - Hq - Hkv)) * kLanesPerRow + sub);
  };
  // the first batch of rows is in flight while the angles are formed
  RowPiece pc[kBatch];
#pragma unroll
  for (int it = 0; it < kBatch; ++it) {
    pc[it].r = it * kStride + row_in_step;
    pc[it].u = load(pc[it].r);
  }
  const int pos = positions[b] + t;
  const bool in_cache = positions[b] >= 0 && pos < Lmax;
  if (threadIdx.x == 0 && !in_cache) raise_error(err, kDevErrBadPosition);
  if (threadIdx.x < D / 2) {
    // the angle in turns, u = pos * theta^(-2i/d) / (2 pi), in double precision;
    // its fractional part r in [-1/2, 1/2] (exact in float32 to 2^-25) gives
    // cos and sin of 2 pi r = the angle modulo 2 pi, in float32
    const double u = static_cast<double>(pos) * turns.t[threadIdx.x];
    const float r = static_cast<float>(u - rint(u));
    float sn, cs;
    sincospif(2.0f * r, &sn, &cs);
    s_cos[threadIdx.x] = cs;
    s_sin[threadIdx.x] = sn;
  }
  __syncthreads();
  const size_t crow0 = in_cache ? (static_cast<size_t>(b) * Lmax + pos) * Hkv : 0;
  const bool low = sub < kHalf;                     // channels below d/2
  const int i0 = 8 * (low ? sub : sub - kHalf);     // pair index of this lane's first channel
  // this lane's channels never change: its norm weights, cosines and sines
  // are held in registers for every row it handles
  float wq[8], wk[8], cs8[8], sn8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    wq[e] = q_w[8 * sub + e];
    wk[e] = k_w[8 * sub + e];
    cs8[e] = s_cos[i0 + e];
    sn8[e] = low ? -s_sin[i0 + e] : s_sin[i0 + e];   // the low half subtracts its partner's share
  }

  for (int base = 0; base < rows; base += kBatch * kStride) {
#pragma unroll
    for (int it = 0; it < kBatch; ++it) {
      const int r = pc[it].r;
      const uint4 u = pc[it].u;
      // prefetch the same slot of the next batch
      const int rn = r + kBatch * kStride;
      if (base + kBatch * kStride < rows) pc[it].u = load(rn);
      pc[it].r = rn;
      const bool live = r < rows;
      const bool is_q = r < Hq, is_k = !is_q && r < Hq + Hkv;
      if (live && !is_q && !is_k) {
        if (in_cache) v_cache[(crow0 + (r - Hq - Hkv)) * kLanesPerRow + sub] = u;   // V: appended as is
      }
      // the shuffles below run on every lane of the warp (uniform trip count)
      float x[8];
      bf16x8_to_f32(u, x);
      float ss = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
      for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      const float inv = 1.0f / sqrtf(ss * (1.0f / D) + eps);
      float y[8], yp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = (live && (is_q || is_k)) ? (is_q ? wq[e] : wk[e]) * (x[e] * inv) : 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) yp[e] = __shfl_xor_sync(0xFFFFFFFFu, y[e], kHalf);
      if (live && (is_q || is_k)) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float o0 = fmaf(yp[e], sn8[e], y[e] * cs8[e]);
          const float o1 = fmaf(yp[e + 1], sn8[e + 1], y[e + 1] * cs8[e + 1]);
          pk[e / 2] = pack_bf16x2(o0, o1);
        }
        const uint4 o = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        if (is_q) __stcs(q_out + (qrow0 + r) * kLanesPerRow + sub, o);
        else if (in_cache) k_cache[(crow0 + (r - Hq)) * kLanesPerRow + sub] = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_prologue(const void* q, const void* k, const void* v, const float* q_w, const float* k_w,
                            float eps, float theta, const int32_t* positions, int B, int L, int Lmax, int Hq, int Hkv,
                            int d, void* q_out, void* k_cache, void* v_cache, uint32_t* err, cudaStream_t s) {
  const long long tokens = static_cast<long long>(B) * L;
  if (tokens > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (d != 64 && d != 128) return cudaErrorInvalidValue;
  RopeTurns turns{};
  const double log_theta = log(static_cast<double>(theta));
  for (int i = 0; i < d / 2; ++i) turns.t[i] = exp(-2.0 * i / d * log_theta) * 0.15915494309189535;   // / (2 pi)
  const dim3 grid(static_cast<unsigned>(tokens)), block(kPrologueThreads);
  if (d == 64)
    prologue_kernel<64><<<grid, block, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v), q_w, k_w, eps,
        turns, positions, L, Lmax, Hq, Hkv, static_cast<uint4*>(q_out), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), err);
  else if (d == 128)
    prologue_kernel<128><<<grid, block, 0, s>>>(
        static_cast<const uint4*>(q), static_cast<const uint4*>(k), static_cast<const uint4*>(v), q_w, k_w, eps,
        turns, positions, L, Lmax, Hq, Hkv, static_cast<uint4*>(q_out), static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), err);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace dma
