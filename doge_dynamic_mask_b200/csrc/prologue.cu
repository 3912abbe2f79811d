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
// Persistent CTAs (two per SM) walk the tokens.  A token's q, k and v rows are
// contiguous in each tensor, so one thread brings them into a ring of shared
// memory stages with three bulk copies per token; with the ring several
// tokens ahead, each SM keeps about 64 KB of reads in flight, which is what
// the HBM latency needs.  The d/2 angles of a position are formed in double
// precision (a position of 10^5 times a frequency near 1 would lose about
// 2^-7 rad of its angle in float32, the size of a bf16 rounding) as turns
// (pos times theta^(-2i/d) / (2 pi), the factors formed once per call by the
// launcher), reduced to their fractional part, and their cosines and sines
// taken in float32 (sincospi); they are formed one token ahead, while the
// current token's rows are processed.  Each group of d/8 threads owns one
// head row as sixteen-byte vectors (eight bf16 channels per thread): the mean
// square is a group shuffle reduction, and channel i's rotation partner
// i + d/2 sits in the thread d/16 positions away, one shuffle.  A thread's
// channels are the same for every row and token it handles, so its norm
// weights stay in registers.  Arithmetic is float32 with one rounding to bf16
// at the end; V rows are copied bit for bit.
#include <cuda_runtime.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kPrologueThreads = 256;
constexpr int kPrologueMaxStages = 2;
constexpr int kPrologueMinBlocks = 2;             // CTAs per SM (128 registers a thread)
constexpr int kPrologueMaxTokens = 16;            // tokens per stage
constexpr int kPrologueAngles = kPrologueMaxTokens * 64 / kPrologueThreads;   // angles per thread and stage, at most
constexpr int kPrologueStageBytes = 32 * 1024;   // rows of one ring stage (whole tokens)

__device__ __forceinline__ unsigned long long mul_f32x2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// two bf16 channels (one 32-bit word, low channel first) as packed float32
__device__ __forceinline__ unsigned long long widen_bf16x2(uint32_t w) {
  return f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from global to shared memory, completing on `bar` (complete-tx).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// theta^(-2i/d) / (2 pi) for i < d/2: each angle in turns is pos times one of
// these, formed once per call in double precision by the launcher
struct RopeTurns {
  double t[64];
};

// One ring stage holds the rows of `nts` consecutive tokens of the CTA's
// chunk: [q rows of those tokens][k rows][v rows], each region one bulk copy.
// Its angles (cosines, then sines, per token and pair index) and each token's
// cache row (-1 outside the cache) sit in one of two slots, formed while the
// previous stage is processed.
template <int D>
__global__ void __launch_bounds__(kPrologueThreads, kPrologueMinBlocks)
    prologue_kernel(const unsigned char* __restrict__ q, const unsigned char* __restrict__ k,
                    const unsigned char* __restrict__ v, const float* __restrict__ q_w,
                    const float* __restrict__ k_w, float eps, const __grid_constant__ RopeTurns turns,
                    const int32_t* __restrict__ positions, int L, int Lmax, int Hq, int Hkv, int ntok, int chunk,
                    int nts, int stages, uint4* __restrict__ q_out, uint4* __restrict__ k_cache,
                    uint4* __restrict__ v_cache, uint32_t* err) {
  constexpr int kLanesPerRow = D / 8;               // 16-byte vectors per head row
  constexpr int kHalf = kLanesPerRow / 2;           // lane distance of channel i's partner i + d/2
  static_assert(kPrologueThreads % kLanesPerRow == 0, "a thread keeps its channels");
  extern __shared__ __align__(128) unsigned char dyn[];
  __shared__ uint64_t full[kPrologueMaxStages];

  const uint32_t qbytes = static_cast<uint32_t>(Hq) * D * 2, kvbytes = static_cast<uint32_t>(Hkv) * D * 2;
  const size_t sbytes = static_cast<size_t>(nts) * (qbytes + 2 * kvbytes);   // one stage
  float* ang = reinterpret_cast<float*>(dyn + static_cast<size_t>(stages) * sbytes);   // [2][nts][2][D/2]
  int* crow_s = reinterpret_cast<int*>(ang + 2 * nts * D);                              // [2][nts]
  const int tid = threadIdx.x;
  const int sub = tid % kLanesPerRow;               // this thread's 8 channels: [8 sub, 8 sub + 8)
  const int t_begin = static_cast<int>(blockIdx.x) * chunk;
  const int t_end = min(ntok, t_begin + chunk);
  const int nst = t_end > t_begin ? (t_end - t_begin + nts - 1) / nts : 0;   // stages of this CTA

  if (tid == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(full + s, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // stage i of this CTA into ring slot s (thread 0)
  auto issue = [&](int i, int s) {
    const int t0 = t_begin + i * nts;
    const uint32_t n = static_cast<uint32_t>(min(nts, t_end - t0));
    unsigned char* st = dyn + static_cast<size_t>(s) * sbytes;
    mbar_arrive_expect_tx(full + s, n * (qbytes + 2 * kvbytes));
    bulk_load(st, q + static_cast<size_t>(t0) * qbytes, n * qbytes, full + s);
    bulk_load(st + n * qbytes, k + static_cast<size_t>(t0) * kvbytes, n * kvbytes, full + s);
    bulk_load(st + n * (qbytes + kvbytes), v + static_cast<size_t>(t0) * kvbytes, n * kvbytes, full + s);
  };
  int issued = nst < stages ? nst : stages;
  if (tid == 0)
    for (int i = 0; i < issued; ++i) issue(i, i);

  // angles of stage i's tokens into slot i & 1: the angle in turns
  // u = pos * theta^(-2i/d) / (2 pi) in double precision; its fractional part
  // r in [-1/2, 1/2] (exact in float32 to 2^-25) gives cos and sin of
  // 2 pi r = the angle modulo 2 pi, in float32.  The positions are read first
  // (pos_of), the angles formed later (angles), so the load's latency is hidden.
  auto pos_of = [&](int i, int (&pv)[kPrologueAngles]) {
#pragma unroll
    for (int m = 0; m < kPrologueAngles; ++m) pv[m] = 0;
    if (i >= nst) return;
    const int t0 = t_begin + i * nts;
    const int n = min(nts, t_end - t0);
#pragma unroll
    for (int m = 0; m < kPrologueAngles; ++m) {
      const int e = tid + m * kPrologueThreads;
      if (e < n * (D / 2)) {
        const int token = t0 + e / (D / 2);
        pv[m] = positions[token / L];
      }
    }
  };
  auto angles = [&](int i, const int (&pv)[kPrologueAngles]) {
    if (i >= nst) return;
    const int t0 = t_begin + i * nts;
    const int n = min(nts, t_end - t0);
    float* a = ang + (i & 1) * nts * D;
#pragma unroll
    for (int m = 0; m < kPrologueAngles; ++m) {
      const int e = tid + m * kPrologueThreads;
      if (e < n * (D / 2)) {
        const int j = e / (D / 2), c = e % (D / 2);
        const int token = t0 + j;
        const int b = token / L;
        const int pos0 = pv[m], pos = pos0 + (token - b * L);
        if (c == 0) {
          const bool in_cache = pos0 >= 0 && pos < Lmax;
          if (!in_cache) raise_error(err, kDevErrBadPosition);
          crow_s[(i & 1) * nts + j] = in_cache ? b * Lmax + pos : -1;
        }
        const double u = static_cast<double>(pos) * turns.t[c];
        const float r = static_cast<float>(u - rint(u));
        float sn, cs;
        sincospif(2.0f * r, &sn, &cs);
        a[j * D + c] = cs;
        a[j * D + D / 2 + c] = sn;
      }
    }
  };
  int pv[kPrologueAngles];
  pos_of(0, pv);
  angles(0, pv);
  const bool low = sub < kHalf;                     // channels below d/2
  const int i0 = 8 * (low ? sub : sub - kHalf);     // pair index of this thread's first channel
  const float inv_hq = 1.0f / static_cast<float>(Hq), inv_hkv = 1.0f / static_cast<float>(Hkv);
  // norm weights of this thread's channels and, with the rotation's sign
  // (the low half subtracts its partner's share), of its partner's channels
  const int psub = sub ^ kHalf;
  const float sg = low ? -1.0f : 1.0f;
  unsigned long long wq[4], wk[4], wpq[4], wpk[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    wq[c] = f32x2(q_w[8 * sub + 2 * c], q_w[8 * sub + 2 * c + 1]);
    wk[c] = f32x2(k_w[8 * sub + 2 * c], k_w[8 * sub + 2 * c + 1]);
    wpq[c] = f32x2(sg * q_w[8 * psub + 2 * c], sg * q_w[8 * psub + 2 * c + 1]);
    wpk[c] = f32x2(sg * k_w[8 * psub + 2 * c], sg * k_w[8 * psub + 2 * c + 1]);
  }

  int i = 0;
  for (; i < nst; ++i) {
    const int s = i % stages;
    const int t0 = t_begin + i * nts;
    const int n = min(nts, t_end - t0);
    pos_of(i + 1, pv);   // the next stage's positions, used after this stage's rows
    const bool ok = mbar_wait(full + s, static_cast<uint32_t>(i / stages) & 1u, err, kDevErrTimeoutBase + 50);
    if (__syncthreads_or(!ok)) break;   // also publishes this stage's angles
    const uint4* st = reinterpret_cast<const uint4*>(dyn + static_cast<size_t>(s) * sbytes);
    const float* a = ang + (i & 1) * nts * D;
    const int* crow_t = crow_s + (i & 1) * nts;
    const int nq = n * Hq * kLanesPerRow, nk = n * Hkv * kLanesPerRow;
    const int npieces = nq + 2 * nk;
    const int nsteps = (npieces + 2 * kPrologueThreads - 1) / (2 * kPrologueThreads);
    // two pieces per thread and step, kPrologueThreads apart: their chains
    // (load, partner shuffle, mean-square reduction, rotation, store) are
    // independent and overlap.  The shuffles run on every thread of the warp
    // (uniform trip count).
    for (int k2 = 0; k2 < nsteps; ++k2) {
      bool live[2];
      int kind[2], j[2], head[2], token[2];
      size_t crow[2];
      bool in_cache[2];
      uint4 u[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int piece = (2 * k2 + h) * kPrologueThreads + tid;   // in stage order: q rows, k rows, v rows
        live[h] = piece < npieces;
        kind[h] = piece < nq ? 0 : (piece < nq + nk ? 1 : 2);   // q, k or v
        const int pr = (kind[h] == 0 ? piece : (kind[h] == 1 ? piece - nq : piece - nq - nk)) / kLanesPerRow;
        const int hh = kind[h] == 0 ? Hq : Hkv;
        // token of the stage and head of the row: pr / hh through the float
        // reciprocal, exact here (pr < 2^12, hh <= 2^7: the quotient is at
        // least 1/(2 hh) from an integer, far above the rounding)
        j[h] = live[h] ? __float2int_rz((static_cast<float>(pr) + 0.5f) * (kind[h] == 0 ? inv_hq : inv_hkv)) : 0;
        head[h] = live[h] ? pr - j[h] * hh : 0;
        token[h] = t0 + j[h];
        const int cr = kind[h] == 0 ? 0 : crow_t[j[h]];
        in_cache[h] = cr >= 0;
        crow[h] = static_cast<size_t>(cr) * Hkv + head[h];
        u[h] = live[h] ? st[piece] : make_uint4(0u, 0u, 0u, 0u);
        if (live[h] && kind[h] == 2 && in_cache[h]) v_cache[crow[h] * kLanesPerRow + sub] = u[h];   // V: as is
      }
      if (__all_sync(0xFFFFFFFFu, (!live[0] || kind[0] == 2) && (!live[1] || kind[1] == 2))) continue;
      // the rotation partner's raw channels, d/16 threads away in the same row
      uint32_t pw[2][4];
      unsigned long long xv[2][4];
      float ss[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t uw[4] = {u[h].x, u[h].y, u[h].z, u[h].w};
        unsigned long long acc = 0ull;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          pw[h][c] = __shfl_xor_sync(0xFFFFFFFFu, uw[c], kHalf);
          xv[h][c] = widen_bf16x2(uw[c]);
          acc = fma_f32x2(xv[h][c], xv[h][c], acc);
        }
        float a0, a1;
        f32x2_split(acc, a0, a1);
        ss[h] = a0 + a1;
      }
#pragma unroll
      for (int o = kLanesPerRow / 2; o >= 1; o >>= 1) {
        ss[0] += __shfl_xor_sync(0xFFFFFFFFu, ss[0], o);
        ss[1] += __shfl_xor_sync(0xFFFFFFFFu, ss[1], o);
      }
      // out = inv (w x cos + w' x' sin): the row's norm factor, this channel's
      // weight and the partner's signed weight
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (!live[h] || kind[h] == 2) continue;
        const float inv = rsqrtf(ss[h] * (1.0f / D) + eps);
        const unsigned long long inv2 = f32x2(inv, inv);
        const float4* cp = reinterpret_cast<const float4*>(a + j[h] * D + i0);
        const float4* sp = reinterpret_cast<const float4*>(a + j[h] * D + D / 2 + i0);
        const float4 c0 = cp[0], c1 = cp[1], s0 = sp[0], s1 = sp[1];
        const unsigned long long cs2[4] = {f32x2(c0.x, c0.y), f32x2(c0.z, c0.w), f32x2(c1.x, c1.y), f32x2(c1.z, c1.w)};
        const unsigned long long sn2[4] = {f32x2(s0.x, s0.y), f32x2(s0.z, s0.w), f32x2(s1.x, s1.y), f32x2(s1.z, s1.w)};
        const bool isq = kind[h] == 0;
        uint32_t pk[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const unsigned long long y = mul_f32x2(xv[h][c], isq ? wq[c] : wk[c]);
          const unsigned long long yp = mul_f32x2(widen_bf16x2(pw[h][c]), isq ? wpq[c] : wpk[c]);
          const unsigned long long t = mul_f32x2(fma_f32x2(yp, sn2[c], mul_f32x2(y, cs2[c])), inv2);
          float lo, hi;
          f32x2_split(t, lo, hi);
          pk[c] = pack_bf16x2(lo, hi);
        }
        const uint4 o = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        if (isq) __stcs(q_out + (static_cast<size_t>(token[h]) * Hq + head[h]) * kLanesPerRow + sub, o);
        else if (in_cache[h]) k_cache[crow[h] * kLanesPerRow + sub] = o;
      }
    }
    angles(i + 1, pv);   // the next stage's, while the others finish this one
    __syncthreads();   // ring slot s has been read
    if (tid == 0 && issued < nst) {
      fence_proxy_async_smem();   // the reads above come before the copy's writes
      issue(issued, issued % stages);
      ++issued;
    }
  }
  // a wait that gave up: the copies still in flight land before the CTA exits
  if (tid == 0)
    for (int j = i; j < issued; ++j)
      mbar_wait(full + j % stages, static_cast<uint32_t>(j / stages) & 1u, err, kDevErrTimeoutBase + 51);
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
  const long long tbytes = static_cast<long long>(Hq + 2 * Hkv) * d * 2;   // one token's rows
  // tokens per stage: about 32 KB of rows (at most 16 tokens), two stages
  long long nts = kPrologueStageBytes / tbytes;
  nts = nts < 1 ? 1 : (nts > kPrologueMaxTokens ? kPrologueMaxTokens : nts);
  const int stages = kPrologueMaxStages;
  const long long smem = stages * nts * tbytes + 2LL * nts * d * 4 + 2LL * nts * 4;
  if (smem > 200 * 1024) return cudaErrorInvalidValue;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  // persistent: kPrologueMinBlocks CTAs per SM, each a contiguous chunk of tokens
  const long long nres = static_cast<long long>(kPrologueMinBlocks) * nsm;
  const long long nblocks = tokens < nres ? tokens : nres;
  const long long chunk = (tokens + nblocks - 1) / nblocks;
  const dim3 grid(static_cast<unsigned>(nblocks)), block(kPrologueThreads);
  const auto* qb = static_cast<const unsigned char*>(q);
  const auto* kb = static_cast<const unsigned char*>(k);
  const auto* vb = static_cast<const unsigned char*>(v);
  cudaError_t e;
  if (d == 64) {
    if ((e = ensure_dyn_smem(reinterpret_cast<const void*>(prologue_kernel<64>), static_cast<int>(smem))) != cudaSuccess) return e;
    prologue_kernel<64><<<grid, block, static_cast<size_t>(smem), s>>>(qb, kb, vb, q_w, k_w, eps, turns, positions, L, Lmax, Hq, Hkv,
                                                  static_cast<int>(tokens), static_cast<int>(chunk), static_cast<int>(nts), stages,
                                                  static_cast<uint4*>(q_out),
                                                  static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), err);
  } else {
    if ((e = ensure_dyn_smem(reinterpret_cast<const void*>(prologue_kernel<128>), static_cast<int>(smem))) != cudaSuccess) return e;
    prologue_kernel<128><<<grid, block, static_cast<size_t>(smem), s>>>(qb, kb, vb, q_w, k_w, eps, turns, positions, L, Lmax, Hq, Hkv,
                                                   static_cast<int>(tokens), static_cast<int>(chunk), static_cast<int>(nts), stages,
                                                  static_cast<uint4*>(q_out),
                                                   static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), err);
  }
  return cudaGetLastError();
}

}  // namespace dma
