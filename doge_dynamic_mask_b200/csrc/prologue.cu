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
// Persistent CTAs (two per SM) walk contiguous chunks of tokens, with eight
// compute warps and one copy warp each.  A token's q, k and v rows are
// contiguous in each tensor, so the copy warp brings a stage of tokens into a
// three-stage shared-memory ring with three bulk copies, and, once the
// compute warps report the stage done on an mbarrier, sends each token's rows
// out again with one bulk copy per tensor; a stage is refilled as soon as its
// stores have read it.  The compute warps never wait for the copies: they
// sync among themselves on a named barrier.  The d/2 angles of a position
// are formed in double precision (a position of 10^5 times a frequency near
// 1 would lose about 2^-7 rad of its angle in float32, the size of a bf16
// rounding) as turns (pos times theta^(-2i/d) / (2 pi), the factors formed
// once per call by the launcher), reduced to their fractional part, and
// their cosines and sines taken in float32 (sincospi); they are formed one
// stage ahead, while the current stage's rows are processed.  Two adjacent
// lanes own each q or k row of the stage and rewrite it in place, each
// taking every other 16-byte vector: one pass for the mean square (the two
// halves joined by one shuffle), one for the scaled rotation of channel
// pairs (i, i + d/2), both reading the vectors in an order rotated by the row
// index so that a warp's reads spread over all banks.  Arithmetic is float32
// (packed pairs) with one rounding to bf16 at the end; V rows are copied bit
// for bit.
#include <cuda_runtime.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kPrologueCompute = 256;                          // warps 0-7: the rows
constexpr int kPrologueThreads = kPrologueCompute + 32;        // warp 8: loads and stores
constexpr int kPrologueCrowSlots = 4;                          // cache-row slots (stage % 4)
constexpr int kPrologueStages = 3;
constexpr int kLanes = 2;                         // adjacent lanes sharing one row
constexpr int kPrologueMinBlocks = 2;             // CTAs per SM
constexpr int kPrologueMaxTokens = 16;            // tokens per stage
constexpr int kPrologueAngles = kPrologueMaxTokens * 64 / kPrologueCompute;   // angles per thread and stage, at most
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

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned)
// from shared to global memory (bulk async-group completion).
__device__ __forceinline__ void bulk_store(void* dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(reinterpret_cast<uint64_t>(dst)),
               "r"(smem_u32(src)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Named barrier 1 over the kPrologueCompute compute threads; true when any of
// them passed a true flag.
__device__ __forceinline__ bool compute_barrier_or(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(flag)), "n"(kPrologueCompute)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// theta^(-2i/d) / (2 pi) for i < d/2: each angle in turns is pos times one of
// these, formed once per call in double precision by the launcher
struct RopeTurns {
  double t[64];
};

// One ring stage holds the rows of `nts` consecutive tokens of the CTA's
// chunk: [q rows of those tokens][k rows][v rows], each region one bulk copy
// in.  Pairs of lanes of the compute warps normalise and rotate the q and k
// rows in place (a row per pair, read in an order rotated by the row index so
// that a warp's 16-byte reads spread over every bank); then the copy warp
// sends each token's q, k and v rows out with a bulk copy per tensor.  A
// stage's angles (cosines, then sines, per token and pair index) sit in one
// of two slots and each token's cache row (-1 outside the cache) in one of
// four, formed while the previous stage is processed; four cache-row slots
// keep the compute warps from overwriting a stage's cache-row entries before
// the copy warp has read them (it reads stage i's before it loads stage i + 3, and the
// compute warps write stage i + 4's only after that load has landed).
template <int D>
__global__ void __launch_bounds__(kPrologueThreads, kPrologueMinBlocks)
    prologue_kernel(const unsigned char* __restrict__ q, const unsigned char* __restrict__ k,
                    const unsigned char* __restrict__ v, const float* __restrict__ q_w,
                    const float* __restrict__ k_w, float eps, const __grid_constant__ RopeTurns turns,
                    const int32_t* __restrict__ positions, int L, int Lmax, int Hq, int Hkv, int ntok, int chunk,
                    int nts, unsigned char* __restrict__ q_out, unsigned char* __restrict__ k_cache,
                    unsigned char* __restrict__ v_cache, uint32_t* err) {
  constexpr int kChunks = D / 8;          // 16-byte chunks (eight channels) per row
  constexpr int kHalfC = kChunks / 2;     // chunk c pairs with chunk c + kHalfC (channel i with i + d/2)
  extern __shared__ __align__(128) unsigned char dyn[];
  __shared__ uint64_t full[kPrologueStages];   // a stage's rows have landed
  __shared__ uint64_t done[kPrologueStages];   // the compute warps have rewritten a stage's rows
  __shared__ int abort_flag;
  __shared__ __align__(16) float s_w[2][D];   // q_norm and k_norm weights

  const uint32_t qbytes = static_cast<uint32_t>(Hq) * D * 2, kvbytes = static_cast<uint32_t>(Hkv) * D * 2;
  const size_t sbytes = static_cast<size_t>(nts) * (qbytes + 2 * kvbytes);   // one stage
  float* ang = reinterpret_cast<float*>(dyn + static_cast<size_t>(kPrologueStages) * sbytes);   // [2][nts][2][D/2]
  int* crow_s = reinterpret_cast<int*>(ang + 2 * nts * D);                  // [kPrologueCrowSlots][nts]
  const int tid = threadIdx.x;
  const int t_begin = static_cast<int>(blockIdx.x) * chunk;
  const int t_end = min(ntok, t_begin + chunk);
  const int nst = t_end > t_begin ? (t_end - t_begin + nts - 1) / nts : 0;   // stages of this CTA

  if (tid == 0) {
    for (int s = 0; s < kPrologueStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(done + s, kPrologueCompute / 32);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  for (int c = tid; c < D; c += kPrologueThreads) {
    s_w[0][c] = q_w[c];
    s_w[1][c] = k_w[c];
  }
  __syncthreads();

  if (tid >= kPrologueCompute) {
    // ===== warp 8, lane 0: loads in, stores out =====
    if (tid != kPrologueCompute) return;
    // stage i of this CTA into ring slot s
    auto issue = [&](int i, int s) {
      const int t0 = t_begin + i * nts;
      const uint32_t n = static_cast<uint32_t>(min(nts, t_end - t0));
      unsigned char* st = dyn + static_cast<size_t>(s) * sbytes;
      mbar_arrive_expect_tx(full + s, n * (qbytes + 2 * kvbytes));
      bulk_load(st, q + static_cast<size_t>(t0) * qbytes, n * qbytes, full + s);
      bulk_load(st + n * qbytes, k + static_cast<size_t>(t0) * kvbytes, n * kvbytes, full + s);
      bulk_load(st + n * (qbytes + kvbytes), v + static_cast<size_t>(t0) * kvbytes, n * kvbytes, full + s);
    };
    const int first = nst < kPrologueStages ? nst : kPrologueStages;
    for (int i = 0; i < first; ++i) issue(i, i);
    int issued = first;
    for (int i = 0; i < nst; ++i) {
      // the slot of stage i - 1 takes stage i + 2 as soon as its stores have read it
      if (i >= 1 && issued < nst) {
        bulk_wait_read_0();
        fence_proxy_async_smem();
        issue(issued, issued % kPrologueStages);
        ++issued;
      }
      // stage i's rows rewritten by the compute warps (or the CTA gave up)
      const int s = i % kPrologueStages;
      const uint32_t par = static_cast<uint32_t>(i / kPrologueStages) & 1u;
      bool ok = mbar_try_wait(done + s, par);
      if (!ok) {
        const long long t0 = clock64();
        while (!(ok = mbar_try_wait_suspend(done + s, par, 20000u))) {
          if (*reinterpret_cast<volatile int*>(&abort_flag)) break;
          if (clock64() - t0 > kWaitLimitCycles) {
            raise_error(err, kDevErrTimeoutBase + 52);
            break;
          }
        }
      }
      if (!ok) break;
      // each token's rows out: q to q_out, k and v to its cache row
      const int t0 = t_begin + i * nts;
      const int n = min(nts, t_end - t0);
      const unsigned char* st = dyn + static_cast<size_t>(s) * sbytes;
      const int* crow_t = crow_s + (i % kPrologueCrowSlots) * nts;
      for (int jj = 0; jj < n; ++jj) {
        const int token = t0 + jj;
        bulk_store(q_out + static_cast<size_t>(token) * qbytes, st + static_cast<size_t>(jj) * qbytes, qbytes);
        const int cr = crow_t[jj];
        if (cr >= 0) {
          bulk_store(k_cache + static_cast<size_t>(cr) * kvbytes,
                     st + static_cast<size_t>(n) * qbytes + static_cast<size_t>(jj) * kvbytes, kvbytes);
          bulk_store(v_cache + static_cast<size_t>(cr) * kvbytes,
                     st + static_cast<size_t>(n) * (qbytes + kvbytes) + static_cast<size_t>(jj) * kvbytes, kvbytes);
        }
      }
      bulk_commit();
    }
    bulk_wait_all();   // every store has been applied before the CTA exits
    // the CTA gave up: loads still in flight (at most the last three issued,
    // one per slot, so each wait's parity is unambiguous) land first
    if (*reinterpret_cast<volatile int*>(&abort_flag)) {
      for (int j = issued > kPrologueStages ? issued - kPrologueStages : 0; j < issued; ++j)
        mbar_wait(full + j % kPrologueStages, static_cast<uint32_t>(j / kPrologueStages) & 1u, err,
                  kDevErrTimeoutBase + 51);
    }
    return;
  }

  // ===== warps 0-7: the rows =====
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
      const int e = tid + m * kPrologueCompute;
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
      const int e = tid + m * kPrologueCompute;
      if (e < n * (D / 2)) {
        const int j = e / (D / 2), c = e % (D / 2);
        const int token = t0 + j;
        const int b = token / L;
        const int pos0 = pv[m], pos = pos0 + (token - b * L);
        if (c == 0) {
          const bool in_cache = pos0 >= 0 && pos < Lmax;
          if (!in_cache) raise_error(err, kDevErrBadPosition);
          crow_s[(i % kPrologueCrowSlots) * nts + j] = in_cache ? b * Lmax + pos : -1;
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

  const int h = tid & (kLanes - 1);
  for (int i = 0; i < nst; ++i) {
    const int s = i % kPrologueStages;
    const int t0 = t_begin + i * nts;
    const int n = min(nts, t_end - t0);
    pos_of(i + 1, pv);   // the next stage's positions, used after this stage's rows
    const bool ok = mbar_wait(full + s, static_cast<uint32_t>(i / kPrologueStages) & 1u, err, kDevErrTimeoutBase + 50);
    // the compute warps only (named barrier 1): every one has its rows, and
    // this stage's angles (written by all of them) are visible
    if (compute_barrier_or(!ok)) {
      if (tid == 0) *reinterpret_cast<volatile int*>(&abort_flag) = 1;
      break;
    }
    unsigned char* st = dyn + static_cast<size_t>(s) * sbytes;
    const float* a = ang + (i & 1) * nts * D;
    const int nqr = n * Hq, nrows = n * (Hq + Hkv);   // q rows, then k rows (v rows pass through)
    // kLanes adjacent lanes per row: lane h takes chunks kLanes * v + h
    for (int base = 0; base < nrows; base += kPrologueCompute / kLanes) {
      const int r = base + tid / kLanes;
      const bool act = r < nrows;
      const unsigned mask = __ballot_sync(0xffffffffu, act);
      if (!act) continue;
      const bool is_q = r < nqr;
      const int j = is_q ? r / Hq : (r - nqr) / Hkv;   // token of the stage
      uint4* row = reinterpret_cast<uint4*>(st + static_cast<size_t>(r) * D * 2);
      const float* w = s_w[is_q ? 0 : 1];
      const float* cs = a + j * D;            // cos of pair index i at cs[i], sin at cs[D/2 + i]
      // mean square of the row: this lane's chunks 2v + h, v in an order
      // rotated by the row index, then the partner lane's share
      unsigned long long acc = 0ull;
#pragma unroll
      for (int c = 0; c < kChunks / kLanes; ++c) {
        const uint4 u = row[kLanes * ((c + r) % (kChunks / kLanes)) + h];
        acc = fma_f32x2(widen_bf16x2(u.x), widen_bf16x2(u.x), acc);
        acc = fma_f32x2(widen_bf16x2(u.y), widen_bf16x2(u.y), acc);
        acc = fma_f32x2(widen_bf16x2(u.z), widen_bf16x2(u.z), acc);
        acc = fma_f32x2(widen_bf16x2(u.w), widen_bf16x2(u.w), acc);
      }
      float a0, a1;
      f32x2_split(acc, a0, a1);
      float ss = a0 + a1;
#pragma unroll
      for (int o = 1; o < kLanes; o <<= 1) ss += __shfl_xor_sync(mask, ss, o);
      const float inv = rsqrtf(ss * (1.0f / D) + eps);
      const unsigned long long inv2 = f32x2(inv, inv);
      // the rotation of channel pairs (i, i + d/2), eight pairs per step:
      // this lane's low chunks 2v + h
#pragma unroll 2
      for (int c = 0; c < kHalfC / kLanes; ++c) {
        const int cl = kLanes * ((c + r) % (kHalfC / kLanes)) + h, ch = cl + kHalfC;
        // at d = 64 a row is 128 bytes, so rows r and r + 4 / kLanes would read the
        // same bank positions: one of them takes the high chunk first
        const bool swap = kHalfC < 8 && ((r / (4 / kLanes)) & 1);
        const uint4 u0 = row[swap ? ch : cl], u1 = row[swap ? cl : ch];
        const uint4 ul = swap ? u1 : u0, uh = swap ? u0 : u1;
        const uint32_t xl[4] = {ul.x, ul.y, ul.z, ul.w}, xh[4] = {uh.x, uh.y, uh.z, uh.w};
        const float4* wl4 = reinterpret_cast<const float4*>(w + 8 * cl);
        const float4* wh4 = reinterpret_cast<const float4*>(w + 8 * ch);
        const float4* c4 = reinterpret_cast<const float4*>(cs + 8 * cl);
        const float4* s4 = reinterpret_cast<const float4*>(cs + D / 2 + 8 * cl);
        const float4 wl0 = wl4[0], wl1 = wl4[1], wh0 = wh4[0], wh1 = wh4[1];
        const float4 c0 = c4[0], c1 = c4[1], s0 = s4[0], s1 = s4[1];
        const unsigned long long wlv[4] = {f32x2(wl0.x, wl0.y), f32x2(wl0.z, wl0.w), f32x2(wl1.x, wl1.y),
                                           f32x2(wl1.z, wl1.w)};
        const unsigned long long whv[4] = {f32x2(wh0.x, wh0.y), f32x2(wh0.z, wh0.w), f32x2(wh1.x, wh1.y),
                                           f32x2(wh1.z, wh1.w)};
        const unsigned long long cv[4] = {f32x2(c0.x, c0.y), f32x2(c0.z, c0.w), f32x2(c1.x, c1.y), f32x2(c1.z, c1.w)};
        const unsigned long long sv[4] = {f32x2(s0.x, s0.y), f32x2(s0.z, s0.w), f32x2(s1.x, s1.y), f32x2(s1.z, s1.w)};
        uint32_t ol[4], oh[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const unsigned long long yl = mul_f32x2(mul_f32x2(widen_bf16x2(xl[e]), wlv[e]), inv2);
          const unsigned long long yh = mul_f32x2(mul_f32x2(widen_bf16x2(xh[e]), whv[e]), inv2);
          // out_i = y_i cos - y_{i+d/2} sin,  out_{i+d/2} = y_{i+d/2} cos + y_i sin
          const unsigned long long lo = sub_f32x2(mul_f32x2(yl, cv[e]), mul_f32x2(yh, sv[e]));
          const unsigned long long hi = fma_f32x2(yl, sv[e], mul_f32x2(yh, cv[e]));
          float p0, p1;
          f32x2_split(lo, p0, p1);
          ol[e] = pack_bf16x2(p0, p1);
          f32x2_split(hi, p0, p1);
          oh[e] = pack_bf16x2(p0, p1);
        }
        const uint4 vl = make_uint4(ol[0], ol[1], ol[2], ol[3]), vh = make_uint4(oh[0], oh[1], oh[2], oh[3]);
        row[swap ? ch : cl] = swap ? vh : vl;
        row[swap ? cl : ch] = swap ? vl : vh;
      }
    }
    fence_proxy_async_smem();   // the rows written above are read by the bulk stores
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive(done + s);
    angles(i + 1, pv);   // the next stage's, while the store warp sends this one out
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
  const long long tbytes = static_cast<long long>(Hq + 2 * Hkv) * d * 2;   // one token's rows
  // tokens per stage: about 32 KB of rows (at most 16 tokens), three stages
  long long nts = kPrologueStageBytes / tbytes;
  nts = nts < 1 ? 1 : (nts > kPrologueMaxTokens ? kPrologueMaxTokens : nts);
  const long long smem = kPrologueStages * nts * tbytes + 2LL * nts * d * 4 + kPrologueCrowSlots * nts * 4LL;
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
                                                  static_cast<int>(tokens), static_cast<int>(chunk), static_cast<int>(nts),
                                                  static_cast<unsigned char*>(q_out),
                                                  static_cast<unsigned char*>(k_cache), static_cast<unsigned char*>(v_cache), err);
  } else {
    if ((e = ensure_dyn_smem(reinterpret_cast<const void*>(prologue_kernel<128>), static_cast<int>(smem))) != cudaSuccess) return e;
    prologue_kernel<128><<<grid, block, static_cast<size_t>(smem), s>>>(qb, kb, vb, q_w, k_w, eps, turns, positions, L, Lmax, Hq, Hkv,
                                                   static_cast<int>(tokens), static_cast<int>(chunk), static_cast<int>(nts),
                                                  static_cast<unsigned char*>(q_out),
                                                   static_cast<unsigned char*>(k_cache), static_cast<unsigned char*>(v_cache), err);
  }
  return cudaGetLastError();
}

}  // namespace dma
