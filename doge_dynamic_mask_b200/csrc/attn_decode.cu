// S4 attention part: one query per (batch, query head) against its kept keys.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 4 (scores scaled by
// head_dim^-0.5 plus the additive mask, softmax in float32) applied to the
// decode query, whose mask is the top-keep_window_size of the cached keys.
//
// Design.  The work is a gather of w kept K and V rows per (batch, kv head)
// shared by the Hq/Hkv query heads of the group: pure HBM traffic with ~2 FLOP
// per byte, so the kernel is a bandwidth kernel on CUDA cores.  Split-K: one
// CTA per (batch, kv head, 128-key chunk of the kept list); each lane owns 8
// head dims (one 16-byte piece per row) and d/8 lanes cover a row.  The rows
// travel by cp.async into shared memory, K in one group and V in a second:
// all of a lane's row copies are in flight at once without holding
// registers, and the scores are computed while the V rows are still
// arriving.  Every lane reads back only the pieces it copied itself.  Each
// CTA writes an unnormalised partial (o, running max m in log2 units, sum l);
// a second kernel merges the splits of each query head.
#include "common.cuh"

namespace dma {
namespace {

constexpr int kDecThreads = 256;
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kKeysPerWarp = kDecodeChunk / kDecWarps;   // 16
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// dynamic shared memory of one decode CTA: the chunk's K and V rows
template <int D>
constexpr int dec_smem_bytes() { return 2 * kDecodeChunk * D * 2; }

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&x)[8]) {
  x[0] = __uint_as_float(u.x << 16);
  x[1] = __uint_as_float(u.x & 0xFFFF0000u);
  x[2] = __uint_as_float(u.y << 16);
  x[3] = __uint_as_float(u.y & 0xFFFF0000u);
  x[4] = __uint_as_float(u.z << 16);
  x[5] = __uint_as_float(u.z & 0xFFFF0000u);
  x[6] = __uint_as_float(u.w << 16);
  x[7] = __uint_as_float(u.w & 0xFFFF0000u);
}

template <int D, int NREP>
__global__ void __launch_bounds__(kDecThreads) decode_attn_kernel(const uint16_t* __restrict__ q,
                                                                   const uint16_t* __restrict__ kc,
                                                                   const uint16_t* __restrict__ vc, int Lk,
                                                                   int Hkv, float scale, DecodePlan plan) {
  constexpr int LPK = D / 8;              // lanes per key row
  constexpr int KPS = 32 / LPK;           // keys per warp step
  constexpr int STEPS = kKeysPerWarp / KPS;
  __shared__ float s_p[NREP][kDecodeChunk];
  __shared__ float s_red[kDecWarps][NREP][D];
  __shared__ float s_m[NREP], s_l[NREP];
  extern __shared__ uint4 dyn[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(dyn);   // [kDecodeChunk][D]
  uint16_t* sV = sK + kDecodeChunk * D;

  pdl_wait();      // the kept lists come from the previous kernel
  pdl_trigger();   // the combine may be scheduled
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int Hq = Hkv * NREP;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const int count = plan.count[bg];
  const int c0 = split * kDecodeChunk;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = lane / LPK;              // key slot within a step
  const int dl = (lane % LPK) * 8;        // first head dim owned by this lane
  const int32_t* idx = plan.idx + bg * plan.cap + c0;
  const float* bias = plan.bias + bg * plan.cap + c0;

  // query slices
  float qf[NREP][8];
#pragma unroll
  for (int r = 0; r < NREP; ++r) {
    const uint4 u = *reinterpret_cast<const uint4*>(q + (static_cast<size_t>(b) * Hq + g * NREP + r) * D + dl);
    bf16x8_to_f32(u, qf[r]);
  }

  // issue every K row copy of this lane, then every V row copy
  int key_local[STEPS];
  size_t rows[STEPS];
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    key_local[s] = warp * kKeysPerWarp + s * KPS + kg;
    // entries past the list's count are never read (key 0 stands in), so the
    // kernel does not depend on what the rest of the list buffer holds
    const int j = c0 + key_local[s] < count ? idx[key_local[s]] : 0;
    rows[s] = ((static_cast<size_t>(b) * Lk + j) * Hkv + g) * D + dl;
    cp_async16(sK + key_local[s] * D + dl, kc + rows[s]);
  }
  cp_async_commit();
#pragma unroll
  for (int s = 0; s < STEPS; ++s) cp_async16(sV + key_local[s] * D + dl, vc + rows[s]);
  cp_async_commit();
  cp_async_wait<1>();   // this lane's K pieces have landed

  // scores (log2 units)
  const float sl = scale * kLog2e;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    float kf[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(sK + key_local[s] * D + dl), kf);
    const bool valid = c0 + key_local[s] < count;
    const float bl = bias[key_local[s]] * kLog2e;
#pragma unroll
    for (int r = 0; r < NREP; ++r) {
      float acc = 0.0f;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = fmaf(qf[r][e], kf[e], acc);
#pragma unroll
      for (int o = LPK / 2; o >= 1; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
      if ((lane % LPK) == 0) s_p[r][key_local[s]] = valid ? fmaf(acc, sl, bl) : -INFINITY;
    }
  }
  __syncthreads();

  // per-head max, probabilities and sum over the chunk
  for (int r = warp; r < NREP; r += kDecWarps) {
    float m = -INFINITY;
    for (int i = lane; i < kDecodeChunk; i += 32) m = fmaxf(m, s_p[r][i]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    float l = 0.0f;
    for (int i = lane; i < kDecodeChunk; i += 32) {
      const float p = m == -INFINITY ? 0.0f : fast_exp2(s_p[r][i] - m);
      s_p[r][i] = p;
      l += p;
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xFFFFFFFFu, l, o);
    if (lane == 0) {
      s_m[r] = m;
      s_l[r] = l;
    }
  }
  __syncthreads();

  // P V
  cp_async_wait<0>();   // this lane's V pieces have landed
  float acc[NREP][8];
#pragma unroll
  for (int r = 0; r < NREP; ++r)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[r][e] = 0.0f;
#pragma unroll
  for (int s = 0; s < STEPS; ++s) {
    float vf[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(sV + key_local[s] * D + dl), vf);
#pragma unroll
    for (int r = 0; r < NREP; ++r) {
      const float p = s_p[r][key_local[s]];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(p, vf[e], acc[r][e]);
    }
  }
  // sum the KPS key slots of the warp (lanes with equal dims)
#pragma unroll
  for (int o = 16; o >= LPK; o >>= 1)
#pragma unroll
    for (int r = 0; r < NREP; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[r][e] += __shfl_xor_sync(0xFFFFFFFFu, acc[r][e], o);
  if (kg == 0) {
#pragma unroll
    for (int r = 0; r < NREP; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_red[warp][r][dl + e] = acc[r][e];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NREP * D; i += kDecThreads) {
    const int r = i / D, e = i % D;
    float o = 0.0f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) o += s_red[w][r][e];
    float* part = plan.part + ((static_cast<size_t>(b) * Hq + g * NREP + r) * plan.n_split + split) * (D + 2);
    part[e] = o;
    if (e == 0) {
      part[D] = s_m[r];
      part[D + 1] = s_l[r];
    }
  }
}

template <int D>
__global__ void decode_combine_kernel(DecodePlan plan, int Hq, uint16_t* __restrict__ out) {
  pdl_wait();      // the partials come from the previous kernel
  const int bh = blockIdx.x;
  const float* part = plan.part + static_cast<size_t>(bh) * plan.n_split * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < plan.n_split; ++s) M = fmaxf(M, part[s * (D + 2) + D]);
  float num = 0.0f, den = 0.0f;
  const int e = threadIdx.x;
  for (int s = 0; s < plan.n_split; ++s) {
    const float m = part[s * (D + 2) + D];
    if (m == -INFINITY) continue;
    const float wgt = fast_exp2(m - M);
    num = fmaf(wgt, part[s * (D + 2) + e], num);
    den = fmaf(wgt, part[s * (D + 2) + D + 1], den);
  }
  const __nv_bfloat16 y = __float2bfloat16_rn(num / den);
  out[static_cast<size_t>(bh) * D + e] = *reinterpret_cast<const uint16_t*>(&y);
}

template <int D, int NREP>
cudaError_t launch_dec(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                       const DecodePlan& plan, void* out, cudaStream_t s) {
  constexpr int smem = dec_smem_bytes<D>();
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(decode_attn_kernel<D, NREP>), smem);
  if (e != cudaSuccess) return e;
  dim3 grid(plan.n_split, g.Hkv, g.B);
  e = launch_after(decode_attn_kernel<D, NREP>, grid, dim3(kDecThreads), smem, s, static_cast<const uint16_t*>(q),
                   static_cast<const uint16_t*>(k), static_cast<const uint16_t*>(v), g.Lk, g.Hkv, scale, plan);
  if (e != cudaSuccess) return e;
  return launch_after(decode_combine_kernel<D>, dim3(g.B * g.Hq), dim3(D), 0, s, plan, g.Hq,
                      static_cast<uint16_t*>(out));
}

}  // namespace

cudaError_t launch_attn_decode(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                               const DecodePlan& plan, void* out, cudaStream_t s) {
  const int nrep = g.Hq / g.Hkv;
#define DMA_DEC_CASE(DD, NR) \
  if (g.d == DD && nrep == NR) return launch_dec<DD, NR>(q, k, v, g, scale, plan, out, s);
  DMA_DEC_CASE(64, 1) DMA_DEC_CASE(64, 2) DMA_DEC_CASE(64, 4) DMA_DEC_CASE(64, 8)
  DMA_DEC_CASE(128, 1) DMA_DEC_CASE(128, 2) DMA_DEC_CASE(128, 4) DMA_DEC_CASE(128, 8)
#undef DMA_DEC_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dma
