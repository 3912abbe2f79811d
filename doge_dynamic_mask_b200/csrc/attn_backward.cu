// Backward of the prefill path with the kept-key selection held fixed
// (sm_100a, tcgen05 + TMA), and the backward of the dt chain.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码": step 3's closing
// paragraph says dt comes from the cached value states so that training learns
// end to end which history tokens to mask; step 4 gives the attention.  The top-k
// is a selection with no gradient: every row's kept set is held fixed and the
// gradient reaches dt through the kept keys' bias.  For L = sum(out * dout):
//   dP = dO V^T, D_i = dO_i . O_i, dS = P (dP - D), dQ = scale dS K,
//   dK = scale dS^T Q, dV = P^T dO, d_dt[g, j] = sum over heads and rows of dS[., j],
//   dt = exp(A softplus(x)), x = v_flat W:  dA = sum d_dt dt softplus(x),
//   dx = d_dt dt A sigmoid(x),  dW = v_flat^T dx,  dv_flat += dx W^T.
//
// Design.  attn_bwd_kernel: one CTA of four warps per (batch, kv group, 128-row
// tile, query head); thread r owns row r of the tile.  It walks the row tile's
// kept-key list (the forward's plan, 128 keys per tile) twice:
//   * pass 1 recomputes each row's softmax statistics (max and sum) from
//     S = Q K^T + bias on the tensor core, unless the forward pass handed
//     over each row's log-sum-exp;
//   * pass 2, per key tile: S = Q K^T and dP = dO V^T into TMEM; each thread
//     forms its row of P and dS = P (dP - D) in float32 and stores them as bf16
//     in shared memory (128-byte swizzle, [row][key]: the same bytes serve as
//     a K-major operand for dQ and as an MN-major operand, i.e. transposed, for
//     dK and dV); then dQ += dS K accumulates in TMEM across the whole list,
//     dV_t = P^T dO and dK_t = dS^T [Q | 1] land in the columns S and dP used.
//     The extra B block of ones turns one more column of the dK product into
//     the column sum of dS, the bias (d_dt) gradient of each key.  Thread r then
//     owns key r of the tile and adds its dK, dV and d_dt rows to float32
//     accumulators in global memory (keys are shared by many row tiles and by
//     the group's heads).
// dt_bwd_token_kernel (one warp per token) recomputes x = v_flat W, forms dx and
// the dA contribution, and writes dv = dV + dx W^T and dk, rounded to bf16;
// dt_bwd_weight_kernel reduces dW = v_flat^T dx over the tokens.
// Every mbarrier wait is bounded; a wait that gives up records an error.
#include <cuda.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kBwdThreads = 128;
constexpr float kLog2eB = 1.4426950408889634f;

template <int D>
struct BwdCfg {
  static constexpr int kSlabs = D / 64;
  static constexpr int kQBytes = kRowTile * D * 2;       // Q or dO tile
  static constexpr int kSlabBytes = kRowTile * 128;      // 128 rows x 64 bf16
  static constexpr int kKVBytes = kKeyTile * D * 2;
  static constexpr int kPBytes = kRowTile * kKeyTile * 2; // P, then dS: two 64-key chunks
  static constexpr int kStages = 1;
  static constexpr int kOnesBytes = 16 * kRowTile * 2;    // the d_dt operand: 16 x 128 rows, K-major
  static constexpr int kOffQ = 0;
  static constexpr int kOffDO = kOffQ + kQBytes;
  static constexpr int kOffK = kOffDO + kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffP = kOffV + kStages * kKVBytes;
  static constexpr int kOffOnes = kOffP + kPBytes;
  static constexpr int kOffMeta = kOffOnes + kOnesBytes;  // per stage: bias[128] f32, span[128] u32, key[128] i32
  static constexpr int kMetaBytes = 3 * kKeyTile * 4;
  static constexpr int kOffBar = kOffMeta + kStages * kMetaBytes;
  static constexpr int kSmemBytes = kOffBar + 128 + 1024;
  // TMEM: S, then dP, at [0, 128), then dK_t at [0, D) once dP is read;
  // dV_t = P^T dO at [128, 128 + D); dQ after it; d_dt (16 columns, of which
  // the first is used) in the free part of [0, 128) at d = 64, else after dQ
  static constexpr uint32_t kColDK = 0;
  static constexpr uint32_t kColDV = 128;
  static constexpr uint32_t kColDQ = 128 + D;
  static constexpr uint32_t kColDDT = D == 64 ? 64 : 128 + 2 * D;
  static constexpr uint32_t kTmemCols = D == 64 ? 256 : 512;
  static constexpr int kMinBlocks = D == 64 ? 2 : 1;     // d = 64: two CTAs share an SM (TMEM 2 x 256)
  static_assert(kColDQ + D <= kTmemCols && kColDDT + 16 <= kTmemCols, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(D != 64 || 2 * (kSmemBytes + 1024) <= 233472, "two CTAs per SM at d = 64");
};

__device__ __forceinline__ unsigned long long mul_f32x2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float ld_bf16(const uint16_t* p) { return __uint_as_float(static_cast<uint32_t>(*p) << 16); }

// TMA reduce-add of a shared-memory box into a 3-D float32 tensor map
// (bulk async-group completion)
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, const void* src, int c0, int c1, int c2) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(tmap)),
               "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// red.global.add on four consecutive floats (16-byte aligned)
__device__ __forceinline__ void red_add_v4(float* dst, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(kBwdThreads, BwdCfg<D>::kMinBlocks)
    attn_bwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
                    const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                    const __grid_constant__ CUtensorMap tmap_k3, const __grid_constant__ CUtensorMap tmap_v3,
                    const __grid_constant__ CUtensorMap tmap_dk, const __grid_constant__ CUtensorMap tmap_dv,
                    PrefillPlan plan, int B, int L, int Hq, int Hkv, float scale, const uint16_t* __restrict__ out,
                    const uint16_t* __restrict__ dout, const float* __restrict__ lse_in, uint16_t* __restrict__ dq,
                    float* __restrict__ dk32, float* __restrict__ dv32, float* __restrict__ ddt32, uint32_t* err) {
  using C = BwdCfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bar;             // Q and dO landed
  uint64_t* kv_full = bar + 1;        // [stages]
  uint64_t* mma_done = bar + 3;       // every MMA issued so far completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 4);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // work item: (b, g, t, head r of the group), the row tile slowest and the
  // last (heaviest: the longest causal list) first, so the long CTAs start in
  // the first waves and the light ones fill the end
  const int nrep = Hq / Hkv;
  int w = blockIdx.x;
  const int r_in_group = w % nrep;
  w /= nrep;
  const int g = w % Hkv;
  w /= Hkv;
  const int b = w % B;
  w /= B;
  const int t = plan.n_row_tiles - 1 - w;
  const int h = g * nrep + r_in_group;
  const size_t tile = (static_cast<size_t>(b) * Hkv + g) * plan.n_row_tiles + t;
  const int r0 = t * kRowTile;
  const int nrows = min(kRowTile, L - r0);
  const int row = tid;
  const bool row_valid = row < nrows;
  const int base_row = b * L;

  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sOnes = smem + C::kOffOnes;
  unsigned char* sDO = smem + C::kOffDO;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  unsigned char* sP = smem + C::kOffP;     // P, then dS, of the current key tile
  unsigned char* sMeta = smem + C::kOffMeta;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) mbar_init(kv_full + s, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_do);
  }
  // the d_dt operand, K-major over the tile's 128 rows: row n = 0 all ones,
  // rows 1..15 zero (the 128-byte swizzle only permutes the 16-byte units of
  // a row, and every unit of row 0 is alike), so column 0 of dS^T x it is the
  // column sum of dS
  {
    const int kc = tid >> 6, n = (tid >> 2) & 15, u0 = (tid & 3) * 2;   // 128 threads x 32 bytes
    const uint4 val = n == 0 ? make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u) : make_uint4(0u, 0u, 0u, 0u);
    unsigned char* rowp = sOnes + kc * 2048 + n * 128;
    *reinterpret_cast<uint4*>(rowp + u0 * 16) = val;
    *reinterpret_cast<uint4*>(rowp + (u0 + 1) * 16) = val;
    fence_proxy_async_smem();
  }
  if (warp == 0) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
  // everything above overlaps the previous kernel; the key lists and their
  // counts come from it (the selector)
  pdl_wait();
  const int2 cnt = plan.counts[tile];
  const int n_full = cnt.x;   // list entries below n_full are kept by every row of the tile
  const int n_total = cnt.y;
  const int n_kt = (n_total + kKeyTile - 1) / kKeyTile;

  // D_r = dO_r . O_r (float32, from the rows in global memory)
  float Dr = 0.0f;
  if (row_valid) {
    const uint16_t* orow = out + ((static_cast<size_t>(base_row) + r0 + row) * Hq + h) * D;
    const uint16_t* grow = dout + ((static_cast<size_t>(base_row) + r0 + row) * Hq + h) * D;
    for (int c = 0; c < D; c += 8) {
      const uint4 a = *reinterpret_cast<const uint4*>(orow + c);
      const uint4 bb = *reinterpret_cast<const uint4*>(grow + c);
      const uint32_t x[4] = {a.x, a.y, a.z, a.w}, y[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        Dr = fmaf(__uint_as_float(x[i] << 16), __uint_as_float(y[i] << 16), Dr);
        Dr = fmaf(__uint_as_float(x[i] & 0xFFFF0000u), __uint_as_float(y[i] & 0xFFFF0000u), Dr);
      }
    }
  }

  // producer helpers (thread 0): Q and dO tiles; the K (and V) rows of list tile j into stage s
  const int32_t* idx_t = plan.idx + tile * plan.cap;
  const int32_t* kbase_t = plan.kbase + tile * (plan.cap / kKeyTile);
  const float* bias_t = plan.bias + tile * plan.cap;
  const uint32_t* span_t = plan.span + tile * plan.cap;
  uint32_t phase_kv[2] = {0u, 0u};
  uint32_t phase_mma = 0;
  auto load_tile = [&](int j, int s, bool with_v) {
    // list metadata of the tile for every thread (bias, row span, key index)
    float* mb = reinterpret_cast<float*>(sMeta + s * C::kMetaBytes);
    uint32_t* ms = reinterpret_cast<uint32_t*>(mb + kKeyTile);
    int32_t* mk = reinterpret_cast<int32_t*>(ms + kKeyTile);
    const int e = j * kKeyTile + tid;
    mb[tid] = bias_t[e];
    ms[tid] = e < n_total ? span_t[e] : 0u;
    mk[tid] = idx_t[e];
    if (warp == 0) {
      const int kb0 = kbase_t[j];
      const uint32_t bytes = (with_v ? 2 : 1) * C::kKVBytes;
      if (lane == 0) mbar_arrive_expect_tx(kv_full + s, bytes);
      __syncwarp();
      if (kb0 >= 0) {
        if (lane == 0) {
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl) {
            tma_load_3d(sK + s * C::kKVBytes + sl * C::kSlabBytes, &tmap_k3, kv_full + s, sl * 64, g, base_row + kb0);
            if (with_v)
              tma_load_3d(sV + s * C::kKVBytes + sl * C::kSlabBytes, &tmap_v3, kv_full + s, sl * 64, g,
                          base_row + kb0);
          }
        }
      } else {
        int4 ix = *reinterpret_cast<const int4*>(idx_t + j * kKeyTile + lane * 4);
        ix.x = (base_row + ix.x) * Hkv + g;
        ix.y = (base_row + ix.y) * Hkv + g;
        ix.z = (base_row + ix.z) * Hkv + g;
        ix.w = (base_row + ix.w) * Hkv + g;
#pragma unroll
        for (int sl = 0; sl < C::kSlabs; ++sl) {
          tma_gather4(sK + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_k, kv_full + s, sl * 64, ix.x,
                      ix.y, ix.z, ix.w);
          if (with_v)
            tma_gather4(sV + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_v, kv_full + s, sl * 64, ix.x,
                        ix.y, ix.z, ix.w);
        }
      }
    }
  };

  bool ok = true;
  if (tid == 0) {
    mbar_arrive_expect_tx(q_full, 2 * C::kQBytes);
#pragma unroll
    for (int sl = 0; sl < C::kSlabs; ++sl) {
      tma_load_3d(sQ + sl * C::kSlabBytes, &tmap_q, q_full, sl * 64, h, base_row + r0);
      tma_load_3d(sDO + sl * C::kSlabBytes, &tmap_do, q_full, sl * 64, h, base_row + r0);
    }
  }
  ok = mbar_wait(q_full, 0, err, kDevErrTimeoutBase + 40);

  const uint32_t idesc_s = make_idesc_bf16(128, 128, false, false);          // S, dP
  const uint32_t idesc_dq = make_idesc_bf16(128, D, false, true);            // dS (K-major) x K (MN-major)
  const uint32_t idesc_dv = make_idesc_bf16(128, D, true, true);             // P^T (MN-major) x dO (MN-major)
  const uint32_t idesc_dk = make_idesc_bf16(128, D, true, true);            // dS^T x Q
  const uint32_t idesc_ddt = make_idesc_bf16(128, 16, true, false);         // dS^T x ones (K-major)
  const uint32_t q_lo = desc_lo(smem_u32(sQ), 16), do_lo = desc_lo(smem_u32(sDO), 16);
  const uint32_t qmn_lo = desc_lo(smem_u32(sQ), C::kSlabBytes);              // Q as an MN-major B
  const uint32_t domn_lo = desc_lo(smem_u32(sDO), C::kSlabBytes);
  const uint32_t ones_lo = desc_lo(smem_u32(sOnes), 16);
  const uint32_t ds_k_lo = desc_lo(smem_u32(sP), 16);                        // the buffer as a K-major A
  const uint32_t p_mn_lo = desc_lo(smem_u32(sP), 16384);                    // ... and as an MN-major A (transposed)

  // S = X K_s^T (X = Q or dO, K-major both) into TMEM column col
  auto issue_xkt = [&](uint32_t x_lo, uint32_t k_lo, uint32_t col) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t off = static_cast<uint32_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
      if (kk == 0) umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem + col, x_lo, k_lo, idesc_s);
      else umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem + col, x_lo + off, k_lo + off, idesc_s);
    }
  };
  auto wait_mma = [&]() -> bool {
    const bool r = mbar_wait(mma_done, phase_mma & 1, err, kDevErrTimeoutBase + 41);
    ++phase_mma;
    return r;
  };

  // ---- pass 1: row statistics (log2 units): m = max, l = sum 2^(x - m) ----------
  // (skipped when the forward pass handed over each row's log-sum-exp)
  float m = -INFINITY, l = 0.0f;
  int gs = 0;   // tiles loaded so far (both passes), for the ring phases
  const int n_kt1 = lse_in ? 0 : n_kt;
  if (ok && n_kt1 > 0) load_tile(0, 0, false);
  for (int j = 0; ok && j < n_kt1; ++j, ++gs) {
    const int s = gs % C::kStages;
    ok = mbar_wait(kv_full + s, phase_kv[s] & 1, err, kDevErrTimeoutBase + 42);
    phase_kv[s] ^= 1u;
    __syncthreads();   // the tile's metadata is visible to every thread
    // two stages: the other stage's tile (j - 1) is done, fetch tile j + 1 into it now
    if (C::kStages == 2 && j + 1 < n_kt1) load_tile(j + 1, (gs + 1) % C::kStages, false);
    if (ok && tid == 0) {
      tc_fence_after();
      issue_xkt(q_lo, desc_lo(smem_u32(sK + s * C::kKVBytes), 16), 0);
      umma_commit(mma_done);
    }
    ok = __syncthreads_and(ok && wait_mma());
    if (!ok) break;
    tc_fence_after();
    const float* mb = reinterpret_cast<const float*>(sMeta + s * C::kMetaBytes);
    const uint32_t* ms = reinterpret_cast<const uint32_t*>(mb + kKeyTile);
    float tmax = -INFINITY;
    float xs[128];
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t r[32];
      DMA_TMEM_LD32(tmem + lane_base + c0, r);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const uint32_t sp = ms[c0 + c];
        const bool kept = static_cast<uint32_t>(row - static_cast<int>(sp & 0xFFFFu)) < ((sp >> 16) - (sp & 0xFFFFu));
        const float x = kept ? (__uint_as_float(r[c]) * scale + mb[c0 + c]) * kLog2eB : -INFINITY;
        xs[c0 + c] = x;
        tmax = fmaxf(tmax, x);
      }
    }
    const float m_new = fmaxf(m, tmax);
    if (m_new != -INFINITY) {
      float sum = 0.0f;
#pragma unroll
      for (int c = 0; c < 128; ++c) sum += exp2f(xs[c] - m_new);
      l = l * exp2f(m - m_new) + sum;
      m = m_new;
    }
    tc_fence_before();
    __syncthreads();   // S read by all before the next tile's MMA overwrites it
    if (C::kStages == 1 && j + 1 < n_kt1) load_tile(j + 1, (gs + 1) % C::kStages, false);
  }
  const float lse = lse_in ? (row_valid ? lse_in[(static_cast<size_t>(b) * Hq + h) * L + r0 + row] : 0.0f)
                           : ((m == -INFINITY) ? 0.0f : m + log2f(l));

  // ---- pass 2: gradients ------------------------------------------------------
  // per key tile: S = Q K^T; P (float32, kept in registers) stored as bf16;
  // dP = dO V^T into the same TMEM columns with dV_t = P^T dO beside them;
  // dS = P (dP - D) over P in shared memory; then dQ += dS K, dK_t = dS^T Q
  // and d_dt = dS^T 1; thread r adds key r's dV, dK and d_dt to the
  // accumulators
  if (ok && n_kt > 0) load_tile(0, gs % C::kStages, true);
  for (int j = 0; ok && j < n_kt; ++j, ++gs) {
    const int s = gs % C::kStages;
    ok = mbar_wait(kv_full + s, phase_kv[s] & 1, err, kDevErrTimeoutBase + 43);
    phase_kv[s] ^= 1u;
    __syncthreads();
    const uint32_t k_lo = desc_lo(smem_u32(sK + s * C::kKVBytes), 16);
    const uint32_t v_lo = desc_lo(smem_u32(sV + s * C::kKVBytes), 16);
    if (ok && tid == 0) {
      tc_fence_after();
      issue_xkt(q_lo, k_lo, 0);              // S
      umma_commit(mma_done);
      bulk_wait_read_all();   // the previous tile's staged dV / dK boxes have been read
    }
    ok = __syncthreads_and(ok && wait_mma());
    if (!ok) break;
    tc_fence_after();
    const float* mb = reinterpret_cast<const float*>(sMeta + s * C::kMetaBytes);
    const uint32_t* ms = reinterpret_cast<const uint32_t*>(mb + kKeyTile);
    // P of this row, 32 keys at a time, kept in float32 and stored as bf16
    // [row][key] (128-byte swizzle): keys c0 .. c0+31 are chunk c0 / 64, 16-byte units u0 .. u0+3
    float pr[128];
    auto store_row = [&](int c0, const uint32_t (&pk)[16]) {
      const int kc = c0 / 64, u0 = (c0 % 64) / 8;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t off = kc * 16384 + row * 128 + ((((u0 + u) ^ (row & 7))) << 4);
        *reinterpret_cast<uint4*>(sP + off) = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      }
    };
    // x = log2e (scale q.k + bias) - lse as one FMA per key: scale log2e is a
    // constant, log2e bias - lse comes from the key's bias; on a key tile kept
    // by every row the row intervals need no check (rows past the sequence
    // still get P = 0)
    const bool full_tile = (j + 1) * kKeyTile <= n_full;
    const float sl2e = scale * kLog2eB;
    const float4* mb4 = reinterpret_cast<const float4*>(mb);
    const uint4* ms4 = reinterpret_cast<const uint4*>(ms);
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t rs[32];
      DMA_TMEM_LD32(tmem + lane_base + c0, rs);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int c4 = 0; c4 < 8; ++c4) {
        const float4 bb = mb4[c0 / 4 + c4];
        const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
        uint32_t spv[4] = {0u, 0u, 0u, 0u};
        if (!full_tile) {
          const uint4 sp4 = ms4[c0 / 4 + c4];
          spv[0] = sp4.x; spv[1] = sp4.y; spv[2] = sp4.z; spv[3] = sp4.w;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = 4 * c4 + e;
          const bool kept = full_tile ? row_valid
                                      : static_cast<uint32_t>(row - static_cast<int>(spv[e] & 0xFFFFu)) <
                                            ((spv[e] >> 16) - (spv[e] & 0xFFFFu));
          const float x = fmaf(__uint_as_float(rs[c]), sl2e, fmaf(bv[e], kLog2eB, -lse));
          pr[c0 + c] = kept ? fast_exp2(x) : 0.0f;
        }
      }
#pragma unroll
      for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pr[c0 + 2 * c], pr[c0 + 2 * c + 1]);
      store_row(c0, pk);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      issue_xkt(do_lo, v_lo, 0);             // dP over S's columns
      // dV_t = P^T dO  (M = keys, K = rows: both operands MN-major)
#pragma unroll
      for (int kk = 0; kk < kRowTile / 16; ++kk) {
        const uint32_t step = static_cast<uint32_t>((kk * 2048) >> 4);
        if (kk == 0) umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem + C::kColDV, p_mn_lo, domn_lo, idesc_dv);
        else umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem + C::kColDV, p_mn_lo + step, domn_lo + step, idesc_dv);
      }
      umma_commit(mma_done);
    }
    ok = __syncthreads_and(ok && wait_mma());
    if (!ok) break;
    tc_fence_after();
    // dS = P (dP - D) over P in shared memory (dV_t, its reader, is done)
#pragma unroll
    for (int c0 = 0; c0 < 128; c0 += 32) {
      uint32_t rp[32];
      DMA_TMEM_LD32(tmem + lane_base + c0, rp);
      tmem_wait_ld();
      uint32_t dd[16];
      const unsigned long long dr2 = f32x2(Dr, Dr);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const unsigned long long ds2 =
            mul_f32x2(f32x2(pr[c0 + 2 * c], pr[c0 + 2 * c + 1]),
                      sub_f32x2(f32x2(__uint_as_float(rp[2 * c]), __uint_as_float(rp[2 * c + 1])), dr2));
        float d0, d1;
        f32x2_split(ds2, d0, d1);
        dd[c] = pack_bf16x2(d0, d1);
      }
      store_row(c0, dd);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      // dQ += dS K  (M = rows, N = D, K = keys; K is the MN-major B like V in the forward)
      const uint32_t kmn_lo = desc_lo(smem_u32(sK + s * C::kKVBytes), C::kSlabBytes);
#pragma unroll
      for (int kk = 0; kk < kKeyTile / 16; ++kk) {
        const uint32_t a = ds_k_lo + static_cast<uint32_t>(((kk / 4) * 16384 + (kk % 4) * 32) >> 4);
        const uint32_t bb = kmn_lo + static_cast<uint32_t>((kk * 2048) >> 4);
        if (kk == 0 && j == 0) umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem + C::kColDQ, a, bb, idesc_dq);
        else umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem + C::kColDQ, a, bb, idesc_dq);
      }
      // dK_t = dS^T Q and d_dt = dS^T 1  (M = keys, K = rows; dS^T is the MN-major view)
#pragma unroll
      for (int kk = 0; kk < kRowTile / 16; ++kk) {
        const uint32_t step = static_cast<uint32_t>((kk * 2048) >> 4);
        const uint32_t ostep = static_cast<uint32_t>(((kk / 4) * 2048 + (kk % 4) * 32) >> 4);
        if (kk == 0) {
          umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem + C::kColDK, p_mn_lo, qmn_lo, idesc_dk);
          umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem + C::kColDDT, p_mn_lo, ones_lo, idesc_ddt);
        } else {
          umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem + C::kColDK, p_mn_lo + step, qmn_lo + step, idesc_dk);
          umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem + C::kColDDT, p_mn_lo + step, ones_lo + ostep, idesc_ddt);
        }
      }
      umma_commit(mma_done);
    }
    ok = __syncthreads_and(ok && wait_mma());
    if (!ok) break;
    tc_fence_after();
    // thread = key of the tile: add its dV, dK and d_dt rows to the accumulators.
    // Every MMA of the tile is done, so the next tile's K, V and list metadata
    // can load now, under the reductions (each thread first takes its own key
    // index out of the metadata slot the load rewrites).
    {
      const int e = j * kKeyTile + tid;
      const int key = reinterpret_cast<const int32_t*>(ms + kKeyTile)[tid];
      const bool live = e < n_total;
      const size_t krow = (static_cast<size_t>(base_row) + key) * Hkv + g;
      if (j + 1 < n_kt) load_tile(j + 1, (gs + 1) % C::kStages, true);
      const int kb0 = kbase_t[j];
      if (kb0 >= 0) {
        // the tile's keys are the run kb0 .. kb0 + 127: 32 columns of dV, then
        // of dK, at a time (one box, 128-byte swizzle) are staged in one half
        // of the P/dS buffer (free now) and TMA adds them into the
        // accumulators; the halves alternate, so a box's read overlaps the
        // staging of the next.  Rows of list padding are zero (P = 0 there).
        constexpr int kRounds = 2 * (D / 32);
#pragma unroll 1
        for (int rnd = 0; rnd < kRounds; ++rnd) {
          const bool is_k = rnd >= D / 32;
          const int col0 = (rnd % (D / 32)) * 32;
          const float mul = is_k ? scale : 1.0f;
          unsigned char* buf = sP + (rnd & 1) * 16384;
          uint32_t r[32];
          DMA_TMEM_LD32(tmem + lane_base + (is_k ? C::kColDK : C::kColDV) + col0, r);
          tmem_wait_ld();
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint32_t off = row * 128 + ((ch ^ (row & 7)) << 4);
            *reinterpret_cast<float4*>(buf + off) =
                make_float4(__uint_as_float(r[4 * ch]) * mul, __uint_as_float(r[4 * ch + 1]) * mul,
                            __uint_as_float(r[4 * ch + 2]) * mul, __uint_as_float(r[4 * ch + 3]) * mul);
          }
          fence_proxy_async_smem();
          __syncthreads();
          if (tid == 0) {
            tma_reduce_add_3d(is_k ? &tmap_dk : &tmap_dv, buf, col0, g, base_row + kb0);
            bulk_commit();
            bulk_wait_read_1();   // the other half (the previous box) has been read
          }
          if (rnd + 1 < kRounds) __syncthreads();
        }
        // the last box is read before the next tile writes P (thread 0 waits there)
      } else {
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t rv[32], rk[32];
          DMA_TMEM_LD32(tmem + lane_base + C::kColDV + c0, rv);
          DMA_TMEM_LD32(tmem + lane_base + C::kColDK + c0, rk);
          tmem_wait_ld();
          if (live) {
#pragma unroll
            for (int c = 0; c < 32; c += 4) {
              red_add_v4(dv32 + krow * D + c0 + c, __uint_as_float(rv[c]), __uint_as_float(rv[c + 1]),
                         __uint_as_float(rv[c + 2]), __uint_as_float(rv[c + 3]));
              red_add_v4(dk32 + krow * D + c0 + c, __uint_as_float(rk[c]) * scale, __uint_as_float(rk[c + 1]) * scale,
                         __uint_as_float(rk[c + 2]) * scale, __uint_as_float(rk[c + 3]) * scale);
            }
          }
        }
      }
      uint32_t rb[16];
      DMA_TMEM_LD16(tmem + lane_base + C::kColDDT, rb);
      tmem_wait_ld();
      if (live) atomicAdd(ddt32 + (static_cast<size_t>(b) * Hkv + g) * L + key, __uint_as_float(rb[0]));
    }
    tc_fence_before();
    __syncthreads();   // TMEM and the P/dS buffer are free for the next tile
  }

  // dQ = scale * (dS K) summed over the list
  if (ok && n_kt > 0) {
    tc_fence_after();
    uint16_t* qrow = dq + ((static_cast<size_t>(base_row) + r0 + row) * Hq + h) * D;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t r[32];
      DMA_TMEM_LD32(tmem + lane_base + C::kColDQ + c0, r);
      tmem_wait_ld();
      if (row_valid) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c)
          pk[c] = pack_bf16x2(__uint_as_float(r[2 * c]) * scale, __uint_as_float(r[2 * c + 1]) * scale);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(qrow + c0 + c * 8) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
    }
  }
  if (tid == 0) bulk_wait_all();   // every TMA reduction has been applied
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, C::kTmemCols);
}

// ---- the dt chain, one warp per token ------------------------------------------------

constexpr int kDtBwdThreads = 256;

// x = v_flat . W[:, g] for every g, then dx, dA, and the token's dv and dk rows (bf16).
template <int HKV>
__global__ void __launch_bounds__(kDtBwdThreads)
    dt_bwd_token_kernel(const uint16_t* __restrict__ v, const float* __restrict__ W, const float* __restrict__ A,
                        const float* __restrict__ ddt32, const float* __restrict__ dk32, const float* __restrict__ dv32,
                        int B, int L, int d, float* __restrict__ dx_out, float* __restrict__ dA,
                        uint16_t* __restrict__ dk, uint16_t* __restrict__ dv) {
  const int C = HKV * d;
  const int lane = threadIdx.x & 31;
  const long long tok = static_cast<long long>(blockIdx.x) * (kDtBwdThreads / 32) + (threadIdx.x >> 5);
  const long long ntok = static_cast<long long>(B) * L;
  __shared__ float s_dA[HKV];
  if (threadIdx.x < HKV) s_dA[threadIdx.x] = 0.0f;
  __syncthreads();
  if (tok < ntok) {
    const long long bb = tok / L, j = tok - bb * L;
    const uint16_t* vrow = v + tok * C;
    float x[HKV];
#pragma unroll
    for (int gg = 0; gg < HKV; ++gg) x[gg] = 0.0f;
    for (int c = lane; c < C; c += 32) {
      const float vc = ld_bf16(vrow + c);
#pragma unroll
      for (int gg = 0; gg < HKV; ++gg) x[gg] = fmaf(vc, W[c * HKV + gg], x[gg]);
    }
    float dx[HKV];
#pragma unroll
    for (int gg = 0; gg < HKV; ++gg) {
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) x[gg] += __shfl_xor_sync(0xFFFFFFFFu, x[gg], o);
      const float sp = fmaxf(x[gg], 0.0f) + log1pf(expf(-fabsf(x[gg])));
      const float dtv = expf(A[gg] * sp);
      const float gdt = ddt32[(bb * HKV + gg) * L + j];
      const float sig = 1.0f / (1.0f + expf(-x[gg]));
      dx[gg] = gdt * dtv * A[gg] * sig;
      if (lane == 0) {
        dx_out[tok * HKV + gg] = dx[gg];
        atomicAdd(&s_dA[gg], gdt * dtv * sp);
      }
    }
    // dv = dV (attention) + dx W^T;  dk from its accumulator
    for (int c = lane; c < C; c += 32) {
      float acc = dv32[tok * C + c];
#pragma unroll
      for (int gg = 0; gg < HKV; ++gg) acc = fmaf(dx[gg], W[c * HKV + gg], acc);
      const __nv_bfloat16 bv = __float2bfloat16_rn(acc);
      const __nv_bfloat16 bk = __float2bfloat16_rn(dk32[tok * C + c]);
      dv[tok * C + c] = *reinterpret_cast<const uint16_t*>(&bv);
      dk[tok * C + c] = *reinterpret_cast<const uint16_t*>(&bk);
    }
  }
  __syncthreads();
  if (threadIdx.x < HKV) atomicAdd(dA + threadIdx.x, s_dA[threadIdx.x]);
}

// dW[c, g] = sum over tokens of v_flat[tok, c] dx[tok, g]: every thread owns
// channels, the CTA a range of tokens; one atomic per (channel, g) per CTA.
template <int HKV>
__global__ void __launch_bounds__(kDtBwdThreads)
    dt_bwd_weight_kernel(const uint16_t* __restrict__ v, const float* __restrict__ dx, long long ntok, int C,
                         int tok_per_cta, float* __restrict__ dW) {
  const long long t0 = static_cast<long long>(blockIdx.x) * tok_per_cta;
  const long long t1 = min(ntok, t0 + tok_per_cta);
  for (int c = threadIdx.x; c < C; c += kDtBwdThreads) {
    float acc[HKV];
#pragma unroll
    for (int gg = 0; gg < HKV; ++gg) acc[gg] = 0.0f;
    for (long long tk = t0; tk < t1; ++tk) {
      const float vc = ld_bf16(v + tk * C + c);
#pragma unroll
      for (int gg = 0; gg < HKV; ++gg) acc[gg] = fmaf(vc, dx[tk * HKV + gg], acc[gg]);
    }
#pragma unroll
    for (int gg = 0; gg < HKV; ++gg) atomicAdd(dW + c * HKV + gg, acc[gg]);
  }
}

template <int D>
cudaError_t launch_bwd_d(const void* q, const void* k, const void* v, const void* out, const void* dout,
                         const float* lse_in, const Geometry& g, float scale, const PrefillPlan& plan, void* dq,
                         float* dk32, float* dv32, float* ddt32, uint32_t* err, cudaStream_t s) {
  using C = BwdCfg<D>;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const uint64_t BL = static_cast<uint64_t>(g.B) * g.Lk;
  CUtensorMap tq, tdo, tk, tv, tk3, tv3;
  const void* qsrc[2] = {q, dout};
  CUtensorMap* qmaps[2] = {&tq, &tdo};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.Hq), BL};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(g.Hq) * D * 2};
    cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kRowTile)};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(qmaps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(qsrc[i]), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const void* kv[2] = {k, v};
  CUtensorMap* maps[2] = {&tk, &tv};
  CUtensorMap* maps3[2] = {&tk3, &tv3};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), BL * g.Hkv};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t es[2] = {1, 1};
    if (enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kv[i]), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    cuuint64_t dims3[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.Hkv), BL};
    cuuint64_t strides3[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(g.Hkv) * D * 2};
    cuuint32_t box3[3] = {64, 1, static_cast<cuuint32_t>(kKeyTile)};
    cuuint32_t es3[3] = {1, 1, 1};
    if (enc(maps3[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv[i]), dims3, strides3, box3, es3,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // the float32 accumulators [B*L, Hkv, d] as TMA reduce-add targets: boxes of
  // 32 columns x 128 consecutive keys of one kv head
  CUtensorMap tdk, tdv;
  float* acc[2] = {dk32, dv32};
  CUtensorMap* amaps[2] = {&tdk, &tdv};
  for (int i = 0; i < 2; ++i) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.Hkv), BL};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(g.Hkv) * D * 4};
    cuuint32_t box[3] = {32, 1, static_cast<cuuint32_t>(kKeyTile)};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(amaps[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, acc[i], dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(attn_bwd_kernel<D>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const long long n_cta = static_cast<long long>(plan.n_row_tiles) * g.B * g.Hq;
  if (n_cta > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  return launch_after(attn_bwd_kernel<D>, dim3(static_cast<unsigned>(n_cta)), dim3(kBwdThreads), C::kSmemBytes, s, tq,
                      tdo, tk, tv, tk3, tv3, tdk, tdv, plan, g.B, g.Lk, g.Hq, g.Hkv, scale, static_cast<const uint16_t*>(out),
                      static_cast<const uint16_t*>(dout), lse_in, static_cast<uint16_t*>(dq), dk32, dv32, ddt32, err);
}

}  // namespace

cudaError_t launch_attn_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                                 const float* lse_in, const Geometry& g, float scale, const PrefillPlan& plan,
                                 void* dq, float* dk32, float* dv32, float* ddt32, uint32_t* err, cudaStream_t s) {
  if (g.d == 64) return launch_bwd_d<64>(q, k, v, out, dout, lse_in, g, scale, plan, dq, dk32, dv32, ddt32, err, s);
  if (g.d == 128) return launch_bwd_d<128>(q, k, v, out, dout, lse_in, g, scale, plan, dq, dk32, dv32, ddt32, err, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_dt_backward(const void* v, const float* W, const float* A, const float* ddt32, const float* dk32,
                               const float* dv32, int B, int L, int Hkv, int d, float* dx, float* dW, float* dA,
                               void* dk, void* dv, cudaStream_t s) {
  const long long ntok = static_cast<long long>(B) * L;
  const int warps = kDtBwdThreads / 32;
  const long long grid = (ntok + warps - 1) / warps;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int C = Hkv * d;
  const long long nblk_w = 4LL * sm_count();
  const int tok_per_cta = static_cast<int>((ntok + nblk_w - 1) / nblk_w);
  const int grid_w = static_cast<int>((ntok + tok_per_cta - 1) / tok_per_cta);
#define DMA_DTB(H)                                                                                                 \
  if (Hkv == H) {                                                                                                  \
    dt_bwd_token_kernel<H><<<static_cast<unsigned>(grid), kDtBwdThreads, 0, s>>>(                                  \
        static_cast<const uint16_t*>(v), W, A, ddt32, dk32, dv32, B, L, d, dx, dA, static_cast<uint16_t*>(dk),    \
        static_cast<uint16_t*>(dv));                                                                               \
    cudaError_t e = cudaGetLastError();                                                                            \
    if (e != cudaSuccess) return e;                                                                                \
    dt_bwd_weight_kernel<H><<<grid_w, kDtBwdThreads, 0, s>>>(static_cast<const uint16_t*>(v), dx, ntok, C,        \
                                                              tok_per_cta, dW);                                    \
    return cudaGetLastError();                                                                                     \
  }
  DMA_DTB(1) DMA_DTB(2) DMA_DTB(4) DMA_DTB(8) DMA_DTB(16)
#undef DMA_DTB
  return cudaErrorInvalidValue;
}

}  // namespace dma
