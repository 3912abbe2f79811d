// S3: block-sparse GQA prefill attention with the dt bias (sm_100a, tcgen05 + TMA).
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 4: scores scaled by
// head_dim^-0.5 plus the additive dynamic mask (dt on kept keys, min_dtype
// elsewhere), softmax in float32, times V.
//
// Design.  One CTA per (row tile of 128 queries, pair of query heads of one kv
// group).  The selector's list for the row tile names the at most
// w + 127 keys any of its rows keeps; the kernel streams those keys in tiles of
// 128 and never touches a key the tile does not keep.
//   * warp 0 (producer): TMA loads the two Q tiles once, then for every key
//     tile fetches the 128 listed K rows and V rows into a ring of
//     shared-memory stages (128-byte swizzle): one box copy per 64-column slab
//     when the listed keys are one ascending run, else tile::gather4 (four
//     listed rows per instruction); it copies the tile's dt bias and row
//     intervals next to them.
//   * warp 1 (one thread): issues tcgen05.mma.  S_h = Q_h K^T (M=128, N=128,
//     K=d) into TMEM, and O_h += P_h V (A = P read from TMEM, B = V from shared
//     memory, N=d).  The two heads ping-pong: while one head's softmax runs the
//     tensor core works on the other head.
//   * warp 2 allocates and frees the 512 TMEM columns (S_0, S_1, O_0, O_1).
//   * warps 4-7 / 8-11 (softmax, one thread per query row): read S from TMEM,
//     add the dt bias, apply the row interval mask on tiles that are not kept
//     by every row, run the float32 online softmax in log2 units, write P as
//     bf16 over S in TMEM, and rescale O only when the running max grew by more
//     than 2^8 (exact: the final division uses the same stale max).
//   * epilogue: O / l in float32, rounded to bf16.
// Every wait is bounded; a wait that gives up records an error and the CTA
// drains its in-flight copies and MMAs before it frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kThreads = 384;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
template <int D>
struct Cfg {
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr int kSlabs = D / 64;                       // 128-byte swizzle atoms along d
  static constexpr int kQBytes = kRowTile * D * 2;            // one head's Q tile
  static constexpr int kKVBytes = kKeyTile * D * 2;           // one K (or V) stage
  static constexpr int kSlabBytes = kKeyTile * 128;           // 128 rows x 128 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kQBytes;
  static constexpr int kOffV = kOffK + kStages * kKVBytes;
  static constexpr int kOffMeta = kOffV + kStages * kKVBytes;
  static constexpr int kMetaBytes = kKeyTile * 8;             // bias[128] f32 + span[128] u32
  static constexpr int kOffBar = kOffMeta + kStages * kMetaBytes;
  static constexpr int kNumBars = 1 + 3 * kStages + 6 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;     // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static_assert(2 * 128 + 2 * D <= 512, "TMEM budget");
};

struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;
  uint64_t* v_full;
  uint64_t* kv_empty;
  uint64_t* s_full;    // [2]
  uint64_t* p_ready;   // [2]
  uint64_t* o_done;    // [2]
  uint64_t* fin;
};

__device__ __forceinline__ bool aborted(volatile int* flag) { return *flag != 0; }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_k3,
                        const __grid_constant__ CUtensorMap tmap_v3, PrefillPlan plan, int B, int L, int Hq,
                        int Hkv, float scale_log2, uint16_t* __restrict__ out, uint32_t* err) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  Bars bars{bar, bar + 1, bar + 1 + C::kStages, bar + 1 + 2 * C::kStages, bar + 1 + 3 * C::kStages,
            bar + 3 + 3 * C::kStages, bar + 5 + 3 * C::kStages, bar + 7 + 3 * C::kStages};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  // ---- work item: heavy row tiles first ------------------------------------
  const int n_rt = plan.n_row_tiles;
  const int nrep = Hq / Hkv;
  const int npairs = (nrep + 1) / 2;
  int id = blockIdx.x;
  const int pair = id % npairs;
  id /= npairs;
  const int g = id % Hkv;
  id /= Hkv;
  const int b = id % B;
  const int t = n_rt - 1 - id / B;
  const int nh = min(2, nrep - 2 * pair);            // query heads in this CTA
  const int h0 = g * nrep + 2 * pair;                // first query head
  const int r0 = t * kRowTile;
  const int nrows = min(kRowTile, L - r0);
  const size_t tile = (static_cast<size_t>(b) * Hkv + g) * n_rt + t;
  const int2 cnt = plan.counts[tile];
  const int n_full = cnt.x, n_total = cnt.y;
  const int n_kt = (n_total + kKeyTile - 1) / kKeyTile;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars.k_full + s, 1);
      mbar_init(bars.v_full + s, 1);
      mbar_init(bars.kv_empty + s, 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bars.s_full + h, 1);
      mbar_init(bars.p_ready + h, kRowTile);
      mbar_init(bars.o_done + h, 1);
    }
    mbar_init(bars.fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_q);
    prefetch_tmap(&tmap_k);
    prefetch_tmap(&tmap_v);
    prefetch_tmap(&tmap_k3);
    prefetch_tmap(&tmap_v3);
  }
  if (warp == 2) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sV = smem + C::kOffV;
  unsigned char* sMeta = smem + C::kOffMeta;

  if (warp == 0) {
    // ======================= producer =======================================
    int issued = 0;
    if (lane == 0) mbar_arrive_expect_tx(bars.q_full, nh * C::kQBytes);
    __syncwarp();
    if (lane < nh * C::kSlabs) {
      const int h = lane / C::kSlabs, sl = lane % C::kSlabs;
      tma_load_3d(sQ + h * C::kQBytes + sl * C::kSlabBytes, &tmap_q, bars.q_full, sl * 64, h0 + h,
                  b * L + r0);
    }
    const int32_t* idx_t = plan.idx + tile * plan.cap;
    const int32_t* kbase_t = plan.kbase + tile * (plan.cap / kKeyTile);
    const float* bias_t = plan.bias + tile * plan.cap;
    const uint32_t* span_t = plan.span + tile * plan.cap;
    for (int j = 0; j < n_kt; ++j) {
      const int s = j % C::kStages;
      const int u = j / C::kStages;
      if (j >= C::kStages) {
        if (!mbar_wait(bars.kv_empty + s, (u - 1) & 1, err, kDevErrTimeoutBase + 1)) {
          *abort_flag = 1;
          break;
        }
      }
      if (aborted(abort_flag)) break;
      const int e = j * kKeyTile + lane * 4;
      const int kb0 = kbase_t[j];
      const float4 bi = *reinterpret_cast<const float4*>(bias_t + e);
      const uint4 sp = *reinterpret_cast<const uint4*>(span_t + e);
      float* mb = reinterpret_cast<float*>(sMeta + s * C::kMetaBytes);
      uint32_t* ms = reinterpret_cast<uint32_t*>(sMeta + s * C::kMetaBytes + kKeyTile * 4);
      *reinterpret_cast<float4*>(mb + lane * 4) =
          make_float4(bi.x * kLog2e, bi.y * kLog2e, bi.z * kLog2e, bi.w * kLog2e);
      *reinterpret_cast<uint4*>(ms + lane * 4) = sp;
      const int base_row = b * L;
      __syncwarp();
      if (kb0 >= 0) {
        // one ascending run of keys: a 128-row box per 64-column slab
        if (lane == 0) {
          mbar_arrive_expect_tx(bars.k_full + s, C::kKVBytes);
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d(sK + s * C::kKVBytes + sl * C::kSlabBytes, &tmap_k3, bars.k_full + s, sl * 64, g,
                        base_row + kb0);
          mbar_arrive_expect_tx(bars.v_full + s, C::kKVBytes);
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d(sV + s * C::kKVBytes + sl * C::kSlabBytes, &tmap_v3, bars.v_full + s, sl * 64, g,
                        base_row + kb0);
        }
      } else {
        const int4 ix = *reinterpret_cast<const int4*>(idx_t + e);
        const int r_0 = (base_row + ix.x) * Hkv + g;
        const int r_1 = (base_row + ix.y) * Hkv + g;
        const int r_2 = (base_row + ix.z) * Hkv + g;
        const int r_3 = (base_row + ix.w) * Hkv + g;
        if (lane == 0) mbar_arrive_expect_tx(bars.k_full + s, C::kKVBytes);
        __syncwarp();
#pragma unroll
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_gather4(sK + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_k, bars.k_full + s, sl * 64,
                      r_0, r_1, r_2, r_3);
        if (lane == 0) mbar_arrive_expect_tx(bars.v_full + s, C::kKVBytes);
        __syncwarp();
#pragma unroll
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_gather4(sV + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_v, bars.v_full + s, sl * 64,
                      r_0, r_1, r_2, r_3);
      }
      issued = j + 1;
    }
    // drain: every copy issued must have landed before the CTA can leave
    if (lane == 0) {
      mbar_wait(bars.q_full, 0, err, kDevErrTimeoutBase + 2);
      for (int j = issued - C::kStages < 0 ? 0 : issued - C::kStages; j < issued; ++j) {
        const int s = j % C::kStages, u = j / C::kStages;
        mbar_wait(bars.k_full + s, u & 1, err, kDevErrTimeoutBase + 3);
        mbar_wait(bars.v_full + s, u & 1, err, kDevErrTimeoutBase + 3);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =====================================
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(128, 128, false, false);
      const uint32_t idesc_pv = make_idesc_bf16(128, D, false, true);
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = mbar_wait(bars.q_full, 0, err, kDevErrTimeoutBase + 4);
      auto issue_qk = [&](int h, int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kSlabBytes + (kk % 4) * 32;
          const uint64_t a = make_sw128_desc(q_addr + h * C::kQBytes + off, 16, 1024);
          const uint64_t bd = make_sw128_desc(k_addr + s * C::kKVBytes + off, 16, 1024);
          umma_ss(tS[h], a, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(bars.s_full + h);
      };
      auto issue_pv = [&](int h, int s, bool first) {
#pragma unroll
        for (int kk = 0; kk < kKeyTile / 16; ++kk) {
          const uint64_t bd = make_sw128_desc(v_addr + s * C::kKVBytes + kk * 2048, C::kSlabBytes, 1024);
          umma_ts(tO[h], tS[h] + kk * 8, bd, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(bars.o_done + h);
      };
      if (ok && n_kt > 0) {
        ok = mbar_wait(bars.k_full, 0, err, kDevErrTimeoutBase + 5);
        if (ok) {
          tc_fence_after();
          for (int h = 0; h < nh; ++h) issue_qk(h, 0);
        }
      }
      for (int j = 0; ok && j < n_kt; ++j) {
        const int s = j % C::kStages, u = j / C::kStages;
        const bool has_next = j + 1 < n_kt;
        const int s1 = (j + 1) % C::kStages, u1 = (j + 1) / C::kStages;
        ok = mbar_wait(bars.v_full + s, u & 1, err, kDevErrTimeoutBase + 6);
        if (ok && has_next) ok = mbar_wait(bars.k_full + s1, u1 & 1, err, kDevErrTimeoutBase + 7);
        for (int h = 0; ok && h < nh; ++h) {
          ok = mbar_wait(bars.p_ready + h, j & 1, err, kDevErrTimeoutBase + 8);
          if (!ok) break;
          tc_fence_after();
          issue_pv(h, s, j == 0);
          if (has_next) issue_qk(h, s1);
        }
        if (ok) umma_commit(bars.kv_empty + s);
        if (aborted(abort_flag)) ok = false;
      }
      if (!ok) *abort_flag = 1;
      // drain every MMA before TMEM is released
      umma_commit(bars.fin);
      mbar_wait(bars.fin, 0, err, kDevErrTimeoutBase + 9);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ======================= softmax / epilogue ============================
    const int h = (warp - 4) / 4;             // which head of the pair
    const int row = (warp % 4) * 32 + lane;   // TMEM lane = query row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + h * 128;
    const uint32_t tO = tmem + lane_base + 256 + h * D;
    const bool row_valid = row < nrows;
    if (h < nh) {
      float m = -INFINITY, l = 0.0f;
      bool ok = true;
      for (int j = 0; j < n_kt; ++j) {
        const int s = j % C::kStages;
        ok = mbar_wait(bars.s_full + h, j & 1, err, kDevErrTimeoutBase + 10);
        // the stage's bias/interval table was published with k_full (acquire it directly)
        if (ok) ok = mbar_wait(bars.k_full + s, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 13);
        if (!ok || aborted(abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        uint32_t r[128];
        DMA_TMEM_LD32(tS + 0, (r + 0));
        DMA_TMEM_LD32(tS + 32, (r + 32));
        DMA_TMEM_LD32(tS + 64, (r + 64));
        DMA_TMEM_LD32(tS + 96, (r + 96));
        tmem_wait_ld();
        // dt bias (log2 units) and row intervals of this key tile.  The table is
        // read 16 columns at a time, each group's address chained through the
        // previous group's result so the loads are not all hoisted (register
        // pressure: the whole S row is live here).
        const float4* mb4 = reinterpret_cast<const float4*>(sMeta + s * C::kMetaBytes);
        const uint4* ms4 = reinterpret_cast<const uint4*>(sMeta + s * C::kMetaBytes + kKeyTile * 4);
        const bool full = (j + 1) * kKeyTile <= n_full || !row_valid;
        float tmax = -INFINITY;
        if (full) {
#pragma unroll
          for (int g16 = 0; g16 < 8; ++g16) {
            const float4* gp = mb4 + g16 * 4;
            asm volatile("" : "+l"(gp) : "f"(tmax));
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 bb = gp[q4];
              const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = g16 * 16 + q4 * 4 + e;
                const float x = fmaf(__uint_as_float(r[c]), scale_log2, bv[e]);
                r[c] = __float_as_uint(x);
                tmax = fmaxf(tmax, x);
              }
            }
          }
        } else {
#pragma unroll
          for (int g16 = 0; g16 < 8; ++g16) {
            const float4* gp = mb4 + g16 * 4;
            const uint4* gs = ms4 + g16 * 4;
            asm volatile("" : "+l"(gp), "+l"(gs) : "f"(tmax));
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const float4 bb = gp[q4];
              const uint4 ss = gs[q4];
              const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
              const uint32_t sv[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = g16 * 16 + q4 * 4 + e;
                const uint32_t sp = sv[e];
                const bool kept = static_cast<uint32_t>(row - static_cast<int>(sp & 0xFFFFu)) <
                                  ((sp >> 16) - (sp & 0xFFFFu));
                const float x = kept ? fmaf(__uint_as_float(r[c]), scale_log2, bv[e]) : -INFINITY;
                r[c] = __float_as_uint(x);
                tmax = fmaxf(tmax, x);
              }
            }
          }
        }
        const float m_new = fmaxf(m, tmax);
        float alpha = 1.0f;
        if (m_new - m > kRescaleThreshold) {   // false while both are -inf
          alpha = fast_exp2(m - m_new);
          m = m_new;
          l *= alpha;
        }
        const float m_use = m == -INFINITY ? 0.0f : m;
        float rs = 0.0f;
        // P in two halves of 64 keys (32 packed columns each): fewer live registers
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const float p0 = fast_exp2(__uint_as_float(r[64 * half + 2 * c]) - m_use);
            const float p1 = fast_exp2(__uint_as_float(r[64 * half + 2 * c + 1]) - m_use);
            rs += p0 + p1;
            pk[c] = pack_bf16x2(p0, p1);
          }
          DMA_TMEM_ST32(tS + 32 * half, pk);
        }
        l += rs;
        if (j > 0) {
          // consume every o_done phase in order (PV of the previous tile), so
          // the parity of the epilogue's wait is never ambiguous
          ok = mbar_wait(bars.o_done + h, (j - 1) & 1, err, kDevErrTimeoutBase + 11);
          if (!ok) {
            *abort_flag = 1;
            tmem_wait_st();
            break;
          }
          // rescale O (only warps where some row's max moved far enough)
          if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
            tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < D; c0 += 32) {
              uint32_t o[32];
              DMA_TMEM_LD32(tO + c0, o);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
              DMA_TMEM_ST32(tO + c0, o);
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bars.p_ready + h);
      }
      // epilogue
      if (ok && !aborted(abort_flag) && n_kt > 0) {
        ok = mbar_wait(bars.o_done + h, (n_kt - 1) & 1, err, kDevErrTimeoutBase + 12);
        if (ok) {
          tc_fence_after();
          const float inv = 1.0f / l;
          uint16_t* orow = out + ((static_cast<size_t>(b) * L + r0 + row) * Hq + h0 + h) * D;
#pragma unroll
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            DMA_TMEM_LD32(tO + c0, o);
            tmem_wait_ld();
            if (row_valid) {
              uint32_t pk2[16];
#pragma unroll
              for (int c = 0; c < 16; ++c)
                pk2[c] = pack_bf16x2(__uint_as_float(o[2 * c]) * inv, __uint_as_float(o[2 * c + 1]) * inv);
#pragma unroll
              for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(orow + c0 + c * 8) =
                    make_uint4(pk2[4 * c], pk2[4 * c + 1], pk2[4 * c + 2], pk2[4 * c + 3]);
            }
          }
        } else {
          *abort_flag = 1;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, C::kTmemCols);
}

// ---- host: tensor maps -------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int D>
cudaError_t launch_d(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                     const PrefillPlan& plan, void* out, uint32_t* err, cudaStream_t s) {
  using C = Cfg<D>;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  const uint64_t BL = static_cast<uint64_t>(g.B) * g.Lk;
  CUtensorMap tq, tk, tv;
  {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.Hq), BL};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(g.Hq) * D * 2};
    cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kRowTile)};
    cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const void* kv[2] = {k, v};
  CUtensorMap* maps[2] = {&tk, &tv};
  CUtensorMap tk3, tv3;
  CUtensorMap* maps3[2] = {&tk3, &tv3};
  for (int i = 0; i < 2; ++i) {
    // rows (b, j, g) of [B*L*Hkv, d], fetched four listed rows at a time
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), BL * g.Hkv};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t es[2] = {1, 1};
    if (enc(maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kv[i]), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    // [B*L, Hkv, d]: 128 consecutive keys of one kv head per box
    cuuint64_t dims3[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(g.Hkv), BL};
    cuuint64_t strides3[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(g.Hkv) * D * 2};
    cuuint32_t box3[3] = {64, 1, static_cast<cuuint32_t>(kKeyTile)};
    cuuint32_t es3[3] = {1, 1, 1};
    if (enc(maps3[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(kv[i]), dims3, strides3, box3, es3,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int nrep = g.Hq / g.Hkv;
  const int npairs = (nrep + 1) / 2;
  const long long nblocks = static_cast<long long>(plan.n_row_tiles) * g.B * g.Hkv * npairs;
  attn_prefill_kernel<D><<<static_cast<unsigned>(nblocks), kThreads, C::kSmemBytes, s>>>(
      tq, tk, tv, tk3, tv3, plan, g.B, g.Lk, g.Hq, g.Hkv, scale * kLog2e, static_cast<uint16_t*>(out), err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_prefill(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                                const PrefillPlan& plan, void* out, uint32_t* err, cudaStream_t s) {
  if (g.d == 64) return launch_d<64>(q, k, v, g, scale, plan, out, err, s);
  if (g.d == 128) return launch_d<128>(q, k, v, g, scale, plan, out, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace dma
