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
//   * warp 0 (K producer): TMA loads the two Q tiles once; for every key tile
//     it fetches the 128 listed K rows into a ring of shared-memory stages
//     (128-byte swizzle): one box copy per 64-column slab when the listed keys
//     are one ascending run, else tile::gather4 (four listed rows per
//     instruction).  It also writes the tile's bias columns (below) and row
//     intervals.
//   * warp 2 (V producer): the same for V, on its own ring release, so a slow
//     V stage never holds back the next K tile.
//   * warp 1: allocates the 512 TMEM columns (S_0, S_1, O_0, O_1, and at
//     d = 64 also P_0, P_1) and, one thread, issues tcgen05.mma.  S_h = Q_h K^T (M=128, N=128, K=d) plus one
//     more K=16 step that adds the dt bias: Q gets three columns of ones and
//     each key row three columns holding dt/scale split into three bf16 terms
//     (hi + mid + lo reproduce the float32 value; products with 1 are exact and
//     the tensor core accumulates in float32), so S_h * scale = scale q.k + dt.
//     O_h += P_h V with A = P read from TMEM and B = V from shared memory.
//     At d = 64, P has its own TMEM columns: the softmax releases S as soon as
//     it has read it, so QK_h(j+1) runs during the softmax of tile j.  At
//     d = 128 P is written over S and the order per key tile is PV_0(j),
//     QK_0(j+1), PV_1(j), QK_1(j+1): while one head's softmax runs the tensor
//     core works for the other head.
//   * warps 3-6 / 7-10 (softmax, one thread per query row; four consecutive
//     warps cover the four TMEM lane quarters): read S from TMEM, mask rows
//     outside a key's row interval on the few tiles not kept by every row,
//     take the row max of the raw scores, and form p = 2^(S*scale*log2e - m)
//     with packed f32x2 arithmetic; P goes back over S in TMEM as bf16.  O is
//     rescaled only when the running max grew by more than 2^8 (exact: the
//     final division uses the same stale max).
//   * epilogue: O / l in float32, rounded to bf16.
// Every wait is bounded; a wait that gives up records an error and the CTA
// drains its in-flight copies and MMAs before it frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"

namespace dma {
namespace {

constexpr int kThreads = 352;   // 11 warps: K producer, MMA/TMEM, V producer, 2 x 4 softmax
// (registers come from each SM sub-partition's own file: with 11 warps three share one, so
// 168 per thread is the most one CTA per SM can have)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units
constexpr int kXBytes = kKeyTile * 32;       // 128 rows x 16 bf16 extra K columns (bias / ones)

template <int D>
struct Cfg {
  static constexpr int kStages = D == 128 ? 2 : 4;
  static constexpr int kSlabs = D / 64;                       // 128-byte swizzle atoms along d
  static constexpr int kQBytes = kRowTile * D * 2;            // one head's Q tile
  static constexpr int kKVBytes = kKeyTile * D * 2;           // one K (or V) stage
  static constexpr int kSlabBytes = kKeyTile * 128;           // 128 rows x 128 B
  static constexpr int kMetaSlots = 2 * kStages;
  static constexpr int kMetaBytes = kKeyTile * 4;             // span[128] u32
  static constexpr int kOffQ = 0;
  static constexpr int kOffQx = kOffQ + 2 * kQBytes;
  static constexpr int kOffK = kOffQx + 2 * kXBytes;
  static constexpr int kOffKx = kOffK + kStages * kKVBytes;
  static constexpr int kOffV = kOffKx + kStages * kXBytes;
  static constexpr int kOffMeta = kOffV + kStages * kKVBytes;
  static constexpr int kOffBar = kOffMeta + kMetaSlots * kMetaBytes;
  static constexpr int kNumBars = 1 + 4 * kStages + kMetaSlots + 8 + 1;
  // d = 64 leaves TMEM room for P in its own columns (S 2x128, O 2x64, P 2x64):
  // the softmax releases S as soon as it has read it, and the next S = Q K^T
  // overlaps the current softmax.  At d = 128 (O 2x128) P is written over S.
  static constexpr bool kSepP = D == 64;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;     // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  static_assert(2 * 128 + 2 * D <= 512, "TMEM budget");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

// Barriers.  K and V stages are released separately (a K stage is free as soon
// as both heads' S = Q K^T are done, long before the V stage).  The row-interval
// table of key tile j lives in meta slot j % (2 * stages) and is published by
// meta_full: the producer can only refill a slot after the softmax of the tile
// that used it two rounds earlier has finished, so a waiter is never more than
// one phase behind.
struct Bars {
  uint64_t* q_full;
  uint64_t* k_full;     // [stages]
  uint64_t* v_full;     // [stages]
  uint64_t* k_empty;    // [stages]
  uint64_t* v_empty;    // [stages]
  uint64_t* meta_full;  // [2 * stages]
  uint64_t* s_full;     // [2]
  uint64_t* s_free;     // [2] (separate-P layout only)
  uint64_t* p_ready;    // [2]
  uint64_t* o_done;     // [2]
  uint64_t* fin;
};

__device__ __forceinline__ bool aborted(volatile int* flag) { return *flag != 0; }

// byte offset of row r, 16-byte chunk c (0 or 1) in a no-swizzle K-major
// [128 rows x 16 bf16] block: 8-row x 16-byte core matrices, chunk halves 128 B
// apart, 8-row groups 256 B apart
__device__ __forceinline__ uint32_t xoff(int r, int c) { return (r >> 3) * 256 + c * 128 + (r & 7) * 16; }

__device__ __forceinline__ uint32_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&b));
}

// key row's bias columns: dt/scale as hi + mid + lo bf16 terms, then zeros
__device__ __forceinline__ uint4 bias_columns(float c) {
  const uint32_t hi = bf16_bits(c);
  const float r1 = c - __uint_as_float(hi << 16);
  const uint32_t mid = bf16_bits(r1);
  const float r2 = r1 - __uint_as_float(mid << 16);
  const uint32_t lo = bf16_bits(r2);
  return make_uint4(hi | (mid << 16), lo, 0u, 0u);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_k3,
                        const __grid_constant__ CUtensorMap tmap_v3, PrefillPlan plan, int B, int L, int Hq,
                        int Hkv, float scale_log2, float inv_scale, uint16_t* __restrict__ out, uint32_t* err) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  Bars bars;
  {
    uint64_t* p = bar;
    bars.q_full = p; p += 1;
    bars.k_full = p; p += C::kStages;
    bars.v_full = p; p += C::kStages;
    bars.k_empty = p; p += C::kStages;
    bars.v_empty = p; p += C::kStages;
    bars.meta_full = p; p += C::kMetaSlots;
    bars.s_full = p; p += 2;
    bars.s_free = p; p += 2;
    bars.p_ready = p; p += 2;
    bars.o_done = p; p += 2;
    bars.fin = p;
  }
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
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sQx = smem + C::kOffQx;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sKx = smem + C::kOffKx;
  unsigned char* sV = smem + C::kOffV;
  unsigned char* sMeta = smem + C::kOffMeta;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bars.k_full + s, 1);
      mbar_init(bars.v_full + s, 1);
      mbar_init(bars.k_empty + s, 1);
      mbar_init(bars.v_empty + s, 1);
    }
    for (int s = 0; s < C::kMetaSlots; ++s) mbar_init(bars.meta_full + s, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(bars.s_full + h, 1);
      mbar_init(bars.s_free + h, kRowTile);
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
  if (warp >= 3) {
    // constant parts of the extra K=16 block: Q's columns of ones, the zero
    // half of every key stage's bias block
    const int i = threadIdx.x - 96;    // 0..255
    const int r = i & 127;
    const int hq = i >> 7;
    *reinterpret_cast<uint4*>(sQx + hq * kXBytes + xoff(r, 0)) = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    *reinterpret_cast<uint4*>(sQx + hq * kXBytes + xoff(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
    for (int s = hq; s < C::kStages; s += 2)
      *reinterpret_cast<uint4*>(sKx + s * kXBytes + xoff(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
  }
  if (warp == 1) tmem_alloc(tmem_slot, C::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int32_t* idx_t = plan.idx + tile * plan.cap;
  const int32_t* kbase_t = plan.kbase + tile * (plan.cap / kKeyTile);
  const float* bias_t = plan.bias + tile * plan.cap;
  const uint32_t* span_t = plan.span + tile * plan.cap;
  const int base_row = b * L;

  if (warp == 0) {
    // ======================= K producer =====================================
    int issued = 0;
    if (lane == 0) mbar_arrive_expect_tx(bars.q_full, nh * C::kQBytes);
    __syncwarp();
    if (lane < nh * C::kSlabs) {
      const int h = lane / C::kSlabs, sl = lane % C::kSlabs;
      tma_load_3d(sQ + h * C::kQBytes + sl * C::kSlabBytes, &tmap_q, bars.q_full, sl * 64, h0 + h,
                  base_row + r0);
    }
    for (int j = 0; j < n_kt; ++j) {
      const int s = j % C::kStages;
      const int u = j / C::kStages;
      const int ms_slot = j % C::kMetaSlots;
      if (j >= C::kStages && !mbar_wait(bars.k_empty + s, (u - 1) & 1, err, kDevErrTimeoutBase + 1)) {
        *abort_flag = 1;
        break;
      }
      if (aborted(abort_flag)) break;
      const int e = j * kKeyTile + lane * 4;
      const int kb0 = kbase_t[j];
      {
        const float4 bi = *reinterpret_cast<const float4*>(bias_t + e);
        const uint4 sp = *reinterpret_cast<const uint4*>(span_t + e);
        *reinterpret_cast<uint4*>(sMeta + ms_slot * C::kMetaBytes + lane * 16) = sp;
        const float bv[4] = {bi.x, bi.y, bi.z, bi.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<uint4*>(sKx + s * kXBytes + xoff(lane * 4 + q, 0)) = bias_columns(bv[q] * inv_scale);
      }
      fence_proxy_async_smem();   // the bias block is read by the tensor core
      int4 ix = make_int4(0, 0, 0, 0);
      if (kb0 < 0) {
        ix = *reinterpret_cast<const int4*>(idx_t + e);
        ix.x = (base_row + ix.x) * Hkv + g;
        ix.y = (base_row + ix.y) * Hkv + g;
        ix.z = (base_row + ix.z) * Hkv + g;
        ix.w = (base_row + ix.w) * Hkv + g;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bars.meta_full + ms_slot);
        mbar_arrive_expect_tx(bars.k_full + s, C::kKVBytes);
      }
      __syncwarp();
      if (kb0 >= 0) {
        // one ascending run of keys: a 128-row box per 64-column slab
        if (lane == 0) {
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d(sK + s * C::kKVBytes + sl * C::kSlabBytes, &tmap_k3, bars.k_full + s, sl * 64, g,
                        base_row + kb0);
        }
      } else {
#pragma unroll
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_gather4(sK + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_k, bars.k_full + s, sl * 64,
                      ix.x, ix.y, ix.z, ix.w);
      }
      issued = j + 1;
    }
    // drain: every copy issued must have landed before the CTA can leave
    if (lane == 0) {
      mbar_wait(bars.q_full, 0, err, kDevErrTimeoutBase + 2);
      for (int j = issued - C::kStages < 0 ? 0 : issued - C::kStages; j < issued; ++j)
        mbar_wait(bars.k_full + j % C::kStages, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 3);
    }
  } else if (warp == 2) {
    // ======================= V producer =====================================
    int issued = 0;
    for (int j = 0; j < n_kt; ++j) {
      const int s = j % C::kStages;
      const int u = j / C::kStages;
      if (j >= C::kStages && !mbar_wait(bars.v_empty + s, (u - 1) & 1, err, kDevErrTimeoutBase + 14)) {
        *abort_flag = 1;
        break;
      }
      if (aborted(abort_flag)) break;
      const int kb0 = kbase_t[j];
      int4 ix = make_int4(0, 0, 0, 0);
      if (kb0 < 0) {
        ix = *reinterpret_cast<const int4*>(idx_t + j * kKeyTile + lane * 4);
        ix.x = (base_row + ix.x) * Hkv + g;
        ix.y = (base_row + ix.y) * Hkv + g;
        ix.z = (base_row + ix.z) * Hkv + g;
        ix.w = (base_row + ix.w) * Hkv + g;
      }
      if (lane == 0) mbar_arrive_expect_tx(bars.v_full + s, C::kKVBytes);
      __syncwarp();
      if (kb0 >= 0) {
        if (lane == 0) {
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_load_3d(sV + s * C::kKVBytes + sl * C::kSlabBytes, &tmap_v3, bars.v_full + s, sl * 64, g,
                        base_row + kb0);
        }
      } else {
#pragma unroll
        for (int sl = 0; sl < C::kSlabs; ++sl)
          tma_gather4(sV + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_v, bars.v_full + s, sl * 64,
                      ix.x, ix.y, ix.z, ix.w);
      }
      issued = j + 1;
    }
    if (lane == 0) {
      for (int j = issued - C::kStages < 0 ? 0 : issued - C::kStages; j < issued; ++j)
        mbar_wait(bars.v_full + j % C::kStages, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 3);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =====================================
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(128, 128, false, false);
      const uint32_t idesc_pv = make_idesc_bf16(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), qx_addr = smem_u32(sQx), k_addr = smem_u32(sK),
                     kx_addr = smem_u32(sKx), v_addr = smem_u32(sV);
      bool ok = mbar_wait_hot(bars.q_full, 0, err, kDevErrTimeoutBase + 4);
      // Descriptor bases, computed once: a stage, a head or a K step only moves
      // the 14-bit start-address field (16-byte units; shared memory < 256 KB),
      // so every MMA below costs a couple of integer adds to issue.
      const uint64_t qd0 = make_sw128_desc(q_addr, 16, 1024);
      const uint64_t kd0 = make_sw128_desc(k_addr, 16, 1024);
      const uint64_t vd0 = make_sw128_desc(v_addr, C::kSlabBytes, 1024);
      const uint64_t qxd0 = make_noswizzle_desc(qx_addr, 128, 256);
      const uint64_t kxd0 = make_noswizzle_desc(kx_addr, 128, 256);
      auto issue_qk = [&](int h, int s) {
        const uint64_t qa = qd0 + static_cast<uint64_t>(h * (C::kQBytes >> 4));
        const uint64_t kb = kd0 + static_cast<uint64_t>(s * (C::kKVBytes >> 4));
        const uint32_t dS = tmem + h * 128;
        umma_ss_c<0>(dS, qa, kb, idesc_qk);
#pragma unroll
        for (int kk = 1; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::kSlabBytes + (kk % 4) * 32) >> 4);
          umma_ss_c<1>(dS, qa + off, kb + off, idesc_qk);
        }
        // + dt/scale through the extra K=16 block (ones x bias columns)
        umma_ss_c<1>(dS, qxd0 + static_cast<uint64_t>(h * (kXBytes >> 4)),
                     kxd0 + static_cast<uint64_t>(s * (kXBytes >> 4)), idesc_qk);
        umma_commit(bars.s_full + h);
      };
      auto issue_pv = [&](int h, int s, bool first) {
        const uint64_t vb = vd0 + static_cast<uint64_t>(s * (C::kKVBytes >> 4));
        const uint32_t dO = tmem + 256 + h * D;
        const uint32_t tp = C::kSepP ? tmem + 384 + h * 64 : tmem + h * 128;
        if (first) umma_ts_c<0>(dO, tp, vb, idesc_pv); else umma_ts_c<1>(dO, tp, vb, idesc_pv);
#pragma unroll
        for (int kk = 1; kk < kKeyTile / 16; ++kk)
          umma_ts_c<1>(dO, tp + kk * 8, vb + static_cast<uint64_t>((kk * 2048) >> 4), idesc_pv);
        umma_commit(bars.o_done + h);
      };
      // Event-driven issue: poll every pending barrier and issue whichever MMA
      // is ready, so one head never waits on the other's progress (the tensor
      // core still executes in issue order).
      //   QK_h(j): needs K(j) landed and S_h free (separate P: S_h(j-1) read by
      //            the softmax; P over S: PV_h(j-1) issued before it)
      //   PV_h(j): needs P_h(j) written and V(j) landed
      // A K stage is released once both heads' QK of it are issued, a V stage
      // once both PVs are.
      int next_qk[2] = {0, 0}, next_pv[2] = {0, 0};
      long long t_last = clock64();   // last time an MMA was issued
      while (ok) {
        bool all_done = true, progressed = false;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (h >= nh) continue;
          const int jq = next_qk[h];
          if (jq < n_kt) {
            all_done = false;
            const bool s_ready = jq == 0 || (C::kSepP ? mbar_test(bars.s_free + h, (jq - 1) & 1)
                                                      : next_pv[h] >= jq);
            if (s_ready && mbar_test(bars.k_full + jq % C::kStages, (jq / C::kStages) & 1)) {
              tc_fence_after();
              issue_qk(h, jq % C::kStages);
              next_qk[h] = jq + 1;
              progressed = true;
              if (next_qk[0] >= jq + 1 && (nh < 2 || next_qk[1] >= jq + 1)) umma_commit(bars.k_empty + jq % C::kStages);
            }
          }
          const int jp = next_pv[h];
          if (jp < n_kt) {
            all_done = false;
            if (jp < next_qk[h] && mbar_test(bars.p_ready + h, jp & 1) &&
                mbar_test(bars.v_full + jp % C::kStages, (jp / C::kStages) & 1)) {
              tc_fence_after();
              issue_pv(h, jp % C::kStages, jp == 0);
              next_pv[h] = jp + 1;
              progressed = true;
              if (next_pv[0] >= jp + 1 && (nh < 2 || next_pv[1] >= jp + 1)) umma_commit(bars.v_empty + jp % C::kStages);
            }
          }
        }
        if (all_done) break;
        if (progressed) {
          t_last = clock64();
        } else {
          if (aborted(abort_flag) || clock64() - t_last > kWaitLimitCycles) {
            raise_error(err, kDevErrTimeoutBase + 16);
            ok = false;
          }
        }
      }
      if (!ok) *abort_flag = 1;
      // drain every MMA before TMEM is released
      umma_commit(bars.fin);
      mbar_wait_hot(bars.fin, 0, err, kDevErrTimeoutBase + 9);
    }
    __syncwarp();
  } else {
    // ======================= softmax / epilogue ============================
    const int h = (warp - 3) / 4;             // which head of the pair (warps 3-6, 7-10)
    const int row = (warp % 4) * 32 + lane;   // TMEM lane = query row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + h * 128;
    const uint32_t tO = tmem + lane_base + 256 + h * D;
    const bool row_valid = row < nrows;
    if (h < nh) {
      float m = -INFINITY, l = 0.0f;
      bool ok = true;
      const unsigned long long scale2 = f32x2(scale_log2, scale_log2);
      for (int j = 0; j < n_kt; ++j) {
        const int ms_slot = j % C::kMetaSlots;
        ok = mbar_wait(bars.s_full + h, j & 1, err, kDevErrTimeoutBase + 10);
        // the tile's row-interval table (published by the K producer)
        if (ok) ok = mbar_wait(bars.meta_full + ms_slot, (j / C::kMetaSlots) & 1, err, kDevErrTimeoutBase + 13);
        if (!ok || aborted(abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        uint32_t r[128];   // S row: scale * log2e * r = log2e * (scale q.k + dt)
        DMA_TMEM_LD32(tS + 0, (r + 0));
        DMA_TMEM_LD32(tS + 32, (r + 32));
        DMA_TMEM_LD32(tS + 64, (r + 64));
        DMA_TMEM_LD32(tS + 96, (r + 96));
        tmem_wait_ld();
        if constexpr (C::kSepP) {
          tc_fence_before();
          mbar_arrive(bars.s_free + h);   // S may be overwritten by the next Q K^T
        }
        if (!((j + 1) * kKeyTile <= n_full || !row_valid)) {
          // key tile not kept by every row: drop keys outside this row's interval
          const uint4* ms4 = reinterpret_cast<const uint4*>(sMeta + ms_slot * C::kMetaBytes);
#pragma unroll
          for (int c4 = 0; c4 < 32; ++c4) {
            const uint4 ss = ms4[c4];
            const uint32_t sv[4] = {ss.x, ss.y, ss.z, ss.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t sp = sv[e];
              const bool kept = static_cast<uint32_t>(row - static_cast<int>(sp & 0xFFFFu)) <
                                ((sp >> 16) - (sp & 0xFFFFu));
              if (!kept) r[4 * c4 + e] = __float_as_uint(-INFINITY);
            }
          }
        }
        // row max of the raw scores (scale > 0), four short chains
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 128; c += 8) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mx[k] = max3f(mx[k], __uint_as_float(r[c + 2 * k]), __uint_as_float(r[c + 2 * k + 1]));
        }
        const float tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale_log2;
        const float m_new = fmaxf(m, tmax);
        float alpha = 1.0f;
        if (m_new - m > kRescaleThreshold) {   // false while both are -inf
          alpha = fast_exp2(m - m_new);
          m = m_new;
          l *= alpha;
        }
        const float nm = m == -INFINITY ? 0.0f : -m;
        const unsigned long long nm2 = f32x2(nm, nm);
        if constexpr (C::kSepP) {
          // P's columns and O are free once PV of the previous tile is done
          if (j > 0) {
            ok = mbar_wait(bars.o_done + h, (j - 1) & 1, err, kDevErrTimeoutBase + 11);
            if (!ok) {
              *abort_flag = 1;
              break;
            }
            tc_fence_after();
          }
        }
        const uint32_t tP = C::kSepP ? tmem + lane_base + 384 + h * 64 : tS;
        unsigned long long sa = 0ull, sb = 0ull;   // two packed partial sums
        // P in two halves of 64 keys (32 packed columns each)
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            const int k = 64 * half + 2 * c;
            const unsigned long long x2 =
                fma_f32x2(f32x2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), scale2, nm2);
            float x0, x1;
            f32x2_split(x2, x0, x1);
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            if (c & 1) sb = add_f32x2(sb, f32x2(p0, p1)); else sa = add_f32x2(sa, f32x2(p0, p1));
            pk[c] = pack_bf16x2(p0, p1);
          }
          DMA_TMEM_ST32(tP + 32 * half, pk);
        }
        {
          float a0, a1, b0, b1;
          f32x2_split(sa, a0, a1);
          f32x2_split(sb, b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        if (j > 0) {
          // consume every o_done phase in order (PV of the previous tile), so
          // the parity of the epilogue's wait is never ambiguous
          if constexpr (!C::kSepP) ok = mbar_wait(bars.o_done + h, (j - 1) & 1, err, kDevErrTimeoutBase + 11);
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
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
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
      tq, tk, tv, tk3, tv3, plan, g.B, g.Lk, g.Hq, g.Hkv, scale * kLog2e, 1.0f / scale, static_cast<uint16_t*>(out),
      err);
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
