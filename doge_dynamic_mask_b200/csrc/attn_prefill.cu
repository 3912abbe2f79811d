// S3: block-sparse GQA prefill attention with the dt bias (sm_100a, tcgen05 + TMA).
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 4: scores scaled by
// head_dim^-0.5 plus the additive dynamic mask (dt on kept keys, min_dtype
// elsewhere), softmax in float32, times V.
//
// Design.  A work item is a row tile of 128 queries and a pair of query heads
// of one kv group.  The selector's list for the row tile names the at most
// w + 127 keys any of its rows keeps (or, without top-k, the kernel derives
// the list itself: the keys up to the tile's last visible row); the kernel
// streams those keys in tiles of 128 and never touches a key the tile does
// not keep.  The kernel is persistent: one CTA per SM walks the work items,
// heaviest row tiles first (at d = 64 in a static snake order, at d = 128
// drawn from a global counter), and every role counts key tiles across items
// so rings and barrier phases carry on from item to item.
// 384 threads in three warpgroups:
//   * warp 0 (K producer): TMA loads the item's Q tiles (after the previous
//     item's last Q K^T, signalled by q_empty); for every key tile it fetches
//     the 128 listed K rows into a ring of shared-memory stages (128-byte
//     swizzle): one box copy per 64-column slab when the listed keys are one
//     ascending run, else tile::gather4 (four listed rows per instruction).
//     It also writes the tile's bias columns (below) and row intervals.
//   * warp 2 (V producer): the same for V, on its own ring release.
//   * warp 3 (gather helper, d = 128): a third of the four-row groups of
//     every gathered K and V tile, since one warp issues its copies one at a
//     time.
//   * warp 1: allocates the 512 TMEM columns and, one thread, issues
//     tcgen05.mma from 32-bit descriptor low words (the high words are
//     constants).  S_h = Q_h K^T (M=128, N=128, K=d) plus one more K=16 step
//     that adds the dt bias: Q gets three columns of ones and each key row
//     three columns holding dt/scale split into three bf16 terms (hi + mid +
//     lo reproduce the float32 value; products with 1 are exact and the tensor
//     core accumulates in float32), so S_h * scale = scale q.k + dt.
//     O_h += P_h V with A = P read from TMEM and B = V from shared memory.
//     d = 64 (S_0 S_1 O_0 O_1 P_0 P_1): the two heads run in lockstep with
//     interleaved MMAs; QK(j+1) is issued as soon as the softmax has read
//     S(j) and runs during the softmax of tile j.  d = 128 (P written over S):
//     fixed ping-pong order PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1), so the
//     tensor core works for one head while the other head's softmax runs.
//     Warpgroup 0 gives registers back (setmaxnreg.dec) to the softmax
//     warpgroups (setmaxnreg.inc).
//   * warpgroups 1 and 2 (softmax, one per head of the pair, one thread per
//     query row; four consecutive warps cover the four TMEM lane quarters):
//     read S from TMEM, mask rows outside a key's row interval on the few
//     tiles not kept by every row, take the row max of the raw scores, and form
//     p = 2^(S*scale*log2e - m) with packed f32x2 arithmetic (a fixed share of
//     the pairs by a cubic on the FMA pipe, the rest by the MUFU ex2); P goes
//     to TMEM as bf16.  O is rescaled only when the running max grew by more
//     than 2^8 (exact: the final division uses the same stale max).  After
//     the item's last tile they write O / l in float32, rounded to bf16, while
//     the next item's first Q K^T already runs.
// Every wait is bounded; a wait that gives up records an error and the CTA
// drains its in-flight copies and MMAs before it frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"

namespace dma {
namespace {

// 12 warps in three warpgroups: warpgroup 0 = K producer, MMA issuer (and TMEM
// owner), V producer and gather helper; warpgroups 1 and 2 = the softmax of the
// pair's two heads (four warps each, one per TMEM lane quarter).  The block is
// launched with at most 168 registers per thread; warpgroup 0 then gives
// registers back (setmaxnreg.dec) and the softmax warpgroups take them
// (setmaxnreg.inc), so the 128-column score row and its probabilities stay in
// registers.  128 x kRegsControl + 256 x kRegsSoftmax must not exceed what the
// block was launched with: the launcher checks it before every launch.
constexpr int kThreads = 384;
constexpr int kRegsControl = 88;
constexpr int kRegsSoftmax = 208;
static_assert(kRegsControl % 8 == 0 && kRegsSoftmax % 8 == 0, "setmaxnreg takes multiples of 8");
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;   // log2 units

constexpr int kXBytes = kKeyTile * 32;       // 128 rows x 16 bf16 extra K columns (bias / ones)
// A gathered K or V tile is 32 groups of four listed rows, one tile::gather4
// per group and 64-column slab.  A warp issues its lanes' copies one after
// another (about 70 cycles each), so at d = 128 the copies of a tile are split
// over three warps: the K and the V producer take groups [0, kGatherSplit) of
// their tensor, the helper warp the remaining groups of both (44 / 44 / 40
// copies per tile).
constexpr int kGatherSplit = 22;
// At d = 128 work items reach a CTA through a global counter (heaviest
// first), fetched by the K producer and handed to the other roles through a
// ring of kItemRing slots in shared memory.
constexpr int kItemRing = 8;

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
  static constexpr int kNumBars = 2 + 4 * kStages + kMetaSlots + 8 + 1 + 2 * kItemRing;
  // d = 64 leaves TMEM room for P in its own columns (S 2x128, O 2x64, P 2x64):
  // the softmax releases S as soon as it has read it, and the next S = Q K^T
  // overlaps the current softmax.  At d = 128 (O 2x128) P is written over S.
  static constexpr bool kSepP = D == 64;
  // every kPolyEvery-th pair of probabilities in a row is computed on the FMA
  // pipe (exp2_poly_x2), the rest on the MUFU: measured best at 1/5 for d = 64
  // (both heads' exponentials run at once) and 1/8 for d = 128
  static constexpr int kPolyEvery = D == 128 ? 8 : 5;
  // d = 128 splits its gathers over a third warp (kGatherSplit); at d = 64 a
  // tile is half as many copies and the split measured slower, so the K and
  // V producers issue all of theirs
  static constexpr bool kHelper = D == 128;
  // d = 128 draws its work items from a global counter (their costs vary with
  // the kept-key unions, ~14 items per CTA on long context); at d = 64 the
  // static order measured faster (fewer, more even items per CTA)
  static constexpr bool kDynamic = D == 128;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffRing = kOffMisc + 64;              // kItemRing work-item numbers
  static constexpr int kSmemBytes = kOffRing + kItemRing * 4 + 1024;   // + alignment slack
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
  uint64_t* q_empty;    // the CTA's Q tile may be refilled (all Q K^T of the item done)
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
  uint64_t* item_full;    // [kItemRing] the slot holds the next work item's number
  uint64_t* item_empty;   // [kItemRing] every other role has read the slot
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

// 2^x for two values at once on the FMA pipe, x <= 8 (the lazy rescale lets x
// exceed 0 by up to its threshold).  x = n + f with n = round(x) and f in
// [-1/2, 1/2]: 2^f comes from a cubic fitted to 2^f over that interval
// (relative error below 7.5e-5, far under the bf16 rounding P goes through
// next), and n is added straight into the exponent field.  Inputs are clamped
// at -126 so the exponent field never underflows (masked keys, x = -inf, give
// 2^-126 or less instead of 0: negligible next to the row maximum's weight 1).
// Used for a fixed share of each row's probabilities, so that the
// exponentials are split between this path and the MUFU ex2 unit.
__device__ __forceinline__ void exp2_poly_x2(float x0, float x1, float& p0, float& p1) {
  const unsigned long long xa = f32x2(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const unsigned long long magic = f32x2(12582912.0f, 12582912.0f);   // 1.5 * 2^23
  const unsigned long long t = add_f32x2(xa, magic);   // round(x) in the low mantissa bits
  const unsigned long long f = sub_f32x2(xa, sub_f32x2(t, magic));
  unsigned long long q = fma_f32x2(f, f32x2(0.0551716573536396f, 0.0551716573536396f),
                                   f32x2(0.2426111400127411f, 0.2426111400127411f));
  q = fma_f32x2(q, f, f32x2(0.6932609677314758f, 0.6932609677314758f));
  q = fma_f32x2(q, f, f32x2(0.9999280571937561f, 0.9999280571937561f));
  float q0, q1, t0, t1;
  f32x2_split(q, q0, q1);
  f32x2_split(t, t0, t1);
  p0 = __uint_as_float(__float_as_uint(q0) + (__float_as_uint(t0) << 23));
  p1 = __uint_as_float(__float_as_uint(q1) + (__float_as_uint(t1) << 23));
}

// Tensor-memory columns: S_h at h * 128, O_h at 256 + h * D and, at d = 64,
// P_h at 384 + h * 64 (otherwise P_h is written over S_h).
//
// S_h = Q_h K^T (+ dt/scale through the extra K=16 block) for the NH heads
// h0 .. h0+NH-1 from K stage descriptors k_lo / kx_lo.  With two heads their
// K steps alternate, so consecutive MMAs write different accumulators.
template <int D, int NH>
__device__ __forceinline__ void issue_qk(uint32_t tmem, int h0, uint32_t q_lo, uint32_t k_lo, uint32_t qx_lo,
                                         uint32_t kx_lo, uint32_t idesc) {
  constexpr uint32_t kQStep = (kRowTile * D * 2) >> 4;   // one head's Q tile, in 16-byte units
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = static_cast<uint32_t>(((kk / 4) * (kKeyTile * 128) + (kk % 4) * 32) >> 4);
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      const uint32_t h = static_cast<uint32_t>(h0 + i);
      if (kk == 0)
        umma_ss_w<0, kDescHiSw128, kDescHiSw128>(tmem + h * 128, q_lo + h * kQStep, k_lo, idesc);
      else
        umma_ss_w<1, kDescHiSw128, kDescHiSw128>(tmem + h * 128, q_lo + h * kQStep + off, k_lo + off, idesc);
    }
  }
#pragma unroll
  for (int i = 0; i < NH; ++i) {
    const uint32_t h = static_cast<uint32_t>(h0 + i);
    umma_ss_w<1, kDescHiPlain, kDescHiPlain>(tmem + h * 128, qx_lo + h * (kXBytes >> 4), kx_lo, idesc);
  }
}

// O_h += P_h V for the NH heads h0 .. h0+NH-1 from V stage descriptor v_lo, K
// steps alternating between heads.
template <int D, int NH, bool SEP_P>
__device__ __forceinline__ void issue_pv(uint32_t tmem, int h0, uint32_t v_lo, uint32_t idesc, bool first) {
#pragma unroll
  for (int kk = 0; kk < kKeyTile / 16; ++kk) {
#pragma unroll
    for (int i = 0; i < NH; ++i) {
      const uint32_t h = static_cast<uint32_t>(h0 + i);
      const uint32_t dO = tmem + 256 + h * D;
      const uint32_t tp = (SEP_P ? tmem + 384 + h * 64 : tmem + h * 128) + kk * 8;
      const uint32_t b = v_lo + static_cast<uint32_t>((kk * 2048) >> 4);
      if (kk == 0 && first) umma_ts_w<0, kDescHiSw128>(dO, tp, b, idesc);
      else umma_ts_w<1, kDescHiSw128>(dO, tp, b, idesc);
    }
  }
}

// Work item (heavy row tiles first): pair of query heads, kv head g, batch b, row tile t.
struct Item {
  int pair, g, b, t;
};
__device__ __forceinline__ Item decode_item(int w, int npairs, int Hkv, int B, int n_rt) {
  Item it;
  it.pair = w % npairs;
  w /= npairs;
  it.g = w % Hkv;
  w /= Hkv;
  it.b = w % B;
  it.t = n_rt - 1 - w / B;
  return it;
}

// The i-th work item of this CTA in the static order: rounds of gridDim.x
// items, taken forwards in even rounds and backwards in odd ones, so every CTA
// gets a similar mix of heavy and light row tiles.
__device__ __forceinline__ int item_of(int i) {
  const int P = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  return i * P + ((i & 1) ? P - 1 - c : c);
}

// Persistent kernel: one CTA per SM walks its share of the work items; every
// role counts key tiles across items, so barrier phases and ring slots carry on
// from one item to the next and the next item's Q, K, V and first S = Q K^T
// are in flight while the softmax warps finish the current item's output.
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_k3,
                        const __grid_constant__ CUtensorMap tmap_v3, PrefillPlan plan, int B, int L, int Hq,
                        int Hkv, float scale_log2, float inv_scale, uint16_t* __restrict__ out,
                        float* __restrict__ lse_out, uint32_t* err) {
  using C = Cfg<D>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                         ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  Bars bars;
  {
    uint64_t* p = bar;
    bars.q_full = p; p += 1;
    bars.q_empty = p; p += 1;
    bars.k_full = p; p += C::kStages;
    bars.v_full = p; p += C::kStages;
    bars.k_empty = p; p += C::kStages;
    bars.v_empty = p; p += C::kStages;
    bars.meta_full = p; p += C::kMetaSlots;
    bars.s_full = p; p += 2;
    bars.s_free = p; p += 2;
    bars.p_ready = p; p += 2;
    bars.o_done = p; p += 2;
    bars.fin = p; p += 1;
    bars.item_full = p; p += kItemRing;
    bars.item_empty = p;
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

  const int n_rt = plan.n_row_tiles;
  const int nrep = Hq / Hkv;
  const int npairs = (nrep + 1) / 2;
  const int n_items = n_rt * B * Hkv * npairs;
  // Softmax head slots taking part in the lockstep (separate-P) barriers: when
  // a pair has a single head (odd nrep), the other slot's warps still arrive
  // on them without doing any work, so their counts never change.
  const int hw = nrep >= 2 ? 2 : 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sQx = smem + C::kOffQx;
  unsigned char* sK = smem + C::kOffK;
  unsigned char* sKx = smem + C::kOffKx;
  unsigned char* sV = smem + C::kOffV;
  unsigned char* sMeta = smem + C::kOffMeta;

  if (threadIdx.x == 0) {
    mbar_init(bars.q_full, 1);
    mbar_init(bars.q_empty, 1);
    for (int s = 0; s < C::kStages; ++s) {
      // the producer's expect-tx arrival and the gather helper's arrival
      mbar_init(bars.k_full + s, C::kHelper ? 2 : 1);
      mbar_init(bars.v_full + s, C::kHelper ? 2 : 1);
      mbar_init(bars.k_empty + s, 1);
      mbar_init(bars.v_empty + s, 1);
    }
    for (int s = 0; s < C::kMetaSlots; ++s) mbar_init(bars.meta_full + s, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(bars.s_full + h, 1);
      // the lockstep (separate-P) layout uses index 0 for both heads; one
      // arrival per softmax warp (four per head)
      mbar_init(bars.s_free + h, C::kSepP ? hw * 4 : 4);
      mbar_init(bars.p_ready + h, C::kSepP ? hw * 4 : 4);
      mbar_init(bars.o_done + h, 1);
    }
    mbar_init(bars.fin, 1);
    for (int r = 0; r < kItemRing; ++r) {
      mbar_init(bars.item_full + r, 1);
      // V producer, MMA issuer, gather helper (d = 128) and the eight softmax warps
      mbar_init(bars.item_empty + r, 2 + (C::kHelper ? 1 : 0) + 8);
    }
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
  if (warp >= 4) {
    // constant parts of the extra K=16 block: Q's columns of ones, the zero
    // half of every key stage's bias block
    const int i = threadIdx.x - 128;    // 0..255
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
  // everything above overlaps the previous kernel's tail; dt, the lists and
  // their counts come from it
  pdl_wait();

  // work item i of this CTA: false when there is none left
  struct ItemInfo {
    Item it;
    int nh, n_kt, n_full, n_total;
    size_t tile;
  };
  // The i-th work item of this CTA.  d = 64: the static order (item_of).
  // d = 128: item 0 is blockIdx.x; later ones come
  // from the counter (offset by the grid), heaviest first, so CTAs that drew
  // light items take more.  The K producer fetches (one item ahead, so the
  // atomic's latency is hidden) and publishes each number in ring slot
  // i % kItemRing; the other roles wait for the slot, read it and release it.
  // The last CTA to finish resets the counter (the workspace starts zeroed).
  uint32_t* sched = err + kHdrItemWord;        // items handed out beyond the first wave
  uint32_t* sched_done = err + kHdrDoneWord;   // CTAs finished
  int* ring = reinterpret_cast<int*>(smem + C::kOffRing);
  int next_w = 0;                    // the K producer's prefetched number
  auto fetch_item = [&](int i) -> int {
    if constexpr (!C::kDynamic) return item_of(i);
    const int slot = i % kItemRing;
    const int lane_ = threadIdx.x & 31;
    if (warp == 0) {
      int wv = 0;
      if (lane_ == 0) {
        if (i == 0) {
          wv = static_cast<int>(blockIdx.x);
        } else {
          wv = next_w;
        }
        next_w = static_cast<int>(atomicAdd(sched, 1u)) + static_cast<int>(gridDim.x);
        if (i >= kItemRing &&
            !mbar_wait(bars.item_empty + slot, ((i / kItemRing) - 1) & 1, err, kDevErrTimeoutBase + 23)) {
          *abort_flag = 1;
          wv = n_items;   // stop
        }
        ring[slot] = wv;
        mbar_arrive(bars.item_full + slot);
      }
      return __shfl_sync(0xFFFFFFFFu, wv, 0);
    }
    int wv = n_items;   // stop on a wait that gives up
    if (mbar_wait(bars.item_full + slot, (i / kItemRing) & 1, err, kDevErrTimeoutBase + 24)) wv = ring[slot];
    else *abort_flag = 1;
    if (warp == 1) {
      mbar_arrive(bars.item_empty + slot);   // the issuing thread alone runs its loop
    } else {
      __syncwarp();
      if (lane_ == 0) mbar_arrive(bars.item_empty + slot);
    }
    return wv;
  };
  auto item_info = [&](int i, ItemInfo& x) -> bool {
    const int w = fetch_item(i);
    if (w >= n_items) return false;
    x.it = decode_item(w, npairs, Hkv, B, n_rt);
    x.nh = min(2, nrep - 2 * x.it.pair);
    x.tile = (static_cast<size_t>(x.it.b) * Hkv + x.it.g) * n_rt + x.it.t;
    int n_total;
    if (plan.no_topk) {
      // keys 0 .. q in order: q = the tile's last row, or the last valid key
      int len = plan.lengths ? plan.lengths[x.it.b] : L;
      if (len < 1 || len > L) {
        raise_error(err, kDevErrBadLength);
        len = len < 1 ? 1 : L;
      }
      const int r0 = x.it.t * kRowTile;
      const int q = min(r0 + min(kRowTile, L - r0) - 1, len - 1);
      x.n_full = min(r0, q) + 1;
      n_total = q + 1;
    } else {
      const int2 cnt = plan.counts[x.tile];
      x.n_full = cnt.x;
      n_total = cnt.y;
    }
    x.n_total = n_total;
    x.n_kt = (n_total + kKeyTile - 1) / kKeyTile;
    return true;
  };

  if (warp < 4) {
  // warpgroup 0 gives registers back to the softmax warpgroups
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  if (warp == 0) {
    // ======================= K producer =====================================
    int gk = 0, nq = 0;   // K tiles and Q tiles issued so far
    bool stop = false;
    ItemInfo x;
    for (int i = 0; !stop && item_info(i, x); ++i) {
      if (x.n_kt == 0) continue;
      const int g = x.it.g, base_row = x.it.b * L;
      const int h0 = g * nrep + 2 * x.it.pair;
      // Q: the previous item's Q K^T must be complete
      if (nq > 0 && !mbar_wait(bars.q_empty, (nq - 1) & 1, err, kDevErrTimeoutBase + 15)) {
        *abort_flag = 1;
        break;
      }
      if (aborted(abort_flag)) break;
      if (lane == 0) mbar_arrive_expect_tx(bars.q_full, x.nh * C::kQBytes);
      __syncwarp();
      if (lane < x.nh * C::kSlabs) {
        const int h = lane / C::kSlabs, sl = lane % C::kSlabs;
        tma_load_3d(sQ + h * C::kQBytes + sl * C::kSlabBytes, &tmap_q, bars.q_full, sl * 64, h0 + h,
                    base_row + x.it.t * kRowTile);
      }
      ++nq;
      const int32_t* idx_t = plan.idx + x.tile * plan.cap;
      const int32_t* kbase_t = plan.kbase + x.tile * (plan.cap / kKeyTile);
      const float* bias_t = plan.bias + x.tile * plan.cap;
      const uint32_t* span_t = plan.span + x.tile * plan.cap;
      const float* dt_row = plan.dt_src + (static_cast<size_t>(x.it.b) * Hkv + g) * L;
      // One tile's list metadata for this lane's four entries: bias, row
      // intervals, key indices and the tile's run start.  The loads of tile
      // j + 1 are issued before waiting for tile j + 1's stage, so their
      // latency overlaps that wait instead of following it.
      struct TileMeta {
        float bv[4];
        uint4 sp;
        int4 ix;
        int kb0;
      };
      auto fetch_meta = [&](int j) {
        TileMeta mt;
        const int e = j * kKeyTile + lane * 4;
        if (plan.no_topk) {
          // list entry e is key e; padding past the last visible key has span 0
          const int r0 = x.it.t * kRowTile, nrows = min(kRowTile, L - r0);
          uint32_t spv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int key = e + q;
            const bool live = key < x.n_total;
            mt.bv[q] = live ? dt_row[key] : 0.0f;
            spv[q] = live ? static_cast<uint32_t>(key > r0 ? key - r0 : 0) | (static_cast<uint32_t>(nrows) << 16) : 0u;
          }
          mt.sp = make_uint4(spv[0], spv[1], spv[2], spv[3]);
          mt.kb0 = j * kKeyTile;
          mt.ix = make_int4(0, 0, 0, 0);
        } else {
          const float4 bi = *reinterpret_cast<const float4*>(bias_t + e);
          mt.sp = *reinterpret_cast<const uint4*>(span_t + e);
          mt.bv[0] = bi.x; mt.bv[1] = bi.y; mt.bv[2] = bi.z; mt.bv[3] = bi.w;
          mt.kb0 = kbase_t[j];
          mt.ix = *reinterpret_cast<const int4*>(idx_t + e);
        }
        return mt;
      };
      TileMeta nxt = fetch_meta(0);
      for (int j = 0; j < x.n_kt; ++j, ++gk) {
        const TileMeta cur = nxt;
        if (j + 1 < x.n_kt) nxt = fetch_meta(j + 1);
        const int s = gk % C::kStages;
        const int u = gk / C::kStages;
        const int ms_slot = gk % C::kMetaSlots;
        if (gk >= C::kStages && !mbar_wait(bars.k_empty + s, (u - 1) & 1, err, kDevErrTimeoutBase + 1)) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        if (aborted(abort_flag)) {
          stop = true;
          break;
        }
        const int kb0 = cur.kb0;
        {
          const float* bv = cur.bv;
          const uint4 sp = cur.sp;
          *reinterpret_cast<uint4*>(sMeta + ms_slot * C::kMetaBytes + lane * 16) = sp;
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(sKx + s * kXBytes + xoff(lane * 4 + q, 0)) = bias_columns(bv[q] * inv_scale);
        }
        fence_proxy_async_smem();   // the bias block is read by the tensor core
        int4 ix = make_int4(0, 0, 0, 0);
        if (kb0 < 0) {
          ix = cur.ix;
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
        } else if (lane < (C::kHelper ? kGatherSplit : 32)) {
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_gather4(sK + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_k, bars.k_full + s, sl * 64,
                        ix.x, ix.y, ix.z, ix.w);
        }
      }
    }
    // drain: every copy issued must have landed before the CTA can leave
    if (lane == 0) {
      if (nq > 0) mbar_wait(bars.q_full, (nq - 1) & 1, err, kDevErrTimeoutBase + 2);
      for (int j = gk - C::kStages < 0 ? 0 : gk - C::kStages; j < gk; ++j)
        mbar_wait(bars.k_full + j % C::kStages, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 3);
    }
  } else if (warp == 2) {
    // ======================= V producer =====================================
    int gv = 0;
    bool stop = false;
    ItemInfo x;
    for (int i = 0; !stop && item_info(i, x); ++i) {
      const int g = x.it.g, base_row = x.it.b * L;
      const int32_t* idx_t = plan.idx + x.tile * plan.cap;
      const int32_t* kbase_t = plan.kbase + x.tile * (plan.cap / kKeyTile);
      // the next tile's run start and key indices are fetched one tile ahead
      auto fetch_kb = [&](int j) { return plan.no_topk ? j * kKeyTile : kbase_t[j]; };
      auto fetch_ix = [&](int j) {
        return plan.no_topk ? make_int4(0, 0, 0, 0) : *reinterpret_cast<const int4*>(idx_t + j * kKeyTile + lane * 4);
      };
      int nkb = x.n_kt > 0 ? fetch_kb(0) : 0;
      int4 nix = x.n_kt > 0 ? fetch_ix(0) : make_int4(0, 0, 0, 0);
      for (int j = 0; j < x.n_kt; ++j, ++gv) {
        const int kb0 = nkb;
        int4 ix = nix;
        if (j + 1 < x.n_kt) {
          nkb = fetch_kb(j + 1);
          nix = fetch_ix(j + 1);
        }
        const int s = gv % C::kStages;
        const int u = gv / C::kStages;
        if (gv >= C::kStages && !mbar_wait(bars.v_empty + s, (u - 1) & 1, err, kDevErrTimeoutBase + 14)) {
          *abort_flag = 1;
          stop = true;
          break;
        }
        if (aborted(abort_flag)) {
          stop = true;
          break;
        }
        if (kb0 < 0) {
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
        } else if (lane < (C::kHelper ? kGatherSplit : 32)) {
#pragma unroll
          for (int sl = 0; sl < C::kSlabs; ++sl)
            tma_gather4(sV + s * C::kKVBytes + sl * C::kSlabBytes + lane * 512, &tmap_v, bars.v_full + s, sl * 64,
                        ix.x, ix.y, ix.z, ix.w);
        }
      }
    }
    if (lane == 0) {
      for (int j = gv - C::kStages < 0 ? 0 : gv - C::kStages; j < gv; ++j)
        mbar_wait(bars.v_full + j % C::kStages, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 3);
    }
  } else if (warp == 3 && C::kHelper) {
    // ======================= K/V gather helper ==============================
    // Row groups [kGatherSplit, 32) of every gathered K and V tile.  It arrives
    // on every tile's full barriers (a run loaded as boxes included), so a
    // full phase needs it and it can never fall two phases behind on the
    // empty barriers it waits on.
    const int rg = kGatherSplit + lane;
    const bool active = rg < kKeyTile / 4;
    int gh = 0;
    bool stop = false;
    ItemInfo x;
    for (int i = 0; !stop && item_info(i, x); ++i) {
      const int g = x.it.g, base_row = x.it.b * L;
      const int32_t* idx_t = plan.idx + x.tile * plan.cap;
      const int32_t* kbase_t = plan.kbase + x.tile * (plan.cap / kKeyTile);
      auto fetch_kb = [&](int j) { return plan.no_topk ? j * kKeyTile : kbase_t[j]; };
      auto fetch_ix = [&](int j) {
        return plan.no_topk || !active ? make_int4(0, 0, 0, 0)
                                       : *reinterpret_cast<const int4*>(idx_t + j * kKeyTile + rg * 4);
      };
      int nkb = x.n_kt > 0 ? fetch_kb(0) : 0;
      int4 nix = x.n_kt > 0 ? fetch_ix(0) : make_int4(0, 0, 0, 0);
      for (int j = 0; !stop && j < x.n_kt; ++j, ++gh) {
        const int kb0 = nkb;
        int4 ix = nix;
        if (j + 1 < x.n_kt) {
          nkb = fetch_kb(j + 1);
          nix = fetch_ix(j + 1);
        }
        if (kb0 < 0) {
          ix.x = (base_row + ix.x) * Hkv + g;
          ix.y = (base_row + ix.y) * Hkv + g;
          ix.z = (base_row + ix.z) * Hkv + g;
          ix.w = (base_row + ix.w) * Hkv + g;
        }
        const int s = gh % C::kStages;
        const int u = gh / C::kStages;
        for (int kv = 0; kv < 2; ++kv) {
          uint64_t* empty = (kv == 0 ? bars.k_empty : bars.v_empty) + s;
          uint64_t* full = (kv == 0 ? bars.k_full : bars.v_full) + s;
          if (gh >= C::kStages && !mbar_wait(empty, (u - 1) & 1, err, kDevErrTimeoutBase + 16 + kv)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          if (aborted(abort_flag)) {
            stop = true;
            break;
          }
          if (kb0 < 0 && active) {
            unsigned char* dst = (kv == 0 ? sK : sV) + s * C::kKVBytes + rg * 512;
            const CUtensorMap* tm = kv == 0 ? &tmap_k : &tmap_v;
#pragma unroll
            for (int sl = 0; sl < C::kSlabs; ++sl)
              tma_gather4(dst + sl * C::kSlabBytes, tm, full, sl * 64, ix.x, ix.y, ix.z, ix.w);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(full);
        }
      }
    }
    // drain: this warp's copies must have landed before the CTA can leave
    if (lane == 0) {
      for (int j = gh - C::kStages < 0 ? 0 : gh - C::kStages; j < gh; ++j) {
        mbar_wait(bars.k_full + j % C::kStages, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 18);
        mbar_wait(bars.v_full + j % C::kStages, (j / C::kStages) & 1, err, kDevErrTimeoutBase + 18);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =====================================
    if (lane == 0) {
      const uint32_t idesc_qk = make_idesc_bf16(128, 128, false, false);
      const uint32_t idesc_pv = make_idesc_bf16(128, D, false, true);
      // descriptor low words of every operand base (the high words are constants)
      const uint32_t q_lo = desc_lo(smem_u32(sQ), 16), k_lo = desc_lo(smem_u32(sK), 16),
                     v_lo = desc_lo(smem_u32(sV), C::kSlabBytes), qx_lo = desc_lo(smem_u32(sQx), 128),
                     kx_lo = desc_lo(smem_u32(sKx), 128);
      constexpr uint32_t kKVStep = C::kKVBytes >> 4, kXStep = kXBytes >> 4;
      // Issue-wait: polls the barrier, gives up on a CTA abort or after the cycle limit.
      auto wait = [&](uint64_t* b, uint32_t parity, uint32_t site) -> bool {
        if (mbar_try_wait(b, parity)) return true;
        const long long t0 = clock64();
        while (true) {
          if (mbar_try_wait(b, parity)) return true;
          if (aborted(abort_flag)) return false;
          if (clock64() - t0 > kWaitLimitCycles) {
            raise_error(err, kDevErrTimeoutBase + site);
            return false;
          }
        }
      };
      bool ok = true;
      int g = 0, nq = 0, t1 = 0;   // key tiles so far (all items), items started, head-1 key tiles (d = 128)
      ItemInfo x;
      for (int i = 0; ok && item_info(i, x); ++i) {
        const int n_kt = x.n_kt, nh = x.nh;
        if (n_kt == 0) continue;
        ok = wait(bars.q_full, nq & 1, 4);
        ++nq;
        if (!ok) break;
        if constexpr (C::kSepP) {
          // Both heads in lockstep (one S/P/O barrier set for the pair).  The
          // softmax releases S right after reading it, so QK(j+1) goes in as
          // soon as that happens and runs during the softmax of tile j; PV(j)
          // follows once both heads' P(j) are written.  Queue: ... PV(j-1),
          // QK(j+1), PV(j) ...; the next item's first QK follows the current
          // item's last PV, and runs while the softmax warps write the output.
          ok = (g == 0 || wait(bars.s_free, (g - 1) & 1, 5)) &&
               wait(bars.k_full + g % C::kStages, (g / C::kStages) & 1, 1);
          if (!ok) break;
          tc_fence_after();
          {
            const uint32_t kl = k_lo + (g % C::kStages) * kKVStep, kxl = kx_lo + (g % C::kStages) * kXStep;
            if (nh == 2) issue_qk<D, 2>(tmem, 0, q_lo, kl, qx_lo, kxl, idesc_qk);
            else issue_qk<D, 1>(tmem, 0, q_lo, kl, qx_lo, kxl, idesc_qk);
          }
          umma_commit(bars.s_full);
          umma_commit(bars.k_empty + g % C::kStages);
          if (n_kt == 1) umma_commit(bars.q_empty);
          for (int j = 0; ok && j < n_kt; ++j) {
            const int gt = g + j, s = gt % C::kStages;
            if (j + 1 < n_kt) {
              const int s1 = (gt + 1) % C::kStages;
              ok = wait(bars.s_free, gt & 1, 5) && wait(bars.k_full + s1, ((gt + 1) / C::kStages) & 1, 6);
              if (!ok) break;
              tc_fence_after();
              const uint32_t kl = k_lo + s1 * kKVStep, kxl = kx_lo + s1 * kXStep;
              if (nh == 2) issue_qk<D, 2>(tmem, 0, q_lo, kl, qx_lo, kxl, idesc_qk);
              else issue_qk<D, 1>(tmem, 0, q_lo, kl, qx_lo, kxl, idesc_qk);
              umma_commit(bars.s_full);
              umma_commit(bars.k_empty + s1);
              if (j + 2 == n_kt) umma_commit(bars.q_empty);
            }
            ok = wait(bars.p_ready, gt & 1, 7) && wait(bars.v_full + s, (gt / C::kStages) & 1, 8);
            if (!ok) break;
            tc_fence_after();
            if (nh == 2) issue_pv<D, 2, true>(tmem, 0, v_lo + s * kKVStep, idesc_pv, j == 0);
            else issue_pv<D, 1, true>(tmem, 0, v_lo + s * kKVStep, idesc_pv, j == 0);
            umma_commit(bars.o_done);
            umma_commit(bars.v_empty + s);
          }
        } else {
          // P is written over S, so QK_h(j+1) can only follow PV_h(j).  Fixed
          // ping-pong order PV_0(j), QK_0(j+1), PV_1(j), QK_1(j+1): while one
          // head's softmax runs, the tensor core works through the other head's
          // PV and next QK.  Head 0 counts every key tile, head 1 only those of
          // items where the pair has two heads.
          ok = wait(bars.k_full + g % C::kStages, (g / C::kStages) & 1, 1);
          if (!ok) break;
          tc_fence_after();
          for (int h = 0; h < nh; ++h) {
            issue_qk<D, 1>(tmem, h, q_lo, k_lo + (g % C::kStages) * kKVStep, qx_lo,
                           kx_lo + (g % C::kStages) * kXStep, idesc_qk);
            umma_commit(bars.s_full + h);
          }
          umma_commit(bars.k_empty + g % C::kStages);
          if (n_kt == 1) umma_commit(bars.q_empty);
          for (int j = 0; ok && j < n_kt; ++j) {
            const int gt = g + j, s = gt % C::kStages, s1 = (gt + 1) % C::kStages;
            for (int h = 0; ok && h < nh; ++h) {
              const int ph = h == 0 ? gt : t1 + j;
              ok = wait(bars.p_ready + h, ph & 1, 7) && (h > 0 || wait(bars.v_full + s, (gt / C::kStages) & 1, 8));
              if (!ok) break;
              tc_fence_after();
              issue_pv<D, 1, false>(tmem, h, v_lo + s * kKVStep, idesc_pv, j == 0);
              umma_commit(bars.o_done + h);
              if (j + 1 < n_kt) {
                ok = h > 0 || wait(bars.k_full + s1, ((gt + 1) / C::kStages) & 1, 6);
                if (!ok) break;
                tc_fence_after();
                issue_qk<D, 1>(tmem, h, q_lo, k_lo + s1 * kKVStep, qx_lo, kx_lo + s1 * kXStep, idesc_qk);
                umma_commit(bars.s_full + h);
              }
            }
            if (!ok) break;
            umma_commit(bars.v_empty + s);
            if (j + 1 < n_kt) {
              umma_commit(bars.k_empty + s1);
              if (j + 2 == n_kt) umma_commit(bars.q_empty);
            }
          }
          if (nh == 2) t1 += n_kt;
        }
        g += n_kt;
      }
      if (!ok) *abort_flag = 1;
      // drain every MMA before TMEM is released
      umma_commit(bars.fin);
      mbar_wait_hot(bars.fin, 0, err, kDevErrTimeoutBase + 9);
    }
    __syncwarp();
  }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    // ======================= softmax / epilogue ============================
    const int h = (warp - 4) / 4;             // which head of the pair (warps 4-7, 8-11)
    const int row = (warp % 4) * 32 + lane;   // TMEM lane = query row in the tile
    const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
    const uint32_t tS = tmem + lane_base + h * 128;
    const uint32_t tO = tmem + lane_base + 256 + h * D;
    // barrier index: the lockstep layout (separate P) has one set for the pair
    const int hb = C::kSepP ? 0 : h;
    const unsigned long long scale2 = f32x2(scale_log2, scale_log2);
    bool ok = true;
    int g = 0, th = 0;   // key tiles so far (all items), key tiles this head took part in
    ItemInfo x;
    for (int i = 0; ok && item_info(i, x); ++i) {
      const int n_kt = x.n_kt;
      if (n_kt == 0) continue;
      if (h >= x.nh) {
        if (C::kSepP && hw == 2) {
          // the pair has one head: keep the lockstep barriers' counts, in the
          // same order as a working head (s_free as soon as S is there; p_ready
          // only after PV of the previous tile, so it cannot count toward that
          // tile's phase)
          for (int j = 0; ok && j < n_kt; ++j) {
            const int gt = g + j;
            ok = mbar_wait(bars.s_full, gt & 1, err, kDevErrTimeoutBase + 10) && !aborted(abort_flag);
            if (!(ok = __all_sync(0xFFFFFFFFu, ok))) break;
            mbar_arrive_warp(bars.s_free);
            if (j > 0) ok = mbar_wait(bars.o_done, (gt - 1) & 1, err, kDevErrTimeoutBase + 11);
            if (!(ok = __all_sync(0xFFFFFFFFu, ok))) break;
            mbar_arrive_warp(bars.p_ready);
          }
          if (!ok) *abort_flag = 1;
        }
        g += n_kt;
        continue;
      }
      const int ph0 = C::kSepP ? g : th;   // phase counter of this head's S/P/O barriers
      const int n_full = x.n_full;
      const int r0 = x.it.t * kRowTile;
      const int nrows = min(kRowTile, L - r0);
      const bool row_valid = row < nrows;
      float m = -INFINITY, l = 0.0f;
      for (int j = 0; j < n_kt; ++j) {
        const int gt = g + j, ph = ph0 + j;
        const int ms_slot = gt % C::kMetaSlots;
        ok = mbar_wait(bars.s_full + hb, ph & 1, err, kDevErrTimeoutBase + 10);
        // the tile's row-interval table (published by the K producer)
        if (ok) ok = mbar_wait(bars.meta_full + ms_slot, (gt / C::kMetaSlots) & 1, err, kDevErrTimeoutBase + 13);
        // warp-uniform from here on (the warp arrives on barriers as one)
        ok = __all_sync(0xFFFFFFFFu, ok && !aborted(abort_flag));
        if (!ok) break;
        tc_fence_after();
        uint32_t r[128];   // S row: scale * log2e * r = log2e * (scale q.k + dt)
        DMA_TMEM_LD32(tS + 0, (r + 0));
        DMA_TMEM_LD32(tS + 32, (r + 32));
        DMA_TMEM_LD32(tS + 64, (r + 64));
        DMA_TMEM_LD32(tS + 96, (r + 96));
        tmem_wait_ld();
        if constexpr (C::kSepP) {
          tc_fence_before();
          mbar_arrive_warp(bars.s_free);   // S may be overwritten by the next Q K^T
        }
        if (plan.no_topk && !((j + 1) * kKeyTile <= n_full || !row_valid)) {
          // every visible key kept: list entry e is key e, kept up to this
          // row's causal limit and the last valid key
          const int lim = min(r0 + row, x.n_total - 1) - j * kKeyTile;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c > lim) r[c] = __float_as_uint(-INFINITY);
        } else if (!((j + 1) * kKeyTile <= n_full || !row_valid)) {
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
        unsigned long long sa = 0ull, sb = 0ull;   // two packed partial sums
        // p = 2^(x * scale * log2e - m) for two keys, packed as bf16x2
        auto p_pair = [&](int k) -> uint32_t {
          const unsigned long long x2 =
              fma_f32x2(f32x2(__uint_as_float(r[k]), __uint_as_float(r[k + 1])), scale2, nm2);
          float x0, x1, p0, p1;
          f32x2_split(x2, x0, x1);
          if (((k >> 1) % C::kPolyEvery) == C::kPolyEvery - 1) {
            exp2_poly_x2(x0, x1, p0, p1);
          } else {
            p0 = fast_exp2(x0);
            p1 = fast_exp2(x1);
          }
          if ((k >> 1) & 1) sb = add_f32x2(sb, f32x2(p0, p1)); else sa = add_f32x2(sa, f32x2(p0, p1));
          return pack_bf16x2(p0, p1);
        };
        if constexpr (C::kSepP) {
          // all of P in registers first: only its store has to wait for PV of
          // the previous tile (which reads P's columns)
          uint32_t pk[64];
#pragma unroll
          for (int c = 0; c < 64; ++c) pk[c] = p_pair(2 * c);
          if (j > 0) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bars.o_done, (gt - 1) & 1, err, kDevErrTimeoutBase + 11));
            if (!ok) break;
            tc_fence_after();
          }
          const uint32_t tP = tmem + lane_base + 384 + h * 64;
          DMA_TMEM_ST32(tP, pk);
          DMA_TMEM_ST32(tP + 32, (pk + 32));
        } else {
          // P over S, in two halves of 64 keys (32 packed columns each)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) pk[c] = p_pair(64 * half + 2 * c);
            DMA_TMEM_ST32(tS + 32 * half, pk);
          }
          // consume every o_done phase in order (PV of the previous tile), so
          // the parity of the epilogue's wait is never ambiguous
          if (j > 0) {
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(bars.o_done + h, (ph - 1) & 1, err, kDevErrTimeoutBase + 11));
            if (!ok) {
              tmem_wait_st();
              break;
            }
            tc_fence_after();
          }
        }
        {
          float a0, a1, b0, b1;
          f32x2_split(sa, a0, a1);
          f32x2_split(sb, b0, b1);
          l += (a0 + a1) + (b0 + b1);
        }
        // rescale O (only warps where some row's max moved far enough); PV of
        // the previous tile is complete (waited above)
        if (j > 0 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
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
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(bars.p_ready + hb);
      }
      // epilogue: O / l once PV of the item's last key tile is done
      if (ok) ok = mbar_wait(bars.o_done + hb, (ph0 + n_kt - 1) & 1, err, kDevErrTimeoutBase + 12);
      if (!(ok = __all_sync(0xFFFFFFFFu, ok))) break;
      tc_fence_after();
      const float inv = 1.0f / l;
      const int head = x.it.g * nrep + 2 * x.it.pair + h;
      uint16_t* orow = out + ((static_cast<size_t>(x.it.b) * L + r0 + row) * Hq + head) * D;
      // the row's log-sum-exp in log2 units (m is the max the sum l was taken
      // against), for a backward pass that reuses it; 0 for a row with no key
      if (lse_out && row_valid)
        lse_out[(static_cast<size_t>(x.it.b) * Hq + head) * L + r0 + row] = m == -INFINITY ? 0.0f : m + log2f(l);
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
      // O may be overwritten by the next item's first PV (after this thread's
      // next p_ready arrival)
      tc_fence_before();
      g += n_kt;
      th += n_kt;
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
  if (C::kDynamic && threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(sched_done, 1u) == gridDim.x - 1) {
      // every CTA has drawn its last number: the next launch starts from zero
      *sched = 0u;
      *sched_done = 0u;
      __threadfence();
    }
  }
}

// ---- host: tensor maps -------------------------------------------------------

template <int D>
cudaError_t launch_d(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                     const PrefillPlan& plan, void* out, float* lse_out, uint32_t* err, cudaStream_t s) {
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
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(attn_prefill_kernel<D>), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  {
    // the warpgroups' register split must fit in what the block is launched
    // with (a property of the compiled kernel: checked once)
    static int num_regs = 0;
    if (num_regs == 0) {
      cudaFuncAttributes fa;
      e = cudaFuncGetAttributes(&fa, attn_prefill_kernel<D>);
      if (e != cudaSuccess) return e;
      num_regs = fa.numRegs;
    }
    if (num_regs * kThreads < 128 * kRegsControl + 256 * kRegsSoftmax) return cudaErrorInvalidConfiguration;
  }
  const int nrep = g.Hq / g.Hkv;
  const int npairs = (nrep + 1) / 2;
  const long long n_items = static_cast<long long>(plan.n_row_tiles) * g.B * g.Hkv * npairs;
  if (n_items > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const long long nblocks = n_items < nsm ? n_items : nsm;   // persistent: one CTA per SM
  return launch_after(attn_prefill_kernel<D>, dim3(static_cast<unsigned>(nblocks)), dim3(kThreads), C::kSmemBytes, s,
                      tq, tk, tv, tk3, tv3, plan, g.B, g.Lk, g.Hq, g.Hkv, scale * kLog2e, 1.0f / scale,
                      static_cast<uint16_t*>(out), lse_out, err);
}

}  // namespace

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

cudaError_t launch_attn_prefill(const void* q, const void* k, const void* v, const Geometry& g, float scale,
                                const PrefillPlan& plan, void* out, float* lse_out, uint32_t* err, cudaStream_t s) {
  if (g.d == 64) return launch_d<64>(q, k, v, g, scale, plan, out, lse_out, err, s);
  if (g.d == 128) return launch_d<128>(q, k, v, g, scale, plan, out, lse_out, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace dma
