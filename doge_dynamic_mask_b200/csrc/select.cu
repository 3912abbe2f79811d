// S2: the dynamic mask's causal top-k, as compact plans for the attention kernels.
//
// Method: page "Transformers 中的 Doge 小语言模型完全指南", section
// "动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 3
// (prepare_dynamic_mask: dt broadcast over the query rows, padding set to
// min_dtype, and above keep_window_size only the keep_window_size best
// positions of each row survive).  Causal masking is merged before the top-k,
// ties go to the lower key index.
//
// Prefill (one CTA per (batch, kv head, run of consecutive 128-row tiles)).
// dt does not depend on the query, so the row threshold tau_i (the composite
// key of row i's worst kept key) never decreases along the rows: each key is
// kept on one contiguous interval of rows, and the union U of the kept sets of
// a row tile is the w keys kept at its first row plus at most 127 newer keys.
// The CTA keeps U sorted by key.  For each tile of its run it
//   1. has K, the kept set at the tile's first row, sorted: for the run's first
//      tile by selecting the w-th largest key over the prefix (radix
//      histogram, then one collection pass) and sorting the w keys in shared
//      memory; for every later tile it is the previous tile's K(q), the first
//      w keys of the previous union, less at most its smallest key,
//   2. merges the tile's new keys that pass the first-row threshold into K,
//      giving U,
//   3. resolves tau_i for each row among the 128 smallest keys of U (the tail,
//      in which every row's tau lies),
//   4. gives each key its row interval [lo, hi) inside the tile (a key above
//      the tail is never evicted in the tile) and writes the list: keys kept
//      by every row first, then the rest, each with its dt bias and interval
//      (the order inside a class carries no meaning).
// Tiles whose rows see at most w keys (and every tile when Lk <= w) keep
// every visible key and skip the selection; their lists are in index order.
//
// Decode (one CTA per (batch, kv head)): the single query at len_b - 1 keeps
// the w best of its len_b keys, selected and collected like a run's first
// prefill tile and listed in any order.
#include <algorithm>

#include "select_common.cuh"

namespace dma {
namespace {

struct SelectSmem {
  uint32_t hist[kBins];
  uint64_t cand[kCandCap];
  uint32_t red[64];
  uint64_t vars[8];
};

// Prefill selector state; the candidate buffer of the prefix selection shares
// the dynamic region with the two key buffers (it is dead before they are
// written).
struct PrefillSelSmem {
  uint32_t hist[kBins];
  uint32_t red[64];
  uint64_t vars[8];
  uint64_t newk[kRowTile];      // the tile's new keys that pass tau0 (0: none), then sorted
  uint64_t news[kRowTile];      // the passing new keys, descending
  int32_t ins[kRowTile];        // keys of K above each of them
  uint64_t tau_s[kRowTile];     // tau of each row of the tile
  int32_t pos_s[kRowTile];      // ascending tail position of each row's tau (-1: the row keeps every visible key)
  int16_t rowpos[kRowTile];     // tail position of the union key whose index is r0 + offset, or -1
  uint32_t newmask[kRowTile / 32];    // row offsets j - r0 of the union's keys newer than the first row
  uint32_t oldmask[kRowTile / 32];    // tail positions of keys every row sees
  uint32_t wor[kRowTile / 32][kRowTile / 32];   // per-warp OR of the rows' new-key tail bits
  uint8_t hi_tail[kRowTile];    // first row whose tau lies above the tail key
  uint32_t cnt[2][kRowTile / 32];    // per-warp counts of the tail's evicted and dead keys
  uint32_t tot[4];
  uint64_t nextk;               // composite key of the next tile's first row
  // followed in dynamic shared memory by two key buffers of ucap keys
};

// prefill selector CTA: threads, and CTAs resident per SM (64 registers a thread)
// Two CTA shapes (threads, CTAs per SM at 64 registers a thread or fewer):
// 512 x 2 for sequences of fewer than kSelLongRowTiles row tiles, 256 x 3
// beyond (smaller blocks pay less at the per-tile barriers, and the longer
// prefix selections of long sequences spread over more CTAs).  Measured: the
// padded sparse workload (64 row tiles) 0.074 ms with 512 x 2 and 0.076 ms
// with 256 x 3; the long one (256 row tiles) 0.108 and 0.100 ms.
constexpr int kSelPrefillThreads = 512;
constexpr int kSelPrefillMinBlocks = 2;
constexpr int kSelPrefillThreadsLong = 256;
constexpr int kSelPrefillMinBlocksLong = 3;
constexpr int kSelLongRowTiles = 128;

// at most this many consecutive row tiles per prefill-selector CTA (see
// select_prefill_kernel); the launcher picks fewer when the grid would not
// fill the GPU
constexpr int kSelTilesPerCtaMax = 8;

__device__ __forceinline__ int clamp_len(const int32_t* lengths, int b, int L, uint32_t* err) {
  int len = lengths ? lengths[b] : L;
  if (len < 1 || len > L) {
    if (threadIdx.x == 0) raise_error(err, kDevErrBadLength);
    len = len < 1 ? 1 : L;
  }
  return len;
}

// Bit position of the k-th (1-based) set bit of b; 1 <= k <= popc(b).
__device__ __forceinline__ int nth_set_bit(uint32_t b, int k) {
  int pos = 0;
#pragma unroll
  for (int width = 16; width >= 1; width >>= 1) {
    const int c = __popc(b & ((1u << width) - 1u));
    if (c < k) {
      k -= c;
      b >>= width;
      pos += width;
    }
  }
  return pos;
}

// Number of set bits at offsets [0, lim] of a 128-bit mask (0 when lim < 0).
__device__ __forceinline__ int popc_upto(const uint32_t* m, int lim) {
  int c = 0;
#pragma unroll
  for (int wd = 0; wd < 4; ++wd) {
    const int top = lim - 32 * wd;
    if (top >= 31) c += __popc(m[wd]);
    else if (top >= 0) c += __popc(m[wd] & ((2u << top) - 1u));
  }
  return c;
}

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
  const uint32_t lo = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v), m);
  const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, static_cast<uint32_t>(v >> 32), m);
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Number of entries of the descending array a[0, n) greater than v (v not in a).
__device__ __forceinline__ int count_greater(const uint64_t* a, int n, uint64_t v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] > v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// Bitonic compare-exchange stages with partner distance j <= 16 for block size k,
// on one key per lane; e is the key's position in the whole sequence (its
// bits pick the direction: the lower position keeps the larger key where
// (e & k) == 0, so the final sequence is descending).
__device__ __forceinline__ uint64_t bitonic_warp_stages(uint64_t v, int e, int k) {
#pragma unroll
  for (int j = 16; j > 0; j >>= 1) {
    if (j < k) {
      const uint64_t o = shfl_xor64(v, j);
      const bool keep_max = ((e & j) == 0) == ((e & k) == 0);
      v = keep_max ? (o > v ? o : v) : (o < v ? o : v);
    }
  }
  return v;
}

// Sorts the n distinct keys (all > 0) of a[0, n) in descending order, in
// place; a must have room for pow2 = max(32, next power of two >= n) keys
// (the rest is padded with 0, which sorts last).  Stages with partner distance
// up to 16 run on registers (one key per lane, shuffles), the longer ones as
// pair passes over shared memory.  Every thread must call it.
__device__ void block_bitonic_desc(uint64_t* a, int n) {
  int pow2 = 32;
  while (pow2 < n) pow2 <<= 1;
  for (int e = n + threadIdx.x; e < pow2; e += blockDim.x) a[e] = 0ull;
  __syncthreads();
  const int lane = static_cast<int>(lane_id()), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int base = warp * 32; base < pow2; base += nw * 32) {   // blocks of 2 .. 32
    const int e = base + lane;
    uint64_t v = a[e];
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) v = bitonic_warp_stages(v, e, k);
    a[e] = v;
  }
  __syncthreads();
  for (int k = 64; k <= pow2; k <<= 1) {
    for (int j = k >> 1; j >= 32; j >>= 1) {
      for (int i = threadIdx.x; i < (pow2 >> 1); i += blockDim.x) {
        const int x = ((i & ~(j - 1)) << 1) | (i & (j - 1)), y = x + j;
        const uint64_t u = a[x], v = a[y];
        const uint64_t big = u > v ? u : v, small = u > v ? v : u;
        const bool desc = (x & k) == 0;
        a[x] = desc ? big : small;
        a[y] = desc ? small : big;
      }
      __syncthreads();
    }
    for (int base = warp * 32; base < pow2; base += nw * 32) {
      const int e = base + lane;
      a[e] = bitonic_warp_stages(a[e], e, k);
    }
    __syncthreads();
  }
}

// Sorts the n distinct keys of a[0, n) in descending order into a, with tmp
// (n keys) as scratch and hist (kBins words): keys are bucketed by the 11
// bits below the highest bit in which they differ, each bucket taking the
// range of positions its rank among the buckets gives, and each key is then
// placed by its rank inside its bucket.  Returns false, with a unchanged, when
// a bucket holds more than 32 keys (the caller sorts another way).  Every
// thread must call it.
__device__ bool block_bucket_sort_desc(uint64_t* a, uint64_t* tmp, int n, uint32_t* hist, uint32_t* red) {
  uint64_t vor = 0ull, vand = ~0ull;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    vor |= a[e];
    vand &= a[e];
  }
  uint64_t O, A;
  block_or_and64(vor, vand, red, O, A);
  const uint64_t vary = O ^ A;
  if (vary == 0ull) return true;   // at most one key
  const int hb = 63 - __clzll(static_cast<long long>(vary));
  const int sh = hb >= 10 ? hb - 10 : 0;
  auto digit = [&](uint64_t k) { return static_cast<int>((k >> sh) & static_cast<uint64_t>(kBins - 1)); };
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += blockDim.x) atomicAdd(&hist[digit(a[e])], 1u);
  __syncthreads();
  // bucket starts from the top bucket down: off[d] = keys in buckets above d
  const int per = (kBins + blockDim.x - 1) / blockDim.x;
  const int top = kBins - static_cast<int>(threadIdx.x) * per;   // this thread's buckets [top - per, top)
  uint32_t local = 0, biggest = 0;
  for (int d = top - 1; d >= top - per && d >= 0; --d) {
    const uint32_t h = hist[d];
    local += h;
    biggest = h > biggest ? h : biggest;
  }
  if (__syncthreads_or(biggest > 32u)) return false;
  uint32_t total;
  uint32_t run = block_exclusive_scan(local, red, &total);
  for (int d = top - 1; d >= top - per && d >= 0; --d) {
    const uint32_t h = hist[d];
    hist[d] = run;
    run += h;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const uint64_t k = a[e];
    tmp[atomicAdd(&hist[digit(k)], 1u)] = k;
  }
  __syncthreads();
  // hist[d] is now the end of bucket d, and bucket d starts where bucket d + 1 ends
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const uint64_t k = tmp[e];
    const int d = digit(k);
    const int st = d + 1 < kBins ? static_cast<int>(hist[d + 1]) : 0, en = static_cast<int>(hist[d]);
    int r = 0;
    for (int f = st; f < en; ++f) r += tmp[f] > k;
    a[st + r] = k;
  }
  __syncthreads();
  return true;
}

// Appends, in any order, the composite keys of positions [0, n) of a dt row
// that are >= tau to X (at most cap are stored); returns their number.  Each warp
// reserves room for sixteen keys per lane with one shared-memory atomic.
// Every thread must call it.
__device__ int row_collect_ge(const uint32_t* __restrict__ bits, int n, uint64_t tau, uint64_t* X, int cap,
                              unsigned long long* counter) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const uint32_t lane = lane_id(), lt = lanemask_lt();
  if (tid == 0) *counter = 0ull;
  __syncthreads();
  const bool vec = (reinterpret_cast<uintptr_t>(bits) & 15u) == 0;
  const int nq = vec ? (n >> 2) : 0;
  const uint4* qv = reinterpret_cast<const uint4*>(bits);
  for (int r0 = 0; r0 < nq; r0 += 4 * nt) {   // same trip count in every thread
    uint32_t v[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = r0 + u * nt + tid;
      const uint4 x = i < nq ? __ldg(qv + i) : make_uint4(0u, 0u, 0u, 0u);
      v[4 * u] = x.x;
      v[4 * u + 1] = x.y;
      v[4 * u + 2] = x.z;
      v[4 * u + 3] = x.w;
    }
    uint32_t vote[16];
    uint32_t total = 0;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = r0 + (c >> 2) * nt + tid;
      const bool m = i < nq && composite_key(v[c], static_cast<uint32_t>(4 * i + (c & 3))) >= tau;
      vote[c] = __ballot_sync(0xFFFFFFFFu, m);
      total += __popc(vote[c]);
    }
    uint32_t base = 0;
    if (lane == 0 && total) base = static_cast<uint32_t>(atomicAdd(counter, static_cast<unsigned long long>(total)));
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = r0 + (c >> 2) * nt + tid;
      if ((vote[c] >> lane) & 1u) {
        const uint32_t pos = base + __popc(vote[c] & lt);
        if (pos < static_cast<uint32_t>(cap)) X[pos] = composite_key(v[c], static_cast<uint32_t>(4 * i + (c & 3)));
      }
      base += __popc(vote[c]);
    }
  }
  for (int j0 = nq << 2; j0 < n; j0 += nt) {   // the rest of the row (or a row not 16-byte aligned)
    const int j = j0 + tid;
    uint64_t key = 0ull;
    const bool m = j < n && (key = composite_key(__ldg(bits + j), static_cast<uint32_t>(j))) >= tau;
    const uint32_t vote = __ballot_sync(0xFFFFFFFFu, m);
    uint32_t base = 0;
    if (lane == 0 && vote) base = static_cast<uint32_t>(atomicAdd(counter, static_cast<unsigned long long>(__popc(vote))));
    base = __shfl_sync(0xFFFFFFFFu, base, 0);
    if (m) {
      const uint32_t pos = base + __popc(vote & lt);
      if (pos < static_cast<uint32_t>(cap)) X[pos] = key;
    }
  }
  __syncthreads();
  const int r = static_cast<int>(*counter);
  __syncthreads();
  return r;   // may exceed cap (only cap keys were stored)
}

// Collects the composite keys of positions [0, n) of a dt row by class:
// cls(v) == 1 appends the key at the front of out (positions 0, 1, ...),
// cls(v) == 2 at the back (positions cap - 1, cap - 2, ...), any order within
// a class; counters[0] and counters[1] end as the two counts.  Each warp
// reserves room for sixteen keys per lane with one shared-memory atomic per
// class.  Every thread must call it.
template <class Cls>
__device__ void row_collect2(const uint32_t* __restrict__ bits, int n, Cls cls, uint64_t* out, int cap,
                             unsigned long long* counters) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const uint32_t lane = lane_id(), lt = lanemask_lt();
  if (tid < 2) counters[tid] = 0ull;
  __syncthreads();
  auto place = [&](uint32_t vf, uint32_t vb, uint32_t& bf, uint32_t& bb, uint64_t key) {
    if ((vf >> lane) & 1u) {
      const uint32_t pos = bf + __popc(vf & lt);
      if (pos < static_cast<uint32_t>(cap)) out[pos] = key;
    } else if ((vb >> lane) & 1u) {
      const uint32_t pos = bb + __popc(vb & lt);
      if (pos < static_cast<uint32_t>(cap)) out[cap - 1 - pos] = key;
    }
    bf += __popc(vf);
    bb += __popc(vb);
  };
  const bool vec = (reinterpret_cast<uintptr_t>(bits) & 15u) == 0;
  const int nq = vec ? (n >> 2) : 0;
  const uint4* qv = reinterpret_cast<const uint4*>(bits);
  for (int r0 = 0; r0 < nq; r0 += 4 * nt) {   // same trip count in every thread
    uint32_t v[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = r0 + u * nt + tid;
      const uint4 x = i < nq ? __ldg(qv + i) : make_uint4(0u, 0u, 0u, 0u);
      v[4 * u] = x.x;
      v[4 * u + 1] = x.y;
      v[4 * u + 2] = x.z;
      v[4 * u + 3] = x.w;
    }
    uint32_t vf[16], vb[16];
    uint32_t tf = 0, tb = 0;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = r0 + (c >> 2) * nt + tid;
      const int k = i < nq ? cls(v[c]) : 0;
      vf[c] = __ballot_sync(0xFFFFFFFFu, k == 1);
      vb[c] = __ballot_sync(0xFFFFFFFFu, k == 2);
      tf += __popc(vf[c]);
      tb += __popc(vb[c]);
    }
    uint32_t bf = 0, bb = 0;
    if (lane == 0) {
      if (tf) bf = static_cast<uint32_t>(atomicAdd(counters, static_cast<unsigned long long>(tf)));
      if (tb) bb = static_cast<uint32_t>(atomicAdd(counters + 1, static_cast<unsigned long long>(tb)));
    }
    bf = __shfl_sync(0xFFFFFFFFu, bf, 0);
    bb = __shfl_sync(0xFFFFFFFFu, bb, 0);
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const int i = r0 + (c >> 2) * nt + tid;
      place(vf[c], vb[c], bf, bb, composite_key(v[c], static_cast<uint32_t>(4 * i + (c & 3))));
    }
  }
  for (int j0 = nq << 2; j0 < n; j0 += nt) {   // the rest of the row (or a row not 16-byte aligned)
    const int j = j0 + tid;
    const uint32_t b = j < n ? __ldg(bits + j) : 0u;
    const int k = j < n ? cls(b) : 0;
    const uint32_t vf = __ballot_sync(0xFFFFFFFFu, k == 1), vb = __ballot_sync(0xFFFFFFFFu, k == 2);
    uint32_t bf = 0, bb = 0;
    if (lane == 0) {
      if (vf) bf = static_cast<uint32_t>(atomicAdd(counters, static_cast<unsigned long long>(__popc(vf))));
      if (vb) bb = static_cast<uint32_t>(atomicAdd(counters + 1, static_cast<unsigned long long>(__popc(vb))));
    }
    bf = __shfl_sync(0xFFFFFFFFu, bf, 0);
    bb = __shfl_sync(0xFFFFFFFFu, bb, 0);
    place(vf, vb, bf, bb, composite_key(b, static_cast<uint32_t>(j)));
  }
  __syncthreads();
}

// K(p) for n > w: the w largest composite keys among positions [0, n) of a dt
// row, in any order, into out[0, w); *tau gets the w-th largest.  Three passes
// over the row: which dt bits vary (OR / AND), an 11-bit histogram of the
// highest varying bits, and one collection of every key in or above the bin
// B holding the w-th largest (keys above B from the front of out, keys in B
// from its back); tau is then selected among B's keys in shared memory and
// B's keys at or above it join the front.  Returns false, with nothing
// written, when B's keys would not fit beside the w (the caller selects and
// collects another way).  Every thread must call it.
static __device__ __noinline__ bool prefix_topw(const uint32_t* __restrict__ bits, int n, int w, uint64_t* out, int cap,
                                               SelScratch sc,
                            unsigned long long* counters, uint64_t* tau) {
  if (w > cap) return false;
  uint32_t vor = 0u, vand = ~0u;
  row_for_each(bits, n, [&](uint32_t v, int, bool ok) {
    if (ok) {
      vor |= v;
      vand &= v;
    }
  });
  uint64_t O, A;
  block_or_and64(vor, vand, sc.red, O, A);
  const uint32_t vary = static_cast<uint32_t>(O ^ A) ;
  if (vary == 0u) {   // one dt value: the lowest w indices rank highest
    for (int e = threadIdx.x; e < w; e += blockDim.x) out[e] = composite_key(static_cast<uint32_t>(A), e);
    *tau = composite_key(static_cast<uint32_t>(A), static_cast<uint32_t>(w - 1));
    __syncthreads();
    return true;
  }
  const int hb = 31 - __clz(vary);
  const int sh = hb >= 10 ? hb - 10 : 0;
  const int nb = 1 << (hb - sh + 1);
  const uint32_t mask = static_cast<uint32_t>(nb - 1);
  for (int i = threadIdx.x; i < nb; i += blockDim.x) sc.hist[i] = 0u;
  __syncthreads();
  row_for_each(bits, n, [&](uint32_t v, int, bool ok) {
    if (ok) atomicAdd(&sc.hist[(v >> sh) & mask], 1u);
  });
  __syncthreads();
  uint32_t k_in_bin, cnt_b;
  const uint32_t B = find_bin_from_top(sc.hist, nb, static_cast<uint32_t>(w), sc.red, sc.vars, &k_in_bin, &cnt_b);
  const int above = w - static_cast<int>(k_in_bin);
  if (w + static_cast<int>(cnt_b) > cap) return false;
  row_collect2(
      bits, n, [&](uint32_t v) { const uint32_t d = (v >> sh) & mask; return d > B ? 1 : (d == B ? 2 : 0); }, out, cap,
      counters);
  // tau: the k_in_bin-th largest of B's keys, out[cap - cnt_b, cap)
  uint64_t* binb = out + (cap - static_cast<int>(cnt_b));
  const uint64_t t = select_kth_smem(binb, static_cast<int>(cnt_b), k_in_bin, sc);
  if (threadIdx.x == 0) counters[0] = 0ull;
  __syncthreads();
  for (int e = threadIdx.x; e < static_cast<int>(cnt_b); e += blockDim.x) {
    const uint64_t k = binb[e];
    if (k >= t) out[above + static_cast<int>(atomicAdd(counters, 1ull))] = k;
  }
  __syncthreads();
  *tau = t;
  return true;
}

// Collects, in any order, the composite keys of positions [0, n) of a dt row
// that are >= tau into out[0, cap): warp w appends to its own region of
// cap / warps keys with a running offset (no atomics), and pads the rest of
// the region with 0 (below every key).  The row is read as 16-byte pieces,
// four per thread per step, with the next step's pieces prefetched into L2
// before this step's are loaded.  Returns the number of keys, or -1 when some warp's
// region overflowed.  Every thread must call it.
static __device__ __noinline__ int row_collect_ge_regions(const uint32_t* __restrict__ bits, int n, uint64_t tau,
                                                         uint64_t* out, int cap, uint32_t* red) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = static_cast<int>(lane_id()), warp = tid >> 5, nw = nt >> 5;
  const uint32_t lt = lanemask_lt();
  const int rcap = cap / nw;
  uint64_t* reg = out + warp * rcap;
  int run = 0;   // keys this warp found (may pass rcap: then only rcap are stored)
  auto put = [&](bool m, uint64_t key) {
    const uint32_t vote = __ballot_sync(0xFFFFFFFFu, m);
    if (m) {
      const int pos = run + __popc(vote & lt);
      if (pos < rcap) reg[pos] = key;
    }
    run += __popc(vote);
  };
  const bool vec = (reinterpret_cast<uintptr_t>(bits) & 15u) == 0;
  const int nq = vec ? (n >> 2) : 0;
  const uint4* qv = reinterpret_cast<const uint4*>(bits);
  for (int r0 = 0; r0 < nq; r0 += 4 * nt) {   // same trip count in every thread
    // the next step's pieces go to L2 now, so its loads do not wait on memory
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = r0 + 4 * nt + u * nt + tid;
      if (i < nq) asm volatile("prefetch.global.L2 [%0];" ::"l"(qv + i));
    }
    uint4 cur[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = r0 + u * nt + tid;
      cur[u] = i < nq ? __ldg(qv + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = r0 + u * nt + tid;
      const bool ok = i < nq;
      const uint32_t x[4] = {cur[u].x, cur[u].y, cur[u].z, cur[u].w};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint64_t key = composite_key(x[c], static_cast<uint32_t>(4 * i + c));
        put(ok && key >= tau, key);
      }
    }
  }
  for (int j0 = nq << 2; j0 < n; j0 += nt) {   // the rest of the row (or a row not 16-byte aligned)
    const int j = j0 + tid;
    const uint64_t key = j < n ? composite_key(__ldg(bits + j), static_cast<uint32_t>(j)) : 0ull;
    put(j < n && key >= tau, key);
  }
  for (int e = run + lane; e < rcap; e += 32) reg[e] = 0ull;
  if (lane == 0) red[warp] = static_cast<uint32_t>(run);
  __syncthreads();
  int total = 0;
  bool over = false;
  for (int k = 0; k < nw; ++k) {
    total += static_cast<int>(red[k]);
    over |= static_cast<int>(red[k]) > rcap;
  }
  __syncthreads();
  return over ? -1 : total;
}

constexpr int kSampleMax = 4096;

// The keys of positions [0, n) of a dt row at or above a threshold t_lo that
// lies a little below the w-th largest: t_lo is the r-th largest of a sample
// of kSampleMax keys, 64 runs of 64 consecutive keys spread evenly over the
// row (r = 3/2 of w's share of the sample, plus 16), so about 3/2 w keys pass
// (for i.i.d. scores fewer than w is a 5.5 sigma event at the decode sizes).  One pass collects them into out (any order).  Returns
// their number c; the caller uses them when w <= c <= cap (then the w-th
// largest overall is the w-th largest among them), else falls back to an
// exact selection.  Every thread must call it.
__device__ int sampled_collect(const uint32_t* __restrict__ bits, int n, int w, uint64_t* out, int cap, SelScratch sc,
                               unsigned long long* counter) {
  const int S = n < kSampleMax ? n : kSampleMax;
  if (S > cap) return -1;
  // the sample: 64 runs of 64 consecutive keys (two 128-byte lines each)
  // spread evenly over the row, or the whole row when it is short
  auto pos_of = [&](int s) { return S < kSampleMax ? s : (s >> 6) * (n / 64) + (s & 63); };
  for (int s0 = 0; s0 < S; s0 += 8 * blockDim.x) {   // eight independent loads in flight per thread
    uint32_t v[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int s = s0 + r * blockDim.x + threadIdx.x;
      v[r] = s < S ? __ldg(bits + pos_of(s)) : 0u;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int s = s0 + r * blockDim.x + threadIdx.x;
      if (s < S) out[s] = composite_key(v[r], static_cast<uint32_t>(pos_of(s)));
    }
  }
  __syncthreads();
  long long r = (static_cast<long long>(w) * S * 3) / (static_cast<long long>(n) * 2) + 16;
  if (r > S) r = S;
  const uint64_t t_lo = select_kth_smem(out, S, static_cast<uint32_t>(r), sc);
  return row_collect_ge_regions(bits, n, t_lo, out, cap, sc.red);
}

// A row tile that lies wholly past its sequence's last valid row: every row
// sees the same keys and keeps K (w keys, sorted by key), so its tau is K's
// smallest key and the list is K, each kept by every row.  Every thread must
// call it.
static __device__ __noinline__ void list_whole_set(const uint64_t* K, int w, int nrows, uint64_t* tau_rows,
                                                   PrefillPlan plan, size_t tile) {
  int32_t* idx_o = plan.idx + tile * plan.cap;
  float* bias_o = plan.bias + tile * plan.cap;
  uint32_t* span_o = plan.span + tile * plan.cap;
  const uint64_t tau_last = K[w - 1];
  for (int i = threadIdx.x; i < nrows; i += blockDim.x) tau_rows[i] = tau_last;
  for (int e = threadIdx.x; e < w; e += blockDim.x) {
    const uint64_t key = K[e];
    idx_o[e] = static_cast<int32_t>(composite_index(key));
    bias_o[e] = __uint_as_float(static_cast<uint32_t>(key >> 32));
    span_o[e] = static_cast<uint32_t>(nrows) << 16;
  }
  const int padded = (w + kKeyTile - 1) / kKeyTile * kKeyTile;
  for (int j = w + threadIdx.x; j < padded; j += blockDim.x) {
    idx_o[j] = 0;
    bias_o[j] = 0.0f;
    span_o[j] = 0u;
  }
  int32_t* kb = plan.kbase + tile * (plan.cap / kKeyTile);
  for (int kt = threadIdx.x; kt * kKeyTile < w; kt += blockDim.x) kb[kt] = -1;   // listed by key, not by index
  if (threadIdx.x == 0) plan.counts[tile] = make_int2(w, w);
}

// One CTA per (batch, kv head, run of tpc consecutive row tiles).
//
// The CTA keeps the union U of a tile (the keys any of its rows keeps) sorted
// by composite key, descending.  All of U is visible at the tile's last row q,
// so the kept set there, K(q), is U's first w keys: it carries to the next
// tile as is.  The next tile's first-row threshold tau0 is the w-th largest of
// K(q) and the key of its first row p (tau_last = U[w-1], second smallest
// U[w-2]); its union is K(q) without the keys below tau0 (at most the last)
// merged with its new keys (q, q'] at or above tau0, sorted.  The first tile of
// a run selects tau0 over its prefix, collects K(p) and sorts it.
//
// Every row's tau lies among the 128 smallest keys of U (a row sees at most
// |U| - w keys fewer than U holds), the tail of the sorted union: row i's tau
// is its rank-th visible tail key in ascending order, rank = (visible keys of
// U) - w + 1, with the tail keys every row sees and the prefix-OR over rows of
// the new ones.  A key above the tail is never evicted inside the tile; a tail
// key is kept up to the first row whose tau lies above it.  The list holds the
// keys every row keeps, then the others, each class in U's (descending key)
// order; consecutive lanes write consecutive entries.
template <int kThreads_, int kMinBlocks_>
__global__ void __launch_bounds__(kThreads_, kMinBlocks_) select_prefill_kernel(const float* __restrict__ dt,
                                                                     const int32_t* __restrict__ lengths, int Hkv,
                                                                     int L, int w, int tpc, PrefillPlan plan,
                                                                     uint32_t* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  PrefillSelSmem& sm = *reinterpret_cast<PrefillSelSmem*>(smem_raw);
  pdl_wait();      // dt comes from the previous kernel
  pdl_trigger();   // the attention may be scheduled
  const int ucap = w + kRowTile;
  uint64_t* Ubuf = reinterpret_cast<uint64_t*>(smem_raw + sizeof(PrefillSelSmem));   // two buffers of ucap keys
  SelScratch sc{sm.hist, Ubuf, sm.red, sm.vars};   // the candidate buffer is dead before Ubuf is written

  // grid (kv head, batch, run): blocks start in that order, so the runs are
  // taken from the end of the sequence backwards (the late runs, whose first
  // tile selects over the longest prefix, start in the first wave)
  const int g = blockIdx.x, b = blockIdx.y;
  const int run = static_cast<int>(gridDim.z - 1 - blockIdx.z);
  const int len = clamp_len(lengths, b, L, err);
  const bool topk = L > w;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(dt) + bg * L;
  uint64_t* tau_g = plan.tau + bg * L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nw = static_cast<int>(blockDim.x >> 5);
  const uint32_t lt = lanemask_lt();
  const int t_first = run * tpc;
  const int t_last = min(plan.n_row_tiles, t_first + tpc);
  bool have = false;      // K(q') of the previous tile and this tile's tau0 carry over
  int cur = 0;            // buffer whose head holds K
  int q_prev = 0;
  uint64_t tau0 = 0ull;
  uint32_t pre_bits = 0u;   // dt bits of this tile's new key q' + 1 + tid (prefetched)

  for (int t = t_first; t < t_last; ++t) {
    const int r0 = t * kRowTile;
    const int nrows = min(kRowTile, L - r0);
    const int p = min(r0, len - 1);                 // effective position of the first row
    const int q = min(r0 + nrows - 1, len - 1);     // effective position of the last row
    const size_t tile = bg * plan.n_row_tiles + t;
    int32_t* idx_o = plan.idx + tile * plan.cap;
    float* bias_o = plan.bias + tile * plan.cap;
    uint32_t* span_o = plan.span + tile * plan.cap;

    if (!topk || q + 1 <= w) {
      // every visible key of every row is kept: keys <= r0 by all rows, key j > r0 from row j on
      const int n_full = min(r0, q) + 1;
      const int n_total = q + 1;
      for (int i = tid; i < nrows; i += blockDim.x) tau_g[r0 + i] = 0ull;
      for (int j = tid; j < n_total; j += blockDim.x) {
        idx_o[j] = j;
        bias_o[j] = __uint_as_float(bits[j]);
        const int lo = j > r0 ? j - r0 : 0;
        span_o[j] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(nrows) << 16);
      }
      const int padded = (n_total + kKeyTile - 1) / kKeyTile * kKeyTile;
      for (int j = n_total + tid; j < padded; j += blockDim.x) {
        idx_o[j] = 0;
        bias_o[j] = 0.0f;
        span_o[j] = 0u;
      }
      int32_t* kb = plan.kbase + tile * (plan.cap / kKeyTile);
      for (int kt = tid; kt * kKeyTile < n_total; kt += blockDim.x) kb[kt] = kt * kKeyTile;   // [0, q] in order
      if (tid == 0) plan.counts[tile] = make_int2(n_full, n_total);
      have = false;
      continue;
    }

    // the next tile of the run: its first row, last row and new keys (q, q_next],
    // whose dt loads are issued now and used one tile later
    const bool more = t + 1 < t_last;
    const int p_next = min(r0 + kRowTile, len - 1);
    const int q_next = more ? min(r0 + kRowTile + min(kRowTile, L - r0 - kRowTile) - 1, len - 1) : q;
    uint32_t pre_next = 0u;
    if (more && tid < q_next - q) pre_next = __ldg(bits + q + 1 + tid);

    if (have && p == q_prev) {
      // the whole tile lies past the sequence's last valid row: every row
      // keeps the carried K; K, cur and tau0 carry over unchanged
      list_whole_set(Ubuf + static_cast<size_t>(cur) * ucap, w, nrows, tau_g + r0, plan, tile);
      q_prev = q;
      have = more;
      continue;
    }

    // K, the kept set at p (tau0 and above, at or before p), sorted, in buffer cur
    int n_keep, j_new;   // keys of K at or above tau0; the new keys are (j_new, q]
    uint32_t new_bits;
    if (have) {
      uint64_t* K = Ubuf + static_cast<size_t>(cur) * ucap;
      n_keep = K[w - 1] >= tau0 ? w : w - 1;   // only the smallest key can fall below tau0
      j_new = q_prev;
      new_bits = pre_bits;
    } else {
      // K(p) = the keys at or before p at or above tau0 (the w-th largest), then sorted
      tau0 = 0ull;
      unsigned long long* ctr = reinterpret_cast<unsigned long long*>(&sm.vars[6]);
      if (p + 1 > w && prefix_topw(bits, p + 1, w, Ubuf, 2 * ucap, sc, ctr, &tau0)) {
        n_keep = w;
      } else {
        if (p + 1 > w) tau0 = select_kth_global(bits, p + 1, static_cast<uint32_t>(w), sc);
        n_keep = min(row_collect_ge(bits, p + 1, tau0, Ubuf, ucap, ctr), ucap);
      }
      if (!block_bucket_sort_desc(Ubuf, Ubuf + ucap, n_keep, sm.hist, sm.red)) block_bitonic_desc(Ubuf, n_keep);
      cur = 0;
      j_new = p;
      new_bits = (tid < q - p) ? __ldg(bits + p + 1 + tid) : 0u;
    }
    uint64_t* K = Ubuf + static_cast<size_t>(cur) * ucap;
    uint64_t* U = Ubuf + static_cast<size_t>(cur ^ 1) * ucap;

    // the new keys (j_new, q] at or above tau0, sorted: rank among them by count
    const int n_new = q - j_new;
    uint64_t nkey = 0ull;
    if (tid < n_new) {
      nkey = composite_key(new_bits, static_cast<uint32_t>(j_new + 1 + tid));
      if (nkey < tau0) nkey = 0ull;
    }
    if (tid < kRowTile) {
      sm.newk[tid] = nkey;
      const uint32_t v = __ballot_sync(0xFFFFFFFFu, nkey != 0ull);
      if (lane == 0) sm.cnt[0][warp] = __popc(v);
    }
    if (tid < kRowTile / 32) {
      sm.newmask[tid] = 0u;
      sm.oldmask[tid] = 0u;
    }
    if (tid == 0 && more) sm.nextk = composite_key(pre_next, static_cast<uint32_t>(p_next));
    __syncthreads();
    int n_pass = 0;
#pragma unroll
    for (int k = 0; k < kRowTile / 32; ++k) n_pass += static_cast<int>(sm.cnt[0][k]);
    if (nkey != 0ull) {
      int rank = 0;
#pragma unroll 16
      for (int m = 0; m < kRowTile; ++m) rank += sm.newk[m] > nkey;
      sm.news[rank] = nkey;
      const int o = j_new + 1 + tid - r0;   // row offset of a key newer than the first row
      if (o >= 1 && o < kRowTile) atomicOr(&sm.newmask[o >> 5], 1u << (o & 31));
    }
    __syncthreads();

    // U = merge of K's first n_keep keys and the sorted new keys: each new key's
    // insertion point in K, then each key of K shifts by the new keys above it
    if (tid < n_pass) sm.ins[tid] = count_greater(K, n_keep, sm.news[tid]);
    __syncthreads();
    {
      int insl[kRowTile / 32];   // lane l holds ins[l + 32 k] (n_keep + 1 past the end: never counted)
#pragma unroll
      for (int k = 0; k < kRowTile / 32; ++k) insl[k] = lane + 32 * k < n_pass ? sm.ins[lane + 32 * k] : n_keep + 1;
      for (int e0 = warp * 32; e0 < n_keep; e0 += nw * 32) {
        int c0 = 0;   // new keys inserted at or before e0
#pragma unroll
        for (int k = 0; k < kRowTile / 32; ++k) c0 += __popc(__ballot_sync(0xFFFFFFFFu, insl[k] <= e0));
        const int e = e0 + lane;
        int c = c0;
        for (int m = c0; m < n_pass && sm.ins[m] <= e0 + 31; ++m) c += sm.ins[m] <= e;
        if (e < n_keep) U[e + c] = K[e];
      }
    }
    if (tid < n_pass) U[tid + sm.ins[tid]] = sm.news[tid];
    const int nU = n_keep + n_pass;
    const int n_old = p + 1 > w ? w : p + 1;
    const int nbot = min(nU, kRowTile);
    if (tid < kRowTile) sm.rowpos[tid] = -1;
    __syncthreads();

    // the tail (nbot smallest keys of U, ascending position s = nU - 1 - e):
    // keys every row sees, and the row at which each newer key appears
    if (tid < kRowTile) {
      bool old = false;
      if (tid < nbot) {
        const int j = static_cast<int>(composite_index(U[nU - 1 - tid]));
        old = j <= r0;
        if (!old && j - r0 < kRowTile) sm.rowpos[j - r0] = static_cast<int16_t>(tid);
      }
      const uint32_t v = __ballot_sync(0xFFFFFFFFu, old);
      if (lane == 0) sm.oldmask[warp] = v;
    }
    __syncthreads();
    // tau of every row: the rank-th set bit of (old tail keys | tail keys new by this row)
    uint32_t vis[kRowTile / 32] = {0u, 0u, 0u, 0u};
    if (tid < kRowTile) {
      const int rp = sm.rowpos[tid];
      if (rp >= 0) vis[rp >> 5] = 1u << (rp & 31);
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
#pragma unroll
        for (int k = 0; k < kRowTile / 32; ++k) {
          const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, vis[k], d);
          if (lane >= d) vis[k] |= x;
        }
      }
      if (lane == 31) {
#pragma unroll
        for (int k = 0; k < kRowTile / 32; ++k) sm.wor[warp][k] = vis[k];
      }
    }
    __syncthreads();
    if (tid < nrows) {
      for (int ww = 0; ww < warp; ++ww) {
#pragma unroll
        for (int k = 0; k < kRowTile / 32; ++k) vis[k] |= sm.wor[ww][k];
      }
      const int ip = min(r0 + tid, len - 1);
      uint64_t tau = 0ull;
      int pos = -1;
      if (ip + 1 > w) {
        int rank = n_old + popc_upto(sm.newmask, ip - r0) - w + 1;
#pragma unroll
        for (int k = 0; k < kRowTile / 32; ++k) {
          const uint32_t v = vis[k] | sm.oldmask[k];
          const int c = __popc(v);
          if (pos < 0) {
            if (rank <= c) pos = 32 * k + nth_set_bit(v, rank);
            else rank -= c;
          }
        }
        if (pos < 0 || pos >= nbot) pos = nbot - 1;   // unreachable: every row's tau is a visible tail key
        tau = U[nU - 1 - pos];
      }
      tau_g[r0 + tid] = tau;
      sm.tau_s[tid] = tau;
      sm.pos_s[tid] = pos;
    }
    __syncthreads();

    // each tail key is kept up to the first row whose tau lies above it; the
    // tail decides the class sizes (a key above the tail is kept from its row
    // to the end of the tile): n_full = keys seen by every row minus those of
    // them evicted in the tile, the rest = newer keys kept by some row plus the
    // evicted ones
    if (tid < kRowTile) {
      bool ev_old = false, dead_new = false;
      if (tid < nbot) {
        int a = 0, c = nrows;
        while (a < c) {
          const int mid = (a + c) >> 1;
          if (sm.pos_s[mid] <= tid) a = mid + 1; else c = mid;
        }
        sm.hi_tail[tid] = static_cast<uint8_t>(a);
        const int j = static_cast<int>(composite_index(U[nU - 1 - tid]));
        const int lo = j > r0 ? j - r0 : 0;
        ev_old = lo == 0 && a < nrows;
        dead_new = lo > 0 && a <= lo;
      }
      const uint32_t v1 = __ballot_sync(0xFFFFFFFFu, ev_old), v2 = __ballot_sync(0xFFFFFFFFu, dead_new);
      if (lane == 0) {
        sm.cnt[0][warp] = __popc(v1);
        sm.cnt[1][warp] = __popc(v2);
      }
    }
    if (tid == 0) {
      sm.tot[2] = 0u;
      sm.tot[3] = 0u;
    }
    // the next tile's tau0: the w-th largest of K(q) = U[0, w) and the key of its first row
    uint64_t tau0n = 0ull;
    if (more) {
      const uint64_t tau_last = U[w - 1];
      tau0n = tau_last;
      if (p_next != q) {
        const uint64_t a2 = w >= 2 ? U[w - 2] : ~0ull;
        const uint64_t nk = sm.nextk;
        tau0n = nk < tau_last ? tau_last : (nk < a2 ? nk : a2);
      }
    }
    __syncthreads();
    int n_ev = 0, n_dead = 0;
#pragma unroll
    for (int k = 0; k < kRowTile / 32; ++k) {
      n_ev += static_cast<int>(sm.cnt[0][k]);
      n_dead += static_cast<int>(sm.cnt[1][k]);
    }
    const int n_lo0 = nU - static_cast<int>(__popc(sm.newmask[0]) + __popc(sm.newmask[1]) + __popc(sm.newmask[2]) +
                                              __popc(sm.newmask[3]));   // keys at or before r0
    const int n_full = n_lo0 - n_ev;
    const int n_total = n_full + (nU - n_lo0) - n_dead + n_ev;

    // the list: keys every row keeps, then the others.  Each warp takes a
    // contiguous segment of U, counts its keys of both classes, reserves room
    // for them with one atomic per class, then writes them.
    int32_t* stage = reinterpret_cast<int32_t*>(K);   // K is dead once U is built
    {
      const int seg = ((nU + nw - 1) / nw + 31) / 32 * 32;
      const int s0 = warp * seg, s1 = min(nU, s0 + seg);
      auto classify = [&](int e, uint64_t& key, int& lo, int& hi, bool& f, bool& pp) {
        key = U[e];
        const int j = static_cast<int>(composite_index(key));
        lo = j > r0 ? j - r0 : 0;
        const int s_ = nU - 1 - e;
        hi = s_ < nbot ? static_cast<int>(sm.hi_tail[s_]) : nrows;
        f = lo == 0 && hi == nrows;
        pp = !f && hi > lo;
      };
      uint32_t cf = 0, cp = 0;
      for (int j0 = s0; j0 < s1; j0 += 32) {
        const int e = j0 + lane;
        uint64_t key = 0ull;
        int lo = 0, hi = 0;
        bool f = false, pp = false;
        if (e < s1) classify(e, key, lo, hi, f, pp);
        cf += __popc(__ballot_sync(0xFFFFFFFFu, f));
        cp += __popc(__ballot_sync(0xFFFFFFFFu, pp));
      }
      uint32_t run_f = 0, run_p = 0;
      if (lane == 0) {
        if (cf) run_f = atomicAdd(&sm.tot[2], cf);
        if (cp) run_p = atomicAdd(&sm.tot[3], cp);
      }
      run_f = __shfl_sync(0xFFFFFFFFu, run_f, 0);
      run_p = __shfl_sync(0xFFFFFFFFu, run_p, 0) + static_cast<uint32_t>(n_full);
      for (int j0 = s0; j0 < s1; j0 += 32) {
        const int e = j0 + lane;
        uint64_t key = 0ull;
        int lo = 0, hi = 0;
        bool f = false, pp = false;
        if (e < s1) classify(e, key, lo, hi, f, pp);
        const uint32_t vf = __ballot_sync(0xFFFFFFFFu, f), vp = __ballot_sync(0xFFFFFFFFu, pp);
        if (f || pp) {
          const uint32_t pos = f ? run_f + __popc(vf & lt) : run_p + __popc(vp & lt);
          if (pos < static_cast<uint32_t>(ucap)) {
            const int j = static_cast<int>(composite_index(key));
            idx_o[pos] = j;
            bias_o[pos] = __uint_as_float(static_cast<uint32_t>(key >> 32));
            span_o[pos] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
            stage[pos] = j;
          }
        }
        run_f += __popc(vf);
        run_p += __popc(vp);
      }
    }
    const int padded = (n_total + kKeyTile - 1) / kKeyTile * kKeyTile;
    for (int j = n_total + tid; j < padded; j += blockDim.x) {
      idx_o[j] = 0;
      bias_o[j] = 0.0f;
      span_o[j] = 0u;
    }
    if (tid == 0) plan.counts[tile] = make_int2(n_full, n_total);
    __syncthreads();
    // key tiles whose listed keys are one ascending run j0, j0+1, ... can be
    // fetched with a single box copy instead of a row gather
    int32_t* kb = plan.kbase + tile * (plan.cap / kKeyTile);
    for (int kt = warp; kt * kKeyTile < n_total; kt += nw) {
      const int e0 = kt * kKeyTile;
      const int j0 = stage[e0];
      bool ok = true;
      for (int e = e0 + lane; e < min(n_total, e0 + kKeyTile); e += 32) ok &= stage[e] == j0 + (e - e0);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (lane == 0) kb[kt] = ok ? j0 : -1;
    }
    __syncthreads();   // the stage (in K's buffer) is read before the next tile writes there

    // carried to the next tile: K(q) = U[0, w) and its tau0
    tau0 = tau0n;
    q_prev = q;
    pre_bits = pre_next;
    cur ^= 1;
    have = more;
  }
}

// decode selector CTA: threads, and CTAs resident per SM (64 registers a thread)
constexpr int kSelDecodeThreads = 256;
constexpr int kSelDecodeMinBlocks = 4;

// One CTA per (batch, kv head).  dt of a long cache row is read from memory,
// not from L2, so passes over it count: a sampled threshold lets one pass
// collect about 3/2 w keys that surely hold the w kept ones, which are then
// selected in shared memory and written from there.  When the sample misjudges
// (fewer than w or more than the buffer), three passes select exactly (which
// bits vary, an 11-bit histogram, one collection of the keys in and above the
// w-th largest's bin), and rows whose keys crowd one bin select and compact in
// two more.
__global__ void __launch_bounds__(kSelDecodeThreads, kSelDecodeMinBlocks) select_decode_kernel(const float* __restrict__ dt,
                                                                    const int32_t* __restrict__ lengths, int Hkv,
                                                                    int Lk, int w, DecodePlan plan, uint32_t* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  SelScratch sc{sm.hist, sm.cand, sm.red, sm.vars};
  pdl_wait();      // dt comes from the previous kernel
  pdl_trigger();   // the decode attention may be scheduled
  const int g = blockIdx.x, b = blockIdx.y;
  const int len = clamp_len(lengths, b, Lk, err);
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(dt) + bg * Lk;
  int32_t* idx_o = plan.idx + bg * plan.cap;
  float* bias_o = plan.bias + bg * plan.cap;
  const int tid = threadIdx.x;
  int n;
  uint64_t tau = 0ull;
  int c = -1;
  unsigned long long* ctr = reinterpret_cast<unsigned long long*>(&sm.vars[6]);
  if (Lk > w && len > w) c = sampled_collect(bits, len, w, sm.cand, kCandCap, sc, ctr);
  if (c >= w) {
    // the w-th largest among the collected keys (the zero padding ranks last),
    // then the keys at or above it
    c = kCandCap;
    tau = select_kth_smem(sm.cand, c, static_cast<uint32_t>(w), sc);
    if (tid == 0) *ctr = 0ull;
    __syncthreads();
    const uint32_t lane = lane_id(), lt = lanemask_lt();
    for (int e0 = 0; e0 < c; e0 += blockDim.x) {   // same trip count in every thread
      const int e = e0 + tid;
      const uint64_t key = e < c ? sm.cand[e] : 0ull;
      const bool keep = e < c && key >= tau;
      const uint32_t vote = __ballot_sync(0xFFFFFFFFu, keep);
      uint32_t base = 0;
      if (lane == 0 && vote) base = static_cast<uint32_t>(atomicAdd(ctr, static_cast<unsigned long long>(__popc(vote))));
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
      if (keep) {
        const uint32_t pos = base + __popc(vote & lt);
        idx_o[pos] = static_cast<int32_t>(composite_index(key));
        bias_o[pos] = __uint_as_float(static_cast<uint32_t>(key >> 32));
      }
    }
    n = w;
  } else if (Lk > w && len > w && prefix_topw(bits, len, w, sm.cand, kCandCap, sc, ctr, &tau)) {
    n = w;
    for (int e = tid; e < w; e += blockDim.x) {
      const uint64_t key = sm.cand[e];
      idx_o[e] = static_cast<int32_t>(composite_index(key));
      bias_o[e] = __uint_as_float(static_cast<uint32_t>(key >> 32));
    }
  } else if (Lk > w && len > w) {
    tau = select_kth_global(bits, len, static_cast<uint32_t>(w), sc);
    n = ordered_compact_row(
        bits, len, [&](uint32_t v, int j) { return composite_key(v, j) >= tau; },
        [&](int pos, int j, uint32_t v) {
          idx_o[pos] = j;
          bias_o[pos] = __uint_as_float(v);
        },
        sc);
  } else {
    n = len;
    for (int j = tid; j < len; j += blockDim.x) {
      idx_o[j] = j;
      bias_o[j] = __uint_as_float(bits[j]);
    }
  }
  const int padded = (n + kDecodeChunk - 1) / kDecodeChunk * kDecodeChunk;
  for (int j = n + tid; j < padded; j += blockDim.x) {
    idx_o[j] = 0;
    bias_o[j] = 0.0f;
  }
  if (tid == 0) {
    plan.count[bg] = n;
    plan.tau[bg] = tau;
  }
}

// Dense bitmask [B, Hkv, L, ceil(L/32)] from the prefill plan (tests/debug).
__global__ void prefill_bitmask_kernel(PrefillPlan plan, int Hkv, int L, uint32_t* bm) {
  const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const size_t tile = bg * plan.n_row_tiles + t;
  const int words = (L + 31) / 32;
  const int2 cnt = plan.counts[tile];
  const int r0 = t * kRowTile;
  for (int e = threadIdx.x; e < cnt.y; e += blockDim.x) {
    const int j = plan.idx[tile * plan.cap + e];
    const uint32_t sp = plan.span[tile * plan.cap + e];
    const int lo = sp & 0xFFFF, hi = sp >> 16;
    for (int r = lo; r < hi; ++r)
      atomicOr(&bm[(bg * L + r0 + r) * words + (j >> 5)], 1u << (j & 31));
  }
}

__global__ void decode_bitmask_kernel(DecodePlan plan, int Hkv, int Lk, uint32_t* bm) {
  const int g = blockIdx.x, b = blockIdx.y;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const int words = (Lk + 31) / 32;
  const int n = plan.count[bg];
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int j = plan.idx[bg * plan.cap + e];
    atomicOr(&bm[bg * words + (j >> 5)], 1u << (j & 31));
  }
}

size_t select_smem_bytes() { return sizeof(SelectSmem); }

// prefill: the static part, then two key buffers of ucap keys (which also
// hold the candidates of the prefix selection)
size_t select_prefill_smem_bytes(int ucap) {
  const size_t keys = static_cast<size_t>(ucap) * 2 > static_cast<size_t>(kCandCap) ? static_cast<size_t>(ucap) * 2
                                                                                     : static_cast<size_t>(kCandCap);
  return sizeof(PrefillSelSmem) + keys * sizeof(uint64_t);
}

}  // namespace

cudaError_t launch_select_prefill(const float* dt, const int32_t* lengths, const Geometry& g,
                                  const PrefillPlan& plan, uint32_t* err, cudaStream_t s) {
  const int L = g.Lk;
  const int ucap = L > g.w ? g.w + kRowTile : 0;
  const size_t smem = select_prefill_smem_bytes(ucap);
  const bool long_rows = plan.n_row_tiles >= kSelLongRowTiles;
  const void* kfn = long_rows
                        ? reinterpret_cast<const void*>(select_prefill_kernel<kSelPrefillThreadsLong, kSelPrefillMinBlocksLong>)
                        : reinterpret_cast<const void*>(select_prefill_kernel<kSelPrefillThreads, kSelPrefillMinBlocks>);
  cudaError_t e = ensure_dyn_smem(kfn, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // row tiles per CTA: a run's first tile selects over its prefix and sorts
  // its kept set, every later one only merges its new keys, so runs should be
  // long; the grid should still fill one wave of resident CTAs with the tiles
  // that need the top-k (rows below keep_window_size keep every visible key
  // and cost little).  Measured on the sparse and long workloads: 3 and 8
  // tiles per CTA with 512-thread CTAs (this rule gives 3 and 7); the long
  // workload's 256-thread CTAs get 5.
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const long long free_tiles = L > g.w ? std::min<long long>(plan.n_row_tiles, g.w / kRowTile) : plan.n_row_tiles;
  const long long topk_tiles = (static_cast<long long>(plan.n_row_tiles) - free_tiles) * g.Hkv * g.B;
  const long long slots =
      static_cast<long long>(long_rows ? kSelPrefillMinBlocksLong : kSelPrefillMinBlocks) * nsm;
  long long tpc = (topk_tiles + slots - 1) / slots;
  tpc = tpc < 1 ? 1 : (tpc > kSelTilesPerCtaMax ? kSelTilesPerCtaMax : tpc);
  dim3 grid(g.Hkv, g.B, static_cast<unsigned>((plan.n_row_tiles + tpc - 1) / tpc));
  if (long_rows)
    return launch_after(select_prefill_kernel<kSelPrefillThreadsLong, kSelPrefillMinBlocksLong>, grid,
                        dim3(kSelPrefillThreadsLong), smem, s, dt, lengths, g.Hkv, L, g.w, static_cast<int>(tpc), plan,
                        err);
  return launch_after(select_prefill_kernel<kSelPrefillThreads, kSelPrefillMinBlocks>, grid, dim3(kSelPrefillThreads),
                      smem, s, dt, lengths, g.Hkv, L, g.w, static_cast<int>(tpc), plan, err);
}

cudaError_t launch_select_decode(const float* dt, const int32_t* lengths, const Geometry& g,
                                 const DecodePlan& plan, uint32_t* err, cudaStream_t s) {
  const size_t smem = select_smem_bytes();
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(select_decode_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(g.Hkv, g.B);
  return launch_after(select_decode_kernel, grid, dim3(kSelDecodeThreads), smem, s, dt, lengths, g.Hkv, g.Lk, g.w, plan,
                      err);
}

cudaError_t launch_prefill_bitmask(const PrefillPlan& plan, const Geometry& g, uint32_t* bitmask, cudaStream_t s) {
  dim3 grid(plan.n_row_tiles, g.Hkv, g.B);
  prefill_bitmask_kernel<<<grid, 256, 0, s>>>(plan, g.Hkv, g.Lk, bitmask);
  return cudaGetLastError();
}

cudaError_t launch_decode_bitmask(const DecodePlan& plan, const Geometry& g, uint32_t* bitmask, cudaStream_t s) {
  dim3 grid(g.Hkv, g.B);
  decode_bitmask_kernel<<<grid, 256, 0, s>>>(plan, g.Hkv, g.Lk, bitmask);
  return cudaGetLastError();
}

}  // namespace dma
