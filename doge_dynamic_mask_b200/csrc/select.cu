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
// kept on one contiguous interval of rows, and the union of the kept sets of a
// row tile is the w keys kept at its first row plus at most 127 newer keys.
// For each tile of its run the CTA
//   1. finds tau at the tile's first row: by radix selection over the keys
//      that row sees (the run's first tile), or from the previous tile's
//      last-row kept set plus at most one new key (every later tile),
//   2. collects the union U (keys <= the tile's last visible row whose key is
//      >= that tau) in index order: from the prefix in global memory, or from
//      the previous tile's union and the tile's own new keys,
//   3. takes the 128 smallest keys of U, in which every later row's tau lies,
//      and resolves tau_i for each row of the tile,
//   4. gives each key of U its row interval [lo, hi) inside the tile and writes
//      the list: keys kept by every row first, then the rest (index order in
//      each class), each with its dt bias and interval.
// Tiles whose rows see at most w keys (and every tile when Lk <= w) keep
// every visible key and skip the selection.
//
// Decode (one CTA per (batch, kv head)): the single query at len_b - 1 keeps
// the w best of its len_b keys; radix-select the w-th key, then compact the
// kept keys in index order.
#include "select_common.cuh"

namespace dma {
namespace {

struct SelectSmem {
  uint32_t hist[kBins];
  uint64_t cand[kCandCap];
  uint32_t red[64];
  uint64_t vars[8];
  uint64_t tau_s[kRowTile];
  uint64_t bot[kRowTile];
  uint64_t bot_raw[kRowTile];
  int misc[8];
  // followed by two unions U[ucap] (uint64) in dynamic shared memory
};

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

// Minimum of the keys of U[0, n) above `floor` (~0 when there is none).
__device__ __forceinline__ uint64_t block_min_above(const uint64_t* U, int n, uint64_t floor, uint64_t* scratch) {
  uint64_t m = ~0ull;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const uint64_t k = U[e];
    if (k > floor && k < m) m = k;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const uint64_t x = __shfl_xor_sync(0xFFFFFFFFu, m, o);
    m = x < m ? x : m;
  }
  const int warp = threadIdx.x >> 5;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) scratch[warp] = m;
  __syncthreads();
  uint64_t r = ~0ull;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) r = scratch[w] < r ? scratch[w] : r;
  __syncthreads();
  return r;
}

// One CTA per (batch, kv head, run of tpc consecutive row tiles).
// The first tile of the run whose rows need the top-k does the full
// selection over its prefix.  Each following tile is derived from the one
// before, in shared memory: the kept set at the previous tile's last visible
// row K(q') (the w keys of the previous union U' at or above that row's tau)
// plus at most one new key (the tile's first row, when it is a valid row)
// gives the tile's first-row threshold as the w-th largest of w+1 keys, and
// the new union is U' filtered by that threshold followed by the tile's own
// new keys (q', q] that pass it.
__global__ void __launch_bounds__(kSelThreads, 2) select_prefill_kernel(const float* __restrict__ dt,
                                                                     const int32_t* __restrict__ lengths, int Hkv,
                                                                     int L, int w, int tpc, PrefillPlan plan,
                                                                     uint32_t* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelectSmem& sm = *reinterpret_cast<SelectSmem*>(smem_raw);
  pdl_wait();      // dt comes from the previous kernel
  pdl_trigger();   // the attention may be scheduled
  const int ucap = w + kRowTile;
  uint64_t* Ubuf = reinterpret_cast<uint64_t*>(smem_raw + sizeof(SelectSmem));   // two unions of ucap keys
  SelScratch sc{sm.hist, sm.cand, sm.red, sm.vars};

  const int g = blockIdx.y, b = blockIdx.z;
  const int len = clamp_len(lengths, b, L, err);
  const bool topk = L > w;
  const size_t bg = static_cast<size_t>(b) * Hkv + g;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(dt) + bg * L;
  uint64_t* tau_g = plan.tau + bg * L;
  const int tid = threadIdx.x;
  const int t_first = blockIdx.x * tpc;
  const int t_last = min(plan.n_row_tiles, t_first + tpc);
  bool have = false;      // the previous tile's union and last-row tau carry over
  int cur = 0;            // buffer holding the previous tile's union
  int nU_prev = 0, q_prev = 0;
  uint64_t tau_last = 0ull;

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

    uint64_t* U = Ubuf + (cur ^ 1) * ucap;
    int nU;
    if (have) {
      // 1. threshold at the first row from the previous tile's last kept set
      const uint64_t* Up = Ubuf + cur * ucap;
      uint64_t tau0 = tau_last;
      if (p != q_prev) {   // p == q_prev + 1: one new key competes
        const uint64_t nk = composite_key(bits[p], static_cast<uint32_t>(p));
        const uint64_t a2 = block_min_above(Up, nU_prev, tau_last, sm.bot_raw);   // second worst kept key
        tau0 = nk < tau_last ? tau_last : (nk < a2 ? nk : a2);
      }
      // 2. the union: kept keys of the previous union, then the new keys (q_prev, q]
      const int n_new = q - q_prev;
      nU = ordered_compact(
          nU_prev + n_new,
          [&](int e) {
            const uint64_t k = e < nU_prev ? Up[e]
                                           : composite_key(bits[q_prev + 1 + (e - nU_prev)],
                                                           static_cast<uint32_t>(q_prev + 1 + (e - nU_prev)));
            return k >= tau0;
          },
          [&](int pos, int e) {
            U[pos] = e < nU_prev ? Up[e]
                                 : composite_key(bits[q_prev + 1 + (e - nU_prev)],
                                                 static_cast<uint32_t>(q_prev + 1 + (e - nU_prev)));
          },
          sc);
    } else {
      // 1. threshold at the first row over its prefix
      uint64_t tau0 = 0ull;
      if (p + 1 > w) tau0 = select_kth_global(bits, p + 1, static_cast<uint32_t>(w), sc);
      // 2. the union U of kept keys, in index order
      nU = ordered_compact_row(
          bits, q + 1, [&](uint32_t v, int j) { return composite_key(v, j) >= tau0; },
          [&](int pos, int j, uint32_t v) { U[pos] = composite_key(v, j); }, sc);
    }
    __syncthreads();
    const int n_old = p + 1 > w ? w : p + 1;

    // 3. the kRowTile smallest keys of U, ascending; then tau for every row
    const int nbot = min(nU, kRowTile);
    uint64_t sigma = ~0ull;
    if (nU > kRowTile) sigma = select_kth_smem(U, nU, static_cast<uint32_t>(nU - kRowTile + 1), sc);
    if (tid == 0) sm.misc[0] = 0;
    __syncthreads();
    for (int e = tid; e < nU; e += blockDim.x) {
      if (U[e] <= sigma) {
        const int pos = atomicAdd(&sm.misc[0], 1);
        if (pos < kRowTile) sm.bot_raw[pos] = U[e];
      }
    }
    __syncthreads();
    if (tid < nbot) {
      const uint64_t key = sm.bot_raw[tid];
      int rank = 0;
      for (int f = 0; f < nbot; ++f) rank += sm.bot_raw[f] < key;
      sm.bot[rank] = key;
    }
    __syncthreads();
    if (tid < kRowTile) {
      uint64_t tau = ~0ull;   // rows past the end of the sequence axis: unused
      if (tid < nrows) {
        const int ip = min(r0 + tid, len - 1);
        if (ip + 1 <= w) {
          tau = 0ull;
        } else {
          // keys of U visible to this row: the n_old old keys plus new keys j <= ip
          int lo = n_old, hi = nU;
          while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (static_cast<int>(composite_index(U[mid])) <= ip) lo = mid + 1; else hi = mid;
          }
          const int rank = lo - w + 1;   // ascending rank of the row's w-th best key
          int c = 0;
          tau = 0ull;
          for (int e = 0; e < nbot; ++e) {
            const uint64_t key = sm.bot[e];
            if (static_cast<int>(composite_index(key)) <= ip && ++c == rank) {
              tau = key;
              break;
            }
          }
        }
        tau_g[r0 + tid] = tau;
      }
      sm.tau_s[tid] = tau;
    }
    __syncthreads();

    // 4. row intervals and the two-class ordered list
    const int per = (nU + blockDim.x - 1) / blockDim.x;
    const int e0 = tid * per, e1 = min(nU, e0 + per);
    uint32_t nf = 0, np = 0;
    for (int e = e0; e < e1; ++e) {
      const uint64_t key = U[e];
      const int j = static_cast<int>(composite_index(key));
      const int lo = j > r0 ? j - r0 : 0;
      int a = 0, c = nrows;   // first row whose tau exceeds the key
      while (a < c) {
        const int mid = (a + c) >> 1;
        if (sm.tau_s[mid] > key) c = mid; else a = mid + 1;
      }
      const int hi = a;
      if (hi > lo) {
        if (lo == 0 && hi == nrows) ++nf; else ++np;
      }
    }
    uint32_t total;
    const uint32_t base = block_exclusive_scan(nf | (np << 16), sm.red, &total);
    const int n_full = static_cast<int>(total & 0xFFFFu);
    const int n_total = n_full + static_cast<int>(total >> 16);
    uint32_t pf = base & 0xFFFFu, pp = n_full + (base >> 16);
    for (int e = e0; e < e1; ++e) {
      const uint64_t key = U[e];
      const int j = static_cast<int>(composite_index(key));
      const int lo = j > r0 ? j - r0 : 0;
      int a = 0, c = nrows;
      while (a < c) {
        const int mid = (a + c) >> 1;
        if (sm.tau_s[mid] > key) c = mid; else a = mid + 1;
      }
      const int hi = a;
      if (hi > lo) {
        const uint32_t pos = (lo == 0 && hi == nrows) ? pf++ : pp++;
        idx_o[pos] = j;
        bias_o[pos] = __uint_as_float(static_cast<uint32_t>(key >> 32));
        span_o[pos] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
      }
    }
    const int padded = (n_total + kKeyTile - 1) / kKeyTile * kKeyTile;
    for (int j = n_total + tid; j < padded; j += blockDim.x) {
      idx_o[j] = 0;
      bias_o[j] = 0.0f;
      span_o[j] = 0u;
    }
    if (tid == 0) plan.counts[tile] = make_int2(n_full, n_total);
    // key tiles whose listed keys are one ascending run j0, j0+1, ... can be
    // fetched with a single box copy instead of a row gather
    __syncthreads();
    int32_t* kb = plan.kbase + tile * (plan.cap / kKeyTile);
    const int lane = tid & 31;
    for (int kt = tid >> 5; kt * kKeyTile < n_total; kt += blockDim.x >> 5) {
      const int e0 = kt * kKeyTile;
      const int j0 = idx_o[e0];
      bool ok = true;
      for (int e = e0 + lane; e < min(n_total, e0 + kKeyTile); e += 32) ok &= idx_o[e] == j0 + (e - e0);
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (lane == 0) kb[kt] = ok ? j0 : -1;
    }

    // carried to the next tile: this union and the tau of its last visible row
    tau_last = sm.tau_s[nrows - 1];
    nU_prev = nU;
    q_prev = q;
    cur ^= 1;
    have = true;
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kSelThreads, 4) select_decode_kernel(const float* __restrict__ dt,
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
  if (Lk > w && len > w) {
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

size_t select_smem_bytes(int ucap) { return sizeof(SelectSmem) + static_cast<size_t>(ucap) * sizeof(uint64_t); }

}  // namespace

cudaError_t launch_select_prefill(const float* dt, const int32_t* lengths, const Geometry& g,
                                  const PrefillPlan& plan, uint32_t* err, cudaStream_t s) {
  const int L = g.Lk;
  const int ucap = L > g.w ? g.w + kRowTile : 0;
  const size_t smem = select_smem_bytes(2 * ucap);
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(select_prefill_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  // row tiles per CTA: runs amortise the full selection, but the grid should
  // still hold about four CTAs per SM (measured on the sparse and long
  // workloads: 2 and 4 tiles per CTA); rows of 8 tiles or more use runs of at
  // least 2
  const int nsm = sm_count();
  if (nsm <= 0) return cudaErrorInvalidDevice;
  const long long tiles = static_cast<long long>(plan.n_row_tiles) * g.Hkv * g.B;
  long long tpc = (tiles + 4LL * nsm - 1) / (4LL * nsm);
  if (plan.n_row_tiles >= 8 && tpc < 2) tpc = 2;
  tpc = tpc < 1 ? 1 : (tpc > kSelTilesPerCtaMax ? kSelTilesPerCtaMax : tpc);
  dim3 grid(static_cast<unsigned>((plan.n_row_tiles + tpc - 1) / tpc), g.Hkv, g.B);
  return launch_after(select_prefill_kernel, grid, dim3(kSelThreads), smem, s, dt, lengths, g.Hkv, L, g.w,
                      static_cast<int>(tpc), plan, err);
}

cudaError_t launch_select_decode(const float* dt, const int32_t* lengths, const Geometry& g,
                                 const DecodePlan& plan, uint32_t* err, cudaStream_t s) {
  const size_t smem = select_smem_bytes(0);
  cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(select_decode_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(g.Hkv, g.B);
  return launch_after(select_decode_kernel, grid, dim3(kSelThreads), smem, s, dt, lengths, g.Hkv, g.Lk, g.w, plan,
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
