// Block-level selection primitives for the dynamic-mask top-k.
//
// Keys are the 64-bit composite (bits(dt) << 32) | (0xFFFFFFFF - j): dt >= 0,
// so the float32 bit pattern orders like the value, and on equal dt the lower
// key index ranks higher.  Every key is distinct, so "the k-th largest key" is
// unique and the kept set of a row is exactly {j : key_j >= that key}.
//
// select_kth_global finds the k-th largest key over a dt row held in global
// memory by most-significant-digit radix selection: bits common to every
// candidate are skipped, 11-bit digits are histogrammed in shared memory, and
// once the candidates fit kCandCap they are compacted into shared memory and
// the remaining digits (down into the index bits) are resolved there.  A row
// whose candidates still exceed kCandCap after all 32 dt bits are fixed
// (massive exact ties, e.g. A = 0 gives dt == 1 everywhere) is resolved by an
// ordered count of the tied indices.
#pragma once

#include "common.cuh"

namespace dma {

constexpr int kSelThreads = 512;
constexpr int kBins = 2048;      // 11-bit digits
constexpr int kCandCap = 5632;   // shared-memory candidate buffer (704 keys per warp of a 256-thread CTA)

struct SelScratch {
  uint32_t* hist;   // [kBins]
  uint64_t* cand;   // [kCandCap]
  uint32_t* red;    // [64]
  uint64_t* vars;   // [8]
};

__device__ __forceinline__ bool hi_match(uint64_t x, uint64_t p, int hb) {
  // bits above position hb agree (hb = 63: nothing fixed yet)
  return hb >= 63 ? true : ((x >> (hb + 1)) == (p >> (hb + 1)));
}

__device__ __forceinline__ void block_or_and64(uint64_t vor, uint64_t vand, uint32_t* red, uint64_t& out_or,
                                               uint64_t& out_and) {
  const uint32_t lane = lane_id(), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t o_lo = __reduce_or_sync(0xFFFFFFFFu, static_cast<uint32_t>(vor));
  uint32_t o_hi = __reduce_or_sync(0xFFFFFFFFu, static_cast<uint32_t>(vor >> 32));
  uint32_t a_lo = __reduce_and_sync(0xFFFFFFFFu, static_cast<uint32_t>(vand));
  uint32_t a_hi = __reduce_and_sync(0xFFFFFFFFu, static_cast<uint32_t>(vand >> 32));
  __syncthreads();
  if (lane == 0) {
    red[warp * 4 + 0] = o_lo;
    red[warp * 4 + 1] = o_hi;
    red[warp * 4 + 2] = a_lo;
    red[warp * 4 + 3] = a_hi;
  }
  __syncthreads();
  uint32_t ol = 0, oh = 0, al = 0xFFFFFFFFu, ah = 0xFFFFFFFFu;
  for (uint32_t w = 0; w < nw; ++w) {
    ol |= red[w * 4 + 0];
    oh |= red[w * 4 + 1];
    al &= red[w * 4 + 2];
    ah &= red[w * 4 + 3];
  }
  out_or = (static_cast<uint64_t>(oh) << 32) | ol;
  out_and = (static_cast<uint64_t>(ah) << 32) | al;
  __syncthreads();
}

// Given hist[0, nb), find bin B with  sum_{b > B} hist[b] < k <= sum_{b >= B} hist[b].
// Returns B; *k_in_bin = k - sum_{b > B} hist[b]; *bin_count = hist[B].
__device__ __forceinline__ uint32_t find_bin_from_top(const uint32_t* hist, int nb, uint32_t k, uint32_t* red,
                                                      uint64_t* vars, uint32_t* k_in_bin, uint32_t* bin_count) {
  const int per = (nb + blockDim.x - 1) / blockDim.x;
  const int hi = nb - static_cast<int>(threadIdx.x) * per;        // exclusive
  const int lo = hi - per;
  uint32_t local = 0;
  for (int b = hi - 1; b >= lo; --b)
    if (b >= 0 && b < nb) local += hist[b];
  uint32_t total;
  const uint32_t above = block_exclusive_scan(local, red, &total);
  if (above < k && above + local >= k) {
    uint32_t acc = above;
    for (int b = hi - 1; b >= lo; --b) {
      if (b < 0 || b >= nb) continue;
      const uint32_t h = hist[b];
      if (acc + h >= k) {
        vars[0] = static_cast<uint64_t>(b);
        vars[1] = static_cast<uint64_t>(k - acc);
        vars[2] = static_cast<uint64_t>(h);
        break;
      }
      acc += h;
    }
  }
  __syncthreads();
  const uint32_t B = static_cast<uint32_t>(vars[0]);
  *k_in_bin = static_cast<uint32_t>(vars[1]);
  *bin_count = static_cast<uint32_t>(vars[2]);
  __syncthreads();
  return B;
}

// k-th largest (1-based) of n distinct keys held in shared memory.
static __device__ __noinline__ uint64_t select_kth_smem(const uint64_t* keys, int n, uint32_t k, SelScratch sc) {
  uint64_t vor = 0, vand = ~0ull;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    vor |= keys[e];
    vand &= keys[e];
  }
  uint64_t O, A;
  block_or_and64(vor, vand, sc.red, O, A);
  const uint64_t vary = O ^ A;
  int hb = vary ? 63 - __clzll(static_cast<long long>(vary)) : -1;
  uint64_t prefix = hb < 0 ? A : (hb >= 63 ? 0ull : (A & ~((2ull << hb) - 1ull)));
  uint32_t count = static_cast<uint32_t>(n);
  while (count > 1 && hb >= 0) {
    const int s = hb >= 10 ? hb - 10 : 0;
    const int nb = 1 << (hb - s + 1);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) sc.hist[i] = 0;
    __syncthreads();
    for (int e = threadIdx.x; e < n; e += blockDim.x) {
      const uint64_t key = keys[e];
      if (hi_match(key, prefix, hb)) atomicAdd(&sc.hist[(key >> s) & static_cast<uint64_t>(nb - 1)], 1u);
    }
    __syncthreads();
    uint32_t kk, cnt;
    const uint32_t B = find_bin_from_top(sc.hist, nb, k, sc.red, sc.vars, &kk, &cnt);
    k = kk;
    count = cnt;
    prefix |= static_cast<uint64_t>(B) << s;
    hb = s - 1;
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const uint64_t key = keys[e];
    if (hi_match(key, prefix, hb)) sc.vars[3] = key;
  }
  __syncthreads();
  const uint64_t r = sc.vars[3];
  __syncthreads();
  return r;
}

// Index of the k-th (1-based) position j in [0, n) with bits[j] == val, in increasing j.
static __device__ __noinline__ int kth_matching_index(const uint32_t* __restrict__ bits, int n, uint32_t val, uint32_t k,
                                               SelScratch sc) {
  const uint32_t lane = lane_id(), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int seg = ((n + nw - 1) / nw + 31) / 32 * 32;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);
  uint32_t cnt = 0;
  for (int j0 = s0; j0 < s1; j0 += 32) {
    const int j = j0 + lane;
    const bool m = j < s1 && bits[j] == val;
    cnt += __popc(__ballot_sync(0xFFFFFFFFu, m));
  }
  if (lane == 0) sc.red[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t acc = 0;
    for (uint32_t w = 0; w < nw; ++w) {
      if (acc + sc.red[w] >= k) {
        sc.vars[4] = w;
        sc.vars[5] = k - acc;
        break;
      }
      acc += sc.red[w];
    }
  }
  __syncthreads();
  if (warp == sc.vars[4]) {
    const uint32_t kl = static_cast<uint32_t>(sc.vars[5]);
    uint32_t run = 0;
    for (int j0 = s0; j0 < s1; j0 += 32) {
      const int j = j0 + lane;
      const bool m = j < s1 && bits[j] == val;
      uint32_t mask = __ballot_sync(0xFFFFFFFFu, m);
      const uint32_t c = __popc(mask);
      if (run + c >= kl) {
        for (uint32_t r = run + 1; r < kl; ++r) mask &= mask - 1;  // drop the lower matches
        if (lane == 0) sc.vars[6] = static_cast<uint64_t>(j0 + __ffs(mask) - 1);
        break;
      }
      run += c;
    }
  }
  __syncthreads();
  const int r = static_cast<int>(sc.vars[6]);
  __syncthreads();
  return r;
}

// Visits every position j in [0, n) of a dt row as f(bits, j, valid), each
// thread a strided subset.  A 16-byte-aligned row is read four keys per 16-byte
// load, four loads in flight per thread, so a pass over a long row is limited by
// bandwidth rather than by one load's latency per key.  Every thread of the
// block makes the same number of calls (valid = false past the end), so f may
// use warp-wide votes.
template <class F>
__device__ __forceinline__ void row_for_each(const uint32_t* __restrict__ bits, int n, F&& f) {
  const int tid = threadIdx.x, nt = blockDim.x;
  int done = 0;
  if ((reinterpret_cast<uintptr_t>(bits) & 15u) == 0) {
    const int nq = n >> 2;
    const uint4* q = reinterpret_cast<const uint4*>(bits);
    for (int r0 = 0; r0 < nq; r0 += 4 * nt) {   // same trip count in every thread
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = r0 + u * nt + tid;
        v[u] = i < nq ? __ldg(q + i) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = r0 + u * nt + tid;
        const bool ok = i < nq;
        f(v[u].x, 4 * i, ok);
        f(v[u].y, 4 * i + 1, ok);
        f(v[u].z, 4 * i + 2, ok);
        f(v[u].w, 4 * i + 3, ok);
      }
    }
    done = nq << 2;
  }
  for (int j0 = done; j0 < n; j0 += nt) {
    const int j = j0 + tid;
    const bool ok = j < n;
    f(ok ? __ldg(bits + j) : 0u, j, ok);
  }
}

// k-th largest composite key (1 <= k <= n) among positions [0, n) of a dt row.
static __device__ __noinline__ uint64_t select_kth_global(const uint32_t* __restrict__ bits, int n, uint32_t k,
                                                   SelScratch sc) {
  uint32_t vor = 0u, vand = ~0u;
  row_for_each(bits, n, [&](uint32_t b, int, bool ok) {
    if (ok) {
      vor |= b;
      vand &= b;
    }
  });
  uint64_t O, A;
  block_or_and64(vor, vand, sc.red, O, A);
  O &= 0xFFFFFFFFull;
  A &= 0xFFFFFFFFull;
  const uint64_t vary = O ^ A;
  int hb = vary ? 63 - __clzll(static_cast<long long>(vary)) : -1;   // <= 31
  uint64_t prefix = hb >= 0 ? (A & ~((2ull << hb) - 1ull)) : A;
  uint32_t count = static_cast<uint32_t>(n);
  while (hb >= 0 && count > static_cast<uint32_t>(kCandCap)) {
    const int s = hb >= 10 ? hb - 10 : 0;
    const int nb = 1 << (hb - s + 1);
    for (int i = threadIdx.x; i < nb; i += blockDim.x) sc.hist[i] = 0;
    __syncthreads();
    row_for_each(bits, n, [&](uint32_t b, int, bool ok) {
      if (ok && hi_match(b, prefix, hb)) atomicAdd(&sc.hist[(b >> s) & static_cast<uint32_t>(nb - 1)], 1u);
    });
    __syncthreads();
    uint32_t kk, cnt;
    const uint32_t B = find_bin_from_top(sc.hist, nb, k, sc.red, sc.vars, &kk, &cnt);
    k = kk;
    count = cnt;
    prefix |= static_cast<uint64_t>(B) << s;
    hb = s - 1;
  }
  if (count <= static_cast<uint32_t>(kCandCap)) {
    if (threadIdx.x == 0) sc.vars[7] = 0;
    __syncthreads();
    // candidates appended with one shared-memory atomic per warp and vote
    const uint32_t lane = lane_id();
    row_for_each(bits, n, [&](uint32_t b, int j, bool ok) {
      const bool m = ok && hi_match(b, prefix, hb);
      const uint32_t vote = __ballot_sync(0xFFFFFFFFu, m);
      if (vote) {
        uint32_t base = 0;
        if (lane == 0) base = static_cast<uint32_t>(
            atomicAdd(reinterpret_cast<unsigned long long*>(&sc.vars[7]), static_cast<unsigned long long>(__popc(vote))));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        if (m) {
          const uint32_t pos = base + __popc(vote & lanemask_lt());
          if (pos < static_cast<uint32_t>(kCandCap)) sc.cand[pos] = composite_key(b, j);
        }
      }
    });
    __syncthreads();
    const int c = static_cast<int>(sc.vars[7]);
    __syncthreads();
    return select_kth_smem(sc.cand, c, k, sc);
  }
  // every candidate has dt bits == prefix; the lower index ranks higher
  const int j = kth_matching_index(bits, n, static_cast<uint32_t>(prefix), k, sc);
  return composite_key(static_cast<uint32_t>(prefix), static_cast<uint32_t>(j));
}

// Stable compaction of the positions j in [0, n) with pred(j): emit(pos, j) for
// pos = 0, 1, ... in increasing j.  Returns the count.  Every thread must call it.
template <class Pred, class Emit>
__device__ __forceinline__ int ordered_compact(int n, Pred pred, Emit emit, SelScratch sc) {
  const uint32_t lane = lane_id(), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int seg = ((n + nw - 1) / nw + 31) / 32 * 32;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);
  uint32_t cnt = 0;
  for (int j0 = s0; j0 < s1; j0 += 32) {
    const int j = j0 + lane;
    cnt += __popc(__ballot_sync(0xFFFFFFFFu, j < s1 && pred(j)));
  }
  __syncthreads();
  if (lane == 0) sc.red[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t acc = 0;
    for (uint32_t w = 0; w < nw; ++w) {
      const uint32_t c = sc.red[w];
      sc.red[w] = acc;
      acc += c;
    }
    sc.red[32] = acc;
  }
  __syncthreads();
  uint32_t run = sc.red[warp];
  for (int j0 = s0; j0 < s1; j0 += 32) {
    const int j = j0 + lane;
    const bool p = j < s1 && pred(j);
    const uint32_t m = __ballot_sync(0xFFFFFFFFu, p);
    if (p) emit(static_cast<int>(run + __popc(m & lanemask_lt())), j);
    run += __popc(m);
  }
  const int total = static_cast<int>(sc.red[32]);
  __syncthreads();
  return total;
}

// Stable compaction over a dt row: emit(pos, j, bits[j]) for the positions j
// in [0, n) with pred(bits[j], j), pos = 0, 1, ... in increasing j; returns
// the count.  Each warp owns a contiguous segment, read as 16-byte quads (a
// lane holds four consecutive keys), with two quads in flight per lane.
template <class Pred, class Emit>
__device__ __forceinline__ int ordered_compact_row(const uint32_t* __restrict__ bits, int n, Pred pred, Emit emit,
                                                   SelScratch sc) {
  if ((reinterpret_cast<uintptr_t>(bits) & 15u) != 0)
    return ordered_compact(
        n, [&](int j) { return pred(bits[j], j); }, [&](int pos, int j) { emit(pos, j, bits[j]); }, sc);
  const uint32_t lane = lane_id(), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int seg = ((n + nw - 1) / nw + 127) / 128 * 128;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);
  // the four keys of this lane at chunk start c0 (positions past s1 read as 0)
  auto load4 = [&](int c0, uint32_t (&v)[4]) {
    const int j = c0 + 4 * static_cast<int>(lane);
    if (j + 3 < s1) {
      const uint4 q = __ldg(reinterpret_cast<const uint4*>(bits + j));
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = j + e < s1 ? __ldg(bits + j + e) : 0u;
    }
  };
  uint32_t cnt = 0;
  for (int c0 = s0; c0 < s1; c0 += 256) {
    uint32_t v0[4], v1[4];
    load4(c0, v0);
    load4(c0 + 128, v1);
    const int j = c0 + 4 * static_cast<int>(lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      cnt += (j + e < s1 && pred(v0[e], j + e)) ? 1u : 0u;
      cnt += (j + 128 + e < s1 && pred(v1[e], j + 128 + e)) ? 1u : 0u;
    }
  }
  cnt = __reduce_add_sync(0xFFFFFFFFu, cnt);
  __syncthreads();
  if (lane == 0) sc.red[warp] = cnt;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t acc = 0;
    for (uint32_t w = 0; w < nw; ++w) {
      const uint32_t c = sc.red[w];
      sc.red[w] = acc;
      acc += c;
    }
    sc.red[32] = acc;
  }
  __syncthreads();
  uint32_t run = sc.red[warp];
  const uint32_t lt = lanemask_lt();
  for (int c0 = s0; c0 < s1; c0 += 128) {
    uint32_t v[4];
    load4(c0, v);
    const int j = c0 + 4 * static_cast<int>(lane);
    bool p[4];
    uint32_t c = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      p[e] = j + e < s1 && pred(v[e], j + e);
      c += p[e] ? 1u : 0u;
    }
    // exclusive prefix of c (0..4) over the lanes, from its three bits
    const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, c & 1u), b1 = __ballot_sync(0xFFFFFFFFu, c & 2u),
                   b2 = __ballot_sync(0xFFFFFFFFu, c & 4u);
    uint32_t pos = run + __popc(b0 & lt) + 2u * __popc(b1 & lt) + 4u * __popc(b2 & lt);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (p[e]) emit(static_cast<int>(pos++), j + e, v[e]);
    run += __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
  }
  const int total = static_cast<int>(sc.red[32]);
  __syncthreads();
  return total;
}

}  // namespace dma
