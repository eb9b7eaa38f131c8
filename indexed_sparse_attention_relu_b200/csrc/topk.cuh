// topk.cuh -- per-row Top-K of the indexer scores (radix select).
//
// Selection (Top-K step of the Lightning Indexer, section 1 of "Day-0
// Inference Optimization for a New Sparse Attention Architecture"): the K
// best positions of row t under the order (score desc, position asc), among
// its n_valid(t) = min(q_pos + 1, seq_len) causal candidates; fewer than K
// candidates -> all of them, padded with -1. Output ascending by position.
//
// Method: scores map to order-preserving uint32 keys (-0 == +0); one CTA per
// row finds the K-th largest key tau and `need` = how many keys equal to tau
// must be taken (the lowest positions win). topk_reg_kernel (rows of at most
// 16384 positions) reads the row once into registers; topk_bitmap_kernel
// (every row whose position bitmaps fit in shared memory) needs two
// streaming passes over the row; topk_kernel (longer rows) one pass per
// 8-bit radix digit.
// Both emit the selected positions in position order with two block-wide
// exclusive scans, so the output comes out sorted with no sort. The result
// depends only on the scores (bit-deterministic).
#pragma once
#include <cub/block/block_scan.cuh>

#include "dsa_common.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;
  int64_t ld;
  const int32_t* cu_q;
  const int32_t* q_pos;
  const int32_t* seq_lens;
  int32_t B;
  int32_t L_max;
  int32_t K;
  int32_t* idx;
  int32_t cache_cap;  // keys that fit in the dynamic shared-memory cache (radix kernels),
                      // candidate slots of the threshold bin (bitmap kernel)
  int32_t bm_words;   // words of each position bitmap (bitmap kernel): >= ceil(L_max / 32), even
};

template <int THREADS>
__global__ void __launch_bounds__(THREADS) topk_kernel(const TopkParams p) {
  constexpr int IPT = 4;
  constexpr int CHUNK = THREADS * IPT;
  using Scan = cub::BlockScan<int, THREADS>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int hist[256];
  __shared__ int sel_digit, sel_krem, chunk_total;
  extern __shared__ uint32_t key_cache[];

  const int t = blockIdx.x;
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int n = max(0, min(__ldg(p.q_pos + t) + 1, len));
  int32_t* out = p.idx + static_cast<int64_t>(t) * p.K;
  const float* row = p.scores + static_cast<int64_t>(t) * p.ld;
  pdl_launch_dependents();  // the attention may be scheduled; it waits for these indices
  pdl_wait_prior();         // the indexer's scores (and anything before it) are complete

  if (n <= p.K) {
    for (int i = threadIdx.x; i < p.K; i += THREADS) out[i] = (i < n) ? i : -1;
    return;
  }

  const bool cached = n <= p.cache_cap;
  if (cached) {
    // Batched loads: 8 independent reads in flight per thread before any store,
    // so the row costs one memory latency, not one per element.
    constexpr int BATCH = 8;
    for (int base = 0; base < n; base += THREADS * BATCH) {
      float v[BATCH];
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const int i = base + u * THREADS + threadIdx.x;
        v[u] = (i < n) ? ld_dep(row + i) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const int i = base + u * THREADS + threadIdx.x;
        if (i < n) key_cache[i] = float_order_key(v[u]);
      }
    }
    __syncthreads();
  }
  auto key_at = [&](int i) -> uint32_t { return cached ? key_cache[i] : float_order_key(ld_dep(row + i)); };

  uint32_t prefix = 0u, mask = 0u;
  int krem = p.K;
  const int lane = lane_id();
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += THREADS) hist[i] = 0;
    __syncthreads();
    // Every lane of a warp runs the same trip count (THREADS is a multiple of
    // 32), so all lanes reach __ballot_sync / __match_any_sync together.
    constexpr int HB = 4;
    for (int base = 0; base < n; base += THREADS * HB) {
      uint32_t kk[HB];
#pragma unroll
      for (int u = 0; u < HB; ++u) {
        const int i = base + u * THREADS + threadIdx.x;
        kk[u] = (i < n) ? key_at(i) : 0u;
      }
#pragma unroll
      for (int u = 0; u < HB; ++u) {
        const int i = base + u * THREADS + threadIdx.x;
        const bool mine = (i < n) && ((kk[u] & mask) == prefix);
        const unsigned active = __ballot_sync(0xffffffffu, mine);
        if (mine) {
          const uint32_t digit = (kk[u] >> shift) & 0xFFu;
          const unsigned peers = __match_any_sync(active, digit);
          if ((__ffs(peers) - 1) == lane) atomicAdd(&hist[digit], __popc(peers));
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      int local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) local += hist[255 - 8 * lane - j];
      int incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const int before = incl - local;
      if (before < krem && krem <= incl) {
        int acc = before;
        for (int j = 0; j < 8; ++j) {
          const int d = 255 - 8 * lane - j;
          if (acc + hist[d] >= krem) {
            sel_digit = d;
            sel_krem = krem - acc;
            break;
          }
          acc += hist[d];
        }
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_digit) << shift;
    mask |= 0xFFu << shift;
    krem = sel_krem;
    __syncthreads();
  }
  const uint32_t tau = prefix;   // the K-th largest key
  const int need = krem;         // keys equal to tau that are taken (lowest positions)

  int eq_run = 0, out_run = 0;
#pragma unroll 1
  for (int base = 0; base < n; base += CHUNK) {
    const int i0 = base + threadIdx.x * IPT;
    uint32_t k[IPT];
    int n_eq = 0;
#pragma unroll
    for (int u = 0; u < IPT; ++u) {
      k[u] = (i0 + u < n) ? key_at(i0 + u) : 0u;
      n_eq += (i0 + u < n && k[u] == tau) ? 1 : 0;
    }
    int eq_before, eq_total;
    Scan(scan_tmp).ExclusiveSum(n_eq, eq_before, eq_total);
    __syncthreads();
    eq_before += eq_run;
    bool sel[IPT];
    int n_sel = 0;
#pragma unroll
    for (int u = 0; u < IPT; ++u) {
      const bool valid = i0 + u < n;
      bool s = valid && k[u] > tau;
      if (valid && k[u] == tau) {
        s = eq_before < need;
        ++eq_before;
      }
      sel[u] = s;
      n_sel += s ? 1 : 0;
    }
    int out_before, out_total;
    Scan(scan_tmp).ExclusiveSum(n_sel, out_before, out_total);
    __syncthreads();
    out_before += out_run;
#pragma unroll
    for (int u = 0; u < IPT; ++u) {
      if (sel[u] && out_before < p.K) out[out_before++] = i0 + u;
    }
    eq_run += eq_total;
    out_run += out_total;
  }
  (void)chunk_total;
}

// ---------------------------------------------------------------------------
// Rows of any length whose position bitmaps fit in shared memory: two
// streaming passes over the row instead of one pass per radix digit.
//  A. Histogram of the top 11 key bits (2048 bins, four copies against
//     atomic contention); a block scan from the top bin down finds the bin
//     b* that holds the K-th largest key and the count `above` of keys in
//     higher bins.
//  B. Every position in a higher bin is selected: its bit is set in the
//     selection bitmap (a warp covers 32 aligned positions, so it writes whole
//     words). Keys in b* are appended (key, position) to a candidate list.
// The K - above largest candidates are found with radix passes over the 21
// remaining key bits (on the candidate list; by streaming the row restricted
// to b* when the list overflowed), giving the K-th largest key tau and the
// number `need` of keys equal to tau to take (the lowest positions). Keys
// above tau join the selection bitmap, keys equal to tau an "equal" bitmap.
// Emission walks the bitmaps in position order with two block scans (the
// first ranks the equal keys, the second places the outputs), so the indices
// come out ascending with no sort.
// Rows of at most THREADS * PER positions. Thread `tid` owns positions
// [tid * PER, tid * PER + PER) and loads their keys once into registers. The
// K-th largest key tau is built from four 8-bit digits, most significant
// first; each digit is counted in per-warp histograms (no two warps share a
// counter) among the keys that match the digits found so far, and the bin
// holding the remaining rank is found with one scan over the 256 bins in
// descending order. Emission: keys above tau, plus the `need` lowest-position
// keys equal to tau, written in position order after one block scan of the
// packed (equal, above) counts: the equal keys taken before a thread are
// min(equal keys before it, need).
template <int THREADS, int PER>
__global__ void __launch_bounds__(THREADS, 1) topk_reg_kernel(const TopkParams p) {
  static_assert(PER % 4 == 0 && PER <= 32, "whole float4 groups, one mask word");
  static_assert(THREADS >= 256, "one thread per digit bin");
  static_assert(THREADS * PER < 65536, "packed 16-bit counts in the emission scan");
  constexpr int NWARP = THREADS / 32;
  using Scan = cub::BlockScan<int, THREADS>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ uint32_t hist[NWARP][256];
  __shared__ int wsum[8];
  __shared__ int s_digit, s_krem;

  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = lane_id();
  const int warp = warp_id();
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int n = max(0, min(__ldg(p.q_pos + t) + 1, len));
  int32_t* out = p.idx + static_cast<int64_t>(t) * p.K;
  const float* row = p.scores + static_cast<int64_t>(t) * p.ld;
  pdl_launch_dependents();  // the attention may be scheduled; it waits for these indices
  pdl_wait_prior();         // the indexer's scores (and anything before it) are complete

  if (n <= p.K) {
    for (int i = tid; i < p.K; i += THREADS) out[i] = (i < n) ? i : -1;
    return;
  }
  const int base = tid * PER;
  uint32_t key[PER];
  uint32_t valid = 0u;
  if (base + PER <= n && (reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
#pragma unroll
    for (int c = 0; c < PER / 4; ++c) {
      const float4 v = ld_dep4(row + base + 4 * c);
      key[4 * c] = float_order_key(v.x);
      key[4 * c + 1] = float_order_key(v.y);
      key[4 * c + 2] = float_order_key(v.z);
      key[4 * c + 3] = float_order_key(v.w);
    }
    valid = (PER == 32) ? ~0u : ((1u << PER) - 1u);
  } else {
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      key[u] = 0u;
      if (base + u < n) {
        key[u] = float_order_key(ld_dep(row + base + u));
        valid |= 1u << u;
      }
    }
  }

  // ---- the K-th largest key, 8 bits at a time
  uint32_t prefix = 0u, pmask = 0u;
  int kr = p.K;  // rank of tau among the keys that match the prefix
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    uint32_t* h = hist[warp];
#pragma unroll
    for (int i = lane; i < 256; i += 32) h[i] = 0u;
    __syncwarp();
#pragma unroll
    for (int u = 0; u < PER; ++u)
      if (((valid >> u) & 1u) && (key[u] & pmask) == prefix) atomicAdd(&h[(key[u] >> shift) & 255u], 1u);
    __syncthreads();
    int cnt = 0, incl = 0;
    if (tid < 256) {
      const int d = 255 - tid;  // descending digit order
#pragma unroll 8
      for (int w = 0; w < NWARP; ++w) cnt += static_cast<int>(hist[w][d]);
      incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      if (lane == 31) wsum[warp] = incl;
    }
    __syncthreads();
    if (tid < 256) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += wsum[w];
      incl += before;
      const int excl = incl - cnt;
      if (excl < kr && kr <= incl) {
        s_digit = 255 - tid;
        s_krem = kr - excl;
      }
    }
    __syncthreads();
    kr = s_krem;
    prefix |= static_cast<uint32_t>(s_digit) << shift;
    pmask |= 255u << shift;
  }
  const uint32_t tau = prefix;
  const int need = kr;  // keys equal to tau that are taken, lowest positions first

  // ---- emission in position order
  uint32_t selm = 0u, eqm = 0u;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    if (!((valid >> u) & 1u)) continue;
    if (key[u] > tau) selm |= 1u << u;
    else if (key[u] == tau) eqm |= 1u << u;
  }
  const int ce = __popc(eqm);
  int packed_before;
  Scan(scan_tmp).ExclusiveSum((ce << 16) | __popc(selm), packed_before);
  const int eq_before = packed_before >> 16;
  const int take = max(0, min(ce, need - eq_before));
  int o = (packed_before & 0xffff) + min(eq_before, need);
  int e = 0;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const bool sel = (selm >> u) & 1u;
    const bool eq = (eqm >> u) & 1u;
    if (sel || (eq && e < take)) {
      if (o < p.K) out[o] = base + u;
      ++o;
    }
    if (eq) ++e;
  }
}

template <int THREADS>
__device__ __forceinline__ void topk_find_digit(const uint32_t* h256, int width, int& kr, int* wsum, int* s_digit,
                                                int* s_krem) {
  // bins in descending digit order among the 2^width used ones; threads 0..255
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  int cnt = 0, incl = 0;
  if (tid < 256) {
    const int d = 255 - tid;
    cnt = (d < (1 << width)) ? static_cast<int>(h256[d]) : 0;
    incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
  }
  __syncthreads();
  if (tid < 256) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    incl += before;
    const int excl = incl - cnt;
    if (excl < kr && kr <= incl) {
      *s_digit = 255 - tid;
      *s_krem = kr - excl;
    }
  }
  __syncthreads();
  kr = *s_krem;
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS, 1) topk_bitmap_kernel(const TopkParams p) {
  constexpr int HBITS = 11;
  constexpr int NB = 1 << HBITS;
  constexpr int HCOPIES = 4;
  constexpr int LOW = 32 - HBITS;  // key bits below the first digit
  static_assert(2 * THREADS == NB, "two first-digit bins per thread");
  using Scan = cub::BlockScan<int, THREADS>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int wsum[8];
  __shared__ int s_bin, s_above, s_ncand, s_digit, s_krem;
  extern __shared__ __align__(16) uint32_t sm[];
  uint32_t* hist = sm;                                         // [HCOPIES][NB]
  uint32_t* selb = hist + HCOPIES * NB;                        // [bm_words]
  uint32_t* eqb = selb + p.bm_words;                           // [bm_words]
  uint2* cands = reinterpret_cast<uint2*>(eqb + p.bm_words);   // [cache_cap] (key, position)

  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = lane_id();
  const int warp = warp_id();
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int n = max(0, min(__ldg(p.q_pos + t) + 1, len));
  int32_t* out = p.idx + static_cast<int64_t>(t) * p.K;
  const float* row = p.scores + static_cast<int64_t>(t) * p.ld;
  pdl_launch_dependents();  // the attention may be scheduled; it waits for these indices
  pdl_wait_prior();         // the indexer's scores (and anything before it) are complete

  if (n <= p.K) {
    for (int i = tid; i < p.K; i += THREADS) out[i] = (i < n) ? i : -1;
    return;
  }
  const int nw = (n + 31) >> 5;
  for (int i = tid; i < HCOPIES * NB; i += THREADS) hist[i] = 0u;
  for (int i = tid; i < nw; i += THREADS) {
    selb[i] = 0u;
    eqb[i] = 0u;
  }
  if (tid == 0) s_ncand = 0;
  __syncthreads();

  // ---- A: first-digit histogram (four 16-byte loads in flight per thread on
  // aligned rows: the streaming passes are bound by loads in flight)
  {
    uint32_t* myh = hist + (warp & (HCOPIES - 1)) * NB;
    int done = 0;
    if ((reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
      const int n4 = n >> 2;  // whole groups of four positions
      for (int g0 = tid; g0 < n4; g0 += 4 * THREADS) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
          v[u] = (g0 + u * THREADS < n4) ? ld_dep4(row + 4 * (g0 + u * THREADS)) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (g0 + u * THREADS < n4) {
            atomicAdd(&myh[float_order_key(v[u].x) >> LOW], 1u);
            atomicAdd(&myh[float_order_key(v[u].y) >> LOW], 1u);
            atomicAdd(&myh[float_order_key(v[u].z) >> LOW], 1u);
            atomicAdd(&myh[float_order_key(v[u].w) >> LOW], 1u);
          }
        }
      }
      done = 4 * n4;
    }
    for (int i0 = done + tid; i0 < n; i0 += 4 * THREADS) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = (i0 + u * THREADS < n) ? ld_dep(row + i0 + u * THREADS) : 0.0f;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + u * THREADS < n) atomicAdd(&myh[float_order_key(v[u]) >> LOW], 1u);
    }
  }
  __syncthreads();
  {
    const int b1 = NB - 1 - 2 * tid, b2 = b1 - 1;
    int h1 = 0, h2 = 0;
#pragma unroll
    for (int c = 0; c < HCOPIES; ++c) {
      h1 += static_cast<int>(hist[c * NB + b1]);
      h2 += static_cast<int>(hist[c * NB + b2]);
    }
    int before;
    Scan(scan_tmp).ExclusiveSum(h1 + h2, before);
    if (before < p.K && p.K <= before + h1 + h2) {
      if (before + h1 >= p.K) {
        s_bin = b1;
        s_above = before;
      } else {
        s_bin = b2;
        s_above = before + h1;
      }
    }
  }
  __syncthreads();
  const uint32_t bstar = static_cast<uint32_t>(s_bin);
  int kr = p.K - s_above;  // keys to take from bin b*

  // ---- B: positions in higher bins -> selection bitmap; keys in b* -> candidates
  // (a warp covers 32 consecutive positions per chunk; four chunks' loads in flight)
  for (int i00 = warp * 32; i00 < n; i00 += 4 * THREADS) {
    float x[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = i00 + k * THREADS + lane;
      x[k] = (i < n) ? ld_dep(row + i) : 0.0f;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i0 = i00 + k * THREADS;  // warp-uniform
      if (i0 >= n) break;
      const int i = i0 + lane;
      const bool valid = i < n;
      const uint32_t key = valid ? float_order_key(x[k]) : 0u;
      const uint32_t kb = key >> LOW;
      const unsigned selmask = __ballot_sync(0xffffffffu, valid && kb > bstar);
      if (lane == 0 && selmask) selb[i0 >> 5] = selmask;
      const unsigned cmask = __ballot_sync(0xffffffffu, valid && kb == bstar);
      if (cmask) {
        int base = 0;
        if (lane == 0) base = atomicAdd(&s_ncand, __popc(cmask));
        base = __shfl_sync(0xffffffffu, base, 0);
        if ((cmask >> lane) & 1u) {
          const int slot = base + __popc(cmask & ((1u << lane) - 1u));
          if (slot < p.cache_cap) cands[slot] = make_uint2(key, static_cast<uint32_t>(i));
        }
      }
    }
  }
  __syncthreads();

  // ---- exact threshold inside b*: digits of 8, 8 and 5 bits
  const int ncand = s_ncand;
  const bool listed = ncand <= p.cache_cap;
  uint32_t prefix = bstar << LOW, mask = ~0u << LOW;
  uint32_t* h256 = hist;  // reuse
  const int shifts[3] = {LOW - 8, LOW - 16, 0};
  const int widths[3] = {8, 8, LOW - 16};
#pragma unroll 1
  for (int ps = 0; ps < 3; ++ps) {
    const int shift = shifts[ps];
    const uint32_t wm = (1u << widths[ps]) - 1u;
    if (tid < 256) h256[tid] = 0u;
    __syncthreads();
    if (listed) {
      for (int c = tid; c < ncand; c += THREADS) {
        const uint32_t key = cands[c].x;
        if ((key & mask) == prefix) atomicAdd(&h256[(key >> shift) & wm], 1u);
      }
    } else {
      for (int i = tid; i < n; i += THREADS) {
        const uint32_t key = float_order_key(ld_dep(row + i));
        if ((key & mask) == prefix) atomicAdd(&h256[(key >> shift) & wm], 1u);
      }
    }
    __syncthreads();
    topk_find_digit<THREADS>(h256, widths[ps], kr, wsum, &s_digit, &s_krem);
    prefix |= static_cast<uint32_t>(s_digit) << shift;
    mask |= wm << shift;
  }
  const uint32_t tau = prefix;  // the K-th largest key
  const int need = kr;          // keys equal to tau that are taken (lowest positions first)
  if (listed) {
    for (int c = tid; c < ncand; c += THREADS) {
      const uint2 kp = cands[c];
      if (kp.x > tau) atomicOr(&selb[kp.y >> 5], 1u << (kp.y & 31));
      else if (kp.x == tau) atomicOr(&eqb[kp.y >> 5], 1u << (kp.y & 31));
    }
  } else {
    for (int i = tid; i < n; i += THREADS) {
      const uint32_t key = float_order_key(ld_dep(row + i));
      if ((key >> LOW) != bstar) continue;
      if (key > tau) atomicOr(&selb[i >> 5], 1u << (i & 31));
      else if (key == tau) atomicOr(&eqb[i >> 5], 1u << (i & 31));
    }
  }
  __syncthreads();

  // ---- emission in position order
  const int wpt = (nw + THREADS - 1) / THREADS;
  const int w0 = min(nw, tid * wpt), w1 = min(nw, w0 + wpt);
  int cs = 0, ce = 0;
  for (int w = w0; w < w1; ++w) {
    cs += __popc(selb[w]);
    ce += __popc(eqb[w]);
  }
  int eq_before;
  Scan(scan_tmp).ExclusiveSum(ce, eq_before);
  __syncthreads();
  const int take_eq = max(0, min(ce, need - eq_before));
  int out_before;
  Scan(scan_tmp).ExclusiveSum(cs + take_eq, out_before);
  int o = out_before, e = eq_before;
  for (int w = w0; w < w1; ++w) {
    const uint32_t sb = selb[w], eb = eqb[w];
    uint32_t all = sb | eb;
    while (all) {
      const int bit = __ffs(all) - 1;
      all &= all - 1u;
      const int pos = w * 32 + bit;
      if ((sb >> bit) & 1u) {
        if (o < p.K) out[o++] = pos;
      } else {
        if (e < need && o < p.K) out[o++] = pos;
        ++e;
      }
    }
  }
}

}  // namespace dsa
