// topk.cuh -- per-row Top-K of the indexer scores (radix select).
//
// Selection (Top-K step of the Lightning Indexer, section 1 of "Day-0
// Inference Optimization for a New Sparse Attention Architecture"): the K
// best positions of row t under the order (score desc, position asc), among
// its n_valid(t) = min(q_pos + 1, seq_len) causal candidates; fewer than K
// candidates -> all of them, padded with -1. Output ascending by position.
//
// Method: scores map to order-preserving uint32 keys (-0 == +0). One CTA per
// row finds the K-th largest key tau with four 8-bit most-significant-digit
// histogram passes (warp-aggregated shared atomics), which also yields
// `need` = how many keys equal to tau must be taken. A final pass walks the
// row in position order with two block-wide exclusive scans: the first ranks
// the keys equal to tau (the lowest positions win), the second places every
// selected position, so the output comes out sorted with no sort. Rows that
// fit in shared memory are cached there; longer rows are re-read from L2/HBM
// on each pass. The result depends only on the scores (bit-deterministic).
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
  int32_t cache_cap;  // keys that fit in the dynamic shared-memory cache
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
// Rows of up to THREADS * IPT candidates (decode and most prefill rows).
// Thread i owns the contiguous positions [i*IPT, (i+1)*IPT): its keys are
// cached in shared memory, every radix pass adds into a per-warp histogram
// (conflicts only inside a warp), 256 threads reduce and scan the 256 bins in
// parallel, and the final emission needs just two block-wide scans because
// ownership is already in position order.
template <int THREADS, int IPT>
__global__ void __launch_bounds__(THREADS, 1) topk_row_kernel(const TopkParams p) {
  static_assert(IPT % 4 == 0, "IPT must be a multiple of 4");
  constexpr int WARPS = THREADS / 32;
  using Scan = cub::BlockScan<int, THREADS>;
  __shared__ typename Scan::TempStorage scan_tmp;
  __shared__ int whist[WARPS][256];
  __shared__ int wsum[8];
  __shared__ int sel_digit, sel_krem;
  extern __shared__ __align__(16) uint32_t keys[];  // THREADS * IPT

  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = lane_id();
  const int warp = warp_id();
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int n = max(0, min(__ldg(p.q_pos + t) + 1, len));
  int32_t* out = p.idx + static_cast<int64_t>(t) * p.K;
  const float* row = p.scores + static_cast<int64_t>(t) * p.ld;
  pdl_launch_dependents();
  pdl_wait_prior();

  if (n <= p.K) {
    for (int i = tid; i < p.K; i += THREADS) out[i] = (i < n) ? i : -1;
    return;
  }
  for (int i = tid; i < WARPS * 256; i += THREADS) (&whist[0][0])[i] = 0;

  // ---- load this thread's contiguous positions (all loads in flight at once)
  const int base = tid * IPT;
  {
    float v[IPT];
    const bool vec = ((p.ld & 3) == 0) && ((reinterpret_cast<uintptr_t>(p.scores) & 15) == 0);
    if (vec && base + IPT <= n) {
#pragma unroll
      for (int u = 0; u < IPT; u += 4) {
        const float4 f = ld_dep4(row + base + u);
        v[u] = f.x;
        v[u + 1] = f.y;
        v[u + 2] = f.z;
        v[u + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int u = 0; u < IPT; ++u) v[u] = (base + u < n) ? ld_dep(row + base + u) : 0.0f;
    }
#pragma unroll
    for (int u = 0; u < IPT; u += 4) {
      uint4 k4;
      k4.x = (base + u + 0 < n) ? float_order_key(v[u + 0]) : 0u;
      k4.y = (base + u + 1 < n) ? float_order_key(v[u + 1]) : 0u;
      k4.z = (base + u + 2 < n) ? float_order_key(v[u + 2]) : 0u;
      k4.w = (base + u + 3 < n) ? float_order_key(v[u + 3]) : 0u;
      *reinterpret_cast<uint4*>(keys + base + u) = k4;
    }
  }
  const int mine = max(0, min(IPT, n - base));  // valid positions owned by this thread
  __syncthreads();

  uint32_t prefix = 0u, mask = 0u;
  int krem = p.K;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
#pragma unroll
    for (int u = 0; u < IPT; u += 4) {
      const uint4 k4 = *reinterpret_cast<const uint4*>(keys + base + u);
      const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (u + j < mine && (kk[j] & mask) == prefix) atomicAdd(&whist[warp][(kk[j] >> shift) & 0xFFu], 1);
    }
    __syncthreads();
    // 256 threads: bin total (descending digit order), reset, inclusive scan
    int cnt = 0, incl = 0;
    if (tid < 256) {
      const int d = 255 - tid;
#pragma unroll 4
      for (int w = 0; w < WARPS; ++w) {
        cnt += whist[w][d];
        whist[w][d] = 0;
      }
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
      int before_warp = 0;
      for (int w = 0; w < warp; ++w) before_warp += wsum[w];
      incl += before_warp;
      const int excl = incl - cnt;
      if (excl < krem && krem <= incl) {
        sel_digit = 255 - tid;
        sel_krem = krem - excl;
      }
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(sel_digit) << shift;
    mask |= 0xFFu << shift;
    krem = sel_krem;
  }
  const uint32_t tau = prefix;   // the K-th largest key
  const int need = krem;         // keys equal to tau that are taken (lowest positions first)

  int n_eq = 0;
#pragma unroll
  for (int u = 0; u < IPT; ++u) n_eq += (u < mine && keys[base + u] == tau) ? 1 : 0;
  int eq_before, eq_total;
  Scan(scan_tmp).ExclusiveSum(n_eq, eq_before, eq_total);
  __syncthreads();
  int n_sel = 0;
  {
    int e = eq_before;
#pragma unroll
    for (int u = 0; u < IPT; ++u) {
      if (u >= mine) break;
      const uint32_t k = keys[base + u];
      if (k > tau) {
        ++n_sel;
      } else if (k == tau) {
        n_sel += (e < need) ? 1 : 0;
        ++e;
      }
    }
  }
  int out_before, out_total;
  Scan(scan_tmp).ExclusiveSum(n_sel, out_before, out_total);
  {
    int e = eq_before, o = out_before;
#pragma unroll
    for (int u = 0; u < IPT; ++u) {
      if (u >= mine) break;
      const uint32_t k = keys[base + u];
      bool take = k > tau;
      if (k == tau) {
        take = e < need;
        ++e;
      }
      if (take && o < p.K) out[o++] = base + u;
    }
  }
  (void)eq_total;
  (void)out_total;
}

}  // namespace dsa
