// sparse_mla_pipe.cuh -- sparse MLA attention for 128 query heads over the
// 576-dim latent rows (d_c = 512, d_rope = 64), on a pipeline of two CTAs:
// Sparse Flash Attention of "Day-0 Inference Optimization for a New Sparse
// Attention Architecture", section 1, over the rows the Lightning Indexer
// selected. Same result as sparse_mla_kernel:
//   z_i = softmax_scale * q[t,h,:] . kv[b,s_i,:]          (all 576 dims)
//   out[t,h,:] = sum_i softmax(z)_i * kv[b,s_i,0:512]     (value = latent part)
//   lse[t,h] = log sum_i exp(z_i)
//
// Why two CTAs. With all 128 heads in one tensor-core tile (M = 128, the full
// datapath rate) the output accumulator alone is 128 x 512 fp32 = all of an
// SM's tensor memory, leaving no room for the scores. So each (query, key
// split) gets a cluster pair:
//  * the score CTA gathers whole rows, computes S = Q K^T with M = 128 (Q and
//    S in tensor memory), runs the online softmax (a thread per head row) and
//    writes P (bf16, already in the 128-byte-swizzled shared-memory image the
//    PV product reads) and the per-row rescale factors of the tile into a
//    small ring in global memory (L2);
//  * the value CTA gathers the latent part of the same rows (L2 hits), copies
//    P into shared memory, rescales O rows when the score CTA raised a row
//    maximum by more than 2^8, and accumulates O += P V (M = 128, N = 256 x 2)
//    with all 512 output columns in its tensor memory.
// Bulk data crosses through L2 (distributed shared memory is far slower for
// it); the pair signals through mbarriers in each other's shared memory:
// "P of tile j is in ring slot j % NP" (score -> value) and "slot free"
// (value -> score). Key splits of one query form the rest of the cluster and
// merge through the workspace after the cluster barrier, as in the 64-head
// kernel. Every wait is bounded.
#pragma once
#include "dsa_common.cuh"
#include "sparse_mla.cuh"

namespace dsa {

struct PipeParams {
  const int32_t* cu_q;
  const int32_t* seq_lens;
  int32_t B;
  int32_t L_max;
  int32_t T;
  int32_t K;
  const int32_t* idx;        // [T, K]
  float scale_log2;          // softmax_scale * log2(e)
  int32_t keys_per_split;    // multiple of 64
  int32_t splits;            // pairs per query (cluster = 2 x splits CTAs)
  __nv_bfloat16* out;        // [T, 128, 512]
  float* lse;                // [T, 128] or null
  uint8_t* ring;             // [RING_SMS, NP] slots of SLOT_BYTES, indexed by the score CTA's SM
  float2* fin;               // [RING_SMS, 128] final (running max, running sum) per head row
  float* part_o;             // [T, splits][512 / 4][128][4] split partials (splits > 1)
  float2* part_ml;           // [T, splits, 128]
  CacheMap cm;               // cache rows (contiguous or paged)
};

struct PipeCfg {
  static constexpr int D = 576, DC = 512, M = 128, TK = 64;
  static constexpr int KSTEPS = D / 16;                 // 36
  static constexpr int ATOM = 64 * 128;                 // one 64-dim atom column of a 64-row tile
  static constexpr int K_BYTES = 9 * ATOM;              // score CTA: a 64-key tile of whole rows
  static constexpr int NKS = 3;                         // score CTA gather stages
  static constexpr int Q_ATOM = M * 128;                // one 64-dim atom column of the 128-head Q tile
  static constexpr int V_BYTES = 8 * ATOM;              // value CTA: the 512 latent dims of 64 keys
  static constexpr int NVS = 3;                         // value CTA gather stages
  static constexpr int P_IMG = M * 128;                 // P tile image (128 rows x 64 keys bf16, swizzled)
  static constexpr int SLOT_BYTES = P_IMG + M * 4;      // + per-row rescale factors
  static constexpr int P_STAGE = ((SLOT_BYTES + 1023) / 1024) * 1024;  // swizzle base stays aligned
  static constexpr int NPS = 2;                         // value CTA P stages
  static constexpr int RING_SMS = 256;                  // SM ids a ring / statistics record exists for
  static constexpr int NP = 4;                          // ring slots per pair
  static constexpr uint32_t COL_S = 0;                  // score CTA: S double buffer, 2 x 64 columns
  static constexpr uint32_t COL_Q = 128;                // score CTA: Q, 288 columns of bf16 pairs
  // 0-3 softmax / rescale, 4-11 gather, 12 MMA, 13 ring signalling (score CTA) or P copy (value
  // CTA); the epilogue runs on warps 0-11 (three per TMEM sub-partition).
  static constexpr int NGATHER = 8;
  static constexpr int ROWS_PER_GW = TK / NGATHER;          // rows of a tile per gather warp
  static constexpr int MMA_WARP = 4 + NGATHER;
  static constexpr int AUX_WARP = MMA_WARP + 1;
  static constexpr int EPI_WARPS = 4 + NGATHER;
  static constexpr int NUM_WARPS = AUX_WARP + 1;
  static constexpr int THREADS = NUM_WARPS * 32;
  static constexpr int MAX_SPLITS = 4;                  // 1, 2 or 4 (a split owns 128 / S head rows)
  // Merge: the other splits' copies of a split's rows arrive by TMA into the
  // value CTA's (then idle) V stages, one box of 128 / S rows x 512 columns
  // per other split (stored [column / 4][row][4] like the workspace).
  static constexpr int MERGE_BAR = 19;
  static constexpr int box_bytes(int S) { return (M / S) * DC * 4; }
  // score CTA shared memory
  static constexpr int A_OFF_K = 0;
  static constexpr int A_OFF_BAR = NKS * K_BYTES;
  // value CTA shared memory
  static constexpr int B_OFF_P = 0;
  static constexpr int B_OFF_V = NPS * P_STAGE;
  static constexpr int B_OFF_BAR = B_OFF_V + NVS * V_BYTES;
  static constexpr int NUM_BARS = 24;
  static constexpr int MISC_BYTES = 32;
  // score CTA: the split's selected indices, staged once (a load issued while
  // the gathers stream queues behind them for microseconds)
  static constexpr int A_OFF_IDX = A_OFF_BAR + NUM_BARS * 8 + MISC_BYTES;
  static constexpr int MAX_K = 2048;
  static constexpr int A_END = A_OFF_IDX + MAX_K * 4;
  static constexpr int B_END = B_OFF_BAR + NUM_BARS * 8 + MISC_BYTES;
  static constexpr int SMEM_BYTES = A_END > B_END ? A_END : B_END;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(M, TK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(M, 256, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(COL_Q + D / 2 <= 512, "TMEM budget of the score CTA");
  static_assert(2 * K_BYTES >= 9 * Q_ATOM, "Q is staged in gather stages 1 and 2");
  static_assert(P_IMG % 1024 == 0 && SLOT_BYTES % 16 == 0, "ring slot layout");
  static_assert(B_OFF_V % 1024 == 0, "TMA destination alignment");
};
static_assert(PipeCfg::box_bytes(2) <= PipeCfg::NVS * PipeCfg::V_BYTES &&
                  (PipeCfg::MAX_SPLITS - 1) * PipeCfg::box_bytes(PipeCfg::MAX_SPLITS) <= PipeCfg::NVS * PipeCfg::V_BYTES,
              "merge boxes fit in the V stages");

__device__ __forceinline__ void tmem_st16w(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

__device__ __forceinline__ bool mbar_wait_cluster_all(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait_cluster(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// PAGED: the caches are paged (rows translated through the block table);
// contiguous calls run without that code in their gather loops.
template <bool PAGED>
__global__ void __launch_bounds__(PipeCfg::THREADS, 1)
    sparse_mla_pipe_kernel(const __grid_constant__ CUtensorMap kvmap, const __grid_constant__ CUtensorMap qmap,
                           const __grid_constant__ CUtensorMap pmap, const PipeParams p) {
  using C = PipeCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // same in every CTA: all leave or none
    if (threadIdx.x == 0) set_device_status(DSA_ERR_DEVICE_LAYOUT);
    return;
  }
  canary_set(smem, C::SMEM_BYTES);
  const uint32_t crank = cluster_ctarank();
  const bool score_cta = (crank & 1u) == 0;
  const int split = static_cast<int>(crank >> 1);
  const uint32_t partner = crank ^ 1u;
  const int S = p.splits;
  const int t = blockIdx.y;
  const int warp = warp_id();
  const int lane = lane_id();
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.K, k_begin + p.keys_per_split);
  const int n_tiles = (k_end - k_begin + C::TK - 1) / C::TK;  // >= 1 by construction
  const int32_t* idx_row = p.idx + static_cast<int64_t>(t) * p.K;
  const int64_t pair = static_cast<int64_t>(t) * S + split;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (score_cta ? C::A_OFF_BAR : C::B_OFF_BAR));
  // score CTA: [0,3) kv_full, [3,6) kv_empty, 6 q_full, 7 q_moved, [8,10) s_full, [10,12) s_empty,
  //            [12,16) slot_free (remote arrivals from the value CTA), 16 drain, [17,21) p_written,
  //            21 fin_written
  // value CTA: [0,3) v_full, [3,6) v_empty, [6,8) p_full, [8,10) p_empty, [12,16) p_ready (remote
  //            arrivals from the score CTA), 16 drain, [17,19) rescaled (per P stage), 20 o_done,
  //            21 fin_ready (remote)
  // [0] TMEM base, [1] abort, [2] SM id, [4..6) per-tile go flags of the gather warps
  int32_t* misc = reinterpret_cast<int32_t*>(bars + C::NUM_BARS);
  int32_t* sidx = reinterpret_cast<int32_t*>(smem + C::A_OFF_IDX);  // score CTA only
  volatile int* abort_flag = misc + 1;
  if (threadIdx.x == 0) {
    if (score_cta) {
      for (int i = 0; i < C::NKS; ++i) {
        mbar_init(&bars[i], 1);  // the gather leader's arrival (+ the row gathers' bytes)
        mbar_init(&bars[3 + i], 1);
      }
      mbar_init(&bars[6], 1);
      mbar_init(&bars[7], 4);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&bars[8 + i], 1);
        mbar_init(&bars[10 + i], 4);
      }
      for (int i = 0; i < C::NP; ++i) {
        mbar_init(&bars[12 + i], 1);
        mbar_init(&bars[17 + i], 128);  // every softmax thread, after its stores into the slot
      }
      mbar_init(&bars[16], 1);
      mbar_init(&bars[21], 128);
    } else {
      for (int i = 0; i < C::NVS; ++i) {
        mbar_init(&bars[i], 1);
        mbar_init(&bars[3 + i], 1);
      }
      for (int i = 0; i < C::NPS; ++i) {
        mbar_init(&bars[6 + i], 32);  // one asynchronous arrival per P-copy thread
        mbar_init(&bars[8 + i], 1);
      }
      for (int i = 0; i < C::NP; ++i) mbar_init(&bars[12 + i], 1);
      mbar_init(&bars[16], 1);
      mbar_init(&bars[17], 4);
      mbar_init(&bars[18], 4);
      mbar_init(&bars[20], 1);
      mbar_init(&bars[21], 1);
      mbar_init(&bars[C::MERGE_BAR], 1);
    }
    misc[1] = 0;
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    misc[2] = static_cast<int32_t>(smid);
    fence_mbar_init();
    if (score_cta) prefetch_tensormap(&qmap);
    prefetch_tensormap(&kvmap);
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();  // every barrier of the cluster is initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);
  // The ring and the final statistics belong to the score CTA's SM (one
  // score CTA per SM at a time): the value CTA reads its partner's SM id.
  int ring_sm = misc[2];
  if (!score_cta) {
    const uint32_t a = mapa_shared(smem_u32(smem + C::A_OFF_BAR + C::NUM_BARS * 8 + 8), partner);
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(ring_sm) : "r"(a) : "memory");
  }
  const bool ring_ok = ring_sm >= 0 && ring_sm < C::RING_SMS;
  if (!ring_ok) {
    if (threadIdx.x == 0) set_device_status(DSA_ERR_DEVICE_LAYOUT);
    ring_sm = 0;
  }
  uint8_t* ring = p.ring + static_cast<int64_t>(ring_sm) * C::NP * C::SLOT_BYTES;
  float2* fin = p.fin + static_cast<int64_t>(ring_sm) * C::M;

  if (score_cta) {
    // =================================================================== score CTA
    uint64_t* kv_full = bars;
    uint64_t* kv_empty = bars + 3;
    uint64_t* q_full = bars + 6;
    uint64_t* q_moved = bars + 7;
    uint64_t* s_full = bars + 8;
    uint64_t* s_empty = bars + 10;
    uint64_t* slot_free = bars + 12;
    uint64_t* drain = bars + 16;
    uint64_t* p_written = bars + 17;
    uint64_t* fin_written = bars + 21;
    const uint32_t q_stage = smem_u32(smem + C::A_OFF_K + C::K_BYTES);  // stages 1 and 2 hold Q first
    if (warp == C::MMA_WARP && lane == 0) {
      // the query block is an input of the call: load it now (9 atom columns of 128 rows)
      mbar_arrive_expect_tx(q_full, 9 * C::Q_ATOM);
#pragma unroll
      for (int c = 0; c < 9; ++c) tma_load_2d(q_stage + c * C::Q_ATOM, &qmap, c * 64, t * C::M, q_full);
    }
    if (warp < 4) {
      // ---------------------------------------------------------- softmax (a thread per head row)
      const int h = warp * 32 + lane;
      const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
      bool ok = mbar_wait_warp(q_full, 0, abort_flag);
      if (ok) {
        // Q row h -> TMEM columns COL_Q + c (dims 2c, 2c+1), 16 columns at a time
#pragma unroll 1
        for (int g = 0; g < 18; ++g) {
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = 4 * g + u;  // 16-byte chunk of the row (8 dims)
            const uint4 x = *reinterpret_cast<const uint4*>(smem + C::A_OFF_K + C::K_BYTES +
                                                             (chunk >> 3) * C::Q_ATOM + sw128_offset(h, chunk & 7));
            w[4 * u] = x.x;
            w[4 * u + 1] = x.y;
            w[4 * u + 2] = x.z;
            w[4 * u + 3] = x.w;
          }
          tmem_st16w(tmem_base + lane_addr + C::COL_Q + 16 * g, w);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_moved);  // also on failure: every wait stays bounded
      named_bar_sync(2, 32 * (4 + C::NGATHER));  // the gather warps have staged the indices

      float m = -INFINITY, l = 0.0f;
      const int nk = k_end - k_begin;
      for (int j = 0; j < n_tiles; ++j) {
        const int i0 = (j * C::TK + lane < nk) ? sidx[j * C::TK + lane] : -1;
        const int i1 = (j * C::TK + 32 + lane < nk) ? sidx[j * C::TK + 32 + lane] : -1;
        // staged entries: positions (contiguous) or pool rows with -1 for masked keys (paged)
        const unsigned v0 = __ballot_sync(0xffffffffu, i0 >= 0 && (PAGED || i0 < len));
        const unsigned v1 = __ballot_sync(0xffffffffu, i1 >= 0 && (PAGED || i1 < len));
        float v[64];
        if (ok) ok = mbar_wait_warp(&s_full[j & 1], (j >> 1) & 1, abort_flag);
        if (ok) {
          tc_fence_after();
          const uint32_t sa = tmem_base + lane_addr + C::COL_S + 64 * (j & 1);
          tmem_ld16(sa, *reinterpret_cast<float(*)[16]>(v));
          tmem_ld16(sa + 16, *reinterpret_cast<float(*)[16]>(v + 16));
          tmem_ld16(sa + 32, *reinterpret_cast<float(*)[16]>(v + 32));
          tmem_ld16(sa + 48, *reinterpret_cast<float(*)[16]>(v + 48));
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s_empty[j & 1]);
        }
        // logits in log2 units, two per instruction
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 z = mul2(make_float2(v[2 * i], v[2 * i + 1]), sc2);
          v[2 * i] = z.x;
          v[2 * i + 1] = z.y;
        }
        if ((v0 & v1) != 0xffffffffu) {  // keys past the row's end or -1: no weight (warp-uniform test)
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (!(((i < 32 ? v0 : v1) >> (i & 31)) & 1u)) v[i] = -INFINITY;
        }
        float t4[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
        for (int i = 4; i < 64; i += 4) {
#pragma unroll
          for (int u = 0; u < 4; ++u) t4[u] = fmaxf(t4[u], v[i + u]);
        }
        const float tmax = fmaxf(fmaxf(t4[0], t4[1]), fmaxf(t4[2], t4[3]));
        float f = 1.0f;
        const float nm = fmaxf(m, tmax);
        if (nm > m + 8.0f) {  // lazy rescale: P stays <= 2^8
          f = ex2_approx(m - nm);  // 0 when m = -inf
          l *= f;
          m = nm;
        }
        // ring slot j % NP: free once the value CTA has copied tile j - NP
        if (ok) ok = mbar_wait_cluster_all(&slot_free[j % C::NP], ((j / C::NP) & 1) ^ 1u, abort_flag);
        uint8_t* slot = ring + (j % C::NP) * C::SLOT_BYTES;
        if (ok) reinterpret_cast<float*>(slot + C::P_IMG)[h] = f;
        // P = 2^(z - m) (masked keys give 2^-inf = 0; a row with no valid key
        // yet has m = -inf and gets zeros), stored 8 keys (16 bytes) at a
        // time into the swizzled image; the row sum takes the fp32 values
        const bool live = m != -INFINITY;
        const float2 nm2 = make_float2(live ? -m : 0.0f, live ? -m : 0.0f);
        float2 la = make_float2(0.0f, 0.0f), lb = la;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w4[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i = 4 * c + u;
            const float2 z = add2(make_float2(v[2 * i], v[2 * i + 1]), nm2);
            float2 e = make_float2(ex2_approx(z.x), ex2_approx(z.y));
            if (!live) e = make_float2(0.0f, 0.0f);
            const __nv_bfloat162 pr = __floats2bfloat162_rn(e.x, e.y);
            w4[u] = *reinterpret_cast<const uint32_t*>(&pr);
            if (u & 1) lb = add2(lb, e); else la = add2(la, e);
          }
          if (ok) *reinterpret_cast<uint4*>(slot + sw128_offset(h, c)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        const float2 ls = add2(la, lb);
        l += ls.x + ls.y;
        // no fence here: the signalling warp publishes the slot to the value
        // CTA (its cluster-scope release covers these stores through this
        // CTA-scope arrival), so the softmax goes on with the next tile
        mbar_arrive(&p_written[j % C::NP]);
      }
      // final statistics of every row, published the same way
      if (ok) fin[h] = make_float2(m, l);
      mbar_arrive(fin_written);
    } else if (warp == C::AUX_WARP) {
      // ---------------------------------------------------------- ring signalling
      // Waits until all 128 softmax threads have stored tile j's P and factors,
      // then releases them to the value CTA at cluster scope. Only this warp
      // waits for the stores to drain to L2.
      if (lane == 0) {
        const uint32_t p_ready_peer = mapa_shared(smem_u32(smem + C::B_OFF_BAR + 12 * 8), partner);
        const uint32_t fin_peer = mapa_shared(smem_u32(smem + C::B_OFF_BAR + 21 * 8), partner);
        bool ok = true;
        // (test hook: a set g_debug_withhold holds back the signal of tile 0,
        // so the value CTA's bounded wait for it runs out)
        const bool withhold = *reinterpret_cast<volatile int*>(&g_debug_withhold) != 0;
        for (int j = 0; j < n_tiles && ok; ++j) {
          ok = mbar_wait(&p_written[j % C::NP], (j / C::NP) & 1, abort_flag);
          if (ok && !(withhold && j == 0)) mbar_arrive_remote(p_ready_peer + (j % C::NP) * 8);
        }
        if (ok && mbar_wait(fin_written, 0, abort_flag)) mbar_arrive_remote(fin_peer);
      }
      __syncwarp();
    } else if (warp < C::MMA_WARP) {
      // ---------------------------------------------------------- gather whole rows
      // TMA row gathers (tile::gather4: four rows x one 64-dim atom column per
      // op, placed in the 128-byte-swizzled K-major layout by the copy engine):
      // 16 row groups x 9 atom columns = 144 ops per tile, one per gather
      // thread. A leader waits for the stage and arms its barrier; the others
      // learn through a per-tile flag whether to go on, so every tile is
      // issued whole or not at all. Invalid rows (-1, or outside the
      // sequence) fetch the sequence's row 0 (paged caches: the pool's row 0)
      // instead: their logits are masked to -inf below and their P is 0.
      pdl_wait_prior();  // the selected indices (Top-K output) are complete from here on
      const int gl = threadIdx.x - 4 * 32;  // 0 .. 32 * NGATHER - 1
      const bool leader = gl == 0;
      const bool active = gl < 16 * 9;
      const int g = gl / 9, a = gl - (gl / 9) * 9;
      const int32_t row0 = b * p.L_max;  // contiguous: the sequence's first row (the stand-in for invalid keys)
      {
        // stage this split's indices (eight independent loads in flight per thread)
        const int nk = k_end - k_begin;
        constexpr int GT = 32 * C::NGATHER;
        for (int base = 0; base < nk; base += 8 * GT) {
          int v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + u * GT + gl;
            v[u] = i < nk ? ld_dep(idx_row + k_begin + i) : -1;
          }
          if constexpr (PAGED) {
            // paged caches: each selected row's pool position, looked up once
            // here rather than before every gather; -1 marks a masked key (-1,
            // or a position outside the sequence, which is reported)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const int i = base + u * GT + gl;
              const int s = v[u];
              if (s >= 0 && s < len) {
                v[u] = p.cm.row_checked(b, s);
              } else {
                if (i < nk && s != -1) set_device_status(DSA_ERR_DEVICE_INDEX);
                v[u] = -1;
              }
            }
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = base + u * GT + gl;
            if (i < nk) sidx[i] = v[u];
          }
        }
      }
      named_bar_sync(2, 32 * (4 + C::NGATHER));  // with the softmax warps
      const int nk = k_end - k_begin;
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int sl = j % C::NKS;
        int cur[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int kk = j * C::TK + 4 * g + i;
          cur[i] = (active && kk < nk) ? sidx[kk] : -1;
        }
        if (leader) {
          bool ok = true;
          if (j == 1) ok = mbar_wait(q_moved, 0, abort_flag);  // stages 1, 2 hold Q until then
          if (ok) ok = mbar_wait(&kv_empty[sl], ((j / C::NKS) & 1) ^ 1u, abort_flag);
          if (ok) mbar_arrive_expect_tx(&kv_full[sl], C::K_BYTES);
          reinterpret_cast<volatile int*>(misc)[4 + (j & 1)] = ok ? 1 : 0;
        }
        named_bar_sync(1, 32 * C::NGATHER);
        if (!reinterpret_cast<volatile int*>(misc)[4 + (j & 1)]) break;
        if (active) {
          int y[4];
          if constexpr (PAGED) {
#pragma unroll
            for (int i = 0; i < 4; ++i) y[i] = cur[i] >= 0 ? cur[i] : 0;  // staged pool rows (masked: row 0)
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const bool v = cur[i] >= 0 && cur[i] < len;
              if (a == 0 && cur[i] != -1 && !v) set_device_status(DSA_ERR_DEVICE_INDEX);
              y[i] = row0 + (v ? cur[i] : 0);
            }
          }
          tma_gather4(smem_u32(smem + C::A_OFF_K + sl * C::K_BYTES + a * C::ATOM + g * 512), &kvmap, a * 64, y[0], y[1],
                      y[2], y[3], &kv_full[sl]);
        }
        ++issued;
      }
      // every tile issued must land before the CTA can retire
      if (leader) {
        for (int j = issued > C::NKS ? issued - C::NKS : 0; j < issued; ++j) {
          volatile int never = 0;
          mbar_wait(&kv_full[j % C::NKS], (j / C::NKS) & 1, &never);
        }
      }
    } else if (warp == C::MMA_WARP) {
      // ---------------------------------------------------------- MMA: S = Q K^T, M = 128
      if (lane == 0) {
        bool ok = mbar_wait(q_moved, 0, abort_flag);
        for (int j = 0; j < n_tiles && ok; ++j) {
          const int sl = j % C::NKS;
          ok = mbar_wait(&kv_full[sl], (j / C::NKS) & 1, abort_flag);
          if (ok && j >= 2) ok = mbar_wait(&s_empty[j & 1], ((j >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          fence_proxy_async_smem();  // cp.async (generic proxy) data -> tensor core reads
          tc_fence_after();
          const uint32_t kb = smem_u32(smem + C::A_OFF_K + sl * C::K_BYTES);
          const uint32_t d = tmem_base + C::COL_S + 64 * (j & 1);
#pragma unroll
          for (int k = 0; k < C::KSTEPS; ++k) {
            const uint64_t bd = smem_desc_sw128(kb + (k >> 2) * C::ATOM + (k & 3) * 32, 16, 1024);
            umma_f16_ts(d, tmem_base + C::COL_Q + 8 * k, bd, C::IDESC_S, k > 0 ? 1u : 0u);
          }
          umma_commit(&kv_empty[sl]);  // the rows are only needed for S
          umma_commit(&s_full[j & 1]);
        }
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never);
      }
      __syncwarp();
    }
  } else {
    // =================================================================== value CTA
    uint64_t* v_full = bars;
    uint64_t* v_empty = bars + 3;
    uint64_t* p_full = bars + 6;
    uint64_t* p_empty = bars + 8;
    uint64_t* p_ready = bars + 12;
    uint64_t* drain = bars + 16;
    uint64_t* rescaled = bars + 17;  // [NPS]
    uint64_t* o_done = bars + 20;
    uint64_t* fin_ready = bars + 21;
    const uint32_t slot_free_peer = mapa_shared(smem_u32(smem + C::A_OFF_BAR + 12 * 8), partner);
    if (warp == C::AUX_WARP) {
      // ---------------------------------------------------------- P copy: ring slot -> P stage
      // Runs up to NPS tiles ahead of the rescale warps and the MMA.
      bool ok = true;
      for (int j = 0; j < n_tiles && ok; ++j) {
        const int ps = j % C::NPS;
        ok = mbar_wait_cluster_all(&p_ready[j % C::NP], (j / C::NP) & 1, abort_flag) &&
             mbar_wait_warp(&p_empty[ps], ((j / C::NPS) & 1) ^ 1u, abort_flag);
        if (!ok) break;
        const uint8_t* slot = ring + (j % C::NP) * C::SLOT_BYTES;
        const uint32_t dst = smem_u32(smem + C::B_OFF_P + ps * C::P_STAGE);
        for (int c = lane; c < C::SLOT_BYTES / 16; c += 32) cp_async_16(dst + 16 * c, slot + 16 * c, 16u);
        cp_async_arrive_noinc(&p_full[ps]);
      }
      cp_async_wait_all();
    } else if (warp < 4) {
      // ---------------------------------------------------------- O rescale
      const int h = warp * 32 + lane;
      const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
      bool ok = true;
      for (int j = 0; j < n_tiles; ++j) {
        const int ps = j % C::NPS;
        if (ok) ok = mbar_wait_warp(&p_full[ps], (j / C::NPS) & 1, abort_flag);
        if (ok) {
          // rows whose running maximum the score CTA raised: rescale O first
          const float f = reinterpret_cast<const float*>(smem + C::B_OFF_P + ps * C::P_STAGE + C::P_IMG)[h];
          if (__any_sync(0xffffffffu, f != 1.0f) && j > 0) {
            ok = mbar_wait_warp(o_done, (j - 1) & 1, abort_flag);  // PV(j - 1) complete
            if (ok) {
              tc_fence_after();
#pragma unroll 1
              for (int c = 0; c < C::DC; c += 16) {
                float o[16];
                tmem_ld16(tmem_base + lane_addr + c, o);
                tmem_wait_ld();
#pragma unroll
                for (int u = 0; u < 16; ++u) o[u] *= f;
                tmem_st16(tmem_base + lane_addr + c, o);
              }
              tmem_wait_st();
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&rescaled[ps]);  // also on failure: every wait stays bounded
      }
    } else if (warp < C::MMA_WARP) {
      // ---------------------------------------------------------- gather the latent part
      // The same TMA row gathers for atom columns 0-7 (the 512 latent dims):
      // 16 row groups x 8 = 128 ops per tile (the score CTA reports bad indices).
      // Indices are read four tiles ahead (a load issued while the gathers
      // stream queues behind them for microseconds).
      pdl_wait_prior();
      const int gl = threadIdx.x - 4 * 32;
      const bool leader = gl == 0;
      const bool active = gl < 16 * 8;
      const int g = gl >> 3, a = gl & 7;
      const int32_t row0 = b * p.L_max;  // contiguous: the sequence's first row (the stand-in for invalid keys)
      auto load_rows = [&](int tile, int (&y)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int k = k_begin + tile * C::TK + 4 * g + i;
          y[i] = (active && tile < n_tiles && k < k_end) ? ld_dep(idx_row + k) : -1;
        }
      };
      // paged caches: the pool rows of the next tile are looked up one tile
      // ahead (from positions loaded three tiles before), so the block-table
      // load is not waited on right before a gather
      auto pool_rows = [&](const int (&s)[4], int (&y)[4]) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          bool rok;
          y[i] = (s[i] >= 0 && s[i] < len) ? p.cm.row(b, s[i], rok) : 0;
        }
      };
      int r0[4], r1[4], r2[4], r3[4];
      load_rows(0, r0);
      load_rows(1, r1);
      load_rows(2, r2);
      load_rows(3, r3);
      int pr[4] = {0, 0, 0, 0};  // pool rows of the tile issued next (paged)
      if constexpr (PAGED) pool_rows(r0, pr);
      int issued = 0;
      bool stop = false;
      for (int j0 = 0; j0 < n_tiles && !stop; j0 += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int j = j0 + u;
          if (j >= n_tiles || stop) break;
          int (&cur)[4] = u == 0 ? r0 : u == 1 ? r1 : u == 2 ? r2 : r3;
          const int (&nxt)[4] = u == 0 ? r1 : u == 1 ? r2 : u == 2 ? r3 : r0;  // tile j + 1's positions
          const int sl = j % C::NVS;
          if (leader) {
            const bool ok = mbar_wait(&v_empty[sl], ((j / C::NVS) & 1) ^ 1u, abort_flag);
            if (ok) mbar_arrive_expect_tx(&v_full[sl], C::V_BYTES);
            reinterpret_cast<volatile int*>(misc)[4 + (j & 1)] = ok ? 1 : 0;
          }
          named_bar_sync(1, 32 * C::NGATHER);
          if (!reinterpret_cast<volatile int*>(misc)[4 + (j & 1)]) {
            stop = true;
            break;
          }
          if (active) {
            int y[4];
            if constexpr (PAGED) {
#pragma unroll
              for (int i = 0; i < 4; ++i) y[i] = pr[i];
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) y[i] = row0 + ((cur[i] >= 0 && cur[i] < len) ? cur[i] : 0);
            }
            tma_gather4(smem_u32(smem + C::B_OFF_V + sl * C::V_BYTES + a * C::ATOM + g * 512), &kvmap, a * 64, y[0],
                        y[1], y[2], y[3], &v_full[sl]);
          }
          ++issued;
          if constexpr (PAGED) pool_rows(nxt, pr);
          load_rows(j + 4, cur);
        }
      }
      if (leader) {
        for (int j = issued > C::NVS ? issued - C::NVS : 0; j < issued; ++j) {
          volatile int never = 0;
          mbar_wait(&v_full[j % C::NVS], (j / C::NVS) & 1, &never);
        }
      }
    } else if (warp == C::MMA_WARP) {
      // ---------------------------------------------------------- MMA: O += P V, M = 128
      if (lane == 0) {
        bool ok = true;
        for (int j = 0; j < n_tiles && ok; ++j) {
          const int vs = j % C::NVS, ps = j % C::NPS;
          ok = mbar_wait(&v_full[vs], (j / C::NVS) & 1, abort_flag) &&
               mbar_wait(&p_full[ps], (j / C::NPS) & 1, abort_flag) &&
               mbar_wait(&rescaled[ps], (j / C::NPS) & 1, abort_flag);
          if (!ok) break;
          // ring slot j % NP has been copied: the score CTA may refill it
          mbar_arrive_remote(slot_free_peer + (j % C::NP) * 8);
          fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t vb = smem_u32(smem + C::B_OFF_V + vs * C::V_BYTES);
          const uint32_t pb = smem_u32(smem + C::B_OFF_P + ps * C::P_STAGE);
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
#pragma unroll
            for (int kk = 0; kk < C::TK / 16; ++kk) {
              const uint64_t a = smem_desc_sw128(pb + kk * 32, 16, 1024);
              // V: 64-dim atom columns ATOM bytes apart (LBO), 8-key row groups 1024 bytes apart (SBO)
              const uint64_t bd = smem_desc_sw128(vb + (4 * nb) * C::ATOM + kk * 16 * 128, C::ATOM, 1024);
              umma_f16(tmem_base + 256 * nb, a, bd, C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&v_empty[vs]);
          umma_commit(&p_empty[ps]);
          umma_commit(o_done);
        }
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never);
      }
      __syncwarp();
    }

    // ------------------------------------------------------------ epilogue (warps 0-11)
    // O is final once the drain commit has landed. Warps w, w + 4, ... read
    // the same 32 TMEM lanes (32 (w % 4) ...) and split the 32 chunks of 16
    // columns between them.
    // With key splits, split s owns the head rows [128 s / S, 128 (s+1) / S):
    // before the cluster barrier every value CTA writes the rows it does not
    // own (unnormalised, with their (max, sum)) to the workspace; after it,
    // each merges its own rows, read straight from tensor memory, with the
    // other splits' copies of them and writes the output.
    const int own_lo = split * C::M / S, own_hi = (split + 1) * C::M / S;
    const int h = (warp & 3) * 32 + lane;
    const bool owned = h >= own_lo && h < own_hi;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    constexpr int GROUPS = C::EPI_WARPS / 4;  // warps per TMEM sub-partition
    const int third = warp >> 2;              // column group 0 .. GROUPS-1
    const int c_lo = 16 * (third * (C::DC / 16) / GROUPS);
    const int c_hi = 16 * ((third + 1) * (C::DC / 16) / GROUPS);
    float2 ml = make_float2(-INFINITY, 0.0f);
    bool ok = false;
    if (warp < C::EPI_WARPS) {
      ok = mbar_wait_cluster_all(fin_ready, 0, abort_flag);
      if (ok) ml = __ldcg(&fin[h]);
      if (ok) ok = mbar_wait_warp(drain, 0, abort_flag);
      if (ok) {
        tc_fence_after();
        if (S == 1) {
          const float inv = (ml.y > 0.0f) ? 1.0f / ml.y : 0.0f;
          const int64_t row = static_cast<int64_t>(t) * C::M + h;
#pragma unroll 1
          for (int c = c_lo; c < c_hi; c += 16) {
            float o[16];
            tmem_ld16(tmem_base + lane_addr + c, o);
            tmem_wait_ld();
            uint32_t w8[8];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
              // a row with no valid key writes zeros whatever its O holds
              const __nv_bfloat162 o2 = inv != 0.0f ? __floats2bfloat162_rn(o[u] * inv, o[u + 1] * inv)
                                                    : __floats2bfloat162_rn(0.0f, 0.0f);
              w8[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * C::DC + c);
            dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
          }
          if (third == 0 && p.lse) p.lse[row] = (ml.y > 0.0f) ? (ml.x + log2f(ml.y)) * 0.69314718055994531f : -INFINITY;
        } else if (__any_sync(0xffffffffu, !owned)) {
          // rows other splits own: unnormalised rows ([column / 4][row] blocks) and statistics -> workspace
          float4* po = reinterpret_cast<float4*>(p.part_o + pair * C::M * C::DC) + h;
#pragma unroll 1
          for (int c = c_lo; c < c_hi; c += 16) {
            float o[16];
            tmem_ld16(tmem_base + lane_addr + c, o);
            tmem_wait_ld();
            if (!owned) {
#pragma unroll
              for (int u = 0; u < 4; ++u)
                po[(c / 4 + u) * C::M] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
            }
          }
          if (third == 0 && !owned) p.part_ml[pair * C::M + h] = ml;
          fence_proxy_async_global();  // the owner reads these rows through the async proxy (TMA)
        }
      }
    }
    if (S > 1) {
      cluster_sync_all();  // every split's rows for the others are in the workspace
      uint64_t* merge_full = bars + C::MERGE_BAR;
      const int own_n = C::M / S;
      const int64_t grp = static_cast<int64_t>(t) * S;
      const int issuer_warp = own_lo / 32;  // the first warp of the owned rows
      if (warp == issuer_warp && lane == 0 && ok) {
        fence_proxy_async_global();
        mbar_arrive_expect_tx(merge_full, (S - 1) * C::box_bytes(S));
        for (int sp = 0, i = 0; sp < S; ++sp) {
          if (sp == split) continue;
          tma_load_2d(smem_u32(smem + C::B_OFF_V + i * C::box_bytes(S)), &pmap, own_lo * 4,
                      static_cast<int32_t>((grp + sp) * (C::DC / 4)), merge_full);
          ++i;
        }
      }
      if (warp < C::EPI_WARPS && ok && __any_sync(0xffffffffu, owned)) {
        // merge the rows this split owns: its own (tensor memory) with the
        // other splits' (shared memory), with a running maximum
        float Mx = ml.x, L = ml.y;
        if (!(L > 0.0f)) {
          Mx = -INFINITY;
          L = 0.0f;
        }
        float fo[C::MAX_SPLITS], fl = 1.0f;  // per-source factors onto the common maximum
        {
          float2 pm[C::MAX_SPLITS];
          float nm = Mx;
#pragma unroll
          for (int sp = 0; sp < C::MAX_SPLITS; ++sp) {
            pm[sp] = make_float2(-INFINITY, 0.0f);
            if (sp < S && sp != split && owned) {
              pm[sp] = __ldcg(&p.part_ml[(grp + sp) * C::M + h]);
              if (!(pm[sp].y > 0.0f)) pm[sp] = make_float2(-INFINITY, 0.0f);
              nm = fmaxf(nm, pm[sp].x);
            }
          }
          const bool any = nm != -INFINITY;
          fl = (any && L > 0.0f) ? exp2f(Mx - nm) : 0.0f;
          float Lt = L * fl;
#pragma unroll
          for (int sp = 0; sp < C::MAX_SPLITS; ++sp) {
            fo[sp] = (any && pm[sp].y > 0.0f) ? exp2f(pm[sp].x - nm) : 0.0f;
            Lt += pm[sp].y * fo[sp];
          }
          Mx = nm;
          L = Lt;
        }
        const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
        const int64_t row = static_cast<int64_t>(t) * C::M + h;
        const int hr = owned ? h - own_lo : 0;
        if (mbar_wait_warp(merge_full, 0, abort_flag)) {
#pragma unroll 1
          for (int c = c_lo; c < c_hi; c += 16) {
            float o[16];
            tmem_ld16(tmem_base + lane_addr + c, o);
            tmem_wait_ld();
            if (owned) {
#pragma unroll
              for (int u = 0; u < 16; ++u) o[u] *= fl;
#pragma unroll
              for (int sp = 0, i = 0; sp < C::MAX_SPLITS; ++sp) {
                if (sp >= S || sp == split) continue;
                const float4* px = reinterpret_cast<const float4*>(smem + C::B_OFF_V + i * C::box_bytes(S)) + hr;
                ++i;
                if (fo[sp] == 0.0f) continue;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const float4 x = px[(c / 4 + u) * own_n];
                  o[4 * u] = fmaf(x.x, fo[sp], o[4 * u]);
                  o[4 * u + 1] = fmaf(x.y, fo[sp], o[4 * u + 1]);
                  o[4 * u + 2] = fmaf(x.z, fo[sp], o[4 * u + 2]);
                  o[4 * u + 3] = fmaf(x.w, fo[sp], o[4 * u + 3]);
                }
              }
              uint32_t w8[8];
#pragma unroll
              for (int u = 0; u < 16; u += 2) {
                // a row with no valid key writes zeros whatever its O holds
                const __nv_bfloat162 o2 = inv != 0.0f ? __floats2bfloat162_rn(o[u] * inv, o[u + 1] * inv)
                                                      : __floats2bfloat162_rn(0.0f, 0.0f);
                w8[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
              }
              uint4* dst = reinterpret_cast<uint4*>(p.out + row * C::DC + c);
              dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
              dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
            }
          }
          if (third == 0 && owned && p.lse) p.lse[row] = (L > 0.0f) ? (Mx + log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
      }
      if (warp == issuer_warp && lane == 0 && ok) {
        volatile int never = 0;  // the copies must land before the CTA can retire
        mbar_wait(merge_full, 0, &never);
      }
      __syncwarp();
    }
  }
  if (score_cta && S > 1) cluster_sync_all();  // pairs with the value CTAs' barrier above

  // The next kernel of the stream may be scheduled now (see the indexer).
  pdl_launch_dependents();

  // No CTA may retire while its partner can still address its shared memory.
  tc_fence_before();
  cluster_sync_all();
  if (warp == C::MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  canary_check(smem, C::SMEM_BYTES);
}

}  // namespace dsa
