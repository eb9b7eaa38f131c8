// indexer.cuh -- Lightning Indexer scores on tcgen05 tensor cores.
//
// Computes, for each query token t and each causal history position s,
//   I[t,s] = sigma_s * sum_j w[t,j] * max(0, q_I[t,j,:] . k[s,:])
// ("relevance scoring" and "head-weight weighting": section 3 of
// "Optimizing Inference for New Model Architectures ..."; section 1 of
// "Day-0 Inference Optimization for a New Sparse Attention Architecture"),
// where sigma_s is the key's FP8 scale (1 for BF16 keys). Because sigma_s >= 0
// and max(0, .) is positively homogeneous, scaling after the head sum equals
// scoring the dequantised key.
//
// Design (swapped AB): one tcgen05.mma tile is M = 128 keys x N = G tokens x
// H_I heads x K = d_I, so the large operand (the key cache, streamed from HBM
// by TMA) is A and the small one (the group's queries, resident in shared
// memory) is B. The fp32 accumulator lives in TMEM (two buffers); the
// epilogue warps read one key row per thread with tcgen05.ld, apply ReLU, the
// head weights, the FP8 scale and the causal / length mask, and store the
// scores coalesced. FP8 keys are TMA-loaded as bytes and widened to bf16 in
// shared memory by four converter warps (exact: every E4M3 value is a bf16).
// Key formats (KF): 0 BF16; 1 FP8 with one fp32 scale per key (sigma_s
// above); 2 MXFP8, one power-of-two (E8M0) scale per 32 elements (Index Q/K
// Uses MXFP8, section 4.2 of "Inference Adaptation and Performance
// Optimization for New Large Language Model Architectures"), applied by the
// converters while widening (exact in bf16; sigma_s = 1), its scale bytes
// copied into the stage with the codes when their rows are 16-byte aligned.
//
// Roles: warp 0 = TMA producer, warp 1 = MMA issuer (+ TMEM owner), then the
// epilogue warps (four; for groups of 64-head tokens up to four per TMEM
// sub-partition, splitting the tokens), then four FP8 converters (FP8 only).
#pragma once
#include "dsa_common.cuh"
#include "quant.cuh"

namespace dsa {

struct IndexerParams {
  const int32_t* cu_q;
  const int32_t* q_pos;
  const int32_t* seq_lens;
  int32_t B;
  int32_t L_max;
  const __nv_bfloat16* q;   // [T, HI, DIN]
  const float* w;           // [T, HI]
  const float* k_scale;     // one scale per cache row (FP8) or null
  const uint8_t* k_mx;      // MXFP8: E8M0 bytes [cache rows, DIN / 32] or null
  int32_t scale_bulk;       // MXFP8: scale bytes are copied into the stage (16-byte aligned rows)
  int64_t rows;             // cache rows (contiguous B * L_max, or the page pool)
  float* scores;            // [T, ld]
  int64_t ld;
  int32_t tiles_per_cta;
  CacheMap cm;              // cache rows (contiguous or paged)
};

template <int HI, int DIN, int G, int KF>
struct IndexerCfg {
  static constexpr bool FP8 = KF != 0;                     // 8-bit codes (FP8 or MXFP8), widened on chip
  static constexpr int SROW = KF == 2 ? DIN / 32 : 0;      // MXFP8 scale bytes per key row (staged)
  static constexpr int DK = DIN < 64 ? 64 : DIN;           // K padded to whole 128-byte atoms
  static constexpr int AK = DK / 64;                       // atom columns along K
  static constexpr int N = ((G * HI + 15) / 16) * 16;      // MMA N
  static constexpr int TILE_BYTES = 128 * DK * 2;          // bf16 key tile (A operand)
  static constexpr int Q_BYTES = N * DK * 2;               // query tile (B operand)
  static constexpr int U8_TILE = 128 * DIN;                // FP8 staging tile
  // Stages: small enough that two CTAs share an SM when the query tile is
  // small (decode), so one CTA's prologue / tail overlaps the other's stream.
  static constexpr int ST = FP8 ? (G == 1 ? 2 : 3) : 3;
  static constexpr int CS = 2;                             // converted bf16 tiles (FP8)
  static constexpr int NACC = 2;                           // TMEM accumulator buffers
  static constexpr int TMEM_COLS = (NACC * N <= 32) ? 32 : (NACC * N <= 64) ? 64 : (NACC * N <= 128) ? 128
                                   : (NACC * N <= 256) ? 256 : 512;
  // epilogue warps: EPI_PARTS per TMEM sub-partition, each taking G / EPI_PARTS
  // of the group's tokens (64-head tokens: four parts for four-token groups of
  // BF16 keys; with 8-bit keys the converter warps leave registers for two)
  static constexpr int EPI_PARTS =
      (G > 1 && HI % 64 == 0) ? ((G % 4 == 0 && KF == 0) ? 4 : G % 2 == 0 ? 2 : 1) : 1;
  static constexpr int EPI_WARPS = 4 * EPI_PARTS;
  static constexpr int CONV_WARPS = FP8 ? 4 : 0;          // 8-bit -> bf16 converters
  static constexpr int NUM_WARPS = 2 + EPI_WARPS + CONV_WARPS;
  static constexpr int THREADS = NUM_WARPS * 32;
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_STAGE = OFF_Q + ((Q_BYTES + 1023) / 1024) * 1024;
  static constexpr int STAGE_BYTES = FP8 ? U8_TILE + 128 * SROW : TILE_BYTES;
  static constexpr int OFF_CONV = OFF_STAGE + ((ST * STAGE_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_BAR = OFF_CONV + (FP8 ? CS * TILE_BYTES : 0);
  static constexpr int NUM_BARS = 2 * ST + 2 * NACC + 2 * CS + 1;
  static constexpr int OFF_W = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_MISC = OFF_W + G * HI * 4;
  // No alignment slack: with no static shared memory the dynamic window
  // starts 1024-byte aligned (checked at run time, see the kernel prologue).
  static constexpr int SMEM_BYTES = OFF_MISC + 64;
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, N, false, false);
  static constexpr int MIN_CTAS = (SMEM_BYTES <= 113 * 1024) ? 2 : 1;  // CTAs per SM the footprint allows
  static_assert(N <= 256, "indexer MMA N must be <= 256");
  static_assert(ST >= 2, "need at least two stages");
};

template <int HI, int DIN, int G, int KF>
__global__ void __launch_bounds__(IndexerCfg<HI, DIN, G, KF>::THREADS, IndexerCfg<HI, DIN, G, KF>::MIN_CTAS)
    indexer_scores_kernel(const __grid_constant__ CUtensorMap kmap, const IndexerParams p) {
  using C = IndexerCfg<HI, DIN, G, KF>;
  constexpr bool FP8 = C::FP8;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-byte alignment
    if (threadIdx.x == 0) set_device_status(DSA_ERR_DEVICE_LAYOUT);
    return;
  }
  canary_set(smem, C::SMEM_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                      // [ST]  TMA -> MMA / converters
  uint64_t* empty = bars + C::ST;             // [ST]  MMA / converters -> TMA
  uint64_t* acc_full = empty + C::ST;         // [NACC] MMA -> epilogue
  uint64_t* acc_empty = acc_full + C::NACC;   // [NACC] epilogue -> MMA
  uint64_t* conv_full = acc_empty + C::NACC;  // [CS] converters -> MMA
  uint64_t* conv_empty = conv_full + C::CS;   // [CS] MMA -> converters
  uint64_t* drain = conv_empty + C::CS;       // teardown
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);
  // misc: [0] b, [1] t0, [2] nt, [3] tile_begin, [4] tile_end, [5] tmem base,
  //       [6] abort, [7..7+G) n_valid per token
  volatile int* abort_flag = misc + 6;

  const int warp = warp_id();
  const int lane = lane_id();
  // Under programmatic dependent launch this grid may start before the
  // previous kernel of the stream has finished, and that kernel may have
  // written any input, so nothing is read before the wait. Only then may the
  // Top-K be scheduled: it reads the batch description before its own wait.
  pdl_wait_prior();
  pdl_launch_dependents();  // the Top-K may be scheduled; it waits for these scores
  if (threadIdx.x == 0) prefetch_tensormap(&kmap);

  // Single-token groups: the query rows depend only on the block index, so
  // their loads go out before the group lookup and overlap it.
  constexpr int QCPR = C::DK / 8;                                   // 16-byte chunks per B row
  constexpr int QPT = (C::N * QCPR + C::THREADS - 1) / C::THREADS;  // chunks per thread
  uint4 qreg[G == 1 ? QPT : 1];
  if constexpr (G == 1) {
    const bool tok_ok = static_cast<int>(blockIdx.x) < __ldg(p.cu_q + p.B);
#pragma unroll
    for (int u = 0; u < QPT; ++u) {
      const int i = threadIdx.x + u * C::THREADS;
      const int n = i / QCPR, c = i % QCPR;
      qreg[u] = make_uint4(0u, 0u, 0u, 0u);
      if (tok_ok && i < C::N * QCPR && n < HI && c * 8 < DIN)
        qreg[u] = __ldg(reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(blockIdx.x) * HI + n) * DIN + c * 8)));
    }
  }

  if (warp == 0) {
    // Locate this CTA's token group: groups are G consecutive tokens of one sequence.
    int b = -1, g = blockIdx.x;
    if constexpr (G == 1) {
      // one token per group: group index == token index
      if (static_cast<int>(blockIdx.x) < __ldg(p.cu_q + p.B)) {
        b = seq_of_token_warp(p.cu_q, p.B, blockIdx.x);
        g = blockIdx.x - __ldg(p.cu_q + b);
      }
    } else {
      // warp-parallel scan of groups-per-sequence, 32 sequences per round
      int before = 0;
      for (int c = 0; c < p.B && b < 0; c += 32) {
        const int bb = c + lane;
        const int ng = (bb < p.B) ? (__ldg(p.cu_q + bb + 1) - __ldg(p.cu_q + bb) + G - 1) / G : 0;
        int incl = ng;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        const int excl = incl - ng;
        const unsigned hit = __ballot_sync(0xffffffffu, ng > 0 && static_cast<int>(blockIdx.x) - before >= excl &&
                                                            static_cast<int>(blockIdx.x) - before < incl);
        if (hit) {
          const int src = __ffs(hit) - 1;
          b = c + src;
          g = static_cast<int>(blockIdx.x) - before - __shfl_sync(0xffffffffu, excl, src);
        }
        before += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
    if (lane == 0) {
      int tb = 0, te = 0, t0 = 0, nt = 0;
      if (b >= 0) {
        t0 = __ldg(p.cu_q + b) + g * G;
        nt = min(G, __ldg(p.cu_q + b + 1) - t0);
        const int len = min(__ldg(p.seq_lens + b), p.L_max);
        int nk = 0;
        for (int i = 0; i < G; ++i) {
          int nv = 0;
          if (i < nt) nv = max(0, min(__ldg(p.q_pos + t0 + i) + 1, len));
          misc[7 + i] = nv;
          nk = max(nk, nv);
        }
        misc[12] = nk;
        const int n_tiles = (nk + 127) / 128;
        tb = blockIdx.y * p.tiles_per_cta;
        te = min(n_tiles, tb + p.tiles_per_cta);
      }
      misc[0] = b;
      misc[1] = t0;
      misc[2] = nt;
      misc[3] = tb;
      misc[4] = te;
      misc[6] = 0;
      for (int i = 0; i < C::ST; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], FP8 ? C::CONV_WARPS : 1);
      }
      for (int i = 0; i < C::NACC; ++i) {
        mbar_init(&acc_full[i], 1);
        mbar_init(&acc_empty[i], C::EPI_WARPS);
      }
      for (int i = 0; i < C::CS; ++i) {
        mbar_init(&conv_full[i], C::CONV_WARPS);
        mbar_init(&conv_empty[i], 1);
      }
      mbar_init(drain, 1);
      fence_mbar_init();
    }
  }
  __syncthreads();
  const int b = misc[0];
  const int tile_begin = misc[3];
  const int tile_end = misc[4];
  if (b < 0 || tile_begin >= tile_end) return;  // uniform across the CTA
  const int t0 = misc[1];
  const int nt = misc[2];
  const int nk = misc[12];  // causal candidates of the group's last token
  const int n_tiles = tile_end - tile_begin;
  const int64_t row0 = static_cast<int64_t>(b) * p.L_max;

  // The first ST key tiles go out now (every stage starts empty), so their
  // latency overlaps the query staging and the TMEM allocation below.
  auto issue_tile = [&](int it) {
    const int st = it % C::ST;
    const int s0 = (tile_begin + it) * 128;  // first key position of the tile
    const uint32_t dst = smem_u32(smem + C::OFF_STAGE + st * C::STAGE_BYTES);
    if (!p.cm.paged()) {
      const int32_t y = static_cast<int32_t>(row0 + s0);
      if constexpr (FP8) {
        // MXFP8: scale rows y .. y + 127, clipped at the end of the cache
        const int64_t left = p.rows - y;
        const uint32_t sbytes = (C::SROW && p.scale_bulk) ? C::SROW * static_cast<uint32_t>(left < 128 ? left : 128) : 0u;
        mbar_arrive_expect_tx(&full[st], C::U8_TILE + sbytes);
        tma_load_2d(dst, &kmap, 0, y, &full[st]);
        if (sbytes) bulk_load(dst + C::U8_TILE, p.k_mx + static_cast<int64_t>(y) * C::SROW, sbytes, &full[st]);
      } else {
        mbar_arrive_expect_tx(&full[st], C::TILE_BYTES);
#pragma unroll
        for (int a = 0; a < C::AK; ++a) tma_load_2d(dst + a * 16384, &kmap, a * 64, y, &full[st]);
      }
    } else {
      // paged: two 64-row boxes (a page holds a whole number of them); a half
      // past the last candidate reloads the first half (its rows are masked)
      mbar_arrive_expect_tx(&full[st], FP8 ? C::U8_TILE + (p.scale_bulk ? 128 * C::SROW : 0) : C::TILE_BYTES);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int32_t y = p.cm.row_checked(b, (s0 + 64 * h < nk) ? s0 + 64 * h : s0);
        if constexpr (FP8) {
          tma_load_2d(dst + h * 64 * DIN, &kmap, 0, y, &full[st]);
          if (C::SROW && p.scale_bulk)
            bulk_load(dst + C::U8_TILE + 64 * C::SROW * h, p.k_mx + static_cast<int64_t>(y) * C::SROW, 64 * C::SROW,
                      &full[st]);
        } else {
#pragma unroll
          for (int a = 0; a < C::AK; ++a) tma_load_2d(dst + a * 16384 + h * 8192, &kmap, a * 64, y, &full[st]);
        }
      }
    }
  };
  const int prologue_tiles = min(n_tiles, C::ST);
  if (threadIdx.x == 0)
    for (int it = 0; it < prologue_tiles; ++it) issue_tile(it);

  // ---- setup: query tile, head weights, TMEM
  // B operand: row n = (token g, head j) = g*HI + j; zero rows beyond the group / padding.
  {
    constexpr int CHUNKS_PER_ROW = C::DK / 8;
    uint8_t* qs = smem + C::OFF_Q;
    if constexpr (G == 1) {
#pragma unroll
      for (int u = 0; u < QPT; ++u) {
        const int i = threadIdx.x + u * C::THREADS;
        if (i < C::N * CHUNKS_PER_ROW) {
          const int n = i / CHUNKS_PER_ROW, c = i % CHUNKS_PER_ROW;
          *reinterpret_cast<uint4*>(qs + (c / 8) * (C::N * 128) + sw128_offset(n, c % 8)) = qreg[u];
        }
      }
    } else {
      for (int i = threadIdx.x; i < C::N * CHUNKS_PER_ROW; i += C::THREADS) {
        const int n = i / CHUNKS_PER_ROW;
        const int c = i % CHUNKS_PER_ROW;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        const int g = n / HI, j = n % HI;
        if (g < nt && c * 8 < DIN)
          v = *reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(t0 + g) * HI + j) * DIN + c * 8));
        *reinterpret_cast<uint4*>(qs + (c / 8) * (C::N * 128) + sw128_offset(n, c % 8)) = v;
      }
    }
    for (int i = threadIdx.x; i < G * HI; i += C::THREADS) {
      const int g = i / HI;
      w_s[i] = (g < nt) ? __ldg(p.w + static_cast<int64_t>(t0 + g) * HI + (i % HI)) : 0.0f;
    }
    if constexpr (FP8 && DIN < C::DK) {
      // zero the converted tiles once: the padding columns are never written again
      uint4* cz = reinterpret_cast<uint4*>(smem + C::OFF_CONV);
      for (int i = threadIdx.x; i < C::CS * C::TILE_BYTES / 16; i += C::THREADS) cz[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc + 5), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(misc[5]);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int issued = prologue_tiles;
      for (int it = prologue_tiles; it < n_tiles; ++it) {
        const int st = it % C::ST;
        if (!mbar_wait(&empty[st], ((it / C::ST) & 1) ^ 1, abort_flag)) break;
        issue_tile(it);
        ++issued;
      }
      // drain: every issued TMA load must land before the CTA can retire
      for (int it = max(0, issued - C::ST); it < issued; ++it) {
        const int st = it % C::ST;
        volatile int never = 0;
        mbar_wait(&full[st], (it / C::ST) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int it = 0; it < n_tiles; ++it) {
        const int acc = it % C::NACC;
        uint32_t a_base;
        if constexpr (FP8) {
          const int cs = it % C::CS;
          if (!mbar_wait(&conv_full[cs], (it / C::CS) & 1, abort_flag)) break;
          a_base = smem_u32(smem + C::OFF_CONV + cs * C::TILE_BYTES);
        } else {
          const int st = it % C::ST;
          if (!mbar_wait(&full[st], (it / C::ST) & 1, abort_flag)) break;
          a_base = smem_u32(smem + C::OFF_STAGE + st * C::TILE_BYTES);
        }
        if (!mbar_wait(&acc_empty[acc], ((it / C::NACC) & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t b_base = smem_u32(smem + C::OFF_Q);
        const uint32_t d_tmem = tmem_base + acc * C::N;
#pragma unroll
        for (int k = 0; k < C::DK / 16; ++k) {
          const uint64_t adesc = smem_desc_sw128(a_base + (k / 4) * 16384 + (k % 4) * 32, 16, 1024);
          const uint64_t bdesc = smem_desc_sw128(b_base + (k / 4) * (C::N * 128) + (k % 4) * 32, 16, 1024);
          umma_f16(d_tmem, adesc, bdesc, C::IDESC, k > 0 ? 1u : 0u);
        }
        if constexpr (FP8)
          umma_commit(&conv_empty[it % C::CS]);
        else
          umma_commit(&empty[it % C::ST]);
        umma_commit(&acc_full[acc]);
      }
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else if (warp >= 2 && warp < 2 + C::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int sub = warp & 3;                 // TMEM sub-partition this warp may access
    const int part = (warp - 2) / 4;          // this warp's share of the group's tokens
    const int r = sub * 32 + lane;            // key row inside the tile
    const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
    int nv[G];
#pragma unroll
    for (int g = 0; g < G; ++g) nv[g] = misc[7 + g];
    for (int it = 0; it < n_tiles; ++it) {
      const int acc = it % C::NACC;
      if (!mbar_wait_warp(&acc_full[acc], (it / C::NACC) & 1, abort_flag)) break;
      tc_fence_after();
      float score[G];
#pragma unroll
      for (int g = 0; g < G; ++g) score[g] = 0.0f;
      if constexpr (C::N <= 64) {
        // all N columns in flight at once, one wait
        float v[C::N / 16][16];
#pragma unroll
        for (int c = 0; c < C::N / 16; ++c) tmem_ld16(tmem_base + lane_addr + acc * C::N + c * 16, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < C::N / 16; ++c) {
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int col = c * 16 + u;
            const int g = col / HI;
            if (g < G) score[g] = fmaf(w_s[col], fmaxf(v[c][u], 0.0f), score[g]);
          }
        }
      } else if constexpr (HI % 64 == 0) {
        // wide tiles, 64 heads per token: one token's 64 columns per TMEM
        // round trip (four loads in flight, one wait); each warp takes the
        // columns of its share of the tokens
        constexpr int COLS = C::N / C::EPI_PARTS;
#pragma unroll 1
        for (int c = part * COLS; c < (part + 1) * COLS; c += 64) {
          float v[4][16];
#pragma unroll
          for (int q = 0; q < 4; ++q) tmem_ld16(tmem_base + lane_addr + acc * C::N + c + 16 * q, v[q]);
          tmem_wait_ld();
          float t4[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // four partial sums (short dependency chains)
#pragma unroll
          for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int u = 0; u < 16; ++u) t4[u & 3] = fmaf(w_s[c + 16 * q + u], fmaxf(v[q][u], 0.0f), t4[u & 3]);
          const float tok = (t4[0] + t4[1]) + (t4[2] + t4[3]);
          const int g = c / HI;
#pragma unroll
          for (int gg = 0; gg < G; ++gg)
            if (gg == g) score[gg] += tok;
        }
      } else {
        // wide tiles (HI >= 16): a 16-column chunk never straddles two tokens
        static_assert(HI % 16 == 0, "wide indexer tiles need HI % 16 == 0");
#pragma unroll 1
        for (int c = 0; c < C::N; c += 16) {
          float v[16];
          tmem_ld16(tmem_base + lane_addr + acc * C::N + c, v);
          tmem_wait_ld();
          float t4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
          for (int u = 0; u < 16; ++u) t4[u & 3] = fmaf(w_s[c + u], fmaxf(v[u], 0.0f), t4[u & 3]);
          const float chunk = (t4[0] + t4[1]) + (t4[2] + t4[3]);
          const int g = c / HI;
#pragma unroll
          for (int gg = 0; gg < G; ++gg)
            if (gg == g) score[gg] += chunk;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[acc]);
      const int64_t s = static_cast<int64_t>(tile_begin + it) * 128 + r;
      float sigma = 1.0f;
      if constexpr (KF == 1) {
        if (s < nk) {
          bool ok;
          const int32_t kr = p.cm.row(b, static_cast<int>(s), ok);
          sigma = __ldg(p.k_scale + (p.cm.paged() ? static_cast<int64_t>(kr) : row0 + s));
        }
      }
      if (s < p.ld) {
        constexpr int GPART = G / C::EPI_PARTS;  // tokens this warp scores
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (g < nt && g / GPART == part) {
            const float val = (s < nv[g]) ? score[g] * sigma : -INFINITY;
            p.scores[static_cast<int64_t>(t0 + g) * p.ld + s] = val;
          }
        }
      }
    }
  } else if constexpr (FP8) {
    // ------------------------------------------------------------ FP8 -> bf16 converters
    constexpr int CT = 32 * C::CONV_WARPS;                 // converter threads
    const int ct = threadIdx.x - (2 + C::EPI_WARPS) * 32;  // 0 .. CT - 1
    constexpr int CPR = DIN / 16;         // 16-byte input chunks per key row
    for (int it = 0; it < n_tiles; ++it) {
      const int st = it % C::ST;
      const int cs = it % C::CS;
      if (!mbar_wait(&full[st], (it / C::ST) & 1, abort_flag)) break;
      if (!mbar_wait(&conv_empty[cs], ((it / C::CS) & 1) ^ 1, abort_flag)) break;
      const uint8_t* src = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
      uint8_t* dst = smem + C::OFF_CONV + cs * C::TILE_BYTES;
      const int s0 = (tile_begin + it) * 128;  // first key position of the tile
      // all of the thread's chunks (and MXFP8 scale bytes) are loaded first
      static_assert((128 * CPR) % CT == 0, "whole chunks per converter thread");
      constexpr int PER = 128 * CPR / CT;
      uint4 raws[PER];
      int bytes[PER];
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int i = ct + u * CT;
        const int row = i / CPR;
        const int c = i % CPR;
        raws[u] = *reinterpret_cast<const uint4*>(src + row * DIN + c * 16);
        bytes[u] = 127;
        if constexpr (KF == 2) {
          if (p.scale_bulk) {
            bytes[u] = src[C::U8_TILE + row * (DIN / 32) + c / 2];
          } else {
            // rows past the last candidate are masked; read a row that exists
            bool rok;
            const int sr = s0 + row < nk ? s0 + row : s0;
            bytes[u] = __ldg(p.k_mx + static_cast<int64_t>(p.cm.row(b, sr, rok)) * (DIN / 32) + c / 2);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int i = ct + u * CT;
        const int row = i / CPR;
        const int c = i % CPR;
        const uint32_t words[4] = {raws[u].x, raws[u].y, raws[u].z, raws[u].w};
        // MXFP8: 2^e of the chunk's 32-element group (exact scaling)
        const float m = KF == 2 ? exp2_int(bytes[u] - 127) : 1.0f;
        uint32_t outw[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __half2_raw h01 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(words[q] & 0xFFFF), __NV_E4M3);
          const __half2_raw h23 = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(words[q] >> 16), __NV_E4M3);
          float2 f01 = __half22float2(__half2(h01));
          float2 f23 = __half22float2(__half2(h23));
          if constexpr (KF == 2) {
            f01.x *= m;
            f01.y *= m;
            f23.x *= m;
            f23.y *= m;
          }
          const __nv_bfloat162 b01 = __float22bfloat162_rn(f01);
          const __nv_bfloat162 b23 = __float22bfloat162_rn(f23);
          outw[2 * q] = *reinterpret_cast<const uint32_t*>(&b01);
          outw[2 * q + 1] = *reinterpret_cast<const uint32_t*>(&b23);
        }
        const int q0 = 2 * c;  // 16-byte bf16 chunk index along the row
        *reinterpret_cast<uint4*>(dst + (q0 / 8) * 16384 + sw128_offset(row, q0 % 8)) =
            make_uint4(outw[0], outw[1], outw[2], outw[3]);
        const int q1 = q0 + 1;
        *reinterpret_cast<uint4*>(dst + (q1 / 8) * 16384 + sw128_offset(row, q1 % 8)) =
            make_uint4(outw[4], outw[5], outw[6], outw[7]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&empty[st]);
        mbar_arrive(&conv_full[cs]);
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  canary_check(smem, C::SMEM_BYTES);
}

}  // namespace dsa
