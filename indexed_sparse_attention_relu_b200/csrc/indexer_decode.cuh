// indexer_decode.cuh -- Lightning Indexer scores when every group is one query
// token (decode): the same scores as indexer_scores_kernel,
//   I[t,s] = sigma_s * sum_j w[t,j] * max(0, q_I[t,j,:] . k[s,:]),
// ("relevance scoring" and "head-weight weighting": section 3 of "Optimizing
// Inference for New Model Architectures ..."; section 1 of "Day-0 Inference
// Optimization for a New Sparse Attention Architecture"), with the work laid
// out for HBM rather than per token.
//
// Work split. The key tiles of all tokens (128 causal candidates each) form
// one flattened list; each of the grid's CTAs (one per SM) takes an equal
// contiguous range of it, so every SM streams the same number of key bytes
// whatever the context lengths, and a range may run across several tokens
// ("segments"). Every CTA computes the same list from cu_q / q_pos /
// seq_lens (a warp scan over the sequences) and keeps its segments in shared
// memory.
//
// Pipeline: warp 0 issues, per segment, the token's query tile (TMA, straight
// into the MMA's swizzled B layout) and head weights into one of two query
// buffers, and per key tile a TMA load into one of ST stages. Warp 1 issues
// tcgen05.mma with M = 128 keys, N = heads, K = d_I into two TMEM
// accumulators. Epilogue warps read one key row per thread, apply ReLU,
// the weights, the key's scale (FP8) and the causal / length mask and store
// the scores. 8-bit codes are widened to bf16 by converter warps (exact:
// every E4M3 value is a bf16). Key formats (KF): BF16; FP8 with one fp32 scale
// per key, applied after the head sum; MXFP8 with one power-of-two (E8M0)
// scale per 32 elements, applied by the converters while widening (still
// exact in bf16), with queries given in bf16 (the host widens MXFP8 queries
// first). A tile's scales ride in its stage (one bulk copy per 64 or 128
// rows) when the scale rows are 16-byte aligned; otherwise each reader loads
// them from global memory. FP8 / MXFP8 stages are freed by the epilogue,
// after every reader of the stage is done. Every wait is bounded.
#pragma once
#include "dsa_common.cuh"
#include "quant.cuh"

namespace dsa {

struct IdxDecParams {
  const int32_t* cu_q;
  const int32_t* q_pos;
  const int32_t* seq_lens;
  const float* k_scale;     // FP8 keys: one fp32 scale per cache row
  const uint8_t* k_mx;      // MXFP8 keys: E8M0 bytes [cache rows, d_I / 32]
  int32_t scale_bulk;       // scales are copied into the stage (16-byte aligned rows)
  int64_t rows;          // cache rows (contiguous B * L_max, or the page pool)
  int32_t B;
  int32_t T;
  int32_t L_max;
  float* scores;  // [T, ld]
  int64_t ld;
  CacheMap cm;    // cache rows (contiguous or paged)
};

// Key formats of the indexer kernels.
constexpr int KF_BF16 = 0, KF_FP8 = 1, KF_MX = 2;

template <int HI, int DIN, int KF>
struct IdxDecCfg {
  static constexpr bool FP8 = KF != KF_BF16;             // 8-bit codes, widened by converter warps
  static constexpr int SROW = KF == KF_FP8 ? 4 : KF == KF_MX ? DIN / 32 : 0;  // scale bytes per key row
  static constexpr int EPI_G = KF != KF_BF16 ? 2 : 1;
  static constexpr int CONV_W = KF == KF_FP8 ? 6 : KF == KF_MX ? 8 : 0;
  static constexpr int DK = DIN < 64 ? 64 : DIN;         // K padded to whole 128-byte atoms
  static constexpr int AK = DK / 64;                     // atom columns along K
  static constexpr int N = ((HI + 15) / 16) * 16;        // MMA N (zero rows beyond HI)
  static constexpr int TILE_BYTES = 128 * DK * 2;        // bf16 key tile (A operand)
  static constexpr int U8_TILE = 128 * DIN;              // FP8 codes of a tile
  static constexpr int STAGE_BYTES = FP8 ? U8_TILE + 128 * SROW : TILE_BYTES;  // codes + the tile's scales
  static constexpr int ST = FP8 ? 6 : 5;                 // key stages
  static constexpr int CS = 2;                           // converted bf16 tiles (FP8)
  static constexpr int NACC = 2;                         // TMEM accumulators
  static constexpr int TMEM_COLS = (NACC * N <= 32) ? 32 : (NACC * N <= 64) ? 64 : (NACC * N <= 128) ? 128 : 256;
  static constexpr int QB_BYTES = N * DK * 2;            // one query buffer (B operand)
  static constexpr int Q_TX = AK * HI * 128;             // bytes the query TMA writes per buffer
  static constexpr int W_BYTES = ((HI * 4 + 15) / 16) * 16;
  static constexpr int MAXSEG = 256;                     // segments a CTA can hold (tokens <= MAXSEG)
  // Epilogue groups of four warps: with 8-bit keys two groups, group g taking
  // the tiles with it % 2 == g (accumulator g), so two tiles' epilogues run at
  // once (measured 6 % faster on a ragged FP8 decode, 1 % with MXFP8 keys,
  // whose widening also applies the block scales and keeps eight converter
  // warps); BF16 keys keep one group.
  static constexpr int EPI_GROUPS = EPI_G;
  static constexpr int EPI_WARPS = 4 * EPI_GROUPS;
  static constexpr int CONV_WARPS = CONV_W;              // 8-bit -> bf16 converters
  static constexpr int NUM_WARPS = 2 + EPI_WARPS + CONV_WARPS;
  static constexpr int THREADS = NUM_WARPS * 32;
  // shared memory (offsets from the 1024-byte-aligned window)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_STAGE = OFF_Q + 2 * QB_BYTES;
  static constexpr int OFF_CONV = ((OFF_STAGE + ST * STAGE_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_W = OFF_CONV + (FP8 ? CS * TILE_BYTES : 0);
  static constexpr int NUM_BARS = 2 * ST + 2 * NACC + 2 * CS + 4 + 1;
  static constexpr int OFF_BAR = OFF_W + 2 * W_BYTES;
  static constexpr int OFF_SEG = OFF_BAR + NUM_BARS * 8;
  static constexpr int OFF_MISC = OFF_SEG + 5 * MAXSEG * 4;
  static constexpr int SMEM_BYTES = OFF_MISC + 64;
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, N, false, false);
  static_assert(QB_BYTES % 1024 == 0 && OFF_STAGE % 1024 == 0 && TILE_BYTES % 1024 == 0, "swizzled operands");
  static_assert(STAGE_BYTES % 16 == 0 && U8_TILE % 16 == 0, "TMA destinations");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(N <= 256, "MMA N");
};

template <int HI, int DIN, int KF>
__global__ void __launch_bounds__(IdxDecCfg<HI, DIN, KF>::THREADS, 1)
    indexer_decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                          const float* __restrict__ w, const IdxDecParams p) {
  using C = IdxDecCfg<HI, DIN, KF>;
  constexpr bool FP8 = C::FP8;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {  // swizzled tiles need 1024-byte alignment (same in every CTA)
    if (threadIdx.x == 0) set_device_status(DSA_ERR_DEVICE_LAYOUT);
    return;
  }
  canary_set(smem, C::SMEM_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                       // [ST]   producer -> MMA (BF16) or converters + epilogue (FP8)
  uint64_t* empty = full + C::ST;              // [ST]   MMA (BF16) or epilogue (FP8) -> producer
  uint64_t* acc_full = empty + C::ST;          // [NACC] MMA -> epilogue
  uint64_t* acc_empty = acc_full + C::NACC;    // [NACC] epilogue -> MMA
  uint64_t* conv_full = acc_empty + C::NACC;   // [CS]   converters -> MMA
  uint64_t* conv_empty = conv_full + C::CS;    // [CS]   MMA -> converters
  uint64_t* q_full = conv_empty + C::CS;       // [2]    producer -> MMA, epilogue
  uint64_t* q_empty = q_full + 2;              // [2]    MMA + epilogue -> producer
  uint64_t* drain = q_empty + 2;
  int32_t* seg_tok = reinterpret_cast<int32_t*>(smem + C::OFF_SEG);  // token of the segment
  int32_t* seg_t0 = seg_tok + C::MAXSEG;                              // first key tile (within the token)
  int32_t* seg_nt = seg_t0 + C::MAXSEG;                               // key tiles of the segment
  int32_t* seg_nv = seg_nt + C::MAXSEG;                               // causal candidates of the token
  int32_t* seg_b = seg_nv + C::MAXSEG;                                // sequence of the token
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);     // [0] segments, [1] TMEM, [2] abort, [3] tiles
  volatile int* abort_flag = misc + 2;
  float* w_s = reinterpret_cast<float*>(smem + C::OFF_W);
  const int warp = warp_id();
  const int lane = lane_id();
  // Under programmatic dependent launch this grid may start before the
  // previous kernel of the stream has finished, and that kernel may have
  // written any input (queries, keys, weights, the batch description), so
  // nothing is read before the wait. Only then may the Top-K be scheduled: it
  // reads the batch description before its own wait.
  pdl_wait_prior();
  pdl_launch_dependents();  // the Top-K may be scheduled; it waits for these scores

  if (warp == 0) {
    // ---- this CTA's range of the flattened key-tile list, as segments
    if (lane == 0) {
      prefetch_tensormap(&kmap);
      prefetch_tensormap(&qmap);
    }
    // per-sequence key tiles, 32 sequences a round (lane = sequence); the
    // first round is kept in registers for the segment walk below
    auto seq_info = [&](int b, int& t0, int& t1, int& len) -> int {
      int tiles = 0;
      t0 = t1 = len = 0;
      if (b < p.B) {
        t0 = __ldg(p.cu_q + b);
        t1 = __ldg(p.cu_q + b + 1);
        len = min(__ldg(p.seq_lens + b), p.L_max);
        for (int t = t0; t < t1; ++t) tiles += (max(0, min(__ldg(p.q_pos + t) + 1, len)) + 127) / 128;
      }
      return tiles;
    };
    int f_t0, f_t1, f_len;
    const int f_tiles = seq_info(lane, f_t0, f_t1, f_len);
    int64_t total = 0;  // every CTA computes the same list
    for (int c = 0; c < p.B; c += 32) {
      int a0, a1, al;
      int tiles = c == 0 ? f_tiles : seq_info(c + lane, a0, a1, al);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, off);
      total += tiles;
    }
    const int64_t lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
    // segments: walk the sequences again, 32 at a time
    int nseg = 0;
    int64_t before = 0;  // key tiles of the sequences already walked
    for (int c = 0; c < p.B && before < hi; c += 32) {
      int t0 = f_t0, t1 = f_t1, len = f_len, tiles = f_tiles;
      if (c > 0) tiles = seq_info(c + lane, t0, t1, len);
      int incl = tiles;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      const int64_t s_lo = before + incl - tiles, s_hi = before + incl;  // this lane's sequence
      unsigned hit = __ballot_sync(0xffffffffu, tiles > 0 && s_lo < hi && s_hi > lo);
      while (hit) {
        const int src = __ffs(hit) - 1;
        hit &= hit - 1;
        const int bt0 = __shfl_sync(0xffffffffu, t0, src), bt1 = __shfl_sync(0xffffffffu, t1, src);
        const int bb = c + src;
        const int blen = __shfl_sync(0xffffffffu, len, src);
        int64_t pos = __shfl_sync(0xffffffffu, s_lo, src);  // flattened index of the token's first tile
        if (lane == 0) {
          for (int t = bt0; t < bt1 && pos < hi; ++t) {
            const int nv = max(0, min(__ldg(p.q_pos + t) + 1, blen));
            const int nt = (nv + 127) / 128;
            const int64_t a = max(pos, lo), e = min(pos + nt, hi);
            if (a < e && nseg < C::MAXSEG) {
              seg_tok[nseg] = t;
              seg_t0[nseg] = static_cast<int>(a - pos);
              seg_nt[nseg] = static_cast<int>(e - a);
              seg_nv[nseg] = nv;
              seg_b[nseg] = bb;
              ++nseg;
            }
            pos += nt;
          }
        }
      }
      before += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      misc[0] = nseg;
      misc[2] = 0;
      misc[3] = static_cast<int>(hi - lo);
      for (int i = 0; i < C::ST; ++i) {
        mbar_init(&full[i], 1);
        mbar_init(&empty[i], FP8 ? 4 : 1);  // FP8: the tile's epilogue group
      }
      for (int i = 0; i < C::NACC; ++i) {
        mbar_init(&acc_full[i], 1);
        mbar_init(&acc_empty[i], 4);  // the accumulator's epilogue group
      }
      for (int i = 0; i < C::CS; ++i) {
        mbar_init(&conv_full[i], C::CONV_WARPS);
        mbar_init(&conv_empty[i], 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(&q_full[i], 1);
        mbar_init(&q_empty[i], 1 + C::EPI_WARPS);
      }
      mbar_init(drain, 1);
      fence_mbar_init();
    }
  } else if (warp == 1) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc + 1), C::TMEM_COLS);
    tmem_relinquish();
  } else if (C::N > HI || C::DK > DIN) {
    // query rows beyond H_I and columns beyond d_I are never written by the
    // query TMA (it fills only its box): zero both buffers once
    for (int i = threadIdx.x - 64; i < 2 * C::QB_BYTES / 16; i += C::THREADS - 64)
      reinterpret_cast<uint4*>(smem + C::OFF_Q)[i] = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (FP8) {
      if (C::DK > DIN) {
        uint4* cz = reinterpret_cast<uint4*>(smem + C::OFF_CONV);
        for (int i = threadIdx.x - 64; i < C::CS * C::TILE_BYTES / 16; i += C::THREADS - 64) cz[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int nseg = misc[0];
  const int n_tiles = misc[3];
  const uint32_t tmem_base = static_cast<uint32_t>(misc[1]);

  if (n_tiles > 0) {
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        const uint8_t* scale_src = KF == KF_MX ? p.k_mx : reinterpret_cast<const uint8_t*>(p.k_scale);
        int it = 0, kq = 0;
        bool ok = true;
        for (int k = 0; k < nseg && ok; ++k) {
          const int buf = k & 1;
          const int t = seg_tok[k];
          if (k >= 2) ok = mbar_wait(&q_empty[buf], ((k >> 1) - 1) & 1, abort_flag);
          if (!ok) break;
          ++kq;
          mbar_arrive_expect_tx(&q_full[buf], C::Q_TX + C::W_BYTES);
#pragma unroll
          for (int a = 0; a < C::AK; ++a)
            tma_load_2d(smem_u32(smem + C::OFF_Q + buf * C::QB_BYTES + a * C::N * 128), &qmap, a * 64, t * HI, &q_full[buf]);
          bulk_load(smem_u32(w_s + buf * (C::W_BYTES / 4)), w + static_cast<int64_t>(t) * HI, C::W_BYTES, &q_full[buf]);
          const int bb = seg_b[k];
          const int nv = seg_nv[k];
          for (int i = 0; i < seg_nt[k]; ++i, ++it) {
            const int st = it % C::ST;
            if (!mbar_wait(&empty[st], ((it / C::ST) & 1) ^ 1u, abort_flag)) {
              ok = false;
              break;
            }
            const int s0 = (seg_t0[k] + i) * 128;  // first key position of the tile
            const uint32_t dst = smem_u32(smem + C::OFF_STAGE + st * C::STAGE_BYTES);
            if (!p.cm.paged()) {
              const int32_t y = bb * p.L_max + s0;
              if constexpr (FP8) {
                // scale rows y .. y + 127, clipped at the end of the cache
                const int64_t left = p.rows - y;
                const uint32_t sbytes =
                    p.scale_bulk ? C::SROW * static_cast<uint32_t>(left < 128 ? left : 128) : 0u;
                mbar_arrive_expect_tx(&full[st], C::U8_TILE + sbytes);
                tma_load_2d(dst, &kmap, 0, y, &full[st]);
                if (sbytes) bulk_load(dst + C::U8_TILE, scale_src + static_cast<int64_t>(y) * C::SROW, sbytes, &full[st]);
              } else {
                mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
#pragma unroll
                for (int a = 0; a < C::AK; ++a) tma_load_2d(dst + a * 16384, &kmap, a * 64, y, &full[st]);
              }
            } else {
              // paged: two 64-row boxes; a half past the last candidate
              // reloads the first half (its rows are masked)
              mbar_arrive_expect_tx(&full[st], FP8 ? C::U8_TILE + (p.scale_bulk ? 128 * C::SROW : 0) : C::STAGE_BYTES);
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int32_t y = p.cm.row_checked(bb, (s0 + 64 * h < nv) ? s0 + 64 * h : s0);
                if constexpr (FP8) {
                  tma_load_2d(dst + h * 64 * DIN, &kmap, 0, y, &full[st]);
                  if (p.scale_bulk)
                    bulk_load(dst + C::U8_TILE + 64 * C::SROW * h, scale_src + static_cast<int64_t>(y) * C::SROW,
                              64 * C::SROW, &full[st]);
                } else {
#pragma unroll
                  for (int a = 0; a < C::AK; ++a)
                    tma_load_2d(dst + a * 16384 + h * 8192, &kmap, a * 64, y, &full[st]);
                }
              }
            }
          }
        }
        // every load issued must land before the CTA can retire
        for (int j = it > C::ST ? it - C::ST : 0; j < it; ++j) {
          volatile int never = 0;
          mbar_wait(&full[j % C::ST], (j / C::ST) & 1, &never);
        }
        for (int k = kq > 2 ? kq - 2 : 0; k < kq; ++k) {
          volatile int never = 0;
          mbar_wait(&q_full[k & 1], (k >> 1) & 1, &never);
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        int it = 0;
        bool ok = true;
        for (int k = 0; k < nseg && ok; ++k) {
          const int buf = k & 1;
          ok = mbar_wait(&q_full[buf], (k >> 1) & 1, abort_flag);
          for (int i = 0; i < seg_nt[k] && ok; ++i, ++it) {
            const int acc = it % C::NACC;
            uint32_t a_base;
            if constexpr (FP8) {
              const int cs = it % C::CS;
              ok = mbar_wait(&conv_full[cs], (it / C::CS) & 1, abort_flag);
              a_base = smem_u32(smem + C::OFF_CONV + cs * C::TILE_BYTES);
            } else {
              const int st = it % C::ST;
              ok = mbar_wait(&full[st], (it / C::ST) & 1, abort_flag);
              a_base = smem_u32(smem + C::OFF_STAGE + st * C::TILE_BYTES);
            }
            if (ok) ok = mbar_wait(&acc_empty[acc], ((it / C::NACC) & 1) ^ 1u, abort_flag);
            if (!ok) break;
            tc_fence_after();
            const uint32_t b_base = smem_u32(smem + C::OFF_Q + buf * C::QB_BYTES);
            const uint32_t d_tmem = tmem_base + acc * C::N;
#pragma unroll
            for (int kk = 0; kk < C::DK / 16; ++kk) {
              const uint64_t adesc = smem_desc_sw128(a_base + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(b_base + (kk / 4) * (C::N * 128) + (kk % 4) * 32, 16, 1024);
              umma_f16(d_tmem, adesc, bdesc, C::IDESC, kk > 0 ? 1u : 0u);
            }
            if constexpr (FP8)
              umma_commit(&conv_empty[it % C::CS]);
            else
              umma_commit(&empty[it % C::ST]);
            umma_commit(&acc_full[acc]);
          }
          if (ok) umma_commit(&q_empty[buf]);  // the query buffer is free once these MMAs complete
        }
        umma_commit(drain);
        volatile int never = 0;
        mbar_wait(drain, 0, &never);
      }
      __syncwarp();
    } else if (warp < 2 + C::EPI_WARPS) {
      // ---------------------------------------------------------- epilogue
      static_assert(C::EPI_GROUPS == 1 || C::EPI_GROUPS == C::NACC, "one epilogue group per accumulator");
      const int grp = (warp - 2) >> 2;  // with two groups: this group's tiles have it % 2 == grp
      const int sub = warp & 3;
      const int r = sub * 32 + lane;  // key row inside the tile
      const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
      int it = 0;
      bool ok = true;
      for (int k = 0; k < nseg && ok; ++k) {
        const int buf = k & 1;
        const int t = seg_tok[k];
        const int nv = seg_nv[k];
        ok = mbar_wait_warp(&q_full[buf], (k >> 1) & 1, abort_flag);
        const float* ws = w_s + buf * (C::W_BYTES / 4);
        const int bb = seg_b[k];
        for (int i = 0; i < seg_nt[k] && ok; ++i, ++it) {
          if (C::EPI_GROUPS == 2 && (it & 1) != grp) continue;
          const int acc = it % C::NACC;
          const int64_t s = static_cast<int64_t>(seg_t0[k] + i) * 128 + r;  // key position of this row
          float sigma = 1.0f;
          if constexpr (FP8) {
            // the stage (codes + scales) stays ours until this warp frees it
            const int st = it % C::ST;
            ok = mbar_wait_warp(&full[st], (it / C::ST) & 1, abort_flag);
            if constexpr (KF != KF_FP8) {
              // MXFP8: the scales were applied while widening
            } else if (p.scale_bulk) {
              if (ok) sigma = reinterpret_cast<const float*>(smem + C::OFF_STAGE + st * C::STAGE_BYTES + C::U8_TILE)[r];
            } else if (s < nv) {
              // the key's scale from global memory (only causal candidates,
              // so only rows inside the sequence)
              bool rok;
              sigma = __ldg(p.k_scale + p.cm.row(bb, static_cast<int>(s), rok));
            }
          }
          if (ok) ok = mbar_wait_warp(&acc_full[acc], (it / C::NACC) & 1, abort_flag);
          if (!ok) break;
          tc_fence_after();
          float score;
          if constexpr (C::N <= 64) {
            float v[C::N / 16][16];
#pragma unroll
            for (int c = 0; c < C::N / 16; ++c) tmem_ld16(tmem_base + lane_addr + acc * C::N + c * 16, v[c]);
            tmem_wait_ld();
            float t4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int c = 0; c < C::N / 16; ++c)
#pragma unroll
              for (int u = 0; u < 16; ++u)
                if (c * 16 + u < HI) t4[u & 3] = fmaf(ws[c * 16 + u], fmaxf(v[c][u], 0.0f), t4[u & 3]);
            score = (t4[0] + t4[1]) + (t4[2] + t4[3]);
          } else {
            float t4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll 1
            for (int c = 0; c < C::N; c += 64) {
              float v[4][16];
#pragma unroll
              for (int q = 0; q < 4; ++q) tmem_ld16(tmem_base + lane_addr + acc * C::N + c + 16 * q, v[q]);
              tmem_wait_ld();
#pragma unroll
              for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int u = 0; u < 16; ++u) t4[u & 3] = fmaf(ws[c + 16 * q + u], fmaxf(v[q][u], 0.0f), t4[u & 3]);
            }
            score = (t4[0] + t4[1]) + (t4[2] + t4[3]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&acc_empty[acc]);
            if constexpr (FP8) mbar_arrive(&empty[it % C::ST]);  // codes converted, scales read
          }
          if (s < p.ld) p.scores[static_cast<int64_t>(t) * p.ld + s] = (s < nv) ? score * sigma : -INFINITY;
        }
        __syncwarp();
        if (ok && lane == 0) mbar_arrive(&q_empty[buf]);  // weights of this buffer read for good
      }
    } else if constexpr (FP8) {
      // ---------------------------------------------------------- FP8 -> bf16 converters
      // Each thread loads all its 16-byte code chunks of the tile first (and,
      // for MXFP8, their scale bytes), then widens and stores them.
      constexpr int CT = C::CONV_WARPS * 32;
      const int ct = threadIdx.x - (2 + C::EPI_WARPS) * 32;  // 0 .. CT - 1
      constexpr int CPR = DIN / 16;                            // 16-byte code chunks per key row
      constexpr int PER = (128 * CPR + CT - 1) / CT;           // chunks per thread
      int it = 0;
      bool ok = true;
      for (int k = 0; k < nseg && ok; ++k) {
        const int bb = seg_b[k];
        for (int i = 0; i < seg_nt[k]; ++i, ++it) {
          const int st = it % C::ST;
          const int cs = it % C::CS;
          ok = mbar_wait_warp(&full[st], (it / C::ST) & 1, abort_flag) &&
               mbar_wait_warp(&conv_empty[cs], ((it / C::CS) & 1) ^ 1u, abort_flag);
          if (!ok) break;
          const uint8_t* src = smem + C::OFF_STAGE + st * C::STAGE_BYTES;
          uint8_t* dst = smem + C::OFF_CONV + cs * C::TILE_BYTES;
          const int s0 = (seg_t0[k] + i) * 128;  // first key position of the tile
          uint4 raws[PER];
          int bytes[PER];
#pragma unroll
          for (int u = 0; u < PER; ++u) {
            const int e = ct + u * CT;
            const int row = e / CPR;
            const int c = e % CPR;
            raws[u] = make_uint4(0u, 0u, 0u, 0u);
            bytes[u] = 127;
            if (e < 128 * CPR) {
              raws[u] = *reinterpret_cast<const uint4*>(src + row * DIN + c * 16);
              if constexpr (KF == KF_MX) {
                if (p.scale_bulk) {
                  bytes[u] = src[C::U8_TILE + row * (DIN / 32) + c / 2];
                } else {
                  // rows past the sequence are masked; read a row that exists
                  bool rok;
                  const int sr = s0 + row < seg_nv[k] ? s0 + row : s0;
                  bytes[u] = __ldg(p.k_mx + static_cast<int64_t>(p.cm.row(bb, sr, rok)) * (DIN / 32) + c / 2);
                }
              }
            }
          }
#pragma unroll
          for (int u = 0; u < PER; ++u) {
            const int e = ct + u * CT;
            if (e >= 128 * CPR) break;
            const int row = e / CPR;
            const int c = e % CPR;
            const uint32_t words[4] = {raws[u].x, raws[u].y, raws[u].z, raws[u].w};
            // MXFP8: 2^e of the chunk's 32-element group (exact scaling)
            const float m = KF == KF_MX ? exp2_int(bytes[u] - 127) : 1.0f;
            uint32_t outw[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const __half2_raw h01 =
                  __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(words[q] & 0xFFFF), __NV_E4M3);
              const __half2_raw h23 =
                  __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(words[q] >> 16), __NV_E4M3);
              float2 f01 = __half22float2(__half2(h01)), f23 = __half22float2(__half2(h23));
              if constexpr (KF == KF_MX) {
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
          if (lane == 0) mbar_arrive(&conv_full[cs]);
        }
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
