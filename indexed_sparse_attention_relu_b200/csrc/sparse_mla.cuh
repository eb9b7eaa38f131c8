// sparse_mla.cuh -- sparse MLA attention over the selected latent KV rows
// (Sparse Flash Attention, section 1 of "Day-0 Inference Optimization for a
// New Sparse Attention Architecture": it reads the KV-cache entries named by
// the Lightning Indexer's indices and attends over them only).
//
// For query token t (sequence b), head h and selected rows s_i:
//   z_i = softmax_scale * q[t,h,:] . kv[b,s_i,:]          (all D = d_c + d_rope dims)
//   out[t,h,:] = sum_i softmax(z)_i * kv[b,s_i,0:d_c]     (value = latent part)
//   lse[t,h] = log sum_i exp(z_i)
//
// One CTA = (token, 64-head block, key split); the key splits of one
// (token, head block) form a thread-block cluster. Per tile of 64 selected keys:
//  * four producer warps gather the 64 rows with 16-byte cp.async straight
//    into the 128-byte-swizzled K-major layout (one warp instruction moves
//    512 contiguous bytes of a row, three cover a 1152-byte row); each thread
//    signals its copies through an asynchronous mbarrier arrival, so the
//    producers run one tile ahead without blocking; an index of -1 or out of
//    range zero-fills its row (two-stage ring);
//  * one thread issues S = Q K^T (M = 64 heads, N = 64 keys, K = D) and
//    O += P V (M = 64, N = d_c in 256-wide pieces, K = 64 keys) on tcgen05;
//    the value operand is the same shared-memory tile read as an MN-major
//    matrix, so each row is gathered once;
//  * with M = 64 an accumulator uses lanes 0-15 of each TMEM sub-partition,
//    so O (all d_c columns) sits at lane offset 0 and S at lane offset 16 of
//    the same columns: both fit in one SM's TMEM;
//  * 4 softmax warps read S with 16-lane TMEM loads, so all 32 threads work:
//    thread t holds head rows t/4 and t/4 + 8 of its warp's 16 and 16 of the
//    64 keys; they run an online softmax in the exp2 domain with lazy
//    rescaling: O is only rescaled (TMEM load/scale/store) when a row maximum
//    grows by more than 2^8, which keeps P <= 256 and the result exact;
//  * P is written as bf16 to shared memory (A operand of the PV product).
// The split partials (O, running max, running sum) are merged inside the
// cluster: every CTA sends each head row to the CTA that owns that head
// (owner = head mod splits) through distributed shared memory, and the owner
// writes the bf16 output and the lse. All cross-CTA handshakes are mbarriers
// with bounded waits.
#pragma once
#include "dsa_common.cuh"

namespace dsa {

struct MlaParams {
  const int32_t* cu_q;
  const int32_t* seq_lens;
  int32_t B;
  int32_t L_max;
  int32_t T;
  int32_t H;
  int32_t K;
  const int32_t* idx;        // [T, K]
  float scale_log2;          // softmax_scale * log2(e)
  int32_t keys_per_split;    // multiple of 64
  int32_t splits;            // == cluster size along z
  __nv_bfloat16* out;        // [T, H, DC]
  float* lse;                // [T, H] or null
};

template <int D, int DC>
struct MlaCfg {
  static constexpr int DP = ((D + 63) / 64) * 64;   // K extent of the QK^T product (whole atoms)
  static constexpr int AKQ = DP / 64;               // 128-byte atom columns per row
  static constexpr int HB = 64;                     // heads per CTA (MMA M)
  static constexpr int TK = 64;                     // keys per tile (QK^T N, PV K)
  static constexpr int ATOM_COL = 64 * 128;         // bytes of one atom column of a 64-row tile
  static constexpr int Q_BYTES = HB * DP * 2;
  static constexpr int KV_BYTES = TK * DP * 2;
  static constexpr int P_BYTES = HB * TK * 2;
  static constexpr int NST = 2;
  static constexpr int N_PV = DC < 256 ? DC : 256;
  static constexpr int PV_MMAS = DC / N_PV;
  static constexpr int TMEM_COLS = DC <= 32 ? 32 : DC <= 64 ? 64 : DC <= 128 ? 128 : DC <= 256 ? 256 : 512;
  static constexpr int NUM_WARPS = 9;  // 0-3 softmax/epilogue, 4-7 gather producers, 8 MMA + TMEM owner
  static constexpr int THREADS = NUM_WARPS * 32;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_P = OFF_KV + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int NUM_BARS = 2 * NST + 8;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;
  static constexpr int MAX_SPLITS = 8;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(64, TK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(64, N_PV, false, true);
  static_assert(DC % N_PV == 0 && DC % 64 == 0, "latent dim must be a multiple of 64");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // merge buffers reuse the KV ring (partial O rows) and the P tile (statistics);
  // S * ceil(64 / S) entries, at most 70 (S = 7) for S <= 8
  static_assert(70 * DC * 4 <= NST * KV_BYTES, "merge buffer must fit in the KV ring");
  static_assert(70 * 8 <= P_BYTES, "merge statistics must fit in the P tile");
};

template <int D, int DC>
__global__ void __launch_bounds__(MlaCfg<D, DC>::THREADS, 1)
    sparse_mla_kernel(const __nv_bfloat16* __restrict__ kv, const __grid_constant__ CUtensorMap qmap,
                      const MlaParams p) {
  using C = MlaCfg<D, DC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;             // [NST] gather producers -> MMA
  uint64_t* kv_empty = bars + C::NST;   // [NST] MMA (PV done) -> gather producers
  uint64_t* q_full = kv_empty + C::NST; // TMA -> MMA
  uint64_t* s_full = q_full + 1;        // MMA (S ready) -> softmax
  uint64_t* s_empty = s_full + 1;       // softmax (S read) -> MMA
  uint64_t* p_full = s_empty + 1;       // softmax (P written) -> MMA
  uint64_t* o_done = p_full + 1;        // MMA (PV done) -> softmax
  uint64_t* drain = o_done + 1;
  uint64_t* ready = drain + 1;          // merge: every CTA of the cluster has finished its loop
  uint64_t* recv = ready + 1;           // merge: every partial row destined here has arrived
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);
  // misc: [0] TMEM base, [1] abort
  volatile int* abort_flag = misc + 1;

  const int t = blockIdx.x;
  const int h0 = blockIdx.y * C::HB;
  const int split = blockIdx.z;
  const int S = p.splits;
  const int warp = warp_id();
  const int lane = lane_id();
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.K, k_begin + p.keys_per_split);
  const int n_tiles = (k_end - k_begin + C::TK - 1) / C::TK;  // >= 1 by construction
  const int32_t* idx_row = p.idx + static_cast<int64_t>(t) * p.K;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&kv_full[i], 128);  // one asynchronous arrival per producer thread
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    mbar_init(ready, S);
    mbar_init(recv, 64 * S);
    misc[1] = 0;
    fence_mbar_init();
    prefetch_tensormap(&qmap);
  }
  if (warp == 8) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  if (S > 1)
    cluster_sync_all();  // peers' barriers are initialised before any remote arrive
  else
    __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);
  const uint32_t tmem_s = tmem_base + (16u << 16);  // S at lane offset 16 (M = 64 layout)

  if (warp == 8 && lane == 0) {
    // the query block is an input of the call, not of the Top-K: load it now
    mbar_arrive_expect_tx(q_full, C::Q_BYTES);
    const uint32_t qs = smem_u32(smem + C::OFF_Q);
#pragma unroll
    for (int c = 0; c < C::AKQ; ++c) tma_load_2d(qs + c * C::ATOM_COL, &qmap, c * 64, t * p.H + h0, q_full);
  }
  pdl_wait_prior();  // the selected indices (Top-K output) are complete from here on

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ gather producers (4 warps)
    // warp pw copies rows 16pw .. 16pw+15 of each 64-key tile; for one row the
    // whole warp issues 16-byte chunks 32 at a time (512 contiguous bytes)
    constexpr int CPR = C::DP / 8;                // 16-byte chunks per padded row
    constexpr int ROUNDS = (CPR + 31) / 32;
    const int pw = warp - 4;
    const __nv_bfloat16* kv_seq = kv + static_cast<int64_t>(b) * p.L_max * D;
    // index of this lane's row (lanes 0..15), fetched one tile ahead; the rows
    // of the tile after next are prefetched into L2 (no shared memory needed),
    // so the gather that fills a freed stage reads from L2
    auto row_index = [&](int tile) -> int {
      const int k = k_begin + tile * C::TK + 16 * pw + lane;
      return (lane < 16 && tile < n_tiles && k < k_end) ? ld_dep(idx_row + k) : -1;
    };
    auto prefetch_rows = [&](int s_row) {
      if (s_row >= 0 && s_row < len) prefetch_l2(kv_seq + static_cast<int64_t>(s_row) * D, D * 2);
    };
    int nxt = row_index(0);
    int nxt2 = row_index(1);
    prefetch_rows(nxt);
    prefetch_rows(nxt2);
    int issued = 0;
    for (int it = 0; it < n_tiles; ++it) {
      const int st = it & 1;
      const int cur = nxt;
      nxt = nxt2;
      nxt2 = row_index(it + 2);  // in flight during the stage wait and the gather
      if (!mbar_wait_warp(&kv_empty[st], ((it >> 1) & 1) ^ 1, abort_flag)) break;
      const bool ok = cur >= 0 && cur < len;
      if (lane < 16 && cur != -1 && !ok) set_device_status(DSA_ERR_DEVICE_INDEX);
      const uint32_t stage = smem_u32(smem + C::OFF_KV + st * C::KV_BYTES);
#pragma unroll 4
      for (int rr = 0; rr < 16; ++rr) {
        const int r = 16 * pw + rr;                         // key slot in the tile
        const int srow = __shfl_sync(0xffffffffu, ok ? cur : -1, rr);
        const __nv_bfloat16* src_row = kv_seq + static_cast<int64_t>(srow < 0 ? 0 : srow) * D;
#pragma unroll
        for (int q = 0; q < ROUNDS; ++q) {
          const int c = 32 * q + lane;                      // 16-byte chunk of the row
          if (c < CPR) {
            const bool has = srow >= 0 && c * 8 < D;
            cp_async_16(stage + (c / 8) * C::ATOM_COL + sw128_offset(r, c % 8), has ? src_row + c * 8 : kv,
                        has ? 16u : 0u);
          }
        }
      }
      cp_async_arrive_noinc(&kv_full[st]);
      prefetch_rows(nxt2);
      ++issued;
    }
    cp_async_wait_all();  // nothing may still be landing when the CTA retires
    (void)issued;
  } else if (warp == 8) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + C::OFF_Q);
      const uint32_t p_base = smem_u32(smem + C::OFF_P);
      auto issue_s = [&](int it) {
        const uint32_t kvb = smem_u32(smem + C::OFF_KV + (it & 1) * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < C::DP / 16; ++k) {
          const uint64_t a = smem_desc_sw128(q_base + (k / 4) * C::ATOM_COL + (k % 4) * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(kvb + (k / 4) * C::ATOM_COL + (k % 4) * 32, 16, 1024);
          umma_f16(tmem_s, a, bd, C::IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
      };
      // Order: S(0), then per tile PV(it) followed by S(it+1). The gather of
      // tile it+1 only waits for PV(it-1), which is issued before S(it+1).
      bool ok = mbar_wait(q_full, 0, abort_flag) && mbar_wait(&kv_full[0], 0, abort_flag);
      if (ok) {
        fence_proxy_async_smem();  // cp.async (generic proxy) data -> tensor core reads
        tc_fence_after();
        issue_s(0);
      }
      for (int it = 0; ok && it < n_tiles; ++it) {
        if (!(ok = mbar_wait(p_full, it & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t kvb = smem_u32(smem + C::OFF_KV + (it & 1) * C::KV_BYTES);
#pragma unroll
        for (int nb = 0; nb < C::PV_MMAS; ++nb) {
#pragma unroll
          for (int kk = 0; kk < C::TK / 16; ++kk) {
            const uint64_t a = smem_desc_sw128(p_base + kk * 32, 16, 1024);
            // V = first DC dims of the gathered rows, MN-major: 64-dim atom columns
            // ATOM_COL bytes apart (LBO), 8-key row groups 1024 bytes apart (SBO).
            const uint64_t bd =
                smem_desc_sw128(kvb + (nb * (C::N_PV / 64)) * C::ATOM_COL + kk * 16 * 128, C::ATOM_COL, 1024);
            umma_f16(tmem_base + nb * C::N_PV, a, bd, C::IDESC_PV, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&kv_empty[it & 1]);
        umma_commit(o_done);
        if (it + 1 < n_tiles) {
          if (!(ok = mbar_wait(s_empty, it & 1, abort_flag))) break;
          if (!(ok = mbar_wait(&kv_full[(it + 1) & 1], ((it + 1) >> 1) & 1, abort_flag))) break;
          fence_proxy_async_smem();
          tc_fence_after();
          issue_s(it + 1);
        }
      }
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0..3)
    const int sw = warp;                                   // TMEM sub-partition
    const uint32_t lane_addr = static_cast<uint32_t>(sw * 32) << 16;
    const bool is_s = lane >= 16;                          // threads 16..31 own S rows
    const int h_local = sw * 16 + (lane & 15);             // head row inside the block
    // Rows of S this thread handles in the 16-lane layout: head rows ra, ra+8
    // of the warp's 16 (h_local = sw*16 + row) and key columns 8j + cc, +1.
    const int ra = lane >> 2;
    const int cc = 2 * (lane & 3);
    float m_a = -INFINITY, m_b = -INFINITY;  // running max per row (log2 domain)
    float l_a = 0.0f, l_b = 0.0f;            // this thread's share of the running sums
    bool ok = true;
    uint8_t* p_tile = smem + C::OFF_P;
    // indices of the next tile (for the validity mask), one tile ahead
    int i0n = (k_begin + lane < k_end) ? ld_dep(idx_row + k_begin + lane) : -1;
    int i1n = (k_begin + 32 + lane < k_end) ? ld_dep(idx_row + k_begin + 32 + lane) : -1;
    for (int it = 0; it < n_tiles; ++it) {
      const int i0 = i0n, i1 = i1n;
      if (it + 1 < n_tiles) {
        const int kn = k_begin + (it + 1) * C::TK;
        i0n = (kn + lane < k_end) ? ld_dep(idx_row + kn + lane) : -1;
        i1n = (kn + 32 + lane < k_end) ? ld_dep(idx_row + kn + 32 + lane) : -1;
      }
      const unsigned v0 = __ballot_sync(0xffffffffu, i0 >= 0 && i0 < len);
      const unsigned v1 = __ballot_sync(0xffffffffu, i1 >= 0 && i1 < len);
      if (!(ok = mbar_wait_warp(s_full, it & 1, abort_flag))) break;
      tc_fence_after();
      float v[32];
      tmem_ld16x256_x8(tmem_s + lane_addr, v);
      tmem_wait_ld();
      // v[4j + 0/1] = row ra, cols 8j+cc, +1; v[4j + 2/3] = row ra+8, same cols
      float ta = -INFINITY, tb = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = 8 * j + cc + e;
          const bool valid = (col < 32) ? ((v0 >> col) & 1u) : ((v1 >> (col - 32)) & 1u);
          v[4 * j + e] = valid ? v[4 * j + e] * p.scale_log2 : -INFINITY;
          v[4 * j + 2 + e] = valid ? v[4 * j + 2 + e] * p.scale_log2 : -INFINITY;
          ta = fmaxf(ta, v[4 * j + e]);
          tb = fmaxf(tb, v[4 * j + 2 + e]);
        }
      }
      ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 1));
      ta = fmaxf(ta, __shfl_xor_sync(0xffffffffu, ta, 2));
      tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 1));
      tb = fmaxf(tb, __shfl_xor_sync(0xffffffffu, tb, 2));
      float fa = 1.0f, fb = 1.0f;
      const float na = fmaxf(m_a, ta), nb = fmaxf(m_b, tb);
      const bool need_a = na > m_a + 8.0f, need_b = nb > m_b + 8.0f;
      if (need_a) {
        fa = ex2_approx(m_a - na);  // 0 when m_a = -inf
        l_a *= fa;
        m_a = na;
      }
      if (need_b) {
        fb = ex2_approx(m_b - nb);
        l_b *= fb;
        m_b = nb;
      }
      bool o_waited = false;
      if (__any_sync(0xffffffffu, (need_a || need_b) && it > 0)) {
        // O already holds earlier tiles: wait for PV(it-1), then rescale those rows
        if (!(ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag))) break;
        o_waited = true;
        tc_fence_after();
        // O row r (lanes 0..15 in the 32-lane layout) is row ra of thread 4(r%8) (a if r < 8, else b)
        const int src = 4 * (lane & 7);
        const float ga = __shfl_sync(0xffffffffu, fa, src);
        const float gb = __shfl_sync(0xffffffffu, fb, src);
        const float fo = (lane < 8) ? ga : gb;
        for (int c = 0; c < DC; c += 16) {
          float o[16];
          tmem_ld16(tmem_base + lane_addr + c, o);
          tmem_wait_ld();
          if (lane < 16) {
#pragma unroll
            for (int u = 0; u < 16; ++u) o[u] *= fo;
          }
          tmem_st16(tmem_base + lane_addr + c, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      // P = 2^(s - m) in bf16; the sums add the rounded values PV actually uses
      uint32_t pa[8], pb[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float a0 = (m_a == -INFINITY) ? 0.0f : ex2_approx(v[4 * j] - m_a);
        const float a1 = (m_a == -INFINITY) ? 0.0f : ex2_approx(v[4 * j + 1] - m_a);
        const float b0 = (m_b == -INFINITY) ? 0.0f : ex2_approx(v[4 * j + 2] - m_b);
        const float b1 = (m_b == -INFINITY) ? 0.0f : ex2_approx(v[4 * j + 3] - m_b);
        const __nv_bfloat162 qa = __floats2bfloat162_rn(a0, a1);
        const __nv_bfloat162 qb = __floats2bfloat162_rn(b0, b1);
        l_a += __low2float(qa) + __high2float(qa);
        l_b += __low2float(qb) + __high2float(qb);
        pa[j] = *reinterpret_cast<const uint32_t*>(&qa);
        pb[j] = *reinterpret_cast<const uint32_t*>(&qb);
      }
      if (it > 0 && !o_waited) {
        if (!(ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag))) break;  // P buffer free
      }
      {
        const int ha = sw * 16 + ra, hb = ha + 8;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          *reinterpret_cast<uint32_t*>(p_tile + sw128_offset(ha, j) + 2 * cc) = pa[j];
          *reinterpret_cast<uint32_t*>(p_tile + sw128_offset(hb, j) + 2 * cc) = pb[j];
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    // full row sums: add the four threads sharing each row
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
    l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
    l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
    // hand (max, sum) of head row r to O lane r (the 32-lane layout below)
    float m_used, l;
    {
      const int src = 4 * (lane & 7);
      const float xa = __shfl_sync(0xffffffffu, m_a, src), xb = __shfl_sync(0xffffffffu, m_b, src);
      const float ya = __shfl_sync(0xffffffffu, l_a, src), yb = __shfl_sync(0xffffffffu, l_b, src);
      m_used = ((lane & 15) < 8) ? xa : xb;
      l = ((lane & 15) < 8) ? ya : yb;
    }
    if (ok) ok = mbar_wait_warp(o_done, (n_tiles - 1) & 1, abort_flag);
    const float l_h = l;        // lane r < 16 owns O row r; lanes 16..31 mirror it
    const float m_h = m_used;
    const int h = h0 + h_local;
    if (ok) tc_fence_after();
    if (S == 1) {
      if (ok) {
        const bool writer = !is_s && h < p.H;
        const float inv = (l_h > 0.0f) ? 1.0f / l_h : 0.0f;
        const int64_t row = static_cast<int64_t>(t) * p.H + h;
        for (int c = 0; c < DC; c += 16) {
          float v[16];
          tmem_ld16(tmem_base + lane_addr + c, v);
          tmem_wait_ld();
          if (writer) {
            uint32_t w8[8];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
              const __nv_bfloat162 o2 = __floats2bfloat162_rn(v[u] * inv, v[u + 1] * inv);
              w8[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * DC + c);
            dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
          }
        }
        if (writer && p.lse) p.lse[row] = (l_h > 0.0f) ? (m_h + log2f(l_h)) * 0.69314718055994531f : -INFINITY;
      }
    } else {
      // ---------------- merge the S split partials inside the cluster
      // Head row h_local belongs to CTA owner = h_local % S (slot h_local / S).
      // Each CTA sends its unnormalised O row with (running max, running sum)
      // into the owner's buffer (entry src * HPC + slot); the owner combines.
      const uint32_t me = cluster_ctarank();
      const int HPC = (64 + S - 1) / S;
      const uint32_t recv_base = smem_u32(smem + C::OFF_KV);
      const uint32_t stat_base = smem_u32(smem + C::OFF_P);
      if (ok && threadIdx.x == 0) {
        // this CTA's loop is done (all PV products complete, no TMA in flight):
        // its KV ring and P tile may now be overwritten by peers
        for (int r = 0; r < S; ++r) mbar_arrive_remote(mapa_shared(smem_u32(ready), r));
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(ready, 0, abort_flag));
      if (ok) {
        const uint32_t owner = static_cast<uint32_t>(h_local % S);
        const int entry = static_cast<int>(me) * HPC + h_local / S;
        const uint32_t o_dst = mapa_shared(recv_base + entry * DC * 4, owner);
        for (int c = 0; c < DC; c += 16) {
          float v[16];
          tmem_ld16(tmem_base + lane_addr + c, v);
          tmem_wait_ld();
          if (!is_s) {
#pragma unroll
            for (int u = 0; u < 16; u += 4) st_cluster_v4(o_dst + (c + u) * 4, v[u], v[u + 1], v[u + 2], v[u + 3]);
          }
        }
        if (!is_s) {
          st_cluster_v2(mapa_shared(stat_base + entry * 8, owner), m_h, l_h);
          // 64 O-row threads per CTA arrive on every CTA's recv barrier (count
          // 64 * S); release order makes each thread's stores visible first
          for (int r = 0; r < S; ++r) mbar_arrive_remote(mapa_shared(smem_u32(recv), r));
        }
      }
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait_cluster(recv, 0, abort_flag));
      if (ok) {
        // finalise the heads this CTA owns: warp sw takes slots sw, sw+4, ...
        const float* obuf = reinterpret_cast<const float*>(smem + C::OFF_KV);
        const float2* sbuf = reinterpret_cast<const float2*>(smem + C::OFF_P);
        for (int slot = sw; slot < HPC; slot += 4) {
          const int hl = slot * S + static_cast<int>(me);
          if (hl >= 64 || h0 + hl >= p.H) continue;
          float M = -INFINITY;
          for (int src = 0; src < S; ++src) M = fmaxf(M, sbuf[src * HPC + slot].x);
          float L = 0.0f;
          for (int src = 0; src < S; ++src) {
            const float2 st = sbuf[src * HPC + slot];
            if (st.y > 0.0f) L += exp2f(st.x - M) * st.y;
          }
          const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
          const int64_t row = static_cast<int64_t>(t) * p.H + h0 + hl;
          for (int d0 = lane * 8; d0 < DC; d0 += 32 * 8) {
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int src = 0; src < S; ++src) {
              const float2 st = sbuf[src * HPC + slot];
              if (!(st.y > 0.0f)) continue;
              const float wgt = exp2f(st.x - M) * inv;
              const float4* o4 = reinterpret_cast<const float4*>(obuf + (src * HPC + slot) * DC + d0);
              const float4 a = o4[0], c4 = o4[1];
              acc[0] = fmaf(wgt, a.x, acc[0]);
              acc[1] = fmaf(wgt, a.y, acc[1]);
              acc[2] = fmaf(wgt, a.z, acc[2]);
              acc[3] = fmaf(wgt, a.w, acc[3]);
              acc[4] = fmaf(wgt, c4.x, acc[4]);
              acc[5] = fmaf(wgt, c4.y, acc[5]);
              acc[6] = fmaf(wgt, c4.z, acc[6]);
              acc[7] = fmaf(wgt, c4.w, acc[7]);
            }
            uint32_t w4[4];
#pragma unroll
            for (int u = 0; u < 8; u += 2) {
              const __nv_bfloat162 o2 = __floats2bfloat162_rn(acc[u], acc[u + 1]);
              w4[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            *reinterpret_cast<uint4*>(p.out + row * DC + d0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          if (lane == 0 && p.lse) p.lse[row] = (L > 0.0f) ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dsa
