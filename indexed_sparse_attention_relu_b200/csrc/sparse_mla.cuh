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
//  * a producer warp gathers the 64 rows with TMA tile::gather4 (four rows per
//    instruction, 128-byte swizzle applied by the tensor map) into a
//    two-stage ring; an index of -1 or out of range becomes an out-of-bounds
//    row, which TMA fills with zeros;
//  * one thread issues S = Q K^T (M = 64 heads, N = 64 keys, K = D) and
//    O += P V (M = 64, N = d_c in 256-wide pieces, K = 64 keys) on tcgen05;
//    the value operand is the same shared-memory tile read as an MN-major
//    matrix, so each row is gathered once;
//  * with M = 64 an accumulator uses lanes 0-15 of each TMEM sub-partition,
//    so O (all d_c columns) sits at lane offset 0 and S at lane offset 16 of
//    the same columns: both fit in one SM's TMEM;
//  * 4 softmax warps (threads 16-31 hold the S rows, threads 0-15 the O rows
//    of the same heads) run an online softmax in the exp2 domain with lazy
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
  static constexpr int NUM_WARPS = 6;  // 0-3 softmax/epilogue, 4 TMA producer, 5 MMA
  static constexpr int THREADS = NUM_WARPS * 32;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_P = OFF_KV + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int NUM_BARS = 2 * NST + 8;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
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
    sparse_mla_kernel(const __grid_constant__ CUtensorMap kvmap, const __grid_constant__ CUtensorMap qmap,
                      const MlaParams p) {
  using C = MlaCfg<D, DC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;             // [NST] TMA -> MMA
  uint64_t* kv_empty = bars + C::NST;   // [NST] MMA (PV done) -> TMA
  uint64_t* q_full = kv_empty + C::NST; // TMA -> MMA
  uint64_t* s_full = q_full + 1;        // MMA (S ready) -> softmax
  uint64_t* s_empty = s_full + 1;       // softmax (S read) -> MMA
  uint64_t* p_full = s_empty + 1;       // softmax (P written) -> MMA
  uint64_t* o_done = p_full + 1;        // MMA (PV done) -> softmax
  uint64_t* drain = o_done + 1;
  uint64_t* ready = drain + 1;          // merge: every CTA of the cluster has finished its loop
  uint64_t* recv = ready + 1;           // merge: every partial row destined here has arrived
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);
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
      mbar_init(&kv_full[i], 1);
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
    prefetch_tensormap(&kvmap);
    prefetch_tensormap(&qmap);
  }
  if (warp == 5) {
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

  if (warp == 4 && lane == 0) {
    // the query block is an input of the call, not of the Top-K: load it now
    mbar_arrive_expect_tx(q_full, C::Q_BYTES);
    const uint32_t qs = smem_u32(smem + C::OFF_Q);
#pragma unroll
    for (int c = 0; c < C::AKQ; ++c) tma_load_2d(qs + c * C::ATOM_COL, &qmap, c * 64, t * p.H + h0, q_full);
  }
  pdl_wait_prior();  // the selected indices (Top-K output) are complete from here on

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer (one warp)
    const int32_t row_base = b * p.L_max;
    const int32_t oob_row = p.B * p.L_max;  // past the end: TMA zero-fills the row
    int issued = 0;
    for (int it = 0; it < n_tiles; ++it) {
      const int st = it & 1;
      if (!mbar_wait_warp(&kv_empty[st], ((it >> 1) & 1) ^ 1, abort_flag)) break;
      ++issued;
      const int kb = k_begin + it * C::TK;
      const int s0 = (kb + lane < k_end) ? __ldg(idx_row + kb + lane) : -1;
      const int s1 = (kb + 32 + lane < k_end) ? __ldg(idx_row + kb + 32 + lane) : -1;
      const bool ok0 = s0 >= 0 && s0 < len, ok1 = s1 >= 0 && s1 < len;
      if ((s0 != -1 && !ok0) || (s1 != -1 && !ok1)) set_device_status(DSA_ERR_DEVICE_INDEX);
      const int32_t r0 = ok0 ? row_base + s0 : oob_row;
      const int32_t r1 = ok1 ? row_base + s1 : oob_row;
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[st], C::KV_BYTES);
      __syncwarp();
      // lane g < 16 gathers keys 4g .. 4g+3 of the tile
      int32_t y[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = 4 * (lane & 15) + j;  // key slot
        const int32_t lo = __shfl_sync(0xffffffffu, r0, k & 31);
        const int32_t hi = __shfl_sync(0xffffffffu, r1, k & 31);
        y[j] = (k < 32) ? lo : hi;
      }
      if (lane < 16) {
        const uint32_t dst = smem_u32(smem + C::OFF_KV + st * C::KV_BYTES) + lane * 4 * 128;
#pragma unroll
        for (int c = 0; c < C::AKQ; ++c)
          tma_gather4(dst + c * C::ATOM_COL, &kvmap, c * 64, y[0], y[1], y[2], y[3], &kv_full[st]);
      }
    }
    // drain: no TMA copy may still be landing when the CTA retires (matters
    // only after a timeout; otherwise every phase below has completed)
    if (lane == 0) {
      volatile int never = 0;
      mbar_wait(q_full, 0, &never);
      for (int it = issued > 2 ? issued - 2 : 0; it < issued; ++it) mbar_wait(&kv_full[it & 1], (it >> 1) & 1, &never);
    }
  } else if (warp == 5) {
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
    float m_used = -INFINITY;                              // running max (log2 domain)
    float l = 0.0f;                                        // running sum of P
    bool ok = true;
    uint8_t* p_tile = smem + C::OFF_P;
    for (int it = 0; it < n_tiles; ++it) {
      if (!(ok = mbar_wait_warp(s_full, it & 1, abort_flag))) break;
      tc_fence_after();
      float s[64];
      {
        float v[4][16];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld16(tmem_base + lane_addr + c * 16, v[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int u = 0; u < 16; ++u) s[c * 16 + u] = v[c][u];
      }
      // validity of the 64 keys of this tile (same for every head)
      const int kb = k_begin + it * C::TK;
      const int i0 = (kb + lane < k_end) ? __ldg(idx_row + kb + lane) : -1;
      const int i1 = (kb + 32 + lane < k_end) ? __ldg(idx_row + kb + 32 + lane) : -1;
      const unsigned v0 = __ballot_sync(0xffffffffu, i0 >= 0 && i0 < len);
      const unsigned v1 = __ballot_sync(0xffffffffu, i1 >= 0 && i1 < len);
      float mt = -INFINITY;
#pragma unroll
      for (int j = 0; j < 64; ++j) {
        const bool valid = (j < 32) ? ((v0 >> j) & 1u) : ((v1 >> (j - 32)) & 1u);
        s[j] = valid ? s[j] * p.scale_log2 : -INFINITY;
        mt = fmaxf(mt, s[j]);
      }
      float factor = 1.0f;
      bool need = false;
      if (is_s) {
        const float m_new = fmaxf(m_used, mt);
        need = m_new > m_used + 8.0f;
        if (need) {
          factor = exp2f(m_used - m_new);
          l *= factor;
          m_used = m_new;
        }
      }
      bool o_waited = false;
      if (__any_sync(0xffffffffu, need && it > 0)) {
        // O already holds earlier tiles: wait for PV(it-1), then rescale those rows.
        if (!(ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag))) break;
        o_waited = true;
        tc_fence_after();
        const float fo = __shfl_sync(0xffffffffu, factor, lane | 16);
        for (int c = 0; c < DC; c += 16) {
          float v[16];
          tmem_ld16(tmem_base + lane_addr + c, v);
          tmem_wait_ld();
          if (!is_s) {
#pragma unroll
            for (int u = 0; u < 16; ++u) v[u] *= fo;
          }
          tmem_st16(tmem_base + lane_addr + c, v);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      // P = 2^(s - m) in bf16; l sums the rounded values actually used by PV
      uint32_t packed[32];
#pragma unroll
      for (int j = 0; j < 64; j += 2) {
        const float a = (s[j] == -INFINITY || m_used == -INFINITY) ? 0.0f : exp2f(s[j] - m_used);
        const float c2 = (s[j + 1] == -INFINITY || m_used == -INFINITY) ? 0.0f : exp2f(s[j + 1] - m_used);
        const __nv_bfloat162 pr = __floats2bfloat162_rn(a, c2);
        l += __low2float(pr) + __high2float(pr);
        packed[j / 2] = *reinterpret_cast<const uint32_t*>(&pr);
      }
      if (it > 0 && !o_waited) {
        if (!(ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag))) break;  // P buffer free
      }
      if (is_s) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(p_tile + sw128_offset(h_local, c)) =
              make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = mbar_wait_warp(o_done, (n_tiles - 1) & 1, abort_flag);
    const float l_h = __shfl_sync(0xffffffffu, l, lane | 16);
    const float m_h = __shfl_sync(0xffffffffu, m_used, lane | 16);
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
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dsa
