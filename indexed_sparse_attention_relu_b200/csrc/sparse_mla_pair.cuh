// sparse_mla_pair.cuh -- sparse MLA attention for 128 query heads over the
// 576-dim latent rows (d_c = 512, d_rope = 64): Sparse Flash Attention of
// "Day-0 Inference Optimization for a New Sparse Attention Architecture",
// section 1, on the KV-cache rows the Lightning Indexer selected.
//
// For query token t, head h and selected rows s_i:
//   z_i = softmax_scale * q[t,h,:] . kv[b,s_i,:]          (all 576 dims)
//   out[t,h,:] = sum_i softmax(z)_i * kv[b,s_i,0:512]     (value = latent part)
//   lse[t,h] = log sum_i exp(z_i)
//
// Work split. The two CTAs of a pair split the dims of every row: CTA half
// dh gathers latent dims [256 dh, 256 dh + 256) and rope dims
// [512 + 32 dh, 512 + 32 dh + 32) of each selected row (576 of the 1152 bytes,
// so every byte of a row crosses HBM once), and owns the output columns
// [256 dh, 256 dh + 256) of all 128 heads. Per tile of 64 selected keys:
//  * S_dh = Q_dh K_dh^T is a partial score over the CTA's 288 dims
//    (tcgen05, M = 128 heads at full rate, N = 64 keys, K = 288);
//  * the softmax warps swap partial scores with the peer CTA through
//    distributed shared memory; both CTAs then hold S = S_0 + S_1 (fp32
//    addition commutes, so both compute bit-identical softmax statistics and
//    probabilities and never need to agree on anything else);
//  * O_dh += P V_dh (M = 128, N = 256 value dims, K = 64 keys).
// Q (288 dims per head) and P live in tensor memory as the A operands, so
// shared memory holds only the gathered rows (four 40 KB stages) and the
// exchange buffers. TMEM columns: O [0,256), S [256,320), P [320,352),
// Q [352,496).
//
// Roles (13 warps): 0-7 softmax and epilogue (warp w reads TMEM lanes
// 32 (w % 4) .. +31, i.e. head rows, and key columns 32 (w / 4) .. +31 of S),
// 8-11 gather producers (16-byte cp.async straight into the 128-byte-swizzled
// K-major tile; an index of -1 or out of range zero-fills its row), 12 MMA
// issuer and TMEM owner. Key splits of one token (when the grid has more SMs
// than tokens) merge their partial O rows inside the cluster, as in the
// 64-head kernel. Every wait is bounded.
#pragma once
#include "dsa_common.cuh"
#include "sparse_mla.cuh"

namespace dsa {

struct PairCfg {
  static constexpr int D = 576;                      // d_c + d_rope
  static constexpr int DC = 512;                     // value (latent) dims
  static constexpr int DCH = 256;                    // latent dims per CTA
  static constexpr int DRH = 32;                     // rope dims per CTA
  static constexpr int M = 128;                      // heads = MMA M
  static constexpr int TK = 64;                      // keys per tile
  static constexpr int KSTEPS = (DCH + DRH) / 16;    // 18 K steps of the QK^T product
  static constexpr int ATOM_COL = TK * 128;          // one 64-dim atom column of a 64-row tile
  static constexpr int KV_BYTES = 5 * ATOM_COL;      // 4 latent atoms + the rope atom (first half used)
  static constexpr int NST = 4;                      // gather stages
  static constexpr int X_BYTES = M * TK * 4;         // one partial-score tile (fp32)
  static constexpr int NX = 2;                       // exchange buffers
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_X = OFF_KV + NST * KV_BYTES;
  static constexpr int OFF_RED = OFF_X + NX * X_BYTES;
  static constexpr int RED_BYTES = 2 * 2 * M * 4;    // [tile parity][key half][head] row maxima
  static constexpr int OFF_BAR = OFF_RED + RED_BYTES;
  static constexpr int NUM_BARS = 2 * NST + 6 + 2 * NX + 2;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr uint32_t COL_O = 0, COL_S = 256, COL_P = 320, COL_Q = 352;
  static constexpr int TMEM_COLS = 512;
  static constexpr int NUM_WARPS = 13;
  static constexpr int THREADS = NUM_WARPS * 32;
  static constexpr int MAX_SPLITS = 4;               // cluster = 2 x splits CTAs <= 8
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(M, TK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(M, DCH, false, true);
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(COL_Q + (DCH + DRH) / 2 <= TMEM_COLS, "TMEM budget");
  // merge buffers: S * ceil(128 / S) <= 129 partial rows (S <= 4) reuse the
  // gather ring, their statistics the exchange buffers
  static_assert(129 * DCH * 4 <= NST * KV_BYTES, "merge rows must fit in the gather ring");
  static_assert(129 * 8 <= NX * X_BYTES, "merge statistics must fit in the exchange buffers");
};

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// Asynchronous 16-byte store into a cluster peer's shared memory that
// completes 16 bytes of the transaction count of the peer's barrier.
__device__ __forceinline__ void st_async_v4(uint32_t cluster_addr, float a, float b, float c, float d,
                                            uint32_t cluster_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
                   cluster_addr),
               "f"(a), "f"(b), "f"(c), "f"(d), "r"(cluster_bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_wait_cluster_warp(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait_cluster(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

__global__ void __launch_bounds__(PairCfg::THREADS, 1)
    sparse_mla_pair_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ kv,
                           const MlaParams p) {
  using C = PairCfg;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled tiles need 1024-byte alignment; the dynamic window starts
  // at the same offset in every CTA, so either all CTAs leave here or none.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) set_device_status(DSA_ERR_DEVICE_LAYOUT);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;               // [NST] gather producers -> MMA
  uint64_t* kv_empty = bars + C::NST;     // [NST] MMA (PV done) -> producers
  uint64_t* q_full = kv_empty + C::NST;   // softmax warps (Q in TMEM) -> MMA
  uint64_t* s_full = q_full + 1;          // MMA (partial S ready) -> softmax
  uint64_t* s_empty = s_full + 1;         // softmax (S read) -> MMA
  uint64_t* p_full = s_empty + 1;         // softmax (P in TMEM) -> MMA
  uint64_t* o_done = p_full + 1;          // MMA (PV done) -> softmax
  uint64_t* drain = o_done + 1;
  uint64_t* xfull = drain + 1;            // [NX] peer's partial S has landed here
  uint64_t* xfree = xfull + C::NX;        // [NX] peer has read the partial S sent to it
  uint64_t* ready = xfree + C::NX;        // merge: every same-half CTA finished its loop
  uint64_t* recv = ready + 1;             // merge: every partial row for this CTA arrived
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);  // [0] TMEM base, [1] abort
  volatile int* abort_flag = misc + 1;

  const uint32_t crank = cluster_ctarank();
  const int dh = static_cast<int>(crank & 1u);   // dim half
  const int split = static_cast<int>(crank >> 1);
  const uint32_t peer = crank ^ 1u;
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

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&kv_full[i], 128);  // one asynchronous arrival per producer thread
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 8);
    mbar_init(s_full, 1);
    mbar_init(s_empty, 8);
    mbar_init(p_full, 8);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    for (int i = 0; i < C::NX; ++i) {
      mbar_init(&xfull[i], 1);    // armed by thread 0; the peer's stores complete its bytes
      mbar_init(&xfree[i], 8);    // one arrival per softmax warp of the peer
    }
    mbar_init(ready, S);
    mbar_init(recv, 256 * S);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();  // the peers' barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);

  if (warp < 8) {
    // ------------------------------------------------------------ softmax + epilogue (warps 0..7)
    const int q4 = warp & 3;          // TMEM lane quarter
    const int half = warp >> 2;       // key half of S; column half of this CTA's O
    const int h = q4 * 32 + lane;     // head row
    const uint32_t lane_addr = static_cast<uint32_t>(q4 * 32) << 16;
    // Q -> TMEM (a call input, independent of the preceding kernels). Thread
    // (h, half 0) writes latent dims [256 dh, +128) to Q columns 0..63;
    // (h, half 1) latent dims [256 dh + 128, +128) to 64..127 and the rope
    // dims [512 + 32 dh, +32) to 128..143 (two bf16 per column).
    {
      const bool hv = h < p.H;
      const uint4* qrow = reinterpret_cast<const uint4*>(q + (static_cast<int64_t>(t) * p.H + (hv ? h : 0)) * C::D);
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      uint4 buf[20];
      const int lat = (C::DCH * dh + 128 * half) / 8;
#pragma unroll
      for (int i = 0; i < 16; ++i) buf[i] = hv ? __ldg(qrow + lat + i) : z;
      const int rope = (C::DC + C::DRH * dh) / 8;
#pragma unroll
      for (int i = 0; i < 4; ++i) buf[16 + i] = (hv && half) ? __ldg(qrow + rope + i) : z;
      const int groups = half ? 5 : 4;
#pragma unroll
      for (int g = 0; g < 5; ++g) {
        if (g < groups) {
          uint32_t w[16];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            w[4 * u + 0] = buf[4 * g + u].x;
            w[4 * u + 1] = buf[4 * g + u].y;
            w[4 * u + 2] = buf[4 * g + u].z;
            w[4 * u + 3] = buf[4 * g + u].w;
          }
          tmem_st16u(tmem_base + lane_addr + C::COL_Q + 64 * half + 16 * g, w);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    pdl_wait_prior();  // the selected indices (Top-K output) are complete from here on

    const uint32_t x_local = smem_u32(smem + C::OFF_X);
    const uint32_t x_peer = mapa_shared(x_local, peer);
    const uint32_t xfull_peer = mapa_shared(smem_u32(xfull), peer);
    const uint32_t xfree_peer = mapa_shared(smem_u32(xfree), peer);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    const uint32_t rowoff = static_cast<uint32_t>(h) * 256u;
    float m_run = -INFINITY;  // running row maximum (log2 domain), identical in both CTAs
    float l_part = 0.0f;      // this thread's share (its 32 key columns) of the running sum
    bool ok = true;
    // Receive buffer b holds the peer's partial scores of tiles b, b + 2, ...
    // Its barrier completes when thread 0 has armed it with one tile's byte
    // count and the peer's asynchronous stores have delivered those bytes
    // (stores landing before the arming are allowed: the count goes negative).
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(&xfull[0], C::X_BYTES);
      if (n_tiles > 1) mbar_arrive_expect_tx(&xfull[1], C::X_BYTES);
    }
    // Reads partial S(it) from TMEM, hands the S buffer back to the MMA and
    // sends the values to the peer: row h, key chunks 8 half .. +7 (16-byte
    // chunks, XOR-swizzled by h & 15 against bank conflicts), as asynchronous
    // stores that complete on the peer's barrier, so no thread waits for them.
    auto load_send = [&](int it, float (&v)[32]) -> bool {
      if (!mbar_wait_warp(s_full, it & 1, abort_flag)) return false;
      tc_fence_after();
      float va[16], vb[16];
      tmem_ld16(tmem_base + lane_addr + C::COL_S + 32 * half, va);
      tmem_ld16(tmem_base + lane_addr + C::COL_S + 32 * half + 16, vb);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        v[i] = va[i];
        v[16 + i] = vb[i];
      }
      const int xb = it & 1;
      // the peer has consumed tile it - 2 from this buffer
      if (!mbar_wait_cluster_warp(&xfree[xb], ((it >> 1) & 1) ^ 1u, abort_flag)) return false;
      const uint32_t dst = x_peer + xb * C::X_BYTES + rowoff;
      const uint32_t bar = xfull_peer + xb * 8;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t chunk = static_cast<uint32_t>(8 * half + k) ^ (static_cast<uint32_t>(h) & 15u);
        st_async_v4(dst + chunk * 16u, v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3], bar);
      }
      return true;
    };
    // index of this lane's key column of a tile (validity mask), loaded a
    // tile before its ballot
    auto raw_idx = [&](int tile) -> int {
      const int k = k_begin + tile * C::TK + 32 * half + lane;
      return (tile < n_tiles && k < k_end) ? ld_dep(idx_row + k) : -1;
    };
    int raw_cur = raw_idx(0);
    int raw_nxt = raw_idx(1);
    float cur[32], nxt[32];
    ok = load_send(0, cur);
    // Software pipeline: iteration it first loads and sends tile it + 1, then
    // finishes tile it with the peer's partial scores, which were sent while
    // this CTA worked on tile it - 1.
    for (int it = 0; it < n_tiles; ++it) {
      if (ok && it + 1 < n_tiles) ok = load_send(it + 1, nxt);
      const unsigned vmask = __ballot_sync(0xffffffffu, raw_cur >= 0 && raw_cur < len);
      const int raw_after = raw_idx(it + 2);
      float tmax = -INFINITY;
      if (ok) {
        const int xb = it & 1;
        ok = mbar_wait_cluster_warp(&xfull[xb], (it >> 1) & 1, abort_flag);
        if (ok) {
          const uint32_t src = x_local + xb * C::X_BYTES + rowoff;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t chunk = static_cast<uint32_t>(8 * half + k) ^ (static_cast<uint32_t>(h) & 15u);
            const float4 w = ld_shared_v4(src + chunk * 16u);
            cur[4 * k] += w.x;
            cur[4 * k + 1] += w.y;
            cur[4 * k + 2] += w.z;
            cur[4 * k + 3] += w.w;
          }
          __syncwarp();
          // re-arm for tile it + 2 (this phase is complete), then free the buffer
          if (threadIdx.x == 0 && it + 2 < n_tiles) mbar_arrive_expect_tx(&xfull[xb], C::X_BYTES);
          if (lane == 0) mbar_arrive_remote(xfree_peer + xb * 8);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            cur[i] = ((vmask >> i) & 1u) ? cur[i] * p.scale_log2 : -INFINITY;
            tmax = fmaxf(tmax, cur[i]);
          }
        }
      }
      // row maximum across the two warps holding the row's key halves (both
      // warps run every iteration, so the named barrier always matches)
      red[(it & 1) * 256 + half * 128 + h] = tmax;
      named_bar_sync(1 + q4, 64);
      tmax = fmaxf(tmax, red[(it & 1) * 256 + (1 - half) * 128 + h]);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) {
        float f = 1.0f;
        const float nm = fmaxf(m_run, tmax);
        const bool need = nm > m_run + 8.0f;  // lazy rescale: P stays <= 2^8
        if (need) {
          f = ex2_approx(m_run - nm);  // 0 when m_run = -inf
          l_part *= f;
          m_run = nm;
        }
        bool o_waited = false;
        if (__any_sync(0xffffffffu, need && it > 0)) {
          // O holds earlier tiles: wait for PV(it-1), then rescale this thread's 128 columns
          ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag);
          o_waited = true;
          if (ok) {
            tc_fence_after();
            for (int c = 0; c < 128; c += 16) {
              float o[16];
              tmem_ld16(tmem_base + lane_addr + C::COL_O + 128 * half + c, o);
              tmem_wait_ld();
              if (need) {
#pragma unroll
                for (int u = 0; u < 16; ++u) o[u] *= f;
              }
              tmem_st16(tmem_base + lane_addr + C::COL_O + 128 * half + c, o);
            }
            tmem_wait_st();
          }
        }
        // P = 2^(s - m) in bf16, two keys per TMEM column; the sums add the
        // rounded values the PV product uses
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float a0 = (m_run == -INFINITY) ? 0.0f : ex2_approx(cur[2 * i] - m_run);
          const float a1 = (m_run == -INFINITY) ? 0.0f : ex2_approx(cur[2 * i + 1] - m_run);
          const __nv_bfloat162 pr = __floats2bfloat162_rn(a0, a1);
          l_part += __low2float(pr) + __high2float(pr);
          pk[i] = *reinterpret_cast<const uint32_t*>(&pr);
        }
        if (ok && it > 0 && !o_waited) {
          ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag);  // P(it-1) consumed
          if (ok) tc_fence_after();
        }
        if (ok) {
          tmem_st16u(tmem_base + lane_addr + C::COL_P + 16 * half, pk);
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(p_full);
        }
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) cur[i] = nxt[i];
      raw_cur = raw_nxt;
      raw_nxt = raw_after;
    }
    // full row sum: add the partner warp's share (slot parity n_tiles & 1 was
    // last read before the previous iteration's barrier)
    red[(n_tiles & 1) * 256 + half * 128 + h] = l_part;
    named_bar_sync(1 + q4, 64);
    const float l = l_part + red[(n_tiles & 1) * 256 + (1 - half) * 128 + h];
    if (ok) ok = mbar_wait_warp(o_done, (n_tiles - 1) & 1, abort_flag);
    if (ok) tc_fence_after();
    const uint32_t o_addr = tmem_base + lane_addr + C::COL_O + 128 * half;
    if (S == 1) {
      if (ok) {
        const bool writer = h < p.H;
        const float inv = (l > 0.0f) ? 1.0f / l : 0.0f;
        const int64_t row = static_cast<int64_t>(t) * p.H + h;
        __nv_bfloat16* dst = p.out + row * C::DC + C::DCH * dh + 128 * half;
        for (int c = 0; c < 128; c += 16) {
          float o[16];
          tmem_ld16(o_addr + c, o);
          tmem_wait_ld();
          if (writer) {
            uint32_t w8[8];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
              const __nv_bfloat162 o2 = __floats2bfloat162_rn(o[u] * inv, o[u + 1] * inv);
              w8[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
            d4[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            d4[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
          }
        }
        if (writer && dh == 0 && half == 0 && p.lse)
          p.lse[row] = (l > 0.0f) ? (m_run + log2f(l)) * 0.69314718055994531f : -INFINITY;
      }
    } else {
      // ---------------- merge the key-split partials of this dim half
      // Head h belongs to split owner = h % S (slot h / S). Every CTA sends
      // its unnormalised O row half with (running max, row sum) into the
      // owner's buffer (entry split * HPC + slot); the owner combines.
      const int HPC = (C::M + S - 1) / S;
      const uint32_t obuf = smem_u32(smem + C::OFF_KV);
      const uint32_t sbuf = smem_u32(smem + C::OFF_X);
      if (ok && threadIdx.x == 0) {
        // this CTA's loop is done (all products complete, every gathered tile
        // consumed, the peer's last partial scores read): its gather ring and
        // exchange buffers may now be overwritten by the same-half CTAs
        for (int s2 = 0; s2 < S; ++s2) mbar_arrive_remote(mapa_shared(smem_u32(ready), 2 * s2 + dh));
      }
      if (ok) ok = mbar_wait_cluster_warp(ready, 0, abort_flag);
      if (ok) {
        const uint32_t owner = static_cast<uint32_t>(2 * (h % S) + dh);
        const int entry = split * HPC + h / S;
        const uint32_t o_dst = mapa_shared(obuf + entry * C::DCH * 4 + half * 512, owner);
        for (int c = 0; c < 128; c += 16) {
          float o[16];
          tmem_ld16(o_addr + c, o);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 16; u += 4) st_cluster_v4(o_dst + (c + u) * 4, o[u], o[u + 1], o[u + 2], o[u + 3]);
        }
        if (half == 0) st_cluster_v2(mapa_shared(sbuf + entry * 8, owner), m_run, l);
        for (int s2 = 0; s2 < S; ++s2) mbar_arrive_remote(mapa_shared(smem_u32(recv), 2 * s2 + dh));
      }
      if (ok) ok = mbar_wait_cluster_warp(recv, 0, abort_flag);
      if (ok) {
        const float* ob = reinterpret_cast<const float*>(smem + C::OFF_KV);
        const float2* sb = reinterpret_cast<const float2*>(smem + C::OFF_X);
        for (int slot = warp; slot < HPC; slot += 8) {
          const int hh = slot * S + split;
          if (hh >= C::M || hh >= p.H) continue;
          float Mx = -INFINITY;
          for (int src = 0; src < S; ++src) Mx = fmaxf(Mx, sb[src * HPC + slot].x);
          float L = 0.0f;
          for (int src = 0; src < S; ++src) {
            const float2 st = sb[src * HPC + slot];
            if (st.y > 0.0f) L += exp2f(st.x - Mx) * st.y;
          }
          const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
          const int64_t row = static_cast<int64_t>(t) * p.H + hh;
          const int d0 = lane * 8;
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
          for (int src = 0; src < S; ++src) {
            const float2 st = sb[src * HPC + slot];
            if (!(st.y > 0.0f)) continue;
            const float wgt = exp2f(st.x - Mx) * inv;
            const float4* o4 = reinterpret_cast<const float4*>(ob + (src * HPC + slot) * C::DCH + d0);
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
          *reinterpret_cast<uint4*>(p.out + row * C::DC + C::DCH * dh + d0) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          if (lane == 0 && dh == 0 && p.lse)
            p.lse[row] = (L > 0.0f) ? (Mx + log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
      }
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ gather producers (warps 8..11)
    // warp pw copies rows 16 pw .. 16 pw + 15 of each tile: one warp
    // instruction moves the 512 latent bytes of a row (32 chunks of 16 bytes),
    // one more the 64 rope bytes of 8 rows (4 chunks each)
    pdl_wait_prior();
    const int pw = warp - 8;
    const __nv_bfloat16* kv_seq = kv + static_cast<int64_t>(b) * p.L_max * C::D;
    auto row_index = [&](int tile) -> int {
      const int k = k_begin + tile * C::TK + 16 * pw + lane;
      return (lane < 16 && tile < n_tiles && k < k_end) ? ld_dep(idx_row + k) : -1;
    };
    int nxt = row_index(0);
    for (int it = 0; it < n_tiles; ++it) {
      const int sl = it % C::NST;
      const uint32_t use = static_cast<uint32_t>(it / C::NST);
      const int cur = nxt;
      nxt = row_index(it + 1);  // in flight during the stage wait and the copies
      if (!mbar_wait_warp(&kv_empty[sl], (use & 1u) ^ 1u, abort_flag)) break;
      const bool okr = cur >= 0 && cur < len;
      if (lane < 16 && cur != -1 && !okr) set_device_status(DSA_ERR_DEVICE_INDEX);
      const int mine = okr ? cur : -1;
      const uint32_t stage = smem_u32(smem + C::OFF_KV + sl * C::KV_BYTES);
#pragma unroll 4
      for (int rr = 0; rr < 16; ++rr) {
        const int r = 16 * pw + rr;
        const int srow = __shfl_sync(0xffffffffu, mine, rr);
        const bool has = srow >= 0;
        const __nv_bfloat16* src =
            kv_seq + static_cast<int64_t>(has ? srow : 0) * C::D + C::DCH * dh + lane * 8;
        cp_async_16(stage + (lane >> 3) * C::ATOM_COL + sw128_offset(r, lane & 7), has ? src : kv, has ? 16u : 0u);
      }
#pragma unroll
      for (int g = 0; g < 2; ++g) {
        const int rl = 8 * g + (lane >> 2);
        const int r = 16 * pw + rl;
        const int c = lane & 3;
        const int srow = __shfl_sync(0xffffffffu, mine, rl);
        const bool has = srow >= 0;
        const __nv_bfloat16* src =
            kv_seq + static_cast<int64_t>(has ? srow : 0) * C::D + C::DC + C::DRH * dh + c * 8;
        cp_async_16(stage + 4 * C::ATOM_COL + sw128_offset(r, c), has ? src : kv, has ? 16u : 0u);
      }
      cp_async_arrive_noinc(&kv_full[sl]);
    }
    cp_async_wait_all();  // nothing may still be landing when the CTA retires
  } else {
    // ------------------------------------------------------------ MMA issuer (warp 12)
    if (lane == 0) {
      auto issue_s = [&](int it) {
        const uint32_t kvb = smem_u32(smem + C::OFF_KV + (it % C::NST) * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k) {
          const int atom = k < 16 ? (k >> 2) : 4;
          const int sub = k < 16 ? (k & 3) : (k - 16);
          const uint64_t bd = smem_desc_sw128(kvb + atom * C::ATOM_COL + sub * 32, 16, 1024);
          umma_f16_ts(tmem_base + C::COL_S, tmem_base + C::COL_Q + 8 * k, bd, C::IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
      };
      auto issue_pv = [&](int it) {
        const uint32_t kvb = smem_u32(smem + C::OFF_KV + (it % C::NST) * C::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < C::TK / 16; ++kk) {
          // V = the CTA's 256 latent dims of the gathered rows, MN-major:
          // 64-dim atom columns ATOM_COL bytes apart (LBO), 8-key row groups
          // 1024 bytes apart (SBO)
          const uint64_t bd = smem_desc_sw128(kvb + kk * 16 * 128, C::ATOM_COL, 1024);
          umma_f16_ts(tmem_base + C::COL_O, tmem_base + C::COL_P + 8 * kk, bd, C::IDESC_PV,
                      (it > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[it % C::NST]);
        umma_commit(o_done);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag);
      int s_next = 0, pv_next = 0;
      uint64_t t0 = globaltimer();
      // Issue whichever product is ready: S(j) needs tile j gathered and the
      // softmax done reading S(j-1) (one S buffer); PV(j) needs P(j).
      while (ok && pv_next < n_tiles) {
        bool progressed = false;
        if (s_next < n_tiles) {
          const int sl = s_next % C::NST;
          const uint32_t use = static_cast<uint32_t>(s_next / C::NST);
          if ((s_next == 0 || mbar_try(smem_u32(s_empty), (s_next - 1) & 1)) &&
              mbar_try(smem_u32(&kv_full[sl]), use & 1u)) {
            fence_proxy_async_smem();  // cp.async (generic proxy) data -> tensor core reads
            tc_fence_after();
            issue_s(s_next);
            ++s_next;
            progressed = true;
          }
        }
        if (pv_next < s_next && mbar_try(smem_u32(p_full), pv_next & 1)) {
          tc_fence_after();
          issue_pv(pv_next);
          ++pv_next;
          progressed = true;
        }
        if (progressed) {
          t0 = globaltimer();
        } else if (*abort_flag) {
          ok = false;
        } else if (globaltimer() - t0 > kWaitLimitNs) {
          set_device_status(DSA_ERR_DEVICE_TIMEOUT);
          *abort_flag = 1;
          ok = false;
        }
      }
      umma_commit(drain);
      volatile int never = 0;
      mbar_wait(drain, 0, &never);
    }
    __syncwarp();
  }

  // No CTA may retire while a cluster peer can still address its shared
  // memory (exchange buffers, merge rows, remote barrier arrivals).
  tc_fence_before();
  cluster_sync_all();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace dsa
