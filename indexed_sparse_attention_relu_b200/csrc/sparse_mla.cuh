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
// One CTA = (token, 64-head block, key split). Per tile of 64 selected keys:
//  * 4 producer warps gather the 64 rows (D bf16 each) with 16-byte cp.async
//    straight into the 128-byte-swizzled K-major layout tcgen05 reads, zero-
//    filling rows whose index is -1 or out of range (two-stage ring);
//  * one thread issues S = Q K^T (M = 64 heads, N = 64 keys, K = D) and
//    O += P V (M = 64, N = d_c in 256-wide pieces, K = 64 keys); the value
//    operand is the same shared-memory tile read as an MN-major matrix;
//  * with M = 64 an accumulator uses lanes 0-15 of each TMEM sub-partition,
//    so O (all d_c columns) sits at lane offset 0 and S at lane offset 16 of
//    the same columns: both fit in one SM's TMEM;
//  * 4 softmax warps (threads 16-31 hold the S rows, threads 0-15 the O rows
//    of the same heads) run an online softmax in the exp2 domain with lazy
//    rescaling: O is only rescaled (TMEM load/scale/store) when a row maximum
//    grows by more than 2^8, which keeps P <= 256 and exact final results;
//  * P is written as bf16 to shared memory (A operand of the PV product).
// With several key splits each CTA writes (O / l, lse) partials and a small
// combine kernel merges them with log-sum-exp weights.
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
  const __nv_bfloat16* q;    // [T, H, D]
  const __nv_bfloat16* kv;   // [B, L_max, D]
  const int32_t* idx;        // [T, K]
  float scale_log2;          // softmax_scale * log2(e)
  int32_t keys_per_split;    // multiple of 64
  int32_t splits;
  __nv_bfloat16* out;        // [T, H, DC]
  float* lse;                // [T, H] or null
  float* part_o;             // [splits, T, H, DC]
  float* part_lse;           // [splits, T, H]
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
  static constexpr int NUM_WARPS = 9;  // 0-3 producers, 4-7 softmax/epilogue, 8 MMA
  static constexpr int THREADS = NUM_WARPS * 32;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_KV = OFF_Q + Q_BYTES;
  static constexpr int OFF_P = OFF_KV + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int NUM_BARS = 2 * NST + 5;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(64, TK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(64, N_PV, false, true);
  static_assert(DC % N_PV == 0 && DC % 64 == 0, "latent dim must be a multiple of 64");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int D, int DC>
__global__ void __launch_bounds__(MlaCfg<D, DC>::THREADS, 1) sparse_mla_kernel(const MlaParams p) {
  using C = MlaCfg<D, DC>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;             // [NST] producers -> MMA
  uint64_t* kv_empty = bars + C::NST;   // [NST] MMA (PV done) -> producers
  uint64_t* s_full = kv_empty + C::NST; // MMA (S ready) -> softmax
  uint64_t* s_empty = s_full + 1;       // softmax (S read) -> MMA
  uint64_t* p_full = s_empty + 1;       // softmax (P written) -> MMA
  uint64_t* o_done = p_full + 1;        // MMA (PV done) -> softmax
  uint64_t* drain = o_done + 1;
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = misc + 1;

  const int t = blockIdx.x;
  const int h0 = blockIdx.y * C::HB;
  const int split = blockIdx.z;
  const int warp = warp_id();
  const int lane = lane_id();
  const int b = seq_of_token(p.cu_q, p.B, t);
  const int len = min(__ldg(p.seq_lens + b), p.L_max);
  const int k_begin = split * p.keys_per_split;
  const int k_end = min(p.K, k_begin + p.keys_per_split);
  const int n_tiles = (k_end - k_begin + C::TK - 1) / C::TK;  // >= 1 by construction
  const int32_t* idx_row = p.idx + static_cast<int64_t>(t) * p.K;
  const __nv_bfloat16* kv_seq = p.kv + static_cast<int64_t>(b) * p.L_max * D;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&kv_full[i], 128);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  // Q block: rows = heads h0..h0+63 (zero beyond H), K = D padded to DP with zeros.
  {
    constexpr int CPR = C::DP / 8;
    const uint32_t qs = smem_u32(smem + C::OFF_Q);
    for (int i = threadIdx.x; i < C::HB * CPR; i += C::THREADS) {
      const int r = i / CPR, c = i % CPR;
      const bool has = (h0 + r < p.H) && (c * 8 < D);
      const __nv_bfloat16* src = has ? p.q + (static_cast<int64_t>(t) * p.H + h0 + r) * D + c * 8 : p.q;
      cp_async_16(qs + (c / 8) * C::ATOM_COL + sw128_offset(r, c % 8), src, has ? 16u : 0u);
    }
    cp_async_commit();
    cp_async_wait_all();
  }
  fence_proxy_async_smem();
  if (warp == 8) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);
  const uint32_t tmem_s = tmem_base + (16u << 16);  // S at lane offset 16 (M = 64 layout)

  if (warp < 4) {
    // ------------------------------------------------------------ gather producers
    const int pt = threadIdx.x;  // 0..127
    constexpr int CPR = C::DP / 8;
    for (int it = 0; it < n_tiles; ++it) {
      const int st = it & 1;
      if (!mbar_wait(&kv_empty[st], ((it >> 1) & 1) ^ 1, abort_flag)) break;
      const uint32_t base = smem_u32(smem + C::OFF_KV + st * C::KV_BYTES);
      for (int i = pt; i < C::TK * CPR; i += 128) {
        const int r = i / CPR, c = i % CPR;
        const int kpos = k_begin + it * C::TK + r;
        const int s = (kpos < k_end) ? __ldg(idx_row + kpos) : -1;
        const bool ok = (s >= 0) && (s < len);
        if (c == 0 && s != -1 && !ok) set_device_status(DSA_ERR_DEVICE_INDEX);
        const bool has = ok && (c * 8 < D);
        const __nv_bfloat16* src = has ? kv_seq + static_cast<int64_t>(s) * D + c * 8 : p.kv;
        cp_async_16(base + (c / 8) * C::ATOM_COL + sw128_offset(r, c % 8), src, has ? 16u : 0u);
      }
      // Signal this tile as soon as it lands: the MMA issuer must never wait on
      // a tile whose signal depends on a later PV product.
      cp_async_commit();
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      mbar_arrive(&kv_full[st]);
    }
    cp_async_wait_group<0>();
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
      bool ok = mbar_wait(&kv_full[0], 0, abort_flag);
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
    // ------------------------------------------------------------ softmax + epilogue (warps 4..7)
    const int sw = warp & 3;                               // TMEM sub-partition
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
        float v[16];
#pragma unroll
        for (int c = 0; c < 64; c += 16) {
          tmem_ld16(tmem_base + lane_addr + c, v);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 16; ++u) s[c + u] = v[u];
        }
      }
      // validity of the 64 keys of this tile (same for every head)
      const int kb = k_begin + it * C::TK;
      int i0 = (kb + lane < k_end) ? __ldg(idx_row + kb + lane) : -1;
      int i1 = (kb + 32 + lane < k_end) ? __ldg(idx_row + kb + 32 + lane) : -1;
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
    if (ok) {
      tc_fence_after();
      const float l_h = __shfl_sync(0xffffffffu, l, lane | 16);
      const float m_h = __shfl_sync(0xffffffffu, m_used, lane | 16);
      const int h = h0 + h_local;
      const bool writer = !is_s && h < p.H;
      const float inv = (l_h > 0.0f) ? 1.0f / l_h : 0.0f;
      const float lse_h = (l_h > 0.0f) ? (m_h + log2f(l_h)) * 0.69314718055994531f : -INFINITY;
      const int64_t row = static_cast<int64_t>(t) * p.H + h;
      for (int c = 0; c < DC; c += 16) {
        float v[16];
        tmem_ld16(tmem_base + lane_addr + c, v);
        tmem_wait_ld();
        if (writer) {
          if (p.splits == 1) {
            uint32_t w8[8];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
              const __nv_bfloat162 o2 = __floats2bfloat162_rn(v[u] * inv, v[u + 1] * inv);
              w8[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * DC + c);
            dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
          } else {
            float4* dst = reinterpret_cast<float4*>(p.part_o + (static_cast<int64_t>(split) * p.T * p.H + row) * DC + c);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_float4(v[4 * u] * inv, v[4 * u + 1] * inv, v[4 * u + 2] * inv, v[4 * u + 3] * inv);
          }
        }
      }
      if (writer) {
        if (p.splits == 1) {
          if (p.lse) p.lse[row] = lse_h;
        } else {
          p.part_lse[static_cast<int64_t>(split) * p.T * p.H + row] = lse_h;
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

// Merge split-K partials: out = sum_s e^{lse_s - lse} O_s, lse = log sum_s e^{lse_s}.
__global__ void __launch_bounds__(128) mla_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_lse, int splits, int T,
                                                          int H, int DC, __nv_bfloat16* __restrict__ out,
                                                          float* __restrict__ lse) {
  const int64_t row = blockIdx.x;  // t * H + h
  const int64_t TH = static_cast<int64_t>(T) * H;
  float m = -INFINITY;
  for (int s = 0; s < splits; ++s) m = fmaxf(m, __ldg(part_lse + s * TH + row));
  float wsum = 0.0f;
  for (int s = 0; s < splits; ++s) {
    const float ls = __ldg(part_lse + s * TH + row);
    wsum += (ls == -INFINITY) ? 0.0f : __expf(ls - m);
  }
  const float inv = (wsum > 0.0f) ? 1.0f / wsum : 0.0f;
  for (int d = threadIdx.x * 4; d < DC; d += blockDim.x * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < splits; ++s) {
      const float ls = __ldg(part_lse + s * TH + row);
      if (ls == -INFINITY) continue;
      const float wgt = __expf(ls - m) * inv;
      const float4 o = __ldg(reinterpret_cast<const float4*>(part_o + (s * TH + row) * DC + d));
      acc.x = fmaf(wgt, o.x, acc.x);
      acc.y = fmaf(wgt, o.y, acc.y);
      acc.z = fmaf(wgt, o.z, acc.z);
      acc.w = fmaf(wgt, o.w, acc.w);
    }
    const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 c = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&a);
    pk.y = *reinterpret_cast<const uint32_t*>(&c);
    *reinterpret_cast<uint2*>(out + row * DC + d) = pk;
  }
  if (threadIdx.x == 0 && lse) lse[row] = (wsum > 0.0f) ? m + logf(wsum) : -INFINITY;
}

}  // namespace dsa
