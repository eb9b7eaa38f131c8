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
// One CTA = (token, 64-head block, key split). Each CTA gathers whole rows
// (a gather costs the issuing warps per row, not per byte, so whole rows are
// the cheapest unit). Per tile of 64 selected keys:
//  * eight producer warps gather the 64 rows with 16-byte cp.async straight
//    into the 128-byte-swizzled K-major layout; the 16-byte chunks of a warp's
//    eight rows are packed 32 to an instruction (512 contiguous bytes), and
//    every thread signals its copies through an asynchronous mbarrier
//    arrival; an index of -1 or out of range zero-fills its row (three-stage
//    ring);
//  * one thread issues S = Q K^T (M = 64 heads, N = 64 keys, K = D) and
//    O += P V (M = 64, N = d_c in 256-wide pieces, K = 64 keys) on tcgen05;
//    the value operand is the same shared-memory tile read as an MN-major
//    matrix, so each row is gathered once;
//  * with M = 64 an accumulator uses lanes 0-15 of each TMEM sub-partition:
//    O (all d_c columns) sits at lane offset 0; S (64 columns) and Q (the A
//    operand of S = Q K^T, D/2 columns of bf16 pairs) sit at lane offset 16.
//    Q arrives by TMA in the third gather stage, which is handed to the
//    gather once the softmax warps have moved Q into tensor memory;
//  * 4 softmax warps read S with 16-lane TMEM loads (thread t holds head rows
//    t/4 and t/4 + 8 of its warp's 16 and 16 of the 64 keys) and run an
//    online softmax in the exp2 domain with lazy rescaling: O is only
//    rescaled (16-lane TMEM load/scale/store) when a row maximum grows by
//    more than 2^8, which keeps P <= 256 and the result exact;
//  * P is written as bf16 to shared memory (A operand of the PV product).
// Key splits of one (token, head block) form a thread-block cluster: every
// CTA writes its unnormalised O rows and (running max, running sum) to the
// workspace in global memory, the cluster barrier orders those writes, and
// head h is then finalised by the CTA of split h mod splits (distributed
// shared memory is far slower than L2 for bulk data, so it carries none).
// Every wait is bounded.
#pragma once
#include "dsa_common.cuh"
#include "quant.cuh"

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
  int32_t keys_per_split;    // multiple of the tile size
  int32_t splits;            // == cluster size along z
  __nv_bfloat16* out;        // [T, H, DC]
  float* lse;                // [T, H] or null
  float* part_o;             // [T, HB, splits][DC / 4][64][4] split partials (splits > 1)
  float2* part_ml;           // [T, HB, splits, 64] (running max, running sum)
  CacheMap cm;               // cache rows (contiguous or paged)
};

template <int D, int DC>
struct MlaCfg {
  static constexpr int DP = ((D + 63) / 64) * 64;   // K extent of the stored rows (whole atoms)
  static constexpr int AKQ = DP / 64;               // 128-byte atom columns per row
  static constexpr int HB = 64;                     // heads per CTA (MMA M)
  // keys per tile (QK^T N, PV K) and gather stages. 80-key tiles (a QK^T
  // instruction costs about the same at N = 80 as at N = 64) fit only two
  // stages of 576-dim rows; measured slower (the gather then stalls the
  // MMA), so three 64-key stages are used. The kernel supports both.
  static constexpr int TK = 64;
  static constexpr int NST = 3;
  static constexpr int RPW = TK / 8;                // rows per gather warp
  static constexpr int KSTEPS = (D + 15) / 16;      // K steps of QK^T
  static constexpr int ATOM_COL = TK * 128;         // bytes of one atom column of a TK-row tile
  static constexpr int Q_ATOM = 64 * 128;           // bytes of one atom column of the 64-head Q tile
  static constexpr int KV_BYTES = TK * DP * 2;
  static constexpr int Q_BYTES = HB * DP * 2;       // staged in the last gather stage
  static constexpr int P_ATOMS = (TK + 63) / 64;    // 64-key atom columns of P
  static constexpr int P_BYTES = P_ATOMS * HB * 128;
  static constexpr int N_PV = DC < 256 ? DC : 256;
  static constexpr int PV_MMAS = DC / N_PV;
  static constexpr uint32_t COL_S = 0;              // lane offset 16, TK columns
  static constexpr uint32_t COL_Q = ((TK + 63) / 64) * 64;  // lane offset 16, DP/2 columns
  static constexpr int TMEM_NEED = (DC > (int)COL_Q + DP / 2) ? DC : (int)COL_Q + DP / 2;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                   : TMEM_NEED <= 256 ? 256 : 512;
  static constexpr int PRODUCERS = 8;               // gather warps
  static constexpr int NUM_WARPS = 4 + PRODUCERS + 1;  // 0-3 softmax/epilogue, 4-11 gather, 12 MMA + TMEM owner
  static constexpr int THREADS = NUM_WARPS * 32;
  static constexpr int OFF_KV = 0;
  static constexpr int OFF_P = OFF_KV + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int NUM_BARS = 2 * NST + 8;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16;
  static constexpr int MAX_SPLITS = 8;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(64, TK, false, false);
  static constexpr uint32_t IDESC_PV = idesc_bf16_f32(64, N_PV, false, true);
  static_assert(DC % N_PV == 0 && DC % 64 == 0, "latent dim must be a multiple of 64");
  static_assert(TK % 16 == 0 && (TK == 64 || TK == 80), "tile of 64 or 80 keys");
  static_assert(ATOM_COL % 1024 == 0, "swizzle atoms stay 1024-byte aligned");
  static_assert(TMEM_NEED <= 512, "TMEM budget");
  static_assert(Q_BYTES <= KV_BYTES, "Q is staged in one gather stage");
  static_assert((DP / 2) % 32 == 0, "Q columns come in 32-column groups");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// 16 lanes x 256 bits, 8 repetitions (64 columns): the store counterpart of
// tmem_ld16x256_x8 (same register layout).
__device__ __forceinline__ void tmem_st16x256_x8(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}

// 16 lanes x 256 bits, 4 repetitions (32 columns), store.
__device__ __forceinline__ void tmem_st16x256_x4(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// 16 lanes x 256 bits, 2 repetitions (16 columns): the 16x256b register
// layout of tmem_ld16x256_x8 for two 8-column repetitions.
__device__ __forceinline__ void tmem_ld16x256_x2(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ uint2 ld_shared_v2u(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr) : "memory");
  return v;
}

// Packed bf16 pairs of Q for TMEM column `col` (dims 2col, 2col+1) of the
// thread's two head rows, read from the TMA-staged swizzled Q tile.
template <int ATOM_COL>
__device__ __forceinline__ void q_pair(uint32_t q_stage, int ha, int hbr, int col, uint32_t& xa0, uint32_t& xa1,
                                       uint32_t& xb0, uint32_t& xb1) {
  const int d = 2 * col;                                        // first dim of the two columns
  const uint32_t off = (d >> 6) * ATOM_COL + (d & 7) * 2;       // atom column, byte in the chunk
  const uint2 x = ld_shared_v2u(q_stage + off + sw128_offset(ha, (d & 63) >> 3));
  const uint2 y = ld_shared_v2u(q_stage + off + sw128_offset(hbr, (d & 63) >> 3));
  xa0 = x.x;
  xa1 = x.y;
  xb0 = y.x;
  xb1 = y.y;
}

// FP8 latent rows: widen 16 E4M3 codes (one 16-byte chunk) times their tile
// scale to 16 bf16 values (two 16-byte chunks), rounding fl32(code * s) to
// nearest bf16; the tensor cores then see bf16 as for bf16 caches.
__device__ __forceinline__ void fp8x16_to_bf16x16(const uint4& raw, float s, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
  uint32_t o[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __half2_raw hr =
          __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>((w[q] >> (16 * h)) & 0xFFFFu), __NV_E4M3);
      float2 f = __half22float2(__half2(hr));
      f.x *= s;
      f.y *= s;
      const __nv_bfloat162 b = __float22bfloat162_rn(f);
      o[2 * q + h] = *reinterpret_cast<const uint32_t*>(&b);
    }
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

template <int D, int DC, bool FP8KV = false>
__global__ void __launch_bounds__(MlaCfg<D, DC>::THREADS, 1)
    sparse_mla_kernel(const void* __restrict__ kv_ptr, const __grid_constant__ CUtensorMap qmap,
                      const MlaParams p) {
  using C = MlaCfg<D, DC>;
  const __nv_bfloat16* kv = static_cast<const __nv_bfloat16*>(kv_ptr);
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled tiles need 1024-byte alignment; the dynamic window starts at
  // the same offset in every CTA, so either all CTAs leave here or none.
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) set_device_status(DSA_ERR_DEVICE_LAYOUT);
    return;
  }
  canary_set(smem, C::SMEM_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;             // [NST] gather producers -> MMA
  uint64_t* kv_empty = bars + C::NST;   // [NST] MMA (PV done) -> gather producers
  uint64_t* q_full = kv_empty + C::NST; // TMA (Q staged) -> softmax warps
  uint64_t* q_moved = q_full + 1;       // softmax warps (Q in TMEM) -> MMA, and the last stage -> gather
  uint64_t* s_full = q_moved + 1;       // MMA (S ready) -> softmax
  uint64_t* s_empty = s_full + 1;       // softmax (S read) -> MMA
  uint64_t* p_full = s_empty + 1;       // softmax (P written) -> MMA
  uint64_t* o_done = p_full + 1;        // MMA (PV done) -> softmax
  uint64_t* drain = o_done + 1;
  int32_t* misc = reinterpret_cast<int32_t*>(smem + C::OFF_MISC);  // [0] TMEM base, [1] abort
  volatile int* abort_flag = misc + 1;

  const int t = blockIdx.x;
  const int hb = blockIdx.y;
  const int h0 = hb * C::HB;
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
  const uint32_t q_stage = smem_u32(smem + C::OFF_KV + (C::NST - 1) * C::KV_BYTES);

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NST; ++i) {
      mbar_init(&kv_full[i], C::PRODUCERS * 32);  // one asynchronous arrival per producer thread
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_moved, 4);
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    mbar_init(p_full, 4);
    mbar_init(o_done, 1);
    mbar_init(drain, 1);
    misc[1] = 0;
    fence_mbar_init();
    prefetch_tensormap(&qmap);
  }
  if (warp == 12) {
    tmem_alloc(reinterpret_cast<uint32_t*>(misc), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = static_cast<uint32_t>(misc[0]);
  const uint32_t lo16 = 16u << 16;  // lane offset 16: S and Q (M = 64 layout)

  if (warp == 12 && lane == 0) {
    // the query block is an input of the call, not of the Top-K: load it now
    mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
    for (int c = 0; c < C::AKQ; ++c) tma_load_2d(q_stage + c * C::Q_ATOM, &qmap, c * 64, t * p.H + h0, q_full);
  }

  if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------ gather producers (8 warps)
    // Warp pw copies rows RPW pw .. RPW pw + RPW - 1 of each tile. Their
    // 16-byte chunks are numbered row-major (CPR per row) and issued 32 per
    // instruction, so most instructions move 512 contiguous bytes of one row.
    pdl_wait_prior();
    constexpr int CPR = C::DP / 8;                 // 16-byte chunks per stored row
    constexpr int ROUNDS = (C::RPW * CPR + 31) / 32;  // instructions per warp per tile
    const int pw = warp - 4;
    auto row_index = [&](int tile) -> int {
      const int k = k_begin + tile * C::TK + C::RPW * pw + lane;
      return (lane < C::RPW && tile < n_tiles && k < k_end) ? ld_dep(idx_row + k) : -1;
    };
    int nxt = row_index(0);
    bool ok = true;
    if constexpr (FP8KV) {
      // FP8 rows (KvFp8Row layout): every lane loads its 16-byte chunks of
      // the tile (codes with their tile scale, rope chunks) before waiting
      // for the stage, then widens them into the swizzled bf16 stage and
      // arrives once the stores are visible to the tensor cores.
      using R = KvFp8Row<DC, D - DC>;
      constexpr int CC = DC / 16;               // code chunks per row (16 codes each)
      constexpr int RC = (D - DC) / 8;          // rope chunks per row (8 bf16 each)
      constexpr int ZC = (C::DP - D) / 8;       // stored chunks past D (zero)
      constexpr int IPR = CC + RC + ZC;         // work items per row
      constexpr int RND = (C::RPW * IPR + 31) / 32;
      const uint8_t* kv8 = static_cast<const uint8_t*>(kv_ptr);
      for (int it = 0; it < n_tiles && ok; ++it) {
        const int sl = it % C::NST;
        const uint32_t use = static_cast<uint32_t>(it / C::NST);
        const int cur = nxt;
        const bool okr = cur >= 0 && cur < len;
        if (lane < C::RPW && cur != -1 && !okr) set_device_status(DSA_ERR_DEVICE_INDEX);
        const int mine = okr ? p.cm.row_checked(b, cur) : -1;  // cache row of this lane's key
        uint4 raw[RND];
        float sc[RND];
#pragma unroll
        for (int q = 0; q < RND; ++q) {
          const int item = q * 32 + lane;
          const int rl = item / IPR;
          const int c = item - rl * IPR;
          const int srow = __shfl_sync(0xffffffffu, mine, rl < C::RPW ? rl : 0);
          raw[q] = make_uint4(0u, 0u, 0u, 0u);
          sc[q] = 0.0f;
          if (item < C::RPW * IPR && srow >= 0 && c < CC + RC) {
            const uint8_t* rp = kv8 + static_cast<int64_t>(srow) * R::ROW_BYTES;
            if (c < CC) {
              raw[q] = __ldg(reinterpret_cast<const uint4*>(rp + 16 * c));
              sc[q] = __ldg(reinterpret_cast<const float*>(rp + R::SCALE_OFF) + (16 * c) / R::TILE);
            } else {
              raw[q] = __ldg(reinterpret_cast<const uint4*>(rp + R::ROPE_OFF + 16 * (c - CC)));
            }
          }
        }
        nxt = row_index(it + 1);
        if (it == C::NST - 1) ok = mbar_wait_warp(q_moved, 0, abort_flag);
        if (ok) ok = mbar_wait_warp(&kv_empty[sl], (use & 1u) ^ 1u, abort_flag);
        if (!ok) break;
        uint8_t* stage = smem + C::OFF_KV + sl * C::KV_BYTES;
#pragma unroll
        for (int q = 0; q < RND; ++q) {
          const int item = q * 32 + lane;
          const int rl = item / IPR;
          const int c = item - rl * IPR;
          if (item < C::RPW * IPR) {
            const int r = C::RPW * pw + rl;
            if (c < CC) {
              uint4 lo, hi;
              fp8x16_to_bf16x16(raw[q], sc[q], lo, hi);
              const int k0 = 2 * c, k1 = 2 * c + 1;  // bf16 chunks of dims 16c .. 16c + 15
              *reinterpret_cast<uint4*>(stage + (k0 >> 3) * C::ATOM_COL + sw128_offset(r, k0 & 7)) = lo;
              *reinterpret_cast<uint4*>(stage + (k1 >> 3) * C::ATOM_COL + sw128_offset(r, k1 & 7)) = hi;
            } else {
              const int k = c < CC + RC ? DC / 8 + (c - CC) : D / 8 + (c - CC - RC);
              *reinterpret_cast<uint4*>(stage + (k >> 3) * C::ATOM_COL + sw128_offset(r, k & 7)) = raw[q];
            }
          }
        }
        fence_proxy_async_smem();  // generic stores -> the tensor cores' reads
        mbar_arrive(&kv_full[sl]);
      }
    } else
    for (int it = 0; it < n_tiles && ok; ++it) {
      const int sl = it % C::NST;
      const uint32_t use = static_cast<uint32_t>(it / C::NST);
      const int cur = nxt;
      nxt = row_index(it + 1);  // in flight during the stage wait and the copies
      // the last stage holds Q until the softmax warps have moved it to TMEM
      if (it == C::NST - 1) ok = mbar_wait_warp(q_moved, 0, abort_flag);
      if (ok) ok = mbar_wait_warp(&kv_empty[sl], (use & 1u) ^ 1u, abort_flag);
      if (!ok) break;
      const bool okr = cur >= 0 && cur < len;
      if (lane < C::RPW && cur != -1 && !okr) set_device_status(DSA_ERR_DEVICE_INDEX);
      const int mine = okr ? p.cm.row_checked(b, cur) : -1;  // cache row of this lane's key
      const uint32_t stage = smem_u32(smem + C::OFF_KV + sl * C::KV_BYTES);
#pragma unroll 2
      for (int q = 0; q < ROUNDS; ++q) {
        const int flat = q * 32 + lane;                  // chunk number within the warp's rows
        const int rl = flat / CPR;                       // row of the warp (0..RPW-1)
        const int c = flat - rl * CPR;                   // 16-byte chunk of the row
        const int srow = __shfl_sync(0xffffffffu, mine, rl < C::RPW ? rl : 0);
        if (flat < C::RPW * CPR) {
          const int r = C::RPW * pw + rl;
          const bool has = srow >= 0 && c * 8 < D;
          const __nv_bfloat16* src = kv + static_cast<int64_t>(has ? srow : 0) * D + (has ? c * 8 : 0);
          cp_async_16(stage + (c >> 3) * C::ATOM_COL + sw128_offset(r, c & 7), has ? src : kv, has ? 16u : 0u);
        }
      }
      cp_async_arrive_noinc(&kv_full[sl]);
    }
    cp_async_wait_all();  // nothing may still be landing when the CTA retires
  } else if (warp == 12) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t p_base = smem_u32(smem + C::OFF_P);
      const uint32_t tmem_s = tmem_base + lo16 + C::COL_S;
      const uint32_t tmem_q = tmem_base + lo16 + C::COL_Q;
      auto issue_s = [&](int it) {
        const uint32_t kvb = smem_u32(smem + C::OFF_KV + (it % C::NST) * C::KV_BYTES);
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k) {
          const uint64_t bd = smem_desc_sw128(kvb + (k >> 2) * C::ATOM_COL + (k & 3) * 32, 16, 1024);
          umma_f16_ts(tmem_s, tmem_q + 8 * k, bd, C::IDESC_S, k > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
      };
      auto issue_pv = [&](int it) {
        const uint32_t kvb = smem_u32(smem + C::OFF_KV + (it % C::NST) * C::KV_BYTES);
#pragma unroll
        for (int nb = 0; nb < C::PV_MMAS; ++nb) {
#pragma unroll
          for (int kk = 0; kk < C::TK / 16; ++kk) {
            const uint64_t a = smem_desc_sw128(p_base + (kk >> 2) * (C::HB * 128) + (kk & 3) * 32, 16, 1024);
            // V = first DC dims of the gathered rows, MN-major: 64-dim atom columns
            // ATOM_COL bytes apart (LBO), 8-key row groups 1024 bytes apart (SBO).
            const uint64_t bd =
                smem_desc_sw128(kvb + (nb * (C::N_PV / 64)) * C::ATOM_COL + kk * 16 * 128, C::ATOM_COL, 1024);
            umma_f16(tmem_base + nb * C::N_PV, a, bd, C::IDESC_PV, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&kv_empty[it % C::NST]);
        umma_commit(o_done);
      };
      bool ok = mbar_wait(q_moved, 0, abort_flag);
      int s_next = 0, pv_next = 0;
      uint64_t t0 = globaltimer();
      // Issue whichever product is ready (non-blocking tests, so one barrier
      // never holds up another): S(j) needs tile j gathered and the softmax
      // done reading S(j-1) (one S buffer); PV(j) needs P(j).
      while (ok && pv_next < n_tiles) {
        bool progressed = false;
        if (s_next < n_tiles && (s_next == 0 || mbar_test(smem_u32(s_empty), (s_next - 1) & 1)) &&
            mbar_test(smem_u32(&kv_full[s_next % C::NST]), (s_next / C::NST) & 1)) {
          fence_proxy_async_smem();  // cp.async (generic proxy) data -> tensor core reads
          tc_fence_after();
          issue_s(s_next);
          ++s_next;
          progressed = true;
        }
        if (pv_next < s_next && mbar_test(smem_u32(p_full), pv_next & 1)) {
          tc_fence_after();
          issue_pv(pv_next);
          ++pv_next;
          progressed = true;
        }
        if (progressed) {
          t0 = globaltimer();
        } else if (*abort_flag) {
          ok = false;
        } else if (globaltimer() - t0 > wait_limit_ns()) {
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
  } else {
    // ------------------------------------------------------------ softmax + epilogue (warps 0..3)
    const int sw = warp;                                   // TMEM sub-partition
    const uint32_t lane_addr = static_cast<uint32_t>(sw * 32) << 16;
    // Rows this thread handles in the 16-lane layout: head rows ra, ra+8 of
    // the warp's 16 (h_local = sw*16 + row) and columns 8j + cc, +1.
    const int ra = lane >> 2;
    const int cc = 2 * (lane & 3);
    bool ok = mbar_wait_warp(q_full, 0, abort_flag);
    if (ok) {
      // Q -> TMEM (lanes 16..31 of this sub-partition, column COL_Q + c holds
      // dims 2c, 2c+1), in the 16x256b layout of rows ra, ra+8
      const int ha = sw * 16 + ra, hbr = ha + 8;
      constexpr int QCOLS = C::DP / 2;
#pragma unroll
      for (int g = 0; g < QCOLS / 64; ++g) {
        uint32_t v[32];
#pragma unroll
        for (int j = 0; j < 8; ++j)
          q_pair<C::Q_ATOM>(q_stage, ha, hbr, 64 * g + 8 * j + cc, v[4 * j], v[4 * j + 1], v[4 * j + 2],
                              v[4 * j + 3]);
        tmem_st16x256_x8(tmem_base + lane_addr + lo16 + C::COL_Q + 64 * g, v);
      }
      if constexpr (QCOLS % 64 == 32) {
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          q_pair<C::Q_ATOM>(q_stage, ha, hbr, (QCOLS / 64) * 64 + 8 * j + cc, v[4 * j], v[4 * j + 1],
                              v[4 * j + 2], v[4 * j + 3]);
        tmem_st16x256_x4(tmem_base + lane_addr + lo16 + C::COL_Q + (QCOLS / 64) * 64, v);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(q_moved);  // also on failure: every wait stays bounded
    pdl_wait_prior();  // the selected indices (Top-K output) are complete from here on

    float m_a = -INFINITY, m_b = -INFINITY;  // running max per row (log2 domain)
    float l_a = 0.0f, l_b = 0.0f;            // this thread's share of the running sums
    uint8_t* p_tile = smem + C::OFF_P;
    // indices of the next tile (for the validity mask), one tile ahead:
    // lane l holds keys l, 32 + l and (80-key tiles) 64 + l of the tile
    constexpr int REPS = C::TK / 8;   // 8-column repetitions of the 16x256b layout
    auto idx_at = [&](int k) -> int { return k < k_end ? ld_dep(idx_row + k) : -1; };
    int i0n = idx_at(k_begin + lane), i1n = idx_at(k_begin + 32 + lane);
    int i2n = (C::TK > 64 && lane < C::TK - 64) ? idx_at(k_begin + 64 + lane) : -1;
    for (int it = 0; it < n_tiles && ok; ++it) {
      const int i0 = i0n, i1 = i1n, i2 = i2n;
      if (it + 1 < n_tiles) {
        const int kn = k_begin + (it + 1) * C::TK;
        i0n = idx_at(kn + lane);
        i1n = idx_at(kn + 32 + lane);
        if (C::TK > 64) i2n = (lane < C::TK - 64) ? idx_at(kn + 64 + lane) : -1;
      }
      const unsigned v0 = __ballot_sync(0xffffffffu, i0 >= 0 && i0 < len);
      const unsigned v1 = __ballot_sync(0xffffffffu, i1 >= 0 && i1 < len);
      const unsigned v2 = __ballot_sync(0xffffffffu, i2 >= 0 && i2 < len);
      if (!(ok = mbar_wait_warp(s_full, it & 1, abort_flag))) break;
      tc_fence_after();
      float v[4 * REPS];
      {
        float* v8 = v;
        tmem_ld16x256_x8(tmem_base + lane_addr + lo16 + C::COL_S, *reinterpret_cast<float(*)[32]>(v8));
        if constexpr (REPS > 8)
          tmem_ld16x256_x2(tmem_base + lane_addr + lo16 + C::COL_S + 64, *reinterpret_cast<float(*)[8]>(v + 32));
      }
      tmem_wait_ld();
      // the S buffer is free again: the next QK^T may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      // v[4j + 0/1] = row ra, cols 8j+cc, +1; v[4j + 2/3] = row ra+8, same cols
      float ta = -INFINITY, tb = -INFINITY;
#pragma unroll
      for (int j = 0; j < REPS; ++j) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int col = 8 * j + cc + e;
          const unsigned vm = col < 32 ? v0 : col < 64 ? v1 : v2;
          const bool valid = (vm >> (col & 31)) & 1u;
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
        // O already holds earlier tiles: wait for PV(it-1), then rescale
        // rows ra, ra+8 (16-lane accesses touch O's lanes only)
        if (!(ok = mbar_wait_warp(o_done, (it - 1) & 1, abort_flag))) break;
        o_waited = true;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < DC; c += 64) {
          float o[32];
          tmem_ld16x256_x8(tmem_base + lane_addr + c, o);
          tmem_wait_ld();
          uint32_t w[32];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            w[4 * j + 0] = __float_as_uint(o[4 * j + 0] * fa);
            w[4 * j + 1] = __float_as_uint(o[4 * j + 1] * fa);
            w[4 * j + 2] = __float_as_uint(o[4 * j + 2] * fb);
            w[4 * j + 3] = __float_as_uint(o[4 * j + 3] * fb);
          }
          tmem_st16x256_x8(tmem_base + lane_addr + c, w);
        }
        tmem_wait_st();
      }
      // P = 2^(s - m) in bf16; the sums add the rounded values PV actually uses
      uint32_t pa[REPS], pb[REPS];
#pragma unroll
      for (int j = 0; j < REPS; ++j) {
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
        // P in 64-key atom columns (K-major, 128-byte swizzle): keys 8j..8j+7
        // are chunk j % 8 of atom column j / 8
        const int ha = sw * 16 + ra, hbr = ha + 8;
#pragma unroll
        for (int j = 0; j < REPS; ++j) {
          uint8_t* atom = p_tile + (j >> 3) * (C::HB * 128);
          *reinterpret_cast<uint32_t*>(atom + sw128_offset(ha, j & 7) + 2 * cc) = pa[j];
          *reinterpret_cast<uint32_t*>(atom + sw128_offset(hbr, j & 7) + 2 * cc) = pb[j];
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
    float m_h, l_h;
    {
      const int src = 4 * (lane & 7);
      const float xa = __shfl_sync(0xffffffffu, m_a, src), xb = __shfl_sync(0xffffffffu, m_b, src);
      const float ya = __shfl_sync(0xffffffffu, l_a, src), yb = __shfl_sync(0xffffffffu, l_b, src);
      m_h = ((lane & 15) < 8) ? xa : xb;
      l_h = ((lane & 15) < 8) ? ya : yb;
    }
    if (ok) ok = mbar_wait_warp(o_done, (n_tiles - 1) & 1, abort_flag);
    const bool o_row = lane < 16;               // lane r < 16 owns O row r
    const int h_local = sw * 16 + (lane & 15);
    const int h = h0 + h_local;
    if (ok) tc_fence_after();
    if (S == 1) {
      if (ok) {
        const bool writer = o_row && h < p.H;
        const float inv = (l_h > 0.0f) ? 1.0f / l_h : 0.0f;
        const int64_t row = static_cast<int64_t>(t) * p.H + h;
        for (int c = 0; c < DC; c += 16) {
          float o[16];
          tmem_ld16(tmem_base + lane_addr + c, o);
          tmem_wait_ld();
          if (writer) {
            uint32_t w8[8];
#pragma unroll
            for (int u = 0; u < 16; u += 2) {
              const __nv_bfloat162 o2 = __floats2bfloat162_rn(o[u] * inv, o[u + 1] * inv);
              w8[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
            }
            uint4* dst = reinterpret_cast<uint4*>(p.out + row * DC + c);
            dst[0] = make_uint4(w8[0], w8[1], w8[2], w8[3]);
            dst[1] = make_uint4(w8[4], w8[5], w8[6], w8[7]);
          }
        }
        if (writer && p.lse) p.lse[row] = (l_h > 0.0f) ? (m_h + log2f(l_h)) * 0.69314718055994531f : -INFINITY;
      }
    } else if (ok) {
      // this split's unnormalised rows and statistics -> workspace (L2). A
      // partial block is stored as [column / 4][head row][4 floats], so the
      // 16 rows of a warp write 256 contiguous bytes per store.
      const int64_t grp = (static_cast<int64_t>(t) * gridDim.y + hb) * S;
      float4* po = reinterpret_cast<float4*>(p.part_o + (grp + split) * C::HB * DC) + h_local;
#pragma unroll 1
      for (int c = 0; c < DC; c += 32) {
        float o[16], o2[16];
        tmem_ld16(tmem_base + lane_addr + c, o);
        tmem_ld16(tmem_base + lane_addr + c + 16, o2);
        tmem_wait_ld();
        if (o_row) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            po[(c / 4 + u) * C::HB] = make_float4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            po[(c / 4 + 4 + u) * C::HB] = make_float4(o2[4 * u], o2[4 * u + 1], o2[4 * u + 2], o2[4 * u + 3]);
        }
      }
      if (o_row) p.part_ml[(grp + split) * C::HB + h_local] = make_float2(m_h, l_h);
    }
  }

  // The next kernel of the stream (the next call's indexer) may be scheduled
  // now; it completes only after this grid (see the indexer's teardown).
  pdl_launch_dependents();

  if (S > 1) {
    // ---------------- merge the key-split partials through global memory
    // The cluster barrier (release/acquire at cluster scope) orders every
    // CTA's partial writes before any CTA reads them. Head h_local is
    // finalised by split h_local % S, the work spread over all threads.
    cluster_sync_all();
    const int64_t grp = (static_cast<int64_t>(t) * gridDim.y + hb) * S;
    constexpr int SL = 16;                     // columns per item
    constexpr int NSL = DC / SL;
    const int owned = (C::HB - split + S - 1) / S;  // heads split, split + S, ...
    // consecutive threads take consecutive owned heads of one slice, so the
    // [column / 4][head row] partial layout is read in 16-byte runs; splits
    // are folded in with a running maximum, so every load of an item is
    // issued before any of its arithmetic
    for (int item = threadIdx.x; item < owned * NSL; item += C::THREADS) {
      const int hl = split + S * (item % owned);
      const int c0 = (item / owned) * SL;
      const int h = h0 + hl;
      if (h >= p.H) continue;
      float Mx = -INFINITY, L = 0.0f;
      float acc[SL];
#pragma unroll
      for (int u = 0; u < SL; ++u) acc[u] = 0.0f;
      for (int sb = 0; sb < S; sb += 2) {
        float2 ml[2];
        float4 x[2][SL / 4];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (sb + u < S) {
            ml[u] = __ldcg(&p.part_ml[(grp + sb + u) * C::HB + hl]);
            const float4* po = reinterpret_cast<const float4*>(p.part_o + (grp + sb + u) * C::HB * DC) + hl;
#pragma unroll
            for (int v4 = 0; v4 < SL / 4; ++v4) x[u][v4] = __ldcg(po + (c0 / 4 + v4) * C::HB);
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          if (sb + u < S && ml[u].y > 0.0f) {
            const float nm = fmaxf(Mx, ml[u].x);
            const float fo = exp2f(Mx - nm);       // 0 while nothing is accumulated (Mx = -inf)
            const float fn = exp2f(ml[u].x - nm);
            L = L * fo + ml[u].y * fn;
#pragma unroll
            for (int v4 = 0; v4 < SL / 4; ++v4) {
              acc[4 * v4 + 0] = acc[4 * v4 + 0] * fo + x[u][v4].x * fn;
              acc[4 * v4 + 1] = acc[4 * v4 + 1] * fo + x[u][v4].y * fn;
              acc[4 * v4 + 2] = acc[4 * v4 + 2] * fo + x[u][v4].z * fn;
              acc[4 * v4 + 3] = acc[4 * v4 + 3] * fo + x[u][v4].w * fn;
            }
            Mx = nm;
          }
        }
      }
      const float inv = (L > 0.0f) ? 1.0f / L : 0.0f;
      const int64_t row = static_cast<int64_t>(t) * p.H + h;
      uint32_t w[SL / 2];
#pragma unroll
      for (int u = 0; u < SL; u += 2) {
        const __nv_bfloat162 o2 = __floats2bfloat162_rn(acc[u] * inv, acc[u + 1] * inv);
        w[u / 2] = *reinterpret_cast<const uint32_t*>(&o2);
      }
      uint4* dst = reinterpret_cast<uint4*>(p.out + row * DC + c0);
#pragma unroll
      for (int u = 0; u < SL / 8; ++u) dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      if (c0 == 0 && p.lse) p.lse[row] = (L > 0.0f) ? (Mx + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
  canary_check(smem, C::SMEM_BYTES);
}

}  // namespace dsa
