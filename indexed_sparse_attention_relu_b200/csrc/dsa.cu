// dsa.cu -- host side of libdsa.so: argument validation, workspace planning,
// tensor-map encoding and kernel launches for the DSA hot path (the C ABI of
// include/dsa.h). All kernels live in this translation unit so they share the
// device status word.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "dsa_common.cuh"
#include "indexer.cuh"
#include "indexer_decode.cuh"
#include "quant.cuh"
#include "sparse_mla.cuh"
#include "sparse_mla_pipe.cuh"
#include "topk.cuh"

namespace {

using namespace dsa;

thread_local char g_last_error[512] = "";

dsa_status fail(dsa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return s;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

dsa_status check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return DSA_OK;
}

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2-D map over the index-key cache: x = element within a key, y = key row.
// Boxes of 128 key rows (one tile), or 64 for paged caches (a tile is then
// two boxes, each inside one page).
dsa_status make_key_map(CUtensorMap* map, const void* base, int64_t rows, int din, bool fp8, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(din), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(din) * (fp8 ? 1u : 2u)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r;
  if (fp8) {
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(din), static_cast<cuuint32_t>(box_rows)};
    r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};  // one 128-byte swizzle atom column
    r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// 2-D bf16 map with a 128-byte swizzle: x = element within a row (box 64),
// y = row (box box_rows; 1 for tile::gather4 row gathers).
dsa_status make_bf16_rows_map(CUtensorMap* map, const void* base, int64_t rows, int cols, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2u};
  const cuuint32_t estr[2] = {1, 1};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled (rows) failed (%d)", static_cast<int>(r));
  return DSA_OK;
}

// ---------------------------------------------------------------- validation
dsa_status check_batch(const dsa_batch* bt) {
  if (!bt) return fail(DSA_ERR_INVALID_ARGUMENT, "batch is NULL");
  if (bt->batch <= 0 || bt->num_q < 0 || bt->max_seq_len <= 0)
    return fail(DSA_ERR_INVALID_ARGUMENT, "batch=%d num_q=%d max_seq_len=%d must be positive", bt->batch,
                bt->num_q, bt->max_seq_len);
  if (bt->num_q > 0 && (!bt->cu_q || !bt->q_pos || !bt->seq_lens))
    return fail(DSA_ERR_INVALID_ARGUMENT, "cu_q, q_pos and seq_lens must be non-NULL");
  if (static_cast<int64_t>(bt->batch) * bt->max_seq_len >= (int64_t(1) << 31))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "batch * max_seq_len must be < 2^31");
  if (!bt->block_table) {
    if (bt->page_size != 0 || bt->num_pages != 0)
      return fail(DSA_ERR_INVALID_ARGUMENT, "page_size and num_pages must be 0 without a block table");
    return DSA_OK;
  }
  if (bt->page_size <= 0 || bt->page_size % 64 != 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "page_size %d must be a positive multiple of 64", bt->page_size);
  if (bt->num_pages <= 0) return fail(DSA_ERR_INVALID_ARGUMENT, "num_pages %d must be positive", bt->num_pages);
  if (static_cast<int64_t>(bt->num_pages) * bt->page_size >= (int64_t(1) << 31))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "num_pages * page_size must be < 2^31");
  if (reinterpret_cast<uintptr_t>(bt->block_table) & 3u)
    return fail(DSA_ERR_MISALIGNED, "block_table must be 4-byte aligned");
  return DSA_OK;
}

// Rows of every cache: B * L_max (contiguous) or the page pool.
int64_t cache_rows(const dsa_batch* bt) {
  return bt->block_table ? static_cast<int64_t>(bt->num_pages) * bt->page_size
                         : static_cast<int64_t>(bt->batch) * bt->max_seq_len;
}

CacheMap cache_map(const dsa_batch* bt) {
  CacheMap m;
  m.table = bt->block_table;
  m.L_max = bt->max_seq_len;
  m.page_size = bt->block_table ? bt->page_size : 0;
  m.max_pages = bt->block_table ? (bt->max_seq_len + bt->page_size - 1) / bt->page_size : 0;
  m.num_pages = bt->block_table ? bt->num_pages : 0;
  return m;
}

int key_box_rows(const dsa_batch* bt) { return bt->block_table ? 64 : 128; }

dsa_status check_indexer(const dsa_batch* bt, const dsa_indexer_in* in) {
  if (!in) return fail(DSA_ERR_INVALID_ARGUMENT, "indexer input is NULL");
  const bool shape_ok = (in->n_heads == 64 && in->head_dim == 128) || (in->n_heads == 64 && in->head_dim == 32) ||
                        (in->n_heads == 4 && in->head_dim == 32) || (in->n_heads == 4 && in->head_dim == 128);
  if (!shape_ok)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "indexer heads/dim %d/%d not in {4,64} x {32,128}", in->n_heads,
                in->head_dim);
  if (in->key_dtype != DSA_KEY_BF16 && in->key_dtype != DSA_KEY_FP8_E4M3 && in->key_dtype != DSA_KEY_MXFP8)
    return fail(DSA_ERR_INVALID_ARGUMENT, "bad key dtype %d", static_cast<int>(in->key_dtype));
  if (!in->q || !in->w || !in->k_cache) return fail(DSA_ERR_INVALID_ARGUMENT, "indexer q, w, k_cache must be non-NULL");
  if (!aligned16(in->q) || !aligned16(in->w) || !aligned16(in->k_cache))
    return fail(DSA_ERR_MISALIGNED, "indexer q, w, k_cache must be 16-byte aligned");
  if (in->key_dtype == DSA_KEY_FP8_E4M3) {
    if (!in->k_scale) return fail(DSA_ERR_INVALID_ARGUMENT, "FP8 keys need k_scale");
    if (in->scale_group != in->head_dim)
      return fail(DSA_ERR_UNSUPPORTED_SHAPE, "FP8 indexer needs one scale per key (scale_group == head_dim)");
  }
  if (in->key_dtype == DSA_KEY_MXFP8) {
    if (!in->q_scale_e8m0 || !in->k_scale_e8m0)
      return fail(DSA_ERR_INVALID_ARGUMENT, "MXFP8 needs q_scale_e8m0 and k_scale_e8m0");
    if (in->scale_group != 32) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "MXFP8 needs scale_group == 32");
    if (!aligned16(in->q_scale_e8m0)) return fail(DSA_ERR_MISALIGNED, "q_scale_e8m0 must be 16-byte aligned");
  }
  (void)bt;
  return DSA_OK;
}

dsa_status check_mla(const dsa_mla_in* in) {
  if (!in) return fail(DSA_ERR_INVALID_ARGUMENT, "MLA input is NULL");
  const bool dims_ok = (in->d_latent == 512 && in->d_rope == 64) || (in->d_latent == 64 && in->d_rope == 16);
  if (!dims_ok)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "MLA dims (%d,%d) not in {(512,64),(64,16)}", in->d_latent, in->d_rope);
  if (in->n_heads < 1 || in->n_heads > 128 || (in->n_heads > 64 && in->n_heads % 64 != 0))
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "MLA heads %d must be <= 64 or a multiple of 64 up to 128", in->n_heads);
  if (!in->q || !in->kv) return fail(DSA_ERR_INVALID_ARGUMENT, "MLA q and kv must be non-NULL");
  if (!aligned16(in->q) || !aligned16(in->kv)) return fail(DSA_ERR_MISALIGNED, "MLA q and kv must be 16-byte aligned");
  if (!std::isfinite(in->softmax_scale)) return fail(DSA_ERR_INVALID_ARGUMENT, "softmax_scale must be finite");
  if (in->kv_dtype != DSA_KV_BF16 && in->kv_dtype != DSA_KV_FP8_E4M3)
    return fail(DSA_ERR_INVALID_ARGUMENT, "bad kv dtype %d", static_cast<int>(in->kv_dtype));
  return DSA_OK;
}

// ---------------------------------------------------------------- planning
int indexer_group(const dsa_batch* bt) { return bt->num_q > bt->batch ? 4 : 1; }

struct MlaPlan {
  int splits;
  int keys_per_split;
};

// Key splits per (token, head block): enough CTAs to fill the SMs in one
// wave, at most 8 (the splits of one (token, head block) form a cluster; each
// leaves its partial rows in the workspace, in L2, and they merge after the
// cluster barrier).
MlaPlan mla_plan(int T, int HB, int K, int sms, int tk = 64) {
  const int tiles = (K + tk - 1) / tk;
  const int base = T * HB;
  int splits = base >= sms ? 1 : sms / base;
  if (splits > 8) splits = 8;
  if (splits > tiles) splits = tiles;
  if (splits < 1) splits = 1;
  const int tps = (tiles + splits - 1) / splits;
  splits = (tiles + tps - 1) / tps;
  return MlaPlan{splits, tps * tk};
}

// Workspace of the attention: with key splits, every split CTA leaves its
// unnormalised O rows (64 x d_latent fp32) and per-row (max, sum) in global
// memory for the merge. Sized for the largest supported latent dim.
constexpr int kMlaMaxLatent = 512;

size_t mla_part_bytes(int T, int hb, int splits, int dc) {
  if (splits <= 1) return 0;
  const size_t rows = static_cast<size_t>(T) * hb * splits * 64;
  return align256(rows * dc * sizeof(float)) + align256(rows * sizeof(float2));
}

// How many clusters of `size` pipeline CTAs the device holds at once (a
// cluster must fit inside one GPC, so this is below sms / size when the GPCs
// do not divide evenly). Queried once per size; `fallback` when the query
// is unavailable.
int pipe_max_clusters(int size, int fallback);

// The two-CTA pipeline for 128 heads (one score CTA and one value CTA per
// pair; the pairs of one query form one cluster of 2 x splits CTAs). The
// time of a launch is about (waves of clusters) x (key tiles per split), so
// take the split count, at most PipeCfg::MAX_SPLITS, that minimises that
// product, the fewer splits on ties (less merging). `max_clusters(s)` is the
// number of clusters of 2s CTAs resident at once.
template <typename MaxClusters>
MlaPlan pipe_plan_with(int T, int K, MaxClusters max_clusters) {
  using C = PipeCfg;
  const int tiles = (K + C::TK - 1) / C::TK;
  int best = 1;
  int64_t best_cost = -1;
  for (int sp = 1; sp <= C::MAX_SPLITS && sp <= tiles; sp *= 2) {  // 1, 2, 4: a split owns 128 / S rows
    if ((sp - 1) * ((tiles + sp - 1) / sp) >= tiles) continue;     // the last split would get no tile
    const int mc = max_clusters(sp);
    if (mc < 1) break;
    const int64_t waves = (static_cast<int64_t>(T) + mc - 1) / mc;
    const int64_t cost = waves * ((tiles + sp - 1) / sp);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = sp;
    }
  }
  const int tps = (tiles + best - 1) / best;
  return MlaPlan{best, tps * C::TK};  // the last split may get fewer tiles (never none: best <= tiles)
}

MlaPlan pipe_plan(int T, int K, int sms) {
  return pipe_plan_with(T, K, [sms](int sp) { return pipe_max_clusters(2 * sp, sms / (2 * sp)); });
}

// Workspace of the pipeline: the P rings and final row statistics (one per
// SM a score CTA can run on), then the split partials (128 rows per pair).
size_t pipe_ring_bytes() {
  using C = PipeCfg;
  return align256(static_cast<size_t>(C::RING_SMS) * C::NP * C::SLOT_BYTES) +
         align256(static_cast<size_t>(C::RING_SMS) * C::M * sizeof(float2));
}

size_t pipe_ws_bytes(int T, int splits) {
  size_t b = pipe_ring_bytes();
  if (splits > 1) {
    const size_t rows = static_cast<size_t>(T) * splits * PipeCfg::M;
    b += align256(rows * PipeCfg::DC * sizeof(float)) + align256(rows * sizeof(float2));
  }
  return b;
}

// Upper bound over the kernels a call can use: the 64-head kernel with 1 or
// 2 head blocks, and the two-CTA pipeline.
size_t mla_ws_bytes(const dsa_batch* bt, int k) {
  const int T = bt->num_q;
  size_t need = 0;
  for (int hb = 1; hb <= 2; ++hb) {
    const MlaPlan pl = mla_plan(T, hb, k, num_sms());
    const size_t b = mla_part_bytes(T, hb, pl.splits, kMlaMaxLatent);
    need = b > need ? b : need;
  }
  const size_t bp = pipe_ws_bytes(T, pipe_plan(T, k, num_sms()).splits);
  return bp > need ? bp : need;
}

// ---------------------------------------------------------------- debug build
#ifdef DSA_DEBUG
// Host check of every index the attention is about to gather: copies the
// indices and the batch metadata to the host (synchronising the stream) and
// requires each to be -1 or a position inside its sequence.
dsa_status debug_check_indices(const dsa_batch* bt, const int32_t* idx, int k, cudaStream_t st) {
  const int T = bt->num_q, B = bt->batch;
  std::vector<int32_t> h_idx(static_cast<size_t>(T) * k), cu(B + 1), lens(B);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e == cudaSuccess) e = cudaMemcpy(h_idx.data(), idx, h_idx.size() * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(cu.data(), bt->cu_q, cu.size() * 4, cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(lens.data(), bt->seq_lens, lens.size() * 4, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "DSA_DEBUG index check: %s", cudaGetErrorString(e));
  int b = 0;
  for (int t = 0; t < T; ++t) {
    while (b + 1 < B && cu[b + 1] <= t) ++b;
    const int len = lens[b] < bt->max_seq_len ? lens[b] : bt->max_seq_len;
    for (int i = 0; i < k; ++i) {
      const int v = h_idx[static_cast<size_t>(t) * k + i];
      if (v != -1 && (v < 0 || v >= len))
        return fail(DSA_ERR_INVALID_ARGUMENT, "DSA_DEBUG: idx[%d][%d] = %d outside [-1, %d)", t, i, v, len);
    }
  }
  return DSA_OK;
}
#endif

// ---------------------------------------------------------------- launches
// Dynamic shared memory of a tensor-core kernel: its layout, plus (DSA_DEBUG)
// the canary after it.
int smem_request(int layout_bytes) { return kCanaryBytes ? canary_offset(layout_bytes) + kCanaryBytes : layout_bytes; }

template <typename Kern>
dsa_status set_smem(Kern k, int bytes) {
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  return DSA_OK;
}

// Key format of a call (the kernels' KF template argument).
int key_format(const dsa_indexer_in* in) {
  return in->key_dtype == DSA_KEY_MXFP8 ? KF_MX : in->key_dtype == DSA_KEY_FP8_E4M3 ? KF_FP8 : KF_BF16;
}

// Scale rows of 8-bit keys start on 16-byte boundaries at every tile (128
// rows, or 64 when paged) when the base is aligned and, for contiguous
// caches, L_max times the row's scale bytes is a multiple of 16.
bool scale_rows_aligned(const dsa_batch* bt, const void* base, int row_bytes) {
  return base && aligned16(base) && (bt->block_table || (static_cast<int64_t>(bt->max_seq_len) * row_bytes) % 16 == 0);
}

template <int HI, int DIN, int G, int KF>
dsa_status launch_indexer_t(const dsa_batch* bt, const dsa_indexer_in* in, float* scores, int64_t ld,
                            cudaStream_t st, bool pdl) {
  using C = IndexerCfg<HI, DIN, G, KF>;
  constexpr bool FP8 = C::FP8;
  CUtensorMap map;
  dsa_status s = make_key_map(&map, in->k_cache, cache_rows(bt), DIN, FP8, key_box_rows(bt));
  if (s != DSA_OK) return s;
  auto kern = indexer_scores_kernel<HI, DIN, G, KF>;
  if ((s = set_smem(kern, smem_request(C::SMEM_BYTES))) != DSA_OK) return s;
  const int sms = num_sms();
  const int64_t groups64 = static_cast<int64_t>((bt->num_q + G - 1) / G) + bt->batch;
  const int groups = static_cast<int>(groups64 < bt->num_q ? groups64 : bt->num_q);
  const int max_tiles = (bt->max_seq_len + 127) / 128;
  // Key tiles per CTA: split each group's key range so the grid fills the
  // resident CTA slots (C::MIN_CTAS per SM) about once; at least 2 tiles so
  // the prologue stays amortised, at most 64 (ragged / causal rows then
  // spread over several CTAs and the hardware scheduler balances them).
  const int slots = sms * C::MIN_CTAS;
  int per_group = slots / (groups > 0 ? groups : 1);
  if (per_group < 1) per_group = 1;
  int tpc = (max_tiles + per_group - 1) / per_group;
  if (tpc < 2) tpc = 2;
  if (tpc > 64) tpc = 64;
  // Single-token groups (decode): at most 16 tiles per CTA, so a ragged batch
  // (most sequences shorter than the longest, whose length sets max_tiles)
  // spreads its work over many short CTAs that the scheduler balances.
  if (G == 1 && tpc > 16) tpc = 16;
  const int gy = (max_tiles + tpc - 1) / tpc;
  IndexerParams p;
  p.cu_q = bt->cu_q;
  p.q_pos = bt->q_pos;
  p.seq_lens = bt->seq_lens;
  p.B = bt->batch;
  p.L_max = bt->max_seq_len;
  p.cm = cache_map(bt);
  p.q = static_cast<const __nv_bfloat16*>(in->q);
  p.w = in->w;
  p.k_scale = KF == KF_FP8 ? in->k_scale : nullptr;
  p.k_mx = KF == KF_MX ? in->k_scale_e8m0 : nullptr;
  p.scale_bulk = KF == KF_MX && scale_rows_aligned(bt, in->k_scale_e8m0, DIN / 32);
  p.rows = cache_rows(bt);
  p.scores = scores;
  p.ld = ld;
  p.tiles_per_cta = tpc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(groups, gy);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem_request(C::SMEM_BYTES);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, map, p);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "indexer launch: %s", cudaGetErrorString(e));
  return check_launch("indexer_scores");
}

// One query token per group (decode): one CTA per SM, each taking an equal
// range of the flattened key-tile list of all tokens.
template <int HI, int DIN, int KF>
dsa_status launch_indexer_decode(const dsa_batch* bt, const dsa_indexer_in* in, float* scores, int64_t ld,
                                 cudaStream_t st, bool pdl) {
  using C = IdxDecCfg<HI, DIN, KF>;
  constexpr bool FP8 = C::FP8;
  CUtensorMap kmap, qmap;
  dsa_status s = make_key_map(&kmap, in->k_cache, cache_rows(bt), DIN, FP8, key_box_rows(bt));
  if (s != DSA_OK) return s;
  if ((s = make_bf16_rows_map(&qmap, in->q, static_cast<int64_t>(bt->num_q) * HI, DIN, HI)) != DSA_OK) return s;
  auto kern = indexer_decode_kernel<HI, DIN, KF>;
  if ((s = set_smem(kern, smem_request(C::SMEM_BYTES))) != DSA_OK) return s;
  IdxDecParams p;
  p.cu_q = bt->cu_q;
  p.q_pos = bt->q_pos;
  p.seq_lens = bt->seq_lens;
  p.k_scale = KF == KF_FP8 ? in->k_scale : nullptr;
  p.k_mx = KF == KF_MX ? in->k_scale_e8m0 : nullptr;
  // the scales ride in the key stage when every tile's scale rows start on a
  // 16-byte boundary
  p.scale_bulk = FP8 && scale_rows_aligned(bt, KF == KF_MX ? static_cast<const void*>(in->k_scale_e8m0)
                                                           : static_cast<const void*>(in->k_scale), C::SROW);
  p.rows = cache_rows(bt);
  p.B = bt->batch;
  p.T = bt->num_q;
  p.L_max = bt->max_seq_len;
  p.cm = cache_map(bt);
  p.scores = scores;
  p.ld = ld;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(num_sms());
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem_request(C::SMEM_BYTES);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, kmap, qmap, in->w, p);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "indexer (decode) launch: %s", cudaGetErrorString(e));
  return check_launch("indexer_scores (decode)");
}

template <int HI, int DIN>
dsa_status launch_indexer_g(const dsa_batch* bt, const dsa_indexer_in* in, float* scores, int64_t ld,
                            cudaStream_t st, bool pdl) {
  const int kf = key_format(in);
  // decode (one token per group): the balanced one-CTA-per-SM kernel while a
  // CTA's segment list (at most one entry per token) fits
  if (indexer_group(bt) == 1 && bt->num_q <= IdxDecCfg<HI, DIN, KF_BF16>::MAXSEG) {
    if (kf == KF_MX) return launch_indexer_decode<HI, DIN, KF_MX>(bt, in, scores, ld, st, pdl);
    if (kf == KF_FP8) return launch_indexer_decode<HI, DIN, KF_FP8>(bt, in, scores, ld, st, pdl);
    return launch_indexer_decode<HI, DIN, KF_BF16>(bt, in, scores, ld, st, pdl);
  }
  if (indexer_group(bt) == 4) {
    if (kf == KF_MX) return launch_indexer_t<HI, DIN, 4, KF_MX>(bt, in, scores, ld, st, pdl);
    if (kf == KF_FP8) return launch_indexer_t<HI, DIN, 4, KF_FP8>(bt, in, scores, ld, st, pdl);
    return launch_indexer_t<HI, DIN, 4, KF_BF16>(bt, in, scores, ld, st, pdl);
  }
  if (kf == KF_MX) return launch_indexer_t<HI, DIN, 1, KF_MX>(bt, in, scores, ld, st, pdl);
  if (kf == KF_FP8) return launch_indexer_t<HI, DIN, 1, KF_FP8>(bt, in, scores, ld, st, pdl);
  return launch_indexer_t<HI, DIN, 1, KF_BF16>(bt, in, scores, ld, st, pdl);
}

// pdl: launch with programmatic stream serialization, so the prologue may
// overlap the tail of the previous kernel in the stream (the kernel itself
// still completes only after that kernel, see its teardown).
// Bytes of the widened (bf16) MXFP8 queries in a workspace.
size_t mx_q_bytes(int T, int h_i, int d_i) { return align256(static_cast<size_t>(T) * h_i * d_i * 2); }

// q_ws: MXFP8 calls only, mx_q_bytes() of 16-byte aligned workspace that
// receives the widened queries (exact in bf16) before the scoring kernel.
dsa_status launch_indexer(const dsa_batch* bt, const dsa_indexer_in* in_, float* scores, int64_t ld,
                          cudaStream_t st, bool pdl = false, void* q_ws = nullptr) {
  dsa_indexer_in local = *in_;
  const dsa_indexer_in* in = &local;
  if (in_->key_dtype == DSA_KEY_MXFP8) {
    const int64_t n = static_cast<int64_t>(bt->num_q) * in_->n_heads * in_->head_dim;
    const int64_t blocks64 = (n / 4 + 255) / 256;
    const int blocks = static_cast<int>(blocks64 < num_sms() * 32 ? blocks64 : num_sms() * 32);
    mx_dequantize_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint8_t*>(in_->q), in_->q_scale_e8m0, n,
                                                 static_cast<__nv_bfloat16*>(q_ws));
    dsa_status s = check_launch("mx_dequantize (queries)");
    if (s != DSA_OK) return s;
    local.q = q_ws;
    pdl = false;  // the scoring kernel reads the queries that kernel writes
  }
  if (in->n_heads == 64 && in->head_dim == 128) return launch_indexer_g<64, 128>(bt, in, scores, ld, st, pdl);
  if (in->n_heads == 64 && in->head_dim == 32) return launch_indexer_g<64, 32>(bt, in, scores, ld, st, pdl);
  if (in->n_heads == 4 && in->head_dim == 128) return launch_indexer_g<4, 128>(bt, in, scores, ld, st, pdl);
  return launch_indexer_g<4, 32>(bt, in, scores, ld, st, pdl);
}

constexpr int kTopkThreads = 512;
constexpr int kTopkCacheMax = 49152;  // keys (192 KB)

template <typename Kern>
dsa_status launch_topk_kernel(Kern kern, int threads, int smem, const TopkParams& p, int rows, cudaStream_t st,
                              bool pdl) {
  dsa_status s = set_smem(kern, smem);
  if (s != DSA_OK) return s;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "topk launch: %s", cudaGetErrorString(e));
  return check_launch("topk");
}

dsa_status launch_topk(const dsa_batch* bt, const float* scores, int64_t ld, int k, int32_t* idx, cudaStream_t st,
                       bool pdl = false) {
  TopkParams p;
  p.scores = scores;
  p.ld = ld;
  p.cu_q = bt->cu_q;
  p.q_pos = bt->q_pos;
  p.seq_lens = bt->seq_lens;
  p.B = bt->batch;
  p.L_max = bt->max_seq_len;
  p.K = k;
  p.idx = idx;
  p.bm_words = 0;
  const int L = bt->max_seq_len;
  // short rows: one read of the row into registers (8 or 16 keys a thread)
  if (L <= 1024 * 8) return launch_topk_kernel(topk_reg_kernel<1024, 8>, 1024, 0, p, bt->num_q, st, pdl);
  if (L <= 1024 * 16) return launch_topk_kernel(topk_reg_kernel<1024, 16>, 1024, 0, p, bt->num_q, st, pdl);
  // two streaming passes with position bitmaps in shared memory: the bitmaps
  // and first-digit histogram are fixed; the candidate list of the threshold
  // bin gets a quarter of a row (at least 2048, at most 16384 slots) within
  // the shared-memory budget (a longer list streams the row instead)
  {
    const int bm_words = ((L + 31) / 32 + 1) & ~1;
    const int fixed = 4 * 2048 * 4 + 2 * bm_words * 4;
    const int budget = 232448 - 6144 - fixed;  // static shared memory of the kernel included
    int cap = L / 4;
    if (cap < 2048) cap = 2048;
    if (cap > 16384) cap = 16384;
    if (cap * 8 > budget) cap = budget / 8;
    if (cap >= 1024) {
      p.bm_words = bm_words;
      p.cache_cap = cap;
      return launch_topk_kernel(topk_bitmap_kernel<1024>, 1024, fixed + cap * 8, p, bt->num_q, st, pdl);
    }
  }
  // longer rows: multi-pass select streaming the row from L2 / HBM
  const int cap = L < kTopkCacheMax ? L : kTopkCacheMax;
  p.cache_cap = cap;
  return launch_topk_kernel(topk_kernel<kTopkThreads>, kTopkThreads, cap * 4, p, bt->num_q, st, pdl);
}

template <int D, int DC, bool FP8KV = false>
dsa_status launch_mla_t(const dsa_batch* bt, const dsa_mla_in* in, const int32_t* idx, int k, void* out,
                        float* lse, void* ws, size_t ws_bytes, cudaStream_t st, const MlaPlan& pl, bool pdl) {
  using C = MlaCfg<D, DC>;
  auto kern = sparse_mla_kernel<D, DC, FP8KV>;
  dsa_status s = set_smem(kern, smem_request(C::SMEM_BYTES));
  if (s != DSA_OK) return s;
  const int T = bt->num_q, H = in->n_heads;
  CUtensorMap qmap;
  if ((s = make_bf16_rows_map(&qmap, in->q, static_cast<int64_t>(T) * H, D, 64)) != DSA_OK) return s;
  MlaParams p;
  p.cu_q = bt->cu_q;
  p.seq_lens = bt->seq_lens;
  p.B = bt->batch;
  p.L_max = bt->max_seq_len;
  p.cm = cache_map(bt);
  p.T = T;
  p.H = H;
  p.K = k;
  p.idx = idx;
  p.scale_log2 = in->softmax_scale * 1.4426950408889634f;
  p.keys_per_split = pl.keys_per_split;
  p.splits = pl.splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  const int hb = (H + 63) / 64;
  p.part_o = nullptr;
  p.part_ml = nullptr;
  if (pl.splits > 1) {
    const size_t need = mla_part_bytes(T, hb, pl.splits, DC);
    if (!ws || ws_bytes < need)
      return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "attention workspace %zu < %zu bytes", ws_bytes, need);
    if (!aligned16(ws)) return fail(DSA_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    const size_t rows = static_cast<size_t>(T) * hb * pl.splits * 64;
    p.part_o = static_cast<float*>(ws);
    p.part_ml = reinterpret_cast<float2*>(static_cast<uint8_t*>(ws) + align256(rows * DC * sizeof(float)));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(T, hb, pl.splits);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem_request(C::SMEM_BYTES);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pl.splits > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = pl.splits;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, in->kv, qmap, p);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "sparse_mla launch: %s", cudaGetErrorString(e));
  return check_launch("sparse_mla");
}

int pipe_max_clusters(int size, int fallback) {
  static std::mutex mu;
  static int cache[2 * PipeCfg::MAX_SPLITS + 1] = {};
  if (size < 1 || size > 2 * PipeCfg::MAX_SPLITS) return fallback;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[size] == 0) {
    int n = 0;
    // (no error message is recorded here: a size query may run without a device)
    if (cudaFuncSetAttribute(sparse_mla_pipe_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_request(PipeCfg::SMEM_BYTES)) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(size, 1, 1);
      cfg.blockDim = dim3(PipeCfg::THREADS);
      cfg.dynamicSmemBytes = smem_request(PipeCfg::SMEM_BYTES);
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = size;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, sparse_mla_pipe_kernel<false>, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();  // clear a failed query's error state
    cache[size] = n > 0 ? n : -1;
  }
  return cache[size] > 0 ? cache[size] : fallback;
}

dsa_status launch_mla_pipe(const dsa_batch* bt, const dsa_mla_in* in, const int32_t* idx, int k, void* out,
                           float* lse, void* ws, size_t ws_bytes, cudaStream_t st, bool pdl) {
  using C = PipeCfg;
  auto kern = bt->block_table ? sparse_mla_pipe_kernel<true> : sparse_mla_pipe_kernel<false>;
  dsa_status s = set_smem(kern, smem_request(C::SMEM_BYTES));
  if (s != DSA_OK) return s;
  const int T = bt->num_q;
  const MlaPlan pl = pipe_plan(T, k, num_sms());
  const size_t need = pipe_ws_bytes(T, pl.splits);
  if (!ws || ws_bytes < need)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "attention workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned16(ws)) return fail(DSA_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  CUtensorMap qmap, kvmap;
  if ((s = make_bf16_rows_map(&qmap, in->q, static_cast<int64_t>(T) * C::M, C::D, C::M)) != DSA_OK) return s;
  if ((s = make_bf16_rows_map(&kvmap, in->kv, cache_rows(bt), C::D, 1)) != DSA_OK)
    return s;
  PipeParams p;
  p.cu_q = bt->cu_q;
  p.seq_lens = bt->seq_lens;
  p.B = bt->batch;
  p.L_max = bt->max_seq_len;
  p.cm = cache_map(bt);
  p.T = T;
  p.K = k;
  p.idx = idx;
  p.scale_log2 = in->softmax_scale * 1.4426950408889634f;
  p.keys_per_split = pl.keys_per_split;
  p.splits = pl.splits;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  uint8_t* w = static_cast<uint8_t*>(ws);
  p.ring = w;
  w += align256(static_cast<size_t>(C::RING_SMS) * C::NP * C::SLOT_BYTES);
  p.fin = reinterpret_cast<float2*>(w);
  w += align256(static_cast<size_t>(C::RING_SMS) * C::M * sizeof(float2));
  p.part_o = nullptr;
  p.part_ml = nullptr;
  if (pl.splits > 1) {
    const size_t rows = static_cast<size_t>(T) * pl.splits * C::M;
    p.part_o = reinterpret_cast<float*>(w);
    p.part_ml = reinterpret_cast<float2*>(w + align256(rows * C::DC * sizeof(float)));
  }
  // the split partials as a 2-D fp32 tensor: x = head row x 4 (512 floats, a
  // [row][4] block per 4 output columns), y = (pair, column / 4)
  CUtensorMap pmap;
  std::memset(&pmap, 0, sizeof(pmap));
  if (pl.splits > 1) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C::M) * 4,
                                static_cast<cuuint64_t>(T) * pl.splits * (C::DC / 4)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C::M) * 4 * sizeof(float)};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(C::M / pl.splits * 4), static_cast<cuuint32_t>(C::DC / 4)};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(&pmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.part_o, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DSA_ERR_CUDA, "cuTensorMapEncodeTiled (partials) failed (%d)", static_cast<int>(r));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pl.splits, T, 1);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = smem_request(C::SMEM_BYTES);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeClusterDimension;
  attr[na].val.clusterDim.x = 2 * pl.splits;
  attr[na].val.clusterDim.y = 1;
  attr[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, kern, kvmap, qmap, pmap, p);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "sparse_mla_pipe launch: %s", cudaGetErrorString(e));
  return check_launch("sparse_mla_pipe");
}

dsa_status launch_mla(const dsa_batch* bt, const dsa_mla_in* in, const int32_t* idx, int k, void* out, float* lse,
                      void* ws, size_t ws_bytes, cudaStream_t st, bool pdl = false) {
  const int hb = (in->n_heads + 63) / 64;
  if (in->kv_dtype == DSA_KV_FP8_E4M3) {
    // FP8 rows: the one-CTA-per-head-block kernel widens them on chip
    if (in->d_latent == 512) {
      const MlaPlan pl = mla_plan(bt->num_q, hb, k, num_sms(), MlaCfg<576, 512>::TK);
      return launch_mla_t<576, 512, true>(bt, in, idx, k, out, lse, ws, ws_bytes, st, pl, pdl);
    }
    const MlaPlan pl = mla_plan(bt->num_q, hb, k, num_sms(), MlaCfg<80, 64>::TK);
    return launch_mla_t<80, 64, true>(bt, in, idx, k, out, lse, ws, ws_bytes, st, pl, pdl);
  }
  if (in->d_latent == 512 && in->n_heads == PipeCfg::M && bt->num_q <= 65535)  // queries on grid y
    return launch_mla_pipe(bt, in, idx, k, out, lse, ws, ws_bytes, st, pdl);
  if (in->d_latent == 512) {
    const MlaPlan pl = mla_plan(bt->num_q, hb, k, num_sms(), MlaCfg<576, 512>::TK);
    return launch_mla_t<576, 512>(bt, in, idx, k, out, lse, ws, ws_bytes, st, pl, pdl);
  }
  const MlaPlan pl = mla_plan(bt->num_q, hb, k, num_sms(), MlaCfg<80, 64>::TK);
  return launch_mla_t<80, 64>(bt, in, idx, k, out, lse, ws, ws_bytes, st, pl, pdl);
}

// Test hook: a kernel that lets programmatic dependents start at once, then
// waits delay_ns of wall time (a bounded sleep loop) and only then copies src
// to dst, so a dependent that read dst before its own wait would see the old
// contents.
__global__ void debug_delayed_copy_kernel(uint4* dst, const uint4* src, int64_t n16, uint64_t delay_ns) {
  pdl_launch_dependents();
  const uint64_t t0 = globaltimer();
  while (globaltimer() - t0 < delay_ns) __nanosleep(2000);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}

}  // namespace

// ============================================================================ C ABI
extern "C" {

const char* dsa_version(void) { return "dsa-b200 0.1 (sm_100a)"; }

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DSA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_DEVICE_INDEX: return "device: out-of-range index skipped";
    case DSA_ERR_DEVICE_TIMEOUT: return "device: bounded wait gave up";
    case DSA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case DSA_ERR_DEVICE_LAYOUT:
      return "device: shared memory window misaligned, or an SM id outside the per-SM workspace records";
  }
  return "unknown status";
}

const char* dsa_last_error(void) { return g_last_error; }

size_t dsa_workspace_size(int op, const dsa_batch* batch, int32_t k, int32_t h_i, int32_t d_i) {
  if (!batch || batch->num_q <= 0) return 0;
  const int T = batch->num_q;
  const size_t qb = (h_i > 0 && d_i > 0) ? mx_q_bytes(T, h_i, d_i) : 0;
  if (op == DSA_OP_INDEXER_SCORES) return qb;
  if (k <= 0) return 0;
  switch (op) {
    case DSA_OP_TOPK:
      return 0;
    case DSA_OP_SPARSE_MLA:
      return mla_ws_bytes(batch, k);
    case DSA_OP_FUSED_DECODE:
      return align256(static_cast<size_t>(T) * batch->max_seq_len * sizeof(float)) +
             align256(static_cast<size_t>(T) * k * sizeof(int32_t)) + mla_ws_bytes(batch, k) + qb;
    default:
      return 0;
  }
}

dsa_status dsa_indexer_scores(const dsa_batch* batch, const dsa_indexer_in* in, float* scores, int64_t score_ld,
                              void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_indexer(batch, in)) != DSA_OK) return s;
  if (!scores) return fail(DSA_ERR_INVALID_ARGUMENT, "scores is NULL");
  if (score_ld < batch->max_seq_len) return fail(DSA_ERR_INVALID_ARGUMENT, "score_ld < max_seq_len");
  if (batch->num_q == 0) return DSA_OK;
  if (in->key_dtype == DSA_KEY_MXFP8) {
    const size_t need = mx_q_bytes(batch->num_q, in->n_heads, in->head_dim);
    if (!ws || ws_bytes < need) return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes, need);
    if (!aligned16(ws)) return fail(DSA_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  }
  return launch_indexer(batch, in, scores, score_ld, reinterpret_cast<cudaStream_t>(stream), false, ws);
}

dsa_status dsa_topk(const dsa_batch* batch, const float* scores, int64_t score_ld, int32_t k, int32_t* idx,
                    void* ws, size_t ws_bytes, dsa_stream_t stream) {
  (void)ws;
  (void)ws_bytes;
  dsa_status s = check_batch(batch);
  if (s != DSA_OK) return s;
  if (!scores || !idx) return fail(DSA_ERR_INVALID_ARGUMENT, "scores and idx must be non-NULL");
  if (k < 1 || k > 2048) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, 2048]", k);
  if (score_ld < batch->max_seq_len) return fail(DSA_ERR_INVALID_ARGUMENT, "score_ld < max_seq_len");
  if (batch->num_q == 0) return DSA_OK;
  return launch_topk(batch, scores, score_ld, k, idx, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_sparse_mla_attn(const dsa_batch* batch, const dsa_mla_in* in, const int32_t* idx, int32_t k,
                               void* out, float* lse, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  dsa_status s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_mla(in)) != DSA_OK) return s;
  if (!idx || !out) return fail(DSA_ERR_INVALID_ARGUMENT, "idx and out must be non-NULL");
  if (!aligned16(out) || !aligned16(idx)) return fail(DSA_ERR_MISALIGNED, "idx and out must be 16-byte aligned");
  if (k < 1 || k > 2048) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, 2048]", k);
  if (batch->num_q == 0) return DSA_OK;
#ifdef DSA_DEBUG
  if ((s = debug_check_indices(batch, idx, k, reinterpret_cast<cudaStream_t>(stream))) != DSA_OK) return s;
#endif
  return launch_mla(batch, in, idx, k, out, lse, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

dsa_status dsa_fused_decode(const dsa_batch* batch, const dsa_indexer_in* idx_in, const dsa_mla_in* mla_in,
                            int32_t k, void* out, float* lse, int32_t* idx_out, void* ws, size_t ws_bytes,
                            const dsa_event_t* stage_events, dsa_stream_t stream) {
  dsa_status s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_indexer(batch, idx_in)) != DSA_OK) return s;
  if ((s = check_mla(mla_in)) != DSA_OK) return s;
  if (!out) return fail(DSA_ERR_INVALID_ARGUMENT, "out is NULL");
  if (!aligned16(out) || (idx_out && !aligned16(idx_out)))
    return fail(DSA_ERR_MISALIGNED, "out and idx_out must be 16-byte aligned");
  if (k < 1 || k > 2048) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, 2048]", k);
  if (batch->num_q == 0) return DSA_OK;
  const int T = batch->num_q;
  const size_t sc_bytes = align256(static_cast<size_t>(T) * batch->max_seq_len * sizeof(float));
  const size_t id_bytes = align256(static_cast<size_t>(T) * k * sizeof(int32_t));
  const size_t mla_bytes = mla_ws_bytes(batch, k);
  const size_t q_bytes = idx_in->key_dtype == DSA_KEY_MXFP8 ? mx_q_bytes(T, idx_in->n_heads, idx_in->head_dim) : 0;
  const size_t need = sc_bytes + id_bytes + mla_bytes + q_bytes;
  if (!ws || ws_bytes < need) return fail(DSA_ERR_WORKSPACE_TOO_SMALL, "workspace %zu < %zu bytes", ws_bytes, need);
  if (!aligned16(ws)) return fail(DSA_ERR_MISALIGNED, "workspace must be 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* scores = static_cast<float*>(ws);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + sc_bytes);
  auto rec = [&](int i) -> dsa_status {
    if (!stage_events) return DSA_OK;
    const cudaError_t e = cudaEventRecord(reinterpret_cast<cudaEvent_t>(stage_events[i]), st);
    return e == cudaSuccess ? DSA_OK : fail(DSA_ERR_CUDA, "cudaEventRecord: %s", cudaGetErrorString(e));
  };
  // Programmatic dependent launch on every edge: each kernel is scheduled
  // while the previous one finishes and waits on the device for what it
  // consumes. The indexer waits before it reads anything (whatever ran
  // before the call may have written its inputs) and only then lets the
  // Top-K be scheduled, so the Top-K and the attention, which read the
  // batch description and the queries before their own waits, see complete
  // inputs. Not used when stage events sit between the kernels.
  const bool pdl = stage_events == nullptr;
  if ((s = rec(0)) != DSA_OK) return s;
  if ((s = launch_indexer(batch, idx_in, scores, batch->max_seq_len, st, pdl,
                          static_cast<uint8_t*>(ws) + sc_bytes + id_bytes + mla_bytes)) != DSA_OK)
    return s;
  if ((s = rec(1)) != DSA_OK) return s;
  if ((s = launch_topk(batch, scores, batch->max_seq_len, k, idx, st, pdl)) != DSA_OK) return s;
#ifdef DSA_DEBUG
  if ((s = debug_check_indices(batch, idx, k, st)) != DSA_OK) return s;
#endif
  if ((s = rec(2)) != DSA_OK) return s;
  if ((s = launch_mla(batch, mla_in, idx, k, out, lse, static_cast<uint8_t*>(ws) + sc_bytes + id_bytes, mla_bytes, st,
                      pdl)) != DSA_OK)
    return s;
  return rec(3);
}

dsa_status dsa_quantize_index_keys(const void* k_bf16, int64_t n_keys, int32_t dim, int32_t group, uint8_t* k8,
                                   float* scale, dsa_stream_t stream) {
  if (!k_bf16 || !k8 || !scale) return fail(DSA_ERR_INVALID_ARGUMENT, "k_bf16, k8, scale must be non-NULL");
  if (n_keys < 0) return fail(DSA_ERR_INVALID_ARGUMENT, "n_keys < 0");
  if (group != 32 && group != 64 && group != 128) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "group %d not in {32,64,128}", group);
  if (dim <= 0 || dim > 1024 || dim % group != 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "dim %d must be a multiple of group and <= 1024", dim);
  if (!aligned16(k_bf16) || !aligned16(k8) || !aligned16(scale))
    return fail(DSA_ERR_MISALIGNED, "k_bf16, k8, scale must be 16-byte aligned");
  if (n_keys == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms();
  const int64_t blocks64 = (n_keys + 7) / 8;
  const int blocks = static_cast<int>(blocks64 < sms * 16 ? blocks64 : sms * 16);
  const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(k_bf16);
  if (group == 32)
    quantize_keys_kernel<32><<<blocks, 256, 0, st>>>(k, n_keys, dim, k8, scale);
  else if (group == 64)
    quantize_keys_kernel<64><<<blocks, 256, 0, st>>>(k, n_keys, dim, k8, scale);
  else
    quantize_keys_kernel<128><<<blocks, 256, 0, st>>>(k, n_keys, dim, k8, scale);
  return check_launch("quantize_index_keys");
}

dsa_status dsa_quantize_mxfp8(const void* x_bf16, int64_t n_rows, int32_t dim, uint8_t* codes, uint8_t* scales,
                              dsa_stream_t stream) {
  if (!x_bf16 || !codes || !scales) return fail(DSA_ERR_INVALID_ARGUMENT, "x_bf16, codes, scales must be non-NULL");
  if (n_rows < 0) return fail(DSA_ERR_INVALID_ARGUMENT, "n_rows < 0");
  if (dim <= 0 || dim > 1024 || dim % 32 != 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "dim %d must be a multiple of 32 and <= 1024", dim);
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales))
    return fail(DSA_ERR_MISALIGNED, "x_bf16, codes, scales must be 16-byte aligned");
  if (n_rows == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms();
  const int64_t blocks64 = (n_rows + 7) / 8;
  const int blocks = static_cast<int>(blocks64 < sms * 16 ? blocks64 : sms * 16);
  mx_quantize_kernel<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x_bf16), n_rows, dim, codes, scales);
  return check_launch("quantize_mxfp8");
}

size_t dsa_kv_fp8_row_bytes(int32_t d_latent, int32_t d_rope) {
  if (d_latent == 512 && d_rope == 64) return KvFp8Row<512, 64>::ROW_BYTES;
  if (d_latent == 64 && d_rope == 16) return KvFp8Row<64, 16>::ROW_BYTES;
  return 0;
}

dsa_status dsa_quantize_kv(const void* kv_bf16, int64_t n_rows, int32_t d_latent, int32_t d_rope, uint8_t* kv_fp8,
                           dsa_stream_t stream) {
  if (!kv_bf16 || !kv_fp8) return fail(DSA_ERR_INVALID_ARGUMENT, "kv_bf16 and kv_fp8 must be non-NULL");
  if (n_rows < 0) return fail(DSA_ERR_INVALID_ARGUMENT, "n_rows < 0");
  if (dsa_kv_fp8_row_bytes(d_latent, d_rope) == 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "KV dims (%d,%d) not in {(512,64),(64,16)}", d_latent, d_rope);
  if (!aligned16(kv_bf16) || !aligned16(kv_fp8)) return fail(DSA_ERR_MISALIGNED, "kv_bf16 and kv_fp8 must be 16-byte aligned");
  if (n_rows == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms();
  const int64_t blocks64 = (n_rows + 7) / 8;
  const int blocks = static_cast<int>(blocks64 < sms * 16 ? blocks64 : sms * 16);
  const __nv_bfloat16* kv = static_cast<const __nv_bfloat16*>(kv_bf16);
  if (d_latent == 512)
    quantize_kv_kernel<512, 64><<<blocks, 256, 0, st>>>(kv, n_rows, kv_fp8);
  else
    quantize_kv_kernel<64, 16><<<blocks, 256, 0, st>>>(kv, n_rows, kv_fp8);
  return check_launch("quantize_kv");
}

dsa_status dsa_dequantize_index_keys(const uint8_t* k8, const float* scale, int64_t n_keys, int32_t dim,
                                     int32_t group, float* out, dsa_stream_t stream) {
  if (!k8 || !scale || !out) return fail(DSA_ERR_INVALID_ARGUMENT, "k8, scale, out must be non-NULL");
  if (n_keys < 0) return fail(DSA_ERR_INVALID_ARGUMENT, "n_keys < 0");
  if (group != 32 && group != 64 && group != 128) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "group %d not in {32,64,128}", group);
  if (dim <= 0 || dim > 1024 || dim % group != 0)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "dim %d must be a multiple of group and <= 1024", dim);
  if (!aligned16(k8) || !aligned16(out) || !aligned16(scale))
    return fail(DSA_ERR_MISALIGNED, "k8, scale, out must be 16-byte aligned");
  if (n_keys == 0) return DSA_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n = n_keys * dim;
  const int64_t blocks64 = (n / 4 + 255) / 256;
  const int sms = num_sms();
  const int blocks = static_cast<int>(blocks64 < sms * 32 ? blocks64 : sms * 32);
  dequantize_keys_kernel<<<blocks, 256, 0, st>>>(k8, scale, n, dim, group, out);
  return check_launch("dequantize_index_keys");
}

dsa_status dsa_read_device_status(dsa_stream_t stream, int32_t* code_out) {
  if (!code_out) return fail(DSA_ERR_INVALID_ARGUMENT, "code_out is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, dsa::g_device_status, sizeof(int));
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "reading device status: %s", cudaGetErrorString(e));
  const int zero = 0;
  e = cudaMemcpyToSymbol(dsa::g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "clearing device status: %s", cudaGetErrorString(e));
  *code_out = v;
  return DSA_OK;
}

dsa_status dsa_debug_set_wait_limit(uint64_t limit_ns) {
  const uint64_t v = limit_ns ? limit_ns : dsa::kDefaultWaitLimitNs;
  const cudaError_t e = cudaMemcpyToSymbol(dsa::g_wait_limit_ns, &v, sizeof(v));
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "setting the wait limit: %s", cudaGetErrorString(e));
  return DSA_OK;
}

dsa_status dsa_debug_delayed_copy(void* dst, const void* src, size_t bytes, uint64_t delay_ns, dsa_stream_t stream) {
  if (!dst || !src) return fail(DSA_ERR_INVALID_ARGUMENT, "dst and src must be non-NULL");
  if ((reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src) | bytes) & 15u)
    return fail(DSA_ERR_INVALID_ARGUMENT, "dst, src and bytes must be multiples of 16");
  if (delay_ns > 1000000000ull) return fail(DSA_ERR_INVALID_ARGUMENT, "delay_ns above 1 s");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  debug_delayed_copy_kernel<<<64, 256, 0, st>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src),
                                                 static_cast<int64_t>(bytes / 16), delay_ns);
  return check_launch("debug_delayed_copy");
}

dsa_status dsa_debug_withhold_signal(int32_t on) {
  const int v = on ? 1 : 0;
  const cudaError_t e = cudaMemcpyToSymbol(dsa::g_debug_withhold, &v, sizeof(v));
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "setting the test hook: %s", cudaGetErrorString(e));
  return DSA_OK;
}

}  // extern "C"

// ============================================================================ allocation-free variant
//
// dsa_fused_decode_noalloc runs the same chain as dsa_fused_decode but takes
// no workspace: its scratch (the fp32 score rows and, when the caller passes
// no idx_out, the selected indices) lives in one fixed device array compiled
// into this library. It exists for callers that cannot hand out device
// memory at call time -- a plugin host or inference runtime that owns every
// byte of device memory through its own pool and gives extensions no
// workspace, or a caller on a latency-critical serving path that must never
// enter the CUDA allocator. The attention runs with one key split per query,
// so no split-K partials are needed.
//
// The array is kNoAllocScratchBytes (32 MiB) on every device that loads the
// library, held until the process exits. Calls that would need more scratch
// are rejected. Nothing in it has to start at zero: the indexer writes every
// score the Top-K reads and the Top-K writes every index the attention
// reads, so contents left by an earlier call are never used. All calls share
// the one array: two calls whose work overlaps on the GPU (different streams,
// or different host threads on one device) race on it and must be ordered by
// the caller.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};  // context the address belongs to

// Unique id of the calling thread's current CUDA context (0 if unavailable).
// Ids are never reused, so a reset device (a new primary context, the module
// loaded again, possibly at another address) is told apart from the old one.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = []() -> GetCurrentFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<GetCurrentFn>(p);
  }();
  static GetIdFn get_id = []() -> GetIdFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<GetIdFn>(p);
  }();
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch array on the current device. The host-side
// symbol is only a stand-in, so the address is looked up with that device
// current (on the first call there, and again whenever the device's context
// has changed, e.g. after cudaDeviceReset) and cached.
dsa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(DSA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(DSA_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const unsigned long long ctx = current_context_id();  // 0: no context bound to this thread yet
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);  // binds the device's context if needed
    if (e != cudaSuccess || !p)
      return fail(DSA_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_context_id();
  }
  *out = g_noalloc_ptr[dev];
  return DSA_OK;
}

// Attention with one key split per query (writes out / lse directly).
dsa_status launch_mla_unsplit(const dsa_batch* bt, const dsa_mla_in* in, const int32_t* idx, int k, void* out,
                              float* lse, cudaStream_t st) {
  const MlaPlan pl{1, ((k + 63) / 64) * 64};
  const bool f8 = in->kv_dtype == DSA_KV_FP8_E4M3;
  if (in->d_latent == 512)
    return f8 ? launch_mla_t<576, 512, true>(bt, in, idx, k, out, lse, nullptr, 0, st, pl, false)
              : launch_mla_t<576, 512>(bt, in, idx, k, out, lse, nullptr, 0, st, pl, false);
  return f8 ? launch_mla_t<80, 64, true>(bt, in, idx, k, out, lse, nullptr, 0, st, pl, false)
            : launch_mla_t<80, 64>(bt, in, idx, k, out, lse, nullptr, 0, st, pl, false);
}

}  // namespace

extern "C" dsa_status dsa_fused_decode_noalloc(const dsa_batch* batch, const dsa_indexer_in* idx_in,
                                               const dsa_mla_in* mla_in, int32_t k, void* out, float* lse,
                                               int32_t* idx_out, dsa_stream_t stream) {
  dsa_status s = check_batch(batch);
  if (s != DSA_OK) return s;
  if ((s = check_indexer(batch, idx_in)) != DSA_OK) return s;
  if ((s = check_mla(mla_in)) != DSA_OK) return s;
  if (idx_in->key_dtype == DSA_KEY_MXFP8)
    return fail(DSA_ERR_UNSUPPORTED_SHAPE, "dsa_fused_decode_noalloc does not take MXFP8 index inputs");
  if (!out) return fail(DSA_ERR_INVALID_ARGUMENT, "out is NULL");
  if (!aligned16(out) || (idx_out && !aligned16(idx_out)))
    return fail(DSA_ERR_MISALIGNED, "out and idx_out must be 16-byte aligned");
  if (k < 1 || k > 2048) return fail(DSA_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, 2048]", k);
  if (batch->num_q == 0) return DSA_OK;
  const int T = batch->num_q;
  const size_t sc_bytes = align256(static_cast<size_t>(T) * batch->max_seq_len * sizeof(float));
  const size_t id_bytes = idx_out ? 0 : align256(static_cast<size_t>(T) * k * sizeof(int32_t));
  if (sc_bytes + id_bytes > kNoAllocScratchBytes)
    return fail(DSA_ERR_WORKSPACE_TOO_SMALL,
                "dsa_fused_decode_noalloc needs %zu bytes of scratch (num_q * max_seq_len * 4%s); its built-in "
                "array holds %zu bytes",
                sc_bytes + id_bytes, idx_out ? "" : " + num_q * k * 4", kNoAllocScratchBytes);
  void* scratch = nullptr;
  if ((s = noalloc_scratch(&scratch)) != DSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  float* scores = static_cast<float*>(scratch);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + sc_bytes);
  if ((s = launch_indexer(batch, idx_in, scores, batch->max_seq_len, st)) != DSA_OK) return s;
  if ((s = launch_topk(batch, scores, batch->max_seq_len, k, idx, st)) != DSA_OK) return s;
  return launch_mla_unsplit(batch, mla_in, idx, k, out, lse, st);
}
