/*
 * dsa.h -- C ABI of libdsa.so: the indexed sparse attention (DSA) hot path on
 * NVIDIA B200 (sm_100a).
 *
 * The path (section 1 of "Day-0 Inference Optimization for a New Sparse
 * Attention Architecture"; section 3 of "Optimizing Inference for New Model
 * Architectures: Co-Designing Sparse Attention, State Recurrence, and
 * Long-Sequence Partitioning"):
 *   1. Lightning Indexer: relevance scoring of each query token against every
 *      causal history position, weighted over indexer heads,
 *        I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]),  s <= pos(t);
 *   2. Top-K: the K highest-scoring positions per query row (ties: higher
 *      score, then lower position);
 *   3. Sparse Flash Attention over multi-head latent attention (MLA) rows:
 *      every query head attends only over the selected latent KV rows; a row
 *      has d_latent + d_rope dims, the value is its first d_latent dims.
 * "Inference Adaptation and Performance Optimization for New Large Language
 * Model Architectures" (section 6, fused execution of the sparse attention
 * path) splits the path into an indexer step that turns the query and the
 * index-key cache into selected positions, and an attention step that reads
 * only those cache rows. The calls below follow that split:
 * dsa_indexer_scores + dsa_topk form the indexer, dsa_sparse_mla_attn the
 * attention, dsa_fused_decode the whole chain. The index-key cache can be
 * BF16 or FP8 E4M3 with a per-group fp32 scale (Tiered Quantization of
 * "Day-0 Inference Adaptation and Performance Optimization for
 * New-Architecture Large Language Models"); both key types go through the
 * same calls with the same meaning, so a caller switches precision by the
 * key_dtype field alone (Layered Quantization of "Inference Optimization for
 * New Open-Source LLM Architectures").
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers unless stated, row-major, owned
 *    by the caller. No call allocates device memory (the one fixed array that
 *    dsa_fused_decode_noalloc uses is part of the loaded library), keeps
 *    per-call state or synchronises (except dsa_read_device_status).
 *  - Calls are asynchronous on `stream` (0 = legacy default stream).
 *  - Argument, shape and alignment errors return a status before anything is
 *    enqueued; dsa_last_error() then describes the problem.
 *  - A failed kernel launch returns DSA_ERR_CUDA.
 *  - Errors found on the device (an index that is neither -1 nor inside
 *    [0, seq_len), or a bounded wait inside a kernel that gave up) never trap:
 *    the offending element is skipped and a sticky per-device status word is
 *    set; read it with dsa_read_device_status().
 *  - Supported shapes (anything else returns DSA_ERR_UNSUPPORTED_SHAPE):
 *      indexer (H_I, d_I): (4, 32), (4, 128), (64, 32), (64, 128)
 *      MLA (d_latent, d_rope): (512, 64), (64, 16)
 *      MLA heads H: 1..64, or 128
 *      top-K k: 1..2048
 *      paged caches: page_size a positive multiple of 64
 *    FP8 index keys need scale_group == d_I (one scale per key); MXFP8 index
 *    inputs need scale_group == 32. FP8 latent KV rows come in the packed
 *    layout of dsa_quantize_kv for either MLA shape.
 *  - Alignment: every tensor pointer must be 16-byte aligned (the block table:
 *    4-byte aligned).
 *  - Debug build (libdsa_debug.so, compiled with DSA_DEBUG): before the
 *    attention gathers any row, the host checks every index (the call then
 *    synchronises its stream) and returns DSA_ERR_INVALID_ARGUMENT naming the
 *    first one that is neither -1 nor inside its sequence; the tensor-core
 *    kernels guard the end of their shared-memory layout with a canary and
 *    report DSA_ERR_DEVICE_LAYOUT if it was overwritten. Calls of the debug
 *    build cannot be captured in a CUDA graph.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dsa_stream_t; /* same type as cudaStream_t */
typedef struct CUevent_st *dsa_event_t;   /* same type as cudaEvent_t */

typedef enum {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARGUMENT = 1,   /* null pointer, negative size, bad enum */
    DSA_ERR_UNSUPPORTED_SHAPE = 2,  /* outside the supported shapes above */
    DSA_ERR_WORKSPACE_TOO_SMALL = 3,/* ws_bytes < dsa_workspace_size(...) */
    DSA_ERR_CUDA = 4,               /* a CUDA runtime call or launch failed */
    DSA_ERR_DEVICE_INDEX = 5,       /* device status: an index out of range was skipped */
    DSA_ERR_DEVICE_TIMEOUT = 6,     /* device status: a bounded wait gave up */
    DSA_ERR_MISALIGNED = 7,         /* a pointer is not 16-byte aligned */
    DSA_ERR_DEVICE_LAYOUT = 8       /* device status: a kernel found its shared memory misaligned,
                                       or an SM id outside its per-SM workspace records */
} dsa_status;

/* Index query / key formats:
 *   DSA_KEY_BF16      bf16 queries and keys;
 *   DSA_KEY_FP8_E4M3  bf16 queries, E4M3 key codes with one fp32 scale per key;
 *   DSA_KEY_MXFP8     E4M3 codes for queries AND keys, one E8M0 (power-of-two)
 *                     scale per 32 elements of each (Index Q/K Uses MXFP8,
 *                     section 4.2 of "Inference Adaptation and Performance
 *                     Optimization for New Large Language Model
 *                     Architectures"); see dsa_quantize_mxfp8. */
typedef enum { DSA_KEY_BF16 = 0, DSA_KEY_FP8_E4M3 = 1, DSA_KEY_MXFP8 = 2 } dsa_key_dtype;

/* Ops for dsa_workspace_size(). */
typedef enum {
    DSA_OP_INDEXER_SCORES = 0,
    DSA_OP_TOPK = 1,
    DSA_OP_SPARSE_MLA = 2,
    DSA_OP_FUSED_DECODE = 3
} dsa_op;

/* The batch: B sequences, T query tokens packed sequence after sequence.
 *   cu_q     [B+1] int32 device: tokens of sequence b are [cu_q[b], cu_q[b+1]);
 *                  cu_q[0] = 0, non-decreasing, cu_q[B] = T.
 *   q_pos    [T]   int32 device: position of each query token inside its
 *                  sequence; its causal history is s <= q_pos.
 *   seq_lens [B]   int32 device: valid cache rows of sequence b (<= max_seq_len).
 *   max_seq_len    L_max: the longest sequence the caches hold, and the row
 *                  stride of the score rows. Contiguous caches (block_table
 *                  NULL): sequence b's row s is cache row b * L_max + s.
 *   block_table    [B, max_pages] int32 device, or NULL. Paged caches (the
 *                  fused indexer reading the paged key cache directly:
 *                  section 3 of "Optimizing Inference for New Model
 *                  Architectures ..."): every cache -- index keys, their FP8
 *                  scales and the latent KV rows -- is a pool of num_pages
 *                  pages of page_size rows, all under this one table, and
 *                  sequence b's row s is pool row
 *                    block_table[b * max_pages + s / page_size] * page_size
 *                      + s % page_size,
 *                  max_pages = ceil(max_seq_len / page_size). Only the
 *                  entries of pages that hold rows s < seq_lens[b] are read.
 *                  An entry outside [0, num_pages) is never dereferenced: the
 *                  row reads as pool row 0 and DSA_ERR_DEVICE_INDEX is set.
 *                  Positions (scores, indices) stay logical.
 *   page_size      rows per page, a positive multiple of 64 (paged), else 0.
 *   num_pages      pages in the pool (paged), else 0; num_pages * page_size
 *                  must be below 2^31.
 * A query's candidate count is n_valid(t) = min(q_pos[t] + 1, seq_lens[b]). */
typedef struct {
    int32_t batch;
    int32_t num_q;
    int32_t max_seq_len;
    const int32_t *cu_q;
    const int32_t *q_pos;
    const int32_t *seq_lens;
    const int32_t *block_table;
    int32_t page_size;
    int32_t num_pages;
} dsa_batch;

/* Lightning Indexer inputs.
 *   q        [T, n_heads, head_dim]            indexer queries q_I: bf16, or
 *            E4M3 codes (DSA_KEY_MXFP8)
 *   w        fp32 [T, n_heads]                 head weights
 *   k_cache  [rows, head_dim]                  index keys, bf16 or e4m3 codes;
 *            rows = B * L_max (contiguous) or num_pages * page_size (paged)
 *   k_scale  fp32 [rows, head_dim/scale_group] per-group scales (FP8_E4M3
 *            only; the key value is decode(code) * scale), else NULL
 *   scale_group: elements per scale; head_dim for FP8_E4M3 (one scale per
 *            key), 32 for MXFP8.
 *   q_scale_e8m0  uint8 [T, n_heads, head_dim/32], k_scale_e8m0 uint8
 *            [rows, head_dim/32]: MXFP8 scale bytes (value = decode(code) *
 *            2^(byte - 127)), else NULL. */
typedef struct {
    int32_t n_heads;
    int32_t head_dim;
    const void *q;
    const float *w;
    dsa_key_dtype key_dtype;
    const void *k_cache;
    const float *k_scale;
    int32_t scale_group;
    const uint8_t *q_scale_e8m0;
    const uint8_t *k_scale_e8m0;
} dsa_indexer_in;

/* Latent KV cache element types. */
typedef enum { DSA_KV_BF16 = 0, DSA_KV_FP8_E4M3 = 1 } dsa_kv_dtype;

/* Sparse MLA inputs.
 *   q   bf16 [T, n_heads, d_latent + d_rope]
 *   kv  latent rows (rows as for k_cache); value = first d_latent dims:
 *       DSA_KV_BF16:     bf16 [rows, d_latent + d_rope]
 *       DSA_KV_FP8_E4M3: packed FP8 rows [rows, dsa_kv_fp8_row_bytes()] as
 *                        written by dsa_quantize_kv (block-wise FP8 KV cache:
 *                        section 4 of "Optimizing Inference for New Model
 *                        Architectures ..."). The rows are widened to bf16
 *                        on chip (fl32(decode(code) * tile scale) rounded to
 *                        nearest bf16); q and the products stay bf16/fp32.
 *   softmax_scale: multiplies q . kv before the softmax.
 *   kv_dtype: DSA_KV_BF16 (0) or DSA_KV_FP8_E4M3. */
typedef struct {
    int32_t n_heads;
    int32_t d_latent;
    int32_t d_rope;
    float softmax_scale;
    const void *q;
    const void *kv;
    dsa_kv_dtype kv_dtype;
} dsa_mla_in;

/* Lightning Indexer scores (relevance scoring + head-weight weighting +
 * causal/ragged mask).
 * scores: fp32 [T, score_ld], score_ld >= max_seq_len. Row t gets
 *   I[t,s] for s < n_valid(t) and -inf for n_valid(t) <= s < the end of the
 *   last 128-key tile that holds a valid key; entries beyond are not written.
 * FP8 keys: I = scale_s * sum_j w_j * max(0, q_j . decode(code_s)), which
 * equals the score of the dequantised key because scale_s >= 0.
 * MXFP8: the scores of the dequantised queries and keys; every dequantised
 * element is exact in bf16, so the products are exact and only the fp32
 * sums round, as for bf16 inputs.
 * ws: workspace of dsa_workspace_size(DSA_OP_INDEXER_SCORES, ...) bytes,
 * 16-byte aligned; used only by MXFP8 (the widened queries: T * n_heads *
 * head_dim * 2 bytes), may be NULL otherwise. */
dsa_status dsa_indexer_scores(const dsa_batch *batch, const dsa_indexer_in *in, float *scores,
                              int64_t score_ld, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Per-row Top-K of the indexer scores: the selection step that ends the
 * Lightning Indexer ("Day-0 Inference Optimization for a New Sparse
 * Attention Architecture", section 1: only the Top-K history positions of a
 * query are passed on to the attention).
 * scores: fp32 [T, score_ld]; only columns [0, n_valid(t)) are read.
 * idx: int32 [T, k]: the min(k, n_valid(t)) best positions of row t under the
 *   order (score desc, position asc) with -0 == +0, written in ascending
 *   position order and padded with -1. Bit-identical for identical scores. */
dsa_status dsa_topk(const dsa_batch *batch, const float *scores, int64_t score_ld, int32_t k,
                    int32_t *idx, void *ws, size_t ws_bytes, dsa_stream_t stream);

/* Sparse MLA attention over the selected rows.
 * idx: int32 [T, k]; -1 entries are skipped; entries outside [0, seq_len) are
 *   skipped and set DSA_ERR_DEVICE_INDEX in the device status word.
 * out: bf16 [T, n_heads, d_latent]:  sum_i softmax_i(scale * q.kv_i) * kv_i[0:d_latent]
 * lse: fp32 [T, n_heads] natural-log sum-exp of the scaled logits, or NULL.
 * A row with no valid index gets out = 0 and lse = -inf.
 * ws: at least dsa_workspace_size(DSA_OP_SPARSE_MLA, ...) bytes, 16-byte
 *   aligned, owned by the caller and not kept after the call's kernels end.
 *   The size is an upper bound over the head counts a call may use (the
 *   query does not take n_heads); it includes about 17.6 MB of P rings for
 *   128-head calls. A call that needs less may pass less.
 * Work split. 128 heads with d_latent = 512: a pair of CTAs per (query, key
 *   split): a score CTA computes Q K^T for all heads and the softmax and
 *   hands P to a value CTA (which holds O) through a per-SM ring in ws.
 *   Other shapes: one CTA per (query, 64-head block, key split). In both,
 *   the key splits of a query form a thread-block cluster; each leaves its
 *   unnormalised output rows and (max, sum) statistics in ws and, after the
 *   cluster barrier, the rows are merged with a running maximum.
 * DSA_ERR_WORKSPACE_TOO_SMALL if ws is smaller than that call needs. */
dsa_status dsa_sparse_mla_attn(const dsa_batch *batch, const dsa_mla_in *in, const int32_t *idx,
                               int32_t k, void *out, float *lse, void *ws, size_t ws_bytes,
                               dsa_stream_t stream);

/* The whole decode chain: indexer scores -> Top-K -> sparse MLA, enqueued
 * back to back on `stream` with intermediates in the workspace. The three
 * kernels are chained with programmatic dependent launch: the first one may
 * be scheduled while the stream's previous kernel finishes, but waits for it
 * before reading any input, so inputs written by earlier work on the stream
 * (including a kernel that itself allows programmatic dependents) are seen
 * complete.
 * idx_out: if non-NULL, int32 [T, k] receives the selected indices.
 * stage_events: NULL, or 4 caller-created events recorded before the indexer,
 *   before the Top-K, before the attention and after the attention (timing).
 * ws: dsa_workspace_size(DSA_OP_FUSED_DECODE, ...) bytes. */
dsa_status dsa_fused_decode(const dsa_batch *batch, const dsa_indexer_in *idx_in,
                            const dsa_mla_in *mla_in, int32_t k, void *out, float *lse,
                            int32_t *idx_out, void *ws, size_t ws_bytes,
                            const dsa_event_t *stage_events, dsa_stream_t stream);

/* The decode chain of dsa_fused_decode without a workspace argument, for
 * callers that cannot provide device memory at call time: for example an
 * inference runtime or plugin host that reserves all device memory in its own
 * pool and hands extensions no workspace, or a serving path that must never
 * enter the CUDA allocator. The paper has no counterpart for this entry
 * point; it is a service of this library.
 * Scratch (score rows, and the indices when idx_out is NULL) lives in one
 * fixed 32 MiB device array inside libdsa.so, held on every device that loads
 * the library until the process exits. The call allocates and frees nothing.
 * Limit: num_q * max_seq_len * 4 bytes (+ num_q * k * 4 when idx_out is NULL,
 * each rounded up to 256) must not exceed 33554432; larger calls return
 * DSA_ERR_WORKSPACE_TOO_SMALL with the required size in dsa_last_error().
 * The attention runs with one key split per query, so results agree with
 * dsa_fused_decode within rounding (indices are identical).
 * The first call on a device looks up the array's device address with that
 * device current, and so does the first call after the device's context has
 * changed (e.g. after cudaDeviceReset); make such a call before any stream
 * capture.
 * All calls share the array: calls whose work overlaps on the GPU (other
 * streams, other threads) race on it and must be serialised by the caller.
 * Nothing in the array needs to start at zero; stale contents are never read.
 * MXFP8 index inputs are not accepted here (DSA_ERR_UNSUPPORTED_SHAPE): their
 * widened queries would need more scratch. */
dsa_status dsa_fused_decode_noalloc(const dsa_batch *batch, const dsa_indexer_in *idx_in,
                                    const dsa_mla_in *mla_in, int32_t k, void *out, float *lse,
                                    int32_t *idx_out, dsa_stream_t stream);

/* Index-key cache write: per-group dynamic FP8 quantisation, the scheme of
 * the Tiered Quantization table of "Day-0 Inference Adaptation and
 * Performance Optimization for New-Architecture Large Language Models"
 * (indexer keys in 8-bit floating point, one scale per group of elements
 * computed from the group's absolute maximum) and of its block-wise
 * quantisation example.
 * k_bf16: bf16 [n_keys, dim]; for every group of `group` elements
 *   scale = fl32(max|k| / 448); scale == 0 -> codes 0;
 *   else code = e4m3 round-to-nearest-even, saturating, of fl32(k / scale).
 * k8: uint8 [n_keys, dim]; scale: fp32 [n_keys, dim/group].
 * group in {32, 64, 128}, dim a multiple of group and of 4, dim <= 1024. */
dsa_status dsa_quantize_index_keys(const void *k_bf16, int64_t n_keys, int32_t dim, int32_t group,
                                   uint8_t *k8, float *scale, dsa_stream_t stream);

/* Latent KV cache write, FP8 (Block-Wise Quantization for Key-Value Cache,
 * section 4 of "Optimizing Inference for New Model Architectures ..."; the
 * Tiered Quantization table of "Day-0 Inference Adaptation ..."): per token
 * row of kv_bf16 [n_rows, d_latent + d_rope], the d_latent dims in tiles of
 * min(128, d_latent) elements, each with scale = fl32(max|x| / 448) and codes
 * as in dsa_quantize_index_keys; the d_rope dims are kept in bf16. One packed
 * row of dsa_kv_fp8_row_bytes(d_latent, d_rope) bytes per token:
 *   bytes [0, d_latent)                       E4M3 codes
 *   bytes [d_latent, d_latent + 2 d_rope)     rope dims, bf16
 *   then one fp32 scale per tile, then zeros up to a multiple of 16 bytes
 *   ((512, 64): 656 bytes; (64, 16): 112 bytes).
 * (d_latent, d_rope) in {(512, 64), (64, 16)}; both pointers 16-byte aligned.
 * Writes kv_fp8 only. */
dsa_status dsa_quantize_kv(const void *kv_bf16, int64_t n_rows, int32_t d_latent, int32_t d_rope,
                           uint8_t *kv_fp8, dsa_stream_t stream);

/* Bytes of one packed FP8 latent row (see dsa_quantize_kv); 0 for
 * unsupported dims. */
size_t dsa_kv_fp8_row_bytes(int32_t d_latent, int32_t d_rope);

/* MXFP8 quantisation of index queries or keys (Index Q/K Uses MXFP8, section
 * 4.2 of "Inference Adaptation and Performance Optimization for New Large
 * Language Model Architectures"; 32 elements share one scale). For each
 * group of 32 elements of x_bf16 [n_rows, dim]: e = the least integer with
 * 448 * 2^e >= max|x| (the group pseudocode's max / 448 rounded up to a power
 * of two, so nothing saturates), kept in [-127, 127] (-127 for an all-zero
 * group); scales[group] = e + 127 (E8M0); codes = E4M3 round-to-nearest-even
 * of x * 2^-e (an exact product). dim a multiple of 32, <= 1024; all
 * pointers 16-byte aligned. Writes codes [n_rows, dim] and scales
 * [n_rows, dim / 32]. */
dsa_status dsa_quantize_mxfp8(const void *x_bf16, int64_t n_rows, int32_t dim, uint8_t *codes, uint8_t *scales,
                              dsa_stream_t stream);

/* Inverse of the cache write above (same passage): the value a key's FP8
 * code stands for, out = fl32(decode(code) * scale), fp32 [n_keys, dim].
 * Same group and dim rules as dsa_quantize_index_keys. */
dsa_status dsa_dequantize_index_keys(const uint8_t *k8, const float *scale, int64_t n_keys,
                                     int32_t dim, int32_t group, float *out, dsa_stream_t stream);

/* Workspace bytes `op` needs for this batch, k and indexer shape (h_i, d_i),
 * enough for every index-key format (MXFP8 needs room for the widened
 * queries); the MLA shape is fixed by the supported set, the largest is
 * assumed. Host-only: reads no device memory. */
size_t dsa_workspace_size(int op, const dsa_batch *batch, int32_t k, int32_t h_i, int32_t d_i);

/* Waits for `stream`, then returns in *code_out the sticky device status
 * (DSA_OK or a DSA_ERR_DEVICE_* code) of the current device and clears it. */
dsa_status dsa_read_device_status(dsa_stream_t stream, int32_t *code_out);

/* Test hooks for the failure-detection path (not for production use; both
 * act on the current device and are synchronous with respect to the host).
 * dsa_debug_set_wait_limit: wall-time limit in ns of every bounded wait
 *   inside the kernels (0 restores the default of 2 s). A shorter limit lets
 *   a test make a wait run out quickly; it must stay far above the longest
 *   legal wait of the calls the test makes.
 * dsa_debug_withhold_signal: on != 0 makes the 128-head attention's score
 *   CTA hold back its first "P ready" signal to the value CTA, so the value
 *   CTA's wait for it runs out: the kernel records DSA_ERR_DEVICE_TIMEOUT in
 *   the device status word, every role leaves its loop, tensor memory is
 *   released and the kernel returns (the call's outputs are then undefined).
 *   on = 0 restores normal operation. */
dsa_status dsa_debug_set_wait_limit(uint64_t limit_ns);
dsa_status dsa_debug_withhold_signal(int32_t on);

/* Test hook for the ordering of the chained calls: enqueues on `stream` a
 * kernel that lets programmatically dependent launches start at once, then
 * waits delay_ns (at most 1 s) and only then copies `bytes` from src to dst
 * (device memory; both addresses and bytes multiples of 16). A call enqueued
 * next on the stream must still see dst's new contents.
 * DSA_ERR_INVALID_ARGUMENT for NULL, misaligned or too long a delay. */
dsa_status dsa_debug_delayed_copy(void *dst, const void *src, size_t bytes, uint64_t delay_ns,
                                  dsa_stream_t stream);

/* Text for a status code (static storage). */
const char *dsa_status_string(dsa_status s);

/* Detail of the last non-OK return on the calling thread (static per thread). */
const char *dsa_last_error(void);

/* Library version string. */
const char *dsa_version(void);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H_ */
