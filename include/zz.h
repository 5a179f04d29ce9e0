/*
 * libzz — zigzag context-parallel prefill attention for NVIDIA B200 (sm_100a).
 *
 * The method (page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
 * module docstring): with cp_size c every sequence is cut into 2c blocks; rank r
 * owns block r (its "prev" half) and block 2c-1-r (its "next" half).  K/V are
 * all-gathered in rank order, reranged back to token order and written into a
 * paged KV pool; then each rank's two query halves run causal attention against
 * the K/V prefix that ends at their own block.  On one GPU all c ranks are
 * "virtual" and are computed by one launch.
 *
 * Conventions for every entry point:
 *   - Returns zz_status_t; zz_last_error() gives a thread-local message for the
 *     last failing call on this thread.  No C++ exception crosses the ABI.
 *   - The caller owns every device buffer (inputs, outputs, workspace).  The
 *     library owns only the opaque host-side plan object.
 *   - Kernel entry points allocate no device memory, do not synchronise the
 *     host, and enqueue all work on the caller's stream (a cudaStream_t passed
 *     as void*; NULL means the legacy default stream).
 *   - Device pointers must be 16-byte aligned.  Integer tables are int32 unless
 *     stated; pool slot indices are int64.
 *   - bf16 is IEEE binary16-brain (1-8-7); fp32 is IEEE binary32.
 */
#ifndef ZZ_H_
#define ZZ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ZZ_OK = 0,
  ZZ_ERR_INVALID_ARG = 1,      /* null/misaligned pointer, bad size, h_q % h_kv != 0, ... */
  ZZ_ERR_NOT_APPLICABLE = 2,   /* zigzag CP refuses the batch (zigzag.py, can_apply)      */
  ZZ_ERR_UNSUPPORTED = 3,      /* valid request the library does not implement (d, dtype) */
  ZZ_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed                        */
  ZZ_ERR_DEVICE_TIMEOUT = 5    /* a bounded device-side wait gave up (zz_plan_device_status) */
} zz_status_t;

typedef enum { ZZ_BF16 = 0, ZZ_FP32 = 1 } zz_dtype_t;

typedef struct zz_plan zz_plan_t;

/* Lists of zigzag.py ZigzagContextParallelMetadata, plus derived tables. */
typedef enum {
  ZZ_FIELD_EXTEND_LENS = 0,        /* [bs]      extend lengths after the pad fold-in          */
  ZZ_FIELD_PREFIX = 1,             /* [bs]      cached-prefix tokens per sequence             */
  ZZ_FIELD_SPLIT_LIST = 2,         /* [bs*2c]   block sizes, sequence-major                    */
  ZZ_FIELD_ZIGZAG_INDEX = 3,       /* [2*bs]    per rank: prev chunks then next chunks         */
  ZZ_FIELD_CP_REVERSE_INDEX = 4,   /* [bs*2c]   gathered chunk -> natural order                */
  ZZ_FIELD_REVERSE_SPLIT_LEN = 5,  /* [c*2*bs]  chunk sizes of the gathered buffer             */
  ZZ_FIELD_PER_RANK_TOKENS = 6,    /* [c]       per_rank_actual_token                          */
  ZZ_FIELD_MAX_RANK_LEN = 7,       /* [c]       max_rank_len (all equal, M)                    */
  ZZ_FIELD_KV_LEN_PREV = 8,        /* [bs]      per rank                                       */
  ZZ_FIELD_KV_LEN_NEXT = 9,        /* [bs]      per rank                                       */
  ZZ_FIELD_Q_LEN_PREV = 10,        /* [bs]      per rank (actual_seq_q_prev)                   */
  ZZ_FIELD_Q_LEN_NEXT = 11,        /* [bs]      per rank (actual_seq_q_next)                   */
  ZZ_FIELD_CU_SEQLENS_Q_PREV = 12, /* [bs+1]    per rank, local exclusive prefix sums          */
  ZZ_FIELD_CU_SEQLENS_Q_NEXT = 13, /* [bs+1]    per rank                                       */
  ZZ_FIELD_SRC_ROW = 14,           /* [T]       natural token -> row of the [c*M] layout       */
  ZZ_FIELD_RANK_TOK = 15           /* [c*M]     row of the [c*M] layout -> natural token, -1 pad */
} zz_field_t;

typedef struct {
  int32_t cp_size;
  int32_t bs;
  int64_t total_tokens;     /* T = sum of extend lengths after the pad fold-in        */
  int32_t max_rank_len;     /* M: rows per rank in the padded gathered / Q layouts    */
  int32_t total_q_prev;     /* of the rank asked for in zz_plan_info                  */
  int32_t total_q_next;
  int32_t max_seqlen_q_prev;
  int32_t max_seqlen_q_next;
  int64_t causal_pairs;     /* visible (q,k) pairs over all ranks and halves          */
} zz_plan_info_t;

/* Thread-local message of the last failing call on this thread ("" if none). */
const char* zz_last_error(void);

/*
 * Build the zigzag metadata for ALL c ranks on the host
 * (zigzag.py, ZigzagCPStrategy.can_apply and build_metadata).
 *   extend_lens [bs]  tokens to prefill per sequence; may be NULL (then
 *                     seq_lens is used, or one sequence of num_tokens, bs = 1).
 *   seq_lens    [bs]  total lengths incl. cached prefix; may be NULL (prefix 0).
 *   num_tokens        >= sum(extend_lens); the surplus is folded into the last
 *                     sequence (and into seq_lens[bs-1] when given).
 * Errors: ZZ_ERR_NOT_APPLICABLE if cp_size <= 1, num_tokens < 2c or any extend
 * length < 2c; ZZ_ERR_INVALID_ARG for bs <= 0, negative lengths, num_tokens <
 * sum(extend_lens), or sizes beyond int32 rows.  *out is owned by the caller and
 * released with zz_plan_destroy.  Host only; needs no GPU.
 */
zz_status_t zz_plan_create(int cp_size, int bs, const int32_t* extend_lens,
                           const int32_t* seq_lens, int64_t num_tokens, zz_plan_t** out);
void zz_plan_destroy(zz_plan_t* plan);

/* Scalars of the plan; the per-rank ones are for `rank`. */
zz_status_t zz_plan_info(const zz_plan_t* plan, int rank, zz_plan_info_t* out);

/*
 * Copy one list into host memory.  `rank` selects the rank for per-rank
 * fields and is ignored otherwise.  On success *count is the list length;
 * with dst == NULL only *count is written.  ZZ_ERR_INVALID_ARG if capacity is
 * too small or rank is out of range.
 */
zz_status_t zz_plan_get(const zz_plan_t* plan, int rank, zz_field_t field,
                        int32_t* dst, int64_t capacity, int64_t* count);

/* Bytes of device workspace zz_plan_upload needs (256-byte aligned sections). */
size_t zz_plan_workspace_bytes(const zz_plan_t* plan);

/*
 * Enqueue the host-to-device copy of the plan's device tables (token -> row
 * map, half descriptors, longest-first work lists) into `dev_workspace`
 * (caller-owned, >= zz_plan_workspace_bytes, 256-byte aligned) on `stream`,
 * and remember that address for later calls.  The plan must outlive the copy.
 * The first upload of a plan lays its tables out in pinned host memory owned
 * by the plan (cudaMallocHost, freed by zz_plan_destroy; make that first call
 * outside stream capture).  Every upload is then one small kernel on `stream`
 * that reads that image through its device mapping: it does not block the
 * calling thread, and unlike a copy-engine transfer it does not queue behind
 * other streams' host<->device copies (e.g. the next batch's inputs).  The
 * upload also clears the status word.
 */
zz_status_t zz_plan_upload(zz_plan_t* plan, void* dev_workspace, size_t bytes, void* stream);

/*
 * Read (and optionally clear) the device status word that the kernels of this
 * plan set: bit 0 (value 1) when a bounded device-side wait gave up instead of
 * hanging, bit 2 (value 4) when the attention read a page_table entry that
 * points outside the pool (those keys were read as zeros).  Synchronises
 * `stream` (a diagnostic, not a hot-path call).  Returns ZZ_ERR_DEVICE_TIMEOUT
 * when bit 0 is set, else ZZ_ERR_INVALID_ARG when bit 2 is set, else ZZ_OK.
 * zz_plan_upload clears the word.  When the plan's last zz_attn_prefill_noalloc
 * call ran on the current device, the status word of the library's static
 * array is read (and cleared) too, and *flags is the OR of both words.
 * ZZ_ERR_INVALID_ARG if the plan was neither uploaded nor used by
 * zz_attn_prefill_noalloc.
 */
zz_status_t zz_plan_device_status(const zz_plan_t* plan, int32_t* flags, int clear, void* stream);

/*
 * Shard rows from natural token order into the rank-ordered padded layout
 * [c*M, row_bytes] (zigzag.py, shard_hidden_states / shard_position_ids for
 * every rank, stacked as _all_gather_reorganized would deliver them).
 * Padding rows are not written.  src: [T, row_bytes], dst: [c*M, row_bytes].
 * row_bytes: a multiple of 4 (16-byte rows and pointers take the wide path);
 * pointers 4-byte aligned.  Position ids of shape [3, T] (mrope) are sharded
 * as rows of their transpose [T, 3].
 */
zz_status_t zz_shard_rows(const zz_plan_t* plan, const void* src, void* dst,
                          int64_t row_bytes, void* stream);

/*
 * Inverse of zz_shard_rows: dst[t] = src[row of token t], rank-ordered padded
 * [c*M, row_bytes] back to token order [T, row_bytes] (zigzag.py,
 * gather_hidden_states after the all-gather: trim, reverse split, cat).
 * Same row/alignment rules as zz_shard_rows.
 */
zz_status_t zz_gather_rows(const zz_plan_t* plan, const void* src, void* dst,
                           int64_t row_bytes, void* stream);

/*
 * One rank's zigzag shard taken from a token-order tensor: dst is that rank's
 * rank-local rows [per_rank_actual_token[rank], row_bytes] (prev blocks of
 * every sequence, then next blocks), src is [T, row_bytes].  This is the
 * take-back that follows a reduction done in token order: each rank keeps its
 * own zigzag rows, picked by token position rather than by rank-major row
 * blocks (sgl-project/sglang pull request #39724, the CP-TP group sharing
 * commit on token-order moves).  ZZ_ERR_INVALID_ARG if rank is outside
 * [0, cp_size).  Same row/alignment rules as zz_shard_rows.
 */
zz_status_t zz_take_back_rows(const zz_plan_t* plan, int rank, const void* src, void* dst,
                              int64_t row_bytes, void* stream);

/*
 * Rerange the all-gathered K and V into the paged pool, in one pass
 * (zigzag.py, _all_gather_reorganized trim + gather_kv_cache + the
 * set_kv_buffer of materialize_full_kv, with unit k/v scales):
 *     k_pool[out_cache_loc[t]] = k_gathered[src_row[t]]  for every token t,
 * and the same for V.
 *   k_gathered, v_gathered: [c*M, h_kv, d] rank-ordered, padded to M per rank.
 *   k_pool, v_pool:         [num_slots, h_kv, d].
 *   out_cache_loc:          [T] int64 pool slots in natural token order.
 * v_gathered and v_pool may both be NULL (one tensor only).  Slots outside
 * [0, num_slots) are skipped, never written.  Bit-exact copy: any dtype whose
 * row h_kv*d*sizeof(dtype) is a multiple of 16 bytes.
 */
zz_status_t zz_rerange_kv_to_pool(const zz_plan_t* plan, const void* k_gathered,
                                  const void* v_gathered, void* k_pool, void* v_pool,
                                  const int64_t* out_cache_loc, int64_t num_slots,
                                  int h_kv, int d, zz_dtype_t dtype, void* stream);

/*
 * zz_rerange_kv_to_pool into an FP8 (E4M3, no infinities, max 448) pool with
 * per-tensor scales (zigzag.py, materialize_full_kv passes layer.k_scale and
 * layer.v_scale to set_kv_buffer):
 *     k_pool[out_cache_loc[t]] = e4m3(k_gathered[src_row[t]] / k_scale)
 * and the same for V.  The division is rounded in fp32; the conversion rounds
 * to nearest even and saturates finite overflow to +-448; NaN stays NaN.
 *   k_gathered, v_gathered: [c*M, h_kv, d] bf16; k_pool, v_pool: [num_slots,
 *   h_kv, d] bytes.  h_kv*d a multiple of 16; scales positive and finite.
 * v_gathered/v_pool may both be NULL.  Slots outside [0, num_slots) are skipped.
 */
zz_status_t zz_rerange_kv_to_pool_fp8(const zz_plan_t* plan, const void* k_gathered,
                                      const void* v_gathered, void* k_pool, void* v_pool,
                                      const int64_t* out_cache_loc, int64_t num_slots,
                                      int h_kv, int d, float k_scale, float v_scale, void* stream);

/* Most destination pools one zz_rerange_push_kv call writes. */
enum { ZZ_MAX_PUSH_DST = 16 };

/*
 * All-gather and rerange fused, push style: rank `rank` writes its own K/V rows
 * straight into the pool of every rank, so no gathered buffer and no separate
 * rerange pass exist (zigzag.py, _all_gather_reorganized + materialize_full_kv:
 * the all-gather of every rank's K/V followed by set_kv_buffer, with unit
 * scales).  For every local row i < per_rank_actual_token[rank] holding
 * natural token t, and every destination j < n_dst:
 *     k_pools[j][out_cache_locs[j][t]] = k_local[i]
 * and the same for V.
 *   k_local, v_local: [>= per_rank_actual_token[rank], h_kv, d] this rank's
 *     rank-local rows (prev blocks of every sequence, then next blocks), on the
 *     calling GPU.
 *   k_pools, v_pools: host arrays of n_dst device pointers, each a pool
 *     [num_slots, h_kv, d] in the calling GPU's address space: its own pool or
 *     a peer's pool mapped with zz_ipc_import (or peer access).  Stores to a
 *     peer travel over NVLink as plain 16-byte stores; no TMA is used.
 *   out_cache_locs: host array of n_dst device pointers to [T] int64 slot maps
 *     readable by the calling GPU (one map may serve every destination).
 * v_local and v_pools may both be NULL (one tensor).  1 <= n_dst <=
 * ZZ_MAX_PUSH_DST.  Slots outside [0, num_slots) are skipped.  The call only
 * enqueues the kernel; the caller orders it against the other ranks both ways:
 *   - read after write: before any rank reads its pool, every rank's push into
 *     it must have completed (e.g. a stream-ordered collective after each
 *     rank's push kernel);
 *   - write after read: before a rank pushes new rows into the pools, every
 *     rank must have finished reading the previous contents of its own pool
 *     (its attention), e.g. a stream-ordered collective after each rank's
 *     attention, or pools used in alternation (double buffering).
 * Bit-exact copy; row h_kv*d*sizeof(dtype) a multiple of 16 bytes and every
 * pointer 16-byte aligned.
 * The pages gather first and rerange after; the push form is this library's
 * own, and on one GPU it equals zz_rerange_kv_to_pool run per rank.
 */
zz_status_t zz_rerange_push_kv(const zz_plan_t* plan, int rank, const void* k_local,
                               const void* v_local, void* const* k_pools, void* const* v_pools,
                               const int64_t* const* out_cache_locs, int n_dst, int64_t num_slots,
                               int h_kv, int d, zz_dtype_t dtype, void* stream);

/* Bytes of an inter-process memory handle (cudaIpcMemHandle_t). */
enum { ZZ_IPC_HANDLE_BYTES = 64 };

/*
 * Export a device buffer to other processes: `handle` (ZZ_IPC_HANDLE_BYTES,
 * caller-owned host memory) names the allocation that contains dev_ptr and
 * *offset is dev_ptr's distance from the allocation's start.  The allocation
 * must come from cudaMalloc (as PyTorch's caching allocator does by default).
 * No counterpart on the pages: it is how the push form reaches peers' pools.
 */
zz_status_t zz_ipc_export(const void* dev_ptr, void* handle, int64_t* offset);

/*
 * Map another process's exported buffer into this process: *base is the
 * mapping of the whole allocation (pass it to zz_ipc_close), *dev_ptr =
 * *base + offset.  Works between processes on the same GPU and between GPUs
 * with peer access.  A handle exported by the calling process itself is
 * rejected by CUDA (ZZ_ERR_CUDA).
 */
zz_status_t zz_ipc_import(const void* handle, int64_t offset, void** base, void** dev_ptr);

/* Unmap a base returned by zz_ipc_import. */
zz_status_t zz_ipc_close(void* base);

/*
 * Zigzag prefill attention for ranks [rank_begin, rank_begin + rank_count)
 * in ONE launch (zigzag.py, run_attention: prev half then next half).  For
 * every rank r, half h, sequence s and query head i:
 *     O = softmax(scale * Q K^T + causal mask) V
 * over keys [0, kv_len_h[s]), query row j of the half sitting at position
 * kv_len_h[s] - Lq + j and seeing keys <= that position; K/V head = i / (h_q/h_kv).
 *   q, out: [rank_count, M, h_q, d] rank-local rows (prev halves from row 0,
 *           next halves from row total_q_prev of that rank); padding rows are
 *           neither read for any valid output nor written.
 *   k_pool, v_pool: [num_slots, h_kv, d]; page_table [bs, max_pages] int32;
 *           slot of key t of sequence s = page_table[s][t/page_size]*page_size
 *           + t%page_size.  Only the first ceil(kv_len/page_size) entries of a
 *           row are read.  An entry whose slots fall outside [0, num_slots)
 *           is not dereferenced: its keys read as zeros and bit 2 of the
 *           plan's status word is set (see zz_plan_device_status).
 *   lse: optional [rank_count, M, h_q] fp32 natural-log sum of exponentials.
 *   softmax_scale <= 0 selects 1/sqrt(d).
 * Errors: ZZ_ERR_INVALID_ARG when h_q % h_kv != 0 (message names "multiple of
 * num_kv_heads"), null or misaligned pointers, rank range outside [0,c);
 * ZZ_ERR_UNSUPPORTED for d not in {64,128}, or for bf16 a page_size that is
 * neither 8, 16, 32, 64 nor a multiple of 128.
 * bf16 runs the tcgen05/TMEM/TMA kernel (fp32 accumulate and softmax): for
 * d = 128 on pairs of CTAs (clusters of two that share each MMA; each CTA
 * loads half of every K and V tile), for d = 64 on single CTAs.  fp32 runs a
 * CUDA-core kernel in full fp32.  The d = 128 kernel is persistent: a running
 * cluster takes the work of clusters of the same launch that have not started
 * (cluster launch control), so the work each cluster does varies from launch
 * to launch, but every output row is computed by one cluster in a fixed order
 * and the result is the same bit for bit.  Launches that share a plan on
 * different streams may run at the same time: they only read the plan's
 * tables, and a status bit either of them sets lands in the plan's one
 * status word.
 */
zz_status_t zz_attn_prefill(const zz_plan_t* plan, int rank_begin, int rank_count,
                            const void* q, const void* k_pool, const void* v_pool,
                            int64_t num_slots, const int32_t* page_table, int max_pages,
                            int page_size, void* out, float* lse, int h_q, int h_kv, int d,
                            float softmax_scale, zz_dtype_t dtype, void* stream);

/*
 * Diagnostic: launch one thread that waits, with the same bounded mbarrier
 * wait every pipeline stage of zz_attn_prefill uses, on a barrier that nothing
 * arrives at.  The wait must give up after `timeout_ns` and the kernel must
 * return normally, leaving the context usable.  Writes dev_status[0] = 1 when
 * the wait gave up (0 if it returned early, which would be a bug) and
 * dev_status[1] = elapsed nanoseconds.  dev_status: 2 x int64 device memory.
 * ZZ_ERR_INVALID_ARG unless 0 < timeout_ns <= 10 s.
 */
zz_status_t zz_debug_wait_timeout(int64_t timeout_ns, int64_t* dev_status, void* stream);

/* Flags of zz_attn_prefill_ex. */
enum { ZZ_ATTN_NONCAUSAL = 1 };

/*
 * zz_attn_prefill with flags.  ZZ_ATTN_NONCAUSAL drops the causal mask: every
 * query row of a half attends to all keys of its sequence, prefix included
 * (kv_len_next of rank 0, i.e. prefix + the whole extend length).  This is
 * the local-Q / global-KV attention of an AllGather-KV layout, which is
 * non-causal ("Compose Ulysses with AllGather-KV as a 2D SP topology",
 * vllm-omni pull request #7937: local Q against the gathered global K/V).
 * flags = 0 is exactly zz_attn_prefill.  Unknown flag bits: ZZ_ERR_INVALID_ARG.
 */
zz_status_t zz_attn_prefill_ex(const zz_plan_t* plan, int rank_begin, int rank_count,
                               const void* q, const void* k_pool, const void* v_pool,
                               int64_t num_slots, const int32_t* page_table, int max_pages,
                               int page_size, void* out, float* lse, int h_q, int h_kv, int d,
                               float softmax_scale, zz_dtype_t dtype, uint32_t flags, void* stream);

/*
 * zz_attn_prefill without a workspace (bf16, causal).  The zigzag pages have
 * no counterpart to this call.  It is for callers that cannot hand the library
 * device memory of their own: a host runtime whose device memory all belongs
 * to its own arena and that gives plug-ins no allocation call, or a process
 * that must keep its device footprint fixed after start-up and so may not
 * call cudaMalloc (or an allocator that ends in it) per request.
 *
 * Same arguments and results as zz_attn_prefill (bit for bit: the same kernel
 * reads the same tables).  zz_plan_upload is not needed.  The half table, the
 * work list and a status word live in a file-scope __device__ array of 1 MiB
 * inside the library instead of a workspace; every GPU that loads libzz holds
 * that array until the process exits.  The call allocates nothing, host or
 * device: it calls no cudaMalloc, cudaMallocHost or cudaFree.  The tables
 * travel to the array as kernel parameters of small copy launches (1 per
 * 32 640 bytes of tables) enqueued on `stream` before the attention launch,
 * so the call neither waits for the stream nor blocks the calling thread.
 *   - Plans whose tables need more than 1 MiB (half table plus work list,
 *     about 130 000 work items) are rejected with ZZ_ERR_INVALID_ARG, like
 *     every other invalid call, before anything is enqueued.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - All calls share the one array and the last call's tables stay in it.
 *     Each call clears the status word before its attention launch.  Calls
 *     whose work overlaps on the GPU (other streams, other host threads) race
 *     on the array and must be serialised by the caller.
 *   - Device-side errors (a bounded wait that gave up, a page_table entry
 *     outside the pool) set the array's status word; zz_plan_device_status on
 *     the same plan, with the same device current, reads and clears it.
 */
zz_status_t zz_attn_prefill_noalloc(const zz_plan_t* plan, int rank_begin, int rank_count,
                                    const void* q, const void* k_pool, const void* v_pool,
                                    int64_t num_slots, const int32_t* page_table, int max_pages,
                                    int page_size, void* out, float* lse, int h_q, int h_kv, int d,
                                    float softmax_scale, zz_dtype_t dtype, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* ZZ_H_ */
