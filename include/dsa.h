/*
 * dsa.h -- C ABI of libdsa_b200: DeepSeek Sparse Attention (DSA) adapted to a GQA
 * decoder, for NVIDIA B200 (sm_100a).
 *
 * The method (Keye-VL-2.0 technical-report summary, mqxn.cn/news/1966, section 1):
 * a lightweight "Lightning Indexer" with one MQA-shared indexer key per position scores
 * every visible context position for each query token; each token keeps its top-k
 * (k = 2048 in the report) positions; GQA attention then runs only over those
 * positions, so attention cost falls from O(L^2) to O(L*k).  The indexer is trained in a
 * dense warm-up stage by a KL divergence to the full attention distribution, then the
 * whole model trains through sparse attention (same section).  Section 8 of the same
 * summary asks for a deterministic top-k and a DSA-specific decode path.
 *
 * Shared conventions for every call below
 * ---------------------------------------
 * - Pointers named as device data are caller-owned device pointers.  The library never
 *   allocates device memory, never synchronises the device, and keeps no pointer after
 *   the work it enqueued has completed.  Scratch memory, where a call needs it, is a
 *   caller-provided workspace whose size the matching *_workspace_size() call returns.
 * - Tensors are dense, row-major (last index fastest).  "bf16" is the 16-bit bfloat16
 *   bit pattern.  Every base pointer must be 16-byte aligned.
 * - Varlen packing: B sequences are concatenated along the token axis.
 *   cu_seqlens_q / cu_seqlens_k are device int32 arrays [B+1] of offsets (0 first,
 *   non-decreasing).  Query row r belongs to the sequence b with
 *   cu_seqlens_q[b] <= r < cu_seqlens_q[b+1]; its sequence-local index is
 *   i = r - cu_seqlens_q[b]; Lq = cu_seqlens_q[b+1]-cu_seqlens_q[b], Lk likewise.
 * - Causality is bottom-right aligned: query i sees the sequence-local key positions
 *   0 .. vis-1 with vis = clamp(i + Lk - Lq + 1, 0, Lk).  Prefill uses Lq == Lk (query i
 *   sees keys 0..i); decode uses Lq == 1 (the query sees its whole cache).
 * - Key positions in `indices` are sequence-local (0-based within the sequence); -1 marks
 *   an unused slot.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call only
 *   enqueues work on it and returns; errors of that work surface through the stream.
 * - Return value: DSA_OK, or a negative dsa_status.  Argument errors are detected on the
 *   host before anything is enqueued.  DSA_ERR_CUDA reports a failed launch.
 * - Device-side waits (pipeline barriers inside kernels) are bounded: a wait that runs
 *   out records DSA_ERR_TIMEOUT in a device status word that dsa_get_device_status()
 *   reads, and the kernel returns instead of hanging.
 */
#ifndef DSA_B200_H
#define DSA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define DSA_API __attribute__((visibility("default")))
#else
#define DSA_API
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = -1, /* a null pointer, bad size, misaligned pointer, bad ld */
  DSA_ERR_UNSUPPORTED = -2, /* a valid shape this build has no kernel for */
  DSA_ERR_WORKSPACE = -3,   /* workspace missing or smaller than *_workspace_size() */
  DSA_ERR_CUDA = -4,        /* a CUDA runtime call or kernel launch failed */
  DSA_ERR_TIMEOUT = -5      /* a bounded device-side wait ran out (device status word) */
} dsa_status;

/* How dsa_index_topk finds the selected sets. */
typedef enum {
  DSA_PATH_AUTO = 0,      /* the fused indexer -> top-k where it is the faster, else the separate passes */
  DSA_PATH_SEPARATE = 1,  /* always the separate passes: dsa_index then dsa_topk per row chunk */
  DSA_PATH_FUSED = 2      /* the fused form wherever its shapes allow (the same sets, whatever the speed) */
} dsa_path;

/* Human-readable name of a dsa_status value.  Never returns NULL. */
DSA_API const char* dsa_status_string(int status);

/* Library ABI version (major*10000 + minor*100 + patch). */
DSA_API int dsa_version(void);

/* The cudaError_t code behind the most recent DSA_ERR_CUDA returned on this host thread
 * (0 if none), and, if message is not NULL, its text (a static string). */
DSA_API int dsa_last_cuda_error(const char** message);

/* Reads and clears the device status word on the current device.  Synchronises the
 * device first (a debugging helper, not for hot paths).  *status_out receives DSA_OK or
 * DSA_ERR_TIMEOUT; *detail_out (may be NULL) receives a kernel-specific code of where
 * the wait ran out.  Returns DSA_ERR_CUDA if the synchronisation itself failed. */
DSA_API int dsa_get_device_status(int* status_out, int* detail_out);

/* Self-test of the bounded device waits (a diagnostic; the method has no counterpart).
 * Launches one small kernel that waits, with the same bounded-wait routine the pipelined
 * kernels use, on a barrier that nothing arrives at, for limit_ns nanoseconds (1 ns .. 1 s);
 * the wait then gives up, records DSA_ERR_TIMEOUT with detail code 900 in the device status
 * word, and the kernel returns.  Read the result with dsa_get_device_status().  The kernel
 * holds no copies, tensor-core work or tensor memory when it gives up, so the context stays
 * usable.  Returns DSA_ERR_INVALID_ARG for a limit outside that range. */
DSA_API int dsa_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* ---------------------------------------------------------------------------------
 * (1) Lightning indexer scores.  Source: report summary section 1 (an MQA-shared
 * scout scans all positions).  For every query row r in [row_begin, row_end):
 *     scores[(r-row_begin)*ld_scores + s] = sum_j w[r,j] * max(0, q_idx[r,j,:] . k_idx[k0+s,:])
 * for s in [0, vis(r)), where k0 = cu_seqlens_k[b].  Products are bf16 x bf16 with fp32
 * accumulation (tensor cores); ReLU, the w-weighting and the head sum are fp32.
 *   q_idx  device bf16 [total_q, H_I, d_I]   indexer queries
 *   k_idx  device bf16 [total_k, d_I]        indexer keys (one per position, shared)
 *   w      device bf16 [total_q, H_I]        per-token indexer head weights
 *   total_q, total_k  host: rows of q_idx/w and of k_idx (cu_seqlens_q[B], cu_seqlens_k[B])
 *   max_seqlen_q  host int >= every Lq (used only to size the launch)
 *   scores device fp32 [row_end-row_begin, ld_scores]; only columns s < vis(r) are
 *          written, the rest is left untouched.  ld_scores >= the longest Lk and a
 *          multiple of 4.
 * Supported: (H_I, d_I) in {(64,128), (32,128), (16,128), (4,32), (8,64)}.
 * ------------------------------------------------------------------------------- */
DSA_API int dsa_index(const void* q_idx, const void* k_idx, const void* w,
                      const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                      int64_t total_q, int64_t total_k, int max_seqlen_q, int max_seqlen_k,
                      int H_I, int d_I, int64_t row_begin, int64_t row_end, float* scores,
                      int64_t ld_scores, void* stream);

/* ---------------------------------------------------------------------------------
 * (2) Deterministic top-k.  Source: report summary section 1 (each token keeps its 2048
 * most relevant positions) and section 8 (the selection must be deterministic so that
 * training and inference select the same set).  For each row r in [row_begin, row_end)
 * the selected set is the k largest scores[(r-row_begin)*ld_scores + s], s < vis(r),
 * where equal scores are ranked by the lower position and +0.0 equals -0.0.  If
 * vis(r) <= k every visible position is selected.  Output:
 *   indices device int32 [row_end-row_begin, k]: the selected positions in ascending
 *           order, then -1 in the unused slots.  Bit-for-bit reproducible.
 *   workspace  optional caller-owned device scratch (16-byte aligned) of at least
 *           dsa_topk_workspace_size(row_end-row_begin, ld_scores, k) bytes.  That size is
 *           non-zero only for a few long rows (the decode shape), where the workspace lets
 *           the call spread each row over many blocks; NULL (or a smaller buffer) selects
 *           a method that needs none, with the same result.  Its contents on entry do not
 *           matter; it must not be shared with work that overlaps this call on the GPU.
 * Supported: 1 <= k <= 4096.
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_topk_workspace_size(int64_t rows, int64_t ld_scores, int k);
DSA_API int dsa_topk(const float* scores, int64_t ld_scores, const int32_t* cu_seqlens_q,
                     const int32_t* cu_seqlens_k, int batch, int64_t row_begin, int64_t row_end,
                     int k, int32_t* indices, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (2b) Indexer and top-k together: the selected sets of the query rows [row_begin,
 * row_end), i.e. (2) applied to the scores of (1), without handing the scores to the
 * caller.  Source: report summary section 1 (the indexer scans every position; each token
 * keeps its k best) and section 8 (deterministic top-k).  Rows are processed in chunks of
 * at most `chunk_rows`.
 *   indices device int32 [row_end-row_begin, k]: as (2), ascending, -1 padded, bit-for-bit
 *           the sets (2) returns on the scores of (1) (the same scores, the same tie rule).
 *           While the call runs, slots k-2 and k-1 of each row hold that row's working state
 *           (the fused form's bound and candidate count).
 *   path    DSA_PATH_AUTO: for (H_I, d_I) in {(64,128), (32,128)} with score rows of
 *           65536 to 524288 positions and room for 2k candidates per row in the scratch,
 *           the fused form: the indexer first scores every S-th key (S a power of two,
 *           about 1024 samples per full row) to bound each row's k-th largest score from
 *           below, then scores every key again but keeps only the (score, position) pairs
 *           that reach the bound, and an exact select over those pairs writes the sets;
 *           rows the bound failed for (fewer than k pairs kept, or more than fit) are
 *           recomputed in full and selected by the exact method.  For one self-attention
 *           sequence (batch 1, total_q == total_k) the leading chunks, whose rows see few
 *           positions, still take the separate passes.  DSA_PATH_FUSED takes the fused
 *           form whenever the shapes and scratch allow it, whatever the row lengths.
 *           Otherwise, and with DSA_PATH_SEPARATE, (1) then (2) per chunk.
 *   workspace  device scratch of dsa_index_topk_workspace_size(chunk_rows, max_seqlen_k)
 *           bytes (16-byte aligned): one chunk of fp32 score rows plus 256 bytes.
 * Supported: the shapes of (1); 1 <= k <= 4096.
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_index_topk_workspace_size(int64_t chunk_rows, int max_seqlen_k);
DSA_API int dsa_index_topk(const void* q_idx, const void* k_idx, const void* w, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, int batch, int64_t total_q, int64_t total_k,
                           int max_seqlen_q, int max_seqlen_k, int H_I, int d_I, int k, int64_t row_begin,
                           int64_t row_end, int64_t chunk_rows, int path, int32_t* indices, void* workspace,
                           size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (3) Sparse GQA attention, prefill/varlen.  Source: report summary section 1 (attention
 * only over the selected positions, O(L*k); GQA adapted to DSA: the one selected set of a
 * token is shared by all its query heads).  For row r, head h, KV head g = h/(Hq/Hkv),
 * set S = the entries of indices[r,:] inside [0, vis(r)) (a -1 slot, or a position the
 * row cannot see, including one past the end of its sequence, is ignored):
 *     O[r,h,:]  = sum_{s in S} softmax_s(scale * Q[r,h,:].K[k0+s,g,:]) V[k0+s,g,:]
 *     lse[r,h]  = natural log of sum_{s in S} exp(scale * Q[r,h,:].K[k0+s,g,:])
 * An empty set gives O = 0 and lse = -inf.
 *   Q  device bf16 [total_q, Hq, d];  K, V device bf16 [total_k, Hkv, d]
 *   indices device int32 [total_q, k] (as produced by dsa_topk)
 *   O  device bf16 [total_q, Hq, d];  lse device fp32 [total_q, Hq] (may be NULL)
 * Supported: d in {64, 128}; Hq/Hkv in {4, 8}; k a multiple of 16, <= 4096.
 * ------------------------------------------------------------------------------- */
DSA_API int dsa_sparse_attn_prefill(const void* Q, const void* K, const void* V,
                                    const int32_t* indices, const int32_t* cu_seqlens_q,
                                    const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                                    int Hq, int Hkv, int d, int k, float scale, void* O,
                                    float* lse, void* stream);

/* ---------------------------------------------------------------------------------
 * (3b) The operation of (3) on the tensor cores, tile by tile over the selected slots.
 * Source: report summary section 1 (attention over the selected positions, one set per
 * token shared by the query heads of its KV group).  Same inputs, outputs, validity rule
 * and rounding bound as (3); a separate entry point because (3)'s warp-level kernel is the
 * faster one on B200 at the shapes measured (the selected K/V rows come from L2 at a
 * latency of microseconds, and its per-warp rings keep more bytes in flight than this
 * kernel's shared tile rings).  Per (row, KV head), 128 selected slots at a time: K and V
 * rows are gathered into shared memory, S^T = K.Q^T and O^T += V^T.P^T run as tcgen05 MMAs
 * with M = 128 slots and the accumulators in tensor memory.
 * Supported: d = 128, Hq = 8 Hkv, k a multiple of 16 and <= 2048, indices 16-byte aligned
 * (DSA_ERR_UNSUPPORTED otherwise).
 * ------------------------------------------------------------------------------- */
DSA_API int dsa_sparse_attn_prefill_tc(const void* Q, const void* K, const void* V,
                                       const int32_t* indices, const int32_t* cu_seqlens_q,
                                       const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                                       int Hq, int Hkv, int d, int k, float scale, void* O,
                                       float* lse, void* stream);

/* ---------------------------------------------------------------------------------
 * (3c) Sparse GQA attention, prefill, with adjacent-query reuse.  Source: report summary
 * section 8 (adjacent queries select highly similar top-k sets; the sets of adjacent
 * queries are deduplicated and the attention kernel applies a mask laid out for the MMA's
 * threads: at 128K and k = 2048, 16 adjacent queries touch about 8000 distinct positions
 * instead of 16 x 2048).  Same inputs, outputs and result as (3).  Per block of 16
 * consecutive rows of a sequence (rows i0 .. i0+15 of sequence b, i0 a multiple of 16), the
 * sorted union of the rows' sets S (as defined in (3)) is formed.  A block whose union
 * holds at most 12288 positions runs on tensor cores over the union, gathered 128 positions
 * at a time (each K and V row loaded once for the block's 16 rows x 8 query heads), with a
 * per-(row, position) selection mask on the logits; the rows of the other blocks run the
 * gather kernel of (3).  O and lse agree with (3) within the same rounding bound.
 *   max_seqlen_k: host int >= every Lk; total_k: rows of K and V.
 *   workspace: dsa_sparse_attn_prefill_reuse_workspace_size(total_q, Hq, batch,
 *     max_seqlen_k) bytes, 16-byte aligned (DSA_ERR_WORKSPACE if NULL or smaller);
 *     about 75 KiB per block of 16 rows at max_seqlen_k >= 12288.
 *   lse may be NULL (the workspace holds it then).
 *   block_union: device int32 [(total_q + 15) / 16 + batch] or NULL: receives per block,
 *     numbered over the sequences in order (ceil(Lq_b / 16) blocks for sequence b), the
 *     size of its union (also where it exceeds 12288); the entries past the last block are
 *     0.  Where no union is formed (see below) every entry is -1.
 *   The tensor-core form needs d = 128, Hq = 8 Hkv and max_seqlen_k <= 262144; for other
 *   supported shapes every row runs the gather kernel of (3).
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_sparse_attn_prefill_reuse_workspace_size(int64_t total_q, int Hq, int batch,
                                                            int max_seqlen_k);
DSA_API int dsa_sparse_attn_prefill_reuse(const void* Q, const void* K, const void* V,
                                          const int32_t* indices, const int32_t* cu_seqlens_q,
                                          const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                                          int64_t total_k, int max_seqlen_k, int Hq, int Hkv, int d,
                                          int k, float scale, void* O, float* lse,
                                          int32_t* block_union, void* workspace,
                                          size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (4) Sparse GQA attention, decode.  Source: report summary section 8 (a decode path
 * specific to DSA).  Same arithmetic as (3) for one query row per sequence (Lq == 1), with
 * the k selected keys split over several thread blocks and their partial softmax states
 * merged by log-sum-exp.  The query of sequence b sees its whole cache (vis = Lk_b):
 * entries of indices outside [0, Lk_b) are ignored like -1.
 *   Q device bf16 [batch, Hq, d]; K, V device bf16 [total_k, Hkv, d] (sequence b's cache
 *   is rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1); indices device int32 [batch, k];
 *   O device bf16 [batch, Hq, d]; lse device fp32 [batch, Hq] (may be NULL).
 *   workspace: device scratch of dsa_sparse_attn_decode_workspace_size() bytes.
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_sparse_attn_decode_workspace_size(int batch, int Hq, int d, int k);
DSA_API int dsa_sparse_attn_decode(const void* Q, const void* K, const void* V,
                                   const int32_t* indices, const int32_t* cu_seqlens_k, int batch,
                                   int Hq, int Hkv, int d, int k, float scale, void* O, float* lse,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (4b) Decode attention without any caller workspace.  The paper has no counterpart: this
 * is a library convenience for callers that cannot allocate device memory where they run
 * decode (a host that owns a preallocated pool and offers plugins no allocator, or a
 * latency-critical loop that must not call cudaMalloc) and have no scratch buffer to pass.
 * Same inputs, outputs and arithmetic as (4); the split-K scratch lives in a fixed 8 MiB
 * device array inside the library, held on every GPU that loads the library until exit.
 *   - Arguments are checked as in (4), in the same order (DSA_ERR_INVALID_ARG, then
 *     DSA_ERR_UNSUPPORTED); then it returns DSA_ERR_WORKSPACE when (4) would need more than
 *     8 MiB of scratch, i.e. when dsa_sparse_attn_decode_workspace_size(batch, Hq, d, k) >
 *     8388608 (at d = 128 and k = 2048 that allows batch * Hq <= 992).
 *   - Device ordinals 0..63 are served; on a device numbered 64 or more it returns
 *     DSA_ERR_UNSUPPORTED.
 *   - The first call on a device looks up the array's device address with that device
 *     current (a one-time set-up); make that first call before any stream capture.
 *   - All calls on a device share the one array; calls that can overlap on the GPU race
 *     and must be ordered by the caller.  Nothing in it needs clearing between calls.
 * ------------------------------------------------------------------------------- */
DSA_API int dsa_sparse_attn_decode_noalloc(const void* Q, const void* K, const void* V,
                                           const int32_t* indices, const int32_t* cu_seqlens_k,
                                           int batch, int Hq, int Hkv, int d, int k, float scale,
                                           void* O, float* lse, void* stream);

/* ---------------------------------------------------------------------------------
 * (5) Whole DSA forward for prefill: (2b) with DSA_PATH_AUTO over row chunks of at most
 * `chunk_rows` query rows (bounding the fp32 score scratch), then (3).
 *   max_seqlen_q / max_seqlen_k: host ints >= every Lq / Lk.
 *   indices device int32 [total_q, k] receives the selected sets.
 *   workspace: dsa_prefill_workspace_size(chunk_rows, max_seqlen_k) bytes.
 *   The attention step, with the same O and lse (within the same rounding bound) whichever
 *   runs: when the selected sets are dense (d = 128, Hq = 8 Hkv, 8 k >= max_seqlen_k), lse
 *   is not NULL and the score scratch also holds total_q * ceil(max_seqlen_k / 128) * 16
 *   bytes of selection bits plus total_q * Hq * 4 bytes, masked dense tensor-core passes;
 *   else, when the score scratch holds the workspace of (3c), (3c); else the gather kernel
 *   of (3).
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_prefill_workspace_size(int64_t chunk_rows, int max_seqlen_k);
DSA_API int dsa_prefill(const void* q_idx, const void* k_idx, const void* w, const void* Q,
                        const void* K, const void* V, const int32_t* cu_seqlens_q,
                        const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                        int64_t total_k, int max_seqlen_q,
                        int max_seqlen_k, int Hq, int Hkv, int d, int H_I, int d_I, int k,
                        float scale, int64_t chunk_rows, int32_t* indices, void* O, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (5b) Whole DSA forward for prefill from HOST buffers.  Same computation as (5): per row
 * chunk of at most `chunk_rows` rows, (2b) with DSA_PATH_AUTO, then (3c) on the chunk's rows
 * (its query offsets shifted to the chunk); the O rows agree with (5)'s sparse path bit for
 * bit.  The inputs are copied in and O copied out inside the call's stream order: per
 * chunk, the key-side rows (k_idx, K, V) its rows can see that earlier chunks did not need,
 * then its q_idx, w and Q rows, so that a chunk's copies overlap its neighbours' kernels;
 * each chunk's O rows are copied back as soon as they are ready.
 *   q_idx, k_idx, w, Q, K, V, cu_seqlens_q, cu_seqlens_k: HOST memory, layouts as in (5)
 *     (pinned memory for the copies to overlap the kernels);
 *   O: HOST bf16 [total_q, Hq, d], written when the work enqueued on `stream` completes;
 *   workspace: DEVICE memory of dsa_prefill_host_workspace_size() bytes, 16-byte aligned
 *     (DSA_ERR_WORKSPACE if NULL or smaller): it holds the device copies of the inputs, the
 *     selected sets, O, and the scratch of (2b) and (3c).
 * The copies run on two copy streams the library creates on first use on each device (and
 * keeps); `stream` is made to wait for them, so synchronising `stream` covers the whole
 * call, including the copy of O.  Host pointers must stay valid until then.  Devices
 * numbered 64 or more return DSA_ERR_UNSUPPORTED.
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_prefill_host_workspace_size(int batch, int64_t total_q, int64_t total_k,
                                               int max_seqlen_k, int Hq, int Hkv, int d, int H_I,
                                               int d_I, int k, int64_t chunk_rows);
DSA_API int dsa_prefill_host(const void* q_idx, const void* k_idx, const void* w, const void* Q,
                             const void* K, const void* V, const int32_t* cu_seqlens_q,
                             const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                             int64_t total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv,
                             int d, int H_I, int d_I, int k, float scale, int64_t chunk_rows,
                             void* O, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (6) Whole DSA decode step: (1) with one query row per sequence over its cache, (2),
 * then (4).  q_idx device bf16 [batch, H_I, d_I]; w device bf16 [batch, H_I]; k_idx
 * device bf16 [total_k, d_I]; Q/K/V/O as in (4); indices device int32 [batch, k].
 *   workspace: dsa_decode_workspace_size(batch, max_seqlen_k, Hq, d, k) bytes.
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_decode_workspace_size(int batch, int max_seqlen_k, int Hq, int d, int k);
DSA_API int dsa_decode(const void* q_idx, const void* k_idx, const void* w, const void* Q,
                       const void* K, const void* V, const int32_t* cu_seqlens_k, int batch,
                       int64_t total_k, int max_seqlen_k, int Hq, int Hkv, int d, int H_I, int d_I, int k,
                       float scale, int32_t* indices, void* O, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (7) Sparse attention backward.  Source: report summary section 1, sparse-adaptation
 * stage (the whole model trains through sparse attention); QbitAI launch article
 * (news.chathome.org): varlen DSA training kernels.  For the fixed sets in `indices` and
 * the forward's O and lse:
 *     P[s] = exp(scale*Q[r,h].K[s,g] - lse[r,h]),  D = dO[r,h].O[r,h]
 *     dS[s] = P[s] * (dO[r,h].V[s,g] - D)
 *     dQ[r,h] = scale * sum_s dS[s] K[s,g]
 *     dK[s,g] += scale * dS[s] Q[r,h],   dV[s,g] += P[s] dO[r,h]   (over all r, h)
 *   dQ device bf16 [total_q, Hq, d]; dK, dV device bf16 [total_k, Hkv, d].
 *   max_seqlen_k: the longest sequence of keys (bounds the selected positions).
 *   Two paths, chosen from the shapes: when d = 128, Hq = 8 Hkv and 8 k >= max_seqlen_k
 *   (dense selected sets), a masked dense pass on tensor cores: each key's dK and dV are
 *   written once, dQ is accumulated in fp32 (float atomics); otherwise one warp per (token,
 *   KV head) over its selected keys, with dK and dV accumulated in fp32 (float atomics).
 *   Float atomics make the summation order, and so the last bits, vary between runs; every
 *   fp32 accumulator is rounded to bf16 once at the end.  As in (3), -1 slots and
 *   positions outside [0, vis(r)) are ignored.
 *   workspace: dsa_sparse_attn_bwd_workspace_size(total_q, total_k, Hq, Hkv, d,
 *   max_seqlen_k) bytes (enough for either path).
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_sparse_attn_bwd_workspace_size(int64_t total_q, int64_t total_k, int Hq,
                                                  int Hkv, int d, int max_seqlen_k);
DSA_API int dsa_sparse_attn_prefill_bwd(const void* Q, const void* K, const void* V,
                                        const void* O, const void* dO, const float* lse,
                                        const int32_t* indices, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                                        int64_t total_k, int max_seqlen_k, int Hq, int Hkv, int d,
                                        int k, float scale, void* dQ, void* dK, void* dV,
                                        void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (8) Indexer KL loss (dense warm-up).  Source: report summary section 1 (the indexer is
 * trained to match the full attention distribution by minimising a KL divergence, with
 * dense attention kept).  For each query row t with visible keys s < vis(t):
 *     p[t,s] = (1/Hq) sum_h softmax_s(scale * Q[t,h].K[s,g(h)])   (target, a constant)
 *     q[t,s] = softmax_s(I[t,s]),  I = the indexer score of (1)
 *     kl[t]  = sum_s p log(p/q)  (0 log 0 = 0);   *loss = (1/total_q) sum_t kl[t]
 * and the gradients of *loss:
 *     dw[t,j]       = sum_s g[t,s] max(0, x[t,j,s])
 *     dq_idx[t,j,:] = w[t,j] sum_s g[t,s] [x[t,j,s] > 0] k_idx[s,:]
 *     dk_idx[s,:]   = sum_t sum_j g[t,s] w[t,j] [x[t,j,s] > 0] q_idx[t,j,:]
 * with g = (q - p)/total_q and x[t,j,s] = q_idx[t,j].k_idx[s].
 *   loss device fp32 [1]; kl device fp32 [total_q]; dq_idx bf16 [total_q,H_I,d_I];
 *   dk_idx bf16 [total_k, d_I]; dw bf16 [total_q, H_I].
 *   workspace: dsa_indexer_kl_loss_workspace_size(...) bytes.
 * Supported: H_I in {16, 32, 64} with d_I = 128; d in {64, 128}; Hq/Hkv in {4, 8}; Hkv <= 8;
 * self-attention packing (Lq == Lk per sequence).  dk_idx is accumulated in fp32 in the
 * workspace from per-(key tile, row block) partials added in a fixed order (no atomics:
 * bit-reproducible).
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_indexer_kl_loss_workspace_size(int64_t total_q, int64_t total_k,
                                                  int max_seqlen_k, int Hq, int H_I, int d_I,
                                                  int64_t chunk_rows, int batch);
DSA_API int dsa_indexer_kl_loss(const void* Q, const void* K, const void* q_idx, const void* k_idx,
                                const void* w, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                                int64_t total_k, int max_seqlen_q, int max_seqlen_k, int Hq,
                                int Hkv, int d, int H_I, int d_I, float scale, int64_t chunk_rows,
                                float* loss, float* kl, void* dq_idx, void* dk_idx, void* dw,
                                void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------
 * (9) Indexer KL loss, sparse-adaptation form.  Source: report summary section 1, second
 * training stage (the whole model trains through sparse attention; the indexer keeps
 * learning from the attention over the positions it selects).  As (8) with every sum over
 * the visible positions replaced by a sum over row t's selected set S_t (the entries of
 * indices[t,:] inside [0, vis(t)), -1 unused):
 *     p[t,s] = (1/Hq) sum_h softmax_{s in S_t}(scale * Q[t,h].K[s,g(h)])   (a constant)
 *     q[t,s] = softmax_{s in S_t}(I[t,s]),  kl[t] = sum_{s in S_t} p log(p/q)
 *     *loss = (1/total_q) sum_t kl[t]
 * and the gradients of (8) with g[t,s] = (q - p)/total_q on S_t and 0 elsewhere.
 *   indices device int32 [total_q, k] (as produced by dsa_topk / dsa_index_topk).
 *   workspace: dsa_indexer_kl_loss_sparse_workspace_size(...) bytes (that of (8) plus the
 *   selection bits, total_q * ceil(max_seqlen_k / 128) * 16 bytes).
 * Supported: d = 128 with Hq = 8 Hkv, Hkv <= 4; H_I in {16, 32, 64} with d_I = 128; k <= 4096;
 * Lq == Lk per sequence.  Deterministic like (8).
 * ------------------------------------------------------------------------------- */
DSA_API size_t dsa_indexer_kl_loss_sparse_workspace_size(int64_t total_q, int64_t total_k, int max_seqlen_k,
                                                         int Hq, int H_I, int d_I, int64_t chunk_rows, int batch);
DSA_API int dsa_indexer_kl_loss_sparse(const void* Q, const void* K, const void* q_idx, const void* k_idx,
                                       const void* w, const int32_t* indices, int k,
                                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                       int64_t total_q, int64_t total_k, int max_seqlen_q, int max_seqlen_k,
                                       int Hq, int Hkv, int d, int H_I, int d_I, float scale,
                                       int64_t chunk_rows, float* loss, float* kl, void* dq_idx, void* dk_idx,
                                       void* dw, void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DSA_B200_H */
