// C ABI of libdsa_b200 (declared in include/dsa.h): argument checks, launch selection,
// and the chunked prefill / decode pipelines.  Every check happens on the host before
// anything is enqueued; the library never allocates and never synchronises.
#include <algorithm>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace dsa {
__global__ void iota_kernel(int* dst, int n, int step) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i <= n) dst[i] = i * step;
}

// Self-test of the bounded wait every pipelined kernel uses: one thread waits, through the
// same mbar_wait, on a shared-memory barrier that nothing ever arrives at.  The wait runs
// out after limit_ns and records DSA_ERR_TIMEOUT with the site code kSelftestWaitSite; the
// kernel then returns.  No copy, tensor-core or tensor-memory work is in flight.
constexpr int kSelftestWaitSite = 900;
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, kSelftestWaitSite, limit_ns);
  __syncthreads();
}
}  // namespace dsa

namespace dsa_host {

// kernels implemented in the sibling translation units of this unity build
int indexer_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                   int batch, long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k,
                   int H_I, int d_I, long long row_begin, long long row_end, float* scores, long long ld,
                   cudaStream_t stream);
size_t topk_ws_bytes(long long rows, long long max_vis);
int topk_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                long long row_begin, long long row_end, int k, int* indices, int max_vis, void* ws,
                size_t ws_bytes, cudaStream_t stream);
int sparse_attn_prefill_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                               const int* cu_k, int batch, long long total_q, int Hq, int Hkv, int d, int k,
                               float scale, void* O, float* lse, cudaStream_t stream, const uint8_t* skip_rows);
bool sa_gather_tc_eligible(int Hq, int Hkv, int d, int k, const void* indices);
int sa_gather_tc_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                        const int* cu_k, int batch, long long total_q, int Hq, int Hkv, int k, float scale, void* O,
                        float* lse, cudaStream_t stream, const uint8_t* skip_rows);
size_t sa_block_reuse_scratch_bytes(long long total_q, int Hq, int batch, int max_seqlen_k, int max_chunks);
bool sa_block_reuse_eligible(int Hq, int Hkv, int d, int max_seqlen_k);
int sa_block_reuse_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                          const int* cu_k, int batch, long long total_q, long long total_k, int Hq, int Hkv, int k,
                          int max_seqlen_k, int max_chunks, float scale, void* O, float* lse, void* ws,
                          int* ucount_out, cudaStream_t s);
// At most this many chunks of 128 positions in a 16-row block's union for the tensor-core
// passes (union form); the cost rule in sparse_attn_tc.cu decides below that.
constexpr int kUnionMaxChunks = 96;
size_t decode_workspace_bytes(int batch, int Hq, int d, int k);
int sparse_attn_decode_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_k,
                              int batch, int Hq, int Hkv, int d, int k, float scale, void* O, float* lse,
                              void* ws, cudaStream_t stream);

size_t sparse_attn_bwd_workspace_bytes(long long total_k, int Hkv, int d);
bool sa_bwd_tc_eligible(int Hq, int Hkv, int d, int k, int max_seqlen_k);
bool sa_fwd_tc_eligible(int Hq, int Hkv, int d, int k, int max_seqlen_k);
size_t sa_fwd_tc_scratch_bytes(long long total_q, int Hq, int max_seqlen_k);
int sa_fwd_tc_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                     const int* cu_k, int batch, long long total_q, long long total_k, int Hq, int Hkv, int k,
                     int max_seqlen_k, float scale, void* O, float* lse, void* mask_ws, cudaStream_t s);
size_t sa_bwd_tc_workspace_bytes(long long total_q, int Hq, int max_seqlen_k);
int sa_bwd_tc_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* lse,
                     const int* indices, const int* cu_q, const int* cu_k, int batch, long long total_q,
                     long long total_k, int Hq, int Hkv, int k, int max_seqlen_k, float scale, void* dQ, void* dK,
                     void* dV, void* ws, cudaStream_t s);
int sparse_attn_bwd_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                           const float* lse, const int* indices, const int* cu_q, const int* cu_k, int batch,
                           long long total_q, long long total_k, int Hq, int Hkv, int d, int k, float scale,
                           void* dQ, void* dK, void* dV, void* ws, cudaStream_t stream);

size_t index_topk_workspace_bytes(long long chunk_rows, int max_seqlen_k);
int index_topk_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                      int batch, long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k, int H_I,
                      int d_I, int k, long long row_begin, long long row_end, long long chunk_rows, int* indices,
                      void* ws, int fused, cudaStream_t stream);

struct KLWorkspace;
size_t kl_workspace_bytes(long long T, long long Tk, int max_seqlen_k, int Hq, int H_I, int d_I, long long chunk_rows,
                          int batch, bool sparse);
int indexer_kl_loss_launch(const void* Q, const void* K, const void* q_idx, const void* k_idx, const void* w,
                           const int* cu_q, const int* cu_k, int batch, long long T, long long Tk,
                           int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d, int H_I, int d_I,
                           float scale, long long chunk_rows, float* loss, float* kl, void* dq, void* dk, void* dw,
                           void* ws, cudaStream_t s, const int* indices, int k);

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

int make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint64_t row_pitch_bytes,
                      uint32_t box_rows, uint32_t box_cols, int swizzle_bytes) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return DSA_ERR_CUDA;
  if (rows == 0) rows = 1;  // an empty operand is never read; keep the descriptor valid
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_pitch_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_INVALID_ARG;
}

// 3-D bf16 TMA descriptor: dims[0] innermost (elements), strides in bytes of dims 1 and 2,
// box[3] elements per dimension, 128-byte swizzle.
int make_tmap_bf16_3d(CUtensorMap* map, const void* base, const uint64_t dims[3], const uint64_t strides[2],
                      const uint32_t box[3]) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) return DSA_ERR_CUDA;
  cuuint64_t d[3] = {dims[0], dims[1] > 0 ? dims[1] : 1, dims[2] > 0 ? dims[2] : 1};
  cuuint64_t st[2] = {strides[0], strides[1]};
  cuuint32_t bx[3] = {box[0], box[1], box[2]};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), d, st, bx, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DSA_OK : DSA_ERR_INVALID_ARG;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

static thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return DSA_ERR_CUDA;
}

int last_launch_status() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return DSA_OK;
  g_last_cuda_error = (int)e;
  return DSA_ERR_CUDA;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

static bool index_shape_supported(int H_I, int d_I) {
  return (H_I == 64 && d_I == 128) || (H_I == 32 && d_I == 128) || (H_I == 16 && d_I == 128) ||
         (H_I == 8 && d_I == 64) || (H_I == 4 && d_I == 32);
}

static bool attn_shape_supported(int Hq, int Hkv, int d) {
  if (Hq <= 0 || Hkv <= 0 || Hq % Hkv) return false;
  const int G = Hq / Hkv;
  return (d == 64 || d == 128) && (G == 4 || G == 8);
}

// Argument checks of the decode attention calls, in their documented order: pointers and
// alignment, then sizes (DSA_ERR_INVALID_ARG), then shapes without a kernel
// (DSA_ERR_UNSUPPORTED).
int decode_attn_args_status(const void* Q, const void* K, const void* V, const int32_t* indices,
                            const int32_t* cu_seqlens_k, int batch, int Hq, int Hkv, int d, int k, float scale,
                            const void* O) {
  if (!Q || !K || !V || !indices || !cu_seqlens_k || !O) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return DSA_ERR_INVALID_ARG;
  if (batch < 1 || k < 1 || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || k % 16 != 0 || k > 4096) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

}  // namespace dsa_host

using namespace dsa_host;

extern "C" {

DSA_API const char* dsa_status_string(int status) {
  switch (status) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    default: return "DSA_ERR_UNKNOWN";
  }
}

DSA_API int dsa_version(void) { return 1 * 10000 + 0 * 100 + 0; }

DSA_API int dsa_last_cuda_error(const char** message) {
  const int e = g_last_cuda_error;
  if (message) *message = cudaGetErrorString((cudaError_t)e);
  return e;
}

DSA_API int dsa_get_device_status(int* status_out, int* detail_out) {
  if (!status_out) return DSA_ERR_INVALID_ARG;
  if (const cudaError_t e_ = cudaDeviceSynchronize(); e_ != cudaSuccess) return cuda_fail(e_);
  int st = 0, det = 0, zero = 0;
  if (const cudaError_t e_ = cudaMemcpyFromSymbol(&st, dsa::g_status, sizeof(int)); e_ != cudaSuccess) return cuda_fail(e_);
  if (const cudaError_t e_ = cudaMemcpyFromSymbol(&det, dsa::g_status_detail, sizeof(int)); e_ != cudaSuccess) return cuda_fail(e_);
  if (const cudaError_t e_ = cudaMemcpyToSymbol(dsa::g_status, &zero, sizeof(int)); e_ != cudaSuccess) return cuda_fail(e_);
  if (const cudaError_t e_ = cudaMemcpyToSymbol(dsa::g_status_detail, &zero, sizeof(int)); e_ != cudaSuccess) return cuda_fail(e_);
  *status_out = st;
  if (detail_out) *detail_out = det;
  return DSA_OK;
}

DSA_API int dsa_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return DSA_ERR_INVALID_ARG;
  dsa::bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)limit_ns);
  return last_launch_status();
}

DSA_API int dsa_index(const void* q_idx, const void* k_idx, const void* w, const int32_t* cu_seqlens_q,
                      const int32_t* cu_seqlens_k, int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                      int max_seqlen_k, int H_I, int d_I, int64_t row_begin, int64_t row_end, float* scores,
                      int64_t ld_scores, void* stream) {
  if (!q_idx || !k_idx || !w || !cu_seqlens_q || !cu_seqlens_k || !scores) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) || !aligned16(scores)) return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0) return DSA_ERR_INVALID_ARG;
  if (row_begin < 0 || row_end < row_begin || row_end > total_q) return DSA_ERR_INVALID_ARG;
  if (ld_scores < max_seqlen_k || (ld_scores % 4) != 0) return DSA_ERR_INVALID_ARG;
  if (total_q * (int64_t)H_I > 0x7FFFFFFFLL || total_k > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  if (!index_shape_supported(H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  if (row_end == row_begin) return DSA_OK;
  return indexer_launch(q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                        max_seqlen_k, H_I, d_I, row_begin, row_end, scores, ld_scores,
                        static_cast<cudaStream_t>(stream));
}

DSA_API size_t dsa_topk_workspace_size(int64_t rows, int64_t ld_scores, int k) {
  if (rows < 1 || ld_scores < 1 || k < 1) return 0;
  return topk_ws_bytes(rows, ld_scores);
}

DSA_API int dsa_topk(const float* scores, int64_t ld_scores, const int32_t* cu_seqlens_q,
                     const int32_t* cu_seqlens_k, int batch, int64_t row_begin, int64_t row_end, int k,
                     int32_t* indices, void* workspace, size_t workspace_bytes, void* stream) {
  if (!scores || !cu_seqlens_q || !cu_seqlens_k || !indices) return DSA_ERR_INVALID_ARG;
  if (!aligned16(scores) || (ld_scores % 4) != 0 || ld_scores <= 0) return DSA_ERR_INVALID_ARG;
  if (batch < 1 || row_begin < 0 || row_end < row_begin) return DSA_ERR_INVALID_ARG;
  if (k < 1) return DSA_ERR_INVALID_ARG;
  if (k > 4096) return DSA_ERR_UNSUPPORTED;
  if (workspace && !aligned16(workspace)) return DSA_ERR_INVALID_ARG;
  // the row length is bounded by ld_scores (>= the longest visible range)
  const int max_vis = ld_scores > 0x7FFFFFFF ? 0x7FFFFFFF : (int)ld_scores;
  return topk_launch(scores, ld_scores, cu_seqlens_q, cu_seqlens_k, batch, row_begin, row_end, k, indices, max_vis,
                     workspace, workspace ? workspace_bytes : 0, static_cast<cudaStream_t>(stream));
}

DSA_API int dsa_sparse_attn_prefill(const void* Q, const void* K, const void* V, const int32_t* indices,
                                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                    int64_t total_q, int Hq, int Hkv, int d, int k, float scale, void* O,
                                    float* lse, void* stream) {
  if (!Q || !K || !V || !indices || !cu_seqlens_q || !cu_seqlens_k || !O) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(indices))
    return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || k < 1 || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || k % 16 != 0 || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (total_q == 0) return DSA_OK;
  return sparse_attn_prefill_launch(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, Hq, Hkv, d, k,
                                    scale, O, lse, static_cast<cudaStream_t>(stream), nullptr);
}

DSA_API int dsa_sparse_attn_prefill_tc(const void* Q, const void* K, const void* V, const int32_t* indices,
                                       const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                       int64_t total_q, int Hq, int Hkv, int d, int k, float scale, void* O,
                                       float* lse, void* stream) {
  if (!Q || !K || !V || !indices || !cu_seqlens_q || !cu_seqlens_k || !O) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(indices))
    return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || k < 1 || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  if (!sa_gather_tc_eligible(Hq, Hkv, d, k, indices)) return DSA_ERR_UNSUPPORTED;
  if (total_q == 0) return DSA_OK;
  return sa_gather_tc_launch(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, Hq, Hkv, k, scale, O, lse,
                             static_cast<cudaStream_t>(stream), nullptr);
}

static size_t reuse_lse_bytes(int64_t total_q, int Hq) { return round_up((size_t)total_q * Hq * 4, 256); }

DSA_API size_t dsa_sparse_attn_prefill_reuse_workspace_size(int64_t total_q, int Hq, int batch, int max_seqlen_k) {
  if (total_q < 0 || Hq < 1 || batch < 1 || max_seqlen_k < 0) return 0;
  return reuse_lse_bytes(total_q, Hq) +
         sa_block_reuse_scratch_bytes(total_q, Hq, batch, std::max(max_seqlen_k, 1), kUnionMaxChunks);
}

DSA_API int dsa_sparse_attn_prefill_reuse(const void* Q, const void* K, const void* V, const int32_t* indices,
                                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                                          int64_t total_q, int64_t total_k, int max_seqlen_k, int Hq, int Hkv, int d,
                                          int k, float scale, void* O, float* lse, int32_t* block_union,
                                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!Q || !K || !V || !indices || !cu_seqlens_q || !cu_seqlens_k || !O) return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(indices))
    return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || max_seqlen_k < 0 || k < 1 || !(scale > 0.f))
    return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || k % 16 != 0 || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < dsa_sparse_attn_prefill_reuse_workspace_size(total_q, Hq, batch, max_seqlen_k))
    return DSA_ERR_WORKSPACE;
  if (total_q == 0) return DSA_OK;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!sa_block_reuse_eligible(Hq, Hkv, d, max_seqlen_k)) {
    if (block_union) {
      const size_t n_blocks = (size_t)((total_q + 15) / 16 + batch);
      if (const cudaError_t e_ = cudaMemsetAsync(block_union, 0xff, n_blocks * 4, s); e_ != cudaSuccess)
        return cuda_fail(e_);
    }
    return sparse_attn_prefill_launch(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, Hq, Hkv, d, k,
                                      scale, O, lse, s, nullptr);
  }
  float* lse_buf = lse ? lse : static_cast<float*>(workspace);
  void* ws = static_cast<uint8_t*>(workspace) + reuse_lse_bytes(total_q, Hq);
  return sa_block_reuse_launch(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, Hq, Hkv, k,
                               max_seqlen_k, kUnionMaxChunks, scale, O, lse_buf, ws, block_union, s);
}

DSA_API size_t dsa_sparse_attn_decode_workspace_size(int batch, int Hq, int d, int k) {
  if (batch < 1 || Hq < 1 || d < 1 || k < 1) return 0;
  return decode_workspace_bytes(batch, Hq, d, k);
}

DSA_API int dsa_sparse_attn_decode(const void* Q, const void* K, const void* V, const int32_t* indices,
                                   const int32_t* cu_seqlens_k, int batch, int Hq, int Hkv, int d, int k,
                                   float scale, void* O, float* lse, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (const int st = decode_attn_args_status(Q, K, V, indices, cu_seqlens_k, batch, Hq, Hkv, d, k, scale, O);
      st != DSA_OK)
    return st;
  if (!workspace || !aligned16(workspace) || workspace_bytes < decode_workspace_bytes(batch, Hq, d, k))
    return DSA_ERR_WORKSPACE;
  return sparse_attn_decode_launch(Q, K, V, indices, cu_seqlens_k, batch, Hq, Hkv, d, k, scale, O, lse, workspace,
                                   static_cast<cudaStream_t>(stream));
}

DSA_API size_t dsa_index_topk_workspace_size(int64_t chunk_rows, int max_seqlen_k) {
  if (chunk_rows < 1 || max_seqlen_k < 0) return 0;
  return index_topk_workspace_bytes(chunk_rows, max_seqlen_k);
}

DSA_API int dsa_index_topk(const void* q_idx, const void* k_idx, const void* w, const int32_t* cu_seqlens_q,
                           const int32_t* cu_seqlens_k, int batch, int64_t total_q, int64_t total_k, int max_seqlen_q,
                           int max_seqlen_k, int H_I, int d_I, int k, int64_t row_begin, int64_t row_end,
                           int64_t chunk_rows, int path, int32_t* indices, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!q_idx || !k_idx || !w || !cu_seqlens_q || !cu_seqlens_k || !indices) return DSA_ERR_INVALID_ARG;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w)) return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || chunk_rows < 1 || k < 1)
    return DSA_ERR_INVALID_ARG;
  if (row_begin < 0 || row_end < row_begin || row_end > total_q) return DSA_ERR_INVALID_ARG;
  if (path != DSA_PATH_AUTO && path != DSA_PATH_SEPARATE && path != DSA_PATH_FUSED) return DSA_ERR_INVALID_ARG;
  if (total_q * (int64_t)H_I > 0x7FFFFFFFLL || total_k > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  if (!index_shape_supported(H_I, d_I) || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) || workspace_bytes < dsa_index_topk_workspace_size(chunk_rows, max_seqlen_k))
    return DSA_ERR_WORKSPACE;
  if (row_end == row_begin) return DSA_OK;
  return index_topk_launch(q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, max_seqlen_q,
                           max_seqlen_k, H_I, d_I, k, row_begin, row_end, chunk_rows, indices, workspace,
                           path == DSA_PATH_SEPARATE ? 0 : path == DSA_PATH_AUTO ? 1 : 2,
                           static_cast<cudaStream_t>(stream));
}

DSA_API size_t dsa_prefill_workspace_size(int64_t chunk_rows, int max_seqlen_k) {
  return dsa_index_topk_workspace_size(chunk_rows, max_seqlen_k);
}

DSA_API int dsa_prefill(const void* q_idx, const void* k_idx, const void* w, const void* Q, const void* K,
                        const void* V, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                        int64_t total_q, int64_t total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv,
                        int d, int H_I, int d_I, int k, float scale, int64_t chunk_rows, int32_t* indices,
                        void* O, float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!indices || !O || chunk_rows < 1) return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || !index_shape_supported(H_I, d_I) || k % 16 != 0 || k > 4096)
    return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) || workspace_bytes < dsa_prefill_workspace_size(chunk_rows, max_seqlen_k))
    return DSA_ERR_WORKSPACE;
  if (const int st = dsa_index_topk(q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                    max_seqlen_q, max_seqlen_k, H_I, d_I, k, 0, total_q, chunk_rows, DSA_PATH_AUTO,
                                    indices, workspace, workspace_bytes, stream);
      st != DSA_OK)
    return st;
  // dense selected sets: masked dense tensor-core passes, their selection words and row
  // maxima in the score scratch (free once the last chunk is selected)
  if (lse && sa_fwd_tc_eligible(Hq, Hkv, d, k, max_seqlen_k) &&
      sa_fwd_tc_scratch_bytes(total_q, Hq, max_seqlen_k) <= workspace_bytes) {
    if (batch < 1 || total_q < 0 || total_k < 0 || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return DSA_ERR_INVALID_ARG;
    return sa_fwd_tc_launch(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, Hq, Hkv, k,
                            max_seqlen_k, scale, O, lse, workspace, static_cast<cudaStream_t>(stream));
  }
  // sparse sets: blocks of 16 adjacent rows whose selected sets overlap (small union) run on
  // the tensor cores over the gathered union (each key loaded once for the block), the rest
  // on the gather kernel, when the score scratch holds the union plans
  if (sa_block_reuse_eligible(Hq, Hkv, d, max_seqlen_k) &&
      dsa_sparse_attn_prefill_reuse_workspace_size(total_q, Hq, batch, max_seqlen_k) <= workspace_bytes)
    return dsa_sparse_attn_prefill_reuse(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                         max_seqlen_k, Hq, Hkv, d, k, scale, O, lse, nullptr, workspace,
                                         workspace_bytes, stream);
  return dsa_sparse_attn_prefill(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, Hq, Hkv, d, k, scale,
                                 O, lse, stream);
}

DSA_API size_t dsa_decode_workspace_size(int batch, int max_seqlen_k, int Hq, int d, int k) {
  if (batch < 1 || max_seqlen_k < 0 || Hq < 1 || d < 1 || k < 1) return 0;
  const size_t ld = round_up((size_t)(max_seqlen_k > 0 ? max_seqlen_k : 1), 4);
  return round_up((size_t)(batch + 1) * sizeof(int), 256) + round_up((size_t)batch * ld * sizeof(float), 256) +
         round_up(topk_ws_bytes(batch, (long long)ld), 256) + round_up(decode_workspace_bytes(batch, Hq, d, k), 256);
}

DSA_API int dsa_decode(const void* q_idx, const void* k_idx, const void* w, const void* Q, const void* K,
                       const void* V, const int32_t* cu_seqlens_k, int batch, int64_t total_k, int max_seqlen_k,
                       int Hq, int Hkv, int d, int H_I, int d_I, int k, float scale, int32_t* indices, void* O,
                       float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  if (!indices || !O || batch < 1) return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || !index_shape_supported(H_I, d_I) || k % 16 != 0 || k > 4096)
    return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < dsa_decode_workspace_size(batch, max_seqlen_k, Hq, d, k))
    return DSA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* cu_q = reinterpret_cast<int*>(ws);
  ws += round_up((size_t)(batch + 1) * sizeof(int), 256);
  const int64_t ld = (int64_t)round_up((size_t)(max_seqlen_k > 0 ? max_seqlen_k : 1), 4);
  float* scores = reinterpret_cast<float*>(ws);
  ws += round_up((size_t)batch * ld * sizeof(float), 256);
  const size_t topk_bytes = topk_ws_bytes(batch, ld);
  void* topk_ws = topk_bytes ? ws : nullptr;
  ws += round_up(topk_bytes, 256);
  dsa::iota_kernel<<<(batch + 1 + 255) / 256, 256, 0, s>>>(cu_q, batch, 1);
  if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  int st = dsa_index(q_idx, k_idx, w, cu_q, cu_seqlens_k, batch, batch, total_k, 1, max_seqlen_k, H_I, d_I, 0, batch,
                     scores, ld, stream);
  if (st != DSA_OK) return st;
  st = dsa_topk(scores, ld, cu_q, cu_seqlens_k, batch, 0, batch, k, indices, topk_ws, topk_bytes, stream);
  if (st != DSA_OK) return st;
  return dsa_sparse_attn_decode(Q, K, V, indices, cu_seqlens_k, batch, Hq, Hkv, d, k, scale, O, lse, ws,
                                workspace_bytes - (size_t)(ws - static_cast<uint8_t*>(workspace)), stream);
}

DSA_API size_t dsa_sparse_attn_bwd_workspace_size(int64_t total_q, int64_t total_k, int Hq, int Hkv, int d,
                                                  int max_seqlen_k) {
  if (total_q < 0 || total_k < 0 || Hq < 1 || Hkv < 1 || d < 1 || max_seqlen_k < 0) return 0;
  size_t bytes = sparse_attn_bwd_workspace_bytes(total_k, Hkv, d);
  if (d == 128 && Hq == 8 * Hkv) bytes = std::max(bytes, sa_bwd_tc_workspace_bytes(total_q, Hq, max_seqlen_k));
  return bytes;
}

DSA_API int dsa_sparse_attn_prefill_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                        const float* lse, const int32_t* indices, const int32_t* cu_seqlens_q,
                                        const int32_t* cu_seqlens_k, int batch, int64_t total_q, int64_t total_k,
                                        int max_seqlen_k, int Hq, int Hkv, int d, int k, float scale, void* dQ,
                                        void* dK, void* dV, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  if (!Q || !K || !V || !O || !dO || !lse || !indices || !cu_seqlens_q || !cu_seqlens_k || !dQ || !dK || !dV)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
      !aligned16(dK) || !aligned16(dV))
    return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || k < 1 || !(scale > 0.f) || max_seqlen_k < 0)
    return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || k % 16 != 0 || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace)) return DSA_ERR_WORKSPACE;
  if (sa_bwd_tc_eligible(Hq, Hkv, d, k, max_seqlen_k)) {
    if (workspace_bytes < sa_bwd_tc_workspace_bytes(total_q, Hq, max_seqlen_k)) return DSA_ERR_WORKSPACE;
    return sa_bwd_tc_launch(Q, K, V, O, dO, lse, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k, Hq,
                            Hkv, k, max_seqlen_k, scale, dQ, dK, dV, workspace, static_cast<cudaStream_t>(stream));
  }
  if (workspace_bytes < sparse_attn_bwd_workspace_bytes(total_k, Hkv, d)) return DSA_ERR_WORKSPACE;
  return sparse_attn_bwd_launch(Q, K, V, O, dO, lse, indices, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                Hq, Hkv, d, k, scale, dQ, dK, dV, workspace, static_cast<cudaStream_t>(stream));
}

DSA_API size_t dsa_indexer_kl_loss_workspace_size(int64_t total_q, int64_t total_k, int max_seqlen_k, int Hq,
                                                  int H_I, int d_I, int64_t chunk_rows, int batch) {
  if (total_q < 0 || total_k < 0 || max_seqlen_k < 0 || Hq < 1 || H_I < 1 || d_I < 1 || chunk_rows < 1 || batch < 1)
    return 0;
  return kl_workspace_bytes(total_q, total_k, max_seqlen_k, Hq, H_I, d_I, chunk_rows, batch, false);
}

// Argument checks shared by the dense and the sparse-adaptation KL loss.
static int kl_args_status(const void* Q, const void* K, const void* q_idx, const void* k_idx, const void* w,
                          const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                          int64_t total_k, int max_seqlen_k, int Hq, int Hkv, int d, int H_I, int d_I, float scale,
                          int64_t chunk_rows, float* loss, float* kl, void* dq_idx, void* dk_idx, void* dw) {
  if (!Q || !K || !q_idx || !k_idx || !w || !cu_seqlens_q || !cu_seqlens_k || !loss || !kl || !dq_idx || !dk_idx ||
      !dw)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w) ||
      !aligned16(dq_idx) || !aligned16(dk_idx) || !aligned16(dw))
    return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || chunk_rows < 1 || !(scale > 0.f) || max_seqlen_k < 0)
    return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || Hkv > 8) return DSA_ERR_UNSUPPORTED;
  if (!((H_I == 64 || H_I == 32 || H_I == 16) && d_I == 128)) return DSA_ERR_UNSUPPORTED;
  if (total_q * (int64_t)H_I > 0x7FFFFFFFLL || total_k > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

DSA_API int dsa_indexer_kl_loss(const void* Q, const void* K, const void* q_idx, const void* k_idx, const void* w,
                                const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch, int64_t total_q,
                                int64_t total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d, int H_I,
                                int d_I, float scale, int64_t chunk_rows, float* loss, float* kl, void* dq_idx,
                                void* dk_idx, void* dw, void* workspace, size_t workspace_bytes, void* stream) {
  if (const int st = kl_args_status(Q, K, q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                    max_seqlen_k, Hq, Hkv, d, H_I, d_I, scale, chunk_rows, loss, kl, dq_idx, dk_idx,
                                    dw);
      st != DSA_OK)
    return st;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < kl_workspace_bytes(total_q, total_k, max_seqlen_k, Hq, H_I, d_I, chunk_rows, batch, false))
    return DSA_ERR_WORKSPACE;
  return indexer_kl_loss_launch(Q, K, q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                max_seqlen_q, max_seqlen_k, Hq, Hkv, d, H_I, d_I, scale, chunk_rows, loss, kl, dq_idx,
                                dk_idx, dw, workspace, static_cast<cudaStream_t>(stream), nullptr, 0);
}

DSA_API size_t dsa_indexer_kl_loss_sparse_workspace_size(int64_t total_q, int64_t total_k, int max_seqlen_k, int Hq,
                                                         int H_I, int d_I, int64_t chunk_rows, int batch) {
  if (total_q < 0 || total_k < 0 || max_seqlen_k < 0 || Hq < 1 || H_I < 1 || d_I < 1 || chunk_rows < 1 || batch < 1)
    return 0;
  return kl_workspace_bytes(total_q, total_k, max_seqlen_k, Hq, H_I, d_I, chunk_rows, batch, true);
}

DSA_API int dsa_indexer_kl_loss_sparse(const void* Q, const void* K, const void* q_idx, const void* k_idx,
                                       const void* w, const int32_t* indices, int k, const int32_t* cu_seqlens_q,
                                       const int32_t* cu_seqlens_k, int batch, int64_t total_q, int64_t total_k,
                                       int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d, int H_I, int d_I,
                                       float scale, int64_t chunk_rows, float* loss, float* kl, void* dq_idx,
                                       void* dk_idx, void* dw, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  if (const int st = kl_args_status(Q, K, q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                    max_seqlen_k, Hq, Hkv, d, H_I, d_I, scale, chunk_rows, loss, kl, dq_idx, dk_idx,
                                    dw);
      st != DSA_OK)
    return st;
  if (!indices || k < 1) return DSA_ERR_INVALID_ARG;
  if (!(d == 128 && Hq == 8 * Hkv && Hkv <= 4) || k > 4096) return DSA_ERR_UNSUPPORTED;
  if (!workspace || !aligned16(workspace) ||
      workspace_bytes < kl_workspace_bytes(total_q, total_k, max_seqlen_k, Hq, H_I, d_I, chunk_rows, batch, true))
    return DSA_ERR_WORKSPACE;
  return indexer_kl_loss_launch(Q, K, q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, batch, total_q, total_k,
                                max_seqlen_q, max_seqlen_k, Hq, Hkv, d, H_I, d_I, scale, chunk_rows, loss, kl, dq_idx,
                                dk_idx, dw, workspace, static_cast<cudaStream_t>(stream), indices, k);
}

}  // extern "C"
