// Whole DSA prefill from host buffers (declared in include/dsa.h, (5b)): the inputs are
// copied in, each row chunk runs the (fused) indexer + top-k and the attention with
// adjacent-query reuse, and its output rows are copied back, with the copies of one chunk
// overlapping the kernels of its neighbours on three streams.  Same kernels, chunking and
// results as (5) run on device copies of the inputs.
//
// Part of the unity build: api.cu (the entry points it calls) comes first.
#include <mutex>
#include <vector>

#include "common.cuh"

namespace dsa {

// Per row chunk c (rows [c * chunk_rows, ...)), the query offsets of the sequences shifted to
// the chunk's first row and clamped to the chunk: the cu_seqlens_q of the chunk's rows.
__global__ void chunk_offsets_kernel(const int* cu_q, int batch, long long total_q, long long chunk_rows, int nchunks,
                                     int* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nchunks * (batch + 1)) return;
  const int c = i / (batch + 1), b = i % (batch + 1);
  const long long r0 = (long long)c * chunk_rows;
  const long long r1 = min(total_q, r0 + chunk_rows);
  out[i] = (int)min(max((long long)cu_q[b] - r0, 0LL), r1 - r0);
}

}  // namespace dsa

namespace dsa_host {

// Device layout of the host-input prefill's workspace: the device copies of the inputs, the
// chunks' query offsets, the selected sets and O, and the two passes' scratch.
struct PrefillHostLayout {
  size_t q_idx, k_idx, w, Q, K, V, cu_q, cu_k, cu_chunks, indices, O, it_ws, reuse_ws, total;
};

static PrefillHostLayout prefill_host_layout(int batch, int64_t total_q, int64_t total_k, int max_seqlen_k, int Hq,
                                             int Hkv, int d, int H_I, int d_I, int k, int64_t chunk_rows) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const int64_t nchunks = (total_q + chunk_rows - 1) / chunk_rows;
  PrefillHostLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += up(bytes);
    return at;
  };
  L.q_idx = take((size_t)total_q * H_I * d_I * 2);
  L.k_idx = take((size_t)total_k * d_I * 2);
  L.w = take((size_t)total_q * H_I * 2);
  L.Q = take((size_t)total_q * Hq * d * 2);
  L.K = take((size_t)total_k * Hkv * d * 2);
  L.V = take((size_t)total_k * Hkv * d * 2);
  L.cu_q = take((size_t)(batch + 1) * 4);
  L.cu_k = take((size_t)(batch + 1) * 4);
  L.cu_chunks = take((size_t)nchunks * (batch + 1) * 4);
  L.indices = take((size_t)total_q * k * 4);
  L.O = take((size_t)total_q * Hq * d * 2);
  L.it_ws = take(dsa_index_topk_workspace_size(chunk_rows, max_seqlen_k));
  L.reuse_ws = take(dsa_sparse_attn_prefill_reuse_workspace_size(chunk_rows, Hq, batch, max_seqlen_k));
  L.total = off;
  return L;
}

// Two copy streams per device (host to device, device to host), created on first use and
// kept for the process: the library's own streams, not device memory.
static int copy_streams(cudaStream_t& h2d, cudaStream_t& d2h) {
  static std::mutex mu;
  static cudaStream_t streams[64][2] = {};
  int dev = 0;
  if (const cudaError_t e_ = cudaGetDevice(&dev); e_ != cudaSuccess) return cuda_fail(e_);
  if (dev < 0 || dev >= 64) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < 2; ++i)
    if (!streams[dev][i])
      if (const cudaError_t e_ = cudaStreamCreateWithFlags(&streams[dev][i], cudaStreamNonBlocking); e_ != cudaSuccess)
        return cuda_fail(e_);
  h2d = streams[dev][0];
  d2h = streams[dev][1];
  return DSA_OK;
}

}  // namespace dsa_host

using namespace dsa_host;

DSA_API size_t dsa_prefill_host_workspace_size(int batch, int64_t total_q, int64_t total_k, int max_seqlen_k, int Hq,
                                               int Hkv, int d, int H_I, int d_I, int k, int64_t chunk_rows) {
  if (batch < 1 || total_q < 0 || total_k < 0 || max_seqlen_k < 0 || Hq < 1 || Hkv < 1 || d < 1 || H_I < 1 ||
      d_I < 1 || k < 1 || chunk_rows < 1)
    return 0;
  return prefill_host_layout(batch, total_q, total_k, max_seqlen_k, Hq, Hkv, d, H_I, d_I, k, chunk_rows).total;
}

DSA_API int dsa_prefill_host(const void* q_idx, const void* k_idx, const void* w, const void* Q, const void* K,
                             const void* V, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int batch,
                             int64_t total_q, int64_t total_k, int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv,
                             int d, int H_I, int d_I, int k, float scale, int64_t chunk_rows, void* O,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (!q_idx || !k_idx || !w || !Q || !K || !V || !cu_seqlens_q || !cu_seqlens_k || !O) return DSA_ERR_INVALID_ARG;
  if (batch < 1 || total_q < 0 || total_k < 0 || max_seqlen_q < 0 || max_seqlen_k < 0 || chunk_rows < 1 || k < 1 ||
      !(scale > 0.f))
    return DSA_ERR_INVALID_ARG;
  if (!attn_shape_supported(Hq, Hkv, d) || !index_shape_supported(H_I, d_I) || k % 16 != 0 || k > 4096)
    return DSA_ERR_UNSUPPORTED;
  const size_t need = dsa_prefill_host_workspace_size(batch, total_q, total_k, max_seqlen_k, Hq, Hkv, d, H_I, d_I, k,
                                                      chunk_rows);
  if (!workspace || !aligned16(workspace) || workspace_bytes < need) return DSA_ERR_WORKSPACE;
  if (total_q == 0) return DSA_OK;
  const PrefillHostLayout L =
      prefill_host_layout(batch, total_q, total_k, max_seqlen_k, Hq, Hkv, d, H_I, d_I, k, chunk_rows);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const cudaStream_t main = static_cast<cudaStream_t>(stream);
  cudaStream_t h2d, d2h;
  if (const int st = copy_streams(h2d, d2h); st != DSA_OK) return st;
  const int nchunks = (int)((total_q + chunk_rows - 1) / chunk_rows);
  // events: start, offsets landed, per chunk inputs landed and outputs ready, copies out done
  std::vector<cudaEvent_t> ev(3 + 2 * (size_t)nchunks, nullptr);
  int status = DSA_OK;
  auto check = [&](cudaError_t e_) {
    if (e_ != cudaSuccess && status == DSA_OK) status = cuda_fail(e_);
    return status == DSA_OK;
  };
  for (auto& e : ev)
    if (!check(cudaEventCreateWithFlags(&e, cudaEventDisableTiming))) break;
  cudaEvent_t e_start = ev[0], e_keys = ev[1], e_out_done = ev[2];
  cudaEvent_t* e_in = ev.data() + 3;
  cudaEvent_t* e_out = ev.data() + 3 + nchunks;
  auto h2d_copy = [&](size_t dst_off, const void* src, size_t bytes) {
    return check(cudaMemcpyAsync(ws + dst_off, src, bytes, cudaMemcpyHostToDevice, h2d));
  };
  const auto* qi = static_cast<const uint8_t*>(q_idx);
  const auto* wi = static_cast<const uint8_t*>(w);
  const auto* Qi = static_cast<const uint8_t*>(Q);
  auto* Oh = static_cast<uint8_t*>(O);
  const size_t qi_row = (size_t)H_I * d_I * 2, w_row = (size_t)H_I * 2, q_row = (size_t)Hq * d * 2;
  if (status == DSA_OK) {
    // the copy streams start after the caller's earlier work (the workspace is free then)
    check(cudaEventRecord(e_start, main)) && check(cudaStreamWaitEvent(h2d, e_start, 0)) &&
        check(cudaStreamWaitEvent(d2h, e_start, 0));
  }
  // the offsets first; then per chunk, the key-side rows its rows can see that earlier
  // chunks did not need (whole 256-key tiles ahead, since the indexer loads keys by tile),
  // then the chunk's query rows: the first chunk starts after its own keys, not all of them
  const auto* ki = static_cast<const uint8_t*>(k_idx);
  const auto* Ki = static_cast<const uint8_t*>(K);
  const auto* Vi = static_cast<const uint8_t*>(V);
  const size_t ki_row = (size_t)d_I * 2, kv_row = (size_t)Hkv * d * 2;
  int64_t keys_done = 0;
  auto copy_keys_to = [&](int64_t kend) {
    kend = std::min<int64_t>(total_k, kend);
    if (kend <= keys_done) return true;
    const int64_t k0 = keys_done, nk = kend - keys_done;
    keys_done = kend;
    return h2d_copy(L.k_idx + k0 * ki_row, ki + k0 * ki_row, nk * ki_row) &&
           h2d_copy(L.K + k0 * kv_row, Ki + k0 * kv_row, nk * kv_row) &&
           h2d_copy(L.V + k0 * kv_row, Vi + k0 * kv_row, nk * kv_row);
  };
  // the end of the keys that rows below r1 see (bottom-right causal alignment per sequence)
  auto key_end = [&](int64_t r1) {
    int b = 0;
    while (b + 1 < batch && cu_seqlens_q[b + 1] <= r1 - 1) ++b;
    const int64_t Lq = cu_seqlens_q[b + 1] - cu_seqlens_q[b], Lk = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
    const int64_t vis = std::min(Lk, std::max<int64_t>(0, (r1 - 1 - cu_seqlens_q[b]) + (Lk - Lq) + 1));
    return cu_seqlens_k[b] + (vis + 511) / 256 * 256;
  };
  if (status == DSA_OK && h2d_copy(L.cu_q, cu_seqlens_q, (size_t)(batch + 1) * 4) &&
      h2d_copy(L.cu_k, cu_seqlens_k, (size_t)(batch + 1) * 4) && check(cudaEventRecord(e_keys, h2d))) {
    for (int c = 0; c < nchunks && status == DSA_OK; ++c) {
      const int64_t r0 = (int64_t)c * chunk_rows, n = std::min(total_q, r0 + chunk_rows) - r0;
      copy_keys_to(c + 1 == nchunks ? total_k : key_end(r0 + n)) &&
          h2d_copy(L.q_idx + r0 * qi_row, qi + r0 * qi_row, n * qi_row) &&
          h2d_copy(L.w + r0 * w_row, wi + r0 * w_row, n * w_row) && h2d_copy(L.Q + r0 * q_row, Qi + r0 * q_row, n * q_row) &&
          check(cudaEventRecord(e_in[c], h2d));
    }
  }
  if (status == DSA_OK && check(cudaStreamWaitEvent(main, e_keys, 0))) {
    const int n = nchunks * (batch + 1);
    dsa::chunk_offsets_kernel<<<(unsigned)((n + 255) / 256), 256, 0, main>>>(
        reinterpret_cast<const int*>(ws + L.cu_q), batch, total_q, chunk_rows, nchunks,
        reinterpret_cast<int*>(ws + L.cu_chunks));
    if (const int st = last_launch_status(); st != DSA_OK) status = st;
  }
  const int* cu_q_d = reinterpret_cast<const int*>(ws + L.cu_q);
  const int* cu_k_d = reinterpret_cast<const int*>(ws + L.cu_k);
  for (int c = 0; c < nchunks && status == DSA_OK; ++c) {
    const int64_t r0 = (int64_t)c * chunk_rows, n = std::min(total_q, r0 + chunk_rows) - r0;
    if (!check(cudaStreamWaitEvent(main, e_in[c], 0))) break;
    int32_t* idx = reinterpret_cast<int32_t*>(ws + L.indices) + r0 * k;
    int st = dsa_index_topk(ws + L.q_idx, ws + L.k_idx, ws + L.w, cu_q_d, cu_k_d, batch, total_q, total_k,
                            max_seqlen_q, max_seqlen_k, H_I, d_I, k, r0, r0 + n, chunk_rows, DSA_PATH_AUTO, idx,
                            ws + L.it_ws, L.reuse_ws - L.it_ws, main);
    if (st == DSA_OK)
      st = dsa_sparse_attn_prefill_reuse(ws + L.Q + r0 * q_row, ws + L.K, ws + L.V, idx,
                                         reinterpret_cast<const int*>(ws + L.cu_chunks) + (size_t)c * (batch + 1),
                                         cu_k_d, batch, n, total_k, max_seqlen_k, Hq, Hkv, d, k, scale,
                                         ws + L.O + r0 * q_row, nullptr, nullptr, ws + L.reuse_ws,
                                         L.total - L.reuse_ws, main);
    if (st != DSA_OK) {
      status = st;
      break;
    }
    check(cudaEventRecord(e_out[c], main)) && check(cudaStreamWaitEvent(d2h, e_out[c], 0)) &&
        check(cudaMemcpyAsync(Oh + r0 * q_row, ws + L.O + r0 * q_row, n * q_row, cudaMemcpyDeviceToHost, d2h));
  }
  // the caller's stream is ordered after every copy (also after an error, so that no copy
  // of this call is left running unseen)
  if (e_out_done) {
    cudaEventRecord(e_out_done, d2h);
    cudaStreamWaitEvent(main, e_out_done, 0);
    cudaEventRecord(e_out_done, h2d);
    cudaStreamWaitEvent(main, e_out_done, 0);
  }
  for (auto& e : ev)
    if (e) cudaEventDestroy(e);  // released once the device has passed them
  return status;
}
