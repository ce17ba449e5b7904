// Allocation-free variant of the split-K decode attention.
//
// Some callers cannot allocate device memory at the point where they run decode: hosts
// that hand their whole device-memory budget to a preallocated pool and expose no
// allocator to plugins, or latency-critical loops where a cudaMalloc (which can
// synchronise the device) is not acceptable and where no caller-owned scratch buffer is
// available.  For them, dsa_sparse_attn_decode_noalloc keeps its split-K scratch in a
// fixed, file-scope device array instead of a caller workspace.
//
// The array is part of the library image: every GPU that loads the library holds its
// kDecodeScratchBytes until the process exits.  All calls on a device share it and it
// keeps whatever the previous call left there; the decode kernel overwrites every
// scratch entry it later reads, so nothing needs clearing between calls.  Calls whose
// work overlaps on the GPU (different streams, no ordering between them) race on the
// array and must be serialised by the caller.
#include <mutex>

#include "common.cuh"

namespace dsa {

constexpr size_t kDecodeScratchBytes = size_t(8) << 20;  // 8 MiB
static __device__ __align__(256) uint8_t g_decode_scratch[kDecodeScratchBytes];

}  // namespace dsa

namespace dsa_host {

int decode_attn_args_status(const void* Q, const void* K, const void* V, const int32_t* indices,
                            const int32_t* cu_seqlens_k, int batch, int Hq, int Hkv, int d, int k, float scale,
                            const void* O);

constexpr int kMaxScratchDevices = 64;  // device ordinals this entry point serves

// Device address of the scratch array, looked up once per device (with that device
// current).  In host code the array's name is only a host-side stand-in, so the kernel
// must be given this address, never the symbol itself.  A failed CUDA call is recorded
// for dsa_last_cuda_error(); a device ordinal of kMaxScratchDevices or more is
// DSA_ERR_UNSUPPORTED.
static void* decode_scratch_address(int* status) {
  static void* addr[kMaxScratchDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (const cudaError_t e = cudaGetDevice(&dev); e != cudaSuccess) {
    *status = cuda_fail(e);
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxScratchDevices) {
    *status = DSA_ERR_UNSUPPORTED;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (const cudaError_t e = cudaGetSymbolAddress(&p, dsa::g_decode_scratch); e != cudaSuccess || !p) {
      *status = e != cudaSuccess ? cuda_fail(e) : DSA_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *status = DSA_OK;
  return addr[dev];
}

}  // namespace dsa_host

extern "C" DSA_API int dsa_sparse_attn_decode_noalloc(const void* Q, const void* K, const void* V,
                                                      const int32_t* indices, const int32_t* cu_seqlens_k,
                                                      int batch, int Hq, int Hkv, int d, int k, float scale,
                                                      void* O, float* lse, void* stream) {
  // the same checks, in the same order, as dsa_sparse_attn_decode; then the scratch limit
  if (const int st = dsa_host::decode_attn_args_status(Q, K, V, indices, cu_seqlens_k, batch, Hq, Hkv, d, k, scale,
                                                       O);
      st != DSA_OK)
    return st;
  const size_t need = dsa_sparse_attn_decode_workspace_size(batch, Hq, d, k);
  if (need == 0) return DSA_ERR_INVALID_ARG;
  if (need > dsa::kDecodeScratchBytes) return DSA_ERR_WORKSPACE;  // beyond the fixed scratch
  int st = DSA_OK;
  void* scratch = dsa_host::decode_scratch_address(&st);
  if (st != DSA_OK) return st;
  return dsa_sparse_attn_decode(Q, K, V, indices, cu_seqlens_k, batch, Hq, Hkv, d, k, scale, O, lse, scratch,
                                dsa::kDecodeScratchBytes, stream);
}
