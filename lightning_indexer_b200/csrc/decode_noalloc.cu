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

// Device address of the scratch array, looked up once per device (with that device
// current).  In host code the array's name is only a host-side stand-in, so the kernel
// must be given this address, never the symbol itself.
static void* decode_scratch_address(int* status) {
  constexpr int kMaxDevices = 64;
  static void* addr[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = DSA_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, dsa::g_decode_scratch) != cudaSuccess || !p) {
      *status = DSA_ERR_CUDA;
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
  if (!Q || !K || !V || !indices || !cu_seqlens_k || !O) return DSA_ERR_INVALID_ARG;
  if (batch < 1 || k < 1 || !(scale > 0.f)) return DSA_ERR_INVALID_ARG;
  const size_t need = dsa_sparse_attn_decode_workspace_size(batch, Hq, d, k);
  if (need == 0) return DSA_ERR_INVALID_ARG;
  if (need > dsa::kDecodeScratchBytes) return DSA_ERR_WORKSPACE;  // beyond the fixed scratch
  int st = DSA_OK;
  void* scratch = dsa_host::decode_scratch_address(&st);
  if (st != DSA_OK) return st;
  return dsa_sparse_attn_decode(Q, K, V, indices, cu_seqlens_k, batch, Hq, Hkv, d, k, scale, O, lse, scratch,
                                dsa::kDecodeScratchBytes, stream);
}
