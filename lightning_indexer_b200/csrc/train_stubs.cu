// Placeholder entry points for the training calls until their kernels land.
#include "common.cuh"
extern "C" {
DSA_API size_t dsa_sparse_attn_bwd_workspace_size(int64_t, int64_t, int, int, int) { return 0; }
DSA_API int dsa_sparse_attn_prefill_bwd(const void*, const void*, const void*, const void*, const void*,
                                        const float*, const int32_t*, const int32_t*, const int32_t*, int,
                                        int64_t, int64_t, int, int, int, int, float, void*, void*, void*, void*,
                                        size_t, void*) {
  return DSA_ERR_UNSUPPORTED;
}
DSA_API size_t dsa_indexer_kl_loss_workspace_size(int64_t, int64_t, int, int, int, int, int64_t) { return 0; }
DSA_API int dsa_indexer_kl_loss(const void*, const void*, const void*, const void*, const void*, const int32_t*,
                                const int32_t*, int, int64_t, int64_t, int, int, int, int, int, int, int, float,
                                int64_t, float*, float*, void*, void*, void*, void*, size_t, void*) {
  return DSA_ERR_UNSUPPORTED;
}
}
