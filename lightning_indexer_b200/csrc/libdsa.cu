// Unity build of libdsa_b200: every kernel and the C ABI in one translation unit, so the
// device status word is shared without relocatable device code.
#include "api.cu"
#include "indexer.cu"
#include "indexer2.cu"
#include "topk.cu"
#include "sparse_attn.cu"
#include "sparse_attn_bwd.cu"
#include "sparse_attn_bwd_tc.cu"
#include "kl_bwd_tc.cu"
#include "kl_dense_tc.cu"
#include "sparse_attn_tc.cu"
#include "kl_loss.cu"
#include "decode_noalloc.cu"
