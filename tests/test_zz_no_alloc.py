"""The allocation-free decode entry point gives the same result as the regular one.

dsa_sparse_attn_decode_noalloc exists for callers that cannot allocate device memory
where they run decode (a host that owns a preallocated memory pool and gives plugins no
allocator, or a latency-critical loop that must not call cudaMalloc) and that have no
scratch buffer to hand over.  It keeps its split-K scratch in a fixed array inside the
library.  This test calls it through the C ABI twice in a row (the second call runs on
whatever the first left in that shared array) and compares each result with
dsa_sparse_attn_decode given a caller-allocated workspace.  The file name makes pytest
collect it after every other test file.

Both entry points run the same kernels with the same split count and scratch layout, so
their outputs must be bit-identical, not merely close.  The largest request the fixed
scratch holds (batch * Hq = 992 at d = 128, k = 2048) is run too, and the next larger ones
are refused with DSA_ERR_WORKSPACE.
"""
import math

import numpy as np
import pytest
import torch

from lightning_indexer_b200 import _lib
from workloads import generators as gen

pytestmark = pytest.mark.gpu

ATTN_ATOL = 1e-2  # the max-abs bound the other attention tests use (bf16 outputs)


def _dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _case(seed, B, N, Hq=32, Hkv=4):
    wl = gen.make_decode(B, N, Hq, Hkv, 128, 64, 128, 2048, seed=seed, layout="video")
    rng = np.random.default_rng(seed)
    idx = np.stack([np.sort(rng.choice(N, size=2048, replace=False)) for _ in range(B)]).astype(np.int32)
    idx[0, -100:] = -1  # some unused slots
    return wl, torch.from_numpy(idx).cuda()


def test_noalloc_decode_matches_workspace_decode_twice():
    lib = _lib.load()
    stream = torch.cuda.current_stream().cuda_stream
    # the second and third cases follow the first on the same scratch; the third is the
    # largest request the 8 MiB scratch holds (31 x 32 = 992 heads at d = 128, k = 2048)
    for seed, B, N in ((61, 16, 9000), (62, 7, 5000), (63, 31, 3000)):
        wl, idx = _case(seed, B, N)
        Q, K, V = _dev(wl.Q), _dev(wl.K), _dev(wl.V)
        cu_k = torch.from_numpy(wl.cu_seqlens_k.astype(np.int32)).cuda()
        scale = 1.0 / math.sqrt(128)
        ws = torch.empty(lib.dsa_sparse_attn_decode_workspace_size(B, 32, 128, 2048), dtype=torch.uint8,
                         device="cuda")
        O_ref = torch.empty_like(Q)
        lse_ref = torch.empty((B, 32), dtype=torch.float32, device="cuda")
        assert lib.dsa_sparse_attn_decode(Q.data_ptr(), K.data_ptr(), V.data_ptr(), idx.data_ptr(),
                                          cu_k.data_ptr(), B, 32, 4, 128, 2048, scale, O_ref.data_ptr(),
                                          lse_ref.data_ptr(), ws.data_ptr(), ws.numel(), stream) == 0
        O = torch.full_like(Q, float("nan"))
        lse = torch.full((B, 32), float("nan"), dtype=torch.float32, device="cuda")
        assert lib.dsa_sparse_attn_decode_noalloc(Q.data_ptr(), K.data_ptr(), V.data_ptr(), idx.data_ptr(),
                                                  cu_k.data_ptr(), B, 32, 4, 128, 2048, scale, O.data_ptr(),
                                                  lse.data_ptr(), stream) == 0
        torch.cuda.synchronize()
        assert torch.isfinite(O.float()).all() and torch.isfinite(lse).all()
        # same kernels, split count and scratch layout: bit-identical results
        assert torch.equal(O, O_ref)
        assert torch.equal(lse, lse_ref)
        # and within the attention tolerance of the other tests, as a sanity bound
        assert (O.float() - O_ref.float()).abs().max().item() <= ATTN_ATOL


def test_noalloc_decode_rejects_requests_beyond_its_scratch():
    lib = _lib.load()
    fake = 1 << 20  # never dereferenced: the size check fails first
    # batch 64 x 32 heads at d=128, k=2048 needs about 17 MiB of split scratch (> 8 MiB)
    assert lib.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, 64, 32, 4, 128, 2048, 0.1, fake,
                                              None, None) == -3
    # the first sizes past the 992-head limit: 32 x 32 = 1024 heads, and 249 x 4 = 996 heads
    assert lib.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, 32, 32, 4, 128, 2048, 0.1, fake,
                                              None, None) == -3
    assert lib.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, 249, 4, 1, 128, 2048, 0.1, fake,
                                              None, None) == -3
    # the limit itself is accepted by the size check (248 x 4 = 992 heads fit)
    assert lib.dsa_sparse_attn_decode_workspace_size(248, 4, 128, 2048) <= 8 << 20
    assert lib.dsa_sparse_attn_decode_workspace_size(31, 32, 128, 2048) <= 8 << 20
