"""C ABI checks that need no GPU: the library loads, exports every entry point that
include/dsa.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from lightning_indexer_b200 import _lib

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dsa.h")


def declared_functions():
    text = open(HDR).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    names = declared_functions()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), "binding signatures out of sync with the header"


def test_status_strings_and_version():
    lib = _lib.load()
    assert lib.dsa_status_string(0) == b"DSA_OK"
    assert lib.dsa_status_string(-3) == b"DSA_ERR_WORKSPACE"
    assert lib.dsa_status_string(12345) == b"DSA_ERR_UNKNOWN"
    assert lib.dsa_version() >= 10000


def test_host_side_argument_errors():
    lib = _lib.load()
    fake = 1 << 20  # never dereferenced: every call below fails its host checks first
    mis = fake + 2  # misaligned
    # null pointer
    assert lib.dsa_index(None, fake, fake, fake, fake, 1, 8, 8, 8, 8, 64, 128, 0, 8, fake, 8, None) == -1
    # misaligned operand
    assert lib.dsa_index(mis, fake, fake, fake, fake, 1, 8, 8, 8, 8, 64, 128, 0, 8, fake, 8, None) == -1
    # row range outside [0, total_q]
    assert lib.dsa_index(fake, fake, fake, fake, fake, 1, 8, 8, 8, 8, 64, 128, 0, 9, fake, 8, None) == -1
    # ld not a multiple of 4 / smaller than max_seqlen_k
    assert lib.dsa_index(fake, fake, fake, fake, fake, 1, 8, 8, 8, 8, 64, 128, 0, 8, fake, 6, None) == -1
    assert lib.dsa_index(fake, fake, fake, fake, fake, 1, 8, 8, 8, 16, 64, 128, 0, 8, fake, 8, None) == -1
    # unsupported indexer shape
    assert lib.dsa_index(fake, fake, fake, fake, fake, 1, 8, 8, 8, 8, 48, 128, 0, 8, fake, 8, None) == -2
    # top-k bounds
    assert lib.dsa_topk(fake, 8, fake, fake, 1, 0, 8, 0, fake, None, 0, None) == -1
    assert lib.dsa_topk(fake, 8, fake, fake, 1, 0, 8, 5000, fake, None, 0, None) == -2
    assert lib.dsa_topk(fake, 8, fake, fake, 1, 0, 8, 16, fake, mis, 1024, None) == -1  # misaligned workspace
    # top-k workspace: asked for few long rows only
    assert lib.dsa_topk_workspace_size(16, 262144, 2048) > 0
    assert lib.dsa_topk_workspace_size(8192, 131072, 2048) == 0
    assert lib.dsa_topk_workspace_size(16, 4096, 2048) == 0
    # attention shapes
    assert lib.dsa_sparse_attn_prefill(fake, fake, fake, fake, fake, fake, 1, 8, 32, 4, 96, 64, 0.1, fake,
                                       None, None) == -2
    assert lib.dsa_sparse_attn_prefill(fake, fake, fake, fake, fake, fake, 1, 8, 32, 4, 128, 40, 0.1, fake,
                                       None, None) == -2
    assert lib.dsa_sparse_attn_prefill(fake, fake, fake, fake, fake, fake, 1, 8, 32, 4, 128, 64, -1.0, fake,
                                       None, None) == -1
    # the tensor-core entry: d = 128, Hq = 8 Hkv, k a multiple of 16 up to 2048, aligned indices
    for Hq, Hkv, d, k in ((32, 4, 64, 64), (16, 4, 128, 64), (32, 4, 128, 40), (32, 4, 128, 4096)):
        assert lib.dsa_sparse_attn_prefill_tc(fake, fake, fake, fake, fake, fake, 1, 8, Hq, Hkv, d, k, 0.1, fake,
                                              None, None) == -2, (Hq, Hkv, d, k)
    assert lib.dsa_sparse_attn_prefill_tc(fake, fake, fake, mis, fake, fake, 1, 8, 32, 4, 128, 64, 0.1, fake,
                                          None, None) == -1  # misaligned indices
    assert lib.dsa_sparse_attn_prefill_tc(fake, fake, fake, fake, fake, fake, 1, 8, 32, 4, 128, 64, 0.0, fake,
                                          None, None) == -1
    # attention with adjacent-query reuse: shape and scale checks as (3), then the workspace
    wsz = lib.dsa_sparse_attn_prefill_reuse_workspace_size(131072, 32, 1, 131072)
    assert 620e6 < wsz < 680e6  # per 16-row block: 12288 union positions, their selection words, lse and maxima
    assert lib.dsa_sparse_attn_prefill_reuse_workspace_size(-1, 32, 1, 4096) == 0
    assert lib.dsa_sparse_attn_prefill_reuse(fake, fake, fake, fake, fake, fake, 1, 8, 8, 8, 32, 4, 96, 64, 0.1,
                                             fake, None, None, fake, wsz, None) == -2
    assert lib.dsa_sparse_attn_prefill_reuse(fake, fake, fake, fake, fake, fake, 1, 8, 8, 8, 32, 4, 128, 64, 0.0,
                                             fake, None, None, fake, wsz, None) == -1
    small = lib.dsa_sparse_attn_prefill_reuse_workspace_size(8, 32, 1, 8)
    assert lib.dsa_sparse_attn_prefill_reuse(fake, fake, fake, fake, fake, fake, 1, 8, 8, 8, 32, 4, 128, 64, 0.1,
                                             fake, None, None, fake, small - 16, None) == -3
    assert lib.dsa_sparse_attn_prefill_reuse(fake, fake, fake, fake, fake, fake, 1, 8, 8, 8, 32, 4, 128, 64, 0.1,
                                             fake, None, None, None, small, None) == -3
    assert lib.dsa_sparse_attn_prefill_reuse(fake, fake, fake, fake, fake, fake, 1, 0, 0, 8, 32, 4, 128, 64, 0.1,
                                             fake, None, None, fake, wsz, None) == 0  # nothing to do
    # host-input prefill: argument checks before anything is enqueued
    hw = lib.dsa_prefill_host_workspace_size(1, 131072, 131072, 131072, 32, 4, 128, 64, 128, 2048, 8192)
    assert hw > 131072 * (64 * 128 * 2 + 32 * 128 * 2 * 2 + 2048 * 4)  # device copies of the inputs, O, indices
    assert lib.dsa_prefill_host_workspace_size(0, 8, 8, 8, 32, 4, 128, 64, 128, 64, 8) == 0
    args = [fake] * 8 + [1, 8, 8, 8, 8, 32, 4, 128, 64, 128, 64, 0.1, 8, fake]
    bad = list(args)
    bad[15] = 96  # d
    assert lib.dsa_prefill_host(*bad, fake, hw, None) == -2
    bad = list(args)
    bad[18] = 40  # k not a multiple of 16
    assert lib.dsa_prefill_host(*bad, fake, hw, None) == -2
    bad = list(args)
    bad[19] = 0.0  # scale
    assert lib.dsa_prefill_host(*bad, fake, hw, None) == -1
    need_small = lib.dsa_prefill_host_workspace_size(1, 8, 8, 8, 32, 4, 128, 64, 128, 64, 8)
    assert lib.dsa_prefill_host(*args, fake, need_small - 16, None) == -3
    assert lib.dsa_prefill_host(*args, None, need_small, None) == -3
    # workspace too small
    need = lib.dsa_sparse_attn_decode_workspace_size(16, 32, 128, 2048)
    assert need > 0
    assert lib.dsa_sparse_attn_decode(fake, fake, fake, fake, fake, 16, 32, 4, 128, 2048, 0.1, fake, None,
                                      fake, need - 1, None) == -3
    # the allocation-free decode checks its arguments in the same order as the regular one,
    # and only then its fixed scratch limit
    big = 64  # batch 64 x 32 heads at d = 128, k = 2048 needs more than the 8 MiB scratch
    assert lib.dsa_sparse_attn_decode_noalloc(None, fake, fake, fake, fake, big, 32, 4, 128, 2048, 0.1, fake,
                                              None, None) == -1
    assert lib.dsa_sparse_attn_decode_noalloc(mis, fake, fake, fake, fake, big, 32, 4, 128, 2048, 0.1, fake,
                                              None, None) == -1
    assert lib.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, big, 32, 4, 128, 2008, 0.1, fake,
                                              None, None) == -2  # k not a multiple of 16
    assert lib.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, big, 32, 4, 96, 2048, 0.1, fake,
                                              None, None) == -2  # head dim without a kernel
    assert lib.dsa_sparse_attn_decode_noalloc(fake, fake, fake, fake, fake, big, 32, 4, 128, 2048, 0.1, fake,
                                              None, None) == -3
    # bounded-wait self-test: limits outside 1 ns .. 1 s are refused before any launch
    assert lib.dsa_selftest_bounded_wait(0, None) == -1
    assert lib.dsa_selftest_bounded_wait(2_000_000_000, None) == -1
    assert lib.dsa_prefill_workspace_size(8192, 131072) >= 8192 * 131072 * 4
    # sparse backward: the masked dense path (d = 128, 8 heads per KV head) needs the fp32 dQ
    # accumulator; the gather path the fp32 dK and dV accumulators
    T, Tk = 4096, 4096
    dense = lib.dsa_sparse_attn_bwd_workspace_size(T, Tk, 32, 4, 128, 4096)
    assert dense >= T * 32 * 128 * 4 + T * 32 * 8
    gather = lib.dsa_sparse_attn_bwd_workspace_size(T, Tk, 8, 2, 64, 4096)
    assert gather >= 2 * Tk * 2 * 64 * 4
    assert lib.dsa_sparse_attn_bwd_workspace_size(T, Tk, 32, 4, 128, -1) == 0
    # dense path chosen (8 k >= max_seqlen_k) with a workspace only the gather path fits
    small = 2 * Tk * 4 * 128 * 4
    assert small < dense
    assert lib.dsa_sparse_attn_prefill_bwd(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, T, Tk, 4096,
                                           32, 4, 128, 512, 0.1, fake, fake, fake, fake, small, None) == -3
    assert lib.dsa_sparse_attn_prefill_bwd(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, T, Tk, -1,
                                           32, 4, 128, 512, 0.1, fake, fake, fake, fake, dense, None) == -1
    # KL loss workspace: needs the batch (dk work items per row chunk), grows with it
    assert lib.dsa_indexer_kl_loss_workspace_size(T, Tk, 4096, 32, 64, 128, 1024, 0) == 0
    w1 = lib.dsa_indexer_kl_loss_workspace_size(T, Tk, 4096, 32, 64, 128, 1024, 1)
    w8 = lib.dsa_indexer_kl_loss_workspace_size(T, Tk, 4096, 32, 64, 128, 1024, 8)
    assert 0 < w1 < w8


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.load()
