"""DSA (lightning indexer + deterministic top-k + sparse GQA attention) for B200.

Thin torch-facing binding over the C ABI of libdsa_b200.so: it checks tensors, allocates
outputs and workspaces with torch (plumbing), and passes raw pointers and the current CUDA
stream.  Every step of the computation runs in the library's sm_100a kernels; there is
no Python or CPU fallback.
"""
import math
from typing import Optional, Tuple

import torch

from . import _lib
from ._lib import DSAError, call

__all__ = ["index", "topk", "topk_workspace_bytes", "index_topk", "index_topk_workspace_bytes", "prefill_from_host", "prefill_host_workspace_bytes", "sparse_attn_prefill", "sparse_attn_prefill_reuse", "sparse_attn_prefill_reuse_workspace_bytes", "sparse_attn_decode", "prefill", "decode",
           "sparse_attn_prefill_bwd", "indexer_kl_loss", "indexer_kl_loss_sparse", "device_status", "DSAError"]


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _check(t: torch.Tensor, name: str, dtype, ndim=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {t.dim()}")


def _ld(max_seqlen_k: int) -> int:
    return max(4, (max_seqlen_k + 3) // 4 * 4)


def index(q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
          row_begin: int = 0, row_end: Optional[int] = None, scores: Optional[torch.Tensor] = None):
    """Indexer scores for query rows [row_begin, row_end): fp32 [rows, ld] (see dsa_index)."""
    _check(q_idx, "q_idx", torch.bfloat16, 3)
    _check(k_idx, "k_idx", torch.bfloat16, 2)
    _check(w, "w", torch.bfloat16, 2)
    _check(cu_seqlens_q, "cu_seqlens_q", torch.int32, 1)
    _check(cu_seqlens_k, "cu_seqlens_k", torch.int32, 1)
    total_q, H_I, d_I = q_idx.shape
    row_end = total_q if row_end is None else row_end
    if scores is None:
        scores = torch.full((row_end - row_begin, _ld(max_seqlen_k)), float("-inf"), dtype=torch.float32,
                            device=q_idx.device)
    _check(scores, "scores", torch.float32, 2)
    call("dsa_index", _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
         cu_seqlens_q.numel() - 1, total_q, k_idx.shape[0], max_seqlen_q, max_seqlen_k, H_I, d_I,
         row_begin, row_end, _ptr(scores), scores.shape[1], _stream())
    return scores


def topk_workspace_bytes(rows: int, ld_scores: int, k: int) -> int:
    return _lib.load().dsa_topk_workspace_size(rows, ld_scores, k)


def topk(scores, cu_seqlens_q, cu_seqlens_k, k: int, row_begin: int = 0, row_end: Optional[int] = None,
         indices: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None):
    """Deterministic top-k of each score row: int32 [rows, k], ascending, -1 padded.

    A workspace of dsa_topk_workspace_size bytes is allocated when the library asks for
    one (few long rows) and none is given."""
    _check(scores, "scores", torch.float32, 2)
    row_end = row_begin + scores.shape[0] if row_end is None else row_end
    if indices is None:
        indices = torch.empty((row_end - row_begin, k), dtype=torch.int32, device=scores.device)
    _check(indices, "indices", torch.int32, 2)
    if workspace is None:
        nbytes = topk_workspace_bytes(row_end - row_begin, scores.shape[1], k)
        if nbytes:
            workspace = torch.empty(nbytes, dtype=torch.uint8, device=scores.device)
    call("dsa_topk", _ptr(scores), scores.shape[1], _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
         cu_seqlens_q.numel() - 1, row_begin, row_end, k, _ptr(indices), _ptr(workspace),
         0 if workspace is None else workspace.numel(), _stream())
    return indices


PATH_AUTO, PATH_SEPARATE, PATH_FUSED = 0, 1, 2


def index_topk_workspace_bytes(chunk_rows: int, max_seqlen_k: int) -> int:
    return _lib.load().dsa_index_topk_workspace_size(chunk_rows, max_seqlen_k)


def index_topk(q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int, k: int,
               chunk_rows: int = 8192, path: int = PATH_AUTO, indices: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, row_begin: int = 0, row_end: Optional[int] = None):
    """Selected sets of the query rows [row_begin, row_end) (indexer + top-k, fused where it
    applies): int32 [rows, k], ascending, -1 padded (see dsa_index_topk)."""
    _check(q_idx, "q_idx", torch.bfloat16, 3)
    _check(k_idx, "k_idx", torch.bfloat16, 2)
    _check(w, "w", torch.bfloat16, 2)
    total_q, H_I, d_I = q_idx.shape
    row_end = total_q if row_end is None else row_end
    chunk_rows = max(1, min(chunk_rows, max(row_end - row_begin, 1)))
    if indices is None:
        indices = torch.empty((row_end - row_begin, k), dtype=torch.int32, device=q_idx.device)
    _check(indices, "indices", torch.int32, 2)
    if workspace is None:
        workspace = torch.empty(index_topk_workspace_bytes(chunk_rows, max_seqlen_k), dtype=torch.uint8,
                                device=q_idx.device)
    call("dsa_index_topk", _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k),
         cu_seqlens_q.numel() - 1, total_q, k_idx.shape[0], max_seqlen_q, max_seqlen_k, H_I, d_I, k, row_begin,
         row_end, chunk_rows, path, _ptr(indices), _ptr(workspace), workspace.numel(), _stream())
    return indices


def sparse_attn_prefill(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, scale: Optional[float] = None,
                        with_lse: bool = True, out=None, kernel: str = "gather") -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Sparse GQA attention of every packed query row over its selected keys.  `out` may
    give (O, lse) tensors to write (lse may be None).  kernel="tensor_core" calls the
    tcgen05 entry point (d = 128, Hq = 8 Hkv, k <= 2048) instead of the default one."""
    entry = {"gather": "dsa_sparse_attn_prefill", "tensor_core": "dsa_sparse_attn_prefill_tc"}[kernel]
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _check(t, n, torch.bfloat16, 3)
    _check(indices, "indices", torch.int32, 2)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is not None:
        O, lse = out
        _check(O, "O", torch.bfloat16, 3)
    else:
        O = torch.empty_like(Q)
        lse = torch.empty((T, Hq), dtype=torch.float32, device=Q.device) if with_lse else None
    call(entry, _ptr(Q), _ptr(K), _ptr(V), _ptr(indices), _ptr(cu_seqlens_q),
         _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, T, Hq, Hkv, d, indices.shape[1], scale, _ptr(O),
         _ptr(lse), _stream())
    return O, lse


def sparse_attn_prefill_reuse_workspace_bytes(total_q: int, Hq: int, batch: int, max_seqlen_k: int) -> int:
    return _lib.load().dsa_sparse_attn_prefill_reuse_workspace_size(total_q, Hq, batch, max_seqlen_k)


def sparse_attn_prefill_reuse(Q, K, V, indices, cu_seqlens_q, cu_seqlens_k, max_seqlen_k: int,
                              scale: Optional[float] = None, out=None, workspace: Optional[torch.Tensor] = None,
                              block_union: Optional[torch.Tensor] = None):
    """Sparse GQA attention with adjacent-query reuse: the same (O, lse) as
    sparse_attn_prefill, with 16-row blocks whose selections overlap computed on tensor cores
    over the union of their sets.  `block_union` (int32, (T + 15) // 16 + batch entries) may
    receive each block's union size."""
    for t, n in ((Q, "Q"), (K, "K"), (V, "V")):
        _check(t, n, torch.bfloat16, 3)
    _check(indices, "indices", torch.int32, 2)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    batch = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is not None:
        O, lse = out
        _check(O, "O", torch.bfloat16, 3)
    else:
        O = torch.empty_like(Q)
        lse = torch.empty((T, Hq), dtype=torch.float32, device=Q.device)
    if workspace is None:
        workspace = torch.empty(sparse_attn_prefill_reuse_workspace_bytes(T, Hq, batch, max_seqlen_k),
                                dtype=torch.uint8, device=Q.device)
    if block_union is not None:
        _check(block_union, "block_union", torch.int32, 1)
        if block_union.numel() < (T + 15) // 16 + batch:
            raise ValueError("block_union needs (T + 15) // 16 + batch entries")
    call("dsa_sparse_attn_prefill_reuse", _ptr(Q), _ptr(K), _ptr(V), _ptr(indices), _ptr(cu_seqlens_q),
         _ptr(cu_seqlens_k), batch, T, K.shape[0], max_seqlen_k, Hq, Hkv, d, indices.shape[1], scale, _ptr(O),
         _ptr(lse), _ptr(block_union), _ptr(workspace), workspace.numel(), _stream())
    return O, lse


def decode_attn_workspace_bytes(batch: int, Hq: int, d: int, k: int) -> int:
    return _lib.load().dsa_sparse_attn_decode_workspace_size(batch, Hq, d, k)


def sparse_attn_decode(Q, K, V, indices, cu_seqlens_k, scale: Optional[float] = None,
                       workspace: Optional[torch.Tensor] = None):
    """Decode attention (one query row per sequence), split over the selected keys."""
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    k = indices.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    nbytes = _lib.load().dsa_sparse_attn_decode_workspace_size(B, Hq, d, k)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=Q.device)
    O = torch.empty_like(Q)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=Q.device)
    call("dsa_sparse_attn_decode", _ptr(Q), _ptr(K), _ptr(V), _ptr(indices), _ptr(cu_seqlens_k), B, Hq, Hkv, d,
         k, scale, _ptr(O), _ptr(lse), _ptr(workspace), workspace.numel(), _stream())
    return O, lse


def prefill_workspace_bytes(chunk_rows: int, max_seqlen_k: int) -> int:
    return _lib.load().dsa_prefill_workspace_size(chunk_rows, max_seqlen_k)


def prefill(q_idx, k_idx, w, Q, K, V, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
            k: int, chunk_rows: int = 8192, scale: Optional[float] = None,
            workspace: Optional[torch.Tensor] = None, out=None):
    """Whole DSA prefill forward: indexer + top-k (row-chunked) then sparse attention.

    Returns (indices [T, k] int32, O [T, Hq, d] bf16, lse [T, Hq] fp32).
    """
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    H_I, d_I = q_idx.shape[1], q_idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    chunk_rows = max(1, min(chunk_rows, T))
    if workspace is None:
        workspace = torch.empty(prefill_workspace_bytes(chunk_rows, max_seqlen_k), dtype=torch.uint8,
                                device=Q.device)
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=Q.device), torch.empty_like(Q),
               torch.empty((T, Hq), dtype=torch.float32, device=Q.device))
    indices, O, lse = out
    call("dsa_prefill", _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(Q), _ptr(K), _ptr(V), _ptr(cu_seqlens_q),
         _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, T, K.shape[0], max_seqlen_q, max_seqlen_k, Hq, Hkv, d,
         H_I, d_I, k, scale, chunk_rows, _ptr(indices), _ptr(O), _ptr(lse), _ptr(workspace), workspace.numel(),
         _stream())
    return indices, O, lse


def prefill_host_workspace_bytes(batch: int, total_q: int, total_k: int, max_seqlen_k: int, Hq: int, Hkv: int, d: int,
                                 H_I: int, d_I: int, k: int, chunk_rows: int) -> int:
    return _lib.load().dsa_prefill_host_workspace_size(batch, total_q, total_k, max_seqlen_k, Hq, Hkv, d, H_I, d_I, k,
                                                       chunk_rows)


def prefill_from_host(q_idx, k_idx, w, Q, K, V, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                      k: int, chunk_rows: int = 8192, scale: Optional[float] = None, O=None,
                      device: Optional[torch.device] = None, buffers: Optional[dict] = None):
    """Whole DSA prefill whose inputs and output live in host memory (pin them for overlap),
    through the library's dsa_prefill_host: the key side is copied first, each row chunk's
    query rows are copied while its neighbours run their indexer + top-k and attention, and
    each chunk's O rows are copied back as soon as they are ready.  `buffers` (a dict,
    filled on first use) keeps the device workspace between calls.  Returns O (host, bf16
    [T, Hq, d]); the current stream is ordered after every copy."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    for t, n in ((q_idx, "q_idx"), (k_idx, "k_idx"), (w, "w"), (Q, "Q"), (K, "K"), (V, "V")):
        if t.dtype != torch.bfloat16 or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous bfloat16 host tensor")
    for t, n in ((cu_seqlens_q, "cu_seqlens_q"), (cu_seqlens_k, "cu_seqlens_k")):
        if t.dtype != torch.int32 or t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous int32 host tensor")
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    H_I, d_I = q_idx.shape[1], q_idx.shape[2]
    B = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    chunk_rows = max(1, min(chunk_rows, T))
    buf = {} if buffers is None else buffers
    nbytes = prefill_host_workspace_bytes(B, T, K.shape[0], max_seqlen_k, Hq, Hkv, d, H_I, d_I, k, chunk_rows)
    if "ws" not in buf or buf["ws"].numel() < nbytes or buf["ws"].device != dev:
        buf["ws"] = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    if O is None:
        O = torch.empty(Q.shape, dtype=torch.bfloat16, pin_memory=True)
    with torch.cuda.device(dev):
        call("dsa_prefill_host", _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(Q), _ptr(K), _ptr(V), _ptr(cu_seqlens_q),
             _ptr(cu_seqlens_k), B, T, K.shape[0], max_seqlen_q, max_seqlen_k, Hq, Hkv, d, H_I, d_I, k, scale,
             chunk_rows, _ptr(O), _ptr(buf["ws"]), buf["ws"].numel(), _stream())
    return O


def decode_workspace_bytes(batch: int, max_seqlen_k: int, Hq: int, d: int, k: int) -> int:
    return _lib.load().dsa_decode_workspace_size(batch, max_seqlen_k, Hq, d, k)


def decode(q_idx, k_idx, w, Q, K, V, cu_seqlens_k, max_seqlen_k: int, k: int, scale: Optional[float] = None,
           workspace: Optional[torch.Tensor] = None, out=None):
    """Whole DSA decode step for one new query row per sequence.

    Returns (indices [B, k] int32, O [B, Hq, d] bf16, lse [B, Hq] fp32).
    """
    B, Hq, d = Q.shape
    Hkv = K.shape[1]
    H_I, d_I = q_idx.shape[1], q_idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(B, max_seqlen_k, Hq, d, k), dtype=torch.uint8,
                                device=Q.device)
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=Q.device), torch.empty_like(Q),
               torch.empty((B, Hq), dtype=torch.float32, device=Q.device))
    indices, O, lse = out
    call("dsa_decode", _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(Q), _ptr(K), _ptr(V), _ptr(cu_seqlens_k), B,
         K.shape[0], max_seqlen_k, Hq, Hkv, d, H_I, d_I, k, scale, _ptr(indices), _ptr(O), _ptr(lse),
         _ptr(workspace), workspace.numel(), _stream())
    return indices, O, lse


def sparse_attn_prefill_bwd(Q, K, V, O, dO, lse, indices, cu_seqlens_q, cu_seqlens_k,
                            scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                            max_seqlen_k: Optional[int] = None):
    """Gradients dQ, dK, dV of sparse attention for fixed selected sets.

    max_seqlen_k: the longest key sequence; read from cu_seqlens_k (a device sync) if None.
    """
    T, Hq, d = Q.shape
    Tk, Hkv, _ = K.shape
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if max_seqlen_k is None:
        max_seqlen_k = int((cu_seqlens_k[1:] - cu_seqlens_k[:-1]).max().item()) if cu_seqlens_k.numel() > 1 else 0
    nbytes = _lib.load().dsa_sparse_attn_bwd_workspace_size(T, Tk, Hq, Hkv, d, max_seqlen_k)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=Q.device)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    call("dsa_sparse_attn_prefill_bwd", _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(dO), _ptr(lse), _ptr(indices),
         _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, T, Tk, max_seqlen_k, Hq, Hkv, d,
         indices.shape[1], scale, _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(workspace), workspace.numel(), _stream())
    return dQ, dK, dV


def indexer_kl_loss(Q, K, q_idx, k_idx, w, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                    scale: Optional[float] = None, chunk_rows: int = 4096,
                    workspace: Optional[torch.Tensor] = None):
    """Indexer KL loss against the dense attention distribution, with its gradients.

    Returns (loss [1] fp32, kl [T] fp32, dq_idx, dk_idx, dw) (gradients bf16).
    """
    T, Hq, d = Q.shape
    Tk, Hkv, _ = K.shape
    H_I, d_I = q_idx.shape[1], q_idx.shape[2]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    chunk_rows = max(1, min(chunk_rows, T))
    nbytes = _lib.load().dsa_indexer_kl_loss_workspace_size(T, Tk, max_seqlen_k, Hq, H_I, d_I, chunk_rows,
                                                            cu_seqlens_q.numel() - 1)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=Q.device)
    loss = torch.empty(1, dtype=torch.float32, device=Q.device)
    kl = torch.empty(T, dtype=torch.float32, device=Q.device)
    dq, dk, dw = torch.empty_like(q_idx), torch.empty_like(k_idx), torch.empty_like(w)
    call("dsa_indexer_kl_loss", _ptr(Q), _ptr(K), _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(cu_seqlens_q),
         _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, T, Tk, max_seqlen_q, max_seqlen_k, Hq, Hkv, d, H_I, d_I,
         scale, chunk_rows, _ptr(loss), _ptr(kl), _ptr(dq), _ptr(dk), _ptr(dw), _ptr(workspace),
         workspace.numel(), _stream())
    return loss, kl, dq, dk, dw


def indexer_kl_loss_sparse(Q, K, q_idx, k_idx, w, indices, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                           max_seqlen_k: int, scale: Optional[float] = None, chunk_rows: int = 4096,
                           workspace: Optional[torch.Tensor] = None):
    """Sparse-adaptation indexer KL loss over each row's selected set, with its gradients.

    Returns (loss [1] fp32, kl [T] fp32, dq_idx, dk_idx, dw) (gradients bf16).
    """
    T, Hq, d = Q.shape
    Tk, Hkv, _ = K.shape
    H_I, d_I = q_idx.shape[1], q_idx.shape[2]
    _check(indices, "indices", torch.int32, 2)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    chunk_rows = max(1, min(chunk_rows, T))
    nbytes = _lib.load().dsa_indexer_kl_loss_sparse_workspace_size(T, Tk, max_seqlen_k, Hq, H_I, d_I, chunk_rows,
                                                                   cu_seqlens_q.numel() - 1)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=Q.device)
    loss = torch.empty(1, dtype=torch.float32, device=Q.device)
    kl = torch.empty(T, dtype=torch.float32, device=Q.device)
    dq, dk, dw = torch.empty_like(q_idx), torch.empty_like(k_idx), torch.empty_like(w)
    call("dsa_indexer_kl_loss_sparse", _ptr(Q), _ptr(K), _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(indices),
         indices.shape[1], _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), cu_seqlens_q.numel() - 1, T, Tk, max_seqlen_q,
         max_seqlen_k, Hq, Hkv, d, H_I, d_I, scale, chunk_rows, _ptr(loss), _ptr(kl), _ptr(dq), _ptr(dk), _ptr(dw),
         _ptr(workspace), workspace.numel(), _stream())
    return loss, kl, dq, dk, dw


def device_status():
    """(status, detail) of the library's device status word; synchronises and clears it."""
    import ctypes
    st, det = ctypes.c_int(0), ctypes.c_int(0)
    call("dsa_get_device_status", ctypes.byref(st), ctypes.byref(det))
    return st.value, det.value
