"""Seeded synthetic inputs for the DSA hot path (lightning indexer, top-k, sparse GQA attention).

This module holds random-number generation and data layout only: shapes, the
fp32 -> bf16 rounding of samples, the varlen length draw and the long-video token
layout.  None of the method's arithmetic lives here.  The fp64 oracle and the CUDA
path both read the arrays built here, and nothing else is shared between them.

Where the inputs come from (the pages describe no dataset that is available here):

* Long video (Keye-VL-2.0 report summary, mqxn.cn/news/1966, section 3 on the
  timestamped frame layout): every frame is preceded by a few natural-language
  timestamp tokens.  The synthetic stand-in uses 8 timestamp tokens followed by 256
  frame tokens; keys and indexer keys inside a frame share a frame-mean vector
  N(0, 1) plus N(0, 0.25) noise, so frames are clustered and redundant.
* Varlen training (same summary, section 3 pixel budget of 12.5/25/50/100 %): the
  packed batch draws sequence lengths uniformly from {1/8, 1/4, 1/2, 1} x 16384.

All bf16 tensors are returned as ``numpy.uint16`` bit patterns (numpy has no bf16).
Random streams are counter-keyed per fixed-size chunk, so the result does not depend
on the number of threads used to produce it.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

_CHUNK = 1 << 22  # elements per independently seeded chunk
VIDEO_PERIOD = 264  # 8 timestamp tokens + 256 frame tokens
VIDEO_TEXT_PER_FRAME = 8

# stream ids: one independent random stream per tensor role
_S_QIDX, _S_KIDX, _S_W, _S_Q, _S_K, _S_V, _S_DO, _S_MEANK, _S_MEANKI, _S_LENS = range(1, 11)
_S_MEANQI, _S_MEANW = 11, 12


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 samples to bf16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + rounding) >> np.uint32(16)).astype(np.uint16)


def _rng(seed: int, stream: int, chunk: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, chunk])))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _normal_bf16(seed: int, stream: int, shape, row_mean: Optional[np.ndarray] = None,
                 mean_rows: Optional[np.ndarray] = None, noise_std: float = 1.0) -> np.ndarray:
    """bf16 bits of N(0,1) samples, or of ``mean + noise_std * N(0,1)`` where a row has a mean.

    ``shape`` is (rows, cols...).  ``mean_rows[r]`` is -1 for an unclustered row (plain
    N(0, 1)) or an index into ``row_mean`` (shape [n_means, cols...]) whose vector is added
    to ``noise_std`` times the noise of that row.
    """
    shape = tuple(int(s) for s in shape)
    rows = shape[0]
    row_elems = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    out = np.empty(rows * row_elems, dtype=np.uint16)
    rows_per_chunk = max(1, _CHUNK // row_elems)
    n_chunks = (rows + rows_per_chunk - 1) // rows_per_chunk

    def work(c: int) -> None:
        r0 = c * rows_per_chunk
        r1 = min(rows, r0 + rows_per_chunk)
        z = _rng(seed, stream, c).standard_normal((r1 - r0) * row_elems, dtype=np.float32)
        if mean_rows is not None:
            z = z.reshape(r1 - r0, row_elems)
            m = mean_rows[r0:r1]
            clustered = m >= 0
            if clustered.any():
                z[clustered] = row_mean.reshape(row_mean.shape[0], row_elems)[m[clustered]] \
                    + np.float32(noise_std) * z[clustered]
            z = z.reshape(-1)
        out[r0 * row_elems:r1 * row_elems] = f32_to_bf16_bits(z)

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(work, range(n_chunks)))
    return out.reshape(shape)


def _softmax_weights_bf16(seed: int, rows: int, H_I: int, row_mean: Optional[np.ndarray] = None,
                          mean_rows: Optional[np.ndarray] = None, noise_std: float = 1.0) -> np.ndarray:
    """Indexer head weights: per token, a softmax over H_I of N(0, 1) logits, stored bf16;
    where a row has a mean (as in ``_normal_bf16``) the logits are mean + noise_std * N(0, 1)."""
    z = _rng(seed, _S_W, 0).standard_normal((rows, H_I), dtype=np.float32)
    if mean_rows is not None:
        clustered = mean_rows >= 0
        z[clustered] = row_mean[mean_rows[clustered]] + np.float32(noise_std) * z[clustered]
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return f32_to_bf16_bits(e / e.sum(axis=1, keepdims=True))


def video_frame_ids(length: int, max_frames: Optional[int] = None) -> np.ndarray:
    """Per position: the frame id of a visual token, or -1 for a text/timestamp token.

    Layout: repeated blocks of 8 timestamp tokens then 256 frame tokens, starting at
    position 0.  Blocks at or beyond ``max_frames`` are text (the question after the
    video).
    """
    p = np.arange(length, dtype=np.int64)
    block = p // VIDEO_PERIOD
    r = p % VIDEO_PERIOD
    fid = np.where(r < VIDEO_TEXT_PER_FRAME, -1, block)
    if max_frames is not None:
        fid = np.where(block >= max_frames, -1, fid)
    return fid.astype(np.int64)


@dataclass
class Workload:
    """One batch of synthetic DSA inputs.  bf16 arrays are uint16 bit patterns.

    Token-major packed layout (varlen): query rows of all sequences are concatenated,
    and so are key rows; ``cu_seqlens_q/k`` hold the int32 offsets [B+1].
    """
    name: str
    kind: str  # "prefill" | "decode" | "train"
    Hq: int
    Hkv: int
    d: int
    H_I: int
    d_I: int
    topk: int
    cu_seqlens_q: np.ndarray
    cu_seqlens_k: np.ndarray
    q_idx: np.ndarray  # [Tq, H_I, d_I]
    k_idx: np.ndarray  # [Tk, d_I]
    w: np.ndarray  # [Tq, H_I]
    Q: np.ndarray  # [Tq, Hq, d]
    K: np.ndarray  # [Tk, Hkv, d]
    V: np.ndarray  # [Tk, Hkv, d]
    dO: Optional[np.ndarray] = None  # [Tq, Hq, d] (training only)
    seed: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return len(self.cu_seqlens_q) - 1

    @property
    def Tq(self) -> int:
        return int(self.cu_seqlens_q[-1])

    @property
    def Tk(self) -> int:
        return int(self.cu_seqlens_k[-1])

    @property
    def seqlens_q(self) -> np.ndarray:
        return np.diff(self.cu_seqlens_q)

    @property
    def seqlens_k(self) -> np.ndarray:
        return np.diff(self.cu_seqlens_k)

    def causal_pairs(self) -> int:
        """Number of (query, key) pairs with the key visible to the query (bottom-right causal)."""
        tot = 0
        for lq, lk in zip(self.seqlens_q.tolist(), self.seqlens_k.tolist()):
            i = np.arange(lq, dtype=np.int64)
            tot += int(np.clip(i + (lk - lq) + 1, 0, lk).sum())
        return tot

    def selected_pairs(self) -> int:
        """Number of (query, key) pairs attended after top-k: min(visible, topk) per query."""
        tot = 0
        for lq, lk in zip(self.seqlens_q.tolist(), self.seqlens_k.tolist()):
            i = np.arange(lq, dtype=np.int64)
            tot += int(np.minimum(np.clip(i + (lk - lq) + 1, 0, lk), self.topk).sum())
        return tot


def _cu(lens) -> np.ndarray:
    return np.concatenate([[0], np.cumsum(np.asarray(lens, dtype=np.int64))]).astype(np.int32)


def make_prefill(seqlens, Hq: int, Hkv: int, d: int, H_I: int, d_I: int, topk: int, seed: int,
                 layout: str = "gaussian", with_dO: bool = False, name: str = "prefill",
                 max_frames: Optional[int] = None, kind: str = "prefill") -> Workload:
    """Causal self-attention prefill over packed sequences (queries == keys per sequence).

    layout:
      "gaussian": every tensor N(0,1); w = softmax over H_I of N(0,1).
      "integer":  q_idx, k_idx integers uniform in [-8, 8] (inclusive); w uniform over
                  {1/2, 1/4, 1/8}; Q/K/V N(0,1).  Indexer scores are exact in fp32.
      "video":    per sequence, the timestamped-frame layout; K (per KV head) and k_idx of
                  frame tokens are frame-mean N(0,1) + N(0, 0.25) noise; the rest N(0,1).
      "video_coherent": "video", and the indexer queries q_idx of a frame's tokens also
                  share a frame mean N(0,1) (per head) plus N(0, 0.25) noise, so adjacent
                  tokens of a frame select partly the same positions.
      "video_overlap": "video_coherent" with N(0, 0.01) query noise around the frame mean and
                  head-weight logits that are a frame mean N(0,1) plus N(0, 0.01) noise, so the
                  16 adjacent tokens of a block select mostly the same positions (the overlap
                  the report summary gives for 128K video: about 8000 distinct positions for
                  16 queries at k = 2048).
    """
    seqlens = [int(x) for x in seqlens]
    T = sum(seqlens)
    cu = _cu(seqlens)
    if layout == "integer":
        g = _rng(seed, _S_QIDX, 0)
        q_idx = f32_to_bf16_bits(g.integers(-8, 9, size=(T, H_I, d_I)).astype(np.float32))
        g = _rng(seed, _S_KIDX, 0)
        k_idx = f32_to_bf16_bits(g.integers(-8, 9, size=(T, d_I)).astype(np.float32))
        g = _rng(seed, _S_W, 0)
        w = f32_to_bf16_bits(np.array([0.5, 0.25, 0.125], np.float32)[g.integers(0, 3, size=(T, H_I))])
        mean_rows_k = None
    else:
        q_idx = None
        w = None
        if layout in ("video", "video_coherent", "video_overlap"):
            fids = np.concatenate([video_frame_ids(L, max_frames) for L in seqlens])
            # frame ids are made unique across sequences
            offs = np.concatenate([[0], np.cumsum([L // VIDEO_PERIOD + 1 for L in seqlens])[:-1]])
            seq_of = np.repeat(np.arange(len(seqlens)), seqlens)
            mean_rows_k = np.where(fids >= 0, fids + offs[seq_of], -1)
            n_means = int(mean_rows_k.max()) + 1 if (mean_rows_k >= 0).any() else 1
            mean_ki = _normal_bf16_f32(seed, _S_MEANKI, (n_means, d_I))
            k_idx = _normal_bf16(seed, _S_KIDX, (T, d_I), row_mean=mean_ki, mean_rows=mean_rows_k,
                                 noise_std=0.5)
            if layout in ("video_coherent", "video_overlap"):
                mean_qi = _normal_bf16_f32(seed, _S_MEANQI, (n_means, H_I, d_I))
                q_idx = _normal_bf16(seed, _S_QIDX, (T, H_I, d_I), row_mean=mean_qi, mean_rows=mean_rows_k,
                                     noise_std=0.5 if layout == "video_coherent" else 0.1)
            if layout == "video_overlap":
                mean_w = _normal_bf16_f32(seed, _S_MEANW, (n_means, H_I))
                w = _softmax_weights_bf16(seed, T, H_I, row_mean=mean_w, mean_rows=mean_rows_k, noise_std=0.1)
        elif layout == "gaussian":
            mean_rows_k = None
            k_idx = _normal_bf16(seed, _S_KIDX, (T, d_I))
        else:
            raise ValueError(f"unknown layout {layout!r}")
        if q_idx is None:
            q_idx = _normal_bf16(seed, _S_QIDX, (T, H_I, d_I))
        if w is None:
            w = _softmax_weights_bf16(seed, T, H_I)
    Q = _normal_bf16(seed, _S_Q, (T, Hq, d))
    if layout in ("video", "video_coherent", "video_overlap"):
        mean_k = _normal_bf16_f32(seed, _S_MEANK, (int(mean_rows_k.max()) + 1, Hkv, d))
        K = _normal_bf16(seed, _S_K, (T, Hkv, d), row_mean=mean_k, mean_rows=mean_rows_k, noise_std=0.5)
    else:
        K = _normal_bf16(seed, _S_K, (T, Hkv, d))
    V = _normal_bf16(seed, _S_V, (T, Hkv, d))
    dO = _normal_bf16(seed, _S_DO, (T, Hq, d)) if with_dO else None
    return Workload(name=name, kind=kind, Hq=Hq, Hkv=Hkv, d=d, H_I=H_I, d_I=d_I, topk=topk,
                    cu_seqlens_q=cu, cu_seqlens_k=cu.copy(), q_idx=q_idx, k_idx=k_idx, w=w,
                    Q=Q, K=K, V=V, dO=dO, seed=seed, meta={"layout": layout, "seqlens": seqlens})


def _normal_bf16_f32(seed: int, stream: int, shape) -> np.ndarray:
    """N(0,1) frame-mean vectors in fp32 (they are summed with noise before rounding)."""
    return _rng(seed, stream, 0).standard_normal(shape, dtype=np.float32)


def make_decode(B: int, N: int, Hq: int, Hkv: int, d: int, H_I: int, d_I: int, topk: int,
                seed: int, layout: str = "video", name: str = "decode") -> Workload:
    """B independent sequences, each with an N-token K/V + indexer-key cache and one new query.

    The cache of sequence b is rows [b*N, (b+1)*N) of K, V, k_idx (so [B, N, Hkv, d] in
    memory); the query sees all N cached positions (the new token's own K/V is the last).
    With layout "video", the timestamped-frame pattern repeats from position 0 and is cut
    at N.
    """
    cu_q = _cu([1] * B)
    cu_k = _cu([N] * B)
    Tk = B * N
    q_idx = _normal_bf16(seed, _S_QIDX, (B, H_I, d_I))
    w = _softmax_weights_bf16(seed, B, H_I)
    Q = _normal_bf16(seed, _S_Q, (B, Hq, d))
    if layout == "video":
        fid = video_frame_ids(N)
        per_seq = int(fid.max()) + 1
        mean_rows = np.concatenate([np.where(fid >= 0, fid + b * per_seq, -1) for b in range(B)])
        mean_ki = _normal_bf16_f32(seed, _S_MEANKI, (B * per_seq, d_I))
        mean_k = _normal_bf16_f32(seed, _S_MEANK, (B * per_seq, Hkv, d))
        k_idx = _normal_bf16(seed, _S_KIDX, (Tk, d_I), row_mean=mean_ki, mean_rows=mean_rows, noise_std=0.5)
        K = _normal_bf16(seed, _S_K, (Tk, Hkv, d), row_mean=mean_k, mean_rows=mean_rows, noise_std=0.5)
    elif layout == "gaussian":
        k_idx = _normal_bf16(seed, _S_KIDX, (Tk, d_I))
        K = _normal_bf16(seed, _S_K, (Tk, Hkv, d))
    else:
        raise ValueError(f"unknown layout {layout!r}")
    V = _normal_bf16(seed, _S_V, (Tk, Hkv, d))
    return Workload(name=name, kind="decode", Hq=Hq, Hkv=Hkv, d=d, H_I=H_I, d_I=d_I, topk=topk,
                    cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, q_idx=q_idx, k_idx=k_idx, w=w,
                    Q=Q, K=K, V=V, seed=seed, meta={"layout": layout, "N": N})


def pixel_budget_lengths(total: int, seed: int, base: int = 16384) -> list:
    """Varlen draw: lengths uniform over {base/8, base/4, base/2, base} until the next draw
    would overflow ``total``; the last sequence takes the remainder."""
    g = _rng(seed, _S_LENS, 0)
    choices = [base // 8, base // 4, base // 2, base]
    lens, acc = [], 0
    while acc < total:
        L = choices[int(g.integers(0, 4))]
        if acc + L > total:
            lens.append(total - acc)
            break
        lens.append(L)
        acc += L
    return lens


# ---------------------------------------------------------------------------------------
# The five named workloads.  Head shapes of the three large ones follow the
# Qwen3-30B-A3B attention layer (Hq=32, Hkv=4, d=128) that hosts DSA in Keye-VL-2.0.
# ---------------------------------------------------------------------------------------

def tiny_integer_1k() -> Workload:
    """L=1024 causal prefill; Hq=8, Hkv=2, d=64; H_I=4, d_I=32, k=128; integer indexer inputs."""
    return make_prefill([1024], 8, 2, 64, 4, 32, 128, seed=0, layout="integer", name="tiny_integer_1k")


def prefill_32k() -> Workload:
    """L=32768 causal prefill, batch 1, all tensors N(0,1)."""
    return make_prefill([32768], 32, 4, 128, 64, 128, 2048, seed=1, layout="gaussian", name="prefill_32k")


def video_prefill_128k() -> Workload:
    """L=131072 long-video prefill: 480 x (8 timestamp + 256 frame tokens) + 4352 text tokens."""
    return make_prefill([131072], 32, 4, 128, 64, 128, 2048, seed=2, layout="video",
                        name="video_prefill_128k", max_frames=480)


def video_prefill_128k_coherent() -> Workload:
    """The 128K long-video prefill with frame-coherent indexer queries (high set overlap)."""
    return make_prefill([131072], 32, 4, 128, 64, 128, 2048, seed=2, layout="video_coherent",
                        name="video_prefill_128k_coherent", max_frames=480)


def video_prefill_128k_overlap() -> Workload:
    """The 128K long-video prefill with the report's adjacent-query overlap (high set overlap)."""
    return make_prefill([131072], 32, 4, 128, 64, 128, 2048, seed=2, layout="video_overlap",
                        name="video_prefill_128k_overlap", max_frames=480)


def decode_256k() -> Workload:
    """Decode: 16 sequences, 262144 cached tokens each, clustered like the video prefill."""
    return make_decode(16, 262144, 32, 4, 128, 64, 128, 2048, seed=3, layout="video", name="decode_256k")


def train_varlen_64k() -> Workload:
    """Training step: 65536 packed tokens, pixel-budget varlen lengths, with dO."""
    lens = pixel_budget_lengths(65536, seed=4)
    return make_prefill(lens, 32, 4, 128, 64, 128, 2048, seed=4, layout="gaussian", with_dO=True,
                        name="train_varlen_64k", kind="train")


NAMED = {
    "tiny_integer_1k": tiny_integer_1k,
    "prefill_32k": prefill_32k,
    "video_prefill_128k": video_prefill_128k,
    "decode_256k": decode_256k,
    "train_varlen_64k": train_varlen_64k,
}
