"""fp64 CPU oracle for DeepSeek Sparse Attention (DSA) on a GQA decoder.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with the
CUDA library (``lightning_indexer_b200``) and never imports it; it reads only the
seeded inputs from ``workloads.generators`` (bf16 bit patterns), converts them to fp64
itself, and computes every result as the plain definition in fp64.

Sources (web pages describing the method; they print no formulas, so the formulas
below are the plainest reading of their prose):

* [S1] Keye-VL-2.0 technical-report summary, mqxn.cn/news/1966, section 1 (sparse
  attention): a lightweight "Lightning Indexer" scans every position with a single
  MQA-shared set of indexer keys; each query then keeps its 2048 most relevant
  positions and attends only to them, so O(L^2) becomes O(L*k); GQA is adapted to DSA
  (the indexer's selection is shared by all heads).  Training has a dense warm-up stage
  in which only the indexer is trained, by minimising the KL divergence between the
  indexer's distribution and the full attention distribution, then a sparse-adaptation
  stage in which gradients flow through sparse attention.
* [S8] Same summary, section 8 (inference/training systems): DSA-specific decode;
  the top-k must be deterministic so that training and inference select identical sets.
* [P2] QbitAI launch article, news.chathome.org: DSA is tuned for varlen (packed)
  sequences in long-sequence training.

Readings where the pages are silent (each listed again in the design notes):

* Indexer score  I[t,s] = sum_j w[t,j] * max(0, q_I[t,j,:] . k_I[s,:]), no extra scale.
* Causality is bottom-right aligned per sequence: query i of a sequence with Lq queries
  and Lk keys sees keys s <= i + (Lk - Lq).  Prefill has Lq == Lk; decode has Lq == 1.
* Top-k: the k largest scores among visible keys; equal scores are ordered by the lower
  key index; fewer than k visible keys selects all of them; the result is the ascending
  list of sequence-local key positions, padded with -1.  +0.0 and -0.0 compare equal.
* Attention over the selected set: softmax(Q.K^T * scale) V with scale = 1/sqrt(d),
  one set per token shared by every head (MQA indexer, [S1]); head h reads KV head
  h // (Hq/Hkv).  LSE is the natural-log log-sum-exp of the scaled logits.
* KL loss (dense warm-up, [S1]): target p[t,s] = (1/Hq) sum_h softmax_s(dense causal
  logits of head h), the L1-normalised head sum; indexer distribution q = softmax_s(I)
  over the same causal positions; KL_t = sum_s p (log p - log q) with 0 log 0 = 0;
  loss = mean of KL_t over all packed tokens; p is a constant for the gradient.
* Sparse-attention backward ([S1] sparse adaptation): the exact gradient of the
  forward above with respect to Q, K, V for a fixed selected set.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np


# ---------------------------------------------------------------------------------------
# bf16 decoding
# ---------------------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode uint16 bf16 bit patterns: the bf16 value is the fp32 with these 16 high bits."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------------------
# Causality
# ---------------------------------------------------------------------------------------

def visible_keys(i: int, Lq: int, Lk: int) -> int:
    """How many keys query i of a sequence sees: keys 0 .. i + (Lk - Lq), clipped to [0, Lk]."""
    return int(min(max(i + (Lk - Lq) + 1, 0), Lk))


# ---------------------------------------------------------------------------------------
# (a1) Lightning indexer  [S1]
# ---------------------------------------------------------------------------------------

def indexer_scores_row(q_idx_t: np.ndarray, w_t: np.ndarray, k_idx_vis: np.ndarray) -> np.ndarray:
    """Scores of one query token against its visible indexer keys, in fp64.

    q_idx_t [H_I, d_I], w_t [H_I], k_idx_vis [n, d_I]  ->  I [n]
    I[s] = sum_j w_t[j] * max(0, q_idx_t[j] . k_idx_vis[s]).
    """
    logits = k_idx_vis @ q_idx_t.T  # [n, H_I]: one dot product per (key, indexer head)
    return np.maximum(logits, 0.0) @ w_t


# ---------------------------------------------------------------------------------------
# (a2) Top-k selection  [S1] (2048 positions per token), [S8] (deterministic)
# ---------------------------------------------------------------------------------------

def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Ascending positions of the k largest scores; ties go to the lower position; -1 pad.

    ``scores`` holds the visible keys only (position s = array index).  The ranking key is
    (-score, position), so every selected score is >= every unselected one and, among equal
    scores, lower positions are selected first.
    """
    n = scores.shape[0]
    take = min(k, n)
    out = np.full(k, -1, dtype=np.int64)
    if take == 0:
        return out
    # +0.0 == -0.0 under numeric comparison, so they tie and fall back to position order
    order = np.lexsort((np.arange(n), -scores))
    out[:take] = np.sort(order[:take])
    return out


# ---------------------------------------------------------------------------------------
# (a3) Sparse GQA attention over the selected positions  [S1]
# ---------------------------------------------------------------------------------------

def sparse_attention_row(Q_t: np.ndarray, K_sel: np.ndarray, V_sel: np.ndarray, scale: float):
    """One query token, all heads, attending to the already-gathered selected keys.

    Q_t [Hq, d], K_sel/V_sel [n, Hkv, d] (the rows of the selected positions).
    Returns O [Hq, d] and LSE [Hq] (natural log; -inf and O = 0 for an empty set).
    """
    Hq, d = Q_t.shape
    Hkv = K_sel.shape[1]
    G = Hq // Hkv
    O = np.zeros((Hq, d))
    lse = np.full(Hq, -np.inf)
    if K_sel.shape[0] == 0:
        return O, lse
    for h in range(Hq):
        g = h // G
        x = (K_sel[:, g, :] @ Q_t[h]) * scale
        m = x.max()
        e = np.exp(x - m)
        z = e.sum()
        O[h] = (e @ V_sel[:, g, :]) / z
        lse[h] = m + math.log(z)
    return O, lse


# ---------------------------------------------------------------------------------------
# Whole-workload forward (prefill or decode)
# ---------------------------------------------------------------------------------------

class Decoded:
    """A workload with lazy fp64 decoding (large caches are decoded only where read)."""

    def __init__(self, wl):
        self.wl = wl
        self.cu_q = np.asarray(wl.cu_seqlens_q, dtype=np.int64)
        self.cu_k = np.asarray(wl.cu_seqlens_k, dtype=np.int64)
        self.scale = 1.0 / math.sqrt(wl.d)
        self._full = {}

    def full(self, name: str) -> np.ndarray:
        """The whole tensor ``name`` in fp64 (small workloads only)."""
        if name not in self._full:
            self._full[name] = bf16_to_f64(getattr(self.wl, name))
        return self._full[name]

    def rows(self, name: str, sel) -> np.ndarray:
        """Rows ``sel`` (a slice or an index array) of tensor ``name`` in fp64."""
        if name in self._full:
            return self._full[name][sel]
        return bf16_to_f64(getattr(self.wl, name)[sel])

    def seq_of_row(self, r: int):
        b = int(np.searchsorted(self.cu_q, r, side="right") - 1)
        i = r - int(self.cu_q[b])
        Lq = int(self.cu_q[b + 1] - self.cu_q[b])
        Lk = int(self.cu_k[b + 1] - self.cu_k[b])
        return b, i, Lq, Lk


def forward_row(D: Decoded, r: int, k: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Indexer scores, top-k set, attention output and LSE for packed query row ``r``."""
    k = D.wl.topk if k is None else k
    b, i, Lq, Lk = D.seq_of_row(r)
    k0 = int(D.cu_k[b])
    n = visible_keys(i, Lq, Lk)
    scores = indexer_scores_row(D.rows("q_idx", r), D.rows("w", r), D.rows("k_idx", slice(k0, k0 + n)))
    idx = topk_row(scores, k)
    sel = idx[idx >= 0] + k0
    O, lse = sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
    return {"scores": scores, "idx": idx, "O": O, "lse": lse}


def forward(D: Decoded, rows: Optional[Sequence[int]] = None, k: Optional[int] = None):
    """Forward over ``rows`` (default: all packed query rows).  Returns stacked arrays."""
    rows = range(D.wl.Tq) if rows is None else rows
    outs = [forward_row(D, int(r), k) for r in rows]
    return {
        "idx": np.stack([o["idx"] for o in outs]),
        "O": np.stack([o["O"] for o in outs]),
        "lse": np.stack([o["lse"] for o in outs]),
        "scores": [o["scores"] for o in outs],
    }


# ---------------------------------------------------------------------------------------
# Dense attention (used by the KL target, and as the k >= L special case)
# ---------------------------------------------------------------------------------------

def dense_attention_row(Q_t: np.ndarray, K_vis: np.ndarray, V_vis: np.ndarray, scale: float):
    """Full causal attention of one token over all visible keys (all positions selected)."""
    return sparse_attention_row(Q_t, K_vis, V_vis, scale)


def dense_target_row(Q_t: np.ndarray, K_vis: np.ndarray, scale: float) -> np.ndarray:
    """KL target for one token: p[s] = (1/Hq) sum_h softmax_s(Q_t[h] . K_vis[s, g(h)] * scale)."""
    Hq = Q_t.shape[0]
    G = Hq // K_vis.shape[1]
    p = np.zeros(K_vis.shape[0])
    for h in range(Hq):
        x = (K_vis[:, h // G, :] @ Q_t[h]) * scale
        e = np.exp(x - x.max())
        p += e / e.sum()
    return p / Hq


# ---------------------------------------------------------------------------------------
# (a5) Indexer KL loss and its gradient  [S1] dense warm-up
# ---------------------------------------------------------------------------------------

def kl_row(I_row: np.ndarray, p_row: np.ndarray):
    """KL(p || softmax(I)) for one token and its gradient with respect to I.

    Returns (KL, dKL/dI) with dKL/dI = softmax(I) - p (p is a constant).
    """
    m = I_row.max()
    logz = m + math.log(np.exp(I_row - m).sum())
    logq = I_row - logz
    pos = p_row > 0
    kl = float(np.sum(p_row[pos] * (np.log(p_row[pos]) - logq[pos])))
    return kl, np.exp(logq) - p_row


def indexer_kl_loss(D: Decoded):
    """Loss, per-token KL, and gradients w.r.t. q_idx, k_idx and w for a packed batch.

    loss = (1/T) sum_t KL_t.  With g[t,s] = dloss/dI[t,s] = (softmax(I_t) - p_t)[s] / T and
    x[t,j,s] = q_idx[t,j] . k_idx[s]:
      dw[t,j]       = sum_s g[t,s] * max(0, x[t,j,s])
      dq_idx[t,j,:] = w[t,j] * sum_s g[t,s] * [x[t,j,s] > 0] * k_idx[s,:]
      dk_idx[s,:]   = sum_t sum_j g[t,s] * w[t,j] * [x[t,j,s] > 0] * q_idx[t,j,:]
    (the derivative of max(0, x) is taken as 0 at x = 0).
    """
    T = D.wl.Tq
    q_idx, k_idx, w, Q, K = (D.full(n) for n in ("q_idx", "k_idx", "w", "Q", "K"))
    kl = np.zeros(T)
    dq = np.zeros_like(q_idx)
    dk = np.zeros_like(k_idx)
    dw = np.zeros_like(w)
    for r in range(T):
        kl[r], g, x = kl_row_terms(D, r)
        if x is None:
            continue
        b, i, Lq, Lk = D.seq_of_row(r)
        k0 = int(D.cu_k[b])
        kv = k_idx[k0:k0 + x.shape[0]]
        g = g / T
        gm = (g[:, None] * (x > 0)) * w[r][None, :]  # [n, H_I] = dloss/dx
        dw[r] = np.maximum(x, 0.0).T @ g
        dq[r] = gm.T @ kv
        dk[k0:k0 + x.shape[0]] += gm @ q_idx[r]
    return {"loss": float(kl.mean()), "kl": kl, "dq_idx": dq, "dk_idx": dk, "dw": dw}


def kl_row_terms(D: Decoded, r: int):
    """KL_r, dKL_r/dI[r, :] (not yet divided by T) and the indexer logits x [n, H_I] of row r."""
    b, i, Lq, Lk = D.seq_of_row(r)
    k0 = int(D.cu_k[b])
    n = visible_keys(i, Lq, Lk)
    if n == 0:
        return 0.0, None, None
    kv = D.rows("k_idx", slice(k0, k0 + n))
    x = kv @ D.rows("q_idx", r).T  # [n, H_I]
    I_row = np.maximum(x, 0.0) @ D.rows("w", r)
    p_row = dense_target_row(D.rows("Q", r), D.rows("K", slice(k0, k0 + n)), D.scale)
    kl, gI = kl_row(I_row, p_row)
    return kl, gI, x


def indexer_kl_grad_row(D: Decoded, r: int, T: int):
    """Row-local outputs of the KL loss for row r: KL_r, dw[r] and dq_idx[r] (fp64)."""
    kl, g, x = kl_row_terms(D, r)
    wr = D.rows("w", r)
    if x is None:
        return kl, np.zeros_like(wr), np.zeros((wr.shape[0], D.wl.d_I))
    b, i, Lq, Lk = D.seq_of_row(r)
    k0 = int(D.cu_k[b])
    kv = D.rows("k_idx", slice(k0, k0 + x.shape[0]))
    g = g / T
    gm = (g[:, None] * (x > 0)) * wr[None, :]
    return kl, np.maximum(x, 0.0).T @ g, gm.T @ kv


def indexer_kl_loss_sparse(D: Decoded, idx: np.ndarray):
    """Sparse-adaptation KL loss [S1]: the indexer KL of the dense warm-up restricted to each
    token's selected set, with its gradients w.r.t. q_idx, k_idx and w.

    [S1]'s second stage trains the whole model through sparse attention while the indexer
    keeps learning from the attention it selects for.  Reading: for row t with selected set
    S_t (sequence-local positions idx[t] >= 0),
      p[t,s] = (1/Hq) sum_h softmax_{s in S_t}(scale * Q[t,h] . K[s, g(h)])   (a constant:
               the head mean of the sparse attention weights)
      q[t,s] = softmax_{s in S_t}(I[t,s])
      KL_t   = sum_{s in S_t} p log(p/q);   loss = (1/T) sum_t KL_t
    and the gradients of indexer_kl_loss with g[t,s] = (q - p)[s] / T on S_t, 0 elsewhere.
    """
    T = D.wl.Tq
    q_idx, k_idx, w, Q, K = (D.full(n) for n in ("q_idx", "k_idx", "w", "Q", "K"))
    kl = np.zeros(T)
    dq = np.zeros_like(q_idx)
    dk = np.zeros_like(k_idx)
    dw = np.zeros_like(w)
    for r in range(T):
        b, i, Lq, Lk = D.seq_of_row(r)
        k0 = int(D.cu_k[b])
        sel = idx[r][idx[r] >= 0] + k0
        if sel.size == 0:
            continue
        kv = k_idx[sel]
        x = kv @ q_idx[r].T  # [n, H_I]
        I_row = np.maximum(x, 0.0) @ w[r]
        p_row = dense_target_row(Q[r], K[sel], D.scale)
        kl[r], gI = kl_row(I_row, p_row)
        g = gI / T
        gm = (g[:, None] * (x > 0)) * w[r][None, :]
        dw[r] = np.maximum(x, 0.0).T @ g
        dq[r] = gm.T @ kv
        np.add.at(dk, sel, gm @ q_idx[r])
    return {"loss": float(kl.mean()), "kl": kl, "dq_idx": dq, "dk_idx": dk, "dw": dw}


# ---------------------------------------------------------------------------------------
# (a6) Sparse-attention backward  [S1] sparse adaptation, [P2] varlen
# ---------------------------------------------------------------------------------------

def sparse_attention_backward(D: Decoded, idx: np.ndarray, O: np.ndarray, lse: np.ndarray,
                              dO: np.ndarray):
    """Gradients of the sparse attention forward for fixed selected sets.

    idx [Tq, k] (sequence-local positions, -1 pad), O [Tq, Hq, d], lse [Tq, Hq] (the
    forward's own fp64 outputs), dO [Tq, Hq, d].  For token t, head h, set S:
      P[s]  = exp(scale * Q[t,h].K[s] - lse[t,h])
      dS[s] = P[s] * (dO[t,h].V[s] - dO[t,h].O[t,h])
      dQ[t,h] = scale * sum_s dS[s] K[s];  dK[s] += scale * dS[s] Q[t,h];  dV[s] += P[s] dO[t,h]
    """
    wl = D.wl
    Hq, Hkv = wl.Hq, wl.Hkv
    G = Hq // Hkv
    Q, K, V = D.full("Q"), D.full("K"), D.full("V")
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for r in range(wl.Tq):
        b, i, Lq, Lk = D.seq_of_row(r)
        k0 = int(D.cu_k[b])
        sel = idx[r][idx[r] >= 0] + k0
        if sel.size == 0:
            continue
        for g in range(Hkv):
            hs = slice(g * G, (g + 1) * G)  # the query heads that read KV head g
            Ks = K[sel, g, :]
            Vs = V[sel, g, :]
            P = np.exp(D.scale * (Ks @ Q[r, hs].T) - lse[r, hs])                   # [n, G]
            dS = P * (Vs @ dO[r, hs].T - np.sum(dO[r, hs] * O[r, hs], axis=1))    # [n, G]
            dQ[r, hs] = D.scale * (dS.T @ Ks)
            # the sums over the group's heads (dS.Q and P.dO) are matrix products
            np.add.at(dK[:, g, :], sel, D.scale * (dS @ Q[r, hs]))
            np.add.at(dV[:, g, :], sel, P @ dO[r, hs])
    return {"dQ": dQ, "dK": dK, "dV": dV}


# ---------------------------------------------------------------------------------------
# Sampled-row helpers for workloads too large for the full oracle
# ---------------------------------------------------------------------------------------

def sample_rows(Tq: int, seed: int, n_first: int = 64, n_last: int = 64, n_mid: int = 128) -> List[int]:
    """The first ``n_first`` rows, the last ``n_last`` rows and ``n_mid`` uniform rows (seeded)."""
    rng = np.random.default_rng(seed)
    rows = set(range(min(n_first, Tq))) | set(range(max(0, Tq - n_last), Tq))
    if Tq > 0:
        rows |= set(int(x) for x in rng.integers(0, Tq, size=n_mid))
    return sorted(rows)
