"""Full-size parity on the four large workloads, in the launch configuration bench.py
times (prefill in 8192-row chunks), against the fp64 oracle on sampled rows.

Sampled rows: the first 64, the last 64 and 128 seeded uniform rows (each row's scores,
set and attention output are independent of the other rows, so the oracle computes them
one by one).  Column reductions that couple every row (dk_idx, dK, dV) are checked with
identities that hold at any size.
"""
import numpy as np
import pytest
import torch

import lightning_indexer_b200 as dsa
from oracle import dsa_oracle as orc
from workloads import generators as gen

from dsa_testutil import set_mismatch_ok, to_device

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ATTN_ATOL = 1e-2
SCORE_RTOL = 2e-5  # fp32 accumulation of 128-term bf16 products vs fp64, relative to the row max


def _rows(T, seed):
    return orc.sample_rows(T, seed=seed, n_first=64, n_last=64, n_mid=128)


def _check_prefill(wl, chunk=8192, seed=0):
    t = to_device(wl)
    D = orc.Decoded(wl)
    L = t["max_k"]
    ld = (L + 3) // 4 * 4
    rows = _rows(wl.Tq, seed)
    # scores of sampled rows, chunk by chunk exactly as the pipeline computes them
    scores = torch.empty((chunk, ld), dtype=torch.float32, device="cuda")
    got_scores = {}
    for r0 in range(0, wl.Tq, chunk):
        r1 = min(wl.Tq, r0 + chunk)
        want = [r for r in rows if r0 <= r < r1]
        if not want:
            continue
        dsa.index(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], L, r0, r1,
                  scores=scores[: r1 - r0])
        sel = torch.tensor([r - r0 for r in want], device="cuda")
        block = scores[sel].cpu().numpy()
        for j, r in enumerate(want):
            got_scores[r] = block[j]
    idx, O, lse = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                              t["max_q"], L, wl.topk, chunk_rows=chunk)
    idx, O, lse = idx.cpu().numpy(), O.float().cpu().numpy(), lse.cpu().numpy()
    exact_rows = 0
    for r in rows:
        ref = orc.forward_row(D, r)
        n = ref["scores"].size
        err = np.max(np.abs(got_scores[r][:n] - ref["scores"]))
        assert err <= SCORE_RTOL * np.max(np.abs(ref["scores"])) + 1e-6, (r, err)
        ok, nsw = set_mismatch_ok(idx[r], ref["idx"], ref["scores"])
        assert ok, r
        if nsw == 0:
            exact_rows += 1
            assert np.max(np.abs(O[r] - ref["O"])) <= ATTN_ATOL, r
            assert np.max(np.abs(lse[r] - ref["lse"])) <= 2e-3, r
    assert exact_rows >= 0.8 * len(rows)
    return t, idx, O, lse


def test_prefill_32k_sampled_rows():
    t, idx, O, lse = _check_prefill(gen.prefill_32k(), seed=1)
    # the tensor-core entry point on the same selections: every row against the gather
    # kernel's, each within its own bound of the oracle, so within twice that of each other
    O2, l2 = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], torch.from_numpy(idx).cuda(), t["cu_q"], t["cu_k"],
                                     kernel="tensor_core")
    assert np.max(np.abs(O2.float().cpu().numpy() - O)) <= 2 * ATTN_ATOL
    assert np.max(np.abs(l2.cpu().numpy() - lse)) <= 2 * 2e-3


def test_video_prefill_128k_sampled_rows():
    _check_prefill(gen.video_prefill_128k(), seed=2)


def test_decode_256k_all_rows():
    wl = gen.decode_256k()
    t = to_device(wl)
    idx, O, lse = dsa.decode(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_k"], t["max_k"],
                             wl.topk)
    idx, O, lse = idx.cpu().numpy(), O.float().cpu().numpy(), lse.cpu().numpy()
    D = orc.Decoded(wl)
    for r in range(wl.B):
        ref = orc.forward_row(D, r)
        ok, nsw = set_mismatch_ok(idx[r], ref["idx"], ref["scores"])
        assert ok, r
        if nsw == 0:
            assert np.max(np.abs(O[r] - ref["O"])) <= ATTN_ATOL, r
            assert np.max(np.abs(lse[r] - ref["lse"])) <= 2e-3, r


def _one_sequence(wl, b):
    """Sequence b of a packed training workload as a workload of its own (same arrays)."""
    q0, q1 = int(wl.cu_seqlens_q[b]), int(wl.cu_seqlens_q[b + 1])
    k0, k1 = int(wl.cu_seqlens_k[b]), int(wl.cu_seqlens_k[b + 1])
    cu_q = np.array([0, q1 - q0], np.int32)
    cu_k = np.array([0, k1 - k0], np.int32)
    return gen.Workload(name=f"{wl.name}[{b}]", kind=wl.kind, Hq=wl.Hq, Hkv=wl.Hkv, d=wl.d, H_I=wl.H_I,
                        d_I=wl.d_I, topk=wl.topk, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
                        q_idx=wl.q_idx[q0:q1], k_idx=wl.k_idx[k0:k1], w=wl.w[q0:q1], Q=wl.Q[q0:q1],
                        K=wl.K[k0:k1], V=wl.V[k0:k1], dO=wl.dO[q0:q1], seed=wl.seed)


def _rel(got, ref):
    return float(np.max(np.abs(got - ref)) / max(float(np.max(np.abs(ref))), 1e-30))


def test_train_varlen_64k_sampled_rows_and_identities():
    wl = gen.train_varlen_64k()
    t = to_device(wl)
    D = orc.Decoded(wl)
    L = t["max_k"]
    # forward + sparse backward (the training step's calls)
    idx, O, lse = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                              t["max_q"], L, wl.topk, chunk_rows=8192)
    dQ, dK, dV = dsa.sparse_attn_prefill_bwd(t["Q"], t["K"], t["V"], O, t["dO"], lse, idx, t["cu_q"], t["cu_k"])
    loss, kl, dq, dk, dw = dsa.indexer_kl_loss(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"], t["cu_q"],
                                               t["cu_k"], t["max_q"], L, chunk_rows=8192)
    idx_h, dQ_h = idx.cpu().numpy(), dQ.float().cpu().numpy()
    dK_h, dV_h = dK.float().cpu().numpy(), dV.float().cpu().numpy()
    kl_h, dq_h, dw_h = kl.cpu().numpy(), dq.float().cpu().numpy(), dw.float().cpu().numpy()
    rows = _rows(wl.Tq, 4)
    for r in rows:
        # KL row terms and the row-local gradients
        kl_r, dw_r, dq_r = orc.indexer_kl_grad_row(D, r, wl.Tq)
        assert abs(kl_h[r] - kl_r) <= 1e-4 * max(abs(kl_r), 1.0), r
        assert np.max(np.abs(dw_h[r] - dw_r)) <= 1.5e-2 * np.max(np.abs(dw_r)) + 1e-12, r
        assert np.max(np.abs(dq_h[r] - dq_r)) <= 1.5e-2 * np.max(np.abs(dq_r)) + 1e-12, r
        # sparse-attention dQ of rows whose selected set equals the oracle's
        ref = orc.forward_row(D, r)
        if np.array_equal(idx_h[r], ref["idx"]):
            b, i, Lq, Lk = D.seq_of_row(r)
            sel = ref["idx"][ref["idx"] >= 0] + int(D.cu_k[b])
            Ks, Vs, Qr, dOr = D.rows("K", sel), D.rows("V", sel), D.rows("Q", r), D.rows("dO", r)
            G = wl.Hq // wl.Hkv
            dq_ref = np.zeros_like(Qr)
            for h in range(wl.Hq):
                g = h // G
                P = np.exp(D.scale * (Ks[:, g] @ Qr[h]) - ref["lse"][h])
                dS = P * (Vs[:, g] @ dOr[h] - float(dOr[h] @ ref["O"][h]))
                dq_ref[h] = D.scale * (dS @ Ks[:, g])
            assert np.max(np.abs(dQ_h[r] - dq_ref)) <= 1.5e-2 * np.max(np.abs(dq_ref)) + 1e-6, r
    # identities over all rows
    assert abs(loss.item() - kl_h.mean()) <= 1e-5 * max(abs(kl_h.mean()), 1.0)
    grp = t["dO"].double().reshape(wl.Tq, wl.Hkv, wl.Hq // wl.Hkv, wl.d).sum(dim=(0, 2)).cpu().numpy()
    np.testing.assert_allclose(dV_h.sum(0), grp, rtol=2e-2, atol=2e-2 * np.abs(grp).max())
    assert np.max(np.abs(dK_h.sum(0))) <= 2e-2 * np.abs(dK_h).max() * np.sqrt(wl.Tk)
    a = float((t["k_idx"].float() * dk.float()).sum())
    b = float((t["w"].float() * dw.float()).sum())
    c = float((t["q_idx"].float() * dq.float()).sum())
    scale = max(abs(a), abs(b), abs(c), 1e-30)
    assert abs(a - b) <= 3e-2 * scale and abs(a - c) <= 3e-2 * scale

    # Element-wise on whole sequences: attention and the KL loss are block-diagonal over
    # the packed sequences, so the oracle run on one sequence alone gives every gradient
    # of that sequence's rows and keys (the KL gradients divided by the packed T, not the
    # sequence's).  The 2048-long sequences sit in the middle and at the end of the pack,
    # so their key tiles, dk work items and row offsets come after those of the 16384-long
    # sequences.
    seqlens = np.diff(wl.cu_seqlens_q)
    dk_h = dk.float().cpu().numpy()
    for b in [i for i, L in enumerate(seqlens) if L == 2048]:
        sub = _one_sequence(wl, b)
        Ds = orc.Decoded(sub)
        q0, q1 = int(wl.cu_seqlens_q[b]), int(wl.cu_seqlens_q[b + 1])
        # k = 2048 covers every visible key of a 2048-long sequence: the sets are exact
        ref_f = orc.forward(Ds)
        assert np.array_equal(idx_h[q0:q1], ref_f["idx"]), b
        ref_b = orc.sparse_attention_backward(Ds, ref_f["idx"], ref_f["O"], ref_f["lse"], Ds.full("dO"))
        assert _rel(dQ_h[q0:q1], ref_b["dQ"]) <= 1.5e-2, b
        assert _rel(dK_h[q0:q1], ref_b["dK"]) <= 1.5e-2, b
        assert _rel(dV_h[q0:q1], ref_b["dV"]) <= 1.5e-2, b
        ref_kl = orc.indexer_kl_loss(Ds)
        f = sub.Tq / wl.Tq  # the oracle divides g by the sequence's rows, the packed loss by all rows
        assert np.max(np.abs(kl_h[q0:q1] - ref_kl["kl"])) <= 1e-4 * np.max(np.abs(ref_kl["kl"])) + 1e-6, b
        assert _rel(dq_h[q0:q1], f * ref_kl["dq_idx"]) <= 1.5e-2, b
        assert _rel(dw_h[q0:q1], f * ref_kl["dw"]) <= 1.5e-2, b
        assert _rel(dk_h[q0:q1], f * ref_kl["dk_idx"]) <= 1.5e-2, b

    # Conditional check of dK and dV at 64 sampled key positions of the long sequences:
    # each sampled key's gradient is summed by the oracle over every row whose GPU-selected
    # set holds it, using the GPU's O and lse for those rows (both verified above on the
    # sampled rows), as the definition of the backward prescribes.
    O_h = O.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    rng = np.random.default_rng(44)
    long_seqs = [i for i, L in enumerate(seqlens) if L >= 8192]
    G = wl.Hq // wl.Hkv
    sampled = []
    for j in range(64):
        b = long_seqs[j % len(long_seqs)]
        L = int(seqlens[b])
        s = (0, L - 1, L // 2)[j // len(long_seqs)] if j < 3 * len(long_seqs) else int(rng.integers(0, L))
        sampled.append((b, s))
    got_k, got_v, want_k, want_v = [], [], [], []
    for b, s in sampled:
        q0, q1 = int(wl.cu_seqlens_q[b]), int(wl.cu_seqlens_q[b + 1])
        kg = int(wl.cu_seqlens_k[b]) + s
        rows = q0 + torch.nonzero((idx[q0:q1] == s).any(dim=1)).flatten().cpu().numpy()
        Kk, Vk = D.rows("K", kg), D.rows("V", kg)  # [Hkv, d]
        Qr = D.rows("Q", rows).reshape(len(rows), wl.Hkv, G, wl.d)
        dOr = D.rows("dO", rows).reshape(len(rows), wl.Hkv, G, wl.d)
        Or = O_h[rows].astype(np.float64).reshape(len(rows), wl.Hkv, G, wl.d)
        lr = lse_h[rows].astype(np.float64).reshape(len(rows), wl.Hkv, G)
        P = np.exp(D.scale * np.einsum("rgjc,gc->rgj", Qr, Kk) - lr)
        dS = P * (np.einsum("rgjc,gc->rgj", dOr, Vk) - np.sum(dOr * Or, axis=3))
        want_k.append(D.scale * np.einsum("rgj,rgjc->gc", dS, Qr))
        want_v.append(np.einsum("rgj,rgjc->gc", P, dOr))
        got_k.append(dK_h[kg])
        got_v.append(dV_h[kg])
    assert _rel(np.stack(got_k), np.stack(want_k)) <= 1.5e-2
    assert _rel(np.stack(got_v), np.stack(want_v)) <= 1.5e-2
