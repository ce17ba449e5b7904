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
    _check_prefill(gen.prefill_32k(), seed=1)


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
    dK_h, dV_h = dK.float().cpu().numpy(), dV.float().cpu().numpy()
    grp = t["dO"].double().reshape(wl.Tq, wl.Hkv, wl.Hq // wl.Hkv, wl.d).sum(dim=(0, 2)).cpu().numpy()
    np.testing.assert_allclose(dV_h.sum(0), grp, rtol=2e-2, atol=2e-2 * np.abs(grp).max())
    assert np.max(np.abs(dK_h.sum(0))) <= 2e-2 * np.abs(dK_h).max() * np.sqrt(wl.Tk)
    a = float((t["k_idx"].float() * dk.float()).sum())
    b = float((t["w"].float() * dw.float()).sum())
    c = float((t["q_idx"].float() * dq.float()).sum())
    scale = max(abs(a), abs(b), abs(c), 1e-30)
    assert abs(a - b) <= 3e-2 * scale and abs(a - c) <= 3e-2 * scale
