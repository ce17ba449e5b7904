"""GPU parity of the training rows: sparse-attention backward and the indexer KL loss
(with its gradients), through the C ABI, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import lightning_indexer_b200 as dsa
from oracle import dsa_oracle as orc
from workloads import generators as gen

from dsa_testutil import set_mismatch_ok, to_device

pytestmark = pytest.mark.gpu


def _rel_err(got, ref):
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


@pytest.mark.parametrize("Hq,Hkv,d,k", [(8, 2, 64, 32), (32, 4, 128, 64), (16, 4, 64, 48), (32, 4, 128, 16)])
def test_sparse_attention_backward(Hq, Hkv, d, k):
    # d = 128, 8 heads per KV head: k = 64 takes the masked dense path (8 k >= 211), k = 16 the gather path
    wl = gen.make_prefill([150, 33, 211], Hq, Hkv, d, 4, 32, k, seed=51, with_dO=True, layout="video")
    D = orc.Decoded(wl)
    ref_f = orc.forward(D, k=k)
    ref = orc.sparse_attention_backward(D, ref_f["idx"], ref_f["O"], ref_f["lse"], D.full("dO"))
    t = to_device(wl)
    idx = torch.from_numpy(ref_f["idx"].astype(np.int32)).cuda()
    O, lse = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], idx, t["cu_q"], t["cu_k"])
    dQ, dK, dV = dsa.sparse_attn_prefill_bwd(t["Q"], t["K"], t["V"], O, t["dO"], lse, idx, t["cu_q"], t["cu_k"])
    dQ, dK, dV = (x.float().cpu().numpy() for x in (dQ, dK, dV))
    # bf16 weights inside the products and bf16 outputs: ~2^-8 relative per element
    assert _rel_err(dQ, ref["dQ"]) <= 1.5e-2
    assert _rel_err(dK, ref["dK"]) <= 1.5e-2
    assert _rel_err(dV, ref["dV"]) <= 1.5e-2
    # the identities that hold at any size
    assert np.max(np.abs(dK.reshape(-1, Hkv, d).sum(0))) <= 2e-2 * np.max(np.abs(ref["dK"])) * np.sqrt(wl.Tk)
    grp = D.full("dO").reshape(wl.Tq, Hkv, Hq // Hkv, d).sum(axis=(0, 2))
    np.testing.assert_allclose(dV.sum(0), grp, rtol=2e-2, atol=2e-2 * np.abs(grp).max())


@pytest.mark.parametrize("Hq,Hkv,d", [(8, 2, 64), (16, 2, 128)])
def test_sparse_attention_backward_padded_sets(Hq, Hkv, d):
    # d = 128 with 8 query heads per KV head takes the masked dense tensor-core path
    wl = gen.make_prefill([40], Hq, Hkv, d, 4, 32, 32, seed=52, with_dO=True)
    D = orc.Decoded(wl)
    idx = np.full((40, 32), -1, np.int64)
    for r in range(40):
        n = min(r + 1, 32 if r % 3 else 5)
        idx[r, :n] = np.sort(np.random.default_rng(r).choice(r + 1, size=n, replace=False))
    O, lse = [], []
    for r in range(40):
        sel = idx[r][idx[r] >= 0]
        o, l = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        O.append(o)
        lse.append(l)
    ref = orc.sparse_attention_backward(D, idx, np.stack(O), np.stack(lse), D.full("dO"))
    t = to_device(wl)
    tidx = torch.from_numpy(idx.astype(np.int32)).cuda()
    Og, lg = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], tidx, t["cu_q"], t["cu_k"])
    dQ, dK, dV = dsa.sparse_attn_prefill_bwd(t["Q"], t["K"], t["V"], Og, t["dO"], lg, tidx, t["cu_q"], t["cu_k"])
    assert _rel_err(dQ.float().cpu().numpy(), ref["dQ"]) <= 1.5e-2
    assert _rel_err(dK.float().cpu().numpy(), ref["dK"]) <= 1.5e-2
    assert _rel_err(dV.float().cpu().numpy(), ref["dV"]) <= 1.5e-2


@pytest.mark.parametrize("H_I,Hq,Hkv,d", [(16, 8, 2, 64), (64, 32, 4, 128), (32, 16, 4, 128), (64, 16, 2, 128)])
def test_indexer_kl_loss(H_I, Hq, Hkv, d):
    wl = gen.make_prefill([260, 1, 129, 75], Hq, Hkv, d, H_I, 128, 64, seed=53, layout="video")
    D = orc.Decoded(wl)
    ref = orc.indexer_kl_loss(D)
    t = to_device(wl)
    for chunk in (wl.Tq, 100):
        loss, kl, dq, dk, dw = dsa.indexer_kl_loss(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"], t["cu_q"],
                                                   t["cu_k"], t["max_q"], t["max_k"], chunk_rows=chunk)
        kl = kl.cpu().numpy()
        assert abs(loss.item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-6
        assert np.max(np.abs(kl - ref["kl"])) <= 1e-4 * np.max(np.abs(ref["kl"])) + 1e-6
        assert _rel_err(dq.float().cpu().numpy(), ref["dq_idx"]) <= 1.5e-2
        assert _rel_err(dk.float().cpu().numpy(), ref["dk_idx"]) <= 1.5e-2
        assert _rel_err(dw.float().cpu().numpy(), ref["dw"]) <= 1.5e-2


def test_indexer_kl_gradient_homogeneity_identity():
    # I is positively homogeneous of degree 1 in k_idx, in w and in q_idx, so
    # sum_s k.dk = sum_{t,j} w.dw = sum_{t,j} q.dq = sum_{t,s} g I  (any size)
    wl = gen.make_prefill([500, 300], 16, 4, 64, 64, 128, 64, seed=54)
    t = to_device(wl)
    loss, kl, dq, dk, dw = dsa.indexer_kl_loss(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"], t["cu_q"],
                                               t["cu_k"], t["max_q"], t["max_k"])
    a = float((t["k_idx"].float() * dk.float()).sum())
    b = float((t["w"].float() * dw.float()).sum())
    c = float((t["q_idx"].float() * dq.float()).sum())
    scale = max(abs(a), abs(b), abs(c), 1e-30)
    assert abs(a - b) <= 3e-2 * scale and abs(a - c) <= 3e-2 * scale


def test_training_medium_varlen_elementwise():
    # Four packed sequences [2048, 1024, 512, 512], k = 512, Hq = 8, Hkv = 1, d = 128,
    # H_I = 64, d_I = 128: every training kernel takes its tensor-core path (8 k >= 2048),
    # the 2048-long sequence spans 16 key tiles of 128 and 8 KL dk items of 256 rows per
    # tile, rows past 512 select a sparse set, and the later sequences sit at non-zero
    # offsets of the pack.  Every element of dQ, dK, dV, dq_idx, dk_idx and dw is compared
    # with the oracle.
    wl = gen.make_prefill([2048, 1024, 512, 512], 8, 1, 128, 64, 128, 512, seed=55, with_dO=True,
                          layout="video")
    D = orc.Decoded(wl)
    ref_f = orc.forward(D)
    t = to_device(wl)
    # the pipeline (indexer, top-k, masked dense attention) on the selected sets
    idx_p, O_p, lse_p = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                                    t["max_q"], t["max_k"], wl.topk, chunk_rows=1024)
    idx_p, O_p, lse_p = idx_p.cpu().numpy(), O_p.float().cpu().numpy(), lse_p.cpu().numpy()
    exact = 0
    for r in range(wl.Tq):
        ok, nsw = set_mismatch_ok(idx_p[r], ref_f["idx"][r], ref_f["scores"][r])
        assert ok, r
        if nsw == 0:
            exact += 1
            assert np.max(np.abs(O_p[r] - ref_f["O"][r])) <= 1e-2, r
            assert np.max(np.abs(lse_p[r] - ref_f["lse"][r])) <= 2e-3, r
    assert exact >= 0.9 * wl.Tq
    # backward on the oracle's sets, from the GPU forward's O and lse
    ref_b = orc.sparse_attention_backward(D, ref_f["idx"], ref_f["O"], ref_f["lse"], D.full("dO"))
    idx = torch.from_numpy(ref_f["idx"].astype(np.int32)).cuda()
    O, lse = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], idx, t["cu_q"], t["cu_k"])
    dQ, dK, dV = dsa.sparse_attn_prefill_bwd(t["Q"], t["K"], t["V"], O, t["dO"], lse, idx, t["cu_q"], t["cu_k"],
                                             max_seqlen_k=t["max_k"])
    assert _rel_err(dQ.float().cpu().numpy(), ref_b["dQ"]) <= 1.5e-2
    assert _rel_err(dK.float().cpu().numpy(), ref_b["dK"]) <= 1.5e-2
    assert _rel_err(dV.float().cpu().numpy(), ref_b["dV"]) <= 1.5e-2
    # indexer KL loss and its gradients, in row chunks of 1024 and in one chunk
    ref = orc.indexer_kl_loss(D)
    for chunk in (1024, wl.Tq):
        loss, kl, dq, dk, dw = dsa.indexer_kl_loss(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"], t["cu_q"],
                                                   t["cu_k"], t["max_q"], t["max_k"], chunk_rows=chunk)
        kl = kl.cpu().numpy()
        assert abs(loss.item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-6
        assert np.max(np.abs(kl - ref["kl"])) <= 1e-4 * np.max(np.abs(ref["kl"])) + 1e-6
        assert _rel_err(dq.float().cpu().numpy(), ref["dq_idx"]) <= 1.5e-2
        assert _rel_err(dk.float().cpu().numpy(), ref["dk_idx"]) <= 1.5e-2
        assert _rel_err(dw.float().cpu().numpy(), ref["dw"]) <= 1.5e-2


@pytest.mark.parametrize("H_I,Hq,Hkv", [(64, 32, 4), (32, 16, 2), (64, 8, 1)])
def test_indexer_kl_loss_sparse(H_I, Hq, Hkv):
    # sparse-adaptation KL over the oracle's selected sets (k = 64: rows past 64 select a
    # strict subset), in one chunk and in chunks of 100 rows
    wl = gen.make_prefill([260, 1, 129, 75], Hq, Hkv, 128, H_I, 128, 64, seed=56, layout="video")
    D = orc.Decoded(wl)
    idx = np.stack([orc.forward_row(D, r, 64)["idx"] for r in range(wl.Tq)])
    ref = orc.indexer_kl_loss_sparse(D, idx)
    t = to_device(wl)
    tidx = torch.from_numpy(idx.astype(np.int32)).cuda()
    for chunk in (wl.Tq, 100):
        loss, kl, dq, dk, dw = dsa.indexer_kl_loss_sparse(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"], tidx,
                                                          t["cu_q"], t["cu_k"], t["max_q"], t["max_k"],
                                                          chunk_rows=chunk)
        kl = kl.cpu().numpy()
        assert abs(loss.item() - ref["loss"]) <= 1e-4 * abs(ref["loss"]) + 1e-6
        assert np.max(np.abs(kl - ref["kl"])) <= 1e-4 * np.max(np.abs(ref["kl"])) + 1e-6
        assert _rel_err(dq.float().cpu().numpy(), ref["dq_idx"]) <= 1.5e-2
        assert _rel_err(dk.float().cpu().numpy(), ref["dk_idx"]) <= 1.5e-2
        assert _rel_err(dw.float().cpu().numpy(), ref["dw"]) <= 1.5e-2
        # keys no row selected get exactly zero gradient
        chosen = np.zeros(wl.Tk, bool)
        for r in range(wl.Tq):
            b = D.seq_of_row(r)[0]
            chosen[idx[r][idx[r] >= 0] + int(D.cu_k[b])] = True
        assert np.all(dk.float().cpu().numpy()[~chosen] == 0)


def test_indexer_kl_loss_sparse_with_every_position_selected_matches_dense():
    # k >= every row's visible count: the sparse-adaptation loss is the dense warm-up loss
    wl = gen.make_prefill([300, 200], 32, 4, 128, 64, 128, 512, seed=57, layout="video")
    D = orc.Decoded(wl)
    idx = np.stack([orc.forward_row(D, r, 512)["idx"] for r in range(wl.Tq)])
    t = to_device(wl)
    dense = dsa.indexer_kl_loss(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"],
                                t["max_k"])
    sparse = dsa.indexer_kl_loss_sparse(t["Q"], t["K"], t["q_idx"], t["k_idx"], t["w"],
                                        torch.from_numpy(idx.astype(np.int32)).cuda(), t["cu_q"], t["cu_k"],
                                        t["max_q"], t["max_k"])
    assert abs(dense[0].item() - sparse[0].item()) <= 1e-5 * abs(dense[0].item())
    for a, b in zip(dense[1:], sparse[1:]):
        a, b = a.float().cpu().numpy(), b.float().cpu().numpy()
        assert np.max(np.abs(a - b)) <= 1e-2 * max(np.max(np.abs(a)), 1e-30)
