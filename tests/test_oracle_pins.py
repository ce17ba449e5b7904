"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test checks the oracle against a hand-worked example, a closed form, an identity
of the definition, a library routine that the definition reduces to in a special case,
a brute-force count, or central finite differences, chosen so that a dropped term,
a wrong sign or index, or a transposed operand in the oracle fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as orc
from workloads import generators as gen

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


def f64(a):
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------- indexer

def test_indexer_hand_worked():
    g = GOLD["indexer"]
    got = orc.indexer_scores_row(f64(g["q_idx"]), f64(g["w"]), f64(g["k_idx"]))
    np.testing.assert_array_equal(got, f64(g["expected"]))


def test_indexer_relu_odd_part_identity():
    # relu(x) - relu(-x) = x, so I(q) - I(-q) = k . (sum_j w_j q_j): a plain weighted sum
    rng = np.random.default_rng(1)
    q = rng.standard_normal((5, 7))
    w = rng.standard_normal(5)
    k = rng.standard_normal((11, 7))
    lhs = orc.indexer_scores_row(q, w, k) - orc.indexer_scores_row(-q, w, k)
    qbar = sum(w[j] * q[j] for j in range(5))
    rhs = np.array([sum(k[s, c] * qbar[c] for c in range(7)) for s in range(11)])
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)


def test_indexer_homogeneity_and_all_negative():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((4, 8))
    w = np.abs(rng.standard_normal(4))
    k = rng.standard_normal((9, 8))
    base = orc.indexer_scores_row(q, w, k)
    np.testing.assert_allclose(orc.indexer_scores_row(2.5 * q, w, k), 2.5 * base, rtol=1e-13)
    np.testing.assert_allclose(orc.indexer_scores_row(q, 3.0 * w, k), 3.0 * base, rtol=1e-13)
    # keys anti-aligned with every head give all-negative dot products -> score exactly 0
    qpos = np.abs(q)
    kneg = -np.abs(k)
    assert np.all(orc.indexer_scores_row(qpos, w, kneg) == 0.0)


def test_indexer_single_head_is_relu_dot():
    # H_I = 1, w = 1: the score is max(0, q . k) for each key, written out by hand
    q = f64([[1.0, -2.0, 0.5]])
    k = f64([[2.0, 1.0, 4.0], [0.0, 1.0, 0.0], [-1.0, -1.0, 2.0]])
    # dots: 2-2+2 = 2 ; -2 -> 0 ; -1+2+1 = 2
    np.testing.assert_array_equal(orc.indexer_scores_row(q, f64([1.0]), k), f64([2.0, 0.0, 2.0]))


def test_integer_config_scores_exact_in_fp32():
    # the tiny integer workload's scores are multiples of 1/8 below 2^13: exact in fp32
    wl = gen.tiny_integer_1k()
    D = orc.Decoded(wl)
    for r in (0, 17, 511, 1023):
        s = orc.forward_row(D, r)["scores"]
        assert np.all(s.astype(np.float32).astype(np.float64) == s)
        assert np.all(s * 8 == np.round(s * 8))


# ----------------------------------------------------------------------------- top-k

@pytest.mark.parametrize("case", GOLD["topk"])
def test_topk_hand_worked(case):
    got = orc.topk_row(f64(case["scores"]), case["k"])
    assert got.tolist() == case["expected"]


def _rank_by_count(scores):
    """Brute-force rank: how many positions beat s (larger score, or equal score and lower)."""
    n = len(scores)
    return [sum(1 for u in range(n) if scores[u] > scores[s] or (scores[u] == scores[s] and u < s))
            for s in range(n)]


@pytest.mark.parametrize("seed", range(6))
def test_topk_against_pairwise_rank_count(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 200))
    k = int(rng.integers(1, 64))
    scores = rng.integers(-4, 5, size=n).astype(np.float64)  # many ties
    if seed % 2:
        scores = rng.standard_normal(n)
    rank = _rank_by_count(scores.tolist())
    expected = sorted(s for s in range(n) if rank[s] < k)
    got = orc.topk_row(scores, k)
    assert got[:len(expected)].tolist() == expected
    assert np.all(got[len(expected):] == -1)


def test_topk_invariants_large():
    rng = np.random.default_rng(7)
    scores = np.round(rng.standard_normal(5000) * 4) / 4  # quarter steps: lots of ties
    k = 300
    sel = orc.topk_row(scores, k)
    assert np.all(np.diff(sel) > 0) and sel.shape == (k,)
    mask = np.zeros(5000, bool)
    mask[sel] = True
    kth = scores[mask].min()
    assert scores[~mask].max() <= kth
    # at the boundary value the chosen positions are the lowest ones
    tie = np.flatnonzero(scores == kth)
    chosen = tie[mask[tie]]
    assert np.all(chosen == tie[:chosen.size])


# ----------------------------------------------------------------------------- attention

def test_attention_hand_worked():
    g = GOLD["attention"]
    O, lse = orc.sparse_attention_row(f64(g["Q"]), f64(g["K_sel"]), f64(g["V_sel"]), g["scale"])
    np.testing.assert_allclose(O, f64(g["expected_O"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, f64(g["expected_lse"]), rtol=0, atol=1e-15)


def _torch_dense_causal(Q, K, V, scale):
    """Dense causal GQA attention by torch's SDPA routine in fp64 (one sequence)."""
    T, Hq, d = Q.shape
    G = Hq // K.shape[1]
    q = torch.from_numpy(Q).permute(1, 0, 2)
    k = torch.from_numpy(K).repeat_interleave(G, dim=1).permute(1, 0, 2)
    v = torch.from_numpy(V).repeat_interleave(G, dim=1).permute(1, 0, 2)
    return q, k, v


def test_sparse_equals_dense_sdpa_when_k_covers_all():
    # k >= L: every visible key is selected, so DSA is dense causal attention
    wl = gen.make_prefill([48], 8, 2, 16, 4, 8, 64, seed=11)
    D = orc.Decoded(wl)
    out = orc.forward(D)
    q, k, v = _torch_dense_causal(D.full("Q"), D.full("K"), D.full("V"), D.scale)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=D.scale)
    np.testing.assert_allclose(out["O"], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
    logits = (q @ k.transpose(1, 2)) * D.scale
    mask = torch.triu(torch.ones(48, 48, dtype=torch.bool), 1)
    lse_ref = torch.logsumexp(logits.masked_fill(mask, -math.inf), dim=-1).T.numpy()
    np.testing.assert_allclose(out["lse"], lse_ref, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    rng = np.random.default_rng(3)
    K = rng.standard_normal((9, 2, 8))
    V = rng.standard_normal((9, 2, 8))
    # zero query: uniform weights -> O = mean of V, lse = ln n
    O, lse = orc.sparse_attention_row(np.zeros((4, 8)), K, V, 0.3)
    np.testing.assert_allclose(O[0], V[:, 0].mean(0), rtol=1e-13)
    np.testing.assert_allclose(O[3], V[:, 1].mean(0), rtol=1e-13)
    np.testing.assert_allclose(lse, np.full(4, math.log(9)), rtol=1e-14)
    # a single selected key: O = V of that key, lse = its scaled logit
    q = rng.standard_normal((4, 8))
    O, lse = orc.sparse_attention_row(q, K[5:6], V[5:6], 0.3)
    np.testing.assert_allclose(O[1], V[5, 0], rtol=1e-14)
    np.testing.assert_allclose(O[2], V[5, 1], rtol=1e-14)
    np.testing.assert_allclose(lse[2], 0.3 * q[2] @ K[5, 1], rtol=1e-14)
    # V = 1 everywhere: softmax weights sum to one
    O, _ = orc.sparse_attention_row(q, K, np.ones_like(V), 0.3)
    np.testing.assert_allclose(O, 1.0, rtol=1e-14)
    # empty set
    O, lse = orc.sparse_attention_row(q, K[:0], V[:0], 0.3)
    assert np.all(O == 0) and np.all(np.isneginf(lse))


def test_causality_future_perturbation():
    wl = gen.make_prefill([64], 4, 2, 16, 4, 8, 8, seed=5)
    D1 = orc.Decoded(wl)
    r = 30
    a = orc.forward_row(D1, r)
    for name in ("k_idx", "K", "V"):
        arr = getattr(wl, name).copy()
        arr[r + 1:] = gen.f32_to_bf16_bits(np.full(arr[r + 1:].shape, 7.0, np.float32))
        setattr(wl, name, arr)
    b = orc.forward_row(orc.Decoded(wl), r)
    assert np.array_equal(a["idx"], b["idx"])
    np.testing.assert_array_equal(a["O"], b["O"])
    assert np.all(a["idx"][a["idx"] >= 0] <= r)


def test_decode_sees_whole_cache_and_matches_dense():
    wl = gen.make_decode(2, 40, 8, 2, 16, 4, 8, 64, seed=6, layout="gaussian")
    D = orc.Decoded(wl)
    for b in range(2):
        o = orc.forward_row(D, b)
        assert o["idx"][:40].tolist() == list(range(40))  # k >= N: everything
        K = D.rows("K", slice(40 * b, 40 * b + 40))
        V = D.rows("V", slice(40 * b, 40 * b + 40))
        O, lse = orc.dense_attention_row(D.rows("Q", b), K, V, D.scale)
        np.testing.assert_allclose(o["O"], O, rtol=1e-14)


# ----------------------------------------------------------------------------- KL loss

def test_kl_hand_worked():
    g = GOLD["kl"]
    kl, grad = orc.kl_row(f64(g["I"]), f64(g["p"]))
    assert abs(kl - g["expected_kl"]) < 1e-15
    np.testing.assert_allclose(grad, f64(g["expected_grad"]), atol=1e-15)


def test_kl_zero_when_indexer_equals_target():
    rng = np.random.default_rng(4)
    p = rng.random(50)
    p /= p.sum()
    kl, grad = orc.kl_row(np.log(p) + 3.7, p)  # any shift of log p is the same distribution
    assert abs(kl) < 1e-13
    np.testing.assert_allclose(grad, 0, atol=1e-15)


def test_kl_closed_form_uniform_target():
    # p uniform over n; I = [a, 0, ..., 0]: KL = ln(e^a + n - 1) - a/n - ln n
    n, a = 7, 1.3
    I = np.zeros(n)
    I[0] = a
    kl, _ = orc.kl_row(I, np.full(n, 1.0 / n))
    assert abs(kl - (math.log(math.exp(a) + n - 1) - a / n - math.log(n))) < 1e-14


def test_dense_target_closed_forms():
    rng = np.random.default_rng(8)
    K = rng.standard_normal((6, 2, 4))
    p = orc.dense_target_row(np.zeros((4, 4)), K, 0.5)  # zero query: uniform
    np.testing.assert_allclose(p, 1.0 / 6, rtol=1e-14)
    p = orc.dense_target_row(rng.standard_normal((4, 4)), K, 0.5)
    assert abs(p.sum() - 1.0) < 1e-14 and np.all(p > 0)


def test_dense_target_hand_worked_gqa():
    # two KV heads, two query heads each: catches a wrong query-head -> KV-head mapping
    # and a dropped softmax scale (the derivation lists what each mistake would give)
    g = GOLD["dense_target_gqa"]
    p = orc.dense_target_row(f64(g["Q"]), f64(g["K_vis"]), g["scale"])
    np.testing.assert_allclose(p, f64(g["expected_p"]), rtol=0, atol=1e-15)


def test_dense_target_is_head_mean_of_sdpa_with_identity_values():
    # With V = the identity over the visible keys, attention of head h returns its softmax
    # row itself, so the head mean of torch's SDPA outputs (fp64, GQA by repeat_interleave,
    # the same scale) is the target p.  A dropped scale or KV head h % Hkv fails here.
    rng = np.random.default_rng(12)
    for Hq, Hkv, d, n in ((8, 2, 16, 11), (32, 4, 8, 5), (4, 1, 32, 9)):
        G = Hq // Hkv
        Q = rng.standard_normal((Hq, d))
        K = rng.standard_normal((n, Hkv, d))
        scale = 1.0 / math.sqrt(d)
        p = orc.dense_target_row(Q, K, scale)
        q = torch.from_numpy(Q)[:, None, :]                                         # [Hq, 1, d]
        k = torch.from_numpy(K).repeat_interleave(G, dim=1).permute(1, 0, 2)       # [Hq, n, d]
        v = torch.eye(n, dtype=torch.float64).expand(Hq, n, n)                     # [Hq, n, n]
        out = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale)
        np.testing.assert_allclose(p, out[:, 0, :].mean(0).numpy(), rtol=1e-12, atol=1e-15)


def test_kl_gradients_by_finite_differences():
    wl = gen.make_prefill([9, 14], 4, 2, 8, 3, 4, 4, seed=9)
    D = orc.Decoded(wl)
    res = orc.indexer_kl_loss(D)
    assert res["loss"] > 0 and np.all(res["kl"] >= -1e-15)
    # perturb the decoded fp64 inputs directly (bypassing bf16 rounding)
    base = {n: D.full(n).copy() for n in ("q_idx", "k_idx", "w", "Q", "K")}

    def loss_with(name, index, delta):
        arrs = {n: v.copy() for n, v in base.items()}
        arrs[name][index] += delta
        D2 = orc.Decoded(wl)
        D2._full.update(arrs)
        return orc.indexer_kl_loss(D2)["loss"]

    rng = np.random.default_rng(0)
    h = 1e-6
    for name, grad in (("q_idx", res["dq_idx"]), ("k_idx", res["dk_idx"]), ("w", res["dw"])):
        for _ in range(6):
            index = tuple(int(rng.integers(0, s)) for s in base[name].shape)
            fd = (loss_with(name, index, h) - loss_with(name, index, -h)) / (2 * h)
            assert abs(fd - grad[index]) < 1e-7 + 1e-5 * abs(fd), (name, index, fd, grad[index])


def test_sparse_kl_with_every_position_selected_is_the_dense_kl():
    # sets that hold every visible position reduce the sparse-adaptation loss to the dense
    # warm-up loss (itself pinned above)
    wl = gen.make_prefill([9, 14], 4, 2, 8, 3, 4, 16, seed=10)
    D = orc.Decoded(wl)
    idx = np.stack([orc.forward_row(D, r, 16)["idx"] for r in range(wl.Tq)])
    sp = orc.indexer_kl_loss_sparse(D, idx)
    de = orc.indexer_kl_loss(D)
    assert abs(sp["loss"] - de["loss"]) < 1e-14
    for n in ("kl", "dq_idx", "dk_idx", "dw"):
        np.testing.assert_allclose(sp[n], de[n], rtol=1e-12, atol=1e-15)


def test_sparse_kl_gradients_by_finite_differences_and_unselected_keys():
    wl = gen.make_prefill([12, 10], 4, 2, 8, 3, 4, 5, seed=13)
    D = orc.Decoded(wl)
    rng = np.random.default_rng(13)
    idx = np.full((wl.Tq, 5), -1, np.int64)
    for r in range(wl.Tq):
        b, i, Lq, Lk = D.seq_of_row(r)
        n = min(i + 1, 5 if r % 4 else 2)
        idx[r, :n] = np.sort(rng.choice(i + 1, size=n, replace=False))
    res = orc.indexer_kl_loss_sparse(D, idx)
    assert res["loss"] > 0 and np.all(res["kl"] >= -1e-15)
    # a key no row selected gets no gradient
    chosen = set()
    for r in range(wl.Tq):
        b = D.seq_of_row(r)[0]
        chosen |= set(int(s) + int(D.cu_k[b]) for s in idx[r] if s >= 0)
    for s in range(wl.Tk):
        if s not in chosen:
            assert np.all(res["dk_idx"][s] == 0)
    # the order of a row's entries does not matter (a set)
    perm = idx.copy()
    for r in range(wl.Tq):
        perm[r] = perm[r][rng.permutation(5)]
    res_p = orc.indexer_kl_loss_sparse(D, perm)
    np.testing.assert_allclose(res_p["dk_idx"], res["dk_idx"], rtol=1e-12, atol=1e-16)
    assert abs(res_p["loss"] - res["loss"]) < 1e-14
    base = {n: D.full(n).copy() for n in ("q_idx", "k_idx", "w", "Q", "K")}

    def loss_with(name, index, delta):
        arrs = {n: v.copy() for n, v in base.items()}
        arrs[name][index] += delta
        D2 = orc.Decoded(wl)
        D2._full.update(arrs)
        return orc.indexer_kl_loss_sparse(D2, idx)["loss"]

    h = 1e-6
    for name, grad in (("q_idx", res["dq_idx"]), ("k_idx", res["dk_idx"]), ("w", res["dw"])):
        for _ in range(6):
            index = tuple(int(rng.integers(0, n)) for n in base[name].shape)
            fd = (loss_with(name, index, h) - loss_with(name, index, -h)) / (2 * h)
            assert abs(fd - grad[index]) <= 1e-6 * max(1.0, abs(fd)), (name, index, fd, grad[index])


# ----------------------------------------------------------------------------- backward

def _oracle_bwd(wl, k):
    D = orc.Decoded(wl)
    out = orc.forward(D, k=k)
    return D, out, orc.sparse_attention_backward(D, out["idx"], out["O"], out["lse"], D.full("dO"))


def test_backward_equals_torch_autograd_dense():
    wl = gen.make_prefill([20], 8, 2, 16, 4, 8, 32, seed=12, with_dO=True)
    D, out, g = _oracle_bwd(wl, 32)  # k >= L: dense
    q, k, v = _torch_dense_causal(D.full("Q"), D.full("K"), D.full("V"), D.scale)
    q.requires_grad_(True)
    kk = torch.from_numpy(D.full("K")).requires_grad_(True)
    vv = torch.from_numpy(D.full("V")).requires_grad_(True)
    G = 4
    o = torch.nn.functional.scaled_dot_product_attention(
        q, kk.repeat_interleave(G, 1).permute(1, 0, 2), vv.repeat_interleave(G, 1).permute(1, 0, 2),
        is_causal=True, scale=D.scale)
    o.backward(torch.from_numpy(D.full("dO")).permute(1, 0, 2))
    np.testing.assert_allclose(g["dQ"], q.grad.permute(1, 0, 2).numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dK"], kk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(g["dV"], vv.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_sparse_finite_differences_and_sums():
    wl = gen.make_prefill([24, 10], 4, 2, 8, 4, 8, 5, seed=13, with_dO=True)
    D, out, g = _oracle_bwd(wl, 5)
    dO = D.full("dO")
    idx = out["idx"]

    def objective(name, index, delta):
        D2 = orc.Decoded(wl)
        arr = D.full(name).copy()
        arr[index] += delta
        D2._full[name] = arr
        for n in ("Q", "K", "V"):
            if n != name:
                D2._full[n] = D.full(n)
        tot = 0.0
        for r in range(wl.Tq):  # fixed sets: the forward with the same idx
            b, i, Lq, Lk = D2.seq_of_row(r)
            sel = idx[r][idx[r] >= 0] + int(D2.cu_k[b])
            O, _ = orc.sparse_attention_row(D2._full["Q"][r], D2._full["K"][sel], D2._full["V"][sel], D2.scale)
            tot += float(np.sum(O * dO[r]))
        return tot

    rng = np.random.default_rng(1)
    h = 1e-6
    for name, grad in (("Q", g["dQ"]), ("K", g["dK"]), ("V", g["dV"])):
        for _ in range(5):
            index = tuple(int(rng.integers(0, s)) for s in D.full(name).shape)
            fd = (objective(name, index, h) - objective(name, index, -h)) / (2 * h)
            assert abs(fd - grad[index]) < 1e-7 + 1e-6 * abs(fd), (name, index)
    # identities that hold at any size: sum_s dK = 0 per KV head; sum_s dV = sum of dO over the group
    np.testing.assert_allclose(g["dK"].sum(0), 0, atol=1e-12)
    grp = dO.reshape(wl.Tq, wl.Hkv, wl.Hq // wl.Hkv, wl.d).sum(axis=(0, 2))
    np.testing.assert_allclose(g["dV"].sum(0), grp, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- workloads

def test_video_layout_counts():
    fid = gen.video_frame_ids(131072, max_frames=480)
    assert len(np.unique(fid[fid >= 0])) == 480
    assert (fid >= 0).sum() == 480 * 256
    assert np.all(fid[126720:] == -1) and 131072 - 126720 == 4352
    fid = gen.video_frame_ids(262144)
    assert fid.max() == 992 and (fid == 992).sum() == 248


def test_pixel_budget_lengths():
    lens = gen.pixel_budget_lengths(65536, seed=4)
    assert sum(lens) == 65536
    assert all(L in (2048, 4096, 8192, 16384) for L in lens[:-1])
    assert lens[-1] % 2048 == 0 and lens[-1] > 0


def test_generator_bf16_rounding_and_determinism():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-3], np.float32)
    # 1 + 2^-8 is halfway between bf16 1.0 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-8 -> up to 1 + 2^-6
    bits = gen.f32_to_bf16_bits(x)
    assert bits[0] == 0x3F80 and bits[1] == 0x3F80 and bits[2] == 0x3F82
    a = gen.make_prefill([100], 4, 2, 16, 4, 8, 8, seed=3, layout="video")
    b = gen.make_prefill([100], 4, 2, 16, 4, 8, 8, seed=3, layout="video")
    assert np.array_equal(a.K, b.K) and np.array_equal(a.k_idx, b.k_idx)
