"""GPU parity of the forward hot path (indexer, top-k, sparse attention, prefill and
decode pipelines) against the fp64 oracle, through the C ABI."""
import math

import numpy as np
import pytest
import torch

import lightning_indexer_b200 as dsa
from oracle import dsa_oracle as orc
from workloads import generators as gen

from dsa_testutil import bf16_dev, set_mismatch_ok, to_device

pytestmark = pytest.mark.gpu

ATTN_ATOL = 1e-2  # max-abs on O: bf16 I/O, fp32 accumulation, unit-variance inputs
LSE_ATOL = 2e-3   # fp32 softmax statistics vs fp64


def _oracle_scores(D, r):
    b, i, Lq, Lk = D.seq_of_row(r)
    k0 = int(D.cu_k[b])
    n = orc.visible_keys(i, Lq, Lk)
    return orc.indexer_scores_row(D.rows("q_idx", r), D.rows("w", r), D.rows("k_idx", slice(k0, k0 + n)))


# ------------------------------------------------------------------------- indexer

def test_indexer_integer_bit_exact():
    wl = gen.tiny_integer_1k()
    t = to_device(wl)
    s = dsa.index(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"]).cpu().numpy()
    D = orc.Decoded(wl)
    for r in range(wl.Tq):
        ref = _oracle_scores(D, r)
        assert np.array_equal(s[r, :ref.size].astype(np.float64), ref), r


@pytest.mark.parametrize("H_I,d_I", [(64, 128), (32, 128), (16, 128), (8, 64), (4, 32)])
def test_indexer_gaussian_varlen_chunks(H_I, d_I):
    # three sequences with ragged tails (not multiples of the 128-key tile or token block)
    wl = gen.make_prefill([300, 1, 777], 8, 2, 64, H_I, d_I, 64, seed=21)
    t = to_device(wl)
    D = orc.Decoded(wl)
    for (r0, r1) in [(0, wl.Tq), (5, 301), (301, wl.Tq)]:
        s = dsa.index(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"],
                      row_begin=r0, row_end=r1).cpu().numpy()
        for r in range(r0, r1):
            ref = _oracle_scores(D, r)
            got = s[r - r0, :ref.size].astype(np.float64)
            tol = 2e-5 * np.abs(ref).max() + 1e-6
            assert np.max(np.abs(got - ref)) <= tol, (r, np.max(np.abs(got - ref)), tol)
            # columns past the visible range are never written
            assert np.all(np.isneginf(s[r - r0, ref.size:min(ref.size + 200, s.shape[1])]))


def test_indexer_decode_shape():
    wl = gen.make_decode(3, 5000, 32, 4, 128, 64, 128, 256, seed=22, layout="video")
    t = to_device(wl)
    s = dsa.index(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], 1, t["max_k"]).cpu().numpy()
    D = orc.Decoded(wl)
    for r in range(3):
        ref = _oracle_scores(D, r)
        tol = 2e-5 * np.abs(ref).max() + 1e-6
        assert np.max(np.abs(s[r, :5000] - ref)) <= tol


# ------------------------------------------------------------------------- top-k

def _topk_case(rows_vis, k, seed, ties=False):
    rng = np.random.default_rng(seed)
    B = len(rows_vis)
    cu_q = np.arange(B + 1, dtype=np.int32)
    cu_k = np.concatenate([[0], np.cumsum(rows_vis)]).astype(np.int32)
    ld = (max(rows_vis) + 3) // 4 * 4
    sc = np.full((B, ld), np.nan, np.float32)
    for b, n in enumerate(rows_vis):
        if ties:
            v = rng.integers(-6, 7, size=n).astype(np.float32) * np.float32(0.5)
            v[rng.random(n) < 0.05] = -0.0
        else:
            v = rng.standard_normal(n).astype(np.float32)
        sc[b, :n] = v
    return sc, cu_q, cu_k


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("k", [1, 16, 128, 2048])
def test_topk_bit_exact(k, ties):
    vis = [1, 5, 127, 128, 129, 2047, 2048, 2049, 5000, 33333]
    sc, cu_q, cu_k = _topk_case(vis, k, seed=k + 7 * ties, ties=ties)
    idx = dsa.topk(torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                   k).cpu().numpy()
    for b, n in enumerate(vis):
        ref = orc.topk_row(sc[b, :n].astype(np.float64), k)
        assert np.array_equal(idx[b], ref), (b, n)


def test_topk_long_rows_decode_length():
    vis = [262144, 262143, 131072]
    sc, cu_q, cu_k = _topk_case(vis, 2048, seed=3, ties=True)
    idx = dsa.topk(torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                   2048).cpu().numpy()
    for b, n in enumerate(vis):
        assert np.array_equal(idx[b], orc.topk_row(sc[b, :n].astype(np.float64), 2048))


@pytest.mark.parametrize("n_rows,n", [(3, 262144), (600, 40000)])
def test_topk_candidate_overflow_paths(n_rows, n):
    # few distinct values: the threshold bin holds far more candidates than fit in shared
    # memory, so the kernel keeps reading the row from global memory; 3 rows use a
    # cluster of blocks per row, 600 rows one block per row
    rng = np.random.default_rng(n_rows)
    vis = [n - (r % 3) for r in range(n_rows)]
    cu_q = np.arange(n_rows + 1, dtype=np.int32)
    cu_k = np.concatenate([[0], np.cumsum(vis)]).astype(np.int32)
    ld = (n + 3) // 4 * 4
    sc = np.zeros((n_rows, ld), np.float32)
    for r in range(n_rows):
        sc[r, :vis[r]] = rng.integers(0, 3, size=vis[r]).astype(np.float32)
    idx = dsa.topk(torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                   2048).cpu().numpy()
    for r in range(0, n_rows, max(1, n_rows // 8)):
        assert np.array_equal(idx[r], orc.topk_row(sc[r, :vis[r]].astype(np.float64), 2048)), r


@pytest.mark.parametrize("case", ["decode_length", "adversarial"])
def test_topk_few_long_rows_without_workspace(case):
    # an empty workspace selects the single-launch path (one cluster per row, the row held
    # in registers); the result must equal the two-launch path's and the oracle's
    if case == "decode_length":
        vis = [262144, 262143, 131072, 200000]
        sc, cu_q, cu_k = _topk_case(vis, 2048, seed=13, ties=False)
    else:
        n = 131072
        rng = np.random.default_rng(12)
        sc = rng.standard_normal((3, n)).astype(np.float32)
        sc[0, ((2 * np.arange(1024) + 1) * n) // 2048] = 10.0   # the sample sees only huge values
        sc[1] = 1.0                                            # all ties
        sc[2, ::3] = 7.0
        vis = [n] * 3
        cu_q = np.arange(4, dtype=np.int32)
        cu_k = (np.arange(4) * n).astype(np.int32)
    args = (torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(), 2048)
    a = dsa.topk(*args, workspace=torch.empty(0, dtype=torch.uint8, device="cuda")).cpu().numpy()
    b = dsa.topk(*args).cpu().numpy()
    assert np.array_equal(a, b)
    for r, n in enumerate(vis):
        assert np.array_equal(a[r], orc.topk_row(sc[r, :n].astype(np.float64), 2048)), r


@pytest.mark.parametrize("ties", [False, True])
def test_topk_many_rows_stream_path(ties):
    # 400 rows of 3000..70000 positions, one block per row: ordered candidate lists built
    # tile by tile (Gaussian scores); with heavy ties most rows overflow the list and are
    # finished by the exact kernel
    vis = [3000 + (r * 167) % 67000 for r in range(400)]
    sc, cu_q, cu_k = _topk_case(vis, 2048, seed=21 + ties, ties=ties)
    idx = dsa.topk(torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                   2048).cpu().numpy()
    for b in range(0, 400, 23):
        assert np.array_equal(idx[b], orc.topk_row(sc[b, :vis[b]].astype(np.float64), 2048)), b


def test_topk_many_long_rows_cluster_path():
    # 120 rows of ~100K positions: too many rows for one cluster per row with the row in
    # registers, so the sampled-threshold kernel runs with a small cluster per row
    vis = [100000 - 37 * r for r in range(120)]
    sc, cu_q, cu_k = _topk_case(vis, 2048, seed=5, ties=True)
    idx = dsa.topk(torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                   2048).cpu().numpy()
    for b in range(0, 120, 13):
        assert np.array_equal(idx[b], orc.topk_row(sc[b, :vis[b]].astype(np.float64), 2048)), b


def test_topk_adversarial_rows():
    # rows built so that a strided sample of the row misjudges the threshold: the largest
    # values sit exactly on evenly spaced positions, or everywhere except there; the
    # selected set must still be exact
    n, k = 131072, 2048
    rng = np.random.default_rng(11)
    sc = np.zeros((4, n), np.float32)
    spots = ((2 * np.arange(1024) + 1) * n) // 2048
    sc[0] = rng.standard_normal(n).astype(np.float32)
    sc[0, spots] = 10.0                       # 1024 huge values on the sampled positions
    sc[1] = rng.standard_normal(n).astype(np.float32) - 5.0
    sc[1, spots] = 10.0
    sc[1, np.arange(7, n, 64)] = 3.0          # the rest of the top-k between the samples
    sc[2] = 1.0
    sc[2, spots] = -1.0                       # everything ties except the sampled ones
    sc[3] = -np.arange(n, dtype=np.float32)   # strictly decreasing
    cu_q = np.arange(5, dtype=np.int32)
    cu_k = (np.arange(5) * n).astype(np.int32)
    idx = dsa.topk(torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(),
                   k).cpu().numpy()
    for r in range(4):
        assert np.array_equal(idx[r], orc.topk_row(sc[r].astype(np.float64), k)), r


def test_topk_deterministic_repeat():
    sc, cu_q, cu_k = _topk_case([70000] * 4, 2048, seed=9, ties=True)
    args = (torch.from_numpy(sc).cuda(), torch.from_numpy(cu_q).cuda(), torch.from_numpy(cu_k).cuda(), 2048)
    a = dsa.topk(*args)
    b = dsa.topk(*args)
    assert torch.equal(a, b)


# ------------------------------------------------------------------------- sparse attention

def _oracle_sets(D, k):
    wl = D.wl
    return np.stack([orc.forward_row(D, r, k)["idx"] for r in range(wl.Tq)])


# "tensor_core": the tcgen05 entry point (d = 128, 8 query heads per KV head)
@pytest.mark.parametrize("Hq,Hkv,d,kernel", [(32, 4, 128, "gather"), (32, 4, 128, "tensor_core"), (8, 2, 64, "gather"),
                                             (16, 4, 64, "gather"), (16, 4, 128, "gather")])
def test_sparse_attention_prefill_given_sets(Hq, Hkv, d, kernel):
    wl = gen.make_prefill([200, 57, 400], Hq, Hkv, d, 4, 32, 64, seed=31)
    D = orc.Decoded(wl)
    idx = _oracle_sets(D, 64)
    t = to_device(wl)
    O, lse = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], torch.from_numpy(idx.astype(np.int32)).cuda(),
                                     t["cu_q"], t["cu_k"], kernel=kernel)
    O = O.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for r in range(wl.Tq):
        b, i, Lq, Lk = D.seq_of_row(r)
        sel = idx[r][idx[r] >= 0] + int(D.cu_k[b])
        Or, lr = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        assert np.max(np.abs(O[r] - Or)) <= ATTN_ATOL, r
        assert np.max(np.abs(lse[r] - lr)) <= LSE_ATOL, r


def _reuse_sets(cu, k, seed):
    """Selected sets with a known union structure, for the adjacent-query reuse path: in
    every other 16-row block the rows draw from one pool of 1.5 k positions that all of the
    block's rows can see (small union: the tensor-core form), in the others each row draws
    from its whole visible range (a union that outgrows 12288 positions late in a long
    sequence: the gather kernel).  A few -1 slots end each row, and a row that has room also
    lists the position just past its causal limit, which every path must ignore."""
    rng = np.random.default_rng(seed)
    idx = np.full((int(cu[-1]), k), -1, np.int32)
    for b in range(len(cu) - 1):
        L = int(cu[b + 1] - cu[b])
        for i0 in range(0, L, 16):
            pool = rng.choice(i0 + 1, size=min(i0 + 1, 3 * k // 2), replace=False) if (i0 // 16) % 2 == 0 else None
            for i in range(i0, min(L, i0 + 16)):
                src = pool if pool is not None else np.arange(i + 1)
                n = min(len(src), k - int(rng.integers(1, 8)))
                row = idx[cu[b] + i]
                row[:n] = np.sort(rng.choice(src, size=n, replace=False))
                if i + 1 < L:
                    row[n] = i + 1
    return idx


def test_sparse_attention_reuse_given_sets():
    wl = gen.make_prefill([14000, 1000], 32, 4, 128, 4, 32, 2048, seed=33)
    cu = wl.cu_seqlens_q.astype(np.int64)
    idx = _reuse_sets(cu, 2048, seed=33)
    t = to_device(wl)
    idx_d = torch.from_numpy(idx).cuda()
    nb = (wl.Tq + 15) // 16 + wl.B
    bu = torch.full((nb,), -7, dtype=torch.int32, device="cuda")
    O, lse = dsa.sparse_attn_prefill_reuse(t["Q"], t["K"], t["V"], idx_d, t["cu_q"], t["cu_k"], t["max_k"],
                                           block_union=bu)
    Og, lg = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], idx_d, t["cu_q"], t["cu_k"])
    # per-block union sizes, exactly (entries past the last block are 0)
    want = []
    for b in range(wl.B):
        L = int(cu[b + 1] - cu[b])
        for i0 in range(0, L, 16):
            rows = idx[cu[b] + i0:cu[b] + min(L, i0 + 16)]
            vis = np.arange(i0, min(L, i0 + 16))[:, None] + 1
            want.append(np.unique(rows[(rows >= 0) & (rows < vis)]).size)
    got = bu.cpu().numpy()
    assert np.array_equal(got[:len(want)], np.array(want)) and (got[len(want):] == 0).all()
    assert (np.array(want) <= 12288).sum() > 100 and (np.array(want) > 12288).sum() > 10  # both paths ran
    O, lse, Og, lg = O.float().cpu().numpy(), lse.cpu().numpy(), Og.float().cpu().numpy(), lg.cpu().numpy()
    assert np.max(np.abs(O - Og)) <= 2 * ATTN_ATOL and np.max(np.abs(lse - lg)) <= 2 * LSE_ATOL
    D = orc.Decoded(wl)
    for r in orc.sample_rows(wl.Tq, seed=33, n_first=40, n_last=40, n_mid=120) + [14000 + 37, 14999]:
        b, i, Lq, Lk = D.seq_of_row(r)
        row = idx[r]
        sel = row[(row >= 0) & (row <= i)] + int(D.cu_k[b])
        Or, lr = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        assert np.max(np.abs(O[r] - Or)) <= ATTN_ATOL, r
        assert np.max(np.abs(lse[r] - lr)) <= LSE_ATOL, r


def _fused_vs_separate(wl, k, chunk):
    """Selected sets by dsa_index_topk on its fused path and on the separate passes."""
    t = to_device(wl)
    args = (t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"], k)
    fused = dsa.index_topk(*args, chunk_rows=chunk, path=dsa.PATH_FUSED).cpu().numpy()
    separate = dsa.index_topk(*args, chunk_rows=chunk, path=dsa.PATH_SEPARATE).cpu().numpy()
    return fused, separate


def test_index_topk_fused_integer_bit_exact():
    # integer indexer inputs (exact fp32 scores, many ties) at H_I = 64, d_I = 128: the fused
    # path must return exactly the oracle's sets and exactly the separate path's, in one
    # chunk and in chunks of 700 rows
    wl = gen.make_prefill([1500, 700, 1200], 8, 2, 64, 64, 128, 128, seed=36, layout="integer")
    D = orc.Decoded(wl)
    ref = _oracle_sets(D, 128)
    for chunk in (wl.Tq, 700):
        fused, separate = _fused_vs_separate(wl, 128, chunk)
        np.testing.assert_array_equal(fused, separate)
        np.testing.assert_array_equal(fused, ref)


def test_index_topk_fused_gaussian_matches_separate_and_oracle():
    wl = gen.make_prefill([3000, 1000], 8, 2, 64, 64, 128, 64, seed=37, layout="video")
    fused, separate = _fused_vs_separate(wl, 64, 1024)
    np.testing.assert_array_equal(fused, separate)
    # a row range (crossing the sequence boundary) gives the same rows
    t = to_device(wl)
    part = dsa.index_topk(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"], 64,
                          chunk_rows=700, row_begin=2500, row_end=3600, path=dsa.PATH_FUSED).cpu().numpy()
    np.testing.assert_array_equal(part, fused[2500:3600])
    D = orc.Decoded(wl)
    for r in range(0, wl.Tq, 3):
        o = orc.forward_row(D, r, 64)
        ok, _ = set_mismatch_ok(fused[r], o["idx"], o["scores"])
        assert ok, r


def test_index_topk_fused_repair_rows():
    # Rows the sampled bound fails for must still come out exact.  The keys at the sampled
    # positions (packed rows that are multiples of the stride, 4 here) get the largest
    # scores and every other key a small one, so a bound taken from the samples lets through
    # only the sampled positions: fewer than k = 256 for rows that see under 1024 keys (too
    # few candidates), and rows whose q_idx is zero score 0 everywhere (every position ties,
    # too many candidates).  Both kinds are recomputed and selected by the exact method.
    wl = gen.make_prefill([2000, 1500], 8, 2, 64, 64, 128, 256, seed=38, layout="integer")
    rng = np.random.default_rng(38)
    k_idx = rng.integers(-1, 2, size=(wl.Tk, 128)).astype(np.float32)
    k_idx[np.arange(wl.Tk) % 4 == 0] = 8.0
    q_idx = rng.integers(1, 9, size=(wl.Tq, 64, 128)).astype(np.float32)
    q_idx[1200:1300] = 0.0  # they see more positions (1201..1300) than a row's 992 candidate slots
    q_idx[2900:2950] = 0.0
    wl.k_idx = gen.f32_to_bf16_bits(k_idx)
    wl.q_idx = gen.f32_to_bf16_bits(q_idx)
    D = orc.Decoded(wl)
    ref = _oracle_sets(D, 256)
    for chunk in (wl.Tq, 1024):
        fused, separate = _fused_vs_separate(wl, 256, chunk)
        np.testing.assert_array_equal(fused, ref)
        np.testing.assert_array_equal(separate, ref)


def test_index_topk_fused_repeat_is_bit_identical():
    # candidate lists arrive in a timing-dependent order; the selected sets must not
    wl = gen.make_prefill([4000], 8, 2, 64, 64, 128, 128, seed=39, layout="video")
    t = to_device(wl)
    args = (t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"], 128)
    first = dsa.index_topk(*args, chunk_rows=1000, path=dsa.PATH_FUSED)
    for _ in range(3):
        assert torch.equal(dsa.index_topk(*args, chunk_rows=1000, path=dsa.PATH_FUSED), first)


@pytest.mark.parametrize("Hq,Hkv,d,k,kernel", [(8, 2, 64, 32, "gather"), (16, 2, 128, 48, "gather"),
                                               (16, 2, 128, 48, "tensor_core"), (16, 2, 128, 176, "tensor_core")])
def test_sparse_attention_empty_and_padded_sets(Hq, Hkv, d, k, kernel):
    # on the tensor-core kernel k = 48 is one partial tile of 128 slots, k = 176 a full tile
    # and a ragged one
    wl = gen.make_prefill([40], Hq, Hkv, d, 4, 32, 32, seed=32)
    D = orc.Decoded(wl)
    idx = np.full((40, k), -1, np.int32)
    idx[39, :5] = [0, 1, 7, 20, 39]
    idx[12, 3] = 11  # a single selected key in the middle of the padding
    idx[20, k - 1] = 4  # a key in the last slot of the last tile
    t = to_device(wl)
    O, lse = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], torch.from_numpy(idx).cuda(), t["cu_q"], t["cu_k"],
                                     kernel=kernel)
    O = O.float().cpu().numpy()
    lse = lse.cpu().numpy()
    assert np.all(O[0] == 0) and np.all(np.isneginf(lse[0]))
    for r in (39, 12, 20):
        sel = idx[r][idx[r] >= 0]
        Or, lr = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        assert np.max(np.abs(O[r] - Or)) <= ATTN_ATOL
        assert np.max(np.abs(lse[r] - lr)) <= LSE_ATOL


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 4, 128), (8, 2, 64)])
def test_sparse_attention_ignores_positions_the_row_cannot_see(Hq, Hkv, d):
    # Two packed sequences [300, 200], k = 64.  In every full set the last slot is replaced
    # by a position the row cannot see: one past its causal range (inside its sequence),
    # one in the next sequence of the pack (still inside the K/V tensors), or past the end
    # of the last sequence (past the end of the tensors).  Such entries must be ignored like
    # -1, in the forward and in the backward, with no memory read behind them.
    wl = gen.make_prefill([300, 200], Hq, Hkv, d, 4, 32, 64, seed=35, with_dO=True)
    D = orc.Decoded(wl)
    good = _oracle_sets(D, 64)
    bad = good.copy()
    kept = good.copy()
    for r in range(wl.Tq):
        b, i, Lq, Lk = D.seq_of_row(r)
        if i < 64:
            continue
        bad[r, -1] = (i + 1 + r % 7, Lk + r % 13, 10 * Lk)[r % 3]
        kept[r, -1] = -1
    t = to_device(wl)
    O, lse = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], torch.from_numpy(bad.astype(np.int32)).cuda(),
                                     t["cu_q"], t["cu_k"])
    Oh, lh = O.float().cpu().numpy(), lse.cpu().numpy()
    O_ref, lse_ref = [], []
    for r in range(wl.Tq):
        b, i, Lq, Lk = D.seq_of_row(r)
        sel = kept[r][kept[r] >= 0] + int(D.cu_k[b])
        Or, lr = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        assert np.max(np.abs(Oh[r] - Or)) <= ATTN_ATOL, r
        assert np.max(np.abs(lh[r] - lr)) <= LSE_ATOL, r
        O_ref.append(Or)
        lse_ref.append(lr)
    if d == 128 and Hq == 8 * Hkv:  # the tensor-core entry point applies the same rule
        O2, l2 = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], torch.from_numpy(bad.astype(np.int32)).cuda(),
                                         t["cu_q"], t["cu_k"], kernel="tensor_core")
        O2, l2 = O2.float().cpu().numpy(), l2.cpu().numpy()
        for r in range(wl.Tq):
            assert np.max(np.abs(O2[r] - O_ref[r])) <= ATTN_ATOL, r
            assert np.max(np.abs(l2[r] - lse_ref[r])) <= LSE_ATOL, r
    # the backward of the same sets (gather path at d = 64, masked dense path at d = 128)
    ref = orc.sparse_attention_backward(D, kept, np.stack(O_ref), np.stack(lse_ref), D.full("dO"))
    dQ, dK, dV = dsa.sparse_attn_prefill_bwd(t["Q"], t["K"], t["V"], O, t["dO"], lse,
                                             torch.from_numpy(bad.astype(np.int32)).cuda(), t["cu_q"], t["cu_k"],
                                             max_seqlen_k=t["max_k"])
    for got, name in ((dQ, "dQ"), (dK, "dK"), (dV, "dV")):
        g = got.float().cpu().numpy()
        assert np.max(np.abs(g - ref[name])) <= 1.5e-2 * np.max(np.abs(ref[name])), name


@pytest.mark.parametrize("kernel", ["gather", "tensor_core"])
def test_sparse_attention_large_rising_logits(kernel):
    """Logits of tens of units that grow along the key order: the running max moves in
    most chunks, by more than the rescale threshold, and the weights span many octaves."""
    wl = gen.make_prefill([300], 32, 4, 128, 4, 32, 128, seed=34)
    Qf = wl.Q.astype(np.uint32) << 16
    Kf = wl.K.astype(np.uint32) << 16
    # powers of two keep every value exact in bf16: Q x 8, K x 1/2/4/8 by position band
    q = (Qf.view(np.float32) * np.float32(8.0)).view(np.uint32)
    band = np.minimum(np.arange(300) // 75, 3).astype(np.float32)
    kk = (Kf.view(np.float32) * (np.float32(2.0) ** band)[:, None, None]).view(np.uint32)
    wl.Q = (q >> 16).astype(np.uint16)
    wl.K = (kk >> 16).astype(np.uint16)
    D = orc.Decoded(wl)
    idx = np.full((300, 128), -1, np.int32)
    for r in range(300):
        n = min(r + 1, 128)
        idx[r, :n] = np.linspace(0, r, n).astype(np.int64)  # step >= 1: distinct, ascending
    t = to_device(wl)
    O, lse = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], torch.from_numpy(idx).cuda(), t["cu_q"], t["cu_k"],
                                     kernel=kernel)
    O = O.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for r in range(0, 300, 7):
        sel = idx[r][idx[r] >= 0]
        Or, lr = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        assert np.max(np.abs(O[r] - Or)) <= ATTN_ATOL, r
        assert np.max(np.abs(lse[r] - lr)) <= 1e-4 * max(1.0, float(np.max(np.abs(lr)))) + LSE_ATOL, r


def test_sparse_attention_decode_given_sets():
    wl = gen.make_decode(5, 3000, 32, 4, 128, 64, 128, 2048, seed=33, layout="video")
    D = orc.Decoded(wl)
    idx = _oracle_sets(D, 2048)
    t = to_device(wl)
    O, lse = dsa.sparse_attn_decode(t["Q"], t["K"], t["V"], torch.from_numpy(idx.astype(np.int32)).cuda(),
                                    t["cu_k"])
    O = O.float().cpu().numpy()
    lse = lse.cpu().numpy()
    for r in range(5):
        sel = idx[r][idx[r] >= 0] + int(D.cu_k[r])
        Or, lr = orc.sparse_attention_row(D.rows("Q", r), D.rows("K", sel), D.rows("V", sel), D.scale)
        assert np.max(np.abs(O[r] - Or)) <= ATTN_ATOL
        assert np.max(np.abs(lse[r] - lr)) <= LSE_ATOL


# ------------------------------------------------------------------------- pipelines

def test_prefill_pipeline_integer_bit_exact_sets():
    wl = gen.tiny_integer_1k()
    t = to_device(wl)
    idx, O, lse = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                              t["max_q"], t["max_k"], wl.topk, chunk_rows=300)
    idx = idx.cpu().numpy()
    O = O.float().cpu().numpy()
    D = orc.Decoded(wl)
    ref = orc.forward(D)
    assert np.array_equal(idx, ref["idx"])
    assert np.max(np.abs(O - ref["O"])) <= ATTN_ATOL
    assert np.max(np.abs(lse.cpu().numpy() - ref["lse"])) <= LSE_ATOL


def test_prefill_pipeline_gaussian_varlen():
    # d = 128, 8 heads per KV head and 8 k >= the longest sequence: the pipeline takes the
    # masked dense attention passes; the gather kernel on the same sets must agree on every row
    wl = gen.make_prefill([1500, 700, 2300], 32, 4, 128, 64, 128, 512, seed=41, layout="video")
    t = to_device(wl)
    idx_t, O_t, lse_t = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                                    t["max_q"], t["max_k"], wl.topk, chunk_rows=1024)
    O_g, lse_g = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], idx_t, t["cu_q"], t["cu_k"])
    # two bf16-rounded results, each within ATTN_ATOL of the exact value
    assert torch.max(torch.abs(O_t.float() - O_g.float())).item() <= 2 * ATTN_ATOL
    assert torch.max(torch.abs(lse_t - lse_g)).item() <= LSE_ATOL
    idx, O, lse = idx_t.cpu().numpy(), O_t.float().cpu().numpy(), lse_t.cpu().numpy()
    D = orc.Decoded(wl)
    rows = orc.sample_rows(wl.Tq, seed=5, n_first=32, n_last=32, n_mid=96) + [1499, 1500, 2199, 2200]
    swaps = 0
    for r in rows:
        ref = orc.forward_row(D, r)
        ok, nsw = set_mismatch_ok(idx[r], ref["idx"], ref["scores"])
        assert ok, r
        swaps += nsw
        if nsw == 0:
            assert np.array_equal(idx[r], ref["idx"])
            assert np.max(np.abs(O[r] - ref["O"])) <= ATTN_ATOL, r
            assert np.max(np.abs(lse[r] - ref["lse"])) <= LSE_ATOL, r


def _check_prefill_rows(wl, rows, chunk):
    """dsa.prefill against the oracle on the given rows (sets by the swap rule; O and lse
    where the sets are identical), and against the gather kernel on the same sets."""
    t = to_device(wl)
    idx, O, lse = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                              t["max_q"], t["max_k"], wl.topk, chunk_rows=chunk)
    Og, lg = dsa.sparse_attn_prefill(t["Q"], t["K"], t["V"], idx, t["cu_q"], t["cu_k"])
    idx_h, O_h, lse_h = idx.cpu().numpy(), O.float().cpu().numpy(), lse.cpu().numpy()
    # two kernels, each within the tolerance of the exact result, so within twice it of each
    # other (two bf16 roundings of one value of magnitude 2..4 can differ by 2^-6 > 1e-2)
    assert np.max(np.abs(O_h - Og.float().cpu().numpy())) <= 2 * ATTN_ATOL
    assert np.max(np.abs(lse_h - lg.cpu().numpy())) <= 2 * LSE_ATOL
    D = orc.Decoded(wl)
    exact = 0
    for r in rows:
        ref = orc.forward_row(D, r)
        ok, nsw = set_mismatch_ok(idx_h[r], ref["idx"], ref["scores"])
        assert ok, r
        if nsw == 0:
            exact += 1
            assert np.max(np.abs(O_h[r] - ref["O"])) <= ATTN_ATOL, r
            assert np.max(np.abs(lse_h[r] - ref["lse"])) <= LSE_ATOL, r
    assert exact >= 0.8 * len(rows)


def test_prefill_union_coherent_video():
    # frame-coherent indexer queries, k = 64 over 3000 and 1000 positions (sparse sets: 8 k
    # < L): every 16-row block's union of selections fits the union form, so attention runs
    # on the tensor-core passes over the gathered union of each block
    wl = gen.make_prefill([3000, 1000], 32, 4, 128, 64, 128, 64, seed=40, layout="video_coherent")
    _check_prefill_rows(wl, list(range(0, wl.Tq, 5)), 1024)


def test_prefill_union_mixed_blocks():
    # i.i.d. queries, k = 2048 over 20480 positions: blocks of rows that see at most 12288
    # positions take the union form, the later blocks' unions (about 16 x 2048 positions with
    # little overlap) exceed it and their rows run on the gather kernel
    wl = gen.make_prefill([20480], 8, 1, 128, 64, 128, 2048, seed=41, layout="gaussian")
    rows = orc.sample_rows(wl.Tq, seed=41, n_first=32, n_last=48, n_mid=64)
    _check_prefill_rows(wl, rows, 4096)


def test_prefill_union_high_overlap_video():
    # the high-overlap video layout at the 128K heads, 20480 positions, k = 2048: most blocks'
    # unions (the report's regime: a few thousand distinct positions per 16 queries) take the
    # union form
    wl = gen.make_prefill([20480], 32, 4, 128, 64, 128, 2048, seed=42, layout="video_overlap", max_frames=80)
    rows = orc.sample_rows(wl.Tq, seed=42, n_first=16, n_last=32, n_mid=48)
    _check_prefill_rows(wl, rows, 4096)


def test_prefill_from_host_matches_device_prefill():
    # host inputs, chunks of 100 rows crossing the sequence boundaries: the same kernels on
    # the same rows, so the result is identical to the device-side pipeline's
    wl = gen.make_prefill([300, 57, 400], 16, 4, 64, 16, 128, 64, seed=41)
    t = to_device(wl)
    _, O_ref, _ = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"],
                              t["max_q"], t["max_k"], 64, chunk_rows=100)

    def host(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()

    cu_q = torch.from_numpy(wl.cu_seqlens_q.astype(np.int32))
    cu_k = torch.from_numpy(wl.cu_seqlens_k.astype(np.int32))
    bufs = {}
    for _ in range(2):  # the second call reuses the device buffers
        O = dsa.prefill_from_host(host(wl.q_idx), host(wl.k_idx), host(wl.w), host(wl.Q), host(wl.K), host(wl.V),
                                  cu_q, cu_k, t["max_q"], t["max_k"], 64, chunk_rows=100, buffers=bufs)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(O.view(torch.int16), O_ref.cpu().view(torch.int16))


def test_prefill_from_host_tensor_core_shape():
    # the native host-input pipeline at the 128K heads (d = 128, 8 query heads per KV head),
    # two sequences, row chunks of 2048 crossing the sequence boundary: sets by the swap rule
    # and O against the oracle on sampled rows, and the same O as the device-side calls
    # (index + top-k, then the reuse attention) chunk by chunk
    wl = gen.make_prefill([3000, 1500], 32, 4, 128, 64, 128, 256, seed=44)
    t = to_device(wl)

    def host(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()

    cu_q = torch.from_numpy(wl.cu_seqlens_q.astype(np.int32))
    cu_k = torch.from_numpy(wl.cu_seqlens_k.astype(np.int32))
    O = dsa.prefill_from_host(host(wl.q_idx), host(wl.k_idx), host(wl.w), host(wl.Q), host(wl.K), host(wl.V), cu_q,
                              cu_k, t["max_q"], t["max_k"], wl.topk, chunk_rows=2048)
    torch.cuda.current_stream().synchronize()
    idx = torch.empty((wl.Tq, wl.topk), dtype=torch.int32, device="cuda")
    O_dev = torch.empty_like(t["Q"])
    for r0 in range(0, wl.Tq, 2048):
        r1 = min(wl.Tq, r0 + 2048)
        dsa.index_topk(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"], wl.topk,
                       chunk_rows=2048, indices=idx[r0:r1], row_begin=r0, row_end=r1)
        cq = torch.from_numpy(np.clip(wl.cu_seqlens_q.astype(np.int64) - r0, 0, r1 - r0).astype(np.int32)).cuda()
        dsa.sparse_attn_prefill_reuse(t["Q"][r0:r1], t["K"], t["V"], idx[r0:r1], cq, t["cu_k"], t["max_k"],
                                      out=(O_dev[r0:r1], None))
    torch.cuda.synchronize()
    assert torch.equal(O.view(torch.int16), O_dev.cpu().view(torch.int16))
    D = orc.Decoded(wl)
    Oh, idx_h = O.float().numpy(), idx.cpu().numpy()
    exact = 0
    rows = list(range(0, wl.Tq, 75))
    for r in rows:
        ref = orc.forward_row(D, r)
        ok, nsw = set_mismatch_ok(idx_h[r], ref["idx"], ref["scores"])
        assert ok, r
        if nsw == 0:
            exact += 1
            assert np.max(np.abs(Oh[r] - ref["O"])) <= ATTN_ATOL, r
    assert exact >= 0.8 * len(rows)


def test_decode_pipeline():
    wl = gen.make_decode(4, 20000, 32, 4, 128, 64, 128, 2048, seed=42, layout="video")
    t = to_device(wl)
    idx, O, lse = dsa.decode(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_k"], t["max_k"],
                             wl.topk)
    idx, O = idx.cpu().numpy(), O.float().cpu().numpy()
    D = orc.Decoded(wl)
    for r in range(4):
        ref = orc.forward_row(D, r)
        ok, nsw = set_mismatch_ok(idx[r], ref["idx"], ref["scores"])
        assert ok, r
        if nsw == 0:
            assert np.max(np.abs(O[r] - ref["O"])) <= ATTN_ATOL


def test_no_device_timeouts_recorded():
    assert dsa.device_status() == (0, 0)


def test_bounded_wait_runs_out_and_reports():
    # A wait with a 100 us limit on a barrier nothing arrives at (the same wait routine the
    # pipelined kernels use) gives up, records DSA_ERR_TIMEOUT with its site code, and the
    # kernel returns; the context stays usable and the status word is cleared on reading.
    from lightning_indexer_b200 import _lib
    assert dsa.device_status() == (0, 0)
    assert _lib.load().dsa_selftest_bounded_wait(100_000, torch.cuda.current_stream().cuda_stream) == 0
    assert dsa.device_status() == (-5, 900)
    assert dsa.device_status() == (0, 0)
    wl = gen.tiny_integer_1k()
    t = to_device(wl)
    sc = dsa.index(t["q_idx"], t["k_idx"], t["w"], t["cu_q"], t["cu_k"], t["max_q"], t["max_k"])
    D = orc.Decoded(wl)
    np.testing.assert_array_equal(sc[777, :778].cpu().numpy(), _oracle_scores(D, 777).astype(np.float32))
    assert dsa.device_status() == (0, 0)
