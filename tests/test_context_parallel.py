"""Context-parallel prefill of one sequence over ranks: the partition, the key all-gather
and the per-block bottom-right alignment.

CPU tests run two or three gloo ranks whose per-block computation is the fp64 oracle: the
concatenated result of the ranks must equal the oracle's whole-sequence forward at the
same positions (an integer-valued indexer input makes every score exact, so the sets are
compared bit for bit).  The GPU test runs the library's prefill on each zig-zag block of
a sequence (what each rank computes after the gather) and compares it with the
whole-sequence prefill.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from lightning_indexer_b200 import context_parallel as cp  # noqa: E402
from workloads import generators as gen  # noqa: E402


def _small_workload(L=203):
    return gen.make_prefill([L], 4, 2, 32, 4, 32, 24, seed=7, layout="integer", name="cp_small")


@pytest.mark.parametrize("L", [7, 203, 1000, 131072])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_zigzag_partition(L, world):
    seen = np.zeros(L, dtype=np.int64)
    work = []
    for r in range(world):
        rows = cp.local_rows(L, world, r).numpy()
        seen[rows] += 1
        work.append(int((rows + 1).sum()))  # causal keys each row sees
        (a0, b0), (a1, b1) = cp.rank_blocks(L, world, r)
        assert a0 <= b0 <= a1 <= b1
    assert (seen == 1).all()
    if L >= 1000:
        # an early and a late block per rank balance the causal work
        assert max(work) / min(work) < 1.05


def _oracle_block(k, scale):
    from oracle import dsa_oracle as orc

    def fn(q_idx, w, Q, k_idx_full, K_full, V_full, a, b):
        n = b - a
        idx_out, O_out, lse_out = [], [], []
        for i in range(n):
            nvis = orc.visible_keys(i, n, b)
            s = orc.indexer_scores_row(q_idx[i].numpy(), w[i].numpy(), k_idx_full[:nvis].numpy())
            idx = orc.topk_row(s, k)
            sel = idx[idx >= 0]
            O, lse = orc.sparse_attention_row(Q[i].numpy(), K_full[sel].numpy(), V_full[sel].numpy(), scale)
            idx_out.append(idx)
            O_out.append(O)
            lse_out.append(lse)
        return (torch.from_numpy(np.stack(idx_out)), torch.from_numpy(np.stack(O_out)),
                torch.from_numpy(np.stack(lse_out)))
    return fn


def _rank_main(rank, world, port, L, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from oracle import dsa_oracle as orc
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    wl = _small_workload(L)
    rows = cp.local_rows(L, world, rank).numpy()
    loc = {n: torch.from_numpy(orc.bf16_to_f64(getattr(wl, n))[rows]) for n in ("q_idx", "k_idx", "w", "Q", "K", "V")}
    scale = 1.0 / np.sqrt(wl.d)
    idx, O, lse = cp.prefill_context_parallel(loc["q_idx"], loc["k_idx"], loc["w"], loc["Q"], loc["K"], loc["V"],
                                              L, wl.topk, block_fn=_oracle_block(wl.topk, scale))
    dist.barrier()
    q.put((rank, rows, idx.numpy(), O.numpy(), lse.numpy()))
    dist.destroy_process_group()


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("L,world", [(203, 2), (96, 2), (203, 3)])
def test_gloo_ranks_match_whole_sequence_oracle(L, world):
    import torch.multiprocessing as mp
    from oracle import dsa_oracle as orc
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, L, q)) for r in range(world)]
    for p in procs:
        p.start()
    outs = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    wl = _small_workload(L)
    ref = orc.forward(orc.Decoded(wl))
    covered = np.zeros(L, dtype=bool)
    for rank, rows, idx, O, lse in outs:
        covered[rows] = True
        assert np.array_equal(idx, ref["idx"][rows]), rank
        assert np.allclose(O, ref["O"][rows], rtol=0, atol=1e-12), rank
        assert np.allclose(lse, ref["lse"][rows], rtol=0, atol=1e-12), rank
    assert covered.all()


@pytest.mark.gpu
@pytest.mark.parametrize("world", [2, 4])
def test_gpu_blocks_match_whole_sequence(world):
    """Each rank's two blocks, run through the library's prefill with the whole key side
    (as after the gather), give the whole-sequence prefill's rows: the same selected sets,
    and outputs within the attention tolerance (a short block may take the dense-set
    tensor-core pass where the whole sequence takes the sparse one)."""
    import lightning_indexer_b200 as dsa
    from dsa_testutil import to_device
    L = 20480
    wl = gen.make_prefill([L], 32, 4, 128, 64, 128, 2048, seed=11, layout="video", name="cp_20k", max_frames=60)
    t = to_device(wl)
    whole = dsa.prefill(t["q_idx"], t["k_idx"], t["w"], t["Q"], t["K"], t["V"], t["cu_q"], t["cu_k"], L, L,
                        wl.topk, chunk_rows=4096)
    torch.cuda.synchronize()
    for r in range(world):
        rows = cp.local_rows(L, world, r).cuda()
        qi_r, w_r, Q_r = t["q_idx"][rows], t["w"][rows], t["Q"][rows]
        off = 0
        for a, b in cp.rank_blocks(L, world, r):
            sl = slice(off, off + b - a)
            idx, O, lse = cp.prefill_block(qi_r[sl], w_r[sl], Q_r[sl], t["k_idx"], t["K"], t["V"], a, b, wl.topk,
                                           chunk_rows=4096)
            torch.cuda.synchronize()
            assert torch.equal(idx, whole[0][a:b]), (r, a, b)
            assert (O.float() - whole[1][a:b].float()).abs().max().item() <= 2e-2, (r, a, b)
            assert (lse - whole[2][a:b]).abs().max().item() <= 4e-3, (r, a, b)
            off += b - a
