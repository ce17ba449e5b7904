"""Helpers shared by the GPU tests: moving seeded workloads onto the device (marshalling
only) and the set-comparison rule for top-k on floating-point scores."""
import numpy as np
import torch


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> a contiguous torch.bfloat16 CUDA tensor (no rounding)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def to_device(wl):
    d = {
        "q_idx": bf16_dev(wl.q_idx), "k_idx": bf16_dev(wl.k_idx), "w": bf16_dev(wl.w),
        "Q": bf16_dev(wl.Q), "K": bf16_dev(wl.K), "V": bf16_dev(wl.V),
        "cu_q": torch.from_numpy(wl.cu_seqlens_q.astype(np.int32)).cuda(),
        "cu_k": torch.from_numpy(wl.cu_seqlens_k.astype(np.int32)).cuda(),
        "max_q": int(wl.seqlens_q.max()), "max_k": int(wl.seqlens_k.max()),
    }
    if wl.dO is not None:
        d["dO"] = bf16_dev(wl.dO)
    return d


def set_mismatch_ok(gpu_idx: np.ndarray, ref_idx: np.ndarray, ref_scores: np.ndarray, rel: float = 1e-3):
    """Top-k parity rule for floating-point scores.

    The sets must have the same size, and every position in one set but not the other
    must have an oracle score within ``rel`` (relative) of the oracle's k-th score.
    Returns (ok, number of swapped positions).
    """
    g = set(int(x) for x in gpu_idx if x >= 0)
    r = set(int(x) for x in ref_idx if x >= 0)
    if len(g) != len(r):
        return False, -1
    diff = g.symmetric_difference(r)
    if not diff:
        return True, 0
    kth = ref_scores[np.array(sorted(r))].min()
    tol = rel * max(abs(kth), 1e-30)
    ok = all(abs(ref_scores[s] - kth) <= tol for s in diff if 0 <= s < len(ref_scores))
    ok = ok and all(0 <= s < len(ref_scores) for s in diff)
    return ok, len(diff) // 2
