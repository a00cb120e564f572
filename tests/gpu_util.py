"""Helpers shared by the GPU parity tests (comparison logic only)."""
import numpy as np
import torch

import oracle


def np_u16(t: torch.Tensor) -> np.ndarray:
    """bf16 torch tensor -> uint16 bit patterns (host)."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def to_bf16_dev(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / (den if den > 0 else 1.0))


def check_selection(sel_gpu: np.ndarray, score_oracle: np.ndarray, S_oracle: np.ndarray, k: int, rel: float = 1e-6):
    """Selected channel sets agree bit-exactly except for channels whose score
    is within `rel` (relative) of the k-th largest score."""
    sel_gpu = np.asarray(sel_gpu)[:k]
    assert len(set(sel_gpu.tolist())) == k
    assert np.all(np.diff(sel_gpu) > 0), "selection not ascending"
    if k == 0:
        return
    kth = np.sort(score_oracle)[::-1][k - 1]
    exempt = set(np.nonzero(np.abs(score_oracle - kth) <= rel * kth)[0].tolist())
    a = set(sel_gpu.tolist()) - exempt
    b = set(np.asarray(S_oracle).tolist()) - exempt
    assert a == b, f"selection differs outside the tie window: {sorted(a ^ b)[:10]}"


def unswizzle(scales_gpu: torch.Tensor, rows: int, K: int) -> np.ndarray:
    return oracle.unswizzle_scales(scales_gpu.cpu().numpy(), rows, K)
