"""Helpers shared by the GPU parity tests (marshalling only)."""
import numpy as np
import torch


def to_dev(x: np.ndarray) -> torch.Tensor:
    """numpy bf16 bits (uint16) or float32 -> CUDA tensor of the same bytes."""
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    torch.cuda.synchronize()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def mismatch_report(got: np.ndarray, ref: np.ndarray, name: str) -> str:
    bad = np.argwhere(got != ref)
    return f"{name}: {len(bad)} mismatches of {ref.size}; first at {bad[:5].tolist()}: got {got[tuple(bad[0])] if len(bad) else None} want {ref[tuple(bad[0])] if len(bad) else None}"
