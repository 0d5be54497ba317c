"""Helpers shared by the GPU parity tests (no operator arithmetic here)."""
import numpy as np
import torch


def dev(t):
    return t.to("cuda").contiguous()


def maxabs(gpu_out, ref) -> float:
    g = gpu_out.detach().float().cpu().numpy().astype(np.float64)
    return float(np.abs(g - np.asarray(ref, dtype=np.float64)).max())


def poison_like(t):
    """Output buffers start as NaN so an element the kernel never writes fails the check."""
    return torch.full_like(t, float("nan"))
