"""Turn generator outputs (torch tensors) into the raw numpy storage the oracle reads."""

import numpy as np
import torch


def raw(t: torch.Tensor) -> np.ndarray:
    """Raw storage of a CPU/GPU tensor as numpy: bf16 -> uint16 bits, fp8 -> uint8."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype in (torch.float8_e4m3fn,):
        return t.view(torch.uint8).numpy()
    return t.numpy()


def linear_np(case: dict) -> dict:
    spec = case["spec"]
    d = dict(fmt=spec.fmt, K=spec.K, group=spec.group, b=spec.b, splits=tuple(spec.splits),
             codes=raw(case["codes"]), scales=raw(case["scales"]), X=raw(case["X"]), Q=raw(case["Q"]))
    if "dY" in case:
        d["dY"] = raw(case["dY"])
    return d
