"""Helpers for the GPU parity tests: move seeded numpy problems to the device,
run the library through its binding, bring BF16 results back as bit patterns."""
import numpy as np
import torch


def to_device(prob, device="cuda"):
    return {
        "x": torch.from_numpy(prob["x"].view(np.int16)).to(device).view(torch.bfloat16),
        "wq": torch.from_numpy(prob["wq"].view(np.int32)).to(device),
        "scales": torch.from_numpy(prob["scales"].view(np.int16)).to(device).view(torch.bfloat16),
        "biases": torch.from_numpy(prob["biases"].view(np.int16)).to(device).view(torch.bfloat16),
    }


def bits(t):
    """bf16 tensor -> numpy uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_y(prob, rows=None):
    import oracle
    x = prob["x"] if rows is None else prob["x"][rows]
    return oracle.matmul(x, prob["wq"], prob["scales"], prob["biases"])
