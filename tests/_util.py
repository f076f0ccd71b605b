"""Small helpers shared by the tests (no method arithmetic here)."""
import numpy as np
import torch


def to_np(t: torch.Tensor) -> np.ndarray:
    """Torch tensor -> numpy in storage form: bf16 becomes its uint16 bit pattern."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def inputs_np(d: dict) -> dict:
    return {k: to_np(v) for k, v in d.items()}


def bits_to_bf16_tensor(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def bf16_bits_to_f64_torch(a: np.ndarray) -> np.ndarray:
    """BF16 bits -> float64 through torch's own conversion (independent of the oracle's)."""
    return bits_to_bf16_tensor(np.asarray(a, dtype=np.uint16)).to(torch.float64).numpy()
