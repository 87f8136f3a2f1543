import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")


@pytest.fixture(scope="session")
def rng():
    import numpy as np
    return np.random.default_rng(12345)


# ------------------------------------------------------------ shared helpers
def to_device(b, device="cuda"):
    """synth.Batch (numpy) -> dict of device tensors in the batch dtype."""
    import torch
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32}[b.dtype]
    return dict(q=torch.from_numpy(b.q).to(device).to(tdt), k=torch.from_numpy(b.k).to(device).to(tdt),
                v=torch.from_numpy(b.v).to(device).to(tdt), alpha=torch.from_numpy(b.alpha).to(device),
                beta=torch.from_numpy(b.beta).to(device),
                cu_seqlens=torch.from_numpy(b.cu_seqlens).to(device), cu_host=[int(x) for x in b.cu_seqlens])


def bits(t):
    """Raw bit patterns of a tensor / array, for bitwise comparison."""
    import numpy as np
    import torch
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        return t.numpy().view(np.uint32 if t.dtype == torch.float32 else np.uint8)
    return np.ascontiguousarray(t).view(np.uint32 if t.dtype == np.float32 else np.uint16)
