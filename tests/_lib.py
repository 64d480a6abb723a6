"""Test helpers: build the CUDA library if needed and move NumPy data to the GPU."""
import importlib.util
import os

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_dispatch_combine.h")


def build_module():
    """The package's build script, loaded without importing the package itself."""
    path = os.path.join(ROOT, "combine_route_meta_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_moe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def ensure_built():
    return build_module().build()


def bf16_to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_from_dev(t) -> np.ndarray:
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()
