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


def silu_pairs_near_rounding_boundaries(rel=2.0 ** -36):
    """(gate, up) bf16 bit pairs whose activation g u / (1 + e^-g) lies within
    about `rel` (relative) of a point halfway between two binary32 numbers.

    An fp64 screen over every finite bf16 gate value with |g| <= 60 and every
    up significand in [1, 2): the fp64 value is within a few units of 2^-50 of
    the real one, and its 29 low significand bits give its distance to the
    nearest binary32 halfway point.  These are the pairs where an evaluation
    must carry more than binary32 precision to round correctly.
    """
    bits = np.arange(0, 0x10000, dtype=np.uint32)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF].astype(np.uint16)
    g = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    keep = (np.abs(g) <= 60) & (g != 0)
    bits, g = bits[keep], g[keep]
    sig = 1.0 + np.arange(128) / 128.0                      # up significands
    a = (g / (1.0 + np.exp(-g)))[:, None] * sig[None, :]
    b = a.view(np.uint64)
    low = (b & np.uint64((1 << 29) - 1)).astype(np.int64)
    dist = np.abs(low - (1 << 28))
    normal = np.abs(a) >= 2.0 ** -126
    gi, ui = np.nonzero((dist < rel * 2.0 ** 52) & normal)
    ubits = (0x3F80 + np.arange(128)).astype(np.uint16)
    return bits[gi], ubits[ui]
