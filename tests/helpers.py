"""Shared helpers of the test suite (no method arithmetic here: comparisons,
layout un-tiling written from the header's layout definition, tolerances)."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nvfp4moe.h")

# BF16 output tolerances: max |gpu - ref| <= 1e-2 * RMS(ref), ||gpu - ref||_F / ||ref||_F <= 5e-3,
# where ref is the oracle's FP64 result rounded once to BF16 (the exact answer in the output format).
MAX_ABS_REL_RMS = 1e-2
REL_FRO = 5e-3


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"NVFP4_API\s+[\w\s\*]+?\b((?:nvfp4|moe)_\w+)\s*\(", text)))


def untile_sf(sf_tiled, rows, K):
    """NVFP4_SF_MMA_TILED bytes -> row-major [rows, K/16] (layout as documented in the header)."""
    flat = np.ascontiguousarray(sf_tiled).reshape(-1)
    r = np.arange(rows)[:, None]
    b = np.arange(K // 16)[None, :]
    off = ((r // 128) * (K // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + (b % 4)
    return flat[off]


def bf16_to_f64(bits):
    bits = np.ascontiguousarray(bits).view(np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def compare_bf16(gpu_bits, ref_bits, what=""):
    """Compare BF16 outputs (bit patterns) against the BF16-rounded oracle; returns a stats dict."""
    g = bf16_to_f64(gpu_bits)
    r = bf16_to_f64(ref_bits)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    diff = np.abs(g - r)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    fro = float(np.linalg.norm(r))
    stats = {
        "n": int(r.size),
        "rms": rms,
        "max_abs": float(diff.max()) if r.size else 0.0,
        "rel_fro": float(np.linalg.norm(g - r) / fro) if fro > 0 else float(np.linalg.norm(g - r)),
        "exact_frac": float(np.mean(g == r)) if r.size else 1.0,
        "over_tol": int(np.sum(diff > MAX_ABS_REL_RMS * rms)),
    }
    assert stats["max_abs"] <= MAX_ABS_REL_RMS * rms + 1e-30, f"{what}: {stats}"
    assert stats["rel_fro"] <= REL_FRO, f"{what}: {stats}"
    return stats


def gpu_bf16(bits):
    """numpy uint16 BF16 bit patterns -> CUDA bfloat16 tensor."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def host_bits(t):
    """CUDA bfloat16 tensor -> numpy uint16 bit patterns."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t):
    return t.detach().contiguous().cpu().numpy()


def require_gpu():
    import pytest
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device (run them with -m gpu on a B200)")
    from nvfp4_block_scaled_09_b200 import build as nvbuild
    nvbuild.build()
