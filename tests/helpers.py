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
# A kernel that computes in FP32 can land on the other side of a BF16 rounding midpoint when the exact
# value sits right at it; for |v| > 2.56 RMS one BF16 ulp already exceeds the max-abs bound. A one-ulp
# disagreement counts as a rounding tie (not an error) only when the exact FP64 value lies within the
# element's own error bound `band` of the midpoint between the two BF16 neighbours -- the bound of the
# kernel's FP32 arithmetic that the oracle derives per element (grouped_gemm_bound: exact 16-element
# block partials, FP32 accumulation over the K/16 blocks, FP32 epilogue). Ties must also stay rare.
TIE_MAX_FRAC = 1e-3


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


def kstage_sf_to_rowmajor(sf_kstage, rows, K, sel=None):
    """NVFP4_SF_KSTAGE bytes -> row-major [rows, K/16] (or only the rows in `sel`). The header's definition:
    one [rows x 16 bytes] slab per 256-element K step, row r's scale of block b at
    ((b // 16) * rows + r) * 16 + b % 16 -- i.e. the bytes form an array [ceil(K/256), rows, 16], whose last
    slab holds 8 scales and 8 zero bytes per row when K % 256 == 128 (checked here)."""
    ns = (K + 255) // 256
    slabs = np.ascontiguousarray(sf_kstage).reshape(ns, rows, 16)
    if sel is not None:
        slabs = slabs[:, np.asarray(sel), :]
    if K % 256:
        assert not slabs[-1, :, 8:].any(), "the padding of the last K-stage slab must be zero scales"
    return np.ascontiguousarray(slabs.transpose(1, 0, 2)).reshape(-1, ns * 16)[:, : K // 16]


def rowmajor_sf_to_kstage(sf_rowmajor, rows, K):
    """Row-major [rows, K/16] scales -> the NVFP4_SF_KSTAGE array [ceil(K/256), rows, 16] (zero-padded)."""
    ns = (K + 255) // 256
    padded = np.zeros((rows, ns * 16), dtype=np.uint8)
    padded[:, : K // 16] = np.asarray(sf_rowmajor).reshape(rows, K // 16)
    return np.ascontiguousarray(padded.reshape(rows, ns, 16).transpose(1, 0, 2))


def bf16_to_f64(bits):
    bits = np.ascontiguousarray(bits).view(np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def compare_bf16(gpu_bits, ref_bits, what="", exact=None, band=None):
    """Compare BF16 outputs (bit patterns) against the BF16-rounded oracle `ref_bits`. With `exact` (the
    oracle's unrounded FP64 value) and `band` (the per-element bound on the kernel's FP32 error, same shape),
    one-ulp disagreements whose exact value lies within `band` of the rounding midpoint are ties. Returns a
    stats dict (printed, with the band next to the largest tie distance)."""
    gb = np.ascontiguousarray(gpu_bits).view(np.uint16)
    rb = np.ascontiguousarray(ref_bits).view(np.uint16)
    g = bf16_to_f64(gb)
    r = bf16_to_f64(rb)
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), f"{what}: non-finite GPU output"
    diff = np.abs(g - r)
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    fro = float(np.linalg.norm(r))
    ties = np.zeros(diff.shape, dtype=bool)
    tie_dist = tie_ratio = 0.0
    band_max = band_med = 0.0
    if exact is not None:
        assert band is not None, "a tie needs the element's derived error bound"
        ex = np.asarray(exact, dtype=np.float64).reshape(g.shape)
        bd = np.broadcast_to(np.asarray(band, dtype=np.float64).reshape(-1) if np.ndim(band) else band,
                             (g.size,)).reshape(g.shape)
        assert np.all(np.isfinite(bd)) and np.all(bd >= 0), f"{what}: bad bound"
        same_sign = (gb >> 15) == (rb >> 15)
        adjacent = same_sign & (np.abs(gb.astype(np.int32) - rb.astype(np.int32)) == 1)
        dist = np.abs(ex - 0.5 * (g + r))
        ties = adjacent & (diff > 0) & (dist <= bd)
        flips = adjacent & (diff > 0)
        if np.any(flips):
            tie_dist = float(dist[flips].max() / rms)
            tie_ratio = float(np.max(dist[flips] / np.maximum(bd[flips], 1e-300)))
        band_max = float(bd.max() / rms) if rms > 0 and bd.size else 0.0
        band_med = float(np.median(bd) / rms) if rms > 0 and bd.size else 0.0
    eff = np.where(ties, 0.0, diff)
    stats = {
        "n": int(r.size),
        "rms": rms,
        "max_abs": float(eff.max()) if r.size else 0.0,
        "max_abs_raw": float(diff.max()) if r.size else 0.0,
        "rel_fro": float(np.linalg.norm(g - r) / fro) if fro > 0 else float(np.linalg.norm(g - r)),
        "exact_frac": float(np.mean(g == r)) if r.size else 1.0,
        "tie_flips": int(np.sum(ties)),
        "max_tie_dist_rms": tie_dist,
        "max_tie_dist_over_band": tie_ratio,
        "band_max_rms": band_max,
        "band_median_rms": band_med,
        "over_tol_raw": int(np.sum(diff > MAX_ABS_REL_RMS * rms)),
    }
    print(f"[parity] {what}: {stats}")
    assert stats["max_abs"] <= MAX_ABS_REL_RMS * rms + 1e-30, f"{what}: {stats}"
    assert stats["rel_fro"] <= REL_FRO, f"{what}: {stats}"
    assert stats["tie_flips"] <= TIE_MAX_FRAC * max(1, r.size) + 1, f"{what}: {stats}"
    return stats


def combine_band(y_bits, inv_perm, topk_w):
    """Per-output bound of the combine's FP64 accumulation: k terms, each an exact FP32 x BF16 product, summed
    in FP64 (gamma_k in double precision times the sum of |terms|); the final rounding to BF16 is the
    reference's own."""
    import oracle
    y_abs = np.ascontiguousarray(y_bits).view(np.uint16) & np.uint16(0x7FFF)
    k = np.asarray(topk_w).shape[1]
    s = oracle.combine(y_abs, inv_perm, np.abs(np.asarray(topk_w, dtype=np.float32)))
    nu = k * 2.0 ** -53
    return s * (nu / (1 - nu)) * 1.01


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


def unpack_weights(packed, rows, K):
    """Packed weight tiles (layout of nvfp4_pack_weights in the header) -> (codes [rows, K/2],
    row-major scales [rows, K/16]). When K % 256 == 128 the last tile's padding must be zero (checked)."""
    flat = np.ascontiguousarray(packed).reshape(-1)
    kt_n = (K + 255) // 256
    tiles = flat.reshape(rows // 128, kt_n, 18432)
    codes = tiles[:, :, :16384].reshape(rows // 128, kt_n, 128, 8, 16)      # [rb, kt, r, swizzled piece, byte]
    r = np.arange(128)[:, None]
    c = np.arange(8)[None, :]
    logical = codes[:, :, r, c ^ (r & 7), :]                                  # [rb, kt, r, c, byte]
    q = logical.transpose(0, 2, 1, 3, 4).reshape(rows, kt_n * 128)
    sc = tiles[:, :, 16384:].reshape(rows // 128, kt_n, 4, 512)               # [rb, kt, kc, atom]
    rr = np.arange(128)[:, None]
    j = np.arange(4)[None, :]
    off = (rr % 32) * 16 + (rr // 32) * 4 + j                                  # [r, j]
    s = sc[:, :, :, off]                                                       # [rb, kt, kc, r, j]
    sf = s.transpose(0, 3, 1, 2, 4).reshape(rows, kt_n * 16)
    if K % 256:
        assert not q[:, K // 2:].any() and not sf[:, K // 16:].any(), "the last packed tile's padding must be zero"
    return q[:, : K // 2], sf[:, : K // 16]
