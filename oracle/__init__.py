"""CPU oracle for the NVFP4 block-scaled MoE path (numpy front end over plain C).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package. The
CUDA library never links, imports or calls it, and the two share no code.

Every function here is a thin marshalling layer over ``nvfp4_oracle.c``; the
arithmetic, with its citations of the pages, lives in that file:

- ``quantize``: per-tensor amax -> FP32 global scale, per-16 E4M3 block scale,
  E2M1 codes ("Peering into the CUTLASS SharedStorage", Input Knowledge
  Required item 3: two FP4 values per byte, one FP8 scale per 16 elements).
- ``permute``: explicit counting of routed (token, slot) pairs per expert,
  stable in (t, j) ("Peering into the CUTLASS Kernel Cache", Knowledge
  Required: each expert multiplies the subset of tokens routed to it).
- ``grouped_gemm`` / ``grouped_gemm_at``: per-expert block-scaled dot products
  in FP64, global scales, optional SwiGLU on gate/up halves.
- ``route_topk``: the router -- top-k logits per token (lower index first
  among equal values) and the softmax of the chosen k (the pages describe no
  router; the reading is stated in the C source).
- ``combine``: top-k weighted sum of expert outputs in FP64 (the final MoE
  output write of "Peering into the CUTLASS Kernel", Input Knowledge Required
  item 5).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64, i32, f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float
        L.oracle_bf16_to_float.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_float.restype = f32
        L.oracle_bf16_from_double.argtypes = [ctypes.c_double]
        L.oracle_bf16_from_double.restype = ctypes.c_uint16
        L.oracle_bf16_from_double_array.argtypes = [P, i64, P]
        L.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e2m1_decode.restype = ctypes.c_double
        L.oracle_e2m1_encode.argtypes = [f32]
        L.oracle_e2m1_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [f32]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_amax.argtypes = [P, i64]
        L.oracle_amax.restype = f32
        L.oracle_quantize.argtypes = [P, i64, i64, P, P, P, P]
        L.oracle_quantize_amax.argtypes = [P, i64, i64, f32, P, P, P]
        L.oracle_dequantize.argtypes = [P, P, f32, i64, i64, P]
        L.oracle_permute.argtypes = [P, i32, i32, i32, P, P, P]
        L.oracle_permute.restype = ctypes.c_int
        L.oracle_gather_rows.argtypes = [P, i64, P, i64, P]
        L.oracle_grouped_gemm.argtypes = [P, P, f32, P, P, P, P, i32, i64, i64, i32, P]
        L.oracle_grouped_gemm_at.argtypes = [P, P, f32, P, P, P, P, i32, i64, i64, i32, P, P, i64, P]
        L.oracle_combine.argtypes = [P, P, P, i32, i32, i64, P]
        L.oracle_route_topk.argtypes = [P, i32, i32, i32, P, P]
        L.oracle_grouped_gemm_bound.argtypes = [P, P, f32, P, P, P, P, i32, i64, i64, i32, P]
        L.oracle_grouped_gemm_bound_at.argtypes = [P, P, f32, P, P, P, P, i32, i64, i64, i32, P, P, i64, P]
        L.oracle_num_threads.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return ctypes.c_void_p(a.ctypes.data)


def _u16(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != np.uint16:
        raise TypeError("BF16 tensors are passed as their uint16 bit patterns")
    return np.ascontiguousarray(a)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


# --- scalar codecs -----------------------------------------------------------

def e2m1_decode(code: int) -> float:
    return float(lib().oracle_e2m1_decode(int(code)))


def e2m1_encode(y: float) -> int:
    return int(lib().oracle_e2m1_encode(float(y)))


def e4m3_decode(b: int) -> float:
    return float(lib().oracle_e4m3_decode(int(b)))


def e4m3_encode(s: float) -> int:
    return int(lib().oracle_e4m3_encode(float(s)))


def bf16_to_float(b: int) -> float:
    return float(lib().oracle_bf16_to_float(int(b)))


def bf16_from_double(v: float) -> int:
    return int(lib().oracle_bf16_from_double(float(v)))


def bf16_round(v: np.ndarray) -> np.ndarray:
    """FP64 array -> BF16 bit patterns (uint16), round-to-nearest-even."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    lib().oracle_bf16_from_double_array(_p(v), v.size, _p(out))
    return out


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --- tensor operations -----------------------------------------------------

def amax(x_bf16: np.ndarray) -> float:
    x = _u16(x_bf16)
    return float(lib().oracle_amax(_p(x), x.size))


def quantize(x_bf16: np.ndarray, global_scale=None):
    """x [rows, K] BF16 bits -> (q [rows, K/2] u8, sf [rows, K/16] u8 row-major, g_dec f32)."""
    x = _u16(x_bf16)
    rows, K = x.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    q = np.empty((rows, K // 2), dtype=np.uint8)
    sf = np.empty((rows, K // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    gin = None
    if global_scale is not None:
        gin = np.array([global_scale], dtype=np.float32)
    lib().oracle_quantize(_p(x), rows, K, _p(gin) if gin is not None else None, _p(q), _p(sf), _p(g))
    return q, sf, np.float32(g[0])


def quantize_with_amax(x_bf16: np.ndarray, amax_value: float):
    """quantize() of rows that belong to a larger tensor whose amax is amax_value (one global scale per
    tensor, reading 8): the same steps with the given amax."""
    x = _u16(x_bf16)
    rows, K = x.shape
    if K % 16:
        raise ValueError("K must be a multiple of 16")
    q = np.empty((rows, K // 2), dtype=np.uint8)
    sf = np.empty((rows, K // 16), dtype=np.uint8)
    g = np.zeros(1, dtype=np.float32)
    lib().oracle_quantize_amax(_p(x), rows, K, np.float32(amax_value), _p(q), _p(sf), _p(g))
    return q, sf, np.float32(g[0])


def dequantize(q: np.ndarray, sf: np.ndarray, g_dec: float) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    rows, half = q.shape
    K = half * 2
    out = np.empty((rows, K), dtype=np.float64)
    lib().oracle_dequantize(_p(q), _p(sf), float(g_dec), rows, K, _p(out))
    return out


def permute(topk_ids: np.ndarray, num_experts: int):
    """topk_ids [T, k] int32 -> (offsets [E+1], perm_src [T*k], inv_perm [T*k])."""
    ids = np.ascontiguousarray(topk_ids, dtype=np.int32)
    T, k = ids.shape
    off = np.empty(num_experts + 1, dtype=np.int32)
    src = np.empty(T * k, dtype=np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    rc = lib().oracle_permute(_p(ids), T, k, num_experts, _p(off), _p(src), _p(inv))
    if rc != 0:
        raise ValueError(f"oracle_permute failed ({rc}): expert id out of range")
    return off, src, inv


def gather_rows(src: np.ndarray, idx: np.ndarray) -> np.ndarray:
    src = np.ascontiguousarray(src)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    row_bytes = src.strides[0]
    out = np.empty((idx.size,) + src.shape[1:], dtype=src.dtype)
    lib().oracle_gather_rows(_p(src), row_bytes, _p(idx), idx.size, _p(out))
    return out


def grouped_gemm(a_q, a_sf, a_g, w_q, w_sf, w_g, offsets, N, K, swiglu: bool) -> np.ndarray:
    """FP64 result [rows, N or N/2] for every routed row (weights' sf row-major)."""
    a_q = np.ascontiguousarray(a_q, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    w_q = np.ascontiguousarray(w_q, dtype=np.uint8)
    w_sf = np.ascontiguousarray(w_sf, dtype=np.uint8)
    w_g = np.ascontiguousarray(w_g, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    E = off.size - 1
    rows = int(off[-1])
    nout = N // 2 if swiglu else N
    out = np.empty((rows, nout), dtype=np.float64)
    lib().oracle_grouped_gemm(_p(a_q), _p(a_sf), float(a_g), _p(w_q), _p(w_sf), _p(w_g), _p(off),
                              E, N, K, 1 if swiglu else 0, _p(out))
    return out


def grouped_gemm_at(a_q, a_sf, a_g, w_q, w_sf, w_g, offsets, N, K, swiglu: bool, rows, cols) -> np.ndarray:
    """FP64 result at the selected (row, col) points only."""
    a_q = np.ascontiguousarray(a_q, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    w_q = np.ascontiguousarray(w_q, dtype=np.uint8)
    w_sf = np.ascontiguousarray(w_sf, dtype=np.uint8)
    w_g = np.ascontiguousarray(w_g, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    r = np.ascontiguousarray(rows, dtype=np.int64)
    c = np.ascontiguousarray(cols, dtype=np.int64)
    out = np.empty(r.size, dtype=np.float64)
    lib().oracle_grouped_gemm_at(_p(a_q), _p(a_sf), float(a_g), _p(w_q), _p(w_sf), _p(w_g), _p(off),
                                 off.size - 1, N, K, 1 if swiglu else 0, _p(r), _p(c), r.size, _p(out))
    return out


def route_topk(logits: np.ndarray, k: int):
    """Router: logits [T, E] FP32 -> (topk_ids [T, k] int32, topk_w [T, k] float32)."""
    z = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = z.shape
    if not 1 <= k <= E:
        raise ValueError("need 1 <= k <= E")
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float32)
    lib().oracle_route_topk(_p(z), T, E, int(k), _p(ids), _p(w))
    return ids, w


def grouped_gemm_bound(a_q, a_sf, a_g, w_q, w_sf, w_g, offsets, N, K, swiglu: bool, rows=None, cols=None):
    """Per-output bound on |FP32-path result - exact result| (the error model of the tensor-core path: exact
    16-element block partials, FP32 accumulation over the K/16 blocks, FP32 epilogue; see the C source).
    Every output like grouped_gemm(), or only the (rows, cols) points like grouped_gemm_at()."""
    a_q = np.ascontiguousarray(a_q, dtype=np.uint8)
    a_sf = np.ascontiguousarray(a_sf, dtype=np.uint8)
    w_q = np.ascontiguousarray(w_q, dtype=np.uint8)
    w_sf = np.ascontiguousarray(w_sf, dtype=np.uint8)
    w_g = np.ascontiguousarray(w_g, dtype=np.float32)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    if rows is None:
        nout = N // 2 if swiglu else N
        out = np.empty((int(off[-1]), nout), dtype=np.float64)
        lib().oracle_grouped_gemm_bound(_p(a_q), _p(a_sf), float(a_g), _p(w_q), _p(w_sf), _p(w_g), _p(off),
                                        off.size - 1, N, K, 1 if swiglu else 0, _p(out))
        return out
    r = np.ascontiguousarray(rows, dtype=np.int64)
    c = np.ascontiguousarray(cols, dtype=np.int64)
    out = np.empty(r.size, dtype=np.float64)
    lib().oracle_grouped_gemm_bound_at(_p(a_q), _p(a_sf), float(a_g), _p(w_q), _p(w_sf), _p(w_g), _p(off),
                                       off.size - 1, N, K, 1 if swiglu else 0, _p(r), _p(c), r.size, _p(out))
    return out


def combine(y_bf16: np.ndarray, inv_perm: np.ndarray, topk_w: np.ndarray) -> np.ndarray:
    """FP64 result [T, H] of the top-k weighted combine."""
    y = _u16(y_bf16)
    inv = np.ascontiguousarray(inv_perm, dtype=np.int32)
    w = np.ascontiguousarray(topk_w, dtype=np.float32)
    T, k = w.shape
    H = y.shape[1]
    out = np.empty((T, H), dtype=np.float64)
    lib().oracle_combine(_p(y), _p(inv), _p(w), T, k, H, _p(out))
    return out


__all__ = [
    "lib", "num_threads", "set_num_threads", "e2m1_decode", "e2m1_encode", "e4m3_decode", "e4m3_encode",
    "bf16_to_float", "bf16_from_double", "bf16_round", "bf16_bits_to_f64", "amax", "quantize", "dequantize",
    "permute", "gather_rows", "grouped_gemm", "grouped_gemm_at", "combine", "route_topk", "grouped_gemm_bound",
]
