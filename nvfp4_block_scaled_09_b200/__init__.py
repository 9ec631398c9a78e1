"""NVFP4 block-scaled Mixture-of-Experts hot path for B200 (sm_100a).

A thin Python binding over the C ABI in ``include/nvfp4moe.h`` (library
``lib/libnvfp4moe.so``, built by ``build.py``). Every function here only
marshals torch tensors into pointers, sizes and the current CUDA stream; all
arithmetic runs in the library's CUDA kernels. PyTorch supplies device memory,
streams and workspaces. There is no CPU fallback: without the built library or
without a CUDA device the calls raise.

Calls (same names as the C ABI):
  quantize            -> nvfp4_quantize
  permute             -> moe_permute
  quantize_permute    -> moe_quantize_permute_prefetch (no hint: moe_quantize_permute's bytes)
  grouped_gemm        -> moe_grouped_gemm_nvfp4 (moe_grouped_gemm_nvfp4_amax with amax_out)
  quantize_from_amax  -> nvfp4_quantize_from_amax_prefetch (no hint: nvfp4_quantize_from_amax)
  layer_l2_prefetch_bytes -> moe_layer_l2_prefetch_bytes
  amax                -> nvfp4_amax
  pack_weights        -> nvfp4_pack_weights
  unpermute_combine   -> moe_unpermute_combine
  route_topk          -> moe_route_topk
  moe_layer           -> moe_layer_nvfp4
  moe_layer_from_logits -> moe_layer_nvfp4_from_logits
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "lib", "libnvfp4moe.so")

STATUS = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_MISALIGNED", 3: "NVFP4_ERR_UNSUPPORTED_SHAPE",
    4: "NVFP4_ERR_WORKSPACE", 5: "NVFP4_ERR_SMEM_BUDGET", 6: "NVFP4_ERR_CUDA", 7: "NVFP4_ERR_DEVICE_TIMEOUT",
    8: "NVFP4_ERR_DEVICE_INPUT",
}
OK = 0
EPI_NONE, EPI_SWIGLU = 0, 1
SF_ROWMAJOR, SF_MMA_TILED, SF_KSTAGE = 0, 1, 2


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


class LayerWorkspace(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "q_x", "sf_x", "g_x", "q_perm", "sf_perm", "offsets", "perm_src", "inv_perm", "h", "q_h", "sf_h", "g_h",
        "amax_h", "fin_counters", "y", "scratch", "topk_ids", "topk_w", "total")]


class GemmPlan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "tile_weight_rows", "tile_tokens_max", "stage_k", "stages", "stage_bytes_weights", "stage_bytes_weight_sf",
        "stage_bytes_act_max", "stage_bytes_act_sf", "smem_bytes", "tmem_columns", "threads",
        "wide_tile_tokens_max", "wide_stage_bytes_act_max", "wide_smem_bytes", "wide_min_avg_rows",
        "pair_tile_tokens_max", "pair_smem_bytes", "pair_min_avg_rows")]


_lib = None


def lib():
    """Load the CUDA library (fails loudly when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m nvfp4_block_scaled_09_b200.build` "
                              "(or __graft_entry__.build()) first")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        st = ctypes.c_int
        L.nvfp4_quantize_workspace_size.argtypes = [i64, i64]
        L.nvfp4_quantize_workspace_size.restype = sz
        L.nvfp4_quantize.argtypes = [P, i64, i64, P, P, P, P, ctypes.c_int, P, sz, P]
        L.nvfp4_quantize.restype = st
        L.moe_permute_workspace_size.argtypes = [i32, i32, i32]
        L.moe_permute_workspace_size.restype = sz
        L.moe_permute.argtypes = [P, i32, i32, i32, P, P, i64, P, P, ctypes.c_int, P, P, P, P, sz, P]
        L.moe_quantize_permute_workspace_size.argtypes = [i32, i32, i32, i64]
        L.moe_quantize_permute_workspace_size.restype = sz
        L.moe_quantize_permute.argtypes = [P, i32, i64, P, i32, i32, P, P, ctypes.c_int, P, P, P, P, P, sz, P]
        L.moe_quantize_permute.restype = st
        L.moe_quantize_permute_prefetch.argtypes = [P, i32, i64, P, i32, i32, P, P, ctypes.c_int, P, P, P, P, P, sz,
                                                    P, sz, P]
        L.moe_quantize_permute_prefetch.restype = st
        L.moe_layer_l2_prefetch_bytes.argtypes = [i32, i32, i32, i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.moe_layer_l2_prefetch_bytes.restype = None
        L.moe_permute.restype = st
        L.moe_permute_noalloc.argtypes = [P, i32, i32, i32, P, P, i64, P, P, ctypes.c_int, P, P, P, P]
        L.moe_permute_noalloc.restype = st
        L.moe_grouped_gemm_nvfp4.argtypes = [P, P, P, P, P, P, i32, i64, i64, i64, ctypes.c_int, P, P]
        L.moe_grouped_gemm_nvfp4.restype = st
        L.moe_grouped_gemm_nvfp4_amax.argtypes = [P, P, P, P, P, P, i32, i64, i64, i64, ctypes.c_int, P, P, P]
        L.moe_grouped_gemm_nvfp4_amax.restype = st
        L.nvfp4_quantize_from_amax.argtypes = [P, i64, i64, P, P, P, P, ctypes.c_int, P]
        L.nvfp4_quantize_from_amax.restype = st
        L.nvfp4_quantize_from_amax_prefetch.argtypes = [P, i64, i64, P, P, P, P, ctypes.c_int, P, sz, P]
        L.nvfp4_quantize_from_amax_prefetch.restype = st
        L.nvfp4_amax.argtypes = [P, i64, i64, P, P]
        L.nvfp4_amax.restype = st
        L.moe_unpermute_combine.argtypes = [P, P, P, i32, i32, i64, P, P]
        L.moe_unpermute_combine.restype = st
        L.moe_layer_workspace_layout.argtypes = [i32, i32, i32, i64, i64, ctypes.POINTER(LayerWorkspace)]
        L.moe_layer_workspace_layout.restype = st
        L.moe_layer_workspace_size.argtypes = [i32, i32, i32, i64, i64]
        L.moe_layer_workspace_size.restype = sz
        L.moe_layer_nvfp4.argtypes = [P, P, P, i32, i32, i32, i64, i64, P, P, P, P, P, P, sz, P]
        L.moe_layer_nvfp4_from_logits.argtypes = [P, P, i32, i32, i32, i64, i64, P, P, P, P, P, P, sz, P]
        L.moe_layer_nvfp4_from_logits.restype = st
        L.moe_route_topk.argtypes = [P, i32, i32, i32, P, P, P]
        L.moe_route_topk.restype = st
        L.moe_grouped_gemm_nvfp4_quant.argtypes = [P, P, P, P, P, P, i32, i64, i64, i64, P, P, P, P, P]
        L.moe_grouped_gemm_nvfp4_quant.restype = st
        L.moe_finalize_counters_size.argtypes = [i32, i64]
        L.moe_finalize_counters_size.restype = sz
        L.moe_grouped_gemm_nvfp4_finalize.argtypes = [P, P, P, P, P, P, i32, i64, i64, i64, P, P, P, P, i32, i32, P,
                                                      P, P]
        L.moe_grouped_gemm_nvfp4_finalize.restype = st
        L.nvfp4_packed_weight_bytes.argtypes = [i64, i64]
        L.nvfp4_packed_weight_bytes.restype = sz
        L.nvfp4_pack_weights.argtypes = [P, P, i64, i64, P, P]
        L.nvfp4_pack_weights.restype = st
        L.moe_layer_nvfp4.restype = st
        L.nvfp4_gemm_get_plan.argtypes = [ctypes.POINTER(GemmPlan)]
        L.nvfp4_gemm_get_plan.restype = st
        L.nvfp4_gemm_stage_tx_bytes.argtypes = [i32, i32]
        L.nvfp4_gemm_stage_tx_bytes.restype = i64
        L.nvfp4_can_implement_with_budget.argtypes = [i64, i64, i32, ctypes.c_int, i64]
        L.nvfp4_can_implement_with_budget.restype = st
        L.nvfp4_can_implement.argtypes = [i64, i64, i32, ctypes.c_int]
        L.nvfp4_can_implement.restype = st
        L.nvfp4_get_device_status.argtypes = [P]
        L.nvfp4_get_device_status.restype = st
        L.nvfp4_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
        L.nvfp4_set_wait_timeout_ns.restype = None
        L.nvfp4_get_wait_timeout_ns.restype = ctypes.c_uint64
        L.nvfp4_launch_count.restype = ctypes.c_uint64
        L.nvfp4_debug_set_flags.argtypes = [ctypes.c_uint32]
        L.nvfp4_debug_set_flags.restype = None
        L.nvfp4_status_string.argtypes = [ctypes.c_int]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != OK:
        raise NVFP4Error(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("nvfp4 calls take CUDA tensors only (no CPU fallback)")


def _bits(t: torch.Tensor) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bfloat16 tensor")
    return t.contiguous()


def _need(t: torch.Tensor, nbytes: int, what: str, dtype=None) -> torch.Tensor:
    """A caller-given buffer the library reads or writes `nbytes` of: contiguous, large enough, of `dtype`
    when given (the library sees only a pointer, so a short buffer would be overrun on the device)."""
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{what} holds {have} bytes; the call needs {nbytes}")
    return t


# ----------------------------------------------------------------------------- quantize

def kstage_slabs(K: int) -> int:
    """K-stage scale slabs of a K-element row: one per 256 elements, the last one zero-padded when K % 256."""
    return (K + 255) // 256


def sf_bytes(rows: int, K: int, layout: int) -> int:
    return kstage_slabs(K) * rows * 16 if layout == SF_KSTAGE else rows * K // 16


def _sf_empty(rows: int, K: int, layout: int, dev) -> torch.Tensor:
    """Scale buffer of a [rows, K] tensor: [ceil(K/256), rows, 16] in the K-stage layout, else [rows, K/16]."""
    if layout == SF_KSTAGE:
        return torch.empty((kstage_slabs(K), rows, 16), dtype=torch.uint8, device=dev)
    return torch.empty((rows, K // 16), dtype=torch.uint8, device=dev)


def quantize_workspace_size(rows: int, K: int) -> int:
    return int(lib().nvfp4_quantize_workspace_size(rows, K))


def quantize(x: torch.Tensor, global_scale: torch.Tensor | None = None, layout: int = SF_ROWMAJOR,
             q: torch.Tensor | None = None, sf: torch.Tensor | None = None, g: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream=None):
    """x [rows, K] bf16 -> (q uint8 [rows, K/2], sf uint8, g float32 [1] = g_dec). sf is [rows, K/16] for
    SF_ROWMAJOR and SF_MMA_TILED, [K/256, rows, 16] for SF_KSTAGE (the grouped GEMM's activation scales)."""
    _require_cuda(x, global_scale)
    x = _bits(x)
    rows, K = x.shape
    dev = x.device
    q = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev) if q is None else _need(q, rows * K // 2, "q")
    sf = _sf_empty(rows, K, layout, dev) if sf is None else _need(sf, sf_bytes(rows, K, layout), "sf")
    g = torch.empty(1, dtype=torch.float32, device=dev) if g is None else _need(g, 4, "g", torch.float32)
    if ws is None and global_scale is None:
        ws = torch.empty(max(quantize_workspace_size(rows, K), 16), dtype=torch.uint8, device=dev)
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().nvfp4_quantize(_ptr(x), rows, K, _ptr(global_scale), _ptr(q), _ptr(sf), _ptr(g), layout,
                                _ptr(ws), nbytes, _stream(stream)), "nvfp4_quantize")
    return q, sf, g


def amax(x: torch.Tensor, amax_bits: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Raise amax_bits (device int32 [1], zeroed here when not given) to max |x| as BF16 bits."""
    _require_cuda(x, amax_bits)
    x = _bits(x)
    if amax_bits is None:
        amax_bits = torch.zeros(1, dtype=torch.int32, device=x.device)
    _need(amax_bits, 4, "amax_bits")
    _check(lib().nvfp4_amax(_ptr(x), x.shape[0], x.shape[1], _ptr(amax_bits), _stream(stream)), "nvfp4_amax")
    return amax_bits


def _l2_hint(l2_next, l2_next_bytes):
    """(pointer, bytes) of an L2 prefetch hint: the first l2_next_bytes bytes of the device tensor l2_next (all of
    it by default), or (None, 0)."""
    if l2_next is None:
        return None, 0
    _require_cuda(l2_next)
    n = l2_next.numel() * l2_next.element_size()
    return _ptr(l2_next), n if l2_next_bytes is None else min(int(l2_next_bytes), n)


def layer_l2_prefetch_bytes(T: int, k: int, E: int, H: int, I: int) -> tuple[int, int]:
    """The L2 prefetch hints moe_layer_nvfp4 gives: bytes of the gate/up and of the down packed weights
    (moe_layer_l2_prefetch_bytes)."""
    g, d = ctypes.c_size_t(0), ctypes.c_size_t(0)
    lib().moe_layer_l2_prefetch_bytes(T, k, E, H, I, ctypes.byref(g), ctypes.byref(d))
    return g.value, d.value


def quantize_from_amax(x: torch.Tensor, amax_bits: torch.Tensor, layout: int = SF_ROWMAJOR,
                       q: torch.Tensor | None = None, sf: torch.Tensor | None = None, g: torch.Tensor | None = None,
                       stream=None, l2_next: torch.Tensor | None = None, l2_next_bytes: int | None = None):
    """quantize() with a dynamic global scale from a known amax: amax_bits is a device int32 [1] holding max |x|
    as BF16 bits (e.g. the amax_out of grouped_gemm). l2_next / l2_next_bytes: an L2 prefetch hint for the next
    kernel's constant operand (nvfp4_quantize_from_amax_prefetch); the outputs do not depend on it."""
    _require_cuda(x, amax_bits)
    x = _bits(x)
    rows, K = x.shape
    dev = x.device
    _need(amax_bits, 4, "amax_bits")
    q = torch.empty((rows, K // 2), dtype=torch.uint8, device=dev) if q is None else _need(q, rows * K // 2, "q")
    sf = _sf_empty(rows, K, layout, dev) if sf is None else _need(sf, sf_bytes(rows, K, layout), "sf")
    g = torch.empty(1, dtype=torch.float32, device=dev) if g is None else _need(g, 4, "g", torch.float32)
    pf, pf_bytes = _l2_hint(l2_next, l2_next_bytes)
    _check(lib().nvfp4_quantize_from_amax_prefetch(_ptr(x), rows, K, _ptr(amax_bits), _ptr(q), _ptr(sf), _ptr(g),
                                                   layout, pf, pf_bytes, _stream(stream)),
           "nvfp4_quantize_from_amax_prefetch")
    return q, sf, g


def packed_weight_bytes(rows: int, K: int) -> int:
    return int(lib().nvfp4_packed_weight_bytes(rows, K))


def pack_weights(q: torch.Tensor, sf: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Quantised weights (codes [rows, K/2], row-major scales [rows, K/16]) -> the GEMM's packed tiles."""
    _require_cuda(q, sf)
    rows, half = q.shape[-2], q.shape[-1]
    rows = q.numel() // half
    K = half * 2
    _need(q, rows * K // 2, "q")
    _need(sf, rows * K // 16, "sf")
    if out is None:
        out = torch.empty(packed_weight_bytes(rows, K), dtype=torch.uint8, device=q.device)
    else:
        _need(out, packed_weight_bytes(rows, K), "out")
    _check(lib().nvfp4_pack_weights(_ptr(q), _ptr(sf), rows, K, _ptr(out), _stream(stream)), "nvfp4_pack_weights")
    return out


@dataclass
class PackedWeights:
    packed: torch.Tensor          # [E, packed_weight_bytes(N, K)] bytes, packed tiles
    gscale: torch.Tensor          # [E] FP32 global scales (dequantisation multipliers)
    E: int
    N: int
    K: int
    q: torch.Tensor | None = None   # row-major codes [E, N, K/2] (kept only on request)
    sf: torch.Tensor | None = None  # row-major scales [E, N, K/16] (kept only on request)


def prepare_expert_weights(w: torch.Tensor, keep_rowmajor: bool = False, stream=None) -> PackedWeights:
    """Weights [E, N, K] bf16 -> packed NVFP4 tiles with one global scale per expert matrix.
    One-time preparation: quantise each expert (row-major), then pack."""
    _require_cuda(w)
    E, N, K = w.shape
    dev = w.device
    packed = torch.empty((E, packed_weight_bytes(N, K)), dtype=torch.uint8, device=dev)
    g = torch.empty(E, dtype=torch.float32, device=dev)
    qk = torch.empty((E, N, K // 2), dtype=torch.uint8, device=dev) if keep_rowmajor else None
    sk = torch.empty((E, N, K // 16), dtype=torch.uint8, device=dev) if keep_rowmajor else None
    qt = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    st = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
    ws = torch.empty(max(quantize_workspace_size(N, K), 16), dtype=torch.uint8, device=dev)
    for e in range(E):
        q_e = qk[e] if keep_rowmajor else qt
        s_e = sk[e] if keep_rowmajor else st
        quantize(w[e], q=q_e, sf=s_e, g=g[e:e + 1], ws=ws, stream=stream)
        pack_weights(q_e, s_e, out=packed[e], stream=stream)
    return PackedWeights(packed, g, E, N, K, qk, sk)


# ----------------------------------------------------------------------------- permute

def permute_workspace_size(T: int, k: int, E: int) -> int:
    return int(lib().moe_permute_workspace_size(T, k, E))


@dataclass
class Permuted:
    q_perm: torch.Tensor
    sf_perm: torch.Tensor
    offsets: torch.Tensor
    perm_src: torch.Tensor
    inv_perm: torch.Tensor


def permute(topk_ids: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, num_experts: int, ws=None,
            stream=None, sf_layout: int = SF_KSTAGE) -> Permuted:
    """Group the routed rows by expert. sf is row-major [T, K/16]; sf_perm comes out in sf_layout:
    SF_KSTAGE (what grouped_gemm reads, [K/256, T*k, 16]) or SF_ROWMAJOR ([T*k, K/16])."""
    _require_cuda(topk_ids, q, sf)
    if topk_ids.dtype != torch.int32:
        raise TypeError("topk_ids must be int32")
    topk_ids = topk_ids.contiguous()
    T, k = topk_ids.shape
    K = q.shape[1] * 2
    R = T * k
    dev = q.device
    _need(q, T * K // 2, "q")
    _need(sf, T * K // 16, "sf")
    out = Permuted(
        q_perm=torch.empty((R, K // 2), dtype=torch.uint8, device=dev),
        sf_perm=_sf_empty(R, K, sf_layout, dev),
        offsets=torch.empty(num_experts + 1, dtype=torch.int32, device=dev),
        perm_src=torch.empty(R, dtype=torch.int32, device=dev),
        inv_perm=torch.empty(R, dtype=torch.int32, device=dev),
    )
    if ws is None:
        ws = torch.empty(max(permute_workspace_size(T, k, num_experts), 16), dtype=torch.uint8, device=dev)
    _check(lib().moe_permute(_ptr(topk_ids), T, k, num_experts, _ptr(q), _ptr(sf), K, _ptr(out.q_perm),
                             _ptr(out.sf_perm), sf_layout, _ptr(out.offsets), _ptr(out.perm_src), _ptr(out.inv_perm),
                             _ptr(ws), ws.numel(), _stream(stream)), "moe_permute")
    return out


def quantize_permute(x: torch.Tensor, topk_ids: torch.Tensor, num_experts: int, ws=None, stream=None,
                     sf_layout: int = SF_KSTAGE, l2_next: torch.Tensor | None = None,
                     l2_next_bytes: int | None = None):
    """quantize(x) then permute of the result in one call (moe_quantize_permute): the same bytes.
    Returns (Permuted, g) with g the float32 [1] global scale of x. l2_next / l2_next_bytes: an L2 prefetch
    hint for the next kernel's constant operand (moe_quantize_permute_prefetch)."""
    _require_cuda(x, topk_ids)
    if topk_ids.dtype != torch.int32:
        raise TypeError("topk_ids must be int32")
    topk_ids = topk_ids.contiguous()
    T, k = topk_ids.shape
    if x.dim() != 2 or x.shape[0] != T:
        raise ValueError(f"x must be [T={T}, H]")
    H = x.shape[1]
    _need(x, T * H * 2, "x", torch.bfloat16)
    R = T * k
    dev = x.device
    out = Permuted(
        q_perm=torch.empty((R, H // 2), dtype=torch.uint8, device=dev),
        sf_perm=_sf_empty(R, H, sf_layout, dev),
        offsets=torch.empty(num_experts + 1, dtype=torch.int32, device=dev),
        perm_src=torch.empty(R, dtype=torch.int32, device=dev),
        inv_perm=torch.empty(R, dtype=torch.int32, device=dev),
    )
    g = torch.empty(1, dtype=torch.float32, device=dev)
    need = int(lib().moe_quantize_permute_workspace_size(T, k, num_experts, H))
    if ws is None:
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    else:
        _need(ws, need, "ws")
    pf, pf_bytes = _l2_hint(l2_next, l2_next_bytes)
    _check(lib().moe_quantize_permute_prefetch(_ptr(x), T, H, _ptr(topk_ids), k, num_experts, _ptr(out.q_perm),
                                               _ptr(out.sf_perm), sf_layout, _ptr(g), _ptr(out.offsets),
                                               _ptr(out.perm_src), _ptr(out.inv_perm), _ptr(ws), ws.numel(), pf,
                                               pf_bytes, _stream(stream)),
           "moe_quantize_permute_prefetch")
    return out, g


def permute_noalloc(topk_ids: torch.Tensor, q: torch.Tensor, sf: torch.Tensor, num_experts: int,
                    stream=None, sf_layout: int = SF_KSTAGE) -> Permuted:
    """moe_permute without a workspace: the library's own fixed device array holds the count table
    (for callers that cannot allocate device memory; see moe_permute_noalloc in the header)."""
    _require_cuda(topk_ids, q, sf)
    if topk_ids.dtype != torch.int32:
        raise TypeError("topk_ids must be int32")
    topk_ids = topk_ids.contiguous()
    T, k = topk_ids.shape
    K = q.shape[1] * 2
    R = T * k
    dev = q.device
    _need(q, T * K // 2, "q")
    _need(sf, T * K // 16, "sf")
    out = Permuted(
        q_perm=torch.empty((R, K // 2), dtype=torch.uint8, device=dev),
        sf_perm=_sf_empty(R, K, sf_layout, dev),
        offsets=torch.empty(num_experts + 1, dtype=torch.int32, device=dev),
        perm_src=torch.empty(R, dtype=torch.int32, device=dev),
        inv_perm=torch.empty(R, dtype=torch.int32, device=dev),
    )
    _check(lib().moe_permute_noalloc(_ptr(topk_ids), T, k, num_experts, _ptr(q), _ptr(sf), K, _ptr(out.q_perm),
                                     _ptr(out.sf_perm), sf_layout, _ptr(out.offsets), _ptr(out.perm_src),
                                     _ptr(out.inv_perm), _stream(stream)), "moe_permute_noalloc")
    return out


# ----------------------------------------------------------------------------- grouped GEMM

def grouped_gemm(a_q, a_sf, a_g, w: PackedWeights, offsets, swiglu: bool, out=None, stream=None, amax_out=None):
    """Per-expert NVFP4 GEMM. a_sf holds the activation scales in the K-stage layout ([K/256, rows, 16], as
    permute() and quantize(layout=SF_KSTAGE) write them). Returns bf16 [rows, N] (or [rows, N/2] with SwiGLU).
    With amax_out (device int32 [1], zeroed by the caller) the kernel also raises it to max |out| as BF16 bits."""
    _require_cuda(a_q, a_sf, a_g, w.packed, w.gscale, offsets, amax_out)
    rows = a_q.shape[0]
    if a_sf.dim() != 3 or tuple(a_sf.shape) != (kstage_slabs(w.K), rows, 16):
        raise ValueError(f"a_sf must be K-stage scales of shape {(kstage_slabs(w.K), rows, 16)}, "
                         f"got {tuple(a_sf.shape)}")
    E = offsets.numel() - 1
    N, K = w.N, w.K
    nout = N // 2 if swiglu else N
    _need(a_q, rows * K // 2, "a_q")
    _need(a_sf, sf_bytes(rows, K, SF_KSTAGE), "a_sf")
    if amax_out is not None:
        _need(amax_out, 4, "amax_out")
    if out is None:
        out = torch.empty((rows, nout), dtype=torch.bfloat16, device=a_q.device)
    else:
        _need(out, rows * nout * 2, "out", torch.bfloat16)
    _check(lib().moe_grouped_gemm_nvfp4_amax(_ptr(a_q), _ptr(a_sf), _ptr(a_g), _ptr(w.packed), _ptr(w.gscale),
                                             _ptr(offsets), E, rows, N, K, EPI_SWIGLU if swiglu else EPI_NONE,
                                             _ptr(out), _ptr(amax_out), _stream(stream)), "moe_grouped_gemm_nvfp4_amax")
    return out


def grouped_gemm_quant(a_q, a_sf, a_g, w: PackedWeights, offsets, h_gscale, q_h=None, sf_h=None, amax_out=None,
                       stream=None):
    """Gate/up GEMM (SwiGLU) whose epilogue writes h as NVFP4 with the static global scale h_gscale (device
    float32 [1], g_dec): returns (q_h uint8 [rows, N/4], sf_h uint8 K-stage [ceil((N/2)/256), rows, 16]), the
    bytes nvfp4_quantize(h, global_scale=h_gscale, layout=SF_KSTAGE) gives for the BF16 h grouped_gemm writes.
    amax_out (device int32 [1], zeroed by the caller) is raised to max |h| as BF16 bits."""
    _require_cuda(a_q, a_sf, a_g, w.packed, w.gscale, offsets, h_gscale, amax_out)
    rows = a_q.shape[0]
    N, K = w.N, w.K
    E = offsets.numel() - 1
    hc = N // 2
    if a_sf.dim() != 3 or tuple(a_sf.shape) != (kstage_slabs(K), rows, 16):
        raise ValueError(f"a_sf must be K-stage scales of shape {(kstage_slabs(K), rows, 16)}")
    _need(a_q, rows * K // 2, "a_q")
    _need(a_sf, sf_bytes(rows, K, SF_KSTAGE), "a_sf")
    _need(h_gscale, 4, "h_gscale", torch.float32)
    if amax_out is not None:
        _need(amax_out, 4, "amax_out")
    q_h = torch.empty((rows, hc // 2), dtype=torch.uint8, device=a_q.device) if q_h is None else \
        _need(q_h, rows * hc // 2, "q_h")
    sf_h = _sf_empty(rows, hc, SF_KSTAGE, a_q.device) if sf_h is None else _need(sf_h, sf_bytes(rows, hc, SF_KSTAGE),
                                                                                  "sf_h")
    _check(lib().moe_grouped_gemm_nvfp4_quant(_ptr(a_q), _ptr(a_sf), _ptr(a_g), _ptr(w.packed), _ptr(w.gscale),
                                              _ptr(offsets), E, rows, N, K, _ptr(h_gscale), _ptr(q_h), _ptr(sf_h),
                                              _ptr(amax_out), _stream(stream)), "moe_grouped_gemm_nvfp4_quant")
    return q_h, sf_h


def finalize_counters(T: int, N: int, device="cuda") -> torch.Tensor:
    """Zeroed arrival counters for grouped_gemm_finalize (each call leaves them zero)."""
    n = int(lib().moe_finalize_counters_size(T, N))
    return torch.zeros(max(n // 4, 1), dtype=torch.int32, device=device)


def grouped_gemm_finalize(a_q, a_sf, a_g, w: PackedWeights, offsets, perm_src, inv_perm, topk_w, counters,
                          y=None, out=None, stream=None):
    """Down GEMM (plain epilogue) with the top-k combine fused into its epilogue: returns (out [T, N] bf16,
    y [rows, N] bf16). perm_src / inv_perm as permute() returns them, topk_w [T, k] float32."""
    _require_cuda(a_q, a_sf, a_g, w.packed, w.gscale, offsets, perm_src, inv_perm, topk_w, counters)
    rows = a_q.shape[0]
    T, k = topk_w.shape
    N, K = w.N, w.K
    E = offsets.numel() - 1
    if a_sf.dim() != 3 or tuple(a_sf.shape) != (kstage_slabs(K), rows, 16):
        raise ValueError(f"a_sf must be K-stage scales of shape {(kstage_slabs(K), rows, 16)}")
    _need(a_q, rows * K // 2, "a_q")
    _need(a_sf, sf_bytes(rows, K, SF_KSTAGE), "a_sf")
    _need(perm_src, rows * 4, "perm_src", torch.int32)
    _need(inv_perm, T * k * 4, "inv_perm", torch.int32)
    _need(topk_w, T * k * 4, "topk_w", torch.float32)
    _need(counters, int(lib().moe_finalize_counters_size(T, N)), "counters")
    y = torch.empty((rows, N), dtype=torch.bfloat16, device=a_q.device) if y is None else \
        _need(y, rows * N * 2, "y", torch.bfloat16)
    out = torch.empty((T, N), dtype=torch.bfloat16, device=a_q.device) if out is None else \
        _need(out, T * N * 2, "out", torch.bfloat16)
    _check(lib().moe_grouped_gemm_nvfp4_finalize(_ptr(a_q), _ptr(a_sf), _ptr(a_g), _ptr(w.packed), _ptr(w.gscale),
                                                 _ptr(offsets), E, rows, N, K, _ptr(y), _ptr(perm_src),
                                                 _ptr(inv_perm), _ptr(topk_w), T, k, _ptr(counters), _ptr(out),
                                                 _stream(stream)), "moe_grouped_gemm_nvfp4_finalize")
    return out, y


def can_implement(N: int, K: int, E: int, swiglu: bool, smem_budget: int | None = None) -> int:
    epi = EPI_SWIGLU if swiglu else EPI_NONE
    if smem_budget is None:
        return int(lib().nvfp4_can_implement(N, K, E, epi))
    return int(lib().nvfp4_can_implement_with_budget(N, K, E, epi, smem_budget))


def gemm_plan() -> dict:
    p = GemmPlan()
    _check(lib().nvfp4_gemm_get_plan(ctypes.byref(p)), "nvfp4_gemm_get_plan")
    return {n: getattr(p, n) for n, _ in GemmPlan._fields_}


def gemm_stage_tx_bytes(tokens: int, wide: bool = False) -> int:
    return int(lib().nvfp4_gemm_stage_tx_bytes(tokens, 1 if wide else 0))


# ----------------------------------------------------------------------------- combine

def unpermute_combine(y: torch.Tensor, inv_perm: torch.Tensor, topk_w: torch.Tensor, out=None, stream=None):
    _require_cuda(y, inv_perm, topk_w)
    T, k = topk_w.shape
    H = y.shape[1]
    _need(inv_perm, T * k * 4, "inv_perm", torch.int32)
    _need(topk_w, T * k * 4, "topk_w", torch.float32)
    if y.shape[0] < T * k or inv_perm.numel() < T * k:
        raise ValueError(f"y and inv_perm need {T * k} rows for T={T}, k={k}")
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=y.device)
    else:
        _need(out, T * H * 2, "out", torch.bfloat16)
    _check(lib().moe_unpermute_combine(_ptr(y.contiguous()), _ptr(inv_perm), _ptr(topk_w.contiguous()), T, k, H,
                                       _ptr(out), _stream(stream)), "moe_unpermute_combine")
    return out


# ----------------------------------------------------------------------------- router

def route_topk(logits: torch.Tensor, k: int, ids: torch.Tensor | None = None, w: torch.Tensor | None = None,
               stream=None):
    """Router: logits [T, E] float32 -> (topk_ids int32 [T, k], topk_w float32 [T, k]): the k largest logits
    per token (lower index first among equal values) and the softmax of the chosen k."""
    _require_cuda(logits)
    if logits.dtype != torch.float32:
        raise TypeError("logits must be float32")
    _need(logits, logits.numel() * 4, "logits")
    T, E = logits.shape
    dev = logits.device
    ids = torch.empty((T, k), dtype=torch.int32, device=dev) if ids is None else _need(ids, T * k * 4, "ids",
                                                                                          torch.int32)
    w = torch.empty((T, k), dtype=torch.float32, device=dev) if w is None else _need(w, T * k * 4, "w",
                                                                                      torch.float32)
    _check(lib().moe_route_topk(_ptr(logits), T, E, k, _ptr(ids), _ptr(w), _stream(stream)), "moe_route_topk")
    return ids, w


# ----------------------------------------------------------------------------- layer

@dataclass
class MoEWeights:
    w13: PackedWeights   # gate/up [E, 2I, H]
    w2: PackedWeights    # down [E, H, I]

    @property
    def num_experts(self) -> int:
        return self.w13.E

    @property
    def hidden(self) -> int:
        return self.w13.K

    @property
    def intermediate(self) -> int:
        return self.w13.N // 2


def layer_workspace_layout(T: int, k: int, E: int, H: int, I: int) -> dict:
    L = LayerWorkspace()
    _check(lib().moe_layer_workspace_layout(T, k, E, H, I, ctypes.byref(L)), "moe_layer_workspace_layout")
    return {n: getattr(L, n) for n, _ in LayerWorkspace._fields_}


def layer_workspace(T: int, k: int, E: int, H: int, I: int, device="cuda") -> torch.Tensor:
    n = int(lib().moe_layer_workspace_size(T, k, E, H, I))
    return torch.empty(n, dtype=torch.uint8, device=device)


def moe_layer(x: torch.Tensor, topk_ids: torch.Tensor, topk_w: torch.Tensor, w: MoEWeights, ws=None, out=None,
              stream=None):
    """Whole MoE FFN: quantize -> permute -> gate/up GEMM + SwiGLU -> quantize -> down GEMM -> combine."""
    _require_cuda(x, topk_ids, topk_w)
    x = _bits(x)
    T, H = x.shape
    k = topk_ids.shape[1]
    E, I = w.num_experts, w.intermediate
    if ws is None:
        ws = layer_workspace(T, k, E, H, I, x.device)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, T * H * 2, "out", torch.bfloat16)
    _check(lib().moe_layer_nvfp4(_ptr(x), _ptr(topk_ids.contiguous()), _ptr(topk_w.contiguous()), T, k, E, H, I,
                                 _ptr(w.w13.packed), _ptr(w.w13.gscale), _ptr(w.w2.packed), _ptr(w.w2.gscale),
                                 _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "moe_layer_nvfp4")
    return out


def moe_layer_from_logits(x: torch.Tensor, logits: torch.Tensor, k: int, w: MoEWeights, ws=None, out=None,
                          stream=None):
    """moe_layer() with the routing computed by the router kernel from logits [T, E] float32."""
    _require_cuda(x, logits)
    x = _bits(x)
    T, H = x.shape
    E, I = w.num_experts, w.intermediate
    if logits.dtype != torch.float32 or tuple(logits.shape) != (T, E):
        raise ValueError(f"logits must be float32 [{T}, {E}]")
    _need(logits, T * E * 4, "logits")
    if ws is None:
        ws = layer_workspace(T, k, E, H, I, x.device)
    if out is None:
        out = torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    else:
        _need(out, T * H * 2, "out", torch.bfloat16)
    _check(lib().moe_layer_nvfp4_from_logits(_ptr(x), _ptr(logits), T, k, E, H, I, _ptr(w.w13.packed),
                                             _ptr(w.w13.gscale), _ptr(w.w2.packed), _ptr(w.w2.gscale), _ptr(out),
                                             _ptr(ws), ws.numel(), _stream(stream)), "moe_layer_nvfp4_from_logits")
    return out


# ----------------------------------------------------------------------------- diagnostics

def device_status(stream=None) -> int:
    """Synchronise, read and clear the device status word (returns a status code)."""
    return int(lib().nvfp4_get_device_status(_stream(stream)))


def set_wait_timeout_ns(ns: int) -> None:
    lib().nvfp4_set_wait_timeout_ns(int(ns))


def get_wait_timeout_ns() -> int:
    return int(lib().nvfp4_get_wait_timeout_ns())


def debug_set_flags(flags: int) -> None:
    """Test hook (see nvfp4_debug_set_flags in the header)."""
    lib().nvfp4_debug_set_flags(int(flags))


def launch_count() -> int:
    return int(lib().nvfp4_launch_count())


def status_string(status: int) -> str:
    return lib().nvfp4_status_string(int(status)).decode()
