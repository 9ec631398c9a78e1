"""The C-ABI library builds, loads and exports every call the header declares;
host-side checks (capability predicate, pipeline plan, stage byte accounting,
status strings) run without a GPU."""
import ctypes

import pytest

import nvfp4_block_scaled_09_b200 as nv
from nvfp4_block_scaled_09_b200 import build as nvbuild
from tests.helpers import header_symbols


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def test_every_header_symbol_is_exported(L):
    syms = header_symbols()
    assert len(syms) >= 18, syms
    for s in syms:
        assert hasattr(L, s), f"{s} declared in include/nvfp4moe.h but not exported"


def test_status_strings(L):
    for code, name in nv.STATUS.items():
        assert nv.status_string(code) == name


def test_can_implement_shapes_and_budget(L):
    big = 232448  # B200 opt-in shared memory per block
    plan = nv.gemm_plan()
    assert plan["smem_bytes"] <= big
    assert nv.can_implement(4096, 6144, 256, True, big) == 0
    assert nv.can_implement(6144, 2048, 256, False, big) == 0
    assert nv.can_implement(8192, 8192, 1, False, big) == 0
    assert nv.can_implement(256, 256, 4, False, big) == 0
    # K % 128 and, for the plain epilogue, N % 128; SwiGLU needs N % 256 (gate and up 128-row blocks)
    assert nv.can_implement(128, 128, 4, False, big) == 0
    assert nv.can_implement(384, 384, 4, False, big) == 0
    assert nv.can_implement(4096, 6144 + 128, 256, True, big) == 0
    assert nv.can_implement(4096 + 128, 6144, 256, True, big) == 3
    assert nv.can_implement(4096, 6144 + 64, 256, True, big) == 3
    assert nv.can_implement(128 + 64, 128, 4, False, big) == 3
    assert nv.can_implement(128, 64, 4, False, big) == 3
    assert nv.can_implement(4096, 6144, 1025, True, big) == 3
    assert nv.can_implement(0, 6144, 8, True, big) == 1
    # a budget below either tile shape's shared memory is refused before any launch
    need = max(plan["smem_bytes"], plan["wide_smem_bytes"], plan["pair_smem_bytes"])
    assert need <= big
    assert nv.can_implement(4096, 6144, 256, True, need - 1) == 5
    assert plan["pair_min_avg_rows"] > plan["wide_min_avg_rows"] and plan["pair_tile_tokens_max"] == 256
    assert nv.can_implement(4096, 6144, 256, True, 101376) == 5     # an SM120-sized budget


def test_stage_transaction_bytes_are_tile_sums(L):
    # Per stage: (A tile bits + A scale bits) + (B tile bits + B scale bits), in bytes, for
    # packed E2M1 (4 bits) and one 8-bit scale per 16 elements. The B rows are rounded up to
    # the 16-row TMA box; the B scales (one contiguous run of the K-stage slab) cover exactly
    # the tile's rows.
    plan = nv.gemm_plan()
    bk = plan["stage_k"]
    wrows = plan["tile_weight_rows"]
    a_bits = wrows * bk * 4
    sfa_bits = wrows * (bk // 16) * 8
    for wide, bn_max in ((False, plan["tile_tokens_max"]), (True, plan["wide_tile_tokens_max"])):
        for tokens in (1, 15, 16, 17, 32, 48, 64, 65, 100, 128):
            sfb_bits = tokens * (bk // 16) * 8
            if tokens > bn_max:
                assert nv.gemm_stage_tx_bytes(tokens, wide) == -1
                continue
            bn = -(-tokens // 16) * 16
            b_bits = bn * bk * 4
            assert nv.gemm_stage_tx_bytes(tokens, wide) == (a_bits + sfa_bits + b_bits + sfb_bits) // 8
        assert nv.gemm_stage_tx_bytes(0, wide) == -1
    assert plan["wide_tile_tokens_max"] > plan["tile_tokens_max"]
    # the rings fit the shared-memory budgets they claim
    for act, smem in ((plan["stage_bytes_act_max"], plan["smem_bytes"]),
                      (plan["wide_stage_bytes_act_max"], plan["wide_smem_bytes"])):
        stage = plan["stage_bytes_weights"] + plan["stage_bytes_weight_sf"] + act + plan["stage_bytes_act_sf"]
        assert plan["stages"] * stage <= smem <= 232448
    assert plan["tmem_columns"] in (32, 64, 128, 256, 512)


def test_layer_workspace_layout_is_disjoint_and_aligned(L):
    lay = nv.layer_workspace_layout(512, 8, 256, 6144, 2048)
    names = [n for n in lay if n != "total"]
    offs = sorted(lay[n] for n in names)
    assert all(o % 256 == 0 for o in offs)
    assert len(set(offs)) == len(offs)
    R = 512 * 8
    assert lay["q_perm"] - lay["g_x"] >= 4 and lay["sf_perm"] - lay["q_perm"] >= R * 6144 // 2
    assert lay["total"] >= lay["scratch"]


def test_invalid_arguments_rejected_before_any_cuda_call(L):
    # Null pointers and bad shapes return synchronously (no device needed).
    assert L.nvfp4_quantize(None, 4, 32, None, None, None, None, 0, None, 0, None) == 1
    assert L.moe_unpermute_combine(None, None, None, 1, 1, 8, None, None) == 1
    p = ctypes.c_void_p(16)
    assert L.moe_unpermute_combine(p, p, p, 1, 1, 12, p, None) == 3     # H % 8 != 0
    assert L.moe_permute(p, 4, 8, 2000, p, p, 256, p, p, 2, p, p, p, p, 1 << 20, None) == 3  # E > 1024
    assert L.moe_permute(p, 4, 8, 8, p, p, 256, p, p, 2, p, p, p, None, 0, None) == 4       # no workspace
    assert L.moe_permute(p, 4, 8, 8, p, p, 256, p, p, 1, p, p, p, p, 1 << 20, None) == 1    # tiled sf_perm
    assert L.moe_permute_noalloc(p, 4, 8, 8, p, p, 256, p, p, 7, p, p, p, None) == 1        # unknown layout
    assert L.nvfp4_quantize(p, 4, 64, p, p, p, p, 2, None, 0, None) == 3    # K-stage layout: K % 128 != 0
    assert L.nvfp4_quantize(p, 4, 128, p, p, ctypes.c_void_p(24), p, 2, None, 0, None) == 2  # K-stage sf misaligned
    assert L.moe_permute(p, 4, 8, 8, p, p, 192, p, p, 2, p, p, p, p, 1 << 20, None) == 3    # K % 128 != 0
    assert L.nvfp4_quantize(p, 4, 256, p, p, p, p, 3, None, 0, None) == 1   # unknown layout
    assert L.nvfp4_quantize_from_amax(None, 4, 32, None, None, None, None, 0, None) == 1
    assert L.nvfp4_quantize_from_amax(p, 4, 32, ctypes.c_void_p(18), p, p, p, 0, None) == 2  # amax word misaligned
    assert L.moe_grouped_gemm_nvfp4_amax(p, p, p, p, p, p, 1, 16, 256, 256, 0, p, ctypes.c_void_p(18), None) == 2


def test_layout_helpers_follow_the_header_definitions():
    # The host-side layout converters the GPU tests use, checked byte by byte against the index formulas the
    # header states (K-stage: ((b / 16) * rows + r) * 16 + b % 16; MMA-tiled: 512-byte atoms), on shapes with
    # several K steps and a row count that is not a multiple of anything.
    import numpy as np
    from tests.helpers import kstage_sf_to_rowmajor, rowmajor_sf_to_kstage, untile_sf
    rng = np.random.default_rng(0)
    rows, K = 37, 768
    rm = rng.integers(0, 256, size=(rows, K // 16), dtype=np.uint8)
    ks = rowmajor_sf_to_kstage(rm, rows, K)
    assert ks.shape == (K // 256, rows, 16)
    flat = ks.reshape(-1)
    for r in range(rows):
        for b in range(K // 16):
            assert flat[((b // 16) * rows + r) * 16 + b % 16] == rm[r, b]
    assert np.array_equal(kstage_sf_to_rowmajor(ks, rows, K), rm)
    sel = np.array([36, 0, 17])
    assert np.array_equal(kstage_sf_to_rowmajor(ks, rows, K, sel=sel), rm[sel])
    # K % 256 == 128: ceil(K/256) slabs, the last one's second 8 bytes of every row are zero scales
    K_h = 384
    rm_h = rng.integers(0, 256, size=(rows, K_h // 16), dtype=np.uint8)
    ks_h = rowmajor_sf_to_kstage(rm_h, rows, K_h)
    assert ks_h.shape == (2, rows, 16) and not ks_h[1, :, 8:].any()
    flat_h = ks_h.reshape(-1)
    for r in range(rows):
        for b in range(K_h // 16):
            assert flat_h[((b // 16) * rows + r) * 16 + b % 16] == rm_h[r, b]
    assert np.array_equal(kstage_sf_to_rowmajor(ks_h, rows, K_h), rm_h)
    rows_t, K_t = 256, 128
    rm_t = rng.integers(0, 256, size=(rows_t, K_t // 16), dtype=np.uint8)
    tiled = np.zeros(rows_t * K_t // 16, dtype=np.uint8)
    for r in range(rows_t):
        for b in range(K_t // 16):
            tiled[((r // 128) * (K_t // 64) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4] = rm_t[r, b]
    assert np.array_equal(untile_sf(tiled, rows_t, K_t), rm_t)


def test_binding_rejects_short_or_strided_buffers():
    # The library sees only pointers; the binding refuses caller buffers it would overrun (checked here on
    # host tensors: the same helper guards every caller-given output of the binding).
    import pytest
    import torch
    need = nv._need
    t = torch.empty((4, 8), dtype=torch.uint8)
    assert need(t, 32, "sf") is t
    with pytest.raises(ValueError):
        need(t, 33, "sf")
    with pytest.raises(ValueError):
        need(torch.empty((8, 8), dtype=torch.uint8)[:, ::2], 16, "sf")     # not contiguous
    with pytest.raises(TypeError):
        need(torch.empty(1, dtype=torch.float64), 4, "g", torch.float32)
    assert need(torch.empty((3, 5), dtype=torch.bfloat16), 30, "out", torch.bfloat16).numel() == 15


def test_layer_l2_prefetch_hints_follow_the_header_rule(L):
    # moe_layer_l2_prefetch_bytes: 96 MB of the gate/up and 48 MB of the down weights (or the whole tensor when
    # smaller) for batches under 32 rows per expert; nothing from 32 rows per expert on. Host arithmetic only.
    mb = 1 << 20
    assert nv.layer_l2_prefetch_bytes(512, 8, 256, 6144, 2048) == (96 * mb, 48 * mb)      # decode, 16 rows/expert
    assert nv.layer_l2_prefetch_bytes(1024, 8, 256, 6144, 2048) == (0, 0)                 # Zipf, 32 rows/expert
    assert nv.layer_l2_prefetch_bytes(8192, 8, 256, 6144, 2048) == (0, 0)                 # prefill
    # 4 experts, H = 256, I = 128: w13 = 4 * 256 * (128 + 16) bytes, w2 = 4 * 256 * (64 + 8) bytes
    assert nv.layer_l2_prefetch_bytes(4, 1, 4, 256, 128) == (4 * 256 * 144, 4 * 256 * 72)
    assert nv.layer_l2_prefetch_bytes(0, 8, 256, 6144, 2048) == (0, 0)


def test_prefetch_forms_reject_arguments_like_the_plain_calls(L):
    # the *_prefetch calls validate exactly as the plain ones, before any CUDA call; a hint is never required
    p = ctypes.c_void_p(16)
    assert L.nvfp4_quantize_from_amax_prefetch(None, 4, 32, None, None, None, None, 0, p, 1 << 20, None) == 1
    assert L.nvfp4_quantize_from_amax_prefetch(p, 4, 32, ctypes.c_void_p(18), p, p, p, 0, p, 64, None) == 2
    assert L.nvfp4_quantize_from_amax_prefetch(p, 4, 24, p, p, p, p, 0, None, 0, None) == 3     # K % 16 != 0
    assert L.moe_quantize_permute_prefetch(None, 4, 256, p, 2, 8, p, p, 2, p, p, p, p, p, 1 << 20, p, 64, None) == 1
    assert L.moe_quantize_permute_prefetch(p, 4, 192, p, 2, 8, p, p, 2, p, p, p, p, p, 1 << 20, None, 0, None) == 3
    assert L.moe_quantize_permute_prefetch(p, 4, 256, p, 2, 8, p, p, 2, p, p, p, p, None, 0, p, 64, None) == 4
    # an unaligned hint is refused before any CUDA call (bulk prefetches start on 16 bytes); without bytes it is ignored
    odd = ctypes.c_void_p(24)
    assert L.nvfp4_quantize_from_amax_prefetch(p, 4, 32, p, p, p, p, 0, odd, 64, None) == 2
    assert L.moe_quantize_permute_prefetch(p, 4, 256, p, 2, 8, p, p, 2, p, p, p, p, p, 1 << 20, odd, 64, None) == 2
