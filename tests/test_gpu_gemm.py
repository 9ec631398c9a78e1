"""moe_grouped_gemm_nvfp4 on the GPU against the oracle.

Teacher-forced: the oracle consumes the GPU's own quantised operands (whose
quantisation is itself checked bit-exact against the oracle), computes the
block-scaled dot products in FP64, and the BF16-rounded result is the
reference. Small cases are compared element by element; the full-size cases
(dense 8192^3, the decode layer's two GEMMs) on sampled outputs.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_09_b200 as nv
import oracle
import workloads
from tests.helpers import (compare_bf16, gpu_bf16, host, host_bits, kstage_sf_to_rowmajor, require_gpu,
                           unpack_weights)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def make_case(rows, N, K, seed, a_std=1.0, w_std=0.02, pad_rows=0):
    """Quantised activations [sum(rows) + pad_rows, K] and packed per-expert weights [E, N, K] on the GPU.
    The GEMM's max_rows is the activation row count, so padding rows changes the tile shape it picks."""
    E = len(rows)
    R = int(sum(rows))
    rows_a = max(R + pad_rows, 1)
    a_bits = workloads.random_bf16_bits((rows_a, K), seed=seed, std=a_std)
    a_q, a_sf, a_g = nv.quantize(gpu_bf16(a_bits), layout=nv.SF_KSTAGE)   # the GEMM's activation-scale layout
    w = workloads.normal_bf16((E, N, K), w_std, seed, workloads.TAG_W13, device="cuda")
    pw = nv.prepare_expert_weights(w, keep_rowmajor=True)
    off = np.concatenate([[0], np.cumsum(rows)]).astype(np.int32)
    torch.cuda.synchronize()
    # the GPU's operands are the oracle's operands: check their quantisation first
    oq, osf, og = oracle.quantize(a_bits)
    a_sf_rm = kstage_sf_to_rowmajor(host(a_sf), rows_a, K)
    assert np.array_equal(host(a_q), oq) and np.array_equal(a_sf_rm, osf) and host(a_g)[0] == og
    return dict(a_q=a_q, a_sf=a_sf, a_sf_rm=a_sf_rm, a_g=a_g, pw=pw, off=torch.from_numpy(off).cuda(), off_np=off,
                w=w, E=E, R=R, N=N, K=K)


def oracle_operands(c):
    """Host copies of the GPU's row-major weight codes / scales / global scales."""
    pw = c["pw"]
    return host(pw.q), host(pw.sf), host(pw.gscale)


def check_weights_quantised_and_packed(c, experts):
    pw = c["pw"]
    for e in experts:
        wq, wsf, wg = oracle.quantize(host_bits(c["w"][e]))
        assert np.array_equal(host(pw.q[e]), wq)
        assert np.array_equal(host(pw.sf[e]), wsf)
        assert host(pw.gscale)[e] == wg
        uq, usf = unpack_weights(host(pw.packed[e]), c["N"], c["K"])
        assert np.array_equal(uq, wq) and np.array_equal(usf, wsf)


def run_full(rows, N, K, swiglu, seed, pad_rows=0):
    c = make_case(rows, N, K, seed, pad_rows=pad_rows)
    amax = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = nv.grouped_gemm(c["a_q"], c["a_sf"], c["a_g"], c["pw"], c["off"], swiglu, amax_out=amax)
    assert nv.device_status() == 0
    # the side output is the max |BF16| over the stored rows only (BF16 bits), i.e. what the amax pass of
    # quantize() would find on out[:R]
    got_bits = host_bits(out)[: c["R"]]
    want = int((got_bits & 0x7FFF).max()) if got_bits.size else 0
    assert int(host(amax)[0]) == want
    check_weights_quantised_and_packed(c, range(min(c["E"], 3)))
    w_q, w_sf, w_g = oracle_operands(c)
    R = c["R"]
    ref = oracle.grouped_gemm(host(c["a_q"])[:R], c["a_sf_rm"][:R], host(c["a_g"])[0], w_q, w_sf, w_g,
                              c["off_np"], N, K, swiglu)
    band = oracle.grouped_gemm_bound(host(c["a_q"])[:R], c["a_sf_rm"][:R], host(c["a_g"])[0], w_q, w_sf, w_g,
                                     c["off_np"], N, K, swiglu)
    got = host_bits(out)[: c["R"]]
    return compare_bf16(got, oracle.bf16_round(ref), f"gemm rows={rows} N={N} K={K} swiglu={swiglu}", exact=ref,
                        band=band)


def test_tiny_config():
    # 4 experts x 16 rows, K = N = 256, plain epilogue
    stats = run_full([16, 16, 16, 16], 256, 256, False, seed=0)
    assert stats["exact_frac"] > 0.97


@pytest.mark.parametrize("swiglu", [False, True])
def test_ragged_experts_and_row_tiles(swiglu):
    # empty expert, 1 row, a partial 16-row step, exactly one 64-row tile, 64+1, several tiles
    run_full([0, 1, 17, 64, 65, 130], 512, 512, swiglu, seed=1)


@pytest.mark.parametrize("swiglu", [False, True])
def test_narrow_tiles_several_row_tiles(swiglu):
    # the same ragged experts plus empty ones, so that the mean stays below the wide-tile threshold and the
    # 64-row (narrow) tile shape takes experts of 65 and 130 rows in several row tiles
    rows = [0, 1, 17, 64, 65, 130, 0, 0, 0, 0]
    assert sum(rows) < nv.gemm_plan()["wide_min_avg_rows"] * len(rows)
    run_full(rows, 512, 512, swiglu, seed=12)


@pytest.mark.parametrize("swiglu", [False, True])
def test_wide_tiles_ragged(swiglu):
    # experts averaging >= 32 rows take the 128-row tile shape: empty, partial, exact, 128 + 1, several tiles
    run_full([0, 100, 128, 129, 300, 17], 512, 768, swiglu, seed=6)


@pytest.mark.parametrize("swiglu", [False, True])
def test_pair_tiles_ragged(swiglu):
    # experts averaging >= 192 rows run on CTA pairs (256 weight rows x up to 256 activation rows):
    # empty, partial, exact, 256 + 1, two tiles, a small expert
    run_full([0, 200, 256, 257, 500, 40], 512, 768, swiglu, seed=7)


@pytest.mark.parametrize("swiglu", [False, True])
@pytest.mark.parametrize("K", [512, 384])
def test_pair_tiles_tail_rows(swiglu, K):
    # an expert's rows past its last full 256-row tile ride on that tile when there are at most 32 of them
    # (a second MMA into accumulator columns 256-287): 256 (no tail), 257 / 272 / 288 (tails of 1, 16, 32),
    # 289 (a tile of its own), 512 + 1 and 512 + 32 (tail on the second tile), 545 (third tile), with
    # K % 256 == 128 (a last stage of two K-steps) as well
    rows = [256, 257, 272, 288, 289, 513, 544, 545]
    run_full(rows, 512, K, swiglu, seed=13)


@pytest.mark.parametrize("swiglu", [False, True])
def test_pair_tiles_small_ragged_experts(swiglu):
    # padding the activations to 192 rows per expert selects the CTA-pair kernel for experts of 1-33 rows:
    # one-row tiles, a 32-row tile (one full N step), 33 rows (two N steps), an empty expert
    plan = nv.gemm_plan()
    rows = [1, 0, 31, 32, 33, 7]
    pad = plan["pair_min_avg_rows"] * len(rows) - sum(rows)
    run_full(rows, 512, 512, swiglu, seed=8, pad_rows=pad)


@pytest.mark.parametrize("swiglu", [False, True])
def test_max_experts(swiglu):
    # E = 1024 (the largest the scheduler takes): 0-3 rows per expert, a third of them empty
    rng = np.random.default_rng(9)
    rows = [int(r) for r in rng.integers(0, 4, size=1024)]
    run_full(rows, 256, 256, swiglu, seed=9)


def test_max_experts_pair_tiles():
    # E = 1024 on the CTA-pair kernel (expert offsets and tile starts of all 1024 experts in shared memory)
    plan = nv.gemm_plan()
    rng = np.random.default_rng(10)
    rows = [int(r) for r in rng.integers(0, 40, size=1024)]
    run_full(rows, 256, 256, False, seed=10, pad_rows=plan["pair_min_avg_rows"] * 1024 - sum(rows))


@pytest.mark.parametrize("pad", [64, 600])   # narrow and CTA-pair tile shapes
def test_all_experts_empty_writes_nothing(pad):
    c = make_case([0, 0, 0], 256, 256, seed=11, pad_rows=pad)
    out = torch.full((pad, 256), 3.0, dtype=torch.bfloat16, device="cuda")
    amax = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.grouped_gemm(c["a_q"], c["a_sf"], c["a_g"], c["pw"], c["off"], False, out=out, amax_out=amax)
    assert nv.device_status() == 0
    assert torch.all(out == 3.0) and int(host(amax)[0]) == 0


@pytest.mark.parametrize("swiglu", [False, True])
def test_deeper_k_and_wider_n(swiglu):
    run_full([5, 40, 200], 768, 2048, swiglu, seed=2)


@pytest.mark.parametrize("N,K,swiglu", [(128, 128, False), (384, 384, False), (128, 640, False), (256, 128, True),
                                        (512, 384, True)])
def test_k_and_n_multiples_of_128(N, K, swiglu):
    # the boundary's smallest steps: K at its minimum 128, K % 256 == 128 (a last stage of 128 K-elements over
    # zero-padded weight tiles and scale slabs), and, for the plain epilogue, N % 256 == 128 (a last column
    # tile of one 128-row weight block); narrow tiles
    assert nv.can_implement(N, K, 6, swiglu) == 0
    run_full([0, 5, 16, 33, 64, 1], N, K, swiglu, seed=N + K)


@pytest.mark.parametrize("N,K,swiglu,pad", [(384, 384, False, 1200), (512, 384, True, 1200),
                                            (384, 128, False, 0)])
def test_k_and_n_multiples_of_128_wide_and_pair(N, K, swiglu, pad):
    # the same shapes on the wide one-SM tile (NONE with N % 256 == 128 stays on one SM even when the rows
    # per expert would pick CTA pairs) and on the CTA-pair kernel (SwiGLU, K % 256 == 128)
    run_full([0, 200, 256, 257, 40], N, K, swiglu, seed=N * K, pad_rows=pad)


def test_rows_outside_experts_untouched():
    c = make_case([10, 0, 20], 256, 256, seed=3)
    R = c["R"]
    out = torch.full((R + 8, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    # offsets cover only rows [0, 30); rows 30.. must keep their canary
    nv.grouped_gemm(c["a_q"], c["a_sf"], c["a_g"], c["pw"], c["off"], False, out=out)
    assert nv.device_status() == 0
    assert torch.all(out[R:] == 7.0)


def test_bad_offsets_latch_status_and_skip():
    c = make_case([16, 16], 256, 256, seed=4)
    bad = torch.tensor([0, 20, 10], dtype=torch.int32, device="cuda")   # decreasing
    nv.grouped_gemm(c["a_q"], c["a_sf"], c["a_g"], c["pw"], bad, False)
    assert nv.device_status() == 8


def sampled_check(a_q, a_sf, a_g, c_w, off_np, N, K, swiglu, out, experts, n_cols=64, seed=0):
    """Compare the GPU output against the oracle at every row of `experts` x n_cols random columns."""
    rng = np.random.default_rng(seed)
    nout = N // 2 if swiglu else N
    w_q, w_sf, w_g = c_w(experts)
    rows_l, cols_l, sub_off = [], [], [0]
    a_rows = []
    for i, e in enumerate(experts):
        r0, r1 = int(off_np[e]), int(off_np[e + 1])
        a_rows.extend(range(r0, r1))
        sub_off.append(sub_off[-1] + (r1 - r0))
    a_rows = np.array(a_rows, dtype=np.int64)
    cols = rng.choice(nout, size=min(n_cols, nout), replace=False)
    rr, cc = np.meshgrid(np.arange(a_rows.size), cols, indexing="ij")
    rr, cc = rr.ravel(), cc.ravel()
    aq = host(a_q)[a_rows]
    asf = kstage_sf_to_rowmajor(host(a_sf), a_q.shape[0], K, sel=a_rows)
    ref = oracle.grouped_gemm_at(aq, asf, float(host(a_g)[0]), w_q, w_sf, w_g, np.array(sub_off, np.int32), N, K,
                                 swiglu, rr, cc)
    band = oracle.grouped_gemm_bound(aq, asf, float(host(a_g)[0]), w_q, w_sf, w_g, np.array(sub_off, np.int32), N,
                                     K, swiglu, rr, cc)
    got = host_bits(out)[a_rows[rr], cc]
    return compare_bf16(got, oracle.bf16_round(ref), f"sampled N={N} K={K} swiglu={swiglu}", exact=ref, band=band)


def test_dense_8192_sampled():
    M = N = K = 8192
    a_bits_t = workloads.normal_bf16((M, K), 1.0, 0, workloads.TAG_A, device="cuda")
    a_q, a_sf, a_g = nv.quantize(a_bits_t, layout=nv.SF_KSTAGE)
    b = workloads.normal_bf16((1, N, K), 0.02, 0, workloads.TAG_B, device="cuda")
    pw = nv.prepare_expert_weights(b, keep_rowmajor=True)
    off = torch.tensor([0, M], dtype=torch.int32, device="cuda")
    out = nv.grouped_gemm(a_q, a_sf, a_g, pw, off, False)
    assert nv.device_status() == 0
    # quantisation of a sample of A rows against the oracle
    oq, osf, og = oracle.quantize(host_bits(a_bits_t[:256]), float(host(a_g)[0]))
    a_sf_rm = kstage_sf_to_rowmajor(host(a_sf), M, K)
    assert np.array_equal(host(a_q[:256]), oq) and np.array_equal(a_sf_rm[:256], osf)
    uq, usf = unpack_weights(host(pw.packed[0]), N, K)
    assert np.array_equal(uq, host(pw.q[0])) and np.array_equal(usf, host(pw.sf[0]))
    rng = np.random.default_rng(5)
    rows = np.sort(rng.choice(M, size=48, replace=False))
    cols = rng.choice(N, size=48, replace=False)
    rr, cc = np.meshgrid(rows, cols, indexing="ij")
    rr, cc = rr.ravel(), cc.ravel()
    ref = oracle.grouped_gemm_at(host(a_q), a_sf_rm, float(host(a_g)[0]), host(pw.q), host(pw.sf),
                                 host(pw.gscale), np.array([0, M], np.int32), N, K, False, rr, cc)
    band = oracle.grouped_gemm_bound(host(a_q), a_sf_rm, float(host(a_g)[0]), host(pw.q), host(pw.sf),
                                     host(pw.gscale), np.array([0, M], np.int32), N, K, False, rr, cc)
    compare_bf16(host_bits(out)[rr, cc], oracle.bf16_round(ref), "dense 8192", exact=ref, band=band)


def build_layer_weights(E, N, K, tag, keep):
    """Packed weights of a full-size layer, generated and packed expert by expert; row-major copies (host)
    are kept for the experts in `keep`."""
    packed = torch.empty((E, N * (K // 2 + K // 16)), dtype=torch.uint8, device="cuda")
    g = torch.empty(E, dtype=torch.float32, device="cuda")
    qt = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    st = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    kept = {}
    for e in range(E):
        w = workloads.normal_bf16((N, K), 0.02, 0, tag, e, device="cuda")
        nv.quantize(w, q=qt, sf=st, g=g[e:e + 1])
        nv.pack_weights(qt, st, out=packed[e])
        if e in keep:
            kept[e] = (host_bits(w), host(qt), host(st))
    return nv.PackedWeights(packed, g, E, N, K), kept


@pytest.mark.parametrize("name", ["moe_decode_t512", "moe_zipf_t1024", "moe_prefill_t8192"])
def test_moe_layer_gemms_full_size_sampled(name):
    cfg = workloads.CONFIGS[name]
    T, H, I, E, k = cfg["T"], cfg["H"], cfg["I"], cfg["E"], cfg["k"]
    ids, _ = workloads.config_routing(name)
    off_np, src, _ = oracle.permute(ids, E)
    R = T * k
    counts = np.diff(off_np)
    experts = [int(np.argmax(counts)), int(np.argmin(np.where(counts > 0, counts, 1 << 30))), 0, E - 1]
    experts = sorted(set(e for e in experts if counts[e] > 0))
    # activations already in expert order (permute is tested on its own)
    a = workloads.normal_bf16((R, H), 1.0, 0, workloads.TAG_X, device="cuda")
    a_q, a_sf, a_g = nv.quantize(a, layout=nv.SF_KSTAGE)
    w13, kept13 = build_layer_weights(E, 2 * I, H, workloads.TAG_W13, set(experts))
    off = torch.from_numpy(off_np).cuda()
    h = nv.grouped_gemm(a_q, a_sf, a_g, w13, off, True)
    assert nv.device_status() == 0
    for e in experts[:2]:
        wq, wsf, wg = oracle.quantize(kept13[e][0])
        assert np.array_equal(kept13[e][1], wq) and np.array_equal(kept13[e][2], wsf)
        uq, usf = unpack_weights(host(w13.packed[e]), 2 * I, H)
        assert np.array_equal(uq, wq) and np.array_equal(usf, wsf)

    def host_w(kept, gs):
        return lambda sel: (np.stack([kept[e][1] for e in sel]), np.stack([kept[e][2] for e in sel]),
                            host(gs)[sel])

    sampled_check(a_q, a_sf, a_g, host_w(kept13, w13.gscale), off_np, 2 * I, H, True, h, experts, n_cols=32)

    # down projection on the GPU's own h
    hq, hsf, hg = nv.quantize(h, layout=nv.SF_KSTAGE)
    w2, kept2 = build_layer_weights(E, H, I, workloads.TAG_W2, set(experts))
    y = nv.grouped_gemm(hq, hsf, hg, w2, off, False)
    assert nv.device_status() == 0
    sampled_check(hq, hsf, hg, host_w(kept2, w2.gscale), off_np, H, I, False, y, experts, n_cols=32, seed=1)
