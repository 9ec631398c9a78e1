// grouped_gemm_pair.cu -- the grouped NVFP4 GEMM on CTA pairs (tcgen05
// cta_group::2) for experts with many rows (prefill) and dense GEMMs.
//
// Same computation as grouped_gemm.cu. A cluster of two CTAs on neighbouring
// SMs shares one tile of 256 weight rows x up to 256 activation rows: each CTA
// loads its own 128 weight rows and half of the activation rows, and the even
// CTA issues M = 256 MMAs that read both CTAs' shared memory. Per SM this
// halves the bytes moved per FLOP against a one-SM 256 x 128 tile (each SM
// fetches 128 + 128 rows per K step for a 128 x 256 output), and the N = 256
// MMA runs ~30% faster per FLOP than two N = 128 ones -- the two limits
// (L2 -> SM traffic, MMA time) of the one-SM wide tile on prefill and dense.
//
// SwiGLU: CTA r covers output columns [n0 + 64r, +64). Its 128 A rows interleave
// the gate and up rows 16 at a time (lanes 32q..32q+15: gate rows n0+64r+16q+j,
// lanes 32q+16..32q+31: the matching up rows), so one warp reads both halves of
// its 16 output columns and pairs them with a lane shuffle.
//
// One accumulator per CTA (256 columns, plus 32 for the rows past an expert's
// last full tile that ride on it in the configuration with row tails; the scale
// ring takes the rest of tensor memory), so the epilogue warps first drain it
// into registers as final BF16 values and hand it back to the MMA warp; staging
// and storing those values then overlaps the next tile's main loop. Three
// configurations (Cfg below): row tails, 5 stages and a 3-slot scale ring for up
// to 256 experts (4 stages beyond); 5 stages and a scale slot per stage for one
// expert.
//
// The kernel is a template on the epilogue mode, the configuration and SwiGLU or plain output, so each
// instantiation carries only its own epilogue (measured on B200: a runtime SwiGLU switch cost 1-4% on
// the prefill GEMMs).
//
// The peer's scale-writer and epilogue warps arrive on the even CTA's barriers
// through cluster addresses (mapa); the even CTA's MMA completions reach both
// CTAs' barriers through one commit with a CTA mask (no data moves by multicast;
// measured 1-3% faster than a commit per CTA).
// Work items come from a grid-wide counter (dynamic schedule); the even CTA
// takes each one and writes it into both CTAs' work-item rings. Every wait is
// bounded as in the one-SM kernel; a cluster barrier guards the release of
// tensor memory.
#include <mutex>

#include "common.cuh"



namespace nvfp4 {
namespace gp {
// max |x| over the n BF16 pairs of a chunk, as BF16 bits, counting only the halves whose token is below
// nrows: word i holds tokens stride * i + off (low half) and stride * i + off + stride / 2 (high half)
__device__ __forceinline__ uint32_t absmax_bf16x2(const uint32_t* pk, int n, int nrows, int stride, int off) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < n; i++) {
        const int lo = stride * i + off;
        const uint32_t mask = (lo < nrows ? 0x7FFFu : 0u) | (lo + stride / 2 < nrows ? 0x7FFF0000u : 0u);
        m = __vmaxu2(m, pk[i] & mask);
    }
    return max(m & 0xFFFFu, m >> 16);
}


constexpr int kBM = 128;                          // weight rows per CTA (MMA M = 256 per pair)
constexpr int kBK = 256;                          // K elements per stage
constexpr int kRowBytes = kBK / 2;
constexpr int kKSteps = kBK / 64;
constexpr int kBNMax = 256;                       // activation rows per pair tile (MMA N)
constexpr int kBNStep = 32;                       // N granularity: each CTA holds a multiple of 16 rows
constexpr int kBoxRows = 16;                      // activation TMA box rows
constexpr int kPackedTileBytes = 18432;           // packed weight tile: 16 KB codes + 2 KB scales
constexpr int kCodeBytes = 16384;
constexpr int kTileSFBytes = 2048;
constexpr int kOffA = 0;                          // 128 weight rows x 128 B (SwiGLU: gate/up slabs of 16 rows, interleaved)
constexpr int kOffSFA = kCodeBytes;               // scales of one packed tile (SwiGLU: gate tile's, then up tile's)
constexpr int kThreads = 512;                     // warps: 0 loads, 2 MMA, 4-7 + 12-15 epilogue, 8-11 scales
constexpr int kEpiWarps = 8;                      // two per TMEM lane quadrant, alternating 32-token chunks
constexpr int kChunksPerWarp = kBNMax / 32 / 2;   // 32-token chunks one epilogue warp drains per tile
                                                  // (plus the tail chunk, columns 256-287, on warps 4-7)
constexpr uint32_t kTmemCols = 512;

constexpr int kTileRing = 4;                      // work items the even CTA may publish ahead
constexpr int kTileConsumersPerCta = 13;          // even CTA: MMA warp + 4 scale writers + 8 epilogue warps;
                                                  // odd CTA: its producer + 4 scale writers + 8 epilogue warps
constexpr int kTileConsumers = 2 * kTileConsumersPerCta;

template <int kStagesT, int kTailT, int kMaxET, int kStgElemsT, int kFinTokT>
struct SharedT {
    alignas(16) uint16_t ostage[kEpiWarps][kStgElemsT];  // epilogue: one 32-token chunk of BF16 outputs per warp
    uint64_t tq_full[kTileRing];  // the even CTA published tq[i] (in this CTA's copy of the ring)
    uint64_t tq_empty[kTileRing]; // even CTA: every consumer warp of both CTAs read entry i
    int32_t tq[kTileRing];        // work item index (>= total: no more work)
    uint64_t full_tma[kStagesT];  // this CTA's loads of the stage landed
    uint64_t sf_ready[kStagesT];  // even CTA: both CTAs' scales are in TMEM (8 warp arrivals)
    uint64_t empty[kStagesT];     // the pair's MMAs of the stage completed (commit from the even CTA)
    uint64_t acc_full;            // the pair's MMAs of the tile completed
    uint64_t acc_empty;           // even CTA: both CTAs' epilogues drained TMEM (2 x kEpiWarps arrivals)
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int32_t total_tiles;
    int32_t off[kMaxET + 1];
    int32_t tile_start[kMaxET + 1];
    int32_t fin_tok[kFinTokT];    // fused combine: tokens of this tile whose last row this CTA wrote
    uint64_t fin_bar;             // fused combine: this CTA's 8 epilogue warps meet (bounded waits)
};

// Three configurations of the kernel, chosen per launch (kConf):
// 0 (one expert, dense): 5 stages, one TMEM scale slot per stage.
// 1, 2 (grouped GEMMs): an expert's rows past its last full 256-row tile ride on that tile when there are at
//   most kTailMax = 32 of them (a second MMA of N = 32 into accumulator columns 256-287) instead of taking a tile
//   of their own, which would stream the whole weight tile again for a few rows. The tail's accumulator columns
//   leave TMEM room for a ring of 3 scale slots (a slot is written just before its MMAs, so it needs fewer slots
//   than there are stages). Configuration 2 (up to 256 experts) holds 5 data stages: its scheduler tables are
//   sized for 256 experts, and a SwiGLU tile's staging chunk is half a plain one's. Configuration 1 (up to
//   1024 experts) holds 4. Measured on B200 (prefill, same box): 3 data stages against 4 cost 8% (gate/up) and
//   6% (down).
// The scales of the weight tile take 4 KB of a stage with SwiGLU (the gate and the up tile's) and 2 KB without.
template <int kConf, bool kSw, bool kFin>
struct Cfg {
    static constexpr bool kTails = kConf != 0;
    static constexpr int kTailMax = kTails ? 32 : 0;
    static constexpr int kStages = kConf == 1 ? 4 : 5;
    static constexpr int kMaxE = kConf == 2 ? 256 : 1024;        // experts the scheduler tables hold
    static constexpr int kOffB = kOffSFA + (kSw ? 2 : 1) * kTileSFBytes;  // this CTA's half of the activation rows
    static constexpr int kOffBT = kOffB + (kBNMax / 2) * kRowBytes;       // this CTA's half of the tail rows
    static constexpr int kOffSFB = kOffBT + (kTailMax / 2) * kRowBytes;   // scales of all the tile's rows, 16 B each
    static constexpr int kStageBytes = (kOffSFB + (kBNMax + kTailMax) * 16 + 1023) / 1024 * 1024;
    static constexpr uint32_t kAccCols = kBNMax + kTailMax;    // one accumulator per CTA (+ the tail's columns)
    // TMEM scale slot: SFA 4 columns per K step, SFB 8 (256 rows), tail SFB 4 (one used)
    static constexpr int kSFSlots = kTails ? 3 : kStages;
    static constexpr uint32_t kSFSlot = (kTails ? 16 : 12) * kKSteps;
    static constexpr uint32_t kSFTail = 12 * kKSteps;          // tail SFB of K step kc at slot + kSFTail + 4 kc
    static constexpr uint32_t kTmemSFRing = kAccCols;
    // a staged chunk: 32 tokens x 16 (SwiGLU) or 32 output columns
    using Shared = SharedT<kStages, kTailMax, kMaxE, 32 * (kSw ? 16 : 32), kFin ? kBNMax + kTailMax : 1>;
    static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStageBytes + sizeof(Shared);
    static_assert(kTmemSFRing + kSFSlots * kSFSlot <= kTmemCols, "TMEM budget");
    static_assert(kStageBytes % 1024 == 0 && kOffB % 1024 == 0 && kOffBT % 1024 == 0,
                  "swizzled tiles need 1024-byte alignment");
    static_assert(kSmemBytes + 256 <= 232448, "shared memory budget");
};

struct Params {
    const uint8_t* a_sf;
    const float* a_gscale;
    const uint8_t* w_packed;
    const float* w_gscale;
    const int32_t* offsets;
    uint16_t* out;
    int32_t E;
    int64_t max_rows;
    int64_t N;
    int64_t K;
    int32_t swiglu;
    uint32_t* amax_out;   // nullable: raised to max |out| (BF16 bits)
    uint32_t* sched;      // this launch's work counter [0] and finished-CTA counter [1]; zero at launch
    DeviceCtl ctl;
    Finalize fin;         // fused top-k combine (NONE epilogue), off when fin.out == nullptr
    QuantOut qo;          // quantised h (SWIGLU epilogue), off when qo.q == nullptr
};

struct Tile {
    int32_t e, nt, mt, row0, rows, bn, tail;   // rows = bn-covered rows + tail rows (columns 256..287)
};

// Row tiles of an expert with M rows: 256 rows each, except that a remainder of at most kTailMax rows
// rides on the last full tile (a second MMA of N = 32 into accumulator columns 256-287) instead of
// taking a tile of its own, which would stream the whole weight tile again for a few rows.
template <int kTail>
__device__ __forceinline__ int32_t row_tiles(int32_t M) {
    const int32_t full = M / kBNMax, rem = M - full * kBNMax;
    return full + ((rem > kTail || (full == 0 && rem > 0)) ? 1 : 0);
}

template <int kTail, class S>
__device__ __forceinline__ void decode_tile(const S& sh, int32_t E, int32_t w, Tile& t) {
    int32_t lo = 0, hi = E;  // tile_start[lo] <= w < tile_start[hi]
    while (hi - lo > 1) {
        const int32_t mid = (lo + hi) >> 1;
        if (sh.tile_start[mid] <= w) lo = mid;
        else hi = mid;
    }
    const int32_t M = sh.off[lo + 1] - sh.off[lo];
    const int32_t mtiles = row_tiles<kTail>(M);
    const int32_t local = w - sh.tile_start[lo];
    t.e = lo;
    t.nt = local / mtiles;
    t.mt = local - t.nt * mtiles;
    t.row0 = sh.off[lo] + t.mt * kBNMax;
    t.rows = t.mt == mtiles - 1 ? M - t.mt * kBNMax : kBNMax;
    const int32_t main_rows = min(t.rows, kBNMax);
    t.bn = (main_rows + kBNStep - 1) / kBNStep * kBNStep;
    t.tail = t.rows - main_rows;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, const DeviceCtl& ctl) {
    bool ok = mbar_wait_bounded(bar, parity, abort, ctl);
    return __all_sync(0xFFFFFFFFu, ok);
}

// Arrive on barrier `bar` of the even CTA (locally when this is the even CTA).
__device__ __forceinline__ void arrive_on_leader(uint64_t* bar, uint32_t rank) {
    if (rank == 0) mbar_arrive(bar);
    else mbar_arrive_cluster(cluster_smem_addr(bar, 0));
}

// ---- the pair's work-item ring -------------------------------------------------------------------
// The even CTA's producer takes each work item from the launch's counter and writes it into both CTAs'
// copies of the ring (the odd CTA's through distributed shared memory, released at cluster scope); every
// consumer warp of both CTAs reports on the even CTA's tq_empty once it has read an entry.
template <class S>
__device__ __forceinline__ bool tq_wait(S& sh, uint32_t qi, uint32_t qphase, uint32_t rank, volatile int* abort,
                                        const DeviceCtl& ctl) {
    return rank == 0 ? mbar_wait_bounded(&sh.tq_full[qi], qphase, abort, ctl)
                     : mbar_wait_bounded_acq_cluster(&sh.tq_full[qi], qphase, abort, ctl);
}
template <class S>
__device__ __forceinline__ void tq_release(S& sh, uint32_t qi, uint32_t rank) {
    if (rank == 0) mbar_arrive(&sh.tq_empty[qi]);
    else mbar_arrive_release_cluster(cluster_smem_addr(&sh.tq_empty[qi], 0));
}
// Next work item for a whole consumer warp. False when a wait ran out.
template <class S>
__device__ __forceinline__ bool next_tile_warp(S& sh, uint32_t rank, uint32_t& qi, uint32_t& qphase, int32_t& w,
                                               int lane, volatile int* abort, const DeviceCtl& ctl) {
    const bool ok = __all_sync(0xFFFFFFFFu, tq_wait(sh, qi, qphase, rank, abort, ctl));
    if (!ok) return false;
    w = *reinterpret_cast<volatile int32_t*>(&sh.tq[qi]);
    __syncwarp();
    if (lane == 0) tq_release(sh, qi, rank);
    if (++qi == kTileRing) { qi = 0; qphase ^= 1u; }
    return true;
}
// Next work item for one thread (the odd CTA's producer).
template <class S>
__device__ __forceinline__ bool next_tile_thread(S& sh, uint32_t rank, uint32_t& qi, uint32_t& qphase,
                                                 int32_t& w, volatile int* abort, const DeviceCtl& ctl) {
    if (!tq_wait(sh, qi, qphase, rank, abort, ctl)) return false;
    w = *reinterpret_cast<volatile int32_t*>(&sh.tq[qi]);
    tq_release(sh, qi, rank);
    if (++qi == kTileRing) { qi = 0; qphase ^= 1u; }
    return true;
}
// The even CTA's producer: take the next work item of the grid and publish it to both CTAs.
template <class S>
__device__ __forceinline__ bool publish_tile(S& sh, const Params& p, int32_t total, uint32_t& qi,
                                             uint32_t& qphase, int32_t& w, volatile int* abort) {
    w = (int32_t)min(atomicAdd(p.sched, 1u), (uint32_t)total);
    if (!mbar_wait_bounded_acq_cluster(&sh.tq_empty[qi], qphase ^ 1u, abort, p.ctl)) return false;
    *reinterpret_cast<volatile int32_t*>(&sh.tq[qi]) = w;
    st_shared_cluster_u32(cluster_smem_addr(&sh.tq[qi], 1), (uint32_t)w);
    mbar_arrive(&sh.tq_full[qi]);
    mbar_arrive_release_cluster(cluster_smem_addr(&sh.tq_full[qi], 1));   // orders the store above
    if (++qi == kTileRing) { qi = 0; qphase ^= 1u; }
    return true;
}

// Packed weight tiles of work item t at K step 0 for CTA `rank`: NONE: g = this CTA's 128 rows, u = the
// other CTA's; SWIGLU: g = the gate tile, u = the up tile of the item's 128 output columns (both CTAs).
__device__ __forceinline__ void weight_tiles(const Params& p, const Tile& t, uint32_t rank, int32_t ksteps,
                                             const uint8_t*& g, const uint8_t*& u) {
    const int64_t tile_stride = (int64_t)ksteps * kPackedTileBytes;
    if (p.swiglu) {
        const int64_t gate_base = (int64_t)t.e * p.N + (int64_t)t.nt * kBM;
        g = p.w_packed + (gate_base / kBM) * tile_stride;
        u = p.w_packed + ((gate_base + p.N / 2) / kBM) * tile_stride;
    } else {
        const int64_t base = (int64_t)t.e * p.N + (int64_t)t.nt * 2 * kBM;
        g = p.w_packed + (base / kBM + rank) * tile_stride;
        u = p.w_packed + (base / kBM + (rank ^ 1u)) * tile_stride;
    }
}

// Expert offsets and the first work item of each expert (every CTA builds its own copy).
template <int kTail, class S>
__device__ __forceinline__ void build_schedule(S& sh, const Params& p, int32_t n_col_tiles) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int32_t E = p.E;
    const int e0 = tid * 4;
    int32_t cnt[4];
    int32_t local = 0;
    bool bad = false;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int e = e0 + i;
        cnt[i] = 0;
        if (e < E) {
            const int32_t a = sh.off[e], b = sh.off[e + 1];
            if (a < 0 || b < a || (int64_t)b > p.max_rows) bad = true;  // inconsistent offsets: skip the expert
            else cnt[i] = row_tiles<kTail>(b - a) * n_col_tiles;
        }
        local += cnt[i];
    }
    if (bad) atomicOr(p.ctl.status, kStatusBadInput);
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    __shared__ int32_t warp_tot[kThreads / 32];
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int32_t before = 0;
    for (int w2 = 0; w2 < warp; w2++) before += warp_tot[w2];
    int32_t run = before + incl - local;
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int e = e0 + i;
        if (e < E) sh.tile_start[e] = run;
        run += cnt[i];
    }
    if (tid == kThreads - 1) {
        sh.total_tiles = before + incl;
        sh.tile_start[E] = before + incl;
    }
}

}  // namespace gp
}  // namespace nvfp4

namespace nvfp4 {
namespace gp {

template <int kEpi, int kConf, bool kSw>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a_full,
                             const __grid_constant__ CUtensorMap tm_out, const __grid_constant__ CUtensorMap tm_wsw,
                             const __grid_constant__ CUtensorMap tm_wsf, const Params p) {
    using C = Cfg<kConf, kSw, kEpi == kEpiFinalize>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    typename C::Shared& sh = *reinterpret_cast<typename C::Shared*>(smem + (size_t)C::kStages * C::kStageBytes);
    volatile int* abort = &sh.abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int32_t E = p.E;
    const int32_t n_col_tiles = (int32_t)(kSw ? (p.N / 2) / kBM : p.N / (2 * kBM));
    // K % 256 == 128: the last stage holds 128 K-elements (2 MMA K-steps); weights and activation scales
    // are zero-padded there, and the activation tile's second half is outside the tensor (zero-filled)
    const int32_t ksteps_total = (int32_t)((p.K + kBK - 1) / kBK);
    const int last_ksteps = (p.K % kBK) ? (int)((p.K % kBK) / 64) : kKSteps;

    if (tid == 0) {
        prefetch_tensormap(&tm_a);
        prefetch_tensormap(&tm_a_full);
        prefetch_tensormap(&tm_out);
        if (kSw) {
            prefetch_tensormap(&tm_wsw);
            prefetch_tensormap(&tm_wsf);
        }
        sh.abort = 0;
        for (int s = 0; s < C::kStages; s++) {
            mbar_init(&sh.full_tma[s], 1);
            mbar_init(&sh.sf_ready[s], 8);
            mbar_init(&sh.empty[s], 1);
        }
        mbar_init(&sh.acc_full, 1);
        mbar_init(&sh.acc_empty, 2 * kEpiWarps);
        mbar_init(&sh.drain, 1);
        mbar_init(&sh.fin_bar, kEpiWarps);
        for (int i = 0; i < kTileRing; i++) {
            mbar_init(&sh.tq_full[i], 1);
            mbar_init(&sh.tq_empty[i], kTileConsumers);
        }
        fence_barrier_init();
    }
    // everything above overlaps the previous kernel; global memory only from here on
    pdl_launch_dependents();
    pdl_wait();
    if (E > C::kMaxE) {   // the launcher picks a configuration whose tables hold E; never taken
        if (tid == 0) atomicOr(p.ctl.status, kStatusBadInput);
        return;
    }
    for (int i = tid; i <= E; i += kThreads) sh.off[i] = __ldg(p.offsets + i);
    __syncthreads();
    build_schedule<C::kTailMax>(sh, p, n_col_tiles);
    if (warp == 2) {
        tmem_alloc_pair(&sh.tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // both CTAs' barriers exist before any cross-CTA arrival
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;
    const int32_t total = sh.total_tiles;

    if (warp == 0) {
        // ================= loads of this CTA's halves =================
        uint32_t issued_parity[C::kStages];
        bool issued[C::kStages];
#pragma unroll
        for (int s = 0; s < C::kStages; s++) issued[s] = false, issued_parity[s] = 0;
        if (lane == 0 && !(p.ctl.flags & kCtlStallProducer)) {
            // L2: an expert's activation rows are re-read by each of its column tiles and stay hot on
            // their own; a weight tile is re-read only by the expert's other row tiles, which run
            // alongside (row tile fastest), so it is streamed evict-first when the expert has one
            const uint64_t pol_w_once = l2_policy_evict_first();
            const uint64_t pol_w_reuse = l2_policy_evict_normal();
            const uint64_t pol_a = l2_policy_evict_normal();
            uint32_t stage = 0, phase = 0, qi = 0, qphase = 0;
            // dynamic schedule: work items in increasing order (row tiles of one weight tile side by side).
            // The even CTA publishes the item after the current one before the current one's loads, so
            // the counter's round trip and the cross-CTA publication overlap the MMAs.
            int32_t w = total, w_next = total;
            bool ok;
            if (rank == 0) {
                ok = publish_tile(sh, p, total, qi, qphase, w, abort);
                if (ok && w < total) ok = publish_tile(sh, p, total, qi, qphase, w_next, abort);
            } else {
                ok = next_tile_thread(sh, rank, qi, qphase, w, abort, p.ctl);
            }
            while (ok && w < total) {
                Tile t;
                decode_tile<C::kTailMax>(sh, E, w, t);
                const uint64_t pol_w = row_tiles<C::kTailMax>(sh.off[t.e + 1] - sh.off[t.e]) > 1 ? pol_w_reuse : pol_w_once;
                // weight rows of this CTA, as (packed tile base, byte offset of the first row's codes)
                const uint8_t* g_tile;   // NONE: this CTA's 128-row tile; SWIGLU: the gate tile
                const uint8_t* u_tile;   // NONE: the other CTA's tile; SWIGLU: the up tile
                weight_tiles(p, t, rank, ksteps_total, g_tile, u_tile);
                const uint32_t half = kSw ? rank * 64 : 0;
                const int32_t sw_tile0 = (int32_t)((g_tile - p.w_packed) / kPackedTileBytes);  // SWIGLU: gate tile index at K step 0
                const int32_t my_rows = t.bn / 2;
                const int32_t my_row0 = t.row0 + (int32_t)rank * my_rows;
                // SWIGLU: 16 KB of interleaved gate/up codes + both tiles' 2 KB of scales; NONE: one packed tile
                const uint32_t a_bytes = kSw ? (uint32_t)kCodeBytes + 2u * kTileSFBytes : (uint32_t)kPackedTileBytes;
                // both CTAs stage the scales of all the tile's rows: one contiguous run of the K step's
                // slab (K-stage layout), 16 bytes per row
                // (+ this CTA's 16 tail rows when the tile has a tail)
                const uint32_t tx = a_bytes + (uint32_t)my_rows * kRowBytes +
                                    (C::kTailMax > 0 && t.tail > 0 ? (C::kTailMax / 2) * kRowBytes : 0u) +
                                    (uint32_t)t.rows * 16u;
                const uint8_t* sfb = p.a_sf + (int64_t)t.row0 * 16;
                for (int32_t kt = 0; kt < ksteps_total; kt++) {
                    if (!mbar_wait_bounded(&sh.empty[stage], phase ^ 1u, abort, p.ctl)) { ok = false; break; }
                    uint8_t* sb = stages + (size_t)stage * C::kStageBytes;
                    uint64_t* bar = &sh.full_tma[stage];
                    mbar_arrive_expect_tx(bar, tx);
                    const size_t ko = (size_t)kt * kPackedTileBytes;
                    if (kSw) {
                        // 16-row slabs (2 KB, whole swizzle atoms) of this CTA's half: gate slab q -> A rows
                        // 32q.., up slab q -> 32q+16.. (one box: bytes x rows x gate/up x slab x tile)
                        tma_load_5d(sb + kOffA, &tm_wsw, 0, 0, 0, (int32_t)(half / 16), sw_tile0 + kt, bar, pol_w);
                        // both tiles' 2 KB of scales (slab 8 of each tile's view): one load instead of two
                        // (measured: ~2% on the prefill gate/up GEMM)
                        tma_load_5d(sb + kOffSFA, &tm_wsf, 0, 0, 0, 8, sw_tile0 + kt, bar, pol_w);
                    } else {
                        bulk_load(sb + kOffA, g_tile + ko, kPackedTileBytes, bar, pol_w);   // codes + scales
                    }
                    if (my_rows == kBNMax / 2) {
                        tma_load_2d(sb + C::kOffB, &tm_a_full, kt * kRowBytes, my_row0, bar, pol_a);
                    } else {
                        for (int32_t i = 0; i < my_rows / kBoxRows; i++)
                            tma_load_2d(sb + C::kOffB + i * kBoxRows * kRowBytes, &tm_a, kt * kRowBytes,
                                        my_row0 + i * kBoxRows, bar, pol_a);
                    }
                    if (C::kTailMax > 0 && t.tail > 0)
                        tma_load_2d(sb + C::kOffBT, &tm_a, kt * kRowBytes, t.row0 + kBNMax + (int32_t)rank * (C::kTailMax / 2),
                                    bar, pol_a);
                    bulk_load(sb + C::kOffSFB, sfb + (int64_t)kt * p.max_rows * 16, (uint32_t)t.rows * 16u, bar, pol_a);
                    issued[stage] = true;
                    issued_parity[stage] = phase;
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                if (rank == 0) {
                    w = w_next;
                    if (w < total) ok = publish_tile(sh, p, total, qi, qphase, w_next, abort);
                } else {
                    ok = next_tile_thread(sh, rank, qi, qphase, w, abort, p.ctl);
                }
            }
            if (!ok || *abort) {
                for (int s = 0; s < C::kStages; s++)
                    if (issued[s]) mbar_wait_drain(&sh.full_tma[s], issued_parity[s], 200000000ull);
            }
        }
        __syncwarp();
    } else if (warp >= 8 && warp < 12) {
        // ================= scale writers (one per TMEM lane quadrant) =================
        // SFA: the weight row of lane m at column slot + 4 kc + m/32. SFB: activation row n (all
        // kBNMax rows, both CTAs) at lane n % 32 of every quadrant, column slot + 16 + 8 kc + n/32.
        const int quad = warp & 3;
        const uint32_t lane_addr = (uint32_t)(quad * 32) << 16;
        // row of this lane inside its packed tile, and that tile's scale atom in the stage
        const int tile_row = kSw ? (int)rank * 64 + quad * 16 + (lane & 15) : quad * 32 + lane;
        const uint32_t sfa_off = kOffSFA + ((kSw && lane >= 16) ? kTileSFBytes : 0) + (tile_row & 31) * 16 +
                                 (tile_row >> 5) * 4;
        uint32_t stage = 0, phase = 0, qi = 0, qphase = 0, sfs = 0;
        uint32_t count = 0;   // stages handled so far
        bool ok = true;
        while (ok) {
            int32_t w;
            if (!next_tile_warp(sh, rank, qi, qphase, w, lane, abort, p.ctl) || w >= total) break;
            Tile t;
            decode_tile<C::kTailMax>(sh, E, w, t);
            for (int32_t kt = 0; kt < ksteps_total; kt++) {
                if (!warp_wait(&sh.full_tma[stage], phase, abort, p.ctl)) { ok = false; break; }
                // this stage's scales into registers first (SFA: the word of this lane's row per K step; SFB:
                // rows 32 g + lane, 16 bytes each; the tail rows 256 + lane)
                const uint8_t* sb = stages + (size_t)stage * C::kStageBytes;
                uint32_t sfa[kKSteps], v32[32];
                uint4 xt = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                for (int kc = 0; kc < kKSteps; kc++) sfa[kc] = *reinterpret_cast<const uint32_t*>(sb + sfa_off + kc * 512);
#pragma unroll
                for (int g = 0; g < 8; g++) {
                    const uint4 x = *reinterpret_cast<const uint4*>(sb + C::kOffSFB + (32 * g + lane) * 16);
                    v32[g] = x.x;
                    v32[8 + g] = x.y;
                    v32[16 + g] = x.z;
                    v32[24 + g] = x.w;
                }
                const bool tail = C::kTailMax > 0 && t.tail > 0;
                if (tail) xt = *reinterpret_cast<const uint4*>(sb + C::kOffSFB + (kBNMax + lane) * 16);
                // the TMEM slot's previous stage (kSFSlots back) has had its MMAs completed
                if (C::kSFSlots < C::kStages && count >= (uint32_t)C::kSFSlots) {
                    const uint32_t c0 = count - C::kSFSlots;
                    if (!warp_wait(&sh.empty[c0 % C::kStages], (c0 / C::kStages) & 1u, abort, p.ctl)) { ok = false; break; }
                }
                tc_fence_after();
                const uint32_t slot = tmem + lane_addr + C::kTmemSFRing + sfs * C::kSFSlot;
                // SFA: one column per K-step, the one this quadrant's rows are read from (the other three
                // columns of the step belong to the other quadrants; measured: 1% faster than writing all four)
#pragma unroll
                for (int kc = 0; kc < kKSteps; kc++) tmem_st_32x32b_x1(slot + 4 * kc + quad, sfa[kc]);
                tmem_st_32x32b_x32(slot + 16, v32);
                if (tail) {
                    // tail SFB: tail row 256 + r at lane r of every quadrant, one column per K step
                    tmem_st_32x32b_x1(slot + C::kSFTail, xt.x);
                    tmem_st_32x32b_x1(slot + C::kSFTail + 4, xt.y);
                    tmem_st_32x32b_x1(slot + C::kSFTail + 8, xt.z);
                    tmem_st_32x32b_x1(slot + C::kSFTail + 12, xt.w);
                }
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_on_leader(&sh.sf_ready[stage], rank);
                if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                if (++sfs == (uint32_t)C::kSFSlots) sfs = 0;
                count++;
            }
        }
    } else if (warp == 2) {
        // ================= MMA issuer (even CTA) =================
        if (rank == 0) {
            const uint32_t idesc_base = (1u << 7) | (1u << 10) | ((uint32_t)((2 * kBM) >> 4) << 24);
            const uint32_t idesc_tail = idesc_base | ((uint32_t)(C::kTailMax >> 3) << 17);
            uint32_t stage = 0, phase = 0, aphase = 0, qi = 0, qphase = 0, sfs = 0;
            bool ok = true;
            while (ok) {
                int32_t w;
                if (!next_tile_warp(sh, rank, qi, qphase, w, lane, abort, p.ctl)) { ok = false; break; }
                if (w >= total) break;
                Tile t;
                decode_tile<C::kTailMax>(sh, E, w, t);
                const uint32_t idesc = idesc_base | ((uint32_t)(t.bn >> 3) << 17);
                const bool tail = C::kTailMax > 0 && t.tail > 0;
                if (!warp_wait(&sh.acc_empty, aphase ^ 1u, abort, p.ctl)) { ok = false; break; }
                tc_fence_after();
                for (int32_t kt = 0; kt < ksteps_total; kt++) {
                    // sf_ready alone: it implies both CTAs' loads of the stage landed, since every scale writer
                    // waits for its CTA's loads before arriving (measured: one poll less per stage, 1-4% faster)
                    if (!warp_wait(&sh.sf_ready[stage], phase, abort, p.ctl)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t sb = smem_u32(stages + (size_t)stage * C::kStageBytes);
                        const uint32_t sf = tmem + C::kTmemSFRing + sfs * C::kSFSlot;
                        // the stage's first K-step descriptors; each further K-step is 32 bytes on, +2 in the
                        // address field (bits 0-13 hold address / 16, which stays below 2^14 in shared memory).
                        // Built once per stage with the tail test hoisted out of the K-steps: measured 1-2% faster
                        // on the gate/up GEMM than building each K-step's descriptors (same outputs).
                        const uint64_t a0 = make_smem_desc(sb + kOffA, 16, 1024, 2);
                        const uint64_t b0 = make_smem_desc(sb + C::kOffB, 16, 1024, 2);
                        const uint64_t t0 = make_smem_desc(sb + C::kOffBT, 16, 1024, 2);
                        const uint32_t acc0 = kt != 0 ? 1u : 0u;
                        // the tile's 256 columns, and (with_tail) the tail rows into columns 256-287
                        auto mma_step = [&](int kc, bool with_tail) {
                            const uint32_t acc = kc != 0 ? 1u : acc0;
                            mma_mxf4nvf4_pair(tmem, a0 + 2 * kc, b0 + 2 * kc, idesc, sf + 4 * kc, sf + 16 + 8 * kc, acc);
                            if (with_tail)
                                mma_mxf4nvf4_pair(tmem + kBNMax, a0 + 2 * kc, t0 + 2 * kc, idesc_tail, sf + 4 * kc,
                                                  sf + C::kSFTail + 4 * kc, acc);
                        };
                        if (kt != ksteps_total - 1 || last_ksteps == kKSteps) {
                            if (tail) {
#pragma unroll
                                for (int kc = 0; kc < kKSteps; kc++) mma_step(kc, true);
                            } else {
#pragma unroll
                                for (int kc = 0; kc < kKSteps; kc++) mma_step(kc, false);
                            }
                        } else {
                            // a last stage of 128 K-elements: its first two K-steps
                            for (int kc = 0; kc < last_ksteps; kc++) mma_step(kc, tail);
                        }
                        tc_commit_pair_both(&sh.empty[stage]);
                    }
                    __syncwarp();
                    if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
                    if (++sfs == (uint32_t)C::kSFSlots) sfs = 0;
                }
                if (!ok) break;
                if (lane == 0) {
                    tc_commit_pair_both(&sh.acc_full);
                }
                __syncwarp();
                aphase ^= 1u;
            }
            if (!ok || *abort) {
                if (lane == 0) {
                    tc_commit_pair(cluster_smem_addr(&sh.drain, 0));
                    mbar_wait_drain(&sh.drain, 0, 200000000ull);
                }
                __syncwarp();
            }
        }
    } else if (warp >= 4) {  // warps 4-7 and 12-15
        // ================= epilogue (both CTAs) =================
        // TMEM lane = A row of this CTA, column = token of the tile. Each warp drains its 32-token
        // chunks into registers, releases the accumulator, then per chunk stages a BF16 block in its
        // private shared buffer and stores it (tensor store, or 16-byte row pieces for a partial chunk).
        const int quad = warp & 3;
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const int half = warp >= 12 ? 1 : 0;  // this warp takes the chunks c with c % 2 == half
        uint16_t* stg = sh.ostage[half * 4 + quad];
        const bool up_lane = lane >= 16;
        const float a_g = __ldg(p.a_gscale);
        const float h_genc = kEpi == kEpiQuant ? __fdiv_rn(1.0f, __ldg(p.qo.gdec)) : 0.0f;   // static scale of h
        uint32_t amax = 0;  // max |stored BF16| of this thread, as BF16 bits
        uint32_t aphase = 0, qi = 0, qphase = 0, fphase = 0;
        // this CTA's 8 epilogue warps meet here (fused combine only); false when a wait ran out
        auto epi_sync = [&]() -> bool {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.fin_bar);
            const bool ok = warp_wait(&sh.fin_bar, fphase, abort, p.ctl);
            fphase ^= 1u;
            return ok;
        };
        while (true) {
            int32_t w;
            if (!next_tile_warp(sh, rank, qi, qphase, w, lane, abort, p.ctl) || w >= total) break;
            Tile t;
            decode_tile<C::kTailMax>(sh, E, w, t);
            // the accumulator is a whole main loop away: poll it with short pauses (fewer issue slots
            // and less power spent polling; measured ~1% faster under the power cap, same at full clock)
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_bounded_pause(&sh.acc_full, aphase, abort, p.ctl, 500))) break;
            tc_fence_after();
            const float alpha = a_g * __ldg(p.w_gscale + t.e);
            // Chunk c (columns [32 c, +32), tokens row0 + 32 c ...) as final BF16 values, two per word
            // (SWIGLU: 16 outputs per lane, NONE: 32); quantised h is written here directly
            auto finish = [&](int c, const float (&v)[32], uint32_t (&pk)[16]) {
                const int nrows = min(32, t.rows - c * 32);
                if (kSw) {
                    // lane l < 16 holds gate, lane l + 16 up, of output column 16 quad + l; lane l
                    // produces the even tokens, lane l + 16 the odd ones
                    if (kEpi == kEpiPlain && nrows == 32) {
                        // a whole chunk (the accumulator hold is the epilogue's critical path): two outputs
                        // per step rounded together to a BF16 pair, amax over the pairs at the end (measured
                        // on the prefill gate/up GEMM: 1.3% faster than one output at a time)
#pragma unroll
                        for (int j = 0; j < 16; j += 2) {
                            float hv[2];
#pragma unroll
                            for (int jj = 0; jj < 2; jj++) {
                                const int jx = j + jj;
                                const float send = up_lane ? v[2 * jx] : v[2 * jx + 1];
                                const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
                                hv[jj] = swiglu_f32(alpha * (up_lane ? recv : v[2 * jx]),
                                                    alpha * (up_lane ? v[2 * jx + 1] : recv));
                            }
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(hv[0], hv[1]);
                            pk[j >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                        // word i: tokens 4 i + (up lane) and 4 i + 2 + (up lane)
                        if (p.amax_out != nullptr) amax = max(amax, absmax_bf16x2(pk, 8, nrows, 4, up_lane ? 1 : 0));
                        return;
                    }
#pragma unroll
                    for (int j = 0; j < 16; j++) {
                        const float send = up_lane ? v[2 * j] : v[2 * j + 1];
                        const float recv = __shfl_xor_sync(0xFFFFFFFFu, send, 16);
                        const float g = alpha * (up_lane ? recv : v[2 * j]);
                        const float u = alpha * (up_lane ? v[2 * j + 1] : recv);
                        const uint32_t hb = __bfloat16_as_ushort(__float2bfloat16_rn(swiglu_f32(g, u)));
                        const bool valid = 2 * j + (up_lane ? 1 : 0) < nrows;
                        if (valid) amax = max(amax, hb & 0x7FFFu);
                        if (kEpi == kEpiQuant) {
                            // h as NVFP4: lanes 0-15 hold one 16-column block of token 2j, lanes 16-31
                            // the same block of token 2j + 1
                            uint32_t code;
                            const uint32_t S = quantize_half_warp_block(hb, valid, h_genc, code);
                            const uint32_t hi = __shfl_xor_sync(0xFFFFFFFFu, code, 1);
                            const int64_t hcols = p.N / 2;
                            const int64_t n = (int64_t)t.nt * kBM + (int64_t)rank * 64 + quad * 16 + (lane & 15);
                            const int64_t row = (int64_t)t.row0 + c * 32 + 2 * j + (up_lane ? 1 : 0);
                            if (valid && (lane & 1) == 0)
                                p.qo.q[row * (hcols / 2) + n / 2] = (uint8_t)(code | (hi << 4));
                            if (valid && (lane & 15) == 0) {
                                const int64_t b = n >> 4;
                                uint8_t* piece = p.qo.sf + ((b >> 4) * p.qo.rows_per_slab + row) * 16;
                                piece[b & 15] = (uint8_t)S;
                                if ((hcols & 255) == 128 && b == (hcols >> 4) - 1)   // the last slab's padding
                                    *reinterpret_cast<uint2*>(piece + 8) = make_uint2(0u, 0u);
                            }
                        }
                        if (j & 1) pk[j >> 1] |= hb << 16;
                        else pk[j >> 1] = hb;
                    }
                } else {
                    // alpha applied with packed FP32 multiplies, two outputs rounded per conversion, amax
                    // only when it is asked for (measured on the prefill down GEMM: 5% faster than one
                    // output at a time; the same bits). Word i: tokens 2 i and 2 i + 1.
                    const uint64_t a2 = f32x2_pack(alpha, alpha);
#pragma unroll
                    for (int i = 0; i < 32; i += 2)
                        pk[i >> 1] = f32x2_to_bf16x2(f32x2_mul(f32x2_pack(v[i], v[i + 1]), a2));
                    if (p.amax_out != nullptr) amax = max(amax, absmax_bf16x2(pk, 16, nrows, 2, 0));
                }
            };
            // Chunk c staged as a 32-token block in shared memory and stored
            auto store = [&](int c, const uint32_t (&pk)[16]) {
                const int nrows = min(32, t.rows - c * 32);
                const int32_t r0 = t.row0 + c * 32;
                // the previous chunk's tensor store has finished reading the staging block
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
                int32_t col;      // first output column of this warp's block
                int lane_cols;    // lanes per 16-byte row piece in the direct-store path: 2 (SwiGLU) or 4
                if (kSw) {
#pragma unroll
                    for (int j = 0; j < 16; j++)
                        stg[(2 * j + (up_lane ? 1 : 0)) * 16 + (lane & 15)] =
                            (uint16_t)((j & 1) ? (pk[j >> 1] >> 16) : (pk[j >> 1] & 0xFFFFu));
                    col = t.nt * kBM + (int32_t)rank * 64 + quad * 16;
                    lane_cols = 2;
                } else {
#pragma unroll
                    for (int i = 0; i < 32; i++)
                        stg[i * 32 + lane] = (uint16_t)((i & 1) ? (pk[i >> 1] >> 16) : (pk[i >> 1] & 0xFFFFu));
                    col = t.nt * 2 * kBM + (int32_t)rank * kBM + quad * 32;
                    lane_cols = 4;
                }
                if (nrows == 32 && kEpi != kEpiFinalize) {
                    // a whole chunk of the expert: one asynchronous tensor store of the block
                    // (the fused combine stores directly: its last arrivers read these rows back)
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tm_out, stg, col, r0);
                        bulk_commit_group();
                    }
                } else {
                    // the expert's last, partial chunk: rows past its end belong to the next expert
                    __syncwarp();
                    const int64_t ldo = kSw ? p.N / 2 : p.N;
                    const int row_elems = 8 * lane_cols;
                    const int rows_per_pass = 32 / lane_cols;
                    for (int r = lane / lane_cols; r < nrows; r += rows_per_pass) {
                        const int piece = 8 * (lane % lane_cols);
                        *reinterpret_cast<uint4*>(p.out + (int64_t)(r0 + r) * ldo + col + piece) =
                            *reinterpret_cast<const uint4*>(stg + r * row_elems + piece);
                    }
                    __syncwarp();
                }
            };
            // 0. The tail rows (columns 256-287), on tiles that have them: warps 4-7 finish and store them
            //    while the accumulator is still held
            if (C::kTailMax > 0 && half == 0 && t.tail > 0) {
                float v[32];
                tmem_ld_32x32b_x32(tmem + lane_base + kBNMax, v);
                tmem_ld_wait();
                uint32_t pkt[16];
                finish(kBNMax / 32, v, pkt);
                if (kEpi != kEpiQuant) store(kBNMax / 32, pkt);
            }
            // 1. Drain: this warp's chunks (c = half, half + 2, ...) become final values in registers, and
            //    the accumulator goes back to the MMA warp at once: the next tile's main loop runs while 2.
            //    stages and stores them.
            uint32_t pk[kChunksPerWarp][16];
#pragma unroll
            for (int ci = 0; ci < kChunksPerWarp; ci++) {
                const int c = half + 2 * ci;
                if (c * 32 < t.bn) {
                    float v[32];
                    tmem_ld_32x32b_x32(tmem + lane_base + c * 32, v);
                    tmem_ld_wait();
                    finish(c, v, pk[ci]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_on_leader(&sh.acc_empty, rank);
            // 2. Write out
#pragma unroll
            for (int ci = 0; ci < kChunksPerWarp; ci++) {
                if (kEpi == kEpiQuant) break;
                const int c = half + 2 * ci;
                if (c * 32 < t.bn) store(c, pk[ci]);
            }
            aphase ^= 1u;
            if (kEpi == kEpiFinalize) {
                // Fused combine over this CTA's 128 output columns: count the tile's rows in per (token,
                // 128-column block); the CTA that brings a count to k writes that token's combined output
                // for these columns (see the one-SM kernel: the result does not depend on the order).
                __threadfence();                            // this thread's y stores, device-wide, first
                if (!epi_sync()) break;
                for (int i = (half * 4 + quad) * 32 + lane; i < kBNMax + C::kTailMax; i += 32 * kEpiWarps) {
                    int32_t tok = -1;
                    if (i < t.rows) {
                        const int32_t tk = __ldg(p.fin.src + t.row0 + i);
                        if (tk >= 0 && tk < p.fin.T) {
                            uint32_t* cnt = p.fin.counters + (int64_t)tk * p.fin.col_blocks + 2 * t.nt + rank;
                            if (atomicAdd(cnt, 1u) == (uint32_t)(p.fin.k - 1)) {
                                atomicExch(cnt, 0u);            // left at zero for the next launch
                                tok = tk;
                            }
                        }
                    }
                    sh.fin_tok[i] = tok;
                }
                __threadfence();                            // the other rows' stores are visible before the reads
                if (!epi_sync()) break;
                // one half-warp per token: lane l combines columns [8 (l % 16), +8) of this CTA's 128
                const int64_t col = (int64_t)t.nt * 2 * kBM + (int64_t)rank * kBM + (lane & 15) * 8;
                for (int j = 2 * (half * 4 + quad) + (lane >> 4); j < t.rows; j += 2 * kEpiWarps) {
                    const int32_t tk = sh.fin_tok[j];
                    if (tk >= 0) combine_vec8(p.out, p.N, p.fin.inv, p.fin.w, tk, p.fin.k, col, p.fin.out, p.N);
                }
                if (!epi_sync()) break;                     // fin_tok is rewritten by the next tile
            }
        }
        if (lane == 0) bulk_wait_group0();  // this warp's tensor stores completed
        __syncwarp();
        if (p.amax_out != nullptr) {
            amax = __reduce_max_sync(0xFFFFFFFFu, amax);
            if (lane == 0 && amax != 0u) atomicMax(p.amax_out, amax);
        }
    }

    // ---- teardown: both CTAs have drained their own work; then the pair frees its TMEM ----
    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 2) tmem_dealloc_pair(tmem, kTmemCols);
    // The last CTA to finish leaves the work counters at zero for the next launch that draws this slot.
    if (tid == 0 && atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
        atomicExch(p.sched, 0u);
        atomicExch(p.sched + 1, 0u);
    }
}

}  // namespace gp
}  // namespace nvfp4

using namespace nvfp4;

namespace nvfp4 {

// the largest of the instantiated configurations (SwiGLU, plain, fused combine in each of the three)
template <int kConf>
static constexpr size_t pair_conf_smem() {
    constexpr size_t a = gp::Cfg<kConf, true, false>::kSmemBytes, b = gp::Cfg<kConf, false, false>::kSmemBytes,
                     c = gp::Cfg<kConf, false, true>::kSmemBytes;
    return a > b ? (a > c ? a : c) : (b > c ? b : c);
}
size_t pair_gemm_smem_bytes() {
    constexpr size_t c0 = pair_conf_smem<0>(), c1 = pair_conf_smem<1>(), c2 = pair_conf_smem<2>();
    return c0 > c1 ? (c0 > c2 ? c0 : c2) : (c1 > c2 ? c1 : c2);
}
int pair_gemm_tokens_max() { return gp::kBNMax; }
int pair_gemm_store_cols(int swiglu) { return swiglu ? 16 : 32; }  // 32 tokens x this many BF16 columns

// The shared-memory opt-in of one instantiation, once per device (thread-safe).
template <int kEpi, int kConf, bool kSw>
static bool pair_kernel_configured(int dev) {
    static std::once_flag once[64];
    static bool ok[64] = {};
    std::call_once(once[dev], [&] {
        ok[dev] = cudaFuncSetAttribute(gp::grouped_gemm_pair_kernel<kEpi, kConf, kSw>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)gp::Cfg<kConf, kSw, kEpi == kEpiFinalize>::kSmemBytes) == cudaSuccess;
    });
    return ok[dev];
}

// As many pairs as can be resident at once (the persistent grid), once per device and configuration.
template <int kConf>
static nvfp4_status pair_grid(int dev, int& grid) {
    static std::once_flag once[64];
    static int grid_for[64] = {};
    static nvfp4_status set_result[64] = {};
    std::call_once(once[dev], [&] {
        set_result[dev] = NVFP4_ERR_CUDA;
        // the SwiGLU instantiation: the configuration's largest shared memory but for the fused combine's
        // table, and every instantiation fits one CTA per SM
        if (!pair_kernel_configured<kEpiPlain, kConf, true>(dev)) return;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)device_sm_count() / 2 * 2);
        cfg.blockDim = dim3(gp::kThreads);
        cfg.dynamicSmemBytes = gp::Cfg<kConf, true, false>::kSmemBytes;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = 2;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, gp::grouped_gemm_pair_kernel<kEpiPlain, kConf, true>, &cfg) !=
                cudaSuccess ||
            clusters <= 0) {
            set_result[dev] = NVFP4_ERR_SMEM_BUDGET;
            return;
        }
        grid_for[dev] = 2 * clusters < device_sm_count() ? 2 * clusters : device_sm_count() / 2 * 2;
        set_result[dev] = NVFP4_OK;
    });
    grid = grid_for[dev];
    return set_result[dev];
}

template <int kConf>
static nvfp4_status launch_pair_config(int dev, const CUtensorMap& tm_a, const CUtensorMap& tm_a_full,
                                       const CUtensorMap& tm_out, const CUtensorMap& tm_wsw, const CUtensorMap& tm_wsf,
                                       const gp::Params& prm, cudaStream_t s) {
    int grid = 0;
    const nvfp4_status st = pair_grid<kConf>(dev, grid);
    if (st != NVFP4_OK) return st;
    // every instantiation runs one CTA per SM in clusters of two; quantised h is SWIGLU only, the fused
    // combine NONE only (the caller checked)
    if (prm.qo.q != nullptr) {
        if (!pair_kernel_configured<kEpiQuant, kConf, true>(dev)) return NVFP4_ERR_CUDA;
        launch_pdl(gp::grouped_gemm_pair_kernel<kEpiQuant, kConf, true>, dim3(grid), dim3(gp::kThreads),
                   gp::Cfg<kConf, true, false>::kSmemBytes, s, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm);
    } else if (prm.fin.out != nullptr) {
        if (!pair_kernel_configured<kEpiFinalize, kConf, false>(dev)) return NVFP4_ERR_CUDA;
        launch_pdl(gp::grouped_gemm_pair_kernel<kEpiFinalize, kConf, false>, dim3(grid), dim3(gp::kThreads),
                   gp::Cfg<kConf, false, true>::kSmemBytes, s, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm);
    } else if (prm.swiglu) {
        if (!pair_kernel_configured<kEpiPlain, kConf, true>(dev)) return NVFP4_ERR_CUDA;
        launch_pdl(gp::grouped_gemm_pair_kernel<kEpiPlain, kConf, true>, dim3(grid), dim3(gp::kThreads),
                   gp::Cfg<kConf, true, false>::kSmemBytes, s, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm);
    } else {
        if (!pair_kernel_configured<kEpiPlain, kConf, false>(dev)) return NVFP4_ERR_CUDA;
        launch_pdl(gp::grouped_gemm_pair_kernel<kEpiPlain, kConf, false>, dim3(grid), dim3(gp::kThreads),
                   gp::Cfg<kConf, false, false>::kSmemBytes, s, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm);
    }
    return NVFP4_OK;
}

// Launches the pair kernel; the caller validated every argument (same contract as the one-SM kernel).
// Several experts: a configuration that lets up to 32 rows past a full tile ride on it; one expert (a dense
// GEMM): the configuration without that and with a scale slot per stage.
nvfp4_status launch_grouped_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_a_full,
                                      const CUtensorMap& tm_out, const CUtensorMap& tm_wsw,
                                      const CUtensorMap& tm_wsf, const uint8_t* a_sf,
                                      const float* a_gscale, const uint8_t* w_packed, const float* w_gscale,
                                      const int32_t* offsets, int32_t E, int64_t max_rows, int64_t N, int64_t K,
                                      int swiglu, uint16_t* out, uint32_t* out_amax, const Finalize& fin,
                                      const QuantOut& qo, cudaStream_t s, uint32_t* status) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
    gp::Params prm;
    prm.a_sf = a_sf;
    prm.a_gscale = a_gscale;
    prm.w_packed = w_packed;
    prm.w_gscale = w_gscale;
    prm.offsets = offsets;
    prm.out = out;
    prm.E = E;
    prm.max_rows = max_rows;
    prm.N = N;
    prm.K = K;
    prm.swiglu = swiglu;
    prm.amax_out = out_amax;
    prm.fin = fin;
    prm.qo = qo;
    prm.sched = sched_counter_slot();
    if (!prm.sched) return NVFP4_ERR_CUDA;
    prm.ctl.status = status;
    prm.ctl.timeout_ns = wait_timeout_ns();
    prm.ctl.flags = debug_flags();
    // one expert: no row tails; up to 256 experts: row tails and 5 data stages; more: row tails and 4
    const nvfp4_status st =
        E == 1     ? launch_pair_config<0>(dev, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm, s)
        : E <= 256 ? launch_pair_config<2>(dev, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm, s)
                   : launch_pair_config<1>(dev, tm_a, tm_a_full, tm_out, tm_wsw, tm_wsf, prm, s);
    if (st != NVFP4_OK) return st;
    count_launch();
    return check_launch();
}

}  // namespace nvfp4
