// gemm.cuh -- block-scaled FP8 GEMM on the 5th-generation tensor cores (tcgen05), with the
// per-128-K scales applied when each K group's partial sum is promoted into FP32.
//
// What it computes (DeepSeek-V3 report repost, paragraphs 1 and 4, Figure 7(b);
// "DeepSeek-V3 Technical Report" summary page, Key ideas, FP8 bullet):
//   for each 128-wide K group kb:  P = sum_{k in kb} qA[m,k] qB(k,n)        (tensor cores, FP32)
//                                  acc[m,n] += P * sA[kb][m] * sB(kb, n)    (CUDA cores, FP32)
//   D = acc  (bf16 for Fprop / Dgrad, FP32 for Wgrad).
// The pages' H800 design runs two WGMMA warpgroups so one promotes while the other multiplies.
// Here the overlap comes from the asynchronous tcgen05 pipeline instead:
//   warp 0      TMA producer: A and B tiles (128-byte swizzled) into a STAGES-deep ring;
//               for Wgrad also the per-column scales of each K group (bulk copy).
//   warps 1, 3  MMA issuers: 4 x tcgen05.mma (K = 32 each) per K group into one of two TMEM
//               partial buffers (a fresh accumulation per group), then tcgen05.commit; warp 1
//               issues the groups of buffer 0, warp 3 those of buffer 1.  An issuing warp slows
//               the promotion warps of its SM sub-partition (which gate every buffer hand-back),
//               so the issuing is split over two sub-partitions.
//   warps 4..   promotion (2 or 4 warpgroups): tcgen05.ld the partial of group kb while the
//               tensor cores fill the other buffer, fold in the scales and accumulate in
//               registers (each warp owns 32 rows x BN/kPW columns); after the last group,
//               convert and store the tile.
// The CTA is persistent (one per SM) and walks a static tile list, so the epilogue of one
// tile overlaps the first MMAs of the next.  setmaxnreg moves registers from the producer /
// MMA warpgroup to the promotion warpgroups (see GemmShape).
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "ptx.cuh"
#include "quant.cuh"

namespace fp8q {

enum { kModeFprop = 0, kModeDgrad = 1, kModeWgrad = 2 };

struct GemmArgs {
    const float* sA;          // [KB][M]
    const float* sB;          // Fprop [N/128][KB], Dgrad [KB][N/128] (each x E if grouped); Wgrad [KB][N]
    void* D;                  // [M][N], bf16 (Fprop / Dgrad) or fp32 (Wgrad)
    const int32_t* offsets;   // grouped only: device [E+1]
    int32_t E;                // number of groups (1 unless grouped)
    int32_t M;                // rows of A and D
    int32_t N;
    int32_t KB;               // K / 128
    // Stream-K schedule (ws != nullptr): CTA c owns the (tile, 128-K group) units
    // [units*c/G, units*(c+1)/G) of the tile-major unit space, G = gridDim.x.
    float* ws;                // partial accumulators, one 128 x BN FP32 slot per CTA
    unsigned long long* flags;   // per CTA: == stamp once its slot holds this launch's partial
    unsigned long long stamp; // unique per launch, so flags never need resetting
    int64_t units;            // tiles * KB
    int32_t accumulate;       // Wgrad only: 1 adds the result into D (D += dY^T X), 0 overwrites D
    // Fused 1x128 quantisation of the bf16 output (dense Fprop / Dgrad with 256-wide tiles):
    // q_out [M][N] E4M3 codes and s_out [N/128][M] scales of bf16(D), exactly what the 1x128
    // activation quantiser would produce from the stored D; nullptr = off.  store_d = 0 skips D.
    float* s_out;
    int32_t quant_out;
    int32_t store_d;
    int64_t rows_total;       // grouped: the offsets must end here (rows of A, or tokens for Wgrad)
};

// One piece of work: groups [kb0, kb1) of tile `tile`.
struct WorkItem {
    int tile;
    int kb0;
    int kb1;
};

// Walks a CTA's work items.  Data-parallel: whole tiles c, c + G, ...  Stream-K: the CTA's
// contiguous unit range cut at tile boundaries -- at most one leading item that starts
// mid-tile (its partial goes to the workspace) and at most one trailing item that starts at
// group 0 without reaching the end (it adds the later CTAs' partials, then stores the tile).
struct WorkSched {
    int64_t u, u_end;
    int t;
    bool sk;
};

__device__ __forceinline__ int64_t sk_begin(int64_t units, int c, int G) { return units * c / G; }

__device__ __forceinline__ WorkSched sched_begin(const GemmArgs& a)
{
    WorkSched w;
    w.sk = a.ws != nullptr;
    w.t = (int)blockIdx.x;
    w.u = w.sk ? sk_begin(a.units, (int)blockIdx.x, (int)gridDim.x) : 0;
    w.u_end = w.sk ? sk_begin(a.units, (int)blockIdx.x + 1, (int)gridDim.x) : 0;
    return w;
}

__device__ __forceinline__ bool sched_next(WorkSched& w, int num_tiles, int KB, WorkItem& it)
{
    if (!w.sk) {
        if (w.t >= num_tiles) return false;
        it.tile = w.t;
        it.kb0 = 0;
        it.kb1 = KB;
        w.t += (int)gridDim.x;
        return true;
    }
    if (w.u >= w.u_end) return false;
    it.tile = (int)(w.u / KB);
    it.kb0 = (int)(w.u - (int64_t)it.tile * KB);
    const int64_t n = min((int64_t)(KB - it.kb0), w.u_end - w.u);
    it.kb1 = it.kb0 + (int)n;
    w.u += n;
    return true;
}

// MX: the power-of-two (UE8M0) scale variant.  The tensor core applies the scales itself
// (tcgen05.mma kind::mxf8f6f4, one 8-bit exponent per row / column per 32-element K block), so
// the whole K accumulates in one TMEM accumulator and the promotion warps only drain it once
// per work item.  Warp 2 turns each K group's fp32 power-of-two scales into the scale-factor
// layout the MMA reads and warp 1 copies them into TMEM (tcgen05.cp) ahead of the group's MMAs.
template <int MODE, int BN, bool GROUPED, bool MX = false>
struct GemmShape {
    static constexpr int kBM = 128;
    static constexpr int kBK = 128;
    static constexpr int kABytes = kBM * kBK;
    static constexpr int kBBytes = BN * kBK;
    static constexpr int kStageBytes = kABytes + kBBytes;
    // Wgrad keeps three stages: its promotion, not the operand feed, sets the pace, and the 48 KB
    // freed pay for a second epilogue staging buffer per warp (the fp32 tile leaves in eight 2 KB
    // slabs per warp; with one buffer each slab waited for the previous store to read it).
    // Measured: linear-layer Wgrad (2048 x 7168 x 4096) 104.8 -> 100.0 us; MoE grouped Wgrad
    // (256 experts, 65536 rows) 4.49 -> 4.17 ms.
    static constexpr bool kWgrad3 = MODE == kModeWgrad && !MX && BN == 256;
    static constexpr int kStages = kWgrad3 ? 3 : ((BN == 256) ? 4 : 6);
    static constexpr int kScaleStages = (MODE == kModeWgrad && !MX) ? 4 : 0;
    // MX scale factors per stage: one 512-byte chunk for A's 128 rows and one per 128 columns
    // of B.  Chunk row r (16 bytes, r = 0..31) holds the exponents of rows r, 32 + r, 64 + r,
    // 96 + r as four 32-bit words, each word the same exponent in all four bytes (one per
    // 32-element K block of the 128-wide group); tcgen05.cp 32x128b.warpx4 copies a chunk to
    // 4 TMEM columns of all 128 lanes, the layout the block-scaled MMA reads.
    static constexpr int kSfChunks = MX ? 1 + BN / 128 : 0;
    static constexpr int kSfStageBytes = 512 * kSfChunks;
    static constexpr int kSfCol0 = BN;                   // TMEM: accumulator [0, BN), then 16 columns per stage
    static constexpr int kOffSf = kStages * kStageBytes;
    // Promotion warpgroups.  Each owns BN / kPW columns of the tile (all 128 rows; warp w of a
    // group reads TMEM lanes 32*(w%4) ..).  Two: four groups (640 threads) halve each thread's
    // arithmetic per K group but not its TMEM round trips, which set the fold's length; with
    // 104 registers per thread they measured 6-8 % slower on the linear-layer Fprop / Dgrad and
    // 43 % slower on Wgrad (whose fold then spills).
    static constexpr int kPW = 2;
    static constexpr int kPromoWarps = 4 * kPW;
    static constexpr int kPromoThreads = 128 * kPW;
    static constexpr int kCols = BN / kPW;         // columns per promotion thread
    static constexpr int kTmemCols = 2 * BN;       // two partial buffers
    static constexpr int kThreads = 128 + kPromoThreads;
    static constexpr int kMaxGroups = 1024;
    static constexpr int kOffScales = kOffSf + kStages * kSfStageBytes;
    static constexpr int kOffBars = kOffScales + kScaleStages * BN * 4;
    static constexpr int kNumBars = 2 * kStages + 4 + 2 * kScaleStages + 2 + (MX ? kStages : 0);
    static constexpr int kOffMisc = kOffBars + kNumBars * 8;
    static constexpr int kOffGroups = kOffMisc + 16;
    // Epilogue staging: 2 KB per promotion warp and buffer, 1024-byte aligned (the 64-byte
    // swizzle of the tensor store works on absolute shared-memory address bits).  Two buffers per
    // warp where shared memory allows, so one slab's store reads while the next is written.
    static constexpr int kEpiBufs = kWgrad3 ? 2 : ((MODE == kModeWgrad || GROUPED || kPW == 4 || MX) ? 1 : 2);
    static constexpr int kOffEpi = (kOffGroups + (GROUPED ? 2 * (kMaxGroups + 1) * 4 : 0) + 1023) / 1024 * 1024;
    static constexpr int kSmemBytes = kOffEpi + kPromoWarps * 2048 * kEpiBufs + 1024;
    // Registers (setmaxnreg moves them from the producer / MMA warpgroup to the promotion
    // warpgroups within the launch allocation):
    //   384 threads launched at 168:  128 x 40 + 256 x 232 = 64512 <= 384 x 168
    //   640 threads launched at  96:  128 x 56 + 512 x 104 = 60416 <= 640 x  96
    //   MX, 384 threads at 168:       128 x 72 + 256 x 216 = 64512 (the scale warp keeps two
    //                                 K groups of scales in flight; the drain needs no scales)
    static constexpr int kRegsLow = (kPW == 4) ? 56 : (MX ? 72 : 40);
    static constexpr int kRegsHigh = (kPW == 4) ? 104 : (MX ? 216 : 232);
    static constexpr int kRegsLaunch = (kPW == 4) ? 96 : 168;
    static_assert(kThreads * kRegsLaunch >= 128 * kRegsLow + kPromoThreads * kRegsHigh, "register split");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static_assert(!MX || kSfCol0 + 16 * kStages <= kTmemCols, "MX scale factors fit the TMEM allocation");
    static_assert(!(MX && GROUPED), "the MX variant is dense only");
};

struct TileInfo {
    int32_t row0;      // first row of the 128-row tile (rows of A)
    int32_t row_end;   // rows >= row_end are not part of this tile's group (masked)
    int32_t n0;        // first column
    int32_t e;         // group
    int32_t out_row0;  // first row of the tile in D (K-grouped Wgrad: expert e's dW starts at e*M)
};

// Grouped GEMMs.  Row-grouped (Fprop / Dgrad): the rows of A are split among experts and a
// tile holds one expert's rows.  K-grouped (Wgrad): every expert has the full M x N output, and
// its K range is its own tokens' 128-token groups [g_pre[e], g_pre[e+1]).
template <bool GROUPED, bool KGROUPED>
__device__ __forceinline__ TileInfo decode_tile(int t, int nb_tiles, int bn, const GemmArgs& a,
                                                const int32_t* g_off, const int32_t* g_pre)
{
    TileInfo ti;
    if (KGROUPED) {
        const int per_e = ((a.M + 127) >> 7) * nb_tiles;
        ti.e = t / per_e;
        const int r = t - ti.e * per_e;
        const int mt = r / nb_tiles;
        ti.n0 = (r - mt * nb_tiles) * bn;
        ti.row0 = mt * 128;
        ti.row_end = a.M;
        ti.out_row0 = ti.e * a.M + ti.row0;
        return ti;
    }
    const int mt = t / nb_tiles;
    const int nt = t - mt * nb_tiles;
    ti.n0 = nt * bn;
    if (GROUPED) {
        int lo = 0, hi = a.E;   // g_pre[lo] <= mt < g_pre[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (g_pre[mid] <= mt) lo = mid; else hi = mid;
        }
        ti.e = lo;
        ti.row0 = g_off[lo] + (mt - g_pre[lo]) * 128;
        ti.row_end = g_off[lo + 1];
    } else {
        ti.e = 0;
        ti.row0 = mt * 128;
        ti.row_end = a.M;
    }
    ti.out_row0 = ti.row0;
    return ti;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <int MODE, int BN, bool GROUPED, bool MX = false>
__global__ void __launch_bounds__(GemmShape<MODE, BN, GROUPED, MX>::kThreads, 1)
gemm_blockscaled_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmQ,
                        const GemmArgs args)
{
    using S = GemmShape<MODE, BN, GROUPED, MX>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* col_scales = reinterpret_cast<float*>(smem + S::kOffScales);
    uint32_t* misc = reinterpret_cast<uint32_t*>(smem + S::kOffMisc);   // [0] TMEM base, [1] abort, [2] bad groups
    int32_t* g_off = reinterpret_cast<int32_t*>(smem + S::kOffGroups);
    int32_t* g_pre = g_off + (S::kMaxGroups + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);

    const uint32_t bar0 = smem_u32(smem + S::kOffBars);
    const auto full_bar = [&](int s) { return bar0 + 8u * s; };
    const auto empty_bar = [&](int s) { return bar0 + 8u * (S::kStages + s); };
    const auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * S::kStages + b); };
    const auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * S::kStages + 2 + b); };
    const auto sfull_bar = [&](int s) { return bar0 + 8u * (2 * S::kStages + 4 + s); };
    const auto sempty_bar = [&](int s) { return bar0 + 8u * (2 * S::kStages + 4 + S::kScaleStages + s); };
    const uint32_t drain_bar = bar0 + 8u * (2 * S::kStages + 4 + 2 * S::kScaleStages);
    const uint32_t parked_bar = drain_bar + 8u;   // stream-K: all promotion warps wrote the slot
    const auto sf_full_bar = [&](int s) { return parked_bar + 8u * (1 + s); };   // MX: chunks of stage s built

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    griddep_launch_dependents();

    // ---------------------------------------------------------------- set-up
    if (threadIdx.x == 0) {
        for (int s = 0; s < S::kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), S::kPromoWarps);
        }
        for (int s = 0; s < S::kScaleStages; ++s) {
            mbar_init(sfull_bar(s), 1);
            mbar_init(sempty_bar(s), S::kPromoWarps);
        }
        mbar_init(drain_bar, MX ? 1 : 2);
        mbar_init(parked_bar, S::kPromoWarps);
        if (MX)
            for (int s = 0; s < S::kStages; ++s) mbar_init(sf_full_bar(s), 1);
        misc[1] = 0;
        misc[2] = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(misc), S::kTmemCols);
        tmem_relinquish();
    }
    // Everything above touches only this CTA's own resources; inputs are read from here on.
    griddep_wait();
    if (GROUPED && warp == 2) {
        // Copy the offsets, validate them and build the prefix of 128-row tiles per group with a
        // warp scan (each lane owns a contiguous run of groups).
        const int E = args.E;
        for (int i = lane; i <= E; i += 32) g_off[i] = __ldg(args.offsets + i);
        __syncwarp();
        const int per = (E + 31) >> 5;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int local = 0;
        bool bad = false;
        for (int e = lo; e < hi; ++e) {
            const int cnt = g_off[e + 1] - g_off[e];
            bad |= cnt < 0;
            local += cnt > 0 ? (cnt + 127) >> 7 : 0;
        }
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        int run = incl - local;
        for (int e = lo; e < hi; ++e) {
            g_pre[e] = run;
            const int cnt = g_off[e + 1] - g_off[e];
            run += cnt > 0 ? (cnt + 127) >> 7 : 0;
        }
        if (lane == 31) g_pre[E] = incl;
        if (lane == 0) bad |= (g_off[0] != 0) || ((int64_t)g_off[E] != args.rows_total);
        // K-grouped: the experts' padded token groups must fit the operands' K extent.
        if (MODE == kModeWgrad) bad |= __shfl_sync(0xFFFFFFFFu, incl, 31) > args.KB;
        bad = __any_sync(0xFFFFFFFFu, bad);
        if (bad && lane == 0) {
            misc[2] = 1;
            latch_status(2 /* FP8Q_DEV_BAD_OFFSETS */);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    const uint32_t tmem_base = misc[0];
    const int nb_tiles = args.N / BN;
    constexpr bool kKGrouped = GROUPED && MODE == kModeWgrad;    // K ranges per expert
    constexpr bool kRowGrouped = GROUPED && MODE != kModeWgrad;  // rows per expert
    const int num_m_tiles = kRowGrouped ? (misc[2] ? 0 : g_pre[args.E]) : (args.M + 127) / 128;
    const int num_tiles = (kKGrouped ? (misc[2] ? 0 : args.E) : 1) * num_m_tiles * nb_tiles;
    // K-grouped: a work item's K groups are its expert's padded token groups.
    const auto kgroup_range = [&](WorkItem& it) {
        if (kKGrouped) {
            const int e = it.tile / (num_m_tiles * nb_tiles);
            it.kb0 = g_pre[e];
            it.kb1 = g_pre[e + 1];
        }
    };
    const int KB = args.KB;

    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(S::kRegsLow));
        if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int stage = 0, ss = 0;
            uint32_t phase = 0, sph = 0;
            bool ok = true;
            WorkSched ws = sched_begin(args);
            WorkItem it;
            while (ok && sched_next(ws, num_tiles, KB, it)) {
                kgroup_range(it);
                const TileInfo ti = decode_tile<GROUPED, kKGrouped>(it.tile, nb_tiles, BN, args, g_off, g_pre);
                const int brow = kRowGrouped ? ti.e * args.N + ti.n0 : ti.n0;
                for (int kb = it.kb0; kb < it.kb1; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
                    const uint32_t sa = smem_u32(smem + stage * S::kStageBytes);
                    const uint32_t sb = sa + S::kABytes;
                    mbar_arrive_expect_tx(full_bar(stage), S::kStageBytes);
                    tma_load_2d(sa, &tmA, kb * 128, ti.row0, full_bar(stage));
                    if (MODE == kModeDgrad) {
#pragma unroll
                        for (int h = 0; h < BN / 128; ++h)   // grouped: expert e's K rows start at e * K
                            tma_load_2d(sb + h * 16384, &tmB, ti.n0 + h * 128, (GROUPED ? ti.e * KB * 128 : 0) + kb * 128,
                                        full_bar(stage));
                    } else {
                        tma_load_2d(sb, &tmB, kb * 128, brow, full_bar(stage));
                    }
                    if (MODE == kModeWgrad && !MX) {
                        if (!mbar_wait(sempty_bar(ss), sph ^ 1u, abort_flag)) { ok = false; break; }
                        mbar_arrive_expect_tx(sfull_bar(ss), BN * 4);
                        bulk_load(smem_u32(col_scales + ss * BN), args.sB + (size_t)kb * args.N + ti.n0, BN * 4,
                                  sfull_bar(ss));
                        if (++ss == S::kScaleStages) { ss = 0; sph ^= 1u; }
                    }
                    if (++stage == S::kStages) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok) {
                // Aborting: give copies already in flight time to land before the CTA exits.
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 50000ull) __nanosleep(1000);
            }
        }
        } else if (MX && warp == 1) {
        // ------------------------------------------------------------ MMA issuer (MX)
        // One accumulator: a work item's groups accumulate into TMEM columns [0, BN); the next
        // item starts once the promotion warps have drained it.  Per group: the scale chunks go
        // to this stage's 16 TMEM scale columns (A at +0, B at +4), then 4 MMAs.  The four bytes
        // of a scale word are one group's exponent for its four 32-element K blocks, all equal,
        // so every MMA reads byte 0 (scale-factor id 0).
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, aph = 0;
            bool ok = true;
            WorkSched ws = sched_begin(args);
            WorkItem it;
            while (ok && sched_next(ws, num_tiles, KB, it)) {
                if (!mbar_wait(tempty_bar(0), aph ^ 1u, abort_flag)) { ok = false; break; }
                tc_fence_after();
                for (int kb = it.kb0; kb < it.kb1; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                    if (!mbar_wait(sf_full_bar(stage), phase, abort_flag)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * S::kStageBytes);
                    const uint32_t sb = sa + S::kABytes;
                    const uint32_t sf = smem_u32(smem + S::kOffSf + stage * S::kSfStageBytes);
                    const uint32_t tsf = tmem_base + (uint32_t)(S::kSfCol0 + 16 * stage);
#pragma unroll
                    for (int c = 0; c < S::kSfChunks; ++c) tmem_cp_32x128b_x4(tsf + 4u * c, sdesc_plain(sf + 512u * c, 128));
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const uint64_t ad = sdesc_sw128(sa + k * 32, 16, 1024);
                        const uint64_t bd = (MODE == kModeDgrad) ? sdesc_sw128(sb + k * 4096, 16384, 1024)
                                                                 : sdesc_sw128(sb + k * 32, 16, 1024);
                        constexpr uint32_t idesc = idesc_mx_e4m3(BN, MODE == kModeDgrad, 0u, 0u);
                        mma_mxf8f6f4(tmem_base, ad, bd, idesc, tsf, tsf + 4u, (kb > it.kb0 || k > 0) ? 1u : 0u);
                    }
                    tc_commit(empty_bar(stage));
                    if (++stage == S::kStages) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(tfull_bar(0));
                aph ^= 1u;
            }
            tc_commit(drain_bar);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
            }
        }
        __syncwarp();
        // Release TMEM once the promotion warps have read their last accumulator.
        named_bar_sync(1, 32 + S::kPromoThreads);
        tc_fence_after();
        tmem_dealloc(tmem_base, S::kTmemCols);
        } else if (MX && warp == 2) {
        // ------------------------------------------------------------ scale chunks (MX)
        // Lane l builds chunk row l: the exponents of A rows l + 32j (j = 0..3) and of B columns
        // 128h + l + 32j.  The fp32 scales are loaded two K groups ahead (they come from L2:
        // the item's scales are prefetched at its start); a scale that is not a positive normal
        // power of two latches FP8Q_DEV_BAD_SCALES.
        constexpr int kNB = (MODE == kModeWgrad) ? 4 * (BN / 128) : (BN / 128);   // B scales per lane
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, bad = false;
        WorkSched ws = sched_begin(args);
        WorkItem it;
        while (ok && sched_next(ws, num_tiles, KB, it)) {
            const TileInfo ti = decode_tile<false, false>(it.tile, nb_tiles, BN, args, g_off, g_pre);
            const auto a_ptr = [&](int kb, int j) -> const float* {
                return args.sA + (size_t)kb * args.M + (ti.row0 + lane + 32 * j);
            };
            const auto b_ptr = [&](int kb, int j) -> const float* {
                if (MODE == kModeWgrad) return args.sB + (size_t)kb * args.N + ti.n0 + 128 * (j >> 2) + lane + 32 * (j & 3);
                if (MODE == kModeFprop) return args.sB + (size_t)((ti.n0 >> 7) + j) * KB + kb;
                return args.sB + (size_t)kb * (args.N >> 7) + (ti.n0 >> 7) + j;
            };
            // Pull the item's scales into L2: per group 4 lines of row scales (and for Wgrad 8 of
            // column scales), clamped to rows that exist.
            for (int k = it.kb0 + (lane >> 3); k < it.kb1; k += 4) {
                const int j = lane & 7;
                if (j < 4) prefetch_l2(args.sA + (size_t)k * args.M + min(ti.row0 + 32 * j, args.M - 1));
                if (MODE == kModeWgrad) {
                    if (32 * j < BN) prefetch_l2(args.sB + (size_t)k * args.N + ti.n0 + 32 * j);
                }
                else if (j == 4) prefetch_l2(b_ptr(k, 0));
            }
            float na[3][4], nbv[3][kNB];
            const auto load = [&](int kb, float (&a)[4], float (&b)[kNB]) {
#pragma unroll
                for (int j = 0; j < 4; ++j) a[j] = (kb < it.kb1 && ti.row0 + lane + 32 * j < args.M) ? __ldg(a_ptr(kb, j)) : 1.0f;
#pragma unroll
                for (int j = 0; j < kNB; ++j) b[j] = kb < it.kb1 ? __ldg(b_ptr(kb, j)) : 1.0f;
            };
            load(it.kb0, na[0], nbv[0]);
            load(it.kb0 + 1, na[1], nbv[1]);
            for (int kb = it.kb0; kb < it.kb1; ++kb) {
                load(kb + 2, na[2], nbv[2]);
                const auto expo = [&](float v) -> uint32_t {
                    const uint32_t u = __float_as_uint(v);
                    const uint32_t e = u >> 23;
                    bad |= (u & 0x7FFFFFu) != 0u || e == 0u || e >= 255u;
                    return (e & 0xFFu) * 0x01010101u;
                };
                const uint4 wa = make_uint4(expo(na[0][0]), expo(na[0][1]), expo(na[0][2]), expo(na[0][3]));
                uint4 wb[BN / 128];
#pragma unroll
                for (int h = 0; h < BN / 128; ++h) {
                    if (MODE == kModeWgrad) {
                        wb[h] = make_uint4(expo(nbv[0][4 * h]), expo(nbv[0][4 * h + 1]), expo(nbv[0][4 * h + 2]),
                                           expo(nbv[0][4 * h + 3]));
                    } else {
                        const uint32_t w = expo(nbv[0][h]);
                        wb[h] = make_uint4(w, w, w, w);
                    }
                }
                if (!warp_wait(empty_bar(stage), phase ^ 1u, abort_flag)) { ok = false; break; }
                uint4* chunk = reinterpret_cast<uint4*>(smem + S::kOffSf + stage * S::kSfStageBytes);
                chunk[lane] = wa;
#pragma unroll
                for (int h = 0; h < BN / 128; ++h) chunk[32 * (1 + h) + lane] = wb[h];
                fence_proxy_async_smem();   // generic-proxy writes, read by tcgen05.cp
                __syncwarp();
                if (lane == 0) mbar_arrive(sf_full_bar(stage));
                if (++stage == S::kStages) { stage = 0; phase ^= 1u; }
#pragma unroll
                for (int j = 0; j < 4; ++j) { na[0][j] = na[1][j]; na[1][j] = na[2][j]; }
#pragma unroll
                for (int j = 0; j < kNB; ++j) { nbv[0][j] = nbv[1][j]; nbv[1][j] = nbv[2][j]; }
            }
        }
        if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) latch_status(3 /* FP8Q_DEV_BAD_SCALES */);
        } else if (!MX && (warp == 1 || warp == 3)) {
        // ------------------------------------------------------------ MMA issuers
        // Warp 1 issues the K groups that accumulate into TMEM buffer 0, warp 3 those into buffer
        // 1 (independent accumulators), so the issuing work is split over two SM sub-partitions.
        const int mybuf = (warp == 1) ? 0 : 1;
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_e4m3_f32(BN, MODE == kModeDgrad);
            int stage = 0, tb = 0;
            uint32_t phase = 0, tph = 0;
            bool ok = true;
            WorkSched ws = sched_begin(args);
            WorkItem it;
            while (ok && sched_next(ws, num_tiles, KB, it)) {
                kgroup_range(it);
                for (int kb = it.kb0; kb < it.kb1; ++kb) {
                    if (tb == mybuf) {
                        if (!mbar_wait(tempty_bar(tb), tph ^ 1u, abort_flag)) { ok = false; break; }
                        if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                        tc_fence_after();
                        const uint32_t sa = smem_u32(smem + stage * S::kStageBytes);
                        const uint32_t sb = sa + S::kABytes;
                        const uint32_t d = tmem_base + (uint32_t)(tb * BN);
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const uint64_t ad = sdesc_sw128(sa + k * 32, 16, 1024);
                            const uint64_t bd = (MODE == kModeDgrad) ? sdesc_sw128(sb + k * 4096, 16384, 1024)
                                                                     : sdesc_sw128(sb + k * 32, 16, 1024);
                            mma_f8f6f4(d, ad, bd, idesc, k > 0 ? 1u : 0u);
                        }
                        tc_commit(empty_bar(stage));
                        tc_commit(tfull_bar(tb));
                    }
                    if (++stage == S::kStages) { stage = 0; phase ^= 1u; }
                    if (++tb == 2) { tb = 0; tph ^= 1u; }
                }
            }
            // Drain: every MMA both issuers started has completed before TMEM is released.
            tc_commit(drain_bar);
            if (warp == 1) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain_bar, 0) && globaltimer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
        if (warp == 1) {
            // Release TMEM once the promotion warps have read their last partial.
            named_bar_sync(1, 32 + S::kPromoThreads);
            tc_fence_after();
            tmem_dealloc(tmem_base, S::kTmemCols);
        }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(S::kRegsHigh));
        // ------------------------------------------------------------ promotion + epilogue
        const int pw = warp - 4;
        const int quad = warp & 3;            // TMEM lanes 32*quad .. 32*quad+31
        const int half = pw >> 2;             // column group: [half*kCols, (half+1)*kCols)
        const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
        const int rit = quad * 32 + lane;     // row within the tile
        const int ptid = pw * 32 + lane;      // promotion thread 0..255
        int tb = 0, ss = 0;
        uint32_t tph = 0, sph = 0;
        // Columns per TMEM load.  Each load is a round trip on the promotion's critical path,
        // so chunks are as wide as the registers allow: two 32-column chunks in flight beside
        // the accumulators (16 with four promotion warpgroups, whose threads have fewer registers).
        //
        // Wgrad multiplies every element by its own column's scale, which comes from shared
        // memory; with one row per thread each thread would need all its kCols column scales per K
        // group.  So Wgrad reads TMEM with the 16x256b shape instead: a thread holds 4 rows
        // (t/4 + 8i of the warp's 32) x 2 columns of every 8-column block, i.e. needs a quarter
        // of the column scales (an 8-byte load per block).  Its chunk is 32 columns: two
        // 16x256b.x4 loads (lanes +0 and +16) of 16 registers each, half the round trips of
        // 16-column chunks (104.8 against 106.8 us on the linear-layer Wgrad);
        // acc[kBlocks * i + j] is row i's column pair of block j.
        constexpr int kCW = (S::kCols < 32 || S::kPW == 4) ? 16 : 32;
        constexpr int kHalfW = kCW / 2;   // Wgrad: registers of one 16-lane load
        constexpr int kChunks = S::kCols / kCW;
        constexpr int kBlocks = S::kCols / 8;
        const int wt0 = lane & 3, wt1 = lane >> 2;   // Wgrad: column pair and first row of a thread
        float2 acc[S::kCols / 2];
        WorkSched wsched = sched_begin(args);
        WorkItem it;
        bool alive = true;
        while (alive && sched_next(wsched, num_tiles, KB, it)) {
            kgroup_range(it);
            const TileInfo ti = decode_tile<GROUPED, kKGrouped>(it.tile, nb_tiles, BN, args, g_off, g_pre);
            const int row = ti.row0 + rit;
            const bool in_a = row < args.M;
            const int ncol0 = ti.n0 + half * S::kCols;
            const float* sa_ptr = args.sA + (in_a ? row : 0);
            const float* sb_ptr = args.sB;
            size_t sb_step = 0;
            if (MODE == kModeFprop) {
                sb_ptr = args.sB + (size_t)ti.e * (size_t)(args.N >> 7) * KB + (size_t)(ncol0 >> 7) * KB;
                sb_step = 1;
            } else if (MODE == kModeDgrad) {
                sb_ptr = args.sB + (size_t)ti.e * (size_t)KB * (size_t)(args.N >> 7) + (ncol0 >> 7);
                sb_step = (size_t)(args.N >> 7);
            }
#pragma unroll
            for (int i = 0; i < S::kCols / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            // The row and block scales of the item's groups are pulled into L2 up front (one line
            // per group holds this warp's 32 row scales), so the per-group loads below, issued one
            // group ahead, find them there instead of in HBM.
            for (int k = it.kb0 + 1 + lane; !MX && k < it.kb1; k += 32) {
                prefetch_l2(args.sA + (size_t)k * args.M + min(ti.row0 + quad * 32, args.M - 1));
                if (MODE != kModeWgrad) prefetch_l2(sb_ptr + (size_t)k * sb_step);
            }
            float sa_next = (!MX && in_a) ? __ldg(sa_ptr + (size_t)it.kb0 * args.M) : 0.0f;
            float sb_next = (!MX && MODE != kModeWgrad) ? __ldg(sb_ptr + (size_t)it.kb0 * sb_step) : 1.0f;
            bool ok = true;
            if (MX) {
                // The item's whole K sits in the one TMEM accumulator: copy it into the registers
                // (same layouts as the promotion below: a row per thread, or for Wgrad 4 rows x 2
                // columns per 8-column block), two loads in flight, and hand the accumulator back
                // as soon as the last load has landed.
                if (!warp_wait(tfull_bar(0), tph, abort_flag)) {
                    ok = false;
                } else {
                    tc_fence_after();
                    const uint32_t taddr = tmem_base + lane_base + (uint32_t)(half * S::kCols);
                    const auto tload = [&](int ch, uint32_t (&r)[kCW]) {
                        if (MODE != kModeWgrad) {
                            tmem_ld_async(taddr + ch * kCW, r);
                        } else {
                            tmem_ld_16x256b<kCW / 8>(taddr + ch * kCW, r);
                            tmem_ld_16x256b<kCW / 8>(taddr + (16u << 16) + ch * kCW, r + kHalfW);
                        }
                    };
                    const auto take = [&](uint32_t (&cur)[kCW], int ch) {
                        if (MODE != kModeWgrad) {
#pragma unroll
                            for (int j = 0; j < kCW; j += 2)
                                acc[(ch * kCW + j) / 2] = make_float2(__uint_as_float(cur[j]), __uint_as_float(cur[j + 1]));
                        } else {
#pragma unroll
                            for (int b = 0; b < kCW / 8; ++b)
#pragma unroll
                                for (int h = 0; h < 2; ++h)
#pragma unroll
                                    for (int q = 0; q < 2; ++q) {
                                        const int r0 = kHalfW * h + 4 * b + 2 * q;
                                        acc[kBlocks * (2 * h + q) + (kCW / 8) * ch + b] =
                                            make_float2(__uint_as_float(cur[r0]), __uint_as_float(cur[r0 + 1]));
                                    }
                        }
                    };
                    uint32_t ra[kCW], rb[kCW];
                    tload(0, ra);
                    tmem_wait_ld(ra);
#pragma unroll
                    for (int ch = 0; ch < kChunks; ++ch) {
                        if (ch + 1 < kChunks) {
                            if (ch & 1) tload(ch + 1, ra);
                            else tload(ch + 1, rb);
                        } else {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(tempty_bar(0));
                        }
                        if (ch & 1) take(rb, ch); else take(ra, ch);
                        if (ch + 1 < kChunks) {
                            if (ch & 1) tmem_wait_ld(ra); else tmem_wait_ld(rb);
                        }
                    }
                    tph ^= 1u;
                }
            }
            for (int kb = it.kb0; !MX && kb < it.kb1; ++kb) {
                const float sa = sa_next, sbv = sb_next;
                if (kb + 1 < it.kb1) {
                    sa_next = in_a ? __ldg(sa_ptr + (size_t)(kb + 1) * args.M) : 0.0f;
                    if (MODE != kModeWgrad) sb_next = __ldg(sb_ptr + (size_t)(kb + 1) * sb_step);
                }
                if (!warp_wait(tfull_bar(tb), tph, abort_flag)) { ok = false; break; }
                if (MODE == kModeWgrad) {
                    if (!warp_wait(sfull_bar(ss), sph, abort_flag)) { ok = false; break; }
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + lane_base + (uint32_t)(tb * BN + half * S::kCols);
                const float* cs = col_scales + ss * BN + half * S::kCols;
                const float2 c2 = make_float2(sa * sbv, sa * sbv);
                // Wgrad: the row scales of this thread's 4 rows, from the lanes that loaded them.
                float2 sa2w[4];
                if (MODE == kModeWgrad) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float v = __shfl_sync(0xFFFFFFFFu, sa, wt1 + 8 * i);
                        sa2w[i] = make_float2(v, v);
                    }
                }
                const auto tload = [&](int ch, uint32_t (&r)[kCW]) {
                    if (MODE != kModeWgrad) {
                        tmem_ld_async(taddr + ch * kCW, r);
                    } else {
                        tmem_ld_16x256b<kCW / 8>(taddr + ch * kCW, r);
                        tmem_ld_16x256b<kCW / 8>(taddr + (16u << 16) + ch * kCW, r + kHalfW);
                    }
                };
                // Two register chunks: the TMEM load of chunk ch+1 is in flight while chunk ch is
                // folded into the accumulators.  The buffer is released as soon as its last
                // chunk has landed in registers, before that chunk's arithmetic.
                uint32_t ra[kCW], rb[kCW];
                tload(0, ra);
                tmem_wait_ld(ra);
                const auto fold = [&](uint32_t (&cur)[kCW], int ch) {
                    if (MODE != kModeWgrad) {
#pragma unroll
                        for (int j = 0; j < kCW; j += 2) {
                            const float2 v = make_float2(__uint_as_float(cur[j]), __uint_as_float(cur[j + 1]));
                            acc[(ch * kCW + j) / 2] = __ffma2_rn(v, c2, acc[(ch * kCW + j) / 2]);
                        }
                    } else {
                        // cur[kHalfW*h + 4b + 2q + {0,1}]: row wt1 + 8q + 16h, column pair of block
                        // (kCW/8)*ch + b.
#pragma unroll
                        for (int b = 0; b < kCW / 8; ++b) {
                            const int jb = (kCW / 8) * ch + b;
                            const float2 sc = *reinterpret_cast<const float2*>(cs + 8 * jb + 2 * wt0);
#pragma unroll
                            for (int h = 0; h < 2; ++h) {
#pragma unroll
                                for (int q = 0; q < 2; ++q) {
                                    const int i = 2 * h + q, r0 = kHalfW * h + 4 * b + 2 * q;
                                    const float2 v = make_float2(__uint_as_float(cur[r0]), __uint_as_float(cur[r0 + 1]));
                                    acc[kBlocks * i + jb] = __ffma2_rn(v, __fmul2_rn(sa2w[i], sc), acc[kBlocks * i + jb]);
                                }
                            }
                        }
                    }
                };
                const auto release = [&]() {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty_bar(tb));
                };
#pragma unroll
                for (int ch = 0; ch < kChunks; ++ch) {
                    if (ch + 1 < kChunks) {
                        if (ch & 1) tload(ch + 1, ra);
                        else tload(ch + 1, rb);
                    } else {
                        release();
                    }
                    if (ch & 1) fold(rb, ch); else fold(ra, ch);
                    if (ch + 1 < kChunks) {
                        if (ch & 1) tmem_wait_ld(ra); else tmem_wait_ld(rb);
                    }
                }
                if (MODE == kModeWgrad) {
                    // The column scales were read with ordinary loads; the next bulk copy into this
                    // slot is an async-proxy write, so fence the proxies before releasing it.
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(sempty_bar(ss));
                    if (++ss == S::kScaleStages) { ss = 0; sph ^= 1u; }
                }
                if (++tb == 2) { tb = 0; tph ^= 1u; }
            }
            if (!ok) break;
            if (wsched.sk && it.kb0 > 0) {
                // Leading partial of a tile that another CTA finishes: park it in this CTA's slot.
                // Only the same thread of the finishing CTA reads an entry back, so the slot is
                // interleaved by promotion thread: each warp store moves 512 contiguous bytes.
                float4* slot = reinterpret_cast<float4*>(args.ws + (size_t)blockIdx.x * (128 * BN)) + ptid;
#pragma unroll
                for (int j = 0; j < S::kCols / 2; j += 2)
                    __stcg(slot + (j / 2) * S::kPromoThreads, make_float4(acc[j].x, acc[j].y, acc[j + 1].x, acc[j + 1].y));
                __threadfence();
                __syncwarp();
                if (lane == 0) mbar_arrive(parked_bar);
                if (warp == 4 && lane == 0) {
                    // A CTA parks at most one partial per launch (its first item): phase 0.
                    if (mbar_wait(parked_bar, 0, abort_flag)) st_release_gpu(args.flags + blockIdx.x, args.stamp);
                }
                continue;
            }
            if (wsched.sk && it.kb1 < KB) {
                // This CTA owns group 0 of the tile: add, in CTA order, the partials of the CTAs
                // whose ranges start inside it (they computed them first, so the waits are short).
                const int64_t tile_end = (int64_t)(it.tile + 1) * KB;
                for (int j = (int)blockIdx.x + 1; j < (int)gridDim.x && sk_begin(args.units, j, gridDim.x) < tile_end;
                     ++j) {
                    bool ready = true;
                    if (lane == 0) ready = spin_flag(args.flags + j, args.stamp, abort_flag);
                    if (__shfl_sync(0xFFFFFFFFu, ready ? 1 : 0, 0) == 0) {
                        alive = false;
                        break;
                    }
                    __syncwarp();   // orders the lanes' loads of the slot after lane 0's acquire
                    const float4* slot = reinterpret_cast<const float4*>(args.ws + (size_t)j * (128 * BN)) + ptid;
#pragma unroll
                    for (int q = 0; q < S::kCols / 2; q += 2) {
                        const float4 v = __ldcg(slot + (q / 2) * S::kPromoThreads);
                        acc[q].x += v.x;
                        acc[q].y += v.y;
                        acc[q + 1].x += v.z;
                        acc[q + 1].y += v.w;
                    }
                }
                if (!alive) break;
            }
            // Epilogue.  The warp's 32 rows x kCols columns leave through 2 KB staging buffers in
            // shared memory, one 32-row x 64-byte slab at a time.  16-byte unit p of staged row r
            // sits at unit 4r + (p ^ ((r >> 1) & 3)) -- the tensor map's 64-byte swizzle, and
            // conflict-free for the row-per-lane writes.  Dense GEMMs hand each slab to a bulk
            // tensor store (rows past M are clipped by the tensor bounds); the grouped GEMM,
            // whose next rows belong to another group, stores the slab itself, 8 rows x 64
            // contiguous bytes per instruction, skipping rows at or past the group's end.
            {
                constexpr int kElt = (MODE == kModeWgrad) ? 4 : 2;    // bytes per output element
                constexpr int kSlabCols = 64 / kElt;
                uint4* stage0 = reinterpret_cast<uint4*>(smem + S::kOffEpi) + pw * 128 * S::kEpiBufs;
                const int wrow0 = ti.out_row0 + quad * 32;
                // Fused 1x128 quantisation: this thread's kCols = 128 columns of its row are one
                // group.  Its scale comes from the bf16-rounded outputs, as the activation
                // quantiser would see them in D.
                constexpr bool kCanQuant = (MODE != kModeWgrad) && !GROUPED && S::kCols == 128;
                const bool quant = kCanQuant && args.quant_out;
                float qinv = 0.0f;
                if (quant) {
                    float amax = 0.0f;
#pragma unroll
                    for (int i = 0; i < S::kCols / 2; ++i) {
                        const uint32_t h = pack_bf16x2(acc[i].x, acc[i].y);
                        amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(h)), fabsf(bf16_hi(h))));
                    }
                    float qs;
                    group_scale<MX>(amax, qs, qinv);
                    if (row < args.M) args.s_out[(size_t)(ncol0 >> 7) * (size_t)args.M + row] = qs;
                }
                const bool store_d = GROUPED || MODE == kModeWgrad || args.store_d;
                int nslab = 0;   // slabs staged so far (rotates the staging buffers)
#pragma unroll
                for (int sl = 0; sl < S::kCols / kSlabCols; ++sl) {
                    if (!store_d) break;
                    uint4* stage = stage0 + (nslab++ % S::kEpiBufs) * 128;
                    uint4 u[4];
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        if (MODE == kModeWgrad) {
                            u[p] = make_uint4(0u, 0u, 0u, 0u);   // Wgrad stages 8-byte pieces below
                        } else {
                            const int q = sl * 16 + 4 * p;
                            u[p] = make_uint4(pack_bf16x2(acc[q].x, acc[q].y), pack_bf16x2(acc[q + 1].x, acc[q + 1].y),
                                              pack_bf16x2(acc[q + 2].x, acc[q + 2].y),
                                              pack_bf16x2(acc[q + 3].x, acc[q + 3].y));
                        }
                    }
                    if (!kRowGrouped) {
                        // The buffer is free once the store issued from it kEpiBufs slabs ago has
                        // read it.
                        if (lane == 0) bulk_wait_group_read<S::kEpiBufs - 1>();
                        __syncwarp();
                    }
                    if (MODE == kModeWgrad) {
                        // Slab sl = blocks 2sl, 2sl+1 (16 fp32 columns).  This thread's pair of block
                        // 2sl + b in row r = wt1 + 8i is bytes 32b + 8*wt0 of the 64-byte staged row.
                        float2* st2 = reinterpret_cast<float2*>(stage);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int r = wt1 + 8 * i;
#pragma unroll
                            for (int b = 0; b < 2; ++b) {
                                const int unit = (2 * b + (wt0 >> 1)) ^ ((r >> 1) & 3);
                                st2[r * 8 + unit * 2 + (wt0 & 1)] = acc[kBlocks * i + 2 * sl + b];
                            }
                        }
                    } else {
                        const int wsw = (lane >> 1) & 3;
#pragma unroll
                        for (int p = 0; p < 4; ++p) stage[lane * 4 + (p ^ wsw)] = u[p];
                    }
                    if (!kRowGrouped) {
                        fence_proxy_async_smem();     // the writes above, before the async-proxy read
                        __syncwarp();
                        if (lane == 0) {
                            if (MODE == kModeWgrad && args.accumulate)
                                tma_reduce_add_2d(&tmD, smem_u32(stage), ncol0 + sl * kSlabCols, wrow0);
                            else
                                tma_store_2d(&tmD, smem_u32(stage), ncol0 + sl * kSlabCols, wrow0);
                            bulk_commit_group();
                        }
                    } else {
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int r = (lane >> 2) + 8 * i, p = lane & 3;
                            const uint4 v = stage[r * 4 + (p ^ ((r >> 1) & 3))];
                            const int grow = wrow0 + r;
                            if (grow < ti.row_end) {
                                uint8_t* dst = reinterpret_cast<uint8_t*>(args.D) +
                                               ((size_t)grow * args.N + ncol0 + sl * kSlabCols) * kElt + p * 16;
                                *reinterpret_cast<uint4*>(dst) = v;
                            }
                        }
                        __syncwarp();
                    }
                }
                if (kCanQuant && quant) {
                    // Codes: two 64-column slabs of E4M3 (64 bytes per row), through the same
                    // staging buffers and a tensor map over q_out.
#pragma unroll
                    for (int cs = 0; cs < 2; ++cs) {
                        uint4* stage = stage0 + (nslab++ % S::kEpiBufs) * 128;
                        uint4 u[4];
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            uint32_t wv[4];
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                const int c = cs * 32 + p * 8 + 2 * k;   // float2 index: columns 2c, 2c+1 and 2c+2, 2c+3
                                const uint32_t h0 = pack_bf16x2(acc[c].x, acc[c].y);
                                const uint32_t h1 = pack_bf16x2(acc[c + 1].x, acc[c + 1].y);
                                wv[k] = e4m3x2(__fmul_rn(bf16_lo(h0), qinv), __fmul_rn(bf16_hi(h0), qinv)) |
                                        (e4m3x2(__fmul_rn(bf16_lo(h1), qinv), __fmul_rn(bf16_hi(h1), qinv)) << 16);
                            }
                            u[p] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
                        }
                        if (lane == 0) bulk_wait_group_read<S::kEpiBufs - 1>();
                        __syncwarp();
                        const int wsw = (lane >> 1) & 3;
#pragma unroll
                        for (int p = 0; p < 4; ++p) stage[lane * 4 + (p ^ wsw)] = u[p];
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmQ, smem_u32(stage), ncol0 + cs * 64, wrow0);
                            bulk_commit_group();
                        }
                    }
                }
            }
        }
        // Every store has finished reading shared memory and writing its tile before the CTA
        // (and its shared memory) goes away.
        if (!kRowGrouped && lane == 0) bulk_wait_group<0>();
        __syncwarp();
        tc_fence_before();
        named_bar_arrive(1, 32 + S::kPromoThreads);
    }

}

}  // namespace fp8q
