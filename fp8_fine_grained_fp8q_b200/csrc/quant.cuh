// quant.cuh -- E4M3 group quantisers (HBM-bound streaming kernels).
//
// Group scaling follows the "DeepSeek-V3 Technical Report" summary page (Key ideas, FP8
// mixed-precision bullet): 1x128 tiles for activations, 128x128 blocks for weights; the
// 128x1 token-direction form serves Wgrad, whose inner dimension is the token dimension
// (DeepSeek-V3 report repost, paragraph 4: scaling groups along the GEMM's inner dimension).
//
// Per group: a = max(amax, 2^-100); s = a / 448 (stored); q = E4M3(x * (448 / a)), all IEEE
// binary32 with round-to-nearest (explicit __fdiv_rn / __fmul_rn, so no fast-math flag can
// change them); the conversion is cvt.rn.satfinite.e4m3x2.f32 (nearest-even, saturating).
#pragma once

#include <stdint.h>

#include "ptx.cuh"

namespace fp8q {

constexpr float kE4M3Max = 448.0f;
constexpr float kAmaxFloor = 0x1p-100f;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two E4M3 codes packed little-endian: `first` in the low byte (lower address).
__device__ __forceinline__ uint32_t e4m3x2(float first, float second)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(second), "f"(first));
    return r;
}

__device__ __forceinline__ float amax8(const uint4& v)
{
    float m = fabsf(bf16_lo(v.x));
    m = fmaxf(m, fabsf(bf16_hi(v.x)));
    m = fmaxf(m, fabsf(bf16_lo(v.y)));
    m = fmaxf(m, fabsf(bf16_hi(v.y)));
    m = fmaxf(m, fabsf(bf16_lo(v.z)));
    m = fmaxf(m, fabsf(bf16_hi(v.z)));
    m = fmaxf(m, fabsf(bf16_lo(v.w)));
    m = fmaxf(m, fabsf(bf16_hi(v.w)));
    return m;
}

// 8 bf16 values times `inv` -> 8 E4M3 codes.
__device__ __forceinline__ uint2 quant8(const uint4& v, float inv)
{
    uint2 o;
    o.x = e4m3x2(__fmul_rn(bf16_lo(v.x), inv), __fmul_rn(bf16_hi(v.x), inv)) |
          (e4m3x2(__fmul_rn(bf16_lo(v.y), inv), __fmul_rn(bf16_hi(v.y), inv)) << 16);
    o.y = e4m3x2(__fmul_rn(bf16_lo(v.z), inv), __fmul_rn(bf16_hi(v.z), inv)) |
          (e4m3x2(__fmul_rn(bf16_lo(v.w), inv), __fmul_rn(bf16_hi(v.w), inv)) << 16);
    return o;
}

// POW2 = false: the max-abs scale s = a / 448.  POW2 = true (the UE8M0 variant, a separate
// mode): s = the smallest power of two not below the binary32 quotient r = a / 448, which the
// block-scaled tensor-core MMA can take as an 8-bit exponent; 1 / s is then an exact power of
// two too.  r lies in [2^-109, 2^120), a normal binary32 number, so s and 1 / s are formed
// directly from its biased exponent (rounded up when r has a nonzero fraction).
template <bool POW2>
__device__ __forceinline__ void group_scale(float amax, float& s, float& inv)
{
    const float a = fmaxf(amax, kAmaxFloor);
    if (POW2) {
        const uint32_t r = __float_as_uint(__fdiv_rn(a, kE4M3Max));
        const uint32_t e = (r >> 23) + ((r & 0x7FFFFFu) != 0u ? 1u : 0u);
        s = __uint_as_float(e << 23);
        inv = __uint_as_float((254u - e) << 23);
    } else {
        s = __fdiv_rn(a, kE4M3Max);
        inv = __fdiv_rn(kE4M3Max, a);
    }
}

// ------------------------------------------------------------------------------------------
// 1x128: x[M,K] -> q[M,K], s[K/128][M].  Eight lanes own one tile (8 x 32 B = 256 B of bf16,
// 16 values per lane), so a warp covers 4 consecutive tiles = 1 KB of contiguous input per
// load; the max-abs needs 3 shuffle levels.  Each lane keeps UNR tile-groups of loads in
// flight.  Tiles are visited row-major so the reads stream through HBM sequentially; all index
// arithmetic is 32-bit (the host guarantees M * K/128 < 2^31).
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float amax16(const uint4& a, const uint4& b)
{
    return fmaxf(amax8(a), amax8(b));
}

template <int UNR, bool POW2>
__global__ void __launch_bounds__(256) act_1x128_kernel(const uint16_t* __restrict__ x,
                                                        uint8_t* __restrict__ q,
                                                        float* __restrict__ s, int M, int K)
{
    griddep_launch_dependents();
    griddep_wait();
    const uint32_t KB = (uint32_t)K >> 7;
    const uint32_t ntiles = (uint32_t)M * KB;
    const uint32_t sub = threadIdx.x & 7;                       // lane within the tile
    const uint32_t g8 = ((uint32_t)blockIdx.x * blockDim.x + threadIdx.x) >> 3;   // 8-lane group
    const uint32_t ng8 = ((uint32_t)gridDim.x * blockDim.x) >> 3;

    for (uint32_t base = g8; base < ntiles; base += ng8 * UNR) {
        uint4 v[UNR][2];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const uint32_t t = base + (uint32_t)u * ng8;
            v[u][0] = make_uint4(0u, 0u, 0u, 0u);
            v[u][1] = make_uint4(0u, 0u, 0u, 0u);
            if (t < ntiles) {
                // Tile t = (m, kb) row-major is the 256 B at element offset t * 128.
                const uint4* p = reinterpret_cast<const uint4*>(x + (size_t)t * 128) + 2 * sub;
                v[u][0] = __ldg(p);
                v[u][1] = __ldg(p + 1);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const uint32_t t = base + (uint32_t)u * ng8;
            float amax = amax16(v[u][0], v[u][1]);
            // All 32 lanes take part in the shuffles even when an 8-lane group has no tile.
#pragma unroll
            for (int o = 4; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            float sc, inv;
            group_scale<POW2>(amax, sc, inv);
            if (t < ntiles) {
                const uint2 lo = quant8(v[u][0], inv), hi = quant8(v[u][1], inv);
                reinterpret_cast<uint4*>(q + (size_t)t * 128)[sub] = make_uint4(lo.x, lo.y, hi.x, hi.y);
                if (sub == 0) {
                    const uint32_t m = t / KB, kb = t - m * KB;
                    s[(size_t)kb * M + m] = sc;
                }
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// 128x1 with transposed output: x[T,C] -> qt[C,T], s[T/128][C].  One CTA per 128-token x
// 64-channel tile.  Warp w reads tokens 16w .. 16w+15; lane l owns channels 2l, 2l+1, so each
// 4-byte load of the warp is one coalesced 128-byte row segment and the thread ends up holding
// its 16 tokens x 2 channels in registers (the transpose happens in registers, not in shared
// memory).  Only the per-channel max-abs crosses warps, through a small shared reduction; then
// each thread converts its values and writes 16 consecutive tokens of each of its two channels
// as one 16-byte store each.
// ------------------------------------------------------------------------------------------
// The transposed codes of a tile leave through shared memory: 16-byte unit u (tokens 16u ..
// 16u+15) of code row r sits at unit u ^ ((r >> kSh) & 7) of the row's 128 bytes, so that both the
// per-thread 16-token writes and the whole-row reads are free of bank conflicts, and every row's
// 128 tokens then go out as one 128-byte line (a warp instruction stores 4 rows).  Written as
// scattered 16-byte pieces instead (each line by 8 warps), the 128x1 quantiser of X [4096, 7168]
// ran at 4.55 against 5.97 TB/s.
template <int kSh>
__device__ __forceinline__ int qt_unit(int row, int u) { return row * 8 + (u ^ ((row >> kSh) & 7)); }

// Rows [row0, row0 + 4 * N) of a staged code tile (laid out by qt_unit<kSh>), 4 rows per warp
// instruction, to qt (row pitch `pitch` bytes, first token column col0).
template <int kSh, int N>
__device__ __forceinline__ void qt_store_rows(const uint4* qs, int row0, uint8_t* __restrict__ qt, int64_t c0,
                                              int64_t pitch, int64_t col0, int lane)
{
#pragma unroll
    for (int k = 0; k < N; ++k) {
        const int row = row0 + 4 * k + (lane >> 3), u = lane & 7;
        *reinterpret_cast<uint4*>(qt + (c0 + row) * pitch + col0 + 16 * u) = qs[qt_unit<kSh>(row, u)];
    }
}

constexpr int kT1Tok = 128;
constexpr int kT1Ch = 64;

template <bool POW2>
__global__ void __launch_bounds__(256) act_128x1_t_kernel(const uint16_t* __restrict__ x,
                                                          uint8_t* __restrict__ qt,
                                                          float* __restrict__ s, int64_t T, int64_t C)
{
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float red[8][kT1Ch];
    __shared__ float inv_c[kT1Ch];
    __shared__ __align__(16) uint4 qs[kT1Ch * 8];   // the tile's codes, [channel][128 tokens]

    const int64_t c0 = (int64_t)blockIdx.x * kT1Ch;
    const int64_t tb = blockIdx.y;
    const int64_t t0 = tb * kT1Tok;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Tokens t0 + 16w + i, channels c0 + 2*lane (low half) and c0 + 2*lane + 1 (high half).
    const uint32_t* src = reinterpret_cast<const uint32_t*>(x + (t0 + 16 * w) * C + c0) + lane;
    uint32_t v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __ldg(src + (size_t)i * (size_t)(C >> 1));
    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        m0 = fmaxf(m0, fabsf(bf16_lo(v[i])));
        m1 = fmaxf(m1, fabsf(bf16_hi(v[i])));
    }
    red[w][2 * lane] = m0;
    red[w][2 * lane + 1] = m1;
    __syncthreads();
    if (threadIdx.x < kT1Ch) {
        float a = red[0][threadIdx.x];
#pragma unroll
        for (int k = 1; k < 8; ++k) a = fmaxf(a, red[k][threadIdx.x]);
        float sc, inv;
        group_scale<POW2>(a, sc, inv);
        s[tb * C + c0 + threadIdx.x] = sc;
        inv_c[threadIdx.x] = inv;
    }
    __syncthreads();
    const float inv0 = inv_c[2 * lane], inv1 = inv_c[2 * lane + 1];
    uint32_t q0[4], q1[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        q0[p] = e4m3x2(__fmul_rn(bf16_lo(v[4 * p + 0]), inv0), __fmul_rn(bf16_lo(v[4 * p + 1]), inv0)) |
                (e4m3x2(__fmul_rn(bf16_lo(v[4 * p + 2]), inv0), __fmul_rn(bf16_lo(v[4 * p + 3]), inv0)) << 16);
        q1[p] = e4m3x2(__fmul_rn(bf16_hi(v[4 * p + 0]), inv1), __fmul_rn(bf16_hi(v[4 * p + 1]), inv1)) |
                (e4m3x2(__fmul_rn(bf16_hi(v[4 * p + 2]), inv1), __fmul_rn(bf16_hi(v[4 * p + 3]), inv1)) << 16);
    }
    qs[qt_unit<1>(2 * lane, w)] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
    qs[qt_unit<1>(2 * lane + 1, w)] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
    __syncthreads();
    qt_store_rows<1, 2>(qs, 8 * w, qt, c0, T, t0, lane);
}

// ------------------------------------------------------------------------------------------
// 128x1 with transposed output over expert-grouped rows (the grouped Wgrad operands).  Rows
// offsets[e] .. offsets[e+1]-1 of x[Mtot, C] are expert e's tokens.  Expert e's 128-token groups
// start at its first row; a final partial group takes its max-abs over the tokens it has.  In
// the transposed output qt[C, Kcap] the expert's tokens start at column 128 * P[e],
// P[e] = sum over e' < e of ceil(n_e' / 128), and the rest of its last group holds zero codes;
// st[Kcap/128][C].  CTA (x, y): padded group g = y, channel blocks 8x .. 8x+7 of 64 channels.
// Each CTA rebuilds P from the offsets (validated: 0-based, nondecreasing, ending at Mtot, and
// P[E] <= Kcap/128; otherwise FP8Q_DEV_BAD_OFFSETS is latched and nothing is written).
// ------------------------------------------------------------------------------------------
constexpr int kRgMaxGroups = 1024;
constexpr int kRgChunk = 8;   // 64-channel blocks per CTA

template <bool POW2>
__global__ void __launch_bounds__(256) act_128x1_t_ragged_kernel(const uint16_t* __restrict__ x,
                                                                 const int32_t* __restrict__ offsets, int E,
                                                                 int64_t Mtot, int64_t C, uint8_t* __restrict__ qt,
                                                                 float* __restrict__ s, int64_t Kcap)
{
    griddep_launch_dependents();
    griddep_wait();
    __shared__ int s_off[kRgMaxGroups + 1];
    __shared__ int s_pre[kRgMaxGroups + 1];
    __shared__ float red[8][kT1Ch];
    __shared__ float inv_c[kT1Ch];
    __shared__ __align__(16) uint4 qs[kT1Ch * 8];   // one channel block's codes, [channel][128 tokens]
    __shared__ int s_bad;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (w == 0) {
        for (int i = lane; i <= E; i += 32) s_off[i] = __ldg(offsets + i);
        __syncwarp();
        const int per = (E + 31) >> 5;
        const int lo = min(E, lane * per), hi = min(E, lo + per);
        int local = 0;
        bool bad = false;
        for (int e = lo; e < hi; ++e) {
            const int cnt = s_off[e + 1] - s_off[e];
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
            s_pre[e] = run;
            const int cnt = s_off[e + 1] - s_off[e];
            run += cnt > 0 ? (cnt + 127) >> 7 : 0;
        }
        if (lane == 31) s_pre[E] = incl;
        const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);   // padded groups of all experts
        if (lane == 0) bad |= (s_off[0] != 0) || ((int64_t)s_off[E] != Mtot) || ((int64_t)total * 128 > Kcap);
        bad = __any_sync(0xFFFFFFFFu, bad);
        if (lane == 0) s_bad = bad ? 1 : 0;
    }
    __syncthreads();
    if (s_bad) {
        if (threadIdx.x == 0) latch_status(2 /* FP8Q_DEV_BAD_OFFSETS */);
        return;
    }
    const int g = blockIdx.y;
    if (g >= s_pre[E]) return;
    int lo = 0, hi = E;   // s_pre[lo] <= g < s_pre[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_pre[mid] <= g) lo = mid; else hi = mid;
    }
    const int64_t r0 = (int64_t)s_off[lo] + 128ll * (g - s_pre[lo]);
    const int nvalid = (int)min((int64_t)128, (int64_t)s_off[lo + 1] - r0);

    for (int j = 0; j < kRgChunk; ++j) {
        const int64_t c0 = ((int64_t)blockIdx.x * kRgChunk + j) * kT1Ch;
        if (c0 >= C) break;
        // Tokens 16w + i of the group, channels c0 + 2*lane and + 1; tokens past the expert's
        // end read as zero.
        const uint32_t* src = reinterpret_cast<const uint32_t*>(x + (r0 + 16 * w) * C + c0) + lane;
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = (16 * w + i < nvalid) ? __ldg(src + (size_t)i * (size_t)(C >> 1)) : 0u;
        float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            m0 = fmaxf(m0, fabsf(bf16_lo(v[i])));
            m1 = fmaxf(m1, fabsf(bf16_hi(v[i])));
        }
        red[w][2 * lane] = m0;
        red[w][2 * lane + 1] = m1;
        __syncthreads();
        if (threadIdx.x < kT1Ch) {
            float a = red[0][threadIdx.x];
#pragma unroll
            for (int k = 1; k < 8; ++k) a = fmaxf(a, red[k][threadIdx.x]);
            float sc, inv;
            group_scale<POW2>(a, sc, inv);
            s[(int64_t)g * C + c0 + threadIdx.x] = sc;
            inv_c[threadIdx.x] = inv;
        }
        __syncthreads();
        const float inv0 = inv_c[2 * lane], inv1 = inv_c[2 * lane + 1];
        uint32_t q0[4], q1[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            q0[p] = e4m3x2(__fmul_rn(bf16_lo(v[4 * p + 0]), inv0), __fmul_rn(bf16_lo(v[4 * p + 1]), inv0)) |
                    (e4m3x2(__fmul_rn(bf16_lo(v[4 * p + 2]), inv0), __fmul_rn(bf16_lo(v[4 * p + 3]), inv0)) << 16);
            q1[p] = e4m3x2(__fmul_rn(bf16_hi(v[4 * p + 0]), inv1), __fmul_rn(bf16_hi(v[4 * p + 1]), inv1)) |
                    (e4m3x2(__fmul_rn(bf16_hi(v[4 * p + 2]), inv1), __fmul_rn(bf16_hi(v[4 * p + 3]), inv1)) << 16);
        }
        qs[qt_unit<1>(2 * lane, w)] = make_uint4(q0[0], q0[1], q0[2], q0[3]);
        qs[qt_unit<1>(2 * lane + 1, w)] = make_uint4(q1[0], q1[1], q1[2], q1[3]);
        __syncthreads();
        qt_store_rows<1, 2>(qs, 8 * w, qt, c0, Kcap, (int64_t)g * 128, lane);
        __syncthreads();   // red, inv_c and qs are rewritten by the next channel block
    }
}

// ------------------------------------------------------------------------------------------
// Both activation forms in one pass: x[T,C] -> (q[T,C], s[C/128][T]) as the 1x128 kernel and
// (qt[C,T], st[T/128][C]) as the 128x1 kernel, reading x once.  One CTA per 128-token x
// 128-channel tile, which is a whole group in both directions.  Warp w holds tokens
// 16w .. 16w+15; lane l holds channels 4l .. 4l+3 (one 8-byte load per token row, 256 B per
// warp instruction).  Column max-abs: per thread over its 16 tokens, then across warps in
// shared memory.  Row max-abs: a shuffle reduce-scatter (16 -> 8 -> 4 -> 2 -> 1 values per
// lane, then one all-reduce step) leaves the maximum of row 16w + (l >> 1) on lanes 2r, 2r+1.
// Codes: rows as 4-byte stores (128 B per warp row), columns as 16-byte stores of 16 tokens.
// ------------------------------------------------------------------------------------------
// One 128x128 tile (column block cb, token block tb) of the dual quantiser; red [8][128] and
// inv_c [128] are this CTA's shared scratch.
template <bool POW2>
__device__ __forceinline__ void act_dual_tile(const uint16_t* __restrict__ x, uint8_t* __restrict__ q,
                                              float* __restrict__ s, uint8_t* __restrict__ qt,
                                              float* __restrict__ st, int64_t T, int64_t C, int64_t cb,
                                              int64_t tb, float (*red)[128], float* inv_c, uint4* qs)
{
    const int64_t c0 = cb * 128, t0 = tb * 128;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t trow = t0 + 16 * w;

    const uint2* src = reinterpret_cast<const uint2*>(x + trow * C + c0) + lane;
    uint2 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __ldg(src + (size_t)i * (size_t)(C >> 2));

    float cm0 = 0.0f, cm1 = 0.0f, cm2 = 0.0f, cm3 = 0.0f, rm[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float a0 = fabsf(bf16_lo(v[i].x)), a1 = fabsf(bf16_hi(v[i].x));
        const float a2 = fabsf(bf16_lo(v[i].y)), a3 = fabsf(bf16_hi(v[i].y));
        cm0 = fmaxf(cm0, a0);
        cm1 = fmaxf(cm1, a1);
        cm2 = fmaxf(cm2, a2);
        cm3 = fmaxf(cm3, a3);
        rm[i] = fmaxf(fmaxf(a0, a1), fmaxf(a2, a3));
    }
    *reinterpret_cast<float4*>(&red[w][4 * lane]) = make_float4(cm0, cm1, cm2, cm3);

    // Row max-abs reduce-scatter: at the step with lane bit b, a lane keeps the half of its
    // rows selected by that bit and sends the other half to its partner.
    {
        const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float send = b4 ? rm[i] : rm[i + 8], keep = b4 ? rm[i + 8] : rm[i];
            rm[i] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 16));
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = b3 ? rm[i] : rm[i + 4], keep = b3 ? rm[i + 4] : rm[i];
            rm[i] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 8));
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = b2 ? rm[i] : rm[i + 2], keep = b2 ? rm[i + 2] : rm[i];
            rm[i] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 4));
        }
        {
            const float send = b1 ? rm[0] : rm[1], keep = b1 ? rm[1] : rm[0];
            rm[0] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, 2));
        }
        rm[0] = fmaxf(rm[0], __shfl_xor_sync(0xFFFFFFFFu, rm[0], 1));
    }
    float rsc, rinv;
    group_scale<POW2>(rm[0], rsc, rinv);                      // row 16w + (lane >> 1)
    if (!(lane & 1)) s[cb * T + trow + (lane >> 1)] = rsc;

    __syncthreads();
    if (threadIdx.x < 128) {
        float a = red[0][threadIdx.x];
#pragma unroll
        for (int k = 1; k < 8; ++k) a = fmaxf(a, red[k][threadIdx.x]);
        float sc, inv;
        group_scale<POW2>(a, sc, inv);
        st[tb * C + c0 + threadIdx.x] = sc;
        inv_c[threadIdx.x] = inv;
    }

    // Row-wise codes.
    uint8_t* qrow = q + trow * C + c0 + 4 * lane;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float ri = __shfl_sync(0xFFFFFFFFu, rinv, 2 * i);
        const uint32_t word =
            e4m3x2(__fmul_rn(bf16_lo(v[i].x), ri), __fmul_rn(bf16_hi(v[i].x), ri)) |
            (e4m3x2(__fmul_rn(bf16_lo(v[i].y), ri), __fmul_rn(bf16_hi(v[i].y), ri)) << 16);
        *reinterpret_cast<uint32_t*>(qrow + (size_t)i * (size_t)C) = word;
    }

    __syncthreads();
    const float4 ic = *reinterpret_cast<const float4*>(&inv_c[4 * lane]);
    uint32_t c[4][4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint2 a = v[4 * p], b = v[4 * p + 1], d = v[4 * p + 2], e = v[4 * p + 3];
        c[0][p] = e4m3x2(__fmul_rn(bf16_lo(a.x), ic.x), __fmul_rn(bf16_lo(b.x), ic.x)) |
                  (e4m3x2(__fmul_rn(bf16_lo(d.x), ic.x), __fmul_rn(bf16_lo(e.x), ic.x)) << 16);
        c[1][p] = e4m3x2(__fmul_rn(bf16_hi(a.x), ic.y), __fmul_rn(bf16_hi(b.x), ic.y)) |
                  (e4m3x2(__fmul_rn(bf16_hi(d.x), ic.y), __fmul_rn(bf16_hi(e.x), ic.y)) << 16);
        c[2][p] = e4m3x2(__fmul_rn(bf16_lo(a.y), ic.z), __fmul_rn(bf16_lo(b.y), ic.z)) |
                  (e4m3x2(__fmul_rn(bf16_lo(d.y), ic.z), __fmul_rn(bf16_lo(e.y), ic.z)) << 16);
        c[3][p] = e4m3x2(__fmul_rn(bf16_hi(a.y), ic.w), __fmul_rn(bf16_hi(b.y), ic.w)) |
                  (e4m3x2(__fmul_rn(bf16_hi(d.y), ic.w), __fmul_rn(bf16_hi(e.y), ic.w)) << 16);
    }
    // Channels c0 + 4*lane + j, tokens trow .. trow+15: staged, then written as whole 128-token rows.
#pragma unroll
    for (int j = 0; j < 4; ++j) qs[qt_unit<2>(4 * lane + j, w)] = make_uint4(c[j][0], c[j][1], c[j][2], c[j][3]);
    __syncthreads();
    qt_store_rows<2, 4>(qs, 16 * w, qt, c0, T, t0, lane);
}

template <bool POW2>
__global__ void __launch_bounds__(256, 3) act_dual_kernel(const uint16_t* __restrict__ x,
                                                       uint8_t* __restrict__ q, float* __restrict__ s,
                                                       uint8_t* __restrict__ qt, float* __restrict__ st,
                                                       int64_t T, int64_t C)
{
    griddep_launch_dependents();
    griddep_wait();
    __shared__ __align__(16) float red[8][128];
    __shared__ __align__(16) float inv_c[128];
    __shared__ __align__(16) uint4 qs[128 * 8];   // the tile's transposed codes, [channel][128 tokens]
    act_dual_tile<POW2>(x, q, s, qt, st, T, C, blockIdx.x, blockIdx.y, red, inv_c, qs);
}

// ------------------------------------------------------------------------------------------
// 128x128: w[N,K] -> q[N,K], s[N/128][K/128] (+ optional qt[K,N]).  One CTA per block; each
// thread holds 64 of the block's 16384 values in registers, so the block is read once.
// ------------------------------------------------------------------------------------------
// One 128x128 block (column block kb, row block nb) of the weight quantiser; red [8] and
// codes [128][144] are this CTA's shared scratch (codes only when qt is requested).
template <bool POW2>
__device__ __forceinline__ void weight_tile(const uint16_t* __restrict__ w, uint8_t* __restrict__ q,
                                            float* __restrict__ s, uint8_t* __restrict__ qt, int64_t N,
                                            int64_t K, int64_t kb, int64_t nb, float* red,
                                            uint8_t (*codes)[128 + 16])
{
    const int64_t KB = K >> 7;
    const int tid = threadIdx.x;
    const uint16_t* wb = w + nb * 128 * K + kb * 128;

    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int idx = tid + 256 * i;
        const int r = idx >> 4, c16 = idx & 15;
        v[i] = __ldg(reinterpret_cast<const uint4*>(wb + (int64_t)r * K) + c16);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, amax8(v[i]));
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
    float sc, inv;
    group_scale<POW2>(amax, sc, inv);
    if (tid == 0) s[nb * KB + kb] = sc;

    uint8_t* qb = q + nb * 128 * K + kb * 128;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int idx = tid + 256 * i;
        const int r = idx >> 4, c16 = idx & 15;
        const uint2 o = quant8(v[i], inv);
        reinterpret_cast<uint2*>(qb + (int64_t)r * K)[c16] = o;
        if (qt) *reinterpret_cast<uint2*>(&codes[r][c16 * 8]) = o;
    }
    if (qt) {
        __syncthreads();
        // Thread -> (k = tid / 2, half of the 128 n): 64 codes of column k gathered into 4 x 16 B.
        const int k = tid >> 1, nh = (tid & 1) * 64;
        uint8_t* dst = qt + (kb * 128 + k) * N + nb * 128 + nh;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            uint32_t wv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int n = nh + 16 * p + 4 * u;
                wv[u] = (uint32_t)codes[n][k] | ((uint32_t)codes[n + 1][k] << 8) |
                        ((uint32_t)codes[n + 2][k] << 16) | ((uint32_t)codes[n + 3][k] << 24);
            }
            reinterpret_cast<uint4*>(dst)[p] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
    }
}

template <bool POW2>
__global__ void __launch_bounds__(256) weight_128x128_kernel(const uint16_t* __restrict__ w,
                                                             uint8_t* __restrict__ q,
                                                             float* __restrict__ s,
                                                             uint8_t* __restrict__ qt, int64_t N, int64_t K)
{
    griddep_launch_dependents();
    griddep_wait();
    __shared__ float red[8];
    __shared__ __align__(16) uint8_t codes[128][128 + 16];
    weight_tile<POW2>(w, q, s, qt, N, K, blockIdx.x, blockIdx.y, red, codes);
}

// ------------------------------------------------------------------------------------------
// The forward operands of a linear layer Y = X W^T in one launch: x[T,C] to both activation
// forms (as act_dual_kernel) and w[N,C] to 128x128 blocks (as weight_128x128_kernel).  CTA b
// takes dual tile b (token-block-major) while b < tiles_x, then weight block b - tiles_x; one
// grid instead of two saves a launch and a partly filled last wave.
// ------------------------------------------------------------------------------------------
template <bool POW2>
__global__ void __launch_bounds__(256, 3) forward_operands_kernel(
    const uint16_t* __restrict__ x, uint8_t* __restrict__ xq, float* __restrict__ xs, uint8_t* __restrict__ xqt,
    float* __restrict__ xst, int64_t T, int64_t C, const uint16_t* __restrict__ w, uint8_t* __restrict__ wq,
    float* __restrict__ ws, uint8_t* __restrict__ wqt, int64_t N)
{
    griddep_launch_dependents();
    griddep_wait();
    // Dual tile: staged transposed codes (16 KB), then red (4 KB) and inv_c.  Weight block: codes
    // (128 x 144 B) and its reduction slots.
    __shared__ __align__(16) uint8_t scratch[16384 + 8 * 128 * 4 + 128 * 4];
    static_assert(16384 + 8 * 128 * 4 + 128 * 4 >= 128 * (128 + 16) + 8 * 4, "weight block scratch");
    const int64_t CB = C >> 7;
    const int64_t tiles_x = CB * (T >> 7);
    const int64_t b = blockIdx.x;
    if (b < tiles_x) {
        uint4* qs = reinterpret_cast<uint4*>(scratch);
        float (*red)[128] = reinterpret_cast<float (*)[128]>(scratch + 16384);
        float* inv_c = reinterpret_cast<float*>(scratch + 16384 + 8 * 128 * 4);
        act_dual_tile<POW2>(x, xq, xs, xqt, xst, T, C, b % CB, b / CB, red, inv_c, qs);
    } else {
        const int64_t bw = b - tiles_x;
        uint8_t (*codes)[128 + 16] = reinterpret_cast<uint8_t (*)[128 + 16]>(scratch);
        float* red = reinterpret_cast<float*>(scratch + 128 * (128 + 16));
        weight_tile<POW2>(w, wq, ws, wqt, N, C, bw % CB, bw / CB, red, codes);
    }
}

}  // namespace fp8q
