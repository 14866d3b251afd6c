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

__device__ __forceinline__ void group_scale(float amax, float& s, float& inv)
{
    const float a = fmaxf(amax, kAmaxFloor);
    s = __fdiv_rn(a, kE4M3Max);
    inv = __fdiv_rn(kE4M3Max, a);
}

// ------------------------------------------------------------------------------------------
// 1x128: x[M,K] -> q[M,K], s[K/128][M].  A half-warp owns one tile (16 lanes x 16 B = 256 B of
// bf16); each lane keeps UNR tiles' loads in flight.  Tiles are visited in row-major order so
// the reads stream through HBM sequentially.
// ------------------------------------------------------------------------------------------
template <int UNR>
__global__ void __launch_bounds__(256) act_1x128_kernel(const uint16_t* __restrict__ x,
                                                        uint8_t* __restrict__ q,
                                                        float* __restrict__ s, int64_t M, int64_t K)
{
    const int64_t KB = K >> 7;
    const int64_t ntiles = M * KB;
    const int sub = threadIdx.x & 15;
    const int64_t hw = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int64_t nhw = ((int64_t)gridDim.x * blockDim.x) >> 4;

    for (int64_t base = hw; base < ntiles; base += nhw * UNR) {
        uint4 v[UNR];
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int64_t t = base + (int64_t)u * nhw;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (t < ntiles) {
                const int64_t m = t / KB, kb = t - m * KB;
                v[u] = __ldg(reinterpret_cast<const uint4*>(x + m * K + kb * 128) + sub);
            }
        }
#pragma unroll
        for (int u = 0; u < UNR; ++u) {
            const int64_t t = base + (int64_t)u * nhw;
            float amax = amax8(v[u]);
            // All 32 lanes take part in the shuffles even when one half-warp has no tile.
#pragma unroll
            for (int o = 8; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
            float sc, inv;
            group_scale(amax, sc, inv);
            if (t < ntiles) {
                const int64_t m = t / KB, kb = t - m * KB;
                reinterpret_cast<uint2*>(q + m * K + kb * 128)[sub] = quant8(v[u], inv);
                if (sub == 0) s[kb * M + m] = sc;
            }
        }
    }
}

// ------------------------------------------------------------------------------------------
// 128x1 with transposed output: x[T,C] -> qt[C,T], s[T/128][C].  One CTA per 128-token x
// 64-channel tile: coalesced 16 B row loads into shared memory, column max-abs by warps that
// each scan every 8th token (lanes = channel pairs, conflict-free), then each thread writes
// 16 consecutive tokens of one channel as one 16 B store.
// ------------------------------------------------------------------------------------------
constexpr int kT1Tok = 128;
constexpr int kT1Ch = 64;
constexpr int kT1Pitch = kT1Ch + 8;   // bf16 elements per shared row (144 B, 16 B aligned)

__global__ void __launch_bounds__(256) act_128x1_t_kernel(const uint16_t* __restrict__ x,
                                                          uint8_t* __restrict__ qt,
                                                          float* __restrict__ s, int64_t T, int64_t C)
{
    __shared__ __align__(16) uint16_t tile[kT1Tok][kT1Pitch];
    __shared__ float red[8][kT1Ch];
    __shared__ float inv_c[kT1Ch];

    const int64_t c0 = (int64_t)blockIdx.x * kT1Ch;
    const int64_t tb = blockIdx.y;
    const int64_t t0 = tb * kT1Tok;
    const int tid = threadIdx.x;

    uint4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int idx = tid + 256 * i;
        const int r = idx >> 3, c8 = idx & 7;
        v[i] = __ldg(reinterpret_cast<const uint4*>(x + (t0 + r) * C + c0) + c8);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int idx = tid + 256 * i;
        const int r = idx >> 3, c8 = idx & 7;
        *reinterpret_cast<uint4*>(&tile[r][c8 * 8]) = v[i];
    }
    __syncthreads();

    {
        const int w = tid >> 5, lane = tid & 31;
        float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
        for (int i = 0; i < kT1Tok / 8; ++i) {
            const uint32_t pr = *reinterpret_cast<const uint32_t*>(&tile[8 * i + w][2 * lane]);
            m0 = fmaxf(m0, fabsf(bf16_lo(pr)));
            m1 = fmaxf(m1, fabsf(bf16_hi(pr)));
        }
        red[w][2 * lane] = m0;
        red[w][2 * lane + 1] = m1;
    }
    __syncthreads();
    if (tid < kT1Ch) {
        float a = red[0][tid];
#pragma unroll
        for (int w = 1; w < 8; ++w) a = fmaxf(a, red[w][tid]);
        float sc, inv;
        group_scale(a, sc, inv);
        s[tb * C + c0 + tid] = sc;
        inv_c[tid] = inv;
    }
    __syncthreads();

#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int item = tid + 256 * j;
        const int c = item & (kT1Ch - 1), seg = item >> 6;   // seg: 16-token segment 0..7
        const float inv = inv_c[c];
        uint32_t w4[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
            const int tk = seg * 16 + 4 * p;
            const float f0 = __fmul_rn(__uint_as_float((uint32_t)tile[tk + 0][c] << 16), inv);
            const float f1 = __fmul_rn(__uint_as_float((uint32_t)tile[tk + 1][c] << 16), inv);
            const float f2 = __fmul_rn(__uint_as_float((uint32_t)tile[tk + 2][c] << 16), inv);
            const float f3 = __fmul_rn(__uint_as_float((uint32_t)tile[tk + 3][c] << 16), inv);
            w4[p] = e4m3x2(f0, f1) | (e4m3x2(f2, f3) << 16);
        }
        *reinterpret_cast<uint4*>(qt + (c0 + c) * T + t0 + seg * 16) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
}

// ------------------------------------------------------------------------------------------
// 128x128: w[N,K] -> q[N,K], s[N/128][K/128] (+ optional qt[K,N]).  One CTA per block; each
// thread holds 64 of the block's 16384 values in registers, so the block is read once.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) weight_128x128_kernel(const uint16_t* __restrict__ w,
                                                             uint8_t* __restrict__ q,
                                                             float* __restrict__ s,
                                                             uint8_t* __restrict__ qt, int64_t N, int64_t K)
{
    __shared__ float red[8];
    __shared__ __align__(16) uint8_t codes[128][128 + 16];

    const int64_t kb = blockIdx.x, nb = blockIdx.y;
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
    group_scale(amax, sc, inv);
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

}  // namespace fp8q
