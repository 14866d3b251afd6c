// fp8q.cu -- the C ABI of libfp8q.so (declared in include/fp8q.h): argument checks, TMA
// descriptor set-up and kernel launches.  Every call is asynchronous on the caller's stream
// and allocates no device memory.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <random>

#include "fp8q.h"
#include "gemm.cuh"
#include "ptx.cuh"
#include "quant.cuh"

namespace {

using namespace fp8q;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_fmt(int f) { return f == FP8Q_SCALE_FP32 || f == FP8Q_SCALE_UE8M0; }
bool pow2(int f) { return f == FP8Q_SCALE_UE8M0; }

int sm_count()
{
    static int counts[kMaxDevices] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
    if (counts[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        counts[dev] = n;
    }
    return counts[dev];
}

int launch_status()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

// Launches: every kernel of this library waits (griddepcontrol.wait) for the previous kernel in
// the stream before touching global memory, so each may be launched with programmatic stream
// serialization: its launch and prologue then overlap the previous kernel's tail.
// FP8Q_PDL=0 turns this off (plain stream order).
bool pdl_enabled()
{
    static const bool on = [] {
        const char* e = getenv("FP8Q_PDL");
        return !(e && strcmp(e, "0") == 0);
    }();
    return on;
}

template <typename... KArgs, typename... Args>
int launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool cooperative,
                  Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    int n = 0;
    if (cooperative) {
        attr[n].id = cudaLaunchAttributeCooperative;
        attr[n].val.cooperative = 1;
        ++n;
    }
    const int n_base = n;
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess) return launch_status();
    cudaGetLastError();
    if (n == n_base) return FP8Q_ERR_CUDA;
    cfg.numAttrs = n_base;   // the driver refused the combination: launch in plain stream order
    if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) {
        cudaGetLastError();
        return FP8Q_ERR_CUDA;
    }
    return launch_status();
}

// ------------------------------------------------------------------------------------------
// TMA descriptors (the driver entry point is fetched through the runtime, so the library has
// no link-time dependency on libcuda).
// ------------------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major uint8 matrix [outer][inner] with 128-byte swizzled boxes of box_inner x box_outer.
bool make_tmap_u8(CUtensorMap* tm, const void* base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                  uint32_t box_outer)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Row-major output matrix [outer][inner] of 1-, 2- or 4-byte elements, stored by the GEMM epilogue in
// boxes of 32 rows x 64 bytes with the 64-byte swizzle.
bool make_tmap_out(CUtensorMap* tm, void* base, uint64_t inner, uint64_t outer, int elt_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {inner * (uint64_t)elt_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(64 / elt_bytes), 32};
    const cuuint32_t estr[2] = {1, 1};
    const CUtensorMapDataType dt = elt_bytes == 4   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                   : elt_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_UINT8;
    return fn(tm, dt, 2, base, dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------------------------------
// GEMM launch
// ------------------------------------------------------------------------------------------
template <int MODE, int BN, bool GROUPED, bool MX = false>
int prepare_kernel()
{
    using S = GemmShape<MODE, BN, GROUPED, MX>;
    static int ready[kMaxDevices] = {0};   // 1 ok, -1 unusable
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
    if (ready[dev] == 0) {
        auto kern = gemm_blockscaled_kernel<MODE, BN, GROUPED, MX>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes) != cudaSuccess)
            return FP8Q_ERR_CUDA;
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, kern) != cudaSuccess) return FP8Q_ERR_CUDA;
        // The register hand-over (setmaxnreg) needs the launch-time allocation it redistributes;
        // never launch a build whose allocation is smaller.
        ready[dev] = (attr.numRegs >= S::kRegsLaunch) ? 1 : -1;
    }
    return ready[dev] == 1 ? FP8Q_OK : FP8Q_ERR_UNSUPPORTED;
}

// Workspace of the stream-K schedule for `ctas` persistent CTAs of BN-wide tiles: one FP32
// 128 x BN partial slot per CTA, then one 64-bit ready flag per CTA (256-byte aligned).
size_t sk_slot_bytes(int bn) { return (size_t)128 * bn * sizeof(float); }
size_t sk_workspace_bytes(int ctas, int bn)
{
    return (size_t)ctas * sk_slot_bytes(bn) + (((size_t)ctas * sizeof(uint64_t) + 255) & ~(size_t)255);
}

// Launch stamps: a flag holds the stamp of the launch that published it, so flags are never
// reset.  Bits 40..63 are a nonzero random salt drawn once per process (workspace memory left by
// another process cannot match by accident); bits 0..39 count this process's stream-K launches
// from 1.  Stamps are nonzero and never repeat within a process until 2^40 launches (about 35
// years at one launch per millisecond).
unsigned long long next_stamp()
{
    static std::atomic<unsigned long long> counter{0};
    static const unsigned long long salt = [] {
        std::random_device rd;
        unsigned long long v = ((unsigned long long)rd() << 32) ^ (unsigned long long)rd();
        v &= 0xFFFFFFull;
        return v ? v : 1ull;
    }();
    return (salt << 40) | ((++counter) & 0xFFFFFFFFFFull);
}

// FP8Q_GEMM_SCHED=dp / sk forces the data-parallel / stream-K schedule (tests and tuning).
bool streamk_forced()
{
    const char* env = getenv("FP8Q_GEMM_SCHED");
    return env && strcmp(env, "sk") == 0;
}

// Stream-K pays off when the whole tiles leave the last wave of the persistent grid mostly empty;
// otherwise its partial tiles (parked in the workspace and added by the tile's owner) and the
// extra work items per CTA cost more than the idle SMs of the last wave.  Measured on the
// linear-layer shapes (back-to-back launches, operands in L2): data-parallel is faster at a wave
// occupancy of 0.865 (Fprop 4096x2048x7168: 256 tiles in 2 waves of 148; Dgrad 4096x7168x2048:
// 896 tiles in 7), stream-K at 0.757 and below (Wgrad 2048x7168x4096: 448 tiles in 4; the MLA
// widths 1536 and 512: 192 and 64 tiles).  The switch sits between the two, at 0.8.
bool want_streamk(int64_t tiles, int ctas, int kb)
{
    const char* env = getenv("FP8Q_GEMM_SCHED");
    if (env && strcmp(env, "dp") == 0) return false;
    if (kb < 2) return false;
    if (streamk_forced()) return true;
    if (tiles % ctas == 0) return false;
    const int64_t waves = (tiles + ctas - 1) / ctas;
    return (double)tiles < 0.8 * (double)(waves * ctas);
}

template <int MODE, int BN, bool GROUPED, bool MX = false>
int launch_gemm(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB, void* D,
                const int32_t* offsets, int E, int64_t M, int64_t N, int64_t K, cudaStream_t st,
                void* workspace = nullptr, size_t ws_bytes = 0, bool accumulate = false,
                uint8_t* q_out = nullptr, float* s_out = nullptr, int64_t rows_total = -1)
{
    using S = GemmShape<MODE, BN, GROUPED, MX>;
    const int prep = prepare_kernel<MODE, BN, GROUPED, MX>();
    if (prep != FP8Q_OK) return prep;
    CUtensorMap ta, tb;
    if (!make_tmap_u8(&ta, A, (uint64_t)K, (uint64_t)M, 128, 128)) return FP8Q_ERR_CUDA;
    if (MODE == kModeDgrad) {
        const uint64_t krows = GROUPED ? (uint64_t)E * (uint64_t)K : (uint64_t)K;
        if (!make_tmap_u8(&tb, B, (uint64_t)N, krows, 128, 128)) return FP8Q_ERR_CUDA;
    } else {
        const uint64_t rows = (GROUPED && MODE != kModeWgrad) ? (uint64_t)E * (uint64_t)N : (uint64_t)N;
        if (!make_tmap_u8(&tb, B, (uint64_t)K, rows, 128, BN)) return FP8Q_ERR_CUDA;
    }
    CUtensorMap td, tq;   // the epilogue's store maps (the grouped GEMM stores without them)
    memset(&td, 0, sizeof(td));
    memset(&tq, 0, sizeof(tq));
    // Row-grouped GEMMs store without a map; the K-grouped Wgrad stores expert e's dW at rows e*M.
    const uint64_t d_rows = (GROUPED && MODE == kModeWgrad) ? (uint64_t)E * (uint64_t)M : (uint64_t)M;
    if ((!GROUPED || MODE == kModeWgrad) && D &&
        !make_tmap_out(&td, D, (uint64_t)N, d_rows, MODE == kModeWgrad ? 4 : 2))
        return FP8Q_ERR_CUDA;
    if (q_out && !make_tmap_out(&tq, q_out, (uint64_t)N, (uint64_t)M, 1)) return FP8Q_ERR_CUDA;
    GemmArgs a;
    a.sA = sA;
    a.sB = sB;
    a.D = D;
    a.offsets = offsets;
    a.E = E;
    a.M = (int32_t)M;
    a.N = (int32_t)N;
    a.KB = (int32_t)(K / 128);
    a.ws = nullptr;
    a.flags = nullptr;
    a.stamp = 0;
    a.units = 0;
    a.accumulate = accumulate ? 1 : 0;
    a.s_out = s_out;
    a.quant_out = q_out ? 1 : 0;
    a.store_d = D ? 1 : 0;
    a.rows_total = rows_total >= 0 ? rows_total : M;
    const int sms = sm_count();
    if (sms <= 0) return FP8Q_ERR_CUDA;
    // Row-grouped: at most ceil(Mtot/128) + E row tiles (each group adds at most one partial
    // tile).  K-grouped: E x the dense tiles.
    const int64_t m_tiles = (GROUPED && MODE != kModeWgrad) ? (M + 127) / 128 + E
                            : (GROUPED ? (int64_t)E * ((M + 127) / 128) : (M + 127) / 128);
    const int64_t tiles = m_tiles * (N / BN);
    const int64_t units = tiles * a.KB;
    if (!GROUPED && workspace && want_streamk(tiles, sms, a.KB)) {
        const int grid = (int)(units < sms ? units : sms);
        if (ws_bytes >= sk_workspace_bytes(grid, BN) && (reinterpret_cast<uintptr_t>(workspace) & 255u) == 0) {
            a.ws = static_cast<float*>(workspace);
            a.flags = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) +
                                                            (size_t)grid * sk_slot_bytes(BN));
            a.stamp = next_stamp();
            a.units = units;
            // CTAs wait on each other's partials: launch them co-resident (cooperative launch).
            return launch_kernel(gemm_blockscaled_kernel<MODE, BN, GROUPED, MX>, dim3((unsigned)grid),
                                 dim3(S::kThreads), S::kSmemBytes, st, true, ta, tb, td, tq, a);
        }
    }
    const int grid = (int)(tiles < sms ? tiles : sms);
    if (grid <= 0) return FP8Q_OK;
    return launch_kernel(gemm_blockscaled_kernel<MODE, BN, GROUPED, MX>, dim3((unsigned)grid), dim3(S::kThreads),
                         S::kSmemBytes, st, false, ta, tb, td, tq, a);
}

// Tile width: 256 whenever N allows it (measured faster on every linear-layer and MLA shape: it
// halves the B-tile traffic per MMA and gives the promotion warps twice the MMA time per group);
// FP8Q_GEMM_BN=128 forces the narrow tile (tests and tuning).
int choose_bn(int64_t M, int64_t N, int extra_m_tiles)
{
    (void)M;
    (void)extra_m_tiles;
    const char* env = getenv("FP8Q_GEMM_BN");
    if (env && atoi(env) == 128) return 128;
    return (N % 256 == 0) ? 256 : 128;
}

template <int MODE, bool MX = false>
int gemm_mode(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB, void* D, int64_t M,
              int64_t N, int64_t K, cudaStream_t st, void* ws, size_t ws_bytes, bool accumulate = false)
{
    if (choose_bn(M, N, 0) == 256)
        return launch_gemm<MODE, 256, false, MX>(A, sA, B, sB, D, nullptr, 1, M, N, K, st, ws, ws_bytes, accumulate);
    return launch_gemm<MODE, 128, false, MX>(A, sA, B, sB, D, nullptr, 1, M, N, K, st, ws, ws_bytes, accumulate);
}

// Waits on an mbarrier that nothing ever arrives on, so the bounded wait must expire, latch
// FP8Q_DEV_TIMEOUT and return.  Exercises the kernels' timeout path without a hang or a fault.
__global__ void selftest_wait_kernel(uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_slow(smem_u32(&bar), 0, &abort_flag, limit_ns);
}

// ------------------------------------------------------------------------------------------
// Allocation-free GEMM: the stream-K scratch lives in a file-scope device array instead of a
// caller workspace.  It holds the slots and flags of kNoallocMaxCtas persistent CTAs of
// 256-wide tiles (about 20 MiB), is present on every GPU that loads this library, and lives
// until the process exits.
// ------------------------------------------------------------------------------------------
constexpr int kNoallocMaxCtas = 160;
constexpr size_t kNoallocScratchBytes =
    (size_t)kNoallocMaxCtas * 128 * 256 * sizeof(float) + (((size_t)kNoallocMaxCtas * sizeof(uint64_t) + 255) & ~(size_t)255);
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  In host code the array's name is
// only a host-side stand-in, so the address is looked up once per device (with that device
// current) and cached.  Returns nullptr if the lookup fails.
void* noalloc_scratch()
{
    static void* addr[kMaxDevices] = {nullptr};
    static std::mutex lock;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> guard(lock);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

// ==========================================================================================
// C ABI
// ==========================================================================================
extern "C" {

const char* fp8q_status_string(int status)
{
    switch (status) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_ARG: return "invalid argument";
    case FP8Q_ERR_SHAPE: return "shape: a 128-group dimension is not a multiple of 128";
    case FP8Q_ERR_ALIGN: return "a data pointer is not 16-byte aligned";
    case FP8Q_ERR_CUDA: return "CUDA error";
    case FP8Q_ERR_UNSUPPORTED: return "size or configuration not supported by this build";
    case FP8Q_ERR_DEVICE: return "error reported by the device";
    case FP8Q_ERR_SCRATCH: return "the allocation-free GEMM needs more scratch than its fixed array holds";
    default: return "unknown status";
    }
}

int fp8q_abi_version(void) { return 1; }

int fp8q_act_1x128_fmt(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s, int scale_fmt,
                       fp8q_stream_t stream)
{
    if (M < 0 || K < 0 || !valid_fmt(scale_fmt)) return FP8Q_ERR_ARG;
    if (K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (M == 0 || K == 0) return FP8Q_OK;
    if (!x || !q || !s) return FP8Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s)) return FP8Q_ERR_ALIGN;
    const int sms = sm_count();
    if (sms <= 0) return FP8Q_ERR_CUDA;
    constexpr int kUnr = 4;
    const int64_t ntiles = M * (K / 128);
    if (ntiles >= (1ll << 31) || M >= (1ll << 31)) return FP8Q_ERR_UNSUPPORTED;
    const int64_t want = (ntiles + 32 * kUnr - 1) / (32 * kUnr);   // blocks of 32 eight-lane groups
    const int64_t cap = (int64_t)sms * 8;
    const int grid = (int)(want < cap ? want : cap);
    const auto kern = pow2(scale_fmt) ? act_1x128_kernel<kUnr, true> : act_1x128_kernel<kUnr, false>;
    return launch_kernel(kern, dim3(grid), dim3(256), 0, (cudaStream_t)stream, false, x, q, s, (int)M, (int)K);
}

int fp8q_act_1x128(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s, fp8q_stream_t stream)
{
    return fp8q_act_1x128_fmt(x, M, K, q, s, FP8Q_SCALE_FP32, stream);
}

int fp8q_act_128x1_transposed_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* qt, float* s, int scale_fmt,
                                  fp8q_stream_t stream)
{
    if (T < 0 || C < 0 || !valid_fmt(scale_fmt)) return FP8Q_ERR_ARG;
    if (T % 128 != 0 || C % 64 != 0) return FP8Q_ERR_SHAPE;
    if (T == 0 || C == 0) return FP8Q_OK;
    if (!x || !qt || !s) return FP8Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(qt) || !aligned16(s)) return FP8Q_ERR_ALIGN;
    if (T / 128 > 65535 || C / 64 > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)(C / 64), (unsigned)(T / 128));
    const auto kern = pow2(scale_fmt) ? act_128x1_t_kernel<true> : act_128x1_t_kernel<false>;
    return launch_kernel(kern, grid, dim3(256), 0, (cudaStream_t)stream, false, x, qt, s, T, C);
}

int fp8q_act_128x1_transposed(const uint16_t* x, int64_t T, int64_t C, uint8_t* qt, float* s,
                              fp8q_stream_t stream)
{
    return fp8q_act_128x1_transposed_fmt(x, T, C, qt, s, FP8Q_SCALE_FP32, stream);
}

int fp8q_act_dual_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* q, float* s, uint8_t* qt, float* st,
                      int scale_fmt, fp8q_stream_t stream)
{
    if (T < 0 || C < 0 || !valid_fmt(scale_fmt)) return FP8Q_ERR_ARG;
    if (T % 128 != 0 || C % 128 != 0) return FP8Q_ERR_SHAPE;
    if (T == 0 || C == 0) return FP8Q_OK;
    if (!x || !q || !s || !qt || !st) return FP8Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(q) || !aligned16(s) || !aligned16(qt) || !aligned16(st))
        return FP8Q_ERR_ALIGN;
    if (T / 128 > 65535 || C / 128 > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)(C / 128), (unsigned)(T / 128));
    const auto kern = pow2(scale_fmt) ? act_dual_kernel<true> : act_dual_kernel<false>;
    return launch_kernel(kern, grid, dim3(256), 0, (cudaStream_t)stream, false, x, q, s, qt, st, T, C);
}

int fp8q_act_dual(const uint16_t* x, int64_t T, int64_t C, uint8_t* q, float* s, uint8_t* qt, float* st,
                  fp8q_stream_t stream)
{
    return fp8q_act_dual_fmt(x, T, C, q, s, qt, st, FP8Q_SCALE_FP32, stream);
}

int fp8q_quant_forward_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* xq, float* xs, uint8_t* xqt,
                           float* xst, const uint16_t* w, int64_t N, uint8_t* wq, float* ws, uint8_t* wqt_or_null,
                           int scale_fmt, fp8q_stream_t stream)
{
    if (T < 0 || C < 0 || N < 0 || !valid_fmt(scale_fmt)) return FP8Q_ERR_ARG;
    if (T % 128 != 0 || C % 128 != 0 || N % 128 != 0) return FP8Q_ERR_SHAPE;
    if (C == 0 || (T == 0 && N == 0)) return FP8Q_OK;
    if (!x || !xq || !xs || !xqt || !xst || !w || !wq || !ws) return FP8Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(xq) || !aligned16(xs) || !aligned16(xqt) || !aligned16(xst) || !aligned16(w) ||
        !aligned16(wq) || !aligned16(ws) || !aligned16(wqt_or_null))
        return FP8Q_ERR_ALIGN;
    const int64_t tiles = (T / 128 + N / 128) * (C / 128);
    if (tiles > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
    const auto kern = pow2(scale_fmt) ? forward_operands_kernel<true> : forward_operands_kernel<false>;
    return launch_kernel(kern, dim3((unsigned)tiles), dim3(256), 0, (cudaStream_t)stream, false, x, xq, xs, xqt, xst,
                         T, C, w, wq, ws, wqt_or_null, N);
}

int fp8q_quant_forward(const uint16_t* x, int64_t T, int64_t C, uint8_t* xq, float* xs, uint8_t* xqt, float* xst,
                       const uint16_t* w, int64_t N, uint8_t* wq, float* ws, uint8_t* wqt_or_null,
                       fp8q_stream_t stream)
{
    return fp8q_quant_forward_fmt(x, T, C, xq, xs, xqt, xst, w, N, wq, ws, wqt_or_null, FP8Q_SCALE_FP32, stream);
}

int fp8q_weight_128x128_fmt(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s, uint8_t* qt_or_null,
                            int scale_fmt, fp8q_stream_t stream)
{
    if (N < 0 || K < 0 || !valid_fmt(scale_fmt)) return FP8Q_ERR_ARG;
    if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (N == 0 || K == 0) return FP8Q_OK;
    if (!w || !q || !s) return FP8Q_ERR_ARG;
    if (!aligned16(w) || !aligned16(q) || !aligned16(s) || !aligned16(qt_or_null)) return FP8Q_ERR_ALIGN;
    if (N / 128 > 65535 || K / 128 > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
    const dim3 grid((unsigned)(K / 128), (unsigned)(N / 128));
    const auto kern = pow2(scale_fmt) ? weight_128x128_kernel<true> : weight_128x128_kernel<false>;
    return launch_kernel(kern, grid, dim3(256), 0, (cudaStream_t)stream, false, w, q, s, qt_or_null, N, K);
}

int fp8q_weight_128x128(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s, uint8_t* qt_or_null,
                        fp8q_stream_t stream)
{
    return fp8q_weight_128x128_fmt(w, N, K, q, s, qt_or_null, FP8Q_SCALE_FP32, stream);
}

size_t fp8q_gemm_workspace_size(int mode, int64_t M, int64_t N, int64_t K)
{
    (void)mode;
    if (M <= 0 || N <= 0 || K < 256) return 0;   // one 128-K group: nothing to split
    int sms = sm_count();
    if (sms <= 0) sms = 148;
    return sk_workspace_bytes(sms, 256);
}

int fp8_gemm_blockscaled(int mode, const uint8_t* A, const float* sA, const uint8_t* B, const float* sB, void* D,
                         int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes, fp8q_stream_t stream)
{
    if (mode != FP8Q_FPROP && mode != FP8Q_DGRAD && mode != FP8Q_WGRAD && mode != FP8Q_WGRAD_ACC) return FP8Q_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_ARG;
    if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8Q_OK;
    if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31)) return FP8Q_ERR_UNSUPPORTED;
    if (!A || !sA || !B || !sB || !D) return FP8Q_ERR_ARG;
    if (!aligned16(A) || !aligned16(sA) || !aligned16(B) || !aligned16(sB) || !aligned16(D)) return FP8Q_ERR_ALIGN;
    if (K == 0) {
        // An empty contraction: D = 0 (D += 0 leaves it as it is).
        if (mode == FP8Q_WGRAD_ACC) return FP8Q_OK;
        const size_t bytes = (size_t)M * (size_t)N * (mode == FP8Q_WGRAD ? 4u : 2u);
        return cudaMemsetAsync(D, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
    }
    const cudaStream_t st = (cudaStream_t)stream;
    switch (mode) {
    case FP8Q_FPROP: return gemm_mode<kModeFprop>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes);
    case FP8Q_DGRAD: return gemm_mode<kModeDgrad>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes);
    case FP8Q_WGRAD: return gemm_mode<kModeWgrad>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes);
    default: return gemm_mode<kModeWgrad>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes, true);
    }
}

int fp8_gemm_blockscaled_ue8m0(int mode, const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                               void* D, int64_t M, int64_t N, int64_t K, void* workspace, size_t ws_bytes,
                               fp8q_stream_t stream)
{
    if (mode != FP8Q_FPROP && mode != FP8Q_DGRAD && mode != FP8Q_WGRAD && mode != FP8Q_WGRAD_ACC) return FP8Q_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_ARG;
    if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8Q_OK;
    if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31)) return FP8Q_ERR_UNSUPPORTED;
    if (!A || !sA || !B || !sB || !D) return FP8Q_ERR_ARG;
    if (!aligned16(A) || !aligned16(sA) || !aligned16(B) || !aligned16(sB) || !aligned16(D)) return FP8Q_ERR_ALIGN;
    if (K == 0) {
        if (mode == FP8Q_WGRAD_ACC) return FP8Q_OK;
        const size_t bytes = (size_t)M * (size_t)N * (mode == FP8Q_WGRAD ? 4u : 2u);
        return cudaMemsetAsync(D, 0, bytes, (cudaStream_t)stream) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
    }
    const cudaStream_t st = (cudaStream_t)stream;
    switch (mode) {
    case FP8Q_FPROP: return gemm_mode<kModeFprop, true>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes);
    case FP8Q_DGRAD: return gemm_mode<kModeDgrad, true>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes);
    case FP8Q_WGRAD: return gemm_mode<kModeWgrad, true>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes);
    default: return gemm_mode<kModeWgrad, true>(A, sA, B, sB, D, M, N, K, st, workspace, ws_bytes, true);
    }
}

int fp8_gemm_blockscaled_quant(int mode, const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                               void* D, uint8_t* Dq, float* Ds, int64_t M, int64_t N, int64_t K, void* workspace,
                               size_t ws_bytes, fp8q_stream_t stream)
{
    if (mode != FP8Q_FPROP && mode != FP8Q_DGRAD) return FP8Q_ERR_ARG;
    if (M < 0 || N < 0 || K < 0) return FP8Q_ERR_ARG;
    if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8Q_OK;
    if (M >= (1ll << 31) || N >= (1ll << 31) || K >= (1ll << 31) || K == 0) return FP8Q_ERR_UNSUPPORTED;
    if (!A || !sA || !B || !sB || !Dq || !Ds) return FP8Q_ERR_ARG;
    if (!aligned16(A) || !aligned16(sA) || !aligned16(B) || !aligned16(sB) || !aligned16(D) || !aligned16(Dq) ||
        !aligned16(Ds))
        return FP8Q_ERR_ALIGN;
    const cudaStream_t st = (cudaStream_t)stream;
    if (choose_bn(M, N, 0) == 256) {
        // One 256-wide tile row per promotion warp pair: each thread's 128 columns are a group.
        if (mode == FP8Q_FPROP)
            return launch_gemm<kModeFprop, 256, false>(A, sA, B, sB, D, nullptr, 1, M, N, K, st, workspace,
                                                      ws_bytes, false, Dq, Ds);
        return launch_gemm<kModeDgrad, 256, false>(A, sA, B, sB, D, nullptr, 1, M, N, K, st, workspace, ws_bytes,
                                                  false, Dq, Ds);
    }
    // 128-wide tiles split a group over two warps: run the GEMM, then quantise D.
    if (!D) return FP8Q_ERR_UNSUPPORTED;
    const int rc = fp8_gemm_blockscaled(mode, A, sA, B, sB, D, M, N, K, workspace, ws_bytes, stream);
    if (rc != FP8Q_OK) return rc;
    return fp8q_act_1x128(static_cast<const uint16_t*>(D), M, N, Dq, Ds, stream);
}

int fp8_gemm_blockscaled_noalloc(int mode, const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                                 void* D, int64_t M, int64_t N, int64_t K, fp8q_stream_t stream)
{
    // The stream-K schedule needs one slot per persistent CTA (one per SM); the data-parallel
    // schedule needs none.  When the slots would not fit the fixed array (more SMs than it was
    // sized for) the call runs data-parallel, unless stream-K is forced.
    const size_t need = fp8q_gemm_workspace_size(mode, M, N, K);
    void* scratch = nullptr;
    if (need > kNoallocScratchBytes) {
        if (streamk_forced()) return FP8Q_ERR_SCRATCH;
    } else if (need > 0) {
        scratch = noalloc_scratch();
        if (!scratch) return FP8Q_ERR_CUDA;
    }
    return fp8_gemm_blockscaled(mode, A, sA, B, sB, D, M, N, K, scratch, scratch ? kNoallocScratchBytes : 0, stream);
}

int fp8_grouped_gemm_blockscaled(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                                 const int32_t* offsets, int32_t E, int64_t Mtot, int64_t N, int64_t K, uint16_t* D,
                                 fp8q_stream_t stream)
{
    if (E < 1 || Mtot < 0 || N < 0 || K < 0) return FP8Q_ERR_ARG;
    if (E > 1024) return FP8Q_ERR_UNSUPPORTED;
    if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (Mtot == 0 || N == 0) return FP8Q_OK;
    if (Mtot >= (1ll << 31) || (int64_t)E * N >= (1ll << 31) || K >= (1ll << 31)) return FP8Q_ERR_UNSUPPORTED;
    if (!A || !sA || !B || !sB || !D || !offsets) return FP8Q_ERR_ARG;
    if (!aligned16(A) || !aligned16(sA) || !aligned16(B) || !aligned16(sB) || !aligned16(D)) return FP8Q_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return FP8Q_ERR_ALIGN;
    const cudaStream_t st = (cudaStream_t)stream;
    if (K == 0) {
        return cudaMemsetAsync(D, 0, (size_t)Mtot * (size_t)N * 2u, st) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
    }
    if (choose_bn(Mtot, N, E) == 256)
        return launch_gemm<kModeFprop, 256, true>(A, sA, B, sB, D, offsets, E, Mtot, N, K, st);
    return launch_gemm<kModeFprop, 128, true>(A, sA, B, sB, D, offsets, E, Mtot, N, K, st);
}

int fp8_grouped_gemm_blockscaled_dgrad(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                                       const int32_t* offsets, int32_t E, int64_t Mtot, int64_t N, int64_t K,
                                       uint16_t* D, fp8q_stream_t stream)
{
    if (E < 1 || Mtot < 0 || N < 0 || K < 0) return FP8Q_ERR_ARG;
    if (E > 1024) return FP8Q_ERR_UNSUPPORTED;
    if (N % 128 != 0 || K % 128 != 0) return FP8Q_ERR_SHAPE;
    if (Mtot == 0 || N == 0) return FP8Q_OK;
    if (Mtot >= (1ll << 31) || N >= (1ll << 31) || (int64_t)E * K >= (1ll << 31)) return FP8Q_ERR_UNSUPPORTED;
    if (!A || !sA || !B || !sB || !D || !offsets) return FP8Q_ERR_ARG;
    if (!aligned16(A) || !aligned16(sA) || !aligned16(B) || !aligned16(sB) || !aligned16(D)) return FP8Q_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return FP8Q_ERR_ALIGN;
    const cudaStream_t st = (cudaStream_t)stream;
    if (K == 0) {
        return cudaMemsetAsync(D, 0, (size_t)Mtot * (size_t)N * 2u, st) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
    }
    if (choose_bn(Mtot, N, E) == 256)
        return launch_gemm<kModeDgrad, 256, true>(A, sA, B, sB, D, offsets, E, Mtot, N, K, st);
    return launch_gemm<kModeDgrad, 128, true>(A, sA, B, sB, D, offsets, E, Mtot, N, K, st);
}

int fp8q_act_128x1_transposed_ragged(const uint16_t* x, const int32_t* offsets, int32_t E, int64_t Mtot, int64_t C,
                                     uint8_t* qt, float* s, int64_t Kcap, fp8q_stream_t stream)
{
    if (E < 1 || Mtot < 0 || C < 0 || Kcap < 0) return FP8Q_ERR_ARG;
    if (E > kRgMaxGroups) return FP8Q_ERR_UNSUPPORTED;
    if (C % 64 != 0 || Kcap % 128 != 0) return FP8Q_ERR_SHAPE;
    if (Mtot == 0 || C == 0) return FP8Q_OK;
    if (!x || !offsets || !qt || !s) return FP8Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(qt) || !aligned16(s)) return FP8Q_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return FP8Q_ERR_ALIGN;
    const int64_t groups = (Mtot + 127) / 128 + E;   // padded token groups, at most
    if (groups > 0x7FFFFFFF || Mtot >= (1ll << 31)) return FP8Q_ERR_UNSUPPORTED;
    const int64_t chunks = (C / 64 + kRgChunk - 1) / kRgChunk;
    const dim3 grid((unsigned)chunks, (unsigned)(groups < 65535 ? groups : 65535));
    if (groups > 65535) return FP8Q_ERR_UNSUPPORTED;
    return launch_kernel(act_128x1_t_ragged_kernel<false>, grid, dim3(256), 0, (cudaStream_t)stream, false, x, offsets,
                         (int)E, Mtot, C, qt, s, Kcap);
}

int fp8_grouped_gemm_blockscaled_wgrad(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                                       const int32_t* offsets, int32_t E, int64_t Mtot, int64_t M, int64_t N,
                                       int64_t Kcap, float* D, fp8q_stream_t stream)
{
    if (E < 1 || Mtot < 0 || M < 0 || N < 0 || Kcap < 0) return FP8Q_ERR_ARG;
    if (E > 1024) return FP8Q_ERR_UNSUPPORTED;
    if (M % 128 != 0 || N % 128 != 0 || Kcap % 128 != 0) return FP8Q_ERR_SHAPE;
    if (M == 0 || N == 0) return FP8Q_OK;
    if (Mtot >= (1ll << 31) || (int64_t)E * M >= (1ll << 31) || N >= (1ll << 31) || Kcap >= (1ll << 31))
        return FP8Q_ERR_UNSUPPORTED;
    if ((int64_t)E * (M / 128) * (N / 128) > 0x7FFFFFFF) return FP8Q_ERR_UNSUPPORTED;
    if (!A || !sA || !B || !sB || !D || !offsets) return FP8Q_ERR_ARG;
    if (!aligned16(A) || !aligned16(sA) || !aligned16(B) || !aligned16(sB) || !aligned16(D)) return FP8Q_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(offsets) & 3u) != 0) return FP8Q_ERR_ALIGN;
    const cudaStream_t st = (cudaStream_t)stream;
    if (Kcap == 0) {
        return cudaMemsetAsync(D, 0, (size_t)E * (size_t)M * (size_t)N * 4u, st) == cudaSuccess ? FP8Q_OK
                                                                                             : FP8Q_ERR_CUDA;
    }
    if (choose_bn(M, N, E) == 256)
        return launch_gemm<kModeWgrad, 256, true>(A, sA, B, sB, D, offsets, E, M, N, Kcap, st, nullptr, 0, false,
                                                 nullptr, nullptr, Mtot);
    return launch_gemm<kModeWgrad, 128, true>(A, sA, B, sB, D, offsets, E, M, N, Kcap, st, nullptr, 0, false,
                                             nullptr, nullptr, Mtot);
}

int fp8q_selftest_wait_timeout(uint64_t limit_ns, fp8q_stream_t stream)
{
    if (limit_ns == 0 || limit_ns > 2000000000ull) return FP8Q_ERR_ARG;
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
    return launch_status();
}

int fp8q_device_status(fp8q_stream_t stream, int* out)
{
    if (!out) return FP8Q_ERR_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FP8Q_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, fp8q::g_status, sizeof(int)) != cudaSuccess) return FP8Q_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(fp8q::g_status, &zero, sizeof(int)) != cudaSuccess) return FP8Q_ERR_CUDA;
    *out = v;
    return FP8Q_OK;
}

}  // extern "C"
