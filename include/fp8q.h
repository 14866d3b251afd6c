/*
 * fp8q.h -- C ABI of libfp8q.so: fine-grained FP8 (E4M3) quantisation and the block-scaled
 * FP8 GEMM of DeepSeek-V3's linear layers, hand-written for B200 (sm_100a).
 *
 * Passages these operations follow (pages on the DeepSeek-V3 Technical Report, arXiv
 * 2412.19437):
 *   [SUMMARY] "DeepSeek-V3 Technical Report" summary page (xyznot.com): Key ideas, FP8
 *             mixed-precision bullet -- E4M3 for all tensors, 1x128 tile-wise activation and
 *             128x128 block-wise weight scaling, accumulation copied to FP32 CUDA-core registers
 *             every N_c = 128 elements; Questions, the answer on FP8 training without
 *             divergence -- the same, restated.
 *   [REPOST]  DeepSeek-V3 report repost (why-be.co.kr board post): paragraph 1 -- 128 elements
 *             (4 WGMMAs) is the promotion interval; paragraph 2 and Figure 6 -- Fprop, Dgrad
 *             and Wgrad all run in FP8; paragraph 3 -- master weights and gradients stay in
 *             FP32; paragraph 4 -- per-group scaling factors along the GEMM's inner dimension,
 *             dequantised during the increased-precision accumulation (Figure 7(b)).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer argument is a DEVICE pointer owned by the caller (for example a PyTorch
 *   tensor's data_ptr()).  The library never allocates, frees or retains caller memory.
 * - Every tensor is dense row-major with no padding; bf16 tensors are passed as uint16_t bit
 *   patterns; E4M3 codes as uint8_t (OCP E4M3FN: bias 7, largest finite 448 = 0x7E).
 * - Every data pointer must be 16-byte aligned (FP8Q_ERR_ALIGN otherwise).
 * - Work is enqueued on `stream` (NULL = the legacy default stream) and is complete when the
 *   stream reaches it.  No call synchronises, except fp8q_device_status.
 * - The status returned covers the host-side checks and the launch only.  Errors found on the
 *   device (a malformed offsets array, a pipeline wait that timed out) are latched in a device
 *   status word that fp8q_device_status reads and clears.
 * - A call with an empty problem (M == 0, T == 0, ...) returns FP8Q_OK and launches nothing.
 * - Scale layout: the per-row scales of a [rows, K] operand quantised in groups of 128 along K
 *   are stored group-major, s[K/128][rows], so one 128-row tile's scales for one K group are
 *   one contiguous 512-byte run.
 * - Quantisation of a group g: a = max(max|x| over g, 2^-100); s = a / 448 (stored: the
 *   dequantisation multiplier); q = E4M3(x * (448 / a)) rounded to nearest even with
 *   saturation.  The divisions and the multiply are IEEE binary32, round to nearest.  Codes and
 *   scales are bit-exact functions of the input.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FP8Q_API __attribute__((visibility("default")))
#else
#define FP8Q_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st* fp8q_stream_t;

/* Return codes. */
enum {
    FP8Q_OK = 0,
    FP8Q_ERR_ARG = 1,          /* null pointer where data is required, negative size, bad mode */
    FP8Q_ERR_SHAPE = 2,        /* a dimension that a 128-group spans is not a multiple of 128 */
    FP8Q_ERR_ALIGN = 3,        /* a data pointer is not 16-byte aligned */
    FP8Q_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed (no device, launch error) */
    FP8Q_ERR_UNSUPPORTED = 5,  /* a size beyond what this build supports (see each call) */
    FP8Q_ERR_DEVICE = 6,       /* reported by fp8q_device_status: an error latched on the device */
    FP8Q_ERR_SCRATCH = 7       /* fp8_gemm_blockscaled_noalloc with stream-K forced: scratch need exceeds its fixed array */
};

/* Device status word values (what fp8q_device_status writes to *out). */
enum {
    FP8Q_DEV_OK = 0,
    FP8Q_DEV_TIMEOUT = 1,      /* a bounded pipeline wait expired; the kernel exited early */
    FP8Q_DEV_BAD_OFFSETS = 2,  /* grouped GEMM: offsets not 0-based / nondecreasing / ending at Mtot */
    FP8Q_DEV_BAD_SCALES = 3    /* fp8_gemm_blockscaled_ue8m0: a scale that is not a positive normal
                                  power of two (its result is then unspecified) */
};

/* Scale formats of the quantisers (the *_fmt entry points). */
enum {
    FP8Q_SCALE_FP32 = 0,       /* s = a / 448, the pages' max-abs scale (all other entry points) */
    FP8Q_SCALE_UE8M0 = 1       /* s = the smallest power of two >= fl32(a / 448): see below */
};

/* GEMM modes (the three GEMMs of a linear layer, [REPOST] paragraph 2, Figure 6; the FP32
 * weight gradient is accumulated across micro-batches, [REPOST] paragraph 3). */
enum {
    FP8Q_FPROP = 0,            /* Y  = X  W^T : D bf16 */
    FP8Q_DGRAD = 1,            /* dX = dY W   : D bf16 */
    FP8Q_WGRAD = 2,            /* dW = dY^T X : D fp32 */
    FP8Q_WGRAD_ACC = 3         /* dW += dY^T X : D fp32, accumulated into (gradient accumulation) */
};

/* Human-readable name of a return code (static storage; never NULL). */
FP8Q_API const char* fp8q_status_string(int status);

/* ABI version of this header (incremented on incompatible change). */
FP8Q_API int fp8q_abi_version(void);

/*
 * 1x128 tile-wise activation quantisation ([SUMMARY] Key ideas, FP8 bullet).
 *   x : [M, K] bf16            q : [M, K] E4M3 codes         s : [K/128, M] fp32 scales
 * Group = one row, 128 consecutive columns.  K % 128 == 0 (FP8Q_ERR_SHAPE otherwise); any
 * M >= 0.  x is not modified; q and s are fully overwritten.
 */
FP8Q_API int fp8q_act_1x128(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s,
                   fp8q_stream_t stream);

/*
 * 128x1 token-direction quantisation with transposed output, the operand form of Wgrad, whose
 * inner (scaled) dimension is the token dimension ([REPOST] paragraphs 2 and 4).
 *   x : [T, C] bf16            qt : [C, T] E4M3 codes        s : [T/128, C] fp32 scales
 * Group = one channel c, 128 consecutive tokens.  T % 128 == 0 and C % 64 == 0
 * (FP8Q_ERR_SHAPE otherwise).
 */
FP8Q_API int fp8q_act_128x1_transposed(const uint16_t* x, int64_t T, int64_t C, uint8_t* qt, float* s,
                              fp8q_stream_t stream);

/*
 * Both activation forms of one tensor in a single pass over x: the 1x128 form (as
 * fp8q_act_1x128 with M = T, K = C) and the 128x1 transposed form (as
 * fp8q_act_128x1_transposed).  A linear layer needs both for X (Fprop, Wgrad) and for dY
 * (Dgrad, Wgrad) ([REPOST] paragraphs 2 and 4); reading x once instead of twice saves one
 * full read of the tensor from HBM.  Outputs are bit-identical to the two separate calls.
 *   x : [T, C] bf16
 *   q : [T, C] E4M3 codes,  s  : [C/128, T] fp32   (groups: one token, 128 channels)
 *   qt: [C, T] E4M3 codes,  st : [T/128, C] fp32   (groups: one channel, 128 tokens)
 * T % 128 == 0 and C % 128 == 0 (FP8Q_ERR_SHAPE otherwise); T / 128 <= 65535
 * (FP8Q_ERR_UNSUPPORTED otherwise).  All pointers 16-byte aligned, caller-owned, device.
 */
FP8Q_API int fp8q_act_dual(const uint16_t* x, int64_t T, int64_t C, uint8_t* q, float* s,
                           uint8_t* qt, float* st, fp8q_stream_t stream);

/*
 * The forward operands of a linear layer Y = X W^T in one launch: X to both activation forms
 * (exactly as fp8q_act_dual) and W to 128x128 blocks (exactly as fp8q_weight_128x128 with
 * K = C).  Outputs are bit-identical to the two separate calls; one launch instead of two
 * saves a launch and a partly filled last wave.
 *   x : [T, C] bf16   -> xq [T, C], xs [C/128, T], xqt [C, T], xst [T/128, C]
 *   w : [N, C] bf16   -> wq [N, C], ws [N/128, C/128], wqt [C, N] (optional: NULL skips it)
 * T, C, N multiples of 128 (FP8Q_ERR_SHAPE otherwise).  All pointers 16-byte aligned, caller-owned,
 * device.
 */
FP8Q_API int fp8q_quant_forward(const uint16_t* x, int64_t T, int64_t C, uint8_t* xq, float* xs, uint8_t* xqt,
                                float* xst, const uint16_t* w, int64_t N, uint8_t* wq, float* ws,
                                uint8_t* wqt_or_null, fp8q_stream_t stream);

/*
 * 128x128 block-wise weight quantisation ([SUMMARY] Key ideas, FP8 bullet).
 *   w : [N, K] bf16            q : [N, K] E4M3 codes         s : [N/128, K/128] fp32 scales
 *   qt_or_null : NULL, or [K, N] receiving the same codes transposed.
 * N % 128 == 0 and K % 128 == 0 (FP8Q_ERR_SHAPE otherwise).
 */
FP8Q_API int fp8q_weight_128x128(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s,
                        uint8_t* qt_or_null, fp8q_stream_t stream);

/*
 * Block-scaled FP8 GEMM with FP32 promotion every 128 K ([REPOST] paragraphs 1 and 4;
 * [SUMMARY] FP8 bullet):  D[m, n] = sum_kb sum_{k in kb} A^(m, k) B^(k, n), where each 128-wide
 * K group's tensor-core partial sum is multiplied by its two scales and added into an FP32
 * accumulator.
 *
 *   A  : [M, K] E4M3 codes, sA : [K/128, M] (1x128 or 128x1-transposed scales).
 *   mode FP8Q_FPROP: B = W [N, K] codes, sB = [N/128, K/128] block scales; D = bf16 [M, N].
 *   mode FP8Q_DGRAD: B = W [K, N] codes -- the forward weight [out = K, in = N], used
 *                    transposed, no requantisation; sB = [K/128, N/128]; D = bf16 [M, N].
 *   mode FP8Q_WGRAD: B = X^T [N, K] codes (128x1 along K = tokens), sB = [K/128, N];
 *                    D = fp32 [M, N].
 *   mode FP8Q_WGRAD_ACC: as FP8Q_WGRAD, but the result is added into D (D must hold the
 *                    FP32 gradient so far; each element gets one FP32 addition).
 * Requirements: K % 128 == 0, N % 128 == 0 (FP8Q_ERR_SHAPE); M >= 0 (any M, the last row tile
 * is masked); M, N, K < 2^31 (FP8Q_ERR_UNSUPPORTED).  D is fully overwritten, except in
 * FP8Q_WGRAD_ACC.  K == 0 writes D = 0 (FP8Q_WGRAD_ACC: leaves D unchanged).
 * workspace / ws_bytes: optional scratch for the stream-K schedule (used when whole output tiles
 * would leave the persistent grid's last wave less than 80 % full, and K spans at least two
 * 128-groups): at least fp8q_gemm_workspace_size(...) bytes,
 * 256-byte aligned, device memory owned by the caller, reusable across calls on one stream
 * (never cleared: each launch stamps its flags with a fresh value).  NULL / 0, or a smaller
 * buffer, runs the data-parallel schedule instead -- same results, possibly slower.
 */
FP8Q_API int fp8_gemm_blockscaled(int mode, const uint8_t* A, const float* sA, const uint8_t* B,
                         const float* sB, void* D, int64_t M, int64_t N, int64_t K,
                         void* workspace, size_t ws_bytes, fp8q_stream_t stream);

/* Bytes of workspace fp8_gemm_blockscaled can use for a problem (0: none is useful). */
FP8Q_API size_t fp8q_gemm_workspace_size(int mode, int64_t M, int64_t N, int64_t K);

/*
 * Fprop or Dgrad (mode FP8Q_FPROP / FP8Q_DGRAD, arguments as fp8_gemm_blockscaled) that also
 * quantises its output for the next GEMM: the 1x128 tile-wise E4M3 codes and scales of the bf16
 * output, written from the epilogue while the output tile is still in registers.
 *   D  : [M, N] bf16, or NULL to skip storing the bf16 output (then N % 256 == 0 is required)
 *   Dq : [M, N] E4M3 codes,  Ds : [N/128, M] fp32 scales -- bit-identical to
 *        fp8q_act_1x128(D) applied to the bf16 output this call computes.
 * With N % 256 == 0 (256-wide tiles: each promotion thread holds one row's 128-column group) the
 * quantisation runs in the GEMM epilogue; otherwise the call runs the GEMM and then
 * fp8q_act_1x128 on D (D required).  K > 0; other requirements and errors as
 * fp8_gemm_blockscaled.
 */
FP8Q_API int fp8_gemm_blockscaled_quant(int mode, const uint8_t* A, const float* sA, const uint8_t* B,
                                        const float* sB, void* D, uint8_t* Dq, float* Ds, int64_t M, int64_t N,
                                        int64_t K, void* workspace, size_t ws_bytes, fp8q_stream_t stream);

/*
 * fp8_gemm_blockscaled without a workspace argument, for callers that may not allocate device
 * memory themselves: a plugin running inside a host framework that owns the device memory pool
 * and gives its kernels only their inputs and outputs, or a latency-critical path that cannot
 * afford cudaMalloc's implicit device-wide synchronisation.  (This entry point has no
 * counterpart on the pages; it is packaging, not part of the method.)
 *
 * Same arguments, results and requirements as fp8_gemm_blockscaled.  The stream-K scratch that
 * call would take from `workspace` comes instead from a fixed device array inside the library:
 * room for the partial slots and flags of 160 persistent CTAs of 256-wide tiles, about 20 MiB,
 * held by every GPU that loads the library until the process exits.  Where the slots would not
 * fit it (a device with more than 160 SMs) the call runs the data-parallel schedule, which needs
 * no scratch; only with stream-K forced (FP8Q_GEMM_SCHED=sk) does it return FP8Q_ERR_SCRATCH
 * instead.  No call allocates or frees anything.
 * - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *   that device current) and caches it; make that first call before any stream capture.
 * - Every call shares the one array per device and leaves its contents behind.  Nothing in it
 *   needs clearing: each launch stamps its flags with a value no earlier launch used.
 * - Calls whose GPU work overlaps (on different streams, or from different threads) race on the
 *   shared scratch and give wrong results; order them on one stream or with events.
 */
FP8Q_API int fp8_gemm_blockscaled_noalloc(int mode, const uint8_t* A, const float* sA, const uint8_t* B,
                                          const float* sB, void* D, int64_t M, int64_t N, int64_t K,
                                          fp8q_stream_t stream);

/*
 * Grouped (MoE expert) block-scaled FP8 Fprop over ragged row groups: the rows of A are sorted
 * by expert and rows offsets[e] .. offsets[e+1]-1 multiply expert e's weight.
 *   A  : [Mtot, K] codes, sA : [K/128, Mtot]
 *   B  : [E, N, K] codes, sB : [E, N/128, K/128]
 *   offsets : DEVICE int32 [E + 1], offsets[0] = 0, nondecreasing, offsets[E] = Mtot.  Empty
 *             experts are allowed.  A malformed array is detected on the device: nothing is
 *             written and FP8Q_DEV_BAD_OFFSETS is latched for fp8q_device_status.
 *   D  : [Mtot, N] bf16.
 * Requirements: K % 128 == 0, N % 128 == 0, 1 <= E <= 1024, Mtot < 2^31.
 */
FP8Q_API int fp8_grouped_gemm_blockscaled(const uint8_t* A, const float* sA, const uint8_t* B,
                                 const float* sB, const int32_t* offsets, int32_t E,
                                 int64_t Mtot, int64_t N, int64_t K, uint16_t* D,
                                 fp8q_stream_t stream);

/*
 * Grouped Dgrad over the same ragged row groups: dX_e = dY_e W_e for every expert, the input
 * gradient of the grouped Fprop ([REPOST] paragraph 2: Dgrad in FP8; 256 routed experts,
 * [SUMMARY]).  The expert weights are the forward ones, used transposed without requantisation:
 *   A  : [Mtot, K] codes of dY (K = the experts' output width), sA : [K/128, Mtot] (1x128)
 *   B  : [E, K, N] codes -- expert e's forward weight [out = K, in = N] -- and
 *   sB : [E, K/128, N/128] its forward 128x128 block scales
 *   offsets : as fp8_grouped_gemm_blockscaled (validated on the device the same way)
 *   D  : [Mtot, N] bf16.
 * Requirements and errors as fp8_grouped_gemm_blockscaled, with E * K < 2^31.
 */
FP8Q_API int fp8_grouped_gemm_blockscaled_dgrad(const uint8_t* A, const float* sA, const uint8_t* B,
                                                const float* sB, const int32_t* offsets, int32_t E, int64_t Mtot,
                                                int64_t N, int64_t K, uint16_t* D, fp8q_stream_t stream);

/*
 * 128x1 transposed quantisation over expert-grouped rows: the operand form of the grouped Wgrad
 * (the groups lie along the tokens, [REPOST] paragraph 4).  Rows offsets[e] .. offsets[e+1]-1 of
 * x [Mtot, C] (bf16) are expert e's tokens.  Expert e's 128-token groups start at its first row;
 * a final partial group takes its max-abs over the tokens it has (equivalently: the expert's rows
 * zero-padded to a multiple of 128).  With P[e] = sum over e' < e of ceil(n_e' / 128):
 *   qt : [C, Kcap] codes; expert e's tokens at columns 128 P[e] .., zero codes in its padding
 *   s  : [Kcap / 128, C] fp32 scales; group P[e] + j is expert e's j-th group
 * Columns and groups at or past 128 P[E] are not written.  offsets: DEVICE int32 [E + 1], checked
 * on the device (0-based, nondecreasing, ending at Mtot, 128 P[E] <= Kcap; otherwise
 * FP8Q_DEV_BAD_OFFSETS is latched and nothing is written).  Kcap = 128 (ceil(Mtot/128) + E) always
 * suffices.  C % 64 == 0 and Kcap % 128 == 0 (FP8Q_ERR_SHAPE); E <= 1024.
 */
FP8Q_API int fp8q_act_128x1_transposed_ragged(const uint16_t* x, const int32_t* offsets, int32_t E, int64_t Mtot,
                                              int64_t C, uint8_t* qt, float* s, int64_t Kcap,
                                              fp8q_stream_t stream);

/*
 * Grouped Wgrad: dW_e = dY_e^T X_e for every expert, each summing over its own tokens ([REPOST]
 * paragraphs 2-3: Wgrad in FP8, FP32 gradients).  The operands are the ragged 128x1 forms above:
 *   A  : dY^T codes [M, Kcap],  sA : [Kcap/128, M]   (fp8q_act_128x1_transposed_ragged of dY)
 *   B  : X^T codes [N, Kcap],   sB : [Kcap/128, N]   (the same of X)
 *   offsets : the token offsets [E + 1] both were quantised with (DEVICE int32), Mtot tokens
 *   D  : fp32 [E, M, N]; an expert without tokens gets dW_e = 0.
 * M % 128 == 0, N % 128 == 0, Kcap % 128 == 0 (FP8Q_ERR_SHAPE); E <= 1024.  Malformed offsets
 * (including 128 P[E] > Kcap) latch FP8Q_DEV_BAD_OFFSETS and write nothing.
 */
FP8Q_API int fp8_grouped_gemm_blockscaled_wgrad(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                                                const int32_t* offsets, int32_t E, int64_t Mtot, int64_t M, int64_t N,
                                                int64_t Kcap, float* D, fp8q_stream_t stream);

/*
 * Power-of-two (UE8M0) scale variant.  A separate mode with its own scale semantics, not one the
 * pages describe: the block-scaled tensor-core MMA of sm_100a (tcgen05.mma kind::mxf8f6f4) takes
 * per-32-element scales as 8-bit exponents (UE8M0) and applies them inside the MMA, so the GEMM
 * accumulates the whole K in the tensor core's FP32 accumulator with no per-128-K promotion.
 * Groups stay 1x128, 128x1 and 128x128; only the scale of a group changes:
 *   a = max(max|x| over g, 2^-100);  r = a / 448 (binary32, round to nearest);
 *   s = the smallest power of two >= r (stored as an fp32 value, exactly a power of two);
 *   q = E4M3(x * (1 / s)), 1 / s an exact power of two.
 * The *_fmt quantisers take scale_fmt = FP8Q_SCALE_FP32 (identical to the entry point without
 * the suffix) or FP8Q_SCALE_UE8M0; other arguments, layouts and errors as those entry points
 * (FP8Q_ERR_ARG for an unknown scale_fmt).
 */
FP8Q_API int fp8q_act_1x128_fmt(const uint16_t* x, int64_t M, int64_t K, uint8_t* q, float* s, int scale_fmt,
                                fp8q_stream_t stream);
FP8Q_API int fp8q_act_128x1_transposed_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* qt, float* s,
                                           int scale_fmt, fp8q_stream_t stream);
FP8Q_API int fp8q_act_dual_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* q, float* s, uint8_t* qt,
                               float* st, int scale_fmt, fp8q_stream_t stream);
FP8Q_API int fp8q_quant_forward_fmt(const uint16_t* x, int64_t T, int64_t C, uint8_t* xq, float* xs, uint8_t* xqt,
                                    float* xst, const uint16_t* w, int64_t N, uint8_t* wq, float* ws,
                                    uint8_t* wqt_or_null, int scale_fmt, fp8q_stream_t stream);
FP8Q_API int fp8q_weight_128x128_fmt(const uint16_t* w, int64_t N, int64_t K, uint8_t* q, float* s,
                                     uint8_t* qt_or_null, int scale_fmt, fp8q_stream_t stream);

/*
 * Block-scaled FP8 GEMM for power-of-two scales: D = sum_k A^(m, k) B^(k, n) with the dequantised
 * operands A^ = dec(A) sA, B^ = dec(B) sB, computed by tcgen05.mma kind::mxf8f6f4 with each
 * 128-group's scale exponent replicated over its four 32-element blocks; the products are exact
 * and the whole K is accumulated in FP32 by the tensor core.  Arguments, operand layouts,
 * modes (FP8Q_FPROP, FP8Q_DGRAD, FP8Q_WGRAD, FP8Q_WGRAD_ACC), requirements, workspace and return
 * codes exactly as fp8_gemm_blockscaled, except that every scale read must be a positive normal
 * power of two (the FP8Q_SCALE_UE8M0 quantisers produce only such scales); any other scale latches
 * FP8Q_DEV_BAD_SCALES and leaves D unspecified.  Scales of rows past M are not read.
 */
FP8Q_API int fp8_gemm_blockscaled_ue8m0(int mode, const uint8_t* A, const float* sA, const uint8_t* B,
                                        const float* sB, void* D, int64_t M, int64_t N, int64_t K,
                                        void* workspace, size_t ws_bytes, fp8q_stream_t stream);

/*
 * Synchronise `stream`, then read and clear the device status word of the current device.
 * *out receives FP8Q_DEV_OK or the first error latched since the last call.  Returns FP8Q_OK,
 * FP8Q_ERR_ARG (out == NULL) or FP8Q_ERR_CUDA.
 */
FP8Q_API int fp8q_device_status(fp8q_stream_t stream, int* out);

/*
 * Self-test of the device-side error path (no counterpart on the pages): launches one CTA that
 * waits on a barrier nothing ever completes, with the same bounded wait the GEMM pipeline uses
 * but a limit of `limit_ns` (1 .. 2e9).  The wait expires, FP8Q_DEV_TIMEOUT is latched and the
 * kernel returns; the context stays usable.  Returns FP8Q_ERR_ARG for a limit out of range.
 */
FP8Q_API int fp8q_selftest_wait_timeout(uint64_t limit_ns, fp8q_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
