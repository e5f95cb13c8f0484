/*
 * awq.h -- C ABI of libawq_b200.so: W4A16 group-quantized linear layer on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (TinyChat: Efficient and Lightweight Chatbot with AWQ,
 * README sections "Speed Benchmarks" and "Usage", step 3):
 *   weights are stored as 4-bit unsigned codes q with one fp16 scale s and one
 *   4-bit zero point z per (output channel, group of 128 input channels)
 *   ("--w_bit 4 --q_group_size 128"; Falcon-7B uses groups of 64, and groups
 *   of 32 are taken too), each weight is w = (q - z) * s, and the layer runs
 *   as W4A16: fp16 activations times 4-bit weights, fp16 output.
 *
 *   y[m][n] = sum_k x[m][k] * W^[n][k],   W^[n][k] = fp16_rne((q - z) * s)
 *
 * Orientation: W is [N][K] (N output channels, K input channels, K
 * contiguous), x is [M][K] and y is [M][N], all row-major.
 *
 * ---------------------------------------------------------------------------
 * Packed layout (ours; the README names only a "-w4-g128-awq.pt" checkpoint)
 * ---------------------------------------------------------------------------
 *   qweight  uint32, (N/16)*(K/128) blocks of 16 x 16 words (K*N/2 bytes)
 *            Block (nb, kb) is 1 KiB, holds output channels n = 16*nb + r
 *            (r = 0..15) and input channels 128*kb .. 128*kb + 127. Word w of
 *            row r holds k = 128*kb + k0(w) + i for i = 0..7: the code of even
 *            i at bits 4*(i/2) .. 4*(i/2)+3 and the code of odd i at bits
 *            16 + 4*(i/2) .. 16 + 4*(i/2)+3. So (word >> 4*j) & 0x000F000F
 *            holds the adjacent pair k0 + 2j, k0 + 2j + 1 as two 16-bit lanes.
 *            For group 128, k0(w) = 8*w. For group 64 or 32, with w = 4*t + j
 *            (t, j = 0..3) and J = group/32, k0(w) = group*(j/J) + 8*(t*J +
 *            j%J): the words with the same j hold whole groups (group j/J of
 *            the block), and words 4t .. 4t+3 hold a piece of every group.
 *            Blocks are grouped by 8 row blocks (128 output channels):
 *            group gi = nb/8 holds R = min(8, N/16 - 8*gi) row blocks and is
 *            stored k-block-major, so block (nb, kb) is block number
 *            8*gi*(K/128) + kb*R + nb%8, and the R blocks of one k-block of
 *            one group (128 x 128 weights) are one contiguous run of R KiB.
 *   scales   fp16  [K/group][N]             (2*N*K/group bytes)
 *   zeros    uint8 [K/group][N/2]           (N*K/(2*group) bytes): the zero
 *            point of even n in the low nibble, of odd n in the high nibble.
 *
 * Quantization (awq_pack), per (n, group) over the group's raw values v:
 *   lo = min v, hi = max v, R = max(hi - lo, 1e-5)
 *   s = fp16_rne(R / 15), z = clamp(rint(-lo / s), 0, 15),
 *   q = clamp(rint(v / s) + z, 0, 15)
 * with every division in fp64 against the stored fp16 s and rint rounding
 * half to even. The pages print no formula; this is the plainest reading of
 * asymmetric min-max 4-bit quantization with fp16 scales and 4-bit zeros.
 *
 * ---------------------------------------------------------------------------
 * Conventions for every entry point
 * ---------------------------------------------------------------------------
 *   Shapes     M >= 0 (M = 0 is a no-op), K > 0 and K % 128 == 0, N > 0 and
 *              N % 16 == 0 (else AWQ_ERR_SHAPE); group 128, 64 or 32, and
 *              K, N <= 2^22, M <= 2^24 (else AWQ_ERR_UNSUPPORTED).
 *   Pointers   device pointers unless stated; all non-null (x and y may be
 *              null when M == 0) and 16-byte aligned (AWQ_ERR_INVALID_ARG /
 *              AWQ_ERR_ALIGNMENT). Outputs may not overlap inputs.
 *   Ownership  the caller allocates and owns every buffer, the workspace
 *              included. The library allocates no device memory; it keeps
 *              only per-device launch parameters (SM count, kernel attributes).
 *   Streams    `stream` is a cudaStream_t (NULL = legacy default stream).
 *              Calls are asynchronous on it; only awq_get_status synchronizes.
 *   Debug      the library built with -DAWQ_DEBUG (weight_only_bit_awq_b200/
 *              build.py --debug: libawq_b200_debug.so, same entry points)
 *              checks the index range of every global and shared access of
 *              the pack, dequant, GEMV and GEMM kernels before it happens; a
 *              failed check records AWQ_ERR_BOUNDS in the status word and
 *              skips the access instead of faulting.
 *   Errors     argument errors are returned before anything is launched;
 *              AWQ_ERR_CUDA reports a failed launch. Errors found on the device
 *              (a non-finite weight in awq_pack, a bounded wait that expired)
 *              are recorded in the workspace status word and read back with
 *              awq_get_status.
 *   Workspace  at least awq_workspace_bytes(M, K, N, group) bytes of device
 *              memory, zeroed once with awq_workspace_init before first use.
 *              Only its status word must start at zero; the GEMV's partial
 *              sums of split rows and the GEMM's stream-K parts of split
 *              tiles are written before they are read. One
 *              workspace must not be used by two calls that can run at the
 *              same time (e.g. on two streams).
 */
#ifndef AWQ_B200_H
#define AWQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum awq_status {
  AWQ_OK = 0,
  AWQ_ERR_INVALID_ARG = 1, /* null pointer, overlapping buffers, bad workspace */
  AWQ_ERR_SHAPE = 2,       /* M < 0, K <= 0, N <= 0, K % 128, N % 16, K % group */
  AWQ_ERR_ALIGNMENT = 3,   /* a pointer that is not 16-byte aligned */
  AWQ_ERR_WORKSPACE = 4,   /* ws_bytes below awq_workspace_bytes(...) */
  AWQ_ERR_UNSUPPORTED = 5, /* group not 32, 64 or 128, M above an entry's limit, no sm_100 device */
  AWQ_ERR_CUDA = 6,        /* a CUDA runtime call or kernel launch failed */
  AWQ_ERR_TIMEOUT = 7,     /* device side: a bounded pipeline wait expired */
  AWQ_ERR_NONFINITE = 8,   /* device side: awq_pack met an inf or NaN weight */
  AWQ_ERR_BOUNDS = 9       /* device side, debug build only: an index check failed (the access was skipped) */
} awq_status;

typedef struct awq_packed_sizes {
  size_t qweight_bytes; /* K*N/2 */
  size_t scales_bytes;  /* 2*N*(K/group) */
  size_t zeros_bytes;   /* N*(K/group)/2 */
} awq_packed_sizes;

/* Largest M accepted by awq_w4a16_gemv (the decode path). */
#define AWQ_GEMV_MAX_M 32

/* Sizes of the three packed buffers for a [N][K] weight. Host only.
 * Returns AWQ_ERR_SHAPE / AWQ_ERR_UNSUPPORTED / AWQ_ERR_INVALID_ARG (out NULL).
 * Source: TinyChat README, Usage step 3 (4-bit codes per group of 128
 * inputs); the byte counts follow from the packed layout above. */
awq_status awq_packed_size(int64_t K, int64_t N, int group, awq_packed_sizes* out);

/* Workspace bytes needed by any entry point below for these sizes on the
 * current device: the status word, plus, when the decode GEMV's plan splits
 * rows between CTAs, its partial sums of those rows, and for M >
 * AWQ_GEMV_MAX_M, when the GEMM's schedule is stream-K, its fp32 parts of
 * split tiles (two slots of 128 x 256 floats per SM at most). Host only.
 * Returns 0 for invalid sizes.
 * Source: none on the pages (the kernels' scratch memory, owned by the caller). */
size_t awq_workspace_bytes(int64_t M, int64_t K, int64_t N, int group);

/* Zero `ws_bytes` bytes of workspace on `stream` (needed once, before the
 * first use of a new workspace).
 * Source: none on the pages (workspace set-up). */
awq_status awq_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/* Quantize and pack (TinyChat README, Usage step 3: "--w_bit 4
 * --q_group_size 128 ... --q_backend real"): W fp16 [N][K] -> qweight,
 * scales, zeros in the layout above, bit for bit the quantization stated
 * above. An inf/NaN weight records AWQ_ERR_NONFINITE in the workspace status
 * word (its group's outputs are then unspecified).
 * Source: TinyChat README, Usage step 3 (the quantization knobs). */
awq_status awq_pack(const void* w, int64_t K, int64_t N, int group, void* qweight, void* scales, void* zeros,
                    void* workspace, size_t ws_bytes, void* stream);

/* Dequantize: W^ fp16 [N][K] = fp16_rne((q - z) * s) for every (n, k). The
 * bit-exact test surface of the packed format; w_out must not overlap the
 * packed buffers.
 * Source: TinyChat README, Usage step 3 (the 4-bit weights with a scale and
 * zero point per group, "--q_backend real" storing them packed); w = (q - z) s
 * is the asymmetric reading stated at the top of this header. */
awq_status awq_dequant(const void* qweight, const void* scales, const void* zeros, int64_t K, int64_t N,
                       int group, void* w_out, void* stream);

/* Decode-stage W4A16 GEMV, 1 <= M <= AWQ_GEMV_MAX_M (README "Speed
 * Benchmarks": per-token latency of the generation stage): y fp16 [M][N] =
 * x fp16 [M][K] . W^T. Streams the packed weights once; fp32 accumulation
 * (M <= 2 with groups of 128: exact integer sums of the codes times a block
 * fixed-point form of x, exact except for inputs below 2^-19 of their
 * 128-input block's largest magnitude). Rows whose k-range is split between
 * CTAs are added in a fixed order, so results are deterministic. A non-finite
 * x[m][k] gives non-finite y[m][*]. M > AWQ_GEMV_MAX_M returns
 * AWQ_ERR_UNSUPPORTED.
 * Source: TinyChat README, Speed Benchmarks (per-token generation latency). */
awq_status awq_w4a16_gemv(const void* x, const void* qweight, const void* scales, const void* zeros, void* y,
                          int64_t M, int64_t K, int64_t N, int group, void* workspace, size_t ws_bytes,
                          void* stream);

/* Context-stage (prefill) W4A16 GEMM for any M (README "New Optimization of
 * Context Stage": the prompt is processed as one batch of tokens): same
 * result as awq_w4a16_gemv, on the tcgen05 tensor cores with fp32
 * accumulation in tensor memory. For M > AWQ_GEMV_MAX_M, where whole output
 * tiles would leave the last wave of SMs short, the k-range of the last tiles
 * is split between CTAs ("stream-K") and a second kernel adds the fp32 parts,
 * which live in the workspace, in a fixed order: results are deterministic
 * for a given device (SM count). Where whole 256-token tiles are used
 * without that split (the large prefill shapes), pairs of SMs share each
 * MMA (clusters of two CTAs, 256 channels x 256 tokens per tile).
 * Source: TinyChat README, New Optimization of Context Stage. */
awq_status awq_w4a16_gemm(const void* x, const void* qweight, const void* scales, const void* zeros, void* y,
                          int64_t M, int64_t K, int64_t N, int group, void* workspace, size_t ws_bytes,
                          void* stream);

/* The linear layer: awq_w4a16_gemv for M <= awq_linear_gemv_limit() (16),
 * and for 16 < M <= AWQ_GEMV_MAX_M when the layer has fewer 128-channel tiles
 * than the device has SMs (ceil(N / 128) < SMs); awq_w4a16_gemm otherwise.
 * The split was measured on B200: the GEMV wins every decode layer up to
 * M = 16, the GEMM wins the wide layers from M = 24.
 * Source: TinyChat README, Speed Benchmarks and New Optimization of Context
 * Stage (the same W4A16 linear layers at decode and at prefill). */
awq_status awq_linear(const void* x, const void* qweight, const void* scales, const void* zeros, void* y,
                      int64_t M, int64_t K, int64_t N, int group, void* workspace, size_t ws_bytes,
                      void* stream);

/* ---------------------------------------------------------------------------
 * W4A8-FP8 variant of the prefill GEMM
 * ---------------------------------------------------------------------------
 * The TensorRT-LLM news item on INT4 AWQ on one H200 says its AWQ kernels
 * compute in FP8 on the tensor cores; the pages print no recipe. This variant
 * keeps the packed 4-bit weights of awq_pack unchanged and runs the MMA on
 * E4M3 (OCP 8-bit floating point, 4 exponent bits, bias 7, 3 fraction bits,
 * largest finite value 448) with fp32 accumulation:
 *   sx[m]   = fp32(max_k |x[m][k]|) / 448                (IEEE fp32 division)
 *   x8[m,k] = e4m3(x[m][k] / sx[m])                      (0 when sx[m] == 0)
 *   e[n]    = the largest integer with 15 * max_g s[n,g] * 2^e <= 448
 *   W8[n,k] = e4m3(fp16((q - z) * fp16(s * 2^e[n])))
 *   y[m][n] = fp16(sum_k x8[m,k] W8[n,k] * sx[m] * 2^-e[n])
 * e4m3() rounds to the nearest E4M3 value, ties to even, saturating at +-448.
 * It is a lossy variant: x and the weights each keep 4 significant bits, so y
 * differs from awq_w4a16_gemm by up to about 2^-3 of sum_k |x W^| (2^-4 from
 * each operand). Typical use per weight: awq_fp8_row_exponents once (offline,
 * like awq_pack); per batch: awq_fp8_quantize_x, then awq_w4a8_gemm. */

/* e[n] (int8, one per output channel) from the packed scales fp16 [K/group][N]
 * as awq_pack wrote them (positive). Shapes and group as for every entry
 * point; scales 16-byte aligned; e_out any alignment, not overlapping scales.
 * Source: TensorRT-LLM news item on INT4 AWQ on one H200 (FP8 compute). */
awq_status awq_fp8_row_exponents(const void* scales, int64_t K, int64_t N, int group, void* e_out, void* stream);

/* x fp16 [M][K] -> x8 E4M3 codes uint8 [M][K] and sx fp32 [M] (formulas above).
 * K % 128 == 0; M >= 0 (0 is a no-op); x, x8 and sx 16-byte aligned and not
 * overlapping. A row holding inf or NaN gives codes and sx that are not
 * finite numbers (NaN, or 0 codes with sx = inf).
 * Source: TensorRT-LLM news item on INT4 AWQ on one H200 (FP8 compute). */
awq_status awq_fp8_quantize_x(const void* x, int64_t M, int64_t K, void* x8, void* sx, void* stream);

/* W8 uint8 [N][K] = the E4M3 codes the W4A8 GEMM multiplies (test surface,
 * like awq_dequant): row_exp is e from awq_fp8_row_exponents.
 * Source: TensorRT-LLM news item on INT4 AWQ on one H200 (FP8 compute). */
awq_status awq_dequant_fp8(const void* qweight, const void* scales, const void* zeros, const void* row_exp,
                           int64_t K, int64_t N, int group, void* w8_out, void* stream);

/* y fp16 [M][N] from x8 [M][K] and sx [M] (awq_fp8_quantize_x), the packed
 * weight and row_exp [N] (awq_fp8_row_exponents): tcgen05.mma kind::f8f6f4
 * on E4M3 operands, fp32 accumulation in tensor memory, the weights
 * dequantized to E4M3 in shared memory just ahead of the MMA. Any M >= 0.
 * x8, sx, y, the packed buffers and the workspace 16-byte aligned; y must not
 * overlap any input. The workspace needs only its status word
 * (ws_bytes >= 256); an expired bounded wait records AWQ_ERR_TIMEOUT there.
 * Source: TensorRT-LLM news item on INT4 AWQ on one H200 (FP8 compute). */
awq_status awq_w4a8_gemm(const void* x8, const void* sx, const void* qweight, const void* scales, const void* zeros,
                         const void* row_exp, void* y, int64_t M, int64_t K, int64_t N, int group, void* workspace,
                         size_t ws_bytes, void* stream);

/* The M at and below which awq_linear always takes the GEMV path (above it,
 * up to AWQ_GEMV_MAX_M, only for layers with fewer 128-channel tiles than SMs).
 * Source: none on the pages (a dispatch threshold set from measurements). */
int awq_linear_gemv_limit(void);

/* Size of the library-owned scratch array behind awq_w4a16_gemv_no_alloc:
 * 1 MiB of device memory on every GPU that loads the library, held until the
 * process exits. */
#define AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES (1u << 20)

/* The decode GEMV (awq_w4a16_gemv, same result bit for bit) for callers that
 * cannot allocate device memory -- e.g. code running inside a fixed memory
 * pool it must not grow, or a plug-in whose host process owns every device
 * allocation. The pages have no counterpart of this entry point. Same
 * arguments as awq_w4a16_gemv minus the workspace: the workspace lives
 * in a static device array of AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES inside the
 * library, so nothing is allocated (no cudaMalloc, no allocating library
 * call). Returns AWQ_ERR_WORKSPACE when these sizes need more scratch than
 * that (awq_workspace_bytes(M, K, N, group) > AWQ_GEMV_NO_ALLOC_SCRATCH_BYTES).
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture. Every call uses the same array: calls that can
 * overlap on the GPU race on it. Each call zeroes the status word (a memset
 * on `stream`) before its kernels run.
 * Source: none on the pages (an allocation-free variant for such callers). */
awq_status awq_w4a16_gemv_no_alloc(const void* x, const void* qweight, const void* scales, const void* zeros,
                                   void* y, int64_t M, int64_t K, int64_t N, int group, void* stream);

/* The device-side status word of awq_w4a16_gemv_no_alloc's scratch array on
 * the current device: synchronize `stream`, then return and clear it (AWQ_OK
 * if nothing was recorded; AWQ_ERR_TIMEOUT if a bounded wait of the GEMV
 * expired). Like the workspace status of awq_get_status, a device-side error
 * is only seen here, so call it after the calls whose outcome matters and
 * before the next awq_w4a16_gemv_no_alloc, which clears the word again.
 * Allocates nothing. AWQ_ERR_CUDA if the synchronization or the copy fails.
 * Source: none on the pages (error reporting of the allocation-free variant). */
awq_status awq_get_status_no_alloc(void* stream);

/* Number of kernels awq_linear launches for these sizes on the current device
 * (1, or 2 when the decode GEMV runs its split-row fixup kernel or the GEMM
 * its stream-K fixup kernel; 0 for M == 0 or invalid sizes). Host only. For
 * launch accounting and graph planning.
 * Source: none on the pages. */
int awq_linear_launches(int64_t M, int64_t K, int64_t N, int group);

/* Which kernel awq_linear runs for these sizes on the current device: 1 = the
 * decode GEMV (awq_w4a16_gemv), 2 = the tensor-core GEMM (awq_w4a16_gemm) on
 * one CTA per tile, 3 = the same GEMM on CTA pairs (256-channel x 256-token
 * tiles); 0 for M == 0 or invalid sizes. Host only.
 * Source: none on the pages (dispatch query). */
int awq_linear_path(int64_t M, int64_t K, int64_t N, int group);

/* Self-test of the kernels' failure detection (the pages have no counterpart):
 * launches one thread that waits, through the same bounded-wait routine the
 * GEMM and GEMV pipelines use, on a barrier phase that nothing completes,
 * giving up after `limit_us` microseconds (1 .. 1000000). The expired wait
 * records AWQ_ERR_TIMEOUT in the workspace status word, which awq_get_status
 * then returns; the CUDA context stays usable. Returns AWQ_OK when launched.
 * Source: none on the pages (failure detection of this library). */
awq_status awq_check_bounded_wait(void* workspace, size_t ws_bytes, uint32_t limit_us, void* stream);

/* Synchronize `stream`, then return and clear the device-side status word of
 * `workspace` (AWQ_OK if no device-side error was recorded).
 * Source: none on the pages (error reporting of this library). */
awq_status awq_get_status(void* workspace, void* stream);

/* Static, human-readable name of a status code.
 * Source: none on the pages. */
const char* awq_status_string(awq_status status);

#ifdef __cplusplus
}
#endif

#endif /* AWQ_B200_H */
