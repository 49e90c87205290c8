/*
 * nvq.h - C ABI of the NVFP4 x Q8_0 dequantise-and-dot library (B200, sm_100a).
 *
 * The library computes the fused dequantise-and-dot product used in
 * quantised LLM inference: 4-bit block-scaled weights (NVFP4) times 8-bit
 * block-quantised activations (Q8_0), for decode (matrix-vector, M = 1..16)
 * and prefill (GEMM, M up to thousands of tokens).
 *
 * Sources of the operations (web pages, cited by title and section):
 *  - "HANDOFF: flint CPU optimization (Q4_1 + NVFP4)", section 3 "Code map
 *    (NVFP4 work)": the NVFP4-weight x Q8_0-activation row dot
 *    (ggml_vec_dot_nvfp4_q8_0), weights handled in 64-element blocks with one
 *    scale per 16 elements; the tiled prefill kernels on the same operands;
 *    and the "Bias trick" paragraph: integer weight codes 2*E2M1 (-12..12)
 *    and sum(w*a) = sum((w+12)*a) - 12*bsum16.
 *  - The spke.com tutorial on 2-bit GGUF builds of a 27B model, GGML type
 *    table (download step): Q8_0 = 32 int8 values + one fp16 scale, 34 bytes.
 *  - "TKintegers K5: 3.21x prefill and 3.10x decode throughput vs TorchAO
 *    FP8 on NVIDIA L4": compact weight tiles expanded to FP16 tensor-core
 *    operands with FP32 accumulation (the prefill GEMM's design); and the
 *    NVFP4 tensor-core engines it links to, which run both operands in
 *    NVFP4 (nvq_gemm_nvf4).
 *  - "HANDOFF ...", section 7 "Open items / next steps": item 1, the
 *    mixture-of-experts product (mul_mat_id; nvq_moe_gemv); item 2, the
 *    per-32 costs of the accumulation (the fused requantisation of
 *    nvq_gemv_requant).
 *  - "Roofline-First Decoding: results": a fused 4-bit dequantise-plus-GEMV
 *    on fp16 activations for batch-1 decoding (nvq_gemm_w4a16).
 *
 * Data formats (all planar, row-major, owned by the caller):
 *  - NVFP4 weights W[N, K]:
 *      codes  uint8 [N, K/2]  : E2M1 codes, element 2i in the low nibble of
 *                               byte i and element 2i+1 in the high nibble;
 *                               bit 3 of a code is the sign, codes 0..7 are
 *                               0, .5, 1, 1.5, 2, 3, 4, 6 (OCP MX E2M1).
 *      scales uint8 [N, K/16] : one UE4M3 scale per 16-element subblock
 *                               (E4M3 with sign 0, bias 7; max 448 = 0x7E;
 *                               bytes >= 0x7F are not valid scales).
 *      g      float           : per-tensor scale.
 *      w[n,k] = g * UE4M3(scales[n,k/16]) * E2M1(code[n,k]).
 *  - Q8_0 activations A[M, K]:
 *      q      int8   [M, K]     : codes in -127..127.
 *      d      uint16 [M, K/32]  : IEEE binary16 bit patterns, one per 32.
 *      a[m,k] = fp16(d[m,k/32]) * q[m,k].
 *  - Output y float [M, N], row-major, overwritten (never accumulated into):
 *      y[m,n] = sum_k w[n,k] * a[m,k]
 *             = sum over 16-subblocks sb of g*s_w*d_a*0.5*isum[m,n,sb],
 *      isum[m,n,sb] = sum over the subblock of (2*E2M1(code)) * q.
 *    Accuracy: |y - exact| <= 1e-5 * sum_sb |term_sb| + 1e-6 per element.
 *
 * Conventions shared by every entry point:
 *  - Shapes: the NVFP4 x Q8_0 products take K a positive multiple of 64
 *    (the 64-element blocks of the row dot); each entry point states its
 *    own further conditions.  The empty product (N == 0 or M == 0) is
 *    accepted and does nothing.
 *  - Device pointers must be 16-byte aligned (NVQ_ERR_MISALIGNED).
 *  - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *    stream.  Device entry points only enqueue work and return at once;
 *    results are ready when the stream reaches them.
 *  - The library allocates no device memory and keeps no state beyond a
 *    per-device cache of attributes.  It never prints and never aborts.
 *  - Errors: arguments are validated on the host before anything is
 *    enqueued, so a non-OK status other than NVQ_ERR_CUDA means nothing was
 *    launched.  NVQ_ERR_CUDA reports a CUDA runtime error seen while
 *    launching (cudaGetLastError); nvq_last_cuda_error() names it.
 *  - Entry points may be called from several host threads at once.
 */
#ifndef NVQ_H_
#define NVQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int nvq_status;

#define NVQ_OK                     0
#define NVQ_ERR_INVALID_ARG        1  /* NULL pointer, negative size, bad value */
#define NVQ_ERR_BAD_SHAPE          2  /* K % 64 != 0, M out of the entry's range */
#define NVQ_ERR_MISALIGNED         3  /* a device pointer not 16-byte aligned */
#define NVQ_ERR_CUDA               4  /* CUDA runtime error while launching */
#define NVQ_ERR_UNSUPPORTED_DEVICE 5  /* current device is not sm_100 */
#define NVQ_ERR_WORKSPACE          6  /* workspace missing or too small */

/* Library version, major*10000 + minor*100 + patch. */
int nvq_version(void);

/* Short English description of a status code (a static string). */
const char* nvq_status_string(nvq_status status);

/* Name of the last CUDA error an entry point met on this host thread
 * (a static string; "cudaSuccess" if none). */
const char* nvq_last_cuda_error(void);

/*
 * nvq_pack_nvfp4 - host-side NVFP4 packer of fp32 weights (not timed; used
 * by generators and loaders).
 *
 * w      host float [N, K] row-major, finite values.
 * codes  host uint8 [N, K/2], scales host uint8 [N, K/16], g host float*:
 *        outputs, caller-owned.
 * Recipe, fp32 with one rounding per operation: g = amax(|w|) / (6*448);
 * per 16-element subblock s = UE4M3(amax_blk / (6*g)) (nearest, ties to
 * even, saturating at 448); code = E2M1(w / (g*s)) (nearest, ties to even,
 * saturating at 6, zero stored as +0); a subblock whose s or g*s is 0 stores
 * codes 0.  Requires K % 16 == 0 (K % 64 for the device entry points).
 * Runs on the calling thread plus up to hardware_concurrency helper threads.
 * Errors: NVQ_ERR_INVALID_ARG (NULL, negative sizes, non-finite w),
 * NVQ_ERR_BAD_SHAPE (K % 16 != 0).
 */
nvq_status nvq_pack_nvfp4(const float* w, int64_t N, int64_t K,
                          uint8_t* codes, uint8_t* scales, float* g);

/*
 * nvq_quantize_act_q8_0 - fused Q8_0 activation quantiser (one pass).
 *
 * x  device float [M, K] row-major, finite values.
 * q  device int8 [M, K], d device uint16 (fp16 bits) [M, K/32]: outputs.
 * Per 32-element block, fp32 IEEE arithmetic: amax = max|x|,
 * d32 = amax / 127 (correctly rounded division), q = rint(x / d32) (true
 * division, round half to even) clamped to +-127, d = fp16(d32) (round to
 * nearest even).  A block with d32 == 0 gives q = 0, d = 0.  Bit-exact.
 * Errors: NVQ_ERR_INVALID_ARG, NVQ_ERR_BAD_SHAPE (K % 32 != 0),
 * NVQ_ERR_MISALIGNED, NVQ_ERR_UNSUPPORTED_DEVICE, NVQ_ERR_CUDA.
 */
nvq_status nvq_quantize_act_q8_0(const float* x, int64_t M, int64_t K,
                                 int8_t* q, uint16_t* d, void* stream);

/*
 * nvq_gemv - decode GEMV, y[M, N] = A[M, K] . W[N, K]^T for M = 1..16.
 *
 * HBM-streaming kernel: each weight byte is read once with 128-bit loads;
 * E2M1 codes are decoded in registers to the integer LUT 2*E2M1, the
 * per-subblock integer sums are formed with dp4a, rescaled by s_w*d_a in
 * fp32 and reduced across the warp; y = 0.5*g*acc.
 * Errors: NVQ_ERR_INVALID_ARG, NVQ_ERR_BAD_SHAPE (K % 64 != 0, M outside
 * 1..16), NVQ_ERR_MISALIGNED, NVQ_ERR_UNSUPPORTED_DEVICE, NVQ_ERR_CUDA.
 */
nvq_status nvq_gemv(const uint8_t* codes, const uint8_t* scales, float g,
                    int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                    int64_t M, float* y, void* stream);

/*
 * nvq_gemv_requant - one token's GEMV (nvq_gemv with M = 1) whose epilogue
 * also emits the Q8_0 quantisation of its output, the activation format the
 * next product of a decoder layer reads (y is a layer's output, Q8_0(y) the
 * next layer's input: "HANDOFF: flint CPU optimization (Q4_1 + NVFP4)",
 * section 7 "Open items / next steps", item 2, on the per-32 costs around
 * the NVFP4 x Q8_0 accumulation; the GGML type table of the spke.com 2-bit
 * GGUF tutorial for Q8_0).
 *
 * y       device float [N]: as nvq_gemv.
 * q_out   device int8 [N], d_out device uint16 (fp16 bits) [N/32]: Q8_0 of y,
 *         bit-identical to nvq_quantize_act_q8_0 applied to this y.
 * counters device int32 [N/32], 16-byte aligned: block arrival counters.
 *         They must be zero before the first call; every call that completes
 *         leaves them zero (a call that timed out may not: zero them again).
 *         Calls that overlap on the GPU need their own counters.
 * The block of 32 outputs is quantised by whichever CTA stores its last
 * output.  Requires N % 32 == 0.  For K outside the register schedule (K =
 * 1024 * T, T in {4,5,6,8,10,12,15,16,20,25}) the call runs nvq_gemv and
 * then the quantiser (two launches, same results).
 * Errors: as nvq_gemv; NVQ_ERR_BAD_SHAPE when N % 32 != 0.
 */
nvq_status nvq_gemv_requant(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                            int64_t K, const int8_t* q, const uint16_t* d, float* y,
                            int8_t* q_out, uint16_t* d_out, int32_t* counters, void* stream);

/* One NVFP4 weight matrix W[N, K] in device memory (caller-owned). */
typedef struct nvq_linear {
  const uint8_t* codes;   /* device uint8 [N, K/2]  */
  const uint8_t* scales;  /* device uint8 [N, K/16] */
  float g;                /* per-tensor scale       */
  int64_t N;
  int64_t K;
} nvq_linear;

/*
 * nvq_gemv_grouped - nvq_gemv of several weight matrices with the same K
 * against the same Q8_0 activations (the q, k and v projections of a layer;
 * up and gate), ys[i][M, N_i] = A . W_i^T.
 *
 * linears  host array of `count` descriptors (read during the call).
 * ys       host array of `count` device float pointers.
 * For one token the matrices share launches of the register schedule, up to
 * three per launch with their rows concatenated, so the row ranges of the
 * SMs stay balanced over the group; other M run one nvq_gemv per matrix.
 * Results are those of nvq_gemv on each matrix.
 * Errors: as nvq_gemv; NVQ_ERR_BAD_SHAPE when the K differ.
 */
nvq_status nvq_gemv_grouped(const nvq_linear* linears, int64_t count, const int8_t* q,
                            const uint16_t* d, int64_t M, float* const* ys, void* stream);

/*
 * nvq_moe_gemv - the mixture-of-experts product of decode (mul_mat_id):
 * every token times the weight matrices of the experts its routing selects,
 * y[t, j, :] = A[t, :] . W_{ids[t, j]}^T.  ("HANDOFF: flint CPU optimization
 * (Q4_1 + NVFP4)", section 7 "Open items / next steps", item 1: the NVFP4 x
 * Q8_0 row dot on a mixture-of-experts shape, K = 2048, 256 experts, 6
 * active per token.)
 *
 * codes   device uint8 [E, N, K/2], scales device uint8 [E, N, K/16]: the E
 *         experts' NVFP4 matrices W_e[N, K], stacked.
 * g       device float [E]: per-expert tensor scales.
 * ids     device int32 [T, top_k]: the experts of each token (read on the
 *         device, so the routing may come from a previous kernel).
 * q, d    device Q8_0 activations [T, K], [T, K/32].
 * y       device float [T, top_k, N].
 * Each token's CTAs stream its selected experts' rows (concatenated, split
 * evenly) with the register schedule of nvq_gemv, so the result of every
 * slot is that of nvq_gemv on its expert.  Requires K = 1024 * T' with T' in
 * {2,3,4,5,6,8,10,12,15,16,20,25} and 1 <= top_k <= 8 (NVQ_ERR_BAD_SHAPE
 * otherwise), T <= 65535.  An id outside 0..E-1 is skipped (its slot of y is
 * left as it was) and raises NVQ_FLAG_BAD_INDEX (nvq_error_flags).
 * Errors: NVQ_ERR_INVALID_ARG, NVQ_ERR_BAD_SHAPE, NVQ_ERR_MISALIGNED,
 * NVQ_ERR_UNSUPPORTED_DEVICE, NVQ_ERR_CUDA.
 */
nvq_status nvq_moe_gemv(const uint8_t* codes, const uint8_t* scales, const float* g, int64_t E,
                        int64_t N, int64_t K, const int32_t* ids, int64_t T, int64_t top_k,
                        const int8_t* q, const uint16_t* d, float* y, void* stream);

/*
 * nvq_gemm_workspace_size - bytes of device workspace nvq_gemm needs for
 * M tokens of K features (0 when M == 0).  It holds the activations
 * expanded to the exact fp16 pair (hi, lo) with hi + lo = d*q and, for
 * M > 16, two 64 KB slots of fp32 partial sums per SM of the current device
 * (query it with the device that will run the GEMM current).
 */
size_t nvq_gemm_workspace_size(int64_t M, int64_t N, int64_t K);

/*
 * nvq_gemm - y[M, N] = A[M, K] . W[N, K]^T for any M >= 1: the prefill GEMM
 * on the tcgen05 tensor cores, and the small-batch decode of several
 * sequences.  Three schedules, chosen by the call:
 *
 *  - M <= 4: the decode GEMV (nvq_gemv), which streams the weights faster
 *    there (its integer dot costs little per token); the workspace is unused.
 *  - 5 <= M <= 16 and K % 256 == 0: the small-token tensor-core schedule.
 *    One CTA per SM; the (128-row tile, 256-wide K stage) units are split
 *    into equal contiguous ranges (a tile two CTAs share is added from fp32
 *    partials in the workspace, in a fixed order, by a second launch); 16
 *    warps expand the weights into tensor memory; tcgen05.mma with N = 2 x
 *    (tokens padded to 8 or 16) takes the exact hi/lo activations (below)
 *    from shared memory; accumulators are promoted to fp32 registers every
 *    1024 K.  Results are deterministic.
 *  - otherwise: the prefill schedule on persistent CTA pairs (one per two
 *    SMs): tiles of 128 tokens x 256 weight rows, the weights expanded in
 *    tensor memory, one tcgen05.mma (kind::f16, cta_group::2, M = N = 256,
 *    K = 16) per K-step forming the hi and the lo products in separate
 *    accumulator columns; each chunk of up to 5120 K is added in fp32 (hi +
 *    lo) to the tile's running sum.  Whole tiles go round-robin over the
 *    pairs; the K stages of the last partial wave's tiles are split evenly
 *    over all pairs, whose parts (fp32, in the workspace) a second launch
 *    adds in K order.  Results are deterministic.
 *
 * The tensor-core schedules expand the activations once into `workspace` as
 * fp16 pairs hi = fp16(d*q), lo = fp16(d*q - hi), exact (hi + lo == d*q),
 * and the weights to fp16 w' = E2M1*s_w (exact); every product is exact
 * and only the fp32 accumulation rounds; y = g * sum.
 * workspace: device, caller-owned, >= nvq_gemm_workspace_size(M, N, K)
 * bytes, 16-byte aligned; its contents are scratch.
 * Errors: as nvq_gemv (M >= 1), plus NVQ_ERR_WORKSPACE.
 */
nvq_status nvq_gemm(const uint8_t* codes, const uint8_t* scales, float g,
                    int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                    int64_t M, float* y, void* workspace,
                    size_t workspace_bytes, void* stream);

/*
 * nvq_gemm_w4a16 - NVFP4 weights times fp16 activations (W4A16), the fused
 * 4-bit dequantise-plus-GEMV of batch-1 decoding in "Roofline-First
 * Decoding: results", for M = 1..16 tokens:
 * y[m, n] = sum_k w[n, k] * x[m, k].
 *
 * x          device uint16 [M, K]: IEEE binary16 bit patterns (finite).
 * workspace  device, >= nvq_gemm_w4a16_workspace_size(M, N, K) bytes,
 *            16-byte aligned, scratch.
 * Runs the small-token tensor-core schedule of nvq_gemm with the
 * activations taken as they are (an fp16 value is already an exact operand;
 * the second operand row of each token is zero): w' = E2M1*s_w in fp16,
 * every product exact, fp32 accumulation promoted every 1024 K, y = g*sum.
 * Accuracy: |y - exact| <= 1e-5 * sum_k |w*x| + 1e-6 per element (the
 * products are the terms: there are no integer subblock sums here).
 * Requires K % 256 == 0 and 1 <= M <= 16 (NVQ_ERR_BAD_SHAPE).
 * Errors: as nvq_gemm.
 */
size_t nvq_gemm_w4a16_workspace_size(int64_t M, int64_t N, int64_t K);
nvq_status nvq_gemm_w4a16(const uint8_t* codes, const uint8_t* scales, float g, int64_t N,
                          int64_t K, const uint16_t* x, int64_t M, float* y, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * nvq_quantize_act_nvfp4 - fp32 activations to NVFP4, one fp32 scale per
 * token: the operand of nvq_gemm_nvf4.  The NVFP4 x NVFP4 engines that
 * "TKintegers K5: 3.21x prefill and 3.10x decode throughput vs TorchAO FP8
 * on NVIDIA L4" points to (and the NVFP4 rows of the lab-benchmarks card)
 * quantise activations to the weights' 4-bit format; this library takes the
 * weight recipe of nvq_pack_nvfp4 row by row:
 *   g[m] = amax(|x[m, :]|) / 2688;  per 16 elements s = UE4M3(amax_blk/(6 g[m]));
 *   code = E2M1(x / (g[m] * s)),
 * fp32 with one IEEE rounding per operation, round to nearest with ties to
 * the even code, saturating; a zero magnitude is stored as +0 and a
 * subblock whose 6*g or g*s is 0 stores codes 0.
 * x       device fp32 [M, K] row-major, finite.
 * codes   device uint8 [M, K/2] out: element 2i in the low nibble of byte i.
 * scales  device uint8 [M, K/16] out; g device fp32 [M] out.
 * Requires K % 16 == 0 (NVQ_ERR_BAD_SHAPE).  Results are bit-identical to
 * nvq_pack_nvfp4 applied to each row on its own.
 * Errors: NVQ_ERR_INVALID_ARG, NVQ_ERR_BAD_SHAPE, NVQ_ERR_MISALIGNED,
 * NVQ_ERR_UNSUPPORTED_DEVICE, NVQ_ERR_CUDA.
 */
nvq_status nvq_quantize_act_nvfp4(const float* x, int64_t M, int64_t K, uint8_t* codes,
                                  uint8_t* scales, float* g, void* stream);

/*
 * nvq_gemm_nvf4 - NVFP4 weights times NVFP4 activations on the tensor
 * core's block-scaled FP4 path (tcgen05.mma kind::mxf4nvf4, one UE4M3 scale
 * per 16 elements on both operands):
 *   y[m, n] = g_w * a_g[m] * sum_k (s_w E2M1_w)[n, k] * (s_a E2M1_a)[m, k].
 * w_codes/w_scales/g_w  weights as nvq_pack_nvfp4 writes them ([N, K/2],
 *                       [N, K/16], tensor scale).
 * a_codes/a_scales/a_g  activations as nvq_quantize_act_nvfp4 writes them
 *                       ([M, K/2], [M, K/16], fp32 [M]).
 * y                     device fp32 [M, N] out.
 * Every product of two E2M1 values and two UE4M3 scales is exact in fp32;
 * the sums accumulate in fp32 in tensor memory and are promoted to fp32
 * registers every 1024 K.  Accuracy: |y - exact| <= 1e-5 * sum_k |w*a| +
 * 1e-6 per element, exact being the fp64 product of the dequantised
 * operands.
 * Requires K % 256 == 0 and N <= 65535*128 (NVQ_ERR_BAD_SHAPE).
 * No workspace.  Errors: as nvq_gemm; a pipeline wait that gives up raises
 * NVQ_FLAG_GEMM_TIMEOUT.
 */
nvq_status nvq_gemm_nvf4(const uint8_t* w_codes, const uint8_t* w_scales, float g_w, int64_t N,
                         int64_t K, const uint8_t* a_codes, const uint8_t* a_scales,
                         const float* a_g, int64_t M, float* y, void* stream);

/*
 * nvq_gemm_noalloc - nvq_gemm for callers that cannot allocate device memory
 * and cannot hand the library a workspace.  (An addition of this library;
 * the web pages describing the method have no counterpart.)
 *
 * Some callers may not allocate: code that runs inside a host framework
 * which owns every device allocation (through its own pool or arena) and
 * gives its plugins no scratch, and latency-critical serving loops that must
 * not call cudaMalloc, which can synchronise the device and fragment memory.
 * This entry point needs neither: it keeps the GEMM's scratch (the expanded
 * activations) in a 64 MiB array of device memory that the library itself
 * holds on every GPU that loads it, from load until the process exits.  It
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments, layouts, result and accuracy are those of nvq_gemm (y is the
 * same); there is no workspace argument.  Limit: the problem must fit the
 * scratch, nvq_gemm_workspace_size(M, N, K) <= 64 MiB, i.e. roughly
 * 4 * ceil(M/128)*128 * K bytes plus 128 KB per SM (on a 148-SM B200, for
 * example M = 2048 up to K = 5760, or M = 256 up to K = 46528); larger
 * problems return NVQ_ERR_WORKSPACE and should use nvq_gemm with a caller
 * workspace.
 * Set-up: the first call on a device looks up the scratch's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The address is cached per device and context;
 * a call made in another context (for example after cudaDeviceReset) looks
 * it up again, so that call too must come before any capture.
 * Sharing: every call, on every stream and host thread, uses the same
 * array, so calls whose work overlaps on the GPU race and corrupt each
 * other's results; serialise them (one stream, or events).  The array keeps
 * the last call's contents; nothing in it needs to start at zero, since
 * each call writes every byte it reads before reading it.
 * Errors: as nvq_gemm, with NVQ_ERR_WORKSPACE for problems over the limit.
 */
nvq_status nvq_gemm_noalloc(const uint8_t* codes, const uint8_t* scales, float g,
                            int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                            int64_t M, float* y, void* stream);

/*
 * nvq_debug_subblock_sums - nvq_gemv that also exports the integer per-16
 * subblock sums it forms, for bit-exact checking ("HANDOFF: flint CPU
 * optimization (Q4_1 + NVFP4)", section 3: the row dot forms one integer sum
 * per 16-element subblock; "Bias trick": the decode path stores the codes
 * +12-biased and removes the bias with -12*bsum16).
 *
 * Arguments as nvq_gemv, plus
 * isum  device int32 [M, N, K/16]:
 *       isum[m, n, sb] = sum_{k in sb} (2*E2M1(code[n,k])) * q[m,k]
 *       (|isum| <= 16*12*127), 16-byte aligned.
 * The call dispatches exactly as nvq_gemv does and runs the same schedule,
 * decode (biased or signed LUT) and dp4a code, instantiated to also store
 * the sums; y receives the same values nvq_gemv writes.
 * Errors: as nvq_gemv; NVQ_ERR_INVALID_ARG / NVQ_ERR_MISALIGNED for isum.
 */
nvq_status nvq_debug_subblock_sums(const uint8_t* codes, const uint8_t* scales, float g,
                                   int64_t N, int64_t K, const int8_t* q, const uint16_t* d,
                                   int64_t M, float* y, int32_t* isum, void* stream);

/* Bits of nvq_error_flags. */
#define NVQ_FLAG_GEMV_TIMEOUT 1u  /* a GEMV pipeline wait gave up (4 s)  */
#define NVQ_FLAG_GEMM_TIMEOUT 2u  /* a GEMM pipeline wait gave up (4 s)  */
#define NVQ_FLAG_BAD_INDEX    4u  /* nvq_moe_gemv met a routing id outside 0..E-1 */

/*
 * nvq_error_flags - device-side error flags of the current device.
 *
 * Every pipeline wait inside the kernels (a consumer waiting for a copy, a
 * producer for a free stage, the tensor-core issuer for its operands) is
 * bounded: after 4 s without progress the kernel raises a flag, stops
 * issuing, lets the copies it issued land, frees its tensor memory and
 * returns instead of hanging.  The outputs of a call whose kernel timed out
 * are not valid, and the call itself has already returned NVQ_OK (it only
 * enqueued work), so callers that need the guarantee read the flags after
 * synchronising the streams they used.
 * flags  host uint32 out: NVQ_FLAG_* bits raised since the last clear.
 * clear  nonzero: reset the flags after reading them.
 * The read is synchronous (a device-to-host copy on the legacy stream).
 * Errors: NVQ_ERR_INVALID_ARG (flags NULL), NVQ_ERR_UNSUPPORTED_DEVICE,
 * NVQ_ERR_CUDA.
 */
nvq_status nvq_error_flags(unsigned int* flags, int clear);

/*
 * nvq_debug_stalled_wait - test-only: run one pipeline wait that can never
 * complete (a stage whose copy is never issued), through the same bounded
 * wait as the GEMV kernels, with a limit of limit_ns (1 us .. 1 s).  The
 * kernel gives up after the limit, raises NVQ_FLAG_GEMV_TIMEOUT and returns.
 * result  device int32 [2] (16-byte aligned): result[0] = 1 if the wait
 *         completed (it cannot), result[1] = microseconds spent waiting.
 * Errors: NVQ_ERR_INVALID_ARG (NULL, limit out of range),
 * NVQ_ERR_MISALIGNED, NVQ_ERR_UNSUPPORTED_DEVICE, NVQ_ERR_CUDA.
 */
nvq_status nvq_debug_stalled_wait(uint64_t limit_ns, int* result, void* stream);

/* Linears per decoder layer, in execution order. */
#define NVQ_STACK_LINEARS 7

/*
 * nvq_decoder_stack - every linear layer of a dense decoder stack, layer
 * after layer, on one stream, for M tokens: the decode pass (M <= 16, the
 * GEMV) or the prefill pass (M > 16, the tensor-core GEMM).
 *
 * Each layer holds NVQ_STACK_LINEARS matrices in the order q, k, v, o, up,
 * gate, down (linears[7*l + i]), and runs
 *     (q_a, d_a) = Q8_0(x);          y_q, y_k, y_v = W_q a, W_k a, W_v a
 *     (q_a, d_a) = Q8_0(y_v);        y_o = W_o a
 *     (q_a, d_a) = Q8_0(y_o);        y_up, y_gate = W_up a, W_gate a
 *     (q_a, d_a) = Q8_0(y_up);       y_down = W_down a
 * i.e. 7 products and 4 activation quantisations per layer.  Every layer
 * starts again from the same input x: only the linear layers are modelled
 * (no attention, norms or activation functions), so the chain stays in
 * range over any depth.  Shapes: q, k, v have K = hidden (x is [M, hidden]);
 * o.K = v.N; up.K = gate.K = o.N; down.K = up.N; every layer has the shapes
 * of layer 0.
 *
 * linears   host array of 7 * n_layers descriptors (read during the call).
 * x         device float [M, hidden].
 * outs      host array of 7 device float pointers, outs[i] of [M, N_i];
 *           overwritten by every layer, so they hold the last layer's outputs.
 * workspace device scratch of nvq_decoder_stack_workspace_size(linears, M)
 *           bytes (Q8_0 activations, and the fp16 expansion when M > 16).
 * Errors: as nvq_gemv / nvq_gemm, NVQ_ERR_BAD_SHAPE when the shapes do not
 * chain, NVQ_ERR_WORKSPACE.  Launch errors stop the pass at that point.
 */
nvq_status nvq_decoder_stack(const nvq_linear* linears, int64_t n_layers,
                             const float* x, int64_t M, float* const* outs,
                             void* workspace, size_t workspace_bytes,
                             void* stream);

/* Workspace bytes nvq_decoder_stack needs for M tokens (0 on bad input). */
size_t nvq_decoder_stack_workspace_size(const nvq_linear* linears, int64_t M);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* NVQ_H_ */
