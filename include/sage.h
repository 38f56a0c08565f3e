/*
 * sage.h -- C ABI of the B200 (sm_100a) quantized self-attention library for
 * video diffusion transformers.
 *
 * The operation is the full-sequence self-attention of a video DiT, which
 * page 1 of the TMAP / Taobao Faxiang image-to-video write-up
 * (ai.aiking123.com/155823.html, section "Attention performance
 * optimisation / Background") profiles as aten.scaled_dot_product_flash_attention
 * (73.76% of the model's FLOPs, 72% of runtime), and which it replaces by the
 * SageAttention operator ("attention quantization"), keeping some layers at
 * original precision ("keeping video quality") and guarding the per-channel
 * quantization coefficient against all-zero channels ("operator details").
 *
 * Conventions shared by every entry point:
 *  - Tensors are row-major [B, H, N, d] ("BHND"): tokens contiguous per head,
 *    channels contiguous per token.  d must be 64 or 128, N >= 1, B, H >= 1,
 *    B * H * ceil(N/128) * 128 * d < 2^31.
 *  - Pointers are DEVICE pointers unless a parameter says "host".  Device
 *    pointers must be 16-byte aligned.  The caller owns all memory; the
 *    library allocates nothing and keeps no state between calls, except the
 *    fixed scratch array of sage_quantize_qk_noalloc (see there).
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Calls are asynchronous on that stream; no call synchronises except
 *    sage_status() and sage_attn_fwd_host().
 *  - The device calls allocate nothing and never synchronise, so after one
 *    eager call per device (which sets kernel attributes) they can be
 *    captured into a CUDA graph and replayed; sage_status(),
 *    sage_attn_fwd_host() and the first call of sage_quantize_qk_noalloc on
 *    a device cannot.
 *  - Every function returns SAGE_OK (0) or a negative SAGE_E* code; none
 *    aborts or throws.  Argument errors are detected on the host before any
 *    launch.  Device-side failures (a bounded wait that ran out) are recorded
 *    in the status word inside the workspace and reported by sage_status().
 */
#ifndef SAGE_H
#define SAGE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* attention modes (one per layer, see attn_layer_schedule) */
#define SAGE_MODE_BF16 0      /* exact softmax attention, BF16 tensor-core MMAs */
#define SAGE_MODE_INT8_FP8 1  /* smoothed INT8 QK^T, FP8 e4m3 P.V             */
#define SAGE_MODE_INT8_FP8_QTOKEN 2  /* the same with one Q scale per token  */

/* status codes */
#define SAGE_OK 0
#define SAGE_EINVAL (-1)        /* bad size, null or misaligned pointer, bad mode      */
#define SAGE_EUNSUPPORTED (-2)  /* d not in {64,128}, or the device is not sm_100     */
#define SAGE_ELAUNCH (-3)       /* a CUDA launch or runtime call failed               */
#define SAGE_EWORKSPACE (-4)    /* workspace smaller than sage_workspace_bytes()      */
#define SAGE_ETIMEOUT (-5)      /* a bounded device-side wait ran out (see sage_status) */
#define SAGE_EBOUNDS (-6)       /* a device-side bounds check failed (debug build only) */

/* tile sizes of the quantization blocks and of the attention tiles */
#define SAGE_BLK_Q 128
#define SAGE_BLK_K 128
/* static scale of the FP8 P operand: P8 = e4m3(p * 448), p in [0, 1] */
#define SAGE_P_SCALE 448.0f

/*
 * Bytes of device workspace sage_attn_fwd needs for (B, H, N, d, mode).
 * INT8_FP8: the quantized Q/K/V, their scales, the K mean, prepass partials
 * and a 256-byte status word.  BF16: the status word only.
 * Returns 0 for invalid arguments.
 */
size_t sage_workspace_bytes(int B, int H, int N, int d, int mode);

/*
 * Quantization prepass (steps a1-a4 of the scheme), fused into three kernels:
 *  a1  k_mean[b,h,c] = (1/N) sum_n K[b,h,n,c] (fp64 sums in a fixed order,
 *      rounded once to fp32);
 *  a2  Ks = fp32(K) - k_mean; per 128-token block: amax = max|Ks|,
 *      k_scale = amax/127, k_i8 = clamp(rne(Ks * (127/amax)), -127, 127);
 *  a3  the same for Q without smoothing;
 *  a4  per channel amax over all tokens of V, v_scale = amax/448,
 *      v_f8t = e4m3_rne_satfinite(V * (448/amax)), stored transposed.
 * An all-zero block or channel (amax == 0) gets scale 0 and all-zero codes:
 * no division by zero, no NaN (the fix described under "operator details").
 *
 * q, k, v   bf16 [B,H,N,d]                                  (input)
 * q_i8      int8 [B,H,nQ*128,d], rows >= N zero              (output)
 * q_scale   fp32 [B,H,nQ]                                    (output)
 * k_i8      int8 [B,H,nK*128,d], rows >= N zero              (output)
 * k_scale   fp32 [B,H,nK]                                    (output)
 * k_mean    fp32 [B,H,d]                                     (output)
 * v_f8t     e4m3 [B,H,d,nK*128], token-contiguous, cols >= N zero (output)
 * v_scale   fp32 [B,H,d]                                     (output)
 * scratch   device scratch of sage_prepass_scratch_bytes() bytes (partials)
 * with nQ = nK = ceil(N/128).
 */
size_t sage_prepass_scratch_bytes(int B, int H, int N, int d);
/*
 * The prepass with a choice of Q granularity: q_granularity = 128 is
 * sage_quantize_qk (one Q scale per 128-token block, q_scale [B,H,nQ]);
 * q_granularity = 1 gives one Q scale per token, amax over the token's d
 * channels / 127 with the same rounding and zero guard, q_scale [B,H,nQ*128]
 * (rows >= N get scale 0).  This finer granularity costs nothing in the
 * attention kernel, where each thread owns one query row.  Other values:
 * SAGE_EINVAL.
 */
int sage_quantize_qk_ex(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                        int q_granularity, int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale,
                        float* k_mean, uint8_t* v_f8t, float* v_scale, void* scratch, size_t scratch_bytes,
                        void* stream);
int sage_quantize_qk(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                     int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                     uint8_t* v_f8t, float* v_scale, void* scratch, size_t scratch_bytes,
                     void* stream);

/*
 * Same prepass as sage_quantize_qk, for callers that must not allocate device
 * memory while they run (a service that reserved all of HBM for its own pool,
 * a latency-critical loop that cannot take the implicit synchronisation of
 * cudaMalloc / cudaFree).  The pages this library follows describe no such
 * entry point; it exists for those callers only.
 *  - The prepass partials live in one fixed device array inside the library,
 *    SAGE_NOALLOC_SCRATCH_BYTES (32 MiB) on every device that loads it, held
 *    until the process exits.  The caller passes only inputs and outputs
 *    (same meaning and layout as sage_quantize_qk).
 *  - Problems whose partials need more than that (sage_prepass_scratch_bytes
 *    > SAGE_NOALLOC_SCRATCH_BYTES, e.g. B*H*ceil(N/128)*d above ~1.6M) are
 *    rejected with SAGE_EWORKSPACE before anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.  The address is cached with the id of the
 *    CUDA context it belongs to; the first call in a new context (after
 *    cudaDeviceReset, which also frees the array's old contents) looks it up
 *    again, so that call too must come before any capture.
 *  - Every call shares the one array.  Calls whose kernels may overlap on the
 *    GPU (different streams, or several host threads) race on it and give
 *    wrong results: serialise them on one stream.  Each call overwrites every
 *    partial it later reads, so no clearing is needed between calls.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define SAGE_NOALLOC_SCRATCH_BYTES (32u << 20)
int sage_quantize_qk_noalloc(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                             int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                             uint8_t* v_f8t, float* v_scale, void* stream);

/*
 * Attention over already-quantized operands (steps a5-a9): per 128x128 tile
 * S = Q_i8 K_i8^T in exact int32 (tcgen05 kind::i8), s = S * q_scale * k_scale
 * * log2(e)/sqrt(d), keys >= N masked, online softmax with p = 2^(s - m),
 * P8 = e4m3(p * 448) staged in shared memory (128-byte swizzled K-major tile),
 * O += P8 V8 (tcgen05 kind::f8f6f4 from shared memory, fp32 in tensor
 * memory), O = O * v_scale / (448 * l) rounded to bf16.
 * Operands as written by sage_quantize_qk; o is bf16 [B,H,N,d] (output).
 * status: a 256-byte device status region (e.g. the start of a workspace);
 * failures are OR-ed into its first word.
 */
int sage_attn_quantized(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                        const float* k_scale, const uint8_t* v_f8t, const float* v_scale,
                        void* o, int B, int H, int N, int d, void* status, void* stream);
/* The same with q_scale in the granularity sage_quantize_qk_ex wrote (128 or 1). */
int sage_attn_quantized_ex(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                           const float* k_scale, const uint8_t* v_f8t, const float* v_scale, void* o, int B,
                           int H, int N, int d, int q_granularity, void* status, void* stream);

/*
 * Full-sequence self-attention O = softmax(Q K^T / sqrt(d)) V, non-causal,
 * q, k, v, o bf16 [B,H,N,d].
 * mode SAGE_MODE_INT8_FP8: sage_quantize_qk into the workspace, then
 *   sage_attn_quantized.
 * mode SAGE_MODE_INT8_FP8_QTOKEN: the same with one Q scale per token
 *   (sage_quantize_qk_ex with q_granularity 1).
 * mode SAGE_MODE_BF16: S = Q K^T with BF16 tensor-core MMAs (fp32
 *   accumulate), online softmax in fp32, P rounded to bf16, O += P V
 *   (fp32), O / l rounded to bf16.  Uses only the status word of the workspace.
 * workspace: device buffer of at least sage_workspace_bytes(B,H,N,d,mode)
 * bytes, 256-byte aligned; its first 256 bytes are the status word.
 */
int sage_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int H, int N, int d,
                  int mode, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The same call from host memory, pipelined: the B*H heads are processed in
 * chunks of `chunk_heads` (0: sage_host_chunk_heads()); the host-to-device copy of
 * chunk i+1 and the device-to-host copy of chunk i-1 overlap the attention of
 * chunk i.  Heads are independent (every statistic of the scheme is per head),
 * so the result is bit-for-bit that of sage_attn_fwd on the whole tensor.
 * q_host, k_host, v_host, o_host: HOST bf16 [B,H,N,d]; pinned (page-locked)
 *   memory is needed for the copies to overlap.
 * q_dev, k_dev, v_dev, o_dev: device staging buffers bf16 [B,H,N,d] (caller-owned).
 * workspace: at least sage_host_workspace_bytes(B, H, N, d, mode, chunk_heads)
 *   bytes, 256-byte aligned, zero-filled before the first call: its two halves (each rounded
 *   down to 256 bytes; one when B*H == 1) are the workspaces of alternate
 *   chunks, each with its status word first, at the same offsets whatever the
 *   mode, so one buffer serves calls of every mode.
 * The first and the last chunk take half as many heads (at least one): they
 * are the copies nothing overlaps.  Alternate chunks run on `stream` and on a
 * second compute stream, so one chunk's prepass and attention start while
 * the previous chunk's last wave drains.
 * Runs after earlier work on `stream` and returns when the output is in
 * o_host (it synchronises).  Its three streams (copy in, copy out, second
 * compute stream) and three events are made on the first call on a device
 * (and again in a new CUDA context) and kept until the process exits; calls
 * on one device from several host threads run one after the other.
 * Allocates no device memory.  Returns the status of the call including
 * device-side status (SAGE_ETIMEOUT).
 */
int sage_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host, void* o_host, int B, int H,
                       int N, int d, int mode, void* q_dev, void* k_dev, void* v_dev, void* o_dev,
                       void* workspace, size_t workspace_bytes, int chunk_heads, void* stream);

/*
 * Workspace bytes of sage_attn_fwd_host for this shape, mode and chunk
 * (chunk_heads 0: sage_host_chunk_heads()): two 256-byte aligned copies of
 * sage_workspace_bytes(1, chunk_heads, N, d, mode) (one when B*H == 1).
 * 0 on a bad shape or mode.
 */
size_t sage_host_workspace_bytes(int B, int H, int N, int d, int mode, int chunk_heads);

/*
 * The default chunk of sage_attn_fwd_host: the fewest heads whose attention
 * launch fills four waves of the current device's SMs (148 if no device is
 * usable), at most B*H; 2 heads at the Wan2.1-14B 720p shape.  Small chunks
 * leave less of the first upload and the last download uncovered.  0 on a
 * bad shape.
 */
int sage_host_chunk_heads(int B, int H, int N, int d);

/*
 * Per-layer mode table for selective quantization ("keeping video quality":
 * some attention layers stay at original precision at every denoising step).
 * full_precision_layers (host, n_fp entries, duplicates allowed) -> BF16,
 * every other layer -> INT8_FP8.  modes_out: host int8 [num_layers].
 * Returns SAGE_EINVAL if an index is outside [0, num_layers).
 */
int attn_layer_schedule(int num_layers, const int* full_precision_layers, int n_fp, int8_t* modes_out);

/*
 * Per-layer error calibration for attn_layer_schedule ("keeping video
 * quality": the quantized attention error of each layer is measured over the
 * denoising iterations, and the layers whose error stays large keep the
 * original precision).
 *
 * sage_attn_error_stats: a, b device bf16 [B,H,N,d] (16-byte aligned, d a
 * multiple of 8); stats device fp64 [B*H][4] = per head
 * {sum (a-b)^2, sum b^2, sum a*b, sum a^2} (e.g. a = INT8/FP8 output,
 * b = BF16 output: relative L2 error = sqrt(s0/s1), cosine = s2/sqrt(s1*s3)).
 * Deterministic (fixed summation order).  scratch: device buffer of
 * sage_error_scratch_bytes(B, H) bytes.  Asynchronous on `stream`.
 *
 * sage_attn_rel_l2: the error of one layer at one iteration, the relative L2
 * distance of a from b over every element of the layer (all B*H heads):
 * out = sqrt(sum (a-b)^2 / sum b^2) as one fp64 value written to the device
 * pointer `out` (0 when both sums are 0, +inf when only sum b^2 is).  The
 * per-head sums are formed as in sage_attn_error_stats and added over the
 * heads in ascending order on the device, so the result is deterministic.
 * Same arguments, alignment, scratch and stream rules as
 * sage_attn_error_stats; `out` must be 8-byte aligned.
 *
 * sage_select_full_precision_layers: host layer_err [num_layers][num_iters]
 * (any per-layer, per-iteration error, e.g. sage_attn_rel_l2's); writes, in
 * ascending order, the layers kept at full precision to host
 * layers_out[num_layers] and their count to *n_out; the result feeds
 * attn_layer_schedule.  rule SAGE_SELECT_EVERY_ITERATION (the page's reading:
 * the error is above `threshold` at every iteration) or SAGE_SELECT_MEAN (the
 * mean error over the iterations is above it).  SAGE_EINVAL on a non-finite
 * error, an unknown rule or bad sizes.
 */
enum { SAGE_SELECT_EVERY_ITERATION = 0, SAGE_SELECT_MEAN = 1 };
size_t sage_error_scratch_bytes(int B, int H);
int sage_attn_error_stats(const void* a, const void* b, int B, int H, int N, int d, double* stats,
                          void* scratch, size_t scratch_bytes, void* stream);
int sage_attn_rel_l2(const void* a, const void* b, int B, int H, int N, int d, double* out, void* scratch,
                     size_t scratch_bytes, void* stream);
int sage_select_full_precision_layers(const double* layer_err, int num_layers, int num_iters,
                                      double threshold, int rule, int* layers_out, int* n_out);

/*
 * 8-bit linear layers with 128 x 128 block scales (TMAP write-up, "FFN
 * performance optimisation / linear-layer quantization": the DiT's linear
 * weights and activations in 8 bits -- W8A8 -- with a 128 x 128 per-block
 * quantization operator).  The 8-bit format is symmetric INT8, as in the
 * attention prepass: per block, scale = amax / 127 and
 * code = clamp(rne(x * (127 / amax)), -127, 127); an all-zero block gets
 * scale 0 and codes 0.
 *
 * sage_quantize_blocks_2d: x device bf16 [R, K] row-major (R >= 1, K a
 * positive multiple of 128, ceil(R/128) <= 65535); codes device int8 [R, K];
 * scales device fp32 [ceil(R/128), K/128], scales[rb][kb] for rows
 * 128*rb .. +127 (only the real ones) and columns 128*kb .. +127.  Used for
 * the activations X [M, K] (rows = tokens) and, once, for the weights
 * W [N, K] (rows = output features).
 *
 * sage_linear_w8a8: Y = X W^T + bias from the block-quantized operands:
 *   Y[m, n] = sum over kb = 0 .. K/128-1 (in that order) of
 *             fl(sx[m/128][kb] * sw[n/128][kb]) * S_kb[m, n],
 *   S_kb[m, n] = sum over k in block kb of xq[m, k] * wq[n, k] (exact int32),
 * the sum over kb in fp32 with one fused multiply-add per block, then
 * + bias[n] in fp32 and, for y_dtype SAGE_DTYPE_BF16, rounded to bf16 (RNE).
 *   xq int8 [M, K], sx fp32 [ceil(M/128), K/128]  (sage_quantize_blocks_2d of X)
 *   wq int8 [N, K], sw fp32 [N/128, K/128]        (sage_quantize_blocks_2d of W)
 *   bias bf16 [N] or NULL; y [M, N] bf16 or fp32 (y_dtype).
 * M >= 1; N and K positive multiples of 128.  xq, wq, bias, y 16-byte
 * aligned; sx, sw 4-byte aligned.  status: device memory whose first uint32
 * is the status word (the workspace of the attention calls serves);
 * sage_status() on it reports a bounded wait that ran out.  Asynchronous on
 * `stream`.  Errors: SAGE_EINVAL (sizes, null or misaligned pointers, bad
 * y_dtype), SAGE_EUNSUPPORTED / SAGE_ELAUNCH (device), all before any launch.
 */
#define SAGE_LIN_BLK 128
#define SAGE_DTYPE_BF16 0
#define SAGE_DTYPE_F32 1
int sage_quantize_blocks_2d(const void* x, int R, int K, int8_t* codes, float* scales, void* stream);
int sage_linear_w8a8(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, const void* bias,
                     void* y, int y_dtype, int M, int N, int K, void* status, void* stream);

/*
 * W8A16 and bf16 linear layers (TMAP write-up, FFN section: to keep video
 * quality some layers go back from W8A8 to W8A16 -- the weights stay in
 * 8 bits, the activations and the arithmetic are 16-bit).
 *
 * sage_dequant_blocks_2d: out[r][k] = bf16_rne(fl(scales[r/128][k/128] *
 * codes[r][k])) for codes int8 [R, K] and scales fp32 [ceil(R/128), K/128]
 * as written by sage_quantize_blocks_2d; out device bf16 [R, K].  K a
 * positive multiple of 128, ceil(R/128) <= 65535.
 *
 * sage_linear_bf16: Y = X W^T + bias with x bf16 [M, K], w bf16 [N, K],
 * bias bf16 [N] or NULL, y [M, N] bf16 or fp32 (y_dtype); products and sums
 * in fp32 on the tensor cores (summation order unspecified), bias added in
 * fp32, bf16 output rounded to nearest even.  M >= 1, N a positive multiple
 * of 128, K a positive multiple of 64; x, w, bias, y 16-byte aligned.
 *
 * sage_linear_w8a16: the W8A16 layer, sage_dequant_blocks_2d of (wq, sw)
 * into `workspace` followed by sage_linear_bf16 against it.  K a positive
 * multiple of 128; workspace: device memory of at least
 * sage_linear_w8a16_workspace_bytes(N, K) bytes, 16-byte aligned.
 *
 * status as for sage_linear_w8a8.  Asynchronous on `stream`.  Errors:
 * SAGE_EINVAL (sizes, pointers, y_dtype), SAGE_EWORKSPACE (workspace too
 * small), SAGE_EUNSUPPORTED / SAGE_ELAUNCH (device).
 */
int sage_dequant_blocks_2d(const int8_t* codes, const float* scales, int R, int K, void* out, void* stream);
int sage_linear_bf16(const void* x, const void* w, const void* bias, void* y, int y_dtype, int M, int N, int K,
                     void* status, void* stream);
size_t sage_linear_w8a16_workspace_bytes(int N, int K);
int sage_linear_w8a16(const void* x, const int8_t* wq, const float* sw, const void* bias, void* y, int y_dtype,
                      int M, int N, int K, void* workspace, size_t workspace_bytes, void* status, void* stream);

/*
 * Sequence-parallel (DeepSpeed-Ulysses) attention (TMAP write-up, "Optimising
 * multi-GPU parallelism"): each of P ranks holds Nl = N / P tokens of every
 * head; an all-to-all gives each rank all N tokens of Hl = H / P heads,
 * attention runs on those, and a second all-to-all returns O to the token
 * slices.  The exchange buffers use the layout [P][B][Nl][Hl][d] (bf16):
 * chunk r holds the sending rank's tokens for heads r*Hl .. r*Hl + Hl - 1,
 * token-major, so that chunk p of the receive buffer holds tokens
 * p*Nl .. p*Nl + Nl - 1 of this rank's heads.
 *
 * sage_attn_fwd_seqpar: O = softmax(Q K^T / sqrt(d)) V over the B x Hl heads
 * and N = P * Nl tokens, as sage_attn_fwd, with q, k, v read from and o
 * written to that layout (device pointers; o is the send buffer of the return
 * exchange).  In the INT8/FP8 modes the quantization prepass reads the
 * chunks directly and the attention epilogue writes the chunks directly, so
 * no layout copy runs; in BF16 mode q, k, v are first gathered into the
 * workspace.  workspace: device, 256-byte aligned, at least
 * sage_seqpar_workspace_bytes(P, B, Nl, Hl, d, mode) bytes, status word first
 * (sage_status).  Results are bitwise those of sage_attn_fwd on the same
 * heads in the plain layout.  Errors as sage_attn_fwd (SAGE_EINVAL for
 * P < 1, Nl < 1 or P * Nl above 2^30).
 */
size_t sage_seqpar_workspace_bytes(int P, int B, int Nl, int Hl, int d, int mode);
int sage_attn_fwd_seqpar(const void* q, const void* k, const void* v, void* o, int P, int B, int Nl, int Hl, int d,
                         int mode, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Layout copies around the Ulysses all-to-all (rows of d bf16 values; Hl =
 * H / P, N = P * Nl):
 *   SAGE_ULYSSES_SEND     src [B, Nl, H, d]          -> dst [P][B][Nl][Hl][d]
 *   SAGE_ULYSSES_RECV_O   src [P][B][Nl][Hl][d]      -> dst [B, Nl, H, d]
 *   SAGE_ULYSSES_GATHER   src [P][B][Nl][Hl][d]      -> dst [B, Hl, N, d]
 *   SAGE_ULYSSES_SCATTER  src [B, Hl, N, d]          -> dst [P][B][Nl][Hl][d]
 * At P = 1 SEND and RECV_O are plain copies (the layouts coincide).  The [P]
 * side may be strided: chunk r starts at row base_rows + r * chunk_rows
 * (chunk_rows = 0 means dense, B*Hl*Nl; otherwise at least that), so that
 * several tensors can share one exchange buffer.  H % P == 0, d in {64, 128},
 * B, Nl, P >= 1; src and dst device, 16-byte aligned, disjoint.  Asynchronous
 * on `stream`.  Errors: SAGE_EINVAL (sizes, op, chunk_rows below the dense
 * chunk, pointers), SAGE_EUNSUPPORTED / SAGE_ELAUNCH (device).
 */
#define SAGE_ULYSSES_SEND 0
#define SAGE_ULYSSES_RECV_O 1
#define SAGE_ULYSSES_GATHER 2
#define SAGE_ULYSSES_SCATTER 3
int sage_ulysses_permute(const void* src, void* dst, int B, int Nl, int H, int d, int P, int op,
                         long long chunk_rows, long long base_rows, void* stream);

/*
 * Reads and clears the device status word at the start of `workspace`
 * (synchronises `stream`).  Returns SAGE_OK, SAGE_ETIMEOUT if a bounded
 * device-side wait ran out since the last call, or SAGE_ELAUNCH if the stream
 * reports a CUDA error.
 */
int sage_status(void* workspace, void* stream);

/* Human-readable text of a status code (static storage). */
const char* sage_strerror(int code);

/*
 * Returns SAGE_OK if the current device is an sm_100 part the kernels were
 * built for, SAGE_EUNSUPPORTED otherwise, SAGE_ELAUNCH if no device is usable.
 */
int sage_device_check(void);

/*
 * Debug build.  The same sources compiled with -DSAGE_DEBUG give
 * libsage_debug.so: every global access of the prepass, of the attention
 * kernels' scale loads and output stores, and of the Ulysses permutations
 * whose index is computed is checked against the extent of its buffer
 * first.  A failed check skips that access and records the site and the
 * index of the first failure; nothing traps.  The device entry points of the
 * quantization path, attention and the permutations then synchronise their
 * stream and return SAGE_EBOUNDS if a check failed (so a debug build cannot
 * be captured into a CUDA graph).  A release build has no checks.
 *
 * sage_debug_build: 1 in a debug build, 0 otherwise.
 * sage_debug_last_failure: the site (see csrc/internal.h, DebugSite) and the
 *   index of the first failed check of the last call that returned
 *   SAGE_EBOUNDS; SAGE_EUNSUPPORTED in a release build.
 * sage_dbg_bounds_selftest: runs a one-thread kernel whose single check
 *   fails on purpose (the index equals the extent; no memory is touched) and
 *   returns what a call with a failed check returns: SAGE_EBOUNDS in a debug
 *   build (site 99, index 1); SAGE_EUNSUPPORTED in a release build.
 */
int sage_debug_build(void);
int sage_debug_last_failure(int* site, long long* index);
int sage_dbg_bounds_selftest(void* stream);

/*
 * Diagnostic: copies int32 QK^T tiles computed by the same TMA + tcgen05
 * kind::i8 path the attention kernel uses.  q_i8, k_i8 as written by
 * sage_quantize_qk; tile_list: device int32 [n][4] of (b, h, qb, kb);
 * out: device int32 [n, 128, 128], out[t][i][j] = S[qb*128+i, kb*128+j].
 */
int sage_dbg_qk_tiles(const int8_t* q_i8, const int8_t* k_i8, int B, int H, int N, int d,
                      const int* tile_list, int n, int32_t* out, void* stream);

/*
 * Diagnostic: one 128-row P.V product through the same operand path as the
 * attention kernels: INT8_FP8 writes P from registers into the swizzled
 * shared-memory tile and issues the shared-memory kind::f8f6f4 MMA; BF16
 * writes P into tensor memory and issues the kind::f16 MMA with A there.
 * mode INT8_FP8: p (device, e4m3 [128,128]) times vt (device, e4m3 [d,128],
 *   key-contiguous) -> out fp32 [128,d] = sum_j p[i,j] * vt[c,j].
 * mode BF16: p (device, bf16 [128,128]) times vt (device, bf16 [128,d],
 *   channel-contiguous, i.e. V itself) -> out fp32 [128,d].
 */
int sage_dbg_pv_tile(const void* p, const void* vt, int d, int mode, float* out, void* stream);

/*
 * Diagnostic: one 128x128 BF16 QK^T tile through the BF16 attention path's
 * operand staging.  q, k: device bf16 [128,d]; out fp32 [128,128].
 */
int sage_dbg_qk_bf16_tile(const void* q, const void* k, int d, float* out, void* stream);

/*
 * Test hook of the bounded-wait machinery: runs the quantized attention
 * kernel on the given operands with a wait that no one satisfies and a wait
 * limit of `timeout_cycles` SM clocks, so that the kernel records
 * SAGE_ETIMEOUT in `status` and returns without hanging.  Same operands as
 * sage_attn_quantized.
 */
int sage_dbg_attn_forced_timeout(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                                 const float* k_scale, const uint8_t* v_f8t, const float* v_scale,
                                 void* o, int B, int H, int N, int d, void* status,
                                 long long timeout_cycles, void* stream);

/*
 * Test hook of the bounded-wait machinery of sage_linear_w8a8: the MMA
 * thread first waits on a barrier that no one completes, with a wait limit of
 * `timeout_cycles` SM clocks, so the kernel records SAGE_ETIMEOUT in `status`
 * and returns without hanging.  Same operands as sage_linear_w8a8.
 */
int sage_dbg_linear_forced_timeout(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                   const void* bias, void* y, int y_dtype, int M, int N, int K, void* status,
                                   long long timeout_cycles, void* stream);

/*
 * The same test hook for sage_linear_bf16: its MMA thread first waits on a
 * barrier no one completes, with a limit of `timeout_cycles` SM clocks, so
 * the kernel records SAGE_ETIMEOUT in `status` and returns without hanging.
 */
int sage_dbg_linear_bf16_forced_timeout(const void* x, const void* w, const void* bias, void* y, int y_dtype, int M,
                                        int N, int K, void* status, long long timeout_cycles, void* stream);

/*
 * Tensor-core throughput probe: one CTA per SM (grid = the device's SM
 * count) issues `iters` x 4 back-to-back tcgen05.mma of M=128, N = n (128 or
 * 256) and 32 bytes of K from shared-memory operands into tensor memory, and
 * writes each CTA's elapsed SM clocks to cycles (device int64 [grid]).
 * kind: SAGE_MMA_BF16 (K = 16 bf16), SAGE_MMA_E4M3 (K = 32), SAGE_MMA_I8
 * (K = 32).  MACs per SM per clock = iters * 4 * 128 * n * K / cycles.
 * status as for sage_attn_quantized.  Not part of the attention or linear
 * paths; it measures the rate they are bounded by, at any SM clock.
 */
#define SAGE_MMA_BF16 0
#define SAGE_MMA_E4M3 1
#define SAGE_MMA_I8 2
int sage_dbg_mma_peak(int kind, int n, int iters, long long* cycles, int grid, void* status, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_H */
