/*
 * moe_gemv.h -- C ABI of the B200 (sm_100a) weight-streaming hot path of
 * batch-1 mixture-of-experts decode.
 *
 * What the path computes (sources: the web pages on NVIDIA's "3 ways to boost
 * MoE inference on DGX Spark" write-up; the number formats come from the OCP
 * specifications named below):
 *
 *  - The routed-expert MoE layer.  Each token goes to k of E routed experts
 *    plus one shared expert that always runs (saipien.org essay, "Why one user
 *    waits on weights": 8 of 512 routed experts plus one shared expert).  Its
 *    weights are MXFP4 (same essay, "Why one user waits on weights": an FP4
 *    checkpoint; generativeaipub.com blog, "DGX Spark Can Hold the Whole
 *    Model": MXFP4 weights) and the expert layer is narrow, intermediate 768
 *    (saipien.org essay, "Kernels built for the shape you actually have").  The
 *    verify step scores 4 positions in one pass and wakes up to 32 routed
 *    experts (saipien.org essay, "Draft three tokens, verify four").
 *  - The online-FP8 LM head: the 157,184 x 2,560 BF16 vocabulary projection is
 *    quantised to FP8 once, when the layer is built, which halves the bytes
 *    each token reads (ncijnetwork.com summary, "What are the 3
 *    optimizations?", item 2; generativeaipub.com blog, "2. Compressing the
 *    Output Head").  Decode reads the whole head every token and keeps the
 *    top-k token ids (greedy decoding takes k = 1; the sampled workload on the
 *    same page uses top_k 29).
 *
 * Readings where the pages are silent:
 *  - routing: softmax over the E routed logits (plus an optional per-expert
 *    bias), top-k, renormalised over the selected k; ties go to the lower id;
 *  - each expert is a SwiGLU MLP: h = silu(gate x) * (up x), out = down h;
 *    the shared expert has weight 1;
 *  - FP8 head: per-row fp32 scale s = amax / 448, q = E4M3 RNE satfinite of
 *    w / s; logit = s * sum_j q_j x_j; activations stay bf16;
 *  - MXFP4 per OCP Microscaling Formats v1.0: E2M1 codes (bit 3 = sign),
 *    one E8M0 scale per 32 elements along K, scale exponent
 *    floor(log2(amax)) - 2 clamped to [-127, 127], elements rounded to
 *    nearest even and saturated at +-6, element 2j in the low nibble of byte j;
 *  - E4M3 per the OCP 8-bit Floating Point Specification (bias 7, max 448).
 *
 * Conventions for every call:
 *  - All tensors are row-major and contiguous in device memory that the caller
 *    owns (allocated with cudaMalloc or by torch).  The library never allocates
 *    or frees device memory.  Device pointers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Work is enqueued asynchronously; no call synchronises the host
 *    except moe_workspace_status().
 *  - Argument errors are returned before anything is enqueued.  Argument
 *    checks touch no CUDA API, so they also run on a machine without a GPU.
 *  - Quantised tensors carry a format tag that every call checks: passing a
 *    BF16-tagged head where the FP8 one is expected returns
 *    MOE_ERR_FORMAT_MISMATCH instead of silently reading FP8 bytes as BF16
 *    (the integration trap described in the ncijnetwork.com summary, "What
 *    are the 3 optimizations?", paragraph "The integration trap").
 *  - Calls are reentrant: all mutable state lives in the caller's workspace.
 *    Two calls that run at the same time on the GPU must use different
 *    workspaces.
 */
#ifndef MOE_GEMV_H
#define MOE_GEMV_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,       /* NULL pointer, non-positive size, bad M or top_k  */
    MOE_ERR_UNSUPPORTED_SHAPE = -2, /* a shape this build was not compiled for          */
    MOE_ERR_MISALIGNED = -3,        /* a device pointer not 16-byte aligned             */
    MOE_ERR_FORMAT_MISMATCH = -4,   /* wrong format tag on a quantised tensor           */
    MOE_ERR_WORKSPACE = -5,         /* workspace missing or smaller than required       */
    MOE_ERR_CUDA = -6,              /* a CUDA runtime call failed (launch, query)        */
    MOE_ERR_TIMEOUT = -7,           /* a bounded device-side wait ran out (see status)  */
    MOE_ERR_DEVICE_CHECK = -8       /* a device-side check failed (see status)          */
} moe_status;

typedef enum {
    MOE_FMT_NONE = 0,
    MOE_FMT_BF16 = 1,
    MOE_FMT_MXFP4_E2M1_E8M0_32 = 2,
    MOE_FMT_FP8_E4M3_ROWSCALE_F32 = 3,
    MOE_FMT_MXFP4_MOE_PACKED = 4,
    MOE_FMT_FP8_E4M3_TILED = 5
} moe_format;

/* A stack of `count` MXFP4 matrices, each [rows][K]:
 *   data   [count][rows][K/2] : E2M1 codes, element 2j in the low nibble of byte j
 *   scales [count][rows][K/32]: E8M0 block scales, 2^(code - 127)
 * K must be a multiple of 32.  fmt must be MOE_FMT_MXFP4_E2M1_E8M0_32.          */
typedef struct {
    int32_t fmt;
    int32_t count;
    int64_t rows;
    int64_t K;
    uint8_t* data;
    uint8_t* scales;
} moe_mxfp4_tensor;

/* The experts of one MoE layer, each a SwiGLU MLP:
 *   gate, up: count x [I][H];  down: count x [H][I].
 * The routed bank has count = E; the shared expert is a bank with count = 1.  */
typedef struct {
    moe_mxfp4_tensor gate;
    moe_mxfp4_tensor up;
    moe_mxfp4_tensor down;
} moe_expert_bank;

/* An expert bank re-laid out for moe_decode (moe_pack_experts): the same
 * MXFP4 bytes, grouped by the kernel's work items.  An item (e, j) is 16 rows
 * of expert e's intermediate dimension: gate and up rows 16j .. 16j+15 and
 * down columns 16j .. 16j+15.  The item's 32 gate/up rows (gate 16j ..
 * 16j+15, then up 16j .. 16j+15) enter the tensor core as a 128-row operand:
 * row 32s + R is row R over K segment s (elements s*Ks .. s*Ks + Ks - 1, with
 * Ks = 64 T and T = ceil(hidden / 256) K tiles per segment):
 *   units   [count][inter/16][unit]: item (e, j)'s bytes, one contiguous run
 *           of unit = 4096 T + 256 T + 8 * hidden bytes (25 * hidden when
 *           hidden is a multiple of 256):
 *     A (T tiles x 4096 B): gate/up data as the A operand of a
 *       block-scaled tensor-core MMA (canonical K-major layout, no swizzle):
 *       half c (2048 B) of tile t holds, at 16 r, the 16 bytes of operand
 *       row r = 32s + R: elements s*Ks + 64t + 32c .. +31 of row R, packed
 *       E2M1 with element 2i in the low nibble of byte i; zero past hidden;
 *     B (T x 256 B): byte 256t + 8R + 2s + c = the E8M0 scale of block
 *       2Ts + 2t + c of row R (0 past hidden);
 *     C (hidden/32 groups x 256 B): for 32-row group G and lane l = 4g + t,
 *       8 bytes = 2 bytes (columns 16j + 4t .. 16j + 4t + 3) of each of down
 *       rows 32G + g, 32G + 8 + g, 32G + 16 + g and 32G + 24 + g, with the bits
 *       of each byte's two E2M1 codes re-placed: element 2j's sign, e1, e0, m
 *       go to bits 7, 3, 2, 1 and element 2j+1's to bits 0, 6, 5, 4;
 *   dscales [count][inter/32][hidden]: the down scales of each 32-column
 *           pair p (shared by items 2p and 2p+1); byte 32G + 4g + r is the
 *           scale of down row 32G + 8r + g, block p.
 * fmt must be MOE_FMT_MXFP4_MOE_PACKED.  The pages have no counterpart for
 * this layout; it moves bytes and bits, never changes a value.              */
typedef struct {
    int32_t fmt;
    int32_t count;
    int32_t hidden;
    int32_t inter;
    uint8_t* units;
    uint8_t* dscales;
} moe_packed_bank;

/* The online-FP8 LM head: q E4M3 and row_scale [vocab] fp32.
 *   fmt MOE_FMT_FP8_E4M3_ROWSCALE_F32 (lmhead_quantize_fp8): q [vocab][hidden].
 *   fmt MOE_FMT_FP8_E4M3_TILED (lmhead_tile_fp8; what lmhead_decode reads):
 *     the same bytes in whole 16-row tiles (zero rows past vocab), tile T of
 *     16 * hidden bytes; for each 64-byte K slice s, 1,024 bytes ordered
 *     [half h][lane l][16 bytes] = row 16T + (l >> 2) + 8h, K bytes
 *     64s + 16(l & 3) .. +15.  One 512-byte run is then one warp's A
 *     fragments of an mma.sync m16n8k32 pair.  Values are unchanged.       */
typedef struct {
    int32_t fmt;
    int64_t vocab;
    int64_t hidden;
    uint8_t* q;
    float* row_scale;
} moe_fp8_head;

/* The unquantised BF16 LM head [vocab][hidden] (the comparator path).
 * fmt must be MOE_FMT_BF16.                                                    */
typedef struct {
    int32_t fmt;
    int64_t vocab;
    int64_t hidden;
    uint16_t* w;
} moe_bf16_head;

/* ---- load time ------------------------------------------------------------ */

/* Quantise `count` bf16 matrices w [count][rows][K] into `out`, whose count,
 * rows, K, data and scales the caller fills in (buffers of the sizes above).
 * On success sets out->fmt = MOE_FMT_MXFP4_E2M1_E8M0_32.  Blocks that hold an
 * Inf or NaN get scale code 0xFF (NaN) and element codes 0.  Bit-exact with
 * the OCP MX conversion rule stated at the top of this header.               */
MOE_API moe_status moe_quantize_mxfp4(const uint16_t* w_bf16, moe_mxfp4_tensor* out, void* stream);

/* Bytes of the two packed arrays of a bank with `count` experts (0 if the
 * sizes are unsupported: hidden and inter multiples of 32).                  */
MOE_API size_t moe_packed_units_bytes(int32_t count, int32_t hidden, int32_t inter);
MOE_API size_t moe_packed_dscales_bytes(int32_t count, int32_t hidden, int32_t inter);

/* Re-lay out a quantised bank (`src`: gate and up count x [I][H], down
 * count x [H][I], all tagged MXFP4) into `dst`, whose caller fills count,
 * hidden, inter and the two device arrays (units, dscales: sizes above,
 * 16-byte aligned).
 * Enqueued on `stream`; on success sets dst->fmt.  The source is not needed
 * by moe_decode afterwards.                                                  */
MOE_API moe_status moe_pack_experts(const moe_expert_bank* src, moe_packed_bank* dst, void* stream);

/* Quantise the bf16 head w [vocab][hidden] into `out` (caller fills vocab,
 * hidden, q, row_scale): s_v = fp32(amax_v / 448) (1 for an all-zero row),
 * q = E4M3 RNE satfinite of fp32(w / s_v).  On success sets out->fmt.
 * The ncijnetwork.com summary, "What are the 3 optimizations?", item 2:
 * quantising only this layer to FP8 at load time.                           */
MOE_API moe_status lmhead_quantize_fp8(const uint16_t* w_bf16, moe_fp8_head* out, void* stream);

/* Bytes of the tiled FP8 head for these sizes (0 if unsupported).            */
MOE_API size_t lmhead_tiled_bytes(int64_t vocab, int64_t hidden);

/* Re-lay a quantised head (fmt MOE_FMT_FP8_E4M3_ROWSCALE_F32) into the tiled
 * layout lmhead_decode streams.  The caller fills dst->vocab, hidden (equal
 * to src's), q (lmhead_tiled_bytes bytes, 16-byte aligned) and row_scale
 * (an array holding src's row scales -- src->row_scale itself serves; this
 * call does not touch it).  Enqueued on `stream`; on success sets dst->fmt. */
MOE_API moe_status lmhead_tile_fp8(const moe_fp8_head* src, moe_fp8_head* dst, void* stream);

/* ---- decode --------------------------------------------------------------- */

/* Bytes of workspace moe_decode needs for these sizes (0 if unsupported).    */
MOE_API size_t moe_workspace_bytes(int32_t M, int32_t top_k, int32_t num_experts,
                           int32_t hidden, int32_t inter);

/* One MoE layer for M tokens (1 <= M <= 4):
 *   hidden      [M][H] bf16
 *   router_w    [E][H] fp32;  router_bias [E] fp32 or NULL (added to the logits)
 *   experts     routed bank (count E), shared: bank with count 1; both packed
 *               by moe_pack_experts (host structs, device arrays)
 *   out         [M][H] fp32:  sum_i w_i expert_{id_i}(x) + shared(x)
 *   topk_ids    [M][top_k] int32 or NULL: selected experts, by descending logit
 *   topk_w      [M][top_k] fp32 or NULL:  renormalised softmax weights
 *   workspace   device buffer of at least moe_workspace_bytes(...) bytes,
 *               zeroed once (moe_workspace_reset) before its first use.
 * Supported: H and I multiples of 32, 32 <= H <= 3840, 32 <= I <= 65536,
 * E <= 1024, 1 <= top_k <= 8 and top_k <= E.  The call is one launch of
 * one CTA per SM, all resident (a kernel of another process that holds SMs
 * for over a second makes it return MOE_ERR_TIMEOUT).  Each distinct routed expert is
 * streamed once per call, however many of the M tokens chose it.  The
 * output is the same on every call with the same inputs (a fixed summation
 * order on a given GPU).
 * Arithmetic: gate/up on the tensor core (block-scaled FP4 MMA, fp32
 * accumulation): the E2M1 weights with their E8M0 scales times x written,
 * per token and 32-element block, as eight E2M1 base-4 digits with power-of-
 * two scales: exact for bf16 values within 2^-8 of the block's largest
 * magnitude, rounded to within 2^-16 of it below.  Where a block's weight
 * and activation scales together leave E8M0's range (activations below
 * about 2^-113 or above 2^127), powers of two move between them, and a
 * weight scale pushed out of range saturates.  h, per token and 16 values
 * scaled by a power of two, is split into two f16 parts (about 22
 * significant bits) for the down products.  Down E8M0 scales are decoded
 * by one multiply into the fp32 exponent: code 0 contributes 0 instead of
 * 2^-127 times its elements, and code 255 acts as +inf, so a non-finite
 * block as moe_quantize_mxfp4 writes it (scale 0xFF, zero elements) still
 * turns the rows that read it into NaN; a gate/up weight block with scale
 * 0xFF makes its row NaN.                                                   */
MOE_API moe_status moe_decode(const uint16_t* hidden_bf16, const float* router_w, const float* router_bias,
                      const moe_packed_bank* experts, const moe_packed_bank* shared,
                      int32_t M, int32_t top_k, float* out, int32_t* topk_ids, float* topk_w,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace lmhead_decode / lmhead_decode_bf16 need (0 if unsupported). */
MOE_API size_t lmhead_workspace_bytes(int32_t M, int32_t top_k, int64_t vocab, int64_t hidden);

/* FP8 LM head for M tokens (1 <= M <= 4), fused with top-k:
 *   hidden   [M][H] bf16;  head: the tiled head (fmt MOE_FMT_FP8_E4M3_TILED)
 *   topk_ids [M][top_k] int32, topk_vals [M][top_k] fp32: the top_k largest
 *            logits, descending, ties to the lower token id (top_k = 1 is the
 *            greedy argmax); 1 <= top_k <= 64
 *   logits   [M][vocab] fp32 or NULL: every logit, when the caller wants them
 *   workspace: at least lmhead_workspace_bytes(...), zeroed once before use.
 * Supported: hidden a multiple of 64 and at most 5120, vocab < 2^31, and a
 * vocabulary whose logits fit in shared memory across the GPU's SMs while the
 * head streams (each CTA keeps its rows' M logits and candidates: on a
 * 148-SM B200 with H = 2560, about 1.8 M rows at M = 1 and 430 K rows at
 * M = 4); larger returns MOE_ERR_UNSUPPORTED_SHAPE.                          */
MOE_API moe_status lmhead_decode(const uint16_t* hidden_bf16, const moe_fp8_head* head,
                         int32_t M, int32_t top_k, int32_t* topk_ids, float* topk_vals,
                         float* logits, void* workspace, size_t workspace_bytes, void* stream);

/* The same with the unquantised BF16 head (the comparator the FP8 head halves);
 * hidden a multiple of 32 and at most 2560.                                 */
MOE_API moe_status lmhead_decode_bf16(const uint16_t* hidden_bf16, const moe_bf16_head* head,
                              int32_t M, int32_t top_k, int32_t* topk_ids, float* topk_vals,
                              float* logits, void* workspace, size_t workspace_bytes, void* stream);

/* One draw per token from the head's top-k (ids and values as lmhead_decode
 * returns them: values sorted descending), with temperature and top-p -- the
 * sampled workload of the ncijnetwork.com summary ("What are the 3
 * optimizations?": temperature 0.6, top-p 0.95, top-k 29).  In fp64, in this
 * order, per token m with values v_0 >= v_1 >= ... and u = uniforms[m]:
 *   p_i = exp((v_i - v_0) / temperature), total = p_0 + ... + p_{k-1};
 *   n = the smallest prefix whose mass p_0 + ... + p_{n-1} reaches top_p * total;
 *   i = the first index < n with p_0 + ... + p_i > u * (p_0 + ... + p_{n-1});
 *   out_ids[m] = topk_ids[m][i].
 *   topk_ids [M][top_k] int32, topk_vals [M][top_k] fp32, uniforms [M] fp32 in
 *   [0, 1) (the caller's random numbers), out_ids [M] int32: device memory.
 * 1 <= top_k <= 64, temperature > 0, 0 < top_p <= 1.  Enqueued on `stream`;
 * argument errors are returned before anything is enqueued.                 */
MOE_API moe_status lmhead_sample(const int32_t* topk_ids, const float* topk_vals, int32_t M, int32_t top_k,
                                 float temperature, float top_p, const float* uniforms, int32_t* out_ids,
                                 void* stream);

/* Greedy acceptance of D draft tokens against the D + 1 argmaxes of the
 * verify step (the saipien.org essay, "Draft three tokens, verify four":
 * D = 3).  Draft i is accepted while it equals verify_ids[i] and every
 * earlier draft was accepted; emitted_ids = the accepted drafts followed by
 * verify_ids[accepted]; *n_emitted = accepted + 1 (1 .. D + 1).
 *   draft_ids [D], verify_ids [D + 1], emitted_ids [D + 1], n_emitted [1]:
 *   int32 device memory; 1 <= D <= 64.                                        */
MOE_API moe_status moe_mtp_accept(const int32_t* draft_ids, const int32_t* verify_ids, int32_t D,
                                  int32_t* emitted_ids, int32_t* n_emitted, void* stream);

/* lmhead_decode for callers that cannot provide a workspace: hosts that own
 * every device allocation and give a plugin only its inputs and outputs, or
 * loops that must not call cudaMalloc (it can synchronise the device).  No
 * counterpart on the pages: this is an interface convenience.  The scratch is
 * one fixed device array of MOE_LMHEAD_NOALLOC_SCRATCH_BYTES, held by every
 * GPU that loads the library until the process exits.  It must fit a 64-byte
 * header plus M candidate lists of (SM count) x top_k entries of 8 bytes,
 * each list rounded up to an even entry count: M x top_k <= 220 on a 148-SM
 * B200 (e.g. M = 4, top_k <= 55); larger requests return MOE_ERR_WORKSPACE.
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and should come before any stream capture.  Each
 * call resets the header's counters on `stream` before its kernel but keeps
 * its status word: a device error (a wait that ran out) stays there until
 * lmhead_noalloc_status reads and clears it.  All calls share the array, so
 * calls that overlap on the GPU (different streams, or different threads)
 * race: serialise them.  Allocates nothing.  The head is the tiled one, as
 * for lmhead_decode.                                                         */
#define MOE_LMHEAD_NOALLOC_SCRATCH_BYTES (256u * 1024u)
MOE_API moe_status lmhead_decode_noalloc(const uint16_t* hidden_bf16, const moe_fp8_head* head,
                                         int32_t M, int32_t top_k, int32_t* topk_ids, float* topk_vals,
                                         float* logits, void* stream);

/* The device status of lmhead_decode_noalloc on the current device: waits
 * for `stream` (cudaStreamSynchronize), writes to *status_out the first
 * moe_status a no-alloc launch reported since the last read (MOE_OK if none)
 * and clears it.  Returns MOE_OK, MOE_ERR_INVALID_ARG (status_out NULL) or
 * MOE_ERR_CUDA.  Allocates nothing; do not call it during stream capture.   */
MOE_API moe_status lmhead_noalloc_status(int32_t* status_out, void* stream);

/* ---- between the layers of a decode step ---------------------------------- */

/* The next layer's input from a layer's output, for a stack of MoE layers
 * each re-routed from the previous layer's RMS-normalised output (the decode
 * stream of the workload): out[m][j] = bf16_RNE(y[m][j] / sqrt(mean_j y[m][j]^2
 * + eps)), gain 1.  y [M][H] fp32, out [M][H] bf16; H a multiple of 8.       */
MOE_API moe_status moe_rmsnorm_bf16(const float* y, int32_t M, int32_t H, float eps, uint16_t* out,
                                    void* stream);

/* Greedy feedback: out[m] = table[ids[m * ids_stride]] for the next step
 * (table [V][H] bf16; ids device int32, e.g. the column 0 of lmhead_decode's
 * topk_ids with ids_stride = top_k).  An id outside [0, V) gives a zero row.
 * H a multiple of 8.                                                         */
MOE_API moe_status moe_embed_gather(const uint16_t* table, int64_t V, int64_t H, const int32_t* ids,
                                    int32_t ids_stride, int32_t M, uint16_t* out, void* stream);

/* Measurement aid, not a step of the path: read `bytes` (a multiple of 16)
 * from device memory `src` (16-byte aligned) with 128-bit non-allocating loads
 * from every SM, folding the words into the device word *sink by XOR, so that
 * a caller timing it sees this GPU's practical HBM read ceiling -- the
 * yardstick for the weight streams above.  Enqueued on `stream`.            */
MOE_API moe_status moe_stream_read(const void* src, size_t bytes, uint32_t* sink, void* stream);

/* ---- housekeeping --------------------------------------------------------- */

/* Zero a workspace (async memset on `stream`).  Needed once before first use,
 * and after a call reported MOE_ERR_TIMEOUT.                                 */
MOE_API moe_status moe_workspace_reset(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, read the device status word that kernels set in this
 * workspace (MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE_CHECK), clear it, and
 * return it.  Device-side waits in these kernels are bounded: a wait that
 * runs out sets the status word and the kernel returns instead of hanging.   */
MOE_API moe_status moe_workspace_status(void* workspace, void* stream);

/* Write a NUL-terminated description of the compiled kernels and formats
 * ("sm_100a ...") into buf of n bytes.  The pages advise confirming at startup
 * that each optimisation is live (ncijnetwork.com summary, "The integration
 * trap"); this is the string to log.  A buffer too small for the whole text
 * (1 KB always suffices) gets its first n - 1 characters, NUL-terminated, and
 * the call returns MOE_ERR_INVALID_ARG.                                      */
MOE_API moe_status moe_query_path(char* buf, size_t n);

/* Self-test of the bounded device waits; the pages have no counterpart.
 * Enqueues one small kernel that waits on a word of the workspace header that
 * no kernel ever writes, using the same bounded wait as the decode kernels but
 * with a limit of `limit_us` microseconds (1 .. 1,000,000).  When the limit
 * runs out the kernel records MOE_ERR_TIMEOUT in the workspace's status word
 * and returns; read it with moe_workspace_status.  The decode kernels' own
 * limit is 1 s.  Any workspace of at least 64 bytes serves; calls that
 * overlap on the GPU must not share one.  Returns MOE_ERR_WORKSPACE,
 * MOE_ERR_MISALIGNED or MOE_ERR_INVALID_ARG for bad arguments.             */
MOE_API moe_status moe_selftest_wait_timeout(void* workspace, size_t workspace_bytes, uint32_t limit_us,
                                             void* stream);

/* Text for a status code ("MOE_ERR_FORMAT_MISMATCH", ...); never NULL.       */
MOE_API const char* moe_status_string(moe_status s);

#ifdef __cplusplus
}
#endif
#endif
