/*
 * ivit.h -- C ABI of the integer-only ViT encoder block on B200 (sm_100a).
 *
 * The method is I-ViT's integer-only block: INT8 linear layers whose INT32
 * accumulators are requantised with dyadic numbers, Shiftmax attention,
 * ShiftGELU and I-LayerNorm.  Sources, cited per entry point below:
 *   [IVIT] "I-ViT: Integer-only Quantization for Efficient Vision Transformer
 *          Inference" (mer.run notes), sections 3.1-3.5.
 *   [TRIO] "Trio-ViT" article (cloud.tencent.com), eqs. (1)-(3) and (12);
 *          section IV-D (log2 quantisation).
 *   [FQ]   "FQ-ViT: Post-Training Quantization for Fully Quantized Vision
 *          Transformer" (ijcai.org record), abstract: Power-of-Two Factor
 *          (PTF) for LayerNorm inputs, Log-Int-Softmax (LIS) with 4-bit
 *          attention maps and the BitShift operator.
 *
 * Conventions for every entry point:
 *   - Tensors are device pointers, row-major and contiguous, each 16-byte
 *     aligned.  The caller owns all memory (inputs, outputs, workspace); the
 *     library allocates nothing on these paths.
 *   - ">> c" is an arithmetic (floor) shift; sat_k clamps to the signed k-bit
 *     range.  A dyadic number {b, c} stands for b / 2^c with 0 <= b < 2^31 and
 *     0 <= c <= 31.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Arguments are validated on the host first; a bad
 *     argument returns IVIT_ERR_INVALID_ARG (or IVIT_ERR_UNSUPPORTED for a
 *     shape outside the supported envelope) with nothing enqueued.  A failed
 *     launch returns IVIT_ERR_CUDA.
 *   - Kernels never wait without bound: a wait that exceeds its budget (one
 *     second) records IVIT_ERR_TIMEOUT in a per-device status word, which
 *     ivit_stream_status() reads.
 *   - There is no CPU fallback: without a usable sm_100 device every compute
 *     entry point returns IVIT_ERR_CUDA or IVIT_ERR_UNSUPPORTED.
 */
#ifndef IVIT_H_
#define IVIT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *ivit_stream_t;

typedef enum {
  IVIT_OK = 0,
  IVIT_ERR_INVALID_ARG = 1,
  IVIT_ERR_UNSUPPORTED = 2,
  IVIT_ERR_CUDA = 3,
  IVIT_ERR_TIMEOUT = 4,
  IVIT_ERR_INTERNAL = 5
} ivit_status;

/* b / 2^c: the dyadic number DN(S) of [IVIT] 3.2 / [TRIO] eq. (12). */
typedef struct {
  int32_t b;
  int32_t c;
} ivit_dyadic;

/* Residual addition of two int8 tensors with different scales ([IVIT] 3.1,
 * X^ = MSA(LN(X)) + X and Y = MLP(LN(X^)) + X^): both terms are rescaled to
 * the output scale over one common shift,
 *   y = sat_8((b_skip * skip + b_branch * branch) >> c).              */
typedef struct {
  int32_t b_skip;
  int32_t b_branch;
  int32_t c;
} ivit_residual;

/* Human-readable name of a status code (static string, never NULL). */
const char *ivit_status_string(ivit_status s);

/* ---------------------------------------------------------------------------
 * Host-side parameter helpers (no device work; usable without a GPU)
 * ------------------------------------------------------------------------- */

/* DN(s) of [IVIT] 3.2: c is the largest shift in [0, 31] for which
 * b = round(s * 2^c) (half away from zero) stays below 2^31, so that
 * |b / 2^c - s| <= 2^-(c+1).  s must be finite, >= 0 and < 2^31 - 0.5;
 * otherwise IVIT_ERR_INVALID_ARG.  `out` must not be NULL.                */
ivit_status ivit_dyadic_from_double(double s, ivit_dyadic *out);

/* Two dyadic numbers over a common shift (for ivit_residual): c is the
 * smaller of the two individual DN shifts, b_i = round(s_i * 2^c).        */
ivit_status ivit_residual_from_double(double s_skip, double s_branch, ivit_residual *out);

/* I_0 of the shift-exponential ([IVIT] 3.3): round(1 / S) half away from
 * zero, at least 1.  S must be finite and > 0.                              */
ivit_status ivit_i0_from_scale(double S, int32_t *out);

/* ---------------------------------------------------------------------------
 * Hot-path operators
 * ------------------------------------------------------------------------- */

/* INT8 linear layer with dyadic epilogue ([IVIT] 3.1-3.2; [TRIO] eqs. (1),
 * (12)), optionally followed by a residual addition:
 *   acc_ij = sum_k X[i,k] * W[j,k] + bias[j]                   (int32)
 *   o_ij   = sat_{out_bits}((b[j] * acc_ij) >> c[j])           rounding = 0
 *   o_ij   = sat_{out_bits}((b[j] * acc_ij + 2^(c[j]-1)) >> c[j])   rounding = 1
 *   Y_ij   = skip ? sat_8((res.b_skip * skip[i,j] + res.b_branch * o_ij) >> res.c)
 *                 : o_ij
 * X [M x K] int8; W [N x K] int8 (one output channel per row, i.e. K-major);
 * bias [N] int32 or NULL, |bias| <= 2^30 (the int32 accumulator cannot
 * overflow); b [N] int32 in [0, 2^31); c [N] int8 in [0, 31];
 * skip [M x N] int8 or NULL; Y [M x N] int8.
 * Constraints: M >= 1; 16 <= K <= 16384 and N >= 16, both multiples of 16;
 * 2 <= out_bits <= 8; rounding 0 (the floor shift the page's integer
 * formula writes, the default reading) or 1 (round half up, the variant its
 * ideal form suggests; nothing is added when c[j] = 0).  Runs on the tensor
 * cores (tcgen05 kind::i8).                                                 */
ivit_status ivit_linear_requant(const int8_t *X, int64_t M, int32_t K, const int8_t *W, int32_t N,
                                const int32_t *bias, const int32_t *b, const int8_t *c, int32_t out_bits,
                                int32_t rounding, const int8_t *skip, ivit_residual res, int8_t *Y,
                                ivit_stream_t stream);

/* fc1 of the MLP with ShiftGELU fused into the epilogue ([IVIT] 3.1, 3.2,
 * 3.4): Y = ShiftGELU(sat_8((b[j] * (X W^T + bias)_ij) >> c[j])), with the
 * ShiftGELU of ivit_shiftgelu (I0 = round(1 / S_h) of the requantised fc1
 * output, gelu_out ~ S_h 2^-(k_out-1) / S_g).  Bit-identical to
 * ivit_linear_requant followed by ivit_shiftgelu, without the intermediate
 * tensor in memory.  Same constraints as both; rounding applies to the fc1
 * requant as in ivit_linear_requant.                                        */
ivit_status ivit_linear_shiftgelu(const int8_t *X, int64_t M, int32_t K, const int8_t *W, int32_t N,
                                  const int32_t *bias, const int32_t *b, const int8_t *c, int32_t rounding,
                                  int32_t gelu_I0, int32_t gelu_M, int32_t gelu_k_out, ivit_dyadic gelu_out,
                                  int8_t *Y, ivit_stream_t stream);

/* Multi-head attention core with Shiftmax ([IVIT] 3.1-3.3; [TRIO] eqs.
 * (1)-(3)), fused on chip (the score matrix never reaches memory):
 *   S_ij   = sum_{d<64} Q_id K_jd                                  (int32)
 *   L_ij   = sat_{k_s}((logit.b * S_ij) >> logit.c)   logit ~ S_q S_k / (8 S_L)
 *   P_i.   = Shiftmax(L_i., I0, M, k_out) over the N keys of the image:
 *            I_delta = L - max; e = ShiftExp(I_delta); Dv = floor(2^M / sum e);
 *            P = (Dv * e) >> (M - (k_out - 1))           (u8, <= 2^(k_out-1))
 *   ctx_id = sat_8((out.b * sum_j P_ij V_jd) >> out.c) out ~ S_v 2^-(k_out-1) / S_ctx
 * qkv [B*N x 3*H*64] int8: columns [0, D) are Q (head h at h*64), [D, 2D) K,
 * [2D, 3D) V, D = H*64.  ctx [B*N x D] int8, heads concatenated.
 * Constraints: B, H >= 1; 1 <= N <= 640; 2 <= k_s <= 16; I0 >= 1;
 * k_out - 1 <= M <= 30; 1 <= k_out <= 8.  Logits of up to 8 bits take
 * ShiftExp from a table; wider ones (k_s > 8) compute it per score and need
 * N <= 256 and n_max * I0 < 2^32, where n_max = m + ceil(m/2) - ceil(m/16)
 * with m = 2^k_s - 1 is the largest -I_p (the floor division by I0 is then
 * one exact mul.hi); otherwise IVIT_ERR_UNSUPPORTED, nothing enqueued.     */
ivit_status ivit_attention(const int8_t *qkv, int32_t B, int32_t N, int32_t H, ivit_dyadic logit, int32_t k_s,
                           int32_t I0, int32_t M, int32_t k_out, ivit_dyadic out, int8_t *ctx,
                           ivit_stream_t stream);

/* ShiftGELU, elementwise ([IVIT] 3.4): GELU(x) ~ x * sigmoid(1.702 x) with
 *   I_p = x + (x >> 1) + (x >> 3) + (x >> 4)                   (1.1011b)
 *   sigma = IntDiv(ShiftExp(I_p - m), ShiftExp(I_p - m) + ShiftExp(-m)),
 *           m = max(I_p, 0)                 (scale 2^-(k_out-1))
 *   y = sat_8((out.b * x * sigma) >> out.c)   out ~ S_x 2^-(k_out-1) / S_y
 * x, y: n int8 values (any n >= 0).  I0 = round(1 / S_x) >= 1;
 * k_out - 1 <= M <= 30; 1 <= k_out <= 8.                                   */
ivit_status ivit_shiftgelu(const int8_t *x, int64_t n, int32_t I0, int32_t M, int32_t k_out, ivit_dyadic out,
                           int8_t *y, ivit_stream_t stream);

/* I-LayerNorm, per row of `cols` int8 values ([IVIT] 3.5):
 *   mu = floor(sum x / cols);  V = floor(sum (x - mu)^2 / cols)
 *   sigma = max(isqrt(V), 1), isqrt by exactly 10 Newton steps
 *           I <- (I + floor(V / I)) >> 1 from I = 2^floor(bit(V) / 2)
 *   n_i = ((x_i - mu) * floor(2^M_ln / sigma)) >> (M_ln - F)   (scale 2^-F)
 *   y_i = sat_8((out.b * (n_i * gamma_i + beta_i)) >> out.c)
 * x, y [rows x cols] int8; gamma [cols] int8 (scale S_gamma); beta [cols]
 * int32 (scale S_gamma 2^-F), |beta| <= 2^30.  Constraints: rows >= 0;
 * 16 <= cols <= 2048, multiple of 16; 0 <= F <= 14; F <= M_ln <= 23.        */
ivit_status ivit_layernorm(const int8_t *x, int64_t rows, int32_t cols, const int8_t *gamma,
                           const int32_t *beta, int32_t F, int32_t M_ln, ivit_dyadic out, int8_t *y,
                           ivit_stream_t stream);

/* ---------------------------------------------------------------------------
 * Variants where the pages leave a step open or name an alternative
 * ------------------------------------------------------------------------- */

/* ShiftGELU with a row maximum ([IVIT] 3.4, which multiplies the sigmoid's
 * numerator and denominator by e^(-S I_max) and stops before defining I_max).
 * READING: I_max is the largest exponent of the row, max(0, max_i I_p,i), as
 * Shiftmax subtracts its row maximum (ivit_shiftgelu takes max(I_p, 0) per
 * element instead):
 *   e1 = ShiftExp(I_p - I_max); e2 = ShiftExp(-I_max)
 *   sigma = IntDiv(e1, e1 + e2), and sigma = 0 when e1 + e2 = 0 (both
 *           exponentials underflow: the divisor is taken as 1)
 *   y = sat_8((out.b * x * sigma) >> out.c)
 * x, y [rows x cols] int8, one row per token (e.g. cols = Dm channels of fc1's
 * output).  Constraints: rows >= 0; 16 <= cols <= 16384, multiple of 16;
 * I0 >= 1; k_out - 1 <= M <= 30; 1 <= k_out <= 8.                          */
ivit_status ivit_shiftgelu_rowmax(const int8_t *x, int64_t rows, int32_t cols, int32_t I0, int32_t M,
                                  int32_t k_out, ivit_dyadic out, int8_t *y, ivit_stream_t stream);

/* Attention with Log-Int-Softmax ([FQ] abstract: the attention map quantised
 * to 4 bits on a log2 grid and multiplied with V by BitShift; the log2
 * quantiser clip(round(log2(.)), -a, b) of [TRIO] IV-D).  S and the logits
 * as in ivit_attention; then, READING, per query row:
 *   e = ShiftExp(L - max L), Dv = floor(2^M / sum e)          ([IVIT] 3.3)
 *   P16 = (Dv * e) >> (M - 15)             (16-bit probability, scale 2^-15)
 *   k = clip(15 - round(log2 P16), 0, 15), k = 15 when P16 = 0 (4-bit code;
 *       round(log2 P) rounds up exactly when P^2 >= 2^(2 floor(log2 P) + 1))
 *   ctx_id = sat_8((out.b * sum_j (V_jd << (15 - k_j))) >> out.c)
 *            out ~ S_v 2^-15 / S_ctx
 * (the bit shift at scale 2^-15 is exact; it runs on the tensor cores as two
 * u8 x s8 products over the power-of-two planes 2^(7-k), k <= 7, and
 * 2^(15-k), k >= 8).  Layouts as ivit_attention.  Constraints: B, H >= 1;
 * 1 <= N <= 640; 2 <= k_s <= 8; I0 >= 1; 15 <= M <= 30.                    */
ivit_status ivit_attention_lis(const int8_t *qkv, int32_t B, int32_t N, int32_t H, ivit_dyadic logit,
                               int32_t k_s, int32_t I0, int32_t M, ivit_dyadic out, int8_t *ctx,
                               ivit_stream_t stream);

/* I-LayerNorm of an input quantised with power-of-two factors ([FQ] abstract:
 * PTF against the inter-channel variation of LayerNorm inputs).  READING:
 * channel i of x carries the scale S 2^alpha_i (one layer-wise S, alpha_i in
 * {0, 1, 2, 3}, chosen off-line per channel); the LayerNorm input at the
 * common scale S is x_i << alpha_i, and ivit_layernorm's steps ([IVIT] 3.5)
 * run on it unchanged.  alpha [cols] uint8 (device; only its two low bits are
 * read).  Constraints as ivit_layernorm, with M_ln <= 20 (|x << alpha - mu|
 * < 2^11 keeps (x - mu) * floor(2^M_ln / sigma) below 2^31).               */
ivit_status ivit_layernorm_ptf(const int8_t *x, int64_t rows, int32_t cols, const uint8_t *alpha,
                               const int8_t *gamma, const int32_t *beta, int32_t F, int32_t M_ln,
                               ivit_dyadic out, int8_t *y, ivit_stream_t stream);

/* ---------------------------------------------------------------------------
 * The encoder block ([IVIT] 3.1): X^ = MSA(LN1(X)) + X; Y = MLP(LN2(X^)) + X^
 * ------------------------------------------------------------------------- */

/* Integer parameters of one block.  Pointers are device memory owned by the
 * caller; per-output-channel multiplier tables follow ivit_linear_requant. */
typedef struct {
  int32_t D;  /* model width, = 64 * H */
  int32_t H;  /* heads (head width 64) */
  int32_t Dm; /* MLP width */
  /* I-LayerNorm 1 */
  const int8_t *ln1_gamma;
  const int32_t *ln1_beta;
  ivit_dyadic ln1_out;
  /* QKV projection: W [3D x D], bias / b / c [3D] */
  const int8_t *w_qkv;
  const int32_t *bias_qkv;
  const int32_t *b_qkv;
  const int8_t *c_qkv;
  /* attention */
  ivit_dyadic logit;
  int32_t k_s, attn_I0, attn_M, attn_k_out;
  ivit_dyadic attn_out;
  /* output projection W^O [D x D] + residual 1 */
  const int8_t *w_o;
  const int32_t *bias_o;
  const int32_t *b_o;
  const int8_t *c_o;
  ivit_residual res1;
  /* I-LayerNorm 2 */
  const int8_t *ln2_gamma;
  const int32_t *ln2_beta;
  ivit_dyadic ln2_out;
  /* fc1: W1 [Dm x D] */
  const int8_t *w1;
  const int32_t *bias1;
  const int32_t *b1;
  const int8_t *c1;
  /* ShiftGELU */
  int32_t gelu_I0, gelu_M, gelu_k_out;
  ivit_dyadic gelu_out;
  /* fc2: W2 [D x Dm] + residual 2 */
  const int8_t *w2;
  const int32_t *bias2;
  const int32_t *b2;
  const int8_t *c2;
  ivit_residual res2;
  /* I-LayerNorm constants shared by both norms */
  int32_t ln_F, ln_M;
  /* requant rounding of the four linear layers, as ivit_linear_requant's
   * `rounding` (0 floor, 1 round half up) */
  int32_t linear_round;
} ivit_block_params;

/* Bytes of device workspace ivit_block_forward needs for B images of N
 * tokens (intermediate activations; 256-byte aligned sub-buffers).         */
size_t ivit_block_workspace_bytes(int32_t B, int32_t N, int32_t D, int32_t Dm);

/* One encoder block over B images of N tokens.  x, y [B*N x D] int8 (may not
 * alias); workspace: at least ivit_block_workspace_bytes(B, N, D, Dm) bytes,
 * 256-byte aligned, owned by the caller and not used concurrently by another
 * call.  Enqueues LN1, QKV, attention, W^O (+residual), LN2, fc1 with the
 * ShiftGELU fused into its epilogue, and fc2 (+residual) on `stream`.  The
 * same constraints as the individual operators apply (N <= 640, D = 64 H,
 * D and Dm multiples of 16).                                                */
ivit_status ivit_block_forward(const ivit_block_params *p, const int8_t *x, int8_t *y, void *workspace,
                               size_t workspace_bytes, int32_t B, int32_t N, ivit_stream_t stream);

/* Size of the device array that ivit_block_forward_static keeps its
 * intermediates in: 32 MiB on every GPU that loads the library.            */
#define IVIT_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/* The encoder block without a workspace argument and without allocating.
 * The pages have no counterpart: this is a deployment convenience.
 *
 * For callers that cannot allocate device memory at all: an inference-server
 * plugin whose host gives it no allocator, code inside a framework whose
 * caching allocator already holds the whole device, or a latency-critical
 * loop that cannot pay for cudaMalloc/cudaFree (which may synchronise the
 * device).  The intermediates that ivit_block_forward keeps in the caller's
 * workspace live instead in one fixed array of IVIT_STATIC_SCRATCH_BYTES in
 * device memory, defined by the library; every GPU that loads the library
 * holds it until the process exits.  The caller still passes the inputs x,
 * the outputs y and the parameters, exactly as for ivit_block_forward.
 *
 * - Returns IVIT_ERR_UNSUPPORTED, with nothing enqueued, when
 *   ivit_block_workspace_bytes(B, N, p->D, p->Dm) exceeds
 *   IVIT_STATIC_SCRATCH_BYTES (e.g. more than 22 images of 197 tokens at
 *   ViT-B width); all other checks and errors are those of
 *   ivit_block_forward.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  No call allocates or frees memory.
 * - Every call on a device shares the one array, and it keeps whatever the
 *   last call left in it (no intermediate needs to start at zero).  Calls
 *   whose work overlaps on the GPU -- on different streams, or from different
 *   threads without ordering -- race on the array and corrupt each other's
 *   results; order them on one stream.                                       */
ivit_status ivit_block_forward_static(const ivit_block_params *p, const int8_t *x, int8_t *y, int32_t B,
                                      int32_t N, ivit_stream_t stream);

/* ---------------------------------------------------------------------------
 * Steps either side of the blocks.  [IVIT] 3.1 quantises every linear layer
 * of the ViT with the same int8 x int8 -> int32 -> dyadic scheme; READING:
 * the patch projection (a P x P convolution with stride P, i.e. a linear
 * layer over flattened patches) and the classifier are two more such layers,
 * and the position embedding joins the tokens through the same two-scale
 * dyadic addition as the residual connections.
 * ------------------------------------------------------------------------- */

/* Bytes of device workspace ivit_patch_embed needs (flattened patches and
 * their embeddings; 256-byte aligned sub-buffers).                         */
size_t ivit_patch_embed_workspace_bytes(int32_t B, int32_t C, int32_t Hi, int32_t Wi, int32_t P, int32_t D);

/* Patch embedding.  img [B x C x Hi x Wi] int8 (NCHW), Np = (Hi/P)(Wi/P)
 * patches in row-major patch order.  The patch at (py, px) flattens to
 * z[(ch P + ky) P + kx] = img[b, ch, py P + ky, px P + kx] (the [D x C x P x P]
 * layout of a convolution weight) and
 *   e[b, p] = sat_8((b_j * (sum_k z_k W_jk + bias_j)) >> c_j)   W [D x C P P]
 * x [B*(Np+1) x D] int8 gets, per image, the class token then the patches:
 *   x[b, 0]     = sat_8((pos_add.b_skip * cls_j    + pos_add.b_branch * pos[0, j])     >> pos_add.c)
 *   x[b, 1 + p] = sat_8((pos_add.b_skip * e[b,p]_j + pos_add.b_branch * pos[1 + p, j]) >> pos_add.c)
 * cls [D] int8 is held at the embedding scale; pos [(Np+1) x D] int8.
 * workspace: ivit_patch_embed_workspace_bytes(...) bytes, 256-byte aligned,
 * caller-owned.  Constraints: Hi, Wi multiples of P; C P P and D multiples
 * of 16, each <= 16384; pointers 16-byte aligned.  Errors as for
 * ivit_linear_requant, nothing enqueued on a failed check.                 */
ivit_status ivit_patch_embed(const int8_t *img, int32_t B, int32_t C, int32_t Hi, int32_t Wi, int32_t P,
                             const int8_t *W, int32_t D, const int32_t *bias, const int32_t *b, const int8_t *c,
                             int32_t rounding, const int8_t *cls, const int8_t *pos, ivit_residual pos_add,
                             void *workspace, size_t workspace_bytes, int8_t *x, ivit_stream_t stream);

/* Bytes of device workspace ivit_head needs (the class tokens, normalised). */
size_t ivit_head_workspace_bytes(int32_t B, int32_t D);

/* Classifier head: the class token of every image (row 0 of its Ntok rows
 * in x [B*Ntok x D]), I-LayerNorm (as ivit_layernorm), then an int8 linear
 * layer W [Ncls x D] to int8 logits [B x Ncls] (as ivit_linear_requant).
 * Ncls a multiple of 16 (pad a class count with zero rows of W).  rounding
 * as in ivit_linear_requant (for the classifier; the patch embedding's
 * `rounding` likewise applies to its projection).                          */
ivit_status ivit_head(const int8_t *x, int32_t B, int32_t Ntok, int32_t D, const int8_t *gamma,
                      const int32_t *beta, int32_t F, int32_t M_ln, ivit_dyadic ln_out, const int8_t *W,
                      int32_t Ncls, const int32_t *bias, const int32_t *b, const int8_t *c, int32_t rounding,
                      void *workspace, size_t workspace_bytes, int8_t *logits, ivit_stream_t stream);

/* A whole ViT: patch embedding, n_blocks encoder blocks, classifier head.
 * Device pointers as above; `blocks` is a host array of n_blocks entries
 * (each with the model width D).                                           */
typedef struct {
  int32_t C, P, D, n_blocks, Ncls;
  /* patch embedding: W [D x C P P], bias / b / c [D], class token, position embedding */
  const int8_t *w_pe;
  const int32_t *bias_pe;
  const int32_t *b_pe;
  const int8_t *c_pe;
  const int8_t *cls;
  const int8_t *pos;
  ivit_residual pos_add;
  const ivit_block_params *blocks;
  /* head: I-LayerNorm then W [Ncls x D] */
  const int8_t *head_gamma;
  const int32_t *head_beta;
  int32_t head_ln_F, head_ln_M;
  ivit_dyadic head_ln_out;
  const int8_t *w_head;
  const int32_t *bias_head;
  const int32_t *b_head;
  const int8_t *c_head;
  /* requant rounding of the patch projection and the classifier (the blocks
   * carry their own) */
  int32_t linear_round;
} ivit_model_params;

/* Bytes of device workspace ivit_model_forward needs for B images of
 * Hi x Wi pixels (two token buffers and the largest step's workspace).     */
size_t ivit_model_workspace_bytes(const ivit_model_params *m, int32_t B, int32_t Hi, int32_t Wi);

/* img [B x C x Hi x Wi] int8 -> logits [B x Ncls] int8.  Every check of
 * every step runs before anything is enqueued.                             */
ivit_status ivit_model_forward(const ivit_model_params *m, const int8_t *img, int32_t B, int32_t Hi, int32_t Wi,
                               void *workspace, size_t workspace_bytes, int8_t *logits, ivit_stream_t stream);

/* ---------------------------------------------------------------------------
 * Status
 * ------------------------------------------------------------------------- */

/* Synchronises `stream`, then reads and clears the current device's status
 * word: IVIT_ERR_TIMEOUT if a kernel gave up a bounded wait since the last
 * call, IVIT_ERR_CUDA on a CUDA error, else IVIT_OK.                        */
ivit_status ivit_stream_status(ivit_stream_t stream);

/* Number of kernel launches this library has enqueued in this process (for
 * launch accounting by benchmarks).                                          */
uint64_t ivit_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* IVIT_H_ */
