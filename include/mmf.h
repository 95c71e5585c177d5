/*
 * mmf.h - C ABI of the MatMul-free block forward on NVIDIA B200 (sm_100a).
 *
 * The operations follow the web pages on "Scalable MatMul-free Language
 * Modeling" (arXiv 2406.02528):
 *   [DC] "MatMul-free language models", DataCamp blog:
 *        "Replacing MatMul with ternary operations" (absmean ternary weights,
 *        multiply by -1/0/1 as negate/drop/keep) and "Core components: MLGRU
 *        and GLU" (MLGRU token mixer, MatMul-free GLU, overview figure panels
 *        "MatMul vs. scaled ternary accumulation" and "RMS Norm").
 *   [HL] hysenlabs review of ridgerchu/matmulfreellm: "FusedBitLinear" (RMSNorm
 *        then a fused quantise-and-accumulate kernel) and "HGRN attention"
 *        (f/c/g projections, recurrence, o-projection).
 *
 * Conventions for every call below
 *   - Pointers marked (device) are CUDA device addresses on the current
 *     device; (host) are ordinary host addresses. The caller owns every buffer
 *     it passes; the library never frees or keeps them past the call, except
 *     the weight pointers remembered by mmf_block_create (see there).
 *   - Tensors are dense and row-major (last index fastest). All device pointers
 *     must be 16-byte aligned; row lengths K and d must be multiples of 16.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Compute calls are asynchronous on that stream and do not synchronise,
 *     except mmf_state_get / mmf_state_set / mmf_check, which synchronise it.
 *   - `ws` / `ws_bytes` is caller-owned device scratch; the matching *_ws_size
 *     function gives the minimum size. Workspace contents need no initialisation
 *     and are clobbered. Calls that share a workspace must not overlap in time.
 *   - Every argument is validated on the host before any launch; on error the
 *     call returns a non-zero mmf_status, launches nothing and sets a message
 *     readable with mmf_last_error() (thread-local). No C++ exception, abort or
 *     exit ever crosses this interface.
 *   - Kernels never trap: a device-side fault condition (for example a bounded
 *     wait that ran out) is recorded in a per-device status word which
 *     mmf_check() returns and clears.
 *   - Activation dtypes: MMF_F32 (float) or MMF_BF16 (bfloat16). Internal
 *     arithmetic is int8 x ternary -> int32 for the accumulation and fp32
 *     elsewhere; the recurrent state h is always fp32.
 */
#ifndef MMF_H_
#define MMF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mmf_status {
  MMF_OK = 0,
  MMF_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum */
  MMF_ERR_UNSUPPORTED_SHAPE = 2,  /* K or d not a multiple of 16, too large, gains differ */
  MMF_ERR_MISALIGNED = 3,         /* a device pointer is not 16-byte aligned */
  MMF_ERR_WORKSPACE = 4,          /* ws_bytes smaller than the *_ws_size answer */
  MMF_ERR_CUDA = 5,               /* a CUDA runtime call failed (message has the CUDA error) */
  MMF_ERR_TIMEOUT = 6,            /* a bounded device-side wait ran out (mmf_check) */
  MMF_ERR_NOMEM = 7               /* host or device allocation inside the library failed */
} mmf_status;

typedef enum mmf_dtype { MMF_F32 = 0, MMF_BF16 = 1 } mmf_dtype;

/* Library version string, e.g. "mmf 0.1.0 sm_100a". */
const char* mmf_version(void);

/* Message of the last failed call on this host thread ("" if none). */
const char* mmf_last_error(void);

/* Synchronise `stream`, then return MMF_ERR_CUDA for a pending CUDA error,
 * MMF_ERR_INVALID_ARG if mmf_embed met a token id outside [0, V), or
 * MMF_ERR_TIMEOUT if a kernel recorded a bounded-wait timeout since the last
 * check (the status word is cleared), else MMF_OK. */
mmf_status mmf_check(void* stream);

/* ------------------------------------------------------------------------- */
/* Ternary weights                                                            */
/* ------------------------------------------------------------------------- */

/* A ternary BitLinear layer y = BitLinear(x), x: [M, K] -> y: [M, N].
 *   packed (device) uint32 [N, K/16]: 2-bit codes, K-contiguous. The stored
 *          value is w + 1 in {0,1,2} for w in {-1,0,1}; the code of column
 *          k = 16*j + 4*i + b is in word j at bits [8*b + 2*i, 8*b + 2*i + 2).
 *          Field value 3 is invalid.
 *   gamma  (device) one float: the absmean weight scale of the whole matrix.
 *   gain   (device) float [K] RMSNorm gain, or NULL for all ones.
 *   bias   (device) float [N], or NULL for all zeros.
 *   codes  (device) uint8 [N, K], or NULL: the same stored values one byte per
 *          weight (mmf_unpack_codes builds it). When given, prefill-sized
 *          contractions load it directly instead of expanding `packed` in
 *          shared memory (same results; 4x the memory). It must match `packed`.
 * The struct itself is read during the call only. */
typedef struct mmf_tlinear {
  const uint32_t* packed;
  const float* gamma;
  const float* gain;
  const float* bias;
  int32_t N;
  int32_t K;
  const uint8_t* codes;
} mmf_tlinear;

/* Scratch bytes mmf_quantize_weights needs for an N x K matrix. */
size_t mmf_quantize_weights_ws_size(int32_t N, int32_t K);

/* Absmean ternarisation and 2-bit packing of one latent weight matrix.
 * [DC] "Replacing MatMul with ternary operations": the matrix is scaled by the
 * mean absolute value of its elements and each element is rounded to the
 * nearest of -1, 0, 1. Here gamma = (float)(sum |W| in fp64 / (N*K)) and
 * w = clamp(round_half_even(W / (gamma + 1e-5f)), -1, 1) with one IEEE fp32
 * division. The fp64 sum is reduced in a fixed order, so the result is
 * deterministic for a given N, K.
 *   W      (device) float [N, K] latent weights (read only)
 *   packed (device) uint32 [N, K/16] output codes, format as in mmf_tlinear
 *   gamma  (device) one float, output
 * Errors: INVALID_ARG (null, N or K < 1), UNSUPPORTED_SHAPE (K % 16 != 0),
 *         MISALIGNED, WORKSPACE. */
mmf_status mmf_quantize_weights(const float* W, int32_t N, int32_t K, uint32_t* packed,
                                float* gamma, void* ws, size_t ws_bytes, void* stream);

/* One byte per weight from the packed codes: codes[n, k] = the stored value
 * w + 1 of column k of row n (format as in mmf_tlinear), for the optional
 * mmf_tlinear.codes. Asynchronous on stream.
 *   packed (device) uint32 [N, K/16], read only
 *   codes  (device) uint8 [N, K], output, 16-byte aligned
 * Errors: INVALID_ARG (null, N or K < 1), UNSUPPORTED_SHAPE (K % 16 != 0),
 *         MISALIGNED, CUDA. */
mmf_status mmf_unpack_codes(const uint32_t* packed, int32_t N, int32_t K, uint8_t* codes, void* stream);

/* ------------------------------------------------------------------------- */
/* FusedBitLinear                                                             */
/* ------------------------------------------------------------------------- */

/* Optional device outputs of mmf_bitlinear's intermediate steps (each may be NULL). */
typedef struct mmf_bitlinear_debug {
  int8_t* q;       /* [M, K] int8 activation codes */
  float* scale;    /* [M] per-token quantisation scale s */
  int32_t* acc;    /* [M, N] exact int32 accumulators sum_k q[m,k] * w[n,k] */
} mmf_bitlinear_debug;

/* Scratch bytes mmf_bitlinear needs for M tokens of length K. */
size_t mmf_bitlinear_ws_size(int32_t M, int32_t K);

/* FusedBitLinear forward. [HL] "FusedBitLinear": RMSNorm on the input, then
 * quantisation and accumulation against ternary weights; [DC] "Replacing
 * MatMul with ternary operations" and the overview figure's "MatMul vs. scaled
 * ternary accumulation" panel. Per token m:
 *   x^ = x * (1 / sqrt(mean(x^2) + eps)) * gain        (mean of squares summed in fp64)
 *   s  = 127 / max(max|x^|, 1e-5),  q = clamp(round_half_even(x^ * s), -128, 127)
 *   acc[n] = sum_k q[k] * w[n,k]   exactly, in int32
 *   y[n] = acc[n] * gamma / s + bias[n]
 *   lin (host) layer description; x (device) [M, K] in dtype; y (device) [M, N]
 *   in dtype; eps > 0 is the RMSNorm epsilon; dbg (host struct, device
 *   pointers) may be NULL. M = 0 is allowed and does nothing.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, CUDA. */
mmf_status mmf_bitlinear(const mmf_tlinear* lin, const void* x, mmf_dtype dtype, int32_t M,
                         void* y, float eps, void* ws, size_t ws_bytes, void* stream,
                         const mmf_bitlinear_debug* dbg);

/* ------------------------------------------------------------------------- */
/* MLGRU scan                                                                 */
/* ------------------------------------------------------------------------- */

/* Scratch bytes mmf_mlgru_scan needs for B sequences of T tokens and d channels
 * (a small constant: the scan keeps its state on chip). */
size_t mmf_mlgru_scan_ws_size(int32_t B, int32_t T, int32_t d);

/* MLGRU gates and gated recurrence over T tokens for B sequences.
 * [DC] "Core components: MLGRU and GLU" (token-by-token update of a hidden
 * state through element-wise gates valued in [0,1]); [HL] "HGRN attention".
 * With f~, c~, g~ the pre-activations of token t:
 *   f = sigmoid(f~), c = SiLU(c~), g = sigmoid(g~)
 *   h_t = f * h_{t-1} + (1 - f) * c,   o'_t = g * h_t
 *   pre (device) [B, T, 3, d] in dtype: for each token the rows f~, c~, g~
 *   h   (device) float [B, d]: h_0 on entry, h_T on return (in place)
 *   o   (device) [B, T, d] in dtype: o'
 *   ws  (device) scratch of mmf_mlgru_scan_ws_size(B, T, d) bytes.
 * One CTA owns a block of channels of one sequence and walks the sequence's
 * chunks in order with the state on chip; within a chunk the warps' steps are
 * composed as affine maps. Its waits for the gate tiles it streams in are
 * bounded (a timeout is reported by mmf_check as MMF_ERR_TIMEOUT).
 * T = 0 leaves h unchanged. Errors: INVALID_ARG, UNSUPPORTED_SHAPE (d % 8),
 * MISALIGNED, WORKSPACE, CUDA. */
mmf_status mmf_mlgru_scan(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                          float* h, void* o, void* ws, size_t ws_bytes, void* stream);

/* Scratch bytes mmf_mlgru_scan_backward needs when it is not given the
 * forward states: 4 x B x T x d (0 needed when hs is given). */
size_t mmf_mlgru_scan_backward_ws_size(int32_t B, int32_t T, int32_t d);

/* Training forward: mmf_mlgru_scan (sigmoid output gate) that also stores the
 * states h_t, for mmf_mlgru_scan_backward.
 *   pre, h (in place: h_0 -> h_T) as for mmf_mlgru_scan; o (device) [B, T, d]
 *   in dtype: o', or NULL to skip it; hs (device) float [B, T, d]: h_t.
 * No scratch. Errors: as mmf_mlgru_scan. */
mmf_status mmf_mlgru_scan_states(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                                 float* h, void* o, float* hs, void* stream);

/* Training: gradients of mmf_mlgru_scan (sigmoid output gate) for the
 * upstream gradients dout = dL/do' and dhT = dL/dh_T. The pages give no
 * backward formula ([DC] "Memory efficiency": the models are trained with
 * fused GPU kernels); this is the exact derivative of the forward recurrence.
 * With lambda_t = dL/dh_t and mu_t = f_t lambda_t:
 *   lambda_t = dout_t g_t + mu_{t+1},  mu_T = dhT
 *   dg~_t = dout_t h_t g_t (1 - g_t)
 *   df~_t = lambda_t (h_{t-1} - c_t) f_t (1 - f_t)
 *   dc~_t = lambda_t (1 - f_t) sigmoid(c~_t) (1 + c~_t (1 - sigmoid(c~_t)))
 *   dh0 = mu_0
 *   pre  (device) [B, T, 3, d] in dtype: the forward's pre-activations
 *   h0   (device) float [B, d]: the forward's initial state (read only)
 *   dout (device) [B, T, d] in dtype; dhT (device) float [B, d] or NULL (zero)
 *   hs   (device) float [B, T, d]: the forward states (mmf_mlgru_scan_states),
 *        or NULL: then they are recomputed into ws first (one more launch)
 *   dpre (device) [B, T, 3, d] in dtype: dL/df~, dL/dc~, dL/dg~ per token
 *   dh0  (device) float [B, d]: dL/dh0; must not overlap h0
 *   ws   (device) scratch of mmf_mlgru_scan_backward_ws_size(B, T, d) bytes
 *        (may be NULL when hs is given).
 * Without hs, two launches: the forward scan writing the states h_t into ws, then a
 * reverse chunked scan (one CTA per sequence x 64 channels, chunks from the
 * last to the first, the backward maps mu -> f mu + f dout g composed like
 * the forward ones). T = 0 does nothing. Errors: as mmf_mlgru_scan. */
mmf_status mmf_mlgru_scan_backward(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                                   const float* h0, const void* dout, const float* dhT, const float* hs,
                                   void* dpre, float* dh0, void* ws, size_t ws_bytes, void* stream);

/* Scratch bytes mmf_mlgru_scan_gnorm needs: 4 x B x T x d bytes for
 * v = swish(g~) h in fp32, 4 x B x T x ceil(d / 32) for the partial sums of
 * h^2, and a little padding. */
size_t mmf_mlgru_scan_gnorm_ws_size(int32_t B, int32_t T, int32_t d);

/* The MLGRU recurrence of mmf_mlgru_scan with the g_norm output gate in place
 * of sigmoid(g~) h. [HL] "HGRN attention": the recurrence output passes g_norm,
 * a FusedRMSNormSwishGate (RMSNorm and swish activation fused). Per token t,
 * normalising over the d channels:
 *   o'_t = h_t / sqrt(mean_n h_t[n]^2 + eps) * gain * swish(g~_t),
 *   swish(z) = z sigmoid(z)
 * pre, h, o as for mmf_mlgru_scan; gain (device) float [d], not NULL (a
 * vector of ones for an unscaled norm); eps > 0. Two launches on `stream`:
 * the scan writes v = swish(g~) h and per-token partial sums of h^2 into ws,
 * then a row kernel writes o'. Errors: as mmf_mlgru_scan. */
mmf_status mmf_mlgru_scan_gnorm(const void* pre, mmf_dtype dtype, int32_t B, int32_t T, int32_t d,
                                float* h, const float* gain, float eps, void* o, void* ws,
                                size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Model ends: embedding lookup and greedy next token                         */
/* ------------------------------------------------------------------------- */

/* Token embedding lookup. [HL] "Install and model initialisation": the default
 * configuration has an embedding of 32000 entries at hidden size 2048.
 *   x[m, :] = table[ids[m], :]   for m < M
 *   ids   (device) int32 [M]; table (device) [V, d] in dtype (caller-owned,
 *         16-byte aligned); x (device) [M, d] in dtype, 16-byte aligned.
 * A row copy, bit-exact. An id outside [0, V) writes a zero row and is
 * reported by the next mmf_check (MMF_ERR_INVALID_ARG); the kernel does not
 * read outside the table. M = 0 does nothing. The same call gathers any rows
 * of a [V, d] tensor, e.g. the last token of each sequence of a block's output.
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (d % 16), MISALIGNED, CUDA. */
mmf_status mmf_embed(const int32_t* ids, int32_t M, const void* table, int32_t V, int32_t d,
                     mmf_dtype dtype, void* x, void* stream);

/* Greedy next token over the LM head's logits. [HL] "Official generation
 * example" samples; greedy decoding is the deterministic choice taken here:
 *   ids[m] = the index of the largest of logits[m, 0..V), the lowest index on
 *            ties (a NaN counts as larger than every number)
 *   logits (device) [M, V] in dtype; ids (device) int32 [M].
 * The head itself is a BitLinear d -> V (mmf_bitlinear; [HL] "FusedBitLinear":
 * every linear projection is one). One CTA per row. M = 0 does nothing.
 * Errors: INVALID_ARG, CUDA. */
mmf_status mmf_argmax(const void* logits, mmf_dtype dtype, int32_t M, int32_t V, int32_t* ids,
                      void* stream);

/* ------------------------------------------------------------------------- */
/* MatMul-free GLU                                                            */
/* ------------------------------------------------------------------------- */

/* Scratch bytes mmf_glu needs for M tokens, hidden d, inner size I. */
size_t mmf_glu_ws_size(int32_t M, int32_t d, int32_t I);

/* MatMul-free GLU channel mixer. [DC] "Core components: MLGRU and GLU": two
 * separate BitLinear layers, SiLU on one branch, element-wise product, then a
 * third BitLinear.
 *   p = SiLU(BitLinear_gate(x)) * BitLinear_up(x)   (stored in dtype, [M, I])
 *   y = BitLinear_down(p) (+ residual)
 * gate and up must share one RMSNorm gain (same pointer or both NULL) because x
 * is normalised and quantised once for both.
 *   x (device) [M, d]; residual (device) [M, d] or NULL; y (device) [M, d].
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE (shapes disagree, gains differ),
 * MISALIGNED, WORKSPACE, CUDA. */
mmf_status mmf_glu(const mmf_tlinear* gate, const mmf_tlinear* up, const mmf_tlinear* down,
                   const void* x, const void* residual, void* y, int32_t M, mmf_dtype dtype,
                   float eps, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* Blocks and recurrent state                                                 */
/* ------------------------------------------------------------------------- */

/* Weights of one MatMul-free block: MLGRU projections f, c, g, o (d x d) and
 * GLU gate, up (I x d) and down (d x I). f, c and g share one gain, gate and up
 * share one gain. gnorm (device, float [d], 16-byte aligned) selects the
 * g_norm output gate of mmf_mlgru_scan_gnorm with that gain; NULL selects the
 * sigmoid output gate o' = sigmoid(g~) h. */
typedef struct mmf_block_weights {
  mmf_tlinear f, c, g, o, gate, up, down;
  const float* gnorm;
} mmf_block_weights;

typedef struct mmf_block mmf_block;   /* opaque */
typedef struct mmf_state mmf_state;   /* opaque */

/* Validate a block's weights and build its launch descriptors. The device
 * buffers named in `w` are NOT copied: they must stay valid and unchanged
 * until mmf_block_destroy. The handle is host memory owned by the library.
 * For the prefill contraction the block uses each matrix's codes one byte per
 * weight: the caller's mmf_tlinear.codes when given, otherwise a copy the
 * library makes (4x the packed size, e.g. 303 MB for a 24-block d=1024 /
 * I=2816 stack). The copy is not made here: the block's first forward call
 * with T > 1 and at least 128 tokens allocates it with cudaMalloc on the
 * current device and fills it with one kernel on that call's stream, so make
 * that first prefill call outside stream capture; a decode-only block never
 * allocates it. mmf_block_destroy frees it. The environment variable
 * MMF_PREFILL_UNPACKED=0 turns the copy off, and when the memory cannot be
 * allocated the block goes without it (the contraction then expands the packed
 * codes in shared memory; same results).
 * Errors: INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED, NOMEM, CUDA. */
mmf_status mmf_block_create(const mmf_block_weights* w, int32_t d, int32_t I, mmf_block** out);
void mmf_block_destroy(mmf_block* blk);

/* Free the one-byte code copy that the block's first prefill-sized call made
 * (see mmf_block_create), e.g. before a long decode-only phase, where only the
 * packed codes are read: the block returns to its packed size (plus the
 * caller's own one-byte codes, if it gave any). The next forward call with
 * T > 1 and at least 128 tokens makes the copy again. Synchronises the device
 * first when there is a copy to free, so call it between forward calls; it
 * must not run concurrently with a forward call on the same block.
 * Results are unchanged either way. Errors: INVALID_ARG (null), CUDA. */
mmf_status mmf_block_release_codes(mmf_block* blk);

/* Recurrent state h for L layers x B sequences x d channels, fp32, zeroed.
 * The library allocates it with cudaMalloc on the current device and frees it
 * in mmf_state_destroy. The first decode step (T = 1) that runs as one launch
 * (see mmf_block_forward) also allocates, with cudaMalloc, the state's
 * exchange buffers for that launch (2 x 4 bytes x B x (3 d + I) per layer plus
 * a small header; again for a later call with a larger I), so make that first
 * decode call before any stream capture. Calls that share a state must be
 * ordered on one stream: h and the exchange buffers are updated in place. */
mmf_status mmf_state_create(int32_t L, int32_t B, int32_t d, mmf_state** out);
void mmf_state_destroy(mmf_state* st);
/* Zero every layer's state and reset the decode exchange buffers
 * (asynchronous on stream); also the way to recover after mmf_check reported
 * a decode step whose waits gave up (codes 5 and 6). */
mmf_status mmf_state_reset(mmf_state* st, void* stream);
/* Device address of layer `layer`'s state, float [B, d]; NULL if out of range. */
float* mmf_state_layer(mmf_state* st, int32_t layer);
/* Copy the whole state [L, B, d] fp32 to / from host memory; synchronises stream. */
mmf_status mmf_state_get(const mmf_state* st, float* host_dst, void* stream);
mmf_status mmf_state_set(mmf_state* st, const float* host_src, void* stream);

/* Scratch bytes mmf_block_forward / mmf_stack_forward need for B x T tokens. */
size_t mmf_block_ws_size(const mmf_block* blk, int32_t B, int32_t T);

/* One MatMul-free block on x [B, T, d] -> y [B, T, d] (both device, dtype):
 *   y1 = x + o_proj(MLGRU(x)),  y = y1 + GLU(y1)
 * with the block's output gate (sigmoid, or g_norm when its gnorm gain is set).
 * [HL] "HGRN attention" (the block input is normalised first, then f/c/g
 * projections, recurrence and o-projection) and [DC] "Core components".
 * The MLGRU continues from the state of `layer` in `st` and leaves h_T there,
 * so T = 1 is one decode step and consecutive calls may split a prompt.
 * A decode step (T = 1) of B <= 8 sequences (d and I multiples of 64, at
 * most 3 x 16 rows of each matrix per SM) runs as one cooperative launch:
 * every CTA streams its rows of the four projections through shared memory
 * and the stages hand their outputs over through the state's exchange
 * buffers (mmf_state_create). Each wait in that launch is bounded (about 1 s);
 * one that runs out is reported by mmf_check (MMF_ERR_TIMEOUT, code 5 or 6),
 * after which the state must be reset. Larger batches, other shapes, or the
 * environment variable MMF_DECODE_STEP_KERNEL=0 run four contractions instead
 * (f|c|g with the recurrence step in its epilogue, o, gate|up, down), with the
 * same arithmetic. A g_norm block's decode step runs its prefill sequence
 * (f|c|g contraction, scan and row kernel of mmf_mlgru_scan_gnorm, o, gate|up,
 * down) with T = 1. x and y must not overlap. Errors: INVALID_ARG,
 * UNSUPPORTED_SHAPE, MISALIGNED, WORKSPACE, NOMEM, CUDA. */
mmf_status mmf_block_forward(const mmf_block* blk, int32_t layer, mmf_state* st,
                             const void* x, void* y, int32_t B, int32_t T, mmf_dtype dtype,
                             float eps, void* ws, size_t ws_bytes, void* stream);

/* Optional device outputs of one block step's stored intermediates, for
 * checking each stage on its own (any field may be NULL; M = B * T tokens,
 * activation dtype unless stated):
 *   pre       [M, 3, d]: the f~, c~, g~ pre-activations as the kernels store them
 *   og        [M, d]: o', the output-gated state, the input of the o projection
 *   y1        [M, d]: x + o, the token mixer's output and the GLU's input
 *   p         [M, I]: SiLU(gate) * up, the input of the down projection
 *   q[i]      int8 activation codes of the i-th quantised input (0: x [M, d],
 *             1: o' [M, d], 2: y1 [M, d], 3: p [M, I])
 *   scale[i]  float [M]: their per-token scales s
 * Buffers are 16-byte aligned device memory of at least the sizes above. */
typedef struct mmf_block_debug {
  void* pre;
  void* og;
  void* y1;
  void* p;
  int8_t* q[4];
  float* scale[4];
} mmf_block_debug;

/* mmf_block_forward, also writing the intermediates named in `dbg` (host
 * struct of device pointers; NULL behaves as mmf_block_forward). The stages
 * and their results are those of mmf_block_forward; the extra copies are
 * stream-ordered device-to-device copies, plus code outputs of the
 * contraction kernels that quantise their own input rows.
 * Errors: as mmf_block_forward, and MISALIGNED for a debug buffer. */
mmf_status mmf_block_forward_debug(const mmf_block* blk, int32_t layer, mmf_state* st,
                                   const void* x, void* y, int32_t B, int32_t T, mmf_dtype dtype,
                                   float eps, void* ws, size_t ws_bytes, void* stream,
                                   const mmf_block_debug* dbg);

/* L blocks in sequence (block l uses state layer l): y = block_{L-1}(...block_0(x)).
 * blocks (host) array of L handles. x and y (device) [B, T, d] must not overlap;
 * intermediate activations live in the workspace (mmf_block_ws_size of the
 * largest block). A decode step (T = 1) that qualifies for the one-launch form
 * (mmf_block_forward) covers up to 32 layers per launch. Errors as
 * mmf_block_forward. */
mmf_status mmf_stack_forward(const mmf_block* const* blocks, int32_t L, mmf_state* st,
                             const void* x, void* y, int32_t B, int32_t T, mmf_dtype dtype,
                             float eps, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------- */
/* FusedBitLinear without a workspace                                         */
/* ------------------------------------------------------------------------- */

/* Bytes of the fixed device array mmf_bitlinear_noalloc uses as scratch. */
#define MMF_NOALLOC_SCRATCH_BYTES (2u * 1024u * 1024u)

/* The same computation as mmf_bitlinear (y = BitLinear(x), x [M, K] -> y [M, N]),
 * for callers that can neither allocate device memory nor pass a workspace:
 * a custom-operator plug-in that is handed only its input and output buffers,
 * or a process that reserved its whole device-memory budget up front. The
 * paper has no counterpart to this call; it is a property of this library.
 *
 * Scratch (the int8 activation codes, scales and row sums) lives in one fixed
 * array of MMF_NOALLOC_SCRATCH_BYTES that the library image places in device
 * memory on every GPU that loads it and keeps until the process exits. The
 * call never calls cudaMalloc, cudaFree or any allocating routine. Its size
 * limit: round_up(M*K, 256) + 2 * round_up(4*M, 256) <= MMF_NOALLOC_SCRATCH_BYTES
 * (for example M = 64 tokens of K = 16384, or at most M = 511 of K = 4096); larger calls
 * return MMF_ERR_UNSUPPORTED_SHAPE with a message naming the limit.
 * The first call on a device looks up the array's device address (a one-time
 * set-up with that device current); make that first call before any stream
 * capture. Every call shares the array and it keeps the last call's contents
 * (each call overwrites everything it reads, so nothing needs clearing); calls
 * that overlap on the GPU race on it and must be serialised by the caller.
 * Arguments, layouts and the other errors are those of mmf_bitlinear. */
mmf_status mmf_bitlinear_noalloc(const mmf_tlinear* lin, const void* x, mmf_dtype dtype, int32_t M,
                                 void* y, float eps, void* stream);

/* ------------------------------------------------------------------------- */
/* Kernel timing (tracing)                                                    */
/* ------------------------------------------------------------------------- */

/* When enabled, every kernel launch the library makes is bracketed by two CUDA
 * events recorded on the launch's stream (process-wide switch, off by default;
 * do not enable it while capturing a CUDA graph). Costs two event records per
 * launch and nothing on the device. */
mmf_status mmf_prof_enable(int32_t on);
/* Wait for every recorded event pair and fold the durations into per-kernel
 * totals. Returns the number of kernel kinds seen since the last reset, or -1
 * on a CUDA error (see mmf_last_error). */
int32_t mmf_prof_collect(void);
/* Totals of kernel kind i (0 <= i < mmf_prof_collect()): its name (host buffer,
 * truncated to name_len - 1 bytes), its number of launches and the summed
 * device time in milliseconds. */
mmf_status mmf_prof_get(int32_t i, char* name, size_t name_len, int64_t* launches, double* total_ms);
/* Forget all totals and pending events. */
void mmf_prof_reset(void);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MMF_H_ */
