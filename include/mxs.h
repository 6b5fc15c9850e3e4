/*
 * mxs.h -- C ABI of libmxs: mixed-width MXINT quantisation and GEMM for B200.
 *
 * The method is MXSens (Sensitivity-Aware Mixed-Precision Quantization for
 * Efficient LLM Inference, arXiv 2607.17733).  Citations below name the page
 * and section the operation comes from:
 *   [TS]  gist.science technical summary ("Technische Samenvatting") §1-§5;
 *   [ABS] the paper's abstract (insight.artgrammer.co.kr);
 *   [RP]  researchpod.app summary;
 *   [RV]  romaanj.github.io review.
 * The pages publish no formula beyond H = X^T X, no bit layout and no API;
 * the fixed readings used by this library are stated at each entry point.
 *
 * Conventions (all entry points):
 *   - Pointers marked (device) are CUDA device pointers on the current device;
 *     (host) are host pointers.  The caller allocates and owns every buffer,
 *     including workspaces; the library never allocates device memory.
 *   - Matrices are row-major with unit stride along K (the input dimension);
 *     ld* arguments are row pitches in ELEMENTS.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     Device work is stream-ordered and asynchronous; arguments are checked
 *     on the host before any launch and a non-MXS_OK status means nothing was
 *     launched.  mxs_allocate synchronises the stream in one case only:
 *     budget mode over more than one layer, where the greedy needs the
 *     device-computed group gains on the host.
 *   - Device-side failures (a bounded wait that expired) are recorded in a
 *     per-device status word and returned by mxs_sync.
 *   - Calls are thread-safe apart from that shared status word.
 */
#ifndef MXS_H
#define MXS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXS_OK = 0,
    MXS_ERR_ARG = 1,       /* NULL pointer, negative size, bad enum            */
    MXS_ERR_SHAPE = 2,     /* inconsistent shapes / layouts                    */
    MXS_ERR_ALIGN = 3,     /* pointer or pitch misaligned (16 bytes required)  */
    MXS_ERR_DTYPE = 4,     /* unsupported element type                         */
    MXS_ERR_BUDGET = 5,    /* the fixed 8-bit blocks alone exceed the budget   */
    MXS_ERR_CUDA = 6,      /* a CUDA runtime call failed                       */
    MXS_ERR_TIMEOUT = 7,   /* a device-side bounded wait expired               */
    MXS_ERR_DEVICE = 8,    /* the current device is not sm_100                 */
    MXS_ERR_WORKSPACE = 9  /* workspace NULL, misaligned or too small          */
} mxs_status;

typedef enum { MXS_F32 = 0, MXS_BF16 = 1 } mxs_dtype;

/* One K-segment of the mixed-width layout.  Segments are stored in the order
 * 8-bit, 6-bit, 4-bit; a segment holds k_real columns followed by zero
 * padding up to k_pad = 32*ceil(k_real/32) positions and starts at padded
 * position k_off.  [TS §2.2: three mantissa widths 4/6/8; TS §2.3 last
 * paragraph: the mixed widths live inside MXINT's 32-value blocks.] */
typedef struct {
    int32_t bits;
    int64_t k_real;
    int64_t k_pad;
    int64_t k_off;
} mxs_segment;

/* Column layout of one linear layer: perm (device, K entries, or NULL for
 * the identity) lists the original column of each real position, segment by
 * segment, ascending within a segment.  Build it with mxs_layout_make. */
typedef struct {
    int64_t K;
    int64_t K_pad;
    mxs_segment seg[3];
    const int32_t *perm;
} mxs_layout;

/* A quantised matrix: `rows` rows in layout `lay`.  For segment g:
 *   codes[g]  (device) rows x code_pitch[g] bytes; row r holds k_pad codes of
 *             width bits, two's complement, packed: 4-bit two per byte (even
 *             position in the low nibble), 6-bit four per three bytes (a
 *             24-bit little-endian group, position 4j+i at bits 6i..6i+5),
 *             8-bit one per byte;
 *   scales[g] (device) rows x scale_pitch[g] bytes; one E8M0 byte per block
 *             of 32 positions: byte = e + 127, the block's value is
 *             code * 2^(e - bits + 2).
 * Pitches are multiples of 16 bytes (mxs_mxtensor_bytes gives them); the
 * bytes beyond each row's payload are left as the caller set them.
 * Empty segments (k_pad == 0) may have NULL pointers. */
typedef struct {
    int64_t rows;
    mxs_layout lay;
    uint8_t *codes[3];
    int64_t code_pitch[3];
    uint8_t *scales[3];
    int64_t scale_pitch[3];
} mxs_mxtensor;

enum { MXS_ALLOC_FRACTIONS = 0, MXS_ALLOC_BUDGET = 1, MXS_ALLOC_LAYER = 2 };

/* Bit-allocation policy.
 *   MXS_ALLOC_FRACTIONS: n8 = round(p8*K), n6 = round(p6*K) (half up, exact
 *     rational arithmetic on p = num/den), the rest 4-bit.
 *   MXS_ALLOC_BUDGET: n8 = min(fixed8, K) -- the most sensitive columns, one
 *     MXINT block when fixed8 = 32 [TS §2.2 8-bit, §2.3 fixed high-precision
 *     block]; then greedy 6-bit upgrades of 32-column groups under an average
 *     mantissa-bit budget num/den over all weight elements, E8M0 scales not
 *     counted [TS §2.3 dynamic 6-bit allocation; TS §4 hardware overhead:
 *     4 + 4*32/4096 = 4.03 bits for the fixed block alone].
 *   MXS_ALLOC_LAYER: n8 as in MXS_ALLOC_BUDGET; the 6-bit count of layer l
 *     is proportional to its layer score w_l (mxs_allocate's layer_w, e.g.
 *     from mxs_layer_scores), scaled by one global R that meets the budget
 *     [TS §2.3 "Dynamische 6-bit Allocatie"], in whole 32-column groups:
 *       n6_l(R) = min(K_l - n8_l, 32 * floor(R * w_l / 32)),
 *     R the largest value whose counts fit.  The counts change only at
 *     R = 32 k / w_l; those steps are taken in increasing R (ordered
 *     exactly: k_a w_b against k_b w_a as exact products), all steps of one
 *     R value together, until the next value's steps no longer fit.  No
 *     device data is read, so the call never synchronises. */
typedef struct {
    int32_t mode;
    int64_t num, den;
    int64_t p8_num, p8_den;
    int64_t p6_num, p6_den;
    int64_t fixed8;
} mxs_budget;

/* Human-readable name of a status code (static storage). */
const char *mxs_status_str(mxs_status st);

/* Number of kernels this library has launched in this process so far. */
int64_t mxs_launch_count(void);

/* Waits for `stream`, then returns and clears the device status word of the
 * current device: MXS_ERR_TIMEOUT if a bounded device wait expired since the
 * last call, MXS_ERR_CUDA if the stream reported an error, else MXS_OK. */
mxs_status mxs_sync(void *stream);

/* Diagnostic: sets, on the current device, how many SM clock cycles a
 * pipeline wait of the prefill GEMM's tensor-core kernels (the mxs_gemm
 * calls whose workspace size is non-zero) may spin before the kernel gives up: it records MXS_ERR_TIMEOUT
 * in the status word, stops issuing, lets the copies and MMAs it already
 * issued finish (waits bounded by the default limit), frees its tensor
 * memory and returns; its output is then unspecified.  cycles <= 0 restores
 * the default (4e9 cycles, about 2 s); larger values are clamped to it.
 * Synchronous; applies to GEMM launches made after it returns.  Lets a test
 * make a wait run out without a fault.  Errors: MXS_ERR_CUDA. */
mxs_status mxs_set_wait_limit(int64_t cycles);

/* Fills *out for K columns with counts = {n8, n6, n4} (host, summing to K)
 * and perm (device, K entries; NULL for the identity, e.g. the K/V cache
 * layout {0, 0, K}).  No device access; perm is stored, not read. */
mxs_status mxs_layout_make(int64_t K, const int64_t counts[3], const int32_t *perm,
                           mxs_layout *out);

/* Pitches and byte sizes of the code and scale buffers of a `rows`-row
 * tensor in layout *lay (host outputs, 3 entries each, zero for empty
 * segments; pitches are multiples of 16 bytes). */
mxs_status mxs_mxtensor_bytes(int64_t rows, const mxs_layout *lay,
                              int64_t code_pitch[3], int64_t code_bytes[3],
                              int64_t scale_pitch[3], int64_t scale_bytes[3]);

/* ---------------------------------------------------------------------------
 * mxs_sensitivity -- column sensitivity of one linear layer.
 * [TS §2.1: column-wise sensitivity from the diagonal of H = X^T X.]
 *   H[j] = (2/T) * sum_t X[t][j]^2                 (fp64)
 *   E[j] = sum_i (W[i][j] - Q4(W)[i][j])^2          (fp64)
 *   s[j] = H[j] * E[j]
 * Q4 is the 4-bit MXINT code of each W row in blocks of 32 ORIGINAL columns
 * (a short last block is zero-padded).  Rounding order: rows are summed in
 * chunks of 64 from zero, in row order, and chunk sums are added in chunk
 * order; the result is bit-identical for any launch configuration.
 *   X (device): T x K, dtype xt, pitch ldx (elements); W (device): N x K,
 *   dtype wt, pitch ldw; all values finite (a NaN or Inf makes H, E and s
 *   unspecified).  H, E, s (device): K doubles each (E may be NULL).
 *   ws (device, 256-byte aligned): mxs_sensitivity_workspace_bytes(T, N, K).
 * T, N >= 1, K >= 1. */
mxs_status mxs_sensitivity_workspace_bytes(int64_t T, int64_t N, int64_t K, size_t *bytes);
mxs_status mxs_sensitivity(const void *X, mxs_dtype xt, int64_t T, int64_t K, int64_t ldx,
                           const void *W, mxs_dtype wt, int64_t N, int64_t ldw,
                           double *H, double *E, double *s,
                           void *ws, size_t ws_bytes, void *stream);

/* mxs_sensitivity_noalloc -- mxs_sensitivity without a caller workspace, for
 * callers that cannot allocate device memory (code inside stream capture,
 * runtimes without an allocator).  The pages have no counterpart: this is a
 * library convenience around the same computation.
 *   The chunk partials live in one library-owned device array of 16 MiB per
 *   device (MXS_NOALLOC_SCRATCH_BYTES); shapes whose workspace
 *   (mxs_sensitivity_workspace_bytes) exceeds it return MXS_ERR_WORKSPACE
 *   before any launch.  No memory is allocated.
 *   The first call on a device looks up the array's address (with that
 *   device current); make one call on each device before any stream capture.
 *   A device reset (cudaDeviceReset) moves the array: the first call after
 *   it looks the address up again, so it too belongs outside any capture.
 *   Argument checks and return codes are those of mxs_sensitivity; they run
 *   before the device is touched.
 *   Every call shares the one array: calls that overlap on the GPU (other
 *   streams, other host threads) race on it and must be serialised by the
 *   caller.  Nothing in the array needs to start at zero.
 *   Results are bit-identical to mxs_sensitivity. */
#define MXS_NOALLOC_SCRATCH_BYTES (16u << 20)
mxs_status mxs_sensitivity_noalloc(const void *X, mxs_dtype xt, int64_t T, int64_t K, int64_t ldx,
                                   const void *W, mxs_dtype wt, int64_t N, int64_t ldw,
                                   double *H, double *E, double *s, void *stream);

/* ---------------------------------------------------------------------------
 * mxs_allocate -- 4/6/8-bit widths for n_layers layers and their column
 * permutations.  [TS §2.3: sort columns by sensitivity; the top block gets 8
 * bits; a sensitivity-driven number of 6-bit columns under a global budget;
 * the rest 4 bits.]
 *   Ranking: s descending, ties to the lower column index.
 *   Budget greedy (MXS_ALLOC_BUDGET): candidates are the next 32 ranked
 *   4-bit columns of each layer (fewer at the tail); gain = layer_w[l] * sum
 *   of their s (fp64, rank order), cost = 2 * N[l] * count bits; repeatedly
 *   take the highest gain/cost (compared as gain_a*cost_b > gain_b*cost_a in
 *   fp64, ties to the lower layer) and stop at the first that does not fit
 *   sum_l N_l (4 K_l + 4 n8_l + 2 n6_l) * den <= num * sum_l N_l K_l.
 *   Inputs: K, N (host, n_layers each); s (host array of n_layers device
 *   pointers, K[l] doubles each, finite and >= 0); layer_w (host, n_layers):
 *   in MXS_ALLOC_BUDGET the greedy's gain weights (NULL = all 1), in
 *   MXS_ALLOC_LAYER the layer scores (required, finite, >= 0).
 *   Outputs: perm (host array of device pointers, K[l] int32 each: the
 *   8-bit columns, then 6-bit, then 4-bit, ascending within each);
 *   counts (host, 3*n_layers: n8, n6, n4 per layer).
 *   ws (device): mxs_allocate_workspace_bytes(n_layers, K).
 * The counts depend only on K, N and the policy except in multi-layer budget
 * mode, which synchronises `stream` to read the group gains; otherwise the
 * call is asynchronous.  MXS_ERR_BUDGET if infeasible. */
mxs_status mxs_allocate_workspace_bytes(int32_t n_layers, const int64_t *K, size_t *bytes);
mxs_status mxs_allocate(int32_t n_layers, const int64_t *K, const int64_t *N,
                        const double *const *s, const double *layer_w,
                        const mxs_budget *budget, int32_t *const *perm,
                        int64_t *counts, void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * mxs_quantize_weight / mxs_quantize_act -- mixed-width MXINT quantisation of
 * the rows of a matrix (weights offline, activations and the K/V cache per
 * forward).  [TS §2.2 triplet widths; TS §2.3 last paragraph; RP: widths apply
 * to weights and activations; TS §4 W4A4KV4.]
 *   Row r, segment g, padded position p: x = src[r][perm[real_off_g + p]]
 *   for p < k_real, else 0.  For each block of 32 positions:
 *     e = floor(log2(max |x|)) clamped to [-127, 127], -127 for a zero block;
 *     scale byte = e + 127;
 *     q = clamp(round_half_even(x / 2^(e - m + 2)), -(2^(m-1)-1), 2^(m-1)-1).
 *   src (device): rows x K, dtype, pitch ld (elements), with rows ==
 *   out->rows and K == out->lay.K; out: caller-owned buffers sized by
 *   mxs_mxtensor_bytes.  The two entry points compute the same function;
 *   the K/V cache uses mxs_quantize_act with the identity layout {0, 0, K}. */
mxs_status mxs_quantize_weight(const void *W, mxs_dtype dt, int64_t N, int64_t ldw,
                               const mxs_mxtensor *out, void *stream);
mxs_status mxs_quantize_act(const void *A, mxs_dtype dt, int64_t M, int64_t lda,
                            const mxs_mxtensor *out, void *stream);

/* Decodes a quantised tensor to fp32 in padded-position order:
 * out (device) rows x K_pad, pitch ldo (elements).  A checking aid. */
mxs_status mxs_dequantize(const mxs_mxtensor *in, float *out, int64_t ldo, void *stream);

/* ---------------------------------------------------------------------------
 * mxs_gemm -- the mixed-width MXINT linear layer.
 * [TS §2.3 last paragraph and §4: the layer runs on the mixed MXINT blocks
 * directly, about 1% of the work at more than 4 bits for a 4.03-bit budget.]
 *   Y[m][n] = sum over padded positions k of deq(A)[m][k] * deq(W)[n][k]
 *   with fp32 accumulation, rounded to bf16 (round to nearest even).
 *   A, W: quantised tensors with identical segment tables (and perm);
 *   Y (device): A->rows x W->rows bf16, pitch ldy (elements).
 *   ws (device, 256-byte aligned): mxs_gemm_workspace_bytes(A, W); it holds
 *   the operands re-coded for the tensor cores (4-bit codes as E4M3 with
 *   their E8M0 block scales, 6/8-bit codes as exact bf16 values).
 * Products of decoded values are exact; only the fp32 accumulation and the
 * final bf16 rounding round. */
mxs_status mxs_gemm_workspace_bytes(const mxs_mxtensor *A, const mxs_mxtensor *W, size_t *bytes);
mxs_status mxs_gemm(const mxs_mxtensor *A, const mxs_mxtensor *W, void *Y, int64_t ldy,
                    void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * mxs_attn_decode -- one decode step of grouped-query attention that reads
 * the 4-bit MXINT K/V cache directly.  [TS §4: the W4A4KV4 setting keeps the
 * K/V cache in 4-bit MXINT; RV Validation: A4W4KV4 against A4W4KV16.]  The
 * pages give no attention formula; this is scaled dot-product attention of
 * one query token on the decoded cache:
 *   query head h reads kv head g = h / (n_qh / n_kvh);
 *   s_t = sm_scale * sum_d q[h][d] * deq(K)[t*n_kvh + g][d]      (t < T)
 *   p = softmax(s);   out[h][d] = sum_t p_t * deq(V)[t*n_kvh + g][d]
 *   q (device): n_qh x 128 bf16, pitch ldq (elements; 16-byte aligned rows);
 *   K, V: the caches as mxs_quantize_act writes them with the identity
 *   layout {0, 0, 128}: T*n_kvh rows, row t*n_kvh + g = token t of kv head g
 *   (a [T][n_kvh][128] cache flattened token-major), one 4-bit segment;
 *   out (device): n_qh x 128 fp32, pitch ldo (elements).
 *   Head dimension 128; n_qh a multiple of n_kvh with n_qh / n_kvh <= 8;
 *   T >= 1; block scale bytes <= 249 (values below 2^122).
 *   ws (device, 256-byte aligned): mxs_attn_decode_workspace_bytes(...), the
 *   per-split partial results (the call splits the tokens over CTAs and
 *   merges the splits in a second kernel).
 * Decoded cache values are exact; the dot products accumulate in fp32, the
 * softmax weights enter the output product with 16 significant bits. */
mxs_status mxs_attn_decode_workspace_bytes(int64_t T, int64_t n_qh, int64_t n_kvh, int64_t d, size_t *bytes);
mxs_status mxs_attn_decode(const void *q, int64_t n_qh, int64_t ldq, const mxs_mxtensor *K, const mxs_mxtensor *V,
                           int64_t T, int64_t n_kvh, float sm_scale, float *out, int64_t ldo,
                           void *ws, size_t ws_bytes, void *stream);

/* ---------------------------------------------------------------------------
 * mxs_layer_scores -- layer-wise sensitivity of a decoder stack.
 * [TS §2.1 "Laaggewijze Sensitiviteit": a layer's score is the L2 error at
 * the model's final output when that layer alone is quantised; TS §2.3: the
 * scores set each layer's 6-bit count, mxs_allocate's MXS_ALLOC_LAYER.]
 * The pages name the measure, not the model code; the readings:
 *   - the model is a Llama-architecture decoder stack without embedding
 *     table or LM head: x (T synthetic hidden states) goes in, the final
 *     RMSNorm of the last block's output comes out.  Block: RMSNorm (weight
 *     1, eps rms_eps) -> q, k, v projections -> rotary embedding (pair
 *     (i, i + d/2) of each head turned by t * rope_theta^(-2i/d) at token
 *     t) -> causal softmax attention (scale 1/sqrt(d), query head h on kv
 *     head h / (n_heads / n_kv_heads)) -> o projection + residual ->
 *     RMSNorm -> silu(gate) * up -> down projection + residual;
 *   - "quantised" is this library's W4A4 MXINT4 layer: the linear's fp32
 *     input through mxs_quantize_act and its bf16 weight through
 *     mxs_quantize_weight, both in the uniform 4-bit layout {0, 0, K}, then
 *     mxs_gemm (bf16 output);
 *   - score = Frobenius norm of (output with that layer quantised) minus
 *     (output of the unquantised stack), in fp64.
 * The unquantised stack runs in fp32 (bf16 weights widened exactly).
 *   m: the stack; m->W (host array of 7 * n_blocks device pointers, bf16,
 *   row-major out x in, 16-byte aligned) in the order q (n_heads*d x
 *   hidden), k, v (n_kv_heads*d x hidden), o (hidden x n_heads*d), gate, up
 *   (mlp x hidden), down (hidden x mlp) per block, d = hidden / n_heads.
 *   x (device): T x hidden fp32, pitch ldx; 1 <= T <= 1024.
 *   scores (host): 7 * n_blocks doubles, layer 7 b + j = linear j of block b.
 *   hidden, mlp and n_heads*d multiples of 32; d even, <= 256; n_heads a
 *   multiple of n_kv_heads.
 *   ws (device, 256-byte aligned): mxs_layer_scores_workspace_bytes(m, T).
 * A calibration routine, not a per-token one: it runs 1 + 7 * n_blocks
 * partial forward passes and synchronises `stream` to return the scores. */
typedef struct {
    int32_t n_blocks;
    int32_t hidden, n_heads, n_kv_heads, mlp;
    float rms_eps, rope_theta;
    const void *const *W;
} mxs_stack;
mxs_status mxs_layer_scores_workspace_bytes(const mxs_stack *m, int64_t T, size_t *bytes);
mxs_status mxs_layer_scores(const mxs_stack *m, const float *x, int64_t T, int64_t ldx, double *scores,
                            void *ws, size_t ws_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* MXS_H */
