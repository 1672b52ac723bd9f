/*
 * dstar_fmdq.h -- C ABI of the B200 (sm_100a) FMDQ differential linear layer.
 *
 * FMDQ is the fine-grained mixed-precision differential quantization of
 * DSTAR ("DSTAR: Accelerating Diffusion Transformers via Spatial and Temporal
 * Redundancy Reduction"), section 3.1.  One call computes, for a linear layer
 * Y = X W with int8 weights,
 *
 *   dX  = X_t - X_{t-1}                                  (section 2.2, Eq. 1)
 *   per sub-channel (16 tokens x 1 channel): M_i = max|dX|, PoT (Eq. 3),
 *        bit width b in {2,4,6,8} from the thresholds Thr_0 * 2^(2N),
 *        FPoT (Eq. 4), scale s_i = base * 2^FPoT (Eq. 5), codes q = rne(dX s_i)
 *   2-bit slices of every code, their FPoT lowered by 2 per slice, grouped by
 *        FPoT and encoded with shift counts               (section 3.1, steps 2-4)
 *   acc = shift-aligned accumulation of slice x weight    (section 3.1, step 5)
 *   Y_t = Y_{t-1} + acc * 2^(-lb-g_ref) * w_scale          (section 4.2 inverse
 *        quantization and accumulation units; section 4.3 reverse differential)
 *
 * and refreshes the caches (x_prev <- X_t, y_prev <- Y_t).
 *
 * Conventions for every entry point
 *   - All matrices are row-major in DEVICE memory and owned by the caller; the
 *     library allocates nothing.  Scratch lives in a caller-owned device
 *     workspace (dstar_fmdq_workspace_size bytes), except for
 *     dstar_fmdq_linear_noalloc, which uses a static device array instead.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  All work is enqueued asynchronously on it; nothing synchronises
 *     except dstar_fmdq_status.
 *   - Return value: DSTAR_OK or a negative DSTAR_ERR_* code, decided on the host
 *     before anything is enqueued (arguments) or right after (launch errors).
 *     dstar_fmdq_last_error() gives a one-line reason for the calling thread.
 *   - Data-dependent problems found on the device (non-finite dX, PoT above its
 *     maximum, an exhausted wait) set bits of the workspace's sticky status
 *     word, read and cleared by dstar_fmdq_status.  When a bit is set the
 *     outputs of the calls since the last read are unspecified.
 *   - The entry points are reentrant; two calls that share a workspace must be
 *     ordered on the device (same stream, or events).
 *
 * Interface choices
 *   - The status word lives in the caller's workspace, so the library keeps no
 *     global state (no per-stream or per-device table to create, look up or
 *     free): dstar_fmdq_status takes the workspace whose calls it reports.
 *   - The workspace size depends on M and K only: every section is per token
 *     or per (token tile, channel); N and the quantizer settings do not change
 *     it, so dstar_fmdq_workspace_size takes neither.
 *   - Debug output is requested by passing device buffers (debug_codes,
 *     debug_acc), not by a flag; the bounded device wait is exercised by its
 *     own entry point, dstar_fmdq_selftest_wait, so no flag of the production
 *     call can make a wait run out.
 */
#ifndef DSTAR_FMDQ_H
#define DSTAR_FMDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSTAR_FMDQ_VERSION 2

#if defined(__GNUC__)
#define DSTAR_API __attribute__((visibility("default")))
#else
#define DSTAR_API
#endif

/* return codes */
#define DSTAR_OK 0
#define DSTAR_ERR_INVALID_ARG (-1) /* bad pointer, shape, dtype, alignment, parameter */
#define DSTAR_ERR_WORKSPACE (-2)   /* workspace missing, misaligned or too small */
#define DSTAR_ERR_CUDA (-3)        /* a CUDA runtime call or launch failed */
#define DSTAR_ERR_UNSUPPORTED (-4) /* the current device is not sm_100 */

/* sticky device status bits (dstar_fmdq_status) */
#define DSTAR_STATUS_NONFINITE 1u /* some dX was NaN or infinite; that sub-channel was zeroed */
#define DSTAR_STATUS_RANGE 2u     /* some PoT exceeded DSTAR_POT_MAX and was clamped */
#define DSTAR_STATUS_TIMEOUT 4u   /* a bounded device wait ran out; the kernel returned early */

/* element types of dstar_mat */
#define DSTAR_F32 0
#define DSTAR_BF16 1
#define DSTAR_I8 2

/* tile_cfg.flags */
#define DSTAR_FLAG_NO_XPREV_REFRESH 1u /* leave x_prev untouched (caller swaps buffers) */
#define DSTAR_FLAG_SLICE_PATH 2u       /* compute every tile with the slice-stream kernel */
#define DSTAR_FLAG_DYNAMIC_BASE 4u     /* FMDQ-DYN: base = min M_i of the call (see dstar_fmdq_linear) */
/* Slice-GEMM output tile form, bits 8..10 of flags: 0 = the library's choice
 * (dstar_fmdq_gemm_tile), else one form for the call -- a tuning override;
 * results are the same bit for bit in every form.  The 256-column forms fall
 * back to 128 columns with fp32 outputs. */
#define DSTAR_FLAG_TILE_SHIFT 8
#define DSTAR_FLAG_TILE_MASK (7u << DSTAR_FLAG_TILE_SHIFT)
#define DSTAR_TILE_128x128 1u      /* one CTA */
#define DSTAR_TILE_128x256 2u      /* one CTA; bf16 outputs */
#define DSTAR_TILE_PAIR_256x256 3u /* a cluster of two CTAs (two SMs); bf16 outputs */
#define DSTAR_TILE_PAIR_256x128 4u /* a cluster of two CTAs (two SMs) */

/* limits of this implementation */
#define DSTAR_TILE_TOKENS 16   /* tokens per sub-channel (the only supported tile) */
#define DSTAR_POT_MAX 32       /* largest PoT (Eq. 3); larger ones clamp and set RANGE */
#define DSTAR_K_MAX 8192       /* input channels */
#define DSTAR_BASE_LOG2_MIN (-32)
#define DSTAR_BASE_LOG2_MAX 32
#define DSTAR_NOALLOC_SCRATCH_BYTES (64u << 20) /* static scratch of dstar_fmdq_linear_noalloc */

/* A row-major matrix in device memory: element (r, c) is at
 * data + (r * ld + c) * sizeof(element).  ld is in elements. */
typedef struct {
  void* data;
  int32_t dtype; /* DSTAR_F32, DSTAR_BF16 or DSTAR_I8 */
  int32_t reserved;
  int64_t rows, cols, ld;
} dstar_mat;

/* Per-call quantizer configuration (section 3.1, step 1) and scratch. */
typedef struct {
  int32_t tile_tokens; /* tokens per sub-channel; must be DSTAR_TILE_TOKENS */
  int32_t thr0_log2;   /* t0: Thr_0 = base_scale * 2^t0; Thr_N = Thr_0 * 2^(2N) */
  int32_t force_bits;  /* 0: bit width by the thresholds; 2, 4, 6 or 8: that width everywhere */
  uint32_t flags;      /* DSTAR_FLAG_* */
  void* workspace;     /* device memory, 256-byte aligned, dstar_fmdq_workspace_size bytes,
                          initialised once with dstar_fmdq_workspace_init */
  size_t workspace_bytes;
  int8_t* debug_codes; /* optional device [M x K] int8 (ld = K): every code q */
  int64_t* debug_acc;  /* optional device [M x N] int64 (ld = N): every exact accumulator */
} dstar_tile_cfg;

/* Byte offsets of the sections of a workspace for an (M, K) call.  The
 * sections hold the quantizer's outputs and stay valid until the next call
 * that uses the workspace:
 *   fpot    int8  [T x K]  absolute FPoT of each sub-channel (Eq. 4)
 *   bits    int8  [T x K]  its bit width
 *   g_ref   int32 [T]      finest FPoT of each 16-token tile
 *   count   int32 [T]      number of slice records of the tile
 *   records 8-byte [T x record_cap] records of the tile in (FPoT, channel)
 *           order: { uint32 word; uint16 k; int8 fpot; uint8 j }, where word
 *           holds the 2-bit field of slice j of channel k for the 16 tokens
 *           (token i in bits 2i..2i+1) -- the encoded stream of section 3.1
 *           step 4; the shift before a record is its fpot minus the previous
 *   planes  int32 [T]      tensor-core operand planes the tile needs
 *   plane0/plane1 int8 [M x K]  shift-folded operands of the tensor-core GEMM
 *   mask1   uint32 [T x mask_words]  K-chunks (128 wide) where plane 1 is nonzero
 *   dyn_base fp32 word  the base found by the last DSTAR_FLAG_DYNAMIC_BASE call
 * T = M / 16.  With DSTAR_FLAG_DYNAMIC_BASE, fpot holds FPoT relative to the
 * dynamic base (b - 2 - PoT) and the records carry those tags. */
typedef struct {
  size_t total;
  size_t status;
  size_t plane0, plane1;
  size_t fpot, bits;
  size_t g_ref, planes, count;
  size_t mask1;
  size_t records;
  int64_t mask_words;
  int64_t record_cap;
  size_t dyn_base; /* fp32 word: the dynamic base of the last DSTAR_FLAG_DYNAMIC_BASE call
                      (all bits set when no sub-channel had a nonzero M_i) */
} dstar_fmdq_ws_layout;

/* Workspace bytes needed by calls with M tokens and K input channels.
 * Errors: INVALID_ARG for a NULL `bytes`, negative sizes, K > DSTAR_K_MAX. */
DSTAR_API int dstar_fmdq_workspace_size(int64_t M, int64_t K, size_t* bytes);

/* Section offsets of that workspace (see dstar_fmdq_ws_layout). */
DSTAR_API int dstar_fmdq_workspace_layout(int64_t M, int64_t K, dstar_fmdq_ws_layout* out);

/* Clear the status word of a fresh workspace (enqueued on `stream`).  Call once
 * after allocating it; the other sections need no initialisation. */
DSTAR_API int dstar_fmdq_workspace_init(void* workspace, size_t bytes, void* stream);

/*
 * The FMDQ differential linear (whole hot path).
 *   x_t     [M x K] F32 or BF16: current input X_t (read only)
 *   x_prev  [M x K] same dtype:  cached X_{t-1}; overwritten with X_t unless
 *           DSTAR_FLAG_NO_XPREV_REFRESH (then the caller swaps buffers)
 *   y_prev  [M x N] F32 or BF16: cached Y_{t-1}; holds Y_t afterwards
 *   w_q     [N x K] I8 in [-127, 127]: weights, W_deq[k][n] = w_q[n][k] * w_scale[n]
 *   w_scale [N] fp32 device array: per-output-channel weight scale
 *   base_scale: the static base of Eq. 3 (section 3.1 "predefined static base");
 *           an exact power of two 2^lb, lb in [DSTAR_BASE_LOG2_MIN, DSTAR_BASE_LOG2_MAX].
 *           With DSTAR_FLAG_DYNAMIC_BASE (FMDQ-DYN, the paper's dynamic-base
 *           reference of section 5.2) a first pass over X_t and X_{t-1} finds
 *           base = the minimum of M_i over the sub-channels with a nonzero,
 *           finite M_i, and Eqs. 2-5 use it: PoT = ceil(log2(M_i / base)),
 *           codes q = rne(fl32(dX / base) * 2^(b-2-PoT)), FPoT relative to the
 *           base (b - 2 - PoT), Y_t = Y_{t-1} + acc * 2^-g_ref * base * w_scale.
 *           base_scale then only sets the predefined thresholds,
 *           Thr_N = base_scale * 2^(t0 + 2N) compared with M_i.
 *   tile_cfg: quantizer settings and workspace (see dstar_tile_cfg)
 *   y_out   [M x N] same dtype as y_prev: receives Y_t; may be y_prev itself
 *           (same pointer and ld) or a disjoint buffer, never a partial overlap
 * Shapes: M % 16 == 0 (M == 0 is a no-op), 0 < K <= DSTAR_K_MAX with K % 32 == 0,
 * N >= 0 with N % 16 == 0.  Pointers 16-byte aligned, ld * element size a
 * multiple of 16 bytes; w_q and w_scale are not written.
 */
DSTAR_API int dstar_fmdq_linear(const dstar_mat* x_t, dstar_mat* x_prev, dstar_mat* y_prev, const dstar_mat* w_q,
                      const float* w_scale, float base_scale, const dstar_tile_cfg* tile_cfg,
                      dstar_mat* y_out, void* stream);

/*
 * The chained feed-forward pair of a DiT block with the GELU fused into the
 * first layer's epilogue (section 4.3 "Operator Mapping": the reverse
 * differential and the GELU activation are fused with the linear layer):
 *   Y1_t = Y1_{t-1} + FMDQ(X_t - X_{t-1}) W1        (layer 1, cache y1_prev)
 *   H_t  = GELU(Y1_t) = Y1_t Phi(Y1_t)                written by layer 1's epilogue
 *   Y2_t = Y2_{t-1} + FMDQ(H_t - H_{t-1}) W2        (layer 2, cache y2_prev)
 *   x_t, x_prev   [M x K1]: as in dstar_fmdq_linear (x_prev refreshed unless
 *                 cfg1 has DSTAR_FLAG_NO_XPREV_REFRESH)
 *   y1_prev       [M x N1] F32/BF16: layer 1's cache, updated in place to Y1_t
 *   w1 [N1 x K1] I8, w1_scale [N1]
 *   h_t           [M x N1], y1_prev's dtype: receives H_t = GELU of the stored
 *                 Y1_t value, 0.5 y erfc(-y / sqrt 2): for bf16 from a table of
 *                 every bf16 value (fp64, rounded to fp32 then bf16), filled
 *                 once per CUDA context by the first call (make that call
 *                 outside stream capture); for fp32 in fp32 with erfcf
 *   h_prev        [M x N1]: H_{t-1}; refreshed to H_t unless cfg2 has
 *                 DSTAR_FLAG_NO_XPREV_REFRESH (then the caller swaps h_t, h_prev)
 *   y2_prev       [M x N2] F32/BF16: layer 2's cache, updated in place to Y2_t
 *   w2 [N2 x N1] I8, w2_scale [N2]
 *   cfg1, cfg2    each layer's settings and its own workspace, sized for
 *                 (M, K1) and (M, N1)
 * N1 must be a positive multiple of 32 (it is layer 2's K); h_t, h_prev,
 * y1_prev and y2_prev must not overlap.  Errors as dstar_fmdq_linear.
 */
DSTAR_API int dstar_fmdq_ffn_gelu(const dstar_mat* x_t, dstar_mat* x_prev, dstar_mat* y1_prev, const dstar_mat* w1,
                                  const float* w1_scale, dstar_mat* h_t, dstar_mat* h_prev, dstar_mat* y2_prev,
                                  const dstar_mat* w2, const float* w2_scale, float base_scale,
                                  const dstar_tile_cfg* cfg1, const dstar_tile_cfg* cfg2, void* stream);

/*
 * Sparse attention reuse with INT8 FMDQ operands (section 3.2 "Sparse
 * Attention Reuse"; section 4.3 "Attention Operation": every attention MMA
 * in INT8, activations through FMDQ at 8 bits).  For each of `heads`
 * independent problems (batch x head, stacked along the rows) of S tokens:
 *   cached step (reuse == 0):
 *     K -> int8 per key row (scale = max|row|/127, q = rne(k/scale));
 *     Q -> FMDQ with every width 8 and X_{t-1} = 0 (base base_q);
 *     scores = dequant(Q codes . K codes) * scores_scale, only on the blocks
 *              the mask keeps (block size DSTAR_SAR_BLOCK; pruned blocks are
 *              never computed);
 *     P = softmax of each row over its kept blocks (fp32), 0 elsewhere;
 *     P -> FMDQ with every width 8 and X_{t-1} = 0 (base base_p): this
 *          quantized P is the cache, kept in the workspace;
 *   reused step (reuse != 0): Q, K and the softmax are skipped and the P
 *     cached by the last cached step on this workspace is used;
 *   both: V -> int8 per head dimension; out = dequant(P codes . V codes),
 *     reading only the kept blocks of P.
 * Arguments
 *   q, k, v  [heads*S x d] BF16 or F32 (one dtype), device; d a multiple of
 *            32 (pad with zero channels; they change nothing)
 *   out      [heads*S x d] F32, device: written
 *   cfg      sizes, host block mask, scales and the caller-owned workspace of
 *            dstar_sar_workspace_size bytes (256-byte aligned), initialised
 *            once with dstar_sar_workspace_init
 * S: a positive multiple of DSTAR_SAR_BLOCK up to 32 blocks; every mask row
 * must keep at least one block.  Errors as dstar_fmdq_linear; status bits
 * through dstar_sar_status.
 */
#define DSTAR_SAR_BLOCK 128
typedef struct {
  int64_t heads;             /* independent attention problems (batch x heads) */
  int64_t seq;               /* S: tokens per problem */
  int64_t head_dim;          /* d */
  const uint8_t* block_mask; /* HOST [S/128 x S/128], row-major; nonzero = block kept */
  float scores_scale;        /* multiplies Q K^T (1 / sqrt of the unpadded head dimension) */
  float base_q, base_p;      /* static FMDQ bases of Q and of P (exact powers of two) */
  void* workspace;
  size_t workspace_bytes;
} dstar_sar_cfg;

/* Byte offsets of the attention workspace: ws_p and ws_q are FMDQ workspaces
 * (dstar_fmdq_ws_layout inside) of P (rows heads*S, K = S: the cache of the
 * reused steps) and of Q (K = d); kq int8 [heads*S x d] and ks fp32
 * [heads*S] (the key scales times scores_scale); vqt int8 [heads*d x S] and
 * vs fp32 [heads*d]; scores and probs fp32 [heads*S x S]. */
typedef struct {
  size_t total, ws_p, ws_q, kq, ks, vqt, vs, scores, probs;
} dstar_sar_layout;

DSTAR_API int dstar_sar_workspace_size(int64_t heads, int64_t seq, int64_t head_dim, size_t* bytes);
DSTAR_API int dstar_sar_workspace_layout(int64_t heads, int64_t seq, int64_t head_dim, dstar_sar_layout* out);
/* Clear the status words of a fresh attention workspace (enqueued on `stream`). */
DSTAR_API int dstar_sar_workspace_init(const dstar_sar_cfg* cfg, void* stream);
DSTAR_API int dstar_sar_attention(const dstar_mat* q, const dstar_mat* k, const dstar_mat* v, const dstar_sar_cfg* cfg,
                                  int reuse, dstar_mat* out, void* stream);
/* Synchronise `stream`, report and clear the status bits of the attention
 * workspace described by cfg (both of its FMDQ stages). */
DSTAR_API int dstar_sar_status(const dstar_sar_cfg* cfg, void* stream, uint32_t* status);

/*
 * dstar_fmdq_linear for callers that cannot allocate device memory.  The
 * paper has no counterpart: this is a packaging choice of the library.
 *
 * Who needs it: code that runs where device memory belongs to someone else --
 * a plug-in layer of an inference engine or a custom operator whose host only
 * hands it input and output buffers, a real-time loop that must not call
 * cudaMalloc (it can synchronise the device and take milliseconds), or a
 * framework whose caching allocator must account for every byte.  Such a
 * caller cannot create the workspace dstar_fmdq_linear asks for.
 *
 * Instead the library keeps a static device array of
 * DSTAR_NOALLOC_SCRATCH_BYTES (64 MiB) in its own image.  Every GPU that loads
 * the library's device code holds that array until the process exits (with
 * CUDA's lazy module loading, from this entry point's first call on the
 * device; with eager loading, from context creation).  The call allocates
 * nothing: no cudaMalloc, no cudaFree, no allocating library routine.
 *
 * Arguments, layouts, shapes and results are those of dstar_fmdq_linear, with
 * two differences:
 *   tile_cfg->workspace must be NULL and tile_cfg->workspace_bytes 0
 *           (INVALID_ARG otherwise); the other fields keep their meaning.
 *   status_out: NULL, or a 4-byte aligned word in device memory (or host
 *           memory the device can reach) that receives, in stream order, the
 *           DSTAR_STATUS_* bits of this call; the array's status word is then
 *           cleared, so each call reports only its own problems.
 * Size limit: the call needs dstar_fmdq_workspace_size(M, K) bytes of the
 * array (about 4.1 * M * K; e.g. M = 2048 tokens with K = 4608 channels fits)
 * and returns DSTAR_ERR_WORKSPACE, enqueueing nothing, when that exceeds
 * DSTAR_NOALLOC_SCRATCH_BYTES.
 * Set-up: every call looks up the array's device address with the caller's
 * device current.  The first call in a CUDA context (the first on a device,
 * and again after a device reset) also enqueues the clearing of the array's
 * status word on `stream`.  Make that first call before any stream capture.
 * Sharing: every call on a device uses the same array, which keeps the
 * previous call's contents.  Calls that may overlap on the GPU (different
 * streams without an ordering between them, or several host threads) race on
 * it and give wrong results: order them, for instance on one stream.
 */
DSTAR_API int dstar_fmdq_linear_noalloc(const dstar_mat* x_t, dstar_mat* x_prev, dstar_mat* y_prev,
                                        const dstar_mat* w_q, const float* w_scale, float base_scale,
                                        const dstar_tile_cfg* tile_cfg, dstar_mat* y_out, uint32_t* status_out,
                                        void* stream);

/*
 * First stage alone (section 3.1 steps 1-4, the paper's QPU): dX, max-abs,
 * PoT/bit width/FPoT, codes, 2-bit slices, FPoT-grouped encoded stream, plus
 * the tensor-core operand planes; refreshes x_prev like dstar_fmdq_linear.
 * Outputs go to the workspace sections listed in dstar_fmdq_ws_layout.
 */
DSTAR_API int dstar_fmdq_quantize(const dstar_mat* x_t, dstar_mat* x_prev, float base_scale,
                        const dstar_tile_cfg* tile_cfg, void* stream);

/*
 * Second stage alone (section 3.1 step 5 and the section 4.2/4.3 epilogue):
 * the shift-aligned slice GEMM over the workspace written by the last
 * dstar_fmdq_quantize with the same (M, K) and workspace, then
 * Y_t = Y_{t-1} + dequant(acc) into y_out and y_prev.  Same argument rules as
 * dstar_fmdq_linear; M and K are taken from y_prev and w_q.
 */
DSTAR_API int dstar_fmdq_slice_gemm(const dstar_mat* w_q, const float* w_scale, dstar_mat* y_prev, float base_scale,
                          const dstar_tile_cfg* tile_cfg, dstar_mat* y_out, void* stream);

/* The output tile shape the slice GEMM takes for an M x N output with K input
 * channels on the current device (out_bf16: bf16 outputs): *bm x *bn, and
 * *pair = 1 when a cluster of two CTAs (two SMs) computes each tile, 0 when
 * one CTA does.
 * Shapes: 128 x 128 and 128 x 256 in one CTA; 256 x 128 and 256 x 256 in a
 * pair (the 256-column forms with bf16 outputs only).  It follows from the
 * shape and the SM count alone (a model of the mainloop and the epilogue),
 * not from the data.  Launches nothing.  `pair` may be NULL.
 * Returns DSTAR_OK; DSTAR_ERR_INVALID_ARG for null bm/bn or negative sizes;
 * DSTAR_ERR_UNSUPPORTED / DSTAR_ERR_CUDA when the current device cannot be
 * queried or is not sm_100. */
DSTAR_API int dstar_fmdq_gemm_tile(int64_t M, int64_t N, int64_t K, int out_bf16, int* bm, int* bn, int* pair);

/* Synchronise `stream`, copy the workspace's sticky status word to *status
 * (DSTAR_STATUS_* bits, 0 when clean) and clear it. */
DSTAR_API int dstar_fmdq_status(void* workspace, void* stream, uint32_t* status);

/* Device self-test of the bounded wait used by every pipeline wait in the
 * library: launches one block whose thread waits on a barrier that nothing
 * completes, with a wall-clock limit of `limit_us` microseconds; the wait gives
 * up, the kernel sets DSTAR_STATUS_TIMEOUT in the workspace status word and
 * returns normally (the context stays usable). */
DSTAR_API int dstar_fmdq_selftest_wait(void* workspace, uint32_t limit_us, void* stream);

/* Device self-test of the division by the dynamic base (FMDQ-DYN divides every
 * dX by one base per call with FMA corrections of a correctly rounded
 * reciprocal instead of an IEEE division per element): for every
 * a = (1 + m 2^-23) 2^e -- all 2^23 significands m, e_lo <= e <= e_hi
 * (-126 < e < 128) -- and each of the n_b divisors b[i] (device memory), the
 * quotient is compared bit for bit with CUDA's __fdiv_rn(a, b[i]); the number
 * of differences is added to *count (device memory, 64-bit).  Enqueued on
 * `stream`; DSTAR_ERR_INVALID_ARG for null pointers or exponents out of range. */
DSTAR_API int dstar_fmdq_selftest_div(const float* b, int n_b, int e_lo, int e_hi, unsigned long long* count,
                                      void* stream);

/* Human-readable name of a return code; one-line reason for the last error of
 * the calling thread (empty when none). */
DSTAR_API const char* dstar_fmdq_error_string(int code);
DSTAR_API const char* dstar_fmdq_last_error(void);

DSTAR_API int dstar_fmdq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DSTAR_FMDQ_H */
