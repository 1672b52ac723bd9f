// Internal definitions shared by the host dispatcher and the kernels of the
// FMDQ differential linear library (not part of the C ABI).
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/dstar_fmdq.h"

namespace fmdq {

constexpr int kTile = DSTAR_TILE_TOKENS;  // tokens per sub-channel
constexpr int kBlockM = 128;               // rows of one tensor-core tile (8 token tiles)
constexpr int kChunkK = 128;               // int8 columns per K chunk (one 128-byte swizzle row)
constexpr int kPotMax = DSTAR_POT_MAX;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits give up after 2 s

// Plane split of a shift-folded operand v = q * 2^(g_ref - FPoT):
// v = A0 + 256 * A1 with A0 = the low byte of v read as signed, A1 the rest.
// One plane holds v in [-128, 127]; two planes hold v in [-128*257, 127*257].
constexpr int64_t kPlane1Lo = -128, kPlane1Hi = 127;
constexpr int64_t kPlane2Lo = -128 * 257, kPlane2Hi = 127 * 257;

// A row-major region to pull into L2 ahead of its reader: rows of row_bytes,
// ld_bytes apart (both multiples of 16, base 16-byte aligned).
struct L2Region {
  const uint8_t* base;
  int64_t rows, row_bytes, ld_bytes;
};

struct QuantParams {
  const void* x_t;
  void* x_prev;  // nullptr: X_{t-1} = 0 (the operand itself is quantized; no refresh)
  int64_t ld_xt, ld_xp;
  int64_t M, K;
  int lb, t0, force_bits;
  uint32_t flags;
  uint32_t* status;
  int8_t* plane0;
  int8_t* plane1;
  int8_t* fpot;
  int8_t* bits;
  int32_t* g_ref;
  int32_t* planes;
  int32_t* count;
  uint32_t* mask1;
  uint2* records;
  int64_t record_cap;
  int64_t mask_words;
  int8_t* debug_codes;
  // dynamic base (DSTAR_FLAG_DYNAMIC_BASE): the fp32 bits of min M_i written
  // by the first pass (all ones when none is nonzero); nullptr = static base
  uint32_t* dyn_base;
  // operands of the GEMM that follows in the same call (weights, cached
  // output): prefetched into L2 once the quantizer no longer streams HBM
  L2Region prefetch[2];
};

struct GemmParams {
  int64_t M, N, K;
  int lb;
  uint32_t flags;
  const int32_t* g_ref;
  const int32_t* planes;
  const uint32_t* mask1;
  int64_t mask_words;
  const float* w_scale;
  void* y_prev;
  int64_t ld_yp;
  void* y_out;
  int64_t ld_yo;
  int y_distinct;  // y_out is a different buffer: write both
  uint32_t* status;
  int64_t* debug_acc;
  const uint32_t* dyn_base;  // dynamic base word (nullptr = static base, whose scale is in lb)
  void* h_out;               // GELU(Y_t) output, same dtype as y (nullptr = none)
  int64_t ld_h;
  int tiles_m, tiles_n, num_chunks;
  // encoded stream, for tiles whose operands need more than two planes
  const int8_t* w_q;
  int64_t ld_w;
  const uint2* records;
  int64_t record_cap;
  const int32_t* count;
  const int8_t* bits;
};

// Batched heads and block sparsity of the attention GEMMs (sparse attention
// reuse): rows [h R, (h + 1) R) of the operand planes form head h, whose
// weights are rows [h WR, (h + 1) WR) of W and whose weight scales are
// w_scale[h N + n].  Within a head, only the listed 128 x 128 output tiles
// are computed (local tile id = row block * tiles_n + column block), and
// row block r reads only the K chunks set in chunk_keep[r].
constexpr int kSparseMaxTiles = 1024;
constexpr int kSparseMaxRowBlocks = 32;
struct GemmSparse {
  int64_t heads, rows_per_head, w_rows_per_head;
  int n_listed;                  // listed tiles per head (0: every tile)
  uint16_t list[kSparseMaxTiles];
  uint64_t chunk_keep[kSparseMaxRowBlocks];  // all ones: every chunk
};

// A block mask of one head's score matrix: bit c of bits[r] = block (r, c) kept.
struct BlockMask {
  uint64_t bits[kSparseMaxRowBlocks];
};

struct SliceParams {
  int64_t M, N, K;
  int lb;
  const int8_t* w_q;
  int64_t ld_w;
  const uint2* records;
  int64_t record_cap;
  const int32_t* count;
  const int8_t* bits;
  const int32_t* g_ref;
  const int32_t* planes;
  const float* w_scale;
  void* y_prev;
  int64_t ld_yp;
  void* y_out;
  int64_t ld_yo;
  int y_distinct;
  int all_tiles;  // 1: every tile; 0: only tiles that need more than two planes
  int64_t* debug_acc;
  const uint32_t* dyn_base;
  void* h_out;  // GELU(Y_t) output (nullptr = none)
  int64_t ld_h;
};

// Workspace sections (byte offsets from the workspace base).
struct WsLayout {
  size_t total, status, plane0, plane1, fpot, bits, g_ref, planes, count, mask1, records;
  int64_t mask_words, record_cap;
  size_t dyn_base;  // inside the 256-byte header that starts with the status word
};
WsLayout ws_layout(int64_t M, int64_t K);

// Launchers (return cudaError_t as int).
int launch_quantize(const QuantParams& p, int in_bf16, int num_sms, void* stream);
// First pass of the dynamic base: atomic minimum of the nonzero finite M_i
// into *out (which the caller set to all ones).
int launch_base_min(const void* x_t, const void* x_prev, int64_t ld_xt, int64_t ld_xp, int64_t M, int64_t K,
                    int in_bf16, uint32_t* out, int num_sms, void* stream);
int quantize_cluster_size(int64_t M, int64_t K, int num_sms);
// Exhaustive comparison of the dynamic-base division with __fdiv_rn (see
// dstar_fmdq_selftest_div).
int launch_div_selftest(const float* b, int n_b, int e_lo, int e_hi, unsigned long long* count, void* stream);
// Output tiles of 128 x bn in one CTA, or 256 x bn in a cluster of two CTAs
// (pair); bn = 256 only with bf16 outputs.  tiles_m counts 128-row (256 with
// pair) blocks.  The A0/A1 maps have 128-row boxes, the W map bn-row boxes
// (bn / 2 with pair).
int launch_gemm(const GemmParams& p, const void* maps /* CUtensorMap[5]: A0, A1, W, y_prev, y_out */, int bn,
                int pair, int out_bf16, int num_sms, void* stream);
// The batched, block-sparse form (fp32 outputs, 128-column tiles).
int launch_gemm_sparse(const GemmParams& p, const GemmSparse& sp, const void* maps, int num_sms, void* stream);
int launch_slice_gemm(const SliceParams& p, int out_bf16, int num_sms, void* stream);
// attention operands: per-row int8 (scale_out = scale * scale_mul), per-column
// int8 of each head's V written transposed, and the block-masked softmax
int launch_quant_rows(const void* x, int64_t ld, int64_t rows, int64_t cols, int in_bf16, int8_t* q, int64_t ldq,
                      float* scale_out, float scale_mul, void* stream);
int launch_quant_cols_t(const void* v, int64_t ld, int64_t heads, int64_t S, int64_t d, int in_bf16, int8_t* vqt,
                        float* scale, void* stream);
int launch_masked_softmax(const float* sc, float* pr, int64_t rows, int64_t S, const BlockMask& mk, void* stream);
int launch_selftest_wait(uint32_t* status, uint32_t spin_limit, void* stream);
// Fill the bf16 GELU table of the slice GEMM's activation output (enqueued on stream).
int launch_gelu_table(void* stream);
size_t quantize_smem_bytes(int64_t Kc);  // shared memory of a CTA owning Kc channels
// Raise a kernel's dynamic shared-memory limit once per device (returns a
// cudaError_t as int); later calls only look up the cache, so launches stay
// legal inside stream capture.
int ensure_max_smem(const void* func, int bytes);
size_t gemm_smem_bytes(int bn, int pair);

// Record a one-line reason for dstar_fmdq_last_error() and return `code`.
int report_error(int code, const char* msg);
int report_cuda_error(int cuda_error, const char* what);  // returns DSTAR_ERR_CUDA

}  // namespace fmdq
