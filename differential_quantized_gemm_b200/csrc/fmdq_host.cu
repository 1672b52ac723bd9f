// Host side of the C ABI declared in include/dstar_fmdq.h: argument checks,
// workspace layout, TMA descriptors and kernel launches on the caller's
// stream.  Nothing here allocates device memory.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fmdq_internal.h"

namespace fmdq {

namespace {

thread_local char g_last_error[256] = {0};

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return code;
}

int ok() {
  g_last_error[0] = 0;
  return DSTAR_OK;
}

int cuda_fail(int e, const char* what) {
  return fail(DSTAR_ERR_CUDA, "%s: %s", what, cudaGetErrorString((cudaError_t)e));
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

size_t elem_size(int dtype) { return dtype == DSTAR_F32 ? 4 : dtype == DSTAR_BF16 ? 2 : 1; }

// device properties, cached per device ordinal
struct DevInfo {
  int sms = 0;
  int major = 0, minor = 0;
  bool valid = false;
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

int device_info(DevInfo* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(DSTAR_ERR_UNSUPPORTED, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (!g_dev[dev].valid) {
    DevInfo d;
    if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute");
    d.valid = true;
    g_dev[dev] = d;
  }
  *out = g_dev[dev];
  if (out->major != 10 || out->minor != 0)
    return fail(DSTAR_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev,
                out->major, out->minor);
  return DSTAR_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda)
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D tensor map of a row-major matrix (rows x cols, row pitch ld elements)
// with a box of box_cols x box_rows elements; zero fill outside the matrix.
int make_map(CUtensorMap* map, CUtensorMapDataType dt, int es, const void* base, int64_t rows, int64_t cols,
             int64_t ld, int box_cols, int box_rows, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(DSTAR_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
  const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(DSTAR_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return DSTAR_OK;
}

// int8 operand: box of box_rows x 128 bytes, 128-byte swizzle (the MMA's K-major layout)
int make_map_i8(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  return make_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, rows, cols, ld, kChunkK, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}

// Y tiles of the epilogue: 32 x 32 elements; 64-byte rows (bf16) use the
// 64-byte swizzle, 128-byte rows (fp32) the 128-byte one
int make_map_y(CUtensorMap* map, const dstar_mat* y) {
  const bool bf = y->dtype == DSTAR_BF16;
  return make_map(map, bf ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, bf ? 2 : 4, y->data,
                  y->rows, y->cols, y->ld, 32, 32, bf ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_mat(const dstar_mat* m, const char* name, int64_t rows, int64_t cols, bool want_float) {
  if (!m) return fail(DSTAR_ERR_INVALID_ARG, "%s is NULL", name);
  if (want_float && m->dtype != DSTAR_F32 && m->dtype != DSTAR_BF16)
    return fail(DSTAR_ERR_INVALID_ARG, "%s: dtype must be F32 or BF16", name);
  if (!want_float && m->dtype != DSTAR_I8) return fail(DSTAR_ERR_INVALID_ARG, "%s: dtype must be I8", name);
  if (m->rows != rows || m->cols != cols)
    return fail(DSTAR_ERR_INVALID_ARG, "%s: shape %lldx%lld, expected %lldx%lld", name, (long long)m->rows,
                (long long)m->cols, (long long)rows, (long long)cols);
  if (rows > 0 && cols > 0) {
    if (!m->data) return fail(DSTAR_ERR_INVALID_ARG, "%s: data is NULL", name);
    if (m->ld < cols) return fail(DSTAR_ERR_INVALID_ARG, "%s: ld < cols", name);
    if (!aligned16(m->data) || (m->ld * (int64_t)elem_size(m->dtype)) % 16 != 0)
      return fail(DSTAR_ERR_INVALID_ARG, "%s: data and row pitch must be 16-byte aligned", name);
  }
  return DSTAR_OK;
}

bool overlap(const dstar_mat* a, const dstar_mat* b) {
  if (!a->data || !b->data || a->rows == 0 || b->rows == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a->data), b0 = reinterpret_cast<uintptr_t>(b->data);
  const uintptr_t a1 = a0 + (size_t)((a->rows - 1) * a->ld + a->cols) * elem_size(a->dtype);
  const uintptr_t b1 = b0 + (size_t)((b->rows - 1) * b->ld + b->cols) * elem_size(b->dtype);
  return a0 < b1 && b0 < a1;
}

int base_log2(float base, int* lb) {
  if (!(base > 0.f) || !std::isfinite(base)) return fail(DSTAR_ERR_INVALID_ARG, "base_scale must be positive and finite");
  int e;
  const float f = std::frexp(base, &e);
  if (f != 0.5f) return fail(DSTAR_ERR_INVALID_ARG, "base_scale must be an exact power of two");
  *lb = e - 1;
  if (*lb < DSTAR_BASE_LOG2_MIN || *lb > DSTAR_BASE_LOG2_MAX)
    return fail(DSTAR_ERR_INVALID_ARG, "base_scale 2^%d outside [2^%d, 2^%d]", *lb, DSTAR_BASE_LOG2_MIN,
                DSTAR_BASE_LOG2_MAX);
  return DSTAR_OK;
}

int check_cfg(const dstar_tile_cfg* c, int64_t M, int64_t K) {
  if (!c) return fail(DSTAR_ERR_INVALID_ARG, "tile_cfg is NULL");
  if (c->tile_tokens != DSTAR_TILE_TOKENS) return fail(DSTAR_ERR_INVALID_ARG, "tile_tokens must be 16");
  if (c->force_bits != 0 && c->force_bits != 2 && c->force_bits != 4 && c->force_bits != 6 && c->force_bits != 8)
    return fail(DSTAR_ERR_INVALID_ARG, "force_bits must be 0, 2, 4, 6 or 8");
  if (c->thr0_log2 < -100 || c->thr0_log2 > 100) return fail(DSTAR_ERR_INVALID_ARG, "thr0_log2 out of [-100, 100]");
  if (c->flags & ~(DSTAR_FLAG_NO_XPREV_REFRESH | DSTAR_FLAG_SLICE_PATH | DSTAR_FLAG_DYNAMIC_BASE | DSTAR_FLAG_TILE_MASK))
    return fail(DSTAR_ERR_INVALID_ARG, "unknown flag bits 0x%x", c->flags);
  if (((c->flags & DSTAR_FLAG_TILE_MASK) >> DSTAR_FLAG_TILE_SHIFT) > DSTAR_TILE_PAIR_256x128)
    return fail(DSTAR_ERR_INVALID_ARG, "unknown tile form %u", (c->flags & DSTAR_FLAG_TILE_MASK) >> DSTAR_FLAG_TILE_SHIFT);
  const WsLayout L = ws_layout(M, K);
  if (!c->workspace) return fail(DSTAR_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(c->workspace) & 255u) return fail(DSTAR_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (c->workspace_bytes < L.total)
    return fail(DSTAR_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", c->workspace_bytes, L.total);
  if ((c->debug_codes && !aligned16(c->debug_codes)) || (c->debug_acc && !aligned16(c->debug_acc)))
    return fail(DSTAR_ERR_INVALID_ARG, "debug buffers must be 16-byte aligned");
  return DSTAR_OK;
}

int check_mk(int64_t M, int64_t K) {
  if (M < 0 || M % kTile != 0) return fail(DSTAR_ERR_INVALID_ARG, "M=%lld must be a non-negative multiple of 16", (long long)M);
  if (K <= 0 || K % 32 != 0 || K > DSTAR_K_MAX)
    return fail(DSTAR_ERR_INVALID_ARG, "K=%lld must be a positive multiple of 32 up to %d", (long long)K, DSTAR_K_MAX);
  return DSTAR_OK;
}

template <typename T>
T* ws_ptr(const dstar_tile_cfg* c, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(c->workspace) + off);
}

int do_quantize(const dstar_mat* x_t, dstar_mat* x_prev, int lb, const dstar_tile_cfg* c, int64_t M, int64_t K,
                const DevInfo& dev, void* stream, const dstar_mat* pf_w = nullptr, const dstar_mat* pf_y = nullptr) {
  const WsLayout L = ws_layout(M, K);
  QuantParams q{};
  q.x_t = x_t->data;
  q.x_prev = x_prev->data;
  q.ld_xt = x_t->ld;
  q.ld_xp = x_prev->ld;
  q.M = M, q.K = K;
  q.lb = lb, q.t0 = c->thr0_log2, q.force_bits = c->force_bits, q.flags = c->flags;
  q.status = ws_ptr<uint32_t>(c, L.status);
  q.plane0 = ws_ptr<int8_t>(c, L.plane0);
  q.plane1 = ws_ptr<int8_t>(c, L.plane1);
  q.fpot = ws_ptr<int8_t>(c, L.fpot);
  q.bits = ws_ptr<int8_t>(c, L.bits);
  q.g_ref = ws_ptr<int32_t>(c, L.g_ref);
  q.planes = ws_ptr<int32_t>(c, L.planes);
  q.count = ws_ptr<int32_t>(c, L.count);
  q.mask1 = ws_ptr<uint32_t>(c, L.mask1);
  q.records = ws_ptr<uint2>(c, L.records);
  q.record_cap = L.record_cap;
  q.mask_words = L.mask_words;
  q.debug_codes = c->debug_codes;
  q.dyn_base = nullptr;
  const bool in_bf16 = x_t->dtype == DSTAR_BF16;
  if (c->flags & DSTAR_FLAG_DYNAMIC_BASE) {
    // first pass: base = min of the nonzero M_i (atomic minimum from all ones)
    q.dyn_base = ws_ptr<uint32_t>(c, L.dyn_base);
    cudaError_t ce = cudaMemsetAsync(q.dyn_base, 0xFF, sizeof(uint32_t), (cudaStream_t)stream);
    if (ce != cudaSuccess) return cuda_fail(ce, "clearing the dynamic base");
    const int e = launch_base_min(x_t->data, x_prev->data, x_t->ld, x_prev->ld, M, K, in_bf16, q.dyn_base, dev.sms,
                                  stream);
    if (e) return cuda_fail(e, "dynamic-base launch");
  }
  // L2 prefetch of the next GEMM's operands: only what stays resident until the
  // GEMM reads it (half of the 126 MB L2); a larger region would be evicted
  // before use and only add HBM traffic
  constexpr int64_t kPrefetchBudget = 64ll << 20;
  const dstar_mat* pf[2] = {pf_w, pf_y};
  int64_t budget = kPrefetchBudget;
  for (int i = 0; i < 2; ++i) {
    if (pf[i] && pf[i]->data && pf[i]->rows > 0 && pf[i]->cols > 0) {
      const int64_t es = (int64_t)elem_size(pf[i]->dtype);
      const int64_t bytes = pf[i]->rows * pf[i]->cols * es;
      if (bytes > budget) continue;
      budget -= bytes;
      q.prefetch[i] = L2Region{static_cast<const uint8_t*>(pf[i]->data), pf[i]->rows, pf[i]->cols * es,
                               pf[i]->ld * es};
    }
  }
  const int e = launch_quantize(q, in_bf16, dev.sms, stream);
  if (e) return cuda_fail(e, "quantize launch");
  return DSTAR_OK;
}

// Output tile shape from a model of one tile's period on an SM: the larger of
// its mainloop and its epilogue (the two overlap through the TMEM slots).
// Mainloop: the operand bytes in flight bound it -- with S stages of B bytes,
// S - 1 are on their way while one is consumed, and the L2 -> shared-memory
// rate an SM reaches grows with them (measured with every SM loading: about
// 45 B per clock with 96 KB in flight, 60 with 160 KB, linear between, at
// most 74) -- so a 128-deep K chunk costs the larger of its MMA cycles (the
// SM's 128 rows x BN x 128 int8 MAC at 8192 per clock) and its bytes at that
// rate.  Epilogue: about 1400 + 3000 cycles per 128 output columns of an
// SM's 128 rows (y_prev in, Y_t out, TMEM reads), in one CTA or a pair
// (fitted so that the picks match the fastest measured form of each layer of
// the DiT-XL/2, PixArt and Latte workloads).  The busiest SM's (or pair's) tile count times
// the period decides, ties to the earlier form.  Forms (stages): 128 x 128
// (6 with bf16 outputs, 5 with fp32), 128 x 256 (3), and CTA pairs 256 x 256
// (4; bf16 outputs) and 256 x 128 (8 with bf16 outputs, 6 with fp32), whose
// SMs each hold 128 rows of A and half of W.
struct TileShape {
  int bm, bn, pair;
};

// form: a DSTAR_TILE_* value, 0 for the model's choice
TileShape choose_tile(int64_t M, int64_t N, int64_t K, int sms, bool bf16, unsigned form = 0) {
  switch (form) {
    case DSTAR_TILE_128x128: return {128, 128, 0};
    case DSTAR_TILE_128x256: return bf16 ? TileShape{128, 256, 0} : TileShape{128, 128, 0};
    case DSTAR_TILE_PAIR_256x256: return bf16 ? TileShape{256, 256, 1} : TileShape{256, 128, 1};
    case DSTAR_TILE_PAIR_256x128: return {256, 128, 1};
    default: break;
  }
  auto rate = [](double in_flight) { return std::min(74.0, 45.0 + (in_flight - 96.0 * 1024) / (64.0 * 1024) * 15.0); };
  const double chunks = (double)((K + kChunkK - 1) / kChunkK);
  auto cost = [&](int64_t bn, bool pair, int stages) {
    const int64_t wrows = pair ? bn / 2 : bn;  // one SM's share of the W tile
    const double bytes = (128 + wrows) * 128.0;
    const double chunk = std::max<double>(128.0 * bn * 128.0 / 8192.0, bytes / rate((stages - 1) * bytes));
    const double epi = 1400.0 + 3000.0 * bn / 128.0;
    const int64_t bm = pair ? 256 : 128, units = pair ? sms / 2 : sms;
    const int64_t tiles = ((M + bm - 1) / bm) * ((N + bn - 1) / bn);
    return (double)((tiles + units - 1) / units) * std::max(chunks * chunk, epi);
  };
  TileShape best{128, 128, 0};
  double cb = cost(128, false, bf16 ? 6 : 5);
  auto consider = [&](TileShape t, double c) {
    if (c < cb) best = t, cb = c;
  };
  if (bf16) consider({128, 256, 0}, cost(256, false, 3));
  if (bf16) consider({256, 256, 1}, cost(256, true, 4));
  consider({256, 128, 1}, cost(128, true, bf16 ? 8 : 6));
  return best;
}

int do_gemm(const dstar_mat* w_q, const float* w_scale, dstar_mat* y_prev, int lb, const dstar_tile_cfg* c,
            dstar_mat* y_out, int64_t M, int64_t K, int64_t N, const DevInfo& dev, void* stream,
            dstar_mat* h_out = nullptr) {
  if (N == 0 || M == 0) return DSTAR_OK;
  const WsLayout L = ws_layout(M, K);
  const bool bf16 = y_prev->dtype == DSTAR_BF16;
  const bool distinct = y_out->data != y_prev->data;
  const bool slice_all = (c->flags & DSTAR_FLAG_SLICE_PATH) != 0;
  // with the dynamic base the FPoTs are relative to it: no 2^lb in the epilogue
  const bool dyn = (c->flags & DSTAR_FLAG_DYNAMIC_BASE) != 0;
  const uint32_t* dyn_base = dyn ? ws_ptr<const uint32_t>(c, L.dyn_base) : nullptr;
  if (dyn) lb = 0;
  if (!slice_all) {
    const TileShape ts = choose_tile(M, N, K, dev.sms, bf16, (c->flags & DSTAR_FLAG_TILE_MASK) >> DSTAR_FLAG_TILE_SHIFT);
    const int bn = ts.bn;
    CUtensorMap maps[5];  // A0, A1, W, y_prev, y_out
    int r;
    if ((r = make_map_i8(&maps[0], ws_ptr<void>(c, L.plane0), M, K, K, kBlockM)) != DSTAR_OK) return r;
    if ((r = make_map_i8(&maps[1], ws_ptr<void>(c, L.plane1), M, K, K, kBlockM)) != DSTAR_OK) return r;
    if ((r = make_map_i8(&maps[2], w_q->data, N, K, w_q->ld, ts.pair ? bn / 2 : bn)) != DSTAR_OK) return r;
    if ((r = make_map_y(&maps[3], y_prev)) != DSTAR_OK) return r;
    if ((r = make_map_y(&maps[4], y_out)) != DSTAR_OK) return r;
    GemmParams g{};
    g.M = M, g.N = N, g.K = K;
    g.lb = lb;
    g.flags = c->flags;
    g.g_ref = ws_ptr<int32_t>(c, L.g_ref);
    g.planes = ws_ptr<int32_t>(c, L.planes);
    g.mask1 = ws_ptr<uint32_t>(c, L.mask1);
    g.mask_words = L.mask_words;
    g.w_scale = w_scale;
    g.y_prev = y_prev->data;
    g.ld_yp = y_prev->ld;
    g.y_out = y_out->data;
    g.ld_yo = y_out->ld;
    g.y_distinct = distinct;
    g.status = ws_ptr<uint32_t>(c, L.status);
    g.debug_acc = c->debug_acc;
    g.dyn_base = dyn_base;
    g.h_out = h_out ? h_out->data : nullptr;
    g.ld_h = h_out ? h_out->ld : 0;
    g.tiles_m = (int)((M + ts.bm - 1) / ts.bm);
    g.tiles_n = (int)((N + bn - 1) / bn);
    g.num_chunks = (int)((K + kChunkK - 1) / kChunkK);
    g.w_q = static_cast<const int8_t*>(w_q->data);
    g.ld_w = w_q->ld;
    g.records = ws_ptr<const uint2>(c, L.records);
    g.record_cap = L.record_cap;
    g.count = ws_ptr<const int32_t>(c, L.count);
    g.bits = ws_ptr<const int8_t>(c, L.bits);
    const int e = launch_gemm(g, maps, bn, ts.pair, bf16, dev.sms, stream);
    if (e) return cuda_fail(e, "slice-GEMM launch");
    return DSTAR_OK;  // tiles needing the slice stream are handled inside the GEMM kernel
  }
  SliceParams s{};
  s.M = M, s.N = N, s.K = K;
  s.lb = lb;
  s.w_q = static_cast<const int8_t*>(w_q->data);
  s.ld_w = w_q->ld;
  s.records = ws_ptr<const uint2>(c, L.records);
  s.record_cap = L.record_cap;
  s.count = ws_ptr<const int32_t>(c, L.count);
  s.bits = ws_ptr<const int8_t>(c, L.bits);
  s.g_ref = ws_ptr<const int32_t>(c, L.g_ref);
  s.planes = ws_ptr<const int32_t>(c, L.planes);
  s.w_scale = w_scale;
  s.y_prev = y_prev->data;
  s.ld_yp = y_prev->ld;
  s.y_out = y_out->data;
  s.ld_yo = y_out->ld;
  s.y_distinct = distinct;
  s.all_tiles = 1;
  s.debug_acc = c->debug_acc;
  s.dyn_base = dyn_base;
  s.h_out = h_out ? h_out->data : nullptr;
  s.ld_h = h_out ? h_out->ld : 0;
  const int e = launch_slice_gemm(s, bf16, dev.sms, stream);
  if (e) return cuda_fail(e, "slice-stream launch");
  return DSTAR_OK;
}

int check_gemm_args(const dstar_mat* w_q, const float* w_scale, dstar_mat* y_prev, dstar_mat* y_out, int64_t M,
                    int64_t K, int64_t* N_out) {
  if (!w_q) return fail(DSTAR_ERR_INVALID_ARG, "w_q is NULL");
  const int64_t N = w_q->rows;
  if (N < 0 || N % 16 != 0) return fail(DSTAR_ERR_INVALID_ARG, "N=%lld must be a non-negative multiple of 16", (long long)N);
  int r;
  if ((r = check_mat(w_q, "w_q", N, K, false)) != DSTAR_OK) return r;
  if ((r = check_mat(y_prev, "y_prev", M, N, true)) != DSTAR_OK) return r;
  if ((r = check_mat(y_out, "y_out", M, N, true)) != DSTAR_OK) return r;
  if (y_out->dtype != y_prev->dtype) return fail(DSTAR_ERR_INVALID_ARG, "y_out and y_prev must share a dtype");
  if (N > 0 && M > 0) {
    if (!w_scale) return fail(DSTAR_ERR_INVALID_ARG, "w_scale is NULL");
    if (reinterpret_cast<uintptr_t>(w_scale) & 3u) return fail(DSTAR_ERR_INVALID_ARG, "w_scale must be 4-byte aligned");
    const bool same = y_out->data == y_prev->data && y_out->ld == y_prev->ld;
    if (!same && overlap(y_out, y_prev)) return fail(DSTAR_ERR_INVALID_ARG, "y_out partially overlaps y_prev");
  }
  *N_out = N;
  return DSTAR_OK;
}

// ------------------------------------------------------------ attention

struct SarLayout {
  size_t total, ws_p, ws_q, kq, ks, vqt, vs, scores, probs;
};

SarLayout sar_layout(int64_t G, int64_t S, int64_t d) {
  SarLayout L{};
  const int64_t R = G * S;
  size_t o = 0;
  L.ws_p = o, o = align256(o + ws_layout(R, S).total);
  L.ws_q = o, o = align256(o + ws_layout(R, d).total);
  L.kq = o, o = align256(o + (size_t)(R * d));
  L.ks = o, o = align256(o + (size_t)R * 4);
  L.vqt = o, o = align256(o + (size_t)(G * d * S));
  L.vs = o, o = align256(o + (size_t)(G * d) * 4);
  L.scores = o, o = align256(o + (size_t)(R * S) * 4);
  L.probs = o, o = align256(o + (size_t)(R * S) * 4);
  L.total = o;
  return L;
}

int check_sar_sizes(int64_t G, int64_t S, int64_t d) {
  if (G <= 0) return fail(DSTAR_ERR_INVALID_ARG, "heads must be positive");
  if (S <= 0 || S % DSTAR_SAR_BLOCK != 0 || S / DSTAR_SAR_BLOCK > kSparseMaxRowBlocks)
    return fail(DSTAR_ERR_INVALID_ARG, "seq must be a positive multiple of %d up to %d", DSTAR_SAR_BLOCK,
                DSTAR_SAR_BLOCK * kSparseMaxRowBlocks);
  if (d <= 0 || d % 32 != 0 || d > DSTAR_K_MAX)
    return fail(DSTAR_ERR_INVALID_ARG, "head_dim must be a positive multiple of 32 up to %d", DSTAR_K_MAX);
  return DSTAR_OK;
}

// One FMDQ workspace inside the attention workspace, as a tile_cfg with every width 8.
dstar_tile_cfg sar_cfg_of(void* base, size_t off, int64_t M, int64_t K) {
  dstar_tile_cfg c{};
  c.tile_tokens = DSTAR_TILE_TOKENS;
  c.force_bits = 8;
  c.workspace = static_cast<uint8_t*>(base) + off;
  c.workspace_bytes = ws_layout(M, K).total;
  return c;
}

// The batched, block-sparse slice GEMM: operand planes of the FMDQ workspace
// `c` (R rows, K columns), weights w [w_rows x K] (head h's rows start at h *
// sp.w_rows_per_head), y [R x N] fp32 (Y_{t-1} = 0, not read).
int do_gemm_sparse(const dstar_tile_cfg* c, int64_t R, int64_t K, const int8_t* w, int64_t w_rows, int64_t ldw,
                   const float* w_scale, float* y, int64_t N, int64_t ldy, int lb, const GemmSparse& sp,
                   const DevInfo& dev, void* stream) {
  const WsLayout L = ws_layout(R, K);
  CUtensorMap maps[5];
  dstar_mat ym{y, DSTAR_F32, 0, R, N, ldy};
  int r;
  if ((r = make_map_i8(&maps[0], ws_ptr<void>(c, L.plane0), R, K, K, kBlockM)) != DSTAR_OK) return r;
  if ((r = make_map_i8(&maps[1], ws_ptr<void>(c, L.plane1), R, K, K, kBlockM)) != DSTAR_OK) return r;
  if ((r = make_map_i8(&maps[2], w, w_rows, K, ldw, 128)) != DSTAR_OK) return r;
  if ((r = make_map_y(&maps[3], &ym)) != DSTAR_OK) return r;
  if ((r = make_map_y(&maps[4], &ym)) != DSTAR_OK) return r;
  GemmParams g{};
  g.M = R, g.N = N, g.K = K;
  g.lb = lb;
  g.g_ref = ws_ptr<int32_t>(c, L.g_ref);
  g.planes = ws_ptr<int32_t>(c, L.planes);
  g.mask1 = ws_ptr<uint32_t>(c, L.mask1);
  g.mask_words = L.mask_words;
  g.w_scale = w_scale;
  g.y_prev = y, g.ld_yp = ldy, g.y_out = y, g.ld_yo = ldy;
  g.status = ws_ptr<uint32_t>(c, L.status);
  g.tiles_m = (int)(R / kBlockM);
  g.tiles_n = (int)((N + 127) / 128);
  g.num_chunks = (int)((K + kChunkK - 1) / kChunkK);
  g.w_q = w;
  g.ld_w = ldw;
  g.records = ws_ptr<const uint2>(c, L.records);
  g.record_cap = L.record_cap;
  g.count = ws_ptr<const int32_t>(c, L.count);
  g.bits = ws_ptr<const int8_t>(c, L.bits);
  const int e = launch_gemm_sparse(g, sp, maps, dev.sms, stream);
  if (e) return cuda_fail(e, "sparse slice-GEMM launch");
  return DSTAR_OK;
}

// The bf16 GELU table of the slice GEMM is filled once per CUDA context (a
// device reset or a new context loads the module again), before the first
// GEMM that reads it, on that GEMM's stream.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
std::mutex g_gelu_mu;
unsigned long long g_gelu_ctx[64] = {};
int g_gelu_n = 0, g_gelu_next = 0;

int ensure_gelu_table(void* stream) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
    return fail(DSTAR_ERR_CUDA, "cannot identify the current CUDA context");
  std::lock_guard<std::mutex> lk(g_gelu_mu);
  for (int i = 0; i < g_gelu_n; ++i)
    if (g_gelu_ctx[i] == id) return DSTAR_OK;
  const int e = launch_gelu_table(stream);
  if (e) return cuda_fail(e, "GELU table launch");
  g_gelu_ctx[g_gelu_next] = id;
  g_gelu_next = (g_gelu_next + 1) % 64;
  if (g_gelu_n < 64) ++g_gelu_n;
  return DSTAR_OK;
}

std::mutex g_attr_mu;
struct AttrEntry {
  int dev;
  const void* func;
  int bytes;
};
AttrEntry g_attr[64];
int g_nattr = 0;

}  // namespace

int ensure_max_smem(const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  std::lock_guard<std::mutex> lk(g_attr_mu);
  for (int i = 0; i < g_nattr; ++i)
    if (g_attr[i].dev == dev && g_attr[i].func == func && g_attr[i].bytes >= bytes) return 0;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return (int)e;
  for (int i = 0; i < g_nattr; ++i)
    if (g_attr[i].dev == dev && g_attr[i].func == func) {
      g_attr[i].bytes = bytes;
      return 0;
    }
  if (g_nattr < 64) g_attr[g_nattr++] = AttrEntry{dev, func, bytes};
  return 0;
}

int report_error(int code, const char* msg) { return fail(code, "%s", msg); }
int report_cuda_error(int cuda_error, const char* what) { return cuda_fail(cuda_error, what); }

WsLayout ws_layout(int64_t M, int64_t K) {
  WsLayout L{};
  const int64_t T = M / kTile;
  const int64_t chunks = (K + kChunkK - 1) / kChunkK;
  L.mask_words = (chunks + 31) / 32;
  L.record_cap = 4 * K;
  size_t o = 0;
  L.status = o, o = align256(o + 256);
  L.dyn_base = L.status + 16;
  L.plane0 = o, o = align256(o + (size_t)(M * K));
  L.plane1 = o, o = align256(o + (size_t)(M * K));
  L.fpot = o, o = align256(o + (size_t)(T * K));
  L.bits = o, o = align256(o + (size_t)(T * K));
  L.g_ref = o, o = align256(o + (size_t)T * 4);
  L.planes = o, o = align256(o + (size_t)T * 4);
  L.count = o, o = align256(o + (size_t)T * 4);
  L.mask1 = o, o = align256(o + (size_t)(T * L.mask_words) * 4);
  L.records = o, o = align256(o + (size_t)(T * L.record_cap) * 8);
  L.total = o;
  return L;
}

}  // namespace fmdq

using namespace fmdq;

extern "C" {

int dstar_fmdq_version(void) { return DSTAR_FMDQ_VERSION; }

const char* dstar_fmdq_error_string(int code) {
  switch (code) {
    case DSTAR_OK: return "ok";
    case DSTAR_ERR_INVALID_ARG: return "invalid argument";
    case DSTAR_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DSTAR_ERR_CUDA: return "CUDA error";
    case DSTAR_ERR_UNSUPPORTED: return "unsupported device";
    default: return "unknown error";
  }
}

const char* dstar_fmdq_last_error(void) { return g_last_error; }

int dstar_fmdq_workspace_size(int64_t M, int64_t K, size_t* bytes) {
  if (!bytes) return fail(DSTAR_ERR_INVALID_ARG, "bytes is NULL");
  if (M < 0 || K < 0 || K > DSTAR_K_MAX) return fail(DSTAR_ERR_INVALID_ARG, "bad M or K");
  *bytes = ws_layout(M, K).total;
  return ok();
}

int dstar_fmdq_workspace_layout(int64_t M, int64_t K, dstar_fmdq_ws_layout* out) {
  if (!out) return fail(DSTAR_ERR_INVALID_ARG, "out is NULL");
  if (M < 0 || K < 0 || K > DSTAR_K_MAX) return fail(DSTAR_ERR_INVALID_ARG, "bad M or K");
  const WsLayout L = ws_layout(M, K);
  out->total = L.total;
  out->status = L.status;
  out->plane0 = L.plane0;
  out->plane1 = L.plane1;
  out->fpot = L.fpot;
  out->bits = L.bits;
  out->g_ref = L.g_ref;
  out->planes = L.planes;
  out->count = L.count;
  out->mask1 = L.mask1;
  out->records = L.records;
  out->mask_words = L.mask_words;
  out->record_cap = L.record_cap;
  out->dyn_base = L.dyn_base;
  return ok();
}

int dstar_fmdq_workspace_init(void* workspace, size_t bytes, void* stream) {
  if (!workspace || bytes < 256) return fail(DSTAR_ERR_WORKSPACE, "workspace is NULL or smaller than 256 bytes");
  const cudaError_t e = cudaMemsetAsync(workspace, 0, 256, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  return ok();
}

int dstar_fmdq_quantize(const dstar_mat* x_t, dstar_mat* x_prev, float base_scale, const dstar_tile_cfg* tile_cfg,
                        void* stream) {
  int r;
  if (!x_t || !x_prev) return fail(DSTAR_ERR_INVALID_ARG, "x_t or x_prev is NULL");
  const int64_t M = x_t->rows, K = x_t->cols;
  if ((r = check_mk(M, K)) != DSTAR_OK) return r;
  if ((r = check_mat(x_t, "x_t", M, K, true)) != DSTAR_OK) return r;
  if ((r = check_mat(x_prev, "x_prev", M, K, true)) != DSTAR_OK) return r;
  if (x_t->dtype != x_prev->dtype) return fail(DSTAR_ERR_INVALID_ARG, "x_t and x_prev must share a dtype");
  if (!(x_t->data == x_prev->data && x_t->ld == x_prev->ld) && overlap(x_t, x_prev))
    return fail(DSTAR_ERR_INVALID_ARG, "x_t partially overlaps x_prev");
  int lb = 0;
  if ((r = base_log2(base_scale, &lb)) != DSTAR_OK) return r;
  if ((r = check_cfg(tile_cfg, M, K)) != DSTAR_OK) return r;
  if (M == 0) return ok();
  DevInfo dev;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  if ((r = do_quantize(x_t, x_prev, lb, tile_cfg, M, K, dev, stream)) != DSTAR_OK) return r;
  return ok();
}

int dstar_fmdq_slice_gemm(const dstar_mat* w_q, const float* w_scale, dstar_mat* y_prev, float base_scale,
                          const dstar_tile_cfg* tile_cfg, dstar_mat* y_out, void* stream) {
  int r;
  if (!w_q || !y_prev) return fail(DSTAR_ERR_INVALID_ARG, "w_q or y_prev is NULL");
  const int64_t M = y_prev->rows, K = w_q->cols;
  if ((r = check_mk(M, K)) != DSTAR_OK) return r;
  int64_t N = 0;
  if ((r = check_gemm_args(w_q, w_scale, y_prev, y_out, M, K, &N)) != DSTAR_OK) return r;
  int lb = 0;
  if ((r = base_log2(base_scale, &lb)) != DSTAR_OK) return r;
  if ((r = check_cfg(tile_cfg, M, K)) != DSTAR_OK) return r;
  if (M == 0 || N == 0) return ok();
  DevInfo dev;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  if ((r = do_gemm(w_q, w_scale, y_prev, lb, tile_cfg, y_out, M, K, N, dev, stream)) != DSTAR_OK) return r;
  return ok();
}

int dstar_fmdq_linear(const dstar_mat* x_t, dstar_mat* x_prev, dstar_mat* y_prev, const dstar_mat* w_q,
                      const float* w_scale, float base_scale, const dstar_tile_cfg* tile_cfg, dstar_mat* y_out,
                      void* stream) {
  int r;
  if (!x_t || !x_prev) return fail(DSTAR_ERR_INVALID_ARG, "x_t or x_prev is NULL");
  const int64_t M = x_t->rows, K = x_t->cols;
  if ((r = check_mk(M, K)) != DSTAR_OK) return r;
  if ((r = check_mat(x_t, "x_t", M, K, true)) != DSTAR_OK) return r;
  if ((r = check_mat(x_prev, "x_prev", M, K, true)) != DSTAR_OK) return r;
  if (x_t->dtype != x_prev->dtype) return fail(DSTAR_ERR_INVALID_ARG, "x_t and x_prev must share a dtype");
  if (!(x_t->data == x_prev->data && x_t->ld == x_prev->ld) && overlap(x_t, x_prev))
    return fail(DSTAR_ERR_INVALID_ARG, "x_t partially overlaps x_prev");
  int64_t N = 0;
  if ((r = check_gemm_args(w_q, w_scale, y_prev, y_out, M, K, &N)) != DSTAR_OK) return r;
  int lb = 0;
  if ((r = base_log2(base_scale, &lb)) != DSTAR_OK) return r;
  if ((r = check_cfg(tile_cfg, M, K)) != DSTAR_OK) return r;
  if (M == 0) return ok();
  DevInfo dev;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  if ((r = do_quantize(x_t, x_prev, lb, tile_cfg, M, K, dev, stream, N > 0 ? w_q : nullptr,
                       N > 0 ? y_prev : nullptr)) != DSTAR_OK)
    return r;
  if ((r = do_gemm(w_q, w_scale, y_prev, lb, tile_cfg, y_out, M, K, N, dev, stream)) != DSTAR_OK) return r;
  return ok();
}

int dstar_fmdq_ffn_gelu(const dstar_mat* x_t, dstar_mat* x_prev, dstar_mat* y1_prev, const dstar_mat* w1,
                        const float* w1_scale, dstar_mat* h_t, dstar_mat* h_prev, dstar_mat* y2_prev,
                        const dstar_mat* w2, const float* w2_scale, float base_scale, const dstar_tile_cfg* cfg1,
                        const dstar_tile_cfg* cfg2, void* stream) {
  int r;
  if (!x_t || !x_prev || !w1 || !w2 || !h_t || !h_prev || !y1_prev || !y2_prev)
    return fail(DSTAR_ERR_INVALID_ARG, "a matrix argument is NULL");
  const int64_t M = x_t->rows, K1 = x_t->cols, N1 = w1->rows;
  // layer 1: X (M x K1) -> Y1 (M x N1); its GELU output H is layer 2's input (K2 = N1)
  if ((r = check_mk(M, K1)) != DSTAR_OK) return r;
  if ((r = check_mat(x_t, "x_t", M, K1, true)) != DSTAR_OK) return r;
  if ((r = check_mat(x_prev, "x_prev", M, K1, true)) != DSTAR_OK) return r;
  if (x_t->dtype != x_prev->dtype) return fail(DSTAR_ERR_INVALID_ARG, "x_t and x_prev must share a dtype");
  if (!(x_t->data == x_prev->data && x_t->ld == x_prev->ld) && overlap(x_t, x_prev))
    return fail(DSTAR_ERR_INVALID_ARG, "x_t partially overlaps x_prev");
  int64_t n1 = 0, n2 = 0;
  if ((r = check_gemm_args(w1, w1_scale, y1_prev, y1_prev, M, K1, &n1)) != DSTAR_OK) return r;
  if (N1 <= 0 || N1 % 32 != 0 || N1 > DSTAR_K_MAX)
    return fail(DSTAR_ERR_INVALID_ARG, "N1=%lld (layer 2's K) must be a positive multiple of 32 up to %d",
                (long long)N1, DSTAR_K_MAX);
  if ((r = check_mat(h_t, "h_t", M, N1, true)) != DSTAR_OK) return r;
  if ((r = check_mat(h_prev, "h_prev", M, N1, true)) != DSTAR_OK) return r;
  if (h_t->dtype != y1_prev->dtype || h_prev->dtype != y1_prev->dtype)
    return fail(DSTAR_ERR_INVALID_ARG, "h_t and h_prev must have y1_prev's dtype");
  if (overlap(h_t, h_prev) || overlap(h_t, y1_prev) || overlap(h_prev, y1_prev))
    return fail(DSTAR_ERR_INVALID_ARG, "h_t, h_prev and y1_prev must be disjoint");
  if ((r = check_gemm_args(w2, w2_scale, y2_prev, y2_prev, M, N1, &n2)) != DSTAR_OK) return r;
  if (overlap(y2_prev, h_t) || overlap(y2_prev, h_prev) || overlap(y2_prev, y1_prev))
    return fail(DSTAR_ERR_INVALID_ARG, "y2_prev overlaps another buffer of the pair");
  int lb = 0;
  if ((r = base_log2(base_scale, &lb)) != DSTAR_OK) return r;
  if ((r = check_cfg(cfg1, M, K1)) != DSTAR_OK) return r;
  if ((r = check_cfg(cfg2, M, N1)) != DSTAR_OK) return r;
  if (cfg1->workspace == cfg2->workspace) return fail(DSTAR_ERR_WORKSPACE, "the two layers need two workspaces");
  if (M == 0) return ok();
  DevInfo dev;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  // layer 1, its epilogue also writing H_t = GELU(Y1_t)
  if (h_t->dtype == DSTAR_BF16 && (r = ensure_gelu_table(stream)) != DSTAR_OK) return r;
  if ((r = do_quantize(x_t, x_prev, lb, cfg1, M, K1, dev, stream, w1, y1_prev)) != DSTAR_OK) return r;
  if ((r = do_gemm(w1, w1_scale, y1_prev, lb, cfg1, y1_prev, M, K1, N1, dev, stream, h_t)) != DSTAR_OK) return r;
  // layer 2 on the differential H_t - H_{t-1}
  if ((r = do_quantize(h_t, h_prev, lb, cfg2, M, N1, dev, stream, n2 > 0 ? w2 : nullptr,
                       n2 > 0 ? y2_prev : nullptr)) != DSTAR_OK)
    return r;
  if ((r = do_gemm(w2, w2_scale, y2_prev, lb, cfg2, y2_prev, M, N1, n2, dev, stream)) != DSTAR_OK) return r;
  return ok();
}

int dstar_sar_workspace_size(int64_t heads, int64_t seq, int64_t head_dim, size_t* bytes) {
  if (!bytes) return fail(DSTAR_ERR_INVALID_ARG, "bytes is NULL");
  int r;
  if ((r = check_sar_sizes(heads, seq, head_dim)) != DSTAR_OK) return r;
  *bytes = sar_layout(heads, seq, head_dim).total;
  return ok();
}

int dstar_sar_workspace_layout(int64_t heads, int64_t seq, int64_t head_dim, dstar_sar_layout* out) {
  if (!out) return fail(DSTAR_ERR_INVALID_ARG, "out is NULL");
  int r;
  if ((r = check_sar_sizes(heads, seq, head_dim)) != DSTAR_OK) return r;
  const SarLayout L = sar_layout(heads, seq, head_dim);
  *out = dstar_sar_layout{L.total, L.ws_p, L.ws_q, L.kq, L.ks, L.vqt, L.vs, L.scores, L.probs};
  return ok();
}

namespace {
int check_sar_cfg(const dstar_sar_cfg* cfg, SarLayout* L) {
  if (!cfg) return fail(DSTAR_ERR_INVALID_ARG, "cfg is NULL");
  int r;
  if ((r = check_sar_sizes(cfg->heads, cfg->seq, cfg->head_dim)) != DSTAR_OK) return r;
  *L = sar_layout(cfg->heads, cfg->seq, cfg->head_dim);
  if (!cfg->workspace) return fail(DSTAR_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(cfg->workspace) & 255u) return fail(DSTAR_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (cfg->workspace_bytes < L->total)
    return fail(DSTAR_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", cfg->workspace_bytes, L->total);
  return DSTAR_OK;
}
}  // namespace

int dstar_sar_workspace_init(const dstar_sar_cfg* cfg, void* stream) {
  SarLayout L;
  int r;
  if ((r = check_sar_cfg(cfg, &L)) != DSTAR_OK) return r;
  uint8_t* base = static_cast<uint8_t*>(cfg->workspace);
  cudaError_t e = cudaMemsetAsync(base + L.ws_p, 0, 256, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(base + L.ws_q, 0, 256, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  return ok();
}

int dstar_sar_attention(const dstar_mat* q, const dstar_mat* k, const dstar_mat* v, const dstar_sar_cfg* cfg,
                        int reuse, dstar_mat* out, void* stream) {
  SarLayout L;
  int r;
  if ((r = check_sar_cfg(cfg, &L)) != DSTAR_OK) return r;
  const int64_t G = cfg->heads, S = cfg->seq, d = cfg->head_dim, R = G * S, nb = S / DSTAR_SAR_BLOCK;
  if (!q || !k || !v || !out) return fail(DSTAR_ERR_INVALID_ARG, "q, k, v or out is NULL");
  if (!reuse) {
    if ((r = check_mat(q, "q", R, d, true)) != DSTAR_OK) return r;
    if ((r = check_mat(k, "k", R, d, true)) != DSTAR_OK) return r;
    if (k->dtype != q->dtype) return fail(DSTAR_ERR_INVALID_ARG, "q and k must share a dtype");
  }
  if ((r = check_mat(v, "v", R, d, true)) != DSTAR_OK) return r;
  if ((r = check_mat(out, "out", R, d, true)) != DSTAR_OK) return r;
  if (out->dtype != DSTAR_F32) return fail(DSTAR_ERR_INVALID_ARG, "out must be F32");
  if (!cfg->block_mask) return fail(DSTAR_ERR_INVALID_ARG, "block_mask is NULL");
  if (!(cfg->scores_scale > 0.f) || !std::isfinite(cfg->scores_scale))
    return fail(DSTAR_ERR_INVALID_ARG, "scores_scale must be positive and finite");
  int lb_q = 0, lb_p = 0;
  if ((r = base_log2(cfg->base_q, &lb_q)) != DSTAR_OK) return r;
  if ((r = base_log2(cfg->base_p, &lb_p)) != DSTAR_OK) return r;
  // the mask: per row block, the kept key blocks; the listed score tiles
  GemmSparse sp_s{}, sp_o{};
  BlockMask mk{};
  int listed = 0;
  for (int64_t a = 0; a < nb; ++a) {
    for (int64_t b = 0; b < nb; ++b)
      if (cfg->block_mask[a * nb + b]) {
        mk.bits[a] |= 1ull << b;
        sp_s.list[listed++] = (uint16_t)(a * nb + b);
      }
    if (!mk.bits[a]) return fail(DSTAR_ERR_INVALID_ARG, "block_mask row %lld keeps no block", (long long)a);
  }
  sp_s.heads = sp_o.heads = G;
  sp_s.rows_per_head = sp_o.rows_per_head = S;
  sp_s.w_rows_per_head = S, sp_o.w_rows_per_head = d;
  sp_s.n_listed = listed == nb * nb ? 0 : listed;
  sp_o.n_listed = 0;
  for (int64_t a = 0; a < kSparseMaxRowBlocks; ++a) sp_s.chunk_keep[a] = ~0ull, sp_o.chunk_keep[a] = a < nb ? mk.bits[a] : 0;
  DevInfo dev;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  uint8_t* base = static_cast<uint8_t*>(cfg->workspace);
  const dstar_tile_cfg cp = sar_cfg_of(base, L.ws_p, R, S);
  const dstar_mat none{nullptr, q ? q->dtype : DSTAR_F32, 0, R, d, d};  // X_{t-1} = 0: the operands themselves
  int e;
  if (!reuse) {
    const dstar_tile_cfg cq = sar_cfg_of(base, L.ws_q, R, d);
    e = launch_quant_rows(k->data, k->ld, R, d, k->dtype == DSTAR_BF16, reinterpret_cast<int8_t*>(base + L.kq), d,
                          reinterpret_cast<float*>(base + L.ks), cfg->scores_scale, stream);
    if (e) return cuda_fail(e, "key quantization launch");
    dstar_mat none_q = none;
    if ((r = do_quantize(q, &none_q, lb_q, &cq, R, d, dev, stream)) != DSTAR_OK) return r;
    if ((r = do_gemm_sparse(&cq, R, d, reinterpret_cast<const int8_t*>(base + L.kq), R, d,
                            reinterpret_cast<const float*>(base + L.ks), reinterpret_cast<float*>(base + L.scores), S,
                            S, lb_q, sp_s, dev, stream)) != DSTAR_OK)
      return r;
    e = launch_masked_softmax(reinterpret_cast<const float*>(base + L.scores), reinterpret_cast<float*>(base + L.probs),
                              R, S, mk, stream);
    if (e) return cuda_fail(e, "softmax launch");
    const dstar_mat pm{base + L.probs, DSTAR_F32, 0, R, S, S};
    dstar_mat none_p{nullptr, DSTAR_F32, 0, R, S, S};
    if ((r = do_quantize(&pm, &none_p, lb_p, &cp, R, S, dev, stream)) != DSTAR_OK) return r;
  }
  e = launch_quant_cols_t(v->data, v->ld, G, S, d, v->dtype == DSTAR_BF16, reinterpret_cast<int8_t*>(base + L.vqt),
                          reinterpret_cast<float*>(base + L.vs), stream);
  if (e) return cuda_fail(e, "value quantization launch");
  if ((r = do_gemm_sparse(&cp, R, S, reinterpret_cast<const int8_t*>(base + L.vqt), G * d, S,
                          reinterpret_cast<const float*>(base + L.vs), static_cast<float*>(out->data), d, out->ld,
                          lb_p, sp_o, dev, stream)) != DSTAR_OK)
    return r;
  return ok();
}

int dstar_sar_status(const dstar_sar_cfg* cfg, void* stream, uint32_t* status) {
  SarLayout L;
  int r;
  if (!status) return fail(DSTAR_ERR_INVALID_ARG, "status is NULL");
  if ((r = check_sar_cfg(cfg, &L)) != DSTAR_OK) return r;
  uint32_t a = 0, b = 0;
  uint8_t* base = static_cast<uint8_t*>(cfg->workspace);
  if ((r = dstar_fmdq_status(base + L.ws_p, stream, &a)) != DSTAR_OK) return r;
  if ((r = dstar_fmdq_status(base + L.ws_q, stream, &b)) != DSTAR_OK) return r;
  *status = a | b;
  return ok();
}

int dstar_fmdq_status(void* workspace, void* stream, uint32_t* status) {
  if (!workspace || !status) return fail(DSTAR_ERR_INVALID_ARG, "workspace or status is NULL");
  cudaError_t e = cudaMemcpyAsync(status, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  return ok();
}

int dstar_fmdq_gemm_tile(int64_t M, int64_t N, int64_t K, int out_bf16, int* bm, int* bn, int* pair) {
  if (!bm || !bn) return fail(DSTAR_ERR_INVALID_ARG, "bm and bn must not be NULL");
  if (M < 0 || N < 0 || K < 0) return fail(DSTAR_ERR_INVALID_ARG, "negative size");
  DevInfo dev;
  int r;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  const TileShape ts = choose_tile(M, N, K, dev.sms, out_bf16 != 0);
  *bm = ts.bm, *bn = ts.bn;
  if (pair) *pair = ts.pair;
  return ok();
}

int dstar_fmdq_selftest_div(const float* b, int n_b, int e_lo, int e_hi, unsigned long long* count, void* stream) {
  if (!b || !count) return fail(DSTAR_ERR_INVALID_ARG, "b and count must not be NULL");
  if (n_b < 0 || e_lo <= -127 || e_hi >= 128 || e_hi < e_lo) return fail(DSTAR_ERR_INVALID_ARG, "bad divisor count or exponents");
  DevInfo dev;
  int r;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  const int e = launch_div_selftest(b, n_b, e_lo, e_hi, count, stream);
  if (e) return cuda_fail(e, "division self-test launch");
  return ok();
}

int dstar_fmdq_selftest_wait(void* workspace, uint32_t limit_us, void* stream) {
  if (!workspace) return fail(DSTAR_ERR_WORKSPACE, "workspace is NULL");
  DevInfo dev;
  int r;
  if ((r = device_info(&dev)) != DSTAR_OK) return r;
  const int e = launch_selftest_wait(static_cast<uint32_t*>(workspace), limit_us, stream);
  if (e) return cuda_fail(e, "self-test launch");
  return ok();
}

}  // extern "C"
