// K2+K3: the shift-aligned slice GEMM on tcgen05 tensor cores with the fused
// dequantize / reverse-differential epilogue (DSTAR section 3.1 step 5,
// section 4.2 "Design of MPU" inverse quantization and accumulation units,
// section 4.3 "Operator Mapping": cached outputs added to the partial sum).
//
// The paper's MPU streams 2-bit slices in ascending FPoT order and shifts the
// partial sum by the FPoT difference between groups.  Here every shift is
// folded into the operand before the contraction: slice j of channel k in
// tile T enters with weight 2^(g_ref(T) - FPoT(T,k) + 2j), so the sum of a
// channel's slices is v = q * 2^(g_ref - FPoT), an exact integer that the
// quantizer splits into int8 planes v = A0 + 256 A1.  The tensor cores then
// compute D_p = A_p W^T (int8 x int8 -> int32, exact), and the epilogue forms
// acc = D_0 + 256 D_1 in 64-bit integers -- bit for bit the accumulator that
// ascending-FPoT shift-and-add produces -- then
//   Y_t = Y_{t-1} + ((float)acc * 2^(-lb - g_ref)) * w_scale[n]   (fp32, in this order).
//
// Structure (one CTA per SM, persistent over 128 x BN output tiles; or, with
// PAIR, one cluster of two CTAs per two SMs over 256 x BN tiles, each CTA
// owning 128 rows):
//   warp 0      TMA producer: per K chunk, a 128 x 128-byte tile of the operand
//               plane and a BN x 128-byte tile of W (BN / 2 rows with PAIR);
//               blocks that need the second plane run a second K pass over
//               the chunks where it is nonzero
//   warp 1      TMEM allocator and MMA issuer (one thread; the even CTA's with
//               PAIR): M=128 (256 with PAIR), N=BN, K=32
//   warps 2..9  epilogue, two warps per 32 TMEM lanes (rows), each half of the
//               columns: TMA-load of its 32 x 32 tiles of y_prev into shared
//               memory (issued before the accumulator is ready), tcgen05.ld,
//               fp32 epilogue written in place, TMA-store of Y_t to y_out (and
//               y_prev when distinct)
// TMEM holds 512 columns = 512/BN accumulator slots; a one-plane tile takes one
// slot, a two-plane tile two, so the epilogue of one tile overlaps the MMAs
// of the next.  Tiles whose operands need more than two int8 planes are
// computed by the epilogue warps along the slice stream.  Every wait is
// bounded (wait_parity).  The host picks BN and PAIR per call from a model of
// the mainloop and the epilogue (choose_tile in fmdq_host.cu).
#include <cuda_bf16.h>

#include "fmdq_device.cuh"

namespace fmdq {

namespace {

constexpr int kEpiWarps = 8;                       // two per TMEM lane quarter, each half the columns
constexpr int kGThreads = 64 + 32 * kEpiWarps;     // producer warp, MMA warp, epilogue warps
constexpr int kA0Bytes = kBlockM * kChunkK;        // 16 KB
constexpr int kMaxTileSlots = 32;                  // tiles per CTA whose block info is precomputed
constexpr int kEpiBarrier = 1;                     // named barrier of the epilogue warps
// PAIR: a cluster of two CTAs computes a 256 x BN tile with cta_group::2
// MMAs, each CTA holding its 128 rows of A and half of the BN rows of W, so
// every weight byte brought from L2 feeds twice the work without doubling one
// SM's operand stages.
// The mainloop is bound by the operand bytes in flight (loaded L2 latency
// times rate), so every form takes as many stages as shared memory holds
// beside the epilogue's y boxes: 6 x 32 KB (bf16 outputs), 5 x 32 KB (fp32)
// and, in a pair, 8 x 24 KB (bf16) or 6 x 24 KB (fp32) fill the 227 KB of a
// CTA; 128 x 256 tiles keep 3 x 48 KB beside their 64 KB of y boxes (4 x 32 KB
// in a pair).
template <int BN, bool OUT_BF16, bool PAIR = false>
struct GemmCfg {
  static constexpr int kStages = PAIR ? (BN == 256 ? 4 : (OUT_BF16 ? 8 : 6)) : (BN == 256 ? 3 : (OUT_BF16 ? 6 : 5));
  static constexpr int kWBytes = (PAIR ? BN / 2 : BN) * kChunkK;  // a CTA of a pair holds half of W's rows
  static constexpr int kStageBytes = kA0Bytes + kWBytes;
  static constexpr int kSlots = 512 / BN;                            // TMEM accumulator slots of BN columns
  static_assert(kSlots >= 2, "a two-plane tile takes two accumulator slots");
  static constexpr int kHalfGroups = BN / 64;                        // 32-column groups per epilogue warp
  static constexpr int kOutBytes = OUT_BF16 ? 2 : 4;
  static constexpr int kBoxBytes = 32 * 32 * kOutBytes;              // one 32 x 32 tile of Y
  static constexpr int kYWarpBytes = kHalfGroups * kBoxBytes;        // one epilogue warp's tiles
  // small region first, then the 1024-aligned buffers
  static constexpr int kNumBars = 2 * kStages + 2 * kSlots + kEpiWarps + 2;
  static constexpr int kOffBar = 0;
  static constexpr int kOffMisc = (kOffBar + kNumBars * 8 + 15) & ~15;  // tmem base, abort flag
  static constexpr int kOffWs = kOffMisc + 16;                          // [2][BN] fp32 weight scales
  static constexpr int kOffInfo = (kOffWs + 2 * BN * 4 + 15) & ~15;         // [kMaxTileSlots] int4 block info
  static constexpr int kSmallBytes = kOffInfo + kMaxTileSlots * 16;
  static_assert(kOffWs % 16 == 0 && kOffInfo % 16 == 0, "16-byte aligned shared arrays");
  static constexpr int kOffStages = (kSmallBytes + 1023) & ~1023;
  static constexpr int kOffY = kOffStages + kStages * kStageBytes;
  static constexpr int kBytes = kOffY + kEpiWarps * kYWarpBytes + 1024;  // + base alignment slack
  static_assert(kBytes <= 227 * 1024, "shared memory of one CTA");
};

struct BlockInfo {
  int nplanes;  // 1 or 2 operand planes (plane 0 is computed even when every tile takes the slice stream)
  int any_slice;  // some tile of the row block goes through the slice stream
  uint32_t mask[2];
};

// What the quantizer decided for the token tiles [t0, t0 + n) of an output
// tile's rows (any thread, from global memory).
__device__ __forceinline__ BlockInfo block_info_global(const GemmParams& p, int t0, int n) {
  BlockInfo bi;
  bi.mask[0] = bi.mask[1] = 0;
  bi.any_slice = 0;
  const int T = (int)(p.M / kTile);
  int np = 0;
  bool any = false;
  for (int t = t0; t < min(t0 + n, T); ++t) {
    const int pl = p.planes[t];
    if (pl <= 2) {
      any = true;
      np = max(np, pl);
    } else {
      bi.any_slice = 1;
    }
    for (int w = 0; w < (int)p.mask_words && w < 2; ++w) bi.mask[w] |= p.mask1[(int64_t)t * p.mask_words + w];
  }
  bi.nplanes = (any && np == 2 && (bi.mask[0] | bi.mask[1])) ? 2 : 1;
  return bi;
}

__device__ __forceinline__ bool chunk_has_plane1(const BlockInfo& bi, int c) {
  return bi.nplanes == 2 && ((bi.mask[c >> 5] >> (c & 31)) & 1u);
}

__device__ __forceinline__ float exp2_exact(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ void epi_barrier() {
  asm volatile("bar.sync %0, %1;" ::"n"(kEpiBarrier), "n"(32 * kEpiWarps) : "memory");
}

template <bool OUT_BF16>
struct OutT;
template <>
struct OutT<true> {
  using T = __nv_bfloat16;
};
template <>
struct OutT<false> {
  using T = float;
};

// y = y_prev + (((float)acc * p2) * beta) * ws  -- fp32, no contraction.  beta is
// the dynamic base, or exactly 1 with the static base (whose scale is in p2).
__device__ __forceinline__ float epi(int64_t acc, bool wide, float p2, float beta, float ws, float yp) {
  const float a = wide ? __ll2float_rn(acc) : __int2float_rn((int)acc);
  return __fadd_rn(yp, __fmul_rn(__fmul_rn(__fmul_rn(a, p2), beta), ws));
}

// The dynamic base written by the quantizer's first pass (1 when no M_i was
// nonzero), or 1 with the static base.
__device__ __forceinline__ float dyn_beta(const uint32_t* dyn_base) {
  if (!dyn_base) return 1.f;
  const uint32_t b = *dyn_base;
  return b == 0xFFFFFFFFu ? 1.f : __uint_as_float(b);
}

template <bool OUT_BF16>
__device__ __forceinline__ float load_y(const void* base, int64_t off) {
  if constexpr (OUT_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[off]);
  else return static_cast<const float*>(base)[off];
}

template <bool OUT_BF16>
__device__ __forceinline__ void store_y(void* base, int64_t off, float y) {
  if constexpr (OUT_BF16) static_cast<__nv_bfloat16*>(base)[off] = __float2bfloat16_rn(y);
  else static_cast<float*>(base)[off] = y;
}

// GELU(y) = y Phi(y) = 0.5 y erfc(-y / sqrt 2), the activation between the
// two layers of a DiT feed-forward block (section 4.3 "Operator Mapping"),
// in fp32 with CUDA's erfcf (the erfc form keeps its relative accuracy in
// the negative tail, where 1 + erf cancels).
__device__ __forceinline__ float gelu(float y) {
  return __fmul_rn(__fmul_rn(0.5f, y), erfcf(__fmul_rn(y, -0.70710678118654752f)));
}

}  // namespace

// GELU of every bf16 value (the paper's vector unit computes GELU with
// lookup tables): entry b holds GELU of the bf16 pattern b, evaluated in fp64
// (CUDA's double erfc) and rounded to fp32, then to bf16.  Filled once per
// CUDA context by gelu_table_kernel before the first GEMM that reads it.
__device__ uint16_t g_gelu_bf16[65536];

__global__ void gelu_table_kernel() {
  const uint32_t b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= 65536u) return;
  const double v = (double)__uint_as_float(b << 16);
  const double g = 0.5 * v * erfc(-v * 0.70710678118654752440);
  g_gelu_bf16[b] = __bfloat16_as_ushort(__float2bfloat16_rn((float)g));
}

namespace {

// H = GELU(stored Y_t): the table for bf16 outputs, fp32 erfcf for fp32 ones.
template <bool OUT_BF16>
__device__ __forceinline__ float gelu_of_output(float y) {
  if constexpr (OUT_BF16) return __bfloat162float(__ushort_as_bfloat16(g_gelu_bf16[__bfloat16_as_ushort(__float2bfloat16_rn(y))]));
  else return gelu(y);
}

// The paper's accumulation order literally, for one 16-token tile and one
// output column n: walk the tile's encoded stream in (FPoT, channel) order;
// when the FPoT changes, shift the 16 running sums left by the difference,
// then add digit x w[n][k] (section 3.1 step 5, Fig. 6).  The sums end in
// units of the last FPoT and are shifted to g_ref.
template <bool OUT_BF16>
__device__ void slice_stream_column(const uint2* recs, int cnt, const int8_t* bits_row, int g_ref,
                                    const int8_t* w_row, int64_t t, int64_t n, int lb, float beta, float ws,
                                    void* y_prev, int64_t ld_yp, void* y_out, int64_t ld_yo, int y_distinct,
                                    int64_t* debug_acc, int64_t N, void* h_out, int64_t ld_h) {
  int64_t acc[kTile];
#pragma unroll
  for (int i = 0; i < kTile; ++i) acc[i] = 0;
  int prev = 0;
  for (int r = 0; r < cnt; ++r) {
    const uint2 rec = recs[r];
    const int k = (int)(rec.y & 0xFFFFu);
    const int tag = (int)(int8_t)((rec.y >> 16) & 0xFFu);
    const int j = (int)(rec.y >> 24);
    if (r > 0 && tag != prev) {
      const int sh = tag - prev;
#pragma unroll
      for (int i = 0; i < kTile; ++i) acc[i] *= ((int64_t)1 << sh);
    }
    prev = tag;
    const bool top = j == (bits_row[k] >> 1) - 1;
    const int64_t w = (int64_t)w_row[k];
#pragma unroll
    for (int i = 0; i < kTile; ++i) {
      int d = (int)((rec.x >> (2 * i)) & 3u);
      if (top && d >= 2) d -= 4;
      acc[i] += (int64_t)d * w;
    }
  }
  if (cnt > 0 && g_ref != prev) {
    const int sh = g_ref - prev;
#pragma unroll
    for (int i = 0; i < kTile; ++i) acc[i] *= ((int64_t)1 << sh);
  }
  const float p2 = exp2_exact(-lb - g_ref);
#pragma unroll
  for (int i = 0; i < kTile; ++i) {
    const int64_t row = t * kTile + i;
    // no y_prev: the output has no cached previous value (Y_{t-1} = 0)
    const float y = epi(acc[i], true, p2, beta, ws, y_prev ? load_y<OUT_BF16>(y_prev, row * ld_yp + n) : 0.f);
    store_y<OUT_BF16>(y_out, row * ld_yo + n, y);
    if (y_distinct) store_y<OUT_BF16>(y_prev, row * ld_yp + n, y);
    if (h_out) store_y<OUT_BF16>(h_out, row * ld_h + n, gelu_of_output<OUT_BF16>(y));
    if (debug_acc) debug_acc[row * N + n] = acc[i];
  }
}

// One epilogue group: 32 columns of one row (this lane's), in place in its
// swizzled 32 x 32 shared-memory tile.  acc = d0 (+ 256 d1 for rows of
// two-plane tiles); y = y_prev + (((float)acc * p2) * beta) * w_scale, fp32, no FMA.
// With GELU, the activation of the stored values also goes to hrow (this
// lane's row of the activation output at the group's first column, global
// memory), 16 bytes per chunk, for the first hchunks chunks (columns < N).
template <bool OUT_BF16, bool WIDE, bool GELU, bool ZERO_Y = false>
__device__ __forceinline__ void epi_group(uint8_t* row, int swz, const float* ws32, const uint32_t (&d0)[32],
                                          const uint32_t (&d1)[32], bool wide_row, float p2, float beta,
                                          uint8_t* hrow, int hchunks) {
  constexpr int kOutBytes = OUT_BF16 ? 2 : 4;
  constexpr int E = 16 / kOutBytes;              // outputs per 16-byte chunk
  constexpr int kChunks = 32 * kOutBytes / 16;   // chunks per 32-column row
  const float4* ws4 = reinterpret_cast<const float4*>(ws32);  // 16-byte aligned
#pragma unroll
  for (int c = 0; c < kChunks; ++c) {
    uint4* cp = reinterpret_cast<uint4*>(row + 16 * (c ^ swz));
    const uint4 yv = ZERO_Y ? make_uint4(0u, 0u, 0u, 0u) : *cp;  // ZERO_Y: no cached output (Y_{t-1} = 0)
    const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
    float wsv[E];
#pragma unroll
    for (int h = 0; h < E / 4; ++h) {
      const float4 w = ws4[c * (E / 4) + h];
      wsv[4 * h] = w.x, wsv[4 * h + 1] = w.y, wsv[4 * h + 2] = w.z, wsv[4 * h + 3] = w.w;
    }
    float y[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int i = c * E + e;
      float ypf;
      if constexpr (OUT_BF16) ypf = __uint_as_float((e & 1) ? (yw[e >> 1] & 0xFFFF0000u) : (yw[e >> 1] << 16));
      else ypf = __uint_as_float(yw[e]);
      float a;
      if constexpr (WIDE) a = __ll2float_rn((int64_t)(int32_t)d0[i] + (wide_row ? (int64_t)(int32_t)d1[i] * 256 : 0));
      else a = __int2float_rn((int32_t)d0[i]);
      y[e] = __fadd_rn(ypf, __fmul_rn(__fmul_rn(__fmul_rn(a, p2), beta), wsv[e]));
    }
    if constexpr (OUT_BF16) {
      uint32_t w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(y[2 * q], y[2 * q + 1]);
        w[q] = *reinterpret_cast<const uint32_t*>(&b2);
      }
      *cp = make_uint4(w[0], w[1], w[2], w[3]);
      if constexpr (GELU) {
        if (c < hchunks) {
          uint32_t h[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)  // two table entries per word of stored values
            h[q] = (uint32_t)g_gelu_bf16[w[q] & 0xFFFFu] | ((uint32_t)g_gelu_bf16[w[q] >> 16] << 16);
          *reinterpret_cast<uint4*>(hrow + 16 * c) = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
    } else {
      *cp = make_uint4(__float_as_uint(y[0]), __float_as_uint(y[1]), __float_as_uint(y[2]), __float_as_uint(y[3]));
      if constexpr (GELU) {
        if (c < hchunks)
          *reinterpret_cast<uint4*>(hrow + 16 * c) = make_uint4(
              __float_as_uint(gelu(y[0])), __float_as_uint(gelu(y[1])), __float_as_uint(gelu(y[2])),
              __float_as_uint(gelu(y[3])));
      }
    }
  }
}

}  // namespace

size_t gemm_smem_bytes(int bn, int pair) {
  if (pair) return bn == 256 ? GemmCfg<256, true, true>::kBytes : GemmCfg<128, true, true>::kBytes;
  return bn == 256 ? GemmCfg<256, true>::kBytes : GemmCfg<128, true>::kBytes;
}

// The batched, block-sparse form takes a GemmSparse argument; the plain one
// an empty struct.
struct NoSparse {};
template <bool S>
struct SparseArg {
  using T = NoSparse;
};
template <>
struct SparseArg<true> {
  using T = GemmSparse;
};

template <int BN, bool OUT_BF16, bool GELU, bool SPARSE, bool PAIR>
__global__ void __launch_bounds__(kGThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a0, const __grid_constant__ CUtensorMap tm_a1,
                const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_yp,
                const __grid_constant__ CUtensorMap tm_yo, const GemmParams p,
                const __grid_constant__ typename SparseArg<SPARSE>::T sp) {
  using C = GemmCfg<BN, OUT_BF16, PAIR>;
  static_assert(!SPARSE || !PAIR, "the batched form uses 128-row tiles");
  constexpr int BM = kBlockM * (PAIR ? 2 : 1);  // rows of an output tile
  constexpr int kTilesPerBlock = BM / kTile;
  // With PAIR, CTA crank of cluster `unit` owns rows [crank * 128, +128) of
  // each tile; otherwise every CTA is its own unit.
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = crank == 0;
  const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;
  using TOut = typename OutT<OUT_BF16>::T;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;                       // [kStages] TMA -> MMA
  uint64_t* empty = full + C::kStages;         // [kStages] MMA -> TMA
  uint64_t* tm_full = empty + C::kStages;      // [kSlots] MMA -> epilogue
  uint64_t* tm_empty = tm_full + C::kSlots;    // [kSlots] epilogue -> MMA
  uint64_t* ybar = tm_empty + C::kSlots;       // [kEpiWarps] y_prev tiles landed
  uint64_t* drain = ybar + kEpiWarps;          // MMA completion at exit
  uint64_t* info_bar = drain + 1;              // block info in shared memory
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  float* s_ws = reinterpret_cast<float*>(smem + C::kOffWs);
  int4* s_info = reinterpret_cast<int4*>(smem + C::kOffInfo);  // {nplanes, any_slice, mask0, mask1} per tile
  uint8_t* stages = smem + C::kOffStages;
  uint8_t* ysmem = smem + C::kOffY;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Tile i of the launch -> (row block, column block); with SPARSE, tiles run
  // head by head over the listed tiles of a head (all, when none is listed).
  int num_tiles = p.tiles_m * p.tiles_n, rb_per_head = p.tiles_m, tiles_per_head = num_tiles;
  if constexpr (SPARSE) {
    rb_per_head = (int)(sp.rows_per_head / kBlockM);
    tiles_per_head = sp.n_listed > 0 ? sp.n_listed : rb_per_head * p.tiles_n;
    num_tiles = (int)sp.heads * tiles_per_head;
  }
  auto coords = [&](int i, int& rb, int& nb) {
    if constexpr (SPARSE) {
      const int head = i / tiles_per_head, j = i % tiles_per_head;
      const int id = sp.n_listed > 0 ? (int)sp.list[j] : j;
      rb = head * rb_per_head + id / p.tiles_n, nb = id % p.tiles_n;
    } else {
      rb = i / p.tiles_n, nb = i % p.tiles_n;
    }
  };
  // first row of W for a tile (the head's weights with SPARSE)
  auto w_row = [&](int rb, int nb) -> int {
    if constexpr (SPARSE) return (int)((rb / rb_per_head) * sp.w_rows_per_head) + nb * BN;
    else return nb * BN;
  };
  // K chunk c of plane 0 is read for row block rb
  auto keep0 = [&](int rb, int c) -> bool {
    if constexpr (SPARSE) return ((sp.chunk_keep[rb % rb_per_head] >> c) & 1ull) != 0;
    else return true;
  };
  const int my_tiles = num_tiles > unit ? (num_tiles - 1 - unit) / units + 1 : 0;
  const int T = (int)(p.M / kTile);
  // first row of this CTA's rows of row block rb
  auto row_of = [&](int rb) { return rb * BM + (int)crank * kBlockM; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) mbar_init(&full[i], 1), mbar_init(&empty[i], 1);
    // with PAIR the even CTA's tm_empty counts both CTAs' epilogue warps
    for (int i = 0; i < C::kSlots; ++i) mbar_init(&tm_full[i], 1), mbar_init(&tm_empty[i], (PAIR ? 2 : 1) * kEpiWarps);
    for (int i = 0; i < kEpiWarps; ++i) mbar_init(&ybar[i], 1);
    mbar_init(drain, 1);
    mbar_init(info_bar, 1);
    *s_abort = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_a0);
    prefetch_tmap(&tm_a1);
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_yp);
    prefetch_tmap(&tm_yo);
  }
  // set-up that does not touch memory written by the previous kernel
  for (int i = threadIdx.x; i < kMaxTileSlots; i += kGThreads) s_info[i] = make_int4(0, 0, 0, 0);
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(s_tmem, 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s_tmem, 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  // with PAIR the peer's barriers and TMEM exist before either CTA signals the other
  if constexpr (PAIR) cluster_sync();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  pdl_launch_dependents();

  auto info = [&](int slot, int rb) -> BlockInfo {
    if (slot < kMaxTileSlots) {
      const int4 e = s_info[slot];
      BlockInfo bi;
      bi.mask[0] = (uint32_t)e.z, bi.mask[1] = (uint32_t)e.w;
      bi.any_slice = e.y;
      bi.nplanes = (e.x == 2 && (e.z | e.w)) ? 2 : 1;
      return bi;
    }
    return block_info_global(p, rb * kTilesPerBlock, kTilesPerBlock);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (elect_one()) {
      uint32_t it = 0;
      bool ok = true;
      // With PAIR both CTAs' loads complete on the even CTA's full barrier,
      // which expects the bytes of both.
      const uint32_t full_cl = PAIR ? cluster_smem_addr(full, 0) : 0u;
      auto load = [&](void* dst, const CUtensorMap* m, int s, int x, int y) {
        if constexpr (PAIR) tma_load_2d_pair(dst, m, full_cl + 8u * (uint32_t)s, x, y);
        else tma_load_2d(dst, m, &full[s], x, y);
      };
      auto expect = [&](int s) {
        if (leader) mbar_arrive_expect_tx(&full[s], (PAIR ? 2 : 1) * C::kStageBytes);
      };
      const int w_off = PAIR ? (int)crank * (BN / 2) : 0;  // this CTA's rows of the W tile
      // The weights do not depend on the previous kernel: the W tiles of the
      // first stages are requested before waiting for it.
      uint32_t pre = 0;
      if (my_tiles > 0) {
        int rb0, nb0;
        coords(unit, rb0, nb0);
        for (int c = 0; c < p.num_chunks && pre < (uint32_t)C::kStages; ++c) {
          if (!keep0(rb0, c)) continue;
          expect(pre);
          load(stages + pre * C::kStageBytes + kA0Bytes, &tm_w, pre, c * kChunkK, w_row(rb0, nb0) + w_off);
          ++pre;
        }
      }
      pdl_wait();  // the operand planes are the previous kernel's output
      bool have_info = false;
      for (int slot = 0; slot < my_tiles && ok; ++slot) {
        int rb, nb;
        coords(unit + slot * units, rb, nb);
        const int wr = w_row(rb, nb) + w_off;
        for (int pass = 0; pass < 2 && ok; ++pass) {
          BlockInfo bi{};
          if (pass == 1) {  // plane 1 only where the block needs it
            if (!have_info && !(ok = wait_parity(info_bar, 0, s_abort, p.status, kWaitLimitNs))) break;
            have_info = true;
            bi = info(slot, rb);
            if (bi.nplanes < 2) break;
          }
          const CUtensorMap* tm_a = pass == 0 ? &tm_a0 : &tm_a1;
          for (int c = 0; c < p.num_chunks; ++c) {
            if (pass == 0 && !keep0(rb, c)) continue;
            if (pass == 1 && !chunk_has_plane1(bi, c)) continue;
            const int s = it % C::kStages;
            uint8_t* a = stages + s * C::kStageBytes;
            if (it < pre) {  // the stage's W tile is already on its way
              load(a, tm_a, s, c * kChunkK, row_of(rb));
              ++it;
              continue;
            }
            if (!wait_parity(&empty[s], ((it / C::kStages) & 1) ^ 1, s_abort, p.status, kWaitLimitNs)) {
              ok = false;
              break;
            }
            expect(s);
            load(a, tm_a, s, c * kChunkK, row_of(rb));
            load(a + kA0Bytes, &tm_w, s, c * kChunkK, wr);
            ++it;
          }
        }
      }
      // drain: every stage filled must have landed before the block can exit
      // (with PAIR the even CTA's barriers count both CTAs' loads, and the
      // final cluster barrier holds the odd CTA until then)
      const uint32_t first = it > (uint32_t)C::kStages ? it - C::kStages : 0;
      if (leader)
        for (uint32_t j = first; j < it; ++j)
          wait_parity(&full[j % C::kStages], (j / C::kStages) & 1, s_abort, p.status, kWaitLimitNs, true);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------------- MMA
    if (elect_one() && leader) {  // with PAIR the even CTA issues the pair's MMAs
      pdl_wait();  // block info beyond the shared-memory table is read from global memory
      constexpr uint32_t idesc = idesc_i8(BN, PAIR ? 256 : 128);
      uint32_t it = 0, slot_it = 0;
      bool ok = true, issued = false, have_info = false;
      for (int slot = 0; slot < my_tiles && ok; ++slot) {
        int rb, nb_unused;
        coords(unit + slot * units, rb, nb_unused);
        uint32_t acc0 = 0, acc1 = 0;
        int np = 1;
        for (int pass = 0; pass < 2 && ok; ++pass) {
          BlockInfo bi{};
          if (pass == 1) {
            if (!have_info && !(ok = wait_parity(info_bar, 0, s_abort, p.status, kWaitLimitNs))) break;
            have_info = true;
            bi = info(slot, rb);
            if (bi.nplanes < 2) break;
            np = 2;
          }
          // the pass's accumulator slot
          const uint32_t si = slot_it + pass;
          const uint32_t acc = si % C::kSlots;
          (pass == 0 ? acc0 : acc1) = acc;
          if (!(ok = wait_parity(&tm_empty[acc], ((si / C::kSlots) & 1) ^ 1, s_abort, p.status, kWaitLimitNs)))
            break;
          tc_fence_after();
          const uint32_t d = tmem_base + acc * BN;
          bool first = true;
          for (int c = 0; c < p.num_chunks; ++c) {
            if (pass == 0 && !keep0(rb, c)) continue;
            if (pass == 1 && !chunk_has_plane1(bi, c)) continue;
            const int s = it % C::kStages;
            if (!wait_parity(&full[s], (it / C::kStages) & 1, s_abort, p.status, kWaitLimitNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da = smem_desc_k_sw128(stages + s * C::kStageBytes);
            const uint64_t dw = smem_desc_k_sw128(stages + s * C::kStageBytes + kA0Bytes);
#pragma unroll
            for (int kk = 0; kk < kChunkK / 32; ++kk) {
              if constexpr (PAIR) mma_i8_pair(d, da + 2 * kk, dw + 2 * kk, idesc, (!first || kk > 0) ? 1u : 0u);
              else mma_i8(d, da + 2 * kk, dw + 2 * kk, idesc, (!first || kk > 0) ? 1u : 0u);
            }
            first = false;
            if constexpr (PAIR) mma_commit_pair_mc(&empty[s], 3);  // both CTAs may refill the stage
            else mma_commit(&empty[s]);
            issued = true;
            ++it;
          }
        }
        if (!ok) break;
        if constexpr (PAIR) {  // both CTAs' epilogues read their halves of the slot
          mma_commit_pair_mc(&tm_full[acc0], 3);
          if (np == 2) mma_commit_pair_mc(&tm_full[acc1], 3);
        } else {
          mma_commit(&tm_full[acc0]);
          if (np == 2) mma_commit(&tm_full[acc1]);
        }
        slot_it += np;
      }
      // drain: all MMAs this thread issued complete before TMEM and SMEM go away
      if (issued) {
        if constexpr (PAIR) mma_commit_pair(drain);
        else mma_commit(drain);
        wait_parity(drain, 0, s_abort, p.status, kWaitLimitNs, true);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;           // 0 .. kEpiWarps-1
    const int etid = threadIdx.x - 64; // 0 .. 32*kEpiWarps-1
    const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31 are this warp's rows
    const int half = ew >> 2;          // columns [half*BN/2, (half+1)*BN/2)
    uint8_t* ybuf = ysmem + ew * C::kYWarpBytes;  // this warp's kHalfGroups tiles of 32 x 32
    static_assert(BN <= 32 * kEpiWarps, "one weight scale per epilogue thread and tile");
    static_assert(C::kHalfGroups % 2 == 0, "groups are processed in pairs");
    // TMA swizzle of a 32 x 32 tile: 64-byte rows (bf16) use the 64-byte pattern,
    // 128-byte rows (fp32) the 128-byte one; chunk c of row r sits at chunk c ^ sw(r)
    auto sw = [](int r) { return OUT_BF16 ? ((r >> 1) & 3) : (r & 7); };
    // the slot's tm_empty barrier: the even CTA's with PAIR
    const uint32_t tm_empty_cl = PAIR ? cluster_smem_addr(tm_empty, 0) : 0u;
    // Everything a tile needs besides its accumulator is requested one tile
    // ahead: its y_prev boxes (each as soon as the previous tile's store has
    // read the box), its weight scales (shared memory, double-buffered) and
    // this lane's row data.
    auto weight_scale = [&](int rb_s, int nb_s) -> float {
      const int64_t n = (int64_t)nb_s * BN + etid;
      int64_t off = 0;  // the head's scales with SPARSE
      if constexpr (SPARSE) off = (int64_t)(rb_s / rb_per_head) * p.N;
      return (etid < BN && n < p.N) ? p.w_scale[off + n] : 0.f;
    };
    // this lane's row: plane count (3 beyond M) and g_ref
    auto row_planes = [&](int rb_s, int& pl, int& gref) {
      const int64_t row = (int64_t)row_of(rb_s) + quarter * 32 + lane;
      pl = 3, gref = 0;
      if (row < p.M) pl = p.planes[row / kTile], gref = p.g_ref[row / kTile];
    };
    // With SPARSE there is no cached output: Y_{t-1} = 0 is never read.
    auto load_y_box = [&](int rb_s, int nb_s, int g) {  // lane 0
      if constexpr (SPARSE) return;
      if (g == 0) mbar_arrive_expect_tx(&ybar[ew], C::kYWarpBytes);
      tma_load_2d(ybuf + g * C::kBoxBytes, &tm_yp, &ybar[ew], nb_s * BN + half * (BN / 2) + g * 32,
                  row_of(rb_s) + quarter * 32);
    };
    uint32_t slot_it = 0;
    uint32_t y_issued = 0, y_seen = 0;  // batches of y_prev boxes requested (lane 0) / observed landed
    int ok = 1;
    pdl_wait();  // the quantizer's outputs and the cached output are read from here on
    const float beta = dyn_beta(p.dyn_base);
    // this tile's coordinates and the next one's, advanced once per tile
    int rb_c = 0, nb_c = 0;
    if (my_tiles > 0) coords(unit, rb_c, nb_c);
    if (lane == 0 && my_tiles > 0) {
      for (int g = 0; g < C::kHalfGroups; ++g) load_y_box(rb_c, nb_c, g);
      ++y_issued;
    }
    int pl_cur = 3, gref_cur = 0;
    if (my_tiles > 0) {
      row_planes(rb_c, pl_cur, gref_cur);
      if (etid < BN) s_ws[etid] = weight_scale(rb_c, nb_c);
    }
    // block info of this CTA's first kMaxTileSlots tiles, loaded in parallel,
    // then published to the producer and MMA threads (with PAIR both CTAs
    // compute the same information for the tile's 256 rows)
    for (int i = etid; i < min(my_tiles, kMaxTileSlots) * kTilesPerBlock; i += 32 * kEpiWarps) {
      const int slot = i / kTilesPerBlock, sub = i % kTilesPerBlock;
      int rb_s, nb_s;
      coords(unit + slot * units, rb_s, nb_s);
      const int t = rb_s * kTilesPerBlock + sub;
      if (t < T) {
        const int pl = p.planes[t];
        int* e = reinterpret_cast<int*>(&s_info[slot]);
        if (pl <= 2) atomicMax(&e[0], pl);
        else atomicOr(&e[1], 1);
        if (p.mask_words > 0) atomicOr(reinterpret_cast<unsigned*>(&e[2]), p.mask1[(int64_t)t * p.mask_words]);
        if (p.mask_words > 1) atomicOr(reinterpret_cast<unsigned*>(&e[3]), p.mask1[(int64_t)t * p.mask_words + 1]);
      }
    }
    epi_barrier();
    if (etid == 0) mbar_arrive(info_bar);
    // Every epilogue warp runs every iteration and the named barrier of it,
    // also after a timed-out wait (ok == 0), so no warp can be left waiting
    // at a barrier that another warp skipped.
    for (int slot = 0; slot < my_tiles; ++slot) {
      const int rb = rb_c, nb = nb_c;
      const bool has_next = slot + 1 < my_tiles;
      int rb_n = 0, nb_n = 0;
      if (has_next) coords(unit + (slot + 1) * units, rb_n, nb_n);
      const BlockInfo bi = info(slot, rb);
      const int64_t n_base = (int64_t)nb * BN;
      const int64_t n_half = n_base + half * (BN / 2);
      const int row0 = row_of(rb) + quarter * 32;
      const float* ws_tile = s_ws + (slot & 1) * BN;
      float ws_next = 0.f;
      int pl_next = 3, gref_next = 0;
      if (has_next) {
        ws_next = weight_scale(rb_n, nb_n);
        row_planes(rb_n, pl_next, gref_next);
      }

      if (ok) {
        const int64_t row = row0 + lane;
        const int pl = pl_cur;
        const bool row_ok = row < p.M && pl <= 2;
        const float p2 = row_ok ? exp2_exact(-p.lb - gref_cur) : 0.f;

        uint32_t acc_slot[2];
        for (int q = 0; q < bi.nplanes; ++q) {
          const uint32_t si = slot_it + q;
          acc_slot[q] = si % C::kSlots;
          // one lane polls; the warp follows its verdict (tcgen05.ld needs the whole warp)
          if (lane == 0 && ok)
            ok = wait_parity(&tm_full[acc_slot[q]], (si / C::kSlots) & 1, s_abort, p.status, kWaitLimitNs) ? 1 : 0;
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if constexpr (!SPARSE) {
          if (lane == 0 && ok) ok = wait_parity(&ybar[ew], y_seen & 1, s_abort, p.status, kWaitLimitNs) ? 1 : 0;
          ok = __shfl_sync(0xffffffffu, ok, 0);
        } else {
          if (lane == 0) bulk_wait_read<0>();  // the previous tile's stores have read the boxes
          __syncwarp();
        }
        if (ok) {
          // the landed tiles are visible to the lanes that observe the barrier phase
          if constexpr (!SPARSE) {
            mbar_try_wait(&ybar[ew], y_seen & 1);
            ++y_seen;
          }
          tc_fence_after();
          const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
          const uint32_t col_half = half * (BN / 2);
          const uint32_t t0a = tmem_base + lane_off + acc_slot[0] * BN + col_half;
          const uint32_t t1a = tmem_base + lane_off + (bi.nplanes == 2 ? acc_slot[1] : acc_slot[0]) * BN + col_half;
          const float* ws_h = ws_tile + half * (BN / 2);
          const bool wide_blk = bi.nplanes == 2;  // warp-uniform
          const bool wide_row = pl == 2;
          // Finished 32 x 32 tiles go out through TMA (rows beyond M and columns
          // beyond N are clipped; rows left to the slice stream keep y_prev).
          // Once a store has read its box, the next tile's y_prev box is
          // requested into it.
          auto store_group = [&](int g) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              if (n_half + g * 32 < p.N && row0 < p.M) {  // a store never starts outside the matrix
                tma_store_2d(&tm_yo, ybuf + g * C::kBoxBytes, (int)(n_half + g * 32), row0);
                if (p.y_distinct) tma_store_2d(&tm_yp, ybuf + g * C::kBoxBytes, (int)(n_half + g * 32), row0);
              }
              bulk_commit();
              if (has_next && g > 0) {
                bulk_wait_read<1>();
                load_y_box(rb_n, nb_n, g - 1);
              }
              if (has_next && g == C::kHalfGroups - 1) {
                bulk_wait_read<0>();
                load_y_box(rb_n, nb_n, g);
                ++y_issued;
              }
            }
          };
          auto debug_group = [&](int g, const uint32_t (&d0)[32], const uint32_t (&d1)[32], bool wide) {
            const int64_t n0 = n_half + g * 32;
            for (int i = 0; i < 32 && n0 + i < p.N; ++i)
              p.debug_acc[row * p.N + n0 + i] =
                  (int64_t)(int32_t)d0[i] + (wide && wide_row ? (int64_t)(int32_t)d1[i] * 256 : 0);
          };
          uint8_t* my_row = ybuf + lane * (32 * C::kOutBytes);
          const int swz = sw(lane);
          // this lane's row of the activation output at group g (GELU only)
          auto h_row = [&](int g, int& hch) -> uint8_t* {
            hch = 0;
            if constexpr (!GELU) return nullptr;
            constexpr int E = 16 / C::kOutBytes;
            const int64_t n0 = n_half + g * 32, left = p.N - n0;
            if (left <= 0) return nullptr;
            hch = left >= 32 ? 32 / E : (int)(left / E);
            return static_cast<uint8_t*>(p.h_out) + (row * p.ld_h + n0) * C::kOutBytes;
          };
          auto one_plane_group = [&](int g, const uint32_t (&d)[32]) {
            if (row_ok) {
              int hch;
              uint8_t* hr = h_row(g, hch);
              epi_group<OUT_BF16, false, GELU, SPARSE>(my_row + g * C::kBoxBytes, swz, ws_h + g * 32, d, d, false, p2,
                                                       beta, hr, hch);
              if (p.debug_acc) debug_group(g, d, d, false);
            }
            store_group(g);
          };
          if (!wide_blk) {
            // one plane: groups in pairs, the accumulator of the next group is
            // read from TMEM while the current one is computed
            uint32_t dA[32], dB[32];
            tmem_ld32(t0a, dA);
            tmem_ld_wait(dA);
#pragma unroll 1
            for (int g = 0; g < C::kHalfGroups; g += 2) {
              tmem_ld32(t0a + (g + 1) * 32, dB);
              one_plane_group(g, dA);
              tmem_ld_wait(dB);
              if (g + 2 < C::kHalfGroups) tmem_ld32(t0a + (g + 2) * 32, dA);
              one_plane_group(g + 1, dB);
              if (g + 2 < C::kHalfGroups) tmem_ld_wait(dA);
            }
          } else {
#pragma unroll 1
            for (int g = 0; g < C::kHalfGroups; ++g) {
              uint32_t d0[32], d1[32];
              tmem_ld32(t0a + g * 32, d0);
              tmem_ld32(t1a + g * 32, d1);
              tmem_ld_wait(d0);
              tmem_ld_wait(d1);
              if (row_ok) {
                int hch;
                uint8_t* hr = h_row(g, hch);
                epi_group<OUT_BF16, true, GELU, SPARSE>(my_row + g * C::kBoxBytes, swz, ws_h + g * 32, d0, d1, wide_row,
                                                        p2, beta, hr, hch);
                if (p.debug_acc) debug_group(g, d0, d1, true);
              }
              store_group(g);
            }
          }
          // the slot is free once this warp's TMEM reads are done (with PAIR
          // the even CTA's barrier counts both CTAs' epilogue warps)
          tc_fence_before();
          __syncwarp();
          if (lane == 0)
            for (int q = 0; q < bi.nplanes; ++q) {
              if constexpr (PAIR) mbar_arrive_cluster(tm_empty_cl + 8u * acc_slot[q]);
              else mbar_arrive(&tm_empty[acc_slot[q]]);
            }
          slot_it += bi.nplanes;
        }
      }

      // this CTA's token tiles whose operands need more than two planes: the
      // slice stream, one output column per epilogue thread, after this
      // tile's TMA stores have completed.  Whether the barrier runs depends
      // on the block info alone, the same in every warp, so a warp whose wait
      // gave up (ok == 0) still takes it.
      if (bi.any_slice) {
        if (lane == 0) bulk_wait<0>();
        __syncwarp();
        epi_barrier();
        const int t0 = row_of(rb) / kTile;
        for (int t = ok ? t0 : T; t < min(t0 + kBlockM / kTile, T); ++t) {
          if (p.planes[t] <= 2) continue;
          for (int c = etid; c < BN; c += 32 * kEpiWarps) {
            const int64_t n = n_base + c;
            if (n >= p.N) continue;
            slice_stream_column<OUT_BF16>(p.records + (int64_t)t * p.record_cap, p.count[t], p.bits + (int64_t)t * p.K,
                                          p.g_ref[t], p.w_q + ((int64_t)w_row(rb, 0) + n) * p.ld_w, t, n, p.lb, beta,
                                          ws_tile[c], SPARSE ? nullptr : p.y_prev, p.ld_yp,
                                          p.y_out, p.ld_yo, p.y_distinct, p.debug_acc, p.N, p.h_out, p.ld_h);
          }
        }
      }
      // the next tile's weight scales go to the other buffer, whose readers
      // finished before the previous iteration's barrier
      if (has_next && etid < BN) s_ws[((slot + 1) & 1) * BN + etid] = ws_next;
      pl_cur = pl_next, gref_cur = gref_next;
      rb_c = rb_n, nb_c = nb_n;
      epi_barrier();
    }
    // nothing of this warp's may still be in flight when the block exits:
    // y_prev boxes that were requested but not observed, and the last stores
    y_issued = __shfl_sync(0xffffffffu, y_issued, 0);
    if (lane == 0) {
      if (!SPARSE && y_issued > y_seen)
        wait_parity(&ybar[ew], (y_issued - 1) & 1, s_abort, p.status, kWaitLimitNs, true);
      bulk_wait<0>();
    }
    __syncwarp();
  }

  tc_fence_before();
  // with PAIR neither CTA leaves while the other's MMAs or loads may use its memory
  if constexpr (PAIR) cluster_sync();
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 512);
    else tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------------------
// Slice-stream kernel: every tile through the paper's accumulation order
// (slice_stream_column), one block per (tile, 256 output columns), one output
// column per thread.  Used under DSTAR_FLAG_SLICE_PATH; in the default path
// the tensor-core kernel's epilogue warps run the same routine for the tiles
// that need it.
// ---------------------------------------------------------------------------
template <bool OUT_BF16>
__global__ void __launch_bounds__(256) slice_gemm_kernel(const SliceParams p) {
  const int64_t T = p.M / kTile;
  const int64_t nblk = (p.N + 255) / 256;
  const float beta = dyn_beta(p.dyn_base);
  for (int64_t item = blockIdx.x; item < T * nblk; item += gridDim.x) {
    const int64_t t = item / nblk;
    const int64_t n = (item % nblk) * 256 + threadIdx.x;
    if (!p.all_tiles && p.planes[t] <= 2) continue;
    if (n >= p.N) continue;
    slice_stream_column<OUT_BF16>(p.records + t * p.record_cap, p.count[t], p.bits + t * p.K, p.g_ref[t],
                                  p.w_q + n * p.ld_w, t, n, p.lb, beta, p.w_scale[n], p.y_prev, p.ld_yp, p.y_out, p.ld_yo,
                                  p.y_distinct, p.debug_acc, p.N, p.h_out, p.ld_h);
  }
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// completes; the wait must give up after limit_us and record TIMEOUT.
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    wait_parity(&bar, 0, &abort_flag, status, limit_ns);
  }
}

template <int BN, bool BF, bool GELU, bool SPARSE = false, bool PAIR = false>
static int launch_gemm_t(const GemmParams& p, const CUtensorMap* m, int num_sms, void* stream,
                         const typename SparseArg<SPARSE>::T& sp = {}) {
  int tiles = p.tiles_m * p.tiles_n;
  if constexpr (SPARSE)
    tiles = (int)sp.heads * (sp.n_listed > 0 ? sp.n_listed : (int)(sp.rows_per_head / kBlockM) * p.tiles_n);
  const int units = PAIR ? num_sms / 2 : num_sms;  // CTA pairs are clusters of two
  const int grid = (tiles < units ? tiles : units) * (PAIR ? 2 : 1);
  if (grid == 0) return 0;
  const int smem = GemmCfg<BN, BF, PAIR>::kBytes;
  const int e = ensure_max_smem((const void*)gemm_kernel<BN, BF, GELU, SPARSE, PAIR>, smem);
  if (e != 0) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(kGThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the launch with the quantizer
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = PAIR ? 2 : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = PAIR ? 2 : 1;
  const cudaError_t ce =
      cudaLaunchKernelEx(&cfg, gemm_kernel<BN, BF, GELU, SPARSE, PAIR>, m[0], m[1], m[2], m[3], m[4], p, sp);
  if (ce != cudaSuccess) return (int)ce;
  return (int)cudaGetLastError();
}

// maps: the A0, A1, W, y_prev and y_out tensor maps (CUtensorMap[5]).
template <bool GELU>
static int launch_gemm_g(const GemmParams& p, const CUtensorMap* m, int bn, int pair, int out_bf16, int num_sms,
                         void* stream) {
  if (pair) {
    if (!out_bf16) return launch_gemm_t<128, false, GELU, false, true>(p, m, num_sms, stream);
    return bn == 256 ? launch_gemm_t<256, true, GELU, false, true>(p, m, num_sms, stream)
                     : launch_gemm_t<128, true, GELU, false, true>(p, m, num_sms, stream);
  }
  if (out_bf16)
    return bn == 256 ? launch_gemm_t<256, true, GELU>(p, m, num_sms, stream)
                     : launch_gemm_t<128, true, GELU>(p, m, num_sms, stream);
  return launch_gemm_t<128, false, GELU>(p, m, num_sms, stream);  // fp32 outputs: 128-column tiles
}

int launch_gemm(const GemmParams& p, const void* maps, int bn, int pair, int out_bf16, int num_sms, void* stream) {
  const CUtensorMap* m = static_cast<const CUtensorMap*>(maps);
  if (!(bn == 128 || (bn == 256 && out_bf16))) return (int)cudaErrorInvalidValue;
  return p.h_out ? launch_gemm_g<true>(p, m, bn, pair, out_bf16, num_sms, stream)
                 : launch_gemm_g<false>(p, m, bn, pair, out_bf16, num_sms, stream);
}

int launch_gemm_sparse(const GemmParams& p, const GemmSparse& sp, const void* maps, int num_sms, void* stream) {
  return launch_gemm_t<128, false, false, true>(p, static_cast<const CUtensorMap*>(maps), num_sms, stream, sp);
}

int launch_slice_gemm(const SliceParams& p, int out_bf16, int num_sms, void* stream) {
  const int64_t T = p.M / kTile;
  const int64_t items = T * ((p.N + 255) / 256);
  if (items == 0) return 0;
  const int64_t grid = items < 4LL * num_sms ? items : 4LL * num_sms;
  if (out_bf16) slice_gemm_kernel<true><<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(p);
  else slice_gemm_kernel<false><<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(p);
  return (int)cudaGetLastError();
}

int launch_gelu_table(void* stream) {
  gelu_table_kernel<<<256, 256, 0, (cudaStream_t)stream>>>();
  return (int)cudaGetLastError();
}

int launch_selftest_wait(uint32_t* status, uint32_t limit_us, void* stream) {
  selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status, (uint64_t)limit_us * 1000ull);
  return (int)cudaGetLastError();
}

}  // namespace fmdq
