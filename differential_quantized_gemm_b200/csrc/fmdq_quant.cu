// K1: the FMDQ quantizer (DSTAR section 3.1 steps 1-4; the paper's QPU,
// section 4.2 "Design of QPU", stages 1-5).
//
// One 256-thread block per 16-token tile.  Phase 1 streams the tile's rows of
// X_t and X_{t-1} once with 16-byte loads (coalesced along channels), forms
// dX in fp32, takes the per-channel max |dX| as an integer max over the
// magnitude bits (stage 1 compares the value without its sign), derives PoT
// (Eq. 3), the bit width (threshold bins, stage 2), FPoT (Eq. 4) and the codes
// q = rne(dX * s_i) with s_i = base * 2^FPoT (Eq. 5, stage 3), and keeps the
// codes in shared memory.  Phase 2 knows the tile's finest FPoT (g_ref) and
// writes (a) the tensor-core operand planes: v = q * 2^(g_ref - FPoT), split
// into int8 planes v = A0 + 256 A1, and (b) the encoded stream: one record per
// 2-bit slice, grouped by slice FPoT ascending and channel ascending (stages
// 4-5), located by a per-tag count and exclusive scan instead of a sort.
#include <cuda_bf16.h>

#include "fmdq_device.cuh"

namespace fmdq {

namespace {

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;
constexpr int kMaxTags = 64;  // tag spread within a tile is at most 6 + kPotMax + 6 < 64
constexpr int kMaxMaskWords = (DSTAR_K_MAX / kChunkK + 31) / 32;

template <typename TIn>
struct In;
template <>
struct In<float> {
  static constexpr int kVec = 4;
  __device__ static void load(const void* base, int64_t off, float (&v)[4]) {
    float4 f = *reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
  }
  __device__ static uint4 raw(const void* base, int64_t off) {
    return *reinterpret_cast<const uint4*>(static_cast<const float*>(base) + off);
  }
  __device__ static void store_raw(void* base, int64_t off, uint4 r) {
    *reinterpret_cast<uint4*>(static_cast<float*>(base) + off) = r;
  }
  __device__ static void widen(uint4 r, float (&v)[4]) {
    v[0] = __uint_as_float(r.x), v[1] = __uint_as_float(r.y), v[2] = __uint_as_float(r.z),
    v[3] = __uint_as_float(r.w);
  }
};
template <>
struct In<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ static uint4 raw(const void* base, int64_t off) {
    return *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + off);
  }
  __device__ static void store_raw(void* base, int64_t off, uint4 r) {
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + off) = r;
  }
  // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word.
  __device__ static void widen(uint4 r, float (&v)[8]) {
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
};

__device__ __forceinline__ float exp2_exact(int e) {  // 2^e for e in the normal range
  return __int_as_float((127 + e) << 23);
}

}  // namespace

size_t quantize_smem_bytes(int64_t K) {
  const size_t cs = (size_t)K + 64;                         // padded code row stride
  size_t b = 16 * cs + 4 * (size_t)K;                       // codes + 4 per-column bytes
  b = (b + 15) & ~(size_t)15;
  b += sizeof(int) * (64 + 2 * kQWarps * kMaxTags) + sizeof(uint32_t) * kMaxMaskWords;
  return b;
}

template <typename TIn>
__global__ void __launch_bounds__(kQThreads) quantize_kernel(const QuantParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int VEC = In<TIn>::kVec;
  constexpr int CB = 8 * VEC;  // channels covered by one warp pass (8 lanes x VEC)

  const int64_t K = p.K;
  const int64_t cs = K + 64;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  int8_t* s_codes = reinterpret_cast<int8_t*>(smem);  // [16][cs]
  int8_t* s_fpot = s_codes + 16 * cs;                  // [K]
  int8_t* s_bits = s_fpot + K;
  int8_t* s_qmax = s_bits + K;
  int8_t* s_qmin = s_qmax + K;
  int* s_small = reinterpret_cast<int*>(smem + ((16 * cs + 4 * K + 15) & ~(int64_t)15));
  int* s_hist = s_small + 64;                  // [warps][kMaxTags]
  int* s_off = s_hist + kQWarps * kMaxTags;    // [warps][kMaxTags]
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_off + kQWarps * kMaxTags);
  // s_small: [0,8) warp max FPoT, [8,16) warp min FPoT, [16,24) warp plane need,
  //          [24] flags (1 nonfinite, 2 range), [25] g_ref, [26] min FPoT, [27] planes

  if (tid < kMaxMaskWords) s_mask[tid] = 0;
  if (tid == 0) s_small[24] = 0;
  __syncthreads();

  const int lb = p.lb, t0 = p.t0, fb = p.force_bits;
  const float beta = exp2_exact(lb);
  const bool refresh = !(p.flags & DSTAR_FLAG_NO_XPREV_REFRESH);
  const int rsub = lane >> 3;  // this lane's rows: 4*rsub .. 4*rsub+3
  const int csub = lane & 7;   // this lane's channels: VEC consecutive
  const int nblk = (int)((K + CB - 1) / CB);
  int fmax = -1000, fmin = 1000;
  int flags = 0;

  // ---------------------------------------------------------------- phase 1
  for (int blk = warp; blk < nblk; blk += kQWarps) {
    const int64_t c0 = (int64_t)blk * CB + csub * VEC;
    const bool valid = c0 < K;  // K % 32 == 0: a lane's VEC channels are all valid or all not
    float dx[4][VEC];
    uint4 xt_raw[4], xp_raw[4];
    if (valid) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t row = (int64_t)t * kTile + rsub * 4 + r;
        xt_raw[r] = In<TIn>::raw(p.x_t, row * p.ld_xt + c0);
        xp_raw[r] = In<TIn>::raw(p.x_prev, row * p.ld_xp + c0);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        float a[VEC], b[VEC];
        In<TIn>::widen(xt_raw[r], a);
        In<TIn>::widen(xp_raw[r], b);
#pragma unroll
        for (int c = 0; c < VEC; ++c) dx[r][c] = __fsub_rn(a[c], b[c]);  // Eq. 1, one fp32 subtraction
        if (refresh) {
          const int64_t row = (int64_t)t * kTile + rsub * 4 + r;
          In<TIn>::store_raw(p.x_prev, row * p.ld_xp + c0, xt_raw[r]);
        }
      }
    } else {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < VEC; ++c) dx[r][c] = 0.f;
    }

    // stage 1: max |dX| of each channel over the 16 tokens, on the magnitude bits
    uint32_t mb[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
      uint32_t m = 0;
#pragma unroll
      for (int r = 0; r < 4; ++r) m = max(m, __float_as_uint(dx[r][c]) & 0x7FFFFFFFu);
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 8));
      m = max(m, __shfl_xor_sync(0xffffffffu, m, 16));
      mb[c] = m;
    }

    int8_t qv[4][VEC];
    int fp_c[VEC], b_c[VEC], qmx_c[VEC], qmn_c[VEC];
#pragma unroll
    for (int c = 0; c < VEC; ++c) {
      const bool nonfinite = mb[c] >= 0x7F800000u;
      int P = 0;
      // stage 2, Eq. 3 with the static base: PoT = ceil(log2(M_i / base)), 0 when M_i <= base.
      // M_i > base >= 2^-32 is a normal float: M_i = (1 + f) 2^x  ->  PoT = x - lb + (f != 0).
      if (!nonfinite && __uint_as_float(mb[c]) > beta)
        P = (int)(mb[c] >> 23) - 127 - lb + ((mb[c] & 0x7FFFFFu) != 0u ? 1 : 0);
      if (nonfinite && valid) flags |= 1;
      if (P > kPotMax) {
        P = kPotMax;
        if (valid) flags |= 2;
      }
      // bins Thr_N = base * 2^(t0 + 2N): PoT <= t0 -> 2 bits, <= t0+2 -> 4, <= t0+4 -> 6, else 8
      const int b = fb ? fb : (P <= t0 ? 2 : P <= t0 + 2 ? 4 : P <= t0 + 4 ? 6 : 8);
      const int fpot = b - 2 - 2 * lb - P;         // Eq. 4 with PCeil = 2^(b-2)
      const float s = exp2_exact(b - 2 - lb - P);  // Eq. 5: s_i = base * 2^FPoT
      int qmx = -128, qmn = 127;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int q = nonfinite ? 0 : __float2int_rn(__fmul_rn(dx[r][c], s));  // stage 3
        qv[r][c] = (int8_t)q;
        qmx = max(qmx, q);
        qmn = min(qmn, q);
      }
      qmx = max(qmx, __shfl_xor_sync(0xffffffffu, qmx, 8));
      qmx = max(qmx, __shfl_xor_sync(0xffffffffu, qmx, 16));
      qmn = min(qmn, __shfl_xor_sync(0xffffffffu, qmn, 8));
      qmn = min(qmn, __shfl_xor_sync(0xffffffffu, qmn, 16));
      fp_c[c] = fpot, b_c[c] = b, qmx_c[c] = qmx, qmn_c[c] = qmn;
      if (valid) fmax = max(fmax, fpot), fmin = min(fmin, fpot);
    }

    if (valid) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int row = rsub * 4 + r;
        if constexpr (VEC == 8) {
          uint2 w;
          w.x = (uint32_t)(uint8_t)qv[r][0] | ((uint32_t)(uint8_t)qv[r][1] << 8) |
                ((uint32_t)(uint8_t)qv[r][2] << 16) | ((uint32_t)(uint8_t)qv[r][3] << 24);
          w.y = (uint32_t)(uint8_t)qv[r][4] | ((uint32_t)(uint8_t)qv[r][5] << 8) |
                ((uint32_t)(uint8_t)qv[r][6] << 16) | ((uint32_t)(uint8_t)qv[r][7] << 24);
          *reinterpret_cast<uint2*>(s_codes + row * cs + c0) = w;
          if (p.debug_codes)
            *reinterpret_cast<uint2*>(p.debug_codes + ((int64_t)t * kTile + row) * K + c0) = w;
        } else {
          uint32_t w = (uint32_t)(uint8_t)qv[r][0] | ((uint32_t)(uint8_t)qv[r][1] << 8) |
                       ((uint32_t)(uint8_t)qv[r][2] << 16) | ((uint32_t)(uint8_t)qv[r][3] << 24);
          *reinterpret_cast<uint32_t*>(s_codes + row * cs + c0) = w;
          if (p.debug_codes)
            *reinterpret_cast<uint32_t*>(p.debug_codes + ((int64_t)t * kTile + row) * K + c0) = w;
        }
      }
      if (rsub == 0) {
#pragma unroll
        for (int c = 0; c < VEC; ++c) {
          s_fpot[c0 + c] = (int8_t)fp_c[c];
          s_bits[c0 + c] = (int8_t)b_c[c];
          s_qmax[c0 + c] = (int8_t)qmx_c[c];
          s_qmin[c0 + c] = (int8_t)qmn_c[c];
        }
      }
    }
  }

  // block reductions: finest / coarsest FPoT, flags
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    fmax = max(fmax, __shfl_xor_sync(0xffffffffu, fmax, o));
    fmin = min(fmin, __shfl_xor_sync(0xffffffffu, fmin, o));
    flags |= __shfl_xor_sync(0xffffffffu, flags, o);
  }
  if (lane == 0) {
    s_small[warp] = fmax;
    s_small[8 + warp] = fmin;
    if (flags) atomicOr(&s_small[24], flags);
  }
  __syncthreads();
  if (tid == 0) {
    int g = -1000, gm = 1000;
    for (int w = 0; w < kQWarps; ++w) g = max(g, s_small[w]), gm = min(gm, s_small[8 + w]);
    s_small[25] = g;
    s_small[26] = gm;
    if (s_small[24]) set_status(p.status, (s_small[24] & 1 ? DSTAR_STATUS_NONFINITE : 0u) |
                                              (s_small[24] & 2 ? DSTAR_STATUS_RANGE : 0u));
  }
  __syncthreads();
  const int g = s_small[25];
  const int gmin = s_small[26];

  // planes the tile needs: every v = q 2^(g - FPoT) must fit the split
  int need = 1;
  for (int64_t k = tid; k < K; k += kQThreads) {
    const int S = g - s_fpot[k];
    const int64_t vmax = (int64_t)s_qmax[k] * ((int64_t)1 << S), vmin = (int64_t)s_qmin[k] * ((int64_t)1 << S);
    if (vmin < kPlane1Lo || vmax > kPlane1Hi) need = max(need, 2);
    if (vmin < kPlane2Lo || vmax > kPlane2Hi) need = 3;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) need = max(need, __shfl_xor_sync(0xffffffffu, need, o));
  if (lane == 0) s_small[16 + warp] = need;
  __syncthreads();
  if (tid == 0) {
    int n = 1;
    for (int w = 0; w < kQWarps; ++w) n = max(n, s_small[16 + w]);
    s_small[27] = n;
  }
  __syncthreads();
  const int planes = s_small[27];

  // ------------------------------------------------- phase 2a: operand planes
  if (planes <= 2) {
    const int64_t vpr = K / 16;  // 16-byte vectors per row
    for (int64_t v = tid; v < 16 * vpr; v += kQThreads) {
      const int row = (int)(v / vpr);
      const int64_t c = (v - row * vpr) * 16;
      const uint4 qraw = *reinterpret_cast<const uint4*>(s_codes + row * cs + c);
      const uint4 fraw = *reinterpret_cast<const uint4*>(s_fpot + c);
      const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
      const uint32_t fw[4] = {fraw.x, fraw.y, fraw.z, fraw.w};
      uint32_t a0w[4], a1w[4];
      bool nz1 = false;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a0w[i] = 0, a1w[i] = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int q = (int)(int8_t)(qw[i] >> (8 * j));
          const int S = g - (int)(int8_t)(fw[i] >> (8 * j));
          const int64_t val = (int64_t)q * ((int64_t)1 << S);  // shift-folded code, exact
          const int a0 = (int)(int8_t)(val & 0xFF);
          const int a1 = (int)((val - a0) >> 8);
          a0w[i] |= (uint32_t)(uint8_t)a0 << (8 * j);
          a1w[i] |= (uint32_t)(uint8_t)a1 << (8 * j);
          nz1 |= a1 != 0;
        }
      }
      const int64_t off = ((int64_t)t * kTile + row) * K + c;
      *reinterpret_cast<uint4*>(p.plane0 + off) = make_uint4(a0w[0], a0w[1], a0w[2], a0w[3]);
      if (planes == 2) {
        *reinterpret_cast<uint4*>(p.plane1 + off) = make_uint4(a1w[0], a1w[1], a1w[2], a1w[3]);
        if (nz1) {
          const int chunk = (int)(c / kChunkK);
          atomicOr(&s_mask[chunk >> 5], 1u << (chunk & 31));
        }
      }
    }
  }

  // ------------------------------------- phase 2b: FPoT-grouped encoded stream
  // Slice j of channel k carries tag FPoT(k) - 2j (j < bits/2).  Tags of the
  // tile lie in [gmin - 6, g]; tag index ti = tag - (gmin - 6).  Each warp owns a
  // contiguous channel range, so (tag, k) order is (tag, warp, chunk, lane).
  const int tlo = gmin - 6;
  const int ntags = g - tlo + 1;  // <= 6 + (g - gmin) + 1 < kMaxTags
  const int64_t kw = K / kQWarps;  // K % 32 == 0 -> a multiple of 4
  const int64_t k_lo = warp * kw, k_hi = (warp == kQWarps - 1) ? K : k_lo + kw;

  // pass A: per-warp count of each tag; lane ti % 32 keeps tag ti in cnt[ti / 32]
  int cnt[2] = {0, 0};
  for (int64_t kb = k_lo; kb < k_hi; kb += 32) {
    const int64_t k = kb + lane;
    const bool kv = k < k_hi;
    const int f = kv ? s_fpot[k] : 0, b = kv ? s_bits[k] : 0;
    for (int ti = 0; ti < ntags; ++ti) {
      const int d = f - (tlo + ti);
      const bool has = kv && d >= 0 && !(d & 1) && (d >> 1) < (b >> 1);
      const uint32_t bal = __ballot_sync(0xffffffffu, has);
      if (lane == (ti & 31)) cnt[ti >> 5] += __popc(bal);
    }
  }
  s_hist[warp * kMaxTags + lane] = cnt[0];
  s_hist[warp * kMaxTags + 32 + lane] = cnt[1];
  __syncthreads();
  // exclusive scan over (tag, warp): warp 0, lane handles tags lane and lane + 32
  if (warp == 0) {
    int tot0 = 0, tot1 = 0;
    for (int w = 0; w < kQWarps; ++w) tot0 += s_hist[w * kMaxTags + lane], tot1 += s_hist[w * kMaxTags + 32 + lane];
    int inc0 = tot0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc0, o);
      if (lane >= o) inc0 += y;
    }
    const int sum0 = __shfl_sync(0xffffffffu, inc0, 31);
    int inc1 = tot1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, inc1, o);
      if (lane >= o) inc1 += y;
    }
    int base0 = inc0 - tot0, base1 = sum0 + inc1 - tot1;
    for (int w = 0; w < kQWarps; ++w) {
      const int h0 = s_hist[w * kMaxTags + lane], h1 = s_hist[w * kMaxTags + 32 + lane];
      s_off[w * kMaxTags + lane] = base0;
      s_off[w * kMaxTags + 32 + lane] = base1;
      base0 += h0, base1 += h1;
    }
    if (lane == 31) s_small[28] = sum0 + inc1;  // total records of the tile
  }
  __syncthreads();

  // pass B: write each record at (tag start) + (rank among earlier channels)
  int off[2] = {s_off[warp * kMaxTags + lane], s_off[warp * kMaxTags + 32 + lane]};
  uint2* rec = p.records + (int64_t)t * p.record_cap;
  for (int64_t kb = k_lo; kb < k_hi; kb += 32) {
    const int64_t k = kb + lane;
    const bool kv = k < k_hi;
    const int f = kv ? s_fpot[k] : 0, b = kv ? s_bits[k] : 0;
    uint32_t word[4] = {0, 0, 0, 0};
    if (kv) {
      const uint32_t msk = (1u << b) - 1u;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t u = (uint32_t)(int)s_codes[i * cs + k] & msk;  // b-bit two's complement
#pragma unroll
        for (int j = 0; j < 4; ++j) word[j] |= ((u >> (2 * j)) & 3u) << (2 * i);
      }
    }
    const uint32_t lt = (1u << lane) - 1u;
    for (int ti = 0; ti < ntags; ++ti) {
      const int tag = tlo + ti;
      const int d = f - tag;
      const bool has = kv && d >= 0 && !(d & 1) && (d >> 1) < (b >> 1);
      const uint32_t bal = __ballot_sync(0xffffffffu, has);
      const int base = __shfl_sync(0xffffffffu, off[ti >> 5], ti & 31);
      if (has) {
        const int j = d >> 1;
        const uint32_t w = j == 0 ? word[0] : j == 1 ? word[1] : j == 2 ? word[2] : word[3];
        rec[base + __popc(bal & lt)] =
            make_uint2(w, (uint32_t)k | ((uint32_t)(uint8_t)(int8_t)tag << 16) | ((uint32_t)j << 24));
      }
      if (lane == (ti & 31)) off[ti >> 5] += __popc(bal);
    }
  }

  // per-sub-channel meta and per-tile meta
  for (int64_t k = tid; k < K; k += kQThreads) {
    p.fpot[(int64_t)t * K + k] = s_fpot[k];
    p.bits[(int64_t)t * K + k] = s_bits[k];
  }
  __syncthreads();  // s_mask complete
  if (tid < p.mask_words) p.mask1[(int64_t)t * p.mask_words + tid] = planes == 2 ? s_mask[tid] : 0u;
  if (tid == 0) {
    p.g_ref[t] = g;
    p.planes[t] = planes;
    p.count[t] = s_small[28];
  }
}

int launch_quantize(const QuantParams& p, int in_bf16, void* stream) {
  const int64_t T = p.M / kTile;
  if (T == 0) return 0;
  const size_t smem = quantize_smem_bytes(p.K);
  cudaError_t e;
  if (in_bf16) {
    e = cudaFuncSetAttribute(quantize_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return (int)e;
    quantize_kernel<__nv_bfloat16><<<(unsigned)T, kQThreads, smem, (cudaStream_t)stream>>>(p);
  } else {
    e = cudaFuncSetAttribute(quantize_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    quantize_kernel<float><<<(unsigned)T, kQThreads, smem, (cudaStream_t)stream>>>(p);
  }
  return (int)cudaGetLastError();
}

}  // namespace fmdq
