// K1: the FMDQ quantizer (DSTAR section 3.1 steps 1-4; the paper's QPU,
// section 4.2 "Design of QPU", stages 1-5).
//
// One 256-thread block per 16-token tile.  Phase 1: every thread owns a pair
// of adjacent channels and walks the 16 tokens of the tile, so a warp reads
// whole 128-byte row segments of X_t and X_{t-1} and the per-channel max
// |dX| (stage 1: compare the magnitude bits, sign dropped) stays inside the
// thread.  PoT (Eq. 3), the bit width (threshold bins, stage 2), FPoT (Eq. 4)
// and the codes q = rne(dX * s_i) with s_i = base * 2^FPoT (Eq. 5, stage 3)
// follow per channel; the 16 codes of a channel go to shared memory as one
// 16-byte column.  Phase 2 knows the tile's finest FPoT (g_ref) and writes
// (a) the tensor-core operand planes v = q * 2^(g_ref - FPoT), split into int8
// planes v = A0 + 256 A1, and (b) the encoded stream: one record per 2-bit
// slice, grouped by slice FPoT ascending then channel ascending (stages 4-5),
// placed by per-tag counts and an exclusive scan rather than a sort.
#include <cuda_bf16.h>

#include "fmdq_device.cuh"

namespace fmdq {

namespace {

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;
constexpr int kMaxTags = 64;  // tag spread within a tile is at most 6 + kPotMax + 6 < 64
constexpr int kMaxMaskWords = (DSTAR_K_MAX / kChunkK + 31) / 32;

// Two adjacent channels of one token row.
template <typename TIn>
struct Pair;
template <>
struct Pair<__nv_bfloat16> {
  using Raw = uint32_t;
  __device__ static Raw load(const void* base, int64_t off) {
    return *reinterpret_cast<const uint32_t*>(static_cast<const __nv_bfloat16*>(base) + off);
  }
  __device__ static void store(void* base, int64_t off, Raw r) {
    *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(base) + off) = r;
  }
  // bf16 -> fp32 is exact: the bf16 bits are the high half of the fp32 word
  __device__ static float lo(Raw r) { return __uint_as_float(r << 16); }
  __device__ static float hi(Raw r) { return __uint_as_float(r & 0xFFFF0000u); }
};
template <>
struct Pair<float> {
  using Raw = uint2;
  __device__ static Raw load(const void* base, int64_t off) {
    return *reinterpret_cast<const uint2*>(static_cast<const float*>(base) + off);
  }
  __device__ static void store(void* base, int64_t off, Raw r) {
    *reinterpret_cast<uint2*>(static_cast<float*>(base) + off) = r;
  }
  __device__ static float lo(Raw r) { return __uint_as_float(r.x); }
  __device__ static float hi(Raw r) { return __uint_as_float(r.y); }
};

__device__ __forceinline__ float exp2_exact(int e) {  // 2^e for e in the normal range
  return __int_as_float((127 + e) << 23);
}

// Per-channel parameters from the magnitude bits of M_i (section 3.1 step 1).
struct ColParams {
  int fpot, bits;
  float scale;
  bool nonfinite;
};

__device__ __forceinline__ ColParams col_params(uint32_t mbits, int lb, float beta, int t0, int fb, int& flags) {
  ColParams cp;
  cp.nonfinite = mbits >= 0x7F800000u;
  int P = 0;
  // Eq. 3 with the static base: PoT = ceil(log2(M_i / base)), 0 when M_i <= base.
  // M_i > base >= 2^-32 is a normal float: M_i = (1 + f) 2^x  ->  PoT = x - lb + (f != 0).
  if (!cp.nonfinite && __uint_as_float(mbits) > beta)
    P = (int)(mbits >> 23) - 127 - lb + ((mbits & 0x7FFFFFu) != 0u ? 1 : 0);
  if (cp.nonfinite) flags |= 1;
  if (P > kPotMax) {
    P = kPotMax;
    flags |= 2;
  }
  // bins Thr_N = base * 2^(t0 + 2N): PoT <= t0 -> 2 bits, <= t0+2 -> 4, <= t0+4 -> 6, else 8
  cp.bits = fb ? fb : (P <= t0 ? 2 : P <= t0 + 2 ? 4 : P <= t0 + 4 ? 6 : 8);
  cp.fpot = cp.bits - 2 - 2 * lb - P;          // Eq. 4 with PCeil = 2^(b-2)
  cp.scale = exp2_exact(cp.bits - 2 - lb - P);  // Eq. 5: s_i = base * 2^FPoT
  return cp;
}

// The 2-bit field j of the 16 codes of a channel (byte r of word w = token
// 4w + r), gathered into one word: token i in bits 2i..2i+1.
__device__ __forceinline__ uint32_t slice_word(const uint4 cw, int j) {
  const uint32_t ws[4] = {cw.x, cw.y, cw.z, cw.w};
  uint32_t out = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t x = (ws[w] >> (2 * j)) & 0x03030303u;
    x = (x | (x >> 6)) & 0x000F000Fu;
    x = (x | (x >> 12)) & 0xFFu;
    out |= x << (8 * w);
  }
  return out;
}

__device__ __forceinline__ int code_at(const uint4 cw, int r) {
  const uint32_t w = r < 4 ? cw.x : r < 8 ? cw.y : r < 12 ? cw.z : cw.w;
  return (int)(int8_t)(w >> (8 * (r & 3)));
}

}  // namespace

size_t quantize_smem_bytes(int64_t K) {
  size_t b = 16 * (size_t)K + 4 * (size_t)K;  // column-major codes + 4 per-column bytes
  b = (b + 15) & ~(size_t)15;
  b += sizeof(int) * (64 + 2 * kQWarps * kMaxTags) + sizeof(uint32_t) * kMaxMaskWords;
  return b;
}

template <typename TIn>
__global__ void __launch_bounds__(kQThreads, 2) quantize_kernel(const QuantParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  using PR = Pair<TIn>;

  const int64_t K = p.K;
  const int t = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  int8_t* s_code = reinterpret_cast<int8_t*>(smem);  // [K][16]: the 16 codes of channel k
  int8_t* s_fpot = s_code + 16 * K;                   // [K]
  int8_t* s_bits = s_fpot + K;
  int8_t* s_qmax = s_bits + K;
  int8_t* s_qmin = s_qmax + K;
  int* s_small = reinterpret_cast<int*>(smem + ((20 * K + 15) & ~(int64_t)15));
  int* s_hist = s_small + 64;                  // [warps][kMaxTags]
  int* s_off = s_hist + kQWarps * kMaxTags;    // [warps][kMaxTags]
  uint32_t* s_mask = reinterpret_cast<uint32_t*>(s_off + kQWarps * kMaxTags);
  // s_small: [0,8) warp max FPoT, [8,16) warp min FPoT, [16,24) warp plane need,
  //          [24] flags (1 nonfinite, 2 range), [25] g_ref, [26] min FPoT, [27] planes, [28] records

  if (tid < kMaxMaskWords) s_mask[tid] = 0;
  if (tid == 0) s_small[24] = 0;
  __syncthreads();

  const int lb = p.lb, t0 = p.t0, fb = p.force_bits;
  const float beta = exp2_exact(lb);
  const bool refresh = !(p.flags & DSTAR_FLAG_NO_XPREV_REFRESH);
  const int64_t row0 = (int64_t)t * kTile;
  const int npairs = (int)(K / 2);
  int fmax = -1000, fmin = 1000;
  int flags = 0;

  // ---------------------------------------------------------------- phase 1
  for (int pr = tid; pr < npairs; pr += kQThreads) {
    const int64_t c = 2 * (int64_t)pr;
    typename PR::Raw rt[kTile], rp[kTile];
#pragma unroll
    for (int r = 0; r < kTile; ++r) {
      rt[r] = PR::load(p.x_t, (row0 + r) * p.ld_xt + c);
      rp[r] = PR::load(p.x_prev, (row0 + r) * p.ld_xp + c);
    }
    if (refresh) {
#pragma unroll
      for (int r = 0; r < kTile; ++r) PR::store(p.x_prev, (row0 + r) * p.ld_xp + c, rt[r]);
    }
    float d0[kTile], d1[kTile];
    uint32_t m0 = 0, m1 = 0;
#pragma unroll
    for (int r = 0; r < kTile; ++r) {
      d0[r] = __fsub_rn(PR::lo(rt[r]), PR::lo(rp[r]));  // Eq. 1, one fp32 subtraction
      d1[r] = __fsub_rn(PR::hi(rt[r]), PR::hi(rp[r]));
      m0 = max(m0, __float_as_uint(d0[r]) & 0x7FFFFFFFu);  // stage 1 on the magnitude bits
      m1 = max(m1, __float_as_uint(d1[r]) & 0x7FFFFFFFu);
    }
    const ColParams c0 = col_params(m0, lb, beta, t0, fb, flags);
    const ColParams c1 = col_params(m1, lb, beta, t0, fb, flags);
    uint32_t w0[4] = {0, 0, 0, 0}, w1[4] = {0, 0, 0, 0};
    int qmx0 = -128, qmn0 = 127, qmx1 = -128, qmn1 = 127;
#pragma unroll
    for (int r = 0; r < kTile; ++r) {
      const int q0 = c0.nonfinite ? 0 : __float2int_rn(__fmul_rn(d0[r], c0.scale));  // stage 3
      const int q1 = c1.nonfinite ? 0 : __float2int_rn(__fmul_rn(d1[r], c1.scale));
      w0[r >> 2] |= ((uint32_t)q0 & 0xFFu) << (8 * (r & 3));
      w1[r >> 2] |= ((uint32_t)q1 & 0xFFu) << (8 * (r & 3));
      qmx0 = max(qmx0, q0), qmn0 = min(qmn0, q0);
      qmx1 = max(qmx1, q1), qmn1 = min(qmn1, q1);
      if (p.debug_codes)
        *reinterpret_cast<uint16_t*>(p.debug_codes + (row0 + r) * K + c) =
            (uint16_t)(((uint32_t)q0 & 0xFFu) | (((uint32_t)q1 & 0xFFu) << 8));
    }
    *reinterpret_cast<uint4*>(s_code + 16 * c) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4*>(s_code + 16 * c + 16) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    auto two = [](int a, int b) { return (uint16_t)(((uint32_t)a & 0xFFu) | (((uint32_t)b & 0xFFu) << 8)); };
    *reinterpret_cast<uint16_t*>(s_fpot + c) = two(c0.fpot, c1.fpot);
    *reinterpret_cast<uint16_t*>(s_bits + c) = two(c0.bits, c1.bits);
    *reinterpret_cast<uint16_t*>(s_qmax + c) = two(qmx0, qmx1);
    *reinterpret_cast<uint16_t*>(s_qmin + c) = two(qmn0, qmn1);
    fmax = max(fmax, max(c0.fpot, c1.fpot));
    fmin = min(fmin, min(c0.fpot, c1.fpot));
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
  // Same channel-pair mapping: 2-byte stores, a warp writes 64 contiguous bytes per row.
  if (planes == 1) {
    for (int pr = tid; pr < npairs; pr += kQThreads) {
      const int64_t c = 2 * (int64_t)pr;
      const uint4 q0 = *reinterpret_cast<const uint4*>(s_code + 16 * c);
      const uint4 q1 = *reinterpret_cast<const uint4*>(s_code + 16 * c + 16);
      // a nonzero code of a one-plane tile has a shift <= 7; zero codes stay zero
      const int S0 = min(g - s_fpot[c], 31), S1 = min(g - s_fpot[c + 1], 31);
#pragma unroll
      for (int r = 0; r < kTile; ++r) {
        const uint32_t a = (((uint32_t)code_at(q0, r) << S0) & 0xFFu) | ((((uint32_t)code_at(q1, r) << S1) & 0xFFu) << 8);
        *reinterpret_cast<uint16_t*>(p.plane0 + (row0 + r) * K + c) = (uint16_t)a;
      }
    }
  } else if (planes == 2) {
    for (int pr = tid; pr < npairs; pr += kQThreads) {
      const int64_t c = 2 * (int64_t)pr;
      const uint4 q0 = *reinterpret_cast<const uint4*>(s_code + 16 * c);
      const uint4 q1 = *reinterpret_cast<const uint4*>(s_code + 16 * c + 16);
      // a nonzero code of a two-plane tile has a shift <= 15, so v fits 32 bits
      const int S0 = min(g - s_fpot[c], 24), S1 = min(g - s_fpot[c + 1], 24);
      uint32_t nz = 0;
#pragma unroll
      for (int r = 0; r < kTile; ++r) {
        const int v0 = code_at(q0, r) * (1 << S0), v1 = code_at(q1, r) * (1 << S1);
        const int a00 = (int)(int8_t)(v0 & 0xFF), a01 = (int)(int8_t)(v1 & 0xFF);
        const int a10 = (v0 - a00) >> 8, a11 = (v1 - a01) >> 8;
        nz |= (uint32_t)(a10 | a11);
        *reinterpret_cast<uint16_t*>(p.plane0 + (row0 + r) * K + c) =
            (uint16_t)(((uint32_t)a00 & 0xFFu) | (((uint32_t)a01 & 0xFFu) << 8));
        *reinterpret_cast<uint16_t*>(p.plane1 + (row0 + r) * K + c) =
            (uint16_t)(((uint32_t)a10 & 0xFFu) | (((uint32_t)a11 & 0xFFu) << 8));
      }
      // a warp's 32 pairs are 64 aligned channels: one K chunk
      const uint32_t bal = __ballot_sync(__activemask(), nz != 0);
      if (bal && nz && (__ffs(bal) - 1) == lane) {
        const int chunk = (int)(c / kChunkK);
        atomicOr(&s_mask[chunk >> 5], 1u << (chunk & 31));
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
    uint4 cw = make_uint4(0, 0, 0, 0);
    if (kv) {
      cw = *reinterpret_cast<const uint4*>(s_code + 16 * k);
      p.fpot[(int64_t)t * K + k] = (int8_t)f;
      p.bits[(int64_t)t * K + k] = (int8_t)b;
    }
    const uint32_t lt = (1u << lane) - 1u;
    for (int ti = 0; ti < ntags; ++ti) {
      const int tag = tlo + ti;
      const int d = f - tag;
      const bool has = kv && d >= 0 && !(d & 1) && (d >> 1) < (b >> 1);
      const uint32_t bal = __ballot_sync(0xffffffffu, has);
      const int base = __shfl_sync(0xffffffffu, off[ti >> 5], ti & 31);
      if (has) {
        // the field j < b/2 of the b-bit pattern equals that of the 8-bit pattern
        const int j = d >> 1;
        rec[base + __popc(bal & lt)] =
            make_uint2(slice_word(cw, j), (uint32_t)k | ((uint32_t)(uint8_t)(int8_t)tag << 16) | ((uint32_t)j << 24));
      }
      if (lane == (ti & 31)) off[ti >> 5] += __popc(bal);
    }
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
  const int smem_max = (int)quantize_smem_bytes(DSTAR_K_MAX);  // one setting serves every K
  int e;
  if (in_bf16) {
    if ((e = ensure_max_smem((const void*)quantize_kernel<__nv_bfloat16>, smem_max)) != 0) return e;
    quantize_kernel<__nv_bfloat16><<<(unsigned)T, kQThreads, smem, (cudaStream_t)stream>>>(p);
  } else {
    if ((e = ensure_max_smem((const void*)quantize_kernel<float>, smem_max)) != 0) return e;
    quantize_kernel<float><<<(unsigned)T, kQThreads, smem, (cudaStream_t)stream>>>(p);
  }
  return (int)cudaGetLastError();
}

}  // namespace fmdq
