// K1: the FMDQ quantizer (DSTAR section 3.1 steps 1-4; the paper's QPU,
// section 4.2 "Design of QPU", stages 1-5).
//
// One 16-token tile is handled by a thread-block cluster of C CTAs (C = 1, 2,
// 4 or 8, chosen so that small batches still fill every SM); CTA r owns a
// contiguous range of channels.  Every thread owns pairs of adjacent channels
// and walks the 16 tokens, so a warp reads whole 128-byte row segments of X_t
// and X_{t-1} and the per-channel max |dX| (stage 1: compare the magnitude
// bits, sign dropped) stays inside the thread.  PoT (Eq. 3), the bit width
// (threshold bins, stage 2), FPoT (Eq. 4) and the codes q = rne(dX s_i) with
// s_i = base 2^FPoT (Eq. 5, stage 3) follow per channel; a channel's 16 codes
// go to shared memory as one 16-byte column.
//
// The tile's finest FPoT (g_ref), its plane count and the per-tag record
// counts are combined across the cluster through distributed shared memory.
// Phase 2 writes (a) the tensor-core operand planes v = q 2^(g_ref - FPoT),
// split into int8 planes v = A0 + 256 A1, and (b) the encoded stream: one
// record per 2-bit slice, ordered by slice FPoT ascending then channel
// ascending (stages 4-5).  A record's position is found by counting, not
// sorting: warp ballots per tag rank the channels of a 32-channel chunk, and
// per-tag counts of warps, CTAs and lower tags give the offsets.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "fmdq_device.cuh"

namespace cg = cooperative_groups;

namespace fmdq {

namespace {

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;
constexpr int kMaxCluster = 8;
constexpr int kMaxMaskWords = (DSTAR_K_MAX / kChunkK + 31) / 32;
constexpr int kTagWin = 8;  // tags ranked per pass (one ballot each)

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

// The four 2-bit slice words of a channel from its 16 codes (byte r of code
// word w = token 4w + r): word j holds field j (bits 2j..2j+1) of every code,
// token i in bits 2i..2i+1.  Each code word is a 4 x 4 matrix of 2-bit cells
// (byte i, field j); two delta swaps transpose it to (byte j, field i), and
// byte permutes gather byte j of the four transposed words.
__device__ __forceinline__ void slice_words(const uint4 cw, uint32_t (&out)[4]) {
  uint32_t tw[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    uint32_t x = tw[w], t;
    t = ((x >> 12) ^ x) & 0x0000F0F0u;  // swap the off-diagonal 2 x 2 blocks of cells
    x ^= t ^ (t << 12);
    t = ((x >> 6) ^ x) & 0x00CC00CCu;   // swap the off-diagonal cells inside each block
    x ^= t ^ (t << 6);
    tw[w] = x;
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t sel = (uint32_t)j | ((uint32_t)(4 + j) << 4);
    const uint32_t lo = __byte_perm(tw[0], tw[1], sel), hi = __byte_perm(tw[2], tw[3], sel);
    out[j] = __byte_perm(lo, hi, 0x5410);
  }
}

__device__ __forceinline__ int code_at(const uint4 cw, int r) {
  const uint32_t w = r < 4 ? cw.x : r < 8 ? cw.y : r < 12 ? cw.z : cw.w;
  return (int)(int8_t)(w >> (8 * (r & 3)));
}

// Window slots ti (tag tw + ti, 0 <= ti < 8) that one channel's slices occupy.
__device__ __forceinline__ uint32_t tag_mask(int f, int b, int tw) {
  uint32_t m = 0;
  for (int j = 0; j < (b >> 1); ++j) {  // slice j has tag f - 2j
    const int ti = f - 2 * j - tw;
    if (ti >= 0 && ti < kTagWin) m |= 1u << ti;
  }
  return m;
}

// Cluster-wide barrier; a plain block barrier when the cluster is one CTA.
__device__ __forceinline__ void csync(cg::cluster_group& cluster, int C) {
  if (C > 1) cluster.sync();
  else __syncthreads();
}

struct QSmem {
  // exchanged across the cluster (read remotely)
  int fmax, fmin, need, pad;
  uint32_t mask[kMaxMaskWords];
  int cta_tot[kTagWin];  // this CTA's record count per tag of the current window
  // local
  int warp_a[kQWarps], warp_b[kQWarps];
  int flags;
  int base[kTagWin];       // records before this CTA's first record of the tag
  int warp_cnt[kQWarps][kTagWin];
  // copies of the cluster's exchanged values, fetched one remote word per thread
  int x_fmax[kMaxCluster], x_fmin[kMaxCluster], x_need[kMaxCluster];
  int x_tot[kMaxCluster][kTagWin];
};

}  // namespace

size_t quantize_smem_bytes(int64_t Kc) {
  size_t b = 20 * (size_t)Kc;  // column-major codes + 4 per-column bytes
  b = (b + 15) & ~(size_t)15;
  return b + sizeof(QSmem);
}

int quantize_cluster_size(int64_t M, int64_t K, int num_sms) {
  const int64_t T = M / kTile;
  const int64_t units = K / 32;
  int c = 1;
  // about 1.5 CTAs per SM when the batch is small, at least 256 channels per CTA
  while (c < kMaxCluster && 2 * T * c < 3LL * num_sms && units / (2 * c) >= 8) c *= 2;
  return c;
}

template <typename TIn>
__global__ void __launch_bounds__(kQThreads, 2) quantize_kernel(const QuantParams p, int C, int64_t kc_max) {
  extern __shared__ __align__(16) uint8_t smem[];
  using PR = Pair<TIn>;
  cg::cluster_group cluster = cg::this_cluster();

  const int64_t K = p.K;
  const int rank = (int)cluster.block_rank();
  const int t = (int)(blockIdx.x / C);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t units = K / 32;
  const int64_t k_lo = 32 * (rank * units / C), k_hi = 32 * ((rank + 1) * units / C);
  const int64_t Kc = k_hi - k_lo;

  int8_t* s_code = reinterpret_cast<int8_t*>(smem);  // [Kc][16]: the 16 codes of local channel k
  int8_t* s_fpot = s_code + 16 * kc_max;              // [Kc]
  int8_t* s_bits = s_fpot + kc_max;
  int8_t* s_qmax = s_bits + kc_max;
  int8_t* s_qmin = s_qmax + kc_max;
  QSmem& S = *reinterpret_cast<QSmem*>(smem + ((20 * kc_max + 15) & ~(int64_t)15));

  if (tid < kMaxMaskWords) S.mask[tid] = 0;
  if (tid == 0) S.flags = 0;
  pdl_launch_dependents();
  pdl_wait();  // nothing of global memory is touched before the previous kernel completed
  __syncthreads();

  const int lb = p.lb, t0 = p.t0, fb = p.force_bits;
  const float beta = exp2_exact(lb);
  const bool refresh = !(p.flags & DSTAR_FLAG_NO_XPREV_REFRESH);
  const int64_t row0 = (int64_t)t * kTile;
  const int npairs = (int)(Kc / 2);
  int fmax = -1000, fmin = 1000;
  int flags = 0;

  // ---------------------------------------------------------------- phase 1
  for (int pr = tid; pr < npairs; pr += kQThreads) {
    const int64_t lc = 2 * (int64_t)pr, c = k_lo + lc;
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
    // Eq. 1 (one fp32 subtraction per element) and stage 1 on the magnitude bits
    uint32_t m0 = 0, m1 = 0;
#pragma unroll
    for (int r = 0; r < kTile; ++r) {
      m0 = max(m0, __float_as_uint(__fsub_rn(PR::lo(rt[r]), PR::lo(rp[r]))) & 0x7FFFFFFFu);
      m1 = max(m1, __float_as_uint(__fsub_rn(PR::hi(rt[r]), PR::hi(rp[r]))) & 0x7FFFFFFFu);
    }
    const ColParams c0 = col_params(m0, lb, beta, t0, fb, flags);
    const ColParams c1 = col_params(m1, lb, beta, t0, fb, flags);
    uint32_t w0[4] = {0, 0, 0, 0}, w1[4] = {0, 0, 0, 0};
    int qmx0 = -128, qmn0 = 127, qmx1 = -128, qmn1 = 127;
#pragma unroll
    for (int r = 0; r < kTile; ++r) {  // stage 3 (dX recomputed: the same single subtraction)
      const float d0 = __fsub_rn(PR::lo(rt[r]), PR::lo(rp[r])), d1 = __fsub_rn(PR::hi(rt[r]), PR::hi(rp[r]));
      const int q0 = c0.nonfinite ? 0 : __float2int_rn(__fmul_rn(d0, c0.scale));
      const int q1 = c1.nonfinite ? 0 : __float2int_rn(__fmul_rn(d1, c1.scale));
      w0[r >> 2] |= ((uint32_t)q0 & 0xFFu) << (8 * (r & 3));
      w1[r >> 2] |= ((uint32_t)q1 & 0xFFu) << (8 * (r & 3));
      qmx0 = max(qmx0, q0), qmn0 = min(qmn0, q0);
      qmx1 = max(qmx1, q1), qmn1 = min(qmn1, q1);
    }
    if (p.debug_codes) {
#pragma unroll
      for (int r = 0; r < kTile; ++r)
        *reinterpret_cast<uint16_t*>(p.debug_codes + (row0 + r) * K + c) =
            (uint16_t)(((w0[r >> 2] >> (8 * (r & 3))) & 0xFFu) | (((w1[r >> 2] >> (8 * (r & 3))) & 0xFFu) << 8));
    }
    *reinterpret_cast<uint4*>(s_code + 16 * lc) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
    *reinterpret_cast<uint4*>(s_code + 16 * lc + 16) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
    auto two = [](int a, int b) { return (uint16_t)(((uint32_t)a & 0xFFu) | (((uint32_t)b & 0xFFu) << 8)); };
    *reinterpret_cast<uint16_t*>(s_fpot + lc) = two(c0.fpot, c1.fpot);
    *reinterpret_cast<uint16_t*>(s_bits + lc) = two(c0.bits, c1.bits);
    *reinterpret_cast<uint16_t*>(s_qmax + lc) = two(qmx0, qmx1);
    *reinterpret_cast<uint16_t*>(s_qmin + lc) = two(qmn0, qmn1);
    *reinterpret_cast<uint16_t*>(p.fpot + (int64_t)t * K + c) = two(c0.fpot, c1.fpot);
    *reinterpret_cast<uint16_t*>(p.bits + (int64_t)t * K + c) = two(c0.bits, c1.bits);
    fmax = max(fmax, max(c0.fpot, c1.fpot));
    fmin = min(fmin, min(c0.fpot, c1.fpot));
  }

  // CTA reductions, then the cluster's finest / coarsest FPoT
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    fmax = max(fmax, __shfl_xor_sync(0xffffffffu, fmax, o));
    fmin = min(fmin, __shfl_xor_sync(0xffffffffu, fmin, o));
    flags |= __shfl_xor_sync(0xffffffffu, flags, o);
  }
  if (lane == 0) {
    S.warp_a[warp] = fmax;
    S.warp_b[warp] = fmin;
    if (flags) atomicOr(&S.flags, flags);
  }
  __syncthreads();
  if (tid == 0) {
    int a = -1000, b = 1000;
    for (int w = 0; w < kQWarps; ++w) a = max(a, S.warp_a[w]), b = min(b, S.warp_b[w]);
    S.fmax = a, S.fmin = b;
    if (S.flags)
      set_status(p.status, (S.flags & 1 ? DSTAR_STATUS_NONFINITE : 0u) | (S.flags & 2 ? DSTAR_STATUS_RANGE : 0u));
  }
  csync(cluster, C);
  if (tid < C) {  // one remote read per thread, all in flight together
    const QSmem* R = C > 1 ? cluster.map_shared_rank(&S, tid) : &S;
    S.x_fmax[tid] = R->fmax;
    S.x_fmin[tid] = R->fmin;
  }
  __syncthreads();
  int g = -1000, gmin = 1000;
  for (int q = 0; q < C; ++q) g = max(g, S.x_fmax[q]), gmin = min(gmin, S.x_fmin[q]);

  // planes the tile needs: every v = q 2^(g - FPoT) must fit the split
  int need = 1;
  for (int64_t k = tid; k < Kc; k += kQThreads) {
    const int Sh = g - s_fpot[k];
    const int64_t vmax = (int64_t)s_qmax[k] * ((int64_t)1 << Sh), vmin = (int64_t)s_qmin[k] * ((int64_t)1 << Sh);
    if (vmin < kPlane1Lo || vmax > kPlane1Hi) need = max(need, 2);
    if (vmin < kPlane2Lo || vmax > kPlane2Hi) need = 3;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) need = max(need, __shfl_xor_sync(0xffffffffu, need, o));
  if (lane == 0) S.warp_a[warp] = need;
  __syncthreads();
  if (tid == 0) {
    int n = 1;
    for (int w = 0; w < kQWarps; ++w) n = max(n, S.warp_a[w]);
    S.need = n;
  }
  csync(cluster, C);
  if (tid < C) S.x_need[tid] = (C > 1 ? cluster.map_shared_rank(&S, tid) : &S)->need;
  __syncthreads();
  int planes = 1;
  for (int q = 0; q < C; ++q) planes = max(planes, S.x_need[q]);

  // ------------------------------------------------- phase 2a: operand planes
  // Same channel-pair mapping: 2-byte stores, a warp writes 64 contiguous bytes per row.
  if (planes == 1) {
    for (int pr = tid; pr < npairs; pr += kQThreads) {
      const int64_t lc = 2 * (int64_t)pr, c = k_lo + lc;
      const uint4 q0 = *reinterpret_cast<const uint4*>(s_code + 16 * lc);
      const uint4 q1 = *reinterpret_cast<const uint4*>(s_code + 16 * lc + 16);
      // a nonzero code of a one-plane tile has a shift <= 7; zero codes stay zero
      const int S0 = min(g - s_fpot[lc], 31), S1 = min(g - s_fpot[lc + 1], 31);
#pragma unroll
      for (int r = 0; r < kTile; ++r) {
        const uint32_t a = (((uint32_t)code_at(q0, r) << S0) & 0xFFu) | ((((uint32_t)code_at(q1, r) << S1) & 0xFFu) << 8);
        *reinterpret_cast<uint16_t*>(p.plane0 + (row0 + r) * K + c) = (uint16_t)a;
      }
    }
  } else if (planes == 2) {
    for (int pr = tid; pr < npairs; pr += kQThreads) {
      const int64_t lc = 2 * (int64_t)pr, c = k_lo + lc;
      const uint4 q0 = *reinterpret_cast<const uint4*>(s_code + 16 * lc);
      const uint4 q1 = *reinterpret_cast<const uint4*>(s_code + 16 * lc + 16);
      // a nonzero code of a two-plane tile has a shift <= 15, so v fits 32 bits
      const int S0 = min(g - s_fpot[lc], 24), S1 = min(g - s_fpot[lc + 1], 24);
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
      if (nz) {
        const int chunk = (int)(c / kChunkK);
        atomicOr(&S.mask[chunk >> 5], 1u << (chunk & 31));
      }
    }
  }

  // ------------------------------------- phase 2b: FPoT-grouped encoded stream
  // Slice j of channel k carries tag FPoT(k) - 2j (j < bits/2).  Tags lie in
  // [gmin - 6, g] and are handled in windows of 8 consecutive tags.  Each warp
  // owns a contiguous range of this CTA's channels and walks it 32 channels
  // at a time (lane = channel); one ballot per tag of the window ranks the
  // lanes carrying that tag.  The record of (tag, k) lands after: the tile's
  // records of lower tags, then those of the same tag in lower-ranked CTAs,
  // lower warps of this CTA, earlier chunks of this warp and lower lanes.
  const int tlo = gmin - 6;
  const int ntags = g - tlo + 1;
  const int64_t kw = ((Kc / 32 + kQWarps - 1) / kQWarps) * 32;  // channels per warp, a multiple of 32
  const int64_t w_lo = min(Kc, (int64_t)warp * kw), w_hi = min(Kc, w_lo + kw);
  const uint32_t lt = (1u << lane) - 1u;
  uint2* rec = p.records + (int64_t)t * p.record_cap;
  int records_before_window = 0;  // all CTAs, all lower tags (kept by threads tid < kTagWin)
  for (int wbase = 0; wbase < ntags; wbase += kTagWin) {
    const int tw = tlo + wbase;  // tag of window slot 0
    // pass A: this warp's count of each tag of the window
    int cnt[kTagWin];
#pragma unroll
    for (int ti = 0; ti < kTagWin; ++ti) cnt[ti] = 0;
    for (int64_t kb = w_lo; kb < w_hi; kb += 4 * 32) {  // four independent chunks per iteration
      uint32_t m[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t k = kb + 32 * u + lane;
        m[u] = k < w_hi ? tag_mask(s_fpot[k], s_bits[k], tw) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int ti = 0; ti < kTagWin; ++ti) cnt[ti] += __popc(__ballot_sync(0xffffffffu, (m[u] >> ti) & 1u));
    }
    if (lane == 0) {
#pragma unroll
      for (int ti = 0; ti < kTagWin; ++ti) S.warp_cnt[warp][ti] = cnt[ti];
    }
    __syncthreads();
    if (tid < kTagWin) {
      int tot = 0;
      for (int w = 0; w < kQWarps; ++w) tot += S.warp_cnt[w][tid];
      S.cta_tot[tid] = tot;
    }
    csync(cluster, C);
    // window totals of every CTA -> where this CTA's records of each tag start
    if (tid < C * kTagWin) {
      const int q = tid / kTagWin, u = tid % kTagWin;
      S.x_tot[q][u] = (C > 1 ? cluster.map_shared_rank(&S, q) : &S)->cta_tot[u];
    }
    __syncthreads();
    if (tid < kTagWin) {
      int below = 0, lower_cta = 0, all = 0;
      for (int q = 0; q < C; ++q) {
        for (int u = 0; u < kTagWin; ++u) {
          const int v = S.x_tot[q][u];
          if (u < tid) below += v;
          if (u == tid && q < rank) lower_cta += v;
          all += v;
        }
      }
      S.base[tid] = records_before_window + below + lower_cta;
      records_before_window += all;
    }
    __syncthreads();
    int off[kTagWin];
#pragma unroll
    for (int ti = 0; ti < kTagWin; ++ti) {
      int o = S.base[ti];
      for (int w = 0; w < warp; ++w) o += S.warp_cnt[w][ti];
      off[ti] = o;
    }
    // pass B: rank and write, two independent chunks per iteration
    for (int64_t kb = w_lo; kb < w_hi; kb += 2 * 32) {
      int f[2], b[2];
      uint32_t m[2], bal[2][kTagWin], words[2][4];
      int64_t k[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        k[u] = kb + 32 * u + lane;
        const bool kv = k[u] < w_hi;
        f[u] = kv ? s_fpot[k[u]] : 0, b[u] = kv ? s_bits[k[u]] : 0;
        m[u] = kv ? tag_mask(f[u], b[u], tw) : 0u;
        if (m[u]) slice_words(*reinterpret_cast<const uint4*>(s_code + 16 * k[u]), words[u]);
#pragma unroll
        for (int ti = 0; ti < kTagWin; ++ti) bal[u][ti] = __ballot_sync(0xffffffffu, (m[u] >> ti) & 1u);
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (m[u]) {
#pragma unroll
          for (int ti = 0; ti < kTagWin; ++ti) {
            if ((m[u] >> ti) & 1u) {
              // the field j < b/2 of the b-bit pattern equals that of the 8-bit pattern
              const int j = (f[u] - tw - ti) >> 1;
              const uint32_t w = j == 0 ? words[u][0] : j == 1 ? words[u][1] : j == 2 ? words[u][2] : words[u][3];
              rec[off[ti] + __popc(bal[u][ti] & lt)] = make_uint2(
                  w, (uint32_t)(k_lo + k[u]) | ((uint32_t)(uint8_t)(int8_t)(tw + ti) << 16) | ((uint32_t)j << 24));
            }
          }
        }
#pragma unroll
        for (int ti = 0; ti < kTagWin; ++ti) off[ti] += __popc(bal[u][ti]);
      }
    }
    csync(cluster, C);  // cta_tot and warp_cnt are rewritten by the next window
  }

  // the tile's meta: rank 0 gathers the cluster's mask words
  __syncthreads();
  if (rank == 0) {
    if (tid < p.mask_words) {
      uint32_t m = 0;
      for (int q = 0; q < C; ++q) m |= (C > 1 ? cluster.map_shared_rank(&S, q) : &S)->mask[tid];
      p.mask1[(int64_t)t * p.mask_words + tid] = planes == 2 ? m : 0u;
    }
    if (tid == 0) {
      p.g_ref[t] = g;
      p.planes[t] = planes;
      p.count[t] = records_before_window;
    }
  }
  csync(cluster, C);  // no CTA leaves while another may still read its shared memory
}

int launch_quantize(const QuantParams& p, int in_bf16, int num_sms, void* stream) {
  const int64_t T = p.M / kTile;
  if (T == 0) return 0;
  const int C = quantize_cluster_size(p.M, p.K, num_sms);
  const int64_t units = p.K / 32;
  const int64_t kc_max = 32 * ((units + C - 1) / C);
  const size_t smem = quantize_smem_bytes(kc_max);
  const int smem_max = (int)quantize_smem_bytes(DSTAR_K_MAX);  // one setting serves every K
  const void* fn = in_bf16 ? (const void*)quantize_kernel<__nv_bfloat16> : (const void*)quantize_kernel<float>;
  int e = ensure_max_smem(fn, smem_max);
  if (e != 0) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(T * C), 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the launch with the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t ce;
  if (in_bf16) ce = cudaLaunchKernelEx(&cfg, quantize_kernel<__nv_bfloat16>, p, C, kc_max);
  else ce = cudaLaunchKernelEx(&cfg, quantize_kernel<float>, p, C, kc_max);
  if (ce != cudaSuccess) return (int)ce;
  return (int)cudaGetLastError();
}

}  // namespace fmdq
