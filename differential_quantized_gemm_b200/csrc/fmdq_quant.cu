// K1: the FMDQ quantizer (DSTAR section 3.1 steps 1-4; the paper's QPU,
// section 4.2 "Design of QPU", stages 1-5).
//
// Two kernels share the per-tile stages.  For small batches one 16-token tile
// is handled by a thread-block cluster of C CTAs (C = 1, 2, 4 or 8, chosen so
// that small batches still fill every SM); CTA r owns a contiguous range of
// channels.  For batches of at least two tiles per SM a persistent kernel
// runs phase 1 of one tile and phase 2 of the previous one at the same time
// (see quantize_persistent_kernel).  Every thread owns pairs of adjacent channels
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

// Occupancy settings of the quantizer (compile-time; the defaults are the
// measured best on B200): CTAs per SM the register budget is sized for,
// whether phase 1 keeps the next channel pair's loads in flight, and the
// channel count per CTA above which a tile is split over a cluster even when
// the grid already fills the GPU (0: only to fill the GPU).
#ifndef FMDQ_Q_MIN_BLOCKS
#define FMDQ_Q_MIN_BLOCKS 2
#endif
#ifndef FMDQ_Q_PREFETCH
#define FMDQ_Q_PREFETCH 1
#endif
#ifndef FMDQ_Q_SPLIT_K
#define FMDQ_Q_SPLIT_K 0
#endif

constexpr int kQThreads = 256;
constexpr int kQWarps = kQThreads / 32;
constexpr int kMaxCluster = 8;
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
  __device__ static Raw zero() { return 0u; }
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
  __device__ static Raw zero() { return make_uint2(0u, 0u); }
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

// Normalised form of a positive finite float: value = (sig / 2^23) * 2^exp
// with sig in [2^23, 2^24); subnormals are normalised too.
__device__ __forceinline__ int norm_float(uint32_t bits, uint32_t& sig) {
  const int e = (int)(bits >> 23);
  const uint32_t m = bits & 0x7FFFFFu;
  if (e == 0) {
    const int sh = __clz(m) - 8;
    sig = m << sh;
    return -126 - sh;
  }
  sig = m | 0x800000u;
  return e - 127;
}

// a / b rounded to nearest for one divisor b shared by a whole call (the
// dynamic base), from r = RN(1/b) (CUDA's __frcp_rn) and FMAs: y0 = RN(a r)
// lies within 2 ulp of a/b; one Newton-Raphson correction with the exact
// FMA residual, y1 = RN(y0 + (a - y0 b) r), makes it faithful; then
// Markstein's theorem (IBM J. Res. Dev. 34(1), 1990: for a faithful y and a
// correctly rounded reciprocal r, RN(y + (a - y b) r) is the correctly
// rounded quotient, the residual being exact) gives q.  Used while b lies in
// [2^-100, 2^100], where no product, residual or reciprocal leaves the
// normal range for the quotients that decide codes; otherwise the IEEE
// division itself.  dstar_fmdq_selftest_div compares it with __fdiv_rn.
struct DivBy {
  float b, r;
  bool fast;
};
__device__ __forceinline__ DivBy div_by_setup(float b) {
  DivBy d;
  d.b = b;
  d.r = __frcp_rn(b);
  const float ab = fabsf(b);
  d.fast = ab >= 0x1p-100f && ab <= 0x1p100f;
  return d;
}
__device__ __forceinline__ float div_by(float a, const DivBy& d) {
  if (!d.fast) return __fdiv_rn(a, d.b);
  const float y0 = __fmul_rn(a, d.r);
  const float y1 = __fmaf_rn(__fmaf_rn(-y0, d.b, a), d.r, y0);
  return __fmaf_rn(__fmaf_rn(-y1, d.b, a), d.r, y1);
}

// Per-channel parameters with the dynamic base (FMDQ-DYN): PoT =
// ceil(log2(M_i / base)) exactly, from the normalised exponents and
// significands; the width from the predefined thresholds M_i <= 2^(thr + 2N)
// (thr = lb + t0), i.e. ceil(log2 M_i) <= thr + 2N; FPoT relative to the base.
// The code scale is 2^(b-2-PoT), applied to fl32(dX / base).
__device__ __forceinline__ ColParams col_params_dyn(uint32_t mbits, uint32_t bbits, int thr, int fb, int& flags) {
  ColParams cp;
  cp.nonfinite = mbits >= 0x7F800000u;
  int P = 0, b;
  if (cp.nonfinite) flags |= 1;
  if (!cp.nonfinite && mbits != 0u) {
    uint32_t sm, sb;
    const int em = norm_float(mbits, sm), eb = norm_float(bbits, sb);
    P = max(em - eb + (sm > sb ? 1 : 0), 0);
    if (P > kPotMax) {
      P = kPotMax;
      flags |= 2;
    }
    const int pabs = em + (sm > 0x800000u ? 1 : 0);  // ceil(log2 M_i)
    b = pabs <= thr ? 2 : pabs <= thr + 2 ? 4 : pabs <= thr + 4 ? 6 : 8;
  } else {
    b = 2;  // M_i = 0 lies below every threshold
  }
  cp.bits = fb ? fb : b;
  cp.fpot = cp.bits - 2 - P;
  cp.scale = exp2_exact(cp.bits - 2 - P);
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

// Shift room of a channel whose codes satisfy |q| <= qa: an s with every
// q 2^s inside the one-plane range [-128, 127] (wide = false) or the
// two-plane range [-32896, 32639] (wide = true); 99 when qa is 0.  For
// 0 < qa <= 128, |q| 2^s <= 127 holds when bitlen(qa) + s <= 7 and
// |q| 2^s <= 32639 when bitlen(qa) + s <= 15 (the negative bounds are looser).
__device__ __forceinline__ int shift_room(int qa, bool wide) {
  return qa > 0 ? (wide ? 15 : 7) - (32 - __clz(qa)) : 99;
}

// 16-byte slot of local channel c in the code array.  The XOR swizzle inside
// each 128-byte row keeps three access patterns free of bank conflicts:
// channel pairs per thread (phase 1), four channels per thread (planes) and one
// channel per lane (encoded stream).
__device__ __forceinline__ int code_slot(int c) { return c ^ ((c >> 3) & 7); }

// Window slots (tag - tw, 0..31) of the slices of a channel with FPoT f and
// width b: slice j has tag f - 2j, j < b/2, so the slots are lo, lo + 2, ..,
// lo + b - 2 with lo = f - b + 2 - tw.
__device__ __forceinline__ uint32_t tag_mask32(int f, int b, int tw) {
  const uint32_t pat = 0x55u & ((1u << b) - 1u);
  const int lo = f - b + 2 - tw;
  if (lo >= 32 || lo < -8) return 0u;
  return (uint32_t)(((uint64_t)pat << (lo + 32)) >> 32);
}

// Transpose of a 32 x 32 bit matrix held one row per lane: afterwards lane c
// holds column c (its bit l is bit c of lane l's row).  Five exchange steps
// swap the off-diagonal blocks of halving size.
__device__ __forceinline__ uint32_t warp_bit_transpose(uint32_t x, int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const uint32_t lo = s == 16 ? 0x0000FFFFu : s == 8 ? 0x00FF00FFu : s == 4 ? 0x0F0F0F0Fu : s == 2 ? 0x33333333u
                                                                                                    : 0x55555555u;
    const uint32_t y = __shfl_xor_sync(0xffffffffu, x, s);
    x = (lane & s) ? ((x & ~lo) | ((y & ~lo) >> s)) : ((x & lo) | ((y & lo) << s));
  }
  return x;
}

// Rows 4R..4R+3 of four channels (word R of each channel's 16 codes, one byte
// per row) -> four row words of four channels each.
__device__ __forceinline__ void transpose4(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t (&row)[4]) {
  const uint32_t t0 = __byte_perm(a, b, 0x5140), t1 = __byte_perm(c, d, 0x5140);
  const uint32_t t2 = __byte_perm(a, b, 0x7362), t3 = __byte_perm(c, d, 0x7362);
  row[0] = __byte_perm(t0, t1, 0x5410);
  row[1] = __byte_perm(t0, t1, 0x7632);
  row[2] = __byte_perm(t2, t3, 0x5410);
  row[3] = __byte_perm(t2, t3, 0x7632);
}

// Cluster-wide barrier; a plain block barrier when the cluster is one CTA.
__device__ __forceinline__ void csync(cg::cluster_group& cluster, int C) {
  if (C > 1) cluster.sync();
  else __syncthreads();
}
// The two halves of a cluster barrier, for work that may overlap it.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

constexpr int kTagWin = 16;  // tags handled per pass of the encoded stream
constexpr int kUA = 1;       // chunks per round of ballots when counting
constexpr uint32_t kFull = 0xffffffffu;

struct QSmem {
  // read by the other CTAs of the cluster
  int xv[4];  // finest FPoT, coarsest FPoT, min(FPoT + one-plane room), min(FPoT + two-plane room)
  uint32_t mask[kMaxMaskWords];
  int cta_tot[kTagWin];  // this CTA's record count per tag of the current window
  // local
  int flags;
  int total;
  int red[4][kQWarps];
  int warp_cnt[kQWarps][kTagWin];
  int base[kTagWin];              // first record of this CTA per tag of the window
  int wbase[kQWarps][kTagWin];    // first record of each warp per tag of the window
  int x[kMaxCluster][4];
  int x_tot[kMaxCluster][kTagWin];
};

}  // namespace

size_t quantize_smem_bytes(int64_t Kc) {
  // codes (16 per channel), FPoT and width, rank table (kTagWin 8-byte entries per 32 channels)
  size_t b = 18 * (size_t)Kc + (size_t)Kc / 32 * kTagWin * 8;
  b = (b + 15) & ~(size_t)15;
  return b + sizeof(QSmem);
}

int quantize_cluster_size(int64_t M, int64_t K, int num_sms) {
  const int64_t T = M / kTile;
  const int64_t units = K / 32;
  int c = 1;
  // about 1.5 CTAs per SM when the batch is small, at least 1024 channels per
  // CTA (below that the cluster exchanges cost more than the split gains)
  while (c < kMaxCluster && 2 * T * c < 3LL * num_sms && units / (2 * c) >= 32) c *= 2;
  // a smaller share of channels per CTA lowers its shared memory, so more CTAs fit an SM
  while (FMDQ_Q_SPLIT_K > 0 && c < kMaxCluster && K / c > FMDQ_Q_SPLIT_K && units / (2 * c) >= 32) c *= 2;
  return c;
}

// ------------------------------------------------------------------------
// Per-tile stages, shared by the two quantizer kernels below.  `gt` is the
// thread's index among the `NT` threads that run the stage together.

// The call's constants of steps 1-2 (static or dynamic base).
struct QConst {
  int lb, t0, fb;
  float beta;      // 2^lb
  uint32_t dbits;  // dynamic base (fp32 bits), 1.0 when none
  float dbase;
  bool refresh;
};

template <bool DYN>
__device__ __forceinline__ QConst quant_const(const QuantParams& p) {
  QConst q;
  q.lb = p.lb, q.t0 = p.t0, q.fb = p.force_bits;
  q.beta = exp2_exact(q.lb);
  q.dbits = 0x3F800000u;
  if constexpr (DYN) {  // written by the first pass; all ones when no M_i was nonzero
    q.dbits = *p.dyn_base;
    if (q.dbits == 0xFFFFFFFFu) q.dbits = 0x3F800000u;
  }
  q.dbase = __uint_as_float(q.dbits);
  q.refresh = !(p.flags & DSTAR_FLAG_NO_XPREV_REFRESH) && p.x_prev != nullptr;
  return q;
}

// Reductions phase 1 hands on: finest and coarsest FPoT, the plane-room
// minima and the status flags of the thread's channels.
struct P1Red {
  int fmax, fmin, a1, a2, flags;
};

// Phase 1 (steps 1-3 of section 3.1; QPU stages 1-3) works on channel pairs:
// a thread reads a pair's 16 token rows of X_t and X_{t-1} (a warp reads
// 128-byte row segments), forms dX once (one fp32 subtraction), the magnitude
// max, PoT, width, FPoT and the codes, and puts each channel's 16 codes into
// shared memory as one 16-byte column; FPoT and width go to shared and global
// memory, X_t into the x_prev cache.
template <typename TIn>
__device__ __forceinline__ void load_pair(const QuantParams& p, int64_t row0, int64_t c,
                                          typename Pair<TIn>::Raw (&a)[kTile], typename Pair<TIn>::Raw (&b)[kTile]) {
  const bool diff = p.x_prev != nullptr;  // no x_prev: the operand itself is quantized (X_{t-1} = 0)
#pragma unroll
  for (int i = 0; i < kTile; ++i) {
    a[i] = Pair<TIn>::load(p.x_t, (row0 + i) * p.ld_xt + c);
    b[i] = diff ? Pair<TIn>::load(p.x_prev, (row0 + i) * p.ld_xp + c) : Pair<TIn>::zero();
  }
}

// One channel pair (global channels c, c + 1; local lc, lc + 1) of tile t.
template <typename TIn, bool DYN>
__device__ __forceinline__ void process_pair(const QuantParams& p, const QConst& qc, int64_t t, int64_t c, int lc,
                                             const typename Pair<TIn>::Raw (&rt)[kTile],
                                             const typename Pair<TIn>::Raw (&rp)[kTile], int8_t* s_code,
                                             int8_t* s_fpot, int8_t* s_bits, P1Red& r) {
  using PR = Pair<TIn>;
  const int64_t K = p.K;
  const int64_t row0 = t * kTile;
  if (qc.refresh) {
#pragma unroll
    for (int i = 0; i < kTile; ++i) PR::store(p.x_prev, (row0 + i) * p.ld_xp + c, rt[i]);
  }
  // Eq. 1 (one fp32 subtraction per element, kept) and stage 1 on the magnitude bits
  float d0[kTile], d1[kTile];
  uint32_t m0 = 0, m1 = 0;
#pragma unroll
  for (int i = 0; i < kTile; ++i) {
    d0[i] = __fsub_rn(PR::lo(rt[i]), PR::lo(rp[i]));
    d1[i] = __fsub_rn(PR::hi(rt[i]), PR::hi(rp[i]));
    m0 = max(m0, __float_as_uint(d0[i]) & 0x7FFFFFFFu);
    m1 = max(m1, __float_as_uint(d1[i]) & 0x7FFFFFFFu);
  }
  ColParams c0, c1;
  if constexpr (DYN) {
    c0 = col_params_dyn(m0, qc.dbits, qc.lb + qc.t0, qc.fb, r.flags);
    c1 = col_params_dyn(m1, qc.dbits, qc.lb + qc.t0, qc.fb, r.flags);
  } else {
    c0 = col_params(m0, qc.lb, qc.beta, qc.t0, qc.fb, r.flags);
    c1 = col_params(m1, qc.lb, qc.beta, qc.t0, qc.fb, r.flags);
  }
  // stage 3; a non-finite sub-channel has scale 0, and its NaN products convert to 0
  const float s0 = c0.nonfinite ? 0.f : c0.scale, s1 = c1.nonfinite ? 0.f : c1.scale;
  if constexpr (DYN) {  // fl32(dX / base) first (correctly rounded), then the power-of-two scale
    const DivBy dv = div_by_setup(qc.dbase);
#pragma unroll
    for (int i = 0; i < kTile; ++i) d0[i] = div_by(d0[i], dv), d1[i] = div_by(d1[i], dv);
    m0 = __float_as_uint(div_by(__uint_as_float(m0), dv));
    m1 = __float_as_uint(div_by(__uint_as_float(m1), dv));
  }
  uint32_t w0[4], w1[4];
#pragma unroll
  for (int R = 0; R < 4; ++R) {
    int a[4], b[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      a[e] = __float2int_rn(__fmul_rn(d0[4 * R + e], s0));
      b[e] = __float2int_rn(__fmul_rn(d1[4 * R + e], s1));
    }
    // low bytes of four codes, token 4R + e in byte e
    w0[R] = __byte_perm(__byte_perm(a[0], a[1], 0x0040), __byte_perm(a[2], a[3], 0x0040), 0x5410);
    w1[R] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  }
  // largest |code| of each channel: rne(M_i s_i) bounds every |rne(dX s_i)|
  const int qa0 = c0.nonfinite ? 0 : __float2int_rn(__fmul_rn(__uint_as_float(m0), s0));
  const int qa1 = c1.nonfinite ? 0 : __float2int_rn(__fmul_rn(__uint_as_float(m1), s1));
  if (p.debug_codes) {
#pragma unroll
    for (int i = 0; i < kTile; ++i)
      *reinterpret_cast<uint16_t*>(p.debug_codes + (row0 + i) * K + c) =
          (uint16_t)(((w0[i >> 2] >> (8 * (i & 3))) & 0xFFu) | (((w1[i >> 2] >> (8 * (i & 3))) & 0xFFu) << 8));
  }
  *reinterpret_cast<uint4*>(s_code + 16 * code_slot(lc)) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
  *reinterpret_cast<uint4*>(s_code + 16 * code_slot(lc + 1)) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
  auto two = [](int a, int b) { return (uint16_t)(((uint32_t)a & 0xFFu) | (((uint32_t)b & 0xFFu) << 8)); };
  *reinterpret_cast<uint16_t*>(s_fpot + lc) = two(c0.fpot, c1.fpot);
  *reinterpret_cast<uint16_t*>(s_bits + lc) = two(c0.bits, c1.bits);
  *reinterpret_cast<uint16_t*>(p.fpot + t * K + c) = two(c0.fpot, c1.fpot);
  *reinterpret_cast<uint16_t*>(p.bits + t * K + c) = two(c0.bits, c1.bits);
  r.fmax = max(r.fmax, max(c0.fpot, c1.fpot));
  r.fmin = min(r.fmin, min(c0.fpot, c1.fpot));
  r.a1 = min(r.a1, min(c0.fpot + shift_room(qa0, false), c1.fpot + shift_room(qa1, false)));
  r.a2 = min(r.a2, min(c0.fpot + shift_room(qa0, true), c1.fpot + shift_room(qa1, true)));
}

// warp reduction of the phase-1 values (every lane gets the warp's result)
__device__ __forceinline__ void warp_reduce(P1Red& r) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    r.fmax = max(r.fmax, __shfl_xor_sync(kFull, r.fmax, o));
    r.fmin = min(r.fmin, __shfl_xor_sync(kFull, r.fmin, o));
    r.a1 = min(r.a1, __shfl_xor_sync(kFull, r.a1, o));
    r.a2 = min(r.a2, __shfl_xor_sync(kFull, r.a2, o));
    r.flags |= __shfl_xor_sync(kFull, r.flags, o);
  }
}

// Phase 1 over channels [k_lo, k_lo + Kc) of tile t.  With bf16 inputs the
// row words of the thread's next pair are requested before its current pair
// is processed, so two pairs' loads are in flight per thread (fp32 inputs
// would not fit the registers twice).
template <typename TIn, bool DYN, int NT>
__device__ __forceinline__ P1Red phase1(const QuantParams& p, const QConst& qc, int64_t t, int64_t k_lo, int Kc, int gt,
                                        int8_t* s_code, int8_t* s_fpot, int8_t* s_bits) {
  using Raw = typename Pair<TIn>::Raw;
  const int64_t row0 = t * kTile;
  const int npairs = Kc / 2;
  P1Red r{-1000, 1000, 1000, 1000, 0};
  constexpr bool kAhead = FMDQ_Q_PREFETCH && sizeof(Raw) == 4;
  Raw nt[kTile], np[kTile];
  if (kAhead && gt < npairs) load_pair<TIn>(p, row0, k_lo + 2 * gt, nt, np);
  for (int pr = gt; pr < npairs; pr += NT) {
    Raw rt[kTile], rp[kTile];
    if constexpr (kAhead) {
#pragma unroll
      for (int i = 0; i < kTile; ++i) rt[i] = nt[i], rp[i] = np[i];
      if (pr + NT < npairs) load_pair<TIn>(p, row0, k_lo + 2 * (pr + NT), nt, np);
    } else {
      load_pair<TIn>(p, row0, k_lo + 2 * pr, rt, rp);
    }
    process_pair<TIn, DYN>(p, qc, t, k_lo + 2 * pr, 2 * pr, rt, rp, s_code, s_fpot, s_bits, r);
  }
  warp_reduce(r);
  return r;
}

// Phase 2a: the tensor-core operand planes of tile rows row0..row0+15,
// channels [k_lo, k_lo + Kc).  Four channels per thread: their 16-code
// columns, shifted by g - FPoT, are transposed into 4-byte row words; a warp
// writes 128 contiguous bytes per row.  Chunks where plane 1 is nonzero are
// marked in `mask` (shared memory).
template <int NT>
__device__ __forceinline__ void phase2_planes(const QuantParams& p, int64_t row0, int64_t k_lo, int Kc, int gt, int g,
                                              int planes, const int8_t* s_code, const int8_t* s_fpot, uint32_t* mask) {
  const int64_t K = p.K;
  if (planes == 1) {
    for (int qd = gt; qd < Kc / 4; qd += NT) {
      const int lc = 4 * qd;
      const uint32_t f4 = *reinterpret_cast<const uint32_t*>(s_fpot + lc);
      uint32_t col[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(s_code + 16 * code_slot(lc + i));
        // nonzero codes of a one-plane tile have a shift <= 7; zero codes stay zero
        const int sh = min(g - (int)(int8_t)(f4 >> (8 * i)), 7);
        const uint32_t keep = ((0xFFu << sh) & 0xFFu) * 0x01010101u;  // drops bits carried into the next byte
        col[i][0] = (v.x << sh) & keep, col[i][1] = (v.y << sh) & keep;
        col[i][2] = (v.z << sh) & keep, col[i][3] = (v.w << sh) & keep;
      }
      int8_t* dst = p.plane0 + row0 * K + k_lo + lc;
#pragma unroll
      for (int R = 0; R < 4; ++R) {
        uint32_t row[4];
        transpose4(col[0][R], col[1][R], col[2][R], col[3][R], row);
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint32_t*>(dst + (4 * R + i) * K) = row[i];
      }
    }
  } else if (planes == 2) {
    for (int qd = gt; qd < Kc / 4; qd += NT) {
      const int lc = 4 * qd;
      uint32_t c0w[4][4], c1w[4][4];
      uint32_t nz = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = *reinterpret_cast<const uint4*>(s_code + 16 * code_slot(lc + i));
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
        // nonzero codes of a two-plane tile have a shift <= 15, so q 2^shift fits 32 bits
        const int sh = min(g - (int)s_fpot[lc + i], 24);
#pragma unroll
        for (int R = 0; R < 4; ++R) {
          uint32_t lo = 0, hi = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int val = (int)(int8_t)(vw[R] >> (8 * e)) * (1 << sh);
            const int p0 = (int)(int8_t)(val & 0xFF);
            const int p1 = (val - p0) >> 8;
            nz |= (uint32_t)p1;
            lo |= ((uint32_t)p0 & 0xFFu) << (8 * e);
            hi |= ((uint32_t)p1 & 0xFFu) << (8 * e);
          }
          c0w[i][R] = lo, c1w[i][R] = hi;
        }
      }
      int8_t* d0 = p.plane0 + row0 * K + k_lo + lc;
      int8_t* d1 = p.plane1 + row0 * K + k_lo + lc;
#pragma unroll
      for (int R = 0; R < 4; ++R) {
        uint32_t r0[4], r1[4];
        transpose4(c0w[0][R], c0w[1][R], c0w[2][R], c0w[3][R], r0);
        transpose4(c1w[0][R], c1w[1][R], c1w[2][R], c1w[3][R], r1);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          *reinterpret_cast<uint32_t*>(d0 + (4 * R + i) * K) = r0[i];
          *reinterpret_cast<uint32_t*>(d1 + (4 * R + i) * K) = r1[i];
        }
      }
      if (nz) {
        const int chunk = (int)((k_lo + lc) / kChunkK);
        atomicOr(&mask[chunk >> 5], 1u << (chunk & 31));
      }
    }
  }
}

// Encoded stream, pass A for one window of kTagWin tags starting at tw, over
// the warp's 32-channel chunks [ch_lo, ch_hi): per chunk, a warp bit
// transpose of the lanes' tag masks gives every tag's lane ballot at once
// (lane u: tag tw + u); the ballot and the warp's count of the tag before the
// chunk go to the rank table.  Returns lane u's count of tag tw + u.
__device__ __forceinline__ int count_window(int tw, int ch_lo, int ch_hi, int lane, const int8_t* s_fpot,
                                            const int8_t* s_bits, uint2* s_tab) {
  int cnt = 0;
  for (int ch0 = ch_lo; ch0 < ch_hi; ch0 += kUA) {
    uint32_t col[kUA];
#pragma unroll
    for (int u = 0; u < kUA; ++u) {
      const int c = 32 * (ch0 + u) + lane;
      const uint32_t m = ch0 + u < ch_hi ? tag_mask32(s_fpot[c], s_bits[c], tw) & ((1u << kTagWin) - 1u) : 0u;
      col[u] = warp_bit_transpose(m, lane);
    }
#pragma unroll
    for (int u = 0; u < kUA; ++u) {
      if (ch0 + u < ch_hi && lane < kTagWin) {
        s_tab[(ch0 + u) * kTagWin + lane] = make_uint2(col[u], (uint32_t)cnt);
        cnt += __popc(col[u]);
      }
    }
  }
  return cnt;
}

// Encoded stream, pass B: every lane writes its channel's records of the
// window; record of (tag, k) = the warp's first record of the tag (wb) + the
// warp's count of the tag before the chunk + the set lanes below it in the
// chunk's ballot.
__device__ __forceinline__ void write_window(int tw, int ch_lo, int ch_hi, int lane, int64_t k_lo, const int* wb,
                                             const int8_t* s_code, const int8_t* s_fpot, const int8_t* s_bits,
                                             const uint2* s_tab, uint2* rec) {
  const uint32_t lt = (1u << lane) - 1u;
#pragma unroll 2
  for (int ch = ch_lo; ch < ch_hi; ++ch) {
    const int c = 32 * ch + lane;
    const int f = s_fpot[c], b = s_bits[c];
    uint32_t words[4];
    slice_words(*reinterpret_cast<const uint4*>(s_code + 16 * code_slot(c)), words);
    const uint2* row = s_tab + ch * kTagWin;
    const uint32_t meta_k = (uint32_t)(k_lo + c);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int ti = f - 2 * j - tw;  // window slot of slice j
      if (2 * j < b && ti >= 0 && ti < kTagWin) {
        const uint2 e = row[ti];
        // the field j < b/2 of the b-bit pattern equals that of the 8-bit pattern
        rec[wb[ti] + (int)e.y + __popc(e.x & lt)] =
            make_uint2(words[j], meta_k | ((uint32_t)(uint8_t)(int8_t)(tw + ti) << 16) | ((uint32_t)j << 24));
      }
    }
  }
}

// ------------------------------------------------------------------------
// K1 for small batches: one 16-token tile per cluster of C CTAs, CTA r owning
// a contiguous range of channels; g_ref, plane count and per-tag record
// counts are combined across the cluster through distributed shared memory.
template <typename TIn, bool DYN>
__global__ void __launch_bounds__(kQThreads, FMDQ_Q_MIN_BLOCKS) quantize_kernel(const QuantParams p, int C, int64_t kc_max) {
  extern __shared__ __align__(16) uint8_t smem[];
  cg::cluster_group cluster = cg::this_cluster();

  const int64_t K = p.K;
  const int rank = (int)cluster.block_rank();
  const int t = (int)(blockIdx.x / C);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t units = K / 32;
  const int64_t k_lo = 32 * (rank * units / C), k_hi = 32 * ((rank + 1) * units / C);
  const int Kc = (int)(k_hi - k_lo);

  int8_t* s_code = reinterpret_cast<int8_t*>(smem);  // 16-byte slots: the 16 codes of a local channel
  int8_t* s_fpot = s_code + 16 * kc_max;              // [Kc]
  int8_t* s_bits = s_fpot + kc_max;                   // [Kc]
  // [Kc / 32][kTagWin]: per 32-channel chunk and window tag, the ballot of the
  // lanes carrying the tag and the warp's records of the tag in earlier chunks
  uint2* s_tab = reinterpret_cast<uint2*>(s_bits + kc_max);
  const int64_t tab_bytes = kc_max / 32 * kTagWin * 8;
  QSmem& S = *reinterpret_cast<QSmem*>(smem + ((18 * kc_max + tab_bytes + 15) & ~(int64_t)15));

  if (tid < kMaxMaskWords) S.mask[tid] = 0;
  if (tid == 0) S.flags = 0;
  pdl_launch_dependents();
  pdl_wait();  // nothing of global memory is touched before the previous kernel completed
  __syncthreads();

  const QConst qc = quant_const<DYN>(p);
  const int64_t row0 = (int64_t)t * kTile;

  // ---------------------------------------------------------------- phase 1
  const P1Red r1 = phase1<TIn, DYN, kQThreads>(p, qc, t, k_lo, Kc, tid, s_code, s_fpot, s_bits);

  // CTA reductions, then one exchange across the cluster
  if (lane == 0) {
    S.red[0][warp] = r1.fmax, S.red[1][warp] = r1.fmin, S.red[2][warp] = r1.a1, S.red[3][warp] = r1.a2;
    if (r1.flags) atomicOr(&S.flags, r1.flags);
  }
  __syncthreads();
  if (tid < 4) {
    int v = S.red[tid][0];
    for (int w = 1; w < kQWarps; ++w) v = tid == 0 ? max(v, S.red[tid][w]) : min(v, S.red[tid][w]);
    S.xv[tid] = v;
    if (tid == 0 && S.flags)
      set_status(p.status, (S.flags & 1 ? DSTAR_STATUS_NONFINITE : 0u) | (S.flags & 2 ? DSTAR_STATUS_RANGE : 0u));
  }
  csync(cluster, C);
  if (tid < 4 * C) {  // one remote read per thread, all in flight together
    const int q = tid >> 2, u = tid & 3;
    S.x[q][u] = (C > 1 ? cluster.map_shared_rank(&S, q) : &S)->xv[u];
  }
  __syncthreads();
  int g = -1000, gmin = 1000, A1 = 1000, A2 = 1000;
  for (int q = 0; q < C; ++q) {
    g = max(g, S.x[q][0]), gmin = min(gmin, S.x[q][1]);
    A1 = min(A1, S.x[q][2]), A2 = min(A2, S.x[q][3]);
  }
  // every v = q 2^(g - FPoT) must fit the split: g - FPoT <= room for each channel
  const int planes = g <= A1 ? 1 : g <= A2 ? 2 : 3;
  // HBM is idle from here on: pull the next GEMM's operands into L2
  if (tid == 0) {
    prefetch_region_share(p.prefetch[0], (int)blockIdx.x, (int)gridDim.x);
    prefetch_region_share(p.prefetch[1], (int)blockIdx.x, (int)gridDim.x);
  }

  // ------------------------------------------------- phase 2a: operand planes
  phase2_planes<kQThreads>(p, row0, k_lo, Kc, tid, g, planes, s_code, s_fpot, S.mask);

  // ------------------------------------- phase 2b: FPoT-grouped encoded stream
  // Slice j of channel k carries tag FPoT(k) - 2j (j < bits/2).  Tags lie in
  // [gmin - 6, g] and are handled in windows of 16 consecutive tags (one
  // window unless the tile's FPoT spread exceeds 9).  Each warp owns a
  // contiguous run of 32-channel chunks (lane = channel).  The record of
  // (tag, k) lands after the tile's records of lower tags, then those of the
  // same tag in lower-ranked CTAs, lower warps of this CTA, earlier chunks of
  // this warp and lower lanes of its chunk.
  const int tlo = gmin - 6;
  const int nchunks = Kc / 32;
  const int ch_lo = warp * nchunks / kQWarps, ch_hi = (warp + 1) * nchunks / kQWarps;
  uint2* rec = p.records + (int64_t)t * p.record_cap;
  int total = 0;  // records of lower windows, all CTAs (kept by warp 0)
  bool first = true;
  for (int tw = tlo; tw <= g; tw += kTagWin) {
    if (!first) {
      __syncthreads();             // every warp is done with the previous window's counts and bases
      if (C > 1) cluster_wait();   // and every CTA with its remote reads of them
    }
    first = false;
    const int cnt = count_window(tw, ch_lo, ch_hi, lane, s_fpot, s_bits, s_tab);
    if (lane < kTagWin) S.warp_cnt[warp][lane] = cnt;
    __syncthreads();
    if (tid < kTagWin) {
      int s = 0;
#pragma unroll
      for (int w = 0; w < kQWarps; ++w) s += S.warp_cnt[w][tid];
      S.cta_tot[tid] = s;
    }
    csync(cluster, C);
    if (tid < kTagWin * C) {  // every CTA's window totals, one remote word per thread
      const int q = tid / kTagWin, u = tid % kTagWin;
      S.x_tot[q][u] = (C > 1 ? cluster.map_shared_rank(&S, q) : &S)->cta_tot[u];
    }
    if (tw == tlo && rank == 0 && tid >= 32 * (kQWarps - 1) && tid - 32 * (kQWarps - 1) < p.mask_words) {
      // the tile's plane-1 chunk mask (every CTA finished its planes before the barrier)
      const int wd = tid - 32 * (kQWarps - 1);
      uint32_t m = 0;
      for (int q = 0; q < C; ++q) m |= (C > 1 ? cluster.map_shared_rank(&S, q) : &S)->mask[wd];
      p.mask1[(int64_t)t * p.mask_words + wd] = planes == 2 ? m : 0u;
    }
    __syncthreads();
    if (C > 1) cluster_arrive();  // remote reads of this window done; waited for before reuse or exit
    if (warp == 0) {
      int all = 0, lower = 0;
      for (int q = 0; q < C && lane < kTagWin; ++q) {
        const int v = S.x_tot[q][lane];
        all += v;
        if (q < rank) lower += v;
      }
      int incl = all;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += n;
      }
      if (lane < kTagWin) S.base[lane] = total + incl - all + lower;
      total += __shfl_sync(kFull, incl, 31);
    }
    __syncthreads();
    if (lane < kTagWin) {
      int o = S.base[lane];
      for (int w = 0; w < warp; ++w) o += S.warp_cnt[w][lane];
      S.wbase[warp][lane] = o;
    }
    __syncwarp();
    write_window(tw, ch_lo, ch_hi, lane, k_lo, S.wbase[warp], s_code, s_fpot, s_bits, s_tab, rec);
  }
  if (rank == 0 && tid == 0) {
    p.g_ref[t] = g;
    p.planes[t] = planes;
  }
  if (warp == 0 && lane == 0) S.total = total;
  __syncthreads();
  if (rank == 0 && tid == 0) p.count[t] = S.total;
  if (C > 1) cluster_wait();  // no CTA leaves while another may still read its shared memory
}

// ------------------------------------------------------------------------
// K1 for large batches: persistent (one CTA per SM) and warp-specialised.
// With one CTA per tile, every CTA of a wave streams HBM in phase 1 and then
// leaves it idle while it builds planes and records.  Here two groups of
// eight warps work on consecutive tiles at once: group 1 runs phase 1 of a
// tile into one of two shared-memory buffers while group 2 runs phases 2a
// and 2b of the previous tile from the other, so each SM streams HBM and
// encodes at the same time.  The per-tile arithmetic is that of the kernel
// above (the same stage functions, with one CTA per tile); the buffers pass
// between the groups through mbarriers (full: group 1 -> 2, empty: 2 -> 1)
// whose waits are bounded.
// Two forms, 16 warps of 128 registers per SM either way: one CTA of 8 + 8
// warps, or two CTAs of 4 + 4 warps, whose group barriers take half the
// threads and whose two tile streams cover each other's pipeline fill and
// drain.  The second pays where an SM has few tiles (measured: PixArt's
// 8192-token layers, 3.5 tiles per SM, 1-2 us faster per launch; the Latte
// layers, 6.9 tiles per SM, 3 us slower per step) and needs two CTAs'
// buffers in the SM's shared memory (inputs of up to about 2900 channels).
constexpr int kPMaxWarps = 8;          // warps of a group, at most
constexpr int kBarG1 = 1, kBarG2 = 2;  // named barriers of the groups (0 is __syncthreads)

struct PSmem {
  uint64_t full[2], empty[2];
  int abort;
  int red[4][kPMaxWarps];
  int xv[2][4];  // per buffer: finest FPoT, coarsest FPoT, min(FPoT + one-plane room), min(FPoT + two-plane room)
  uint32_t mask[kMaxMaskWords];
  int warp_cnt[kPMaxWarps][kTagWin];
  int base[kTagWin];
  int wbase[kPMaxWarps][kTagWin];
};

template <int NT>
__device__ __forceinline__ void group_sync(int id) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(NT) : "memory");
}

template <typename TIn, bool DYN, int kPG1Warps, int kPG2Warps, int kMinBlocks>
__global__ void __launch_bounds__(32 * (kPG1Warps + kPG2Warps), kMinBlocks)
    quantize_persistent_kernel(const QuantParams p) {
  static_assert(kPG1Warps <= kPMaxWarps && kPG2Warps <= kPMaxWarps, "shared-memory tables");
  constexpr int kPG1 = 32 * kPG1Warps, kPG2 = 32 * kPG2Warps;  // threads of each group
  extern __shared__ __align__(16) uint8_t smem[];
  const int64_t K = p.K;
  const int Kc = (int)K;
  const int64_t T = p.M / kTile;
  const int tid = threadIdx.x, lane = tid & 31;
  const bool g1 = tid < kPG1;
  const int gt = g1 ? tid : tid - kPG1;  // thread index within the group
  const int gw = gt >> 5;                   // warp index within the group
  // buffer b: codes at 16 K b, FPoT at 32 K + 2 K b, widths right after the FPoTs
  int8_t* const s_base = reinterpret_cast<int8_t*>(smem);
  auto s_code = [&](int b) { return s_base + 16 * K * b; };
  auto s_fpot = [&](int b) { return s_base + 32 * K + 2 * K * b; };
  auto s_bits = [&](int b) { return s_base + 33 * K + 2 * K * b; };
  uint2* s_tab = reinterpret_cast<uint2*>(smem + 36 * K);  // group 2 only
  PSmem& S = *reinterpret_cast<PSmem*>(smem + ((36 * K + K / 32 * kTagWin * 8 + 15) & ~(int64_t)15));
  volatile int* abort_flag = &S.abort;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) mbar_init(&S.full[b], kPG1), mbar_init(&S.empty[b], kPG2);
    S.abort = 0;
    fence_barrier_init();
  }
  pdl_launch_dependents();
  pdl_wait();  // nothing of global memory is touched before the previous kernel completed
  __syncthreads();
  const QConst qc = quant_const<DYN>(p);
  const int ntiles = T > (int64_t)blockIdx.x ? (int)((T - 1 - blockIdx.x) / gridDim.x) + 1 : 0;

  if (g1) {
    // ------------------------------------------------- group 1: phase 1
    using Raw = typename Pair<TIn>::Raw;
    constexpr bool kAhead = FMDQ_Q_PREFETCH && sizeof(Raw) == 4;
    const int npairs = Kc / 2;
    Raw nt[kTile], np[kTile];
    if (kAhead && ntiles > 0 && gt < npairs) load_pair<TIn>(p, (int64_t)blockIdx.x * kTile, 2 * gt, nt, np);
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      const int64_t t = blockIdx.x + (int64_t)i * gridDim.x;
      // buffer b is free once group 2 has finished tile i - 2
      if (gt == 0 && i >= 2 && !wait_parity(&S.empty[b], ((i >> 1) - 1) & 1, abort_flag, p.status, kWaitLimitNs))
        *abort_flag = 1;
      __syncwarp();
      group_sync<kPG1>(kBarG1);  // also: every warp is done with the previous tile's reduction
      if (*abort_flag) break;
      // phase 1; the loads of the thread's first pair of the next tile are
      // issued while its last pair of this tile is processed
      P1Red r{-1000, 1000, 1000, 1000, 0};
      for (int pr = gt; pr < npairs; pr += kPG1) {
        Raw rt[kTile], rp[kTile];
        if constexpr (kAhead) {
#pragma unroll
          for (int j = 0; j < kTile; ++j) rt[j] = nt[j], rp[j] = np[j];
          if (pr + kPG1 < npairs) load_pair<TIn>(p, t * kTile, 2 * (pr + kPG1), nt, np);
          else if (i + 1 < ntiles) load_pair<TIn>(p, (t + gridDim.x) * kTile, 2 * gt, nt, np);
        } else {
          load_pair<TIn>(p, t * kTile, 2 * pr, rt, rp);
        }
        process_pair<TIn, DYN>(p, qc, t, 2 * pr, 2 * pr, rt, rp, s_code(b), s_fpot(b), s_bits(b), r);
      }
      warp_reduce(r);
      if (lane == 0) {
        S.red[0][gw] = r.fmax, S.red[1][gw] = r.fmin, S.red[2][gw] = r.a1, S.red[3][gw] = r.a2;
        if (r.flags)
          set_status(p.status, (r.flags & 1 ? DSTAR_STATUS_NONFINITE : 0u) | (r.flags & 2 ? DSTAR_STATUS_RANGE : 0u));
      }
      group_sync<kPG1>(kBarG1);
      if (gt < 4) {
        int v = S.red[gt][0];
        for (int w = 1; w < kPG1Warps; ++w) v = gt == 0 ? max(v, S.red[gt][w]) : min(v, S.red[gt][w]);
        S.xv[b][gt] = v;
      }
      mbar_arrive(&S.full[b]);  // every thread after its own writes of the tile
    }
    // this CTA no longer reads HBM: pull the next GEMM's operands into L2
    if (gt == 0) {
      prefetch_region_share(p.prefetch[0], (int)blockIdx.x, (int)gridDim.x);
      prefetch_region_share(p.prefetch[1], (int)blockIdx.x, (int)gridDim.x);
    }
  } else {
    // ------------------------------------- group 2: phases 2a and 2b
    const int nchunks = Kc / 32;
    const int ch_lo = gw * nchunks / kPG2Warps, ch_hi = (gw + 1) * nchunks / kPG2Warps;
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      const int64_t t = blockIdx.x + (int64_t)i * gridDim.x;
      if (gt == 0 && !wait_parity(&S.full[b], (i >> 1) & 1, abort_flag, p.status, kWaitLimitNs)) *abort_flag = 1;
      __syncwarp();
      group_sync<kPG2>(kBarG2);  // also: every warp is done with the previous tile
      if (*abort_flag) break;
      const int g = S.xv[b][0], gmin = S.xv[b][1], A1 = S.xv[b][2], A2 = S.xv[b][3];
      const int planes = g <= A1 ? 1 : g <= A2 ? 2 : 3;
      if (gt < kMaxMaskWords) S.mask[gt] = 0;
      group_sync<kPG2>(kBarG2);
      const int64_t row0 = t * kTile;
      phase2_planes<kPG2>(p, row0, 0, Kc, gt, g, planes, s_code(b), s_fpot(b), S.mask);
      const int tlo = gmin - 6;
      uint2* rec = p.records + t * p.record_cap;
      int total = 0;  // records of lower windows (kept by warp 0)
      for (int tw = tlo; tw <= g; tw += kTagWin) {
        if (tw != tlo) group_sync<kPG2>(kBarG2);  // every warp is done with the previous window
        const int cnt = count_window(tw, ch_lo, ch_hi, lane, s_fpot(b), s_bits(b), s_tab);
        if (lane < kTagWin) S.warp_cnt[gw][lane] = cnt;
        group_sync<kPG2>(kBarG2);  // counts written; every plane of the tile written (mask complete)
        if (tw == tlo && gt < p.mask_words) p.mask1[t * p.mask_words + gt] = planes == 2 ? S.mask[gt] : 0u;
        if (gw == 0) {
          int all = 0;
          if (lane < kTagWin)
            for (int w = 0; w < kPG2Warps; ++w) all += S.warp_cnt[w][lane];
          int incl = all;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += n;
          }
          if (lane < kTagWin) S.base[lane] = total + incl - all;
          total += __shfl_sync(kFull, incl, 31);
        }
        group_sync<kPG2>(kBarG2);
        if (lane < kTagWin) {
          int o = S.base[lane];
          for (int w = 0; w < gw; ++w) o += S.warp_cnt[w][lane];
          S.wbase[gw][lane] = o;
        }
        __syncwarp();
        write_window(tw, ch_lo, ch_hi, lane, 0, S.wbase[gw], s_code(b), s_fpot(b), s_bits(b), s_tab, rec);
      }
      if (gt == 0) {
        p.g_ref[t] = g;
        p.planes[t] = planes;
        p.count[t] = total;
      }
      mbar_arrive(&S.empty[b]);  // buffer b may be refilled
    }
  }
  __syncthreads();
}

size_t quantize_persistent_smem_bytes(int64_t K) {
  size_t b = 36 * (size_t)K + (size_t)K / 32 * kTagWin * 8;
  b = (b + 15) & ~(size_t)15;
  return b + sizeof(PSmem);
}

// The persistent kernel takes batches of at least two tiles per SM whose
// double buffers fit shared memory.
bool use_persistent(int64_t M, int64_t K, int num_sms) {
  return M / kTile >= 2LL * num_sms && quantize_persistent_smem_bytes(K) <= 227 * 1024;
}

// Two CTAs of the persistent kernel per SM: at most four tiles per SM, and
// both CTAs fit the SM's 228 KB of shared memory, each with the 1 KB the
// system reserves per CTA.
bool persistent_two_per_sm(int64_t T, int64_t K, int num_sms) {
  return T <= 4LL * num_sms && 2 * (quantize_persistent_smem_bytes(K) + 1024) <= 228 * 1024;
}

template <typename TIn, bool DYN>
int launch_persistent(cudaLaunchConfig_t& cfg, const QuantParams& p, int64_t T, int num_sms) {
  const bool two = persistent_two_per_sm(T, p.K, num_sms);
  const void* fn = two ? (const void*)quantize_persistent_kernel<TIn, DYN, 4, 4, 2>
                       : (const void*)quantize_persistent_kernel<TIn, DYN, 8, 8, 1>;
  const int e = ensure_max_smem(fn, 227 * 1024);
  if (e != 0) return e;
  const int64_t ctas = (int64_t)num_sms * (two ? 2 : 1);
  cfg.gridDim = dim3((unsigned)(T < ctas ? T : ctas), 1, 1);
  cfg.blockDim = dim3(two ? 256 : 512, 1, 1);
  cfg.dynamicSmemBytes = quantize_persistent_smem_bytes(p.K);
  cfg.numAttrs = 1;
  const cudaError_t ce = two ? cudaLaunchKernelEx(&cfg, quantize_persistent_kernel<TIn, DYN, 4, 4, 2>, p)
                             : cudaLaunchKernelEx(&cfg, quantize_persistent_kernel<TIn, DYN, 8, 8, 1>, p);
  if (ce != cudaSuccess) return (int)ce;
  return (int)cudaGetLastError();
}

int launch_quantize(const QuantParams& p, int in_bf16, int num_sms, void* stream) {
  const int64_t T = p.M / kTile;
  if (T == 0) return 0;
  const bool dyn = p.dyn_base != nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the launch with the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cudaError_t ce;
  if (use_persistent(p.M, p.K, num_sms)) {
    if (in_bf16) return dyn ? launch_persistent<__nv_bfloat16, true>(cfg, p, T, num_sms)
                            : launch_persistent<__nv_bfloat16, false>(cfg, p, T, num_sms);
    return dyn ? launch_persistent<float, true>(cfg, p, T, num_sms) : launch_persistent<float, false>(cfg, p, T, num_sms);
  }
  const int C = quantize_cluster_size(p.M, p.K, num_sms);
  const int64_t units = p.K / 32;
  const int64_t kc_max = 32 * ((units + C - 1) / C);
  const size_t smem = quantize_smem_bytes(kc_max);
  const int smem_max = (int)quantize_smem_bytes(DSTAR_K_MAX);  // one setting serves every K
  const void* fn = in_bf16 ? (dyn ? (const void*)quantize_kernel<__nv_bfloat16, true>
                                  : (const void*)quantize_kernel<__nv_bfloat16, false>)
                           : (dyn ? (const void*)quantize_kernel<float, true> : (const void*)quantize_kernel<float, false>);
  int e = ensure_max_smem(fn, smem_max);
  if (e != 0) return e;
  cfg.gridDim = dim3((unsigned)(T * C), 1, 1);
  cfg.blockDim = dim3(kQThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.numAttrs = 2;
  if (in_bf16) ce = dyn ? cudaLaunchKernelEx(&cfg, quantize_kernel<__nv_bfloat16, true>, p, C, kc_max)
                        : cudaLaunchKernelEx(&cfg, quantize_kernel<__nv_bfloat16, false>, p, C, kc_max);
  else ce = dyn ? cudaLaunchKernelEx(&cfg, quantize_kernel<float, true>, p, C, kc_max)
                : cudaLaunchKernelEx(&cfg, quantize_kernel<float, false>, p, C, kc_max);
  if (ce != cudaSuccess) return (int)ce;
  return (int)cudaGetLastError();
}

// ---------------------------------------------------------------------------
// First pass of the dynamic base (section 3.1: the base is the minimum of M_i
// over all sub-channels, which needs a pass over the data before any
// sub-channel can be quantized).  Each thread owns 16 bytes of channels (8
// bf16 or 4 fp32) of one 16-token tile, reads its 16 rows of X_t and X_{t-1},
// forms |dX| with the same fp32 subtraction as the quantizer and keeps the
// per-channel maxima; the smallest nonzero finite one of the warp goes to an
// atomic minimum on the fp32 bits (positive floats order like their bits).
// ---------------------------------------------------------------------------
template <typename TIn>
__global__ void __launch_bounds__(256) base_min_kernel(const TIn* __restrict__ x_t, const TIn* __restrict__ x_prev,
                                                       int64_t ld_xt, int64_t ld_xp, int64_t M, int64_t K,
                                                       uint32_t* out) {
  constexpr int E = 16 / sizeof(TIn);  // channels per thread
  const int64_t groups = K / E, T = M / kTile;
  uint32_t best = 0xFFFFFFFFu;
  pdl_launch_dependents();
  pdl_wait();
  for (int64_t item = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; item < T * groups;
       item += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = item / groups, c = (item % groups) * E;
    uint32_t mx[E];
#pragma unroll
    for (int e = 0; e < E; ++e) mx[e] = 0;
#pragma unroll 8
    for (int r = 0; r < kTile; ++r) {
      const int64_t row = t * kTile + r;
      const uint4 a = *reinterpret_cast<const uint4*>(x_t + row * ld_xt + c);
      const uint4 b = *reinterpret_cast<const uint4*>(x_prev + row * ld_xp + c);
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float xa, xb;
        if constexpr (sizeof(TIn) == 2) {
          xa = __uint_as_float((e & 1) ? (aw[e >> 1] & 0xFFFF0000u) : (aw[e >> 1] << 16));
          xb = __uint_as_float((e & 1) ? (bw[e >> 1] & 0xFFFF0000u) : (bw[e >> 1] << 16));
        } else {
          xa = __uint_as_float(aw[e]);
          xb = __uint_as_float(bw[e]);
        }
        const uint32_t m = __float_as_uint(__fsub_rn(xa, xb)) & 0x7FFFFFFFu;
        mx[e] = max(mx[e], m);  // NaN bits sort above infinity: the channel reads as non-finite
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (mx[e] != 0u && mx[e] < 0x7F800000u) best = min(best, mx[e]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = min(best, __shfl_xor_sync(0xffffffffu, best, o));
  if ((threadIdx.x & 31) == 0 && best != 0xFFFFFFFFu) atomicMin(out, best);
}

// Self-test of div_by against CUDA's __fdiv_rn: every a = (1 + m 2^-23) 2^e,
// all 2^23 significands m and e in [e_lo, e_hi], divided by each of the n_b
// divisors b[]; the number of results that differ in any bit is added to
// *count.  Grid: (significand blocks, n_b, exponents).
__global__ void __launch_bounds__(256) div_selftest_kernel(const float* __restrict__ b, int e_lo,
                                                           unsigned long long* count) {
  const DivBy d = div_by_setup(b[blockIdx.y]);
  const int e = e_lo + (int)blockIdx.z;
  unsigned long long bad = 0;
  for (uint32_t m = blockIdx.x * blockDim.x + threadIdx.x; m < (1u << 23); m += gridDim.x * blockDim.x) {
    const float a = __uint_as_float(((uint32_t)(e + 127) << 23) | m);
    bad += __float_as_uint(div_by(a, d)) != __float_as_uint(__fdiv_rn(a, d.b));
  }
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(count, bad);
}

int launch_div_selftest(const float* b, int n_b, int e_lo, int e_hi, unsigned long long* count, void* stream) {
  if (n_b <= 0 || e_hi < e_lo) return 0;
  const dim3 grid(512, (unsigned)n_b, (unsigned)(e_hi - e_lo + 1));
  div_selftest_kernel<<<grid, 256, 0, (cudaStream_t)stream>>>(b, e_lo, count);
  return (int)cudaGetLastError();
}

int launch_base_min(const void* x_t, const void* x_prev, int64_t ld_xt, int64_t ld_xp, int64_t M, int64_t K,
                    int in_bf16, uint32_t* out, int num_sms, void* stream) {
  const int64_t items = (M / kTile) * (K / (in_bf16 ? 8 : 4));
  if (items == 0) return 0;
  const int64_t want = (items + 255) / 256;
  const int grid = (int)(want < 8LL * num_sms ? want : 8LL * num_sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = (cudaStream_t)stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t ce;
  if (in_bf16)
    ce = cudaLaunchKernelEx(&cfg, base_min_kernel<__nv_bfloat16>, static_cast<const __nv_bfloat16*>(x_t),
                            static_cast<const __nv_bfloat16*>(x_prev), ld_xt, ld_xp, M, K, out);
  else
    ce = cudaLaunchKernelEx(&cfg, base_min_kernel<float>, static_cast<const float*>(x_t),
                            static_cast<const float*>(x_prev), ld_xt, ld_xp, M, K, out);
  if (ce != cudaSuccess) return (int)ce;
  return (int)cudaGetLastError();
}

}  // namespace fmdq
