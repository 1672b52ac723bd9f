/*
 * CPU oracle for the FMDQ differential linear layer (DSTAR, "Accelerating
 * Diffusion Transformers via Spatial and Temporal Redundancy Reduction",
 * section 3.1 "Fine-Grained Mixed-Precision Quantization", Eqs. 1-5, and
 * section 4.2 "Design of MPU" / 4.3 "Operator Mapping").
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
 * CUDA path is checked against.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load it.  It shares no code, header or
 * constant table with the CUDA library, and it never calls into it.
 *
 * Everything here is written for a reader checking it against the paper:
 * one loop per step, no blocking, no fusion.  Integer work is exact (int64).
 * The only floating point that decides an integer is the differential
 * dX = X_t - X_{t-1}, taken as one IEEE fp32 subtraction (the precision the
 * kernels use); every later step up to the accumulator is exact.  The
 * epilogue is provided twice: in the fixed fp32 operation order the kernels
 * use (so bf16 rounding decisions can be compared), and in fp64 (to pin the
 * fp32 order against the exact value).
 *
 * Readings of points the paper leaves open (each is stated where it is used):
 *   - tile of 16 tokens x 1 channel = one sub-channel;
 *   - PoT = ceil(log2(M_i / base)), taken as 0 when M_i <= base (static base);
 *   - PCeil(b) = 2^(b-2), the only choice that keeps Eq. 4 an integer and the
 *     thresholds a x4 series per 2 bits;
 *   - Thr_N = base * 2^(t0 + 2N), so "M_i <= Thr_N" <=> "PoT <= t0 + 2N";
 *   - quantization rounds half to even;
 *   - slices are the base-4 digits of the b-bit two's-complement code, the
 *     top digit signed;
 *   - records are ordered by (FPoT ascending, channel ascending);
 *   - the accumulator of a tile is kept in units of the finest FPoT of the
 *     tile (g_ref = max FPoT), exact in int64.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -shared -fPIC
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_TILE 16     /* tokens per sub-channel */
#define ORC_POT_MAX 32  /* largest PoT accepted; above it the call reports RANGE */

/* status bits reported by fmdq_orc_quantize (same meaning as the library's) */
#define ORC_ST_NONFINITE 1
#define ORC_ST_RANGE 2

/* ---------------------------------------------------------------- helpers */

/* bf16 -> fp32 is exact: the 16 bits are the top half of the fp32 pattern. */
static float bf16_bits_to_float(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* fp32 -> bf16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* ceil(log2(v)) for a finite v > 1, exactly, from the binary exponent:
 * v = f * 2^e with f in [0.5, 1)  ->  log2 v = e + log2 f, log2 f in [-1, 0);
 * it is an integer only when f == 0.5. */
static int ceil_log2_exact(double v) {
  int e;
  double f = frexp(v, &e);
  return (f == 0.5) ? (e - 1) : e;
}

/* ------------------------------------------------------------ quantizer */

/*
 * Step 1 of the computation flow (Fig. 5, steps 1-4):
 *   1  on-the-fly PoT quantization per sub-channel (Eqs. 2-5, static base),
 *   2  decomposition into 2-bit slices (FPoT of slice n lowered by 2n),
 *   3  reordering of the slices by FPoT (ascending),
 *   4  encoding: shift counts = difference of adjacent FPoTs.
 *
 * Inputs
 *   x_t, x_prev : [M x K] fp32 (bf16 inputs are widened exactly by the caller)
 *   M (multiple of 16), K
 *   lb          : base = 2^lb (static base, exact power of two)
 *   t0          : Thr_0 = base * 2^t0
 *   force_bits  : 0 = adaptive, else every sub-channel uses this width
 * Outputs (caller-allocated)
 *   codes [M x K] int8; bits [T x K] int8; fpot [T x K] int8 (absolute FPoT,
 *   Eq. 4); pot [T x K] int16 (PoT_i, Eq. 3); g_ref [T] int32 (max FPoT of
 *   the tile); count [T] int32; per tile up to 4K records, each
 *   {word, k, tag, j}: word holds the 2-bit field of slice j for the 16
 *   tokens (token i in bits 2i..2i+1), tag is the slice's FPoT;
 *   shift [T x 4K] int8: encoded shift before each record.
 * Returns the status bits.
 */
int fmdq_orc_quantize(const float* x_t, const float* x_prev, int64_t M, int64_t K, int lb,
                      int t0, int force_bits, int8_t* codes, int8_t* bits, int8_t* fpot,
                      int16_t* pot, int32_t* g_ref, int32_t* count, uint32_t* rec_word,
                      uint16_t* rec_k, int8_t* rec_tag, uint8_t* rec_j, int8_t* shift) {
  const int64_t T = M / ORC_TILE;
  const int64_t cap = 4 * K;
  const double base = ldexp(1.0, lb);
  int status = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : status)
  for (int64_t t = 0; t < T; ++t) {
    /* per-slice records of this tile before sorting */
    typedef struct {
      int tag;
      int k;
      int j;
      uint32_t word;
    } rec_t;
    rec_t* recs = (rec_t*)malloc((size_t)cap * sizeof(rec_t));
    int64_t nrec = 0;
    int gmax = -1000;

    for (int64_t k = 0; k < K; ++k) {
      /* dX of the sub-channel: one fp32 subtraction per element (Eq. 1). */
      float dx[ORC_TILE];
      for (int i = 0; i < ORC_TILE; ++i) {
        int64_t m = t * ORC_TILE + i;
        dx[i] = x_t[m * K + k] - x_prev[m * K + k];
      }
      /* M_i = max |dX| over the sub-channel (QPU stage 1). */
      double Mi = 0.0;
      int nonfinite = 0;
      for (int i = 0; i < ORC_TILE; ++i) {
        double a = fabs((double)dx[i]);
        if (!isfinite(a)) nonfinite = 1;
        else if (a > Mi) Mi = a;
      }
      if (nonfinite) {
        status |= ORC_ST_NONFINITE;
        Mi = 0.0; /* the sub-channel is treated as all-zero */
        for (int i = 0; i < ORC_TILE; ++i) dx[i] = 0.0f;
      }
      /* Eq. 3 with a static base: PoT_i = ceil(log2(M_i / base)), and 0 when
       * M_i <= base (base is the smallest scale allowed). */
      int PoT = 0;
      if (Mi > base) PoT = ceil_log2_exact(Mi / base);
      if (PoT > ORC_POT_MAX) {
        status |= ORC_ST_RANGE;
        PoT = ORC_POT_MAX;
      }
      /* Precision by binning M_i against Thr_N = Thr_0 * 2^(2N) (QPU stage 2). */
      int b;
      if (force_bits) b = force_bits;
      else if (PoT <= t0) b = 2;
      else if (PoT <= t0 + 2) b = 4;
      else if (PoT <= t0 + 4) b = 6;
      else b = 8;
      /* PCeil = 2^(b-2); Eq. 4: FPoT = log2(PCeil / (base^2 * 2^PoT)). */
      int FPoT = (b - 2) - 2 * lb - PoT;
      /* Eq. 5: s_i = base * 2^FPoT; the code is x * s_i rounded half-to-even. */
      double s_i = ldexp(1.0, lb + FPoT);
      int32_t q[ORC_TILE];
      for (int i = 0; i < ORC_TILE; ++i) {
        double v = (double)dx[i] * s_i; /* exact: power-of-two scaling */
        q[i] = (int32_t)nearbyint(v);   /* default rounding mode: ties to even */
        /* no clipping is ever needed: |dX| <= M_i <= base*2^PoT. */
        if (abs(q[i]) > (1 << (b - 2))) status |= ORC_ST_RANGE;
        codes[(t * ORC_TILE + i) * K + k] = (int8_t)q[i];
      }
      bits[t * K + k] = (int8_t)b;
      fpot[t * K + k] = (int8_t)FPoT;
      pot[t * K + k] = (int16_t)PoT;
      if (FPoT > gmax) gmax = FPoT;

      /* Step 2: b/2 slices of 2 bits; slice j carries FPoT - 2j.  The field of
       * slice j is bits 2j..2j+1 of the b-bit two's-complement pattern. */
      for (int j = 0; j < b / 2; ++j) {
        uint32_t word = 0;
        for (int i = 0; i < ORC_TILE; ++i) {
          uint32_t u = (uint32_t)q[i] & ((1u << b) - 1u);
          uint32_t field = (u >> (2 * j)) & 3u;
          word |= field << (2 * i);
        }
        recs[nrec].tag = FPoT - 2 * j;
        recs[nrec].k = (int)k;
        recs[nrec].j = j;
        recs[nrec].word = word;
        ++nrec;
      }
    }

    /* Step 3: reorder by FPoT ascending, ties by channel ascending.  A plain
     * insertion sort keyed on (tag, k) keeps this obviously correct. */
    for (int64_t a = 1; a < nrec; ++a) {
      rec_t key = recs[a];
      int64_t c = a - 1;
      while (c >= 0 && (recs[c].tag > key.tag || (recs[c].tag == key.tag && recs[c].k > key.k))) {
        recs[c + 1] = recs[c];
        --c;
      }
      recs[c + 1] = key;
    }

    /* Step 4: encoding; the shift before a record is its FPoT minus the
     * previous record's (0 for the first). */
    for (int64_t r = 0; r < nrec; ++r) {
      rec_word[t * cap + r] = recs[r].word;
      rec_k[t * cap + r] = (uint16_t)recs[r].k;
      rec_tag[t * cap + r] = (int8_t)recs[r].tag;
      rec_j[t * cap + r] = (uint8_t)recs[r].j;
      shift[t * cap + r] = (int8_t)(r == 0 ? 0 : recs[r].tag - recs[r - 1].tag);
    }
    count[t] = (int32_t)nrec;
    g_ref[t] = gmax;
    free(recs);
  }
  return status;
}

/* ------------------------------------------------- dynamic base (FMDQ-DYN) */

/*
 * Steps 2-4 for one tile whose codes, widths and FPoTs are known: b/2 slices
 * per sub-channel (slice j carries FPoT - 2j), reordered by (FPoT, channel)
 * ascending, shift counts.  The same rules as in fmdq_orc_quantize.
 */
static void encode_tile(int64_t t, int64_t K, const int8_t* codes, const int8_t* bits,
                        const int8_t* fpot, int32_t* count, uint32_t* rec_word, uint16_t* rec_k,
                        int8_t* rec_tag, uint8_t* rec_j, int8_t* shift) {
  const int64_t cap = 4 * K;
  typedef struct {
    int tag;
    int k;
    int j;
    uint32_t word;
  } rec_t;
  rec_t* recs = (rec_t*)malloc((size_t)cap * sizeof(rec_t));
  int64_t nrec = 0;
  for (int64_t k = 0; k < K; ++k) {
    int b = bits[t * K + k];
    for (int j = 0; j < b / 2; ++j) {
      uint32_t word = 0;
      for (int i = 0; i < ORC_TILE; ++i) {
        uint32_t u = (uint32_t)(int32_t)codes[(t * ORC_TILE + i) * K + k] & ((1u << b) - 1u);
        word |= ((u >> (2 * j)) & 3u) << (2 * i);
      }
      recs[nrec].tag = fpot[t * K + k] - 2 * j;
      recs[nrec].k = (int)k;
      recs[nrec].j = j;
      recs[nrec].word = word;
      ++nrec;
    }
  }
  for (int64_t a = 1; a < nrec; ++a) {
    rec_t key = recs[a];
    int64_t c = a - 1;
    while (c >= 0 && (recs[c].tag > key.tag || (recs[c].tag == key.tag && recs[c].k > key.k))) {
      recs[c + 1] = recs[c];
      --c;
    }
    recs[c + 1] = key;
  }
  for (int64_t r = 0; r < nrec; ++r) {
    rec_word[t * cap + r] = recs[r].word;
    rec_k[t * cap + r] = (uint16_t)recs[r].k;
    rec_tag[t * cap + r] = (int8_t)recs[r].tag;
    rec_j[t * cap + r] = (uint8_t)recs[r].j;
    shift[t * cap + r] = (int8_t)(r == 0 ? 0 : recs[r].tag - recs[r - 1].tag);
  }
  count[t] = (int32_t)nrec;
  free(recs);
}

/*
 * Step 1 with the dynamic base of Eqs. 2-3 (section 3.1: the base is the
 * minimum of M_i over all sub-channels, found by a first pass over the data;
 * the paper's DS-FMDQ-DYN variant of section 5.2, Table 2).  Readings:
 *   - the minimum is taken over the sub-channels with a nonzero, finite M_i
 *     (a zero M_i would make Eq. 3 undefined); with none, every code is 0
 *     and base is reported as 1;
 *   - the bit width still comes from the predefined thresholds,
 *     M_i <= Thr_N = 2^(thr_lb + t0 + 2N) (Thr_0 = 2^(thr_lb + t0));
 *   - PoT_i = ceil(log2(M_i / base)) exactly: the smallest P >= 0 with
 *     M_i <= base * 2^P (both sides exact in double);
 *   - the base is not a power of two, so the relative FPoT b - 2 - PoT is
 *     stored (the absolute one of Eq. 4 differs from it by -2 log2(base),
 *     the same for every sub-channel) and the code is
 *     q = rne(fl32(dX / base) * 2^(b - 2 - PoT)): one IEEE fp32 division,
 *     then an exact power-of-two scaling;
 *   - the dequantized value of a code is q * 2^-(FPoT) * base.
 * Outputs as fmdq_orc_quantize (fpot holds the relative FPoT), plus *base_out.
 */
int fmdq_orc_quantize_dyn(const float* x_t, const float* x_prev, int64_t M, int64_t K, int thr_lb,
                          int t0, int force_bits, float* base_out, int8_t* codes, int8_t* bits,
                          int8_t* fpot, int16_t* pot, int32_t* g_ref, int32_t* count,
                          uint32_t* rec_word, uint16_t* rec_k, int8_t* rec_tag, uint8_t* rec_j,
                          int8_t* shift) {
  const int64_t T = M / ORC_TILE;
  int status = 0;

  /* Pass 1: M_i of every sub-channel, and their minimum over nonzero finite ones. */
  float base = 0.0f;
  int have = 0;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t k = 0; k < K; ++k) {
      float Mi = 0.0f;
      int nonfinite = 0;
      for (int i = 0; i < ORC_TILE; ++i) {
        int64_t m = t * ORC_TILE + i;
        float a = fabsf(x_t[m * K + k] - x_prev[m * K + k]);
        if (!isfinite(a)) nonfinite = 1;
        else if (a > Mi) Mi = a;
      }
      if (nonfinite || Mi == 0.0f) continue;
      if (!have || Mi < base) base = Mi;
      have = 1;
    }
  }
  if (!have) base = 1.0f;
  *base_out = base;

  /* Pass 2: per sub-channel width, PoT, FPoT and codes; then steps 2-4. */
#pragma omp parallel for schedule(dynamic, 1) reduction(| : status)
  for (int64_t t = 0; t < T; ++t) {
    int gmax = -1000;
    for (int64_t k = 0; k < K; ++k) {
      float dx[ORC_TILE];
      float Mi = 0.0f;
      int nonfinite = 0;
      for (int i = 0; i < ORC_TILE; ++i) {
        int64_t m = t * ORC_TILE + i;
        dx[i] = x_t[m * K + k] - x_prev[m * K + k];
        float a = fabsf(dx[i]);
        if (!isfinite(a)) nonfinite = 1;
        else if (a > Mi) Mi = a;
      }
      if (nonfinite) {
        status |= ORC_ST_NONFINITE;
        Mi = 0.0f;
        for (int i = 0; i < ORC_TILE; ++i) dx[i] = 0.0f;
      }
      /* Eq. 3 with the dynamic base: the smallest P >= 0 with M_i <= base * 2^P. */
      int PoT = 0;
      if (Mi > 0.0f)
        while ((double)Mi > ldexp((double)base, PoT) && PoT <= ORC_POT_MAX) ++PoT;
      if (PoT > ORC_POT_MAX) {
        status |= ORC_ST_RANGE;
        PoT = ORC_POT_MAX;
      }
      /* width by binning M_i against the predefined thresholds Thr_N */
      int b;
      if (force_bits) b = force_bits;
      else if ((double)Mi <= ldexp(1.0, thr_lb + t0)) b = 2;
      else if ((double)Mi <= ldexp(1.0, thr_lb + t0 + 2)) b = 4;
      else if ((double)Mi <= ldexp(1.0, thr_lb + t0 + 4)) b = 6;
      else b = 8;
      int FPoT = (b - 2) - PoT; /* relative to the base: PCeil = 2^(b-2) */
      for (int i = 0; i < ORC_TILE; ++i) {
        volatile float u = dx[i] / base;              /* IEEE fp32 division */
        double v = (double)u * ldexp(1.0, b - 2 - PoT); /* exact power-of-two scaling */
        int32_t q = (int32_t)nearbyint(v);             /* ties to even */
        if (abs(q) > (1 << (b - 2))) status |= ORC_ST_RANGE;
        codes[(t * ORC_TILE + i) * K + k] = (int8_t)q;
      }
      bits[t * K + k] = (int8_t)b;
      fpot[t * K + k] = (int8_t)FPoT;
      pot[t * K + k] = (int16_t)PoT;
      if (FPoT > gmax) gmax = FPoT;
    }
    g_ref[t] = gmax;
    encode_tile(t, K, codes, bits, fpot, count, rec_word, rec_k, rec_tag, rec_j, shift);
  }
  return status;
}

/*
 * Epilogue of the dynamic-base variant: the code unit is base * 2^-FPoT, so
 *   a = (float)acc;  a = a * 2^(-g_ref) (exact);  a = a * base;  a = a * w_scale[n];
 *   y = y_prev + a;  bf16 outputs round y to nearest-even.  No FMA.
 */
void fmdq_orc_epilogue_dyn_f32(int64_t M, int64_t N, const int64_t* acc, const int32_t* g_ref,
                               float base, const float* w_scale, const float* y_prev, int out_bf16,
                               float* y_out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    int64_t t = m / ORC_TILE;
    float p2 = (float)ldexp(1.0, -g_ref[t]);
    for (int64_t n = 0; n < N; ++n) {
      volatile float a = (float)acc[m * N + n];
      a = a * p2;
      a = a * base;
      a = a * w_scale[n];
      volatile float y = y_prev[m * N + n] + a;
      float r = y;
      if (out_bf16) r = bf16_bits_to_float(float_to_bf16_bits(y));
      y_out[m * N + n] = r;
    }
  }
}

/* Signed value of the 2-bit field of slice j of a b-bit code: the top slice
 * (j == b/2 - 1) carries the sign of the two's-complement pattern. */
static int slice_digit(uint32_t field, int j, int b) {
  if (j == b / 2 - 1 && field >= 2) return (int)field - 4;
  return (int)field;
}

int fmdq_orc_slice_digit(uint32_t field, int j, int b) { return slice_digit(field, j, b); }

/* ------------------------------------------- runtime requantization (step 5) */

/*
 * Accumulation over the encoded stream of each tile, in ascending FPoT order:
 * before a record whose FPoT differs from the previous one, the running sum is
 * shifted left by the difference (Fig. 6); then slice * weight is added.  The
 * running sum ends in units of the tile's last FPoT and is shifted once more
 * to g_ref, the finest FPoT of the tile.  Weights w_q are [N x K] int8.
 *
 * Only tiles t with tile_mask == NULL or tile_mask[t] != 0 are computed;
 * acc is [M x N] int64.
 */
void fmdq_orc_acc_slices(int64_t M, int64_t K, int64_t N, const uint32_t* rec_word,
                         const uint16_t* rec_k, const int8_t* rec_tag, const uint8_t* rec_j,
                         const int32_t* count, const int8_t* bits, const int32_t* g_ref,
                         const int8_t* w_q, const uint8_t* tile_mask, int64_t* acc) {
  const int64_t T = M / ORC_TILE;
  const int64_t cap = 4 * K;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    if (tile_mask && !tile_mask[t]) continue;
    for (int i = 0; i < ORC_TILE; ++i) {
      int64_t m = t * ORC_TILE + i;
      for (int64_t n = 0; n < N; ++n) {
        int64_t s = 0;
        int prev = 0;
        for (int64_t r = 0; r < count[t]; ++r) {
          int tag = rec_tag[t * cap + r];
          if (r > 0 && tag != prev) s = s * ((int64_t)1 << (tag - prev));
          prev = tag;
          int k = rec_k[t * cap + r];
          int j = rec_j[t * cap + r];
          int b = bits[t * K + k];
          uint32_t field = (rec_word[t * cap + r] >> (2 * i)) & 3u;
          s += (int64_t)slice_digit(field, j, b) * (int64_t)w_q[n * K + k];
        }
        if (count[t] > 0) s = s * ((int64_t)1 << (g_ref[t] - prev));
        acc[m * N + n] = s;
      }
    }
  }
}

/*
 * The same accumulator by its plain definition: every code is brought to the
 * tile's finest scale by 2^(g_ref - FPoT) and the products are summed,
 *   acc[m,n] = sum_k codes[m,k] * 2^(g_ref(t) - FPoT(t,k)) * w_q[n,k].
 */
void fmdq_orc_acc_direct(int64_t M, int64_t K, int64_t N, const int8_t* codes,
                         const int8_t* fpot, const int32_t* g_ref, const int8_t* w_q,
                         const uint8_t* tile_mask, int64_t* acc) {
  const int64_t T = M / ORC_TILE;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t t = 0; t < T; ++t) {
    if (tile_mask && !tile_mask[t]) continue;
    for (int i = 0; i < ORC_TILE; ++i) {
      int64_t m = t * ORC_TILE + i;
      for (int64_t n = 0; n < N; ++n) {
        int64_t s = 0;
        for (int64_t k = 0; k < K; ++k) {
          int64_t v = (int64_t)codes[m * K + k] * ((int64_t)1 << (g_ref[t] - fpot[t * K + k]));
          s += v * (int64_t)w_q[n * K + k];
        }
        acc[m * N + n] = s;
      }
    }
  }
}

/* --------------------------------------------------------------- epilogue */

/*
 * Inverse quantization and reverse differential (section 4.2, inverse
 * quantization unit then accumulation unit; section 4.3, cached outputs added
 * to the partial sum):
 *   dY = acc * 2^(-lb - g_ref) * w_scale[n];   Y_t = Y_{t-1} + dY.
 * fp32, in this order, without fused multiply-add:
 *   a = (float)acc;  a = a * 2^(-lb-g_ref) (exact);  a = a * w_scale[n];
 *   y = y_prev + a;  bf16 outputs round y to nearest-even.
 * y_prev and y_out are fp32 arrays holding the values (bf16 widened exactly);
 * out_bf16 selects the final rounding.  Rows of masked-out tiles are skipped.
 */
void fmdq_orc_epilogue_f32(int64_t M, int64_t N, const int64_t* acc, const int32_t* g_ref, int lb,
                           const float* w_scale, const float* y_prev, int out_bf16,
                           const uint8_t* tile_mask, float* y_out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    int64_t t = m / ORC_TILE;
    if (tile_mask && !tile_mask[t]) continue;
    float p2 = (float)ldexp(1.0, -lb - g_ref[t]);
    for (int64_t n = 0; n < N; ++n) {
      volatile float a = (float)acc[m * N + n];
      a = a * p2;
      a = a * w_scale[n];
      volatile float y = y_prev[m * N + n] + a;
      float r = y;
      if (out_bf16) r = bf16_bits_to_float(float_to_bf16_bits(y));
      y_out[m * N + n] = r;
    }
  }
}

/* The same epilogue evaluated in fp64 without intermediate rounding (used to
 * bound the fp32 order above). */
void fmdq_orc_epilogue_f64(int64_t M, int64_t N, const int64_t* acc, const int32_t* g_ref, int lb,
                           const float* w_scale, const float* y_prev, const uint8_t* tile_mask,
                           double* y_out) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    int64_t t = m / ORC_TILE;
    if (tile_mask && !tile_mask[t]) continue;
    double p2 = ldexp(1.0, -lb - g_ref[t]);
    for (int64_t n = 0; n < N; ++n)
      y_out[m * N + n] = (double)y_prev[m * N + n] + (double)acc[m * N + n] * p2 * (double)w_scale[n];
  }
}

/* ------------------------------------------------------ FFN activation */

/*
 * GELU between the two linear layers of a DiT feed-forward block (section
 * 4.3, "Operator Mapping": the activation is fused with the first layer's
 * output).  The pages name GELU without a variant; this is its definition,
 * GELU(y) = y * Phi(y), with the normal CDF written Phi(y) = erfc(-y / sqrt 2) / 2
 * (the same function as (1 + erf(y / sqrt 2)) / 2, without the cancellation
 * of 1 + erf in the negative tail), evaluated in fp64 on the layer's cached
 * output value y (fp32, or bf16 widened exactly) and rounded to fp32, then
 * to bf16 (RNE) when out_bf16 is set.
 */
void fmdq_orc_gelu(const float* y, int64_t n, int out_bf16, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    double v = (double)y[i];
    double g = 0.5 * v * erfc(-v / sqrt(2.0));
    float r = (float)g;
    if (out_bf16) r = bf16_bits_to_float(float_to_bf16_bits(r));
    out[i] = r;
  }
}

/* ------------------------------------------------------------- attention */

/*
 * Symmetric int8 quantization of each row of a [rows x cols] fp32 matrix
 * (the weight rule of section 5.1, A8W8, applied per row): scale = max|row| /
 * 127 (one fp32 division), q = rne(x / scale) (one fp32 division, then
 * round half to even), so |q| <= 127; an all-zero row gets scale 0 and codes 0.
 * Used for the attention operands K (per key) and V (per head dimension),
 * which section 4.3 runs in INT8.
 */
void fmdq_orc_quant_rows(const float* x, int64_t rows, int64_t cols, int8_t* q, float* scale) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    float mx = 0.0f;
    for (int64_t c = 0; c < cols; ++c) {
      float a = fabsf(x[r * cols + c]);
      if (a > mx) mx = a;
    }
    volatile float s = mx / 127.0f;
    scale[r] = s;
    for (int64_t c = 0; c < cols; ++c) {
      if (mx == 0.0f) {
        q[r * cols + c] = 0;
      } else {
        volatile float v = x[r * cols + c] / s;
        q[r * cols + c] = (int8_t)nearbyintf(v);
      }
    }
  }
}

/*
 * Block-masked softmax over the rows of a [rows x cols] score matrix (section
 * 3.2, Sparse Attention Reuse: pruned blocks of the score matrix are never
 * computed).  Entry (r, c) takes part iff mask[(r / blk) * mask_cols + c / blk]
 * is nonzero; P = exp(s - m) / sum over the row's kept entries, m their
 * maximum, evaluated in fp64 and rounded to fp32; pruned entries are 0.  A
 * row with no kept entry is all 0.
 */
void fmdq_orc_masked_softmax(const float* s, int64_t rows, int64_t cols, const uint8_t* mask, int64_t blk,
                             int64_t mask_cols, float* p) {
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    const uint8_t* mrow = mask + (r / blk) * mask_cols;
    double m = -INFINITY;
    for (int64_t c = 0; c < cols; ++c)
      if (mrow[c / blk] && (double)s[r * cols + c] > m) m = (double)s[r * cols + c];
    double sum = 0.0;
    for (int64_t c = 0; c < cols; ++c)
      if (mrow[c / blk]) sum += exp((double)s[r * cols + c] - m);
    for (int64_t c = 0; c < cols; ++c)
      p[r * cols + c] = mrow[c / blk] ? (float)(exp((double)s[r * cols + c] - m) / sum) : 0.0f;
  }
}

/* bf16 helpers exposed for the tests (exact widening, RNE narrowing). */
void fmdq_orc_bf16_to_f32(const uint16_t* h, int64_t n, float* f) {
  for (int64_t i = 0; i < n; ++i) f[i] = bf16_bits_to_float(h[i]);
}
void fmdq_orc_f32_to_bf16(const float* f, int64_t n, uint16_t* h) {
  for (int64_t i = 0; i < n; ++i) h[i] = float_to_bf16_bits(f[i]);
}

int fmdq_orc_pot_max(void) { return ORC_POT_MAX; }

/* Thread count of the OpenMP loops above (for timing at 1 thread and at all
 * cores); it changes no result. */
#include <omp.h>
void fmdq_orc_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
int fmdq_orc_max_threads(void) { return omp_get_max_threads(); }
