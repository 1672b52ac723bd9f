// Element-wise kernels of sparse attention reuse with INT8 FMDQ operands
// (DSTAR section 3.2 "Sparse Attention Reuse"; section 4.3 "Attention
// Operation": every attention MMA runs in INT8, activations through FMDQ at
// 8 bits).  The contractions themselves run in the FMDQ quantizer and the
// slice GEMM (batched over heads, block-sparse); these kernels prepare the
// weight-side operands and the softmax between the two products.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "fmdq_device.cuh"

namespace fmdq {

namespace cg = cooperative_groups;

namespace {

template <typename TIn>
__device__ __forceinline__ float ld_f(const TIn* p) {
  if constexpr (sizeof(TIn) == 2) return __bfloat162float(*p);
  else return *p;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// 16 bytes of a row as fp32 values: 8 bf16 or 4 fp32 elements.
template <typename TIn>
struct Vec16 {
  static constexpr int N = 16 / (int)sizeof(TIn);
  __device__ static void load(const TIn* p, float (&f)[N]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    if constexpr (sizeof(TIn) == 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) f[2 * i] = __uint_as_float(u[i] << 16), f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) f[i] = __uint_as_float(u[i]);
    }
  }
};

// Symmetric int8 per row (the A8W8 weight rule of section 5.1 applied to the
// key rows): scale = max|row| / 127, q = rne(x / scale), both fp32
// divisions; an all-zero row gets scale 0 and codes 0.  scale_out = scale *
// scale_mul (one fp32 product: the score scaling folded into the weights).
// One warp per row, 16 bytes of the row per lane and step (cols is a
// multiple of 32, rows start on 16-byte boundaries).
template <typename TIn>
__global__ void __launch_bounds__(256) quant_rows_kernel(const TIn* __restrict__ x, int64_t ld, int64_t rows,
                                                         int64_t cols, int8_t* __restrict__ q, int64_t ldq,
                                                         float* __restrict__ scale_out, float scale_mul) {
  using V = Vec16<TIn>;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const TIn* xr = x + row * ld;
  float mx = 0.f;
  for (int64_t c = (int64_t)lane * V::N; c < cols; c += 32 * V::N) {
    float f[V::N];
    V::load(xr + c, f);
#pragma unroll
    for (int i = 0; i < V::N; ++i) mx = fmaxf(mx, fabsf(f[i]));
  }
  mx = warp_max(mx);
  const float s = __fdiv_rn(mx, 127.f);
  if (lane == 0) scale_out[row] = __fmul_rn(s, scale_mul);
  for (int64_t c = (int64_t)lane * V::N; c < cols; c += 32 * V::N) {
    float f[V::N];
    V::load(xr + c, f);
    uint32_t w[V::N / 4];
#pragma unroll
    for (int i = 0; i < V::N / 4; ++i) {
      uint32_t b = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int code = mx == 0.f ? 0 : __float2int_rn(__fdiv_rn(f[4 * i + e], s));
        b |= ((uint32_t)code & 0xFFu) << (8 * e);
      }
      w[i] = b;
    }
    if constexpr (V::N == 8) *reinterpret_cast<uint2*>(q + row * ldq + c) = make_uint2(w[0], w[1]);
    else *reinterpret_cast<uint32_t*>(q + row * ldq + c) = w[0];
  }
}

// The same rule per column of each head's V ([S x d] rows h S .. h S + S - 1),
// written transposed: vqt[(h d + j) S + s] = rne(V[h S + s][j] / scale[h d + j]).
// A cluster of kColsCluster CTAs per (head, 32-column group), each owning
// S / kColsCluster rows: column maxima of its rows, exchanged through
// distributed shared memory, then the codes of its rows (consecutive threads:
// consecutive s).
constexpr int kColsCluster = 8;

template <typename TIn>
__global__ void __cluster_dims__(kColsCluster, 1, 1) __launch_bounds__(256)
    quant_cols_t_kernel(const TIn* __restrict__ v, int64_t ld, int64_t S, int64_t d, int8_t* __restrict__ vqt,
                        float* __restrict__ scale) {
  __shared__ float red[8][32];
  __shared__ float part[32];  // this CTA's column maxima, read by the whole cluster
  __shared__ float sc[32], mxs[32];
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = blockIdx.x / kColsCluster, groups = d / 32;
  const int64_t h = unit / groups, j0 = 32 * (unit % groups);
  const int64_t s_lo = S * rank / kColsCluster, s_hi = S * (rank + 1) / kColsCluster;
  const TIn* base = v + h * S * ld + j0;
  float mx = 0.f;
  for (int64_t s = s_lo + warp; s < s_hi; s += 8) mx = fmaxf(mx, fabsf(ld_f(base + s * ld + lane)));
  red[warp][lane] = mx;
  __syncthreads();
  if (warp == 0) {
    float m = red[0][lane];
    for (int w = 1; w < 8; ++w) m = fmaxf(m, red[w][lane]);
    part[lane] = m;
  }
  cluster.sync();  // every CTA's partial maxima written
  if (warp == 0) {
    float m = 0.f;
    for (int q = 0; q < kColsCluster; ++q) m = fmaxf(m, cluster.map_shared_rank(part, q)[lane]);
    const float s = __fdiv_rn(m, 127.f);
    mxs[lane] = m, sc[lane] = s;
    if (rank == 0) scale[h * d + j0 + lane] = s;
  }
  cluster.sync();  // no CTA leaves while another may still read its maxima; sc visible to the block
  using V = Vec16<TIn>;
  for (int64_t s = s_lo + threadIdx.x; s < s_hi; s += 256) {
    const TIn* row = base + s * ld;
#pragma unroll
    for (int c = 0; c < 32; c += V::N) {
      float f[V::N];
      V::load(row + c, f);
#pragma unroll
      for (int e = 0; e < V::N; ++e) {
        const int j = c + e;
        vqt[(h * d + j0 + j) * S + s] = mxs[j] == 0.f ? (int8_t)0 : (int8_t)__float2int_rn(__fdiv_rn(f[e], sc[j]));
      }
    }
  }
}

// Softmax over the kept blocks of each score row (section 3.2: pruned blocks
// of the score matrix are never computed); pruned entries become 0.  Row r
// is query r mod S of its head; its mask row is bits[(r mod S) / 128] (bit c:
// key block c kept).  The pages leave the softmax's precision open and P
// decides integer codes, so it is evaluated in fp64 (CUDA's double exp, fp64
// sum and division) and rounded once to fp32.  One block of 256 threads per
// row (S <= 4096): each thread holds the kept scores of columns
// tid + 256 i in registers, so every score is read once and every exp is
// evaluated once; the maximum and the sum are block reductions.
constexpr int kSmThreads = 256;
// Four rows per SM at once (at most 64 registers a thread): a row's block waits
// on its score loads and its two reductions, and more resident rows hide
// that (measured on the 32-head, 4096-token step: 3.96 -> 3.03 ms with three
// rows resident before).
constexpr int kSmBlocks = 4;
constexpr int kSmPer = 32 * kBlockM / kSmThreads;  // S <= 32 blocks of 128 columns

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kSmThreads, kSmBlocks) masked_softmax_kernel(const float* __restrict__ sc, float* __restrict__ pr,
                                                                    int64_t S, const __grid_constant__ BlockMask mk) {
  __shared__ float s_max[kSmThreads / 32];
  __shared__ double s_sum[kSmThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = blockIdx.x;
  const uint64_t keep = mk.bits[(r % S) / kBlockM];
  const float* x = sc + r * S;
  float v[kSmPer];
  uint32_t kept = 0;  // bit i: column tid + 256 i is kept
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < kSmPer; ++i) {
    const int64_t c = threadIdx.x + (int64_t)kSmThreads * i;
    v[i] = 0.f;
    if (c < S && ((keep >> (c / kBlockM)) & 1ull)) {
      v[i] = x[c];
      kept |= 1u << i;
      m = fmaxf(m, v[i]);
    }
  }
  m = warp_max(m);
  if (lane == 0) s_max[warp] = m;
  __syncthreads();
  m = s_max[0];
#pragma unroll
  for (int w = 1; w < kSmThreads / 32; ++w) m = fmaxf(m, s_max[w]);
  const double md = (double)m;
  double e[kSmPer];
  double l = 0.0;
#pragma unroll
  for (int i = 0; i < kSmPer; ++i) {
    e[i] = ((kept >> i) & 1u) ? exp((double)v[i] - md) : 0.0;
    l += e[i];
  }
  l = warp_sum_d(l);
  if (lane == 0) s_sum[warp] = l;
  __syncthreads();
  double sum = s_sum[0];
#pragma unroll
  for (int w = 1; w < kSmThreads / 32; ++w) sum += s_sum[w];
  // e / sum for the row's one divisor: q0 = RN(e rs) with rs = RN(1/sum), one
  // Newton-Raphson correction with the exact FMA residual (faithful), then
  // Markstein's correction (IBM J. Res. Dev. 34(1), 1990), which gives the
  // correctly rounded quotient; sum >= 1 (the maximum's own term is 1) and
  // every e in [0, 1], so no step leaves the normal range but for e = 0.
  const double rs = __drcp_rn(sum);
  float* o = pr + r * S;
#pragma unroll
  for (int i = 0; i < kSmPer; ++i) {
    const int64_t c = threadIdx.x + (int64_t)kSmThreads * i;
    if (c >= S) continue;
    float pv = 0.f;
    if ((kept >> i) & 1u) {
      const double q0 = __dmul_rn(e[i], rs);
      const double q1 = __fma_rn(__fma_rn(-q0, sum, e[i]), rs, q0);
      pv = (float)__fma_rn(__fma_rn(-q1, sum, e[i]), rs, q1);
    }
    o[c] = pv;
  }
}

}  // namespace

int launch_quant_rows(const void* x, int64_t ld, int64_t rows, int64_t cols, int in_bf16, int8_t* q, int64_t ldq,
                      float* scale, float scale_mul, void* stream) {
  if (rows == 0) return 0;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (in_bf16)
    quant_rows_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        static_cast<const __nv_bfloat16*>(x), ld, rows, cols, q, ldq, scale, scale_mul);
  else
    quant_rows_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>(static_cast<const float*>(x), ld, rows, cols,
                                                                      q, ldq, scale, scale_mul);
  return (int)cudaGetLastError();
}

int launch_quant_cols_t(const void* v, int64_t ld, int64_t heads, int64_t S, int64_t d, int in_bf16, int8_t* vqt,
                        float* scale, void* stream) {
  if (heads == 0) return 0;
  const dim3 grid((unsigned)(heads * (d / 32) * kColsCluster));
  if (in_bf16)
    quant_cols_t_kernel<__nv_bfloat16><<<grid, 256, 0, (cudaStream_t)stream>>>(
        static_cast<const __nv_bfloat16*>(v), ld, S, d, vqt, scale);
  else
    quant_cols_t_kernel<float><<<grid, 256, 0, (cudaStream_t)stream>>>(static_cast<const float*>(v), ld, S, d, vqt,
                                                                        scale);
  return (int)cudaGetLastError();
}

int launch_masked_softmax(const float* sc, float* pr, int64_t rows, int64_t S, const BlockMask& mk, void* stream) {
  if (rows == 0) return 0;
  if (S > (int64_t)kSmThreads * kSmPer) return (int)cudaErrorInvalidValue;  // the host admits S <= 4096
  masked_softmax_kernel<<<(unsigned)rows, kSmThreads, 0, (cudaStream_t)stream>>>(sc, pr, S, mk);
  return (int)cudaGetLastError();
}

}  // namespace fmdq
