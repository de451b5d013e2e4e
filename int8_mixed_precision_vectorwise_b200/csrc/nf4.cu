// 4-bit NF4 weight-only decode product, blocksize 64 ("Loading an LLM in 4
// bits using bitsandbytes", sections "Normalized Float" and "Double
// Quantization": 4-bit values optimised for normally distributed weights,
// quantised in blocks of 64 that each keep a 32-bit scale, the product
// computed after dequantisation).
//
//   levels  v[0..15]: the NormalFloat values — equal steps in probability on
//           each half of N(0, 1) (8 above zero, 7 below, and 0), divided by the
//           outermost one — computed on the host in double precision with an
//           inverse normal CDF of our own (Newton's method on erfc), stored fp32
//   quant   per block of 64 consecutive weights of a row: a = max |w|,
//           y = w / a (fp32), code = number of level midpoints below y;
//           element 2j of a row in the low nibble of byte j, 2j + 1 in the high
//   dequant W^ = fp16(fl32(v[code] * a))
//   gemv    out[t, n] = fp16(sum_b a_b * sum_{k in b} x[t, k] * v[code[n, k]])
//           (fp32 accumulation, the block scale applied once per half block)
//
// The product streams the packed weight once (K/2 bytes per row plus K/16
// bytes of scales); for few tokens it is bound by HBM and by the unpacking
// work, so it runs on the CUDA cores: each warp takes 4 rows at a time (four
// independent 16-byte loads per lane in flight), X is staged in shared memory
// as fp32 chunks that all warps of the CTA share, and the 16 levels sit in
// shared memory (16 banks: lanes reading different levels never conflict).
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>

#include "kernels.cuh"

namespace i8lt {

namespace {

constexpr int NB = 64;            // weights per scale block
constexpr int NF_WARPS = 8;
constexpr int NF_THREADS = 32 * NF_WARPS;
constexpr int NF_X_FLOATS = 8192; // fp32 elements of X staged per chunk (32 KB)

// Standard normal quantile by Newton's method on Phi(x) = erfc(-x / sqrt 2) / 2.
double normal_quantile(double p) {
  const double rt2 = std::sqrt(2.0), rt2pi = std::sqrt(2.0 * M_PI);
  double x = 0.0;
  for (int it = 0; it < 100; ++it) {
    const double f = 0.5 * std::erfc(-x / rt2) - p;
    const double step = f / (std::exp(-0.5 * x * x) / rt2pi);
    x -= step;
    if (std::fabs(step) <= 1e-17 * std::max(1.0, std::fabs(x))) break;
  }
  return x;
}

}  // namespace

Nf4Tables nf4_tables() {
  const double p_star = 1.0 - (1.0 / 32.0 + 1.0 / 30.0) / 2.0;
  const double top = normal_quantile(p_star);
  double v[16];
  v[7] = 0.0;
  for (int i = 1; i <= 8; ++i) v[7 + i] = normal_quantile(0.5 + i * (p_star - 0.5) / 8.0) / top;
  for (int i = 1; i <= 7; ++i) v[7 - i] = -normal_quantile(0.5 + i * (p_star - 0.5) / 7.0) / top;
  Nf4Tables t;
  for (int i = 0; i < 16; ++i) t.level[i] = static_cast<float>(v[i]);
  for (int i = 0; i < 15; ++i) t.mid[i] = (t.level[i] + t.level[i + 1]) / 2.0f;
  t.mid[15] = 0.f;
  return t;
}

// One warp per block of 64 weights: lane l quantises elements 2l and 2l + 1.
__global__ void __launch_bounds__(256) k_nf4_quantize(const __half* __restrict__ W, int N, int K, Nf4Tables tb,
                                                      uint8_t* __restrict__ packed, float* __restrict__ absmax) {
  const int lane = threadIdx.x & 31;
  const long long nblk = static_cast<long long>(N) * (K / NB);
  for (long long b = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; b < nblk;
       b += (static_cast<long long>(gridDim.x) * blockDim.x) >> 5) {
    const size_t e0 = static_cast<size_t>(b) * NB + 2 * lane;  // blocks tile the row-major weight
    const float2 w = __half22float2(*reinterpret_cast<const __half2*>(W + e0));
    float a = fmaxf(fabsf(w.x), fabsf(w.y));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    uint32_t c[2] = {0u, 0u};
    const float ws[2] = {w.x, w.y};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float y = a > 0.f ? __fdiv_rn(ws[e], a) : 0.f;
#pragma unroll
      for (int i = 0; i < 15; ++i) c[e] += y > tb.mid[i] ? 1u : 0u;
    }
    packed[e0 >> 1] = static_cast<uint8_t>(c[0] | (c[1] << 4));
    if (lane == 0) absmax[b] = a;
  }
}

// W^[n, k] = fp16(fl32(v[code] * a)), two weights (one byte) per thread.
__global__ void __launch_bounds__(256) k_nf4_dequant(const uint8_t* __restrict__ packed,
                                                     const float* __restrict__ absmax, int N, int K, Nf4Tables tb,
                                                     __half* __restrict__ W) {
  __shared__ float lut[16];
  if (threadIdx.x < 16) lut[threadIdx.x] = tb.level[threadIdx.x];
  __syncthreads();
  const size_t nbytes = static_cast<size_t>(N) * K / 2;
  for (size_t j = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; j < nbytes;
       j += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint32_t byte = packed[j];
    const float a = __ldg(absmax + (2 * j) / NB);
    *reinterpret_cast<__half2*>(W + 2 * j) =
        __halves2half2(__float2half_rn(__fmul_rn(lut[byte & 15u], a)), __float2half_rn(__fmul_rn(lut[byte >> 4], a)));
  }
}

// out [M, N] = fp16(X [M, K] . W^T) with MT >= M token slots (a power of two);
// each warp works on R rows at once (fewer for more tokens, to stay in registers).
template <int MT, int R>
__global__ void __launch_bounds__(NF_THREADS) k_nf4_gemv(const __half* __restrict__ X, int M,
                                                         const uint8_t* __restrict__ packed,
                                                         const float* __restrict__ absmax, int N, int K,
                                                         Nf4Tables tb, __half* __restrict__ out) {
  __shared__ float lut[16];
  __shared__ __align__(16) float xs[NF_X_FLOATS];  // [MT][kc] chunk of X as fp32
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < 16) lut[threadIdx.x] = tb.level[threadIdx.x];
  const int kc_max = NF_X_FLOATS / MT;             // a multiple of 512 (MT <= 16)
  const int rows_cta = NF_WARPS * R;
  const size_t row_bytes = static_cast<size_t>(K) / 2;
  const int blocks_row = K / NB;
  for (int g = blockIdx.x; g * rows_cta < N; g += gridDim.x) {
    const int n0 = g * rows_cta + warp * R;        // this warp's rows n0 .. n0 + R - 1
    float acc[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[r][t] = 0.f;
    for (int k0 = 0; k0 < K; k0 += kc_max) {
      const int kc = min(kc_max, K - k0);          // a multiple of 64
      __syncthreads();                             // the previous chunk is no longer read
      for (int i = threadIdx.x; i < MT * (kc / 2); i += NF_THREADS) {
        const int t = i / (kc / 2), j = i - t * (kc / 2);
        float2 f = make_float2(0.f, 0.f);
        if (t < M) f = __half22float2(*reinterpret_cast<const __half2*>(X + static_cast<size_t>(t) * K + k0 + 2 * j));
        *reinterpret_cast<float2*>(xs + t * kc + 2 * j) = f;
      }
      __syncthreads();
      // a lane takes 32 consecutive weights (16 bytes, half a scale block) per row and step
      const int units = kc / 32;
      for (int u0 = 0; u0 < units; u0 += 32) {
        const int u = u0 + lane;
        if (u >= units) continue;
        const int kk = 32 * u;                     // offset in the chunk
        uint4 q[R];
        float a[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const int n = min(n0 + r, N - 1);        // rows past N repeat the last one; never stored
          q[r] = __ldcs(reinterpret_cast<const uint4*>(packed + static_cast<size_t>(n) * row_bytes + (k0 + kk) / 2));
          a[r] = __ldg(absmax + static_cast<size_t>(n) * blocks_row + (k0 + kk) / NB);
        }
        float s[R][MT];
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int t = 0; t < MT; ++t) s[r][t] = 0.f;
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {           // 8 weights (one 32-bit word) per row at a time
          float x[MT][8];
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const float4 lo = *reinterpret_cast<const float4*>(xs + t * kc + kk + 8 * w4);
            const float4 hi = *reinterpret_cast<const float4*>(xs + t * kc + kk + 8 * w4 + 4);
            x[t][0] = lo.x; x[t][1] = lo.y; x[t][2] = lo.z; x[t][3] = lo.w;
            x[t][4] = hi.x; x[t][5] = hi.y; x[t][6] = hi.z; x[t][7] = hi.w;
          }
#pragma unroll
          for (int r = 0; r < R; ++r) {
            const uint32_t wd = w4 == 0 ? q[r].x : (w4 == 1 ? q[r].y : (w4 == 2 ? q[r].z : q[r].w));
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float v = lut[(wd >> (4 * e)) & 15u];
#pragma unroll
              for (int t = 0; t < MT; ++t) s[r][t] = fmaf(x[t][e], v, s[r][t]);
            }
          }
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int t = 0; t < MT; ++t) acc[r][t] = fmaf(a[r], s[r][t], acc[r][t]);
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        float v = acc[r][t];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && t < M && n0 + r < N) out[static_cast<size_t>(t) * N + n0 + r] = __float2half_rn(v);
      }
  }
}

cudaError_t launch_nf4_quantize(const __half* W, int N, int K, uint8_t* packed, float* absmax, int num_sms,
                                cudaStream_t st) {
  const long long nblk = static_cast<long long>(N) * (K / NB);
  const int blocks = static_cast<int>(std::min<long long>((nblk + 7) / 8, static_cast<long long>(num_sms) * 16));
  k_nf4_quantize<<<std::max(blocks, 1), 256, 0, st>>>(W, N, K, nf4_tables(), packed, absmax);
  return cudaGetLastError();
}

cudaError_t launch_nf4_dequant(const uint8_t* packed, const float* absmax, int N, int K, __half* W, int num_sms,
                               cudaStream_t st) {
  const size_t nbytes = static_cast<size_t>(N) * K / 2;
  const int blocks = static_cast<int>(std::min<size_t>((nbytes + 255) / 256, static_cast<size_t>(num_sms) * 16));
  k_nf4_dequant<<<std::max(blocks, 1), 256, 0, st>>>(packed, absmax, N, K, nf4_tables(), W);
  return cudaGetLastError();
}

cudaError_t launch_nf4_gemv(const __half* X, int M, const uint8_t* packed, const float* absmax, int N, int K,
                            __half* out, int num_sms, cudaStream_t st) {
  if (M < 1 || M > kNf4MaxTokens) return cudaErrorInvalidValue;
  const Nf4Tables tb = nf4_tables();
  const int rows = M <= 2 ? 4 : (M <= 4 ? 2 : 1);  // rows per warp of the instantiation below
  const int groups = (N + NF_WARPS * rows - 1) / (NF_WARPS * rows);
  const int grid = std::max(1, std::min(groups, num_sms * 4));
  if (M <= 1) k_nf4_gemv<1, 4><<<grid, NF_THREADS, 0, st>>>(X, M, packed, absmax, N, K, tb, out);
  else if (M <= 2) k_nf4_gemv<2, 4><<<grid, NF_THREADS, 0, st>>>(X, M, packed, absmax, N, K, tb, out);
  else if (M <= 4) k_nf4_gemv<4, 2><<<grid, NF_THREADS, 0, st>>>(X, M, packed, absmax, N, K, tb, out);
  else k_nf4_gemv<8, 1><<<grid, NF_THREADS, 0, st>>>(X, M, packed, absmax, N, K, tb, out);
  return cudaGetLastError();
}

}  // namespace i8lt
