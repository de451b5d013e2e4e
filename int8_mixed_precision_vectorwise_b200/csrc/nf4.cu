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
// bytes of scales).  For few tokens it is bound by HBM and by the unpacking
// work (a shared-memory level lookup per weight), so it runs on the CUDA
// cores with packed fp32 FMAs; the layout is described at k_nf4_gemv.
#include <cuda_fp16.h>

#include <algorithm>
#include <cmath>
#include <cstring>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int NB = 64;            // weights per scale block
constexpr int NF_WARPS = 8;
constexpr int NF_THREADS = 32 * NF_WARPS;
constexpr int NF_XBUF = 4096;     // fp32 elements of X per staging buffer (16 KB, two buffers)
constexpr int NF_STEP = 256;      // weights of a row per step of an octet (128 bytes)

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
#pragma unroll
  for (int i = 0; i < 16; ++i)
    if (threadIdx.x == i) lut[i] = tb.level[i];
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

// out [M, N] = fp16(X [M, K] . W^T), MT >= M token slots (1, 2, 4 or 8).
//
// Layout of the work: eight lanes (an octet) share one row and read its 128-byte
// segment of 256 weights per step, lane q taking the 32 weights k0 + 32q ..
// k0 + 32q + 31 (one 16-byte load, half a scale block).  A warp's four octets take
// four consecutive rows, R such groups at a time, so a CTA of 8 warps owns
// 32R consecutive rows.  The CTA walks its K range (all of K, or 1/S of it
// when S CTAs of a cluster split K) in chunks of X staged as fp32 in shared
// memory, double-buffered: the next chunk is loaded into registers while the
// current one is used and stored behind it, one barrier per chunk.  In a chunk
// the 16-byte granule g of token row t sits at g ^ ((k >> 5) & 7), so the eight
// lanes of an octet, which read the same granule offset of eight different
// 32-weight groups, hit eight different bank groups, and the four octets of a
// warp read the same addresses (broadcast).  The weight codes of the next step
// are loaded while the current step is computed.
//
// Arithmetic (fp32): per row, token and half block, two chains of 16 fused
// multiply-adds (even and odd k, one packed f32x2 FMA per pair of k), their sum
// times the block scale added to the lane's running sum; then a 3-level
// shuffle sum over the octet and, with S > 1, the S partial sums of the cluster
// added in rank order through distributed shared memory.  Deterministic.
template <int MT, int R>
struct Nf4Shape {
  static constexpr int KC = NF_XBUF / MT;          // k per chunk (a multiple of 256)
  static constexpr int ROWS = 32 * R;              // rows per CTA
  static constexpr int STEPS = KC / NF_STEP;       // 256-weight steps per chunk
};

__device__ __forceinline__ float ld_shared_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

__device__ __forceinline__ float lut_at(const float* lut, uint32_t byte_off) {
  return *reinterpret_cast<const float*>(reinterpret_cast<const char*>(lut) + byte_off);
}

template <int MT, int R>
__global__ void __launch_bounds__(NF_THREADS, (MT <= 2 && R <= 2) ? 3 : 2) k_nf4_gemv(const __half* __restrict__ X, int M,
                                                            const uint8_t* __restrict__ packed,
                                                            const float* __restrict__ absmax, int N, int K,
                                                            Nf4Tables tb, int S, __half* __restrict__ out) {
  using Sh = Nf4Shape<MT, R>;
  __shared__ float lut[16];
  __shared__ __align__(16) float xs[2][NF_XBUF];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int oct = lane >> 3, q = lane & 7;
#pragma unroll
  for (int i = 0; i < 16; ++i)                     // constant indices keep the tables in the parameter space
    if (tid == i) lut[i] = tb.level[i];

  // this CTA's rows and K range (S CTAs of one cluster share the rows)
  const int split = S > 1 ? static_cast<int>(blockIdx.x % S) : 0;
  const int rb = S > 1 ? static_cast<int>(blockIdx.x / S) : static_cast<int>(blockIdx.x);
  const int nsteps = (K + NF_STEP - 1) / NF_STEP;
  const int s0 = static_cast<int>(static_cast<long long>(split) * nsteps / S);
  const int s1 = static_cast<int>(static_cast<long long>(split + 1) * nsteps / S);
  const int kb = s0 * NF_STEP, ke = min(K, s1 * NF_STEP);
  const int T = s1 - s0;                           // steps of this CTA
  const int nchunks = (T + Sh::STEPS - 1) / Sh::STEPS;
  const size_t row_bytes = static_cast<size_t>(K) / 2;
  const int blocks_row = K / NB;
  int rows[R];
#pragma unroll
  for (int i = 0; i < R; ++i) rows[i] = rb * Sh::ROWS + (warp * R + i) * 4 + oct;

  // weight codes and block scales of step st for this lane's R rows (zero past the range)
  auto load_step = [&](int st, uint4 (&qv)[R], float (&av)[R]) {
    const int kg = kb + st * NF_STEP + 32 * q;
    const bool ok = kg < ke;
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const size_t n = static_cast<size_t>(min(rows[i], N - 1));  // rows past N repeat the last; never stored
      qv[i] = ok ? __ldcs(reinterpret_cast<const uint4*>(packed + n * row_bytes + kg / 2)) : make_uint4(0, 0, 0, 0);
      av[i] = ok ? __ldg(absmax + n * blocks_row + kg / NB) : 0.f;
    }
  };
  // X chunk c as fp16 pairs in registers (8 per thread), zero past M or the range
  constexpr int XPT = NF_XBUF / 2 / NF_THREADS;
  uint32_t xr[XPT];
  auto load_chunk = [&](int c) {
#pragma unroll
    for (int j = 0; j < XPT; ++j) {
      const int p = tid + NF_THREADS * j;
      const int t = p / (Sh::KC / 2), kp = p % (Sh::KC / 2);
      const int kg = kb + c * Sh::KC + 2 * kp;
      xr[j] = (t < M && kg < ke) ? __ldg(reinterpret_cast<const uint32_t*>(X + static_cast<size_t>(t) * K + kg)) : 0u;
    }
  };
  auto store_chunk = [&](float* buf) {
#pragma unroll
    for (int j = 0; j < XPT; ++j) {
      const int p = tid + NF_THREADS * j;
      const int t = p / (Sh::KC / 2), kp = p % (Sh::KC / 2);
      const int fi = t * Sh::KC + 2 * kp;
      const int phys = (fi >> 2) ^ ((kp >> 4) & 7);
      __half2 h;
      memcpy(&h, &xr[j], 4);
      *reinterpret_cast<float2*>(buf + 4 * phys + (fi & 3)) = __half22float2(h);
    }
  };

  float acc[R][MT];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[i][t] = 0.f;

  uint4 qn[R];
  float an[R];
  if (T > 0) load_step(0, qn, an);
  load_chunk(0);
  store_chunk(xs[0]);
  __syncthreads();
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks) load_chunk(c + 1);
    const float* xb = xs[c & 1];
    for (int j = 0; j < Sh::STEPS; ++j) {
      const int st = c * Sh::STEPS + j;
      if (st >= T) break;
      uint4 qc[R];
      float ac[R];
#pragma unroll
      for (int i = 0; i < R; ++i) { qc[i] = qn[i]; ac[i] = an[i]; }
      if (st + 1 < T) load_step(st + 1, qn, an);
      float2 s[R][MT];
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int t = 0; t < MT; ++t) s[i][t] = make_float2(0.f, 0.f);
      const int g0 = (NF_STEP * j + 32 * q) >> 2;  // granule of this lane's first weight (token 0)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t eb[R], ob[R];                     // byte j: 4 x code of weight 8w + 2j (eb) and 8w + 2j + 1 (ob)
#pragma unroll
        for (int i = 0; i < R; ++i) {
          const uint32_t wd = w == 0 ? qc[i].x : (w == 1 ? qc[i].y : (w == 2 ? qc[i].z : qc[i].w));
          eb[i] = (wd << 2) & 0x3C3C3C3Cu;
          ob[i] = (wd >> 2) & 0x3C3C3C3Cu;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float4 xv[MT];
#pragma unroll
          for (int t = 0; t < MT; ++t)
            xv[t] = *reinterpret_cast<const float4*>(xb + 4 * ((t * (Sh::KC / 4) + g0 + 2 * w + h) ^ q));
#pragma unroll
          for (int i = 0; i < R; ++i) {
            const float2 v01 = make_float2(lut_at(lut, __byte_perm(eb[i], 0, 0x4440 + 2 * h)),
                                           lut_at(lut, __byte_perm(ob[i], 0, 0x4440 + 2 * h)));
            const float2 v23 = make_float2(lut_at(lut, __byte_perm(eb[i], 0, 0x4441 + 2 * h)),
                                           lut_at(lut, __byte_perm(ob[i], 0, 0x4441 + 2 * h)));
#pragma unroll
            for (int t = 0; t < MT; ++t) {
              s[i][t] = __ffma2_rn(make_float2(xv[t].x, xv[t].y), v01, s[i][t]);
              s[i][t] = __ffma2_rn(make_float2(xv[t].z, xv[t].w), v23, s[i][t]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[i][t] = fmaf(ac[i], s[i][t].x + s[i][t].y, acc[i][t]);
    }
    if (c + 1 < nchunks) store_chunk(xs[(c + 1) & 1]);
    __syncthreads();
  }

  // octet sum: lane q == 0 holds the CTA's partial sum of its rows
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float v = acc[i][t];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      acc[i][t] = v;
    }
  if (S == 1) {
    if (q == 0)
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int t = 0; t < MT; ++t)
          if (t < M && rows[i] < N) out[static_cast<size_t>(t) * N + rows[i]] = __float2half_rn(acc[i][t]);
    return;
  }
  // S > 1: partial sums to shared memory (the X buffers are free after the last
  // barrier), then CTA `split` adds the S partials of rows [split, split + 1) * ROWS / S
  // in rank order, reading the other CTAs' shared memory.
  float* red = xs[0];
  if (q == 0)
#pragma unroll
    for (int i = 0; i < R; ++i)
#pragma unroll
      for (int t = 0; t < MT; ++t) red[((warp * R + i) * 4 + oct) * MT + t] = acc[i][t];
  cluster_sync();
  const int r0 = split * Sh::ROWS / S, r1 = (split + 1) * Sh::ROWS / S;
  const uint32_t red_addr = smem_addr(red);
  for (int e = tid; e < (r1 - r0) * MT; e += NF_THREADS) {
    const int rl = r0 + e / MT, t = e % MT;
    float v = 0.f;
    for (int r = 0; r < S; ++r) v += ld_shared_cluster_f32(map_to_rank(red_addr + 4u * (rl * MT + t), r));
    const int n = rb * Sh::ROWS + rl;
    if (t < M && n < N) out[static_cast<size_t>(t) * N + n] = __float2half_rn(v);
  }
  cluster_sync();                                  // keep this CTA's partials alive until all are read
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

namespace {

// Work split of the product: rows per CTA (32R, two choices of R per token
// count) and the number S of CTAs of a cluster that split K.  An SM's time is
// taken as proportional to its share of the work, ceil(CTAs / SMs) times the
// work of one CTA plus one step for its start, times the shared-memory
// wavefronts per 32 weights (1 + MT / R); the smallest estimate wins (fewer,
// larger pieces on ties), keeping at least two steps of 256 weights per CTA.
struct Nf4Plan {
  int R, S, grid;
};

Nf4Plan nf4_plan(int MT, int N, int K, int num_sms) {
  const int r_hi = MT <= 2 ? 4 : 2;
  const int nsteps = (K + NF_STEP - 1) / NF_STEP;
  Nf4Plan best{r_hi, 1, (N + 32 * r_hi - 1) / (32 * r_hi)};
  double best_eff = -1.0;
  for (int R = r_hi; R >= r_hi / 2; R /= 2) {
    const int rb = (N + 32 * R - 1) / (32 * R);
    const double ideal = static_cast<double>(N) * K / num_sms;
    for (int S = 1; S <= 8; ++S) {
      if (S > 1 && nsteps / S < 2) break;
      const long long ctas = static_cast<long long>(rb) * S;
      const long long per_sm = (ctas + num_sms - 1) / num_sms;
      // a CTA's start (X staging, first loads) is counted as one more step of its rows;
      // per 32 weights the lookups take one shared-memory wavefront and the X values
      // MT / R more (each lane reads MT values per k and uses them for R rows)
      // (an SM given a single CTA, 8 warps, hides latency about half as well)
      const double t = static_cast<double>(per_sm) * 32.0 * R * (static_cast<double>(K) / S + NF_STEP) *
                       (1.0 + static_cast<double>(MT) / R) * (per_sm < 2 ? 2.0 : 1.0);
      const double eff = ideal / t * (1.0 + static_cast<double>(MT) / r_hi);
      if (eff > best_eff * 1.02) {
        best_eff = eff;
        best = {R, S, static_cast<int>(ctas)};
      }
    }
  }
  return best;
}

template <int MT, int R>
cudaError_t launch_gemv_t(const Nf4Plan& p, const __half* X, int M, const uint8_t* packed, const float* absmax,
                          int N, int K, const Nf4Tables& tb, __half* out, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(NF_THREADS);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = p.S > 1 ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_nf4_gemv<MT, R>, X, M, packed, absmax, N, K, tb, p.S, out);
}

}  // namespace

cudaError_t launch_nf4_gemv(const __half* X, int M, const uint8_t* packed, const float* absmax, int N, int K,
                            __half* out, int num_sms, cudaStream_t st) {
  if (M < 1 || M > kNf4MaxTokens) return cudaErrorInvalidValue;
  const Nf4Tables tb = nf4_tables();
  const int MT = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
  const Nf4Plan p = nf4_plan(MT, N, K, num_sms);
  const bool hi = p.R == (MT <= 2 ? 4 : 2);
  switch (MT) {
    case 1: return hi ? launch_gemv_t<1, 4>(p, X, M, packed, absmax, N, K, tb, out, st)
                      : launch_gemv_t<1, 2>(p, X, M, packed, absmax, N, K, tb, out, st);
    case 2: return hi ? launch_gemv_t<2, 4>(p, X, M, packed, absmax, N, K, tb, out, st)
                      : launch_gemv_t<2, 2>(p, X, M, packed, absmax, N, K, tb, out, st);
    case 4: return hi ? launch_gemv_t<4, 2>(p, X, M, packed, absmax, N, K, tb, out, st)
                      : launch_gemv_t<4, 1>(p, X, M, packed, absmax, N, K, tb, out, st);
    default: return hi ? launch_gemv_t<8, 2>(p, X, M, packed, absmax, N, K, tb, out, st)
                       : launch_gemv_t<8, 1>(p, X, M, packed, absmax, N, K, tb, out, st);
  }
}

}  // namespace i8lt
