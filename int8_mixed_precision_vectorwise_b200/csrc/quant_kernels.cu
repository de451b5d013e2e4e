// HBM-bound kernels of the LLM.int8() forward:
//   k_quant_rows        fused row absmax calibration + int8 quantisation + outlier
//                       column bitmap ("LLM.int8() Refactoring: Part 1", section
//                       "Improved kernels for inference", int8_vectorwise_quant)
//   k_zero_outlier_cols zero the outlier columns of the codes (the fp16 path owns them)
//   k_outlier_prepare   bitmap -> sorted outlier column list (state.idx), zero CA
//                       columns, gather X[:, O] and fp16(CB[:, O]) for the outlier product
//   k_mm_dequant        int32 -> fp16 with row x column scales / 127^2 + bias
//   k_dequant           int8 weight -> fp16 ("Next steps": int8 dequantize op)
#include <cuda_fp16.h>

#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ uint4 ld_stream_16(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Max |x| over the elements kept on the int8 path and the 8-bit mask of
// elements at or above the threshold, for one vector of 8 fp16 values.
__device__ __forceinline__ void scan8(const uint4& v, float tau, bool use_tau, float& amax, uint32_t& big) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(h[e]);
    const float a0 = fabsf(f.x), a1 = fabsf(f.y);
    if (use_tau && a0 >= tau) big |= 1u << (2 * e); else amax = fmaxf(amax, a0);
    if (use_tau && a1 >= tau) big |= 2u << (2 * e); else amax = fmaxf(amax, a1);
  }
}

__device__ __forceinline__ uint32_t code_byte(float x, float r) {
  int q = __float2int_rn(__fmul_rn(x, r));
  q = max(-127, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

// 8 fp16 values -> 8 int8 codes packed little-endian.
__device__ __forceinline__ uint2 quant8(const uint4& v, float r) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t w[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const float2 a = __half22float2(h[2 * p]);
    const float2 b = __half22float2(h[2 * p + 1]);
    w[p] = code_byte(a.x, r) | (code_byte(a.y, r) << 8) | (code_byte(b.x, r) << 16) | (code_byte(b.y, r) << 24);
  }
  return make_uint2(w[0], w[1]);
}

// OR a vector's outlier bits into the global bitmap.  Must be called by all 32
// lanes of a warp whose lanes hold consecutive vectors (vector index vi).
__device__ __forceinline__ void publish_outliers(uint32_t big, int vi, uint32_t* bitmap) {
  if (!__any_sync(kFull, big != 0)) return;
  uint32_t bits = big << ((vi & 3) * 8);
  bits |= __shfl_xor_sync(kFull, bits, 1);
  bits |= __shfl_xor_sync(kFull, bits, 2);
  if ((threadIdx.x & 3) == 0 && bits) {
    uint32_t* w = bitmap + (vi >> 2);
    if ((__ldcg(w) & bits) != bits) atomicOr(w, bits);   // skip the atomic once set
  }
}

}  // namespace

// One row per group of G threads (G a multiple of 32), 256 threads per block,
// each thread caching up to VPT 16-byte vectors of its row in registers so X
// is read from HBM exactly once.
template <int G, int VPT>
__global__ void __launch_bounds__(256) k_quant_rows(const __half* __restrict__ X, int M, int K, float tau,
                                                    int8_t* __restrict__ CA, float* __restrict__ SCA,
                                                    uint32_t* __restrict__ bitmap) {
  static_assert(G % 32 == 0 && 256 % G == 0, "group size");
  pdl_launch_dependents();
  constexpr int ROWS = 256 / G;
  constexpr int WPR = G / 32;  // warps per row
  __shared__ float red[8];

  const int tid = threadIdx.x;
  const int g = tid / G;
  const int t = tid % G;
  const int row = blockIdx.x * ROWS + g;
  const bool valid = row < M;
  const int nvec = K >> 3;
  const bool use_tau = tau > 0.f;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(valid ? row : 0) * K);

  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = t + i * G;
    v[i] = (valid && vi < nvec) ? ld_stream_16(xr + vi) : make_uint4(0, 0, 0, 0);
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    uint32_t big = 0;
    scan8(v[i], tau, use_tau, amax, big);
    if (use_tau) publish_outliers(big, t + i * G, bitmap);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
  if constexpr (WPR > 1) {
    if ((tid & 31) == 0) red[tid >> 5] = amax;
    __syncthreads();
    amax = red[g * WPR];
#pragma unroll
    for (int w = 1; w < WPR; ++w) amax = fmaxf(amax, red[g * WPR + w]);
  }
  const float r = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
  if (valid) {
    if (t == 0) SCA[row] = amax;
    uint2* cr = reinterpret_cast<uint2*>(CA + static_cast<size_t>(row) * K);
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int vi = t + i * G;
      if (vi < nvec) cr[vi] = quant8(v[i], r);
    }
  }
}

// Rows too long to cache in registers: one block per row, X read twice (the
// second read is served by L2).
__global__ void __launch_bounds__(256) k_quant_rows_stream(const __half* __restrict__ X, int M, int K,
                                                           float tau, int8_t* __restrict__ CA,
                                                           float* __restrict__ SCA, uint32_t* __restrict__ bitmap) {
  __shared__ float red[8];
  pdl_launch_dependents();
  const int row = blockIdx.x;
  const int nvec = K >> 3;
  const bool use_tau = tau > 0.f;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * K);
  float amax = 0.f;
  for (int base = 0; base < nvec; base += 256) {   // uniform trip count for the warp shuffles
    const int vi = base + threadIdx.x;
    const uint4 v = vi < nvec ? xr[vi] : make_uint4(0, 0, 0, 0);
    uint32_t big = 0;
    scan8(v, tau, use_tau, amax, big);
    if (use_tau) publish_outliers(big, vi, bitmap);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float r = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
  if (threadIdx.x == 0) SCA[row] = amax;
  uint2* cr = reinterpret_cast<uint2*>(CA + static_cast<size_t>(row) * K);
  for (int vi = threadIdx.x; vi < nvec; vi += 256) cr[vi] = quant8(xr[vi], r);
}

// Persistent warp-per-row variant for many rows.  Pass 1 streams the row from
// HBM, U 16-byte loads per lane in flight, and reduces |x| with packed fp16
// max (exact: the max of fp16 values is one of them); only vectors whose max
// reaches the threshold take the per-element fp32 path that separates
// outliers.  Pass 2 re-reads the row (now in L2) and writes the codes.  No
// block-level synchronisation: every warp walks its own rows.
template <int U>
__global__ void __launch_bounds__(256) k_quant_rows_warp(const __half* __restrict__ X, int M, int K, float tau,
                                                         int8_t* __restrict__ CA, float* __restrict__ SCA,
                                                         uint32_t* __restrict__ bitmap) {
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  const int nvec = K >> 3;
  const bool use_tau = tau > 0.f;
  for (int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < M; row += nwarps) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * K);
    float amax = 0.f;
    for (int base = 0; base < nvec; base += 32 * U) {  // uniform trip count for the warp votes
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int vi = base + u * 32 + lane;
        v[u] = vi < nvec ? __ldg(xr + vi) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const __half2* h = reinterpret_cast<const __half2*>(&v[u]);
        const __half2 m = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])), __hmax2(__habs2(h[2]), __habs2(h[3])));
        const float vmax = fmaxf(__low2float(m), __high2float(m));
        const bool hot = use_tau && vmax >= tau;  // some element of this vector is an outlier
        if (__any_sync(kFull, hot)) {
          uint32_t big = 0;
          float keep = 0.f;
          if (hot) scan8(v[u], tau, true, keep, big); else keep = vmax;
          amax = fmaxf(amax, keep);
          publish_outliers(big, base + u * 32 + lane, bitmap);
        } else {
          amax = fmaxf(amax, vmax);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
    const float r = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (lane == 0) SCA[row] = amax;
    uint2* cr = reinterpret_cast<uint2*>(CA + static_cast<size_t>(row) * K);
    for (int base = 0; base < nvec; base += 32 * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int vi = base + u * 32 + lane;
        if (vi < nvec) v[u] = __ldcs(xr + vi);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int vi = base + u * 32 + lane;
        if (vi < nvec) cr[vi] = quant8(v[u], r);
      }
    }
  }
}

// Zero every outlier column of CA straight from the bitmap (one warp per row).
__global__ void __launch_bounds__(256) k_zero_outlier_cols(const uint32_t* __restrict__ bitmap, int M, int K,
                                                           int8_t* __restrict__ CA) {
  const int nwords = (K + 31) >> 5;
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * 8;
  for (int row = blockIdx.x * 8 + (threadIdx.x >> 5); row < M; row += warps) {
    int8_t* cr = CA + static_cast<size_t>(row) * K;
    for (int w = lane; w < nwords; w += 32) {
      uint32_t bits = __ldg(bitmap + w);
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        cr[w * 32 + b] = 0;
      }
    }
  }
}

// Outlier preparation for the fused forward.  Every block rebuilds the sorted
// column list from the bitmap in shared memory (a block-wide scan of popcounts),
// then the grid's warps walk rows: X rows (zero CA[:, O], gather X[:, O]) and
// CB rows (gather fp16(CB[:, O])).  Gathered rows are zero-padded to a multiple
// of 64 columns (one 128-byte fp16 tile).  Block 0 publishes the list, the
// counts and the overflow status.
__global__ void __launch_bounds__(256) k_outlier_prepare(const uint32_t* __restrict__ bitmap, int K, int cap,
                                                         int32_t* __restrict__ total_out,
                                                         int32_t* __restrict__ used_out,
                                                         int32_t* __restrict__ idx_out,
                                                         uint32_t* __restrict__ status,
                                                         int8_t* __restrict__ CA, const __half* __restrict__ X,
                                                         int M, __half* __restrict__ XO,
                                                         const int8_t* __restrict__ CB, int N,
                                                         __half* __restrict__ WO, int ld_o) {
  extern __shared__ int32_t idx_s[];
  __shared__ int32_t warp_base[8];
  __shared__ int32_t s_total;
  pdl_launch_dependents();
  pdl_wait();  // the bitmap and codes come from the quantiser
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwords = (K + 31) >> 5;
  const int per = (nwords + 255) / 256;
  const int w0 = min(threadIdx.x * per, nwords), w1 = min(w0 + per, nwords);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(__ldcg(bitmap + w));
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) warp_base[warp] = incl;
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0;
    for (int w = 0; w < 8; ++w) {
      const int x = warp_base[w];
      warp_base[w] = s;
      s += x;
    }
    s_total = s;
  }
  __syncthreads();
  int pos = warp_base[warp] + incl - cnt;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = __ldcg(bitmap + w);
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < cap) idx_s[pos] = w * 32 + b;
      ++pos;
    }
  }
  __syncthreads();
  const int total = s_total;
  const int used = min(total, cap);
  if (blockIdx.x == 0) {
    if (idx_out)
      for (int c = threadIdx.x; c < used; c += 256) idx_out[c] = idx_s[c];
    if (threadIdx.x == 0) {
      if (total_out) *total_out = total;
      if (used_out) *used_out = used;
      if (status && total > cap) atomicCAS(status, kStatusOk, kStatusOutlierOverflow);
    }
  }
  if (used == 0) return;
  const int n_pad = (used + 63) & ~63;
  const int rows_x = (XO != nullptr || CA != nullptr) ? M : 0;
  const int rows_w = WO != nullptr ? N : 0;
  const __half zero = __float2half_rn(0.f);
  for (int r = blockIdx.x * 8 + warp; r < rows_x + rows_w; r += gridDim.x * 8) {
    if (r < rows_x) {
      const size_t base = static_cast<size_t>(r) * K;
      for (int c = lane; c < n_pad; c += 32) {
        const int j = c < used ? idx_s[c] : -1;
        if (XO) XO[static_cast<size_t>(r) * ld_o + c] = j >= 0 ? X[base + j] : zero;
        if (CA && j >= 0) CA[base + j] = 0;
      }
    } else {
      const int n = r - rows_x;
      const size_t base = static_cast<size_t>(n) * K;
      for (int c = lane; c < n_pad; c += 32) {
        const int j = c < used ? idx_s[c] : -1;
        WO[static_cast<size_t>(n) * ld_o + c] = j >= 0 ? __int2half_rn(static_cast<int>(CB[base + j])) : zero;
      }
    }
  }
}

// out = fp16(C * SCA[i] * SCB[n] / 127^2 + bias[n]), four elements per thread.
__global__ void __launch_bounds__(256) k_mm_dequant(const int32_t* __restrict__ C, const float* __restrict__ SCA,
                                                    const float* __restrict__ SCB, const __half* __restrict__ bias,
                                                    int M, int N, __half* __restrict__ out) {
  const size_t total = static_cast<size_t>(M) * N;
  const size_t nq = (total + 3) / 4;
  const bool vec = (N & 3) == 0;
  for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < nq;
       q += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t e0 = q * 4;
    if (vec) {
      const int i = static_cast<int>(e0 / N), n = static_cast<int>(e0 % N);
      const int4 c = __ldcs(reinterpret_cast<const int4*>(C + e0));
      const float sa = __ldg(SCA + i) * (1.0f / 16129.0f);
      const float4 sb = __ldg(reinterpret_cast<const float4*>(SCB + n));
      float b[4] = {0.f, 0.f, 0.f, 0.f};
      if (bias) {
        const uint2 bb = __ldg(reinterpret_cast<const uint2*>(bias + n));
        const float2 b01 = __half22float2(*reinterpret_cast<const __half2*>(&bb.x));
        const float2 b23 = __half22float2(*reinterpret_cast<const __half2*>(&bb.y));
        b[0] = b01.x; b[1] = b01.y; b[2] = b23.x; b[3] = b23.y;
      }
      const __half2 h01 = __floats2half2_rn(fmaf(static_cast<float>(c.x), sa * sb.x, b[0]),
                                            fmaf(static_cast<float>(c.y), sa * sb.y, b[1]));
      const __half2 h23 = __floats2half2_rn(fmaf(static_cast<float>(c.z), sa * sb.z, b[2]),
                                            fmaf(static_cast<float>(c.w), sa * sb.w, b[3]));
      uint2 o;
      o.x = *reinterpret_cast<const uint32_t*>(&h01);
      o.y = *reinterpret_cast<const uint32_t*>(&h23);
      *reinterpret_cast<uint2*>(out + e0) = o;
    } else {
      for (size_t e = e0; e < e0 + 4 && e < total; ++e) {
        const int i = static_cast<int>(e / N), n = static_cast<int>(e % N);
        const float bv = bias ? __half2float(bias[n]) : 0.f;
        out[e] = __float2half_rn(fmaf(static_cast<float>(C[e]), SCA[i] * (1.0f / 16129.0f) * SCB[n], bv));
      }
    }
  }
}

// W = fp16(CB * SCB[n] / 127), sixteen elements per thread (K % 16 == 0).
__global__ void __launch_bounds__(256) k_dequant(const int8_t* __restrict__ CB, const float* __restrict__ SCB,
                                                 int N, int K, __half* __restrict__ W) {
  const size_t nchunks = static_cast<size_t>(N) * K / 16;
  for (size_t q = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; q < nchunks;
       q += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t e0 = q * 16;
    const int n = static_cast<int>(e0 / K);
    const float s = __fdiv_rn(__ldg(SCB + n), 127.0f);
    const int4 c = __ldcs(reinterpret_cast<const int4*>(CB + e0));
    const int8_t* b = reinterpret_cast<const int8_t*>(&c);
    uint32_t h[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const __half2 v = __floats2half2_rn(static_cast<float>(b[2 * e]) * s, static_cast<float>(b[2 * e + 1]) * s);
      h[e] = *reinterpret_cast<const uint32_t*>(&v);
    }
    uint4* o = reinterpret_cast<uint4*>(W + e0);
    o[0] = make_uint4(h[0], h[1], h[2], h[3]);
    o[1] = make_uint4(h[4], h[5], h[6], h[7]);
  }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_quant_rows(const __half* X, int M, int K, float tau, int8_t* CA, float* SCA, uint32_t* bitmap,
                              uint32_t* status, int num_sms, cudaStream_t st) {
  (void)status;
  // Many rows: persistent warps, one row each at a time.
  if (M >= 8 * num_sms) {
    static int blocks_per_sm = 0;
    if (blocks_per_sm == 0) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks_per_sm, k_quant_rows_warp<8>, 256, 0) !=
              cudaSuccess ||
          blocks_per_sm <= 0)
        blocks_per_sm = 4;
    }
    const int warps = (M + 0) < num_sms * blocks_per_sm * 8 ? M : num_sms * blocks_per_sm * 8;
    k_quant_rows_warp<8><<<(warps + 7) / 8, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
    return cudaGetLastError();
  }
  const int nvec = K / 8;
  if (nvec <= 32 * 8) {
    k_quant_rows<32, 8><<<(M + 7) / 8, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 64 * 8) {
    k_quant_rows<64, 8><<<(M + 3) / 4, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 128 * 8) {
    k_quant_rows<128, 8><<<(M + 1) / 2, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 256 * 8) {
    k_quant_rows<256, 8><<<M, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 256 * 16) {
    k_quant_rows<256, 16><<<M, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else {
    k_quant_rows_stream<<<M, 256, 0, st>>>(X, M, K, tau, CA, SCA, bitmap);
  }
  return cudaGetLastError();
}

cudaError_t launch_zero_outlier_cols(const uint32_t* bitmap, int M, int K, int8_t* CA, int num_sms,
                                     cudaStream_t st) {
  const int blocks = max(1, min((M + 7) / 8, num_sms * 4));
  k_zero_outlier_cols<<<blocks, 256, 0, st>>>(bitmap, M, K, CA);
  return cudaGetLastError();
}

cudaError_t launch_outlier_prepare(const uint32_t* bitmap, int K, int cap, int32_t* total_out, int32_t* used_out,
                                   int32_t* idx_out, uint32_t* status, int8_t* CA, const __half* X, int M,
                                   __half* XO, const int8_t* CB, int N, __half* WO, int ld_o, int num_sms,
                                   cudaStream_t st) {
  const int rows = ((XO || CA) ? M : 0) + (WO ? N : 0);
  const int blocks = max(1, min((rows + 7) / 8, num_sms * 4));
  const size_t smem = static_cast<size_t>(max(cap, 1)) * sizeof(int32_t);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_outlier_prepare, bitmap, K, cap, total_out, used_out, idx_out, status, CA, X, M,
                            XO, CB, N, WO, ld_o);
}

cudaError_t launch_mm_dequant(const int32_t* C, const float* SCA, const float* SCB, const __half* bias, int M,
                              int N, __half* out, int num_sms, cudaStream_t st) {
  const size_t nq = (static_cast<size_t>(M) * N + 3) / 4;
  const int blocks = static_cast<int>(std::min<size_t>((nq + 255) / 256, static_cast<size_t>(num_sms) * 16));
  k_mm_dequant<<<max(blocks, 1), 256, 0, st>>>(C, SCA, SCB, bias, M, N, out);
  return cudaGetLastError();
}

cudaError_t launch_dequant(const int8_t* CB, const float* SCB, int N, int K, __half* W, int num_sms,
                           cudaStream_t st) {
  const size_t nq = static_cast<size_t>(N) * K / 16;
  const int blocks = static_cast<int>(std::min<size_t>((nq + 255) / 256, static_cast<size_t>(num_sms) * 16));
  k_dequant<<<max(blocks, 1), 256, 0, st>>>(CB, SCB, N, K, W);
  return cudaGetLastError();
}

}  // namespace i8lt
