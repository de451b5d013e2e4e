// HBM-bound kernels of the LLM.int8() forward:
//   k_quant_rows        fused row absmax calibration + int8 quantisation + outlier
//                       column bitmap ("LLM.int8() Refactoring: Part 1", section
//                       "Improved kernels for inference", int8_vectorwise_quant)
//   k_zero_outlier_cols zero the outlier columns of the codes (the fp16 path owns them)
//   k_outlier_prepare   bitmap -> sorted outlier column list (state.idx), zero CA
//                       columns, gather X[:, O] and fp16(CB[:, O]) for the outlier product
//   k_mm_dequant        int32 -> fp16 with row x column scales / 127^2 + bias
//   k_dequant           int8 weight -> fp16 ("Next steps": int8 dequantize op)
//   k_dequant_t         the same, stored transposed (operand of the input-gradient GEMM)
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

// int8 code of x * r, rounded to nearest even, in the low byte of the result.
// t = fl32(x * r) is rounded once more by adding 1.5 * 2^23: for |t| <= 2^22
// the sum lies in [2^23, 2^24), where fp32 holds exactly the integers, so IEEE
// round-to-nearest-even makes it 1.5 * 2^23 + rne(t), and the low byte of its
// bit pattern is rne(t) as a two's-complement byte (the constant's low 22 bits
// are 0).  This is the reading's code for every element kept on the int8 path
// (|x| <= amax, so |t| <= 127 * (1 + 2^-23) and no clamp is reached).  Larger
// t only occur at or above the threshold, in outlier columns, whose codes are
// zeroed before use.  Two FMA-pipe operations instead of a conversion.
__device__ __forceinline__ uint32_t code_rne(float x, float r) {
  return __float_as_uint(__fadd_rn(__fmul_rn(x, r), 12582912.0f));
}

// 8 fp16 values -> 8 int8 codes packed little-endian.
__device__ __forceinline__ uint2 quant8(const uint4& v, float r) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  uint32_t w[2];
#pragma unroll
  for (int p = 0; p < 2; ++p) {
    const float2 a = __half22float2(h[2 * p]);
    const float2 b = __half22float2(h[2 * p + 1]);
    const uint32_t lo = __byte_perm(code_rne(a.x, r), code_rne(a.y, r), 0x0040);
    const uint32_t hi = __byte_perm(code_rne(b.x, r), code_rne(b.y, r), 0x0040);
    w[p] = __byte_perm(lo, hi, 0x5410);
  }
  return make_uint2(w[0], w[1]);
}

// Max |x| of 8 fp16 values with packed fp16 max (exact: the max of fp16
// values is one of them).
__device__ __forceinline__ float absmax8(const uint4& v) {
  const __half2* h = reinterpret_cast<const __half2*>(&v);
  const __half2 m = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])), __hmax2(__habs2(h[2]), __habs2(h[3])));
  return fmaxf(__low2float(m), __high2float(m));
}

// Fold one vector into the row's running absmax.  A vector whose max reaches
// the threshold takes the per-element path: its outliers are left out of the
// max and OR-ed into the block's shared-memory bitmap (vector vi covers
// columns 8vi .. 8vi+7, i.e. bits 8(vi % 4) .. of word vi / 4).
__device__ __forceinline__ void fold8(const uint4& v, int vi, float tau, bool use_tau, float& amax,
                                      uint32_t* sbm) {
  const float vmax = absmax8(v);
  if (!use_tau || vmax < tau) {
    amax = fmaxf(amax, vmax);
    return;
  }
  uint32_t big = 0;
  scan8(v, tau, true, amax, big);
  atomicOr(sbm + (vi >> 2), big << ((vi & 3) * 8));
}

// The block's outlier bitmap lives in shared memory while its rows are
// scanned; each non-zero word reaches the global bitmap with one atomic.
__device__ __forceinline__ void sbm_clear(uint32_t* sbm, int nwords) {
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) sbm[w] = 0u;
}
__device__ __forceinline__ void sbm_flush(const uint32_t* sbm, int nwords, uint32_t* bitmap) {
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) {
    const uint32_t bits = sbm[w];
    if (bits) atomicOr(bitmap + w, bits);
  }
}

}  // namespace

// One row per group of G threads (G a multiple of 32), 256 threads per block,
// each thread caching up to VPT 16-byte vectors of its row in registers so X
// is read from HBM exactly once.
template <int G, int VPT>
__global__ void __launch_bounds__(256, (VPT > 8 ? 1 : 5)) k_quant_rows(const __half* __restrict__ X, int M, int K, float tau,
                                                    int8_t* __restrict__ CA, float* __restrict__ SCA,
                                                    uint32_t* __restrict__ bitmap) {
  static_assert(G % 32 == 0 && 256 % G == 0, "group size");
  extern __shared__ uint32_t sbm[];
  __shared__ float red[8];
  pdl_launch_dependents();
  constexpr int ROWS = 256 / G;
  constexpr int WPR = G / 32;  // warps per row
  const int tid = threadIdx.x;
  const int g = tid / G;
  const int t = tid % G;
  const int row = blockIdx.x * ROWS + g;
  const bool valid = row < M;
  const int nvec = K >> 3, nwords = (K + 31) >> 5;
  const bool use_tau = tau > 0.f;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(valid ? row : 0) * K);

  uint4 v[VPT];
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int vi = t + i * G;
    v[i] = (valid && vi < nvec) ? ld_stream_16(xr + vi) : make_uint4(0, 0, 0, 0);
  }
  if (use_tau) {
    sbm_clear(sbm, nwords);
    __syncthreads();
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < VPT; ++i) fold8(v[i], t + i * G, tau, use_tau, amax, sbm);
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
  if (use_tau) {
    __syncthreads();
    sbm_flush(sbm, nwords, bitmap);
  }
}

// Rows too long to cache in registers: one block per row, X read twice (the
// second read is served by L2).
__global__ void __launch_bounds__(256) k_quant_rows_stream(const __half* __restrict__ X, int M, int K,
                                                           float tau, int8_t* __restrict__ CA,
                                                           float* __restrict__ SCA, uint32_t* __restrict__ bitmap) {
  extern __shared__ uint32_t sbm[];
  __shared__ float red[8];
  pdl_launch_dependents();
  const int row = blockIdx.x;
  const int nvec = K >> 3, nwords = (K + 31) >> 5;
  const bool use_tau = tau > 0.f;
  const uint4* xr = reinterpret_cast<const uint4*>(X + static_cast<size_t>(row) * K);
  if (use_tau) {
    sbm_clear(sbm, nwords);
    __syncthreads();
  }
  float amax = 0.f;
  for (int vi = threadIdx.x; vi < nvec; vi += 256) fold8(xr[vi], vi, tau, use_tau, amax, sbm);
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
  if (use_tau) sbm_flush(sbm, nwords, bitmap);  // the __syncthreads above ordered every mark before this
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

// Position -> list entry of the gathered outlier operands: within each group
// of 16 columns the entries are stored as (0 1 8 9)(2 3 10 11)(4 5 12 13)
// (6 7 14 15), so a thread of an m16n8k16 fragment reads its four values
// (2t, 2t+1, 2t+8, 2t+9) with one 8-byte load.  A product over the outlier
// columns does not depend on their order, so the tensor-core path that reads
// whole 64-column tiles uses the same layout.
__device__ __forceinline__ int outlier_slot(int pos) {
  const int q = pos & 15;
  return (pos & ~15) + 2 * (q >> 2) + (q & 1) + 8 * ((q >> 1) & 1);
}

// Stored position of list entry e in the gathered operands (the inverse of
// outlier_slot).
__device__ __forceinline__ int outlier_pos(int e) {
  const int q = e & 15;
  return (e & ~15) + 4 * ((q >> 1) & 3) + 2 * ((q >> 3) & 1) + (q & 1);
}

// With at least one listed column per kDenseRowBytes bytes of a weight row,
// most 128-byte lines of every row hold a listed column and the scattered
// gather is bound by its request count; reading the rows whole then costs
// about the same DRAM bytes, in coalesced requests.
constexpr int kDenseRowBytes = 48;
// The dense preparation reads rows in batches of kDenseChunks chunks of 512 bytes (one
// 16-byte load per lane and chunk); the list is indexed by 256-column chunks.
constexpr int kDenseChunk = 512;
constexpr int kDenseChunks = 8;  // chunks per batch
constexpr int kDenseBatch = kDenseChunks * kDenseChunk;
constexpr int kListChunkCols = 256;

// Dynamic shared memory of the preparation: the list (cap entries), then, when
// the dense mode can be taken, the chunk index (K / 256 + 1 entries) and two
// 512-byte staging buffers per warp.
__host__ __device__ inline size_t dense_stage_offset(int cap, int K) {
  const size_t words = static_cast<size_t>(cap > 0 ? cap : 1) + (K + kListChunkCols - 1) / kListChunkCols + 1;
  return (words * sizeof(int32_t) + 15) & ~static_cast<size_t>(15);
}
__host__ __device__ inline bool dense_possible(int cap, int K) {
  return static_cast<long long>(cap) * kDenseRowBytes >= K;
}

__device__ __forceinline__ void load_batch(uint4 (&v)[kDenseChunks], const uint8_t* __restrict__ row, int b0, int row_bytes,
                                           int lane) {
#pragma unroll
  for (int c = 0; c < kDenseChunks; ++c) {
    const int off = b0 + c * kDenseChunk + lane * 16;
    v[c] = off < row_bytes ? __ldcg(reinterpret_cast<const uint4*>(row + off)) : make_uint4(0u, 0u, 0u, 0u);
  }
}

// The listed elements of one batch of a row (kEs bytes per element), starting
// at byte b0.  Each 512-byte chunk goes through one of the warp's two staging
// buffers (wbuf, 2 x 512 bytes); chunk c holds the list entries cst[x0] ..
// cst[x1] - 1 (cst[x] = first entry at or past column 256 x), which the lanes
// take 32 at a time.  X rows (kEs == 2) also zero their codes in ca.
template <int kEs>
__device__ __forceinline__ void take_batch(const uint4 (&v)[kDenseChunks], int b0, int row_bytes, const int32_t* idx_s,
                                           const int32_t* cst, int n_cst, __half* __restrict__ dst,
                                           int8_t* __restrict__ ca, uint8_t* wbuf, int lane) {
#pragma unroll
  for (int c = 0; c < kDenseChunks; ++c) {
    const int lo = b0 + c * kDenseChunk;
    if (lo >= row_bytes) break;
    uint8_t* buf = wbuf + (c & 1) * kDenseChunk;
    // the lanes finished the chunk before the previous one (the last reader of
    // this buffer) before the __syncwarp of the previous chunk
    *reinterpret_cast<uint4*>(buf + lane * 16) = v[c];
    __syncwarp();
    const int x0 = lo / (kEs * kListChunkCols);
    const int x1 = min(x0 + kDenseChunk / (kEs * kListChunkCols), n_cst - 1);
    const int e_hi = cst[x1];
    for (int e = cst[x0] + lane; e < e_hi; e += 32) {
      const int j = idx_s[e];
      const int off = j * kEs - lo;
      unsigned short h;
      if (kEs == 2) {
        h = *reinterpret_cast<const unsigned short*>(buf + off);
        if (ca != nullptr) ca[j] = 0;
      } else {
        h = __half_as_ushort(__int2half_rn(static_cast<int>(reinterpret_cast<const int8_t*>(buf)[off])));
      }
      if (dst != nullptr) dst[outlier_pos(e)] = __ushort_as_half(h);
    }
  }
  __syncwarp();  // the next batch starts again at buffer 0
}

// Rows first, first + stride, ... < rows of one operand, on one warp: the next
// batch (of this row or the next) is requested before the current one is
// taken apart.  dst / ca advance by ld_dst / row_elems per row (ca may be null,
// dst too).  Positions used .. width - 1 of every dst row are zeroed.
template <int kEs>
__device__ __forceinline__ void prepare_rows_dense(const uint8_t* __restrict__ src, int row_elems, int rows,
                                                   int first, int stride, const int32_t* idx_s, const int32_t* cst,
                                                   int n_cst, int used, int width, __half* __restrict__ dst,
                                                   int ld_dst, int8_t* __restrict__ ca, uint8_t* wbuf, int lane) {
  const int row_bytes = row_elems * kEs;
  const int nbat = (row_bytes + kDenseBatch - 1) / kDenseBatch;
  int r = first, b = 0;
  uint4 cur[kDenseChunks], nxt[kDenseChunks];
  if (r < rows) load_batch(cur, src + static_cast<size_t>(r) * row_bytes, 0, row_bytes, lane);
  while (r < rows) {
    int r2 = r, b2 = b + 1;
    if (b2 == nbat) {
      r2 += stride;
      b2 = 0;
    }
    if (r2 < rows) load_batch(nxt, src + static_cast<size_t>(r2) * row_bytes, b2 * kDenseBatch, row_bytes, lane);
    __half* d = dst != nullptr ? dst + static_cast<size_t>(r) * ld_dst : nullptr;
    take_batch<kEs>(cur, b * kDenseBatch, row_bytes, idx_s, cst, n_cst, d,
                    ca != nullptr ? ca + static_cast<size_t>(r) * row_elems : nullptr, wbuf, lane);
    if (b2 == 0 && d != nullptr)
      for (int e = used + lane; e < width; e += 32) d[outlier_pos(e)] = __ushort_as_half(0);
#pragma unroll
    for (int c = 0; c < kDenseChunks; ++c) cur[c] = nxt[c];
    r = r2;
    b = b2;
  }
}

// Outlier preparation for the fused forward.  Every block rebuilds the sorted
// column list from the bitmap in shared memory (a block-wide scan of
// popcounts).  Then, with few listed columns, the grid's threads take work
// items (row, group of 16 list positions) over the X rows (gather X[:, O] into
// X_O, zero CA[:, O]) and the CB rows (gather fp16(CB[:, O]) into W_O): an item
// issues its 16 gathers at once and writes the group as two 16-byte stores, so
// the scattered reads of every (row, column) pair are in flight together across
// the grid.  With many (see kDenseRowBytes), each warp streams whole rows
// instead (prepare_row_dense).  Up to 16 used columns the operands are written
// as one zero-padded group of 16 (the GEMM's epilogue reads exactly that); past
// 16, zero padded to a multiple of 64 (one 128-byte fp16 tile of the tensor-core
// path).  Block 0 publishes the list, the counts and the overflow status.
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
  // up to 4 words per thread (K <= 32768) stay in registers for the second pass
  uint32_t wv[4];
  int cnt = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    wv[q] = w0 + q < w1 ? __ldcg(bitmap + w0 + q) : 0u;
    cnt += __popc(wv[q]);
  }
  for (int w = w0 + 4; w < w1; ++w) cnt += __popc(__ldcg(bitmap + w));
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
  auto list_word = [&](int w, uint32_t bits) {  // the set bits of word w, in order
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (pos < cap) idx_s[pos] = w * 32 + b;
      ++pos;
    }
  };
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (w0 + q < w1) list_word(w0 + q, wv[q]);
  for (int w = w0 + 4; w < w1; ++w) list_word(w, __ldcg(bitmap + w));
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
  const int groups = used <= 16 ? 1 : ((used + 63) & ~63) >> 4;  // 16-position groups written
  const int rows_x = (XO != nullptr || CA != nullptr) ? M : 0;
  const int rows_w = WO != nullptr ? N : 0;
  if (rows_x + rows_w > 0 && static_cast<long long>(used) * kDenseRowBytes >= K) {
    // cst[x] = first list entry at or past column 256 x, x = 0 .. n_cst - 1
    int32_t* cst = idx_s + cap;
    const int n_cst = (K + kListChunkCols - 1) / kListChunkCols + 1;
    uint8_t* wbuf = reinterpret_cast<uint8_t*>(idx_s) + dense_stage_offset(cap, K) + warp * 2 * kDenseChunk;
    for (int e = threadIdx.x; e <= used; e += 256) {
      const int prev = e == 0 ? -1 : idx_s[e - 1] / kListChunkCols;  // chunk of the entry before
      const int here = e == used ? n_cst - 1 : idx_s[e] / kListChunkCols;
      for (int x = prev + 1; x <= here; ++x) cst[x] = e;
    }
    __syncthreads();
    const int gw = blockIdx.x * 8 + warp, nw = gridDim.x * 8;
    const int width = groups * 16;
    if (rows_x > 0)
      prepare_rows_dense<2>(reinterpret_cast<const uint8_t*>(X), K, rows_x, gw, nw, idx_s, cst, n_cst, used, width,
                            XO, ld_o, CA, wbuf, lane);
    if (rows_w > 0)
      prepare_rows_dense<1>(reinterpret_cast<const uint8_t*>(CB), K, rows_w, gw, nw, idx_s, cst, n_cst, used, width,
                            WO, ld_o, nullptr, wbuf, lane);
    return;
  }
  const long long items = static_cast<long long>(rows_x + rows_w) * groups;
  for (long long it = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; it < items;
       it += static_cast<long long>(gridDim.x) * 256) {
    const int r = static_cast<int>(it / groups);
    const int p0 = static_cast<int>(it - static_cast<long long>(r) * groups) * 16;  // first stored position
    const bool is_x = r < rows_x;
    const int row = is_x ? r : r - rows_x;
    const size_t base = static_cast<size_t>(row) * K;
    __half* dst = is_x ? (XO != nullptr ? XO + static_cast<size_t>(row) * ld_o : nullptr)
                       : WO + static_cast<size_t>(row) * ld_o;
    uint32_t h[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (p0 < used) {  // the group holds list entries; the rest of the padding stays 0
      unsigned short v[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        // stored position p0 + q holds list entry outlier_slot(p0 + q)
        const int c = outlier_slot(p0 + q);
        v[q] = 0;
        if (c < used) {
          const int j = idx_s[c];
          v[q] = is_x ? __half_as_ushort(X[base + j])
                      : __half_as_ushort(__int2half_rn(static_cast<int>(CB[base + j])));
        }
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) h[q] = static_cast<uint32_t>(v[2 * q]) | (static_cast<uint32_t>(v[2 * q + 1]) << 16);
      if (is_x && CA != nullptr) {
#pragma unroll
        for (int q = 0; q < 16; ++q)
          if (p0 + q < used) CA[base + idx_s[p0 + q]] = 0;  // the group's columns, in list order
      }
    }
    if (dst != nullptr) {
      uint4* d = reinterpret_cast<uint4*>(dst + p0);
      d[0] = make_uint4(h[0], h[1], h[2], h[3]);
      d[1] = make_uint4(h[4], h[5], h[6], h[7]);
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

// The same dequantised weight, stored transposed: Wt[k, n] = fp16(CB[n, k] * SCB[n] / 127)
// (the operand the input-gradient GEMM reads K-major).  One 64 x 64 tile per
// block through shared memory: each thread reads 16 codes of one weight row and
// writes them as a column of the tile; the tile leaves as 16-byte rows of Wt.
// Requires K % 16 == 0 (a 16-code vector is all inside or all outside) and
// N % 8 == 0 (likewise for an 8-value vector of a Wt row).
constexpr int kDqT = 64;

__global__ void __launch_bounds__(256) k_dequant_t(const int8_t* __restrict__ CB, const float* __restrict__ SCB,
                                                   int N, int K, __half* __restrict__ Wt) {
  __shared__ __align__(16) __half t[kDqT][kDqT + 8];  // [k][n]; 144-byte rows keep 16-byte alignment
  const int n0 = blockIdx.x * kDqT, k0 = blockIdx.y * kDqT;
  {
    // lanes of a warp take consecutive weight rows, so their column writes to
    // the tile fall in distinct banks
    const int r = threadIdx.x & (kDqT - 1), c = (threadIdx.x >> 6) * 16;
    const int n = n0 + r, k = k0 + c;
    int4 v = make_int4(0, 0, 0, 0);
    float sc = 0.f;
    if (n < N && k < K) {
      v = __ldcs(reinterpret_cast<const int4*>(CB + static_cast<size_t>(n) * K + k));
      sc = __fdiv_rn(__ldg(SCB + n), 127.0f);
    }
    const int8_t* b = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
    for (int e = 0; e < 16; ++e) t[c + e][r] = __float2half_rn(static_cast<float>(b[e]) * sc);
  }
  __syncthreads();
#pragma unroll
  for (int q = threadIdx.x; q < kDqT * (kDqT / 8); q += 256) {
    const int kr = q >> 3, nc = (q & 7) * 8;
    const int k = k0 + kr, n = n0 + nc;
    if (k < K && n < N)
      *reinterpret_cast<uint4*>(Wt + static_cast<size_t>(k) * N + n) = *reinterpret_cast<const uint4*>(&t[kr][nc]);
  }
}

// Column blocks gathered from P ranks, G [P, M, Np] (rank-major, as an
// all-gather of each rank's [M, Np] output leaves them), laid out as the
// output of the whole layer: out[m, p * Np + j] = G[p, m, j].  16 bytes per
// thread when Np % 8 == 0, else one element.
__global__ void __launch_bounds__(256) k_gather_column_blocks(const __half* __restrict__ G, int P, int M, int Np,
                                                              __half* __restrict__ out) {
  const bool vec = (Np & 7) == 0;
  const int per_row = vec ? Np >> 3 : Np;  // units per (rank, row)
  const size_t units = static_cast<size_t>(P) * M * per_row;
  const size_t N = static_cast<size_t>(P) * Np;
  for (size_t u = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const size_t pm = u / per_row;
    const int j = static_cast<int>(u - pm * per_row);
    const int p = static_cast<int>(pm / M), m = static_cast<int>(pm - static_cast<size_t>(p) * M);
    if (vec) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(G + pm * Np) + j);
      *reinterpret_cast<uint4*>(out + m * N + static_cast<size_t>(p) * Np + 8 * j) = v;
    } else {
      out[m * N + static_cast<size_t>(p) * Np + j] = G[pm * Np + j];
    }
  }
}

cudaError_t launch_gather_column_blocks(const __half* G, int P, int M, int Np, __half* out, int num_sms,
                                        cudaStream_t st) {
  const size_t units = static_cast<size_t>(P) * M * ((Np & 7) == 0 ? Np / 8 : Np);
  const int blocks = static_cast<int>(std::min<size_t>((units + 255) / 256, static_cast<size_t>(num_sms) * 8));
  k_gather_column_blocks<<<std::max(blocks, 1), 256, 0, st>>>(G, P, M, Np, out);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_quant_rows(const __half* X, int M, int K, float tau, int8_t* CA, float* SCA, uint32_t* bitmap,
                              cudaStream_t st) {
  const size_t smem = tau > 0.f ? static_cast<size_t>((K + 31) / 32) * 4 : 0;
  const int nvec = K / 8;
  // One row per group of threads with the row in registers (one pass over X),
  // grids of many small blocks so that enough rows are in flight per SM; rows
  // beyond 32768 columns stream twice.
  if (nvec <= 32 * 8) {
    k_quant_rows<32, 8><<<(M + 7) / 8, 256, smem, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 64 * 8) {
    k_quant_rows<64, 8><<<(M + 3) / 4, 256, smem, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 128 * 8) {
    k_quant_rows<128, 8><<<(M + 1) / 2, 256, smem, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 256 * 8) {
    k_quant_rows<256, 8><<<M, 256, smem, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else if (nvec <= 256 * 16) {
    k_quant_rows<256, 16><<<M, 256, smem, st>>>(X, M, K, tau, CA, SCA, bitmap);
  } else {
    k_quant_rows_stream<<<M, 256, smem, st>>>(X, M, K, tau, CA, SCA, bitmap);
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
  // work items: (row, 16-position group), at most as many as the capacity
  // allows.  The grid is capped at 2 blocks per SM: the kernel is launched as a
  // programmatic dependent of the quantiser, so its blocks can become resident
  // while the quantiser still runs and would take warp slots from it; the
  // item loop strides over the grid.
  const int rows = ((XO || CA) ? M : 0) + (WO ? N : 0);
  const int groups = cap <= 16 ? 1 : ((cap + 63) / 64) * 4;
  const long long items = static_cast<long long>(rows) * groups;
  const int blocks = static_cast<int>(std::max<long long>(1, std::min<long long>((items + 255) / 256, num_sms * 2LL)));
  const size_t smem = rows > 0 && dense_possible(cap, K) ? dense_stage_offset(cap, K) + 8 * 2 * kDenseChunk
                                                         : static_cast<size_t>(max(cap, 1)) * sizeof(int32_t);
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

cudaError_t launch_dequant_t(const int8_t* CB, const float* SCB, int N, int K, __half* Wt, cudaStream_t st) {
  const dim3 grid((N + kDqT - 1) / kDqT, (K + kDqT - 1) / kDqT, 1);
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  k_dequant_t<<<grid, 256, 0, st>>>(CB, SCB, N, K, Wt);
  return cudaGetLastError();
}

}  // namespace i8lt
