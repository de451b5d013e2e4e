// Few-token (decode) preparation in one launch: for M <= 16 rows the whole
// front half of the LLM.int8() forward -- row absmax calibration, int8
// quantisation, outlier column detection, the sorted outlier list, the
// gather of X[:, O] and the zeroing of CA[:, O] ("LLM.int8() Refactoring:
// Part 1", section "Improved kernels for inference", int8_vectorwise_quant;
// the mixed decomposition of "`bitsandbytes` - `Linear8bitLt` integration
// into `transformers` models", section "About the mixed quantization method
// in few words") -- runs on one cluster of 8 CTAs (16 for long rows of several
// tokens, when the device can place such a cluster).
//
// Each CTA owns a contiguous range of columns for all rows.  A column is an
// outlier column when any of its (at most 16) elements reaches the threshold,
// which the owning CTA decides alone; only the row maxima and the per-CTA
// outlier counts cross CTAs, through distributed shared memory after one
// cluster barrier.  Every word of state the GEMM reads (status, counts,
// split-K counters, list, gathered X) is written here, so no memset precedes
// the kernel.
//
//   pass 1  X -> per-row max |x| over elements below the threshold (packed
//           fp16 max; per-element test only where a vector reaches the
//           threshold) and the CTA's outlier column flags
//   sync    cluster barrier; row maxima and counts read from all CTAs of the cluster
//   pass 2  X (now in L2) -> codes (0 in outlier columns), SCA; the CTA's
//           outlier columns go to idx / X_O at the offset of the CTAs before it
#include <cuda_fp16.h>

#include <atomic>

#include "kernels.cuh"
#include "per_device.h"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int PT = 1024;                 // threads per CTA
constexpr unsigned kAll = 0xffffffffu;
constexpr int PU = 8;                    // X vectors per thread in flight
constexpr int kLocalList = 1024;         // outlier columns per CTA gathered in parallel

__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t code_s8p(float x, float r) {
  uint32_t q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(__fmul_rn(x, r)));
  return q;
}

}  // namespace

// PC: CTAs in the cluster (the launch gives the cluster shape)
template <int PC>
__global__ void __launch_bounds__(1024, 1)
    k_decode_prep(const __half* __restrict__ X, int M, int K, float tau, int cap, int8_t* __restrict__ CA,
                  float* __restrict__ SCA, int32_t* __restrict__ idx, __half* __restrict__ XO, int ld_o,
                  uint32_t* __restrict__ hdr, int32_t* __restrict__ counters, int n_counters) {
  extern __shared__ uint32_t s_flags[];   // outlier flags of this CTA's columns, bit j = column c0 + j
  __shared__ uint32_t s_rowmax[kDecodeMaxTokens];  // fp32 bits of non-negative maxima
  __shared__ int s_count, s_before, s_total;
  __shared__ int s_warp[PT / 32];
  __shared__ float s_r[kDecodeMaxTokens];
  __shared__ int s_list[kLocalList];     // this CTA's outlier columns, in list order

  pdl_launch_dependents();  // the GEMM may be scheduled now; it waits for this grid before reading
  pdl_wait();               // X and the workspace may belong to the work queued before

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  // columns [c0, c1) of this CTA, c0 a multiple of 32 (K is a multiple of 16)
  const int span = ((K + PC - 1) / PC + 31) & ~31;
  const int c0 = min(K, static_cast<int>(rank) * span), c1 = min(K, c0 + span);
  const int nv = (c1 - c0) >> 3;          // 8-column vectors per row
  const int nw = (c1 - c0 + 31) >> 5;     // flag words
  const int items = M * nv;
  const bool use_tau = tau > 0.f;

  for (int w = tid; w < nw; w += PT) s_flags[w] = 0u;
  if (tid < kDecodeMaxTokens) s_rowmax[tid] = 0u;
  __syncthreads();

  // ---------------------------------------------------------------- pass 1
  // Items (row, 8-column vector) in chunks of PU per thread: all PU loads are
  // issued before any is used.  When the CTA's part of X fits in one chunk it
  // stays in registers for pass 2.
  uint4 xv[PU];
  const bool one_chunk = items <= PU * PT;
  for (int base = 0; base < items; base += PU * PT) {  // uniform trip count: whole warps vote below
#pragma unroll
    for (int u = 0; u < PU; ++u) {
      const int it = base + u * PT + tid;
      xv[u] = make_uint4(0, 0, 0, 0);
      if (it < items) {
        const int r = it / nv;
        xv[u] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K + c0) + (it - r * nv));
      }
    }
#pragma unroll
    for (int u = 0; u < PU; ++u) {
      const int it = base + u * PT + tid;
      const bool valid = it < items;
      const int r = valid ? it / nv : -1;
      float keep = 0.f;
      if (valid) {
        const int v = it - r * nv;
        const __half2* h = reinterpret_cast<const __half2*>(&xv[u]);
        const __half2 m = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])), __hmax2(__habs2(h[2]), __habs2(h[3])));
        const float vmax = fmaxf(__low2float(m), __high2float(m));
        if (!use_tau || vmax < tau) {
          keep = vmax;
        } else {
          uint32_t big = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            const float a0 = fabsf(f.x), a1 = fabsf(f.y);
            if (a0 >= tau) big |= 1u << (2 * e); else keep = fmaxf(keep, a0);
            if (a1 >= tau) big |= 2u << (2 * e); else keep = fmaxf(keep, a1);
          }
          atomicOr(s_flags + (v >> 2), big << ((v & 3) * 8));
        }
      }
      // lanes of the same row combine their maxima; one shared atomic per row and warp
      const unsigned same = __match_any_sync(kAll, r);
      const unsigned mx = __reduce_max_sync(same, __float_as_uint(keep));
      if (valid && lane == __ffs(same) - 1) atomicMax(s_rowmax + r, mx);
    }
  }
  __syncthreads();
  int cnt = 0;
  for (int w = tid; w < nw; w += PT) cnt += __popc(s_flags[w]);
  cnt = __reduce_add_sync(kAll, static_cast<unsigned>(cnt));
  if (lane == 0) s_warp[warp] = cnt;
  __syncthreads();
  if (tid == 0) {
    int s = 0;
    for (int w = 0; w < PT / 32; ++w) s += s_warp[w];
    s_count = s;
  }
  cluster_sync();  // every CTA's row maxima and count are final and visible

  // ---------------------------------------------------------------- exchange
  if (tid < M) {
    uint32_t m = 0;
    for (int q = 0; q < PC; ++q) m = max(m, ld_dsmem_u32(map_to_rank(smem_addr(s_rowmax + tid), q)));
    const float amax = __uint_as_float(m);
    s_r[tid] = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (rank == 0) SCA[tid] = amax;
  }
  if (tid == 32) {  // outlier columns of the CTAs before this one, and of all
    const uint32_t a = smem_addr(&s_count);
    int b = 0, t = 0;
    for (int q = 0; q < PC; ++q) {
      const int c = static_cast<int>(ld_dsmem_u32(map_to_rank(a, q)));
      t += c;
      if (q < static_cast<int>(rank)) b += c;
    }
    s_before = b;
    s_total = t;
  }
  __syncthreads();
  const int before = s_before, total = s_total;
  const int used = min(total, cap);

  // ---------------------------------------------------------------- pass 2: codes
  for (int base = 0; base < items; base += PU * PT) {
    if (!one_chunk) {  // X was too large to keep: read the chunk again (from L2)
#pragma unroll
      for (int u = 0; u < PU; ++u) {
        const int it = base + u * PT + tid;
        if (it < items) {
          const int r = it / nv;
          xv[u] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K + c0) + (it - r * nv));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < PU; ++u) {
      const int it = base + u * PT + tid;
      if (it >= items) break;
      const int r = it / nv, v = it - r * nv;
      const float rs = s_r[r];
      const uint32_t fl = (s_flags[v >> 2] >> ((v & 3) * 8)) & 0xffu;
      const __half2* h = reinterpret_cast<const __half2*>(&xv[u]);
      uint32_t w[2];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float2 a = __half22float2(h[2 * p]);
        const float2 b = __half22float2(h[2 * p + 1]);
        const uint32_t lo = __byte_perm(code_s8p(a.x, rs), code_s8p(a.y, rs), 0x0040);
        const uint32_t hi = __byte_perm(code_s8p(b.x, rs), code_s8p(b.y, rs), 0x0040);
        w[p] = __byte_perm(lo, hi, 0x5410);
      }
      if (fl) {  // outlier columns carry code 0
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (fl & (1u << e)) w[e >> 2] &= ~(0xffu << ((e & 3) * 8));
      }
      *reinterpret_cast<uint2*>(CA + static_cast<size_t>(r) * K + c0 + 8 * v) = make_uint2(w[0], w[1]);
    }
  }

  // ---------------------------------------------------------------- outlier list and X_O
  if (use_tau && total > 0) {
    // exclusive scan of the flag words' popcounts over the CTA (word w -> thread w)
    const int nwp = (nw + PT - 1) / PT;  // flag words per thread (1 unless the range is huge)
    int my = 0;
    for (int j = 0; j < nwp; ++j) {
      const int w = tid * nwp + j;
      if (w < nw) my += __popc(s_flags[w]);
    }
    int incl = my;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kAll, incl, o);
      if (lane >= o) incl += y;
    }
    __syncthreads();  // s_warp is reused
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    int wbase = 0;
    for (int q = 0; q < warp; ++q) wbase += s_warp[q];
    int pos = before + wbase + incl - my;
    for (int j = 0; j < nwp; ++j) {
      const int w = tid * nwp + j;
      if (w >= nw) break;
      uint32_t bits = s_flags[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        const int col = c0 + 32 * w + b;
        if (pos < cap) {
          idx[pos] = col;
          if (pos - before < kLocalList) {
            s_list[pos - before] = col;  // gathered below by the whole CTA
          } else {
            for (int r = 0; r < M; ++r) XO[static_cast<size_t>(r) * ld_o + pos] = X[static_cast<size_t>(r) * K + col];
          }
        }
        ++pos;
      }
    }
    __syncthreads();
    // X_O for the first kLocalList outlier columns of this CTA: one element per thread
    const int nl = min(min(s_count, kLocalList), max(cap - before, 0));
    for (int e = tid; e < nl * M; e += PT) {
      const int r = e / nl, i = e - r * nl;
      XO[static_cast<size_t>(r) * ld_o + before + i] = X[static_cast<size_t>(r) * K + s_list[i]];
    }
  }
  if (rank == 0) {
    // X_O is read in steps of 16 columns: zero its rows from `used` to the next multiple of 16
    const int pad = ((used + 15) & ~15) - used;
    if (XO != nullptr)
      for (int e = tid; e < M * pad; e += PT) XO[static_cast<size_t>(e / pad) * ld_o + used + e % pad] = __float2half_rn(0.f);
    for (int e = tid; e < n_counters; e += PT) counters[e] = 0;
    if (tid == 0) {
      hdr[0] = total > cap ? kStatusOutlierOverflow : kStatusOk;
      hdr[1] = static_cast<uint32_t>(used);
      hdr[2] = static_cast<uint32_t>(total);
    }
  }
  cluster_sync();  // no CTA leaves while another may still read its shared memory
}

namespace {

// Whether a cluster of kDecodePrepClusterBig CTAs of this kernel fits the device (a
// non-portable size: it needs 16 SMs of one GPC); checked once per device.
bool big_cluster_ok() {
  static PerDeviceInt state;   // 1 yes, 2 no
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  return state.get(dev, [] {
    bool ok = cudaFuncSetAttribute(k_decode_prep<kDecodePrepClusterBig>,
                                   cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess;
    if (ok) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(kDecodePrepClusterBig, 1, 1);
      cfg.blockDim = dim3(PT, 1, 1);
      cfg.dynamicSmemBytes = 4096;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = kDecodePrepClusterBig;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int clusters = 0;
      ok = cudaOccupancyMaxActiveClusters(&clusters, k_decode_prep<kDecodePrepClusterBig>, &cfg) == cudaSuccess &&
           clusters >= 1;
    }
    cudaGetLastError();   // a refused query leaves no error behind
    return ok ? 1 : 2;
  }) == 1;
}

template <int PC>
cudaError_t launch_prep_t(const __half* X, int M, int K, float tau, int cap, int8_t* CA, float* SCA, int32_t* idx,
                          __half* XO, int ld_o, uint32_t* hdr, int32_t* counters, int n_counters, cudaStream_t st) {
  const int span = ((K + PC - 1) / PC + 31) & ~31;
  const size_t smem = static_cast<size_t>((span + 31) / 32) * 4;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(PC, 1, 1);
  cfg.blockDim = dim3(PT, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = PC;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, k_decode_prep<PC>, X, M, K, tau, cap, CA, SCA, idx, XO, ld_o, hdr, counters,
                            n_counters);
}

}  // namespace

int decode_prep_cluster(int M, int K) {
  return K >= kDecodeLongRow && static_cast<long long>(M) * K >= kDecodeBigPrep && big_cluster_ok()
             ? kDecodePrepClusterBig
             : kDecodePrepCluster;
}

cudaError_t launch_decode_prep(const __half* X, int M, int K, float tau, int cap, int8_t* CA, float* SCA,
                               int32_t* idx, __half* XO, int ld_o, uint32_t* hdr, int32_t* counters, int n_counters,
                               cudaStream_t st) {
  if (decode_prep_cluster(M, K) == kDecodePrepClusterBig)
    return launch_prep_t<kDecodePrepClusterBig>(X, M, K, tau, cap, CA, SCA, idx, XO, ld_o, hdr, counters, n_counters,
                                                st);
  return launch_prep_t<kDecodePrepCluster>(X, M, K, tau, cap, CA, SCA, idx, XO, ld_o, hdr, counters, n_counters, st);
}

}  // namespace i8lt
