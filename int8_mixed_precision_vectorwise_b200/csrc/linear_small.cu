// The whole LLM.int8() Linear8bitLt forward of a small problem in one launch
// (few tokens, a small weight): the mixed int8 / fp16 decomposition of
// "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models"
// (section "About the mixed quantization method in few words") built from the
// int8_vectorwise_quant / int8_linear_matmul / int8_mm_dequant ops of
// "LLM.int8() Refactoring: Part 1" (sections "Improved kernels for
// inference" and "Deprecations").
//
// For such sizes the forward's cost is launches and pipeline start-up, not
// bytes, so everything happens in one grid with no workspace round trip: CTA
// b owns weight rows [128b, 128b + 128).  It
//   1. requests its weight tile through a ring of TMA stages (first of all:
//      the weights do not depend on X);
//   2. quantises all of X itself (X is at most 16 x 4096 fp16): row absmax
//      over the elements below the threshold, the outlier-column flags (every
//      CTA sees every row, so it decides each column alone), codes with the
//      outlier columns zeroed, written straight into shared memory in the
//      128B-swizzled K-major layout the tensor core reads, and the sorted
//      outlier list;
//   3. runs tcgen05 kind::i8 MMAs (M = 128 weight rows, N = 16 token columns,
//      int32 accumulator in TMEM) as weight stages land;
//   4. adds the outlier term X[t, j] * CB[n, j] for the outlier columns from
//      the staged weight tiles (CUDA cores, fp32, columns in ascending order)
//      and applies dequant and bias:
//        out[t, n] = fp16(C * SCA[t] * SCB[n] / 127^2 + bias[n] + (SCB[n] / 127) * D).
// Block 0 writes the status word and the outlier counts.  Every wait is
// bounded by a time limit; on expiry the status becomes I8_ERR_TIMEOUT and
// the CTA leaves after its in-flight copies and MMAs have completed.
#include <cuda_fp16.h>

#include <atomic>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int LM = 128;                       // weight rows per CTA (MMA M)
constexpr int LT = kDecodeMaxTokens;          // token columns (MMA N), zero padded
constexpr int LBOX = LM * 128;                // one 128-byte-deep weight box: 16 KB
constexpr int LSB = 2;                        // weight boxes per ring stage
constexpr int LSTAGE = LSB * LBOX;            // 32 KB
constexpr int LRS = 4;                        // ring stages
constexpr int LCA_BOX = LT * 128;             // one 128-byte-deep box of the 16 code rows: 2 KB
constexpr int LTHREADS = 256;
constexpr int LPU = 8;                        // X vectors per thread in flight while quantising
constexpr uint32_t LTMEM_COLS = 32;
constexpr unsigned kAllLanes = 0xffffffffu;

struct SmallLayout {
  int ca_off, sbm_off, list_off, misc_off, bar_off, total;
  __host__ __device__ SmallLayout(int K) {
    const int nbox = (K + 127) / 128;
    ca_off = LRS * LSTAGE;
    sbm_off = ca_off + nbox * LCA_BOX;
    list_off = sbm_off + ((K + 31) / 32) * 4;
    misc_off = list_off + kSmallListCap * 4;
    bar_off = (misc_off + 3 * LT * 4 + 16 + 7) & ~7;
    total = bar_off + (2 * LRS + 1) * 8 + 1024;  // + slack to align the ring to 1024 bytes
  }
};

__device__ __forceinline__ uint32_t small_code(float x, float r) {
  uint32_t q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(__fmul_rn(x, r)));
  return q;
}

}  // namespace

size_t linear_small_smem(int K) { return static_cast<size_t>(SmallLayout(K).total); }

__global__ void __launch_bounds__(LTHREADS, 1)
    k_linear_small(const __grid_constant__ CUtensorMap tmW, const __half* __restrict__ X, int M, int N, int K,
                   float tau, int cap, const float* __restrict__ SCB, const __half* __restrict__ bias,
                   __half* __restrict__ out, uint32_t* hdr, uint64_t limit_ns, int reset_status) {
  extern __shared__ uint8_t lsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
  const SmallLayout Lay(K);
  uint8_t* ring = smem;
  uint8_t* ca = smem + Lay.ca_off;
  uint32_t* sbm = reinterpret_cast<uint32_t*>(smem + Lay.sbm_off);
  int32_t* s_list = reinterpret_cast<int32_t*>(smem + Lay.list_off);
  uint32_t* s_rowmax = reinterpret_cast<uint32_t*>(smem + Lay.misc_off);  // fp32 bits of maxima
  float* s_r = reinterpret_cast<float*>(s_rowmax + LT);
  float* s_sa = s_r + LT;
  int* s_cnt = reinterpret_cast<int*>(s_sa + LT);        // [0] outlier columns found
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_cnt + 1);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_cnt + 2);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay.bar_off);
  uint64_t* empty = full + LRS;
  uint64_t* acc_full = empty + LRS;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * LM;
  const int nbox = (K + 127) / 128;                 // 128-byte k-boxes
  const int nstage = (nbox + LSB - 1) / LSB;
  const int nvec = K >> 3, nwords = (K + 31) >> 5;
  const bool use_tau = tau > 0.f;

  if (tid == 0) {
    for (int s = 0; s < LRS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);   // the MMAs' commit and the 4 outlier / epilogue warps
    }
    mbar_init(acc_full, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, LTMEM_COLS);
    tmem_relinquish();
  }
  for (int w = tid; w < nwords; w += LTHREADS) sbm[w] = 0u;
  if (tid < LT) s_rowmax[tid] = 0u;
  {  // zero the code tile: rows past M and bytes past K must be 0 for the MMA
    uint4* z = reinterpret_cast<uint4*>(ca);
    for (int i = tid; i < nbox * LCA_BOX / 16; i += LTHREADS) z[i] = make_uint4(0, 0, 0, 0);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  // the weight tile does not depend on X: request the first stages now
  uint32_t filled = 0, fill_parity = 0;
  if (tid == 0) {
    tma_prefetch_desc(&tmW);
    for (int st = 0; st < nstage && st < LRS; ++st) {
      const int b0 = st * LSB, nb = min(LSB, nbox - b0);
      mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(nb * LBOX));
      filled |= 1u << st;
      for (int b = 0; b < nb; ++b) tma_load_2d(ring + st * LSTAGE + b * LBOX, &tmW, &full[st], (b0 + b) * 128, n0);
    }
  }

  // ---------------------------------------------------------------- quantise X (all threads)
  // Items (row, 8-column vector) in chunks of LPU per thread: all LPU loads of
  // a chunk are issued before any is used.  When X fits in one chunk it stays
  // in registers for pass 2; otherwise pass 2 reads each chunk again (from L1/L2).
  const int items = M * nvec;
  const bool one_chunk = items <= LPU * LTHREADS;
  uint4 xv[LPU];
  for (int base = 0; base < items; base += LPU * LTHREADS) {   // pass 1: row maxima below the threshold, column flags
#pragma unroll
    for (int u = 0; u < LPU; ++u) {
      const int it = base + u * LTHREADS + tid;
      xv[u] = make_uint4(0, 0, 0, 0);
      if (it < items) {
        const int r = it / nvec;
        xv[u] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K) + (it - r * nvec));
      }
    }
#pragma unroll
    for (int u = 0; u < LPU; ++u) {   // (uniform trip count: whole warps vote below)
      const int it = base + u * LTHREADS + tid;
      const bool valid = it < items;
      const int r = valid ? it / nvec : -1;
      float keep = 0.f;
      if (valid) {
        const int v = it - r * nvec;
        const __half2* h = reinterpret_cast<const __half2*>(&xv[u]);
        const __half2 m2 = __hmax2(__hmax2(__habs2(h[0]), __habs2(h[1])), __hmax2(__habs2(h[2]), __habs2(h[3])));
        const float vmax = fmaxf(__low2float(m2), __high2float(m2));
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
          atomicOr(sbm + (v >> 2), big << ((v & 3) * 8));
        }
      }
      // lanes of the same row combine their maxima (non-negative floats order like their
      // bits); one shared atomic per row and warp
      const unsigned same = __match_any_sync(kAllLanes, r);
      const unsigned mx = __reduce_max_sync(same, __float_as_uint(keep));
      if (valid && lane == __ffs(same) - 1) atomicMax(s_rowmax + r, mx);
    }
  }
  __syncthreads();
  if (tid < LT) {
    const float amax = tid < M ? __uint_as_float(s_rowmax[tid]) : 0.f;
    s_r[tid] = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
    s_sa[tid] = amax * (1.0f / 16129.0f);
  }
  __syncthreads();
  for (int base = 0; base < items; base += LPU * LTHREADS) {   // pass 2: codes into the swizzled K-major tile
    if (!one_chunk) {
#pragma unroll
      for (int u = 0; u < LPU; ++u) {
        const int it = base + u * LTHREADS + tid;
        if (it < items) {
          const int r = it / nvec;
          xv[u] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K) + (it - r * nvec));
        }
      }
    }
#pragma unroll
    for (int u = 0; u < LPU; ++u) {
      const int it = base + u * LTHREADS + tid;
      if (it >= items) break;
      const int r = it / nvec, v = it - r * nvec;
      const float rs = s_r[r];
      const uint32_t fl = (sbm[v >> 2] >> ((v & 3) * 8)) & 0xffu;
      const __half2* h = reinterpret_cast<const __half2*>(&xv[u]);
      uint32_t w[2];
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const float2 a = __half22float2(h[2 * p]);
        const float2 b = __half22float2(h[2 * p + 1]);
        const uint32_t lo = __byte_perm(small_code(a.x, rs), small_code(a.y, rs), 0x0040);
        const uint32_t hi = __byte_perm(small_code(b.x, rs), small_code(b.y, rs), 0x0040);
        w[p] = __byte_perm(lo, hi, 0x5410);
      }
      if (fl) {  // outlier columns carry code 0
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (fl & (1u << e)) w[e >> 2] &= ~(0xffu << ((e & 3) * 8));
      }
      // byte kk = 8v of row r: box kk / 128, 16-byte chunk q = (kk % 128) / 16 stored at q ^ (r % 8)
      const int kk = 8 * v, box = kk >> 7, q = (kk & 127) >> 4;
      *reinterpret_cast<uint2*>(ca + box * LCA_BOX + r * 128 + ((q ^ (r & 7)) << 4) + (kk & 15)) = make_uint2(w[0], w[1]);
    }
  }
  if (warp == 0) {   // the sorted outlier list (ascending columns)
    const int per = (nwords + 31) / 32;
    const int w0 = min(lane * per, nwords), w1 = min(w0 + per, nwords);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(sbm[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(kAllLanes, incl, o);
      if (lane >= o) incl += y;
    }
    int pos = incl - cnt;
    for (int w = w0; w < w1; ++w) {
      uint32_t bits = sbm[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < kSmallListCap) s_list[pos] = 32 * w + b;
        ++pos;
      }
    }
    if (lane == 31) *s_cnt = incl;
  }
  fence_async_shared();   // the code tile was written by threads; the tensor core reads it
  __syncthreads();
  const int total = use_tau ? *s_cnt : 0;
  const int used = min(total, min(cap, kSmallListCap));
  if (blockIdx.x == 0 && tid == 0) {
    if (reset_status)
      hdr[0] = total > cap ? kStatusOutlierOverflow : kStatusOk;
    else if (total > cap)
      atomicCAS(hdr, kStatusOk, kStatusOutlierOverflow);
    hdr[1] = static_cast<uint32_t>(used);
    hdr[2] = static_cast<uint32_t>(total);
  }

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (the rest of the tile)
    if (lane == 0) {
      for (int st = LRS; st < nstage; ++st) {
        const int s = st % LRS;
        const uint32_t use = static_cast<uint32_t>(st / LRS);
        if (!mbar_wait_bounded(&empty[s], (use - 1) & 1u, s_abort, hdr, limit_ns)) break;
        const int b0 = st * LSB, nb = min(LSB, nbox - b0);
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nb * LBOX));
        filled |= 1u << s;
        fill_parity = (fill_parity & ~(1u << s)) | ((use & 1u) << s);
        for (int b = 0; b < nb; ++b) tma_load_2d(ring + s * LSTAGE + b * LBOX, &tmW, &full[s], (b0 + b) * 128, n0);
      }
      if (*s_abort) {
        int never = 0;
        for (int s = 0; s < LRS; ++s)
          if (filled & (1u << s)) mbar_wait_bounded(&full[s], (fill_parity >> s) & 1u, &never, nullptr, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_i8_s32(LM, LT);
      for (int st = 0; st < nstage && !*s_abort; ++st) {
        const int s = st % LRS;
        if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>(st / LRS) & 1u, s_abort, hdr, limit_ns)) break;
        tc_fence_after_sync();
        const int b0 = st * LSB, nb = min(LSB, nbox - b0);
        for (int b = 0; b < nb; ++b) {
          const uint64_t adesc = smem_desc_k_sw128(smem_addr(ring + s * LSTAGE + b * LBOX));
          const uint64_t bdesc = smem_desc_k_sw128(smem_addr(ca + (b0 + b) * LCA_BOX));
#pragma unroll
          for (int k = 0; k < 4; ++k)   // 32 bytes of K per MMA
            mma_i8(tmem_base, adesc + 2 * k, bdesc + 2 * k, idesc, (b0 + b > 0 || k > 0) ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);   // every MMA issued above has completed when this arrives
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- outlier term + epilogue
    // thread = weight row r of the tile (TMEM lane r: warps 4..7 read lane quadrants 0..3)
    const int quad = warp & 3, r = quad * 32 + lane, n = n0 + r;
    float d[LT];
#pragma unroll
    for (int t = 0; t < LT; ++t) d[t] = 0.f;
    int cur = 0;
    bool ok = true;
    for (int st = 0; st < nstage; ++st) {
      const int s = st % LRS;
      int got = 0;
      if (lane == 0) got = mbar_wait_bounded(&full[s], static_cast<uint32_t>(st / LRS) & 1u, s_abort, hdr, limit_ns);
      if (!__shfl_sync(kAllLanes, got, 0)) {
        ok = false;
        break;
      }
      const uint8_t* sa = ring + s * LSTAGE;
      const int kbeg = st * LSB * 128;
      while (cur < used) {
        const int j = s_list[cur];
        const int kk = j - kbeg;
        if (kk >= LSB * 128) break;
        const int box = kk >> 7, b = kk & 127;
        const float w = static_cast<float>(static_cast<int8_t>(sa[box * LBOX + r * 128 + (((b >> 4) ^ (r & 7)) << 4) + (b & 15)]));
#pragma unroll
        for (int t = 0; t < LT; ++t)
          if (t < M) d[t] = fmaf(__half2float(X[static_cast<size_t>(t) * K + j]), w, d[t]);
        ++cur;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    int acc = 0;
    if (ok && lane == 0) acc = mbar_wait_bounded(acc_full, 0, s_abort, hdr, limit_ns) ? 1 : 0;
    if (__shfl_sync(kAllLanes, acc, 0)) {
      tc_fence_after_sync();
      uint32_t c[LT];
      tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quad * 32) << 16), c);
      tmem_wait_ld();
      if (n < N) {
        const float sb = __ldg(SCB + n);
        const float bv = bias != nullptr ? __half2float(bias[n]) : 0.f;
#pragma unroll
        for (int t = 0; t < LT; ++t) {
          if (t >= M) break;
          const float y = fmaf(d[t], sb * (1.0f / 127.0f), fmaf(static_cast<float>(static_cast<int32_t>(c[t])), s_sa[t] * sb, bv));
          out[static_cast<size_t>(t) * N + n] = __float2half_rn(y);
        }
      }
    }
  }
  // the MMA thread's final commit arrives on acc_full; wait for it here too so
  // that TMEM is never released under an MMA still in flight
  if (warp == 1) {
    int never = 0;
    if (lane == 0) mbar_wait_bounded(acc_full, 0, &never, nullptr, limit_ns);
    __syncwarp();
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, LTMEM_COLS);
  }
}

cudaError_t launch_linear_small(const CUtensorMap& tmW, const __half* X, int M, int N, int K, float tau, int cap,
                                const float* SCB, const __half* bias, __half* out, uint32_t* hdr, uint64_t limit_ns,
                                bool reset_status, cudaStream_t st) {
  const size_t smem = linear_small_smem(K);
  static std::atomic<bool> attr_done[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64 || !attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(k_linear_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(linear_small_smem(kSmallMaxK)));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) attr_done[dev].store(true, std::memory_order_release);
  }
  const int grid = (N + LM - 1) / LM;
  k_linear_small<<<grid, LTHREADS, smem, st>>>(tmW, X, M, N, K, tau, cap, SCB, bias, out, hdr, limit_ns,
                                                reset_status ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace i8lt
