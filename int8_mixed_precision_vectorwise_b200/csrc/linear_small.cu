// The whole LLM.int8() Linear8bitLt forward of a small problem in one launch
// (few tokens, a small weight): the mixed int8 / fp16 decomposition of
// "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models"
// (section "About the mixed quantization method in few words") built from the
// int8_vectorwise_quant / int8_linear_matmul / int8_mm_dequant ops of
// "LLM.int8() Refactoring: Part 1" (sections "Improved kernels for
// inference" and "Deprecations").
//
// For such sizes the forward's cost is launches and latency, not bytes, so
// everything happens in one grid with no workspace round trip, spread over as
// many SMs as the problem allows: a cluster of KS CTAs (1, 2, 4 or 8) owns
// weight rows [128t, 128t + 128), and CTA `rank` of it owns a slice of K (whole
// 128-column boxes).  Each CTA
//   1. requests its slice of the weight tile through TMA (first of all: the
//      weights do not depend on X);
//   2. reads its slice of X: per row the absmax over the elements below the
//      threshold, and the outlier-column flags of its columns; the sorted list
//      of its outlier columns;
//   3. stores its row maxima and outlier count into every CTA of the cluster
//      (distributed shared memory, no remote loads); after one cluster barrier
//      each CTA has them locally: the row scale is the max over all slices, and
//      a column's position in the forward's ascending outlier list is its CTA's
//      offset plus its index in the CTA's list;
//   4. writes its codes (outlier columns zeroed; their X values kept in shared
//      memory for step 5) straight into shared memory in the 128B-swizzled
//      K-major layout the tensor core reads, and runs tcgen05 kind::i8 MMAs
//      (M = 128 weight rows, N = 16 token columns, int32 accumulator in TMEM) as
//      the weight boxes land;
//   5. computes the outlier term X[t, j] * CB[n, j] of its outlier columns from
//      the staged weight boxes (CUDA cores, fp32, ascending columns);
//   6. stores its int32 partial accumulator and fp32 outlier partial sums of
//      each row into the CTA that finishes the row (CTA `rank` owns rows
//      [rank * 128 / KS, (rank + 1) * 128 / KS)); after a second cluster barrier
//      that CTA adds the KS partials in rank order (the int32 sum is exact) and
//      applies dequant and bias:
//        out[t, n] = fp16(C * SCA[t] * SCB[n] / 127^2 + bias[n] + (SCB[n] / 127) * D).
// A first cluster barrier, split into an arrive at the start and a wait before
// the first remote store, makes sure every CTA of the cluster has started.
// Block 0 writes the status word and the outlier counts.  Every mbarrier wait
// is bounded by a time limit; on expiry the status becomes I8_ERR_TIMEOUT and
// the CTA still takes every cluster barrier (after its in-flight copies and
// MMAs have completed), so its peers never wait for it for good.
#include <cuda_fp16.h>

#include <atomic>

#include "kernels.cuh"
#include "per_device.h"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int LM = 128;                       // weight rows per cluster (MMA M)
constexpr int LT = kDecodeMaxTokens;          // token columns (MMA N), zero padded
constexpr int LBOX = LM * 128;                // one 128-byte-deep weight box: 16 KB
constexpr int LSB = 2;                        // weight boxes per ring stage
constexpr int LSTAGE = LSB * LBOX;            // 32 KB
constexpr int LRS = 4;                        // ring stages at most
constexpr int LCA_BOX = LT * 128;             // one 128-byte-deep box of the 16 code rows: 2 KB
constexpr int LTHREADS = 256;
constexpr int LPU = 4;                        // X vectors per thread in flight while quantising
constexpr int LMAXKS = 8;                     // CTAs per cluster at most
constexpr uint32_t LTMEM_COLS = 32;
constexpr unsigned kAllLanes = 0xffffffffu;

// Shared memory of a CTA whose slice has nbl boxes, in a cluster of ks CTAs.  With
// ks > 1 it also receives the other CTAs' row maxima and outlier counts (xch) and, for
// its 128 / ks rows, their partial sums (red: int32 C and fp32 D, [ks][128 / ks][16]).
struct SmallLayout {
  int stages, ca_off, sbm_off, wpre_off, list_off, xo_off, sc_off, xch_off, red_off, misc_off, bar_off, total;
  __host__ __device__ SmallLayout(int nbl, int ks) {
    stages = (nbl + LSB - 1) / LSB < LRS ? (nbl + LSB - 1) / LSB : LRS;
    ca_off = stages * LSTAGE;
    sbm_off = ca_off + nbl * LCA_BOX;
    wpre_off = sbm_off + nbl * 16;                            // 4 bitmap words per box
    list_off = wpre_off + nbl * 16;                           // outlier columns before each word
    xo_off = list_off + kSmallListCap * 4;                    // X of the listed columns, fp16 [cap][16]
    sc_off = xo_off + kSmallListCap * LT * 2;                 // SCB and bias of the tile's rows
    xch_off = sc_off + 2 * LM * 4;
    red_off = xch_off + (ks > 1 ? (LMAXKS * LT + LMAXKS) * 4 : 0);
    misc_off = red_off + (ks > 1 ? 2 * LM * LT * 4 : 0);
    bar_off = (misc_off + 4 * LT * 4 + 32 + 7) & ~7;
    total = bar_off + (2 * LRS + 1) * 8 + 1024;  // + slack to align the ring to 1024 bytes
  }
};

__device__ __forceinline__ uint32_t small_code(float x, float r) {
  uint32_t q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(__fmul_rn(x, r)));
  return q;
}

}  // namespace

size_t linear_small_smem(int K, int ks) {
  const int nbox = (K + 127) / 128;
  return static_cast<size_t>(SmallLayout((nbox + ks - 1) / ks, ks).total);
}

int linear_small_split(int N, int K, int num_sms) {
  const int ntile = (N + LM - 1) / LM, nbox = (K + 127) / 128;
  int ks = LMAXKS;
  while (ks > 1 && (ks > nbox || static_cast<long long>(ntile) * ks > num_sms)) ks /= 2;
  return ks;
}

__global__ void __launch_bounds__(LTHREADS, 1)
    k_linear_small(const __grid_constant__ CUtensorMap tmW, const __half* __restrict__ X, int M, int N, int K,
                   float tau, int cap, const float* __restrict__ SCB, const __half* __restrict__ bias,
                   __half* __restrict__ out, uint32_t* hdr, uint64_t limit_ns, int reset_status, int KS) {
  extern __shared__ uint8_t lsm_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(lsm_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int rank = KS > 1 ? static_cast<int>(blockIdx.x % KS) : 0;
  const int n0 = (KS > 1 ? static_cast<int>(blockIdx.x / KS) : static_cast<int>(blockIdx.x)) * LM;
  const int nbox = (K + 127) / 128;
  const int kb0 = rank * nbox / KS, kb1 = (rank + 1) * nbox / KS;  // this CTA's boxes
  const int nbl = kb1 - kb0;
  const int nbl_max = (nbox + KS - 1) / KS;                         // the layout is the same in every CTA
  const SmallLayout Lay(nbl_max, KS);
  uint8_t* ring = smem;
  uint8_t* ca = smem + Lay.ca_off;
  uint32_t* sbm = reinterpret_cast<uint32_t*>(smem + Lay.sbm_off);
  int32_t* s_wpre = reinterpret_cast<int32_t*>(smem + Lay.wpre_off);
  int32_t* s_list = reinterpret_cast<int32_t*>(smem + Lay.list_off);
  __half* xo = reinterpret_cast<__half*>(smem + Lay.xo_off);
  float* s_sb = reinterpret_cast<float*>(smem + Lay.sc_off);
  float* s_bv = s_sb + LM;
  uint32_t* s_xmax = reinterpret_cast<uint32_t*>(smem + Lay.xch_off);  // [KS][16] row maxima of each CTA
  uint32_t* s_xcnt = s_xmax + LMAXKS * LT;                               // [KS] outlier columns of each CTA
  int32_t* red_c = reinterpret_cast<int32_t*>(smem + Lay.red_off);
  float* red_d = reinterpret_cast<float*>(red_c + LM * LT);
  uint32_t* s_rowmax = reinterpret_cast<uint32_t*>(smem + Lay.misc_off);  // this slice's maxima (fp32 bits)
  float* s_r = reinterpret_cast<float*>(s_rowmax + LT);
  float* s_sa = s_r + LT;
  int* s_cnt = reinterpret_cast<int*>(s_sa + LT);         // [0] this slice's outlier columns
  int* s_base = s_cnt + 1;                                // [0] columns in earlier slices, [1] in all
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(s_cnt + 3);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_cnt + 4);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay.bar_off);
  uint64_t* empty = full + LRS;
  uint64_t* acc_full = empty + LRS;

  const int k0 = kb0 * 128, k1 = min(K, kb1 * 128);       // this CTA's columns
  const int nstage = (nbl + LSB - 1) / LSB;
  const int RS = Lay.stages;
  const int nvec = (k1 - k0) >> 3, nwords = nbl * 4;
  const bool use_tau = tau > 0.f;

  // ---------------------------------------------------------------- set-up (no global memory)
  // The kernel is a programmatic dependent launch: this part may run while the previous
  // kernel of the stream finishes; every global access comes after pdl_wait().
  if (tid == 0) {
    for (int s = 0; s < LRS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);   // the MMAs' commit and the 4 outlier / epilogue warps
    }
    mbar_init(acc_full, 1);
    *s_abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, LTMEM_COLS);
    tmem_relinquish();
  }
  for (int w = tid; w < nwords; w += LTHREADS) sbm[w] = 0u;
  if (tid < LT) s_rowmax[tid] = 0u;
  {  // zero the code tile: rows past M and bytes past K must be 0 for the MMA
    uint4* z = reinterpret_cast<uint4*>(ca);
    for (int i = tid; i < nbl * LCA_BOX / 16; i += LTHREADS) z[i] = make_uint4(0, 0, 0, 0);
  }
  pdl_wait();
  pdl_launch_dependents();   // the next kernel's set-up may overlap the rest of this one

  // the weight slice does not depend on X: thread 0 requests the first stages (its barriers
  // are initialised and fenced above); then every thread requests its first X vectors and
  // this tile's row scales and bias, whose latency the block barrier below overlaps
  uint32_t filled = 0, fill_parity = 0;
  if (tid == 0) {
    for (int st = 0; st < nstage && st < RS; ++st) {
      const int b0 = st * LSB, nb = min(LSB, nbl - b0);
      mbar_arrive_expect_tx(&full[st], static_cast<uint32_t>(nb * LBOX));
      filled |= 1u << st;
      for (int b = 0; b < nb; ++b)
        tma_load_2d(ring + st * LSTAGE + b * LBOX, &tmW, &full[st], (kb0 + b0 + b) * 128, n0);
    }
  }
  const int items = M * nvec;
  const bool one_chunk = items <= LPU * LTHREADS;
  uint4 xv[LPU];
  auto load_x = [&](int base) {
#pragma unroll
    for (int u = 0; u < LPU; ++u) {
      const int it = base + u * LTHREADS + tid;
      xv[u] = make_uint4(0, 0, 0, 0);
      if (it < items) {
        const int r = it / nvec;
        xv[u] = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(r) * K + k0) + (it - r * nvec));
      }
    }
  };
  load_x(0);
  float sb_row = 0.f, bv_row = 0.f;
  if (tid < LM && n0 + tid < N) {
    sb_row = __ldg(SCB + n0 + tid);
    if (bias != nullptr) bv_row = __half2float(bias[n0 + tid]);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;
  // first half of a cluster barrier: its wait (before the first store into another CTA's
  // shared memory) guarantees that every CTA of the cluster has started
  if (KS > 1) cluster_arrive_relaxed();

  // ---------------------------------------------------------------- this slice of X (all threads)
  // Items (row, 8-column vector) in chunks of LPU per thread: all LPU loads of
  // a chunk are issued before any is used.  When the slice fits in one chunk it
  // stays in registers for the codes; otherwise they read each chunk again.
  for (int base = 0; base < items; base += LPU * LTHREADS) {   // row maxima below the threshold, column flags
    if (base > 0) load_x(base);
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
  if (KS > 1) cluster_wait();
  if (warp == 0) {   // this slice's sorted outlier list (ascending columns)
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
      s_wpre[w] = pos;
      uint32_t bits = sbm[w];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < kSmallListCap) s_list[pos] = k0 + 32 * w + b;
        ++pos;
      }
    }
    if (lane == 31) *s_cnt = incl;
    // row maxima and the count go to every CTA of the cluster (this one included)
    if (KS > 1) {
      if (lane < LT) {
        const uint32_t a = smem_addr(s_xmax + rank * LT + lane), m = s_rowmax[lane];
        for (int r = 0; r < KS; ++r) st_cluster_u32(map_to_rank(a, r), m);
      } else if (lane == 31) {
        const uint32_t a = smem_addr(s_xcnt + rank);
        for (int r = 0; r < KS; ++r) st_cluster_u32(map_to_rank(a, r), static_cast<uint32_t>(incl));
      }
    }
  }
  if (tid < LM) {
    s_sb[tid] = sb_row;
    s_bv[tid] = bv_row;
  }
  // ---------------------------------------------------------------- exchange with the cluster
  if (KS > 1) cluster_sync(); else __syncthreads();
  // the pushed values are local now
  if (tid < LT) {
    uint32_t m = s_rowmax[tid];
    for (int r = 0; r < KS && KS > 1; ++r) m = max(m, s_xmax[r * LT + tid]);
    const float amax = tid < M ? __uint_as_float(m) : 0.f;
    s_r[tid] = amax > 0.f ? __fdiv_rn(127.0f, amax) : 0.0f;
    s_sa[tid] = amax * (1.0f / 16129.0f);
  } else if (tid == LT) {
    int before = 0, all = *s_cnt;
    if (KS > 1) {
      all = 0;
      for (int r = 0; r < KS; ++r) {
        const int c = static_cast<int>(s_xcnt[r]);
        if (r < rank) before += c;
        all += c;
      }
    }
    s_base[0] = before;
    s_base[1] = all;
  }
  __syncthreads();
  for (int base = 0; base < items; base += LPU * LTHREADS) {   // codes into the swizzled K-major tile
    if (!one_chunk) load_x(base);
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
      if (fl) {  // outlier columns carry code 0; their X values go to xo at their list position
        const __half* hx = reinterpret_cast<const __half*>(&xv[u]);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (fl & (1u << e)) {
            w[e >> 2] &= ~(0xffu << ((e & 3) * 8));
            const int c = 8 * v + e, wd = c >> 5;
            const int pos = s_wpre[wd] + __popc(sbm[wd] & ((1u << (c & 31)) - 1u));
            if (pos < kSmallListCap) xo[pos * LT + r] = hx[e];
          }
      }
      // byte kk = 8v of row r in the slice: box kk / 128, 16-byte chunk q = (kk % 128) / 16 stored at q ^ (r % 8)
      const int kk = 8 * v, box = kk >> 7, q = (kk & 127) >> 4;
      *reinterpret_cast<uint2*>(ca + box * LCA_BOX + r * 128 + ((q ^ (r & 7)) << 4) + (kk & 15)) = make_uint2(w[0], w[1]);
    }
  }
  fence_async_shared();   // the code tile was written by threads; the tensor core reads it
  __syncthreads();
  const int total = use_tau ? s_base[1] : 0;
  const int used = min(total, min(cap, kSmallListCap));
  // entries [0, lused) of this slice's list are in the forward's first `used` columns
  const int lused = use_tau ? max(0, min(*s_cnt, used - s_base[0])) : 0;
  if (blockIdx.x == 0 && tid == 0) {
    if (reset_status)
      hdr[0] = total > cap ? kStatusOutlierOverflow : kStatusOk;
    else if (total > cap)
      atomicCAS(hdr, kStatusOk, kStatusOutlierOverflow);
    hdr[1] = static_cast<uint32_t>(used);
    hdr[2] = static_cast<uint32_t>(total);
  }

  const int quad = warp & 3, row = quad * 32 + lane;    // epilogue warps 4..7: weight row of the tile
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (the rest of the slice)
    if (lane == 0) {
      for (int st = RS; st < nstage; ++st) {
        const int s = st % RS;
        const uint32_t use = static_cast<uint32_t>(st / RS);
        if (!mbar_wait_bounded(&empty[s], (use - 1) & 1u, s_abort, hdr, limit_ns)) break;
        const int b0 = st * LSB, nb = min(LSB, nbl - b0);
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nb * LBOX));
        filled |= 1u << s;
        fill_parity = (fill_parity & ~(1u << s)) | ((use & 1u) << s);
        for (int b = 0; b < nb; ++b)
          tma_load_2d(ring + s * LSTAGE + b * LBOX, &tmW, &full[s], (kb0 + b0 + b) * 128, n0);
      }
      if (*s_abort) {
        int never = 0;
        for (int s = 0; s < RS; ++s)
          if (filled & (1u << s)) mbar_wait_bounded(&full[s], (fill_parity >> s) & 1u, &never, nullptr, limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_i8_s32(LM, LT);
      for (int st = 0; st < nstage && !*s_abort; ++st) {
        const int s = st % RS;
        if (!mbar_wait_bounded(&full[s], static_cast<uint32_t>(st / RS) & 1u, s_abort, hdr, limit_ns)) break;
        tc_fence_after_sync();
        const int b0 = st * LSB, nb = min(LSB, nbl - b0);
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
    // ---------------------------------------------------------------- outlier term + partial results
    // thread = weight row `row` of the tile (TMEM lane row: warps 4..7 read lane quadrants 0..3)
    float d[LT];
#pragma unroll
    for (int t = 0; t < LT; ++t) d[t] = 0.f;
    int cur = 0;
    bool ok = true;
    for (int st = 0; st < nstage; ++st) {
      const int s = st % RS;
      int got = 0;
      if (lane == 0) got = mbar_wait_bounded(&full[s], static_cast<uint32_t>(st / RS) & 1u, s_abort, hdr, limit_ns);
      if (!__shfl_sync(kAllLanes, got, 0)) {
        ok = false;
        break;
      }
      const uint8_t* sa = ring + s * LSTAGE;
      const int kbeg = k0 + st * LSB * 128;
      while (cur < lused) {
        const int j = s_list[cur];
        const int kk = j - kbeg;
        if (kk >= LSB * 128) break;
        const int box = kk >> 7, b = kk & 127;
        const float w =
            static_cast<float>(static_cast<int8_t>(sa[box * LBOX + row * 128 + (((b >> 4) ^ (row & 7)) << 4) + (b & 15)]));
#pragma unroll
        for (int t = 0; t < LT; ++t)
          if (t < M) d[t] = fmaf(__half2float(xo[cur * LT + t]), w, d[t]);
        ++cur;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    int acc = 0;
    if (ok && lane == 0) acc = mbar_wait_bounded(acc_full, 0, s_abort, hdr, limit_ns) ? 1 : 0;
    uint32_t c[LT];
#pragma unroll
    for (int t = 0; t < LT; ++t) c[t] = 0u;
    if (__shfl_sync(kAllLanes, acc, 0)) {
      tc_fence_after_sync();
      tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quad * 32) << 16), c);
      tmem_wait_ld();
    }
    if (KS == 1) {
      const int n = n0 + row;
      if (n < N) {
        const float sb = s_sb[row], bv = s_bv[row];
#pragma unroll
        for (int t = 0; t < LT; ++t) {
          if (t >= M) break;
          const float y = fmaf(d[t], sb * (1.0f / 127.0f),
                               fmaf(static_cast<float>(static_cast<int32_t>(c[t])), s_sa[t] * sb, bv));
          out[static_cast<size_t>(t) * N + n] = __float2half_rn(y);
        }
      }
    } else {
      // partials of row `row` (16 int32, 16 fp32) go to the CTA that finishes the row
      const int rpr = LM / KS, owner = row / rpr, slot = row - owner * rpr;
      const uint32_t ac = map_to_rank(smem_addr(red_c + (rank * rpr + slot) * LT), owner);
      const uint32_t ad = map_to_rank(smem_addr(red_d + (rank * rpr + slot) * LT), owner);
#pragma unroll
      for (int ch = 0; ch < LT / 4; ++ch) {
        st_cluster_v4(ac + 16u * ch, c[4 * ch], c[4 * ch + 1], c[4 * ch + 2], c[4 * ch + 3]);
        st_cluster_v4(ad + 16u * ch, __float_as_uint(d[4 * ch]), __float_as_uint(d[4 * ch + 1]),
                      __float_as_uint(d[4 * ch + 2]), __float_as_uint(d[4 * ch + 3]));
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
  if (KS > 1) {
    // ---------------------------------------------------------------- sum of the cluster's partials
    cluster_sync();   // every partial of this CTA's rows has arrived; nothing is read remotely after this
    const int rpr = LM / KS;
    for (int e = tid; e < rpr * LT; e += LTHREADS) {
      const int slot = e / LT, t = e % LT, rl = rank * rpr + slot, n = n0 + rl;
      if (t >= M || n >= N) continue;
      int32_t csum = 0;
      float dsum = 0.f;
      for (int r = 0; r < KS; ++r) {   // rank order
        csum += red_c[(r * rpr + slot) * LT + t];
        dsum += red_d[(r * rpr + slot) * LT + t];
      }
      const float sb = s_sb[rl], bv = s_bv[rl];
      const float y = fmaf(dsum, sb * (1.0f / 127.0f), fmaf(static_cast<float>(csum), s_sa[t] * sb, bv));
      out[static_cast<size_t>(t) * N + n] = __float2half_rn(y);
    }
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
                                bool reset_status, int num_sms, cudaStream_t st) {
  const int ks = linear_small_split(N, K, num_sms);
  const size_t smem = linear_small_smem(K, ks);
  static PerDeviceOnce attr_done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  cudaError_t e = cudaSuccess;
  if (!attr_done.run(dev, [&] {
        e = cudaFuncSetAttribute(k_linear_small, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(linear_small_smem(kSmallMaxK, 1)));
        return e == cudaSuccess;
      }))
    return e;
  const int ntile = (N + LM - 1) / LM;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ntile * ks);
  cfg.blockDim = dim3(LTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = ks;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = ks > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, k_linear_small, tmW, X, M, N, K, tau, cap, SCB, bias, out, hdr, limit_ns,
                            reset_status ? 1 : 0, ks);
}

}  // namespace i8lt
