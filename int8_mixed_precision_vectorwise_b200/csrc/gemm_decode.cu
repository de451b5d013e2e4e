// Decode-regime (few tokens) LLM.int8() linear on sm_100a: the weight stream
// is the whole cost, so the tensor cores take the weights as the wide operand
// ("swap AB"):
//
//   C^T[n, t] = sum_k CB[n, k] * CA[t, k]       tcgen05 kind::i8, M = 128 weight rows, N = 16 tokens
//   out[t, n] = fp16(C * SCA[t] * SCB[n] / 127^2 + bias[n]
//                    + (SCB[n] / 127) * sum_{j in O} X[t, j] * CB[n, j])
//
// (the mixed decomposition of "`bitsandbytes` - `Linear8bitLt` integration
// into `transformers` models", section "About the mixed quantization method in
// few words", with the int8_linear_matmul / int8_mm_dequant ops of
// "LLM.int8() Refactoring: Part 1", section "Deprecations").
//
// Work split ("stream-K"): the (128-row tile, 128-byte k-block) grid is cut
// into one contiguous range of k-blocks per CTA, so every SM streams the same
// number of weight bytes.  A tile split across CTAs leaves int32 partials in a
// workspace slot per contributing CTA; per 32-row quarter, a counter tells
// the last contributor, which sums the partials and writes the outputs.
// Outlier columns (CA already zeroed there) are added by that last warp on
// CUDA cores from the gathered X[:, O] and the int8 weight columns.
//
// Block = 6 warps: TMA producer, MMA issuer (+ TMEM owner), 4 epilogue warps
// (one per 32-lane TMEM quadrant).  A 12-stage ring keeps ~200 KB of weights
// in flight per SM.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int DM = 128;                    // weight rows per tile (MMA M)
constexpr int DT = kDecodeMaxTokens;       // token columns (MMA N), zero padded
constexpr int DK = 128;                    // bytes of K per swizzle atom / TMA box
constexpr int DTHREADS = 64 + 128;
constexpr int DA_BYTES = DM * DK;          // 16 KB of weights per box
constexpr int DB_BYTES = DT * DK;          // 2 KB of codes per box
constexpr int DBOX_BYTES = DA_BYTES + DB_BYTES;
constexpr uint32_t DTMEM_COLS = 32;        // two 16-column accumulators

// C boxes (C x 128 bytes of K) per pipeline stage, DRING bytes of ring.
template <int C>
struct DecodeCfg {
  static constexpr int STAGE_BYTES = C * DBOX_BYTES;
  static constexpr int STAGES = (12 * DBOX_BYTES) / STAGE_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 5;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int MISC_OFF = BAR_OFF + ((NUM_BARS * 8 + 15) / 16) * 16;
  static constexpr int SMEM_ALLOC = MISC_OFF + 16 + 1024;
  static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
  static_assert(STAGE_BYTES % 1024 == 0, "stages must keep the 1024-byte swizzle alignment");
};

__device__ __forceinline__ void drain_wait_d(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  int never = 0;
  mbar_wait_bounded(bar, parity, &never, nullptr, limit_ns);
}

// The segments of this CTA's k-block range, in order: (tile, k0, k1).
struct SegIter {
  int kb, pos, end;
  __device__ SegIter(int kb_, int start, int end_) : kb(kb_), pos(start), end(end_) {}
  __device__ bool next(int& tile, int& k0, int& k1) {
    if (pos >= end) return false;
    tile = pos / kb;
    k0 = pos - tile * kb;
    k1 = min(kb, k0 + (end - pos));
    pos += k1 - k0;
    return true;
  }
};

}  // namespace

template <int C>
__global__ void __launch_bounds__(DTHREADS, 1)
    k_gemm_i8_decode(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmC,
                     const DecodeArgs p) {
  using Cfg = DecodeCfg<C>;
  constexpr int DSTAGES = Cfg::STAGES;
  constexpr int DSTAGE_BYTES = Cfg::STAGE_BYTES;
  constexpr int DKS = C * DK;  // bytes of K per stage
  extern __shared__ uint8_t dsmem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::BAR_OFF);
  uint64_t* empty = full + DSTAGES;
  uint64_t* acc_full = empty + DSTAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Cfg::MISC_OFF);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int N = p.N, K = p.K, T = p.M;
  const int kb = (K + DKS - 1) / DKS;  // stages of K per tile
  const int ntiles = (N + DM - 1) / DM;
  const int total = ntiles * kb;
  const int per = (total + gridDim.x - 1) / gridDim.x;  // k-blocks per CTA
  const int start = min(total, static_cast<int>(blockIdx.x) * per);
  const int end = min(total, start + per);

  if (threadIdx.x == 0) {
    for (int s = 0; s < DSTAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmW);
    tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, DTMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // The weights do not depend on the kernels queued just before this one
    // (quantiser, outlier prepare), so the first DSTAGES weight tiles are
    // requested before waiting for them; the code tiles follow the wait.
    if (lane == 0) {
      const int npos = end - start;
      const int npre = min(npos, DSTAGES);
      uint32_t filled = 0;
      for (int i = 0; i < npre; ++i) {  // stages 0..npre-1 of the first pass: free by construction
        const int pos = start + i, tile = pos / kb, k = pos - tile * kb;
        mbar_arrive_expect_tx(&full[i], DSTAGE_BYTES);
        filled |= 1u << i;
#pragma unroll
        for (int c = 0; c < C; ++c)
          tma_load_2d(smem + i * DSTAGE_BYTES + c * DA_BYTES, &tmW, &full[i], k * DKS + c * DK, tile * DM);
      }
      pdl_wait();
      for (int i = 0; i < npre; ++i) {
        const int pos = start + i, k = pos - (pos / kb) * kb;
#pragma unroll
        for (int c = 0; c < C; ++c)
          tma_load_2d(smem + i * DSTAGE_BYTES + C * DA_BYTES + c * DB_BYTES, &tmC, &full[i], k * DKS + c * DK, 0);
      }
      int stage = npre % DSTAGES;
      uint32_t phase = npre == DSTAGES ? 1u : 0u;
      uint32_t fill_parity = 0;
      for (int i = npre; i < npos; ++i) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, p.status, p.wait_limit_ns)) break;
        const int pos = start + i, tile = pos / kb, k = pos - tile * kb;
        uint8_t* sa = smem + stage * DSTAGE_BYTES;
        mbar_arrive_expect_tx(&full[stage], DSTAGE_BYTES);
        filled |= 1u << stage;
        fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
#pragma unroll
        for (int c = 0; c < C; ++c) {
          tma_load_2d(sa + c * DA_BYTES, &tmW, &full[stage], k * DKS + c * DK, tile * DM);
          tma_load_2d(sa + C * DA_BYTES + c * DB_BYTES, &tmC, &full[stage], k * DKS + c * DK, 0);
        }
        if (++stage == DSTAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (*s_abort) {
        for (int s = 0; s < DSTAGES; ++s)
          if (filled & (1u << s)) drain_wait_d(&full[s], (fill_parity >> s) & 1u, p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_i8_s32(DM, DT);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      SegIter seg(kb, start, end);
      int tile, k0, k1;
      while (!*s_abort && seg.next(tile, k0, k1)) {
        const int buf = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait_bounded(&acc_empty[buf], (use & 1u) ^ 1u, s_abort, p.status, p.wait_limit_ns)) break;
        tc_fence_after_sync();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * DT);
        bool ok = true;
        for (int k = k0; k < k1; ++k) {
          if (!mbar_wait_bounded(&full[stage], phase, s_abort, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_addr(smem + stage * DSTAGE_BYTES);
#pragma unroll
          for (int c = 0; c < C; ++c) {
            const uint64_t adesc = smem_desc_k_sw128(a_addr + c * DA_BYTES);
            const uint64_t bdesc = smem_desc_k_sw128(a_addr + C * DA_BYTES + c * DB_BYTES);
#pragma unroll
            for (int j = 0; j < DK / 32; ++j)
              mma_i8(d, adesc + 2 * j, bdesc + 2 * j, idesc, (k > k0 || c > 0 || j > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == DSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
        ++it;
      }
      tc_commit(mma_done);
      drain_wait_d(mma_done, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lanes = weight rows quad*32 .. +31 of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    pdl_wait();  // scales, outlier list and gathered inputs come from the preceding kernels
    const int n_used = p.n_used != nullptr ? min(max(*p.n_used, 0), p.out_cap) : 0;
    int it = 0;
    SegIter seg(kb, start, end);
    int tile, k0, k1;
    while (seg.next(tile, k0, k1)) {
      const int buf = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&acc_full[buf], use & 1u, s_abort, p.status, p.wait_limit_ns) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after_sync();
      uint32_t c[DT];
      tmem_ld_32x32b_x16(tmem_base + lane_off + static_cast<uint32_t>(buf * DT), c);
      tmem_wait_ld();
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);  // the accumulator is in registers now
      ++it;

      const int n = tile * DM + quad * 32 + lane;
      // contributors of this tile: CTAs whose k-block range meets it
      const int first = (tile * kb) / per;
      const int last_cta = ((tile + 1) * kb - 1) / per;
      const int nseg = last_cta - first + 1;
      bool finalize = true;
      if (nseg > 1) {
        const int slot = static_cast<int>(blockIdx.x) - first;
        int32_t* part = p.partials + (static_cast<size_t>(slot) * DT) * N;
        if (n < N) {
#pragma unroll
          for (int t = 0; t < DT; ++t)
            if (t < T) __stcg(part + static_cast<size_t>(t) * N + n, static_cast<int32_t>(c[t]));
        }
        __threadfence();
        __syncwarp();
        int mine = 0;
        if (lane == 0) mine = atomicAdd(p.counters + tile * 4 + quad, 1) == nseg - 1;
        finalize = __shfl_sync(0xffffffffu, mine, 0) != 0;
        if (finalize) {
          __threadfence();
          if (n < N) {
#pragma unroll
            for (int t = 0; t < DT; ++t) {
              if (t >= T) break;
              int32_t sum = 0;
              for (int sl = 0; sl < nseg; ++sl)
                sum += __ldcg(p.partials + (static_cast<size_t>(sl) * DT + t) * N + n);
              c[t] = static_cast<uint32_t>(sum);
            }
          }
        }
      }
      if (!finalize || n >= N) continue;
      // dequant + bias + outlier columns for (t, n), t < T
      const float sb = __ldg(p.SCB + n);
      const float bv = p.bias != nullptr ? __half2float(p.bias[n]) : 0.f;
      float d[DT];
#pragma unroll
      for (int t = 0; t < DT; ++t) d[t] = 0.f;
      const int8_t* cbrow = p.CB + static_cast<size_t>(n) * K;
      for (int j0 = 0; j0 < n_used; j0 += 16) {
        // issue up to 16 outlier-weight loads at once, then use them
        float w[16];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj)
          w[jj] = j0 + jj < n_used ? static_cast<float>(cbrow[__ldg(p.idx + j0 + jj)]) : 0.f;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          if (j0 + jj >= n_used) break;
#pragma unroll
          for (int t = 0; t < DT; ++t)
            if (t < T) d[t] = fmaf(__half2float(p.XO[static_cast<size_t>(t) * p.ld_o + j0 + jj]), w[jj], d[t]);
        }
      }
#pragma unroll
      for (int t = 0; t < DT; ++t) {
        if (t >= T) break;
        const float sa = __ldg(p.SCA + t) * (1.0f / 16129.0f);
        const float y = fmaf(d[t], sb * (1.0f / 127.0f),
                             fmaf(static_cast<float>(static_cast<int32_t>(c[t])), sa * sb, bv));
        p.out[static_cast<size_t>(t) * N + n] = __float2half_rn(y);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, DTMEM_COLS);
  }
}

template <int C>
static cudaError_t launch_decode_c(const CUtensorMap& tmW, const CUtensorMap& tmC, const DecodeArgs& a, int grid,
                                   cudaStream_t st) {
  static bool attr_done = false;
  if (!attr_done) {
    cudaError_t e = cudaFuncSetAttribute(k_gemm_i8_decode<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DecodeCfg<C>::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(DTHREADS, 1, 1);
  cfg.dynamicSmemBytes = DecodeCfg<C>::SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k_gemm_i8_decode<C>, tmW, tmC, a);
}

cudaError_t launch_gemm_decode(const CUtensorMap& tmW, const CUtensorMap& tmC, const DecodeArgs& a, int grid,
                               int boxes_per_stage, cudaStream_t st) {
  switch (boxes_per_stage) {
    case 2: return launch_decode_c<2>(tmW, tmC, a, grid, st);
    case 4: return launch_decode_c<4>(tmW, tmC, a, grid, st);
    default: return launch_decode_c<1>(tmW, tmC, a, grid, st);
  }
}

}  // namespace i8lt
