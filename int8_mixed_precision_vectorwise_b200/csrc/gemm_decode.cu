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
// Work split ("stream-K"): the (128-row tile, k-stage) grid is cut into one
// contiguous range of stages per CTA, so every SM streams the same number of
// weight bytes.  A tile split across CTAs leaves int32 partials (and fp32
// partials of the outlier term) in a workspace slot per contributing CTA; per
// 32-row quarter, a counter tells the last contributor, which sums them and
// writes the outputs.
//
// The outlier columns (CA already zeroed there) are added from the weight
// tiles while they sit in shared memory: every column is streamed exactly
// once, by the CTA whose k-range holds it, so the fp16 term costs no extra
// HBM traffic.
//
// Block = 7 warps: TMA producer, MMA issuer (+ TMEM owner), 4 epilogue warps
// (one per 32-lane TMEM quadrant), and the outlier warp.  A stage is released
// when both the MMAs and the outlier warp are done with it.  A 3-stage ring of
// 72 KB stages keeps ~216 KB of weights in flight per SM.
#include <cuda_fp16.h>

#include <atomic>

#include "kernels.cuh"
#include "per_device.h"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int DM = 128;                    // weight rows per tile (MMA M)
constexpr int DT = kDecodeMaxTokens;       // token columns (MMA N), zero padded
constexpr int DK = 128;                    // bytes of K per swizzle atom / TMA box
constexpr int DL2_AHEAD = 8;               // weight stages past the ring prefetched into L2 before the wait
constexpr int DTHREADS = 64 + 128 + 32;
constexpr int DA_BYTES = DM * DK;          // 16 KB of weights per box
constexpr int DB_BYTES = DT * DK;          // 2 KB of codes per box
constexpr int DBOX_BYTES = DA_BYTES + DB_BYTES;
constexpr uint32_t DTMEM_COLS = 32;        // two 16-column accumulators

// C boxes (C x 128 bytes of K) per pipeline stage, DRING bytes of ring.
constexpr int DS_BYTES = DT * DM * 4;      // one segment's outlier term, fp32 [token][row]
constexpr int XS_COLS = 32;                // outlier columns of X[:, O] kept in shared memory
constexpr int XS_BYTES = DT * XS_COLS * 2; // fp16 [column][token]

// d[i][t] += X[t, j] * CB[row lane + 32 i, j] for tokens t < TT (>= T; the
// rest of d is untouched), list entry c = column j at byte b of the 128-row
// box `box` (128B swizzle: 16-byte chunk q of row r sits at q ^ (r % 8)).
// X[:, j] comes from x_s ([column][token], zero past T) for the first XS_COLS
// entries, else from X_O.
template <int TT>
__device__ __forceinline__ void outlier_column(float (&d)[4][kDecodeMaxTokens], const uint8_t* box, int b, int lane,
                                               const __half* x_s, const __half* XO, int ld_o, int c, int T) {
  float x[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t)
    x[t] = c < XS_COLS ? __half2float(x_s[c * kDecodeMaxTokens + t])
                       : (t < T ? __half2float(XO[static_cast<size_t>(t) * ld_o + c]) : 0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = lane + 32 * i;
    const float w = static_cast<float>(static_cast<int8_t>(box[r * 128 + ((((b >> 4) ^ (r & 7))) << 4) + (b & 15)]));
#pragma unroll
    for (int t = 0; t < TT; ++t) d[i][t] = fmaf(x[t], w, d[i][t]);
  }
}

template <int C>
struct DecodeCfg {
  static constexpr int STAGE_BYTES = C * DBOX_BYTES;
  static constexpr int STAGES = (12 * DBOX_BYTES) / STAGE_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 7;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int DS_OFF = BAR_OFF + ((NUM_BARS * 8 + 15) / 16) * 16;
  static constexpr int XS_OFF = DS_OFF + DS_BYTES;
  static constexpr int MISC_OFF = XS_OFF + XS_BYTES;
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
  uint64_t* d_full = mma_done + 1;       // the outlier term of a segment is in d_s
  uint64_t* d_empty = d_full + 1;        // ... and has been read by the 4 epilogue warps
  float* d_s = reinterpret_cast<float*>(smem + Cfg::DS_OFF);
  __half* x_s = reinterpret_cast<__half*>(smem + Cfg::XS_OFF);
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
      mbar_init(&empty[s], 2);  // the MMAs' commit and the outlier warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(mma_done, 1);
    mbar_init(d_full, 1);
    mbar_init(d_empty, 4);
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
      // the weight stages after the ring go to L2 while the preceding kernel finishes, so
      // HBM keeps streaming during the wait and those stages later load from L2
      for (int i = npre; i < min(npos, npre + DL2_AHEAD); ++i) {
        const int pos = start + i, tile = pos / kb, k = pos - tile * kb;
#pragma unroll
        for (int c = 0; c < C; ++c) tma_prefetch_l2_2d(&tmW, k * DKS + c * DK, tile * DM);
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
  } else if (warp == 6) {
    // ---------------------------------------------------------------- outlier warp
    // Lane l owns rows l, l+32, l+64, l+96 of the tile.  Every stage is waited
    // for and released; stages holding outlier columns add X[t, j] * CB[n, j]
    // (weights read from the swizzled tile) into a per-segment fp32 sum that
    // is handed to the epilogue through d_s at the segment's end.
    pdl_wait();  // outlier list and gathered X come from the preceding kernel
    const int n_used = p.n_used != nullptr ? min(max(*p.n_used, 0), p.out_cap) : 0;
    // the first XS_COLS outlier columns of X, as [column][token], so the
    // per-stage updates read shared memory instead of waiting on global loads
    for (int e = lane; e < min(n_used, XS_COLS) * DT; e += 32) {
      const int j = e / DT, t = e - j * DT;
      x_s[e] = t < T ? p.XO[static_cast<size_t>(t) * p.ld_o + j] : __float2half_rn(0.f);
    }
    __syncwarp();
    int stage = 0;
    uint32_t phase = 0;
    int segi = 0;
    bool ok = true;
    SegIter seg(kb, start, end);
    int tile, k0, k1;
    while (ok && seg.next(tile, k0, k1)) {
      float d[4][DT];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int t = 0; t < DT; ++t) d[i][t] = 0.f;
      // first outlier column at or after this segment's k-range
      int cur = 0;
      while (cur < n_used && __ldg(p.idx + cur) < k0 * DKS) ++cur;
      for (int k = k0; k < k1; ++k) {
        int got = 0;
        if (lane == 0) got = mbar_wait_bounded(&full[stage], phase, s_abort, p.status, p.wait_limit_ns) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        const uint8_t* sa = smem + stage * DSTAGE_BYTES;
        while (cur < n_used) {
          const int j = __ldg(p.idx + cur);
          if (j >= (k + 1) * DKS) break;
          const int kk = j - k * DKS;                // byte within the stage
          const int box = kk >> 7, b = kk & 127;     // 128-byte box, byte within the row
          if (T <= 4)
            outlier_column<4>(d, sa + box * DA_BYTES, b, lane, x_s, p.XO, p.ld_o, cur, T);
          else
            outlier_column<DT>(d, sa + box * DA_BYTES, b, lane, x_s, p.XO, p.ld_o, cur, T);
          ++cur;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == DSTAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      // hand the segment's sum to the epilogue (once it has read the previous one)
      if (segi > 0) {
        int got = 0;
        if (lane == 0) got = mbar_wait_bounded(d_empty, static_cast<uint32_t>(segi - 1) & 1u, s_abort, p.status,
                                               p.wait_limit_ns) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, got, 0)) break;
      }
      if (n_used > 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int t = 0; t < DT; ++t) d_s[t * DM + lane + 32 * i] = d[i][t];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(d_full);
      ++segi;
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lanes = weight rows quad*32 .. +31 of the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    pdl_wait();  // scales and the outlier count come from the preceding kernel
    const bool raw = p.C != nullptr;  // store the int32 sums instead of the dequantised outputs
    const int n_used = p.n_used != nullptr ? min(max(*p.n_used, 0), p.out_cap) : 0;
    const size_t dpart = static_cast<size_t>(p.slots) * DT * N;  // fp32 partials follow the int32 ones
    int it = 0;
    SegIter seg(kb, start, end);
    int tile, k0, k1;
    while (seg.next(tile, k0, k1)) {
      const int buf = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const int n = tile * DM + quad * 32 + lane;
      const float sb = (!raw && n < N) ? __ldg(p.SCB + n) : 0.f;
      const float bv = (!raw && n < N && p.bias != nullptr) ? __half2float(p.bias[n]) : 0.f;
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
      // this segment's outlier term (the outlier warp is done with the segment by now or soon)
      ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(d_full, static_cast<uint32_t>(it) & 1u, s_abort, p.status, p.wait_limit_ns) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      float d[DT];
#pragma unroll
      for (int t = 0; t < DT; ++t) d[t] = (n_used > 0 && t < T) ? d_s[t * DM + quad * 32 + lane] : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(d_empty);
      ++it;

      // contributors of this tile: CTAs whose k-stage range meets it
      const int first = (tile * kb) / per;
      const int last_cta = ((tile + 1) * kb - 1) / per;
      const int nseg = last_cta - first + 1;
      bool finalize = true;
      if (nseg > 1) {
        const int slot = static_cast<int>(blockIdx.x) - first;
        int32_t* part = p.partials + (static_cast<size_t>(slot) * DT) * N;
        float* dp = reinterpret_cast<float*>(p.partials + dpart) + (static_cast<size_t>(slot) * DT) * N;
        if (n < N) {
#pragma unroll
          for (int t = 0; t < DT; ++t) {
            if (t >= T) break;
            __stcg(part + static_cast<size_t>(t) * N + n, static_cast<int32_t>(c[t]));
            if (n_used > 0) __stcg(dp + static_cast<size_t>(t) * N + n, d[t]);
          }
        }
        __threadfence();
        __syncwarp();
        int mine = 0;
        if (lane == 0) mine = atomicAdd(p.counters + tile * 4 + quad, 1) == nseg - 1;
        finalize = __shfl_sync(0xffffffffu, mine, 0) != 0;
        if (finalize) {
          __threadfence();
          if (n < N) {
            // the other contributors' slots: all tokens of a slot in flight at once
            int32_t acc[DT];
#pragma unroll
            for (int t = 0; t < DT; ++t) acc[t] = static_cast<int32_t>(c[t]);
            for (int sl = 0; sl < nseg; ++sl) {
              if (sl == slot) continue;
              const int32_t* src = p.partials + (static_cast<size_t>(sl) * DT) * N + n;
              const float* dsrc = reinterpret_cast<const float*>(p.partials + dpart) + (static_cast<size_t>(sl) * DT) * N + n;
              int32_t v[DT];
              float dv[DT];
#pragma unroll
              for (int t = 0; t < DT; ++t) {
                v[t] = t < T ? __ldcg(src + static_cast<size_t>(t) * N) : 0;
                dv[t] = (n_used > 0 && t < T) ? __ldcg(dsrc + static_cast<size_t>(t) * N) : 0.f;
              }
#pragma unroll
              for (int t = 0; t < DT; ++t) {
                acc[t] += v[t];
                d[t] += dv[t];
              }
            }
#pragma unroll
            for (int t = 0; t < DT; ++t) c[t] = static_cast<uint32_t>(acc[t]);
          }
        }
      }
      if (!finalize || n >= N) continue;
      if (raw) {
        // the exact int32 sums C[t, n], t < T (lanes write consecutive n)
#pragma unroll
        for (int t = 0; t < DT; ++t) {
          if (t >= T) break;
          p.C[static_cast<size_t>(t) * N + n] = static_cast<int32_t>(c[t]);
        }
        continue;
      }
      // dequant + bias + outlier term for (t, n), t < T
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
                                   bool pdl, cudaStream_t st) {
  // the shared-memory opt-in, once per device (calls may come from several host threads)
  static PerDeviceOnce attr_done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  cudaError_t e = cudaSuccess;
  if (!attr_done.run(dev, [&] {
        e = cudaFuncSetAttribute(k_gemm_i8_decode<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DecodeCfg<C>::SMEM_ALLOC);
        return e == cudaSuccess;
      }))
    return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(DTHREADS, 1, 1);
  cfg.dynamicSmemBytes = DecodeCfg<C>::SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_gemm_i8_decode<C>, tmW, tmC, a);
}

cudaError_t launch_gemm_decode(const CUtensorMap& tmW, const CUtensorMap& tmC, const DecodeArgs& a, int grid,
                               int boxes_per_stage, bool pdl, cudaStream_t st) {
  switch (boxes_per_stage) {
    case 2: return launch_decode_c<2>(tmW, tmC, a, grid, pdl, st);
    case 4: return launch_decode_c<4>(tmW, tmC, a, grid, pdl, st);
    default: return launch_decode_c<1>(tmW, tmC, a, grid, pdl, st);
  }
}

}  // namespace i8lt
