// Persistent, warp-specialised int8 tensor-core GEMM for sm_100a with the
// LLM.int8() dequant epilogue fused in.
//
//   C[i, n]  = sum_k CA[i, k] * CB[n, k]                       (tcgen05 kind::i8, int32 in TMEM)
//   D[i, n]  = sum_{j in O} X[i, j] * CB[n, j]                  (tcgen05 kind::f16, fp32 in TMEM)
//   out      = fp16(C * SCA[i] * SCB[n] / 127^2 + bias[n] + D * SCB[n] / 127)
//
// which is the mixed decomposition of "`bitsandbytes` - `Linear8bitLt`
// integration into `transformers` models" (section "About the mixed
// quantization method in few words") with the int8_linear_matmul and
// int8_mm_dequant ops of "LLM.int8() Refactoring: Part 1" (section
// "Deprecations") fused into one kernel.  The raw variant stores C as int32.
//
// Block = 6 warps: warp 0 issues TMA loads (one elected lane), warp 1 owns
// TMEM and issues tcgen05.mma (one lane), warps 2-5 run the epilogue (each
// warp reads the 32 TMEM lanes of its quadrant).  One CTA per SM walks tiles
// of 128 x 256 outputs; K is streamed through a 4-stage ring of
// 128-byte-deep, 128B-swizzled tiles.  The gathered fp16 outlier tiles (64
// fp16 = 128 bytes deep) reuse the same ring after the int8 k-blocks.
// TMEM: 512 columns.  Without outliers, two 256-column int32 accumulators
// alternate between tiles so the epilogue of tile t overlaps the mainloop of
// tile t+1; with outliers, columns [0,256) hold C and [256,512) hold D.
#include <cuda_fp16.h>

#include "kernels.cuh"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int BM = kGemmBM;
constexpr int BN = kGemmBN;
constexpr int BK = kGemmBKBytes;
constexpr int STAGES = 4;
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 5;
constexpr int BAR_OFF = STAGES * STAGE_BYTES;
constexpr int SCALE_OFF = BAR_OFF + ((NUM_BARS * 8 + 15) / 16) * 16;
constexpr int SCALE_BYTES_PER_WARP = 2 * BN * 4;  // SCB and bias of the current tile, per epilogue warp
constexpr int MISC_OFF = SCALE_OFF + EPI_WARPS * SCALE_BYTES_PER_WARP;
constexpr int SMEM_USED = MISC_OFF + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;  // slack to align the ring to 1024 bytes
constexpr uint32_t TMEM_COLS = 512;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(BN == 256, "accumulator layout assumes 256 columns per tile");

// Wait without an abort flag (used for the final drains, which must really
// wait for in-flight asynchronous work), still bounded by `limit_ns`.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  int never = 0;
  mbar_wait_bounded(bar, parity, &never, nullptr, limit_ns);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

template <bool RAW>
__global__ void __launch_bounds__(THREADS, 1)
    k_gemm_i8_tcgen05(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmXO, const __grid_constant__ CUtensorMap tmWO,
                      const GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int M = p.M, N = p.N, K = p.K;
  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  const int kb_int = (K + BK - 1) / BK;
  int n_used = 0;
  if (!RAW && p.n_used != nullptr) n_used = min(max(*p.n_used, 0), p.out_cap);
  const int kb_out = (n_used + 63) / 64;
  const int kb_all = kb_int + kb_out;
  const bool dbl = kb_out == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 32 * EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (kb_out > 0) {
      tma_prefetch_desc(&tmXO);
      tma_prefetch_desc(&tmWO);
    }
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0, fill_parity = 0;  // per stage: ever filled / full-barrier parity of the last fill
      for (int tile = blockIdx.x; tile < tiles && !*s_abort; tile += gridDim.x) {
        const int m0 = (tile % num_m) * BM;
        const int n0 = (tile / num_m) * BN;
        for (int kb = 0; kb < kb_all; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, p.status, p.wait_limit_ns)) break;
          uint8_t* sa = smem + stage * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          filled |= 1u << stage;
          fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
          if (kb < kb_int) {
            tma_load_2d(sa, &tmA, &full[stage], kb * BK, m0);
            tma_load_2d(sb, &tmB, &full[stage], kb * BK, n0);
          } else {
            const int ko = (kb - kb_int) * 64;  // fp16 elements
            tma_load_2d(sa, &tmXO, &full[stage], ko, m0);
            tma_load_2d(sb, &tmWO, &full[stage], ko, n0);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Never leave the CTA while a copy may still be landing in shared memory:
      // every stage this thread filled is either consumed or is waited for here.
      if (*s_abort) {
        for (int s = 0; s < STAGES; ++s)
          if (filled & (1u << s)) drain_wait(&full[s], (fill_parity >> s) & 1u, p.wait_limit_ns);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_i = idesc_i8_s32(BM, BN);
      const uint32_t idesc_f = idesc_f16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < tiles && !*s_abort; tile += gridDim.x, ++it) {
        const int buf = dbl ? (it & 1) : 0;
        const uint32_t use = dbl ? static_cast<uint32_t>(it >> 1) : static_cast<uint32_t>(it);
        if (!mbar_wait_bounded(&acc_empty[buf], (use & 1u) ^ 1u, s_abort, p.status, p.wait_limit_ns)) break;
        tc_fence_after_sync();
        const uint32_t d_int = tmem_base + static_cast<uint32_t>(buf * BN);
        const uint32_t d_fp = tmem_base + static_cast<uint32_t>(BN);
        bool ok = true;
        for (int kb = 0; kb < kb_all; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, s_abort, p.status, p.wait_limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t a_addr = smem_addr(smem + stage * STAGE_BYTES);
          const uint64_t adesc = smem_desc_k_sw128(a_addr);
          const uint64_t bdesc = smem_desc_k_sw128(a_addr + A_BYTES);
          if (kb < kb_int) {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)  // 32 int8 = 32 bytes per MMA
              mma_i8(d_int, adesc + 2 * k, bdesc + 2 * k, idesc_i, (kb > 0 || k > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int k = 0; k < BK / 32; ++k)  // 16 fp16 = 32 bytes per MMA
              mma_f16(d_fp, adesc + 2 * k, bdesc + 2 * k, idesc_f, (kb > kb_int || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
      // Wait for every MMA this thread issued before TMEM is released.
      tc_commit(mma_done);
      drain_wait(mma_done, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;                  // TMEM lanes this warp may read
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const bool vec_ok = RAW ? ((N & 3) == 0) : ((N & 7) == 0);
    // Each epilogue warp keeps its own copy of the tile's column scales and
    // bias, so the four warps never wait on one another.
    float* s_scb = reinterpret_cast<float*>(smem + SCALE_OFF + (warp - 2) * SCALE_BYTES_PER_WARP);
    float* s_bias = s_scb + BN;
    int it = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++it) {  // abort is seen by the wait below
      const int m0 = (tile % num_m) * BM;
      const int n0 = (tile / num_m) * BN;
      if (!RAW) {
        __syncwarp();  // every lane is done with the previous tile's copy
        for (int c = lane; c < BN; c += 32) {
          const int n = n0 + c;
          s_scb[c] = n < N ? p.SCB[n] : 0.f;
          s_bias[c] = (p.bias != nullptr && n < N) ? __half2float(p.bias[n]) : 0.f;
        }
        __syncwarp();
      }
      const int buf = dbl ? (it & 1) : 0;
      const uint32_t use = dbl ? static_cast<uint32_t>(it >> 1) : static_cast<uint32_t>(it);
      // lane 0 waits for the whole warp, so the warp leaves the loop as one
      // (the TMEM loads below are warp-collective)
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&acc_full[buf], use & 1u, s_abort, p.status, p.wait_limit_ns) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after_sync();
      const int row = m0 + quad * 32 + lane;
      const bool row_ok = row < M;
      const float sa = (!RAW && row_ok) ? p.SCA[row] * (1.0f / 16129.0f) : 0.f;
      const uint32_t t_int = tmem_base + lane_off + static_cast<uint32_t>(buf * BN);
      const uint32_t t_fp = tmem_base + lane_off + static_cast<uint32_t>(BN);
#pragma unroll 1
      for (int cc = 0; cc < BN / 32; ++cc) {
        uint32_t ri[32];
        tmem_ld_32x32b_x32(t_int + cc * 32, ri);
        uint32_t rf[32];
        if (!RAW && kb_out > 0) tmem_ld_32x32b_x32(t_fp + cc * 32, rf);
        tmem_wait_ld();
        const int nb = n0 + cc * 32;
        if (!row_ok || nb >= N) continue;
        if (RAW) {
          int32_t* dst = p.C + static_cast<size_t>(row) * N + nb;
          if (vec_ok && nb + 32 <= N) {
#pragma unroll
            for (int q = 0; q < 8; ++q)
              reinterpret_cast<uint4*>(dst)[q] = make_uint4(ri[4 * q], ri[4 * q + 1], ri[4 * q + 2], ri[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < N) dst[j] = static_cast<int32_t>(ri[j]);
          }
        } else {
          float y[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float sb = s_scb[cc * 32 + j];
            float v = fmaf(static_cast<float>(static_cast<int32_t>(ri[j])), sa * sb, s_bias[cc * 32 + j]);
            if (kb_out > 0) v = fmaf(__uint_as_float(rf[j]), sb * (1.0f / 127.0f), v);
            y[j] = v;
          }
          __half* dst = p.out + static_cast<size_t>(row) * N + nb;
          if (vec_ok && nb + 32 <= N) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              reinterpret_cast<uint4*>(dst)[q] =
                  make_uint4(pack_half2(y[8 * q], y[8 * q + 1]), pack_half2(y[8 * q + 2], y[8 * q + 3]),
                             pack_half2(y[8 * q + 4], y[8 * q + 5]), pack_half2(y[8 * q + 6], y[8 * q + 7]));
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < N) dst[j] = __float2half_rn(y[j]);
          }
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&acc_empty[buf]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

cudaError_t launch_gemm(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmXO,
                        const CUtensorMap& tmWO, const GemmArgs& a, bool raw_int32, int num_sms, cudaStream_t st) {
  static bool attr_done[2] = {false, false};
  const int tiles = ((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  if (raw_int32) {
    if (!attr_done[1]) {
      cudaError_t e = cudaFuncSetAttribute(k_gemm_i8_tcgen05<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           SMEM_ALLOC);
      if (e != cudaSuccess) return e;
      attr_done[1] = true;
    }
    k_gemm_i8_tcgen05<true><<<grid, THREADS, SMEM_ALLOC, st>>>(tmA, tmB, tmXO, tmWO, a);
  } else {
    if (!attr_done[0]) {
      cudaError_t e = cudaFuncSetAttribute(k_gemm_i8_tcgen05<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           SMEM_ALLOC);
      if (e != cudaSuccess) return e;
      attr_done[0] = true;
    }
    k_gemm_i8_tcgen05<false><<<grid, THREADS, SMEM_ALLOC, st>>>(tmA, tmB, tmXO, tmWO, a);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------ self test
// One block waits on a barrier that nothing ever completes, through the same
// bounded wait the GEMM pipeline uses; it must give up and report a timeout.
__global__ void k_selftest_wait(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool done = mbar_wait_bounded(&bar, 0, &abort_flag, status, limit_ns);
    if (done) atomicExch(status, 0xFFFFFFFFu);  // impossible: nothing arrives
  }
  __syncthreads();
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t st) {
  k_selftest_wait<<<1, 32, 0, st>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace i8lt
