// Persistent, warp-specialised int8 tensor-core GEMM for sm_100a with the
// LLM.int8() dequant epilogue fused in.
//
//   C[i, n]  = sum_k CA[i, k] * CB[n, k]                       (tcgen05 kind::i8, int32 in TMEM)
//   D[i, n]  = sum_{j in O} X[i, j] * CB[n, j]                  (warp MMAs, or tcgen05 kind::f16)
//   out      = fp16(C * SCA[i] * SCB[n] / 127^2 + bias[n] + D * SCB[n] / 127)
//
// which is the mixed decomposition of "`bitsandbytes` - `Linear8bitLt`
// integration into `transformers` models" (section "About the mixed
// quantization method in few words") with the int8_linear_matmul and
// int8_mm_dequant ops of "LLM.int8() Refactoring: Part 1" (section
// "Deprecations") fused into one kernel.  The raw variant stores C as int32.
//
// The kernel runs on CTA pairs (clusters of 2, tcgen05 cta_group::2): a pair
// computes 256 x 256 output tiles; each CTA loads its own 128 rows of A and its
// own 128 rows of B into its shared memory (plain TMA loads, no multicast) and
// the leader CTA issues one M=256 MMA over both halves.  Each CTA's TMEM holds
// the accumulator rows of its half.
//
// Tiles are handed to pairs round-robin; when the last round would leave
// more than half of the pairs idle, its tiles are split into 256 x 128 halves
// (MMA N = 128), so that round takes about half the time of a full one.
//
// Block = 10 warps: warp 0 issues TMA loads (one lane), warp 1 owns TMEM and,
// in the leader, issues tcgen05.mma (one lane); warps 2-9 run the epilogue
// (two warps per 32-lane TMEM quadrant, one per 128-column half).  K streams
// through a 6-stage ring of 128-byte-deep, 128B-swizzled tiles; the gathered
// fp16 outlier tiles (64 fp16 = 128 bytes deep) use the same ring.  TMEM: 512
// columns.  Two 256-column accumulators alternate so the epilogue of tile t
// overlaps the mainloop of tile t+1.  Up to 16 outlier columns, the epilogue
// adds the (rank <= 16) outlier product itself with warp-level MMAs
// (mma.sync m16n8k16) on the gathered operands.  With more, the epilogue
// first rewrites tile t's int32 accumulator in place as fp32 C * SCA / 127
// (tcgen05.ld, convert, tcgen05.st) and the MMA thread adds tcgen05 kind::f16
// MMAs of the outlier tiles on top of it; it issues them a few k-blocks into
// tile t+1's mainloop, so the tensor pipe does not wait for the conversion.
// The epilogue then scales by SCB / 127 and adds the bias.
// The epilogue writes fp16 32x32 boxes through shared memory with TMA stores.
//
// A third mode runs the same pipeline as a plain fp16 GEMM, out = fp16(XO . WO^T)
// with fp32 accumulation: every k-block is a kind::f16 block, the accumulator
// is double-buffered in TMEM and the epilogue only rounds.  It computes the
// input gradient dX = dY . W^ of a linear layer whose frozen weight W^ is the
// dequantised int8 weight, with XO = dY [M, N] and WO = W^ transposed [K, N].
#include <cuda_fp16.h>

#include <atomic>
#include <type_traits>

#include "kernels.cuh"
#include "per_device.h"
#include "ptx.cuh"

namespace i8lt {

namespace {

constexpr int BM = kGemmBM;          // rows per CTA
constexpr int BN = kGemmBN;          // columns per pair tile
constexpr int BNH = BN / 2;          // B rows per CTA
constexpr int BK = kGemmBKBytes;
constexpr int STAGES = 6;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BNH * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
constexpr int OBOX = kGemmOutBox;                // 32 x 32 fp16 output box
constexpr int STG_BYTES = OBOX * OBOX * 2;       // 2 KB
constexpr int STG_OFF = RING_BYTES;
constexpr int STG_TOTAL = EPI_WARPS * 2 * STG_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 9;
constexpr int BAR_OFF = STG_OFF + STG_TOTAL;
constexpr int MISC_OFF = BAR_OFF + ((NUM_BARS * 8 + 15) / 16) * 16;
constexpr int SMEM_USED = MISC_OFF + 16;
constexpr int SMEM_ALLOC = SMEM_USED + 1024;  // slack to align the ring to 1024 bytes
constexpr uint32_t TMEM_COLS = 512;
constexpr int CHUNKS = BNH / 32;              // 32-column chunks per epilogue warp
constexpr int SMALL_O = kSmallOutliers;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(SMALL_O == 16, "the epilogue's warp MMA covers one k-step of 16 outlier columns");

// Wait without an abort flag (used for the final drains, which must really
// wait for in-flight asynchronous work), still bounded by `limit_ns`.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  int never = 0;
  mbar_wait_bounded(bar, parity, &never, nullptr, limit_ns);
}

// Work units of a pair: tiles [0, full_units) are whole 256 x 256 tiles; past
// them each remaining tile is cut into two 256 x 128 halves, so a last wave
// that would keep at most half of the pairs busy takes half as long (and a
// grid with fewer tiles than half the pairs runs twice as many CTAs).
struct Units {
  int full_units, units;
  __device__ Units(int tiles, int npairs) {
    const int waves = tiles / npairs, rem = tiles - waves * npairs;
    const bool split = rem > 0 && 2 * rem <= npairs;
    full_units = split ? waves * npairs : tiles;
    units = split ? full_units + 2 * rem : tiles;
  }
  // tile of unit u and which column half of it (-1: the whole tile)
  __device__ void at(int u, int& tile, int& half) const {
    if (u < full_units) {
      tile = u;
      half = -1;
    } else {
      tile = full_units + ((u - full_units) >> 1);
      half = (u - full_units) & 1;
    }
  }
};

// Tile order: bands of kRasterRows tile rows (256 rows of A each); inside a
// band the rows of one tile column come first, then the next column.  B is
// read once per band and A once in all, so the band is as tall as possible
// while its rows of A stay in L2 (16 tile rows = 4096 rows, 16.8 MB at
// K = 4096): up to 4096 rows that is plain column order, where the weight is
// read once (bands of 8 read the gate / up weights twice: 108.7 against 64.4 MB
// of DRAM per launch, at the same speed).
constexpr int kRasterRows = 16;
__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& tm, int& tn) {
  const int band = tile / (kRasterRows * num_n);
  const int r = tile - band * kRasterRows * num_n;
  const int rows = min(kRasterRows, num_m - band * kRasterRows);  // the last band may be shorter
  tn = r / rows;
  tm = band * kRasterRows + (r - tn * rows);
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    k_gemm_i8_tcgen05(const __grid_constant__ GemmMaps tm, const GemmArgs p) {
  constexpr bool RAW = MODE == kGemmRaw;
  constexpr bool F16 = MODE == kGemmF16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + BAR_OFF);  // used in the leader only
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2], used in the leader only
  uint64_t* mma_done = acc_empty + 2;
  uint64_t* conv_done = mma_done + 1;   // [2], leader only: accumulator converted to fp32 by the epilogue
  uint64_t* acc_full2 = conv_done + 2;  // [2]: the outlier MMAs on top of it have completed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* s_abort = reinterpret_cast<volatile int*>(s_tmem + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int M = p.M, N = p.N, K = p.K;
  const int num_m = (M + 2 * BM - 1) / (2 * BM);
  const int num_n = (N + BN - 1) / BN;
  const int tiles = num_m * num_n;
  const int kb_int = F16 ? 0 : (K + BK - 1) / BK;
  const Units U(tiles, npairs);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // the leader's expect-tx arrival; the bytes of both CTAs complete it
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&conv_done[b], 2 * EPI_WARPS);
      mbar_init(&acc_full2[b], 1);
    }
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    if constexpr (F16) {
      tma_prefetch_desc(&tm.XO);
      tma_prefetch_desc(&tm.WO);
    } else {
      tma_prefetch_desc(&tm.A);
      tma_prefetch_desc(&tm.B);
    }
    if (!RAW && p.tma_store) tma_prefetch_desc(&tm.Out);
  }
  if (warp == 1) {
    tmem_alloc_pair(s_tmem, TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync();  // barriers initialised and TMEM allocated in both CTAs of the pair
  tc_fence_after_sync();
  const uint32_t tmem_base = *s_tmem;

  // The kernel may be launched while the kernel before it (the outlier
  // preparation) still runs: everything below reads what that kernel and the
  // quantiser wrote, so wait for them here (a no-op without that overlap).
  pdl_wait();
  int n_used = 0;
  if (!RAW && !F16 && p.n_used != nullptr) n_used = min(max(*p.n_used, 0), p.out_cap);
  // Up to 16 outlier columns are added by the epilogue with warp MMAs.  More
  // go through tcgen05 fp16 MMAs accumulated on top of the tile's int8 result:
  // the epilogue first turns the int32 accumulator into fp32 C * SCA / 127 in
  // place, then the MMA thread adds X[:, O] . CB[:, O]^T into the same TMEM
  // columns (its k-blocks are issued a few k-blocks into the next tile's
  // mainloop, by when the conversion is normally done), and the epilogue
  // scales by SCB / 127.  Both ways keep the two accumulators double-buffered.
  // The fp16 mode has only fp16 k-blocks (K fp16 columns).
  const bool small_o = !F16 && n_used > 0 && n_used <= SMALL_O && p.XO != nullptr && p.WO != nullptr;
  const int kb_out = F16 ? (K + 63) / 64 : (small_o ? 0 : (n_used + 63) / 64);
  const bool defer = !F16 && !RAW && kb_out > 0;  // outlier k-blocks issued after the tile's int8 ones
  const int kb_main = F16 ? kb_out : kb_int;      // k-blocks of a unit's own mainloop
  const int j_ins = min(4, kb_main - 1);          // a unit's k-block before which the previous
                                                  // unit's outlier k-blocks are issued

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full0_leader = map_to_rank(smem_addr(&full[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t filled = 0, fill_parity = 0;  // leader: per stage, ever filled / parity of the last fill
      // one stage: k-block x of map pair (ma, mb) at rows (m0, nb0); false on abort
      auto load_stage = [&](const CUtensorMap* ma, const CUtensorMap* mb, int x, int m0, int nb0) -> bool {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, p.status, p.wait_limit_ns)) return false;
        uint8_t* sa = smem + stage * STAGE_BYTES;
        uint8_t* sb = sa + A_BYTES;
        const uint32_t bar = full0_leader + static_cast<uint32_t>(stage) * 8u;
        if (leader) {
          // one arrival that expects the bytes of both CTAs.  The peer's copies
          // may land first (the transaction count goes negative meanwhile); the
          // phase cannot complete before this arrival, and the peer cannot
          // refill the stage before the MMA has consumed it.
          mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
          filled |= 1u << stage;
          fill_parity = (fill_parity & ~(1u << stage)) | (phase << stage);
        }
        tma_load_2d_pair(sa, ma, bar, x, m0);
        tma_load_2d_pair(sb, mb, bar, x, nb0);
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      // the outlier k-blocks (64 fp16 = 128 bytes deep) of a unit
      auto load_outliers = [&](int m0, int nb0) -> bool {
        for (int ko = 0; ko < kb_out; ++ko)
          if (!load_stage(&tm.XO, &tm.WO, ko * 64, m0, nb0)) return false;
        return true;
      };
      bool ok = true, have_prev = false;
      int prev_m0 = 0, prev_nb0 = 0;
      for (int u = pair; ok && u < U.units && !*s_abort; u += npairs) {
        int tile, half;
        U.at(u, tile, half);
        int tmi, tni;
        tile_coords(tile, num_m, num_n, tmi, tni);
        const int m0 = tmi * (2 * BM) + static_cast<int>(rank) * BM;
        // a half tile's 128 columns come as 64 B rows per CTA (the box still
        // carries 128 rows; the MMA reads the first 64)
        const int nb0 = tni * BN +
                        (half < 0 ? static_cast<int>(rank) * BNH : half * BNH + static_cast<int>(rank) * (BNH / 2));
        for (int kb = 0; ok && kb < kb_main; ++kb) {
          if (defer && have_prev && kb == j_ins) ok = load_outliers(prev_m0, prev_nb0);
          if (ok) ok = F16 ? load_stage(&tm.XO, &tm.WO, kb * 64, m0, nb0) : load_stage(&tm.A, &tm.B, kb * BK, m0, nb0);
        }
        prev_m0 = m0;
        prev_nb0 = nb0;
        have_prev = true;
      }
      if (ok && defer && have_prev && !*s_abort) load_outliers(prev_m0, prev_nb0);
      // Never leave while a copy may still be landing in shared memory.  The
      // leader's full barriers count both CTAs' bytes; the peer, which cannot
      // observe them, gives its last copies a bounded grace period.
      if (*s_abort) {
        if (leader) {
          for (int s = 0; s < STAGES; ++s)
            if (filled & (1u << s)) drain_wait(&full[s], (fill_parity >> s) & 1u, p.wait_limit_ns);
        } else {
          const uint64_t t0 = global_timer_ns();
          while (global_timer_ns() - t0 < 200000ull) __nanosleep(1000);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      // one stage: 4 MMAs (32 bytes of K each) into accumulator d; false on abort
      auto mma_stage = [&](uint32_t d, uint32_t idesc, bool f16_block, bool acc0) -> bool {
        if (!mbar_wait_bounded(&full[stage], phase, s_abort, p.status, p.wait_limit_ns)) return false;
        tc_fence_after_sync();
        const uint32_t a_addr = smem_addr(smem + stage * STAGE_BYTES);
        const uint64_t adesc = smem_desc_k_sw128(a_addr);
        const uint64_t bdesc = smem_desc_k_sw128(a_addr + A_BYTES);
        if (f16_block) {
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)  // 16 fp16 = 32 bytes per MMA
            mma_f16_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, (acc0 || k > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int k = 0; k < BK / 32; ++k)  // 32 int8 = 32 bytes per MMA
            mma_i8_pair(d, adesc + 2 * k, bdesc + 2 * k, idesc, (acc0 || k > 0) ? 1u : 0u);
        }
        tc_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      // the outlier k-blocks of an earlier unit, added on top of its converted
      // accumulator (fp32 C * SCA / 127 written back by the epilogue)
      auto outlier_mmas = [&](int b, int nt_b, uint32_t use_b) -> bool {
        if (!mbar_wait_bounded(&conv_done[b], use_b & 1u, s_abort, p.status, p.wait_limit_ns)) return false;
        tc_fence_after_sync();
        const uint32_t idesc_f = idesc_f16_f32(2 * BM, nt_b);
        for (int ko = 0; ko < kb_out; ++ko)
          if (!mma_stage(tmem_base + static_cast<uint32_t>(b * BN), idesc_f, true, true)) return false;
        tc_commit_pair(&acc_full2[b], 0x3);
        return true;
      };
      int it = 0, prev_buf = 0, prev_nt = BN;
      uint32_t prev_use = 0;
      bool ok = true;
      for (int u = pair; ok && u < U.units && !*s_abort; u += npairs, ++it) {
        int tile, half;
        U.at(u, tile, half);
        const int nt = half < 0 ? BN : BNH;
        const uint32_t idesc = F16 ? idesc_f16_f32(2 * BM, nt) : idesc_i8_s32(2 * BM, nt);
        const int buf = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait_bounded(&acc_empty[buf], (use & 1u) ^ 1u, s_abort, p.status, p.wait_limit_ns)) break;
        tc_fence_after_sync();
        const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
        for (int kb = 0; ok && kb < kb_main; ++kb) {
          if (defer && it > 0 && kb == j_ins) ok = outlier_mmas(prev_buf, prev_nt, prev_use);
          if (ok) ok = mma_stage(d, idesc, F16, kb > 0);
        }
        if (!ok) break;
        tc_commit_pair(&acc_full[buf], 0x3);  // both CTAs' accumulator halves are ready
        prev_buf = buf;
        prev_nt = nt;
        prev_use = use;
      }
      if (ok && defer && it > 0 && !*s_abort) outlier_mmas(prev_buf, prev_nt, prev_use);
      // Wait for every MMA this thread issued before TMEM is released.
      tc_commit_pair(mma_done, 0x1);
      drain_wait(mma_done, 0, p.wait_limit_ns);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    // Each warp owns 32 accumulator rows (its TMEM lane quadrant) and 128 of
    // the tile's 256 columns, processed as four 32x32 chunks.  TMEM is read in
    // the mma.m16n8 accumulator layout (thread t: rows t/4 and t/4+8 of each
    // 16-row block, columns 2(t%4), 2(t%4)+1 of each 8-column block), so the
    // few-outlier product can be added with warp MMAs in the same layout.
    const int ew = warp - 2;                    // 0..7
    const int quad = warp & 3;                  // TMEM lanes this warp may read
    const int col_half = ew >> 2;               // which 128 of the tile's 256 columns
    const int g = lane >> 2, tq = lane & 3;     // fragment row / column pair
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t acc_empty0_leader = map_to_rank(smem_addr(&acc_empty[0]), 0);
    const uint32_t conv_done0_leader = map_to_rank(smem_addr(&conv_done[0]), 0);
    uint8_t* stg = smem + STG_OFF + ew * 2 * STG_BYTES;
    int stg_i = 0;
    int it = 0;
    auto run_units = [&](auto defer_tag) {
    constexpr bool DEFER = decltype(defer_tag)::value;  // the value of `defer`, as a constant
    for (int u = pair; u < U.units; u += npairs, ++it) {  // abort is seen by the wait below
      int tile, half;
      U.at(u, tile, half);
      int tmi, tni;
      tile_coords(tile, num_m, num_n, tmi, tni);
      const int row_base = tmi * (2 * BM) + static_cast<int>(rank) * BM + quad * 32;
      // whole tile: 128 columns (4 chunks) per warp; half tile: 64 (2 chunks)
      const int nch = half < 0 ? CHUNKS : CHUNKS / 2;
      const int col_off = col_half * nch * 32;  // TMEM column of this warp's first chunk
      const int n0 = tni * BN + (half < 0 ? 0 : half * BNH) + col_off;
      const int buf = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      // The chunk loop below is deliberately not unrolled: the epilogue runs
      // beside the TMA and MMA warps, and a compact loop keeps their
      // instructions resident in the instruction cache.  Data a chunk needs
      // besides its accumulators is fetched one chunk ahead (the first chunk's
      // before the accumulator wait).
      // Row scales of this thread's four rows: row_base + g + 8i (SCA / 127^2,
      // or SCA / 127 when the outlier MMAs are added on top of the converted
      // accumulator).
      float sa4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = row_base + g + 8 * i;
        sa4[i] = (!RAW && !F16 && r < M) ? __ldg(p.SCA + r) * (DEFER ? (1.0f / 127.0f) : (1.0f / 16129.0f)) : 0.f;
      }
      // Few outliers: the A fragments (X[:, O] rows) of the 16-wide outlier
      // product.  The gathered operands store each group of 16 outlier columns
      // in the order (0 1 8 9)(2 3 10 11)(4 5 12 13)(6 7 14 15): the four
      // values a thread needs from a row (columns 2tq, 2tq+1, 2tq+8, 2tq+9)
      // are one 8-byte load.
      uint32_t af[2][4];
#pragma unroll
      for (int rb = 0; rb < 2; ++rb)
#pragma unroll
        for (int e = 0; e < 4; ++e) af[rb][e] = 0u;
      if (small_o) {
#pragma unroll
        for (int rb = 0; rb < 2; ++rb) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int r = row_base + rb * 16 + g + 8 * hh;
            if (r < M) {
              const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.XO + static_cast<size_t>(r) * p.ld_o + 4 * tq));
              af[rb][hh] = v.x;
              af[rb][2 + hh] = v.y;
            }
          }
        }
      }
      // Per chunk: column scale and bias (lane j holds column nb + j) and the
      // B fragments (CB[:, O] of the chunk's 32 columns).
      float sb_n = 0.f, bi_n = 0.f;
      uint32_t bf_n[4][2];
      auto fetch_chunk = [&](int cc) {
        const int n = n0 + cc * 32 + lane;
        const bool in = !RAW && !F16 && n < N;
        sb_n = in ? __ldg(p.SCB + n) : 0.f;
        bi_n = (in && p.bias != nullptr) ? __half2float(p.bias[n]) : 0.f;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          bf_n[cb][0] = bf_n[cb][1] = 0u;
          const int nf = n0 + cc * 32 + cb * 8 + g;
          if (small_o && nf < N) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.WO + static_cast<size_t>(nf) * p.ld_o + 4 * tq));
            bf_n[cb][0] = v.x;
            bf_n[cb][1] = v.y;
          }
        }
      };
      fetch_chunk(0);
      // lane 0 waits for the whole warp, so the warp leaves the loop as one
      // (the TMEM loads below are warp-collective)
      int ok = 0;
      if (lane == 0) ok = mbar_wait_bounded(&acc_full[buf], use & 1u, s_abort, p.status, p.wait_limit_ns) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after_sync();
      const uint32_t t_int = tmem_base + lane_off + static_cast<uint32_t>(buf * BN + col_off);
      if constexpr (DEFER) {
        // Many outlier columns, phase 1: the int32 accumulator becomes fp32
        // C * SCA / 127 in place; the MMA thread then adds the outlier product
        // onto it (fragment element e of row block rb is row rb*16 + g + 8*((e >> 1) & 1)).
#pragma unroll 1
        for (int cc = 0; cc < nch; ++cc) {
          uint32_t c[2][16];
          tmem_ld_16x256b_x4(t_int + cc * 32, c[0]);
          tmem_ld_16x256b_x4(t_int + (16u << 16) + cc * 32, c[1]);
          tmem_wait_ld();
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
#pragma unroll
            for (int e = 0; e < 16; ++e)
              c[rb][e] = __float_as_uint(static_cast<float>(static_cast<int32_t>(c[rb][e])) * sa4[2 * rb + ((e >> 1) & 1)]);
          tmem_st_16x256b_x4(t_int + cc * 32, c[0]);
          tmem_st_16x256b_x4(t_int + (16u << 16) + cc * 32, c[1]);
        }
        tmem_wait_st();
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(conv_done0_leader + static_cast<uint32_t>(buf) * 8u);
        // phase 2: wait until the outlier MMAs of this tile have completed
        ok = 0;
        if (lane == 0) ok = mbar_wait_bounded(&acc_full2[buf], use & 1u, s_abort, p.status, p.wait_limit_ns) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        tc_fence_after_sync();
      }
#pragma unroll 1
      for (int cc = 0; cc < nch; ++cc) {
        [[maybe_unused]] const float sb_c = sb_n, bi_c = bi_n;  // unused by the raw and fp16 modes
        uint32_t bf_c[4][2];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          bf_c[cb][0] = bf_n[cb][0];
          bf_c[cb][1] = bf_n[cb][1];
        }
        if (cc + 1 < nch) fetch_chunk(cc + 1);
        uint32_t c[2][16];  // int32 accumulators of row blocks 0 / 1
        if (!F16 && !DEFER) {
          tmem_ld_16x256b_x4(t_int + cc * 32, c[0]);
          tmem_ld_16x256b_x4(t_int + (16u << 16) + cc * 32, c[1]);
        }
        // fp32 accumulators: C * SCA / 127 plus the outlier product (many-outlier
        // path) or, in the fp16 mode, the whole product
        uint32_t f[2][16];
        if (F16 || DEFER) {
          tmem_ld_16x256b_x4(t_int + cc * 32, f[0]);
          tmem_ld_16x256b_x4(t_int + (16u << 16) + cc * 32, f[1]);
        }
        tmem_wait_ld();
        const int nb = n0 + cc * 32;
        if constexpr (RAW) {
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
#pragma unroll
            for (int cb = 0; cb < 4; ++cb)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const int r = row_base + rb * 16 + g + 8 * hh;
                const int n = nb + cb * 8 + 2 * tq;
                if (r >= M || n >= N) continue;
                int32_t* dst = p.C + static_cast<size_t>(r) * N + n;
                const uint32_t v0 = c[rb][4 * cb + 2 * hh], v1 = c[rb][4 * cb + 2 * hh + 1];
                if ((N & 1) == 0 && n + 1 < N) {
                  *reinterpret_cast<int2*>(dst) = make_int2(static_cast<int>(v0), static_cast<int>(v1));
                } else {
                  dst[0] = static_cast<int32_t>(v0);
                  if (n + 1 < N) dst[1] = static_cast<int32_t>(v1);
                }
              }
        } else {
        // dequant in fragment layout; halves[rb][cb][hh] = (row rb*16+g+8hh, columns cb*8+2tq, +1)
        uint32_t halves[2][4][2];
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
          [[maybe_unused]] const int j = cb * 8 + 2 * tq;
          [[maybe_unused]] float sb0 = 0.f, sb1 = 0.f, b0 = 0.f, b1 = 0.f;  // stay 0 in the fp16 mode
          if constexpr (!F16) {
            sb0 = __shfl_sync(0xffffffffu, sb_c, j);
            sb1 = __shfl_sync(0xffffffffu, sb_c, j + 1);
            b0 = __shfl_sync(0xffffffffu, bi_c, j);
            b1 = __shfl_sync(0xffffffffu, bi_c, j + 1);
          }
#pragma unroll
          for (int rb = 0; rb < 2; ++rb) {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            if (small_o) {
              mma_16x8x16_f16(d, af[rb], bf_c[cb][0], bf_c[cb][1]);
            } else if (F16 || DEFER) {
#pragma unroll
              for (int e = 0; e < 4; ++e) d[e] = __uint_as_float(f[rb][4 * cb + e]);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              if constexpr (F16) {
                halves[rb][cb][hh] = pack_half2(d[2 * hh], d[2 * hh + 1]);
              } else if constexpr (DEFER) {
                // (C * SCA / 127 + outlier product) * SCB / 127 + bias
                halves[rb][cb][hh] = pack_half2(fmaf(d[2 * hh], sb0 * (1.0f / 127.0f), b0),
                                                fmaf(d[2 * hh + 1], sb1 * (1.0f / 127.0f), b1));
              } else {
                const float sa = sa4[2 * rb + hh];
                const float v0 = fmaf(d[2 * hh], sb0 * (1.0f / 127.0f),
                                      fmaf(static_cast<float>(static_cast<int32_t>(c[rb][4 * cb + 2 * hh])), sa * sb0, b0));
                const float v1 = fmaf(d[2 * hh + 1], sb1 * (1.0f / 127.0f),
                                      fmaf(static_cast<float>(static_cast<int32_t>(c[rb][4 * cb + 2 * hh + 1])), sa * sb1, b1));
                halves[rb][cb][hh] = pack_half2(v0, v1);
              }
            }
          }
        }
        if (p.tma_store) {
          // 32 rows x 32 fp16 box through shared memory with the 64-byte
          // swizzle: 16-byte chunk q of row r sits at chunk q ^ ((r >> 1) & 3)
          uint8_t* box = stg + stg_i * STG_BYTES;
          if (lane == 0) tma_store_wait_read<1>();  // the store that last read this buffer is done
          __syncwarp();
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              // the four 8x8 blocks of rows rb*16 + 8hh .. +7 (one per cb), in the
              // fragment layout; lane l gives the address of row l % 8 of block l / 8
              const int blk = lane >> 3, rr = rb * 16 + 8 * hh + (lane & 7);
              stmatrix_x4(smem_addr(box + rr * 64 + ((blk ^ ((rr >> 1) & 3)) << 4)), halves[rb][0][hh],
                          halves[rb][1][hh], halves[rb][2][hh], halves[rb][3][hh]);
            }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) {
            if (nb < N && row_base < M) tma_store_2d(&tm.Out, box, nb, row_base);
            tma_store_commit();
          }
          stg_i ^= 1;
        } else {
#pragma unroll
          for (int rb = 0; rb < 2; ++rb)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
              for (int cb = 0; cb < 4; ++cb) {
                const int r = row_base + rb * 16 + g + 8 * hh;
                const int n = nb + cb * 8 + 2 * tq;
                if (r >= M || n >= N) continue;
                __half* dst = p.out + static_cast<size_t>(r) * N + n;
                const uint32_t hv = halves[rb][cb][hh];
                if ((N & 1) == 0 && n + 1 < N) {
                  *reinterpret_cast<uint32_t*>(dst) = hv;
                } else {
                  dst[0] = reinterpret_cast<const __half*>(&hv)[0];
                  if (n + 1 < N) dst[1] = reinterpret_cast<const __half*>(&hv)[1];
                }
              }
        }
        }  // RAW / fused
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0_leader + static_cast<uint32_t>(buf) * 8u);
    }
    };
    // one instruction stream per way of adding many outlier columns, so the
    // common path carries no per-element test of it
    if (defer)
      run_units(std::true_type{});
    else
      run_units(std::false_type{});
    if (!RAW && p.tma_store && lane == 0) tma_store_wait_all<0>();
    __syncwarp();
  }

  tc_fence_before_sync();
  cluster_sync();  // no CTA leaves while its pair may still read its shared memory or signal its barriers
  if (warp == 1) {
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

using GemmKernel = void (*)(GemmMaps, GemmArgs);

static GemmKernel gemm_kernel(GemmMode mode) {
  switch (mode) {
    case kGemmRaw: return k_gemm_i8_tcgen05<kGemmRaw>;
    case kGemmF16: return k_gemm_i8_tcgen05<kGemmF16>;
    default: return k_gemm_i8_tcgen05<kGemmFused>;
  }
}

// Number of CTA pairs that fit on the device at once (cached per mode and
// device; calls may come from several host threads, so the cache is atomic).
static int max_pairs(GemmMode mode, int num_sms) {
  static PerDeviceInt cache[3];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  return cache[static_cast<int>(mode)].get(dev, [mode, num_sms] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(num_sms & ~1), 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = SMEM_ALLOC;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&n, gemm_kernel(mode), &cfg);
    if (e != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    return n;
  });
}

cudaError_t launch_gemm(const GemmMaps& maps, const GemmArgs& a, GemmMode mode, int num_sms, cudaStream_t st) {
  if (mode != kGemmFused && mode != kGemmRaw && mode != kGemmF16) return cudaErrorInvalidValue;
  // the shared-memory opt-in is a per-device property of the kernel: done once
  // per mode and device (several host threads may get here at once; setting it
  // twice is harmless)
  static PerDeviceOnce attr_done[3];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  cudaError_t e = cudaSuccess;
  if (!attr_done[static_cast<int>(mode)].run(dev, [&] {
        e = cudaFuncSetAttribute(gemm_kernel(mode), cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC);
        return e == cudaSuccess;
      }))
    return e;
  const int tiles = ((a.M + 2 * BM - 1) / (2 * BM)) * ((a.N + BN - 1) / BN);
  const int pairs_fit = max_pairs(mode, num_sms);
  // fewer tiles than pairs: run each tile as two half tiles where that fits
  const int pairs = tiles >= pairs_fit ? pairs_fit : (2 * tiles <= pairs_fit ? 2 * tiles : tiles);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(THREADS, 1, 1);
  cfg.dynamicSmemBytes = SMEM_ALLOC;
  cfg.stream = st;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel(mode), maps, a);
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
