// Host-side launchers of the library's kernels (all enqueue on the given stream).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace i8lt {

// bitmap: zeroed outlier bitmap to OR into (required when tau > 0).
cudaError_t launch_quant_rows(const __half* X, int M, int K, float tau, int8_t* CA, float* SCA, uint32_t* bitmap,
                              cudaStream_t st);
cudaError_t launch_zero_outlier_cols(const uint32_t* bitmap, int M, int K, int8_t* CA, int num_sms,
                                     cudaStream_t st);
cudaError_t launch_outlier_prepare(const uint32_t* bitmap, int K, int cap, int32_t* total_out, int32_t* used_out,
                                   int32_t* idx_out, uint32_t* status, int8_t* CA, const __half* X, int M,
                                   __half* XO, const int8_t* CB, int N, __half* WO, int ld_o, int num_sms,
                                   cudaStream_t st);
cudaError_t launch_mm_dequant(const int32_t* C, const float* SCA, const float* SCB, const __half* bias, int M,
                              int N, __half* out, int num_sms, cudaStream_t st);
cudaError_t launch_dequant(const int8_t* CB, const float* SCB, int N, int K, __half* W, int num_sms,
                           cudaStream_t st);
// Wt [K, N] = the transpose of launch_dequant's W (K % 16 == 0, N % 8 == 0).
cudaError_t launch_dequant_t(const int8_t* CB, const float* SCB, int N, int K, __half* Wt, cudaStream_t st);
// out [M, P*Np] from P rank-major column blocks G [P, M, Np].
cudaError_t launch_gather_column_blocks(const __half* G, int P, int M, int Np, __half* out, int num_sms,
                                        cudaStream_t st);

// Tensor-core GEMM (tcgen05, TMA-fed, TMEM accumulators).
struct GemmArgs {
  int M, N, K;
  const float* SCA;        // [M]   (fused mode)
  const float* SCB;        // [N]   (fused mode)
  const __half* bias;      // [N] or nullptr
  __half* out;             // [M, N] fp16 (fused mode)
  int32_t* C;              // [M, N] int32 (raw mode)
  const int32_t* n_used;   // device count of gathered outlier columns, or nullptr
  int out_cap;             // capacity of the gathered outlier operands (columns)
  uint32_t* status;        // device status word, or nullptr
  uint64_t wait_limit_ns;  // bound on every pipeline wait
  int tma_store;           // fused mode: write out through tmOut (needs N % 8 == 0)
  // Few outlier columns (n_used <= kSmallOutliers) are added by the epilogue
  // with warp-level MMAs straight from the gathered operands:
  const __half* XO;        // [M, ld_o] gathered X[:, O] (zero padded)
  const __half* WO;        // [N, ld_o] fp16(CB[:, O]) (zero padded)
  int ld_o;
};

// Tensor maps of one GEMM call.  A: CA [M, K] int8 (box 128 rows x 128 B).
// B: CB [N, K] int8 (box 128 rows x 128 B).  XO / WO: gathered fp16 outlier
// operands [M, ld] / [N, ld] (boxes 128 x 64 fp16; used for more than
// kSmallOutliers columns).  Out: out [M, N] fp16 (box 32 x 32; unused unless
// tma_store).
struct GemmMaps {
  CUtensorMap A, B, XO, WO, Out;
};

constexpr int kSmallOutliers = 16;

// What one launch of the GEMM computes:
//   kGemmFused  out = fp16 LLM.int8() forward (int8 codes A/B, outlier operands XO/WO, scales, bias)
//   kGemmRaw    C = A . B^T as int32
//   kGemmF16    out = fp16(XO . WO^T), an fp16 GEMM with fp32 accumulation over K fp16
//               columns: XO [M, K] and WO [N, K] (the A/B maps and every scale are unused)
enum GemmMode : int { kGemmFused = 0, kGemmRaw = 1, kGemmF16 = 2 };

// The kernel runs on CTA pairs.
cudaError_t launch_gemm(const GemmMaps& maps, const GemmArgs& a, GemmMode mode, int num_sms, cudaStream_t st);

// Box sizes the tensor maps above must be encoded with.
constexpr int kGemmBM = 128;        // rows of A per CTA (a CTA pair covers 256 rows)
constexpr int kGemmBN = 256;        // output columns per pair tile (each CTA loads 128 rows of B)
constexpr int kGemmBKBytes = 128;   // bytes of K per pipeline stage
constexpr int kGemmOutBox = 32;     // output box: 32 columns x 32 rows (64-byte swizzle)

// Few-token (decode) GEMM: weights are the wide MMA operand, tokens padded to 16.
constexpr int kDecodeMaxTokens = 16;

struct DecodeArgs {
  int M, N, K;               // M = tokens (<= kDecodeMaxTokens)
  const float* SCA;          // [M]
  const float* SCB;          // [N]
  const __half* bias;        // [N] or nullptr
  __half* out;               // [M, N]
  const int32_t* idx;        // sorted outlier columns
  const int32_t* n_used;     // device count of outlier columns, or nullptr
  int out_cap;
  const __half* XO;          // [M, ld_o] gathered X[:, O]
  int ld_o;
  int32_t* partials;         // [slots][16][N] int32 split-K partial sums, then [slots][16][N] fp32
                             // partial sums of the outlier term
  int slots;                 // decode_slots(N, K)
  int32_t* counters;         // [ceil(N/128) * 4], zero on entry
  uint32_t* status;
  uint64_t wait_limit_ns;
  int32_t* C;                // raw mode when non-null: C[t, n] = sum_k CA[t, k] * CB[n, k] as int32 [M, N]
                             // (no scales, bias or outlier term are read; out is not written)
};

// Partial-sum slots the decode GEMM needs for these sizes (grid <= kDecodeMaxGrid).
constexpr int kDecodeMaxGrid = 256;
inline int decode_slots(int N, int K) {
  const int kb = (K + 127) / 128, ntiles = (N + 127) / 128;
  const int s = kDecodeMaxGrid / ntiles + 2;
  return s < kb ? s : kb;
}

// tmW: CB [N, K] int8, box 128 rows x 128 B; tmC: CA [M, K] int8, box 16 rows x 128 B.
// boxes_per_stage: 128-byte K boxes per pipeline stage (1, 2 or 4).
// pdl: launch as a programmatic dependent of the kernel before it on the
// stream (the weights are then requested before that kernel has finished, so
// it must not write CB).
cudaError_t launch_gemm_decode(const CUtensorMap& tmW, const CUtensorMap& tmC, const DecodeArgs& a, int grid,
                               int boxes_per_stage, bool pdl, cudaStream_t st);

// Few-token preparation on one cluster of decode_prep_cluster(M, K) CTAs (M <= 16):
// codes, SCA, outlier list, X_O (zero padded to a multiple of 16 columns), the
// header words (status, used, total) and zeroed split-K counters, all in one
// launch.  XO may be null when cap == 0.  Clusters of 8 CTAs, or 16 (a
// non-portable size) for long rows of several tokens (K >= kDecodeLongRow and
// M * K >= kDecodeBigPrep) when the device can place one.
constexpr int kDecodePrepCluster = 8;
constexpr int kDecodePrepClusterBig = 16;
constexpr int kDecodeLongRow = 16384;
constexpr long long kDecodeBigPrep = 4LL * 16384;
// A preparation this large keeps its SMs busy long enough that the GEMM after it
// leaves them out of its grid (so does a 16-CTA preparation).
constexpr long long kDecodeHeavyPrep = 16LL * 16384;
int decode_prep_cluster(int M, int K);
cudaError_t launch_decode_prep(const __half* X, int M, int K, float tau, int cap, int8_t* CA, float* SCA,
                               int32_t* idx, __half* XO, int ld_o, uint32_t* hdr, int32_t* counters, int n_counters,
                               cudaStream_t st);

// The whole forward of a small problem in one launch (M <= 16 tokens,
// K <= kSmallMaxK, at most kSmallListCap outlier columns): one CTA per 128
// weight rows quantises X itself and runs its tile on the tensor cores.
// tmW: CB [N, K] int8, box 128 rows x 128 B.  hdr: status word, used and total
// outlier counts (the counts are written by the kernel; the status word is
// set when reset_status, else only raised to an error).  bias may be null.
constexpr int kSmallMaxK = 4096;
constexpr int kSmallListCap = 512;
// The grid is ceil(N / 128) clusters of linear_small_split(N, K, num_sms) CTAs,
// each CTA one slice of K.
int linear_small_split(int N, int K, int num_sms);
size_t linear_small_smem(int K, int ks);
cudaError_t launch_linear_small(const CUtensorMap& tmW, const __half* X, int M, int N, int K, float tau, int cap,
                                const float* SCB, const __half* bias, __half* out, uint32_t* hdr, uint64_t limit_ns,
                                bool reset_status, int num_sms, cudaStream_t st);

// 4-bit NF4 weight-only product, blocksize 64.  Nf4Tables holds the 16 levels
// (ascending, level[7] = 0) and the 15 midpoints between neighbours (fp32),
// computed on the host; passed to the kernels by value.
struct Nf4Tables {
  float level[16];
  float mid[16];
};
constexpr int kNf4MaxTokens = 8;
Nf4Tables nf4_tables();
// W [N, K] fp16 -> packed [N, K/2] (element 2j low nibble of byte j), absmax [N, K/64]; K % 64 == 0.
cudaError_t launch_nf4_quantize(const __half* W, int N, int K, uint8_t* packed, float* absmax, int num_sms,
                                cudaStream_t st);
cudaError_t launch_nf4_dequant(const uint8_t* packed, const float* absmax, int N, int K, __half* W, int num_sms,
                               cudaStream_t st);
// out [M, N] fp16 = X [M, K] . dequantised weight^T, 1 <= M <= kNf4MaxTokens.
cudaError_t launch_nf4_gemv(const __half* X, int M, const uint8_t* packed, const float* absmax, int N, int K,
                            __half* out, int num_sms, cudaStream_t st);

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t st);

}  // namespace i8lt
