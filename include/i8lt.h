/*
 * i8lt.h — C ABI of the B200 (sm_100a) LLM.int8() Linear8bitLt forward library
 * (with the input gradient through a frozen int8 layer).
 *
 * The operation is the mixed int8/fp16 decomposition of
 * "`bitsandbytes` - `Linear8bitLt` integration into `transformers` models"
 * (HF transformers PR #17901, section "About the mixed quantization method in
 * few words": outlier features go through fp16, the rest through int8), built
 * from the ops named in "LLM.int8() Refactoring: Part 1" (bitsandbytes PR
 * #1401): the fused calibration + quantisation kernel of section "Improved
 * kernels for inference" (int8_vectorwise_quant), the int8 GEMM and dequant
 * ops of section "Deprecations" (igemmlt -> int8_linear_matmul, mm_dequant ->
 * int8_mm_dequant), and the int8 dequantize op of section "Next steps".
 *
 * Conventions shared by every entry point
 *   - All matrices are dense row-major.  X / out / bias / W hold IEEE binary16
 *     bits (i8_half); CA / CB hold signed int8 codes in [-127, 127]; SCA / SCB
 *     are fp32 row absmax scales; C is int32.
 *   - Every pointer is a DEVICE pointer unless stated otherwise.  The caller
 *     owns every buffer: the library never allocates or frees memory, keeps no
 *     mutable global state, and may be called concurrently on different
 *     streams as long as the calls do not share output or workspace buffers.
 *     The one exception is i8_linear8bit_forward_static, whose calls share one
 *     scratch array built into the library (see its note).
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and is asynchronous: I8_OK means "arguments valid and
 *     kernels enqueued".  Nothing synchronises the host except i8_read_status.
 *   - Argument errors are returned before anything is enqueued.  Matrix
 *     pointers must be 16-byte aligned and K must be a multiple of 16 (the TMA
 *     row-stride rule; the gradient entry points state their own rule); M, N,
 *     K must be > 0.  The threshold must be finite and
 *     >= 0; 0 turns outlier handling off.
 *   - Errors found on the device (more outlier columns than the workspace
 *     holds, a pipeline wait that ran past its time limit) are written to a
 *     status word in device memory and read back with i8_read_status.
 *   - Numerics: quantisation rounds x * fl32(127 / absmax) to nearest-even in
 *     fp32; the int8 product is exact in int32; dequantisation is fp32 and the
 *     result is rounded once to fp16.
 */
#ifndef I8LT_H_
#define I8LT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define I8_API __attribute__((visibility("default")))
#else
#define I8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t i8_half;          /* IEEE 754 binary16 bit pattern */
typedef struct CUstream_st* i8_stream_t;   /* identical to cudaStream_t */

typedef enum {
  I8_OK = 0,
  I8_ERR_INVALID_ARG = 1,        /* null pointer, non-positive size, bad threshold */
  I8_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 16 != 0, misaligned pointer, size limits */
  I8_ERR_WORKSPACE = 3,          /* workspace too small or misaligned */
  I8_ERR_CUDA = 4,               /* a CUDA runtime / driver call failed */
  I8_ERR_TIMEOUT = 5,            /* device: a pipeline wait ran past its time limit */
  I8_ERR_OUTLIER_OVERFLOW = 6    /* device: more outlier columns than max_outlier_cols */
} i8_status;

/* Human-readable name of a status code (static string, never NULL). */
I8_API const char* i8_status_string(i8_status s);

/*
 * i8_quantize_rowwise — fused row-wise calibration, int8 quantisation and
 * outlier-column detection ("LLM.int8() Refactoring: Part 1", section
 * "Improved kernels for inference": int8_vectorwise_quant; outlier columns are
 * the `state.idx` of the review of bitsandbytes/autograd/_functions.py).
 *
 *   X       [M, K] fp16 input (tokens x features).
 *   CA      [M, K] int8 output codes.
 *   SCA     [M]    fp32 output: per row, the max |x| over the elements whose
 *                  magnitude is below `threshold` (all elements if it is 0).
 *   bitmap  [ceil(K/32)] uint32 output, required when threshold > 0 (may be
 *           NULL otherwise): bit (j % 32) of word j / 32 is set iff some
 *           element of column j has |x| >= threshold.  Overwritten.
 * Codes: CA = clamp(rne(x * fl32(127/SCA)), -127, 127), 0 when SCA == 0, and
 * every outlier column of CA is 0 in every row (that column belongs to the
 * fp16 path).  Uses the caller's `bitmap` as its only scratch.
 */
I8_API i8_status i8_quantize_rowwise(const i8_half* X, int M, int K, float threshold,
                              int8_t* CA, float* SCA, uint32_t* bitmap,
                              i8_stream_t stream);

/*
 * i8_outlier_columns — compact an outlier bitmap into the sorted list of
 * outlier column indices (the `state.idx` of "LLM.int8() Refactoring: Part 1",
 * review of bitsandbytes/autograd/_functions.py).
 *   bitmap [ceil(K/32)] uint32 input; idx [max_cols] int32 output (ascending);
 *   count  one int32 output = number of outlier columns found (may exceed
 *   max_cols; only the first max_cols indices are written).
 */
I8_API i8_status i8_outlier_columns(const uint32_t* bitmap, int K, int32_t* idx,
                             int max_cols, int32_t* count, i8_stream_t stream);

/*
 * i8_int8_linear_matmul — C = A . B^T exactly, int8 x int8 -> int32
 * ("LLM.int8() Refactoring: Part 1", section "Deprecations": igemmlt becomes
 * int8_linear_matmul; row-major operands).
 *   A [M, K] int8, B [N, K] int8 (both K-contiguous), C [M, N] int32 output.
 * |C| <= 127*128*K always fits int32 for K <= 131072.
 */
I8_API i8_status i8_int8_linear_matmul(const int8_t* A, const int8_t* B, int M, int N, int K,
                                int32_t* C, i8_stream_t stream);

/*
 * i8_int8_linear_matmul_ws — the same exact product, C = A . B^T in int32,
 * computed by the kernel the forward itself uses for these sizes: for
 * M <= 16 rows the few-token stream-K kernel (its k-range split across CTAs,
 * partial sums combined in the workspace), for more rows the tensor-core
 * GEMM of i8_int8_linear_matmul.  It lets a caller check that few-token
 * kernel's integer sums on their own, before any scaling.
 *   workspace: device memory, 256-byte aligned, of at least
 *     i8_int8_linear_matmul_workspace_size(M, N, K) bytes (0 for M > 16:
 *     NULL is then accepted).  Its contents on entry do not matter.
 *   status: optional device uint32 (NULL to skip).  The call first sets it to
 *     I8_OK, in stream order; a pipeline wait that ran past its time limit
 *     then sets it to I8_ERR_TIMEOUT (C is unspecified in that case).
 * Same operand rules as i8_int8_linear_matmul.
 */
I8_API size_t i8_int8_linear_matmul_workspace_size(int M, int N, int K);
I8_API i8_status i8_int8_linear_matmul_ws(const int8_t* A, const int8_t* B, int M, int N, int K, int32_t* C,
                                          void* workspace, size_t workspace_bytes, uint32_t* status,
                                          i8_stream_t stream);

/*
 * i8_int8_mm_dequant — out = fp16(C * SCA[i] * SCB[n] / 127^2 + bias[n])
 * ("LLM.int8() Refactoring: Part 1", section "Deprecations": mm_dequant
 * becomes int8_mm_dequant; commit "New naive mm_dequant kernel for row-major").
 *   C [M, N] int32, SCA [M] fp32, SCB [N] fp32, bias [N] fp16 or NULL,
 *   out [M, N] fp16 output.
 */
I8_API i8_status i8_int8_mm_dequant(const int32_t* C, const float* SCA, const float* SCB,
                             const i8_half* bias, int M, int N, i8_half* out,
                             i8_stream_t stream);

/*
 * i8_dequant — int8 weight back to fp16: W = fp16(CB * SCB[n] / 127)
 * ("LLM.int8() Refactoring: Part 1", section "Next steps": int8 dequantize op).
 *   CB [N, K] int8, SCB [N] fp32, W [N, K] fp16 output.
 */
I8_API i8_status i8_dequant(const int8_t* CB, const float* SCB, int N, int K, i8_half* W,
                     i8_stream_t stream);

/*
 * i8_dequant_transposed — the same dequantised weight stored transposed:
 *   Wt[k, n] = fp16(CB[n, k] * SCB[n] / 127), bit for bit the transpose of
 *   i8_dequant's W.  CB [N, K] int8, SCB [N] fp32, Wt [K, N] fp16 output.
 * Requires K % 16 == 0 and N % 8 == 0 (16-byte rows of Wt); K <= 4194240.
 * Wt is the weight operand of i8_linear8bit_backward_input.
 */
I8_API i8_status i8_dequant_transposed(const int8_t* CB, const float* SCB, int N, int K,
                                i8_half* Wt, i8_stream_t stream);

/*
 * i8_gather_column_blocks — the output of a layer split by output columns
 * over P GPUs ("column parallel": the exllama issue #95 discussion of tensor
 * parallelism splits a linear layer's weight between GPUs; the
 * `Linear8bitLt` integration page spreads BLOOM-176B's int8 weights over
 * several A100s).  Rank p holds rows [p*Np, (p+1)*Np) of CB / SCB / bias and
 * computes out_p [M, Np] on the replicated X; an all-gather of the out_p
 * leaves them rank-major in G [P, M, Np] (each block contiguous); this puts
 * them in place:
 *   out[m, p*Np + j] = G[p, m, j],   out [M, P*Np] fp16, row-major.
 * A plain copy (bit for bit).  G and out 16-byte aligned, P*Np < 2^31.
 */
I8_API i8_status i8_gather_column_blocks(const i8_half* G, int P, int M, int Np, i8_half* out,
                                         i8_stream_t stream);

/*
 * 4-bit NF4 weight-only product, blocksize 64 ("Loading an LLM in 4 bits using
 * bitsandbytes", sections "Normalized Float" and "Double Quantization": the
 * nf4 values are optimised for normally distributed weights; weights are
 * quantised in blocks of 64, each with a 32-bit scale; the product is computed
 * after dequantisation).  The page prints neither the values nor the rounding
 * rule; this library takes:
 *   levels  the NormalFloat construction: with Q the standard normal quantile
 *           and p* = 1 - (1/32 + 1/30)/2, Q(1/2 + i(p* - 1/2)/8)/Q(p*) for
 *           i = 1..8, -Q(1/2 + i(p* - 1/2)/7)/Q(p*) for i = 1..7, and 0, as
 *           fp32, ascending (code 7 is 0, codes 0 and 15 are -1 and +1);
 *   codes   per block of 64 consecutive weights of a row (K % 64 == 0):
 *           a = max |w| (fp32), y = fl32(w / a) (0 if a == 0), code = the number
 *           of midpoints fl32((v_i + v_{i+1})/2) below y (nearest level, ties to
 *           the lower); byte j of a row holds element 2j in its low nibble and
 *           element 2j + 1 in its high nibble;
 *   dequant W^ = fp16(fl32(v[code] * a)).
 *
 * i8_nf4_levels — the 16 levels (host memory, 16 floats).  Host only: needs no
 *   device and is safe to call anywhere.
 * i8_nf4_quantize — W [N, K] fp16 -> packed [N, K/2] uint8, absmax [N, K/64] fp32.
 * i8_nf4_dequant — packed, absmax -> W^ [N, K] fp16.
 * i8_nf4_gemv — the decode product out [M, N] fp16 =
 *   fp16(sum_k X[t, k] * v[code[n, k]] * absmax[n, k/64]), 1 <= M <= 8 tokens,
 *   evaluated in fp32 (the block scale applied once per 32 weights).  X [M, K]
 *   fp16 16-byte aligned; packed 16-byte aligned; absmax 4-byte aligned.
 */
I8_API i8_status i8_nf4_levels(float* levels16);
I8_API i8_status i8_nf4_quantize(const i8_half* W, int N, int K, uint8_t* packed, float* absmax,
                                 i8_stream_t stream);
I8_API i8_status i8_nf4_dequant(const uint8_t* packed, const float* absmax, int N, int K, i8_half* W,
                                i8_stream_t stream);
I8_API i8_status i8_nf4_gemv(const i8_half* X, int M, const uint8_t* packed, const float* absmax, int N,
                             int K, i8_half* out, i8_stream_t stream);

/*
 * i8_linear8bit_backward_input — input gradient of the int8 linear layer:
 *   dX[i, k] = fp16( sum_n dY[i, n] * Wt[k, n] ),  fp32 accumulation,
 * i.e. dX = dY . W^ for y = X . W^T + bias with W^ = Wt^T.  With Wt from
 * i8_dequant_transposed, W^ is the dequantised int8 weight, so the gradient
 * flows through the frozen quantised layer to the layers and adapters before
 * it ("`bitsandbytes` - `Linear8bitLt` integration into `transformers`
 * models", discussion of fine-tuning with trainable adapters on top of int8
 * modules; the int8 weight itself is not trained, so there is no weight
 * gradient).  The product has no int8 part and no outlier decomposition: it
 * runs on the tensor cores in fp16 (tcgen05 kind::f16).
 *   dY [M, N] fp16, Wt [K, N] fp16, dX [M, K] fp16 output.
 * Requires N % 8 == 0 (16-byte rows of dY and Wt).  A pipeline wait that ran
 * past its time limit leaves dX unspecified; this entry point does not report
 * it, i8_linear8bit_backward_input_status does.
 */
I8_API i8_status i8_linear8bit_backward_input(const i8_half* dY, const i8_half* Wt, int M, int N,
                                       int K, i8_half* dX, i8_stream_t stream);

/*
 * The same input gradient with a status word: `status` (device uint32, 4-byte
 * aligned, or NULL) is set to I8_OK first, in stream order, and to
 * I8_ERR_TIMEOUT if a pipeline wait ran past its time limit (dX is then
 * unspecified).
 */
I8_API i8_status i8_linear8bit_backward_input_status(const i8_half* dY, const i8_half* Wt, int M, int N,
                                                     int K, i8_half* dX, uint32_t* status,
                                                     i8_stream_t stream);

/*
 * Workspace bytes i8_linear8bit_forward needs for these sizes.  The workspace
 * is caller-owned device memory, 256-byte aligned, that holds CA, SCA, the
 * outlier bitmap / index list, the gathered fp16 outlier operands and the
 * status word.  Returns 0 for invalid sizes.
 */
I8_API size_t i8_linear8bit_workspace_size(int M, int N, int K, int max_outlier_cols);

/*
 * Where i8_linear8bit_prepare leaves its results inside the workspace (byte
 * offsets from its start), so that a caller can read the prepared operands
 * back: after i8_linear8bit_prepare (or a whole forward) has run,
 *   header  uint32 [3]: status word, outlier columns gathered (used = min(total,
 *           max_outlier_cols)), outlier columns found (total);
 *   bitmap  uint32 [ceil(K/32)] outlier-column bitmap (M > 16 only; for M <= 16
 *           the preparation keeps it on chip and this region is unused);
 *   idx     int32 [used]: the outlier columns, ascending (the state.idx of
 *           "LLM.int8() Refactoring: Part 1", review of _functions.py);
 *   sca     fp32 [M] row scales; ca  int8 [M, K] codes, 0 in every outlier column;
 *   x_o     fp16 [M, ld_o] gathered X[:, idx]; w_o  fp16 [N, ld_o] gathered
 *           fp16(CB[:, idx]) (M > 16 only).
 * Order of the gathered columns: for M > 16, within each group of 16 list
 * entries the stored positions hold entries (0 1 8 9)(2 3 10 11)(4 5 12 13)
 * (6 7 14 15) of the group, i.e. position p holds entry
 * 16*(p/16) + 2*((p%16)/4) + (p%2) + 8*((p%4)/2) (the order of an m16n8k16
 * operand fragment), and positions past `used` up to the next multiple of 64
 * (16 when used <= 16) are 0.  For M <= 16, x_o holds the entries in list
 * order, zero up to the next multiple of 16.
 * few_tokens is 1 when M <= 16 (the few-token kernels are used).
 */
typedef struct {
  size_t header, bitmap, idx, sca, ca, x_o, w_o, total;
  int ld_o;
  int few_tokens;
} i8_workspace_layout;
I8_API i8_status i8_linear8bit_workspace_layout(int M, int N, int K, int max_outlier_cols,
                                                i8_workspace_layout* layout);

/*
 * i8_linear8bit_forward — LLM.int8() Linear8bitLt forward
 * ("`bitsandbytes` - `Linear8bitLt` integration into `transformers` models",
 * section "About the mixed quantization method in few words"):
 *
 *   out[i, n] = fp16( C[i,n] * SCA[i] * SCB[n] / 127^2 + bias[n]
 *                     + (SCB[n] / 127) * sum_{j in O} X[i, j] * CB[n, j] )
 *
 * where CA, SCA, O come from i8_quantize_rowwise(X, threshold) and
 * C = CA . CB^T.  X [M, K] fp16; CB [N, K] int8 and SCB [N] fp32 from
 * i8_quantize_rowwise(W, threshold = 0); bias [N] fp16 or NULL; out [M, N]
 * fp16 output.  The outlier term runs on the fp16 tensor-core path; O is read
 * on the device, so the call never waits for the host.
 *   workspace / workspace_bytes: see i8_linear8bit_workspace_size.
 *   max_outlier_cols: capacity for |O|; if more columns reach the threshold,
 *   the status word becomes I8_ERR_OUTLIER_OVERFLOW and out is unspecified.
 * For M > 16 it enqueues one small memset and three kernels: the fused
 * quantiser, the outlier preparation (skipped when threshold == 0) and the
 * tensor-core GEMM with the dequant epilogue.  For M <= 16 it enqueues two
 * kernels: one cluster launch that does the quantisation and the outlier
 * preparation (and writes the status word itself), and the few-token GEMM.
 * Identical to i8_linear8bit_prepare followed by i8_linear8bit_matmul_dequant
 * on the same stream and workspace.
 */
I8_API i8_status i8_linear8bit_forward(const i8_half* X, const int8_t* CB, const float* SCB,
                                const i8_half* bias, int M, int N, int K, float threshold,
                                i8_half* out, void* workspace, size_t workspace_bytes,
                                int max_outlier_cols, i8_stream_t stream);

/*
 * Several linear layers that read the same input X, as the query/key/value
 * projections (or the gate/up projections) of a transformer block do once
 * every nn.Linear is a Linear8bitLt ("`bitsandbytes` - `Linear8bitLt`
 * integration into `transformers` models", which replaces all of a model's
 * linear layers):
 *   out[g] = Linear8bitLt(X; CB[g], SCB[g], bias[g]),  g = 0 .. G-1,
 * each bit for bit what i8_linear8bit_forward returns for that weight alone.
 * The outlier columns are a property of X (any |x| at or above the threshold
 * in the column), so X is quantised, its outlier set found and X[:, O]
 * gathered once for all G weights; then each weight gets its outlier rows
 * fp16(CB[g][:, O]) and its own GEMM launch, in order g = 0 .. G-1.
 *   X [M, K] fp16 device pointer.  CB, SCB, bias, N, out are HOST arrays of
 *   G entries holding device pointers (bias may be NULL, or hold NULL
 *   entries); CB[g] [N[g], K] int8, SCB[g] [N[g]] fp32, out[g] [M, N[g]] fp16.
 *   1 <= G <= 16.  Every weight must pass i8_linear8bit_forward's checks.
 * The workspace comes from i8_linear8bit_multi_workspace_size; status and
 * outlier count are read with i8_read_status, as for the single forward.
 */
I8_API size_t i8_linear8bit_multi_workspace_size(int M, int K, int G, const int* N,
                                          int max_outlier_cols);
I8_API i8_status i8_linear8bit_forward_multi(const i8_half* X, int M, int K, int G,
                                      const int8_t* const* CB, const float* const* SCB,
                                      const i8_half* const* bias, const int* N,
                                      i8_half* const* out, float threshold, void* workspace,
                                      size_t workspace_bytes, int max_outlier_cols,
                                      i8_stream_t stream);

/*
 * The two halves of i8_linear8bit_forward, for callers that want to place
 * work or events between them (same arguments, same workspace, same stream):
 *   i8_linear8bit_prepare: resets the status word, quantises X into the
 *     workspace (CA, SCA) and, when threshold > 0, finds the outlier columns,
 *     builds their sorted list, zeroes CA's outlier columns and gathers the
 *     fp16 operands X[:, O] (and, for M > 16, CB[:, O]).
 *   i8_linear8bit_matmul_dequant: the tensor-core GEMM with the fused
 *     dequant / bias / outlier epilogue, reading the prepared workspace.
 *     Enqueue it right after i8_linear8bit_prepare on the same stream (events
 *     may sit in between, other kernels may not): it is launched as a
 *     programmatic dependent of the preparation and, for few tokens, starts
 *     streaming CB before the preparation has finished.
 */
I8_API i8_status i8_linear8bit_prepare(const i8_half* X, const int8_t* CB, int M, int N, int K,
                                       float threshold, void* workspace, size_t workspace_bytes,
                                       int max_outlier_cols, i8_stream_t stream);
I8_API i8_status i8_linear8bit_matmul_dequant(const int8_t* CB, const float* SCB, const i8_half* bias,
                                              int M, int N, int K, float threshold, i8_half* out,
                                              void* workspace, size_t workspace_bytes,
                                              int max_outlier_cols, i8_stream_t stream);

/*
 * i8_read_status — synchronise `stream` and return the device status word of
 * the last i8_linear8bit_forward that used `workspace` (I8_OK, I8_ERR_TIMEOUT
 * or I8_ERR_OUTLIER_OVERFLOW), or I8_ERR_CUDA if the synchronisation failed.
 * `count` (host pointer, may be NULL) receives the number of outlier columns
 * that call found.
 */
I8_API i8_status i8_read_status(const void* workspace, int32_t* count, i8_stream_t stream);

/*
 * i8_linear8bit_forward_static — the same forward as i8_linear8bit_forward,
 * for callers that cannot hand the library a workspace.  The pages have no
 * counterpart to this entry point.
 *
 * Some callers cannot allocate device memory where they run the forward:
 * plugin and inference-server hooks that are handed a stream but no allocator
 * or workspace, code inside a framework whose own caching allocator owns the
 * device memory, and latency-critical loops that must not call cudaMalloc
 * (it can synchronise the whole device) or take an allocator's locks.  This
 * entry point allocates nothing: its scratch is a
 * fixed 32 MiB device array built into the library (each GPU that loads the
 * library keeps it until the process exits).  The caller still passes X, CB,
 * SCB, bias and out exactly as for i8_linear8bit_forward.
 *   status_out: optional device pointer to 3 uint32 that receive, in stream
 *     order, the status word and the used / total outlier-column counts (the
 *     values i8_read_status reports for a workspace); NULL to skip.
 * Sizes whose workspace (i8_linear8bit_workspace_size) exceeds 32 MiB are
 * rejected with I8_ERR_WORKSPACE before anything is enqueued.
 * The first call on each device looks up the array's device address and must
 * happen before any stream capture that records this call.  The address is
 * kept per device and CUDA context: if the device's context is destroyed and
 * created again (cudaDeviceReset, or a framework that tears its context
 * down), the next call looks the array up again, so that call too must come
 * before any stream capture.  All calls share
 * the one array and it keeps the previous call's contents (each call clears
 * what must start at zero), so calls that can overlap on the GPU — on two
 * streams, or from two host threads — race; serialise them on one stream.
 */
I8_API i8_status i8_linear8bit_forward_static(const i8_half* X, const int8_t* CB, const float* SCB,
                                              const i8_half* bias, int M, int N, int K, float threshold,
                                              i8_half* out, int max_outlier_cols, uint32_t* status_out,
                                              i8_stream_t stream);

/*
 * i8_selftest_bounded_wait — failure-detection self test.  Launches one block
 * that waits on a shared-memory barrier that nothing ever completes, with the
 * same bounded-wait routine the GEMM pipeline uses and a limit of
 * `limit_ns` nanoseconds (1 ms .. 10 s).  The kernel gives up, writes
 * I8_ERR_TIMEOUT to *status (device uint32) and returns; nothing hangs.
 */
I8_API i8_status i8_selftest_bounded_wait(uint32_t* status, uint64_t limit_ns, i8_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* I8LT_H_ */
