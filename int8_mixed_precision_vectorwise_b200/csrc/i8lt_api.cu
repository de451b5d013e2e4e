// C ABI of the library (declared in include/i8lt.h): argument validation,
// workspace layout, TMA tensor-map encoding and kernel launches.  Every check
// that can fail on the host runs before any CUDA call, so argument errors are
// reported without touching the device.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/i8lt.h"
#include "kernels.cuh"
#include "per_device.h"

namespace {

using i8lt::GemmArgs;

constexpr int kMaxOutlierCap = 8192;                   // shared-memory index list of the prepare kernel
constexpr uint64_t kWaitLimitNs = 2000000000ull;       // 2 s bound on every pipeline wait
constexpr size_t kHdrBytes = 256;                      // status, used count, total count

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

constexpr int kMaxGroups = 16;                        // weights per multi-weight forward

struct WsLayout {
  size_t hdr, bitmap, counters, idx, sca, ca, xo, wo, partials, total;
  size_t clear_bytes;  // prefix cleared by every call: header, bitmap, split-K counters
  int ld_o;            // row stride (fp16 elements) of the gathered outlier operands
  bool decode;         // few tokens: the decode GEMM (split-K partials, no W_O gather)
  int n_counters;      // split-K counters of all weights (decode)
};

inline int decode_counters(int N) { return ((N + 127) / 128) * 4; }

// Layout for G weights (N[g] output rows each) that read the same X [M, K]: the
// quantised X, its outlier list and X[:, O] once; per weight its gathered
// outlier rows W_O (more than 16 tokens) or its split-K counters (16 or fewer;
// the partial-sum area is reused by the weights' GEMMs in turn).
bool ws_layout_multi(int M, int K, int G, const int* N, int cap, WsLayout* L) {
  if (M <= 0 || K <= 0 || cap < 0 || G < 1 || G > kMaxGroups || N == nullptr) return false;
  for (int g = 0; g < G; ++g)
    if (N[g] <= 0) return false;
  L->decode = M <= i8lt::kDecodeMaxTokens;
  L->n_counters = 0;
  size_t wo_bytes = 0, partial_bytes = 0;
  for (int g = 0; g < G; ++g) {
    L->n_counters += decode_counters(N[g]);
    const size_t pb = static_cast<size_t>(i8lt::decode_slots(N[g], K)) * i8lt::kDecodeMaxTokens * N[g] * 8;
    partial_bytes = pb > partial_bytes ? pb : partial_bytes;
  }
  L->ld_o = cap > 0 ? ((cap + 63) / 64) * 64 : 0;
  for (int g = 0; g < G; ++g) wo_bytes += align256(static_cast<size_t>(N[g]) * L->ld_o * 2);
  size_t off = 0;
  L->hdr = off;
  off += kHdrBytes;
  L->bitmap = off;
  off += align256(static_cast<size_t>((K + 31) / 32) * 4);
  L->counters = off;
  off += L->decode ? align256(static_cast<size_t>(L->n_counters) * 4) : 0;
  L->clear_bytes = off;
  L->idx = off;
  off += align256(static_cast<size_t>(cap > 0 ? cap : 1) * 4);
  L->sca = off;
  off += align256(static_cast<size_t>(M) * 4);
  L->ca = off;
  off += align256(static_cast<size_t>(M) * K);
  L->xo = off;
  off += align256(static_cast<size_t>(M) * L->ld_o * 2);
  L->wo = off;
  off += L->decode ? 0 : wo_bytes;
  L->partials = off;
  // int32 partials, then fp32 partials of the outlier term
  off += L->decode ? align256(partial_bytes) : 0;
  L->total = off;
  return true;
}

bool ws_layout(int M, int N, int K, int cap, WsLayout* L) { return ws_layout_multi(M, K, 1, &N, cap, L); }

// Byte offsets of weight g's gathered outlier rows and split-K counters.
size_t wo_offset(const WsLayout& L, const int* N, int g) {
  size_t off = L.wo;
  for (int h = 0; h < g; ++h) off += align256(static_cast<size_t>(N[h]) * L.ld_o * 2);
  return off;
}
size_t counters_offset(const WsLayout& L, const int* N, int g) {
  size_t off = L.counters;
  for (int h = 0; h < g; ++h) off += static_cast<size_t>(decode_counters(N[h])) * 4;
  return off;
}

// --------------------------------------------------------------- driver entry point
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major [rows, inner] matrix, boxes of box_inner x box_rows elements.
bool encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t rows,
               uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_rows,
               CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  // A map is a function of these arguments alone (address, sizes, box, swizzle), so the
  // last few encoded per host thread are kept and copied on a repeat: a layer called
  // again with the same weight skips the encoder, a per-call host cost of the small forward.
  struct Entry {
    CUtensorMap map;
    const void* base;
    uint64_t inner, rows, stride;
    uint32_t box_inner, box_rows;
    int dt, swz;
    bool valid;
  };
  static thread_local Entry cache[8];
  static thread_local unsigned next = 0;
  for (const Entry& e : cache)
    if (e.valid && e.base == base && e.inner == inner && e.rows == rows && e.stride == row_stride_bytes &&
        e.box_inner == box_inner && e.box_rows == box_rows && e.dt == static_cast<int>(dt) &&
        e.swz == static_cast<int>(swz)) {
      *tm = e.map;
      return true;
    }
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  if (fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  Entry& e = cache[next++ % 8];
  e = Entry{*tm, base, inner, rows, row_stride_bytes, box_inner, box_rows, static_cast<int>(dt),
            static_cast<int>(swz), true};
  return true;
}

// SM count of the current device, cached per device (calls may come from
// several host threads at once).
int num_sms() {
  static i8lt::PerDeviceInt cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  return cache.get(dev, [dev] {
    int n = 0;
    return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess ? n : 0;
  });
}

inline i8_status cuda_status(cudaError_t e) { return e == cudaSuccess ? I8_OK : I8_ERR_CUDA; }

i8_status check_threshold(float t) {
  if (!std::isfinite(t) || t < 0.f) return I8_ERR_INVALID_ARG;
  return I8_OK;
}

// Shape/pointer rules shared by the GEMM entry points.
i8_status check_gemm_operands(const void* A, const void* B, int M, int N, int K) {
  if (!A || !B) return I8_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (K % 16 != 0 || K > (1 << 17)) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(A) || !aligned16(B)) return I8_ERR_UNSUPPORTED_SHAPE;
  return I8_OK;
}

i8_status run_gemm(const int8_t* A, const int8_t* B, int M, int N, int K, GemmArgs args, bool raw,
                   const __half* XO, const __half* WO, int ld_o, cudaStream_t st) {
  i8lt::GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const uint32_t kbk = i8lt::kGemmBKBytes;
  if (!encode_2d(&maps.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, kbk, i8lt::kGemmBM) ||
      !encode_2d(&maps.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, K, kbk, i8lt::kGemmBN / 2))
    return I8_ERR_CUDA;
  if (XO != nullptr && WO != nullptr && ld_o > 0) {
    const uint64_t ld_bytes = static_cast<uint64_t>(ld_o) * 2;
    if (!encode_2d(&maps.XO, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, XO, ld_o, M, ld_bytes, 64, i8lt::kGemmBM) ||
        !encode_2d(&maps.WO, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, WO, ld_o, N, ld_bytes, 64, i8lt::kGemmBN / 2))
      return I8_ERR_CUDA;
  }
  args.tma_store = 0;
  if (!raw && N % 8 == 0) {
    // fp16 rows must be 16-byte multiples for the TMA store; otherwise plain stores
    if (!encode_2d(&maps.Out, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, args.out, N, M, static_cast<uint64_t>(N) * 2,
                   i8lt::kGemmOutBox, i8lt::kGemmOutBox, CU_TENSOR_MAP_SWIZZLE_64B))
      return I8_ERR_CUDA;
    args.tma_store = 1;
  }
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_gemm(maps, args, raw ? i8lt::kGemmRaw : i8lt::kGemmFused, sms, st));
}

// out [M, Nout] = fp16(Aop [M, Kc] . Bop [Nout, Kc]^T), fp16 operands, fp32 accumulation.
// status: optional device word that a pipeline-wait timeout sets to I8_ERR_TIMEOUT.
i8_status run_gemm_f16(const __half* Aop, const __half* Bop, int M, int Nout, int Kc, __half* out, uint32_t* status,
                       cudaStream_t st) {
  i8lt::GemmMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const uint64_t ld_bytes = static_cast<uint64_t>(Kc) * 2;
  if (!encode_2d(&maps.XO, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Aop, Kc, M, ld_bytes, 64, i8lt::kGemmBM) ||
      !encode_2d(&maps.WO, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, Bop, Kc, Nout, ld_bytes, 64, i8lt::kGemmBN / 2))
    return I8_ERR_CUDA;
  GemmArgs a{};
  a.M = M;
  a.N = Nout;
  a.K = Kc;
  a.out = out;
  a.status = status;
  a.wait_limit_ns = kWaitLimitNs;
  a.tma_store = 0;
  if (Nout % 8 == 0) {
    if (!encode_2d(&maps.Out, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, out, Nout, M, static_cast<uint64_t>(Nout) * 2,
                   i8lt::kGemmOutBox, i8lt::kGemmOutBox, CU_TENSOR_MAP_SWIZZLE_64B))
      return I8_ERR_CUDA;
    a.tma_store = 1;
  }
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_gemm(maps, a, i8lt::kGemmF16, sms, st));
}

// Few-token GEMM: 128-byte K boxes per pipeline stage (512 bytes of each
// weight row per stage) and the grid of the stream-K split (one CTA per SM, at
// most kDecodeMaxGrid, never more CTAs than (tile, stage) work items).
// `M_prep` is the number of rows the preparation kernel before it quantises (0:
// none): when M_prep * K is large, that kernel's cluster keeps its SMs busy for
// several microseconds while the GEMM's CTAs would wait for them with an equal
// share of the weight stream, so the GEMM leaves those SMs out.
constexpr int kDecodeBoxes = 4;
int decode_grid(int N, int K, int sms, int M_prep) {
  const int total = ((N + 127) / 128) * ((K + 128 * kDecodeBoxes - 1) / (128 * kDecodeBoxes));
  if (M_prep > 0) {
    const int pc = i8lt::decode_prep_cluster(M_prep, K);
    if (pc == i8lt::kDecodePrepClusterBig || static_cast<long long>(M_prep) * K >= i8lt::kDecodeHeavyPrep) sms -= pc;
  }
  int grid = sms < i8lt::kDecodeMaxGrid ? sms : i8lt::kDecodeMaxGrid;
  return grid > total ? total : grid;
}

// Workspace of the int8 matmul entry point: for few rows, the split-K
// counters and partial sums of the stream-K kernel; nothing otherwise.
struct MatmulWs {
  size_t partials, total;
};
MatmulWs matmul_ws_layout(int M, int N, int K) {
  MatmulWs w{0, 0};
  if (M > i8lt::kDecodeMaxTokens) return w;
  w.partials = align256(static_cast<size_t>(decode_counters(N)) * 4);
  w.total = w.partials + align256(static_cast<size_t>(i8lt::decode_slots(N, K)) * i8lt::kDecodeMaxTokens * N * 8);
  return w;
}

}  // namespace

namespace {

// Validation shared by the forward and its two stages; fills the layout.
i8_status check_forward(const i8_half* X, const int8_t* CB, const float* SCB, const i8_half* bias, int M, int N,
                        int K, float threshold, const i8_half* out, bool need_out, const void* workspace,
                        size_t workspace_bytes, int max_outlier_cols, WsLayout* L) {
  if (!X || !workspace || (need_out && (!out || !SCB))) return I8_ERR_INVALID_ARG;
  i8_status s = check_gemm_operands(X, CB, M, N, K);
  if (s != I8_OK) return s;
  if (check_threshold(threshold) != I8_OK || max_outlier_cols < 0) return I8_ERR_INVALID_ARG;
  if (max_outlier_cols > kMaxOutlierCap) return I8_ERR_UNSUPPORTED_SHAPE;
  if (need_out && (!aligned16(out) || (bias && !aligned16(bias)))) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!ws_layout(M, N, K, max_outlier_cols, L)) return I8_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < L->total) return I8_ERR_WORKSPACE;
  return I8_OK;
}

struct WsPtrs {
  uint32_t* hdr;
  uint32_t* bitmap;
  int32_t* counters;
  int32_t* partials;
  int32_t* idx;
  float* SCA;
  int8_t* CA;
  __half* XO;
  __half* WO;
};

WsPtrs ws_ptrs(void* workspace, const WsLayout& L) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  return WsPtrs{reinterpret_cast<uint32_t*>(ws + L.hdr), reinterpret_cast<uint32_t*>(ws + L.bitmap),
                reinterpret_cast<int32_t*>(ws + L.counters), reinterpret_cast<int32_t*>(ws + L.partials),
                reinterpret_cast<int32_t*>(ws + L.idx),  reinterpret_cast<float*>(ws + L.sca),
                reinterpret_cast<int8_t*>(ws + L.ca),    reinterpret_cast<__half*>(ws + L.xo),
                reinterpret_cast<__half*>(ws + L.wo)};
}

i8_status enqueue_prepare(const i8_half* X, const int8_t* CB, int M, int N, int K, float threshold, void* workspace,
                          int cap, const WsLayout& L, cudaStream_t st) {
  const WsPtrs w = ws_ptrs(workspace, L);
  const __half* Xh = reinterpret_cast<const __half*>(X);
  const bool outliers = threshold > 0.f;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  if (L.decode) {
    // one cluster launch writes everything the decode GEMMs read, header and counters included
    return cuda_status(i8lt::launch_decode_prep(Xh, M, K, threshold, cap, w.CA, w.SCA, w.idx,
                                                cap > 0 ? w.XO : nullptr, L.ld_o, w.hdr, w.counters, L.n_counters,
                                                st));
  }
  // status word, counts and bitmap are contiguous: one memset clears them
  if (cudaMemsetAsync(workspace, 0, L.clear_bytes, st) != cudaSuccess) return I8_ERR_CUDA;
  i8_status s = cuda_status(i8lt::launch_quant_rows(Xh, M, K, threshold, w.CA, w.SCA, outliers ? w.bitmap : nullptr, st));
  if (s != I8_OK || !outliers) return s;
  return cuda_status(i8lt::launch_outlier_prepare(w.bitmap, K, cap, reinterpret_cast<int32_t*>(w.hdr + 2),
                                                  reinterpret_cast<int32_t*>(w.hdr + 1), w.idx, w.hdr, w.CA, Xh, M,
                                                  cap > 0 ? w.XO : nullptr, CB, N,
                                                  (cap > 0 && !L.decode) ? w.WO : nullptr, L.ld_o, sms, st));
}

// The GEMM of one weight; `counters` / `WO` are that weight's split-K counters
// (decode) or gathered outlier rows (prefill) in the workspace.
i8_status enqueue_gemm(const int8_t* CB, const float* SCB, const i8_half* bias, int M, int N, int K,
                       float threshold, i8_half* out, const WsPtrs& w, int32_t* counters, __half* WO, int cap,
                       const WsLayout& L, cudaStream_t st) {
  const bool with_o = threshold > 0.f && cap > 0;
  if (L.decode) {
    i8lt::DecodeArgs d{};
    d.M = M;
    d.N = N;
    d.K = K;
    d.SCA = w.SCA;
    d.SCB = SCB;
    d.bias = reinterpret_cast<const __half*>(bias);
    d.out = reinterpret_cast<__half*>(out);
    d.idx = w.idx;
    d.n_used = with_o ? reinterpret_cast<const int32_t*>(w.hdr + 1) : nullptr;
    d.out_cap = cap;
    d.XO = w.XO;
    d.ld_o = L.ld_o;
    d.partials = w.partials;
    d.slots = i8lt::decode_slots(N, K);
    d.counters = counters;
    d.status = w.hdr;
    d.wait_limit_ns = kWaitLimitNs;
    CUtensorMap tmW, tmC;
    if (!encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, CB, K, N, K, 128, 128) ||
        !encode_2d(&tmC, CU_TENSOR_MAP_DATA_TYPE_UINT8, w.CA, K, M, K, 128, i8lt::kDecodeMaxTokens))
      return I8_ERR_CUDA;
    const int sms = num_sms();
    if (sms <= 0) return I8_ERR_CUDA;
    return cuda_status(i8lt::launch_gemm_decode(tmW, tmC, d, decode_grid(N, K, sms, M),
                                                kDecodeBoxes, true, st));
  }
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.SCA = w.SCA;
  a.SCB = SCB;
  a.bias = reinterpret_cast<const __half*>(bias);
  a.out = reinterpret_cast<__half*>(out);
  a.n_used = with_o ? reinterpret_cast<const int32_t*>(w.hdr + 1) : nullptr;
  a.out_cap = cap;
  a.XO = with_o ? w.XO : nullptr;
  a.WO = with_o ? WO : nullptr;
  a.ld_o = L.ld_o;
  a.status = w.hdr;
  a.wait_limit_ns = kWaitLimitNs;
  return run_gemm(w.CA, CB, M, N, K, a, false, with_o ? w.XO : nullptr, with_o ? WO : nullptr, L.ld_o, st);
}

i8_status enqueue_matmul_dequant(const int8_t* CB, const float* SCB, const i8_half* bias, int M, int N, int K,
                                 float threshold, i8_half* out, void* workspace, int cap, const WsLayout& L,
                                 cudaStream_t st) {
  const WsPtrs w = ws_ptrs(workspace, L);
  return enqueue_gemm(CB, SCB, bias, M, N, K, threshold, out, w, w.counters, w.WO, cap, L, st);
}

// Small problems run the whole forward as one kernel (k_linear_small): few
// tokens, a row of X that fits the kernel's shared-memory code tile, a weight
// of at most 8 MiB spread over at most one CTA per SM, and an outlier capacity
// the kernel's list holds.  Everything else runs the two-stage path.
constexpr size_t kSmallMaxWeightBytes = size_t(8) << 20;
bool use_small(int M, int N, int K, int cap) {
  if (M > i8lt::kDecodeMaxTokens || K > i8lt::kSmallMaxK || cap > i8lt::kSmallListCap) return false;
  if (static_cast<size_t>(N) * K > kSmallMaxWeightBytes) return false;
  const int sms = num_sms();
  return sms > 0 && (N + 127) / 128 <= sms;
}

// One weight's forward with the prepared quantities kept on chip; the kernel
// writes the status word and outlier counts of the workspace header.
i8_status enqueue_small(const i8_half* X, const int8_t* CB, const float* SCB, const i8_half* bias, int M, int N,
                        int K, float threshold, i8_half* out, void* workspace, int cap, cudaStream_t st) {
  CUtensorMap tmW;
  if (!encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, CB, K, N, K, 128, 128)) return I8_ERR_CUDA;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_linear_small(tmW, reinterpret_cast<const __half*>(X), M, N, K, threshold, cap, SCB,
                                               reinterpret_cast<const __half*>(bias), reinterpret_cast<__half*>(out),
                                               static_cast<uint32_t*>(workspace), kWaitLimitNs, true, sms, st));
}

// The forward of one weight on a workspace laid out by ws_layout.
i8_status enqueue_forward(const i8_half* X, const int8_t* CB, const float* SCB, const i8_half* bias, int M, int N,
                          int K, float threshold, i8_half* out, void* workspace, int cap, const WsLayout& L,
                          cudaStream_t st) {
  if (use_small(M, N, K, cap)) return enqueue_small(X, CB, SCB, bias, M, N, K, threshold, out, workspace, cap, st);
  i8_status s = enqueue_prepare(X, CB, M, N, K, threshold, workspace, cap, L, st);
  if (s != I8_OK) return s;
  return enqueue_matmul_dequant(CB, SCB, bias, M, N, K, threshold, out, workspace, cap, L, st);
}

}  // namespace

// ---------------------------------------------------------------- allocation-free forward
// Built-in scratch for i8_linear8bit_forward_static.  It is a plain device
// array, so every GPU that loads this library holds kStaticScratchBytes of it
// until the process exits, and every call of that entry point shares it.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

namespace {

// Unique id of the calling thread's current CUDA context (driver ids are never
// reused within a process), or 0 if the driver cannot say.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_static_scratch on the current device.  In host code the
// array's name only stands in for the symbol, so the address is looked up with
// cudaGetSymbolAddress while that device is current: once per device and
// context.  If the device's context is torn down and created again (the module
// is then loaded again and the array may move), the new context id triggers a
// fresh lookup.
i8_status static_scratch(void** out) {
  static std::mutex mu;
  static void* addr[64] = {nullptr};
  static unsigned long long ctx_of[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return I8_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return I8_ERR_CUDA;
    addr[dev] = p;
    ctx_of[dev] = current_context_id();  // the lookup has made the device's context current
  }
  *out = addr[dev];
  return I8_OK;
}

}  // namespace

extern "C" {

const char* i8_status_string(i8_status s) {
  switch (s) {
    case I8_OK: return "I8_OK";
    case I8_ERR_INVALID_ARG: return "I8_ERR_INVALID_ARG";
    case I8_ERR_UNSUPPORTED_SHAPE: return "I8_ERR_UNSUPPORTED_SHAPE";
    case I8_ERR_WORKSPACE: return "I8_ERR_WORKSPACE";
    case I8_ERR_CUDA: return "I8_ERR_CUDA";
    case I8_ERR_TIMEOUT: return "I8_ERR_TIMEOUT";
    case I8_ERR_OUTLIER_OVERFLOW: return "I8_ERR_OUTLIER_OVERFLOW";
  }
  return "I8_ERR_UNKNOWN";
}

i8_status i8_quantize_rowwise(const i8_half* X, int M, int K, float threshold, int8_t* CA, float* SCA,
                              uint32_t* bitmap, i8_stream_t stream) {
  if (!X || !CA || !SCA) return I8_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (check_threshold(threshold) != I8_OK) return I8_ERR_INVALID_ARG;
  if (threshold > 0.f && !bitmap) return I8_ERR_INVALID_ARG;
  if (K % 16 != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(CA)) return I8_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const __half* Xh = reinterpret_cast<const __half*>(X);
  if (threshold > 0.f) {
    if (cudaMemsetAsync(bitmap, 0, static_cast<size_t>((K + 31) / 32) * 4, st) != cudaSuccess) return I8_ERR_CUDA;
  }
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  i8_status s = cuda_status(i8lt::launch_quant_rows(Xh, M, K, threshold, CA, SCA, threshold > 0.f ? bitmap : nullptr, st));
  if (s != I8_OK || threshold == 0.f) return s;
  return cuda_status(i8lt::launch_zero_outlier_cols(bitmap, M, K, CA, sms, st));
}

i8_status i8_outlier_columns(const uint32_t* bitmap, int K, int32_t* idx, int max_cols, int32_t* count,
                             i8_stream_t stream) {
  if (!bitmap || !count || K <= 0 || max_cols < 0) return I8_ERR_INVALID_ARG;
  if (max_cols > 0 && !idx) return I8_ERR_INVALID_ARG;
  if (max_cols > kMaxOutlierCap) return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_outlier_prepare(bitmap, K, max_cols, count, nullptr, idx, nullptr, nullptr,
                                                  nullptr, 0, nullptr, nullptr, 0, nullptr, 0, sms,
                                                  reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_int8_linear_matmul(const int8_t* A, const int8_t* B, int M, int N, int K, int32_t* C,
                                i8_stream_t stream) {
  i8_status s = check_gemm_operands(A, B, M, N, K);
  if (s != I8_OK) return s;
  if (!C) return I8_ERR_INVALID_ARG;
  if (!aligned16(C)) return I8_ERR_UNSUPPORTED_SHAPE;
  GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.C = C;
  a.wait_limit_ns = kWaitLimitNs;
  return run_gemm(A, B, M, N, K, a, true, nullptr, nullptr, 0, reinterpret_cast<cudaStream_t>(stream));
}

size_t i8_int8_linear_matmul_workspace_size(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0) return 0;
  return matmul_ws_layout(M, N, K).total;
}

i8_status i8_int8_linear_matmul_ws(const int8_t* A, const int8_t* B, int M, int N, int K, int32_t* C, void* workspace,
                                   size_t workspace_bytes, uint32_t* status, i8_stream_t stream) {
  i8_status s = check_gemm_operands(A, B, M, N, K);
  if (s != I8_OK) return s;
  if (!C) return I8_ERR_INVALID_ARG;
  if (!aligned16(C)) return I8_ERR_UNSUPPORTED_SHAPE;
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u) != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  const MatmulWs w = matmul_ws_layout(M, N, K);
  if (w.total > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
                      workspace_bytes < w.total))
    return I8_ERR_WORKSPACE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (status && cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return I8_ERR_CUDA;
  if (M > i8lt::kDecodeMaxTokens) {
    GemmArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.C = C;
    a.status = status;
    a.wait_limit_ns = kWaitLimitNs;
    return run_gemm(A, B, M, N, K, a, true, nullptr, nullptr, 0, st);
  }
  // Few rows: the forward's stream-K kernel, storing its int32 sums.  Its
  // split-K counters must start at zero.
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, w.partials, st) != cudaSuccess) return I8_ERR_CUDA;
  i8lt::DecodeArgs d{};
  d.M = M;
  d.N = N;
  d.K = K;
  d.C = C;
  d.partials = reinterpret_cast<int32_t*>(ws + w.partials);
  d.slots = i8lt::decode_slots(N, K);
  d.counters = reinterpret_cast<int32_t*>(ws);
  d.status = status;
  d.wait_limit_ns = kWaitLimitNs;
  CUtensorMap tmW, tmC;
  if (!encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, K, 128, 128) ||
      !encode_2d(&tmC, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, M, K, 128, i8lt::kDecodeMaxTokens))
    return I8_ERR_CUDA;
  // no programmatic overlap: B may be written by the work queued just before;
  // no preparation kernel runs beside it
  return cuda_status(i8lt::launch_gemm_decode(tmW, tmC, d, decode_grid(N, K, sms, 0), kDecodeBoxes, false, st));
}

i8_status i8_linear8bit_workspace_layout(int M, int N, int K, int max_outlier_cols, i8_workspace_layout* layout) {
  if (!layout) return I8_ERR_INVALID_ARG;
  if (max_outlier_cols > kMaxOutlierCap) return I8_ERR_UNSUPPORTED_SHAPE;
  WsLayout L;
  if (N <= 0 || !ws_layout(M, N, K, max_outlier_cols, &L)) return I8_ERR_INVALID_ARG;
  layout->header = L.hdr;
  layout->bitmap = L.bitmap;
  layout->idx = L.idx;
  layout->sca = L.sca;
  layout->ca = L.ca;
  layout->x_o = L.xo;
  layout->w_o = L.wo;
  layout->total = L.total;
  layout->ld_o = L.ld_o;
  layout->few_tokens = L.decode ? 1 : 0;
  return I8_OK;
}

i8_status i8_int8_mm_dequant(const int32_t* C, const float* SCA, const float* SCB, const i8_half* bias, int M,
                             int N, i8_half* out, i8_stream_t stream) {
  if (!C || !SCA || !SCB || !out) return I8_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0) return I8_ERR_INVALID_ARG;
  if (!aligned16(C) || !aligned16(SCB) || !aligned16(out) || (bias && !aligned16(bias)))
    return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_mm_dequant(C, SCA, SCB, reinterpret_cast<const __half*>(bias), M, N,
                                             reinterpret_cast<__half*>(out), sms,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_dequant(const int8_t* CB, const float* SCB, int N, int K, i8_half* W, i8_stream_t stream) {
  if (!CB || !SCB || !W) return I8_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (K % 16 != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(CB) || !aligned16(W)) return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_dequant(CB, SCB, N, K, reinterpret_cast<__half*>(W), sms,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_dequant_transposed(const int8_t* CB, const float* SCB, int N, int K, i8_half* Wt,
                                i8_stream_t stream) {
  if (!CB || !SCB || !Wt) return I8_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (K % 16 != 0 || N % 8 != 0 || K > 65535 * 64) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(CB) || !aligned16(Wt)) return I8_ERR_UNSUPPORTED_SHAPE;
  return cuda_status(i8lt::launch_dequant_t(CB, SCB, N, K, reinterpret_cast<__half*>(Wt),
                                            reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_nf4_levels(float* levels16) {
  if (!levels16) return I8_ERR_INVALID_ARG;
  const i8lt::Nf4Tables t = i8lt::nf4_tables();
  for (int i = 0; i < 16; ++i) levels16[i] = t.level[i];
  return I8_OK;
}

i8_status i8_nf4_quantize(const i8_half* W, int N, int K, uint8_t* packed, float* absmax, i8_stream_t stream) {
  if (!W || !packed || !absmax) return I8_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (K % 64 != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || (reinterpret_cast<uintptr_t>(absmax) & 3u) != 0)
    return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_nf4_quantize(reinterpret_cast<const __half*>(W), N, K, packed, absmax, sms,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_nf4_dequant(const uint8_t* packed, const float* absmax, int N, int K, i8_half* W, i8_stream_t stream) {
  if (!W || !packed || !absmax) return I8_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (K % 64 != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(packed) || (reinterpret_cast<uintptr_t>(absmax) & 3u) != 0)
    return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_nf4_dequant(packed, absmax, N, K, reinterpret_cast<__half*>(W), sms,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_nf4_gemv(const i8_half* X, int M, const uint8_t* packed, const float* absmax, int N, int K, i8_half* out,
                      i8_stream_t stream) {
  if (!X || !packed || !absmax || !out) return I8_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (K % 64 != 0 || M > i8lt::kNf4MaxTokens) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(X) || !aligned16(packed) || (reinterpret_cast<uintptr_t>(absmax) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(out) & 1u) != 0)
    return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_nf4_gemv(reinterpret_cast<const __half*>(X), M, packed, absmax, N, K,
                                           reinterpret_cast<__half*>(out), sms,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_gather_column_blocks(const i8_half* G, int P, int M, int Np, i8_half* out, i8_stream_t stream) {
  if (!G || !out) return I8_ERR_INVALID_ARG;
  if (P <= 0 || M <= 0 || Np <= 0) return I8_ERR_INVALID_ARG;
  if (static_cast<long long>(P) * Np > (1LL << 31) - 1) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(G) || !aligned16(out)) return I8_ERR_UNSUPPORTED_SHAPE;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  return cuda_status(i8lt::launch_gather_column_blocks(reinterpret_cast<const __half*>(G), P, M, Np,
                                                       reinterpret_cast<__half*>(out), sms,
                                                       reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_linear8bit_backward_input_status(const i8_half* dY, const i8_half* Wt, int M, int N, int K,
                                              i8_half* dX, uint32_t* status, i8_stream_t stream) {
  if (!dY || !Wt || !dX) return I8_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0) return I8_ERR_INVALID_ARG;
  if (N % 8 != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(dY) || !aligned16(Wt) || !aligned16(dX)) return I8_ERR_UNSUPPORTED_SHAPE;
  if (status && (reinterpret_cast<uintptr_t>(status) & 3u) != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (status && cudaMemsetAsync(status, 0, sizeof(uint32_t), st) != cudaSuccess) return I8_ERR_CUDA;
  return run_gemm_f16(reinterpret_cast<const __half*>(dY), reinterpret_cast<const __half*>(Wt), M, K, N,
                      reinterpret_cast<__half*>(dX), status, st);
}

i8_status i8_linear8bit_backward_input(const i8_half* dY, const i8_half* Wt, int M, int N, int K, i8_half* dX,
                                       i8_stream_t stream) {
  return i8_linear8bit_backward_input_status(dY, Wt, M, N, K, dX, nullptr, stream);
}

size_t i8_linear8bit_workspace_size(int M, int N, int K, int max_outlier_cols) {
  WsLayout L;
  if (max_outlier_cols > kMaxOutlierCap || !ws_layout(M, N, K, max_outlier_cols, &L)) return 0;
  return L.total;
}


i8_status i8_linear8bit_prepare(const i8_half* X, const int8_t* CB, int M, int N, int K, float threshold,
                                void* workspace, size_t workspace_bytes, int max_outlier_cols, i8_stream_t stream) {
  WsLayout L;
  i8_status s = check_forward(X, CB, nullptr, nullptr, M, N, K, threshold, nullptr, false, workspace,
                              workspace_bytes, max_outlier_cols, &L);
  if (s != I8_OK) return s;
  return enqueue_prepare(X, CB, M, N, K, threshold, workspace, max_outlier_cols, L,
                         reinterpret_cast<cudaStream_t>(stream));
}

i8_status i8_linear8bit_matmul_dequant(const int8_t* CB, const float* SCB, const i8_half* bias, int M, int N, int K,
                                       float threshold, i8_half* out, void* workspace, size_t workspace_bytes,
                                       int max_outlier_cols, i8_stream_t stream) {
  WsLayout L;
  // X is not read by this stage; CB stands in for it in the shared pointer checks.
  i8_status s = check_forward(reinterpret_cast<const i8_half*>(CB), CB, SCB, bias, M, N, K, threshold, out, true,
                              workspace, workspace_bytes, max_outlier_cols, &L);
  if (s != I8_OK) return s;
  return enqueue_matmul_dequant(CB, SCB, bias, M, N, K, threshold, out, workspace, max_outlier_cols, L,
                                reinterpret_cast<cudaStream_t>(stream));
}

i8_status i8_linear8bit_forward(const i8_half* X, const int8_t* CB, const float* SCB, const i8_half* bias, int M,
                                int N, int K, float threshold, i8_half* out, void* workspace,
                                size_t workspace_bytes, int max_outlier_cols, i8_stream_t stream) {
  WsLayout L;
  i8_status s = check_forward(X, CB, SCB, bias, M, N, K, threshold, out, true, workspace, workspace_bytes,
                              max_outlier_cols, &L);
  if (s != I8_OK) return s;
  return enqueue_forward(X, CB, SCB, bias, M, N, K, threshold, out, workspace, max_outlier_cols, L,
                         reinterpret_cast<cudaStream_t>(stream));
}

size_t i8_linear8bit_multi_workspace_size(int M, int K, int G, const int* N, int max_outlier_cols) {
  WsLayout L;
  if (max_outlier_cols > kMaxOutlierCap || !ws_layout_multi(M, K, G, N, max_outlier_cols, &L)) return 0;
  return L.total;
}

i8_status i8_linear8bit_forward_multi(const i8_half* X, int M, int K, int G, const int8_t* const* CB,
                                      const float* const* SCB, const i8_half* const* bias, const int* N,
                                      i8_half* const* out, float threshold, void* workspace, size_t workspace_bytes,
                                      int max_outlier_cols, i8_stream_t stream) {
  if (!X || !workspace || !CB || !SCB || !N || !out) return I8_ERR_INVALID_ARG;
  if (G < 1 || G > kMaxGroups) return I8_ERR_INVALID_ARG;
  const int cap = max_outlier_cols;
  WsLayout L;
  for (int g = 0; g < G; ++g) {
    // every weight passes the single-weight checks against the same X and workspace rules
    i8_status s = check_forward(X, CB[g], SCB[g], bias ? bias[g] : nullptr, M, N[g], K, threshold, out[g], true,
                                workspace, ~size_t(0), cap, &L);
    if (s != I8_OK) return s;
  }
  if (!ws_layout_multi(M, K, G, N, cap, &L)) return I8_ERR_INVALID_ARG;
  if (workspace_bytes < L.total) return I8_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // Every weight runs as its own forward would: small ones as the one-launch
  // kernel, the rest on X quantised (and its outlier columns found) once, the
  // first of them with its outlier rows gathered in the same launch.
  int first_big = -1;
  for (int g = 0; g < G && first_big < 0; ++g)
    if (!use_small(M, N[g], K, cap)) first_big = g;
  i8_status s = I8_OK;
  if (first_big >= 0) {
    s = enqueue_prepare(X, CB[first_big], M, N[first_big], K, threshold, workspace, cap, L, st);
    if (s != I8_OK) return s;
  }
  const WsPtrs w = ws_ptrs(workspace, L);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool gather_w = !L.decode && threshold > 0.f && cap > 0;
  const int sms = num_sms();
  if (sms <= 0) return I8_ERR_CUDA;
  for (int g = 0; g < G; ++g) {
    if (use_small(M, N[g], K, cap)) {
      // the status word is reset by the first operation of the call only
      const bool reset = first_big < 0 && g == 0;
      CUtensorMap tmW;
      if (!encode_2d(&tmW, CU_TENSOR_MAP_DATA_TYPE_UINT8, CB[g], K, N[g], K, 128, 128)) return I8_ERR_CUDA;
      s = cuda_status(i8lt::launch_linear_small(tmW, reinterpret_cast<const __half*>(X), M, N[g], K, threshold, cap,
                                                SCB[g], reinterpret_cast<const __half*>(bias ? bias[g] : nullptr),
                                                reinterpret_cast<__half*>(out[g]), w.hdr, kWaitLimitNs, reset, sms,
                                                st));
      if (s != I8_OK) return s;
      continue;
    }
    __half* WO = reinterpret_cast<__half*>(ws + wo_offset(L, N, g));
    int32_t* counters = reinterpret_cast<int32_t*>(ws + counters_offset(L, N, g));
    if (g != first_big && gather_w) {
      // this weight's outlier rows only: the list is rebuilt from the bitmap, X is not touched
      s = cuda_status(i8lt::launch_outlier_prepare(w.bitmap, K, cap, nullptr, nullptr, nullptr, nullptr, nullptr,
                                                   nullptr, 0, nullptr, CB[g], N[g], WO, L.ld_o, sms, st));
      if (s != I8_OK) return s;
    }
    s = enqueue_gemm(CB[g], SCB[g], bias ? bias[g] : nullptr, M, N[g], K, threshold, out[g], w, counters, WO, cap,
                     L, st);
    if (s != I8_OK) return s;
  }
  return I8_OK;
}

i8_status i8_read_status(const void* workspace, int32_t* count, i8_stream_t stream) {
  if (!workspace) return I8_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[3] = {0, 0, 0};
  if (cudaMemcpyAsync(h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return I8_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return I8_ERR_CUDA;
  if (count) *count = static_cast<int32_t>(h[2]);
  return static_cast<i8_status>(h[0]);
}

i8_status i8_selftest_bounded_wait(uint32_t* status, uint64_t limit_ns, i8_stream_t stream) {
  if (!status) return I8_ERR_INVALID_ARG;
  if (limit_ns < 1000000ull || limit_ns > 10000000000ull) return I8_ERR_INVALID_ARG;
  return cuda_status(i8lt::launch_selftest_wait(status, limit_ns, reinterpret_cast<cudaStream_t>(stream)));
}

i8_status i8_linear8bit_forward_static(const i8_half* X, const int8_t* CB, const float* SCB, const i8_half* bias,
                                       int M, int N, int K, float threshold, i8_half* out, int max_outlier_cols,
                                       uint32_t* status_out, i8_stream_t stream) {
  if (!X || !out || !SCB) return I8_ERR_INVALID_ARG;
  i8_status s = check_gemm_operands(X, CB, M, N, K);
  if (s != I8_OK) return s;
  if (check_threshold(threshold) != I8_OK || max_outlier_cols < 0) return I8_ERR_INVALID_ARG;
  if (max_outlier_cols > kMaxOutlierCap) return I8_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(out) || (bias && !aligned16(bias))) return I8_ERR_UNSUPPORTED_SHAPE;
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 3u) != 0) return I8_ERR_UNSUPPORTED_SHAPE;
  WsLayout L;
  if (!ws_layout(M, N, K, max_outlier_cols, &L)) return I8_ERR_INVALID_ARG;
  if (L.total > kStaticScratchBytes) return I8_ERR_WORKSPACE;  // needs more than the built-in 32 MiB
  void* ws = nullptr;
  s = static_scratch(&ws);
  if (s != I8_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the same kernels as i8_linear8bit_forward: the first of them clears (or
  // writes) the status word and counts; every other byte read back is written
  // earlier in the same call
  s = enqueue_forward(X, CB, SCB, bias, M, N, K, threshold, out, ws, max_outlier_cols, L, st);
  if (s != I8_OK || status_out == nullptr) return s;
  return cuda_status(cudaMemcpyAsync(status_out, ws, 3 * sizeof(uint32_t), cudaMemcpyDeviceToDevice, st));
}

}  // extern "C"
