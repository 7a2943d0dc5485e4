// Newton-Schulz orthogonalisation of one matrix without any allocation.
//
// Some callers cannot allocate device memory when they run this: for example a plugin or
// custom-call hook whose host framework owns every allocation and forbids cudaMalloc inside
// its execution callback, or a service that reserves all of its memory at start-up and must not
// allocate afterwards. muon_ns_orthogonalize grows a library workspace with cudaMalloc on first
// use, so those callers cannot use it. This entry point runs the same kernels on a fixed scratch
// area that is part of the library image (a file-scope __device__ array): the caller passes only
// the input and the output, and the call allocates nothing.
//
// Limits and behaviour:
//   - bf16 working precision, no zero-centring; min(m, n) <= 1024 and m * round_up(n, 8) <= 2^21.
//   - The scratch area (about 12.1 MiB) is reserved on every device that loads this library and
//     is held until the process exits.
//   - The first call on a device sets up that device (looks up the scratch address with
//     cudaGetSymbolAddress); make that first call before any stream capture.
//   - Every call uses the same scratch area, which keeps the previous call's contents; the
//     kernels overwrite everything they read, and the status word is cleared at each call. Calls
//     that overlap on the GPU (different streams, not ordered) race on the scratch area.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/muon.h"
#include "muon_internal.h"

namespace muon {

void set_error_message(const std::string& msg);
void note_launches(int64_t n);

namespace {

constexpr int64_t kNaMaxMinDim = 1024;
constexpr int64_t kNaMaxElems = int64_t(1) << 21;
constexpr size_t kNaXBytes = (size_t)kNaMaxElems * 2;
constexpr size_t kNaGramBytes = (size_t)kNaMaxMinDim * kNaMaxMinDim * 2;
constexpr size_t kNaOffX0 = 0;
constexpr size_t kNaOffX1 = kNaXBytes;
constexpr size_t kNaOffA = 2 * kNaXBytes;
constexpr size_t kNaOffB = kNaOffA + kNaGramBytes;
constexpr size_t kNaOffTables = kNaOffB + kNaGramBytes;
constexpr int kNaMaps = 12;     // 4 buffers (X0, X1, A, B) x 3 TMA views
constexpr int kNaProbs = 7;     // gram[2], poly, update-with-B[2], update-with-A[2]

// Per-call tables, written by na_tables_kernel from its by-value parameter.
struct NaHead {
  CUtensorMap maps[kNaMaps];
  GemmProblem probs[kNaProbs];
  MatInfo mat;
};

struct NaTables {
  NaHead head;
  float alpha;
  int status[2];
  float partials[kNaMaxElems / kChunk];
};

constexpr size_t kNaScratchBytes = (kNaOffTables + sizeof(NaTables) + 255) / 256 * 256;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaScratchBytes];

__global__ void na_tables_kernel(const __grid_constant__ NaHead head, NaTables* dst) {
  const uint64_t* src = reinterpret_cast<const uint64_t*>(&head);
  uint64_t* out = reinterpret_cast<uint64_t*>(&dst->head);
  for (size_t i = threadIdx.x; i < sizeof(NaHead) / 8; i += blockDim.x) out[i] = src[i];
  if (threadIdx.x == 0) {
    dst->status[0] = 0;
    dst->status[1] = 0;
  }
}

struct NaDevice {
  bool ready = false;
  char* base = nullptr;
  int sms = 0;
};
constexpr int kNaMaxDevices = 64;
NaDevice g_na[kNaMaxDevices];
std::mutex g_na_mu;

typedef CUresult (*PFN_encode_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                 CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                 CUtensorMapFloatOOBfill);

PFN_encode_t na_encode() {
  static PFN_encode_t fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encode_t>(p);
  }
  return fn;
}

int na_fail(int code, const std::string& msg) {
  set_error_message(msg);
  return code;
}

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// One-time set-up of the current device: checks it is an sm_100 part and looks up the device
// address of the scratch array (host code cannot use the array's name as a device address).
int na_setup(NaDevice** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return na_fail(MUON_ERR_UNSUPPORTED, std::string("no CUDA device: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kNaMaxDevices) return na_fail(MUON_ERR_UNSUPPORTED, "device index out of range");
  NaDevice& d = g_na[dev];
  if (!d.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return na_fail(MUON_ERR_CUDA, std::string("cudaGetDeviceProperties: ") + cudaGetErrorString(e));
    if (prop.major != 10) return na_fail(MUON_ERR_UNSUPPORTED, "this library runs on sm_100 (B200) devices only");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return na_fail(MUON_ERR_CUDA, std::string("cudaGetSymbolAddress(scratch): ") + cudaGetErrorString(e));
    d.base = static_cast<char*>(p);
    d.sms = prop.multiProcessorCount;
    d.ready = true;
  }
  *out = &d;
  return MUON_OK;
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" int muon_ns_orthogonalize_noalloc(const void* G, muon_dtype_t g_dtype, void* X,
                                             muon_dtype_t x_dtype, int64_t m, int64_t n, int steps,
                                             const muon_coeffs_t* coeffs, float eps, int* status,
                                             muon_stream_t stream) {
  // ---- arguments (checked before any device work)
  if (!G || !X) return na_fail(MUON_ERR_INVALID_ARG, "G and X must not be NULL");
  if (g_dtype != MUON_BF16 && g_dtype != MUON_FP32) return na_fail(MUON_ERR_INVALID_ARG, "g_dtype");
  if (x_dtype != MUON_BF16 && x_dtype != MUON_FP32) return na_fail(MUON_ERR_INVALID_ARG, "x_dtype");
  if (m <= 0 || n <= 0) return na_fail(MUON_ERR_INVALID_ARG, "m and n must be positive");
  if (!(eps >= 0.0f) || !std::isfinite(eps)) return na_fail(MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
  if (steps < 0 || steps > MUON_MAX_NS_STEPS)
    return na_fail(MUON_ERR_INVALID_ARG, "steps must be in [0, " + std::to_string(MUON_MAX_NS_STEPS) + "]");
  // m and n are bounded first, so that the products below cannot overflow
  const int64_t mn = std::min(m, n);
  const bool fits = m <= kNaMaxElems && n <= kNaMaxElems && mn <= kNaMaxMinDim &&
                    m * ((n + 7) / 8 * 8) <= kNaMaxElems;
  if (!fits)
    return na_fail(MUON_ERR_INVALID_ARG,
                   "matrix " + std::to_string(m) + "x" + std::to_string(n) +
                       " exceeds the fixed scratch of the no-allocation call (needs min(m, n) <= 1024 and "
                       "m * round_up(n, 8) <= 2097152); use muon_ns_orthogonalize");
  const int64_t ldx = (n + 7) / 8 * 8, ldm = (mn + 7) / 8 * 8;
  muon_coeffs_t co[MUON_MAX_NS_STEPS];
  for (int k = 0; k < steps; ++k) {
    co[k] = coeffs ? coeffs[k] : muon_coeffs_t{3.4445f, -4.7750f, 2.0315f};
    if (!std::isfinite(co[k].a) || !std::isfinite(co[k].b) || !std::isfinite(co[k].c))
      return na_fail(MUON_ERR_INVALID_ARG, "coefficients must be finite");
  }
  {
    const uintptr_t g0 = (uintptr_t)G, g1 = g0 + (uintptr_t)(m * n * (g_dtype == MUON_BF16 ? 2 : 4));
    const uintptr_t x0 = (uintptr_t)X, x1 = x0 + (uintptr_t)(m * n * (x_dtype == MUON_BF16 ? 2 : 4));
    if (g0 < x1 && x0 < g1) return na_fail(MUON_ERR_INVALID_ARG, "G and X overlap");
  }

  std::lock_guard<std::mutex> lk(g_na_mu);
  set_error_message("");
  NaDevice* d = nullptr;
  int rc = na_setup(&d);
  if (rc != MUON_OK) return rc;
  PFN_encode_t encode = na_encode();
  if (!encode) return na_fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");

  // ---- per-call tables, built on the host and written by one small kernel
  char* base = d->base;
  void* bufs[4] = {base + kNaOffX0, base + kNaOffX1, base + kNaOffA, base + kNaOffB};
  NaTables* tables = reinterpret_cast<NaTables*>(base + kNaOffTables);
  const bool tall = m > n;
  const int64_t nn = std::max(m, n);
  NaHead head;
  std::memset(&head, 0, sizeof(head));
  const int64_t rows_of[4] = {m, m, mn, mn}, cols_of[4] = {n, n, mn, mn}, ld_of[4] = {ldx, ldx, ldm, ldm};
  const int boxes[3] = {kTcBM, kTcBN, 64};
  for (int b = 0; b < 4; ++b) {
    for (int v = 0; v < 3; ++v) {
      cuuint64_t gdim[2] = {(cuuint64_t)cols_of[b], (cuuint64_t)rows_of[b]};
      cuuint64_t gstride[1] = {(cuuint64_t)(ld_of[b] * 2)};
      cuuint32_t box[2] = {64u, (cuuint32_t)boxes[v]};
      cuuint32_t estr[2] = {1u, 1u};
      CUresult r = encode(&head.maps[b * 3 + v], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, bufs[b], gdim, gstride,
                          box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return na_fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
    }
  }
  const CUtensorMap* dmaps = tables->head.maps;   // device addresses of the maps
  auto K128 = [&](int b) { return dmaps + b * 3 + 0; };
  auto K256 = [&](int b) { return dmaps + b * 3 + 1; };
  auto MN64 = [&](int b) { return dmaps + b * 3 + 2; };
  const float* alpha = &tables->alpha;
  uint32_t sym_tiles = 0;
  for (int64_t bi = 0; bi < cdiv(mn, kTcBM); ++bi) sym_tiles += (uint32_t)(cdiv(mn, kTcBN) - bi / 2);
  const uint32_t upd_tiles = (uint32_t)(cdiv(m, kTcBM) * cdiv(n, kTcBN));
  for (int p = 0; p < 2; ++p) {
    GemmProblem& g = head.probs[p];
    g.tma_a = tall ? MN64(p) : K128(p);
    g.tma_b = tall ? MN64(p) : K256(p);
    g.a_mn = g.b_mn = tall ? 1 : 0;
    g.d = static_cast<__nv_bfloat16*>(bufs[2]);
    g.ldd = ldm;
    g.alpha = alpha;
    g.M = g.N = (uint32_t)mn;
    g.K = (uint32_t)nn;
    g.tiles_m = (uint32_t)cdiv(mn, kTcBM);
    g.tiles_n = (uint32_t)cdiv(mn, kTcBN);
    g.sym = 1;
    g.n_tiles = sym_tiles;
    for (int which = 0; which < 2; ++which) {   // 0: multiply by B, 1: multiply by A (c = 0)
      GemmProblem& u = head.probs[3 + 2 * which + p];
      const int S = which == 0 ? 3 : 2;
      if (!tall) {
        u.tma_a = K128(S); u.a_mn = 0;
        u.tma_b = MN64(p); u.b_mn = 1;
      } else {
        u.tma_a = K128(p); u.a_mn = 0;
        u.tma_b = K256(S); u.b_mn = 0;
      }
      u.d = static_cast<__nv_bfloat16*>(bufs[1 - p]);
      u.ldd = ldx;
      u.c = static_cast<const __nv_bfloat16*>(bufs[p]);
      u.ldc = ldx;
      u.alpha = alpha;
      u.M = (uint32_t)m; u.N = (uint32_t)n; u.K = (uint32_t)mn;
      u.tiles_m = (uint32_t)cdiv(m, kTcBM);
      u.tiles_n = (uint32_t)cdiv(n, kTcBN);
      u.n_tiles = upd_tiles;
    }
  }
  GemmProblem& q = head.probs[2];
  q.tma_a = K128(2); q.tma_b = K256(2);
  q.d = static_cast<__nv_bfloat16*>(bufs[3]); q.ldd = ldm;
  q.c = static_cast<const __nv_bfloat16*>(bufs[2]); q.ldc = ldm;
  q.alpha = alpha;
  q.M = q.N = q.K = (uint32_t)mn;
  q.tiles_m = (uint32_t)cdiv(mn, kTcBM); q.tiles_n = (uint32_t)cdiv(mn, kTcBN);
  q.sym = 1;
  q.n_tiles = sym_tiles;
  MatInfo& mi = head.mat;
  mi.p = static_cast<float*>(X);
  mi.g = G;
  mi.m = nullptr;
  mi.x0 = bufs[0];
  mi.xf = bufs[steps & 1];
  mi.alpha = &tables->alpha;
  mi.rows = m; mi.cols = n; mi.ldx = ldx;
  mi.rms = 1.0f;
  mi.vec = (n % 8 == 0) && ((uintptr_t)G % 16 == 0) && ((uintptr_t)X % 16 == 0) ? 1 : 0;

  // ---- launches (all on the caller's stream)
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int* st = status ? status : tables->status;
  const MatInfo* dmat = &tables->head.mat;
  const int64_t chunks = cdiv(m * n, kChunk);
  int64_t launches = 0;
  cudaError_t e;
  na_tables_kernel<<<1, 256, 0, s>>>(head, tables);
  ++launches;
  e = cudaGetLastError();
  if (e == cudaSuccess) {
    e = launch_prologue(dmat, 1, chunks, g_dtype == MUON_BF16, 1, 0, 0.0f, 0, 0, tables->partials, st,
                        d->sms * 8, s);
    ++launches;
  }
  if (e == cudaSuccess) { e = launch_alpha(dmat, 1, tables->partials, eps, s); ++launches; }
  const GemmProblem* dprobs = tables->head.probs;
  for (int k = 0; k < steps && e == cudaSuccess; ++k) {
    const int p = k & 1, first = k == 0 ? 1 : 0;
    e = launch_gemm_tc(dprobs + p, 1, sym_tiles, EpiScalars{1.0f, 0.0f, first ? 2 : 0, 0}, st, d->sms, s);
    ++launches;
    if (e != cudaSuccess) break;
    if (co[k].c != 0.0f) {
      e = launch_gemm_tc(dprobs + 2, 1, sym_tiles, EpiScalars{co[k].c, co[k].b, 0, 0}, st, d->sms, s);
      ++launches;
      if (e != cudaSuccess) break;
      e = launch_gemm_tc(dprobs + 3 + p, 1, upd_tiles, EpiScalars{1.0f, co[k].a, first, first}, st, d->sms, s);
    } else {
      e = launch_gemm_tc(dprobs + 5 + p, 1, upd_tiles, EpiScalars{co[k].b, co[k].a, first, first}, st, d->sms, s);
    }
    ++launches;
  }
  if (e == cudaSuccess) {
    e = launch_output(dmat, 1, chunks, 1, x_dtype == MUON_BF16, steps == 0 ? 1 : 0, d->sms * 8, s);
    ++launches;
  }
  note_launches(launches);
  if (e != cudaSuccess) return na_fail(MUON_ERR_CUDA, std::string("launch failed: ") + cudaGetErrorString(e));
  return MUON_OK;
}
