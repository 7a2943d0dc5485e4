// C ABI of the Muon step (see include/muon.h): argument validation, the per-device plan
// (workspace layout, TMA descriptors, grouped problem tables) and the launch sequence.
//
// Launch sequence of one muon_step (all on the caller's stream, no host synchronisation once the
// plan exists), once per wave of matrices (see kWaveElements):
//   [column sums, column means]   only with zero-centring
//   prologue                      momentum, Nesterov, norm partials, U = cast(u)
//   norm                          alpha_j = 1 / (||u_j||_F + eps)
//   per Newton-Schulz iteration k (one grouped launch per phase covering the wave's matrices):
//     gram     A = X X^T                (k = 0: scaled by alpha^2, folding the normalisation)
//     poly     B = b_k A + c_k A A      (skipped when c_k = 0)
//     update   X' = a_k X + B X         (k = 0: scaled by alpha; c_k = 0: X' = a_k X + b_k A X)
//              the last update also applies p = p (1 - lr wd) - lr s O in its epilogue; a separate
//              epilogue kernel does it only when that cannot be fused (bf16 parameters that TMA
//              cannot view) or when steps = 0
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/muon.h"
#include "muon_internal.h"

namespace muon {

namespace {

thread_local std::string t_err;
std::mutex g_mu;
int64_t g_launches = 0;

int fail(int code, const std::string& msg) {
  t_err = msg;
  return code;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(MUON_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define MUON_CUDA(expr)                                   \
  do {                                                    \
    cudaError_t e_ = (expr);                              \
    if (e_ != cudaSuccess) return cuda_fail(e_, #expr);   \
  } while (0)

// ------------------------------------------------------------------ profiling
struct ProfRec {
  int kind;
  int sub;     // phase class of a Newton-Schulz launch, or -1
  cudaEvent_t a, b;
  double flops, exec;
};
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t get_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

template <class F>
cudaError_t timed_launch(int kind, cudaStream_t s, double flops, double exec, F&& launch, int sub = -1) {
  ++g_launches;
  if (!g_prof_on) return launch();
  ProfRec r{kind, sub, get_event(), get_event(), flops, exec};
  cudaEventRecord(r.a, s);
  cudaError_t e = launch();
  cudaEventRecord(r.b, s);
  g_prof.push_back(r);
  return e;
}

// ------------------------------------------------------------------ driver entry point
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled_t get_encode() {
  static PFN_encodeTiled_t fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled_t>(p);
  }
  return fn;
}

// Per-call tables are written in 8-byte words (write_table).
static_assert(sizeof(MatInfo) % 8 == 0 && sizeof(AdamTensor) % 8 == 0, "table rows are 8-byte words");
static_assert(sizeof(GemmProblem) % 8 == 0 && sizeof(GemmProblemX3) % 8 == 0, "table rows are 8-byte words");
static_assert(sizeof(CUtensorMap) % 8 == 0, "table rows are 8-byte words");

// ------------------------------------------------------------------ plan
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

struct Shape {
  int64_t r, c;
  bool operator==(const Shape& o) const { return r == o.r && c == o.c; }
};

struct BufMaps {   // TMA views of one bf16 buffer: operand loads and the epilogue's store view
  int k128 = -1, mn64 = -1, st32 = -1;
};

struct BufMapsX3 {   // TMA views of one two-plane fp32 buffer: K-major and MN-major operand loads
  int k128 = -1, mn32 = -1;
};

// Matrices are processed in waves: consecutive runs of matrices of at most kWaveElements elements
// in total (a larger matrix is a wave of its own). Each wave runs its own prologue, norm and
// Newton-Schulz launches. Within one launch over a few hundred million elements, the output of
// one phase (A, B, the new iterate) is partly still in L2 when the next phase reads it; launches
// over the whole Llama-8B set (7e9 elements) measured 12-25 % slower per step under the power
// cap (lower SM clock at the same board power), with per-wave launch tails costing about 3 %.
constexpr int64_t kWaveElements = int64_t(1) << 29;
int64_t g_wave_elements = kWaveElements;   // muon_set_wave_elements
uint64_t g_wait_ns = 0;                     // muon_set_wait_limit_ns (0: the kernels' default)
// Chained launches (muon_set_chained_launch): a wave whose products all run on 256 x 256 bf16
// tiles may run its whole Newton-Schulz iteration (every phase of every step) as one launch.
// Mode 0: never; 1 (default): when one iteration has at most kChainTilesPerPair tiles per CTA
// pair, where the per-phase launches' fixed costs dominate (a single 256 x 512 matrix 0.31 ->
// 0.18 ms, the cubic 12-matrix set 0.50 -> 0.38 ms), while waves with 25-30 tiles per pair per
// iteration (GPT-2-small, Mamba) measured 2-4 % faster per phase; 2: always.
int g_chain_mode = 1;
constexpr uint32_t kChainTilesPerPair = 8;
constexpr int kMaxChainPhases = 3 * MUON_MAX_NS_STEPS;

// A wave: matrices [j0, j1) of the plan. Every prefix sum in the device tables (elementwise
// chunks, column-sum items, product tiles) restarts at zero at the wave's first matrix, so a
// wave's launches take the table sub-ranges starting at j0 and need no offsets.
struct Wave {
  int j0 = 0, j1 = 0;
  bool wide = false;   // bf16 Gram and update products on 256 x 512 tiles (see build_plan)
  bool chain = false;  // bf16: the iteration runs as one chained launch (g_chain_mode)
  int64_t n_chunks = 0, cs_items = 0, cm_items = 0;
  uint32_t tiles_gram = 0, tiles_poly = 0, tiles_upd = 0;
  double fl_gram = 0, fl_poly = 0, fl_upd = 0;      // nominal flops per launch
  double ex_gram = 0, ex_poly = 0, ex_upd = 0;      // executed (tile) flops per launch
};

// A plan: the layout of one list of shapes (in one working precision and wave budget), its TMA
// descriptors and grouped problem tables. Its tables live in a small allocation of its own; the
// per-wave buffers (iterates, A, B, column-mean scratch, norm partials) live in the device's
// shared buffer arena, which every plan reuses (calls are ordered on the GPU). A plan is valid
// for the arena generation it was built against.
struct Plan {
  std::vector<Shape> shapes;
  int x_bf16 = 1;
  int64_t wave_elements = 0;
  int chain_mode = 1;        // g_chain_mode the plan was built with
  uint64_t arena_gen = 0;
  char* tab = nullptr;       // this plan's tables (cudaMalloc)
  size_t tab_bytes = 0;
  // device tables
  MatInfo* d_mats = nullptr;
  float* d_partials = nullptr;
  std::vector<Wave> waves;
  // per-matrix workspace pointers
  std::vector<void*> x0, x1, A, B;
  std::vector<float*> colmean, colpart, alpha;
  std::vector<int64_t> ldx, ldm;
  // grouped problems
  void* d_gram[2] = {nullptr, nullptr};
  void* d_poly = nullptr;
  void* d_updB[2] = {nullptr, nullptr};
  void* d_updA[2] = {nullptr, nullptr};
  // per-call MatInfo table (written through kernel parameters when it changes)
  std::vector<MatInfo> last_uploaded;
  bool uploaded_once = false;
  // fused last update (tensor-core path): host copies of the update problems, and the per-call
  // table of the last iteration's update problems with TMA views of the caller's parameters
  std::vector<GemmProblem> h_upd[2][2];    // [operand: 0 B, 1 A][parity]
  std::vector<GemmProblemX3> h_upd_x3[2][2];   // the same for the fp32 (3xTF32) mode
  CUtensorMap* d_pmaps = nullptr;
  // chained launches (bf16 waves on 256 x 256 tiles): per-matrix completion targets of the Gram,
  // poly and update phases (eight epilogue warps per tile), the claim and completion counters,
  // and each wave's phase list (rewritten when it changes)
  uint32_t* d_tgt[3] = {nullptr, nullptr, nullptr};
  uint32_t* d_chain_ctr = nullptr;
  PhaseDesc* d_phases = nullptr;
  std::vector<std::vector<PhaseDesc>> last_phases;   // per wave
  void* d_fused = nullptr;                 // GemmProblem (bf16) or GemmProblemX3 (fp32) table
  std::vector<uint8_t> fused_key;

  ~Plan() {
    if (tab) cudaFree(tab);
  }
};

// Plans kept per device (most recently used first). Each holds only its tables (about 2.5 KB per
// matrix); the buffers are shared.
constexpr size_t kMaxPlans = 16;

// Per-device table of an AdamW call: one AdamTensor per tensor, rewritten (through kernel
// parameters) only when the pointers change.
struct AdamPlan {
  std::vector<int64_t> numel;
  AdamTensor* d_tab = nullptr;
  std::vector<AdamTensor> last;
  bool uploaded = false;
  int64_t n_chunks = 0;
  ~AdamPlan() {
    if (d_tab) cudaFree(d_tab);
  }
};

struct DeviceState {
  std::unique_ptr<AdamPlan> adam;
  std::vector<std::unique_ptr<Plan>> plans;   // most recently used first
  char* arena = nullptr;                      // per-wave buffers shared by every plan
  size_t arena_bytes = 0;
  uint64_t arena_gen = 0;                     // bumped whenever the arena moves
  int* d_status = nullptr;  // [0] flags, [1] non-finite count
  int sms = 0;
  int cc_major = 0;
  int pair_capacity = 0;   // resident CTA pairs of the paired tensor-core kernel
  int x3_capacity = 0;     // resident CTA pairs of the 3xTF32 kernel
};

std::map<int, DeviceState> g_dev;

int device_state(DeviceState** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(MUON_ERR_UNSUPPORTED, std::string("no CUDA device: ") + cudaGetErrorString(e));
  DeviceState& ds = g_dev[dev];
  if (ds.sms == 0) {
    cudaDeviceProp prop;
    MUON_CUDA(cudaGetDeviceProperties(&prop, dev));
    ds.sms = prop.multiProcessorCount;
    ds.cc_major = prop.major;
  }
  if (ds.cc_major != 10)
    return fail(MUON_ERR_UNSUPPORTED, "this library runs on sm_100 (B200) devices only");
  if (ds.pair_capacity == 0) ds.pair_capacity = gemm_tc_pair_capacity(ds.sms);
  if (ds.x3_capacity == 0) ds.x3_capacity = gemm_x3_pair_capacity(ds.sms);
  if (!ds.d_status) {
    MUON_CUDA(cudaMalloc(&ds.d_status, 2 * sizeof(int)));
    MUON_CUDA(cudaMemset(ds.d_status, 0, 2 * sizeof(int)));
  }
  *out = &ds;
  return MUON_OK;
}

// Orders the Gram problems of each wave of small matrices (256 x 256 tiles) by descending
// contraction length K (stable), for per-phase launches. Such a launch hands out tiles
// round-robin over the CTA pairs in table order; a wave's Gram tiles differ in K (the longer side
// of each matrix, up to 4x between the matrices of one model), so placing the longest tiles
// first evens out the pairs' loads. Waves of large matrices (256 x 512 tiles, ten or more tiles
// per pair) keep the matrix order, which measured faster there, and so do chained waves: they
// balance by claiming tiles as they go, and a Gram product in another order than the update it
// waits for would start with the matrices whose updates finish last.
template <class Prob>
void order_gram_by_k(std::vector<Prob>& probs, const std::vector<Wave>& waves) {
  for (const Wave& w : waves) {
    if (w.wide || w.chain) continue;
    std::stable_sort(probs.begin() + w.j0, probs.begin() + w.j1,
                     [](const Prob& a, const Prob& b) { return a.K > b.K; });
    uint32_t t = 0;
    for (int j = w.j0; j < w.j1; ++j) {
      probs[j].tile_begin = t;
      t += probs[j].n_tiles;
    }
  }
}

// Finds or builds the plan (TMA descriptors, grouped problem tables, buffer layout) of a list of
// shapes, growing the shared buffer arena when the plan needs more than it holds.
int build_plan(DeviceState& ds, const std::vector<Shape>& shapes, int x_bf16, Plan** out) {
  for (size_t i = 0; i < ds.plans.size(); ++i) {
    const Plan& q = *ds.plans[i];
    if (q.shapes == shapes && q.x_bf16 == x_bf16 && q.wave_elements == g_wave_elements &&
        q.chain_mode == g_chain_mode && q.arena_gen == ds.arena_gen) {
      if (i > 0) std::rotate(ds.plans.begin(), ds.plans.begin() + i, ds.plans.begin() + i + 1);
      *out = ds.plans[0].get();
      return MUON_OK;
    }
  }
  std::unique_ptr<Plan> P(new Plan());
  P->shapes = shapes;
  P->x_bf16 = x_bf16;
  P->wave_elements = g_wave_elements;
  P->chain_mode = g_chain_mode;
  const int n = (int)shapes.size();
  // bf16 mode: one bf16 plane per buffer; fp32 mode: hi and lo fp32 planes (GemmProblemX3)
  const size_t esz = x_bf16 ? 2 : 8;
  const size_t AL = 256;

  // ---- waves
  std::vector<int> wave_of(n);
  {
    int64_t acc = 0;
    for (int j = 0; j < n; ++j) {
      const int64_t el = shapes[j].r * shapes[j].c;
      if (j == 0 || acc + el > P->wave_elements) {
        P->waves.emplace_back();
        P->waves.back().j0 = j;
        acc = 0;
      }
      acc += el;
      P->waves.back().j1 = j + 1;
      wave_of[j] = (int)P->waves.size() - 1;
    }
  }
  auto wave_start = [&](int j) { return P->waves[wave_of[j]].j0 == j; };
  // Tile width of a wave's Gram and update products (bf16). The 256 x 512 tile reads a quarter
  // fewer operand bytes per FLOP, which pays for large matrices (Llama-8B step 15 % faster), but on
  // small ones its column padding and the halved tile count (load balance over the CTA pairs)
  // cost more (GPT-2-small and Mamba steps 25 % slower). Wide tiles are used when matrices with
  // min(rows, cols) >= 2048 carry at least 80 % of the wave's Newton-Schulz FLOPs.
  for (Wave& w : P->waves) {
    double big = 0.0, all = 0.0;
    for (int j = w.j0; j < w.j1; ++j) {
      const double m = (double)std::min(shapes[j].r, shapes[j].c), nn = (double)std::max(shapes[j].r, shapes[j].c);
      const double f = m * m * nn;
      all += f;
      if (m >= 2048) big += f;
    }
    w.wide = all > 0.0 && big >= 0.8 * all;
  }

  // ---- layout
  // The per-matrix buffers (X0, X1, A, B, column-mean scratch) of one wave are laid out from the
  // start of the workspace; the next wave reuses the same region, since waves run one after the
  // other in stream order. The region is as large as the largest wave.
  size_t off = 0, wave_region = 0;
  std::vector<size_t> o_x0(n), o_x1(n), o_A(n), o_B(n), o_cm(n), o_cp(n);
  P->ldx.resize(n);
  P->ldm.resize(n);
  int64_t chunks = 0, cs = 0, cm = 0, max_chunks = 0;
  std::vector<MatInfo> mats(n);
  for (int j = 0; j < n; ++j) {
    if (wave_start(j)) {
      chunks = cs = cm = 0;
      off = 0;
    }
    const int64_t r = shapes[j].r, c = shapes[j].c, m = std::min(r, c);
    const int64_t ldx = align_up(c, 8), ldm = align_up(m, 8);
    P->ldx[j] = ldx;
    P->ldm[j] = ldm;
    o_x0[j] = off; off = align_up(off + (size_t)r * ldx * esz, AL);
    o_x1[j] = off; off = align_up(off + (size_t)r * ldx * esz, AL);
    o_A[j] = off; off = align_up(off + (size_t)m * ldm * esz, AL);
    o_B[j] = off; off = align_up(off + (size_t)m * ldm * esz, AL);
    o_cm[j] = off; off = align_up(off + (size_t)c * 4, AL);
    const int64_t n_rc = ceil_div(r, kCsRows), n_cb = ceil_div(c, kCsCols);
    o_cp[j] = off; off = align_up(off + (size_t)n_rc * c * 4, AL);
    wave_region = std::max(wave_region, off);
    MatInfo& mi = mats[j];
    std::memset(&mi, 0, sizeof(mi));
    mi.rows = r; mi.cols = c; mi.ldx = ldx;
    mi.xlo = x_bf16 ? 0 : r * ldx;
    mi.chunk_begin = chunks; chunks += ceil_div(r * c, kChunk);
    mi.cs_begin = cs; cs += n_rc * n_cb;
    mi.cm_begin = cm; cm += n_cb;
    Wave& w = P->waves[wave_of[j]];
    w.n_chunks = chunks;
    w.cs_items = cs;
    w.cm_items = cm;
    max_chunks = std::max(max_chunks, chunks);
  }
  // the arena: the wave region, then the norm partials of one wave
  const size_t o_part = wave_region;
  const size_t arena_need = align_up(o_part + (size_t)max_chunks * 4, AL);
  // the plan's own tables
  off = 0;
  const size_t o_alpha = off; off = align_up(off + (size_t)n * 4, AL);
  const size_t o_mats = off; off = align_up(off + (size_t)n * sizeof(MatInfo), AL);
  const int maps_per = x_bf16 ? 12 : 8;   // 4 buffers x 3 views (bf16) or x 2 views (fp32)
  const size_t o_maps = off;
  off = align_up(off + (size_t)n * maps_per * sizeof(CUtensorMap), AL);
  const size_t prob_sz = x_bf16 ? sizeof(GemmProblem) : sizeof(GemmProblemX3);
  size_t o_prob[7];
  for (int k = 0; k < 7; ++k) { o_prob[k] = off; off = align_up(off + (size_t)n * prob_sz, AL); }
  const size_t o_pmaps = off;
  if (x_bf16) off = align_up(off + (size_t)n * sizeof(CUtensorMap), AL);
  const size_t o_fused = off;
  off = align_up(off + (size_t)n * prob_sz, AL);
  const size_t o_tgt = off;
  off = align_up(off + 3 * (size_t)n * 4, AL);
  const size_t o_ctr = off;
  off = align_up(off + (1 + (size_t)kMaxChainPhases * n) * 4, AL);
  const size_t o_phases = off;
  off = align_up(off + P->waves.size() * (size_t)kMaxChainPhases * sizeof(PhaseDesc), AL);
  P->tab_bytes = off;

  auto alloc_fail = [](cudaError_t e, const char* what, size_t bytes) {
    cudaGetLastError();
    char buf[200];
    snprintf(buf, sizeof(buf), "%s allocation of %.3f GB failed: %s", what, bytes / 1e9, cudaGetErrorString(e));
    return fail(MUON_ERR_WORKSPACE, buf);
  };
  if (arena_need > ds.arena_bytes) {
    // every cached plan points into the arena that moves: drop them (cudaFree synchronises)
    ds.plans.clear();
    if (ds.arena) cudaFree(ds.arena);
    ds.arena = nullptr;
    ds.arena_bytes = 0;
    ++ds.arena_gen;
    cudaError_t e = cudaMalloc(&ds.arena, arena_need);
    if (e != cudaSuccess) {
      ds.arena = nullptr;
      return alloc_fail(e, "workspace", arena_need);
    }
    ds.arena_bytes = arena_need;
  }
  if (ds.plans.size() >= kMaxPlans) ds.plans.pop_back();   // least recently used
  cudaError_t e = cudaMalloc(&P->tab, P->tab_bytes);
  if (e != cudaSuccess) {
    P->tab = nullptr;
    return alloc_fail(e, "plan table", P->tab_bytes);
  }
  P->arena_gen = ds.arena_gen;
  char* W = ds.arena;   // buffers
  char* T = P->tab;     // tables
  P->d_partials = reinterpret_cast<float*>(W + o_part);
  P->d_mats = reinterpret_cast<MatInfo*>(T + o_mats);
  for (int k = 0; k < 3; ++k) P->d_tgt[k] = reinterpret_cast<uint32_t*>(T + o_tgt) + (size_t)k * n;
  P->d_chain_ctr = reinterpret_cast<uint32_t*>(T + o_ctr);
  P->d_phases = reinterpret_cast<PhaseDesc*>(T + o_phases);
  P->last_phases.assign(P->waves.size(), {});
  for (int j = 0; j < n; ++j) {
    P->x0.push_back(W + o_x0[j]);
    P->x1.push_back(W + o_x1[j]);
    P->A.push_back(W + o_A[j]);
    P->B.push_back(W + o_B[j]);
    P->colmean.push_back(reinterpret_cast<float*>(W + o_cm[j]));
    P->colpart.push_back(reinterpret_cast<float*>(W + o_cp[j]));
    P->alpha.push_back(reinterpret_cast<float*>(T + o_alpha) + j);
  }

  // ---- grouped problems
  // CTA-pair tiles are 256 x 256; a symmetric m x m product computes the T (T + 1) / 2 tiles on or
  // above the diagonal, T = ceil(m / 256).
  auto sym_tiles = [](int64_t m) {
    const int64_t t = ceil_div(m, kTcPairBM);
    return t * (t + 1) / 2;
  };
  // the same on wide tiles (256 x 512): row block bi starts at column block (256 bi) / 512
  auto sym_tiles_wide = [](int64_t m) {
    const int64_t tm = ceil_div(m, kTcPairBM), tn = ceil_div(m, kTcWideBN);
    int64_t t = 0;
    for (int64_t bi = 0; bi < tm; ++bi) t += tn - (bi * kTcPairBM) / kTcWideBN;
    return t;
  };
  if (x_bf16) {
    PFN_encodeTiled_t encode = get_encode();
    if (!encode) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    std::vector<CUtensorMap> maps((size_t)n * maps_per);
    CUtensorMap* d_maps = reinterpret_cast<CUtensorMap*>(T + o_maps);
    int bad = 0;
    // views: 64-wide K-major boxes of 128 rows and 64 x 64 MN-major boxes (128-byte swizzle,
    // operand loads of one CTA of a pair), and 32 x 32 boxes with the 64-byte swizzle (epilogue
    // loads and stores)
    auto make3 = [&](int j, int slot, void* base, int64_t rows, int64_t cols, int64_t ld) {
      BufMaps bm;
      const cuuint32_t bx[3] = {64u, 64u, 32u}, by[3] = {(cuuint32_t)kTcBM, 64u, 32u};
      const CUtensorMapSwizzle sw[3] = {CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_SWIZZLE_128B,
                                        CU_TENSOR_MAP_SWIZZLE_64B};
      int* dst[3] = {&bm.k128, &bm.mn64, &bm.st32};
      for (int b = 0; b < 3; ++b) {
        const int idx = j * maps_per + slot * 3 + b;
        cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
        cuuint64_t gstride[1] = {(cuuint64_t)(ld * 2)};
        cuuint32_t box[2] = {bx[b], by[b]};
        cuuint32_t estr[2] = {1u, 1u};
        CUresult r = encode(&maps[idx], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, gdim, gstride, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw[b],
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) bad = (int)r;
        *dst[b] = idx;
      }
      return bm;
    };
    std::vector<GemmProblem> gram[2], poly, updB[2], updA[2];
    uint32_t tg = 0, tp = 0, tu = 0;
    for (int j = 0; j < n; ++j) {
      if (wave_start(j)) tg = tp = tu = 0;
      Wave& w = P->waves[wave_of[j]];
      const int64_t r = shapes[j].r, c = shapes[j].c, m = std::min(r, c), nn = std::max(r, c);
      const bool tall = r > c;
      BufMaps mx[2] = {make3(j, 0, P->x0[j], r, c, P->ldx[j]), make3(j, 1, P->x1[j], r, c, P->ldx[j])};
      BufMaps mA = make3(j, 2, P->A[j], m, m, P->ldm[j]);
      BufMaps mB = make3(j, 3, P->B[j], m, m, P->ldm[j]);
      auto M_ = [&](int idx) { return d_maps + idx; };
      for (int p = 0; p < 2; ++p) {
        GemmProblem g{};
        g.tma_a = M_(tall ? mx[p].mn64 : mx[p].k128);
        g.tma_b = M_(tall ? mx[p].mn64 : mx[p].k128);
        g.a_mn = g.b_mn = tall ? 1 : 0;
        g.d = static_cast<__nv_bfloat16*>(P->A[j]);
        g.ldd = P->ldm[j];
        g.tma_d = M_(mA.st32);
        g.alpha = P->alpha[j];
        g.M = g.N = (uint32_t)m;
        g.K = (uint32_t)nn;
        g.tiles_m = (uint32_t)ceil_div(m, kTcPairBM);
        g.tiles_n = (uint32_t)ceil_div(m, w.wide ? kTcWideBN : kTcBN);
        g.sym = w.wide ? 1 : 2;   // A whole (mirrored writes) or in the upper-block form
        g.mat = (uint32_t)j;
        g.n_tiles = (uint32_t)(w.wide ? sym_tiles_wide(m) : sym_tiles(m));
        g.tile_begin = tg;
        gram[p].push_back(g);
        for (int which = 0; which < 2; ++which) {   // 0: operand B, 1: operand A
          const BufMaps& mS = which == 0 ? mB : mA;
          GemmProblem u{};
          // B (or A) in the upper-block form: K slices below its diagonal blocks are read
          // transposed through its MN-major view
          const uint32_t half = w.wide ? 0 : 1;
          if (!tall) {
            u.tma_a = M_(mS.k128); u.a_mn = 0;
            u.tma_a_t = M_(mS.mn64); u.a_half = half;
            u.tma_b = M_(mx[p].mn64); u.b_mn = 1;
          } else {
            u.tma_a = M_(mx[p].k128); u.a_mn = 0;
            u.tma_b = M_(mS.k128); u.b_mn = 0;
            u.tma_b_t = M_(mS.mn64); u.b_half = half;
          }
          u.d = static_cast<__nv_bfloat16*>(p == 0 ? P->x1[j] : P->x0[j]);
          u.ldd = P->ldx[j];
          u.tma_d = M_(mx[1 - p].st32);
          u.alpha = P->alpha[j];
          u.M = (uint32_t)r; u.N = (uint32_t)c; u.K = (uint32_t)m;
          u.mat = (uint32_t)j;
          u.tiles_m = (uint32_t)ceil_div(r, kTcPairBM);
          u.tiles_n = (uint32_t)ceil_div(c, w.wide ? kTcWideBN : kTcBN);
          u.n_tiles = u.tiles_m * u.tiles_n;
          u.tile_begin = tu;
          (which == 0 ? updB[p] : updA[p]).push_back(u);
        }
      }
      GemmProblem q{};
      // B = c A A + b A (+ a I on the tensor-core path): A is symmetric, so A A = A A^T; A and B
      // are in the upper-block form
      q.tma_a = M_(mA.k128); q.tma_b = M_(mA.k128);
      q.tma_a_t = M_(mA.mn64); q.tma_b_t = M_(mA.mn64);
      q.a_half = q.b_half = w.wide ? 0 : 1;
      q.mat = (uint32_t)j;
      q.d = static_cast<__nv_bfloat16*>(P->B[j]); q.ldd = P->ldm[j];
      q.tma_d = M_(mB.st32);
      q.tma_c = M_(mA.st32);
      q.alpha = P->alpha[j];
      q.M = q.N = q.K = (uint32_t)m;
      // the polynomial product (K = m) stays on 256 x 256 tiles: its triangle wastes less there
      q.tiles_m = (uint32_t)ceil_div(m, kTcPairBM); q.tiles_n = (uint32_t)ceil_div(m, kTcBN);
      q.sym = w.wide ? 1 : 2;
      q.n_tiles = (uint32_t)sym_tiles(m);
      q.tile_begin = tp;
      poly.push_back(q);
      tg += gram[0].back().n_tiles;
      tp += q.n_tiles;
      tu += updB[0].back().n_tiles;
      w.tiles_gram = tg; w.tiles_poly = tp; w.tiles_upd = tu;
      w.fl_gram += 2.0 * m * m * nn;
      w.fl_poly += 2.0 * m * m * m;
      w.fl_upd += 2.0 * m * m * nn;
      const double tile_fl = 2.0 * kTcPairBM * kTcBN, gu_fl = 2.0 * kTcPairBM * (w.wide ? kTcWideBN : kTcBN);
      w.ex_gram += gu_fl * gram[0].back().n_tiles * (double)(ceil_div(nn, kTcBK) * kTcBK);
      w.ex_poly += tile_fl * q.n_tiles * (double)(ceil_div(m, kTcBK) * kTcBK);
      w.ex_upd += gu_fl * updB[0].back().n_tiles * (double)(ceil_div(m, kTcBK) * kTcBK);
    }
    if (bad) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string(bad));
    MUON_CUDA(cudaMemcpy(d_maps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice));
    {
      // completion targets of a chained launch: eight epilogue warps per tile of each matrix
      std::vector<uint32_t> tgt(3 * (size_t)n);
      for (int j = 0; j < n; ++j) {
        tgt[j] = 8u * gram[0][j].n_tiles;
        tgt[n + j] = 8u * poly[j].n_tiles;
        tgt[2 * (size_t)n + j] = 8u * updB[0][j].n_tiles;
      }
      MUON_CUDA(cudaMemcpy(P->d_tgt[0], tgt.data(), tgt.size() * 4, cudaMemcpyHostToDevice));
    }
    // chained waves: small enough per iteration, and few enough matrices for the 16-bit index
    for (Wave& w : P->waves) {
      const uint32_t tiles = w.tiles_gram + w.tiles_poly + w.tiles_upd;
      w.chain = !w.wide && n <= 65535 &&
                (g_chain_mode == 2 ||
                 (g_chain_mode == 1 && tiles <= kChainTilesPerPair * (uint32_t)std::max(1, ds.pair_capacity)));
    }
    order_gram_by_k(gram[0], P->waves);
    order_gram_by_k(gram[1], P->waves);
    std::vector<GemmProblem>* lists[7] = {&gram[0], &gram[1], &poly, &updB[0], &updB[1], &updA[0], &updA[1]};
    void** dsts[7] = {&P->d_gram[0], &P->d_gram[1], &P->d_poly, &P->d_updB[0], &P->d_updB[1],
                      &P->d_updA[0], &P->d_updA[1]};
    for (int k = 0; k < 7; ++k) {
      *dsts[k] = T + o_prob[k];
      MUON_CUDA(cudaMemcpy(*dsts[k], lists[k]->data(), lists[k]->size() * sizeof(GemmProblem),
                           cudaMemcpyHostToDevice));
    }
    P->h_upd[0][0] = updB[0]; P->h_upd[0][1] = updB[1];
    P->h_upd[1][0] = updA[0]; P->h_upd[1][1] = updA[1];
    P->d_pmaps = reinterpret_cast<CUtensorMap*>(T + o_pmaps);
    P->d_fused = T + o_fused;
  } else {
    PFN_encodeTiled_t encode = get_encode();
    if (!encode) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    std::vector<CUtensorMap> maps((size_t)n * maps_per);
    CUtensorMap* d_maps = reinterpret_cast<CUtensorMap*>(T + o_maps);
    int bad = 0;
    // 3-D views (columns, rows, plane) of a two-plane fp32 buffer, one plane per box: 32-wide
    // K-major boxes of 128 rows (128-byte swizzle) and 32 x 32 MN-major boxes (128-byte swizzle
    // over 32-byte granules, the layout tcgen05 reads MN-major tf32 operands in)
    auto make2 = [&](int j, int slot, void* base, int64_t rows, int64_t cols, int64_t ld) {
      BufMapsX3 bm;
      const cuuint32_t by[2] = {(cuuint32_t)kTcBM, 32u};
      const CUtensorMapSwizzle sw[2] = {CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B};
      int* dst[2] = {&bm.k128, &bm.mn32};
      for (int b = 0; b < 2; ++b) {
        const int idx = j * maps_per + slot * 2 + b;
        cuuint64_t gdim[3] = {(cuuint64_t)cols, (cuuint64_t)rows, 2};
        cuuint64_t gstride[2] = {(cuuint64_t)(ld * 4), (cuuint64_t)(rows * ld * 4)};
        cuuint32_t box[3] = {(cuuint32_t)kX3BK, by[b], 1u};
        cuuint32_t estr[3] = {1u, 1u, 1u};
        CUresult r = encode(&maps[idx], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, gdim, gstride, box,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw[b],
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) bad = (int)r;
        *dst[b] = idx;
      }
      return bm;
    };
    std::vector<GemmProblemX3> gram[2], poly, updB[2], updA[2];
    uint32_t tg = 0, tp = 0, tu = 0;
    for (int j = 0; j < n; ++j) {
      if (wave_start(j)) tg = tp = tu = 0;
      Wave& w = P->waves[wave_of[j]];
      const int64_t r = shapes[j].r, c = shapes[j].c, m = std::min(r, c), nn = std::max(r, c);
      const bool tall = r > c;
      const int64_t ldx = P->ldx[j], ldm = P->ldm[j];
      float* X[2] = {static_cast<float*>(P->x0[j]), static_cast<float*>(P->x1[j])};
      float* A = static_cast<float*>(P->A[j]);
      float* B = static_cast<float*>(P->B[j]);
      BufMapsX3 mx[2] = {make2(j, 0, X[0], r, c, ldx), make2(j, 1, X[1], r, c, ldx)};
      BufMapsX3 mA = make2(j, 2, A, m, m, ldm);
      BufMapsX3 mB = make2(j, 3, B, m, m, ldm);
      auto M_ = [&](int idx) { return d_maps + idx; };
      for (int p = 0; p < 2; ++p) {
        GemmProblemX3 g{};
        g.tma_a = g.tma_b = M_(tall ? mx[p].mn32 : mx[p].k128);
        g.a_mn = g.b_mn = tall ? 1 : 0;
        g.d = A; g.ldd = ldm; g.d_plane = m * ldm;
        g.alpha = P->alpha[j];
        g.M = g.N = (uint32_t)m; g.K = (uint32_t)nn;
        g.tiles_m = (uint32_t)ceil_div(m, kTcPairBM); g.tiles_n = (uint32_t)ceil_div(m, kTcBN);
        g.sym = 1;
        g.n_tiles = (uint32_t)sym_tiles(m);
        g.tile_begin = tg;
        gram[p].push_back(g);
        for (int which = 0; which < 2; ++which) {   // 0: operand B, 1: operand A
          const BufMapsX3& mS = which == 0 ? mB : mA;
          GemmProblemX3 u{};
          if (!tall) {
            u.tma_a = M_(mS.k128); u.a_mn = 0;
            u.tma_b = M_(mx[p].mn32); u.b_mn = 1;
          } else {
            u.tma_a = M_(mx[p].k128); u.a_mn = 0;
            u.tma_b = M_(mS.k128); u.b_mn = 0;
          }
          u.d = X[1 - p]; u.ldd = ldx; u.d_plane = r * ldx;
          u.c = X[p]; u.ldc = ldx; u.c_plane = r * ldx;
          u.alpha = P->alpha[j];
          u.M = (uint32_t)r; u.N = (uint32_t)c; u.K = (uint32_t)m;
          u.tiles_m = (uint32_t)ceil_div(r, kTcPairBM); u.tiles_n = (uint32_t)ceil_div(c, kTcBN);
          u.n_tiles = u.tiles_m * u.tiles_n;
          u.tile_begin = tu;
          (which == 0 ? updB[p] : updA[p]).push_back(u);
        }
      }
      GemmProblemX3 q{};
      // B = c A A + b A: A is symmetric, so A A = A A^T
      q.tma_a = q.tma_b = M_(mA.k128);
      q.d = B; q.ldd = ldm; q.d_plane = m * ldm;
      q.c = A; q.ldc = ldm; q.c_plane = m * ldm;
      q.alpha = P->alpha[j];
      q.M = q.N = q.K = (uint32_t)m;
      q.tiles_m = (uint32_t)ceil_div(m, kTcPairBM); q.tiles_n = (uint32_t)ceil_div(m, kTcBN);
      q.sym = 1;
      q.n_tiles = (uint32_t)sym_tiles(m);
      q.tile_begin = tp;
      poly.push_back(q);
      tg += gram[0].back().n_tiles;
      tp += q.n_tiles;
      tu += updB[0].back().n_tiles;
      w.tiles_gram = tg; w.tiles_poly = tp; w.tiles_upd = tu;
      w.fl_gram += 2.0 * m * m * nn;
      w.fl_poly += 2.0 * m * m * m;
      w.fl_upd += 2.0 * m * m * nn;
      // executed: three tf32 products per tile and K step
      const double tile_fl = 3.0 * 2.0 * kTcPairBM * kTcBN;
      w.ex_gram += tile_fl * gram[0].back().n_tiles * (double)(ceil_div(nn, kX3BK) * kX3BK);
      w.ex_poly += tile_fl * q.n_tiles * (double)(ceil_div(m, kX3BK) * kX3BK);
      w.ex_upd += tile_fl * updB[0].back().n_tiles * (double)(ceil_div(m, kX3BK) * kX3BK);
    }
    if (bad) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed with code " + std::to_string(bad));
    MUON_CUDA(cudaMemcpy(d_maps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice));
    order_gram_by_k(gram[0], P->waves);
    order_gram_by_k(gram[1], P->waves);
    std::vector<GemmProblemX3>* lists[7] = {&gram[0], &gram[1], &poly, &updB[0], &updB[1], &updA[0], &updA[1]};
    void** dsts[7] = {&P->d_gram[0], &P->d_gram[1], &P->d_poly, &P->d_updB[0], &P->d_updB[1],
                      &P->d_updA[0], &P->d_updA[1]};
    for (int k = 0; k < 7; ++k) {
      *dsts[k] = T + o_prob[k];
      MUON_CUDA(cudaMemcpy(*dsts[k], lists[k]->data(), lists[k]->size() * sizeof(GemmProblemX3),
                           cudaMemcpyHostToDevice));
    }
    P->h_upd_x3[0][0] = updB[0]; P->h_upd_x3[0][1] = updB[1];
    P->h_upd_x3[1][0] = updA[0]; P->h_upd_x3[1][1] = updA[1];
    P->d_fused = T + o_fused;
  }

  // ---- per-call table template
  for (int j = 0; j < n; ++j) {
    mats[j].x0 = P->x0[j];
    mats[j].colmean = P->colmean[j];
    mats[j].colpart = P->colpart[j];
    mats[j].alpha = P->alpha[j];
  }
  P->last_uploaded = mats;   // template: pointers of the call are filled in per call
  ds.plans.insert(ds.plans.begin(), std::move(P));
  *out = ds.plans[0].get();
  return MUON_OK;
}

// Writes the per-call table when it differs from the last one written (in stream order, through
// kernel parameters).
int upload_mats(Plan& P, std::vector<MatInfo>& mats, cudaStream_t s) {
  if (P.uploaded_once && std::memcmp(mats.data(), P.last_uploaded.data(), mats.size() * sizeof(MatInfo)) == 0)
    return MUON_OK;
  MUON_CUDA(write_table(P.d_mats, mats.data(), mats.size() * sizeof(MatInfo), s, &g_launches));
  P.last_uploaded = mats;
  P.uploaded_once = true;
  return MUON_OK;
}

// Per-call table of the last Newton-Schulz update with the parameter update fused into its
// epilogue: the plan's update problems plus TMA views (32 x 32 fp32 boxes, 128-byte swizzle) of
// the caller's parameter matrices. Rebuilt and uploaded only when the parameters, the RMS factors
// or the last iteration's operand and parity change. Returns NULL when a parameter matrix cannot
// be viewed by TMA (row length not a multiple of 4 floats, or a base not 16-byte aligned); the
// step then uses the separate update kernel.
std::vector<uint8_t> fused_key_of(float* const* params, const std::vector<int>& idx,
                                  const std::vector<float>& rms, int which, int parity) {
  const int n = (int)idx.size();
  std::vector<uint8_t> key(sizeof(void*) * n + sizeof(float) * n + 2 * sizeof(int));
  uint8_t* k = key.data();
  for (int j = 0; j < n; ++j) { std::memcpy(k, &params[idx[j]], sizeof(void*)); k += sizeof(void*); }
  std::memcpy(k, rms.data(), sizeof(float) * n); k += sizeof(float) * n;
  std::memcpy(k, &which, sizeof(int)); k += sizeof(int);
  std::memcpy(k, &parity, sizeof(int));
  return key;
}

const void* fused_table(Plan& P, float* const* params, const std::vector<int>& idx,
                        const std::vector<float>& rms, int which, int parity, cudaStream_t s, int* rc) {
  *rc = MUON_OK;
  const int n = (int)P.shapes.size();
  for (int j = 0; j < n; ++j)
    if (P.shapes[j].c % 4 != 0 || (uintptr_t)params[idx[j]] % 16 != 0) return nullptr;
  std::vector<uint8_t> key = fused_key_of(params, idx, rms, which, parity);
  if (key == P.fused_key) return P.d_fused;
  PFN_encodeTiled_t encode = get_encode();
  if (!encode) return nullptr;
  std::vector<CUtensorMap> maps(n);
  std::vector<GemmProblem> probs = P.h_upd[which][parity];
  for (int j = 0; j < n; ++j) {
    cuuint64_t gdim[2] = {(cuuint64_t)P.shapes[j].c, (cuuint64_t)P.shapes[j].r};
    cuuint64_t gstride[1] = {(cuuint64_t)(P.shapes[j].c * 4)};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = encode(&maps[j], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, params[idx[j]], gdim, gstride, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return nullptr;
  }
  for (int q = 0; q < n; ++q) {   // table position q holds the update of matrix probs[q].mat
    const int j = probs[q].mat;
    probs[q].tma_p = P.d_pmaps + j;
    probs[q].rms = rms[j];
  }
  cudaError_t e = write_table(P.d_pmaps, maps.data(), n * sizeof(CUtensorMap), s, &g_launches);
  if (e == cudaSuccess) e = write_table(P.d_fused, probs.data(), n * sizeof(GemmProblem), s, &g_launches);
  if (e != cudaSuccess) { *rc = cuda_fail(e, "fused table upload"); return nullptr; }
  P.fused_key = key;
  return P.d_fused;
}

// The same for the fp32 (3xTF32) mode: the epilogue updates the parameters with plain loads and
// stores (16-byte vectors where the rows allow it), so every parameter layout is accepted.
const void* fused_table_x3(Plan& P, float* const* params, const std::vector<int>& idx,
                           const std::vector<float>& rms, int which, int parity, cudaStream_t s, int* rc) {
  *rc = MUON_OK;
  const int n = (int)P.shapes.size();
  std::vector<uint8_t> key = fused_key_of(params, idx, rms, which, parity);
  if (key == P.fused_key) return P.d_fused;
  std::vector<GemmProblemX3> probs = P.h_upd_x3[which][parity];
  for (int j = 0; j < n; ++j) {
    float* p = params[idx[j]];
    probs[j].p = p;
    probs[j].ldp = P.shapes[j].c;
    probs[j].rms = rms[j];
    probs[j].p_vec = (P.shapes[j].c % 4 == 0 && (uintptr_t)p % 16 == 0) ? 1 : 0;
  }
  cudaError_t e = write_table(P.d_fused, probs.data(), n * sizeof(GemmProblemX3), s, &g_launches);
  if (e != cudaSuccess) { *rc = cuda_fail(e, "fused table upload"); return nullptr; }
  P.fused_key = key;
  return P.d_fused;
}

bool finite_f(float x) { return std::isfinite(x); }

int check_coeffs(int steps, const muon_coeffs_t* coeffs, std::vector<muon_coeffs_t>& out) {
  if (steps < 0 || steps > MUON_MAX_NS_STEPS)
    return fail(MUON_ERR_INVALID_ARG, "steps must be in [0, " + std::to_string(MUON_MAX_NS_STEPS) + "]");
  out.resize(steps);
  for (int k = 0; k < steps; ++k) {
    out[k] = coeffs ? coeffs[k] : muon_coeffs_t{3.4445f, -4.7750f, 2.0315f};
    if (!finite_f(out[k].a) || !finite_f(out[k].b) || !finite_f(out[k].c))
      return fail(MUON_ERR_INVALID_ARG, "coefficients must be finite");
  }
  return MUON_OK;
}

int check_shape(int64_t r, int64_t c, const char* what) {
  if (r <= 0 || c <= 0)
    return fail(MUON_ERR_INVALID_ARG, std::string(what) + ": rows and cols must be positive");
  if (r > (1 << 20) || c > (1 << 20) || r * c > (int64_t(1) << 36))
    return fail(MUON_ERR_INVALID_ARG, std::string(what) + ": matrix too large (rows, cols <= 2^20, rows*cols <= 2^36)");
  return MUON_OK;
}

// The whole Newton-Schulz iteration of one wave as one chained launch (bf16, 256 x 256 tiles):
// the same phases, problem tables and epilogue scalars as the per-phase launches of run_ns, with
// each phase waiting (per matrix) for the one whose results it reads: Gram k for update k - 1,
// poly k for Gram k, update k for poly k (Gram k when c_k = 0).
int run_ns_chained(DeviceState& ds, Plan& P, const Wave& w, int wave_idx, const std::vector<muon_coeffs_t>& co,
                   cudaStream_t s, const void* fused_last, float lr, float decay) {
  const int n = w.j1 - w.j0;
  auto tc = [&](void* t) { return static_cast<GemmProblem*>(t) + w.j0; };
  std::vector<PhaseDesc> ph;
  uint32_t tiles = 0;
  double fl = 0.0, ex = 0.0;
  auto add = [&](const void* table, uint32_t n_tiles, const EpiScalars& e, int dep, const uint32_t* tgt) {
    PhaseDesc d{};
    d.probs = static_cast<const GemmProblem*>(table);
    d.dep_target = dep >= 0 ? tgt : nullptr;
    d.tile_begin = tiles;
    d.nprobs = n;
    d.dep = dep;
    d.ep = e;
    d.ep.wait_ns = g_wait_ns;
    ph.push_back(d);
    tiles += n_tiles;
    return (int)ph.size() - 1;
  };
  int prev_update = -1;
  for (size_t k = 0; k < co.size(); ++k) {
    const int p = (int)(k & 1);
    const int first = k == 0 ? 1 : 0;
    const muon_coeffs_t c = co[k];
    // the same epilogue scalars as run_ns's bf16 path
    EpiScalars eg{1.0f, 0.0f, first ? 2 : 0, 0, 0.0f};
    if (c.c == 0.0f) eg = EpiScalars{c.b, 0.0f, first ? 2 : 0, 0, c.a};
    const int gram = add(tc(P.d_gram[p]), w.tiles_gram, eg, prev_update, P.d_tgt[2]);
    fl += w.fl_gram;
    ex += w.ex_gram;
    int dep = gram;
    const uint32_t* dep_tgt = P.d_tgt[0];
    void* upd = P.d_updA[p];
    if (c.c != 0.0f) {
      dep = add(tc(P.d_poly), w.tiles_poly, EpiScalars{c.c, c.b, 0, 0, c.a}, gram, P.d_tgt[0]);
      dep_tgt = P.d_tgt[1];
      upd = P.d_updB[p];
      fl += w.fl_poly;
      ex += w.ex_poly;
    }
    EpiScalars eu{1.0f, 0.0f, first, 0, 0.0f};
    if (fused_last && k + 1 == co.size()) {
      upd = const_cast<void*>(fused_last);
      eu.lr = lr;
      eu.decay = decay;
      eu.fused = 1;
    }
    prev_update = add(tc(upd), w.tiles_upd, eu, dep, dep_tgt);
    fl += w.fl_upd;
    ex += w.ex_upd;
  }
  PhaseDesc* d_ph = P.d_phases + (size_t)wave_idx * kMaxChainPhases;
  std::vector<PhaseDesc>& last = P.last_phases[wave_idx];
  if (last.size() != ph.size() || std::memcmp(last.data(), ph.data(), ph.size() * sizeof(PhaseDesc)) != 0) {
    MUON_CUDA(write_table(d_ph, ph.data(), ph.size() * sizeof(PhaseDesc), s, &g_launches));
    last = ph;
  }
  const int nmats = (int)P.shapes.size();
  MUON_CUDA(cudaMemsetAsync(P.d_chain_ctr, 0, (1 + ph.size() * (size_t)nmats) * 4, s));
  const ChainArgs ca{d_ph, P.d_chain_ctr, P.d_chain_ctr + 1, (int)ph.size(), nmats};
  EpiScalars el{};
  el.wait_ns = g_wait_ns;
  cudaError_t e = timed_launch(MUON_KC_GEMM, s, fl, ex, [&] {
    return launch_gemm_tc_pair_chain(ca, tiles, el, ds.d_status, ds.pair_capacity, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "chained Newton-Schulz launch");
  return MUON_OK;
}

// Runs the Newton-Schulz phases for the matrices of one wave (wave_idx of the plan). fused_last
// (optional) is the per-call table of last-update problems for all matrices of the plan.
int run_ns(DeviceState& ds, Plan& P, const Wave& w, int wave_idx, const std::vector<muon_coeffs_t>& co,
           cudaStream_t s, const void* fused_last = nullptr, float lr = 0.0f, float decay = 1.0f) {
  const int n = w.j1 - w.j0;
  if (P.x_bf16 && w.chain && !co.empty() && co.size() * 3 <= (size_t)kMaxChainPhases)
    return run_ns_chained(ds, P, w, wave_idx, co, s, fused_last, lr, decay);
  // the wave's sub-range of a problem table
  auto tc = [&](void* t) { return static_cast<GemmProblem*>(t) + w.j0; };
  auto x3 = [&](void* t) { return static_cast<GemmProblemX3*>(t) + w.j0; };
  for (size_t k = 0; k < co.size(); ++k) {
    const int p = (int)(k & 1);
    const int first = k == 0 ? 1 : 0;
    const muon_coeffs_t c = co[k];
    cudaError_t e;
    // fp32 (3xTF32) path: gram A = alpha^2k X X^T, poly B = c A A + b A,
    //   update X' = alpha^k (a X + B X)
    //   (c = 0: X' = alpha^k (a X + b A X)).
    // bf16 path: the a X term is folded into the left operand of the update, rounding once:
    //   poly B = c A A + b A + a I (c = 0: gram A = b alpha^2k X X^T + a I), update X' = alpha^k B X.
    EpiScalars eg{1.0f, 0.0f, first ? 2 : 0, 0, 0.0f};
    if (P.x_bf16 && c.c == 0.0f) eg = EpiScalars{c.b, 0.0f, first ? 2 : 0, 0, c.a};
    eg.wait_ns = g_wait_ns;
    if (P.x_bf16) {
      e = timed_launch(MUON_KC_GEMM, s, w.fl_gram, w.ex_gram, [&] {
        return (w.wide ? launch_gemm_tc_pair_wide : launch_gemm_tc_pair)(tc(P.d_gram[p]), n, w.tiles_gram, eg,
                                                                         ds.d_status, ds.pair_capacity, s);
      }, MUON_KC_GEMM_GRAM);
    } else {
      e = timed_launch(MUON_KC_GEMM, s, w.fl_gram, w.ex_gram, [&] {
        return launch_gemm_x3(x3(P.d_gram[p]), n, w.tiles_gram, eg, ds.d_status, ds.x3_capacity, s);
      }, MUON_KC_GEMM_GRAM);
    }
    if (e != cudaSuccess) return cuda_fail(e, "gram launch");
    void* upd;
    EpiScalars eu;
    if (c.c != 0.0f) {
      EpiScalars ep{c.c, c.b, 0, 0, P.x_bf16 ? c.a : 0.0f};
      ep.wait_ns = g_wait_ns;
      if (P.x_bf16) {
        e = timed_launch(MUON_KC_GEMM, s, w.fl_poly, w.ex_poly, [&] {
          return launch_gemm_tc_pair(tc(P.d_poly), n, w.tiles_poly, ep, ds.d_status, ds.pair_capacity, s);
        }, MUON_KC_GEMM_POLY);
      } else {
        e = timed_launch(MUON_KC_GEMM, s, w.fl_poly, w.ex_poly, [&] {
          return launch_gemm_x3(x3(P.d_poly), n, w.tiles_poly, ep, ds.d_status, ds.x3_capacity, s);
        }, MUON_KC_GEMM_POLY);
      }
      if (e != cudaSuccess) return cuda_fail(e, "poly launch");
      upd = P.d_updB[p];
      eu = P.x_bf16 ? EpiScalars{1.0f, 0.0f, first, 0, 0.0f} : EpiScalars{1.0f, c.a, first, first, 0.0f};
    } else {
      upd = P.d_updA[p];
      eu = P.x_bf16 ? EpiScalars{1.0f, 0.0f, first, 0, 0.0f} : EpiScalars{c.b, c.a, first, first, 0.0f};
    }
    eu.wait_ns = g_wait_ns;
    if (fused_last && k + 1 == co.size()) {
      upd = const_cast<void*>(fused_last);
      eu.lr = lr;
      eu.decay = decay;
      eu.fused = 1;
    }
    if (P.x_bf16) {
      e = timed_launch(MUON_KC_GEMM, s, w.fl_upd, w.ex_upd, [&] {
        return (w.wide ? launch_gemm_tc_pair_wide : launch_gemm_tc_pair)(tc(upd), n, w.tiles_upd, eu, ds.d_status,
                                                                         ds.pair_capacity, s);
      }, MUON_KC_GEMM_UPDATE);
    } else {
      e = timed_launch(MUON_KC_GEMM, s, w.fl_upd, w.ex_upd, [&] {
        return launch_gemm_x3(x3(upd), n, w.tiles_upd, eu, ds.d_status, ds.x3_capacity, s);
      }, MUON_KC_GEMM_UPDATE);
    }
    if (e != cudaSuccess) return cuda_fail(e, "update launch");
  }
  return MUON_OK;
}

struct Ranges {   // overlap detection over [begin, end) byte ranges
  std::vector<std::pair<uintptr_t, uintptr_t>> v;
  void add(const void* p, size_t bytes) { v.push_back({(uintptr_t)p, (uintptr_t)p + bytes}); }
  bool overlap() {
    std::sort(v.begin(), v.end());
    for (size_t i = 1; i < v.size(); ++i)
      if (v[i].first < v[i - 1].second) return true;
    return false;
  }
};

}  // namespace

// Hooks for the no-allocation entry point (noalloc.cu): its error message and launch count go
// through the same per-thread message and counter as every other call.
void set_error_message(const std::string& msg) { t_err = msg; }

void note_launches(int64_t n) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_launches += n;
}

}  // namespace muon

using namespace muon;

extern "C" {

int muon_version(void) { return 100; }

const char* muon_last_error(void) { return t_err.c_str(); }

int64_t muon_launch_count(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  return g_launches;
}

int muon_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof_on = on != 0;
  return MUON_OK;
}

int muon_profile_read(int64_t* launches, double* ms, double* flops, double* exec_flops) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!launches || !ms) return fail(MUON_ERR_INVALID_ARG, "launches and ms must not be NULL");
  for (int k = 0; k < MUON_KC_COUNT; ++k) {
    launches[k] = 0;
    ms[k] = 0.0;
    if (flops) flops[k] = 0.0;
    if (exec_flops) exec_flops[k] = 0.0;
  }
  int rc = MUON_OK;
  for (ProfRec& r : g_prof) {
    float t = 0.f;
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, r.a, r.b);
    if (e != cudaSuccess && rc == MUON_OK) rc = cuda_fail(e, "profile event");
    for (int k : {r.kind, r.sub}) {
      if (k < 0) continue;
      launches[k] += 1;
      ms[k] += t;
      if (flops) flops[k] += r.flops;
      if (exec_flops) exec_flops[k] += r.exec;
    }
    g_event_pool.push_back(r.a);
    g_event_pool.push_back(r.b);
  }
  g_prof.clear();
  return rc;
}

int muon_check_status(muon_stream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != MUON_OK) return rc;
  MUON_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  int h[2] = {0, 0};
  MUON_CUDA(cudaMemcpy(h, ds->d_status, sizeof(h), cudaMemcpyDeviceToHost));
  MUON_CUDA(cudaMemset(ds->d_status, 0, sizeof(h)));
  if (h[0] & kStatusTimeout) return fail(MUON_ERR_TIMEOUT, "a kernel wait hit its time limit");
  if (h[1] != 0) return fail(MUON_WARN_NONFINITE, std::to_string(h[1]) + " chunk(s) held NaN or Inf");
  return MUON_OK;
}

int muon_release_workspace(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_OK;
  auto it = g_dev.find(dev);
  if (it == g_dev.end()) return MUON_OK;
  cudaDeviceSynchronize();
  DeviceState& ds = it->second;
  ds.plans.clear();
  if (ds.arena) cudaFree(ds.arena);
  ds.arena = nullptr;
  ds.arena_bytes = 0;
  ++ds.arena_gen;
  ds.adam.reset();
  return MUON_OK;
}

int muon_set_wave_elements(int64_t elements) {
  std::lock_guard<std::mutex> lk(g_mu);
  t_err.clear();
  if (elements < 0) return fail(MUON_ERR_INVALID_ARG, "elements must be >= 0");
  g_wave_elements = elements == 0 ? kWaveElements : elements;
  return MUON_OK;
}

int muon_set_chained_launch(int mode) {
  std::lock_guard<std::mutex> lk(g_mu);
  t_err.clear();
  if (mode < 0 || mode > 2) return fail(MUON_ERR_INVALID_ARG, "mode must be 0, 1 or 2");
  g_chain_mode = mode;
  return MUON_OK;
}

int muon_set_wait_limit_ns(uint64_t ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  t_err.clear();
  g_wait_ns = ns;
  return MUON_OK;
}

int muon_step(int count, float* const* params, const void* const* grads, muon_dtype_t grad_dtype,
              float* const* momentum, const int64_t* rows, const int64_t* cols, float lr, float mu,
              int nesterov, float weight_decay, muon_rms_t rms_scale, int steps,
              const muon_coeffs_t* coeffs, int zero_center, float eps, muon_prec_t prec,
              muon_stream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  t_err.clear();
  // ---- validation (no device work before this passes)
  if (count < 0) return fail(MUON_ERR_INVALID_ARG, "count must be >= 0");
  if (count > 0 && (!params || !grads || !momentum || !rows || !cols))
    return fail(MUON_ERR_INVALID_ARG, "params, grads, momentum, rows and cols must not be NULL");
  if (grad_dtype != MUON_BF16 && grad_dtype != MUON_FP32) return fail(MUON_ERR_INVALID_ARG, "grad_dtype");
  if (prec != MUON_PREC_BF16 && prec != MUON_PREC_FP32) return fail(MUON_ERR_INVALID_ARG, "prec");
  if (rms_scale != MUON_RMS_ONE && rms_scale != MUON_RMS_SQRT_MAX1_ROWS_OVER_COLS)
    return fail(MUON_ERR_INVALID_ARG, "rms_scale");
  if (!finite_f(lr) || !finite_f(weight_decay)) return fail(MUON_ERR_INVALID_ARG, "lr and weight_decay must be finite");
  if (!(mu >= 0.0f && mu < 1.0f)) return fail(MUON_ERR_INVALID_ARG, "mu must be in [0, 1)");
  if (!(eps >= 0.0f) || !finite_f(eps)) return fail(MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
  std::vector<muon_coeffs_t> co;
  int rc = check_coeffs(steps, coeffs, co);
  if (rc != MUON_OK) return rc;
  std::vector<int> idx;
  Ranges written;
  for (int i = 0; i < count; ++i) {
    if (!grads[i]) continue;
    rc = check_shape(rows[i], cols[i], "muon_step");
    if (rc != MUON_OK) return rc;
    if (!params[i] || !momentum[i]) return fail(MUON_ERR_INVALID_ARG, "params[i] and momentum[i] must not be NULL");
    const size_t bytes = (size_t)rows[i] * cols[i] * 4;
    written.add(params[i], bytes);
    written.add(momentum[i], bytes);
    idx.push_back(i);
  }
  if (written.overlap()) return fail(MUON_ERR_INVALID_ARG, "params/momentum buffers overlap");
  if (idx.empty()) return MUON_OK;

  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != MUON_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::vector<Shape> shapes;
  for (int i : idx) shapes.push_back({rows[i], cols[i]});
  const int x_bf16 = prec == MUON_PREC_BF16;
  Plan* P = nullptr;
  rc = build_plan(*ds, shapes, x_bf16, &P);
  if (rc != MUON_OK) return rc;
  const int n = (int)idx.size();
  const int g_bf16 = grad_dtype == MUON_BF16;
  const size_t gsz = g_bf16 ? 2 : 4;
  std::vector<MatInfo> mats = P->last_uploaded;
  for (int j = 0; j < n; ++j) {
    const int i = idx[j];
    MatInfo& mi = mats[j];
    mi.p = params[i];
    mi.g = grads[i];
    mi.m = momentum[i];
    mi.xf = (steps & 1) ? P->x1[j] : P->x0[j];
    mi.rms = rms_scale == MUON_RMS_SQRT_MAX1_ROWS_OVER_COLS
                 ? (float)std::sqrt(std::max(1.0, (double)rows[i] / (double)cols[i])) : 1.0f;
    const bool aligned = ((uintptr_t)params[i] % 16 == 0) && ((uintptr_t)momentum[i] % 16 == 0) &&
                         ((uintptr_t)grads[i] % 16 == 0);
    mi.vec = (cols[i] % 8 == 0) && aligned ? 1 : 0;
    (void)gsz;
  }
  rc = upload_mats(*P, mats, s);
  if (rc != MUON_OK) return rc;
  const void* fused = nullptr;
  if (steps > 0) {
    std::vector<float> rms(n);
    for (int j = 0; j < n; ++j) rms[j] = mats[j].rms;
    const int which = co.back().c != 0.0f ? 0 : 1;
    fused = x_bf16 ? fused_table(*P, params, idx, rms, which, (steps - 1) & 1, s, &rc)
                   : fused_table_x3(*P, params, idx, rms, which, (steps - 1) & 1, s, &rc);
    if (rc != MUON_OK) return rc;
  }

  const int ew_grid = ds->sms * 8;
  for (size_t wi = 0; wi < P->waves.size(); ++wi) {
    const Wave& w = P->waves[wi];
    const MatInfo* dm = P->d_mats + w.j0;
    const int nw = w.j1 - w.j0;
    cudaError_t e;
    if (zero_center) {
      e = timed_launch(MUON_KC_CENTER, s, 0, 0, [&] { return launch_colsum(dm, nw, w.cs_items, g_bf16, s); });
      if (e != cudaSuccess) return cuda_fail(e, "column-sum launch");
      e = timed_launch(MUON_KC_CENTER, s, 0, 0, [&] { return launch_colmean(dm, nw, w.cm_items, s); });
      if (e != cudaSuccess) return cuda_fail(e, "column-mean launch");
    }
    e = timed_launch(MUON_KC_PROLOGUE, s, 0, 0, [&] {
      return launch_prologue(dm, nw, w.n_chunks, g_bf16, x_bf16, 1, mu, nesterov, zero_center,
                             P->d_partials, ds->d_status, ew_grid, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
    e = timed_launch(MUON_KC_NORM, s, 0, 0, [&] { return launch_alpha(dm, nw, P->d_partials, eps, s); });
    if (e != cudaSuccess) return cuda_fail(e, "norm launch");
    rc = run_ns(*ds, *P, w, (int)wi, co, s, fused, lr, 1.0f - lr * weight_decay);
    if (rc != MUON_OK) return rc;
    if (fused) continue;   // the last update product already wrote the parameters
    e = timed_launch(MUON_KC_EPILOGUE, s, 0, 0, [&] {
      return launch_update(dm, nw, w.n_chunks, x_bf16, lr, 1.0f - lr * weight_decay, steps == 0 ? 1 : 0,
                           ew_grid, s);
    });
    if (e != cudaSuccess) return cuda_fail(e, "epilogue launch");
  }
  return MUON_OK;
}

int muon_adamw_step(int count, float* const* params, const void* const* grads, muon_dtype_t grad_dtype,
                    float* const* exp_avg, float* const* exp_avg_sq, const int64_t* numel, int64_t step,
                    float lr, float beta1, float beta2, float eps, float weight_decay, muon_stream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  t_err.clear();
  if (count < 0) return fail(MUON_ERR_INVALID_ARG, "count must be >= 0");
  if (count > 0 && (!params || !grads || !exp_avg || !exp_avg_sq || !numel))
    return fail(MUON_ERR_INVALID_ARG, "params, grads, exp_avg, exp_avg_sq and numel must not be NULL");
  if (grad_dtype != MUON_BF16 && grad_dtype != MUON_FP32) return fail(MUON_ERR_INVALID_ARG, "grad_dtype");
  if (step < 1) return fail(MUON_ERR_INVALID_ARG, "step must be >= 1 (the step count after this step)");
  if (!finite_f(lr) || !finite_f(weight_decay)) return fail(MUON_ERR_INVALID_ARG, "lr and weight_decay must be finite");
  if (!(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f))
    return fail(MUON_ERR_INVALID_ARG, "beta1 and beta2 must be in [0, 1)");
  if (!(eps >= 0.0f) || !finite_f(eps)) return fail(MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
  std::vector<int> idx;
  Ranges written;
  for (int i = 0; i < count; ++i) {
    if (!grads[i] || numel[i] == 0) continue;
    if (numel[i] < 0 || numel[i] > (int64_t(1) << 36)) return fail(MUON_ERR_INVALID_ARG, "numel out of range");
    if (!params[i] || !exp_avg[i] || !exp_avg_sq[i])
      return fail(MUON_ERR_INVALID_ARG, "params[i], exp_avg[i] and exp_avg_sq[i] must not be NULL");
    const size_t bytes = (size_t)numel[i] * 4;
    written.add(params[i], bytes);
    written.add(exp_avg[i], bytes);
    written.add(exp_avg_sq[i], bytes);
    idx.push_back(i);
  }
  if (written.overlap()) return fail(MUON_ERR_INVALID_ARG, "params/exp_avg/exp_avg_sq buffers overlap");
  if (idx.empty()) return MUON_OK;
  DeviceState* ds = nullptr;
  int rc = device_state(&ds);
  if (rc != MUON_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int n = (int)idx.size();
  std::vector<int64_t> nel(n);
  for (int j = 0; j < n; ++j) nel[j] = numel[idx[j]];
  if (!ds->adam || ds->adam->numel != nel) {
    ds->adam.reset();
    std::unique_ptr<AdamPlan> A(new AdamPlan());
    A->numel = nel;
    MUON_CUDA(cudaMalloc(&A->d_tab, (size_t)n * sizeof(AdamTensor)));
    ds->adam = std::move(A);
  }
  AdamPlan& A = *ds->adam;
  std::vector<AdamTensor> tab(n);
  int64_t chunks = 0;
  for (int j = 0; j < n; ++j) {
    const int i = idx[j];
    AdamTensor& t = tab[j];
    std::memset(&t, 0, sizeof(t));
    t.p = params[i];
    t.g = grads[i];
    t.m = exp_avg[i];
    t.v = exp_avg_sq[i];
    t.numel = numel[i];
    t.chunk_begin = chunks;
    chunks += ceil_div(numel[i], kChunk);
    t.vec = ((uintptr_t)params[i] % 16 == 0 && (uintptr_t)grads[i] % 16 == 0 &&
             (uintptr_t)exp_avg[i] % 16 == 0 && (uintptr_t)exp_avg_sq[i] % 16 == 0) ? 1 : 0;
  }
  A.n_chunks = chunks;
  if (!A.uploaded || std::memcmp(tab.data(), A.last.data(), n * sizeof(AdamTensor)) != 0) {
    MUON_CUDA(write_table(A.d_tab, tab.data(), n * sizeof(AdamTensor), s, &g_launches));
    A.last = tab;
    A.uploaded = true;
  }
  const double bc1 = 1.0 - std::pow((double)beta1, (double)step);
  const double bc2 = 1.0 - std::pow((double)beta2, (double)step);
  AdamScalars sc;
  sc.decay = 1.0f - lr * weight_decay;
  sc.beta1 = beta1;
  sc.beta2 = beta2;
  sc.step_size = (float)((double)lr / bc1);
  sc.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  sc.eps = eps;
  const int g_bf16 = grad_dtype == MUON_BF16;
  cudaError_t e = timed_launch(MUON_KC_ADAMW, s, 0, 0, [&] {
    return launch_adamw(A.d_tab, n, A.n_chunks, g_bf16, sc, ds->sms * 4, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "adamw launch");
  return MUON_OK;
}

int muon_ns_orthogonalize(const void* G, muon_dtype_t g_dtype, void* X, muon_dtype_t x_dtype,
                          int64_t m, int64_t n, int steps, const muon_coeffs_t* coeffs,
                          int zero_center, float eps, muon_prec_t prec, muon_stream_t stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  t_err.clear();
  if (!G || !X) return fail(MUON_ERR_INVALID_ARG, "G and X must not be NULL");
  if (g_dtype != MUON_BF16 && g_dtype != MUON_FP32) return fail(MUON_ERR_INVALID_ARG, "g_dtype");
  if (x_dtype != MUON_BF16 && x_dtype != MUON_FP32) return fail(MUON_ERR_INVALID_ARG, "x_dtype");
  if (prec != MUON_PREC_BF16 && prec != MUON_PREC_FP32) return fail(MUON_ERR_INVALID_ARG, "prec");
  if (!(eps >= 0.0f) || !finite_f(eps)) return fail(MUON_ERR_INVALID_ARG, "eps must be finite and >= 0");
  int rc = check_shape(m, n, "muon_ns_orthogonalize");
  if (rc != MUON_OK) return rc;
  std::vector<muon_coeffs_t> co;
  rc = check_coeffs(steps, coeffs, co);
  if (rc != MUON_OK) return rc;
  Ranges rg;
  rg.add(G, (size_t)m * n * (g_dtype == MUON_BF16 ? 2 : 4));
  rg.add(X, (size_t)m * n * (x_dtype == MUON_BF16 ? 2 : 4));
  if (rg.overlap()) return fail(MUON_ERR_INVALID_ARG, "G and X overlap");

  DeviceState* ds = nullptr;
  rc = device_state(&ds);
  if (rc != MUON_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int x_bf16 = prec == MUON_PREC_BF16;
  Plan* P = nullptr;
  rc = build_plan(*ds, {Shape{m, n}}, x_bf16, &P);
  if (rc != MUON_OK) return rc;
  std::vector<MatInfo> mats = P->last_uploaded;
  MatInfo& mi = mats[0];
  mi.p = static_cast<float*>(X);
  mi.g = G;
  mi.m = nullptr;
  mi.xf = (steps & 1) ? P->x1[0] : P->x0[0];
  mi.rms = 1.0f;
  mi.vec = (n % 8 == 0) && ((uintptr_t)G % 16 == 0) && ((uintptr_t)X % 16 == 0) ? 1 : 0;
  rc = upload_mats(*P, mats, s);
  if (rc != MUON_OK) return rc;
  const int g_bf16 = g_dtype == MUON_BF16;
  const int ew_grid = ds->sms * 8;
  const Wave& w = P->waves[0];   // one matrix: one wave
  cudaError_t e;
  if (zero_center) {
    e = timed_launch(MUON_KC_CENTER, s, 0, 0, [&] { return launch_colsum(P->d_mats, 1, w.cs_items, g_bf16, s); });
    if (e != cudaSuccess) return cuda_fail(e, "column-sum launch");
    e = timed_launch(MUON_KC_CENTER, s, 0, 0, [&] { return launch_colmean(P->d_mats, 1, w.cm_items, s); });
    if (e != cudaSuccess) return cuda_fail(e, "column-mean launch");
  }
  e = timed_launch(MUON_KC_PROLOGUE, s, 0, 0, [&] {
    return launch_prologue(P->d_mats, 1, w.n_chunks, g_bf16, x_bf16, 0, 0.0f, 0, zero_center,
                           P->d_partials, ds->d_status, ew_grid, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "prologue launch");
  e = timed_launch(MUON_KC_NORM, s, 0, 0, [&] { return launch_alpha(P->d_mats, 1, P->d_partials, eps, s); });
  if (e != cudaSuccess) return cuda_fail(e, "norm launch");
  rc = run_ns(*ds, *P, w, 0, co, s);
  if (rc != MUON_OK) return rc;
  e = timed_launch(MUON_KC_EPILOGUE, s, 0, 0, [&] {
    return launch_output(P->d_mats, 1, w.n_chunks, x_bf16, x_dtype == MUON_BF16, steps == 0 ? 1 : 0,
                         ew_grid, s);
  });
  if (e != cudaSuccess) return cuda_fail(e, "output launch");
  return MUON_OK;
}

}  // extern "C"
