// Internal structures shared by the host planner and the device kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace muon {

// Elementwise kernels split every matrix into chunks of this many elements; one CTA owns one
// chunk at a time and writes one norm partial per chunk.
constexpr int64_t kChunk = 8192;
constexpr int kEwThreads = 256;

// Zero-centring work items: column sums over blocks of kCsRows rows x kCsCols columns.
constexpr int kCsRows = 64;
constexpr int kCsCols = 256;

// Device status word bits.
constexpr int kStatusTimeout = 1;

// Per-matrix record read by the elementwise kernels.
struct MatInfo {
  float* p;            // fp32 params (muon_step) or output X (orthogonalize), per call
  const void* g;       // gradient / input, per call
  float* m;            // fp32 momentum, per call (NULL for orthogonalize)
  void* x0;            // workspace: U, the unnormalised first iterate (bf16 or fp32)
  void* xf;            // workspace: final iterate X_steps
  float* colmean;      // workspace: column means (zero-centring), else NULL
  float* colpart;      // workspace: column-sum partials (zero-centring), else NULL
  float* alpha;        // workspace: 1 / (||u||_F + eps)
  int64_t rows, cols;  // shape of the stored matrix (row-major)
  int64_t ldx;         // leading dimension of x0 / xf, elements
  int64_t xlo;         // fp32 workspace: offset (elements) of the low plane of x0 / xf (see below)
  int64_t chunk_begin; // first elementwise chunk of this matrix (prefix over matrices)
  int64_t cs_begin;    // first column-sum item
  int64_t cm_begin;    // first column-mean item
  float rms;           // RMS factor s
  int vec;             // 1: 16-byte vector path is legal (cols % 8 == 0, aligned pointers)
};

// One tensor of an AdamW call (any shape, flattened).
struct AdamTensor {
  float* p;
  const void* g;
  float* m;
  float* v;
  int64_t numel;
  int64_t chunk_begin;
  int vec;             // 1: 16-byte vector path is legal (all four pointers 16-byte aligned)
  int pad;
};

// Scalars of one AdamW step: p <- p decay; m <- b1 m + (1-b1) g; v <- b2 v + (1-b2) g^2;
// p <- p - step_size m / (sqrt(v) inv_sqrt_bc2 + eps).
struct AdamScalars {
  float decay, beta1, beta2, step_size, inv_sqrt_bc2, eps;
};

// One problem of a grouped tensor-core launch:
//   D = s_acc * (opA . opB^T) + s_c * C,   D: M x N, contraction over K,
// where opA(i, k) and opB(j, k) are read through TMA from bf16 matrices either K-major
// (k contiguous) or MN-major (i or j contiguous).
struct GemmProblem {
  const CUtensorMap* tma_a;
  const CUtensorMap* tma_b;
  // CTA-pair kernel, a_half / b_half operands: the MN-major view of the same matrix, for the K
  // slices read transposed (see a_half below)
  const CUtensorMap* tma_a_t;
  const CUtensorMap* tma_b_t;
  const CUtensorMap* tma_d;   // CTA-pair kernel: TMA store view (32 x 32 boxes) of d
  const CUtensorMap* tma_c;   // CTA-pair kernel: TMA load view (32 x 32 boxes) of the addend, or NULL
  const CUtensorMap* tma_p;   // CTA-pair kernel, fused last update: fp32 parameters (32 x 32 boxes)
  __nv_bfloat16* d;
  const __nv_bfloat16* c;   // single-CTA kernel: addend, may be NULL when s_c == 0
  const float* alpha;       // per-matrix normalisation 1 / (||u|| + eps)
  int64_t ldd, ldc;
  uint32_t M, N, K;
  uint32_t tiles_m, tiles_n;
  uint32_t tile_begin;      // prefix sum over the problems of the launch
  uint32_t n_tiles;
  float rms;                // fused last update: RMS factor s of this matrix
  // The flags are full 32-bit words: with byte-sized fields, one kernel build read a_half out of
  // the tile record's register copy wrongly (it saw b_mn there) in its MMA-issuing thread.
  uint32_t a_mn, b_mn;      // 1: operand is MN-major
  uint32_t sym;             // D is symmetric: compute the tiles touching the upper triangle, and
                            //   1: write the strictly-upper part also mirrored (whole matrix);
                            //   2 (CTA-pair kernel): write only the 256 x 256 blocks on or above
                            //      the diagonal (the upper-block form)
  uint32_t a_half, b_half;  // 1 (CTA-pair kernel): the operand is a symmetric matrix in the
                            //   upper-block form; a K slice in a 256-block below the operand rows'
                            //   block is read transposed, from the mirror block, through tma_*_t
  uint32_t mat;             // chained launch: the problem's matrix (index within its plan)
};

// fp32 precision mode ("3xTF32"). Every fp32 matrix of the iteration is held as two planes of
// the same shape and leading dimension, the second `plane` elements after the first:
//   hi = the value with its 13 low mantissa bits cleared (exactly a tf32 number),
//   lo = value - hi (exact in fp32),
// so hi + lo is the value itself. One problem of a grouped 3xTF32 launch:
//   D = s_acc * (opA . opB^T) + s_c * C + diag I,
// with opA and opB read through 3-D TMA views (columns, rows, plane), K-major or MN-major.
struct GemmProblemX3 {
  const CUtensorMap* tma_a;
  const CUtensorMap* tma_b;
  float* d;                 // output, hi plane (the fused last update stores no D)
  const float* c;           // addend, hi plane, or NULL
  float* p;                 // fused last update: fp32 parameters, row stride ldp; else NULL
  const float* alpha;       // per-matrix normalisation 1 / (||u|| + eps)
  int64_t ldd, ldc, ldp;
  int64_t d_plane, c_plane; // offset (elements) of the lo plane of d and of c
  uint32_t M, N, K;
  uint32_t tiles_m, tiles_n;
  uint32_t tile_begin;
  uint32_t n_tiles;
  float rms;                // fused last update: RMS factor s of this matrix
  uint32_t a_mn, b_mn;      // 1: operand is MN-major (32-bit words, as in GemmProblem)
  uint32_t sym;             // 1: D is symmetric (upper-triangle tiles, strictly-upper part mirrored)
  uint32_t p_vec;           // 1: p rows are 16-byte aligned (ldp % 4 == 0, p 16-byte aligned)
};

// Epilogue scalars of one launch: D = k_acc alpha^e_acc acc + k_c alpha^e_c C + diag I
// (diag is applied by the CTA-pair kernels only; the bf16 CTA-pair kernel takes alpha^e_c = 1).
// With fused set (CTA-pair kernels, last Newton-Schulz update), O = D is not stored; instead the
// parameters become p (1 - lr wd) - lr s O, with decay = 1 - lr wd and s = rms of the problem.
// wait_ns limits every pipeline wait of the launch (0: the kernels' default of 2 s); a wait that
// gives up makes the launch return early with the timeout bit set in the status word.
struct EpiScalars {
  float k_acc, k_c;
  int e_acc, e_c;
  float diag;
  float lr, decay;
  int fused;
  uint64_t wait_ns;
};

// Chained launch (CTA-pair kernel, 256 x 256 tiles): one launch runs every Newton-Schulz product
// of a wave, phase after phase. Global tile t belongs to the phase with the largest
// tile_begin <= t; its tiles are that phase's problem table, scheduled as in a launch of its own.
// A tile of a phase with a dependency reads results of the phase `dep` for the same matrix: it
// starts once done[dep][mat] (epilogue warps that finished a tile of that matrix, eight per tile)
// has reached dep_target[mat].
struct PhaseDesc {
  const GemmProblem* probs;
  const uint32_t* dep_target;   // per matrix of the plan, or NULL when dep < 0
  uint32_t tile_begin;
  int nprobs;
  int dep;
  int pad;
  EpiScalars ep;
};

struct ChainArgs {
  const PhaseDesc* phases;
  uint32_t* tile_counter;   // tiles claimed so far (zero before the launch)
  uint32_t* done;           // [phase][matrix] finished epilogue warps (zero before the launch)
  int nphases;
  int nmats;                // matrices of the plan (the row length of done)
};

// Per-call tables (pointer tables of a call) travel to the device inside kernel parameters, not
// through a copy engine: a small copy on the caller's stream would otherwise queue behind whatever
// bulk copies the caller has in flight (up to the whole step's gradient upload).
constexpr int kTableWords = 4000;   // 32,000 bytes of payload per launch (parameter limit 32,764)
struct TableChunk {
  uint64_t* dst;
  uint64_t nwords;
  uint64_t w[kTableWords];
};

// ---- launchers (defined in the .cu files) ----
// Writes `bytes` (a multiple of 8) from host memory to device memory at dst, in stream order, with
// ceil(bytes / 32000) launches of a copy kernel; adds the number of launches to *launches.
cudaError_t write_table(void* dst, const void* src, size_t bytes, cudaStream_t s, int64_t* launches);
cudaError_t launch_colsum(const MatInfo* mats, int nmats, int64_t items, int g_bf16, cudaStream_t s);
cudaError_t launch_colmean(const MatInfo* mats, int nmats, int64_t items, cudaStream_t s);
cudaError_t launch_prologue(const MatInfo* mats, int nmats, int64_t chunks, int g_bf16, int x_bf16,
                            int has_momentum, float mu, int nesterov, int zero_center,
                            float* partials, int* status, int grid, cudaStream_t s);
cudaError_t launch_alpha(const MatInfo* mats, int nmats, const float* partials, float eps,
                         cudaStream_t s);
cudaError_t launch_update(const MatInfo* mats, int nmats, int64_t chunks, int x_bf16, float lr,
                          float decay, int scale_by_alpha, int grid, cudaStream_t s);
cudaError_t launch_output(const MatInfo* mats, int nmats, int64_t chunks, int x_bf16, int out_bf16,
                          int scale_by_alpha, int grid, cudaStream_t s);
cudaError_t launch_adamw(const AdamTensor* ts, int n, int64_t chunks, int g_bf16, AdamScalars sc,
                         int grid, cudaStream_t s);
cudaError_t launch_gemm_tc(const GemmProblem* probs, int nprobs, uint32_t total_tiles,
                           EpiScalars ep, int* status, int grid, cudaStream_t s);
cudaError_t launch_gemm_tc_pair(const GemmProblem* probs, int nprobs, uint32_t total_tiles,
                                EpiScalars ep, int* status, int max_pairs, cudaStream_t s);
// The same with 256 x kTcWideBN tiles (problem tables built with tiles_n = ceil(N / kTcWideBN)).
cudaError_t launch_gemm_tc_pair_wide(const GemmProblem* probs, int nprobs, uint32_t total_tiles,
                                     EpiScalars ep, int* status, int max_pairs, cudaStream_t s);
// Every phase of a wave in one launch (256 x 256 tiles); fa's counters must be zero. ep carries
// only the launch's wait limit.
cudaError_t launch_gemm_tc_pair_chain(ChainArgs fa, uint32_t total_tiles, EpiScalars ep, int* status,
                                      int max_pairs, cudaStream_t s);
int gemm_tc_pair_capacity(int sms);
cudaError_t launch_gemm_x3(const GemmProblemX3* probs, int nprobs, uint32_t total_tiles,
                           EpiScalars ep, int* status, int max_pairs, cudaStream_t s);
int gemm_x3_pair_capacity(int sms);

// Tile geometry of the tensor-core kernel: single-CTA tiles are kTcBM x kTcBN, CTA-pair tiles
// kTcPairBM x kTcBN; K advances kTcBK per pipeline stage.
constexpr int kTcBM = 128;
constexpr int kTcPairBM = 256;
constexpr int kTcBN = 256;
constexpr int kTcBK = 64;
constexpr int kTcWideBN = 512;   // CTA-pair wide tiles: kTcPairBM x kTcWideBN (Gram and update products)
// 3xTF32 kernel: CTA-pair tiles kTcPairBM x kTcBN, K advances kX3BK (one 128-byte row of fp32)
// per pipeline stage.
constexpr int kX3BK = 32;

}  // namespace muon
