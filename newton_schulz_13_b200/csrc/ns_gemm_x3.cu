// Newton-Schulz matrix products at fp32 accuracy on the tensor cores ("3xTF32"): the fp32
// precision mode of the iteration of "Muon optimizer ..." `newtonschulz5` (A = X X^T,
// B = b A + c A A, X = a X + B X), which that listing runs in bf16.
//
// Each fp32 matrix is held as two planes, hi (the value with its 13 low mantissa bits cleared,
// exactly a tf32 number) and lo = value - hi. A product of two such matrices is formed from three
// tf32 products accumulated in fp32,
//     x y  ~  x_lo y_hi + x_hi y_lo + x_hi y_hi,
// leaving out x_lo y_lo (about 2^-22 relative) and the tf32 rounding of lo (about 2^-21 of x).
//
// Launch structure (as the bf16 kernel's CTA-pair variant): a persistent grid of CTA pairs, output
// tiles of 256 x 256, one problem list per launch, 192 threads per CTA:
//   warp 0     TMA producer of each CTA: per 32-deep K slice, its 128 rows of opA and its 128 of
//              the 256 opB rows, hi and lo planes (64 KB per stage, 3 stages), per operand
//              K-major boxes of 128 x 32 (128-byte swizzle) or MN-major boxes of 32 x 32 (128-byte
//              swizzle over 32-byte granules, the only MN-major form tcgen05 takes for tf32);
//   warp 1     in the even CTA, one thread issues tcgen05.mma.cta_group::2.kind::tf32, three
//              256 x 256 x 8 MMAs per 8-deep K step, into one of two tensor-memory accumulators,
//              which alternate every 512 of K (see kPromote);
//   warps 2-5  epilogue of each CTA (its 128 accumulator rows): sums the 512-deep partial
//              products in fp32, then D = s_acc acc + s_c C + diag I, written back as hi and lo
//              planes (symmetric products: the upper triangle, and the strictly-upper part again
//              at the mirrored position); for the last update of a Muon step,
//              p <- p decay - lr s D instead, and D is never stored.
// Every mbarrier wait is bounded as in the bf16 kernel: a pipeline wait gives up after the
// launch's limit (EpiScalars::wait_ns, 2 s by default) and raises the abort flag of both CTAs of
// the pair; the status word is set, copies and MMAs in flight are accounted for and drained
// (pair_pipe.cuh), the tensor memory is freed and the CTAs return.
#include <stdint.h>

#include "device_once.h"
#include "muon_internal.h"
#include "pair_pipe.cuh"
#include "ptx.cuh"
#include "tile_sched.cuh"

namespace muon {
namespace {

constexpr int kThreads = 192;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kTileM = kTcPairBM;                   // 256 output rows per pair
constexpr int kTileN = kTcBN;                       // 256 output columns
constexpr int kStages = 3;
constexpr uint32_t kPlaneTile = 128 * kX3BK * 4;    // 16 KB: 128 rows (or columns) x 32 K, one plane
constexpr uint32_t kStageBytes = 4 * kPlaneTile;    // A hi, A lo, B hi, B lo
constexpr uint32_t kMnBox = 32 * kX3BK * 4;         // MN-major box: 32 K rows x 32 M/N columns, 4 KB
constexpr uint32_t kTmemCols = 2 * kTileN;
// The tensor core's fp32 accumulation loses about 2 units in the last place (rounding toward
// zero) per 8-deep K step, a bias that grows with K (about 7e-5 relative at K = 4096, 8e-3 at
// K = 2^20). Each accumulator therefore covers at most kPromote K slices (512 of K, bias about
// 1e-5); the epilogue adds these partial products into an fp32 running sum, rounding to nearest,
// kept in the hi plane of D until the last one.
constexpr uint32_t kPromote = 16;
constexpr size_t kSmemBytes = kStages * kStageBytes + 1024 + 256;
// the 256-byte tail holds full and empty per stage, tfull and tempty per accumulator, drain, the
// tensor-memory address, two flags and the producer's fill count
static_assert((2 * kStages + 2 + 2 + 1) * 8 + 4 * 4 <= 256, "barrier area");
static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA");

// Shared-memory descriptor of one 8-deep K step of an operand plane: K-major tiles use the
// 128-byte swizzle (8-row groups 1024 bytes apart); MN-major tiles the 128-byte swizzle over
// 32-byte granules, which tcgen05 requires for MN-major tf32 (4-row K groups 512 bytes apart,
// 32-column M/N boxes kMnBox apart).
__device__ __forceinline__ uint64_t operand_desc(uint32_t addr, uint8_t mn) {
  return mn ? smem_desc_sw128_atom32(addr, kMnBox, 512u) : smem_desc_sw128(addr, 16u, 1024u);
}

__device__ __forceinline__ float tf32_hi(float v) {
  return __uint_as_float(__float_as_uint(v) & 0xffffe000u);
}

// 128 rows (K-major) or 128 columns (MN-major) of one plane of an operand, 32 deep in K.
__device__ __forceinline__ void load_operand(uint8_t* dst, const CUtensorMap* map, bool mn,
                                             uint32_t bar, int32_t row0, int32_t k0, int32_t plane) {
  if (!mn) {
    tma_load_3d_pair(dst, map, bar, k0, row0, plane);
  } else {
#pragma unroll
    for (int h = 0; h < 4; ++h) tma_load_3d_pair(dst + h * kMnBox, map, bar, row0 + 32 * h, k0, plane);
  }
}

__device__ __forceinline__ void store_split4(float* hi, int64_t lo_off, int g, const float (&v)[32]) {
  const float4 h = make_float4(tf32_hi(v[4 * g]), tf32_hi(v[4 * g + 1]), tf32_hi(v[4 * g + 2]),
                               tf32_hi(v[4 * g + 3]));
  const float4 l = make_float4(v[4 * g] - h.x, v[4 * g + 1] - h.y, v[4 * g + 2] - h.z, v[4 * g + 3] - h.w);
  reinterpret_cast<float4*>(hi)[g] = h;
  reinterpret_cast<float4*>(hi + lo_off)[g] = l;
}

__device__ __forceinline__ void store_split1(float* hi, int64_t lo_off, float v) {
  const float h = tf32_hi(v);
  hi[0] = h;
  hi[lo_off] = v - h;
}

__global__ void __launch_bounds__(kThreads, 1)
    ns_gemm_x3_kernel(const GemmProblemX3* __restrict__ probs, int nprobs, uint32_t total_tiles,
                      EpiScalars ep, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* zero_flag = abort_flag + 1;   // never set: the drain waits poll it
  volatile uint32_t* fill_count = reinterpret_cast<volatile uint32_t*>(zero_flag + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0: the CTA that issues the MMAs
  const uint64_t wait_ns = ep.wait_ns ? ep.wait_ns : kTimeoutNs;   // pipeline waits
  const bool leader = rank == 0;
  const uint32_t unit = blockIdx.x / 2;
  const uint32_t n_units = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 8);   // the four epilogue warps of both CTAs
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *zero_flag = 0;
    *fill_count = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // the odd CTA may signal the even CTA's barriers from now on
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  bool timed_out = false;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, fills = 0;
      for (uint32_t t = unit; t < total_tiles && !timed_out; t += n_units) {
        const Tile tl = decode_tile<kTileM, kTileN>(probs, nprobs, t);
        const GemmProblemX3 P = probs[tl.p];   // in registers: the asm below clobbers memory
        const uint32_t kblocks = (P.K + kX3BK - 1) / kX3BK;
        const int32_t a_row0 = (int32_t)(tl.bi * kTileM + rank * 128);
        const int32_t b_row0 = (int32_t)(tl.bj * kTileN + rank * 128);
        for (uint32_t kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, wait_ns)) {
            timed_out = true;
            break;
          }
          uint8_t* dst = smem + stage * kStageBytes;
          const int32_t k0 = (int32_t)(kb * kX3BK);
          // both CTAs' copies count on the even CTA's barrier
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
#pragma unroll
          for (int pl = 0; pl < 2; ++pl) {
            load_operand(dst + pl * kPlaneTile, P.tma_a, P.a_mn != 0, bar, a_row0, k0, pl);
            load_operand(dst + (2 + pl) * kPlaneTile, P.tma_b, P.b_mn != 0, bar, b_row0, k0, pl);
          }
          ++fills;
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (timed_out) raise_abort(abort_flag, true, rank);
      *fill_count = fills;   // settled with the partner's count at exit (pair_pipe.cuh)
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
      for (uint32_t t = unit; t < total_tiles && !timed_out; t += n_units) {
        const Tile tl = decode_tile<kTileM, kTileN>(probs, nprobs, t);
        const GemmProblemX3 P = probs[tl.p];   // in registers: the asm below clobbers memory
        const uint32_t kblocks = (P.K + kX3BK - 1) / kX3BK;
        const uint32_t idesc = idesc_tf32_f32(kTileM, kTileN, P.a_mn, P.b_mn);
        // 8 K per MMA: 32 bytes along a K-major row, or 8 rows of an MN-major box
        const uint32_t a_kstep = P.a_mn ? 8u * 128u : 32u, b_kstep = P.b_mn ? 8u * 128u : 32u;
        uint32_t d_tmem = 0;
        for (uint32_t kb = 0; kb < kblocks; ++kb) {
          const uint32_t kc = kb % kPromote;   // position inside the current accumulation chunk
          if (kc == 0) {
            if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, wait_ns)) {
              timed_out = true;
              break;
            }
            tc_fence_after();
            d_tmem = tmem_base + acc * kTileN;
          }
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag, wait_ns)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
          const uint32_t base = smem_u32(smem + stage * kStageBytes);
#pragma unroll
          for (uint32_t k = 0; k < kX3BK / 8; ++k) {
            const uint64_t a_hi = operand_desc(base + k * a_kstep, P.a_mn);
            const uint64_t a_lo = operand_desc(base + kPlaneTile + k * a_kstep, P.a_mn);
            const uint64_t b_hi = operand_desc(base + 2 * kPlaneTile + k * b_kstep, P.b_mn);
            const uint64_t b_lo = operand_desc(base + 3 * kPlaneTile + k * b_kstep, P.b_mn);
            // the two small cross terms first, then the leading term
            tc_mma_tf32_pair(d_tmem, a_lo, b_hi, idesc, (kc | k) != 0u);
            tc_mma_tf32_pair(d_tmem, a_hi, b_lo, idesc, 1u);
            tc_mma_tf32_pair(d_tmem, a_hi, b_hi, idesc, 1u);
          }
          tc_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
          if (kc == kPromote - 1 || kb + 1 == kblocks) {   // the chunk is complete
            tc_commit_pair_mc(&tfull[acc], 0x3);
            if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
          }
        }
        if (timed_out) break;
      }
      if (timed_out) raise_abort(abort_flag, true, rank);
      tc_commit_pair(drain);
      mbar_wait_bounded(drain, 0, zero_flag, kTimeoutNs);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    // Lane l of the warp owns accumulator row (warp & 3) * 32 + l of this CTA and handles 32
    // columns at a time. Row-wise stores write 128 contiguous bytes per lane; the mirrored stores
    // of a symmetric output write, for one column, the warp's 32 consecutive rows (coalesced).
    // A product deeper than one chunk keeps its running sum in the hi plane of D, each element
    // read and written by the lane that owns it; only the last chunk applies the epilogue.
    const uint32_t quarter = (uint32_t)(warp & 3);
    uint32_t acc = 0, acc_phase = 0;
    for (uint32_t t = unit; t < total_tiles; t += n_units) {
      const Tile tl = decode_tile<kTileM, kTileN>(probs, nprobs, t);
      const GemmProblemX3 P = probs[tl.p];   // in registers: the asm below clobbers memory
      const float alpha = (ep.e_acc | ep.e_c) ? *P.alpha : 1.0f;
      const float s_acc = ep.k_acc * alpha_pow(alpha, ep.e_acc);
      const float s_c = ep.k_c * alpha_pow(alpha, ep.e_c);
      const bool has_c = P.c != nullptr && s_c != 0.0f;
      const bool fused = ep.fused != 0 && P.p != nullptr;
      const int64_t r0 = (int64_t)tl.bi * kTileM + rank * 128 + quarter * 32;
      const int64_t row = r0 + lane;
      const bool row_ok = row < (int64_t)P.M;
      const int64_t N = P.N;
      const uint32_t kblocks = (P.K + kX3BK - 1) / kX3BK;
      const uint32_t nchunks = (kblocks + kPromote - 1) / kPromote;
      for (uint32_t c = 0; c < nchunks && !timed_out; ++c) {
        const bool last = c + 1 == nchunks;
        const bool ok = __all_sync(0xffffffffu,
                                   mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, wait_ns));
        if (!ok) {
          timed_out = true;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < kTileN / 32; ++ch) {
          uint32_t r[32];
          __syncwarp();
          tmem_ld_32x32b_x32_sync(tmem_base + ((quarter * 32u) << 16) + acc * kTileN + ch * 32, r);
          if (ch == kTileN / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[acc]), 0));
          }
          const int64_t col0 = (int64_t)tl.bj * kTileN + ch * 32;
          if (r0 >= (int64_t)P.M || col0 >= N) continue;   // fully clipped (warp-uniform)
          if (P.sym && col0 + 32 <= r0) continue;           // below the diagonal: mirrored elsewhere
          const bool whole = col0 + 32 <= N;                // all 32 columns inside the matrix
          // the elements this lane owns: its row, columns inside the matrix and, for a symmetric
          // output, on or above the diagonal (the running sums of the chunks live there)
          const bool own_all = whole && (!P.sym || col0 >= row);
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
          if (nchunks > 1 && row_ok) {
            float* srow = P.d + row * P.ldd + col0;
            if (c > 0) {
              if (own_all) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                  const float4 q = reinterpret_cast<const float4*>(srow)[g];
                  v[4 * g + 0] += q.x;
                  v[4 * g + 1] += q.y;
                  v[4 * g + 2] += q.z;
                  v[4 * g + 3] += q.w;
                }
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col0 + i < N && (!P.sym || col0 + i >= row)) v[i] += srow[i];
              }
            }
            if (!last) {
              if (own_all) {
#pragma unroll
                for (int g = 0; g < 8; ++g)
                  reinterpret_cast<float4*>(srow)[g] = make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col0 + i < N && (!P.sym || col0 + i >= row)) srow[i] = v[i];
              }
              continue;
            }
          }
          if (!last) continue;
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= s_acc;
          if (row_ok) {
            if (has_c) {
              const float* c_hi = P.c + row * P.ldc + col0;
              const float* c_lo = c_hi + P.c_plane;
              if (whole) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                  const float4 h = reinterpret_cast<const float4*>(c_hi)[g];
                  const float4 l = reinterpret_cast<const float4*>(c_lo)[g];
                  v[4 * g + 0] += s_c * (h.x + l.x);
                  v[4 * g + 1] += s_c * (h.y + l.y);
                  v[4 * g + 2] += s_c * (h.z + l.z);
                  v[4 * g + 3] += s_c * (h.w + l.w);
                }
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col0 + i < N) v[i] += s_c * (c_hi[i] + c_lo[i]);
              }
            }
            if (ep.diag != 0.0f) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (col0 + i == row) v[i] += ep.diag;
            }
            if (fused) {
              float* prow = P.p + row * P.ldp + col0;
              const float step = ep.lr * P.rms;
              if (whole && P.p_vec) {
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                  float4 q = reinterpret_cast<float4*>(prow)[g];
                  q.x = q.x * ep.decay - step * v[4 * g + 0];
                  q.y = q.y * ep.decay - step * v[4 * g + 1];
                  q.z = q.z * ep.decay - step * v[4 * g + 2];
                  q.w = q.w * ep.decay - step * v[4 * g + 3];
                  reinterpret_cast<float4*>(prow)[g] = q;
                }
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col0 + i < N) prow[i] = prow[i] * ep.decay - step * v[i];
              }
            } else {
              float* drow = P.d + row * P.ldd + col0;
              if (own_all) {
#pragma unroll
                for (int g = 0; g < 8; ++g) store_split4(drow, P.d_plane, g, v);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (col0 + i < N && (!P.sym || col0 + i >= row)) store_split1(drow + i, P.d_plane, v[i]);
              }
            }
          }
          if (P.sym && !fused) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int64_t col = col0 + i;
              if (row_ok && col > row && col < N) store_split1(P.d + col * P.ldd + row, P.d_plane, v[i]);
            }
          }
        }
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (timed_out) break;
    }
    if (timed_out && lane == 0) raise_abort(abort_flag, true, rank);
  }

  if (timed_out) atomicOr(status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  // every role of both CTAs has left its loop and the producers' fill counts are visible; the even
  // CTA's producer accounts for the copies still in flight (pair_pipe.cuh)
  cluster_sync();
  if (warp == 0 && lane == 0 && leader) {
    const uint32_t peer = ld_shared_cluster(mapa_shared(smem_u32((const void*)fill_count), 1u));
    settle_pair_fills<kStages>(full, *fill_count, peer, kStageBytes, zero_flag, kTimeoutNs);
  }
  __syncwarp();
  // the pair leaves together: no CTA exits while a copy may still land in its shared memory, or
  // while its partner may still signal its barriers or (even CTA) write its tensor memory
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

cudaLaunchConfig_t pair_config(uint32_t pairs, cudaStream_t s, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

// Raises the kernel's dynamic shared-memory limit on the current device, once per device (the
// attribute belongs to one device's context).
cudaError_t set_smem_attr() {
  static PerDeviceOnce once;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return (cudaError_t)once.run(dev, [] {
    return (int)cudaFuncSetAttribute(ns_gemm_x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)kSmemBytes);
  });
}

}  // namespace

cudaError_t launch_gemm_x3(const GemmProblemX3* probs, int nprobs, uint32_t total_tiles,
                           EpiScalars ep, int* status, int max_pairs, cudaStream_t s) {
  cudaError_t e = set_smem_attr();
  if (e != cudaSuccess) return e;
  if (total_tiles == 0) return cudaSuccess;
  const uint32_t pairs = (uint32_t)max_pairs < total_tiles ? (uint32_t)max_pairs : total_tiles;
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config(pairs, s, attr);
  return cudaLaunchKernelEx(&cfg, ns_gemm_x3_kernel, probs, nprobs, total_tiles, ep, status);
}

// Largest number of CTA pairs of the 3xTF32 kernel that can be resident at once.
int gemm_x3_pair_capacity(int sms) {
  if (set_smem_attr() != cudaSuccess) {
    cudaGetLastError();
    return sms / 2;
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pair_config((uint32_t)(sms / 2), nullptr, attr);
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ns_gemm_x3_kernel, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return sms / 2;
  }
  return n;
}

}  // namespace muon
