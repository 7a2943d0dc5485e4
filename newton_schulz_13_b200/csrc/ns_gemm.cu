// Newton-Schulz matrix products ("Muon optimizer ..." `newtonschulz5`: A = X X^T,
// B = b A + c A A, X = a X + B X; "AdamW vs Muon" part 3 writes the same iteration as
// M_k = a M + b (M M^T) M + c (M M^T)^2 M).
//
// One kernel template serves all three products. A launch is a list of independent problems (one
// per matrix of a wave of the optimizer step, all at the same iteration and phase), each
//     D = s_acc * (opA . opB^T) + s_c * C + diag I,
// scheduled statically over a persistent grid; or, chained, every phase of a wave's iteration in
// one launch with tiles claimed in order (see CHAIN below). The Muon step uses the CTA-pair
// variants (clusters of two CTAs on two SMs, tcgen05 cta_group::2): 256 x 256 tiles, or 256 x 512
// "wide" tiles for the Gram and update products of large matrices. A single-CTA variant
// (128 x 256 tiles) serves the no-allocation entry point. 320 threads per CTA for the CTA-pair
// launches of one phase (eight epilogue warps), 192 for chained launches and the single CTA:
//   warp 0      TMA producer: 64-deep K slices of opA and opB into a shared-memory ring
//               (128-byte swizzle), K-major or MN-major boxes per operand; in a pair each CTA
//               loads its own 128 opA rows and its 128 of every 256 opB rows, and both CTAs'
//               copies complete on the even CTA's barrier;
//   warp 1      tcgen05.mma issuer (one thread of the even CTA in a pair): bf16 MMAs with fp32
//               accumulation in tensor memory; 256 x 256 tiles alternate between two
//               accumulators, so the epilogue of one tile overlaps the MMAs of the next, and
//               wide tiles use both 256-column slots as the two halves of one accumulator;
//   warps 2-9   epilogue (2-5 when chained or single-CTA): tcgen05.ld of the accumulator, scale, add s_c * C, round to bf16,
//               stage 32 x 32 sub-tiles in shared memory and write them with TMA stores (pair),
//               or store directly (single CTA). For the symmetric products (A = X X^T and
//               A A = A A^T) only tiles that touch the upper triangle are computed; the output
//               is written whole (the strictly-upper part also mirrored) or, on waves of small
//               matrices, in the upper-block form (only the 256-blocks on or above the diagonal;
//               readers take K slices below the diagonal transposed). The last update of a Muon
//               step applies the parameter update instead of storing D.
// Both orientations of the iterate are read in place: a wide iterate X (m x n) is K-major for
// X X^T and MN-major as the right operand of B X; a tall stored matrix G (n x m, iterate G^T)
// is MN-major for G^T G and K-major for G B. So no transposed copies are ever made.
//
// Every wait on an mbarrier is bounded. A pipeline wait (operands, accumulators, epilogue loads)
// gives up after the launch's limit (EpiScalars::wait_ns, 2 s by default); the role then raises
// the abort flag of its CTA and of the partner CTA, so that every other pipeline wait returns at
// once, and the device status word is set. Before the CTAs exit, the MMA thread waits for its
// MMAs, the producers' copies in flight are accounted for and waited for (pair_pipe.cuh), the
// epilogue waits for its loads and stores, and the tensor memory is freed. Those drain waits
// keep the long limit.
#include <cuda_bf16.h>
#include <stdint.h>

#include "device_once.h"
#include "muon_internal.h"
#include "pair_pipe.cuh"
#include "ptx.cuh"
#include "tile_sched.cuh"

namespace muon {
namespace {

constexpr uint32_t kBoxBytes = 64 * 64 * 2;  // one MN-major box: 64 K rows x 64 M/N columns
constexpr uint64_t kTimeoutNs = 2000000000ull;

// Geometry of the variants. Each CTA owns 128 accumulator rows; tensor memory holds 512 columns.
//   single CTA:  output tile 128 x 256, the CTA loads 128 rows of opA and 256 rows of opB; two
//                accumulators of 256 columns (the epilogue of one tile overlaps the next tile).
//   CTA pair:    output tile 256 x 256; each CTA loads its 128 rows of opA and 128 of the 256 opB
//                rows, the even CTA issues 256 x 256 x 16 MMAs that read both CTAs' stages; two
//                accumulators as above.
//   CTA pair, wide: output tile 256 x 512 as two 256-column halves; each CTA loads its 128 rows of
//                opA and 128 opB rows per half, and every opA slice feeds two MMAs (one per half):
//                a quarter fewer operand bytes per FLOP than the 256 x 256 tile. The halves are
//                the two 256-column slots of tensor memory (one accumulator), so the next tile's
//                MMAs wait for the drain: eight epilogue warps (two per 32-lane quarter of tensor
//                memory, each taking alternate groups of four 32-column chunks) drain half 0
//                first, and the next tile's half-0 MMAs overlap the drain of half 1. At the end
//                of a tile the last resident K slices also feed half 0 first, so that half 0
//                completes (tfull[0]) and starts draining while they feed half 1 (tfull[1]).
// CTA-pair launches of one phase run eight epilogue warps, two per 32-lane quarter of tensor
// memory (with four, the 256 x 256 products of short K waited on their epilogue: the MMA thread
// of the update waited for a free accumulator about a quarter of its time at K = 768). Chained
// launches keep four (their tile queue has one reader per epilogue warp).
template <bool PAIR, bool WIDE = false, bool CHAIN = false>
struct TcCfg {
  static_assert(PAIR || !WIDE, "the wide tile is a CTA-pair tile");
  static constexpr int kTileM = PAIR ? 256 : 128;
  static constexpr int kTileN = WIDE ? 512 : 256;
  static constexpr int kHalves = WIDE ? 2 : 1;
  static constexpr int kBRows = PAIR ? 128 * kHalves : 256;
  static constexpr int kStages = PAIR ? (WIDE ? 4 : 6) : 4;
  static constexpr uint32_t kABytes = 128 * kTcBK * 2;
  static constexpr uint32_t kBHalfBytes = 128 * kTcBK * 2;   // 128 opB rows (CTA pair)
  static constexpr uint32_t kBBytes = kBRows * kTcBK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = 512;
  // warps: TMA producer, MMA issuer, then the epilogue warps
  static constexpr int kEpiWarps = (PAIR && !CHAIN) ? 8 : 4;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kWarpChunks = kTileN / 32 / (kEpiWarps / 4);   // 32-column chunks per warp and tile
  static_assert(kWarpChunks * 32 * (kEpiWarps / 4) == kTileN, "chunks per warp");
  // arrivals that free a 256-column accumulator slot: every epilogue warp of both CTAs
  static constexpr uint32_t kEpiArrivals = PAIR ? 2 * kEpiWarps : kEpiWarps;
  // CTA pair: staging per epilogue warp in 2 KB slots (a 32 x 32 bf16 sub-tile each; two make a
  // slot for an fp32 sub-tile or a sub-tile and its mirror), 32 KB in all
  static constexpr uint32_t kSlots = kEpiWarps == 8 ? 2 : 4;
  static constexpr uint32_t kStagingPerWarp = kSlots * 2048;
  static constexpr uint32_t kStagingBytes = PAIR ? kEpiWarps * kStagingPerWarp : 0;
  static constexpr size_t kSmemBytes = kStages * kStageBytes + kStagingBytes + 1024 + 512;
  // the 512-byte tail: full and empty per stage, tfull and tempty per accumulator, drain, 16
  // epilogue operand-load barriers (one per staging slot) and the tile queue's 2 x 8 barriers;
  // then the tensor-memory address, two flags, the producer's fill count and the 8 queued tiles
  static_assert(kEpiWarps * kSlots == 16, "operand-load barriers");
  static_assert((2 * kStages + 2 + 2 + 33) * 8 + 12 * 4 <= 512, "barrier area");
  static_assert(kSmemBytes <= 232448, "dynamic shared memory per CTA");
};

// Whether K slice kb of an operand is read MN-major: always for an MN-major operand; for a
// symmetric operand in the upper-block form (half), when the slice's 256-block of K lies below the
// 256-block `rblk` of the operand's rows, where only the mirror block (K rows, operand columns) is
// stored. Both CTAs of a pair and every 16-deep MMA of a slice make the same choice.
__device__ __forceinline__ bool slice_mn(uint32_t mn, uint32_t half, uint32_t kb, uint32_t rblk) {
  return mn || (half && (kb * (uint32_t)kTcBK) / 256u < rblk);
}

// Byte offset of 16-byte chunk j of row r in a 32-row x 64-byte staging box laid out with the
// 64-byte swizzle the TMA store expects (chunk index XOR bits 1-2 of the row).
__device__ __forceinline__ uint32_t sw64_chunk(uint32_t r, uint32_t j) {
  return r * 64u + ((j ^ ((r >> 1) & 3u)) << 4);
}

// Chained launches: the tile queue's depth, and the roles that read each queued tile (the MMA
// thread, the odd CTA's producer and the eight epilogue warps of the pair).
constexpr int kTileQ = 8;
constexpr uint32_t kTileQReaders = 10;
constexpr uint32_t kNoTile = 0xffffffffu;

// CHAIN (CTA pair, 256 x 256 tiles): the launch runs all the phases of ca (see PhaseDesc). Tiles
// are claimed in order, with an atomic add, by the even CTA's producer and handed to the pair's
// other roles through a queue in shared memory; a tile waits for the phase it reads (per
// matrix) before its operands are loaded, and each epilogue warp counts its finished tiles. A
// claimed tile depends only on tiles claimed before it, so the launch makes progress whether or
// not all of its CTAs are resident.
template <bool PAIR, bool WIDE, bool CHAIN>
__global__ void __launch_bounds__(TcCfg<PAIR, WIDE, CHAIN>::kThreads, 1)
    ns_gemm_tc_kernel(const GemmProblem* __restrict__ probs, int nprobs, uint32_t total_tiles,
                      EpiScalars ep, int* __restrict__ status, ChainArgs ca) {
  static_assert(!CHAIN || (PAIR && !WIDE), "chained launches use 256 x 256 CTA-pair tiles");
  using C = TcCfg<PAIR, WIDE, CHAIN>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t* staging = smem + C::kStages * C::kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::kStagingBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;                       // followed by 16 operand-load barriers
  uint64_t* tq_full = drain + 17;                     // tile queue (chained launches)
  uint64_t* tq_empty = tq_full + kTileQ;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tq_empty + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* zero_flag = abort_flag + 1;   // never set: the drain waits poll it
  volatile uint32_t* fill_count = reinterpret_cast<volatile uint32_t*>(zero_flag + 1);
  volatile uint32_t* tq = fill_count + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;      // 0: the CTA that issues the MMAs
  const uint64_t wait_ns = ep.wait_ns ? ep.wait_ns : kTimeoutNs;   // pipeline waits
  const bool leader = rank == 0;
  const uint32_t unit = PAIR ? blockIdx.x / 2 : blockIdx.x;  // pair (or CTA) index
  const uint32_t n_units = PAIR ? gridDim.x / 2 : gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], C::kEpiArrivals);
    }
    mbar_init(drain, 1);
    for (int w = 0; w < 16; ++w) mbar_init(drain + 1 + w, 1);
    for (int q = 0; q < kTileQ; ++q) {
      mbar_init(&tq_full[q], 1);
      mbar_init(&tq_empty[q], kTileQReaders);
    }
    *abort_flag = 0;
    *zero_flag = 0;
    *fill_count = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) cluster_sync();   // the peer may signal the even CTA's barriers from now on
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  bool timed_out = false;

  // ---- the tiles of this CTA (pair), in order. seq counts the tiles a role has taken; returns
  // false when there are no more (or a wait gave up, and timed_out is set). Static launches walk
  // the tile index with a stride of n_units. Chained launches: the even CTA's producer (claimer)
  // takes the next index with an atomic add and queues it in both CTAs; the other roles read it
  // from their CTA's queue (warp_wide: every lane of an epilogue warp) and release the entry.
  // The claimer reserves one tile ahead: the atomic for the following tile goes out when a tile
  // is handed out, so its latency overlaps that tile's loads instead of stalling the producer.
  uint32_t reserved = kNoTile;
  bool have_reserved = false;
  auto next_tile = [&](uint32_t& seq, uint32_t& t, bool claimer, bool warp_wide) -> bool {
    if constexpr (!CHAIN) {
      t = unit + seq * n_units;
      ++seq;
      return t < total_tiles;
    } else {
      const uint32_t q = seq % kTileQ, par = (seq / kTileQ) & 1u;
      if (claimer) {
        if (!mbar_wait_bounded(&tq_empty[q], par ^ 1u, abort_flag, wait_ns)) {
          timed_out = true;
          return false;
        }
        uint32_t v = have_reserved ? reserved : atomicAdd(ca.tile_counter, 1u);
        if (v >= total_tiles) v = kNoTile;
        have_reserved = v != kNoTile;
        if (have_reserved) reserved = atomicAdd(ca.tile_counter, 1u);   // used at the next call
        tq[q] = v;
        st_shared_cluster(mapa_shared(smem_u32((const void*)&tq[q]), 1u), v);
        mbar_arrive(&tq_full[q]);
        mbar_arrive_cluster(mapa_shared(smem_u32(&tq_full[q]), 1u));
        t = v;
      } else {
        bool ok = mbar_wait_cluster_bounded(&tq_full[q], par, abort_flag, wait_ns);
        if (warp_wide) ok = __all_sync(0xffffffffu, ok);
        if (!ok) {
          timed_out = true;
          return false;
        }
        t = tq[q];
        if (!warp_wide || lane == 0) {
          if (leader) mbar_arrive(&tq_empty[q]);
          else mbar_arrive_cluster(mapa_shared(smem_u32(&tq_empty[q]), 0u));
        }
      }
      ++seq;
      return t != kNoTile;
    }
  };
  // problem, tile coordinates, epilogue scalars and phase of global tile t
  auto decode = [&](uint32_t t, Tile& tl, const GemmProblem*& P, const EpiScalars*& E, int& ph) {
    if constexpr (CHAIN) {
      int lo = 0, hi = ca.nphases - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (ca.phases[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
      }
      const PhaseDesc& D = ca.phases[lo];
      tl = decode_tile<C::kTileM, C::kTileN>(D.probs, D.nprobs, t - D.tile_begin);
      P = &D.probs[tl.p];
      E = &D.ep;
      ph = lo;
    } else {
      tl = decode_tile<C::kTileM, C::kTileN>(probs, nprobs, t);
      P = &probs[tl.p];
      E = &ep;
      ph = 0;
    }
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (every CTA)
    if (lane == 0) {
      int issued_parity[C::kStages];
      for (int s = 0; s < C::kStages; ++s) issued_parity[s] = -1;
      uint32_t stage = 0, phase = 0, fills = 0, seq = 0, t = 0;
      uint32_t dep_done = 0xffffffffu;   // chained: last (phase, matrix) dependency seen complete
      while (!timed_out && next_tile(seq, t, leader, false)) {
        Tile tl;
        const GemmProblem* Pp;
        const EpiScalars* Ep;
        int ph;
        decode(t, tl, Pp, Ep, ph);
        // a copy in registers: the asm statements below clobber memory, which would make every use
        // of a field of the table in global memory a fresh load
        const GemmProblem P = *Pp;
        if constexpr (CHAIN) {
          // the results this tile reads (same matrix, earlier phase) must be complete
          const PhaseDesc& D = ca.phases[ph];
          // completion counts only grow: a dependency seen complete stays complete
          const uint32_t key = ((uint32_t)D.dep << 16) | P.mat;
          if (D.dep >= 0 && key != dep_done) {
            if (!counter_wait_bounded(ca.done + (size_t)D.dep * ca.nmats + P.mat, D.dep_target[P.mat], abort_flag,
                                      wait_ns)) {
              timed_out = true;
              break;
            }
            fence_proxy_async_global();
            dep_done = key;
          }
        }
        const uint32_t kblocks = (P.K + kTcBK - 1) / kTcBK;
        const int32_t a_row0 = (int32_t)(tl.bi * C::kTileM + rank * 128);
        // single CTA: all 256 opB rows of the tile; pair: this CTA's 128 rows of each 256-wide half
        const int32_t b_row0 = (int32_t)(tl.bj * C::kTileN + rank * (PAIR ? 128 : 0));
        // 256-blocks of the operands' rows (symmetric operands in the upper-block form)
        const uint32_t rblk_a = (tl.bi * C::kTileM) / 256u;
        auto rblk_b = [&](int hf) { return (tl.bj * C::kTileN + 256u * (uint32_t)hf) / 256u; };
        for (uint32_t kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, wait_ns)) {
            timed_out = true;
            break;
          }
          uint8_t* a_dst = smem + stage * C::kStageBytes;
          uint8_t* b_dst = a_dst + C::kABytes;
          const int32_t k0 = (int32_t)(kb * kTcBK);
          if constexpr (PAIR) {
            // both halves of the pair count on the even CTA's barrier
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::kStageBytes);
            if (!slice_mn(P.a_mn, P.a_half, kb, rblk_a)) {
              tma_load_2d_pair(a_dst, P.tma_a, bar, k0, a_row0);
            } else {
              const CUtensorMap* map = P.a_mn ? P.tma_a : P.tma_a_t;
              for (int h = 0; h < 2; ++h)
                tma_load_2d_pair(a_dst + h * kBoxBytes, map, bar, a_row0 + 64 * h, k0);
            }
#pragma unroll
            for (int hf = 0; hf < C::kHalves; ++hf) {
              uint8_t* bh = b_dst + hf * C::kBHalfBytes;
              const int32_t brow = b_row0 + 256 * hf;
              if (!slice_mn(P.b_mn, P.b_half, kb, rblk_b(hf))) {
                tma_load_2d_pair(bh, P.tma_b, bar, k0, brow);
              } else {
                const CUtensorMap* map = P.b_mn ? P.tma_b : P.tma_b_t;
                for (int h = 0; h < 2; ++h)
                  tma_load_2d_pair(bh + h * kBoxBytes, map, bar, brow + 64 * h, k0);
              }
            }
          } else {
            mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
            if (!P.a_mn) {
              tma_load_2d(a_dst, P.tma_a, &full[stage], k0, a_row0);
            } else {
              for (int h = 0; h < 2; ++h)
                tma_load_2d(a_dst + h * kBoxBytes, P.tma_a, &full[stage], a_row0 + 64 * h, k0);
            }
            if (!P.b_mn) {
              tma_load_2d(b_dst, P.tma_b, &full[stage], k0, b_row0);
            } else {
              for (int h = 0; h < C::kBRows / 64; ++h)
                tma_load_2d(b_dst + h * kBoxBytes, P.tma_b, &full[stage], b_row0 + 64 * h, k0);
            }
          }
          issued_parity[stage] = (int)phase;
          ++fills;
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (timed_out) raise_abort(abort_flag, PAIR, rank);
      if constexpr (PAIR) {
        *fill_count = fills;   // settled with the partner's count at exit (pair_pipe.cuh)
      } else {
        // copies in flight must land before this CTA's shared memory is released
        for (int s = 0; s < C::kStages; ++s)
          if (issued_parity[s] >= 0)
            mbar_wait_bounded(&full[s], (uint32_t)issued_parity[s], zero_flag, kTimeoutNs);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && leader) {
      uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0, seq = 0, t = 0;
      while (!timed_out && next_tile(seq, t, false, false)) {
        Tile tl;
        const GemmProblem* Pp;
        const EpiScalars* Ep;
        int ph;
        decode(t, tl, Pp, Ep, ph);
        const GemmProblem P = *Pp;   // in registers (see the producer)
        const uint32_t kblocks = (P.K + kTcBK - 1) / kTcBK;
        const uint32_t rblk_a = (tl.bi * C::kTileM) / 256u;
        // the MMAs (kTileM x 256 x 16 each; the wide tile issues them per half) of K slice kb for
        // one 256-column half; the operand layouts follow the producer's choice for that slice
        auto issue = [&](uint32_t stg, int hf, bool first_slice, uint32_t kb) {
          const uint32_t amn = slice_mn(P.a_mn, P.a_half, kb, rblk_a) ? 1u : 0u;
          const uint32_t bmn = slice_mn(P.b_mn, P.b_half, kb, (tl.bj * C::kTileN + 256u * (uint32_t)hf) / 256u) ? 1u : 0u;
          const uint32_t idesc = idesc_bf16_f32(C::kTileM, 256, amn, bmn);
          const uint32_t a_lbo = amn ? kBoxBytes : 16u, b_lbo = bmn ? kBoxBytes : 16u;
          const uint32_t a_kstep = amn ? 16u * 128u : 32u, b_kstep = bmn ? 16u * 128u : 32u;
          const uint32_t a_addr = smem_u32(smem + stg * C::kStageBytes);
          const uint32_t b_addr = a_addr + C::kABytes + hf * C::kBHalfBytes;
          const uint32_t d_tmem = tmem_base + (WIDE ? hf : acc) * 256u;
#pragma unroll
          for (uint32_t k = 0; k < kTcBK / 16; ++k) {
            const uint64_t ad = smem_desc_sw128(a_addr + k * a_kstep, a_lbo, 1024);
            const uint64_t bd = smem_desc_sw128(b_addr + k * b_kstep, b_lbo, 1024);
            const uint32_t accumulate = (!first_slice || k != 0u) ? 1u : 0u;
            if constexpr (PAIR) tc_mma_f16_pair(d_tmem, ad, bd, idesc, accumulate);
            else tc_mma_f16(d_tmem, ad, bd, idesc, accumulate);
          }
        };
        auto release = [&](uint32_t stg) {
          if constexpr (PAIR) tc_commit_pair_mc(&empty[stg], 0x3);
          else tc_commit(&empty[stg]);
        };
        if constexpr (!WIDE) {
          if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, wait_ns)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
          for (uint32_t kb = 0; kb < kblocks; ++kb) {
            if (!mbar_wait_bounded(&full[stage], phase, abort_flag, wait_ns)) {
              timed_out = true;
              break;
            }
            tc_fence_after();
            issue(stage, 0, kb == 0, kb);
            release(stage);
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          }
          if (timed_out) break;
          if constexpr (PAIR) tc_commit_pair_mc(&tfull[acc], 0x3);
          else tc_commit(&tfull[acc]);
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        } else {
          // Half 0 may start as soon as the epilogue has drained half 0 of the previous tile:
          // the first (up to kStages) resident K slices feed half 0 only; once half 1 is free
          // too, the same slices feed half 1 and are released, then both halves go together.
          if (!mbar_wait_bounded(&tempty[0], acc_phase ^ 1u, abort_flag, wait_ns)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
          const uint32_t npre = kblocks < (uint32_t)C::kStages ? kblocks : (uint32_t)C::kStages;
          uint32_t st = stage, ph = phase;
          for (uint32_t i = 0; i < npre; ++i) {
            if (!mbar_wait_bounded(&full[st], ph, abort_flag, wait_ns)) {
              timed_out = true;
              break;
            }
            tc_fence_after();
            issue(st, 0, i == 0, i);
            if (++st == C::kStages) { st = 0; ph ^= 1u; }
          }
          if (timed_out) break;
          if (!mbar_wait_bounded(&tempty[1], acc_phase ^ 1u, abort_flag, wait_ns)) {
            timed_out = true;
            break;
          }
          tc_fence_after();
          for (uint32_t i = 0; i < npre; ++i) {
            issue(stage, 1, i == 0, i);
            release(stage);
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          }
          // the last (up to kStages) K slices feed half 0 first, so that half 0 is complete, and
          // its drain starts, while they still feed half 1
          const uint32_t npost = kblocks - npre < (uint32_t)C::kStages ? kblocks - npre : (uint32_t)C::kStages;
          for (uint32_t kb = npre; kb < kblocks - npost; ++kb) {
            if (!mbar_wait_bounded(&full[stage], phase, abort_flag, wait_ns)) {
              timed_out = true;
              break;
            }
            tc_fence_after();
            issue(stage, 0, false, kb);
            issue(stage, 1, false, kb);
            release(stage);
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          }
          if (timed_out) break;
          st = stage;
          ph = phase;
          for (uint32_t kb = kblocks - npost; kb < kblocks; ++kb) {
            if (!mbar_wait_bounded(&full[st], ph, abort_flag, wait_ns)) {
              timed_out = true;
              break;
            }
            tc_fence_after();
            issue(st, 0, false, kb);
            if (++st == C::kStages) { st = 0; ph ^= 1u; }
          }
          if (timed_out) break;
          tc_commit_pair_mc(&tfull[0], 0x3);   // half 0 of the tile
          for (uint32_t kb = kblocks - npost; kb < kblocks; ++kb) {
            issue(stage, 1, false, kb);
            release(stage);
            if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
          }
          tc_commit_pair_mc(&tfull[1], 0x3);   // half 1
          acc_phase ^= 1u;
        }
      }
      if (timed_out) raise_abort(abort_flag, PAIR, rank);
      // all issued MMAs must finish before the tensor memory is freed
      if constexpr (PAIR) tc_commit_pair(drain);
      else tc_commit(drain);
      mbar_wait_bounded(drain, 0, zero_flag, kTimeoutNs);
    }
    __syncwarp();
  } else if constexpr (PAIR) {
    // ------------------------------------------------------------ epilogue warps 2..9 (pair; 2..5 chained)
    // Each warp owns 32 accumulator rows (a 32-lane quarter of tensor memory; with eight warps,
    // two share a quarter and split its columns). Per 32-column chunk it forms
    //   D = k_acc alpha^e acc + k_c C + diag I
    // in fp32, rounds to bf16, stages the 32 x 32 sub-tile in shared memory (64-byte swizzle) and
    // writes it with a TMA store; rows and columns past the matrix are clipped by the store. A
    // symmetric output is written whole (sym 1: sub-tiles strictly above the diagonal are also
    // staged transposed and stored at the mirrored position, those strictly below are skipped)
    // or in the upper-block form (sym 2: chunks in a 256-block below the diagonal are skipped).
    // The chunks a tile writes ("active") are one contiguous range.
    // A warp's chunks: all eight of a 256-column tile (four warps, chained); with two warps per
    // quarter, chunks 0-3 or 4-7 of a 256-column tile, or alternate groups of four of a 512-column
    // tile, so that half 0 is drained first by both. The warp's active chunks are one contiguous
    // run of its own list.
    // Staging is a ring of 2 KB slots per warp (four with four warps, two with eight) that the
    // active chunks use in turn: one slot per bf16 sub-tile, or pairs of slots for the fused last
    // update (fp32 parameter sub-tiles) and for whole symmetric outputs (a sub-tile and its
    // mirror). A chunk that reads an operand sub-tile (the addend C, or the parameters) has its
    // load issued `ahead` active chunks earlier into the slot it will use (half the ring with 2 KB
    // slots, one less than the ring with 4 KB slots), once the store that used that slot last has
    // read it.
    const uint32_t quarter = (uint32_t)(warp & 3);
    const uint32_t sub = (uint32_t)(warp - 2) >> 2;   // wide tile: which groups of four chunks
    auto ch_of = [&](int i) -> int {
      return WIDE ? ((i >> 2) << 3) + (int)(sub << 2) + (i & 3) : (C::kEpiWarps == 8 ? (int)(sub << 2) + i : i);
    };
    uint8_t* stg = staging + (uint32_t)(warp - 2) * C::kStagingPerWarp;
    uint64_t* cbar = drain + 1 + C::kSlots * (warp - 2);   // this warp's operand-load barriers, one per slot
    uint32_t cph = 0;        // bit s: phase of cbar[s]
    uint32_t inflight = 0;   // bit s: a load into slot s not yet waited for
    uint32_t ring = 0;       // slot of the next active chunk
    int geo = -1;            // slot geometry in use: 0 2 KB slots, 1 4 KB slots
    uint32_t acc = 0, acc_phase = 0, seq = 0, t = 0;
    uint32_t dep_done = 0xffffffffu;   // chained: last (phase, matrix) dependency seen complete
    while (next_tile(seq, t, false, true)) {
      Tile tl;
      const GemmProblem* Pp;
      const EpiScalars* Ep;
      int ph;
      decode(t, tl, Pp, Ep, ph);
      const GemmProblem P = *Pp;   // in registers (see the producer)
      const EpiScalars ep = *Ep;   // this tile's phase (the launch's own scalars when not chained)
      const float alpha = ep.e_acc ? *P.alpha : 1.0f;
      const float s1 = ep.k_acc * alpha_pow(alpha, ep.e_acc);
      const bool has_c = P.tma_c != nullptr && ep.k_c != 0.0f;
      // the wide tile completes half 0 on tfull[0], half 1 on tfull[1] (waited for in step)
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait_bounded(&tfull[WIDE ? 0 : acc], acc_phase, abort_flag, wait_ns));
      if (!ok) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const int32_t r0 = (int32_t)(tl.bi * C::kTileM + rank * 128 + quarter * 32);
      const int32_t col0 = (int32_t)(tl.bj * C::kTileN);
      const bool fused = ep.fused != 0;
      const bool whole_sym = P.sym == 1;
      const int g = (fused || whole_sym) ? 1 : 0;
      if (g != geo) {   // the slots change size: every earlier store has read its slot
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        ring = 0;
        geo = g;
      }
      const uint32_t nslot = g ? C::kSlots / 2 : C::kSlots, slot_bytes = g ? 4096u : 2048u;
      const int ahead = g ? (int)nslot - 1 : (int)nslot / 2;
      // active chunks [lo, hi): inside the matrix and, for a symmetric output, not below the
      // 32 x 32 diagonal (whole form) or in a 256-block on or above the diagonal (upper-block
      // form); the same for every lane
      int lo = 0, hi = 0;
      if (r0 < (int32_t)P.M && col0 < (int32_t)P.N) {
        hi = min(C::kTileN / 32, ((int32_t)P.N - col0 + 31) / 32);
        const int32_t first = whole_sym ? r0 : (P.sym ? (int32_t)(tl.bi * C::kTileM) : col0);
        lo = min(hi, max(0, (first - col0) / 32));
      }
      // this warp's active chunks: positions [i_lo, i_hi) of its list
      int i_lo = 0, i_hi = 0;
#pragma unroll
      for (int i = 0; i < C::kWarpChunks; ++i) {
        i_lo += ch_of(i) < lo ? 1 : 0;
        i_hi += ch_of(i) < hi ? 1 : 0;
      }
      const int n_act = i_hi - i_lo;
      const bool loads = fused || has_c;
      const CUtensorMap* load_map = fused ? P.tma_p : P.tma_c;
      const uint32_t load_bytes = fused ? 4096u : 2048u;
      auto slot_of = [&](int q) { return (ring + (uint32_t)q) % nslot; };
      auto issue_load = [&](int q) {   // lane 0: the operand sub-tile of active chunk q
        const uint32_t sl = slot_of(q);
        mbar_arrive_expect_tx(&cbar[sl], load_bytes);
        tma_load_2d(stg + sl * slot_bytes, load_map, &cbar[sl], col0 + ch_of(i_lo + q) * 32, r0);
      };
      if constexpr (CHAIN) {
        // the addend (the Gram product) was written by other CTAs: the dependency the producer
        // waited for also orders this warp's loads of it
        const PhaseDesc& D = ca.phases[ph];
        const uint32_t key = ((uint32_t)D.dep << 16) | P.mat;
        if (has_c && D.dep >= 0 && key != dep_done) {
          if (lane == 0) {
            counter_wait_bounded(ca.done + (size_t)D.dep * ca.nmats + P.mat, D.dep_target[P.mat], abort_flag, wait_ns);
            fence_proxy_async_global();
          }
          __syncwarp();
          dep_done = key;
        }
      }
      if (loads && n_act > 0) {
        // the stores of earlier tiles have read their slots; the first loads of this tile go out
        if (lane == 0) {
          bulk_wait_group_read<0>();
          for (int q = 0; q < ahead && q < n_act; ++q) issue_load(q);
        }
        for (int q = 0; q < ahead && q < n_act; ++q) inflight |= 1u << slot_of(q);
      }
      const uint32_t tmem_row = (quarter * 32u) << 16;
      auto tmem_col = [&](int c) { return (WIDE ? 0u : acc * 256u) + (uint32_t)c * 32u; };
      // chunk i of this warp's list, whose accumulator values are in r; false when an operand-load
      // wait gave up
      auto chunk = [&](const uint32_t (&r)[32], int i) -> bool {
        // a 256-column slot is free once its last chunks are in registers (wide: half 0 after
        // each warp's first four, so the next tile's half-0 MMAs can start while half 1 drains)
        if (WIDE ? (i & 3) == 3 : i == C::kWarpChunks - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[WIDE ? i >> 2 : acc]), 0));
        }
        if (i < i_lo || i >= i_hi) return true;
        const int q = i - i_lo;
        const int ch = ch_of(i);
        const uint32_t sl = slot_of(q);
        uint8_t* buf = stg + sl * slot_bytes;
        const int32_t c0 = col0 + ch * 32;
        const bool mirror = whole_sym && c0 >= r0 + 32;
        uint8_t* mirr = buf + 2048u;   // the mirrored sub-tile's half of a 4 KB slot
        if (loads) {
          if (q + ahead < n_act) {
            if (lane == 0) {
              // that slot was last used by the store of active chunk q + ahead - nslot
              bulk_wait_group_read_upto(nslot - ahead - 1);
              issue_load(q + ahead);
            }
            inflight |= 1u << slot_of(q + ahead);
          }
          const bool got = __all_sync(0xffffffffu, mbar_wait_bounded(&cbar[sl], (cph >> sl) & 1u, abort_flag,
                                                                     wait_ns));
          if (!got) return false;
          cph ^= 1u << sl;
          inflight &= ~(1u << sl);
        } else {
          // this slot was last used by the store of active chunk q - nslot
          if (lane == 0) bulk_wait_group_read_upto(nslot - 1);
          __syncwarp();
        }
        if (fused) {
          // last update: the slot holds the 32 x 32 fp32 parameter sub-tile (128-byte swizzle); O
          // stays in fp32 and is never stored
          const float step = ep.lr * P.rms * s1;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4* qv = reinterpret_cast<float4*>(buf + (uint32_t)lane * 128u +
                                                   ((((uint32_t)j) ^ ((uint32_t)lane & 7u)) << 4));
            float4 pv = *qv;
            pv.x = pv.x * ep.decay - step * __uint_as_float(r[4 * j + 0]);
            pv.y = pv.y * ep.decay - step * __uint_as_float(r[4 * j + 1]);
            pv.z = pv.z * ep.decay - step * __uint_as_float(r[4 * j + 2]);
            pv.w = pv.w * ep.decay - step * __uint_as_float(r[4 * j + 3]);
            *qv = pv;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(P.tma_p, buf, c0, r0);
            bulk_commit_group();
          }
          return true;
        }
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = s1 * __uint_as_float(r[i]);
        if (has_c) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 raw = *reinterpret_cast<const uint4*>(buf + sw64_chunk((uint32_t)lane, (uint32_t)j));
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __bfloat1622float2(h[i]);
              v[8 * j + 2 * i] += ep.k_c * f.x;
              v[8 * j + 2 * i + 1] += ep.k_c * f.y;
            }
          }
          __syncwarp();   // every lane has read its addend row before the slot is overwritten
        }
        if (P.sym && c0 == r0) {   // a diagonal sub-tile
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i == lane) v[i] += ep.diag;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint4 raw;
          __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
          for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[8 * j + 2 * i], v[8 * j + 2 * i + 1]);
          *reinterpret_cast<uint4*>(buf + sw64_chunk((uint32_t)lane, (uint32_t)j)) = raw;
        }
        if (mirror) {
          // element (row lane, column i) goes to row i, column lane of the transposed box
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const uint32_t off = sw64_chunk((uint32_t)i, (uint32_t)lane >> 3) + ((uint32_t)lane & 7u) * 2u;
            *reinterpret_cast<__nv_bfloat16*>(mirr + off) = __float2bfloat16_rn(v[i]);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(P.tma_d, buf, c0, r0);
          if (mirror) tma_store_2d(P.tma_d, mirr, r0, c0);
          bulk_commit_group();
        }
        return true;
      };
      // Tensor-memory loads run one chunk ahead: the load of the warp's next active chunk is
      // issued before the current chunk is processed and waited for after it.
      auto step = [&](const uint32_t (&cur)[32], uint32_t (&nxt)[32], int i) -> bool {
        __syncwarp();
        // wide: the warp's next chunk is the first of half 1, which completes on tfull[1]
        const bool boundary = WIDE && i == C::kWarpChunks / 2 - 1;
        const bool pre = !boundary && i + 1 >= i_lo && i + 1 < i_hi;
        if (pre) tmem_ld_32x32b_x32_issue(tmem_base + tmem_row + tmem_col(ch_of(i + 1)), nxt);
        bool ok = chunk(cur, i);
        if (pre) tmem_ld_wait_regs(nxt);
        if (boundary && ok) {
          ok = __all_sync(0xffffffffu, mbar_wait_bounded(&tfull[1], acc_phase, abort_flag, wait_ns));
          tc_fence_after();
          __syncwarp();
          if (ok && i + 1 >= i_lo && i + 1 < i_hi)
            tmem_ld_32x32b_x32_sync(tmem_base + tmem_row + tmem_col(ch_of(i + 1)), nxt);
        }
        return ok;
      };
      uint32_t ra[32], rb[32];
      __syncwarp();
      if (i_lo == 0 && i_hi > 0) tmem_ld_32x32b_x32_sync(tmem_base + tmem_row + tmem_col(ch_of(0)), ra);
      bool chunks_ok = true;
#pragma unroll 1
      for (int i = 0; i < C::kWarpChunks && chunks_ok; i += 2) {   // kWarpChunks is even
        chunks_ok = step(ra, rb, i);
        if (chunks_ok) chunks_ok = step(rb, ra, i + 1);
      }
      if (!chunks_ok) timed_out = true;
      if (timed_out) break;
      ring = (ring + (uint32_t)n_act) % nslot;
      if constexpr (CHAIN) {
        // this warp's stores of the tile are complete: count them for the phases that read them
        // (publishing at once measured faster than collecting several tiles per publication)
        if (lane == 0) {
          bulk_wait_group_all();
          fence_proxy_async_global();
          red_release_gpu_add(ca.done + (size_t)ph * ca.nmats + P.mat, 1u);
        }
        __syncwarp();
      }
      if constexpr (WIDE) {
        acc_phase ^= 1u;
      } else if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
    if (timed_out && lane == 0) raise_abort(abort_flag, PAIR, rank);
    // loads still in flight (only after a timeout) must land before the CTA exits
    if (lane == 0)
      for (uint32_t sl = 0; sl < C::kSlots; ++sl)
        if (inflight & (1u << sl)) mbar_wait_bounded(&cbar[sl], (cph >> sl) & 1u, zero_flag, kTimeoutNs);
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue warps 2..5
    const uint32_t quarter = (uint32_t)(warp & 3);
    uint32_t acc = 0, acc_phase = 0;
    for (uint32_t t = unit; t < total_tiles; t += n_units) {
      const Tile tl = decode_tile<C::kTileM, C::kTileN>(probs, nprobs, t);
      const GemmProblem& P = probs[tl.p];
      const float alpha = (ep.e_acc | ep.e_c) ? *P.alpha : 1.0f;
      const float s_acc = ep.k_acc * alpha_pow(alpha, ep.e_acc);
      const float s_c = ep.k_c * alpha_pow(alpha, ep.e_c);
      const bool has_c = (P.c != nullptr) && (s_c != 0.0f);
      // every lane polls; the outcome is made warp-uniform so that the warp stays converged
      // for the .sync.aligned tensor-memory loads below
      const bool ok = __all_sync(0xffffffffu,
                                 mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, wait_ns));
      if (!ok) {
        timed_out = true;
        break;
      }
      tc_fence_after();
      const int64_t row = (int64_t)tl.bi * C::kTileM + rank * 128 + quarter * 32 + lane;
      const bool row_ok = row < (int64_t)P.M;
      const int64_t N = P.N;
#pragma unroll 1
      for (int ch = 0; ch < C::kTileN / 32; ++ch) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld_32x32b_x32_sync(tmem_base + ((quarter * 32u) << 16) + acc * C::kTileN + ch * 32, r);
        if (ch == C::kTileN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[acc]);
        }
        const int64_t col0 = (int64_t)tl.bj * C::kTileN + ch * 32;
        if (!row_ok || col0 >= N) continue;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = s_acc * __uint_as_float(r[i]);
        if (has_c) {
          const __nv_bfloat16* crow = P.c + row * P.ldc;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const int64_t cg = col0 + 8 * g;
            if (cg + 8 <= N) {
              const uint4 raw = *reinterpret_cast<const uint4*>(crow + cg);
              const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h[i]);
                v[8 * g + 2 * i] += s_c * f.x;
                v[8 * g + 2 * i + 1] += s_c * f.y;
              }
            } else {
              for (int e = 0; e < 8; ++e)
                if (cg + e < N) v[8 * g + e] += s_c * __bfloat162float(crow[cg + e]);
            }
          }
        }
        __nv_bfloat16* drow = P.d + row * P.ldd;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int64_t cg = col0 + 8 * g;
          if (cg + 8 <= N && (!P.sym || cg >= row)) {
            uint4 raw;
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[8 * g + 2 * i], v[8 * g + 2 * i + 1]);
            *reinterpret_cast<uint4*>(drow + cg) = raw;
          } else {
            for (int e = 0; e < 8; ++e) {
              const int64_t col = cg + e;
              if (col < N && (!P.sym || col >= row)) drow[col] = __float2bfloat16_rn(v[8 * g + e]);
            }
          }
        }
        if (P.sym) {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int64_t col = col0 + i;
            if (col > row && col < N) P.d[col * P.ldd + row] = __float2bfloat16_rn(v[i]);
          }
        }
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (timed_out && lane == 0) raise_abort(abort_flag, false, rank);
  }

  if (timed_out) atomicOr(status, kStatusTimeout);
  tc_fence_before();
  __syncthreads();
  if constexpr (PAIR) {
    // every role of both CTAs has left its loop and the producers' fill counts are visible; the
    // even CTA's producer accounts for the copies still in flight (pair_pipe.cuh)
    cluster_sync();
    if (warp == 0 && lane == 0 && leader) {
      const uint32_t peer = ld_shared_cluster(mapa_shared(smem_u32((const void*)fill_count), 1u));
      settle_pair_fills<C::kStages>(full, *fill_count, peer, C::kStageBytes, zero_flag, kTimeoutNs);
    }
    __syncwarp();
    // the pair leaves together: no CTA exits while a copy may still land in its shared memory,
    // or while its partner may still signal its barriers or (even CTA) write its tensor memory
    cluster_sync();
  }
  tc_fence_after();
  if (warp == 1) {
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// Raises a kernel's dynamic shared-memory limit on the current device, once per device (the
// attribute belongs to one device's context). `once` is the kernel's own set of flags.
cudaError_t set_smem_limit(const void* kernel, int bytes, PerDeviceOnce& once) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return (cudaError_t)once.run(dev, [&] {
    return (int)cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmProblem* probs, int nprobs, uint32_t total_tiles,
                           EpiScalars ep, int* status, int grid, cudaStream_t s) {
  using C = TcCfg<false>;
  static PerDeviceOnce once;
  cudaError_t e = set_smem_limit((const void*)ns_gemm_tc_kernel<false, false, false>, (int)C::kSmemBytes, once);
  if (e != cudaSuccess) return e;
  if (total_tiles == 0) return cudaSuccess;
  if ((uint32_t)grid > total_tiles) grid = (int)total_tiles;
  ns_gemm_tc_kernel<false, false, false><<<grid, C::kThreads, C::kSmemBytes, s>>>(probs, nprobs, total_tiles, ep, status,
                                                                               ChainArgs{});
  return cudaGetLastError();
}

namespace {

template <bool WIDE, bool CHAIN>
cudaError_t launch_pair(const GemmProblem* probs, int nprobs, uint32_t total_tiles, EpiScalars ep,
                        int* status, int max_pairs, cudaStream_t s, ChainArgs ca) {
  using C = TcCfg<true, WIDE, CHAIN>;
  static PerDeviceOnce once;   // one per instantiation
  cudaError_t e = set_smem_limit((const void*)ns_gemm_tc_kernel<true, WIDE, CHAIN>, (int)C::kSmemBytes, once);
  if (e != cudaSuccess) return e;
  if (total_tiles == 0) return cudaSuccess;
  const uint32_t pairs = (uint32_t)max_pairs < total_tiles ? (uint32_t)max_pairs : total_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, ns_gemm_tc_kernel<true, WIDE, CHAIN>, probs, nprobs, total_tiles, ep, status, ca);
}

}  // namespace

cudaError_t launch_gemm_tc_pair(const GemmProblem* probs, int nprobs, uint32_t total_tiles,
                                EpiScalars ep, int* status, int max_pairs, cudaStream_t s) {
  return launch_pair<false, false>(probs, nprobs, total_tiles, ep, status, max_pairs, s, ChainArgs{});
}

cudaError_t launch_gemm_tc_pair_wide(const GemmProblem* probs, int nprobs, uint32_t total_tiles,
                                     EpiScalars ep, int* status, int max_pairs, cudaStream_t s) {
  return launch_pair<true, false>(probs, nprobs, total_tiles, ep, status, max_pairs, s, ChainArgs{});
}

cudaError_t launch_gemm_tc_pair_chain(ChainArgs ca, uint32_t total_tiles, EpiScalars ep, int* status,
                                      int max_pairs, cudaStream_t s) {
  return launch_pair<false, true>(nullptr, 0, total_tiles, ep, status, max_pairs, s, ca);
}

// Largest number of CTA pairs of the paired kernel that can be resident at once.
int gemm_tc_pair_capacity(int sms) {
  using C = TcCfg<true>;
  static_assert(TcCfg<true, true>::kSmemBytes == C::kSmemBytes && TcCfg<true, false, true>::kSmemBytes == C::kSmemBytes,
                "the pair variants have one occupancy");
  cudaError_t e = cudaFuncSetAttribute(ns_gemm_tc_kernel<true, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::kSmemBytes);
  if (e != cudaSuccess) return sms / 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, ns_gemm_tc_kernel<true, false, false>, &cfg);
  if (e != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return sms / 2;
  }
  return n;
}

}  // namespace muon
