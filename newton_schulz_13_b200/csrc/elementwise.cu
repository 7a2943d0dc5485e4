// Elementwise and reduction kernels of the Muon step (HBM-bound):
//   column sums and means     zero-centring along dim 0 ("Muon meets Mamba" 2.1 `zerocenter`)
//   prologue                  momentum EMA, Nesterov look-ahead, squared-norm partials and the
//                             cast of the update matrix to the Newton-Schulz working type
//                             ("Muon optimizer ..." `Muon.step` and `newtonschulz5` listings)
//   norm                      1 / (||u||_F + eps) per matrix, summed in a fixed order
//   update                    p <- p (1 - lr wd) - lr s O ("AdamW vs Muon" part 3;
//                             "Muon meets Mamba" 4.2)
//   output                    O written to the caller's buffer (orthogonalisation call)
//
// Every kernel is a grid-stride loop over fixed-size chunks of all matrices of the call, so a
// single launch covers every matrix; rows whose length is a multiple of 8 use 16-byte loads and
// stores. The 1 / (||u|| + eps) factor is not applied here: the first Newton-Schulz launch
// folds it into its epilogue, so u is read from HBM once.
#include <cuda_bf16.h>
#include <math.h>

#include <algorithm>
#include <cstring>
#include <memory>


#include "muon_internal.h"

namespace muon {
namespace {

__device__ __forceinline__ int find_mat(const MatInfo* mats, int n, int64_t item, int which) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    const int64_t b = which == 0 ? mats[mid].chunk_begin
                                 : (which == 1 ? mats[mid].cs_begin : mats[mid].cm_begin);
    if (b <= item) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <bool BF16>
__device__ __forceinline__ void load8(const void* base, int64_t idx, float (&v)[8]) {
  if constexpr (BF16) {
    const uint4 raw = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(base) + idx);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx);
    const float4 a = p[0], b = p[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <bool BF16>
__device__ __forceinline__ void store8(void* base, int64_t idx, const float (&v)[8]) {
  if constexpr (BF16) {
    uint4 raw;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(base) + idx) = raw;
  } else {
    float4* p = reinterpret_cast<float4*>(static_cast<float*>(base) + idx);
    p[0] = make_float4(v[0], v[1], v[2], v[3]);
    p[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

template <bool BF16>
__device__ __forceinline__ float load1(const void* base, int64_t idx) {
  if constexpr (BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(base)[idx]);
  else return static_cast<const float*>(base)[idx];
}

template <bool BF16>
__device__ __forceinline__ void store1(void* base, int64_t idx, float v) {
  if constexpr (BF16) static_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  else static_cast<float*>(base)[idx] = v;
}

// The Newton-Schulz iterate: bf16, or fp32 held as two planes lo_off elements apart (hi = the
// value with its 13 low mantissa bits cleared, lo = value - hi; hi + lo is the value exactly).
__device__ __forceinline__ float tf32_hi(float v) {
  return __uint_as_float(__float_as_uint(v) & 0xffffe000u);
}

template <bool X_BF16>
__device__ __forceinline__ void load8x(const void* base, int64_t idx, int64_t lo_off, float (&v)[8]) {
  load8<X_BF16>(base, idx, v);
  if constexpr (!X_BF16) {
    float l[8];
    load8<false>(base, idx + lo_off, l);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] += l[i];
  }
}

template <bool X_BF16>
__device__ __forceinline__ void store8x(void* base, int64_t idx, int64_t lo_off, const float (&v)[8]) {
  if constexpr (X_BF16) {
    store8<true>(base, idx, v);
  } else {
    float h[8], l[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      h[i] = tf32_hi(v[i]);
      l[i] = v[i] - h[i];
    }
    store8<false>(base, idx, h);
    store8<false>(base, idx + lo_off, l);
  }
}

template <bool X_BF16>
__device__ __forceinline__ float load1x(const void* base, int64_t idx, int64_t lo_off) {
  if constexpr (X_BF16) return load1<true>(base, idx);
  else return static_cast<const float*>(base)[idx] + static_cast<const float*>(base)[idx + lo_off];
}

template <bool X_BF16>
__device__ __forceinline__ void store1x(void* base, int64_t idx, int64_t lo_off, float v) {
  if constexpr (X_BF16) {
    store1<true>(base, idx, v);
  } else {
    const float h = tf32_hi(v);
    static_cast<float*>(base)[idx] = h;
    static_cast<float*>(base)[idx + lo_off] = v - h;
  }
}

// Deterministic block sum (fixed shuffle tree, fixed warp order).
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0) {
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
  }
  __syncthreads();
  return s;
}

// ---------------------------------------------------------------- per-call tables
__global__ void __launch_bounds__(256) table_write_kernel(const __grid_constant__ TableChunk c) {
  for (uint64_t i = threadIdx.x; i < c.nwords; i += blockDim.x) c.dst[i] = c.w[i];
}

// ---------------------------------------------------------------- zero-centring
template <bool G_BF16>
__global__ void __launch_bounds__(kCsCols) colsum_kernel(const MatInfo* __restrict__ mats, int nmats,
                                                         int64_t items) {
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int j = find_mat(mats, nmats, it, 1);
    const MatInfo mi = mats[j];
    const int64_t n_cb = (mi.cols + kCsCols - 1) / kCsCols;
    const int64_t local = it - mi.cs_begin;
    const int64_t rc = local / n_cb, cb = local % n_cb;
    const int64_t col = cb * kCsCols + threadIdx.x;
    if (col < mi.cols) {
      const int64_t r0 = rc * kCsRows;
      const int64_t r1 = min(mi.rows, r0 + kCsRows);
      float s = 0.f;
      for (int64_t r = r0; r < r1; ++r) s += load1<G_BF16>(mi.g, r * mi.cols + col);
      mi.colpart[rc * mi.cols + col] = s;
    }
  }
}

__global__ void __launch_bounds__(kCsCols) colmean_kernel(const MatInfo* __restrict__ mats, int nmats,
                                                          int64_t items) {
  for (int64_t it = blockIdx.x; it < items; it += gridDim.x) {
    const int j = find_mat(mats, nmats, it, 2);
    const MatInfo mi = mats[j];
    const int64_t col = (it - mi.cm_begin) * kCsCols + threadIdx.x;
    if (col < mi.cols) {
      const int64_t n_rc = (mi.rows + kCsRows - 1) / kCsRows;
      double s = 0.0;
      for (int64_t rc = 0; rc < n_rc; ++rc) s += (double)mi.colpart[rc * mi.cols + col];
      mi.colmean[col] = (float)(s / (double)mi.rows);
    }
  }
}

// ---------------------------------------------------------------- prologue
template <bool G_BF16, bool X_BF16>
__global__ void __launch_bounds__(kEwThreads, 4) prologue_kernel(const MatInfo* __restrict__ mats, int nmats,
                                                              int64_t nchunks, int has_m, float mu,
                                                              int nesterov, int zc,
                                                              float* __restrict__ partials,
                                                              int* __restrict__ status) {
  __shared__ float red[kEwThreads / 32];
  const float one_m_mu = 1.0f - mu;
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int j = find_mat(mats, nmats, chunk, 0);
    const MatInfo mi = mats[j];
    const int64_t n_el = mi.rows * mi.cols;
    const int64_t e0 = (chunk - mi.chunk_begin) * kChunk;
    const int64_t e1 = min(n_el, e0 + kChunk);
    float sq = 0.f;
    int bad = 0;
    if (mi.vec && e1 - e0 == kChunk) {
      // a full chunk: each thread owns kGroups groups of 8 elements and handles them kBatch at a
      // time, issuing all loads of a batch before any arithmetic (more bytes in flight per thread)
      constexpr int kGroups = (int)(kChunk / (8 * kEwThreads));
      constexpr int kBatch = 2;
#pragma unroll
      for (int b0 = 0; b0 < kGroups; b0 += kBatch) {
        float g[kBatch][8], m[kBatch][8];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int64_t e = e0 + 8 * ((int64_t)threadIdx.x + (int64_t)(b0 + q) * kEwThreads);
          load8<G_BF16>(mi.g, e, g[q]);
          if (has_m) load8<false>(mi.m, e, m[q]);
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int64_t e = e0 + 8 * ((int64_t)threadIdx.x + (int64_t)(b0 + q) * kEwThreads);
          const int64_t row = e / mi.cols, col = e - row * mi.cols;
          float u[8];
          if (zc) {
            const float4* cm = reinterpret_cast<const float4*>(mi.colmean + col);
            const float4 c0 = cm[0], c1 = cm[1];
            g[q][0] -= c0.x; g[q][1] -= c0.y; g[q][2] -= c0.z; g[q][3] -= c0.w;
            g[q][4] -= c1.x; g[q][5] -= c1.y; g[q][6] -= c1.z; g[q][7] -= c1.w;
          }
          if (has_m) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              m[q][i] = mu * m[q][i] + one_m_mu * g[q][i];
              u[i] = nesterov ? mu * m[q][i] + one_m_mu * g[q][i] : m[q][i];
            }
            store8<false>(mi.m, e, m[q]);
          } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) u[i] = g[q][i];
          }
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            sq += u[i] * u[i];
            bad |= !isfinite(u[i]);
          }
          store8x<X_BF16>(mi.x0, row * mi.ldx + col, mi.xlo, u);
        }
      }
    } else if (mi.vec) {
      for (int64_t e = e0 + 8 * (int64_t)threadIdx.x; e < e1; e += 8 * (int64_t)blockDim.x) {
        const int64_t row = e / mi.cols, col = e - row * mi.cols;
        float g[8], u[8];
        load8<G_BF16>(mi.g, e, g);
        if (zc) {
          const float4* cm = reinterpret_cast<const float4*>(mi.colmean + col);
          const float4 c0 = cm[0], c1 = cm[1];
          g[0] -= c0.x; g[1] -= c0.y; g[2] -= c0.z; g[3] -= c0.w;
          g[4] -= c1.x; g[5] -= c1.y; g[6] -= c1.z; g[7] -= c1.w;
        }
        if (has_m) {
          float m[8];
          load8<false>(mi.m, e, m);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            m[i] = mu * m[i] + one_m_mu * g[i];
            u[i] = nesterov ? mu * m[i] + one_m_mu * g[i] : m[i];
          }
          store8<false>(mi.m, e, m);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) u[i] = g[i];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          sq += u[i] * u[i];
          bad |= !isfinite(u[i]);
        }
        store8x<X_BF16>(mi.x0, row * mi.ldx + col, mi.xlo, u);
      }
    } else {
      for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        const int64_t row = e / mi.cols, col = e - row * mi.cols;
        float g = load1<G_BF16>(mi.g, e);
        if (zc) g -= mi.colmean[col];
        float u = g;
        if (has_m) {
          const float m = mu * mi.m[e] + one_m_mu * g;
          mi.m[e] = m;
          u = nesterov ? mu * m + one_m_mu * g : m;
        }
        sq += u * u;
        bad |= !isfinite(u);
        store1x<X_BF16>(mi.x0, row * mi.ldx + col, mi.xlo, u);
      }
    }
    const float total = block_sum(sq, red);
    if (threadIdx.x == 0) partials[chunk] = total;
    if (bad) atomicAdd(status + 1, 1);
  }
}

// One CTA per matrix: alpha = 1 / (sqrt(sum of its partials) + eps), summed in a fixed order.
__global__ void __launch_bounds__(256) alpha_kernel(const MatInfo* __restrict__ mats,
                                                    const float* __restrict__ partials, float eps) {
  __shared__ double red[256];
  const MatInfo mi = mats[blockIdx.x];
  const int64_t n = (mi.rows * mi.cols + kChunk - 1) / kChunk;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) s += (double)partials[mi.chunk_begin + i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *mi.alpha = (float)(1.0 / (sqrt(red[0]) + (double)eps));
}

// ---------------------------------------------------------------- update / output
template <bool X_BF16>
__global__ void __launch_bounds__(kEwThreads, 4) update_kernel(const MatInfo* __restrict__ mats, int nmats,
                                                            int64_t nchunks, float lr, float decay,
                                                            int scale_by_alpha) {
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int j = find_mat(mats, nmats, chunk, 0);
    const MatInfo mi = mats[j];
    const int64_t n_el = mi.rows * mi.cols;
    const int64_t e0 = (chunk - mi.chunk_begin) * kChunk;
    const int64_t e1 = min(n_el, e0 + kChunk);
    const float step = lr * mi.rms * (scale_by_alpha ? *mi.alpha : 1.0f);
    if (mi.vec && e1 - e0 == kChunk) {
      // a full chunk: loads of kBatch groups are issued before their arithmetic
      constexpr int kGroups = (int)(kChunk / (8 * kEwThreads));
      constexpr int kBatch = 2;
#pragma unroll
      for (int b0 = 0; b0 < kGroups; b0 += kBatch) {
        float o[kBatch][8], p[kBatch][8];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int64_t e = e0 + 8 * ((int64_t)threadIdx.x + (int64_t)(b0 + q) * kEwThreads);
          const int64_t row = e / mi.cols, col = e - row * mi.cols;
          load8x<X_BF16>(mi.xf, row * mi.ldx + col, mi.xlo, o[q]);
          load8<false>(mi.p, e, p[q]);
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int64_t e = e0 + 8 * ((int64_t)threadIdx.x + (int64_t)(b0 + q) * kEwThreads);
#pragma unroll
          for (int i = 0; i < 8; ++i) p[q][i] = p[q][i] * decay - step * o[q][i];
          store8<false>(mi.p, e, p[q]);
        }
      }
    } else if (mi.vec) {
      for (int64_t e = e0 + 8 * (int64_t)threadIdx.x; e < e1; e += 8 * (int64_t)blockDim.x) {
        const int64_t row = e / mi.cols, col = e - row * mi.cols;
        float o[8], p[8];
        load8x<X_BF16>(mi.xf, row * mi.ldx + col, mi.xlo, o);
        load8<false>(mi.p, e, p);
#pragma unroll
        for (int i = 0; i < 8; ++i) p[i] = p[i] * decay - step * o[i];
        store8<false>(mi.p, e, p);
      }
    } else {
      for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        const int64_t row = e / mi.cols, col = e - row * mi.cols;
        const float o = load1x<X_BF16>(mi.xf, row * mi.ldx + col, mi.xlo);
        mi.p[e] = mi.p[e] * decay - step * o;
      }
    }
  }
}

template <bool X_BF16, bool OUT_BF16>
__global__ void __launch_bounds__(kEwThreads) output_kernel(const MatInfo* __restrict__ mats, int nmats,
                                                            int64_t nchunks, int scale_by_alpha) {
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int j = find_mat(mats, nmats, chunk, 0);
    const MatInfo mi = mats[j];
    const int64_t n_el = mi.rows * mi.cols;
    const int64_t e0 = (chunk - mi.chunk_begin) * kChunk;
    const int64_t e1 = min(n_el, e0 + kChunk);
    const float s = scale_by_alpha ? *mi.alpha : 1.0f;
    if (mi.vec) {
      for (int64_t e = e0 + 8 * (int64_t)threadIdx.x; e < e1; e += 8 * (int64_t)blockDim.x) {
        const int64_t row = e / mi.cols, col = e - row * mi.cols;
        float o[8];
        load8x<X_BF16>(mi.xf, row * mi.ldx + col, mi.xlo, o);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] *= s;
        store8<OUT_BF16>(mi.p, e, o);
      }
    } else {
      for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        const int64_t row = e / mi.cols, col = e - row * mi.cols;
        store1<OUT_BF16>(mi.p, e, s * load1x<X_BF16>(mi.xf, row * mi.ldx + col, mi.xlo));
      }
    }
  }
}

// ---------------------------------------------------------------- AdamW
// The AdamW step of the parameters Muon leaves out ("Muon meets Mamba" 4.2 `_step_adamw`):
// decoupled decay first, then bias-corrected first and second moments. 4 fp32 arrays plus the
// gradient per element: 26 B (bf16 gradient) or 28 B (fp32) of HBM traffic.
__device__ __forceinline__ int find_tensor(const AdamTensor* ts, int n, int64_t chunk) {
  int lo = 0, hi = n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ts[mid].chunk_begin <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void adam_elem(float& p, float& m, float& v, float g, const AdamScalars& sc) {
  p = p * sc.decay;
  m = sc.beta1 * m + (1.0f - sc.beta1) * g;
  v = sc.beta2 * v + (1.0f - sc.beta2) * g * g;
  p = p - sc.step_size * m / (sqrtf(v) * sc.inv_sqrt_bc2 + sc.eps);
}

template <bool G_BF16>
__global__ void __launch_bounds__(kEwThreads, 4) adamw_kernel(const AdamTensor* __restrict__ ts, int n,
                                                              int64_t nchunks, AdamScalars sc) {
  for (int64_t chunk = blockIdx.x; chunk < nchunks; chunk += gridDim.x) {
    const int j = find_tensor(ts, n, chunk);
    const AdamTensor t = ts[j];
    const int64_t e0 = (chunk - t.chunk_begin) * kChunk;
    const int64_t e1 = min(t.numel, e0 + kChunk);
    if (t.vec) {
      const int64_t nvec = (e1 - e0) / 8;   // whole groups of 8; the rest below
      constexpr int kBatch = 1;             // 4 arrays x 8 values already fill the register budget
      for (int64_t q0 = threadIdx.x; q0 < nvec; q0 += (int64_t)kBatch * blockDim.x) {
        float g[kBatch][8], p[kBatch][8], m[kBatch][8], v[kBatch][8];
        bool ok[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          const int64_t q = q0 + (int64_t)b * blockDim.x;
          ok[b] = q < nvec;
          if (ok[b]) {
            const int64_t e = e0 + 8 * q;
            load8<G_BF16>(t.g, e, g[b]);
            load8<false>(t.p, e, p[b]);
            load8<false>(t.m, e, m[b]);
            load8<false>(t.v, e, v[b]);
          }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
          if (!ok[b]) continue;
          const int64_t e = e0 + 8 * (q0 + (int64_t)b * blockDim.x);
#pragma unroll
          for (int i = 0; i < 8; ++i) adam_elem(p[b][i], m[b][i], v[b][i], g[b][i], sc);
          store8<false>(t.p, e, p[b]);
          store8<false>(t.m, e, m[b]);
          store8<false>(t.v, e, v[b]);
        }
      }
      for (int64_t e = e0 + 8 * nvec + threadIdx.x; e < e1; e += blockDim.x)
        adam_elem(t.p[e], t.m[e], t.v[e], load1<G_BF16>(t.g, e), sc);
    } else {
      for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x)
        adam_elem(t.p[e], t.m[e], t.v[e], load1<G_BF16>(t.g, e), sc);
    }
  }
}

int grid_for(int64_t items, int cap) {
  return (int)(items < (int64_t)cap ? (items < 1 ? 1 : items) : cap);
}

}  // namespace

cudaError_t launch_adamw(const AdamTensor* ts, int n, int64_t chunks, int g_bf16, AdamScalars sc,
                         int grid, cudaStream_t s) {
  grid = grid_for(chunks, grid);
  if (g_bf16) adamw_kernel<true><<<grid, kEwThreads, 0, s>>>(ts, n, chunks, sc);
  else adamw_kernel<false><<<grid, kEwThreads, 0, s>>>(ts, n, chunks, sc);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const MatInfo* mats, int nmats, int64_t items, int g_bf16, cudaStream_t s) {
  const int grid = grid_for(items, 148 * 16);
  if (g_bf16) colsum_kernel<true><<<grid, kCsCols, 0, s>>>(mats, nmats, items);
  else colsum_kernel<false><<<grid, kCsCols, 0, s>>>(mats, nmats, items);
  return cudaGetLastError();
}

cudaError_t write_table(void* dst, const void* src, size_t bytes, cudaStream_t s, int64_t* launches) {
  if (bytes % 8 != 0) return cudaErrorInvalidValue;
  thread_local std::unique_ptr<TableChunk> chunk(new TableChunk());
  const uint64_t* words = static_cast<const uint64_t*>(src);
  const size_t total = bytes / 8;
  for (size_t off = 0; off < total; off += kTableWords) {
    const size_t n = std::min<size_t>(kTableWords, total - off);
    chunk->dst = static_cast<uint64_t*>(dst) + off;
    chunk->nwords = n;
    std::memcpy(chunk->w, words + off, n * 8);
    table_write_kernel<<<1, 256, 0, s>>>(*chunk);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (launches) ++*launches;
  }
  return cudaSuccess;
}

cudaError_t launch_colmean(const MatInfo* mats, int nmats, int64_t items, cudaStream_t s) {
  colmean_kernel<<<grid_for(items, 148 * 16), kCsCols, 0, s>>>(mats, nmats, items);
  return cudaGetLastError();
}

cudaError_t launch_prologue(const MatInfo* mats, int nmats, int64_t chunks, int g_bf16, int x_bf16,
                            int has_momentum, float mu, int nesterov, int zero_center,
                            float* partials, int* status, int grid, cudaStream_t s) {
  grid = grid_for(chunks, grid);
#define MUON_PRO(GB, XB)                                                                        \
  prologue_kernel<GB, XB><<<grid, kEwThreads, 0, s>>>(mats, nmats, chunks, has_momentum, mu,    \
                                                      nesterov, zero_center, partials, status)
  if (g_bf16 && x_bf16) MUON_PRO(true, true);
  else if (g_bf16) MUON_PRO(true, false);
  else if (x_bf16) MUON_PRO(false, true);
  else MUON_PRO(false, false);
#undef MUON_PRO
  return cudaGetLastError();
}

cudaError_t launch_alpha(const MatInfo* mats, int nmats, const float* partials, float eps,
                         cudaStream_t s) {
  alpha_kernel<<<nmats, 256, 0, s>>>(mats, partials, eps);
  return cudaGetLastError();
}

cudaError_t launch_update(const MatInfo* mats, int nmats, int64_t chunks, int x_bf16, float lr,
                          float decay, int scale_by_alpha, int grid, cudaStream_t s) {
  grid = grid_for(chunks, grid);
  if (x_bf16) update_kernel<true><<<grid, kEwThreads, 0, s>>>(mats, nmats, chunks, lr, decay, scale_by_alpha);
  else update_kernel<false><<<grid, kEwThreads, 0, s>>>(mats, nmats, chunks, lr, decay, scale_by_alpha);
  return cudaGetLastError();
}

cudaError_t launch_output(const MatInfo* mats, int nmats, int64_t chunks, int x_bf16, int out_bf16,
                          int scale_by_alpha, int grid, cudaStream_t s) {
  grid = grid_for(chunks, grid);
#define MUON_OUT(XB, OB) output_kernel<XB, OB><<<grid, kEwThreads, 0, s>>>(mats, nmats, chunks, scale_by_alpha)
  if (x_bf16 && out_bf16) MUON_OUT(true, true);
  else if (x_bf16) MUON_OUT(true, false);
  else if (out_bf16) MUON_OUT(false, true);
  else MUON_OUT(false, false);
#undef MUON_OUT
  return cudaGetLastError();
}

}  // namespace muon
