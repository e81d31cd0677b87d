// fa_simt_f32.cuh -- fp32 attention forward and backward on the CUDA cores (FFMA).
//
// For callers that need fp32 accuracy (tensor-core tf32 keeps only 10 mantissa
// bits). Same operation as the bf16 path. The structure follows the pages' own
// CUDA sketches: key/value tiles staged in shared memory with 16-byte (float4)
// loads ("From GPU memory access to code: how FlashAttention makes large-model
// training 3x faster", section 3.1) and row max / row sum by warp-shuffle
// reductions (same page, section 3.2); the forward is the online-softmax loop of
// "FlashAttention optimisation: breaking the performance bottleneck of standard
// attention", section 4.1; the backward recomputes P from the stored log-sum-exp
// (same page, section 4.2) and is deterministic (no atomics):
//   fa_f32_bwd_dot_kernel : D_i = sum_k dO_ik O_ik
//   fa_f32_bwd_dkdv_kernel: per key row j, loop over query rows i
//   fa_f32_bwd_dq_kernel  : per query row i, loop over key rows j
#pragma once

#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "fa_ptx.cuh"  // pdl_wait, pdl_launch_dependents

namespace fa {
namespace f32 {

constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 4;
constexpr int kRowsPerBlock = kWarps * kRowsPerWarp;  // 16 owned rows per block
constexpr int kTile = 32;                             // streamed rows per tile

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Copies `rows` rows (row stride D floats in global) into shared memory with a
// padded stride of D + 4 floats, zero-filling rows beyond `valid`.
template <int D>
__device__ __forceinline__ void load_rows(float* dst, const float* src, int rows, int valid) {
  constexpr int V4 = D / 4;
  for (int idx = threadIdx.x; idx < rows * V4; idx += blockDim.x) {
    const int r = idx / V4, c4 = idx % V4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < valid) v = reinterpret_cast<const float4*>(src + static_cast<size_t>(r) * D)[c4];
    *reinterpret_cast<float4*>(dst + r * (D + 4) + c4 * 4) = v;
  }
}

// ------------------------------------------------------------------ forward

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    fa_f32_fwd_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                      const float* __restrict__ V, float* __restrict__ O, float* __restrict__ LSE,
                      int N, float scale, int causal) {
  pdl_wait();  // the grid before this one has completed
  pdl_launch_dependents();
  constexpr int P = D + 4;
  constexpr int CPL = D / 32;  // output columns per lane
  __shared__ __align__(16) float sQ[kRowsPerBlock * P];
  __shared__ __align__(16) float sK[kTile * P];
  __shared__ __align__(16) float sV[kTile * P];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // grid.x = (batch, head) x row blocks, head-major (grid.y is capped at 65535)
  const int rblocks = (N + kRowsPerBlock - 1) / kRowsPerBlock;
  const size_t bh = blockIdx.x / rblocks;
  const size_t head = bh * N * D;
  const int row0 = static_cast<int>(blockIdx.x % rblocks) * kRowsPerBlock;
  load_rows<D>(sQ, Q + head + static_cast<size_t>(row0) * D, kRowsPerBlock, N - row0);

  float m[kRowsPerWarp], l[kRowsPerWarp], acc[kRowsPerWarp][CPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    m[r] = -INFINITY;
    l[r] = 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[r][c] = 0.f;
  }
  const int last_row = min(row0 + kRowsPerBlock, N) - 1;
  const int kv_end = causal ? last_row + 1 : N;
  for (int j0 = 0; j0 < kv_end; j0 += kTile) {
    __syncthreads();
    load_rows<D>(sK, K + head + static_cast<size_t>(j0) * D, kTile, N - j0);
    load_rows<D>(sV, V + head + static_cast<size_t>(j0) * D, kTile, N - j0);
    __syncthreads();
    const int col = j0 + lane;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int rl = warp * kRowsPerWarp + r;
      const int row = row0 + rl;
      // score of key `col` for this row (lane = key)
      float s = 0.f;
      const float* q = sQ + rl * P;
      const float* k = sK + lane * P;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(q + c);
        const float4 kv = *reinterpret_cast<const float4*>(k + c);
        s = fmaf(qv.x, kv.x, s);
        s = fmaf(qv.y, kv.y, s);
        s = fmaf(qv.z, kv.z, s);
        s = fmaf(qv.w, kv.w, s);
      }
      s *= scale;
      if (col >= N || (causal && col > row)) s = -INFINITY;
      const float m_new = fmaxf(m[r], warp_max(s));
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float pj = expf(s - m_use);
      const float alpha = (m[r] == -INFINITY) ? 0.f : expf(m[r] - m_use);
      l[r] = l[r] * alpha + warp_sum(pj);
      m[r] = m_new;
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[r][c] *= alpha;
#pragma unroll 4
      for (int jj = 0; jj < kTile; ++jj) {
        const float pb = __shfl_sync(0xffffffffu, pj, jj);
        const float* v = sV + jj * P;
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[r][c] = fmaf(pb, v[lane + 32 * c], acc[r][c]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int row = row0 + warp * kRowsPerWarp + r;
    if (row >= N) continue;
    const float inv = l[r] > 0.f ? 1.f / l[r] : 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) O[head + static_cast<size_t>(row) * D + lane + 32 * c] = acc[r][c] * inv;
    if (lane == 0)
      LSE[bh * N + row] = l[r] > 0.f ? m[r] + logf(l[r]) : -INFINITY;
  }
}

// ------------------------------------------------------------------ backward

template <int D>
constexpr size_t dkdv_smem_bytes() {
  return sizeof(float) * (2 * kRowsPerBlock * (D + 4) + 2 * kTile * (D + 4) + 2 * kTile);
}
template <int D>
constexpr size_t dq_smem_bytes() {
  return sizeof(float) * (2 * kRowsPerBlock * (D + 4) + 2 * kTile * (D + 4));
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    fa_f32_bwd_dot_kernel(const float* __restrict__ O, const float* __restrict__ dO,
                          float* __restrict__ Dvec, long long rows) {
  pdl_wait();  // the grid before this one has completed
  pdl_launch_dependents();
  const long long r = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float s = 0.f;
#pragma unroll
  for (int c = lane; c < D; c += 32) s = fmaf(O[r * D + c], dO[r * D + c], s);
  s = warp_sum(s);
  if (lane == 0) Dvec[r] = s;
}

// Each warp owns kRowsPerWarp key rows j; query rows stream through shared memory.
template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    fa_f32_bwd_dkdv_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                           const float* __restrict__ V, const float* __restrict__ dO,
                           const float* __restrict__ LSE, const float* __restrict__ Dvec,
                           float* __restrict__ dK, float* __restrict__ dV, int N, float scale,
                           int causal) {
  pdl_wait();  // the grid before this one has completed
  pdl_launch_dependents();
  constexpr int P = D + 4;
  constexpr int CPL = D / 32;
  extern __shared__ __align__(16) float dsm[];  // dkdv_smem_bytes<D>() bytes
  float* sK = dsm;
  float* sV = sK + kRowsPerBlock * P;
  float* sQ = sV + kRowsPerBlock * P;
  float* sdO = sQ + kTile * P;
  float* sL = sdO + kTile * P;
  float* sD = sL + kTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rblocks = (N + kRowsPerBlock - 1) / kRowsPerBlock;  // grid.x = heads x blocks
  const size_t bh = blockIdx.x / rblocks;
  const size_t head = bh * N * D;
  const size_t hrow = bh * N;
  const int key0 = static_cast<int>(blockIdx.x % rblocks) * kRowsPerBlock;
  load_rows<D>(sK, K + head + static_cast<size_t>(key0) * D, kRowsPerBlock, N - key0);
  load_rows<D>(sV, V + head + static_cast<size_t>(key0) * D, kRowsPerBlock, N - key0);
  float gk[kRowsPerWarp][CPL], gv[kRowsPerWarp][CPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
    for (int c = 0; c < CPL; ++c) gk[r][c] = gv[r][c] = 0.f;
  const int i_start = causal ? (key0 / kTile) * kTile : 0;
  for (int i0 = i_start; i0 < N; i0 += kTile) {
    __syncthreads();
    load_rows<D>(sQ, Q + head + static_cast<size_t>(i0) * D, kTile, N - i0);
    load_rows<D>(sdO, dO + head + static_cast<size_t>(i0) * D, kTile, N - i0);
    if (threadIdx.x < kTile) {
      const int i = i0 + threadIdx.x;
      sL[threadIdx.x] = i < N ? LSE[hrow + i] : 0.f;
      sD[threadIdx.x] = i < N ? Dvec[hrow + i] : 0.f;
    }
    __syncthreads();
    const int i = i0 + lane;  // lane = query row
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int jl = warp * kRowsPerWarp + r;
      const int j = key0 + jl;
      float s = 0.f, dp = 0.f;
      const float* q = sQ + lane * P;
      const float* g = sdO + lane * P;
      const float* k = sK + jl * P;
      const float* v = sV + jl * P;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(q + c);
        const float4 kv = *reinterpret_cast<const float4*>(k + c);
        const float4 gv4 = *reinterpret_cast<const float4*>(g + c);
        const float4 vv = *reinterpret_cast<const float4*>(v + c);
        s = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, s))));
        dp = fmaf(gv4.x, vv.x, fmaf(gv4.y, vv.y, fmaf(gv4.z, vv.z, fmaf(gv4.w, vv.w, dp))));
      }
      const bool live = i < N && j < N && !(causal && j > i);
      const float pij = live ? expf(s * scale - sL[lane]) : 0.f;
      const float dsij = pij * (dp - sD[lane]);
#pragma unroll 4
      for (int ii = 0; ii < kTile; ++ii) {
        const float pb = __shfl_sync(0xffffffffu, pij, ii);
        const float db = __shfl_sync(0xffffffffu, dsij, ii);
        const float* qi = sQ + ii * P;
        const float* gi = sdO + ii * P;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          gv[r][c] = fmaf(pb, gi[lane + 32 * c], gv[r][c]);
          gk[r][c] = fmaf(db, qi[lane + 32 * c], gk[r][c]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int j = key0 + warp * kRowsPerWarp + r;
    if (j >= N) continue;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      dK[head + static_cast<size_t>(j) * D + lane + 32 * c] = gk[r][c] * scale;
      dV[head + static_cast<size_t>(j) * D + lane + 32 * c] = gv[r][c];
    }
  }
}

// Each warp owns kRowsPerWarp query rows i; key/value rows stream through shared memory.
template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    fa_f32_bwd_dq_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                         const float* __restrict__ V, const float* __restrict__ dO,
                         const float* __restrict__ LSE, const float* __restrict__ Dvec,
                         float* __restrict__ dQ, int N, float scale, int causal) {
  pdl_wait();  // the grid before this one has completed
  pdl_launch_dependents();
  constexpr int P = D + 4;
  constexpr int CPL = D / 32;
  extern __shared__ __align__(16) float dsm[];  // dq_smem_bytes<D>() bytes
  float* sQ = dsm;
  float* sdO = sQ + kRowsPerBlock * P;
  float* sK = sdO + kRowsPerBlock * P;
  float* sV = sK + kTile * P;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rblocks = (N + kRowsPerBlock - 1) / kRowsPerBlock;  // grid.x = heads x blocks
  const size_t bh = blockIdx.x / rblocks;
  const size_t head = bh * N * D;
  const size_t hrow = bh * N;
  const int row0 = static_cast<int>(blockIdx.x % rblocks) * kRowsPerBlock;
  load_rows<D>(sQ, Q + head + static_cast<size_t>(row0) * D, kRowsPerBlock, N - row0);
  load_rows<D>(sdO, dO + head + static_cast<size_t>(row0) * D, kRowsPerBlock, N - row0);
  float Lr[kRowsPerWarp], Dr[kRowsPerWarp], gq[kRowsPerWarp][CPL];
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int i = row0 + warp * kRowsPerWarp + r;
    Lr[r] = i < N ? LSE[hrow + i] : 0.f;
    Dr[r] = i < N ? Dvec[hrow + i] : 0.f;
#pragma unroll
    for (int c = 0; c < CPL; ++c) gq[r][c] = 0.f;
  }
  const int last_row = min(row0 + kRowsPerBlock, N) - 1;
  const int kv_end = causal ? last_row + 1 : N;
  for (int j0 = 0; j0 < kv_end; j0 += kTile) {
    __syncthreads();
    load_rows<D>(sK, K + head + static_cast<size_t>(j0) * D, kTile, N - j0);
    load_rows<D>(sV, V + head + static_cast<size_t>(j0) * D, kTile, N - j0);
    __syncthreads();
    const int j = j0 + lane;  // lane = key row
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const int il = warp * kRowsPerWarp + r;
      const int i = row0 + il;
      float s = 0.f, dp = 0.f;
      const float* q = sQ + il * P;
      const float* g = sdO + il * P;
      const float* k = sK + lane * P;
      const float* v = sV + lane * P;
#pragma unroll 8
      for (int c = 0; c < D; c += 4) {
        const float4 qv = *reinterpret_cast<const float4*>(q + c);
        const float4 kv = *reinterpret_cast<const float4*>(k + c);
        const float4 gv4 = *reinterpret_cast<const float4*>(g + c);
        const float4 vv = *reinterpret_cast<const float4*>(v + c);
        s = fmaf(qv.x, kv.x, fmaf(qv.y, kv.y, fmaf(qv.z, kv.z, fmaf(qv.w, kv.w, s))));
        dp = fmaf(gv4.x, vv.x, fmaf(gv4.y, vv.y, fmaf(gv4.z, vv.z, fmaf(gv4.w, vv.w, dp))));
      }
      const bool live = i < N && j < N && !(causal && j > i);
      const float pij = live ? expf(s * scale - Lr[r]) : 0.f;
      const float dsij = pij * (dp - Dr[r]);
#pragma unroll 4
      for (int jj = 0; jj < kTile; ++jj) {
        const float db = __shfl_sync(0xffffffffu, dsij, jj);
        const float* kj = sK + jj * P;
#pragma unroll
        for (int c = 0; c < CPL; ++c) gq[r][c] = fmaf(db, kj[lane + 32 * c], gq[r][c]);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsPerWarp; ++r) {
    const int i = row0 + warp * kRowsPerWarp + r;
    if (i >= N) continue;
#pragma unroll
    for (int c = 0; c < CPL; ++c) dQ[head + static_cast<size_t>(i) * D + lane + 32 * c] = gq[r][c] * scale;
  }
}

}  // namespace f32
}  // namespace fa
