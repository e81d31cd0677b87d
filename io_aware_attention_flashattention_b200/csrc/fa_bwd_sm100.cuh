// fa_bwd_sm100.cuh -- attention backward for sm_100a (bf16 in/out, fp32 accumulate).
//
// Method: recomputation ("FlashAttention optimisation: breaking the performance
// bottleneck of standard attention", section 4.2; "From GPU memory access to code:
// how FlashAttention makes large-model training 3x faster", section 2.2): P is
// rebuilt tile by tile from the stored log-sum-exp instead of being kept, and the
// gradients use the same blocking as the forward. For the loss <dO, O>:
//   D = rowsum(dO o O), P = exp(scale*QK^T - LSE), dP = dO V^T, dS = P o (dP - D),
//   dV = P^T dO, dK = scale * dS^T Q, dQ = scale * dS K.
//
// Three launches:
//   1. fa_bwd_pre_kernel: D_i and L2_i = LSE_i*log2(e) into [B*H, Npad] (padding
//      rows get D = 0, L2 = +inf so that they contribute nothing), and zero the
//      fp32 dQ accumulator.
//   2. fa_bwd_kernel (one CTA per SM, 320 threads): the CTA owns one tile of 128
//      keys K_j, V_j and streams the query tiles Q_i, dO_i (128 rows) through a
//      ring of shared-memory slots with TMA.
//        warp 9 (MMA, one thread): S^T = K_j Q_i^T and dP^T = V_j dO_i^T into TMEM;
//          dV += P^T dO_i and dK += dS^T Q_i with P^T and dS^T read from TMEM;
//          dQ_i = dS K_j with dS read from shared memory.
//        warps 0-3 (one thread per key row): P^T = 2^(S^T c - L2), masked;
//          dS^T = P^T (dP^T - D); both rounded to bf16 and stored back into TMEM
//          over S^T and dP^T, and dS also into shared memory for the dQ MMA.
//          At the end they write dK (times scale) and dV once.
//        warps 4-7 (one thread per query row): read dQ_i from TMEM and add it into
//          the fp32 accumulator with vector reductions (red.global.add.v4.f32).
//        warp 8: TMA producer.
//      TMEM (512 columns): dK [0,D), dV [D,2D), S^T [2D,2D+128), dP^T [2D+128,2D+256);
//      P^T and dS^T (bf16 pairs) alias the first 64 columns of S^T and dP^T. dQ_i
//      uses S^T's columns when D = 128 and its own columns [384,448) when D = 64.
//   3. fa_bwd_dq_kernel: dQ = bf16(scale * accumulator).
// No N x N matrix is written to device memory.
#pragma once

#include "fa_ptx.cuh"

namespace fa {
namespace bwd {

constexpr int BM = 128;        // query rows per step
constexpr int BN = 128;        // key rows per CTA
constexpr int kThreads = 320;
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;

template <int D>
struct Cfg {
  static constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // 128 x D bf16
  static constexpr int kSlots = (D == 128) ? 3 : 6;         // Q/dO ring
  static constexpr int kVecBytes = BM * 4;                   // 128 fp32 (L2 or D)
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kDSOff = kRingOff + kSlots * kTileBytes;  // dS, 128 x 128 bf16
  static constexpr int kDSBytes = 2 * kChunkBytes;
  static constexpr int kVecOff = kDSOff + kDSBytes;  // per slot: L2[128], D[128]
  static constexpr int kBarOff = kVecOff + kSlots * 2 * kVecBytes;
  static constexpr int kBarKV = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = 1 + kSlots;
  static constexpr int kBarS = 1 + 2 * kSlots;
  static constexpr int kBarP = kBarS + 1;
  static constexpr int kBarDQFull = kBarP + 1;
  static constexpr int kBarDQEmpty = kBarDQFull + 1;
  static constexpr int kBarDKDV = kBarDQEmpty + 1;
  static constexpr int kBarDrain = kBarDKDV + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
  static constexpr uint32_t kTmDK = 0, kTmDV = D, kTmS = 2 * D, kTmDP = 2 * D + 128;
  static constexpr uint32_t kTmDQ = (D == 128) ? kTmS : 384;
  static constexpr uint32_t kTmCols = 512;
};

struct Params {
  __nv_bfloat16* dK;
  __nv_bfloat16* dV;
  const float* L2;  // [BH, Npad], LSE * log2(e), +inf in padding
  const float* Dv;  // [BH, Npad]
  float* dQacc;     // [BH, N, D]
  int N;
  int Npad;
  int BH;
  float scale;
  float scale_log2;
  int causal;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_status, kStatusTimeout);
      return;
    }
  }
}

// S^T (or dP^T) = X_j Y_i^T: M = 128 rows of X, N = 128 rows of Y, K = D; both
// operands K-major in 128-byte-swizzled tiles.
template <int D>
__device__ __forceinline__ void issue_xyT(uint32_t tm_d, uint32_t x_smem, uint32_t y_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * Cfg<D>::kChunkBytes + (kk % 4) * 32;
    mma_ss(tm_d, sdesc_sw128(x_smem + off, 16, 1024), sdesc_sw128(y_smem + off, 16, 1024), idesc,
           kk > 0 ? 1u : 0u);
  }
}

// acc[128 x D] (+)= A_tmem[128 x 128] * Y[128 x D], Y a row-major tile in shared
// memory used as the MN-major B operand.
template <int D>
__device__ __forceinline__ void issue_ts_acc(uint32_t tm_acc, uint32_t tm_a, uint32_t y_smem,
                                             bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk)
    mma_ts(tm_acc, tm_a + kk * 8, sdesc_sw128(y_smem + kk * 2048, Cfg<D>::kChunkBytes, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
}

// dQ_i[128 queries x D] = dS[queries x keys] * K_j[keys x D]: A is the dS tile
// (stored key-row-major, i.e. MN-major for A), B is K_j (MN-major).
template <int D>
__device__ __forceinline__ void issue_dq(uint32_t tm_dq, uint32_t ds_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, D, 1, 1);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk)
    mma_ss(tm_dq, sdesc_sw128(ds_smem + kk * 2048, Cfg<D>::kChunkBytes, 1024),
           sdesc_sw128(k_smem + kk * 2048, Cfg<D>::kChunkBytes, 1024), idesc, kk > 0 ? 1u : 0u);
}

// ------------------------------------------------------------------ preprocess

template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_pre_kernel(const __nv_bfloat16* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                      const float* __restrict__ LSE, float* __restrict__ L2,
                      float* __restrict__ Dv, float* __restrict__ dQacc, int N, int Npad,
                      long long total_rows) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= total_rows) return;  // total_rows = BH * Npad
  const long long bh = r / Npad;
  const int i = static_cast<int>(r % Npad);
  if (i >= N) {
    if (lane == 0) {
      L2[r] = INFINITY;
      Dv[r] = 0.f;
    }
    return;
  }
  const long long row = bh * N + i;
  constexpr int PER = D / 32;  // bf16 per lane: 2 or 4
  float s = 0.f;
  if (PER == 4) {
    const uint2 a = reinterpret_cast<const uint2*>(O + row * D)[lane];
    const uint2 b = reinterpret_cast<const uint2*>(dO + row * D)[lane];
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float2 x = __bfloat1622float2(a2[k]), y = __bfloat1622float2(b2[k]);
      s = fmaf(x.x, y.x, fmaf(x.y, y.y, s));
    }
  } else {
    const __nv_bfloat162 a = reinterpret_cast<const __nv_bfloat162*>(O + row * D)[lane];
    const __nv_bfloat162 b = reinterpret_cast<const __nv_bfloat162*>(dO + row * D)[lane];
    const float2 x = __bfloat1622float2(a), y = __bfloat1622float2(b);
    s = fmaf(x.x, y.x, x.y * y.y);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    Dv[r] = s;
    L2[r] = LSE[row] * 1.4426950408889634f;
  }
  float4* z = reinterpret_cast<float4*>(dQacc + row * D);
#pragma unroll
  for (int k = lane; k < D / 4; k += 32) z[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------ dQ convert

template <int D>
__global__ void __launch_bounds__(256)
    fa_bwd_dq_kernel(const float* __restrict__ dQacc, __nv_bfloat16* __restrict__ dQ,
                     long long n4, float scale) {
  for (long long k = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; k < n4;
       k += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(dQacc)[k];
    uint2 out;
    out.x = pack_bf16x2(v.x * scale, v.y * scale);
    out.y = pack_bf16x2(v.z * scale, v.w * scale);
    reinterpret_cast<uint2*>(dQ)[k] = out;
  }
}

// ------------------------------------------------------------------ main kernel

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const Params p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int j = static_cast<int>(blockIdx.x) / p.BH;  // key tile (heaviest first if causal)
  const int bh = static_cast<int>(blockIdx.x) % p.BH;
  const int k0 = j * BN;
  const int n_q = (p.N + BM - 1) / BM;
  const int i_begin = p.causal ? j : 0;  // BM == BN: query tiles i >= j see key tile j
  const int nsteps = n_q - i_begin;

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarKV), 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar(C::kBarFull + s), 1);
      mbar_init(bar(C::kBarEmpty + s), 1);
    }
    mbar_init(bar(C::kBarS), 1);
    mbar_init(bar(C::kBarP), 4);
    mbar_init(bar(C::kBarDQFull), 1);
    mbar_init(bar(C::kBarDQEmpty), 4);
    mbar_init(bar(C::kBarDKDV), 1);
    mbar_init(bar(C::kBarDrain), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Watchdog wd{abort_flag, p.timeout_ns};

  // ring sequence: seq = 2*step + w, w = 0 for Q_i (with L2_i, D_i), 1 for dO_i
  auto slot_of = [&](int seq) { return seq % C::kSlots; };
  auto round_of = [&](int seq) { return seq / C::kSlots; };
  auto slot_smem = [&](int seq) -> uint32_t {
    return base + C::kRingOff + slot_of(seq) * C::kTileBytes;
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      mbar_arrive_expect_tx(bar(C::kBarKV), 2 * C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_3d(base + C::kKOff + c * C::kChunkBytes, &tmK, bar(C::kBarKV), c * 64, k0, bh);
        tma_load_3d(base + C::kVOff + c * C::kChunkBytes, &tmV, bar(C::kBarKV), c * 64, k0, bh);
      }
      int issued = 0;
      bool ok = true;
      for (int s = 0; s < nsteps && ok; ++s) {
        const int i = i_begin + s;
        for (int w = 0; w < 2; ++w) {
          const int seq = 2 * s + w;
          const int slot = slot_of(seq);
          const int rnd = round_of(seq);
          if (rnd > 0 && !mbar_wait(bar(C::kBarEmpty + slot), (rnd - 1) & 1, wd)) {
            ok = false;
            break;
          }
          const uint32_t full = bar(C::kBarFull + slot);
          const uint32_t dst = slot_smem(seq);
          if (w == 0) {
            mbar_arrive_expect_tx(full, C::kTileBytes + 2 * C::kVecBytes);
            const uint32_t vec = base + C::kVecOff + slot * 2 * C::kVecBytes;
            const size_t off = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(i) * BM;
            bulk_load(vec, p.L2 + off, C::kVecBytes, full);
            bulk_load(vec + C::kVecBytes, p.Dv + off, C::kVecBytes, full);
          } else {
            mbar_arrive_expect_tx(full, C::kTileBytes);
          }
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(dst + c * C::kChunkBytes, w ? &tmdO : &tmQ, full, c * 64, i * BM, bh);
          issued = seq + 1;
        }
      }
      for (int seq = max(0, issued - C::kSlots); seq < issued; ++seq)
        drain_wait(bar(C::kBarFull + slot_of(seq)), round_of(seq) & 1, p.timeout_ns);
      drain_wait(bar(C::kBarKV), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t k_smem = base + C::kKOff, v_smem = base + C::kVOff;
      const uint32_t ds_smem = base + C::kDSOff;
      const uint32_t tm_s = tmem + C::kTmS, tm_dp = tmem + C::kTmDP;
      bool ok = mbar_wait(bar(C::kBarKV), 0, wd);
      auto wait_full = [&](int seq) -> bool {
        return mbar_wait(bar(C::kBarFull + slot_of(seq)), round_of(seq) & 1, wd);
      };
      if (ok && nsteps > 0) {
        ok = wait_full(0) && wait_full(1);
        if (ok) {
          tc_fence_after();
          issue_xyT<D>(tm_s, k_smem, slot_smem(0));   // S^T = K Q^T
          issue_xyT<D>(tm_dp, v_smem, slot_smem(1));  // dP^T = V dO^T
          tc_commit(bar(C::kBarS));
        }
      }
      for (int s = 0; s < nsteps && ok; ++s) {
        const int seqQ = 2 * s, seqO = 2 * s + 1;
        if (!mbar_wait(bar(C::kBarP), s & 1, wd)) { ok = false; break; }
        tc_fence_after();
        issue_ts_acc<D>(tmem + C::kTmDV, tm_s, slot_smem(seqO), s > 0);   // dV += P^T dO
        issue_ts_acc<D>(tmem + C::kTmDK, tm_dp, slot_smem(seqQ), s > 0);  // dK += dS^T Q
        if (D == 64 && s > 0) {  // dQ region reused: the previous dQ must have been read
          if (!mbar_wait(bar(C::kBarDQEmpty), (s - 1) & 1, wd)) { ok = false; break; }
          tc_fence_after();
        }
        issue_dq<D>(tmem + C::kTmDQ, ds_smem, k_smem);
        tc_commit(bar(C::kBarDQFull));
        tc_commit(bar(C::kBarEmpty + slot_of(seqQ)));
        tc_commit(bar(C::kBarEmpty + slot_of(seqO)));
        if (s + 1 < nsteps) {
          if (!(wait_full(seqQ + 2) && wait_full(seqO + 2))) { ok = false; break; }
          tc_fence_after();
          issue_xyT<D>(tm_dp, v_smem, slot_smem(seqO + 2));  // dP^T for the next step
          if (D == 128) {  // S^T shares columns with dQ: wait until dQ has been read
            if (!mbar_wait(bar(C::kBarDQEmpty), s & 1, wd)) { ok = false; break; }
            tc_fence_after();
          }
          issue_xyT<D>(tm_s, k_smem, slot_smem(seqQ + 2));
          tc_commit(bar(C::kBarS));
        }
      }
      if (ok) tc_commit(bar(C::kBarDKDV));
      tc_commit(bar(C::kBarDrain));
      drain_wait(bar(C::kBarDrain), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ------------------------------------------------------------ P^T, dS^T (key rows)
    const int krow = warp * 32 + lane;  // key row within the tile = TMEM lane
    const int key = k0 + krow;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tm_s = tmem + lane_off + C::kTmS;
    const uint32_t tm_dp = tmem + lane_off + C::kTmDP;
    const float c = p.scale_log2;
    uint8_t* ds_row = base_ptr + C::kDSOff + krow * 128;
    bool ok = true;
    for (int s = 0; s < nsteps && ok; ++s) {
      const int i = i_begin + s;
      const int q0 = i * BM;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarS), s & 1, wd));
      if (ok && s > 0)  // the previous dQ MMA has finished reading the dS tile
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDQFull), (s - 1) & 1, wd));
      // L2_i and D_i arrived with Q_i: observe that copy's barrier directly
      if (ok)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar(C::kBarFull + slot_of(2 * s)), round_of(2 * s) & 1, wd));
      if (!ok) break;
      tc_fence_after();
      const int slot = slot_of(2 * s);
      const float* Lv = reinterpret_cast<const float*>(base_ptr + C::kVecOff + slot * 2 * C::kVecBytes);
      const float* Dvv = Lv + BM;
      // query columns q0 + [lim, 128) are visible to this key: causal needs q >= key
      const int lim = p.causal ? max(0, key - q0) : 0;
      const bool key_valid = key < p.N;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sv[32], dv[32];
        tmem_ld32(tm_s + cc * 32, sv);
        tmem_ld32(tm_dp + cc * 32, dv);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int qa = cc * 32 + 2 * k, qb = qa + 1;
          float pa = ex2_approx(fmaf(__uint_as_float(sv[2 * k]), c, -Lv[qa]));
          float pb = ex2_approx(fmaf(__uint_as_float(sv[2 * k + 1]), c, -Lv[qb]));
          if (!key_valid || qa < lim) pa = 0.f;
          if (!key_valid || qb < lim) pb = 0.f;
          const float da = pa * (__uint_as_float(dv[2 * k]) - Dvv[qa]);
          const float db = pb * (__uint_as_float(dv[2 * k + 1]) - Dvv[qb]);
          pk[k] = pack_bf16x2(pa, pb);
          dk[k] = pack_bf16x2(da, db);
        }
        tmem_st16(tm_s + cc * 16, pk);
        tmem_st16(tm_dp + cc * 16, dk);
        // dS tile in shared memory: chunk of 64 queries = cc/2, 16-byte units
        // (cc%2)*4 .. +3 of this key's 128-byte row, 128-byte swizzle.
        uint8_t* chunk = ds_row + (cc >> 1) * C::kChunkBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = ((cc & 1) * 4 + u) ^ (krow & 7);
          *reinterpret_cast<uint4*>(chunk + unit * 16) =
              make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
        }
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarP));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDKDV), 0, wd));
    if (ok && nsteps > 0) {
      tc_fence_after();
      const uint32_t tm_dk = tmem + lane_off + C::kTmDK;
      const uint32_t tm_dv = tmem + lane_off + C::kTmDV;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        __nv_bfloat16* out = (which == 0 ? p.dK : p.dV) + (static_cast<size_t>(bh) * p.N + key) * D;
        const float mul = (which == 0) ? p.scale : 1.0f;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t v[32];
          tmem_ld32((which == 0 ? tm_dk : tm_dv) + cc * 32, v);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            pk[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * mul, __uint_as_float(v[2 * k + 1]) * mul);
          if (key < p.N) {
            uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
      }
    } else if (ok && nsteps == 0) {
      // no query tile sees this key tile (cannot happen for square causal attention)
    }
  } else {
    // ------------------------------------------------------------ dQ readout (query rows)
    const int wq = warp - 4;
    const int qrow = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tm_dq = tmem + lane_off + C::kTmDQ;
    bool ok = true;
    for (int s = 0; s < nsteps && ok; ++s) {
      const int q = (i_begin + s) * BM + qrow;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDQFull), s & 1, wd));
      if (!ok) break;
      tc_fence_after();
      uint32_t v[D / 32][32];
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) tmem_ld32(tm_dq + cc * 32, v[cc]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarDQEmpty));
      if (q < p.N) {
        float* dst = p.dQacc + (static_cast<size_t>(bh) * p.N + q) * D;
#pragma unroll
        for (int k = 0; k < D / 4; ++k)
          red_add_v4(dst + 4 * k, __uint_as_float(v[k / 8][(4 * k) % 32]),
                     __uint_as_float(v[k / 8][(4 * k + 1) % 32]),
                     __uint_as_float(v[k / 8][(4 * k + 2) % 32]),
                     __uint_as_float(v[k / 8][(4 * k + 3) % 32]));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

}  // namespace bwd
}  // namespace fa
