// fa_bwd_sm100.cuh -- attention backward for sm_100a (bf16 or f16 in/out, fp32
// accumulate; the element type is the template parameter E).
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
//      rows, and rows that see no key (LSE = -inf), get L2 = +inf so that they
//      contribute nothing), and zero the fp32 dQ accumulator.
//   2. fa_bwd_kernel (one CTA per SM, 512 threads): the CTA owns one tile of 128
//      keys K_j, V_j (or, for a split tile, half of its query tiles) and streams the
//      query tiles Q_i, dO_i (128 rows) through a ring of shared-memory slots with
//      TMA. Each query tile is processed as two halves of 64 queries (h = 0, 1) so
//      that the MMAs of one half overlap the elementwise work of the other.
//      fa_bwd_persistent_kernel, at the end of this file, runs the same roles over a
//      list of key tiles per CTA.
//        warp 13 (MMA, one thread), per half h: S^T_h = K_j Q_ih^T and
//          dP^T_h = V_j dO_ih^T into TMEM; dV += P^T_h dO_ih and dK += dS^T_h Q_ih
//          with P^T_h and dS^T_h read from TMEM; for D = 128, dQ^T_h = K_j^T dS^T_h
//          (M = 128 head-dimension rows, N = 64 queries) into the columns S^T_h
//          used; for D = 64, after both halves, dQ_i = dS K_j into its own columns.
//        warps 4h..4h+3 (one thread per key row, queries of half h): P^T = 2^(S^T c
//          - L2), masked on diagonal and ragged tiles only; dS^T = P^T (dP^T - D);
//          both rounded to bf16 and stored back into TMEM over S^T_h and dP^T_h, and
//          dS also into a 128-byte-swizzled shared tile for the dQ MMA. At the end
//          warps 0-3 write dK (times scale) and warps 4-7 write dV, once.
//        warps 8-11: read dQ from TMEM and add it into the fp32 accumulator. For
//          D = 128 a thread owns one head-dimension element, so a warp's 32 adds
//          for one query hit 128 contiguous bytes; for D = 64 a thread owns a query
//          row and uses 16-byte vector adds.
//        warp 12: TMA producer.
//      TMEM (512 columns): dK [0,D), dV [D,2D), S^T [2D,2D+128), dP^T [2D+128,2D+256),
//      half h at +64h; P^T_h and dS^T_h (bf16 pairs) alias the first 32 columns of
//      their half.
//   3. fa_bwd_dq_kernel: dQ = bf16(scale * accumulator).
// Masks (the forward's: sliding window wl/wr with causal as wr = 0, and a 128 x 128
// block mask): a key tile's CTA walks only the query tiles that can see one of its
// keys, and elements are masked only on steps that cross a window edge. A key tile
// that no query sees gets dK = dV = 0.
// No N x N matrix is written to device memory.
#pragma once

#include <type_traits>

#include "fa_ptx.cuh"

namespace fa {
namespace bwd {

constexpr int BM = 128;        // query rows per step
constexpr int BN = 128;        // key rows per CTA
constexpr int kThreads = 512;
constexpr int kWarpDq = 8;     // first of the 4 dQ warps
constexpr int kWarpTma = 12;
constexpr int kWarpMma = 13;
constexpr int kMaxMaskTiles = 4096;  // largest block mask: 4096 x 4096 tiles (N <= 524288)

template <int D>
struct Cfg {
  static constexpr int kChunkBytes = 128 * 128;  // 128 rows x 64 bf16 (K, V, dS)
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kChunks * kChunkBytes;  // 128 x D bf16
  // Q and dO stream in half tiles (64 rows x D): 64-row chunks of 8 KB
  static constexpr int kHalfChunkBytes = 64 * 128;
  static constexpr int kHalfBytes = kChunks * kHalfChunkBytes;
  static constexpr int kSlots = (D == 128) ? 7 : 12;  // half-tile ring (7 x 16.5 KB fit at D = 128)
  static constexpr int kVecBytes = 64 * 4;             // 64 fp32 (L2 or D of a half)
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kRingOff = 2 * kTileBytes;
  static constexpr int kDSOff = kRingOff + kSlots * kHalfBytes;  // dS: 2 chunks of 64 queries
  static constexpr int kDSBytes = 2 * kChunkBytes;
  static constexpr int kVecOff = kDSOff + kDSBytes;  // per slot: L2[64], D[64]
  static constexpr int kBarOff = kVecOff + kSlots * 2 * kVecBytes;
  static constexpr int kBarKV = 0;
  static constexpr int kBarFull = 1;
  static constexpr int kBarEmpty = 1 + kSlots;
  static constexpr int kBarS = 1 + 2 * kSlots;  // [2]
  static constexpr int kBarP = kBarS + 2;       // [2]
  static constexpr int kBarDQFull = kBarP + 2;  // [2]
  static constexpr int kBarDQEmpty = kBarDQFull + 2;  // [2]
  static constexpr int kBarDKDV = kBarDQEmpty + 2;
  static constexpr int kBarSplitWritten = kBarDKDV + 1;        // split tile: 8 warps' rows written
  static constexpr int kBarSplitDecided = kBarSplitWritten + 1;  // ... and the arrival counted
  static constexpr int kBarKVEmpty = kBarSplitDecided + 1;  // persistent: item's K/V read
  static constexpr int kBarDKDVFree = kBarKVEmpty + 1;      // persistent: dK/dV read out
  static constexpr int kBarDrain = kBarDKDVFree + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kMaskOff = kMiscOff + 16;  // block-mask column of this key tile, as bits
  static constexpr int kSmemBytes = kMaskOff + kMaxMaskTiles / 8 + 1024;
  static constexpr uint32_t kTmDK = 0, kTmDV = D, kTmS = 2 * D, kTmDP = 2 * D + 128;
  static constexpr uint32_t kTmDQ64 = 384;  // D = 64 only
  static_assert(kSmemBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static constexpr uint32_t kTmCols = 512;
};

struct Params {
  uint16_t* dK;  // 16-bit elements (the kernel's element type)
  uint16_t* dV;
  const float* L2;  // [BH, Npad], LSE * log2(e), +inf in padding
  const float* Dv;  // [BH, Npad]
  float* dQacc;     // [BH, N, D]
  int N;
  int Npad;
  int BH;
  float scale;
  float scale_log2;
  int wl;                 // keys j >= i - wl are kept; < 0: no left bound
  int wr;                 // keys j <= i + wr are kept; < 0: no right bound (causal: 0)
  const uint8_t* blocks;  // [n_kt x n_kt] block mask (nonzero = kept), or null
  DropoutParams drop;     // used by the kDropout instances only
  unsigned long long timeout_ns;
  // Split key tiles (no block mask): the last n_split tiles (head-major) have their
  // query steps cut in two segments, [0, a) and [a, steps) with a = steps * split_num /
  // 16 rounded and kept within [1, steps - 1], each run by a CTA of its own. The grid
  // is the whole tiles first, then the larger segments, then the smaller ones. A
  // segment's CTA writes its fp32 dK, dV partial to its slot, counts itself in, and
  // the second to arrive adds the two slots (segment 0 first) and writes dK, dV.
  int n_split;
  int split_num;
  float* part;         // [n_split][2 segments][dK, dV][128 key rows][D] fp32
  unsigned* arrivals;  // [n_split] (zeroed by the preprocess)
  // Grid order of the key tiles: head-major (0: the CTAs resident at one time share one
  // or two heads' Q, dO and dQ accumulator in L2) or rank-major (1: every head's key tile
  // 0, then every head's key tile 1, ...; for causal or windowed launches without splits
  // whose Q, dO and dQ accumulator all fit in L2, so that the heaviest tiles start first).
  int rank_major;
};

// The first segment's step count for a tile of `steps` steps.
__host__ __device__ __forceinline__ int split_point(int steps, int split_num) {
  int a = (steps * split_num + 8) / 16;
  if (a < 1) a = 1;
  if (a > steps - 1) a = steps - 1;
  return a;
}

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

__device__ __forceinline__ void red_add(float* addr, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(a) : "memory");
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

// X_j Y_h^T: M = 128 rows of X, N = 64 rows of the half tile Y_h, K = D; both
// operands K-major (rows of 64 bf16 per 128-byte-swizzled chunk).
template <int D, Elt E>
__device__ __forceinline__ void issue_xyT_half(uint32_t tm_d, uint32_t x_smem, uint32_t yh_smem) {
  constexpr uint32_t idesc = idesc_f32acc<E>(128, 64, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t xo = (kk / 4) * Cfg<D>::kChunkBytes + (kk % 4) * 32;
    const uint32_t yo = (kk / 4) * Cfg<D>::kHalfChunkBytes + (kk % 4) * 32;
    mma_ss_e(tm_d, sdesc_sw128(x_smem + xo, 16, 1024), sdesc_sw128(yh_smem + yo, 16, 1024),
             idesc, kk > 0 ? 1u : 0u);
  }
}

// acc[128 keys x D] (+)= A_tmem[128 keys x 64 queries] * Y_h[64 queries x D] (the half
// tile, row-major in shared memory, used as the MN-major B operand).
template <int D, Elt E>
__device__ __forceinline__ void issue_acc_half(uint32_t tm_acc, uint32_t tm_a, uint32_t yh_smem,
                                               bool accumulate) {
  constexpr uint32_t idesc = idesc_f32acc<E>(128, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < 64 / 16; ++kk)
    mma_ts_e(tm_acc, tm_a + kk * 8,
             sdesc_sw128(yh_smem + kk * 2048, Cfg<D>::kHalfChunkBytes, 1024), idesc,
             (accumulate || kk > 0) ? 1u : 0u);
}

// D = 128: dQ^T_h[128 dims x 64 queries] = K_j^T[dims x keys] * dS_h^T[keys x queries]:
// A = K_j read MN-major (dims contiguous), B = dS chunk h read MN-major (queries
// contiguous in each key row).
template <Elt E>
__device__ __forceinline__ void issue_dqT_half(uint32_t tm_d, uint32_t k_smem, uint32_t ds_chunk) {
  constexpr uint32_t idesc = idesc_f32acc<E>(128, 64, 1, 1);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk)
    mma_ss_e(tm_d, sdesc_sw128(k_smem + kk * 2048, Cfg<128>::kChunkBytes, 1024),
             sdesc_sw128(ds_chunk + kk * 2048, Cfg<128>::kChunkBytes, 1024), idesc,
             kk > 0 ? 1u : 0u);
}

// D = 64: dQ_i[128 queries x 64] = dS[queries x keys] * K_j[keys x 64]: A = the whole
// dS tile (MN-major, two 64-query chunks), B = K_j (MN-major).
template <Elt E>
__device__ __forceinline__ void issue_dq64(uint32_t tm_d, uint32_t ds_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_f32acc<E>(128, 64, 1, 1);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk)
    mma_ss_e(tm_d, sdesc_sw128(ds_smem + kk * 2048, Cfg<64>::kChunkBytes, 1024),
             sdesc_sw128(k_smem + kk * 2048, Cfg<64>::kChunkBytes, 1024), idesc, kk > 0 ? 1u : 0u);
}

// ------------------------------------------------------------------ preprocess

template <int D, Elt E>
__global__ void __launch_bounds__(256)
    fa_bwd_pre_kernel(const uint16_t* __restrict__ O, const uint16_t* __restrict__ dO,
                      const float* __restrict__ LSE, float* __restrict__ L2,
                      float* __restrict__ Dv, float* __restrict__ dQacc, int N, int Npad,
                      long long total_rows, unsigned* __restrict__ arrivals, int n_arrivals) {
  pdl_wait();  // the grid before this one (the forward) has completed
  pdl_launch_dependents();
  if (blockIdx.x == 0)  // the main kernel's arrival counters of split tiles
    for (int k = threadIdx.x; k < n_arrivals; k += blockDim.x) arrivals[k] = 0u;
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
  constexpr int WORDS = D / 64;  // 32-bit words (element pairs) per lane: 1 or 2
  float s = 0.f;
  if (WORDS == 2) {
    const uint2 a = reinterpret_cast<const uint2*>(O + row * D)[lane];
    const uint2 b = reinterpret_cast<const uint2*>(dO + row * D)[lane];
    const float2 x0 = unpack2<E>(a.x), y0 = unpack2<E>(b.x);
    const float2 x1 = unpack2<E>(a.y), y1 = unpack2<E>(b.y);
    s = fmaf(x0.x, y0.x, fmaf(x0.y, y0.y, fmaf(x1.x, y1.x, x1.y * y1.y)));
  } else {
    const uint32_t a = reinterpret_cast<const uint32_t*>(O + row * D)[lane];
    const uint32_t b = reinterpret_cast<const uint32_t*>(dO + row * D)[lane];
    const float2 x = unpack2<E>(a), y = unpack2<E>(b);
    s = fmaf(x.x, y.x, x.y * y.y);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) {
    Dv[r] = s;
    const float lse = LSE[row];
    L2[r] = (lse == -INFINITY) ? INFINITY : lse * 1.4426950408889634f;
  }
  float4* z = reinterpret_cast<float4*>(dQacc + row * D);
#pragma unroll
  for (int k = lane; k < D / 4; k += 32) z[k] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// ------------------------------------------------------------------ dQ convert

template <int D, Elt E>
__global__ void __launch_bounds__(256)
    fa_bwd_dq_kernel(const float* __restrict__ dQacc, uint16_t* __restrict__ dQ, long long n4,
                     float scale) {
  pdl_wait();  // the grid before this one (the main kernel) has completed
  pdl_launch_dependents();
  for (long long k = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; k < n4;
       k += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 v = reinterpret_cast<const float4*>(dQacc)[k];
    uint2 out;
    out.x = pack2<E>(v.x * scale, v.y * scale);
    out.y = pack2<E>(v.z * scale, v.w * scale);
    reinterpret_cast<uint2*>(dQ)[k] = out;
  }
}

// P^T and dS^T of one half step for one key row (this thread, TMEM lane krow): from
// S^T and dP^T in TMEM, P = 2^(S c - L2) and dS = P o (dP - D) (with dropout: P o Z s
// for dV and P o (dP o Z s - D) for dS), both back to TMEM as 16-bit pairs over the
// columns they came from, and dS also into the swizzled shared chunk (the dQ operand).
// kM: test each query against the key's visible range [q_lo, q_hi): query qh0 + x is
// visible iff qoff + x < q_span (unsigned). ctr_head: the dropout counter's head word
// (the call's head_base + the flattened head).
template <Elt E, bool kDropout, bool kM>
__device__ __forceinline__ void p_ds_half(uint32_t tm_s, uint32_t tm_dp, const float4* Lv,
                                          const float4* Dv4, float c, int key, int qh0,
                                          uint32_t ctr_head,
                                          const DropoutParams& drop, int lane, int qoff,
                                          unsigned q_span, uint8_t* ds_row, int krow) {
  uint32_t sv[2][16], dv[2][16];
  tmem_ld16(tm_s, sv[0]);
  tmem_ld16(tm_dp, dv[0]);
  tmem_wait_ld();
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    const int cur = cc & 1;
    if (cc + 1 < 4) {  // the next chunk's loads overlap this chunk's arithmetic
      tmem_ld16(tm_s + 16 * (cc + 1), sv[cur ^ 1]);
      tmem_ld16(tm_dp + 16 * (cc + 1), dv[cur ^ 1]);
    }
    // Dropout bytes of this key for the chunk's 16 queries: byte e of zq[v] is
    // query 16cc + 4v + e of the half. One block covers 4 queries x 4 keys, and
    // the lanes of keys 4g..4g+3 share its counter: lane u draws the block of the
    // query group (qh0 + 16cc) / 4 + u, regroups its bytes by key (zq[b] = byte b
    // of words 0..3) and a 4 x 4 transpose across the four lanes hands each lane
    // its own key's bytes of all four blocks.
    [[maybe_unused]] uint32_t zq[4] = {0u, 0u, 0u, 0u};
    if constexpr (kDropout) {
      const int u = lane & 3;
      const uint4 w = philox4x32_10(
          make_uint4(static_cast<uint32_t>(key >> 2),
                     static_cast<uint32_t>(((qh0 + cc * 16) >> 2) + u),
                     ctr_head, drop.offset),
          drop.seed_lo, drop.seed_hi);
      const uint32_t t0 = __byte_perm(w.x, w.y, 0x5140), t1 = __byte_perm(w.x, w.y, 0x7362);
      const uint32_t t2 = __byte_perm(w.z, w.w, 0x5140), t3 = __byte_perm(w.z, w.w, 0x7362);
      zq[0] = __byte_perm(t0, t2, 0x5410);
      zq[1] = __byte_perm(t0, t2, 0x7632);
      zq[2] = __byte_perm(t1, t3, 0x5410);
      zq[3] = __byte_perm(t1, t3, 0x7632);
      transpose4_lanes(zq, u);
    }
    uint32_t pk[8], dk[8];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 L4 = Lv[cc * 4 + v];
      const float4 D4 = Dv4[cc * 4 + v];
      const float Ls[4] = {L4.x, L4.y, L4.z, L4.w};
      const float Ds[4] = {D4.x, D4.y, D4.z, D4.w};
      float pv[4], dsv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k = 4 * v + e;
        float pe = ex2_approx(fmaf(__uint_as_float(sv[cur][k]), c, -Ls[e]));
        if (kM && static_cast<unsigned>(qoff + cc * 16 + k) >= q_span) pe = 0.f;
        if constexpr (kDropout) {
          // dV takes P o Z * scale and dS = P o (dP o Z * scale - D), with
          // scale = 1 / (1 - threshold / 256)
          const float zs =
              (((zq[v] >> (8 * e)) & 0xffu) >= drop.threshold) ? drop.scale : 0.0f;
          pv[e] = pe * zs;
          dsv[e] = pe * (__uint_as_float(dv[cur][k]) * zs - Ds[e]);
        } else {
          pv[e] = pe;
          dsv[e] = pe * (__uint_as_float(dv[cur][k]) - Ds[e]);
        }
      }
      pk[2 * v] = pack2<E>(pv[0], pv[1]);
      pk[2 * v + 1] = pack2<E>(pv[2], pv[3]);
      dk[2 * v] = pack2<E>(dsv[0], dsv[1]);
      dk[2 * v + 1] = pack2<E>(dsv[2], dsv[3]);
    }
    tmem_st8(tm_s + 8 * cc, pk);
    tmem_st8(tm_dp + 8 * cc, dk);
    // dS into the swizzled shared chunk: 16 queries = 16-byte units 2cc, 2cc+1
    *reinterpret_cast<uint4*>(ds_row + (((2 * cc) ^ (krow & 7)) * 16)) =
        make_uint4(dk[0], dk[1], dk[2], dk[3]);
    *reinterpret_cast<uint4*>(ds_row + (((2 * cc + 1) ^ (krow & 7)) * 16)) =
        make_uint4(dk[4], dk[5], dk[6], dk[7]);
    if (cc + 1 < 4) tmem_wait_ld();
  }
}

// ------------------------------------------------------------------ main kernel

template <int D, Elt E, bool kMasked, bool kDropout = false>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                  const Params p) {
  using C = Cfg<D>;
  if (threadIdx.x == 0) FA_TRACE_CTA(0);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw);
  const uint32_t bars = base + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bars + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + C::kMiscOff + 4);
  volatile unsigned* arrived = reinterpret_cast<volatile unsigned*>(base_ptr + C::kMiscOff + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Without a window's left bound or a block mask (kMasked = false) those are
  // compile-time constants, so the general tile walk folds to the plain / causal one.
  const int wl = kMasked ? p.wl : -1;
  const int wr = p.wr;
  const uint8_t* const blocks = kMasked ? p.blocks : nullptr;

  // Work item: head-major (the resident CTAs share one or two heads' Q, dO and dQ
  // accumulator in L2); within a head, key tile 0 (the heaviest if causal) first.
  const int n_kt = p.Npad / BN;
  const int n_tiles = p.BH * n_kt;
  const int n_whole = n_tiles - p.n_split;
  // this CTA's key tile and, for a split tile, which segment (-1: the whole tile)
  int tile = static_cast<int>(blockIdx.x), seg = -1;
  if (tile >= n_whole) {
    const int c = tile - n_whole;                  // [larger segments][smaller segments]
    const bool second_half = c >= p.n_split;
    tile = n_whole + (second_half ? c - p.n_split : c);
    const bool big_first = p.split_num < 8;        // segment 1 is the larger one
    seg = (second_half == big_first) ? 0 : 1;
  }
  const int bh = p.rank_major ? tile % p.BH : tile / n_kt;
  const int j = p.rank_major ? tile / p.BH : tile % n_kt;
  const int k0 = j * BN;
  const int n_q = (p.N + BM - 1) / BM;
  // query tiles [i_lo, i_hi) hold every query that may see a key of this tile
  const int k1 = min(k0 + BN, p.N) - 1;
  const int i_lo_tile = (wr < 0) ? 0 : max(0, k0 - wr) / BM;
  const int i_hi_tile = (wl < 0) ? n_q : min(n_q, (k1 + wl) / BM + 1);
  // a split tile's segment walks a sub-range of the query tiles (no block mask then)
  int i_lo = i_lo_tile, i_hi = i_hi_tile;
  if (seg >= 0) {
    const int a = split_point(i_hi_tile - i_lo_tile, p.split_num);
    if (seg == 0) i_hi = i_lo_tile + a; else i_lo = i_lo_tile + a;
  }

  // The block-mask column of this key tile as bits: warp w builds words w, w + 16, ...
  uint32_t* mask_bits = reinterpret_cast<uint32_t*>(base_ptr + C::kMaskOff);
  if (blocks != nullptr) pdl_wait();  // the mask may come from the grid before
  if (blocks != nullptr) {
    for (int wi = warp; wi < (n_q + 31) / 32; wi += kThreads / 32) {
      const int i = wi * 32 + lane;
      const bool keep = i < n_q && blocks[static_cast<size_t>(i) * n_kt + j] != 0;
      const uint32_t bits = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) mask_bits[wi] = bits;
    }
  }

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarKV), 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar(C::kBarFull + s), 1);
      mbar_init(bar(C::kBarEmpty + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(C::kBarS + h), 1);
      mbar_init(bar(C::kBarP + h), 4);        // the 4 warps of half h
      mbar_init(bar(C::kBarDQFull + h), 1);
      mbar_init(bar(C::kBarDQEmpty + h), 4);  // the 4 dQ warps
    }
    mbar_init(bar(C::kBarDKDV), 1);
    mbar_init(bar(C::kBarSplitWritten), 8);  // the 8 P/dS warps
    mbar_init(bar(C::kBarSplitDecided), 1);
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
  pdl_wait();  // the grid before this one has completed: global memory is ours
  const Watchdog wd{abort_flag, p.timeout_ns};
  if (threadIdx.x == 0) FA_TRACE_CTA(1);
  if (warp == kWarpMma) FA_TRACE_POINT(0, 0, 0);

  // Does some query of query tile i see a key of this tile?
  auto member = [&](int i) -> bool {
    if (i < i_lo || i >= i_hi) return false;
    return blocks == nullptr || ((mask_bits[i >> 5] >> (i & 31)) & 1u);
  };
  int nsteps = i_hi - i_lo;  // query tiles walked
  if (blocks != nullptr) {
    nsteps = 0;
    for (int i = i_lo; i < i_hi; ++i) nsteps += member(i) ? 1 : 0;
  }

  // ring of half tiles: seq = 4*step + 2*h + w, w = 0 for dO (rows 64h.. of query
  // tile i), w = 1 for Q (with L2 and D of those 64 queries)
  auto seq_of = [](int s, int h, int w) { return 4 * s + 2 * h + w; };
  auto slot_of = [&](int seq) { return seq % C::kSlots; };
  auto round_of = [&](int seq) { return seq / C::kSlots; };
  auto slot_smem = [&](int seq) -> uint32_t {
    return base + C::kRingOff + slot_of(seq) * C::kHalfBytes;
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    // (the whole warp runs the loop; one elected lane issues each copy)
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
    }
    mbar_arrive_expect_tx_e(bar(C::kBarKV), 2 * C::kTileBytes);
    for (int c = 0; c < C::kChunks; ++c) {
      tma_load_3d_e(base + C::kKOff + c * C::kChunkBytes, &tmK, bar(C::kBarKV), c * 64, k0, bh);
      tma_load_3d_e(base + C::kVOff + c * C::kChunkBytes, &tmV, bar(C::kBarKV), c * 64, k0, bh);
    }
    int issued = 0;
    bool ok = true;
    int i = i_lo - 1;
    for (int s = 0; s < nsteps && ok; ++s) {
      do ++i; while (!member(i));
      for (int hw = 0; hw < 4 && ok; ++hw) {
        const int h = hw >> 1, w = hw & 1;
        const int seq = seq_of(s, h, w);
        const int slot = slot_of(seq);
        const int rnd = round_of(seq);
        FA_TRACE_POINT(30, seq, 0);
        if (rnd > 0 && !mbar_wait_warp(bar(C::kBarEmpty + slot), (rnd - 1) & 1, wd)) {
          ok = false;
          break;
        }
        FA_TRACE_POINT(31, seq, 0);
        const uint32_t full = bar(C::kBarFull + slot);
        const uint32_t dst = slot_smem(seq);
        const int row0 = i * BM + 64 * h;
        if (w == 1) {
          mbar_arrive_expect_tx_e(full, C::kHalfBytes + 2 * C::kVecBytes);
          const uint32_t vec = base + C::kVecOff + slot * 2 * C::kVecBytes;
          const size_t off = static_cast<size_t>(bh) * p.Npad + static_cast<size_t>(row0);
          bulk_load_e(vec, p.L2 + off, C::kVecBytes, full);
          bulk_load_e(vec + C::kVecBytes, p.Dv + off, C::kVecBytes, full);
        } else {
          mbar_arrive_expect_tx_e(full, C::kHalfBytes);
        }
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d_e(dst + c * C::kHalfChunkBytes, w ? &tmQ : &tmdO, full, c * 64, row0, bh);
        FA_TRACE_POINT(32, seq, 0);
        issued = seq + 1;
      }
    }
    for (int seq = max(0, issued - C::kSlots); seq < issued; ++seq)
      drain_wait(bar(C::kBarFull + slot_of(seq)), round_of(seq) & 1, p.timeout_ns);
    drain_wait(bar(C::kBarKV), 0, p.timeout_ns);
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // (the whole warp runs the loop; one elected lane issues each MMA and commit)
    const uint32_t k_smem = base + C::kKOff, v_smem = base + C::kVOff;
    const uint32_t ds_smem = base + C::kDSOff;
    const uint32_t tm_s = tmem + C::kTmS, tm_dp = tmem + C::kTmDP;
    bool ok = mbar_wait_warp(bar(C::kBarKV), 0, wd);
    auto wait_full = [&](int seq) -> bool {
      return mbar_wait_warp(bar(C::kBarFull + slot_of(seq)), round_of(seq) & 1, wd);
    };
    // S^T and dP^T of both halves of step s (dP^T first: its columns free up earlier)
    auto issue_sdp = [&](int s) -> bool {
      for (int h = 0; h < 2; ++h) {
        const int seqO = seq_of(s, h, 0), seqQ = seq_of(s, h, 1);
        if (!(wait_full(seqO) && wait_full(seqQ))) return false;
        FA_TRACE_POINT(5, s, h);
        tc_fence_after();
        issue_xyT_half<D, E>(tm_dp + 64 * h, v_smem, slot_smem(seqO));
        if (D == 128 && s > 0) {  // S^T_h shares columns with dQ^T_h of the last step
          if (!mbar_wait_warp(bar(C::kBarDQEmpty + h), (s - 1) & 1, wd)) return false;
          FA_TRACE_POINT(7, s, h);
          tc_fence_after();
        }
        issue_xyT_half<D, E>(tm_s + 64 * h, k_smem, slot_smem(seqQ));
        tc_commit_e(bar(C::kBarS + h));
        FA_TRACE_POINT(8, s, h);
        if (s == 0 && h == 0 && lane == 0) FA_TRACE_CTA(2);
      }
      return true;
    };
    if (ok && nsteps > 0) ok = issue_sdp(0);
    for (int s = 0; s < nsteps && ok; ++s) {
      for (int h = 0; h < 2 && ok; ++h) {
        const int seqO = seq_of(s, h, 0), seqQ = seq_of(s, h, 1);
        FA_TRACE_POINT(1, s, h);
        if (!mbar_wait_warp(bar(C::kBarP + h), s & 1, wd)) { ok = false; break; }
        FA_TRACE_POINT(2, s, h);
        tc_fence_after();
        const bool acc = (s > 0) || (h > 0);
        issue_acc_half<D, E>(tmem + C::kTmDV, tm_s + 64 * h, slot_smem(seqO), acc);   // dV
        issue_acc_half<D, E>(tmem + C::kTmDK, tm_dp + 64 * h, slot_smem(seqQ), acc);  // dK
        // dV and dK are the last readers of this half's dO and Q: free their slots
        // before the dQ product, so that the next loads start a product earlier
        tc_commit_e(bar(C::kBarEmpty + slot_of(seqO)));
        tc_commit_e(bar(C::kBarEmpty + slot_of(seqQ)));
        if constexpr (D == 128) {
          issue_dqT_half<E>(tm_s + 64 * h, k_smem, ds_smem + h * C::kChunkBytes);
          tc_commit_e(bar(C::kBarDQFull + h));
        }
        FA_TRACE_POINT(3, s, h);
      }
      if (!ok) break;
      if constexpr (D == 64) {
        if (s > 0) {  // the dQ columns are reused: the previous dQ must have been read
          if (!mbar_wait_warp(bar(C::kBarDQEmpty), (s - 1) & 1, wd)) { ok = false; break; }
          tc_fence_after();
        }
        issue_dq64<E>(tmem + C::kTmDQ64, ds_smem, k_smem);
        tc_commit_e(bar(C::kBarDQFull));
      }
      if (s + 1 < nsteps) ok = issue_sdp(s + 1);
    }
    if (ok) tc_commit_e(bar(C::kBarDKDV));
    tc_commit_e(bar(C::kBarDrain));
    drain_wait(bar(C::kBarDrain), 0, p.timeout_ns);
    __syncwarp();
    FA_TRACE_POINT(99, 0, 0);
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T, dS^T (key rows)
    const int h = warp >> 2;                  // query half
    const int krow = (warp & 3) * 32 + lane;  // key row within the tile = TMEM lane
    const int key = k0 + krow;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tm_s = tmem + lane_off + C::kTmS + 64 * h;
    const uint32_t tm_dp = tmem + lane_off + C::kTmDP + 64 * h;
    const float c = p.scale_log2;
    uint8_t* ds_row = base_ptr + C::kDSOff + h * C::kChunkBytes + krow * 128;
    const bool ragged_keys = k0 + BN > p.N;
    const int dq_bar = (D == 128) ? C::kBarDQFull + h : C::kBarDQFull;
    // queries that see this key row: [q_lo, q_hi) (empty for a padding key)
    const int q_lo = (wr < 0) ? 0 : key - wr;
    const int q_hi = (key >= p.N) ? q_lo : ((wl < 0) ? p.Npad + BM : key + wl + 1);
    const unsigned q_span = static_cast<unsigned>(q_hi - q_lo);
    const uint32_t ctr_head = p.drop.head_base + static_cast<uint32_t>(bh);  // dropout
    bool ok = true;
    int i = i_lo - 1;
    for (int s = 0; s < nsteps && ok; ++s) {
      do ++i; while (!member(i));
      const int qh0 = i * BM + 64 * h;  // first query of this half
      // The two barriers that completed long ago are observed first, so that the work
      // starts as soon as S^T and dP^T are in TMEM: the dQ MMA of the last step has
      // finished reading this dS chunk, and L2 and D of this half arrived with its Q rows.
      if (s > 0)
        ok = __all_sync(0xffffffffu, mbar_wait(bar(dq_bar), (s - 1) & 1, wd));
      if ((warp & 3) == 0) FA_TRACE_POINT(10, s, h);
      const int seqQ = seq_of(s, h, 1);
      if (ok)
        ok = __all_sync(0xffffffffu,
                        mbar_wait(bar(C::kBarFull + slot_of(seqQ)), round_of(seqQ) & 1, wd));
      if ((warp & 3) == 0) FA_TRACE_POINT(12, s, h);
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarS + h), s & 1, wd));
      if ((warp & 3) == 0) FA_TRACE_POINT(14, s, h);
      if (!ok) break;
      tc_fence_after();
      const float4* Lv = reinterpret_cast<const float4*>(
          base_ptr + C::kVecOff + slot_of(seqQ) * 2 * C::kVecBytes);
      const float4* Dv4 = Lv + 64 / 4;
      // masking is needed only where the half crosses an edge of some key's visible
      // queries (the causal diagonal, a window edge) and on a ragged key tile
      const bool mask = ragged_keys || (wr >= 0 && k0 + BN - 1 - wr > qh0) ||
                        (wl >= 0 && k0 + wl < qh0 + 63);
      const int qoff = qh0 - q_lo;  // query qh0 + x is visible iff qoff + x < q_span (unsigned)
      // The element loop in two compiled forms: with the mask tests only on steps
      // that cross a mask edge, none on all the others.
      if (mask)
        p_ds_half<E, kDropout, true>(tm_s, tm_dp, Lv, Dv4, c, key, qh0, ctr_head, p.drop, lane,
                                     qoff, q_span, ds_row, krow);
      else
        p_ds_half<E, kDropout, false>(tm_s, tm_dp, Lv, Dv4, c, key, qh0, ctr_head, p.drop, lane,
                                      qoff, q_span, ds_row, krow);
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarP + h));
      if ((warp & 3) == 0) FA_TRACE_POINT(16, s, h);
    }
    if (nsteps == 0 && key < p.N) {
      // no query sees this key: dK = dV = 0 (warps 0-3 dK, warps 4-7 dV)
      uint4* dst = reinterpret_cast<uint4*>((h == 0 ? p.dK : p.dV) +
                                            (static_cast<size_t>(bh) * p.N + key) * D);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (ok && nsteps > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDKDV), 0, wd));
    if (threadIdx.x == 0) FA_TRACE_CTA(3);
    if (ok && nsteps > 0) {
      // warps 0-3 write dK (times scale), warps 4-7 write dV; a split tile's segment
      // writes its fp32 partial to its slot instead
      tc_fence_after();
      const uint32_t tm_acc = tmem + lane_off + (h == 0 ? C::kTmDK : C::kTmDV);
      uint16_t* out = (h == 0 ? p.dK : p.dV) + (static_cast<size_t>(bh) * p.N + key) * D;
      const float mul = (h == 0) ? p.scale : 1.0f;
      const int ksplit = tile - n_whole;
      // slot layout: [split tile][segment][dK, dV][128 key rows][D]
      auto slot_row = [&](int sg) -> float* {
        return p.part + ((static_cast<size_t>(ksplit) * 2 + sg) * 2 + h) * (BN * D) +
               static_cast<size_t>(krow) * D;
      };
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tm_acc + cc * 32, v);
        tmem_wait_ld();
        if (seg >= 0) {
          float4* dst = reinterpret_cast<float4*>(slot_row(seg) + cc * 32);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[u] = make_float4(__uint_as_float(v[4 * u]), __uint_as_float(v[4 * u + 1]),
                                 __uint_as_float(v[4 * u + 2]), __uint_as_float(v[4 * u + 3]));
          continue;
        }
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pk[k] = pack2<E>(__uint_as_float(v[2 * k]) * mul, __uint_as_float(v[2 * k + 1]) * mul);
        if (key < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      if (seg >= 0) {
        // Count this segment in once all 8 warps' rows are written (bounded waits); the
        // second to arrive adds slot 0 and slot 1, in that order, and writes dK, dV.
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::kBarSplitWritten));
        if (warp == 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSplitWritten), 0, wd));
          if (ok && lane == 0) {
            __threadfence();
            *arrived = atomicAdd(p.arrivals + ksplit, 1u);
            mbar_arrive(bar(C::kBarSplitDecided));
          }
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSplitDecided), 0, wd));
        if (ok && *arrived == 1u) {
          __threadfence();
          const float4* s0 = reinterpret_cast<const float4*>(slot_row(0));
          const float4* s1 = reinterpret_cast<const float4*>(slot_row(1));
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            float4 a[8], b[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              a[u] = __ldcg(s0 + cc * 8 + u);
              b[u] = __ldcg(s1 + cc * 8 + u);
            }
            uint32_t pk[16];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              pk[2 * u] = pack2<E>((a[u].x + b[u].x) * mul, (a[u].y + b[u].y) * mul);
              pk[2 * u + 1] = pack2<E>((a[u].z + b[u].z) * mul, (a[u].w + b[u].w) * mul);
            }
            if (key < p.N) {
              uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
              for (int u = 0; u < 4; ++u)
                dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
            }
          }
        }
      }
    }
    if (threadIdx.x == 0) FA_TRACE_CTA(5);
  } else if (warp < kWarpTma) {
    // ------------------------------------------------------------ dQ readout
    const int wq = warp - kWarpDq;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int row = wq * 32 + lane;  // TMEM lane: head-dim element (D = 128) or query (D = 64)
    bool ok = true;
    int i = i_lo - 1;
    for (int s = 0; s < nsteps && ok; ++s) {
      do ++i; while (!member(i));
      const int q0 = i * BM;
      if constexpr (D == 128) {
        for (int h = 0; h < 2 && ok; ++h) {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDQFull + h), s & 1, wd));
          if (!ok) break;
          if (warp == kWarpDq) FA_TRACE_POINT(20, s, h);
          tc_fence_after();
          uint32_t v[2][32];
          tmem_ld32(tmem + lane_off + C::kTmS + 64 * h, v[0]);
          tmem_ld32(tmem + lane_off + C::kTmS + 64 * h + 32, v[1]);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::kBarDQEmpty + h));
          if (warp == kWarpDq) FA_TRACE_POINT(22, s, h);
          // element `row` of the head dimension for 64 queries: a warp covers 32
          // consecutive elements of one query row (128 contiguous bytes) per add
          float* dst = p.dQacc + (static_cast<size_t>(bh) * p.N + q0 + 64 * h) * D + row;
          const int nq = min(64, p.N - (q0 + 64 * h));
#pragma unroll
          for (int qq = 0; qq < 64; ++qq)
            if (qq < nq) red_add(dst + static_cast<size_t>(qq) * D, __uint_as_float(v[qq / 32][qq % 32]));
          if (warp == kWarpDq) FA_TRACE_POINT(24, s, h);
        }
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDQFull), s & 1, wd));
        if (!ok) break;
        tc_fence_after();
        uint32_t v[2][32];
        tmem_ld32(tmem + lane_off + C::kTmDQ64, v[0]);
        tmem_ld32(tmem + lane_off + C::kTmDQ64 + 32, v[1]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::kBarDQEmpty));
        const int q = q0 + row;
        if (q < p.N) {
          float* dst = p.dQacc + (static_cast<size_t>(bh) * p.N + q) * D;
#pragma unroll
          for (int k = 0; k < 16; ++k)
            red_add_v4(dst + 4 * k, __uint_as_float(v[k / 8][(4 * k) % 32]),
                       __uint_as_float(v[k / 8][(4 * k + 1) % 32]),
                       __uint_as_float(v[k / 8][(4 * k + 2) % 32]),
                       __uint_as_float(v[k / 8][(4 * k + 3) % 32]));
        }
      }
    }
    if (warp == kWarpDq && lane == 0) FA_TRACE_CTA(6);
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) FA_TRACE_CTA(4);
  pdl_launch_dependents();  // the next grid may launch: this CTA's work is done
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

// The persistent form of fa_bwd_kernel, for launches of many short key tiles:
// min(tiles, SMs) CTAs, each walking a list of key tiles (items) and reusing its
// buffers from one to the next: K/V once the item's last product has read them
// (KVEmpty), dK/dV in TMEM once the epilogue has read them out (DKDVFree). Ring
// indices and barrier phases run on across items, so the next item's first products
// start while the P/dS warps write the last item's dK, dV and the dQ warps add its
// last dQ. The same roles, products and arithmetic; no split tiles and no block mask.
template <int D, Elt E, bool kMasked, bool kDropout>
__global__ void __launch_bounds__(kThreads, 1)
    fa_bwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ,
                             const __grid_constant__ CUtensorMap tmK,
                             const __grid_constant__ CUtensorMap tmV,
                             const __grid_constant__ CUtensorMap tmdO, const Params p) {
  using C = Cfg<D>;
  if (threadIdx.x == 0) FA_TRACE_CTA(0);
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
  const int wl = kMasked ? p.wl : -1;
  const int wr = p.wr;
  const int n_kt = p.Npad / BN;
  const int n_tiles = p.BH * n_kt;
  const int n_q = (p.N + BM - 1) / BM;

  // Items: key tile i of the list (head-major or rank-major, as p.rank_major says); the
  // k-th item of CTA b is k * G + b for even k and k * G + (G - 1 - b) for odd k.
  auto item_of = [&](int k) -> int {
    const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    const int i = k * G + ((k & 1) ? (G - 1 - b) : b);
    return i < n_tiles ? i : -1;
  };
  // An item's (batch, head), key tile and the query tiles [i_lo, i_hi) it walks.
  struct Work {
    int bh, j, k0, i_lo, i_hi;
  };
  auto decode = [&](int tile, Work& w) {
    w.bh = p.rank_major ? tile % p.BH : tile / n_kt;
    w.j = p.rank_major ? tile / p.BH : tile % n_kt;
    w.k0 = w.j * BN;
    const int k1 = min(w.k0 + BN, p.N) - 1;
    w.i_lo = (wr < 0) ? 0 : max(0, w.k0 - wr) / BM;
    w.i_hi = (wl < 0) ? n_q : min(n_q, (k1 + wl) / BM + 1);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarKV), 1);
    mbar_init(bar(C::kBarKVEmpty), 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar(C::kBarFull + s), 1);
      mbar_init(bar(C::kBarEmpty + s), 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(bar(C::kBarS + h), 1);
      mbar_init(bar(C::kBarP + h), 4);        // the 4 warps of half h
      mbar_init(bar(C::kBarDQFull + h), 1);
      mbar_init(bar(C::kBarDQEmpty + h), 4);  // the 4 dQ warps
    }
    mbar_init(bar(C::kBarDKDV), 1);
    mbar_init(bar(C::kBarDKDVFree), 8);  // the 8 P/dS warps
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
  pdl_wait();  // the grid before this one has completed: global memory is ours
  const Watchdog wd{abort_flag, p.timeout_ns};
  if (threadIdx.x == 0) FA_TRACE_CTA(1);

  // ring of half tiles: seq = 4 * step + 2 * h + w over all the CTA's steps, w = 0 for
  // dO (rows 64h.. of query tile i), w = 1 for Q (with L2 and D of those 64 queries)
  auto seq_of = [](int s, int h, int w) { return 4 * s + 2 * h + w; };
  auto slot_of = [&](int seq) { return seq % C::kSlots; };
  auto round_of = [&](int seq) { return seq / C::kSlots; };
  auto slot_smem = [&](int seq) -> uint32_t {
    return base + C::kRingOff + slot_of(seq) * C::kHalfBytes;
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
    }
    int issued = 0;  // ring sequence numbers issued
    int n_kv = 0;    // K/V loads so far (items with steps)
    int s0 = 0;      // steps of the items before
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = item_of(k);
      if (item < 0) break;
      Work w;
      decode(item, w);
      const int nsteps = w.i_hi - w.i_lo;
      if (nsteps == 0) continue;
      // the previous item's products must be done with K and V
      if (n_kv > 0 && !mbar_wait_warp(bar(C::kBarKVEmpty), (n_kv - 1) & 1, wd)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx_e(bar(C::kBarKV), 2 * C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c) {
        tma_load_3d_e(base + C::kKOff + c * C::kChunkBytes, &tmK, bar(C::kBarKV), c * 64, w.k0,
                      w.bh);
        tma_load_3d_e(base + C::kVOff + c * C::kChunkBytes, &tmV, bar(C::kBarKV), c * 64, w.k0,
                      w.bh);
      }
      ++n_kv;
      for (int s = 0; s < nsteps && ok; ++s) {
        const int i = w.i_lo + s;
        for (int hw = 0; hw < 4 && ok; ++hw) {
          const int h = hw >> 1, wv = hw & 1;
          const int seq = seq_of(s0 + s, h, wv);
          const int slot = slot_of(seq);
          const int rnd = round_of(seq);
          if (rnd > 0 && !mbar_wait_warp(bar(C::kBarEmpty + slot), (rnd - 1) & 1, wd)) {
            ok = false;
            break;
          }
          const uint32_t full = bar(C::kBarFull + slot);
          const uint32_t dst = slot_smem(seq);
          const int row0 = i * BM + 64 * h;
          if (wv == 1) {
            mbar_arrive_expect_tx_e(full, C::kHalfBytes + 2 * C::kVecBytes);
            const uint32_t vec = base + C::kVecOff + slot * 2 * C::kVecBytes;
            const size_t off = static_cast<size_t>(w.bh) * p.Npad + static_cast<size_t>(row0);
            bulk_load_e(vec, p.L2 + off, C::kVecBytes, full);
            bulk_load_e(vec + C::kVecBytes, p.Dv + off, C::kVecBytes, full);
          } else {
            mbar_arrive_expect_tx_e(full, C::kHalfBytes);
          }
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d_e(dst + c * C::kHalfChunkBytes, wv ? &tmQ : &tmdO, full, c * 64, row0,
                          w.bh);
          issued = seq + 1;
        }
      }
      s0 += nsteps;
    }
    for (int seq = max(0, issued - C::kSlots); seq < issued; ++seq)
      drain_wait(bar(C::kBarFull + slot_of(seq)), round_of(seq) & 1, p.timeout_ns);
    if (n_kv > 0) drain_wait(bar(C::kBarKV), (n_kv - 1) & 1, p.timeout_ns);
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t k_smem = base + C::kKOff, v_smem = base + C::kVOff;
    const uint32_t ds_smem = base + C::kDSOff;
    const uint32_t tm_s = tmem + C::kTmS, tm_dp = tmem + C::kTmDP;
    auto wait_full = [&](int seq) -> bool {
      return mbar_wait_warp(bar(C::kBarFull + slot_of(seq)), round_of(seq) & 1, wd);
    };
    // S^T and dP^T of both halves of the CTA's step g (dP^T first: its columns free up
    // earlier)
    auto issue_sdp = [&](int g) -> bool {
      for (int h = 0; h < 2; ++h) {
        const int seqO = seq_of(g, h, 0), seqQ = seq_of(g, h, 1);
        if (!(wait_full(seqO) && wait_full(seqQ))) return false;
        tc_fence_after();
        issue_xyT_half<D, E>(tm_dp + 64 * h, v_smem, slot_smem(seqO));
        if (D == 128 && g > 0) {  // S^T_h shares columns with dQ^T_h of the step before
          if (!mbar_wait_warp(bar(C::kBarDQEmpty + h), (g - 1) & 1, wd)) return false;
          tc_fence_after();
        }
        issue_xyT_half<D, E>(tm_s + 64 * h, k_smem, slot_smem(seqQ));
        tc_commit_e(bar(C::kBarS + h));
      }
      return true;
    };
    int n_kv = 0;  // items with steps so far
    int g0 = 0;    // the CTA's step number of the item's first step
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = item_of(k);
      if (item < 0) break;
      Work w;
      decode(item, w);
      const int nsteps = w.i_hi - w.i_lo;
      if (nsteps == 0) continue;
      ok = mbar_wait_warp(bar(C::kBarKV), n_kv & 1, wd);
      if (ok) ok = issue_sdp(g0);
      for (int s = 0; s < nsteps && ok; ++s) {
        const int g = g0 + s;
        for (int h = 0; h < 2 && ok; ++h) {
          const int seqO = seq_of(g, h, 0), seqQ = seq_of(g, h, 1);
          if (!mbar_wait_warp(bar(C::kBarP + h), g & 1, wd)) { ok = false; break; }
          // the item's first dV and dK overwrite the accumulators: the previous item's
          // epilogue must have read them out
          if (s == 0 && h == 0 && n_kv > 0 &&
              !mbar_wait_warp(bar(C::kBarDKDVFree), (n_kv - 1) & 1, wd)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const bool acc = (s > 0) || (h > 0);
          issue_acc_half<D, E>(tmem + C::kTmDV, tm_s + 64 * h, slot_smem(seqO), acc);   // dV
          issue_acc_half<D, E>(tmem + C::kTmDK, tm_dp + 64 * h, slot_smem(seqQ), acc);  // dK
          tc_commit_e(bar(C::kBarEmpty + slot_of(seqO)));
          tc_commit_e(bar(C::kBarEmpty + slot_of(seqQ)));
          if constexpr (D == 128) {
            issue_dqT_half<E>(tm_s + 64 * h, k_smem, ds_smem + h * C::kChunkBytes);
            tc_commit_e(bar(C::kBarDQFull + h));
          }
        }
        if (!ok) break;
        if constexpr (D == 64) {
          if (g > 0) {  // the dQ columns are reused: the previous dQ must have been read
            if (!mbar_wait_warp(bar(C::kBarDQEmpty), (g - 1) & 1, wd)) { ok = false; break; }
            tc_fence_after();
          }
          issue_dq64<E>(tmem + C::kTmDQ64, ds_smem, k_smem);
          tc_commit_e(bar(C::kBarDQFull));
        }
        if (s + 1 < nsteps) ok = issue_sdp(g + 1);
      }
      if (!ok) break;
      tc_commit_e(bar(C::kBarDKDV));     // dK, dV complete
      tc_commit_e(bar(C::kBarKVEmpty));  // K, V no longer read
      ++n_kv;
      g0 += nsteps;
    }
    tc_commit_e(bar(C::kBarDrain));
    drain_wait(bar(C::kBarDrain), 0, p.timeout_ns);
    __syncwarp();
  } else if (warp < 8) {
    // ------------------------------------------------------------ P^T, dS^T (key rows)
    const int h = warp >> 2;                  // query half
    const int krow = (warp & 3) * 32 + lane;  // key row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tm_s = tmem + lane_off + C::kTmS + 64 * h;
    const uint32_t tm_dp = tmem + lane_off + C::kTmDP + 64 * h;
    const float c = p.scale_log2;
    uint8_t* ds_row = base_ptr + C::kDSOff + h * C::kChunkBytes + krow * 128;
    const int dq_bar = (D == 128) ? C::kBarDQFull + h : C::kBarDQFull;
    int n_kv = 0, g0 = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = item_of(k);
      if (item < 0) break;
      Work w;
      decode(item, w);
      const int nsteps = w.i_hi - w.i_lo;
      const int key = w.k0 + krow;
      uint16_t* out = (h == 0 ? p.dK : p.dV) + (static_cast<size_t>(w.bh) * p.N + key) * D;
      if (nsteps == 0) {
        // no query sees this key: dK = dV = 0 (warps 0-3 dK, warps 4-7 dV)
        if (key < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(out);
#pragma unroll
          for (int u = 0; u < D / 8; ++u) dst[u] = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const bool ragged_keys = w.k0 + BN > p.N;
      // queries that see this key row: [q_lo, q_hi) (empty for a padding key)
      const int q_lo = (wr < 0) ? 0 : key - wr;
      const int q_hi = (key >= p.N) ? q_lo : ((wl < 0) ? p.Npad + BM : key + wl + 1);
      const unsigned q_span = static_cast<unsigned>(q_hi - q_lo);
      const uint32_t ctr_head = p.drop.head_base + static_cast<uint32_t>(w.bh);  // dropout
      for (int s = 0; s < nsteps && ok; ++s) {
        const int g = g0 + s;
        const int qh0 = (w.i_lo + s) * BM + 64 * h;  // first query of this half
        // the dQ product of the step before has read this dS chunk; L2 and D of this
        // half arrived with its Q rows; then S^T and dP^T
        if (g > 0) ok = __all_sync(0xffffffffu, mbar_wait(bar(dq_bar), (g - 1) & 1, wd));
        const int seqQ = seq_of(g, h, 1);
        if (ok)
          ok = __all_sync(0xffffffffu,
                          mbar_wait(bar(C::kBarFull + slot_of(seqQ)), round_of(seqQ) & 1, wd));
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarS + h), g & 1, wd));
        if (!ok) break;
        tc_fence_after();
        const float4* Lv = reinterpret_cast<const float4*>(
            base_ptr + C::kVecOff + slot_of(seqQ) * 2 * C::kVecBytes);
        const float4* Dv4 = Lv + 64 / 4;
        const bool mask = ragged_keys || (wr >= 0 && w.k0 + BN - 1 - wr > qh0) ||
                          (wl >= 0 && w.k0 + wl < qh0 + 63);
        const int qoff = qh0 - q_lo;
        if (mask)
          p_ds_half<E, kDropout, true>(tm_s, tm_dp, Lv, Dv4, c, key, qh0, ctr_head, p.drop, lane,
                                       qoff, q_span, ds_row, krow);
        else
          p_ds_half<E, kDropout, false>(tm_s, tm_dp, Lv, Dv4, c, key, qh0, ctr_head, p.drop, lane,
                                        qoff, q_span, ds_row, krow);
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(C::kBarP + h));
      }
      if (!ok) break;
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDKDV), n_kv & 1, wd));
      if (!ok) break;
      // warps 0-3 write dK (times scale), warps 4-7 write dV
      tc_fence_after();
      const uint32_t tm_acc = tmem + lane_off + (h == 0 ? C::kTmDK : C::kTmDV);
      const float mul = (h == 0) ? p.scale : 1.0f;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(tm_acc + cc * 32, v);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int kk = 0; kk < 16; ++kk)
          pk[kk] = pack2<E>(__uint_as_float(v[2 * kk]) * mul, __uint_as_float(v[2 * kk + 1]) * mul);
        if (key < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(out + cc * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        }
      }
      // dK and dV are out of TMEM: the next item's first products may overwrite them
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarDKDVFree));
      ++n_kv;
      g0 += nsteps;
    }
  } else if (warp < kWarpTma) {
    // ------------------------------------------------------------ dQ readout
    const int wq = warp - kWarpDq;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int row = wq * 32 + lane;  // TMEM lane: head-dim element (D = 128) or query (D = 64)
    int g0 = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = item_of(k);
      if (item < 0) break;
      Work w;
      decode(item, w);
      const int nsteps = w.i_hi - w.i_lo;
      for (int s = 0; s < nsteps && ok; ++s) {
        const int g = g0 + s;
        const int q0 = (w.i_lo + s) * BM;
        if constexpr (D == 128) {
          for (int h = 0; h < 2 && ok; ++h) {
            ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDQFull + h), g & 1, wd));
            if (!ok) break;
            tc_fence_after();
            uint32_t v[2][32];
            tmem_ld32(tmem + lane_off + C::kTmS + 64 * h, v[0]);
            tmem_ld32(tmem + lane_off + C::kTmS + 64 * h + 32, v[1]);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarDQEmpty + h));
            // element `row` of the head dimension for 64 queries: a warp covers 32
            // consecutive elements of one query row (128 contiguous bytes) per add
            float* dst = p.dQacc + (static_cast<size_t>(w.bh) * p.N + q0 + 64 * h) * D + row;
            const int nq = min(64, p.N - (q0 + 64 * h));
#pragma unroll
            for (int qq = 0; qq < 64; ++qq)
              if (qq < nq) red_add(dst + static_cast<size_t>(qq) * D, __uint_as_float(v[qq / 32][qq % 32]));
          }
        } else {
          ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarDQFull), g & 1, wd));
          if (!ok) break;
          tc_fence_after();
          uint32_t v[2][32];
          tmem_ld32(tmem + lane_off + C::kTmDQ64, v[0]);
          tmem_ld32(tmem + lane_off + C::kTmDQ64 + 32, v[1]);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::kBarDQEmpty));
          const int q = q0 + row;
          if (q < p.N) {
            float* dst = p.dQacc + (static_cast<size_t>(w.bh) * p.N + q) * D;
#pragma unroll
            for (int kk = 0; kk < 16; ++kk)
              red_add_v4(dst + 4 * kk, __uint_as_float(v[kk / 8][(4 * kk) % 32]),
                         __uint_as_float(v[kk / 8][(4 * kk + 1) % 32]),
                         __uint_as_float(v[kk / 8][(4 * kk + 2) % 32]),
                         __uint_as_float(v[kk / 8][(4 * kk + 3) % 32]));
          }
        }
      }
      g0 += nsteps;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) FA_TRACE_CTA(4);
  pdl_launch_dependents();  // the next grid may launch: this CTA's work is done
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

}  // namespace bwd
}  // namespace fa
