// fa_fwd_sm100.cuh -- fused attention forward for sm_100a (bf16 in, fp32 accumulate).
//
// Method: the blockwise forward of "FlashAttention optimisation: breaking the
// performance bottleneck of standard attention", section 4.1 (for each query
// block, stream the key/value blocks, update the running max m and sum l, rescale
// the partial output, divide by l at the end, write O and the normaliser once),
// with the online-softmax merge of "A survey of key techniques of large language
// model pre-training systems" (Journal of Software 2026(1), p.218: m = max(m1,
// m2), l = e^(m1-m) l1 + e^(m2-m) l2). Causal tiles above the diagonal are skipped
// ("Flash Attention-2: acceleration principle ...", causal-mask item).
//
// B200 mapping (one CTA per SM, 320 threads):
//   * CTA = 2 query tiles of 128 rows (256 rows) of one (batch, head); the two
//     tiles ping-pong so that one tile's softmax overlaps the other's MMAs.
//   * warp 8: TMA producer. Q tiles once; K and V tiles of 128 rows through a ring
//     of NSLOT shared-memory slots (128-byte swizzle), full/empty mbarriers.
//   * warp 9: MMA issuer (one thread). S_t = Q_t K_j^T with tcgen05.mma into TMEM
//     (128 fp32 columns per tile); O_t += P_t V_j with P_t read from TMEM.
//   * warps 0-3 / 4-7: softmax of tile 0 / 1, one thread per query row (TMEM lane).
//     Scores are read with tcgen05.ld, the running max and sum stay in registers,
//     p = 2^(s*c - m) with c = scale*log2(e) folded into one FFMA before ex2, P is
//     rounded to bf16 and stored over the S columns for the PV MMA. O is rescaled
//     in TMEM only when the running max grew by more than 2^8 (exact: O and l
//     always share the same reference max).
//   * TMEM: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D); P_t
//     (bf16 pairs) aliases the first 64 columns of S_t.
//   * Epilogue: O/l rounded to bf16 stored row per thread; LSE = (m + log2 l) ln 2.
#pragma once

#include "fa_ptx.cuh"

namespace fa {
namespace fwd {

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // key/value rows per tile
constexpr int kThreads = 320;  // 8 softmax warps + producer + MMA
constexpr int kWarpTma = 8;
constexpr int kWarpMma = 9;
constexpr float kRescaleThreshold = 8.0f;  // log2 domain: rescale when max grows > 2^8
// When kPolyPeriod > 0, one pair of exponentials in every kPolyPeriod goes to the
// polynomial exp2 on the FMA pipe (exp2_poly2) instead of MUFU. Measured on B200
// at d = 128 the forward is not MUFU-bound (timing is unchanged with the softmax
// arithmetic removed), and moving 12.5% or 25% of the exponentials made it 1.5% and
// 2% slower, so it is off.
constexpr int kPolyPeriod = 0;

template <int D>
struct Cfg {
  static constexpr int kChunkBytes = 128 * 128;      // 128 rows x 64 bf16 (one TMA box)
  static constexpr int kChunks = D / 64;             // boxes per 128 x D tile
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kSlots = (D == 128) ? 5 : 10;  // K/V ring slots
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kSlots * kTileBytes;
  // barriers: q_full[2], kv_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], drain
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKVFull = 2;
  static constexpr int kBarKVEmpty = 2 + kSlots;
  static constexpr int kBarSFull = 2 + 2 * kSlots;
  static constexpr int kBarPFull = kBarSFull + 2;
  static constexpr int kBarOFull = kBarPFull + 2;
  static constexpr int kBarDrain = kBarOFull + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + 1024 for alignment
  static constexpr uint32_t kTmS0 = 0, kTmO0 = 256;
  static constexpr uint32_t kTmCols = 512;
};

struct Params {
  __nv_bfloat16* O;
  float* LSE;
  int N;
  int BH;
  int n_qblk;        // ceil(N / 256)
  float scale_log2;  // scale * log2(e)
  int causal;
  unsigned long long timeout_ns;
};

template <int D>
__device__ __forceinline__ void issue_s(uint32_t tm_d, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, 0, 0);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * Cfg<D>::kChunkBytes + (kk % 4) * 32;
    mma_ss(tm_d, sdesc_sw128(q_smem + off, 16, 1024), sdesc_sw128(k_smem + off, 16, 1024), idesc,
           kk > 0 ? 1u : 0u);
  }
}

template <int D>
__device__ __forceinline__ void issue_pv(uint32_t tm_o, uint32_t tm_p, uint32_t v_smem,
                                         bool accumulate) {
  constexpr uint32_t idesc = idesc_bf16_f32(BM, D, 0, 1);
#pragma unroll
  for (int kk = 0; kk < BN / 16; ++kk) {
    mma_ts(tm_o, tm_p + kk * 8,
           sdesc_sw128(v_smem + kk * 16 * 128, Cfg<D>::kChunkBytes, 1024), idesc,
           (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Drain wait: ignores the abort flag, bounded by its own limit. Used at teardown so
// that no copy or MMA is in flight when the CTA releases TMEM and exits.
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicOr(&g_status, kStatusTimeout);
      return;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
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

  // Work item: heaviest query blocks first (matters for causal).
  const int qb = (p.n_qblk - 1) - static_cast<int>(blockIdx.x) / p.BH;
  const int bh = static_cast<int>(blockIdx.x) % p.BH;
  const int q0 = qb * 2 * BM;
  const int n_kv_total = (p.N + BN - 1) / BN;
  int nk[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r0 = q0 + t * BM;
    nk[t] = (r0 < p.N) ? (p.causal ? min(r0 / BN + 1, n_kv_total) : n_kv_total) : 0;
  }
  const int nkv = max(nk[0], nk[1]);

  if (threadIdx.x == 0) {
    mbar_init(bar(C::kBarQFull + 0), 1);
    mbar_init(bar(C::kBarQFull + 1), 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(bar(C::kBarKVFull + s), 1);
      mbar_init(bar(C::kBarKVEmpty + s), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::kBarSFull + t), 1);
      mbar_init(bar(C::kBarPFull + t), 4);  // one arrival per softmax warp
      mbar_init(bar(C::kBarOFull + t), 1);
    }
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

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      for (int t = 0; t < 2; ++t) {
        if (nk[t] == 0) continue;
        const uint32_t dst = base + C::kQOff + t * C::kTileBytes;
        mbar_arrive_expect_tx(bar(C::kBarQFull + t), C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d(dst + c * C::kChunkBytes, &tmQ, bar(C::kBarQFull + t), c * 64, q0 + t * BM,
                      bh);
      }
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv && ok; ++j) {
        for (int w = 0; w < 2; ++w) {
          const int seq = 2 * j + w;
          const int slot = seq % C::kSlots;
          const int rnd = seq / C::kSlots;
          if (rnd > 0 && !mbar_wait(bar(C::kBarKVEmpty + slot), (rnd - 1) & 1, wd)) {
            ok = false;
            break;
          }
          const uint32_t dst = base + C::kKVOff + slot * C::kTileBytes;
          mbar_arrive_expect_tx(bar(C::kBarKVFull + slot), C::kTileBytes);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d(dst + c * C::kChunkBytes, w ? &tmV : &tmK, bar(C::kBarKVFull + slot),
                        c * 64, j * BN, bh);
          issued = seq + 1;
        }
      }
      // Every issued copy must land before the CTA may exit.
      for (int seq = max(0, issued - C::kSlots); seq < issued; ++seq)
        drain_wait(bar(C::kBarKVFull + seq % C::kSlots), (seq / C::kSlots) & 1, p.timeout_ns);
      for (int t = 0; t < 2; ++t)
        if (nk[t] > 0) drain_wait(bar(C::kBarQFull + t), 0, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int t = 0; t < 2 && ok; ++t)
        if (nk[t] > 0) ok = mbar_wait(bar(C::kBarQFull + t), 0, wd);
      const uint32_t q_smem[2] = {base + C::kQOff, base + C::kQOff + C::kTileBytes};
      auto slot_smem = [&](int seq) -> uint32_t {
        return base + C::kKVOff + (seq % C::kSlots) * C::kTileBytes;
      };
      auto wait_full = [&](int seq) -> bool {
        return mbar_wait(bar(C::kBarKVFull + seq % C::kSlots), (seq / C::kSlots) & 1, wd);
      };
      // Each K/V slot is released by a commit issued right after the last MMA that
      // reads it (a commit fires once every earlier MMA is complete), so the
      // producer can refill it as early as possible.
      // K_j is read by S_t(j) for the tiles with j < nk[t]; V_j by PV_t(j). Tile 1
      // never has fewer key tiles than tile 0 (causal) unless it is empty.
      auto last_tile = [&](int jj) { return (jj < nk[1]) ? 1 : 0; };
      // prologue: S_t(0)
      if (ok && nkv > 0) {
        ok = wait_full(0);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t) {
            if (nk[t] == 0) continue;
            issue_s<D>(tmem + C::kTmS0 + t * 128, q_smem[t], slot_smem(0));
            tc_commit(bar(C::kBarSFull + t));
          }
          tc_commit(bar(C::kBarKVEmpty + 0));
        }
      }
      bool have_v = false, have_k = false;
      for (int j = 0; j < nkv && ok; ++j) {
        const int seqK = 2 * j, seqV = 2 * j + 1;
        have_v = false;
        have_k = false;
        for (int t = 0; t < 2; ++t) {
          if (j >= nk[t]) continue;
          if (!mbar_wait(bar(C::kBarPFull + t), j & 1, wd)) { ok = false; break; }
          if (!have_v) {
            if (!wait_full(seqV)) { ok = false; break; }
            have_v = true;
          }
          tc_fence_after();
          const uint32_t tm_s = tmem + C::kTmS0 + t * 128;
          issue_pv<D>(tmem + C::kTmO0 + t * D, tm_s, slot_smem(seqV), j > 0);
          if (t == last_tile(j)) tc_commit(bar(C::kBarKVEmpty + seqV % C::kSlots));
          if (j + 1 < nk[t]) {
            if (!have_k) {
              if (!wait_full(seqK + 2)) { ok = false; break; }
              have_k = true;
              tc_fence_after();
            }
            issue_s<D>(tm_s, q_smem[t], slot_smem(seqK + 2));
            tc_commit(bar(C::kBarSFull + t));
            if (t == last_tile(j + 1)) tc_commit(bar(C::kBarKVEmpty + (seqK + 2) % C::kSlots));
          } else {
            tc_commit(bar(C::kBarOFull + t));
          }
        }
      }
      // No MMA may be in flight when TMEM is released.
      tc_commit(bar(C::kBarDrain));
      drain_wait(bar(C::kBarDrain), 0, p.timeout_ns);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row_in_tile = wq * 32 + lane;
    const int r0 = q0 + t * BM;
    const int row = r0 + row_in_tile;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tm_s = tmem + lane_off + C::kTmS0 + t * 128;
    const uint32_t tm_o = tmem + lane_off + C::kTmO0 + t * D;
    const float c = p.scale_log2;
    float m_ref = -INFINITY;
    float l = 0.0f;
    bool ok = nk[t] > 0;
    for (int j = 0; j < nk[t] && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + t), j & 1, wd));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld32(tm_s + cc * 32, s[cc]);
      tmem_wait_ld();
      const int kv0 = j * BN;
      const bool need_mask = (p.causal && kv0 + BN - 1 > r0) || (kv0 + BN > p.N);
      if (need_mask) {
        const int lim = p.causal ? min(row + 1, p.N) : p.N;  // first masked column
#pragma unroll
        for (int k = 0; k < 128; ++k)
          if (kv0 + k >= lim) s[k / 32][k % 32] = __float_as_uint(-INFINITY);
      }
      // row max: per 32-column chunk a tree of three-input maxima (short dependency
      // chains, few live temporaries), then across the four chunks
      float cm[4];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float t1[11];
#pragma unroll
        for (int q = 0; q < 10; ++q)
          t1[q] = fmax3(__uint_as_float(s[cc][3 * q]), __uint_as_float(s[cc][3 * q + 1]),
                        __uint_as_float(s[cc][3 * q + 2]));
        t1[10] = fmaxf(__uint_as_float(s[cc][30]), __uint_as_float(s[cc][31]));
        const float a = fmax3(t1[0], t1[1], t1[2]), b = fmax3(t1[3], t1[4], t1[5]);
        const float d2 = fmax3(t1[6], t1[7], t1[8]), e = fmaxf(t1[9], t1[10]);
        cm[cc] = fmax3(a, b, fmaxf(d2, e));
      }
      const float mx = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3]));
      const float m_new = fmaxf(m_ref, mx * c);
      const bool need = m_new > m_ref + kRescaleThreshold;
      // The reference max moves for the whole warp when any row needs it (TMEM
      // accesses are warp-wide); O is rescaled below, after the scores are dead.
      const bool move = __any_sync(0xffffffffu, need);
      float alpha = 1.0f;
      if (move) {
        alpha = (m_ref == -INFINITY) ? 0.0f : ex2_approx(m_ref - m_new);
        m_ref = m_new;
        l *= alpha;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_use, -m_use);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 x = ffma2(make_float2(__uint_as_float(s[cc][2 * k]),
                                             __uint_as_float(s[cc][2 * k + 1])), c2, nm2);
          float2 pe;
          if (kPolyPeriod > 0 && k % (kPolyPeriod > 0 ? kPolyPeriod : 1) == kPolyPeriod - 1) {
            pe = exp2_poly2(x);  // a share of the exponentials on the FMA pipe
          } else {
            pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
          }
          acc[k & 3] = fadd2(acc[k & 3], pe);
          pk[k] = pack_bf16x2(pe.x, pe.y);
        }
        tmem_st16(tm_s + cc * 16, pk);
      }
      const float rowsum = (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y) +
                           (acc[2].x + acc[2].y) + (acc[3].x + acc[3].y);
      l += rowsum;
      if (move && j > 0) {
        // O_t holds the sum up to tile j-1 (PV_t(j-1) completed before S_t(j)'s
        // commit fired); bring it to the new reference max before PV_t(j).
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tm_o + cc * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(tm_o + cc * 32, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarPFull + t));
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarOFull + t), 0, wd));
    if (ok) {
      tc_fence_after();
      const float inv_l = (l > 0.0f) ? 1.0f / l : 0.0f;
      __nv_bfloat16* orow = p.O + (static_cast<size_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tm_o + cc * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pk[k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
        if (row < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
        }
      }
      if (row < p.N)
        p.LSE[static_cast<size_t>(bh) * p.N + row] =
            (l > 0.0f) ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

}  // namespace fwd
}  // namespace fa
