// fa_fwd_sm100.cuh -- fused attention forward for sm_100a (bf16 or f16 in, fp32
// accumulate; the element type is the template parameter E).
//
// Method: the blockwise forward of "FlashAttention optimisation: breaking the
// performance bottleneck of standard attention", section 4.1 (for each query
// block, stream the key/value blocks, update the running max m and sum l, rescale
// the partial output, divide by l at the end, write O and the normaliser once),
// with the online-softmax merge of "A survey of key techniques of large language
// model pre-training systems" (Journal of Software 2026(1), p.218: m = max(m1,
// m2), l = e^(m1-m) l1 + e^(m2-m) l2). Causal tiles above the diagonal are skipped
// ("Flash Attention-2: acceleration principle ...", causal-mask item), and so are
// tiles outside a sliding window (the same item's sliding-window example) or
// outside a 128 x 128 block mask (block-sparse FlashAttention, "FlashAttention
// optimisation ...", section 7). Key j is seen by query i iff
//   j < N, i - wl <= j (wl >= 0), j <= i + wr (wr >= 0; causal is wr = 0), and the
//   block mask keeps (i / 128, j / 128);
// the CTA walks only the key tiles that some of its query rows can see.
//
// B200 mapping (one CTA per SM, 352 threads):
//   * CTA = 2 query tiles of 128 rows (256 rows) of one (batch, head), or one; the two
//     tiles share every K/V tile that is loaded. (fa_fwd_persistent_kernel, at the
//     end of this file, walks a list of such items per CTA.)
//   * warp 8: TMA producer for the Q tiles (once) and the K tiles (128 rows) through
//     a ring of kKSlots shared-memory slots; warp 10: TMA producer for the V tiles
//     (ring of kVSlots). Separate rings let K run further ahead of the MMAs than V.
//   * warp 9: MMA issuer (one thread), per key tile j:
//       S_t(j+1) = Q_t K_{j+1}^T (tcgen05.mma, fp32 into TMEM columns [128t, 128t+128))
//       as soon as the softmax of tile t has read S_t(j) out of TMEM; then
//       O_t += P_t(j) V_j with P_t read from shared memory once it is written.
//     So the tensor cores compute S for the next key tile while the softmax of the
//     current one is still running.
//   * warps 0-3 / 4-7: softmax of tile 0 / 1, one thread per query row (TMEM lane):
//     read S with tcgen05.ld, row max (thread-local), p = 2^(s*c - m) with
//     c = scale*log2(e) folded into one FFMA before ex2, row sum in registers, P
//     rounded to bf16 into a 128-byte-swizzled shared tile (the K-major A operand of
//     the PV MMA). O is rescaled in TMEM only when the running max grew by more than
//     2^8 (exact: O and l always share the same reference max).
//   * TMEM: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D).
//   * Epilogue: O/l rounded to bf16 stored row per thread; LSE = (m + log2 l) ln 2.
#pragma once

#include "fa_ptx.cuh"

namespace fa {
namespace fwd {

constexpr int BM = 128;        // query rows per tile
constexpr int BN = 128;        // key/value rows per tile
constexpr int kThreads = 352;  // 8 softmax warps, K/Q producer, MMA, V producer
constexpr int kWarpTmaK = 8;
constexpr int kWarpMma = 9;
constexpr int kWarpTmaV = 10;
constexpr float kRescaleThreshold = 8.0f;  // log2 domain: rescale when max grows > 2^8
// Largest number of 128-key tiles a block mask may span (N <= 524288).
constexpr int kMaxMaskTiles = 4096;
// When Cfg<D>::kPolyPeriod > 0, one pair of exponentials in every kPolyPeriod goes
// to the polynomial exp2 on the FMA pipe (exp2_poly2) instead of MUFU. The build
// may set the periods with -DFA_FWD_POLY_PERIOD_D64=... / _D128=... (0 = off).
#ifndef FA_FWD_POLY_PERIOD_D64
#define FA_FWD_POLY_PERIOD_D64 0
#endif
#ifndef FA_FWD_POLY_PERIOD_D128
#define FA_FWD_POLY_PERIOD_D128 0
#endif

template <int D>
struct Cfg {
  static constexpr int kChunkBytes = 128 * 128;      // 128 rows x 64 bf16 (one TMA box)
  static constexpr int kChunks = D / 64;             // boxes per 128 x D tile
  static constexpr int kTileBytes = kChunks * kChunkBytes;
  static constexpr int kPBytes = 2 * kChunkBytes;    // P: 128 x 128 bf16
  static constexpr int kKSlots = (D == 128) ? 2 : 3;
  static constexpr int kVSlots = (D == 128) ? 1 : 3;
  static constexpr int kQOff = 0;
  static constexpr int kPOff = 2 * kTileBytes;
  static constexpr int kKOff = kPOff + 2 * kPBytes;
  static constexpr int kVOff = kKOff + kKSlots * kTileBytes;
  static constexpr int kBarOff = kVOff + kVSlots * kTileBytes;
  static constexpr int kBarQFull = 0;                             // [2]
  static constexpr int kBarKFull = 2;                             // [kKSlots]
  static constexpr int kBarKEmpty = kBarKFull + kKSlots;          // [kKSlots]
  static constexpr int kBarVFull = kBarKEmpty + kKSlots;          // [kVSlots]
  static constexpr int kBarVEmpty = kBarVFull + kVSlots;          // [kVSlots]
  static constexpr int kBarSFull = kBarVEmpty + kVSlots;          // [2] S_t(j) in TMEM
  static constexpr int kBarSFree = kBarSFull + 2;                 // [2] S_t(j) read out
  static constexpr int kBarPFull = kBarSFree + 2;                 // [2] P_t(j) written
  static constexpr int kBarPVDone = kBarPFull + 2;                // [2] PV_t(j) complete
  static constexpr int kBarQEmpty = kBarPVDone + 2;               // [2] item's S_t done with Q_t
  static constexpr int kBarOFree = kBarQEmpty + 2;                // [2] item's O_t read out
  static constexpr int kBarDrain = kBarOFree + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem base, abort flag
  static constexpr int kMaskOff = kMiscOff + 16;            // block-mask bits of both tiles
  static constexpr int kMaskWords = kMaxMaskTiles / 32;     // per query tile
  static constexpr int kSmemBytes = kMaskOff + 2 * kMaskWords * 4 + 1024;  // + alignment
  static constexpr uint32_t kTmS0 = 0, kTmO0 = 256;
  static_assert(kSmemBytes <= 232448, "exceeds the 227 KB of shared memory a CTA may use");
  static constexpr uint32_t kTmCols = 512;
  static constexpr int kPolyPeriod = (D == 64) ? FA_FWD_POLY_PERIOD_D64 : FA_FWD_POLY_PERIOD_D128;
};

struct Params {
  uint16_t* O;  // 16-bit elements (bf16 or f16, the kernel's element type)
  float* LSE;
  int N;
  int BH;
  // Work split: per head, pairs_ph items own two consecutive query tiles each (tiles
  // [singles_ph, n_qt)) and singles_ph items own one (tiles [0, singles_ph)). All pair
  // items (n_pair_items = BH * pairs_ph) come first in the list, heaviest first within
  // a head, so the single-tile items (half the work) come last and even out the CTAs'
  // loads. weight_major = 0: the list is head-major (a head's items are consecutive,
  // so the CTAs busy at one time share one or two heads' K/V in L2); 1: rank-major
  // (every head's heaviest item, then every head's second, ...), for causal or
  // windowed launches whose K/V all fit in L2.
  int pairs_ph;
  int singles_ph;
  int n_pair_items;
  int n_items;
  int weight_major;
  float scale_log2;  // scale * log2(e)
  int wl;            // keys j >= i - wl are kept; < 0: no left bound
  int wr;            // keys j <= i + wr are kept; < 0: no right bound (causal: 0)
  const uint8_t* blocks;  // [n_kt x n_kt] block mask (nonzero = kept), or null
  int n_kt;               // ceil(N / 128)
  DropoutParams drop;     // used by the kDropout instances only
  unsigned long long timeout_ns;
};

// S = Q_t K_j^T: M = 128 query rows, N = 128 keys, K = D; both operands K-major.
// Per 64-column chunk, four K = 16 steps 32 bytes apart (2 descriptor units); the
// chunks are kChunkBytes (1024 units) apart.
template <int D, Elt E>
__device__ __forceinline__ void issue_s(uint32_t tm_d, uint32_t q_smem, uint32_t k_smem) {
  constexpr uint32_t idesc = idesc_f32acc<E>(BM, BN, 0, 0);
  constexpr uint64_t kChunk = Cfg<D>::kChunkBytes >> 4;
  const uint64_t qa = sdesc_sw128(q_smem, 16, 1024), kb = sdesc_sw128(k_smem, 16, 1024);
#pragma unroll
  for (int c = 0; c < D / 64; ++c)
    mma_ss_x4<2, 2>(tm_d, qa + c * kChunk, kb + c * kChunk, idesc, c > 0 ? 1u : 0u);
}

// O += P V_j: A = P (128 x 128 keys, K-major in shared memory), B = V_j read MN-major:
// K = 16 keys step 16 rows x 128 bytes (128 descriptor units) down V, 32 bytes along P.
template <int D, Elt E>
__device__ __forceinline__ void issue_pv(uint32_t tm_o, uint32_t p_smem, uint32_t v_smem,
                                         bool accumulate) {
  constexpr uint32_t idesc = idesc_f32acc<E>(BM, D, 0, 1);
  constexpr uint64_t kChunk = Cfg<D>::kChunkBytes >> 4;
  const uint64_t pa = sdesc_sw128(p_smem, 16, 1024);
  const uint64_t vb = sdesc_sw128(v_smem, Cfg<D>::kChunkBytes, 1024);
  mma_ss_x4<2, 128>(tm_o, pa, vb, idesc, accumulate ? 1u : 0u);
  mma_ss_x4<2, 128>(tm_o, pa + kChunk, vb + 4 * 128, idesc, 1u);
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

// The softmax work of one key tile for one query row (this thread, TMEM lane
// row_in_tile of query tile t), once S_t has landed in TMEM: read S_t and release its
// columns (SFree); mask the elements outside the row's visible keys [k_lo, k_hi) on
// tiles that cross an edge; take the row max and move the reference max m_ref when it
// grew by more than 2^8 (rescaling l, lr and, after the previous PV_t, O_t); p = 2^(s*c
// - m_ref), their sum l and, rounded to 16 bits, P_t into the swizzled shared tile (with
// dropout applied after the sum); then PFull. n counts this tile's S and PV products
// before this one (their barrier phases); first: no PV_t of the item yet. Returns false
// if a bounded wait gave up.
template <int D, Elt E, bool kDropout>
__device__ __forceinline__ bool softmax_key_tile(const Params& p, const Watchdog& wd,
                                                 uint32_t tm_s, uint32_t tm_o, uint8_t* p_row,
                                                 uint32_t bar_sfree, uint32_t bar_pvdone,
                                                 uint32_t bar_pfull, int n, bool first, int kt,
                                                 int r0, int row, int row_in_tile, int wl,
                                                 int wr, uint32_t ctr_head, int lane,
                                                 int wq, int t, float& m_ref, float& l,
                                                 float& lr) {
  using C = Cfg<D>;
  const float c = p.scale_log2;
  const int r1 = r0 + BM - 1;
  // visible keys of this row: [k_lo, k_hi)
  const int k_lo = (wl < 0) ? 0 : row - wl;
  const int k_hi = (wr < 0) ? p.N : min(p.N, row + wr + 1);
  tc_fence_after();
  uint32_t s[4][32];
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) tmem_ld32(tm_s + cc * 32, s[cc]);
  tmem_wait_ld();
  // S_t is in registers: the MMA may overwrite it with the next S_t now
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_sfree);
  if (wq == 0) FA_TRACE_POINT(52, n, t);
  const int kv0 = kt * BN;
  // masking only where the tile crosses an edge of some row's visible range
  const bool need_mask = (kv0 + BN > p.N) || (wr >= 0 && kv0 + BN - 1 > r0 + wr) ||
                         (wl >= 0 && kv0 < r1 - wl);
  if (need_mask) {
    // key kv0 + k is visible iff 0 <= kv0 + k - k_lo < k_hi - k_lo
    const int off = kv0 - k_lo;
    const unsigned span = static_cast<unsigned>(max(k_hi - k_lo, 0));
#pragma unroll
    for (int k = 0; k < 128; ++k)
      if (static_cast<unsigned>(off + k) >= span) s[k / 32][k % 32] = __float_as_uint(-INFINITY);
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
    lr *= alpha;
  }
  // the previous PV_t must be complete before P_t is overwritten and O_t rescaled
  if (!first) {
    if (wq == 0) FA_TRACE_POINT(53, n, t);
    const bool ok = __all_sync(0xffffffffu, mbar_wait(bar_pvdone, (n - 1) & 1, wd));
    if (wq == 0) FA_TRACE_POINT(54, n, t);
    if (!ok) return false;
    tc_fence_after();
  }
  const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
  const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_use, -m_use);
  float2 accr[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                   make_float2(0.f, 0.f)};
  // dropout: this row's four words for the current 16 keys (byte b of word m is key
  // 4m + b of the group)
  [[maybe_unused]] uint32_t zw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int cc = 0; cc < 4; ++cc) {
    uint32_t pk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float2 x = ffma2(make_float2(__uint_as_float(s[cc][2 * k]),
                                         __uint_as_float(s[cc][2 * k + 1])), c2, nm2);
      float2 pe;
      constexpr int kPoly = C::kPolyPeriod;
      if (kPoly > 0 && k % (kPoly > 0 ? kPoly : 1) == kPoly - 1) {
        pe = exp2_poly2(x);  // a share of the exponentials on the FMA pipe
      } else {
        pe = make_float2(ex2_approx(x.x), ex2_approx(x.y));
      }
      acc[k & 3] = fadd2(acc[k & 3], pe);  // l is the sum before dropout
      if constexpr (kDropout) {
        // One block covers 4 rows x 4 keys; the lanes of rows 4g..4g+3 share its
        // counter. Every 16 keys, lane u (row mod 4) draws the block of keys
        // 4u..4u+3 of the 16, and a 4 x 4 transpose across the four lanes hands
        // each lane its own row's word of all four blocks.
        if ((k & 7) == 0) {
          const int u = lane & 3;
          const uint4 w = philox4x32_10(
              make_uint4(static_cast<uint32_t>(((kv0 + 32 * cc + 2 * k) >> 2) + u),
                         static_cast<uint32_t>(row >> 2), ctr_head, p.drop.offset),
              p.drop.seed_lo, p.drop.seed_hi);
          zw[0] = w.x;
          zw[1] = w.y;
          zw[2] = w.z;
          zw[3] = w.w;
          transpose4_lanes(zw, u);
        }
        // keys 2k, 2k + 1 of the chunk = keys 2(k mod 8), +1 of the group: word
        // (k mod 8) / 2, bytes 2(k mod 2) and 2(k mod 2) + 1
        const uint32_t wd = zw[(k & 7) >> 1] >> (16 * (k & 1));
        pe.x = ((wd & 0xffu) >= p.drop.threshold) ? pe.x * p.drop.scale : 0.0f;
        pe.y = (((wd >> 8) & 0xffu) >= p.drop.threshold) ? pe.y * p.drop.scale : 0.0f;
      }
      pk[k] = pack2<E>(pe.x, pe.y);
      if constexpr (!kDropout) accr[k & 1] = fadd2(accr[k & 1], unpack2<E>(pk[k]));
    }
    // keys 32cc..32cc+31 = 16-byte units 4cc..4cc+3 of this row's 256 bytes:
    // chunk (cc / 2), units (cc % 2) * 4 + u, 128-byte swizzle by the row
    uint8_t* chunk = p_row + (cc >> 1) * C::kChunkBytes;
#pragma unroll
    for (int u = 0; u < 4; ++u)
      *reinterpret_cast<uint4*>(chunk + ((((cc & 1) * 4 + u) ^ (row_in_tile & 7)) * 16)) =
          make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
  }
  l += (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y) + (acc[2].x + acc[2].y) +
       (acc[3].x + acc[3].y);
  lr += (accr[0].x + accr[0].y) + (accr[1].x + accr[1].y);
  if (move && !first) {
    // bring the sum up to the previous key tile to the new reference max before this PV_t
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t o[32];
      tmem_ld32(tm_o + cc * 32, o);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
      tmem_st32(tm_o + cc * 32, o);
    }
    tmem_wait_st();
  }
  fence_proxy_async_smem();  // P (generic stores) before the MMA reads it
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_pfull);
  if (wq == 0) FA_TRACE_POINT(55, n, t);
  return true;
}

template <int D, Elt E, bool kMasked, bool kDropout = false>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
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
  // Without a window's left bound or a block mask (kMasked = false) those are
  // compile-time constants, so the general tile walk folds to the plain / causal one.
  const int wl = kMasked ? p.wl : -1;
  const int wr = p.wr;
  const uint8_t* const blocks = kMasked ? p.blocks : nullptr;

  // Work item: head-major, so that the CTAs resident at any time cover about two
  // heads and their K/V stay in L2; within a head the heaviest query tiles (causal)
  // go first. Single-tile CTAs, on the lightest tiles, come after all pairs.
  int bh, qt0;
  bool own1;  // does this CTA own query tile 1 (qt0 + 1)?
  // (weight_major: rank-major instead, every head's heaviest pair first)
  if (static_cast<int>(blockIdx.x) < p.n_pair_items) {
    const int c = static_cast<int>(blockIdx.x);
    const int r = p.weight_major ? c / p.BH : c % p.pairs_ph;
    bh = p.weight_major ? c % p.BH : c / p.pairs_ph;
    qt0 = p.singles_ph + 2 * (p.pairs_ph - 1 - r);
    own1 = true;
  } else {
    const int c = static_cast<int>(blockIdx.x) - p.n_pair_items;
    const int r = p.weight_major ? c / p.BH : c % p.singles_ph;
    bh = p.weight_major ? c % p.BH : c / p.singles_ph;
    qt0 = p.singles_ph - 1 - r;
    own1 = false;
  }
  const int q0 = qt0 * BM;
  const int n_kt = p.n_kt;
  // key tiles [lo[t], hi[t]) hold every key a row of query tile t may see
  int lo[2], hi[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int r0 = q0 + t * BM, r1 = min(r0 + BM, p.N) - 1;
    lo[t] = (wl < 0) ? 0 : max(0, r0 - wl) / BN;
    hi[t] = (wr < 0) ? n_kt : min(n_kt, (r1 + wr) / BN + 1);
    if (r0 >= p.N || (t == 1 && !own1)) lo[t] = hi[t] = 0;
  }
  // The CTA's key tiles: the union of both ranges (contiguous: lo[1] <= hi[0]).
  const int kt_lo = (hi[0] > lo[0]) ? lo[0] : lo[1];
  const int kt_hi = max(hi[0], hi[1]);

  // Block mask rows of the two query tiles as bits in shared memory: warp w builds
  // words w, w + 11, ... with one byte per lane and a ballot.
  uint32_t* mask_bits = reinterpret_cast<uint32_t*>(base_ptr + C::kMaskOff);
  if (blocks != nullptr) pdl_wait();  // the mask may come from the grid before
  if (blocks != nullptr) {
    const int nwords = (n_kt + 31) / 32;
    for (int w = warp; w < 2 * nwords; w += kThreads / 32) {
      const int t = w / nwords, wi = w % nwords;
      const int qt = min(qt0 + t, n_kt - 1);
      const int kt = wi * 32 + lane;
      const bool keep = kt < n_kt && blocks[static_cast<size_t>(qt) * n_kt + kt] != 0;
      const uint32_t bits = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) mask_bits[t * C::kMaskWords + wi] = bits;
    }
  }

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::kBarQFull + t), 1);
      mbar_init(bar(C::kBarSFull + t), 1);
      mbar_init(bar(C::kBarSFree + t), 4);  // one arrival per softmax warp
      mbar_init(bar(C::kBarPFull + t), 4);
      mbar_init(bar(C::kBarPVDone + t), 1);
    }
    for (int s = 0; s < C::kKSlots; ++s) {
      mbar_init(bar(C::kBarKFull + s), 1);
      mbar_init(bar(C::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < C::kVSlots; ++s) {
      mbar_init(bar(C::kBarVFull + s), 1);
      mbar_init(bar(C::kBarVEmpty + s), 1);
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
  pdl_wait();  // the grid before this one has completed: global memory is ours
  const Watchdog wd{abort_flag, p.timeout_ns};
  if (threadIdx.x == 0) FA_TRACE_CTA(1);

  // Does query tile t see any key of key tile kt?
  auto member = [&](int kt, int t) -> bool {
    if (kt < lo[t] || kt >= hi[t]) return false;
    return blocks == nullptr || ((mask_bits[t * C::kMaskWords + (kt >> 5)] >> (kt & 31)) & 1u);
  };
  // first key tile >= kt that either query tile sees (kt_hi if none)
  auto next_kt = [&](int kt) -> int {
    while (kt < kt_hi && !(member(kt, 0) || member(kt, 1))) ++kt;
    return kt;
  };
  int nk[2];  // key tiles each query tile sees
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    if (blocks == nullptr) {
      nk[t] = hi[t] - lo[t];
    } else {
      nk[t] = 0;
      for (int kt = lo[t]; kt < hi[t]; ++kt) nk[t] += member(kt, t) ? 1 : 0;
    }
  }

  auto k_smem = [&](int j) -> uint32_t {
    return base + C::kKOff + (j % C::kKSlots) * C::kTileBytes;
  };
  auto v_smem = [&](int j) -> uint32_t {
    return base + C::kVOff + (j % C::kVSlots) * C::kTileBytes;
  };

  if (warp == kWarpTmaK || warp == kWarpTmaV) {
    // ------------------------------------------------------------ producers
    // (the whole warp runs the loop; one elected lane issues each copy)
    const bool is_k = (warp == kWarpTmaK);
    const CUtensorMap* map = is_k ? &tmK : &tmV;
    const int nslots = is_k ? C::kKSlots : C::kVSlots;
    const int bfull = is_k ? C::kBarKFull : C::kBarVFull;
    const int bempty = is_k ? C::kBarKEmpty : C::kBarVEmpty;
    if (lane == 0) tma_prefetch_desc(map);
    if (is_k) {
      if (lane == 0) tma_prefetch_desc(&tmQ);
      for (int t = 0; t < 2; ++t) {
        if (nk[t] == 0) continue;
        const uint32_t dst = base + C::kQOff + t * C::kTileBytes;
        mbar_arrive_expect_tx_e(bar(C::kBarQFull + t), C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d_e(dst + c * C::kChunkBytes, &tmQ, bar(C::kBarQFull + t), c * 64,
                        q0 + t * BM, bh);
      }
    }
    int issued = 0;  // ring index: the issued-th key tile the CTA walks
    for (int kt = next_kt(kt_lo); kt < kt_hi; kt = next_kt(kt + 1)) {
      const int j = issued;
      const int slot = j % nslots, rnd = j / nslots;
      FA_TRACE_POINT(40, j, is_k ? 0 : 1);
      if (rnd > 0 && !mbar_wait_warp(bar(bempty + slot), (rnd - 1) & 1, wd)) break;
      FA_TRACE_POINT(41, j, is_k ? 0 : 1);
      const uint32_t dst = is_k ? k_smem(j) : v_smem(j);
      mbar_arrive_expect_tx_e(bar(bfull + slot), C::kTileBytes);
      for (int c = 0; c < C::kChunks; ++c)
        tma_load_3d_e(dst + c * C::kChunkBytes, map, bar(bfull + slot), c * 64, kt * BN, bh);
      issued = j + 1;
    }
    // Every issued copy must land before the CTA may exit.
    for (int j = max(0, issued - nslots); j < issued; ++j)
      drain_wait(bar(bfull + j % nslots), (j / nslots) & 1, p.timeout_ns);
    if (is_k)
      for (int t = 0; t < 2; ++t)
        if (nk[t] > 0) drain_wait(bar(C::kBarQFull + t), 0, p.timeout_ns);
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // (the whole warp runs the loop; one elected lane issues each MMA and commit)
    FA_TRACE_POINT(0, 0, 0);
    bool ok = true;
    for (int t = 0; t < 2 && ok; ++t)
      if (nk[t] > 0) ok = mbar_wait_warp(bar(C::kBarQFull + t), 0, wd);
    const uint32_t q_smem0 = base + C::kQOff, q_smem1 = base + C::kQOff + C::kTileBytes;
    const uint32_t p_smem0 = base + C::kPOff, p_smem1 = base + C::kPOff + C::kPBytes;
    auto wait_k = [&](int j) {
      return mbar_wait_warp(bar(C::kBarKFull + j % C::kKSlots), (j / C::kKSlots) & 1, wd);
    };
    auto wait_v = [&](int j) {
      return mbar_wait_warp(bar(C::kBarVFull + j % C::kVSlots), (j / C::kVSlots) & 1, wd);
    };
    // ns[t] / npv[t]: S_t and PV_t products issued so far (their barrier phases)
    int ns[2] = {0, 0}, npv[2] = {0, 0};
    // S_t for the key tile at ring index j, for each query tile that sees it, each
    // as soon as the softmax of that tile has read its previous S out of TMEM
    auto issue_s_all = [&](int kt, int j) -> bool {
      bool have_k = false;
      for (int t = 0; t < 2; ++t) {
        if (!member(kt, t)) continue;
        FA_TRACE_POINT(42, ns[t], t);
        if (ns[t] > 0 && !mbar_wait_warp(bar(C::kBarSFree + t), (ns[t] - 1) & 1, wd))
          return false;
        FA_TRACE_POINT(43, ns[t], t);
        if (!have_k) {
          if (!wait_k(j)) return false;
          FA_TRACE_POINT(44, j, 0);
          have_k = true;
        }
        tc_fence_after();
        issue_s<D, E>(tmem + C::kTmS0 + t * 128, t ? q_smem1 : q_smem0, k_smem(j));
        tc_commit_e(bar(C::kBarSFull + t));
        FA_TRACE_POINT(45, ns[t], t);
        ++ns[t];
      }
      tc_commit_e(bar(C::kBarKEmpty + j % C::kKSlots));
      return true;
    };
    int cur = next_kt(kt_lo);
    if (ok && cur < kt_hi) ok = issue_s_all(cur, 0);
    for (int j = 0; cur < kt_hi && ok; ++j) {
      // S for the next key tile before PV of this one
      const int nxt = next_kt(cur + 1);
      if (nxt < kt_hi && !issue_s_all(nxt, j + 1)) { ok = false; break; }
      // O_t += P_t V_cur
      bool have_v = false;
      for (int t = 0; t < 2 && ok; ++t) {
        if (!member(cur, t)) continue;
        FA_TRACE_POINT(46, npv[t], t);
        if (!mbar_wait_warp(bar(C::kBarPFull + t), npv[t] & 1, wd)) { ok = false; break; }
        FA_TRACE_POINT(47, npv[t], t);
        if (!have_v) {
          if (!wait_v(j)) { ok = false; break; }
          FA_TRACE_POINT(48, j, 0);
          have_v = true;
        }
        tc_fence_after();
        issue_pv<D, E>(tmem + C::kTmO0 + t * D, t ? p_smem1 : p_smem0, v_smem(j), npv[t] > 0);
        tc_commit_e(bar(C::kBarPVDone + t));
        FA_TRACE_POINT(49, npv[t], t);
        ++npv[t];
      }
      if (!ok) break;
      tc_commit_e(bar(C::kBarVEmpty + j % C::kVSlots));
      cur = nxt;
    }
    // No MMA may be in flight when TMEM is released.
    tc_commit_e(bar(C::kBarDrain));
    drain_wait(bar(C::kBarDrain), 0, p.timeout_ns);
    __syncwarp();
    FA_TRACE_POINT(99, 0, 0);
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
    uint8_t* p_row = base_ptr + C::kPOff + t * C::kPBytes + row_in_tile * 128;
    float m_ref = -INFINITY;
    float l = 0.0f;
    // lr: the same sum over P as rounded for the PV product. O is divided by lr, so
    // the weights it applies to V sum to exactly 1: the rounding of the largest
    // p (up to 2^8 under the lagging reference max, so up to 2^-8 relative) then
    // cancels instead of showing in O. LSE keeps the unrounded l. With dropout the
    // rounded values carry the keep mask, so there O is divided by l.
    float lr = 0.0f;
    // this tile's range, count and mask bits as scalars (no per-thread array indexing)
    const int t_lo = t ? lo[1] : lo[0], t_hi = t ? hi[1] : hi[0];
    const int t_nk = t ? nk[1] : nk[0];
    const uint32_t* t_bits = mask_bits + t * C::kMaskWords;
    auto t_member = [&](int kt) -> bool {
      if (kt < t_lo || kt >= t_hi) return false;
      return blocks == nullptr || ((t_bits[kt >> 5] >> (kt & 31)) & 1u);
    };
    // the dropout counter's head word: the call's head_base + the flattened head
    const uint32_t ctr_head = p.drop.head_base + static_cast<uint32_t>(bh);
    bool ok = t_nk > 0;
    int kt = t_lo - 1;
    for (int j = 0; j < t_nk && ok; ++j) {
      do ++kt; while (!t_member(kt));
      if (wq == 0) FA_TRACE_POINT(50, j, t);
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + t), j & 1, wd));
      if (wq == 0) FA_TRACE_POINT(51, j, t);
      if (j == 0 && t == 0 && threadIdx.x == 0) FA_TRACE_CTA(2);
      if (!ok) break;
      if (!softmax_key_tile<D, E, kDropout>(p, wd, tm_s, tm_o, p_row, bar(C::kBarSFree + t),
                                            bar(C::kBarPVDone + t), bar(C::kBarPFull + t), j,
                                            j == 0, kt, r0, row, row_in_tile, wl,
                                            wr, ctr_head, lane, wq, t, m_ref, l, lr)) {
        ok = false;
        break;
      }
    }
    if (ok && t_nk > 0)
      ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarPVDone + t), (t_nk - 1) & 1, wd));
    if (t_nk == 0 && row < p.N && (t == 0 || own1)) {
      // a query tile that sees no key: O = 0, LSE = -inf
      uint4* dst = reinterpret_cast<uint4*>(p.O + (static_cast<size_t>(bh) * p.N + row) * D);
#pragma unroll
      for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
      p.LSE[static_cast<size_t>(bh) * p.N + row] = -INFINITY;
    }
    if (ok && t_nk > 0) {
      if (t == 0 && threadIdx.x == 0) FA_TRACE_CTA(3);
      tc_fence_after();
      const float norm = kDropout ? l : lr;
      const float inv_l = (norm > 0.0f) ? 1.0f / norm : 0.0f;
      uint16_t* orow = p.O + (static_cast<size_t>(bh) * p.N + row) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tm_o + cc * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          pk[k] = pack2<E>(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
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
  if (threadIdx.x == 0) FA_TRACE_CTA(4);
  pdl_launch_dependents();  // the next grid may launch: this CTA's work is done
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmCols);
  }
}

// The persistent form of the kernel above, for launches of many short items (few key
// tiles each): min(items, SMs) CTAs, each walking a list of items and reusing its
// buffers from one to the next (Q once the item's last S product has read it, O in
// TMEM once the epilogue has read it out), so one item's epilogue overlaps the next
// item's first loads and products. The same roles, barriers and arithmetic; no block
// mask (its CTA would build the mask rows of every item it walks).
template <int D, Elt E, bool kMasked, bool kDropout>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const Params p) {
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
  // Without a window's left bound (kMasked = false) it is a compile-time constant, so
  // the general tile walk folds to the plain / causal one. Block masks never come here.
  const int wl = kMasked ? p.wl : -1;
  const int wr = p.wr;
  const int n_kt = p.n_kt;

  // Work items: item i < n_pair_items owns two consecutive query tiles, the others
  // one. Every role of the CTA walks the same items, the k-th being k * G + b for even
  // k and k * G + (G - 1 - b) for odd k (b = blockIdx.x, G = gridDim.x), so the heavy
  // items at the front of the list are dealt out back and forth over the CTAs and one
  // item's epilogue overlaps the next one's first loads and products.
  auto item_of = [&](int k) -> int {
    const int G = static_cast<int>(gridDim.x), b = static_cast<int>(blockIdx.x);
    const int i = k * G + ((k & 1) ? (G - 1 - b) : b);
    return i < p.n_items ? i : -1;
  };
  // An item's (batch, head), first query tile, whether it owns the second tile, the
  // key tiles [lo[t], hi[t]) each tile's rows may see and how many of them a tile
  // walks (nk), and the union [kt_lo, kt_hi) the CTA walks for it.
  struct Work {
    int bh, qt0, q0;
    bool own1;
    int lo[2], hi[2], nk[2];
    int kt_lo, kt_hi;
  };
  auto member_w = [&](const Work& w, int kt, int t) -> bool {
    return kt >= (t ? w.lo[1] : w.lo[0]) && kt < (t ? w.hi[1] : w.hi[0]);
  };
  auto decode = [&](int i, Work& w) {
    int r;
    if (i < p.n_pair_items) {
      if (p.weight_major) { r = i / p.BH; w.bh = i % p.BH; }
      else { w.bh = i / p.pairs_ph; r = i % p.pairs_ph; }
      w.qt0 = p.singles_ph + 2 * (p.pairs_ph - 1 - r);
      w.own1 = true;
    } else {
      const int c = i - p.n_pair_items;
      if (p.weight_major) { r = c / p.BH; w.bh = c % p.BH; }
      else { w.bh = c / p.singles_ph; r = c % p.singles_ph; }
      w.qt0 = p.singles_ph - 1 - r;
      w.own1 = false;
    }
    w.q0 = w.qt0 * BM;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int r0 = w.q0 + t * BM, r1 = min(r0 + BM, p.N) - 1;
      w.lo[t] = (wl < 0) ? 0 : max(0, r0 - wl) / BN;
      w.hi[t] = (wr < 0) ? n_kt : min(n_kt, (r1 + wr) / BN + 1);
      if (r0 >= p.N || (t == 1 && !w.own1)) w.lo[t] = w.hi[t] = 0;
    }
    // the union of both ranges (contiguous: lo[1] <= hi[0])
    w.kt_lo = (w.hi[0] > w.lo[0]) ? w.lo[0] : w.lo[1];
    w.kt_hi = max(w.hi[0], w.hi[1]);
#pragma unroll
    for (int t = 0; t < 2; ++t) w.nk[t] = w.hi[t] - w.lo[t];
  };

  if (threadIdx.x == 0) {
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar(C::kBarQFull + t), 1);
      mbar_init(bar(C::kBarQEmpty + t), 1);
      mbar_init(bar(C::kBarSFull + t), 1);
      mbar_init(bar(C::kBarSFree + t), 4);  // one arrival per softmax warp
      mbar_init(bar(C::kBarPFull + t), 4);
      mbar_init(bar(C::kBarPVDone + t), 1);
      mbar_init(bar(C::kBarOFree + t), 4);
    }
    for (int s = 0; s < C::kKSlots; ++s) {
      mbar_init(bar(C::kBarKFull + s), 1);
      mbar_init(bar(C::kBarKEmpty + s), 1);
    }
    for (int s = 0; s < C::kVSlots; ++s) {
      mbar_init(bar(C::kBarVFull + s), 1);
      mbar_init(bar(C::kBarVEmpty + s), 1);
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
  pdl_wait();  // the grid before this one has completed: global memory is ours
  const Watchdog wd{abort_flag, p.timeout_ns};
  if (threadIdx.x == 0) FA_TRACE_CTA(1);

  auto k_smem = [&](int g) -> uint32_t {
    return base + C::kKOff + (g % C::kKSlots) * C::kTileBytes;
  };
  auto v_smem = [&](int g) -> uint32_t {
    return base + C::kVOff + (g % C::kVSlots) * C::kTileBytes;
  };
  // first key tile >= kt that either query tile of the item sees (kt_hi if none)
  auto next_kt = [&](const Work& w, int kt) -> int {
    while (kt < w.kt_hi && !(member_w(w, kt, 0) || member_w(w, kt, 1))) ++kt;
    return kt;
  };

  if (warp == kWarpTmaK || warp == kWarpTmaV) {
    // ------------------------------------------------------------ producers
    // (the whole warp runs the loop; one elected lane issues each copy)
    // Warp 8 streams the K tiles of every item through its ring; warp 10 loads each
    // item's Q tiles (once the previous item's S products have read them: QEmpty)
    // and streams the V tiles. Ring indices run on across items.
    const bool is_k = (warp == kWarpTmaK);
    const CUtensorMap* map = is_k ? &tmK : &tmV;
    const int nslots = is_k ? C::kKSlots : C::kVSlots;
    const int bfull = is_k ? C::kBarKFull : C::kBarVFull;
    const int bempty = is_k ? C::kBarKEmpty : C::kBarVEmpty;
    if (lane == 0) tma_prefetch_desc(map);
    if (!is_k && lane == 0) tma_prefetch_desc(&tmQ);
    int issued = 0;       // ring index: tiles issued so far, over all items
    int nq[2] = {0, 0};   // Q tile loads so far (their barrier phases)
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = item_of(k);
      if (item < 0) break;
      Work w;
      decode(item, w);
      if (!is_k) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if ((t ? w.nk[1] : w.nk[0]) == 0) continue;
          const int n = t ? nq[1] : nq[0];
          if (n > 0 && !mbar_wait_warp(bar(C::kBarQEmpty + t), (n - 1) & 1, wd)) { ok = false; break; }
          const uint32_t dst = base + C::kQOff + t * C::kTileBytes;
          mbar_arrive_expect_tx_e(bar(C::kBarQFull + t), C::kTileBytes);
          for (int c = 0; c < C::kChunks; ++c)
            tma_load_3d_e(dst + c * C::kChunkBytes, &tmQ, bar(C::kBarQFull + t), c * 64,
                          w.q0 + t * BM, w.bh);
          if (t) ++nq[1]; else ++nq[0];
        }
        if (!ok) break;
      }
      for (int kt = next_kt(w, w.kt_lo); kt < w.kt_hi; kt = next_kt(w, kt + 1)) {
        const int g = issued;
        const int slot = g % nslots, rnd = g / nslots;
        FA_TRACE_POINT(40, g, is_k ? 0 : 1);
        if (rnd > 0 && !mbar_wait_warp(bar(bempty + slot), (rnd - 1) & 1, wd)) { ok = false; break; }
        FA_TRACE_POINT(41, g, is_k ? 0 : 1);
        const uint32_t dst = is_k ? k_smem(g) : v_smem(g);
        mbar_arrive_expect_tx_e(bar(bfull + slot), C::kTileBytes);
        for (int c = 0; c < C::kChunks; ++c)
          tma_load_3d_e(dst + c * C::kChunkBytes, map, bar(bfull + slot), c * 64, kt * BN, w.bh);
        issued = g + 1;
      }
    }
    // Every issued copy must land before the CTA may exit.
    for (int g = max(0, issued - nslots); g < issued; ++g)
      drain_wait(bar(bfull + g % nslots), (g / nslots) & 1, p.timeout_ns);
    // (warp 10 made every Q load: the last one's phase covers the earlier ones)
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int n = t ? nq[1] : nq[0];
      if (n > 0) drain_wait(bar(C::kBarQFull + t), (n - 1) & 1, p.timeout_ns);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    // (the whole warp runs the loop; one elected lane issues each MMA and commit)
    FA_TRACE_POINT(0, 0, 0);
    const uint32_t q_smem0 = base + C::kQOff, q_smem1 = base + C::kQOff + C::kTileBytes;
    const uint32_t p_smem0 = base + C::kPOff, p_smem1 = base + C::kPOff + C::kPBytes;
    auto wait_k = [&](int j) {
      return mbar_wait_warp(bar(C::kBarKFull + j % C::kKSlots), (j / C::kKSlots) & 1, wd);
    };
    auto wait_v = [&](int j) {
      return mbar_wait_warp(bar(C::kBarVFull + j % C::kVSlots), (j / C::kVSlots) & 1, wd);
    };
    // Counts over all items so far (their barrier phases): ns[t] / npv[t]: S_t and PV_t
    // products issued; nq[t]: Q_t tiles consumed; no[t]: items whose O_t the softmax has
    // read out. ns0 / npv0: ns / npv at the start of the current item.
    int ns[2] = {0, 0}, npv[2] = {0, 0}, nq[2] = {0, 0}, no[2] = {0, 0};
    int ns0[2] = {0, 0}, npv0[2] = {0, 0};
    Work w;
    auto member = [&](int kt, int t) -> bool { return member_w(w, kt, t); };
    // S_t for the key tile at ring index j, for each query tile that sees it, each
    // as soon as the softmax of that tile has read its previous S out of TMEM
    auto issue_s_all = [&](int kt, int j) -> bool {
      bool have_k = false;
      for (int t = 0; t < 2; ++t) {
        if (!member(kt, t)) continue;
        FA_TRACE_POINT(42, ns[t], t);
        if (ns[t] > 0 && !mbar_wait_warp(bar(C::kBarSFree + t), (ns[t] - 1) & 1, wd))
          return false;
        FA_TRACE_POINT(43, ns[t], t);
        if (!have_k) {
          if (!wait_k(j)) return false;
          FA_TRACE_POINT(44, j, 0);
          have_k = true;
        }
        tc_fence_after();
        issue_s<D, E>(tmem + C::kTmS0 + t * 128, t ? q_smem1 : q_smem0, k_smem(j));
        tc_commit_e(bar(C::kBarSFull + t));
        FA_TRACE_POINT(45, ns[t], t);
        ++ns[t];
        // after the item's last S_t its Q_t buffer may be refilled
        if (ns[t] - ns0[t] == w.nk[t]) tc_commit_e(bar(C::kBarQEmpty + t));
      }
      tc_commit_e(bar(C::kBarKEmpty + j % C::kKSlots));
      return true;
    };
    bool ok = true;
    int j = 0;  // ring index of the current key tile, over all items
    for (int k = 0; ok; ++k) {
      const int item = item_of(k);
      if (item < 0) break;
      decode(item, w);
      for (int t = 0; t < 2 && ok; ++t)
        if (w.nk[t] > 0) ok = mbar_wait_warp(bar(C::kBarQFull + t), nq[t]++ & 1, wd);
      if (!ok) break;
      FA_TRACE_POINT(58, k, 0);
      ns0[0] = ns[0];
      ns0[1] = ns[1];
      npv0[0] = npv[0];
      npv0[1] = npv[1];
      int cur = next_kt(w, w.kt_lo);
      if (cur < w.kt_hi) ok = issue_s_all(cur, j);
      for (; cur < w.kt_hi && ok; ++j) {
        // S for the next key tile before PV of this one
        const int nxt = next_kt(w, cur + 1);
        if (nxt < w.kt_hi && !issue_s_all(nxt, j + 1)) { ok = false; break; }
        // O_t += P_t V_cur
        bool have_v = false;
        for (int t = 0; t < 2 && ok; ++t) {
          if (!member(cur, t)) continue;
          // the item's first PV_t overwrites O_t: the previous item's O_t must be out
          if (npv[t] == npv0[t] && no[t] > 0 &&
              !mbar_wait_warp(bar(C::kBarOFree + t), (no[t] - 1) & 1, wd)) {
            ok = false;
            break;
          }
          FA_TRACE_POINT(46, npv[t], t);
          if (!mbar_wait_warp(bar(C::kBarPFull + t), npv[t] & 1, wd)) { ok = false; break; }
          FA_TRACE_POINT(47, npv[t], t);
          if (!have_v) {
            if (!wait_v(j)) { ok = false; break; }
            FA_TRACE_POINT(48, j, 0);
            have_v = true;
          }
          tc_fence_after();
          issue_pv<D, E>(tmem + C::kTmO0 + t * D, t ? p_smem1 : p_smem0, v_smem(j),
                         npv[t] > npv0[t]);
          tc_commit_e(bar(C::kBarPVDone + t));
          FA_TRACE_POINT(49, npv[t], t);
          ++npv[t];
        }
        if (!ok) break;
        tc_commit_e(bar(C::kBarVEmpty + j % C::kVSlots));
        cur = nxt;
      }
      for (int t = 0; t < 2; ++t)
        if (w.nk[t] > 0) ++no[t];
    }
    // No MMA may be in flight when TMEM is released.
    tc_commit_e(bar(C::kBarDrain));
    drain_wait(bar(C::kBarDrain), 0, p.timeout_ns);
    __syncwarp();
    FA_TRACE_POINT(99, 0, 0);
  } else {
    // ------------------------------------------------------------ softmax
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row_in_tile = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tm_s = tmem + lane_off + C::kTmS0 + t * 128;
    const uint32_t tm_o = tmem + lane_off + C::kTmO0 + t * D;
    uint8_t* p_row = base_ptr + C::kPOff + t * C::kPBytes + row_in_tile * 128;
    // S_t and PV_t products of the items before this one (their barrier phases)
    int n_prev = 0;
    bool ok = true;
    for (int ki = 0; ok; ++ki) {
      const int item = item_of(ki);
      if (item < 0) break;
      Work w;
      decode(item, w);
      const int bh = w.bh;
      const uint32_t ctr_head = p.drop.head_base + static_cast<uint32_t>(bh);  // dropout
      const int r0 = w.q0 + t * BM;
      const int row = r0 + row_in_tile;
      float m_ref = -INFINITY;
      float l = 0.0f;
      // lr: the same sum over P as rounded for the PV product. O is divided by lr, so
      // the weights it applies to V sum to exactly 1: the rounding of the largest
      // p (up to 2^8 under the lagging reference max, so up to 2^-8 relative) then
      // cancels instead of showing in O. LSE keeps the unrounded l. With dropout the
      // rounded values carry the keep mask, so there O is divided by l.
      float lr = 0.0f;
      // this tile's range and count as scalars (no per-thread array indexing)
      const int t_lo = t ? w.lo[1] : w.lo[0], t_hi = t ? w.hi[1] : w.hi[0];
      const int t_nk = t ? w.nk[1] : w.nk[0];
      auto t_member = [&](int kt) -> bool { return kt >= t_lo && kt < t_hi; };
      int kt = t_lo - 1;
      for (int j = 0; j < t_nk && ok; ++j) {
        do ++kt; while (!t_member(kt));
        const int n = n_prev + j;
        if (wq == 0) FA_TRACE_POINT(50, n, t);
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarSFull + t), n & 1, wd));
        if (wq == 0) FA_TRACE_POINT(51, n, t);
        if (ki == 0 && j == 0 && t == 0 && threadIdx.x == 0) FA_TRACE_CTA(2);
        if (j == 0 && wq == 0) FA_TRACE_POINT(57, ki, t);
        if (!ok) break;
        if (!softmax_key_tile<D, E, kDropout>(p, wd, tm_s, tm_o, p_row, bar(C::kBarSFree + t),
                                              bar(C::kBarPVDone + t), bar(C::kBarPFull + t),
                                              n, j == 0, kt, r0, row, row_in_tile,
                                              wl, wr, ctr_head, lane, wq, t, m_ref, l, lr)) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      if (t_nk > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(bar(C::kBarPVDone + t), (n_prev + t_nk - 1) & 1, wd));
        if (!ok) break;
      }
      n_prev += t_nk;
      if (t_nk == 0 && row < p.N && (t == 0 || w.own1)) {
        // a query tile that sees no key: O = 0, LSE = -inf
        uint4* dst = reinterpret_cast<uint4*>(p.O + (static_cast<size_t>(bh) * p.N + row) * D);
#pragma unroll
        for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
        p.LSE[static_cast<size_t>(bh) * p.N + row] = -INFINITY;
      }
      if (t_nk > 0) {
        if (t == 0 && threadIdx.x == 0) FA_TRACE_CTA(3);
        if (wq == 0) FA_TRACE_POINT(56, ki, t);
        tc_fence_after();
        const float norm = kDropout ? l : lr;
        const float inv_l = (norm > 0.0f) ? 1.0f / norm : 0.0f;
        uint16_t* orow = p.O + (static_cast<size_t>(bh) * p.N + row) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tm_o + cc * 32, o);
          tmem_wait_ld();
          if (cc == D / 32 - 1) {
            // O_t is in registers: the next item's first PV_t may overwrite it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(C::kBarOFree + t));
          }
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            pk[k] = pack2<E>(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
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

}  // namespace fwd
}  // namespace fa
