// fa_lib.cu -- the C ABI of include/fa.h: argument validation, TMA tensor-map
// construction, kernel launches and the device status word. All kernels are in
// this one translation unit (they share the status word without relocatable
// device code). The library allocates no device memory.

#include "fa.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cstdlib>
#include <map>
#include <mutex>
#include <queue>
#include <tuple>
#include <utility>
#include <vector>

#include "fa_ptx.cuh"
#include "fa_fwd_sm100.cuh"
#include "fa_bwd_sm100.cuh"
#include "fa_simt_f32.cuh"

namespace fa {
namespace {

// ------------------------------------------------------------------ watchdog kernel

__global__ void watchdog_selftest_kernel(unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  pdl_wait();  // the status word is written below
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must run out and record the timeout.
  const Watchdog wd{&abort_flag, timeout_ns};
  mbar_wait(smem_u32(&bar), 0, wd);
}

// ------------------------------------------------------------------ host helpers

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

unsigned long long watchdog_ns() {
  static const unsigned long long v = [] {
    const char* e = std::getenv("FA_WATCHDOG_MS");
    long long ms = e ? std::atoll(e) : 5000;
    if (ms <= 0) ms = 5000;
    return static_cast<unsigned long long>(ms) * 1000000ull;
  }();
  return v;
}

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context, or 0 if it cannot be
// had. A context that is destroyed and created again (cudaDeviceReset, or the
// primary context released and retained) gets a new id, so per-context state
// cached under the old id is never used with the new context. The runtime makes
// the device's primary context current first (cudaSetDevice initialises it).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (!get_current || !get_id) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaSetDevice(dev) != cudaSuccess) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

constexpr int kMaxDevices = 64;
struct DeviceState {
  bool checked = false;
  bool supported = false;
  int sms = 0;  // streaming multiprocessors
  // The kernels' shared-memory limits are attributes of the context: they are
  // set again whenever the current context's id differs from the one they were
  // set in (0 = never set).
  unsigned long long attrs_ctx = 0;
};
DeviceState g_devices[kMaxDevices];
std::mutex g_mutex;

// Launches `kernel` and returns the status of this launch alone: an error left
// pending by earlier, unrelated CUDA work is neither reported nor cleared. A
// failed launch's own error is cleared, so that it does not surface later in the
// caller's error checks. Launches allow programmatic stream serialization: the
// kernel's set-up may overlap the tail of the kernel before it on the stream, and
// every kernel waits for that one (pdl_wait) before touching global memory.
template <typename... KArgs, typename... Args>
fa_status launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                 Args&&... args) {
  cudaLaunchAttribute attr[1] = {};
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) return FA_OK;
  (void)cudaGetLastError();
  return FA_ERR_CUDA;
}

template <typename Kern>
cudaError_t set_smem(Kern k, size_t bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bytes));
}

template <int D, Elt E>
cudaError_t set_smem_d() {
  constexpr size_t S = fwd::Cfg<D>::kSmemBytes;
  cudaError_t e = set_smem(fwd::fa_fwd_kernel<D, E, false>, S);
  e = e ? e : set_smem(fwd::fa_fwd_kernel<D, E, true>, S);
  e = e ? e : set_smem(fwd::fa_fwd_persistent_kernel<D, E, false, false>, S);
  e = e ? e : set_smem(fwd::fa_fwd_persistent_kernel<D, E, true, false>, S);
  e = e ? e : set_smem(bwd::fa_bwd_kernel<D, E, false>, bwd::Cfg<D>::kSmemBytes);
  e = e ? e : set_smem(bwd::fa_bwd_kernel<D, E, true>, bwd::Cfg<D>::kSmemBytes);
  e = e ? e : set_smem(bwd::fa_bwd_persistent_kernel<D, E, false, false>, bwd::Cfg<D>::kSmemBytes);
  e = e ? e : set_smem(bwd::fa_bwd_persistent_kernel<D, E, true, false>, bwd::Cfg<D>::kSmemBytes);
  return e;
}

template <Elt E>
cudaError_t set_smem_all() {
  cudaError_t e = set_smem_d<64, E>();
  e = e ? e : set_smem_d<128, E>();
  if constexpr (E == Elt::BF16) {  // dropout instances (bf16, general masks)
    e = e ? e : set_smem(fwd::fa_fwd_kernel<64, E, true, true>, fwd::Cfg<64>::kSmemBytes);
    e = e ? e : set_smem(fwd::fa_fwd_kernel<128, E, true, true>, fwd::Cfg<128>::kSmemBytes);
    e = e ? e : set_smem(fwd::fa_fwd_persistent_kernel<64, E, true, true>, fwd::Cfg<64>::kSmemBytes);
    e = e ? e : set_smem(fwd::fa_fwd_persistent_kernel<128, E, true, true>, fwd::Cfg<128>::kSmemBytes);
    e = e ? e : set_smem(bwd::fa_bwd_kernel<64, E, true, true>, bwd::Cfg<64>::kSmemBytes);
    e = e ? e : set_smem(bwd::fa_bwd_kernel<128, E, true, true>, bwd::Cfg<128>::kSmemBytes);
    e = e ? e : set_smem(bwd::fa_bwd_persistent_kernel<64, E, true, true>, bwd::Cfg<64>::kSmemBytes);
    e = e ? e : set_smem(bwd::fa_bwd_persistent_kernel<128, E, true, true>, bwd::Cfg<128>::kSmemBytes);
  }
  return e;
}

// Checks that the current device is an sm_100 part and sets the kernels'
// shared-memory limits once per device.
fa_status prepare_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState& st = g_devices[dev];
  if (!st.checked) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    st.supported = (major == 10 && minor == 0);
    if (cudaDeviceGetAttribute(&st.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    st.checked = true;
  }
  if (!st.supported) return FA_ERR_UNSUPPORTED;
  const unsigned long long ctx = current_ctx_id();
  if (ctx == 0 || st.attrs_ctx != ctx) {
    cudaError_t e = cudaSuccess;
    e = e ? e : set_smem_all<Elt::BF16>();
    e = e ? e : set_smem_all<Elt::F16>();
    e = e ? e : set_smem(f32::fa_f32_bwd_dkdv_kernel<64>, f32::dkdv_smem_bytes<64>());
    e = e ? e : set_smem(f32::fa_f32_bwd_dkdv_kernel<128>, f32::dkdv_smem_bytes<128>());
    e = e ? e : set_smem(f32::fa_f32_bwd_dq_kernel<64>, f32::dq_smem_bytes<64>());
    e = e ? e : set_smem(f32::fa_f32_bwd_dq_kernel<128>, f32::dq_smem_bytes<128>());
    if (e != cudaSuccess) return FA_ERR_CUDA;
    st.attrs_ctx = ctx;
  }
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fa_status check_shape(int B, int H, int N, int d, float scale, int causal) {
  if (B < 1 || H < 1 || N < 0) return FA_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.0f)) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  // Offsets into the tensors are 64-bit. The bound is on the grids: one grid
  // dimension holds every (batch, head) x row block, and the smallest blocks (8 rows
  // of the backward preprocess, 16 of the fp32 kernels) number at most
  // 16 * B * H * ceil(N / 128).
  const long long tiles = static_cast<long long>(B) * H * ((static_cast<long long>(N) + 127) / 128);
  // Row indices stay 32-bit: N <= 2^30 keeps every row + window sum below 2^31.
  if (N > (1 << 30) || static_cast<long long>(B) * H >= (1ll << 31) || 16 * tiles >= (1ll << 31))
    return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

fa_status check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// 3-D view [B*H, N, d] of a 16-bit tensor (bf16 or f16 by E) with boxes of 64
// columns x `box_rows` rows x 1 head, 128-byte swizzle. Rows beyond N read as zero,
// per head.
template <Elt E>
bool make_map(CUtensorMap* map, const void* ptr, int BH, int N, int d, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                                 static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64u, static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  constexpr CUtensorMapDataType dt =
      (E == Elt::BF16) ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return enc(map, dt, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The masks as the kernels take them: window bounds clamped to [-1, N] (-1 = no
// bound; a bound of N or more keeps every key on that side) and causal folded into
// the right bound.
struct MaskSpec {
  int wl, wr;
  const uint8_t* blocks;
  // the general kernels are needed only for a left bound or a block mask; a right
  // bound alone (causal included) is a runtime value of the plain ones
  bool general() const { return wl >= 0 || blocks != nullptr; }
};

fa_status make_mask(int N, int causal, int window_left, int window_right,
                    const uint8_t* block_mask, MaskSpec* m) {
  m->wl = (window_left < 0 || window_left >= N) ? -1 : window_left;
  m->wr = causal ? 0 : ((window_right < 0 || window_right >= N) ? -1 : window_right);
  m->blocks = block_mask;
  if (block_mask != nullptr && (N + 127) / 128 > fwd::kMaxMaskTiles) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// Dropout as the kernels take it: keep iff the element's Philox byte >= threshold,
// where threshold = floor(256 p) (the drop probability is threshold / 256); kept
// values are scaled by 256 / (256 - threshold).
struct DropSpec {
  bool on = false;
  DropoutParams params{};
};

// floor(256 p) for p in [0, 1), the byte threshold; -1 for p outside [0, 1).
int drop_threshold(float p_drop) {
  if (!(p_drop >= 0.0f && p_drop < 1.0f)) return -1;
  const double t = std::floor(static_cast<double>(p_drop) * 256.0);
  return static_cast<int>(std::min(t, 255.0));
}

fa_status make_drop(float p_drop, uint64_t seed, uint32_t offset, int head_base, DropSpec* d) {
  const int ti = drop_threshold(p_drop);
  if (ti < 0 || head_base < 0) return FA_ERR_INVALID_ARG;
  // A rate in (0, 1/256) has threshold 0: it would silently drop nothing.
  if (ti == 0 && p_drop > 0.0f) return FA_ERR_UNSUPPORTED;
  d->on = ti > 0;
  // one byte per element: the drop probability is floor(256 p) / 256
  const double t = ti;
  d->params.threshold = static_cast<uint32_t>(t);
  d->params.scale = static_cast<float>(256.0 / (256.0 - t));
  d->params.seed_lo = static_cast<uint32_t>(seed);
  d->params.seed_hi = static_cast<uint32_t>(seed >> 32);
  d->params.offset = offset;
  // head_base + bh stays below 2^31 + 2^27: the shape checks keep B*H below 2^27
  d->params.head_base = static_cast<uint32_t>(head_base);
  return FA_OK;
}

// ---------------------------------------------------------------- forward work split
//
// A forward item owns two query tiles (they share every K/V tile the CTA loads), or
// one. Per head the lightest `singles` query tiles are single-tile items, listed after
// all pair items, where they even out the CTAs' loads at about half the cost of a
// pair. An item costs the larger key-tile count of its tiles (a pair) or 0.74 of its
// own (a single: measured on B1 H8 N16384 d128, 1024 single-tile CTAs ran at 0.77x
// the rate of 512 pair CTAs).
// Launch forms:
//   * one CTA per item, started in grid order on the first free SM. Each CTA pays
//     its set-up, first loads and epilogue (about 4 us measured on a B200) and the
//     next one on that SM starts about 1 us after it ends.
//   * persistent (fa_fwd_persistent_kernel): min(items, SMs) CTAs deal the list out
//     back and forth (CTA b takes items b, 2G - 1 - b, 2G + b, ...), so one item's
//     epilogue overlaps the next item's first loads and products. Measured on a B200
//     (forward TFLOP/s, one form against the other): short rows gain (B8 H12 N1024
//     causal: d64 225 -> 273, d128 381 -> 434); long rows lose, the per-item
//     bookkeeping slowing the issue loop (B1 H8 N4096 d128, one item per CTA either
//     way: 906 -> 860) and the fixed deal balancing long causal rows worse than the
//     hardware's first-free-SM order (B2 H16 N8192 d128 causal: 949 -> 898).
// So both forms are simulated, each with its best singles count: one CTA per item as
// above, and dealt back and forth with 0.4 key tiles of epilogue per item. The persistent
// form runs when it has more items than SMs and its makespan, 5% longer for its slower
// issue loop, beats that of one CTA per item (charged 1.5 key tiles per CTA for set-up,
// first loads, epilogue and launch gap) by 4%, and never with a block mask (its CTAs would
// build the mask rows of every item they walk). Those constants reproduce which form won
// in the measurements above and in B1 H8 N8192 d128 causal (persistent +14%), B2 H16 N4096
// d128 causal (+5%), B1 H8 N16384 d128 causal (0%) and non-causal (-6%). Cached per shape.
struct FwdSplit {
  int pairs_ph, singles_ph, weight_major, persistent;
};

constexpr double kFwdItemOverhead = 0.4;       // persistent: an item's epilogue, key tiles
constexpr double kFwdGridCtaOverhead = 1.5;    // one CTA per item: set-up, first loads, epilogue, gap
constexpr double kFwdPersistPenalty = 1.05;    // the persistent issue loop's slower key tiles
constexpr double kFwdPersistMargin = 1.04;     // predicted gain the persistent form must beat
// One CTA per item, causal or windowed: rank-major order while all K/V total at most this
// (B200 forward, rank-major against head-major: B1 H8 N16384 causal +4%, B2 H16 N8192
// causal +4%, B1 H16 N16384 causal +6%; at 256 MiB neutral).
constexpr double kFwdGridRankMajorBytes = 256.0 * (1 << 20);
// K and V of every head at most this large: rank-major item order (fits in L2)
constexpr double kFwdWeightMajorBytes = 96.0 * (1 << 20);

// Block-mask launches: one CTA per item, started in grid order on the first free SM.
double fwd_makespan_grid(int BH, int n_qt, int singles, int sms,
                         const std::vector<int>& key_tiles, double overhead = 0.0,
                         bool rank_major = false) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < sms; ++i) free_at.push(0.0);
  double end = 0.0;
  auto run = [&](double cost) {
    const double t = free_at.top() + cost;
    free_at.pop();
    free_at.push(t);
    end = std::max(end, t);
  };
  const int pairs = (n_qt - singles) / 2;
  // grid order: head-major (a head's items heaviest first) or rank-major (every head's
  // heaviest item, then every head's second, ...)
  const int outer_p = rank_major ? pairs : BH, inner_p = rank_major ? BH : pairs;
  for (int a = 0; a < outer_p; ++a)
    for (int b = 0; b < inner_p; ++b) {
      const int k = pairs - 1 - (rank_major ? a : b);
      const int t0 = singles + 2 * k;
      run(std::max(key_tiles[t0], key_tiles[t0 + 1]) + overhead);
    }
  const int outer_s = rank_major ? singles : BH, inner_s = rank_major ? BH : singles;
  for (int a = 0; a < outer_s; ++a)
    for (int b = 0; b < inner_s; ++b) run(0.74 * key_tiles[singles - 1 - (rank_major ? a : b)] + overhead);
  return end;
}

// Persistent launches: the largest load any CTA takes when the items are dealt out
// back and forth, in the kernel's order.
double fwd_makespan_persistent(int BH, int n_qt, int singles, int sms, bool weight_major,
                               const std::vector<int>& key_tiles) {
  const int pairs = (n_qt - singles) / 2;
  const long long n_pair = static_cast<long long>(BH) * pairs;
  const long long n_items = n_pair + static_cast<long long>(BH) * singles;
  const int G = static_cast<int>(std::min<long long>(n_items, sms));
  if (G <= 0) return 0.0;
  std::vector<double> load(G, 0.0);
  for (long long i = 0; i < n_items; ++i) {
    double cost;
    if (i < n_pair) {
      const long long r = weight_major ? i / BH : i % pairs;
      const int t0 = singles + 2 * static_cast<int>(pairs - 1 - r);
      cost = std::max(key_tiles[t0], key_tiles[t0 + 1]);
    } else {
      const long long c = i - n_pair;
      const long long r = weight_major ? c / BH : c % singles;
      cost = 0.74 * key_tiles[singles - 1 - static_cast<int>(r)];
    }
    const long long k = i / G, b = i % G;
    load[(k & 1) ? G - 1 - b : b] += cost + kFwdItemOverhead;
  }
  return *std::max_element(load.begin(), load.end());
}

FwdSplit fwd_split(int BH, int N, int d, int wl, int wr, bool block_mask, int sms) {
  const int n_qt = (N + fwd::BM - 1) / fwd::BM;
  const int n_kt = (N + fwd::BN - 1) / fwd::BN;
  const int min_singles = n_qt % 2;
  FwdSplit plain{(n_qt - min_singles) / 2, min_singles, 0, 0};
  if (sms <= 0) return plain;
  // Singles only help while they fit in the last round: at most about sms / BH per
  // head are tried. The simulation replays every item per candidate, so the total
  // (candidates x items) is bounded too; beyond it the plain split is used.
  const int max_singles = std::min(n_qt, 2 * ((sms + BH - 1) / BH) + 1);
  const long long candidates = (max_singles - min_singles) / 2 + 1;
  if (candidates * BH * n_qt > (1ll << 22)) return plain;
  static std::mutex mu;
  // at most 1024 shapes
  static std::map<std::tuple<int, int, int, int, int, bool, int>, FwdSplit> cache;
  const auto key = std::make_tuple(BH, N, d, wl, wr, block_mask, sms);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  // key tiles each query tile walks (window and causal; a block mask is ignored here)
  std::vector<int> key_tiles(n_qt);
  bool uniform = true;
  for (int t = 0; t < n_qt; ++t) {
    const int r0 = t * fwd::BM, r1 = std::min(r0 + fwd::BM, N) - 1;
    const int lo = (wl < 0) ? 0 : std::max(0, r0 - wl) / fwd::BN;
    const int hi = (wr < 0) ? n_kt : std::min(n_kt, (r1 + wr) / fwd::BN + 1);
    key_tiles[t] = std::max(hi - lo, 1);
    uniform = uniform && key_tiles[t] == key_tiles[0];
  }
  const bool wm = !block_mask && !uniform &&
                  static_cast<double>(BH) * N * d * 4.0 <= kFwdWeightMajorBytes;
  const bool wm_grid = !block_mask && !uniform &&
                       static_cast<double>(BH) * N * d * 4.0 <= kFwdGridRankMajorBytes;
  // each form's best singles count (one CTA per item: the makespan without the per-CTA
  // cost, as first measured; persistent: with its per-item epilogue)
  int sg_grid = min_singles, sg_pers = min_singles;
  double t_grid = fwd_makespan_grid(BH, n_qt, min_singles, sms, key_tiles, 0.0, wm_grid);
  double t_pers = fwd_makespan_persistent(BH, n_qt, min_singles, sms, wm, key_tiles);
  for (int sg = min_singles + 2; sg <= max_singles; sg += 2) {
    const double tg = fwd_makespan_grid(BH, n_qt, sg, sms, key_tiles, 0.0, wm_grid);
    if (tg < t_grid * 0.999) { t_grid = tg; sg_grid = sg; }
    if (!block_mask) {
      const double tp = fwd_makespan_persistent(BH, n_qt, sg, sms, wm, key_tiles);
      if (tp < t_pers * 0.999) { t_pers = tp; sg_pers = sg; }
    }
  }
  // the persistent form only where it is predicted to win by a margin, counting the one-CTA
  // form's set-up, first loads, epilogue and launch gap and the persistent form's slower
  // issue loop
  const long long pers_items = static_cast<long long>(BH) * ((n_qt - sg_pers) / 2 + sg_pers);
  const bool persistent =
      !block_mask && pers_items > sms &&
      fwd_makespan_grid(BH, n_qt, sg_grid, sms, key_tiles, kFwdGridCtaOverhead, wm_grid) >
          kFwdPersistMargin * kFwdPersistPenalty * t_pers;
  FwdSplit best = persistent ? FwdSplit{(n_qt - sg_pers) / 2, sg_pers, wm ? 1 : 0, 1}
                             : FwdSplit{(n_qt - sg_grid) / 2, sg_grid, wm_grid ? 1 : 0, 0};
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= 1024) cache.clear();
  cache[key] = best;
  return best;
}

// ---------------------------------------------------------------- backward tile split
//
// One backward CTA runs one key tile over all its query tiles ("steps"). When the
// key tiles are few (B1 H8 N4096 d128: 256 tiles of 32 steps on 148 SMs, 1.73
// waves) the last wave runs part empty. Cutting some tiles into two segments run
// by two CTAs evens the waves; a split tile pays a partial-sum write and one sum.
// The split is chosen by simulating the launch (CTAs start in grid order on the
// first free SM: whole tiles, then the larger segments, then the smaller ones;
// a CTA costs its steps plus one, a segment half a step more), for tiles of equal
// step counts only (no causal or window bound, no block mask), and kept only when
// the simulated time drops by more than 3%. Cached per shape.
// The simulation leaves out what a segment costs beyond its steps (a second K/V load
// and TMEM set-up, the fp32 partials written and read back), so two limits measured
// on a B200 (d = 128, non-causal, backward time with and without the split) bound it:
//   * only halves are tried: B1 H8 N4096 (108 tiles cut at 3/16) ran 3% slower;
//   * tiles of fewer than kMinSplitSteps query tiles never split: 16 steps gained
//     nothing (B1 H4 N2048 -3%, B1 H12 N2048 0%) and 8 steps lost (B1 H8 N1024 -20%),
//     while 32 steps or more gained (B1 H2 N4096 +24%, B1 H16 N4096 +5%, B1 H3 N8192
//     +19%, B1 H8 N8192 +8%).
// Launches of more than kMaxSplitGrid key tiles (four waves of 148 SMs) never split,
// and at most kMaxSplitTiles tiles split: the workspace makes room for that many.
constexpr int kMaxSplitTiles = 160;
constexpr long long kMaxSplitGrid = 4 * 148;
constexpr int kMinSplitSteps = 32;
constexpr double kBwdRankMajorBytes = 256.0 * (1 << 20);

struct BwdSplit {
  int n_split, split_num;
};

double split_makespan(long long whole, int split, double whole_cost, double seg_a, double seg_b,
                      int sms) {
  std::priority_queue<double, std::vector<double>, std::greater<double>> free_at;
  for (int i = 0; i < sms; ++i) free_at.push(0.0);
  double end = 0.0;
  auto run = [&](double cost) {
    const double t = free_at.top() + cost;
    free_at.pop();
    free_at.push(t);
    end = std::max(end, t);
  };
  for (long long i = 0; i < whole; ++i) run(whole_cost);
  for (int i = 0; i < split; ++i) run(std::max(seg_a, seg_b));
  for (int i = 0; i < split; ++i) run(std::min(seg_a, seg_b));
  return end;
}

// Split tiles in the kernel's order need the larger segment first: segment 1 is the
// larger when split_num < 8 (see bwd::Params).
BwdSplit bwd_split(int BH, int N, bool uniform_tiles, int sms) {
  BwdSplit none{0, 0};
  const int n_kt = (N + 127) / 128;
  const long long n_tiles = static_cast<long long>(BH) * n_kt;
  if (!uniform_tiles || sms <= 0 || n_kt < kMinSplitSteps || n_tiles > 4ll * sms ||
      n_tiles > kMaxSplitGrid)
    return none;
  static std::mutex mu;
  static std::map<std::tuple<int, int, int>, BwdSplit> cache;  // at most 1024 shapes
  const auto key = std::make_tuple(BH, N, sms);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  const int steps = n_kt;
  const double base = split_makespan(n_tiles, 0, steps + 1.0, 0, 0, sms);
  BwdSplit best = none;
  double best_t = base / 1.03;  // must beat the plain launch by more than 3%
  const int max_split = static_cast<int>(std::min<long long>(n_tiles, kMaxSplitTiles));
  const int ns_step = n_tiles < 64 ? 1 : 4;  // at most 64 simulated launches
  for (int ns = ns_step; ns <= max_split; ns += ns_step)
    for (int num : {8}) {
      const int a = bwd::split_point(steps, num);
      const double t = split_makespan(n_tiles - ns, ns, steps + 1.0, a + 1.5, steps - a + 1.5, sms);
      if (t < best_t) {
        best_t = t;
        best = BwdSplit{ns, num};
      }
    }
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() >= 1024) cache.clear();
  cache[key] = best;
  return best;
}

// Split tiles whose partial sums the workspace makes room for: the most a shape can use.
long long bwd_max_split(long long BH, int N) {
  const long long n_kt = (static_cast<long long>(N) + 127) / 128;
  if (n_kt < kMinSplitSteps || BH * n_kt > kMaxSplitGrid) return 0;
  return std::min<long long>(BH * n_kt, kMaxSplitTiles);
}

// Workspace bytes: L2 [BH, Npad] | D [BH, Npad] | dQ accumulator [BH, N, d] (fp32) |
// split-tile partials [S][2][2][128][d] (fp32) | arrival counters [S], for S split slots.
size_t backward_ws_bytes(long long BH, int N, int d, long long S) {
  const size_t bh = static_cast<size_t>(BH);
  const size_t npad = (static_cast<size_t>(N) + 127) / 128 * 128;
  const size_t s = static_cast<size_t>(S);
  return 2 * round256(bh * npad * sizeof(float)) + round256(bh * N * d * sizeof(float)) +
         round256(s * 4 * 128 * d * sizeof(float)) + round256(s * sizeof(unsigned));
}

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::lock_guard<std::mutex> lock(g_mutex);
  return g_devices[dev].sms;
}


}  // namespace
}  // namespace fa

using namespace fa;

namespace {

// The bf16 and f16 entry points share these bodies; E picks the kernels' element
// type and the tensor maps' data type.

template <Elt E, bool kMasked, bool kDropout, bool kPersistent>
fa_status launch_fwd(int d, dim3 grid, cudaStream_t s, const CUtensorMap& mq, const CUtensorMap& mk,
                     const CUtensorMap& mv, const fwd::Params& p) {
  constexpr int T = fwd::kThreads;
  constexpr size_t S64 = fwd::Cfg<64>::kSmemBytes, S128 = fwd::Cfg<128>::kSmemBytes;
  if constexpr (kPersistent) {
    if (d == 64)
      return launch(fwd::fa_fwd_persistent_kernel<64, E, kMasked, kDropout>, grid, T, S64, s,
                    mq, mk, mv, p);
    return launch(fwd::fa_fwd_persistent_kernel<128, E, kMasked, kDropout>, grid, T, S128, s,
                  mq, mk, mv, p);
  } else {
    if (d == 64) return launch(fwd::fa_fwd_kernel<64, E, kMasked, kDropout>, grid, T, S64, s, mq, mk, mv, p);
    return launch(fwd::fa_fwd_kernel<128, E, kMasked, kDropout>, grid, T, S128, s, mq, mk, mv, p);
  }
}

template <Elt E>
fa_status forward_impl(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int H, int N, int d, float scale, int causal, const MaskSpec& mask,
                     const DropSpec& drop, fa_stream_t stream) {
  fa_status st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (N == 0) return FA_OK;
  if ((st = check_ptrs({Q, K, V, O, LSE})) != FA_OK) return st;
  if ((st = prepare_device()) != FA_OK) return st;
  const int BH = B * H;
  CUtensorMap mq, mk, mv;
  if (!make_map<E>(&mq, Q, BH, N, d, fwd::BM) || !make_map<E>(&mk, K, BH, N, d, fwd::BN) ||
      !make_map<E>(&mv, V, BH, N, d, fwd::BN))
    return FA_ERR_CUDA;
  fwd::Params p;
  p.O = static_cast<uint16_t*>(O);
  p.LSE = LSE;
  p.N = N;
  p.BH = BH;
  const bool block_mask = mask.blocks != nullptr;
  const int sms = device_sms();
  const FwdSplit split = fwd_split(BH, N, d, mask.wl, mask.wr, block_mask, sms);
  p.pairs_ph = split.pairs_ph;
  p.singles_ph = split.singles_ph;
  p.n_pair_items = BH * split.pairs_ph;
  p.n_items = BH * (split.pairs_ph + split.singles_ph);
  p.weight_major = split.weight_major;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wl = mask.wl;
  p.wr = mask.wr;
  p.blocks = mask.blocks;
  p.n_kt = (N + fwd::BN - 1) / fwd::BN;
  p.drop = drop.params;
  p.timeout_ns = watchdog_ns();
  // persistent: one CTA per SM at most; else one CTA per item
  const bool pers = split.persistent != 0;
  const dim3 grid(static_cast<unsigned>(pers ? std::min(p.n_items, sms) : p.n_items));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool g = mask.general();
  if constexpr (E == Elt::BF16) {
    if (drop.on) {
      if (pers) return launch_fwd<E, true, true, true>(d, grid, s, mq, mk, mv, p);
      return launch_fwd<E, true, true, false>(d, grid, s, mq, mk, mv, p);
    }
  } else if (drop.on) {
    return FA_ERR_UNSUPPORTED;
  }
  if (g && pers) return launch_fwd<E, true, false, true>(d, grid, s, mq, mk, mv, p);
  if (g) return launch_fwd<E, true, false, false>(d, grid, s, mq, mk, mv, p);
  if (pers) return launch_fwd<E, false, false, true>(d, grid, s, mq, mk, mv, p);
  return launch_fwd<E, false, false, false>(d, grid, s, mq, mk, mv, p);
}

// Shared validation and set-up of the three backward stages. Fills the tensor maps
// only when `maps` is set (the main stage is the only one that needs them).
struct BwdPlan {
  int BH, N, Npad, d;
  float* L2;
  float* Dv;
  float* dQacc;
  float* part;         // partial dK/dV of split tiles
  unsigned* arrivals;  // their arrival counters
  int n_arrivals;
};

// split_ok = false: the workspace holds no split-tile slots (its size is the base
// size, S = 0) and the main kernel splits no tile.
fa_status bwd_plan(const void* const* ptrs, int nptrs, int B, int H, int N, int d,
                          float scale, int causal, void* workspace, size_t workspace_bytes,
                          BwdPlan* plan, bool split_ok = true) {
  fa_status st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  plan->BH = B * H;
  plan->N = N;
  plan->d = d;
  plan->Npad = (N + 127) / 128 * 128;
  if (N == 0) return FA_OK;
  for (int i = 0; i < nptrs; ++i)
    if (ptrs[i] == nullptr || !aligned16(ptrs[i])) return FA_ERR_INVALID_ARG;
  if (workspace == nullptr || !aligned16(workspace)) return FA_ERR_INVALID_ARG;
  const long long smax = split_ok ? bwd_max_split(plan->BH, N) : 0;
  if (workspace_bytes < backward_ws_bytes(plan->BH, N, d, smax)) return FA_ERR_INVALID_ARG;
  if ((st = prepare_device()) != FA_OK) return st;
  // workspace layout: see backward_ws_bytes
  char* ws = static_cast<char*>(workspace);
  const size_t vec_bytes = round256(static_cast<size_t>(plan->BH) * plan->Npad * sizeof(float));
  const size_t acc_bytes = round256(static_cast<size_t>(plan->BH) * N * d * sizeof(float));
  const size_t part_bytes = round256(static_cast<size_t>(smax) * 4 * 128 * d * sizeof(float));
  plan->L2 = reinterpret_cast<float*>(ws);
  plan->Dv = reinterpret_cast<float*>(ws + vec_bytes);
  plan->dQacc = reinterpret_cast<float*>(ws + 2 * vec_bytes);
  plan->part = reinterpret_cast<float*>(ws + 2 * vec_bytes + acc_bytes);
  plan->arrivals = reinterpret_cast<unsigned*>(ws + 2 * vec_bytes + acc_bytes + part_bytes);
  plan->n_arrivals = static_cast<int>(smax);
  return FA_OK;
}

template <Elt E>
fa_status preprocess_impl(const void* O, const void* dO, const float* LSE, int B, int H,
                                 int N, int d, float scale, int causal, void* workspace,
                                 size_t workspace_bytes, fa_stream_t stream,
                                 bool split_ok = true) {
  const void* ptrs[] = {O, dO, LSE};
  BwdPlan pl;
  fa_status st = bwd_plan(ptrs, 3, B, H, N, d, scale, causal, workspace, workspace_bytes, &pl,
                          split_ok);
  if (st != FA_OK || N == 0) return st;
  const long long rows = static_cast<long long>(pl.BH) * pl.Npad;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  const auto* O16 = static_cast<const uint16_t*>(O);
  const auto* dO16 = static_cast<const uint16_t*>(dO);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d == 64)
    return launch(bwd::fa_bwd_pre_kernel<64, E>, blocks, 256, 0, s, O16, dO16, LSE, pl.L2, pl.Dv,
                  pl.dQacc, N, pl.Npad, rows, pl.arrivals, pl.n_arrivals);
  return launch(bwd::fa_bwd_pre_kernel<128, E>, blocks, 256, 0, s, O16, dO16, LSE, pl.L2, pl.Dv,
                pl.dQacc, N, pl.Npad, rows, pl.arrivals, pl.n_arrivals);
}

template <Elt E, bool kMasked, bool kDropout, bool kPersistent>
fa_status launch_bwd(int d, dim3 grid, cudaStream_t s, const CUtensorMap& mq, const CUtensorMap& mk,
                     const CUtensorMap& mv, const CUtensorMap& mdo, const bwd::Params& p) {
  constexpr int T = bwd::kThreads;
  constexpr size_t S64 = bwd::Cfg<64>::kSmemBytes, S128 = bwd::Cfg<128>::kSmemBytes;
  if constexpr (kPersistent) {
    if (d == 64)
      return launch(bwd::fa_bwd_persistent_kernel<64, E, kMasked, kDropout>, grid, T, S64, s, mq,
                    mk, mv, mdo, p);
    return launch(bwd::fa_bwd_persistent_kernel<128, E, kMasked, kDropout>, grid, T, S128, s, mq,
                  mk, mv, mdo, p);
  } else {
    if (d == 64)
      return launch(bwd::fa_bwd_kernel<64, E, kMasked, kDropout>, grid, T, S64, s, mq, mk, mv, mdo,
                    p);
    return launch(bwd::fa_bwd_kernel<128, E, kMasked, kDropout>, grid, T, S128, s, mq, mk, mv, mdo,
                  p);
  }
}

// The persistent backward (fa_bwd_persistent_kernel) runs for every launch of more key
// tiles than SMs without a split tile or a block mask. Measured on a B200 (backward,
// persistent against one CTA per tile): B8 H12 N1024 causal d64 240 -> 252, d128
// 391 -> 428, B4 H16 N2048 d64 causal 341 -> 355, B1 H8 N4096 739 -> 746, B1 H8 N16384
// 880 -> 892 and causal unchanged; no shape measured slower.
bool bwd_persistent(int BH, int N, const MaskSpec& mask, int n_split, int sms) {
  const long long n_tiles = static_cast<long long>(BH) * ((N + 127) / 128);
  return mask.blocks == nullptr && n_split == 0 && sms > 0 && n_tiles > sms;
}

template <Elt E>
fa_status main_impl(const void* Q, const void* K, const void* V, const void* dO, void* dK,
                           void* dV, int B, int H, int N, int d, float scale, int causal,
                           const MaskSpec& mask, const DropSpec& drop, void* workspace,
                           size_t workspace_bytes, fa_stream_t stream, bool split_ok = true) {
  const void* ptrs[] = {Q, K, V, dO, dK, dV};
  BwdPlan pl;
  fa_status st = bwd_plan(ptrs, 6, B, H, N, d, scale, causal, workspace, workspace_bytes, &pl,
                          split_ok);
  if (st != FA_OK || N == 0) return st;
  CUtensorMap mq, mk, mv, mdo;
  // Q and dO stream in half tiles of 64 rows; K and V are loaded as 128-row tiles
  if (!make_map<E>(&mq, Q, pl.BH, N, d, 64) || !make_map<E>(&mk, K, pl.BH, N, d, bwd::BN) ||
      !make_map<E>(&mv, V, pl.BH, N, d, bwd::BN) || !make_map<E>(&mdo, dO, pl.BH, N, d, 64))
    return FA_ERR_CUDA;
  bwd::Params p;
  p.dK = static_cast<uint16_t*>(dK);
  p.dV = static_cast<uint16_t*>(dV);
  p.L2 = pl.L2;
  p.Dv = pl.Dv;
  p.dQacc = pl.dQacc;
  p.N = N;
  p.Npad = pl.Npad;
  p.BH = pl.BH;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wl = mask.wl;
  p.wr = mask.wr;
  p.blocks = mask.blocks;
  p.drop = drop.params;
  p.timeout_ns = watchdog_ns();
  const BwdSplit sp = pl.n_arrivals == 0 ? BwdSplit{0, 0}
                                          : bwd_split(pl.BH, N,
                                                      mask.wl < 0 && mask.wr < 0 &&
                                                          mask.blocks == nullptr,
                                                      device_sms());
  p.n_split = std::min(sp.n_split, pl.n_arrivals);
  p.split_num = sp.split_num;
  p.part = pl.part;
  p.arrivals = pl.arrivals;
  // rank-major order for causal or windowed launches of more than one wave of key tiles
  // whose Q, dO (16-bit) and fp32 dQ accumulator total at most 256 MiB: every head's
  // heaviest key tiles then start first. Measured on a B200 with one CTA per tile
  // (backward, rank-major against head-major): B8 H12 N1024 d64 causal +8%, B8 H12 N1024
  // d128 +6%, B4 H12 N2048 +12%, B2 H16 N4096 +11%, B1 H8 N16384 (128 MiB) +3.5%, B2 H16
  // N8192 (256 MiB) +5%; B4 H16 N8192 (512 MiB, four times the L2) -5%.
  const long long n_tiles = static_cast<long long>(pl.BH) * (pl.Npad / bwd::BN);
  p.rank_major = (mask.wr >= 0 || mask.wl >= 0) && mask.blocks == nullptr && p.n_split == 0 &&
                         n_tiles > device_sms() &&
                         static_cast<double>(pl.BH) * N * d * 8.0 <= kBwdRankMajorBytes
                     ? 1
                     : 0;
  const int sms = device_sms();
  const bool pers = bwd_persistent(pl.BH, N, mask, p.n_split, sms);
  const dim3 grid(pers ? static_cast<unsigned>(std::min<long long>(n_tiles, sms))
                       : static_cast<unsigned>(n_tiles + p.n_split));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const bool g = mask.general();
  if constexpr (E == Elt::BF16) {
    if (drop.on) {
      if (pers) return launch_bwd<E, true, true, true>(d, grid, s, mq, mk, mv, mdo, p);
      return launch_bwd<E, true, true, false>(d, grid, s, mq, mk, mv, mdo, p);
    }
  } else if (drop.on) {
    return FA_ERR_UNSUPPORTED;
  }
  if (g && pers) return launch_bwd<E, true, false, true>(d, grid, s, mq, mk, mv, mdo, p);
  if (g) return launch_bwd<E, true, false, false>(d, grid, s, mq, mk, mv, mdo, p);
  if (pers) return launch_bwd<E, false, false, true>(d, grid, s, mq, mk, mv, mdo, p);
  return launch_bwd<E, false, false, false>(d, grid, s, mq, mk, mv, mdo, p);
}

template <Elt E>
fa_status dq_convert_impl(void* dQ, int B, int H, int N, int d, float scale, void* workspace,
                                 size_t workspace_bytes, fa_stream_t stream,
                                 bool split_ok = true) {
  const void* ptrs[] = {dQ};
  BwdPlan pl;
  fa_status st = bwd_plan(ptrs, 1, B, H, N, d, scale, 0, workspace, workspace_bytes, &pl,
                          split_ok);
  if (st != FA_OK || N == 0) return st;
  const long long n4 = static_cast<long long>(pl.BH) * N * d / 4;
  const unsigned blocks = static_cast<unsigned>(std::min<long long>((n4 + 255) / 256, 148 * 16));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint16_t* dQ16 = static_cast<uint16_t*>(dQ);
  if (d == 64) return launch(bwd::fa_bwd_dq_kernel<64, E>, blocks, 256, 0, s, pl.dQacc, dQ16, n4, scale);
  return launch(bwd::fa_bwd_dq_kernel<128, E>, blocks, 256, 0, s, pl.dQacc, dQ16, n4, scale);
}

template <Elt E>
fa_status backward_impl(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                      const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                      float scale, int causal, const MaskSpec& mask, const DropSpec& drop,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream,
                      bool split_ok = true) {
  const void* ptrs[] = {Q, K, V, O, dO, LSE, dQ, dK, dV};
  BwdPlan pl;
  fa_status st = bwd_plan(ptrs, 9, B, H, N, d, scale, causal, workspace, workspace_bytes, &pl,
                          split_ok);
  if (st != FA_OK || N == 0) return st;
  st = preprocess_impl<E>(O, dO, LSE, B, H, N, d, scale, causal, workspace, workspace_bytes, stream,
                          split_ok);
  if (st != FA_OK) return st;
  st = main_impl<E>(Q, K, V, dO, dK, dV, B, H, N, d, scale, causal, mask, drop, workspace,
                    workspace_bytes, stream, split_ok);
  if (st != FA_OK) return st;
  return dq_convert_impl<E>(dQ, B, H, N, d, scale, workspace, workspace_bytes, stream, split_ok);
}

}  // namespace

extern "C" {

const char* fa_version(void) { return "fa-b200 0.1.0 sm_100a"; }

const char* fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "kernel watchdog timeout";
  }
  return "unknown status";
}

size_t fa_backward_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  const long long bh = static_cast<long long>(B) * H;
  return backward_ws_bytes(bh, N, d, bwd_max_split(bh, N));
}

fa_status fa_launch_plan(int B, int H, int N, int d, int causal, int* fwd_persistent_out,
                         int* bwd_persistent_out, int* bwd_split_out) {
  fa_status st = check_shape(B, H, N, d, 1.0f, causal);
  if (st != FA_OK) return st;
  if ((st = prepare_device()) != FA_OK) return st;
  const int BH = B * H, sms = device_sms();
  int fp = 0, bp = 0, bs = 0;
  if (N > 0) {
    MaskSpec m;
    if ((st = make_mask(N, causal, -1, -1, nullptr, &m)) != FA_OK) return st;
    fp = fwd_split(BH, N, d, m.wl, m.wr, false, sms).persistent;
    const long long smax = bwd_max_split(BH, N);
    if (smax > 0) {
      const BwdSplit sp = bwd_split(BH, N, m.wl < 0 && m.wr < 0, sms);
      bs = static_cast<int>(std::min<long long>(sp.n_split, smax));
    }
    bp = bwd_persistent(BH, N, m, bs, sms) ? 1 : 0;
  }
  if (fwd_persistent_out) *fwd_persistent_out = fp;
  if (bwd_persistent_out) *bwd_persistent_out = bp;
  if (bwd_split_out) *bwd_split_out = bs;
  return FA_OK;
}

float fa_dropout_rate(float p_drop) {
  const int t = drop_threshold(p_drop);
  if (t < 0 || (t == 0 && p_drop > 0.0f)) return -1.0f;
  return static_cast<float>(t) / 256.0f;
}

fa_status fa_get_status(fa_stream_t stream) {
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess)
    return FA_ERR_CUDA;
  return (v & kStatusTimeout) ? FA_ERR_TIMEOUT : FA_OK;
}

fa_status fa_watchdog_selftest(int timeout_ms, fa_stream_t stream) {
  if (timeout_ms < 1 || timeout_ms > 60000) return FA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  if (major != 10) return FA_ERR_UNSUPPORTED;
  return launch(watchdog_selftest_kernel, 1, 32, 0, reinterpret_cast<cudaStream_t>(stream),
                static_cast<unsigned long long>(timeout_ms) * 1000000ull);
}

fa_status fa_forward(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int H, int N, int d, float scale, int causal, fa_stream_t stream) {
  MaskSpec m;
  make_mask(N, causal, -1, -1, nullptr, &m);
  return forward_impl<Elt::BF16>(Q, K, V, O, LSE, B, H, N, d, scale, causal, m, DropSpec{}, stream);
}

fa_status fa_forward_f16(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                         int H, int N, int d, float scale, int causal, fa_stream_t stream) {
  MaskSpec m;
  make_mask(N, causal, -1, -1, nullptr, &m);
  return forward_impl<Elt::F16>(Q, K, V, O, LSE, B, H, N, d, scale, causal, m, DropSpec{}, stream);
}

fa_status fa_forward_masked(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            int B, int H, int N, int d, float scale, int causal,
                            int window_left, int window_right, const uint8_t* block_mask,
                            fa_stream_t stream) {
  MaskSpec m;
  const fa_status st = make_mask(N, causal, window_left, window_right, block_mask, &m);
  if (st != FA_OK) return st;
  return forward_impl<Elt::BF16>(Q, K, V, O, LSE, B, H, N, d, scale, causal, m, DropSpec{}, stream);
}

fa_status fa_backward_preprocess(const void* O, const void* dO, const float* LSE, int B, int H,
                                 int N, int d, float scale, int causal, void* workspace,
                                 size_t workspace_bytes, fa_stream_t stream) {
  return preprocess_impl<Elt::BF16>(O, dO, LSE, B, H, N, d, scale, causal, workspace,
                                    workspace_bytes, stream);
}

fa_status fa_backward_main(const void* Q, const void* K, const void* V, const void* dO, void* dK,
                           void* dV, int B, int H, int N, int d, float scale, int causal,
                           void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  MaskSpec m;
  make_mask(N, causal, -1, -1, nullptr, &m);
  return main_impl<Elt::BF16>(Q, K, V, dO, dK, dV, B, H, N, d, scale, causal, m, DropSpec{},
                              workspace, workspace_bytes, stream);
}

fa_status fa_backward_dq_convert(void* dQ, int B, int H, int N, int d, float scale, void* workspace,
                                 size_t workspace_bytes, fa_stream_t stream) {
  return dq_convert_impl<Elt::BF16>(dQ, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

fa_status fa_backward(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                      const float* LSE, void* dQ, void* dK, void* dV, int B, int H, int N, int d,
                      float scale, int causal, void* workspace, size_t workspace_bytes,
                      fa_stream_t stream) {
  MaskSpec m;
  make_mask(N, causal, -1, -1, nullptr, &m);
  return backward_impl<Elt::BF16>(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, m,
                                  DropSpec{}, workspace, workspace_bytes, stream);
}

fa_status fa_backward_masked(const void* Q, const void* K, const void* V, const void* O,
                             const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                             int B, int H, int N, int d, float scale, int causal,
                             int window_left, int window_right, const uint8_t* block_mask,
                             void* workspace, size_t workspace_bytes, fa_stream_t stream) {
  MaskSpec m;
  const fa_status st = make_mask(N, causal, window_left, window_right, block_mask, &m);
  if (st != FA_OK) return st;
  return backward_impl<Elt::BF16>(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, m,
                                  DropSpec{}, workspace, workspace_bytes, stream);
}

fa_status fa_backward_f16(const void* Q, const void* K, const void* V, const void* O,
                          const void* dO, const float* LSE, void* dQ, void* dK, void* dV, int B,
                          int H, int N, int d, float scale, int causal, void* workspace,
                          size_t workspace_bytes, fa_stream_t stream) {
  MaskSpec m;
  make_mask(N, causal, -1, -1, nullptr, &m);
  return backward_impl<Elt::F16>(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, m,
                                 DropSpec{}, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------- backward without allocation
//
// fa_backward needs a caller-provided device workspace. Some callers cannot make
// one: code that must not call cudaMalloc because the call can synchronise the
// whole device in the middle of latency-critical work, plugins whose host
// application owns every device allocation, or programs that reserved all of the
// device's memory up front for their own pool. For them, fa_backward_noalloc
// keeps the workspace in this fixed array, which the CUDA runtime places in device
// memory when the library's module is loaded on a GPU; it stays there, on every
// GPU that loads the library, until the process exits.
constexpr size_t kNoAllocScratchBytes = 32ull << 20;  // 32 MiB per GPU
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on each GPU, with the id of the context it
// was looked up in. In host code the array's name only stands in for the symbol;
// the address a kernel may use comes from cudaGetSymbolAddress with that GPU
// current. If the context is destroyed and created again (cudaDeviceReset), the
// module is loaded anew and the array may move: a changed context id makes the
// next call look the address up again.
struct NoAllocScratch {
  unsigned long long ctx = 0;
  void* ptr = nullptr;
};
static NoAllocScratch g_noalloc[kMaxDevices];

fa_status fa_backward_noalloc(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                              int B, int H, int N, int d, float scale, int causal,
                              fa_stream_t stream) {
  fa_status st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (N == 0) return FA_OK;
  // Without split-tile slots: the array holds L2, D and the dQ accumulator only.
  if (backward_ws_bytes(static_cast<long long>(B) * H, N, d, 0) > kNoAllocScratchBytes)
    return FA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  void* scratch = nullptr;
  {
    const unsigned long long ctx = current_ctx_id();  // 0: unknown, look up every call
    std::lock_guard<std::mutex> lock(g_mutex);
    NoAllocScratch& e = g_noalloc[dev];
    if (ctx == 0 || e.ctx != ctx || e.ptr == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return FA_ERR_CUDA;
      e.ptr = p;
      e.ctx = ctx;
    }
    scratch = e.ptr;
  }
  // The preprocess stage rewrites every byte of scratch the later stages read
  // (LSE*log2e, D, and the dQ accumulator it zeroes), so whatever an earlier call
  // left in the array does not matter.
  MaskSpec m;
  make_mask(N, causal, -1, -1, nullptr, &m);
  return backward_impl<Elt::BF16>(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, m,
                                  DropSpec{}, scratch, kNoAllocScratchBytes, stream,
                                  /*split_ok=*/false);
}

fa_status fa_forward_dropout(const void* Q, const void* K, const void* V, void* O, float* LSE,
                             int B, int H, int N, int d, float scale, int causal,
                             int window_left, int window_right, const uint8_t* block_mask,
                             float p_drop, uint64_t seed, uint32_t offset, fa_stream_t stream) {
  return fa_forward_dropout_heads(Q, K, V, O, LSE, B, H, N, d, scale, causal, window_left,
                                  window_right, block_mask, p_drop, seed, offset, 0, stream);
}

fa_status fa_forward_dropout_heads(const void* Q, const void* K, const void* V, void* O,
                                   float* LSE, int B, int H, int N, int d, float scale,
                                   int causal, int window_left, int window_right,
                                   const uint8_t* block_mask, float p_drop, uint64_t seed,
                                   uint32_t offset, int head_base, fa_stream_t stream) {
  MaskSpec m;
  DropSpec dr;
  fa_status st = make_drop(p_drop, seed, offset, head_base, &dr);
  if (st != FA_OK) return st;
  if ((st = make_mask(N, causal, window_left, window_right, block_mask, &m)) != FA_OK) return st;
  return forward_impl<Elt::BF16>(Q, K, V, O, LSE, B, H, N, d, scale, causal, m, dr, stream);
}

fa_status fa_backward_dropout(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                              int B, int H, int N, int d, float scale, int causal,
                              int window_left, int window_right, const uint8_t* block_mask,
                              float p_drop, uint64_t seed, uint32_t offset, void* workspace,
                              size_t workspace_bytes, fa_stream_t stream) {
  return fa_backward_dropout_heads(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal,
                                   window_left, window_right, block_mask, p_drop, seed, offset,
                                   0, workspace, workspace_bytes, stream);
}

fa_status fa_backward_dropout_heads(const void* Q, const void* K, const void* V, const void* O,
                                    const void* dO, const float* LSE, void* dQ, void* dK,
                                    void* dV, int B, int H, int N, int d, float scale,
                                    int causal, int window_left, int window_right,
                                    const uint8_t* block_mask, float p_drop, uint64_t seed,
                                    uint32_t offset, int head_base, void* workspace,
                                    size_t workspace_bytes, fa_stream_t stream) {
  MaskSpec m;
  DropSpec dr;
  fa_status st = make_drop(p_drop, seed, offset, head_base, &dr);
  if (st != FA_OK) return st;
  if ((st = make_mask(N, causal, window_left, window_right, block_mask, &m)) != FA_OK) return st;
  return backward_impl<Elt::BF16>(Q, K, V, O, dO, LSE, dQ, dK, dV, B, H, N, d, scale, causal, m,
                                  dr, workspace, workspace_bytes, stream);
}

fa_status fa_forward_f32(const float* Q, const float* K, const float* V, float* O, float* LSE,
                         int B, int H, int N, int d, float scale, int causal,
                         fa_stream_t stream) {
  fa_status st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (N == 0) return FA_OK;
  if ((st = check_ptrs({Q, K, V, O, LSE})) != FA_OK) return st;
  if ((st = prepare_device()) != FA_OK) return st;
  // grid.x = (batch, head) x row blocks (check_shape bounds it below 2^31)
  const dim3 grid(static_cast<unsigned>(static_cast<long long>(B) * H *
                                        ((N + f32::kRowsPerBlock - 1) / f32::kRowsPerBlock)));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  constexpr int T = f32::kWarps * 32;
  if (d == 64) return launch(f32::fa_f32_fwd_kernel<64>, grid, T, 0, s, Q, K, V, O, LSE, N, scale, causal);
  return launch(f32::fa_f32_fwd_kernel<128>, grid, T, 0, s, Q, K, V, O, LSE, N, scale, causal);
}

fa_status fa_backward_f32(const float* Q, const float* K, const float* V, const float* O,
                          const float* dO, const float* LSE, float* dQ, float* dK, float* dV,
                          int B, int H, int N, int d, float scale, int causal, void* workspace,
                          size_t workspace_bytes, fa_stream_t stream) {
  fa_status st = check_shape(B, H, N, d, scale, causal);
  if (st != FA_OK) return st;
  if (N == 0) return FA_OK;
  if ((st = check_ptrs({Q, K, V, O, dO, LSE, dQ, dK, dV, workspace})) != FA_OK) return st;
  if (workspace_bytes < fa_backward_workspace_size(B, H, N, d)) return FA_ERR_INVALID_ARG;
  if ((st = prepare_device()) != FA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* Dvec = static_cast<float*>(workspace);
  const long long rows = static_cast<long long>(B) * H * N;
  const unsigned dot_blocks = static_cast<unsigned>((rows + f32::kWarps - 1) / f32::kWarps);
  const dim3 grid(static_cast<unsigned>(static_cast<long long>(B) * H *
                                        ((N + f32::kRowsPerBlock - 1) / f32::kRowsPerBlock)));
  constexpr int T = f32::kWarps * 32;
  if (d == 64) {
    st = launch(f32::fa_f32_bwd_dot_kernel<64>, dot_blocks, T, 0, s, O, dO, Dvec, rows);
    if (st == FA_OK)
      st = launch(f32::fa_f32_bwd_dkdv_kernel<64>, grid, T, f32::dkdv_smem_bytes<64>(), s, Q, K, V,
                  dO, LSE, Dvec, dK, dV, N, scale, causal);
    if (st == FA_OK)
      st = launch(f32::fa_f32_bwd_dq_kernel<64>, grid, T, f32::dq_smem_bytes<64>(), s, Q, K, V, dO,
                  LSE, Dvec, dQ, N, scale, causal);
  } else {
    st = launch(f32::fa_f32_bwd_dot_kernel<128>, dot_blocks, T, 0, s, O, dO, Dvec, rows);
    if (st == FA_OK)
      st = launch(f32::fa_f32_bwd_dkdv_kernel<128>, grid, T, f32::dkdv_smem_bytes<128>(), s, Q, K,
                  V, dO, LSE, Dvec, dK, dV, N, scale, causal);
    if (st == FA_OK)
      st = launch(f32::fa_f32_bwd_dq_kernel<128>, grid, T, f32::dq_smem_bytes<128>(), s, Q, K, V, dO,
                  LSE, Dvec, dQ, N, scale, causal);
  }
  return st;
}


#ifdef FA_TRACE
// Profiling aid (built only with -DFA_TRACE): arm the timeline trace for one CTA
// of the next launches (clearing it), and read back the slots and the two global
// timer stamps.
int fa_trace_arm(int cta) {
  static std::vector<uint32_t> zeros(kTraceCap, 0u);
  if (cudaMemcpyToSymbol(g_trace, zeros.data(), kTraceCap * sizeof(uint32_t)) != cudaSuccess)
    return -1;
  if (cudaMemcpyToSymbol(g_trace_cta, &cta, sizeof(cta)) != cudaSuccess) return -1;
  static std::vector<unsigned long long> zeros_cta(kTraceCtas * 8u, 0ull);
  if (cudaMemcpyToSymbol(g_trace_cta_ns, zeros_cta.data(), zeros_cta.size() * sizeof(unsigned long long)) !=
      cudaSuccess)
    return -1;
  return 0;
}
int fa_trace_cta_read(unsigned long long* out, int n_ctas) {
  if (n_ctas < 0 || n_ctas > static_cast<int>(kTraceCtas)) return -1;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(out, g_trace_cta_ns, static_cast<size_t>(n_ctas) * 8 * sizeof(unsigned long long)) !=
      cudaSuccess)
    return -1;
  return n_ctas;
}
int fa_trace_read(uint32_t* slots, unsigned long long* ns) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  if (cudaMemcpyFromSymbol(slots, g_trace, kTraceCap * sizeof(uint32_t)) != cudaSuccess)
    return -1;
  if (cudaMemcpyFromSymbol(ns, g_trace_ns, 2 * sizeof(unsigned long long)) != cudaSuccess)
    return -1;
  return static_cast<int>(kTraceCap);
}
#endif

}  // extern "C"
