/*
 * fa.h -- C ABI of the B200 (sm_100a) IO-aware exact-attention library.
 *
 * The operation (per batch b and head h; X[b,h] is an N x d row-major matrix):
 *   S = scale * Q K^T, with S[i][j] = -inf when causal and j > i,
 *   P = softmax(S) row by row, O = P V, LSE[i] = ln sum_j exp(S[i][j]).
 * Definition: "A survey of key techniques of large language model pre-training
 * systems", Journal of Software 2026(1), p.218 (attention definition S = QK^T,
 * P = Softmax(S), O = PV, and the two-block softmax decomposition the kernels use
 * to process keys tile by tile); scaling by 1/sqrt(d): "FlashAttention
 * optimisation: breaking the performance bottleneck of standard attention",
 * section 1; causal masking: "Flash Attention-2: acceleration principle and GPU
 * memory optimisation in deployment", causal-mask item. The forward is the fused,
 * tiled, online-softmax pass of "FlashAttention optimisation ...", section 4.1;
 * the backward recomputes P from LSE ("... ", section 4.2; "From GPU memory access
 * to code: how FlashAttention makes large-model training 3x faster", section 2.2)
 * and forms the gradient of the loss <dO, O>:
 *   dV = P^T dO, dP = dO V^T, D = rowsum(dO o O), dS = P o (dP - D),
 *   dQ = scale * dS K, dK = scale * dS^T Q.
 * No N x N matrix is ever written to device memory.
 *
 * Conventions shared by every entry point:
 *   - Tensors are contiguous row-major [B, H, N, d] (LSE and D are [B, H, N]),
 *     in DEVICE memory, base addresses 16-byte aligned. Q, K and V share one N
 *     (self-attention shape).
 *   - The caller owns every buffer, including the backward workspace; the
 *     library allocates no device memory at run time. Its state: one device
 *     status word per GPU, the fixed scratch array of fa_backward_noalloc (part
 *     of the module image), and on the host each GPU's SM count and a cache of
 *     the forward's work split per shape (thread-safe).
 *   - Calls are asynchronous on `stream` (0 = the legacy default stream).
 *     Argument errors are returned synchronously and launch nothing. A failed
 *     launch returns FA_ERR_CUDA.
 *   - Stream order holds as for any kernel. The library's kernels are launched
 *     with programmatic stream serialization: each may be placed while the
 *     kernel before it on the stream finishes, and waits for that kernel
 *     (griddepcontrol.wait) before touching global memory. A kernel of the
 *     caller's that follows on the stream and is itself launched with that
 *     attribute may start once the library kernel's CTAs have done their work;
 *     it must wait (griddepcontrol.wait / cudaGridDependencySynchronize) before
 *     reading the call's outputs. Kernels launched without it see plain order.
 *   - Every wait inside a kernel is bounded (default 5 s; the environment
 *     variable FA_WATCHDOG_MS, read once per process, overrides it). A wait that
 *     runs out makes the kernel record the error in the device status word and
 *     return early, leaving its outputs undefined; fa_get_status() reports it as
 *     FA_ERR_TIMEOUT.
 *   - Supported: B, H >= 1; N >= 0 (N = 0 is a no-op); d in {64, 128};
 *     causal in {0, 1}; scale finite and > 0; N <= 2^30 and
 *     B*H*ceil(N/128) < 2^27 (a bound on the launch grids; tensor offsets are
 *     64-bit, so one tensor may exceed 2^31 elements). Larger shapes return
 *     FA_ERR_UNSUPPORTED.
 *   - Outputs are overwritten, never accumulated into.
 */
#ifndef FA_B200_FA_H
#define FA_B200_FA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t. */
typedef struct CUstream_st* fa_stream_t;

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad shape, bad scale */
  FA_ERR_UNSUPPORTED = 2, /* valid arguments outside what this library implements */
  FA_ERR_CUDA = 3,        /* a CUDA call or launch failed (no device, bad context) */
  FA_ERR_TIMEOUT = 4      /* a kernel's bounded wait ran out (see fa_get_status) */
} fa_status;

/*
 * Forward, bf16 in / bf16 out, fp32 accumulation (tcgen05 tensor cores).
 *   Q, K, V : bf16 [B,H,N,d], read only.
 *   O       : bf16 [B,H,N,d], written: softmax(S) V rounded to nearest-even.
 *   LSE     : fp32 [B,H,N], written: natural-log log-sum-exp of the scaled,
 *             masked logits of each query row.
 */
fa_status fa_forward(const void* Q, const void* K, const void* V, void* O, float* LSE,
                     int B, int H, int N, int d, float scale, int causal,
                     fa_stream_t stream);

/*
 * Workspace bytes fa_backward and fa_backward_f32 need for this shape, with
 * Npad = N rounded up to a multiple of 128 and T = B*H*Npad/128 key tiles:
 *   LSE*log2(e) (fp32 [B*H, Npad]) + D (fp32 [B*H, Npad]) + dQ accumulator
 *   (fp32 [B,H,N,d]) + room for S split key tiles: fp32 dK and dV partials of
 *   both halves (fp32 [S,2,2,128,d]) and an arrival counter each (u32 [S]);
 *   each region rounded up to 256 bytes. S = min(T, 160) when T <= 592 and
 *   Npad >= 4096 (32 query tiles per key tile), else 0. (A launch of few key
 *   tiles runs some of them as two CTAs, one per half of the query tiles, to
 *   fill the SMs' last wave.)
 * Returns 0 for a shape that is invalid or empty.
 */
size_t fa_backward_workspace_size(int B, int H, int N, int d);

/*
 * Backward, bf16 in / bf16 out, fp32 accumulation (tcgen05 tensor cores).
 *   Q, K, V, O, dO : bf16 [B,H,N,d], read only (O and LSE from fa_forward on the
 *                    same Q, K, V, scale and causal).
 *   LSE            : fp32 [B,H,N], read only.
 *   dQ, dK, dV     : bf16 [B,H,N,d], written (gradients of <dO, O>).
 *   workspace      : device memory of at least fa_backward_workspace_size bytes,
 *                    16-byte aligned; its contents on entry do not matter and are
 *                    undefined on return.
 * dQ is accumulated in fp32 with atomic adds, so its last bits may differ from
 * run to run; dK and dV are deterministic.
 */
fa_status fa_backward(const void* Q, const void* K, const void* V, const void* O,
                      const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                      int B, int H, int N, int d, float scale, int causal,
                      void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * The three stages fa_backward runs, in order, on the same stream and workspace
 * (exposed so that each stage can be timed or scheduled on its own; calling the
 * three in order is exactly fa_backward):
 *   fa_backward_preprocess: D = rowsum(dO o O) and LSE*log2(e) into the workspace
 *                           (rows padded to a multiple of 128), and zeroes the fp32
 *                           dQ accumulator in the workspace.
 *   fa_backward_main      : the fused recomputation kernel: writes dK, dV and adds
 *                           the unscaled dQ into the workspace accumulator.
 *   fa_backward_dq_convert: dQ = bf16(scale * accumulator).
 * Arguments mean what they mean for fa_backward; `causal` is not used by the
 * convert stage. Argument errors are returned before any launch.
 */
fa_status fa_backward_preprocess(const void* O, const void* dO, const float* LSE, int B, int H,
                                 int N, int d, float scale, int causal, void* workspace,
                                 size_t workspace_bytes, fa_stream_t stream);
fa_status fa_backward_main(const void* Q, const void* K, const void* V, const void* dO,
                           void* dK, void* dV, int B, int H, int N, int d, float scale,
                           int causal, void* workspace, size_t workspace_bytes,
                           fa_stream_t stream);
fa_status fa_backward_dq_convert(void* dQ, int B, int H, int N, int d, float scale,
                                 void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_backward without a workspace argument, for callers that cannot allocate
 * device memory (for example code that must not call cudaMalloc because it may
 * synchronise the device, plugins whose host application owns every allocation,
 * or programs whose memory is all reserved by their own pool). The sources this
 * library follows have no counterpart: it is a deployment convenience.
 *   Arguments, outputs and numerics: as for fa_backward.
 *   Scratch: a 32 MiB array built into the library, one per GPU, placed in device
 *     memory when the library's module is loaded on that GPU and held until the
 *     process exits. The call allocates nothing.
 *   Limit: shapes whose LSE*log2(e), D and dQ accumulator regions (the workspace size
 *     with S = 0, see fa_backward_workspace_size) exceed 32 MiB (33554432 bytes)
 *     return FA_ERR_UNSUPPORTED and launch nothing. The array holds no room for
 *     split key tiles: every key tile runs whole, so where fa_backward would
 *     split tiles dK and dV may differ from its result in the last bits.
 *   Set-up: the first call on a GPU looks up the array's device address with
 *     that GPU current (and may load the library's module there); make that first
 *     call before any stream capture. If the GPU's context is destroyed and
 *     created again (cudaDeviceReset), the next call looks the address up again.
 *   Sharing: every call on a GPU uses the same array. Each call rewrites all of
 *     it that it reads (the dQ accumulator is zeroed by the call itself), but two
 *     calls whose kernels can overlap on the GPU (different streams without an
 *     ordering between them, or different host threads) race on it and give
 *     wrong results. Order such calls on one stream.
 */
fa_status fa_backward_noalloc(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                              int B, int H, int N, int d, float scale, int causal,
                              fa_stream_t stream);

/*
 * f16 entry points: fa_forward and fa_backward with IEEE half-precision (f16)
 * tensors in place of bf16 -- Q, K, V, O, dO, dQ, dK, dV are f16 [B,H,N,d]; LSE
 * and the workspace as for the bf16 calls. Same kernels and the same fp32
 * accumulation; P and dS are rounded to f16 before their products (the tensor
 * cores take both operands of one product in one 16-bit type). f16 holds values
 * below 65504 in magnitude: O, dQ, dK and dV beyond that become infinite.
 */
fa_status fa_forward_f16(const void* Q, const void* K, const void* V, void* O, float* LSE,
                         int B, int H, int N, int d, float scale, int causal,
                         fa_stream_t stream);
fa_status fa_backward_f16(const void* Q, const void* K, const void* V, const void* O,
                          const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                          int B, int H, int N, int d, float scale, int causal,
                          void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Masked attention (bf16): fa_forward and fa_backward with two more masks that
 * combine with `causal` by AND -- query i sees key j only if every mask keeps it.
 *   window_left, window_right: a sliding window, key j kept iff
 *       i - window_left <= j <= i + window_right; a negative value leaves that side
 *       unbounded (-1, -1 = no window; window_right = 0 is the causal mask). From
 *       the sliding-window example of "Flash Attention-2: acceleration principle
 *       and GPU memory optimisation in deployment" (causal-mask item: a window-size
 *       pair given together with is_causal).
 *   block_mask: NULL, or DEVICE memory holding a row-major T x T byte matrix,
 *       T = ceil(N / 128), the same for every batch and head; (i, j) is kept iff
 *       block_mask[(i / 128) * T + j / 128] != 0. Block-sparse attention,
 *       "FlashAttention optimisation ...", section 7, at the tile size 128 of the
 *       "Flash Attention-2 ..." page's block strategy. Tiles the mask drops are
 *       never loaded or computed. T <= 4096 (N <= 524288), else
 *       FA_ERR_UNSUPPORTED. Read only; any alignment.
 * A query row that sees no key gets O = 0 and LSE = -inf, and dQ = 0; a key that
 * no query sees gets dK = dV = 0. The backward must be given the same masks as
 * the forward that produced O and LSE. Other arguments as for fa_forward /
 * fa_backward.
 */
fa_status fa_forward_masked(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            int B, int H, int N, int d, float scale, int causal,
                            int window_left, int window_right, const uint8_t* block_mask,
                            fa_stream_t stream);
fa_status fa_backward_masked(const void* Q, const void* K, const void* V, const void* O,
                             const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                             int B, int H, int N, int d, float scale, int causal,
                             int window_left, int window_right, const uint8_t* block_mask,
                             void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Masked attention with dropout on P (bf16): fa_forward_masked / fa_backward_masked
 * plus dropout, one of the operations "A survey of key techniques of large language
 * model pre-training systems" (Journal of Software 2026(1), p.218) lists as fused
 * into the attention kernel. With p_drop in [0, 1), t = floor(256 p_drop) and the drop
 * probability t / 256 (p_drop rounded down to a multiple of 1/256):
 *   Pd = P o Z * 256 / (256 - t),  O = Pd V,  LSE = the log-sum-exp of the logits
 *   (unchanged by dropout); the backward regenerates Z, so nothing N x N is stored.
 * One Philox-4x32-10 block (Salmon, Moraes, Dror and Shaw, "Parallel random numbers:
 * as easy as 1, 2, 3", SC 2011) covers 4 queries x 4 keys: the block at counter
 * (j / 4, i / 4, b * H + h, offset) under key (seed & 0xffffffff, seed >> 32) gives
 * query i its word i mod 4 and key j byte j mod 4 of that word (byte 0 the least
 * significant); Z[i][j] = 0 iff that byte is below t. `offset` lets successive calls
 * draw independent masks under one seed. The backward must be given the same seed,
 * offset, p_drop and masks as the forward. p_drop = 0 is no dropout; p_drop outside
 * [0, 1) (or NaN) is FA_ERR_INVALID_ARG; p_drop in (0, 1/256), which would round
 * down to no dropout, is FA_ERR_UNSUPPORTED. fa_dropout_rate(p_drop) returns the
 * rate actually applied.
 */
fa_status fa_forward_dropout(const void* Q, const void* K, const void* V, void* O, float* LSE,
                             int B, int H, int N, int d, float scale, int causal,
                             int window_left, int window_right, const uint8_t* block_mask,
                             float p_drop, uint64_t seed, uint32_t offset, fa_stream_t stream);
fa_status fa_backward_dropout(const void* Q, const void* K, const void* V, const void* O,
                              const void* dO, const float* LSE, void* dQ, void* dK, void* dV,
                              int B, int H, int N, int d, float scale, int causal,
                              int window_left, int window_right, const uint8_t* block_mask,
                              float p_drop, uint64_t seed, uint32_t offset, void* workspace,
                              size_t workspace_bytes, fa_stream_t stream);

/*
 * The dropout calls for a range of a larger problem's heads: the Philox counter's
 * third word is head_base + b * H + h instead of b * H + h, so a call on the flattened
 * heads [head_base, head_base + B * H) of a [B', H', N, d] problem (given as a
 * [1, B * H, N, d] slice, or any B, H with that product) draws exactly the keep masks
 * the whole call draws for those heads. This is what lets a problem be split by heads
 * over several GPUs with dropout. head_base = 0 is fa_forward_dropout /
 * fa_backward_dropout; head_base < 0 is FA_ERR_INVALID_ARG. Other arguments, errors
 * and ownership as for those calls.
 */
fa_status fa_forward_dropout_heads(const void* Q, const void* K, const void* V, void* O,
                                   float* LSE, int B, int H, int N, int d, float scale,
                                   int causal, int window_left, int window_right,
                                   const uint8_t* block_mask, float p_drop, uint64_t seed,
                                   uint32_t offset, int head_base, fa_stream_t stream);
fa_status fa_backward_dropout_heads(const void* Q, const void* K, const void* V, const void* O,
                                    const void* dO, const float* LSE, void* dQ, void* dK,
                                    void* dV, int B, int H, int N, int d, float scale,
                                    int causal, int window_left, int window_right,
                                    const uint8_t* block_mask, float p_drop, uint64_t seed,
                                    uint32_t offset, int head_base, void* workspace,
                                    size_t workspace_bytes, fa_stream_t stream);

/*
 * The drop probability the dropout calls apply for `p_drop`: floor(256 p_drop) / 256
 * (for example 0.1 gives 25/256 = 0.09765625). Returns -1 for a p_drop those calls
 * refuse (outside [0, 1), NaN, or in (0, 1/256)). Host only; no CUDA call.
 */
float fa_dropout_rate(float p_drop);

/*
 * How the library distributes a plain call (no window, block mask or dropout) of this
 * shape on the current GPU. A planning query: it launches nothing.
 *   *fwd_persistent: 1 if fa_forward runs its persistent kernel (CTAs walking a list
 *     of query-tile items), 0 if one CTA per item.
 *   *bwd_persistent: 1 if the backward's main stage runs its persistent kernel (CTAs
 *     walking a list of key tiles), 0 if one CTA per key tile.
 *   *bwd_split: the number of key tiles the backward runs as two CTAs (0 when
 *     persistent).
 * Output pointers may be null. Returns FA_ERR_INVALID_ARG or FA_ERR_UNSUPPORTED for a
 * shape the calls refuse, FA_ERR_CUDA without a usable sm_100 device.
 */
fa_status fa_launch_plan(int B, int H, int N, int d, int causal, int* fwd_persistent,
                         int* bwd_persistent, int* bwd_split);

/*
 * fp32 entry points: the same operation and arguments with fp32 tensors
 * (float [B,H,N,d]), computed in fp32 on the CUDA cores (FFMA), for callers that
 * need fp32 accuracy; tensor-core fp32 (tf32) cannot reach it. The backward is
 * deterministic. workspace as for fa_backward.
 */
fa_status fa_forward_f32(const float* Q, const float* K, const float* V, float* O,
                         float* LSE, int B, int H, int N, int d, float scale, int causal,
                         fa_stream_t stream);
fa_status fa_backward_f32(const float* Q, const float* K, const float* V, const float* O,
                          const float* dO, const float* LSE, float* dQ, float* dK,
                          float* dV, int B, int H, int N, int d, float scale, int causal,
                          void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * Synchronises `stream`, reads and clears the device status word of the current
 * GPU. Returns FA_ERR_TIMEOUT if a kernel since the last call gave up on a wait,
 * FA_ERR_CUDA if the synchronisation itself failed, else FA_OK.
 */
fa_status fa_get_status(fa_stream_t stream);

/*
 * Launches one kernel that waits, bounded by `timeout_ms`, on a barrier nothing
 * ever completes, so the watchdog path can be exercised without a fault or hang.
 * Afterwards fa_get_status() must return FA_ERR_TIMEOUT.
 */
fa_status fa_watchdog_selftest(int timeout_ms, fa_stream_t stream);

/* Static English text for a status code. */
const char* fa_status_string(fa_status status);

/* Library version string, e.g. "fa-b200 0.1.0 sm_100a". */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_FA_H */
