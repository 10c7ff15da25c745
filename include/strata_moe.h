/*
 * strata_moe.h -- C ABI of the B200 (sm_100a) mixture-of-experts expert layer.
 *
 * One MoE layer applied to a batch of T tokens (a prefill chunk, or a 1..4
 * token decode / speculative-verify batch):
 *
 *   logits = x . W_r (+ bias)                 router
 *   ids, w = top-k(logits), softmax over the k selected logits
 *   rows grouped by expert (histogram -> exclusive scan -> stable scatter)
 *   h      = SiLU(x . Wg_e) * (x . Wu_e)       grouped int4 GEMM, dequant fused
 *   o      = h . Wd_e                           grouped int4 GEMM, dequant fused
 *   y_t    = sum_j w_tj * o_(t,j)               weighted combine
 *
 * Sources.  The method is the MoE expert layer of the Strata local inference
 * engine as described by public write-ups:
 *   - each layer holds 512 experts and a token activates about 10; larger
 *     prefill batches let more tokens reuse each expert: "两天移植，预填充提速8倍：
 *     Strata引擎实测" (kongchang.com), section "Strata快在哪", MoE note;
 *   - the per-layer router picks a subset of experts per token: penglei.dev
 *     "Strata local MoE" post, section "原理一：把显存作为专家缓存";
 *   - 4-bit group quantisation with per-group scales, group 32/64/128:
 *     lqnn.cn static review section 3.1, yfxerp.com review section 3.1;
 *   - dequantisation fused inside the matmul, never materialised: lqnn.cn
 *     review sections 1.2 and 6.2, kongchang.com page section "Strata快在哪"
 *     (MMQ note);
 *   - activation fused with the FFN projection: yfxerp.com review section 5.1.
 * The pages give no API, formula for the router, tie-break, activation or bit
 * layout; the readings used here are stated at each declaration.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library never allocates or frees device memory; scratch space is the
 *     caller's `ws` buffer of at least strata_moe_workspace_bytes(dims) bytes.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No call synchronises the host, so every call can be captured
 *     in a CUDA graph.
 *   - Arguments are validated on the host before any launch.  On error
 *     nothing is launched and a status is returned; no exception crosses the
 *     ABI and no kernel traps.
 *   - Results are bit-identical from run to run (no floating-point atomics).
 *   - bf16 and fp16 values are passed as their 16-bit patterns (uint16_t).
 *   - Device pointers must be 16-byte aligned.
 *
 * Numerics.  The layer input x and output y are bf16; the intermediates h and
 * the per-row expert outputs are fp16, because fp16 carries the dequantised
 * weights q*s to 2^-11 where bf16 would carry them to 2^-8, and bf16-rounded
 * weights alone use up most of a 1.5e-2 * RMS error budget on these layers.
 *   - router logits: fp32 accumulation of exact bf16 products;
 *   - prefill batches (T > 8): tensor-core MMAs on fp16 operands -- x is
 *     converted to fp16 (exact for |x| < 65504; larger values saturate to
 *     infinity and are reported through strata_moe_device_status), each
 *     weight is RNE_fp16(q * s), products accumulate in fp32;
 *   - decode batches (T <= 8): the integer codes q enter the MMA exactly and
 *     the fp16 group scale multiplies each group's fp32 partial sum;
 *   - h = RNE_fp16(SiLU(g) * u), per-row outputs RNE_fp16(o);
 *   - y = RNE_bf16(sum_j w_j * row_j), summed in fp32 in the order j = 0..k-1.
 */
#ifndef STRATA_MOE_H
#define STRATA_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define STRATA_API __attribute__((visibility("default")))
#else
#define STRATA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status of a call.  STRATA_ERR_DEVICE_CHECK is reported by
 * strata_moe_device_status() when a kernel recorded a failed device-side
 * check (an index out of range, or a bounded wait that ran out). */
typedef enum {
  STRATA_OK = 0,
  STRATA_ERR_INVALID_ARG = 1,  /* null pointer, bad dims, misaligned pointer */
  STRATA_ERR_UNSUPPORTED = 2,  /* valid shape this build does not implement */
  STRATA_ERR_WORKSPACE = 3,    /* ws missing or smaller than required       */
  STRATA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed       */
  STRATA_ERR_DEVICE_CHECK = 5  /* a device-side check failed (see above)     */
} strata_status_t;

/* Layer dimensions.
 *   T      tokens in the batch (T = 0 is a valid empty batch: nothing runs and
 *          no pointer is read, except that strata_moe_permute zeroes counts
 *          and offsets)
 *   d      hidden size (reduction dim of gate/up, output dim of down)
 *   E      number of experts
 *   k      experts per token, 1 <= k <= E
 *   n      expert intermediate size
 *   group  int4 group size along K, for all three projections
 * Supported: d, n multiples of 128; group in {32, 64, 128}; E <= 1024;
 * k <= 32; T*k < 2^31.  Other positive shapes return STRATA_ERR_UNSUPPORTED. */
typedef struct {
  int32_t T, d, E, k, n, group;
} strata_moe_dims_t;

/* One group-quantised weight tensor for all E experts, logical W_e[K][N]
 * (K = reduction dim), stored K-major per output feature:
 *   q: [E][N][K/2] bytes.  Byte q[e][nn][kk/2] holds element kk in its low
 *      nibble when kk is even and in its high nibble when kk is odd; nibbles
 *      are two's-complement int4 in [-8, 7].
 *   s: [E][N][K/group] fp16 scales.
 * Element value: W_e[kk][nn] = q * s[e][nn][kk/group] (symmetric, no zero
 * point).  gate/up: N = n, K = d.  down: N = d, K = n.  The pages describe
 * grouped int4 with per-group scales (lqnn.cn review 3.1; yfxerp.com review
 * 3.1) but no bit layout; this layout is the library's own. */
typedef struct {
  const uint8_t* q;
  const uint16_t* s;
} strata_q4_t;

typedef enum {
  STRATA_OP_GATE_UP_SWIGLU = 0, /* h = SiLU(a . Wg_e) * (a . Wu_e), a = gathered x */
  STRATA_OP_DOWN = 1            /* o = a . Wd_e (times row_scale), a = h rows       */
} strata_moe_op_t;

/* A cudaStream_t without including CUDA headers. */
typedef struct CUstream_st* strata_stream_t;

/* Bytes of caller-provided scratch space that strata_moe_forward needs for
 * `dims` (also enough for every other entry point).  Returns 0 for dims that
 * no entry point accepts. */
STRATA_API size_t strata_moe_workspace_bytes(strata_moe_dims_t dims);

/* Static, NUL-terminated description of a status. */
STRATA_API const char* strata_status_string(strata_status_t status);

/* Router + top-k + softmax ("the router of each layer selects a subset of
 * experts for every token": penglei.dev post, section "原理一").
 *   x         [T][d] bf16, row-major
 *   w_router  [d][E] bf16, row-major
 *   bias      [E] fp32 or NULL; added to the logits before selection, and the
 *             biased logits are the ones softmax weights are computed from
 *   topk_ids  [T][k] int32 out: the k largest logits in descending order;
 *             exactly equal logits go to the lower expert index
 *   topk_w    [T][k] fp32 out: w_j = exp(l_j - l_0) / sum_i exp(l_i - l_0)
 *             over the k selected logits (l_0 the largest)
 *   logits_out [T][E] fp32 out or NULL: the fp32 logits selection used
 *   ws/ws_bytes scratch (see strata_moe_workspace_bytes)
 * Logits are accumulated in fp32 from bf16 products. */
STRATA_API strata_status_t strata_moe_route(const uint16_t* x, const uint16_t* w_router,
                                 const float* bias, strata_moe_dims_t dims,
                                 int32_t* topk_ids, float* topk_w,
                                 float* logits_out, void* ws, size_t ws_bytes,
                                 strata_stream_t stream);

/* Grouping of token slots by expert (tokens that share an expert are
 * processed together: kongchang.com page, section "Strata快在哪", MoE note).
 * Slot s = t*k + j is the j-th expert choice of token t.
 *   topk_ids     [T][k] int32 in: expert of every slot, each in [0, E)
 *   counts       [E] int32 out: number of slots routed to each expert
 *   offsets      [E+1] int32 out: exclusive prefix sum of counts; offsets[E]=T*k
 *   sorted_token [T*k] int32 out: row p -> token; rows of expert e are
 *                offsets[e] .. offsets[e+1]-1 in increasing slot order
 *   slot_row     [T*k] int32 out: slot s -> its row p
 * The output is unique (a stable counting sort); ids outside [0, E) are
 * clamped into range and reported through strata_moe_device_status(). */
STRATA_API strata_status_t strata_moe_permute(const int32_t* topk_ids,
                                   strata_moe_dims_t dims, int32_t* counts,
                                   int32_t* offsets, int32_t* sorted_token,
                                   int32_t* slot_row, void* ws, size_t ws_bytes,
                                   strata_stream_t stream);

/* strata_moe_permute without a caller workspace.  The pages describe no such
 * call: it exists for callers that cannot hand the library device memory --
 * a host program that owns only the five tensors it passes (it has no device
 * allocator of its own to carve a workspace from), or a deployment that
 * budgets every device byte up front and forbids allocation once serving
 * starts.  Such callers get the same result as strata_moe_permute (bit for
 * bit: same kernels, same order) with the per-chunk histogram held in a
 * fixed scratch array compiled into the library, one per device.  Nothing is
 * allocated or freed: no cudaMalloc/cudaFree and no allocating library call,
 * on the first call or later.
 *   Arguments and outputs: as strata_moe_permute, minus ws/ws_bytes.
 *   Limit: the scratch holds STRATA_PERMUTE_STATIC_SCRATCH_INTS int32
 *     values (512 KiB); a call needs ceil(T*k / 1024) * E of them (E = 512:
 *     T*k up to 262144 slots; E = 1024: up to 131072).  Larger inputs return
 *     STRATA_ERR_WORKSPACE before anything is launched.
 *   Zero state: none -- every scratch value a call reads was written earlier
 *     in the same call, so the scratch needs no clearing, and nothing carries
 *     over from one call to the next.
 *   Setup: the first call on each device looks up the scratch's device
 *     address (cudaGetSymbolAddress, with that device current) and caches it;
 *     that lookup may synchronise with the device, so make the first call on
 *     a device before any stream capture begins.
 *   Concurrency: all calls on one device share the one scratch array.  Two
 *     calls in flight at the same time on the same device (different
 *     streams, or different host threads without ordering) race on it and
 *     produce wrong groupings; order them on one stream or with events. */
#define STRATA_PERMUTE_STATIC_SCRATCH_INTS 131072
STRATA_API strata_status_t strata_moe_permute_static(const int32_t* topk_ids,
                                          strata_moe_dims_t dims, int32_t* counts,
                                          int32_t* offsets, int32_t* sorted_token,
                                          int32_t* slot_row, strata_stream_t stream);

/* Grouped expert projection with int4 dequantisation fused into the GEMM
 * (dequantise inside the matmul: lqnn.cn review 1.2 / 6.2; expert matmul is
 * the heaviest compute: kongchang.com page, "Strata快在哪"; activation fused
 * with the projection: yfxerp.com review 5.1).
 *   op = STRATA_OP_GATE_UP_SWIGLU:
 *     a      [T][d] bf16 token rows (x); row p reads a[sorted_token[p]]
 *     w0, w1 gate and up weights (N = n, K = d)
 *     out    [T*k][n] fp16: out[p] = SiLU(a.Wg_e) * (a.Wu_e), e = expert of p
 *     row_scale must be NULL
 *   op = STRATA_OP_DOWN:
 *     a      [T*k][n] fp16 rows in grouped order (the gate/up output)
 *     sorted_token ignored (may be NULL); w0 = down weights (N = d, K = n);
 *     w1 ignored
 *     row_scale [T*k] fp32 or NULL: out[p] is multiplied by row_scale[p]
 *     out    [T*k][d] fp16
 *   offsets [E+1] int32: row ranges per expert, as from strata_moe_permute;
 *     offsets that are not non-decreasing from 0 to T*k are reported through
 *     strata_moe_device_status() and nothing is computed
 * Products accumulate in fp32 (see Numerics above). */
STRATA_API strata_status_t strata_moe_expert_gemm_q4(
    strata_moe_op_t op, const uint16_t* a, const int32_t* sorted_token,
    const int32_t* offsets, strata_q4_t w0, strata_q4_t w1,
    const float* row_scale, strata_moe_dims_t dims, uint16_t* out, void* ws,
    size_t ws_bytes, strata_stream_t stream);

/* Weighted combine back to token order:
 *   y[t] = sum_{j=0..k-1} topk_w[t][j] * rows[slot_row[t*k+j]]
 * summed in fp32 in the order j = 0..k-1 and rounded once to bf16.
 *   rows     [T*k][d] fp16 (per-row expert outputs, grouped order)
 *   topk_w   [T][k] fp32, or NULL when the rows are already weighted
 *   slot_row [T*k] int32
 *   y        [T][d] bf16 out */
STRATA_API strata_status_t strata_moe_combine(const uint16_t* rows, const float* topk_w,
                                   const int32_t* slot_row,
                                   strata_moe_dims_t dims, uint16_t* y,
                                   strata_stream_t stream);

/* The whole layer: route -> permute -> gate/up -> down -> combine, stream
 * ordered, all intermediates in `ws`.
 *   x [T][d] bf16, w_router [d][E] bf16, bias [E] fp32 or NULL
 *   gate, up (N = n, K = d), down (N = d, K = n): int4 weights as above
 *   y [T][d] bf16 out
 *   topk_ids_out [T][k] int32 / topk_w_out [T][k] fp32: optional copies of
 *   the routes (NULL = not written) */
STRATA_API strata_status_t strata_moe_forward(const uint16_t* x, const uint16_t* w_router,
                                   const float* bias, strata_q4_t gate,
                                   strata_q4_t up, strata_q4_t down,
                                   strata_moe_dims_t dims, uint16_t* y,
                                   int32_t* topk_ids_out, float* topk_w_out,
                                   void* ws, size_t ws_bytes,
                                   strata_stream_t stream);

/* Row gather for the expert-parallel exchange (no counterpart on the pages):
 *   dst[i] = src[index[i]],  i < rows, rows of `width` 16-bit values (bf16 or
 *   fp16 bit patterns; width a multiple of 8)
 *   src [src_rows][width], index [rows] int32, dst [rows][width]
 * An index outside [0, src_rows) is reported through
 * strata_moe_device_status() and reads row 0. */
STRATA_API strata_status_t strata_moe_gather_rows(const uint16_t* src, const int32_t* index,
                                       int32_t src_rows, int32_t rows, int32_t width,
                                       uint16_t* dst, strata_stream_t stream);

/* Attention over the KV-cache rows an indexer selected.  The pages' model
 * picks about 2000 positions per query with an indexer, and Strata's kernel
 * reads only the selected KV-cache rows where llama.cpp builds a full mask
 * and runs dense flash attention (kongchang.com "两天移植，预填充提速8倍：
 * Strata引擎实测", section "Strata快在哪", attention paragraph).  For query
 * token t and query head h, with KV head hk = h / (Hq / Hkv):
 *   o[t][h] = sum_p softmax_p(scale * q[t][h] . K[p][hk]) V[p][hk],
 *             p over idx[t][0..P) with slots of -1 unused
 *   T   query tokens            L    KV-cache rows
 *   Hq  query heads             Hkv  KV heads (Hq % Hkv == 0, Hq / Hkv <= 16)
 *   D   head size (64 or 128)   P    index slots per query (<= 65536)
 *   q [T][Hq][D] bf16, k_cache / v_cache [L][Hkv][D] bf16, idx [T][P] int32,
 *   out [T][Hq][D] bf16; scale <= 0 means 1 / sqrt(D)
 * Scores, softmax and the weighted sum in fp32; one rounding to bf16.  A
 * query with no selected row gets zeros.  An index >= L is reported through
 * strata_moe_device_status() and skipped.  The pages fix no head counts,
 * head size or index format; these are this library's readings. */
typedef struct {
  int32_t T, L, Hq, Hkv, D, P;
} strata_attn_dims_t;
STRATA_API size_t strata_sparse_attention_workspace_bytes(strata_attn_dims_t dims);
STRATA_API strata_status_t strata_sparse_attention(const uint16_t* q, const uint16_t* k_cache,
                                        const uint16_t* v_cache, const int32_t* idx,
                                        strata_attn_dims_t dims, float scale, uint16_t* out,
                                        void* ws, size_t ws_bytes, strata_stream_t stream);

/* Synchronises `stream`, then reports (and clears) the device-side check word
 * of the current device: STRATA_OK, or STRATA_ERR_DEVICE_CHECK when a kernel
 * since the last call recorded an out-of-range index or a bounded wait that
 * timed out.  This is the one entry point that blocks the host. */
STRATA_API strata_status_t strata_moe_device_status(strata_stream_t stream);

/* Diagnostic: drives the library's bounded waits into their time limit on
 * purpose and lets them give up, so that callers (and the tests) can see the
 * failure path work on their device.  The pages have no counterpart; every
 * wait in the kernels above is bounded in the same way (about one second),
 * after which the kernel records a time-out in the device check word,
 * releases what it holds and returns instead of spinning forever.
 *   out      device int32[10] (16-byte aligned), written by the kernels:
 *            out[0..3]  1 if wait w completed, 0 if it gave up (an mbarrier
 *                       that nothing arrives on; warp 0 waits alone, warps
 *                       1..3 wait as whole warps and see warp 0's abort;
 *                       warp 1 holds 32 columns of tensor memory meanwhile)
 *            out[4]     nanoseconds warp 0 waited before giving up
 *            out[5]     1 once warp 1 released its tensor memory
 *            out[6]     1 if a two-CTA grid barrier that one CTA never
 *                       reaches completed, 0 if it gave up
 *            out[7]     nanoseconds that barrier waited
 *            out[8]     1 if a wait for a count of finished work that
 *                       nothing raises (the form the fused decode kernel
 *                       uses between its phases) completed, 0 if it gave up
 *            out[9]     nanoseconds that wait took
 *   sync_ws  device scratch of 32 bytes (16-byte aligned), overwritten
 * Both kernels take about one second each.  Afterwards
 * strata_moe_device_status() reports STRATA_ERR_DEVICE_CHECK (and clears it);
 * the device stays usable. */
STRATA_API strata_status_t strata_moe_selftest_wait(int32_t* out, void* sync_ws,
                                         strata_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* STRATA_MOE_H */
