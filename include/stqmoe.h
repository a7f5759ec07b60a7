/*
 * stqmoe.h - C ABI of libstqmoe.so: the routed-expert FFN of one MoE layer over
 * packed low-bit expert weights, on one NVIDIA B200 (sm_100a).
 *
 * Two weight formats (the problem as the pages state it):
 *
 *  STQ1_0  3:4 sparse ternary.  "Hy4-preview-GGUF", section 3 "STQ1_0 and the
 *          mixed-precision strategy": weights {-d, 0, +d}, exactly one zero per
 *          four lanes, one FP16 scale per 256 weights, 42 bytes per 256 weights
 *          (1.3125 bpw).  "Hy4-preview-FlashMoE-STQ1_0", "How the STQ1_0 packing
 *          works": 64 four-weight groups per block, 4 x 2^3 = 32 patterns, five
 *          bits each.  The byte layout is this library's own (GGML type 43's
 *          literal codebook is not given on the pages; no byte compatibility is
 *          claimed):
 *            pattern c = 8*z + s: z = zero lane, bit n of s = sign of the n-th
 *            non-zero lane counted upward (1 = negative); weight = d * (0 | +-1);
 *            group j of 256-block b covers k = 256*b + 4*j + lane.
 *            Matrix [rows, K] (rows % 16 == 0, K % 256 == 0) = tiles of 16 rows,
 *            each tile = K/256 tile-blocks of 672 bytes (16 rows x 42 bytes):
 *              [0,32)    word g (g=0..7) = fp16 d(row g) | fp16 d(row g+8) << 16
 *              [32,544)  lane L: words 0..3 of its 160-bit code stream at 32+16L
 *              [544,672) lane L: word 4 at 544+4L
 *            lane L = 4g+t holds rows g, g+8 and groups j = 16t+s (s = 0..15);
 *            code i = 2s+h (row g+8h) sits at stream bits [5i, 5i+5).
 *  MXFP4 x MXFP8 ("W4A8").  "Hy4-preview-SF-WFP4AFP8", "Quant Diff": routed
 *          experts are FP4 E2M1 weights with FP8 E4M3 activations, group 32,
 *          UE8M0 scales.  Weights [rows, K]: codes [rows][K/2] (element 2i in the
 *          low nibble) + scales [rows][K/32]; activations: codes [rows][K] +
 *          scales [rows][K/32].  Element encodings follow the OCP MX spec.
 *
 * Conventions (every entry point):
 *  - Pointers named in the argument lists are DEVICE pointers owned by the
 *    caller, unless the name ends in _host.  The library allocates nothing and
 *    frees nothing.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream) and return
 *    after enqueueing.  Argument errors are detected on the host before any
 *    launch; on error nothing is launched and outputs are untouched.
 *  - Device-side data errors (non-finite weights in a pack, an expert id out of
 *    range, a bounded wait that ran out) are recorded in a caller-owned device
 *    int32 "error word" (first error wins); read it with stq_read_error().
 *  - Device pointers must be 16-byte aligned; sizes are element counts.
 *  - Not thread-safe per workspace / error word.
 */
#ifndef STQMOE_H
#define STQMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* stq_stream_t; /* same type as cudaStream_t */
typedef int32_t stq_status;

enum {
  STQ_OK = 0,
  STQ_ERR_INVALID_ARG = -1, /* null pointer, bad enum, negative size */
  STQ_ERR_SHAPE = -2,       /* K % 256 (STQ1_0), K % 32 (MX), rows % 16, H/I mismatch */
  STQ_ERR_ALIGN = -3,       /* a device pointer is not 16-byte aligned */
  STQ_ERR_NONFINITE = -4,   /* pack: NaN/Inf weight, or an STQ block amax above 65504 */
  STQ_ERR_CUDA = -5,        /* a CUDA runtime call failed (launch, attribute) */
  STQ_ERR_DEVICE = -6,      /* device-detected: expert id out of range */
  STQ_ERR_WORKSPACE = -7,   /* workspace smaller than moe_workspace_bytes() */
  STQ_ERR_TIMEOUT = -8,     /* device-detected: a bounded wait ran out */
  STQ_ERR_UNSUPPORTED = -9  /* valid request this build does not implement */
};

/* Human-readable name of a status code (static string). */
const char* stq_status_string(stq_status s);

/* ABI version of this header (bumped on any signature or layout change). */
#define STQMOE_ABI_VERSION 2
int32_t stq_abi_version(void);

/* Synchronise `stream`, return the error word's value and reset it to 0.
 * `err` is a device int32.  Returns STQ_ERR_CUDA if the synchronisation fails. */
stq_status stq_read_error(int32_t* err, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Packing.  Sources: "Hy4-preview-GGUF" section 3 (upstream quantiser: d = amax, */
/* zero the lane of smallest |w|) for STQ1_0; "Hy4-preview-SF-WFP4AFP8", "Quant   */
/* Diff" for MXFP4 (E2M1 g32, UE8M0).                                             */
/* ------------------------------------------------------------------------- */

/* w: float32 [rows, K] row-major -> out: rows*K/256*42 bytes in the STQ1_0 layout
 * above.  Per 256-block d = fp16_rne(max |w|); per group the zero goes to the
 * first lane of smallest |w|, the other lanes keep sign(w).  d == 0 gives all
 * codes 0.  Exact (pack(unpack(b)) == b) on canonical bytes.  A NaN/Inf weight or
 * a block amax > 65504 sets STQ_ERR_NONFINITE in *err (err may be NULL).
 * rows % 16 == 0, K % 256 == 0. */
stq_status stq1_pack(const float* w, int64_t rows, int64_t K, uint8_t* out,
                     int32_t* err, stq_stream_t stream);

/* The same bytes from the least-squares encoder ("Hy4-preview-GGUF", section 3, "Our
 * encoder"): per 256-block of a row, starting from d = max |w|, three rounds of
 *   1. per group, the zero on the lane j of least v_j * (w_j^2 - (|w_j| - d)^2) (first
 *      lane on ties), the other lanes keeping sign(w);
 *   2. d = sum(v |w|) / sum(v) over the kept lanes (0 if that sum of v is 0);
 * then d is stored as fp16_rne (d == 0: all codes 0).  v = importance[k] per column k
 * (float32 [K], >= 0, e.g. an importance matrix's column weights; NULL = all 1).  The
 * costs and sums are FP64 with explicit roundings, the scale rounded directly from FP64
 * to FP16.  A NaN/Inf weight or a block amax > 65504 sets STQ_ERR_NONFINITE, a negative
 * or non-finite importance STQ_ERR_INVALID_ARG, in *err (may be NULL).  Pointers are
 * device pointers, 16-byte aligned; rows % 16 == 0, K % 256 == 0; rows == 0 or K == 0
 * is a no-op (pointers may then be NULL). */
stq_status stq1_pack_ls(const float* w, const float* importance, int64_t rows, int64_t K,
                        uint8_t* out, int32_t* err, stq_stream_t stream);

/* STQ1_0 bytes -> float32 [rows, K]: +-d on non-zero lanes (sign applied to d),
 * +0 on the zero lane.  Bit-exact. */
stq_status stq1_unpack(const uint8_t* in, int64_t rows, int64_t K, float* w,
                       stq_stream_t stream);

/* w: float32 [rows, K] -> codes [rows, K/2], scales [rows, K/32].  Per 32 along
 * K: e = clamp(k + 127, 0, 254) with k the smallest integer such that
 * max|w| <= 6 * 2^k (e = 127 for an all-zero group); codes = E2M1 round to
 * nearest even of w * 2^-k, sign of w kept (-0 -> code 8).  NaN/Inf weights set
 * STQ_ERR_NONFINITE in *err.  K % 32 == 0. */
stq_status mxfp4_pack(const float* w, int64_t rows, int64_t K, uint8_t* codes,
                      uint8_t* scales, int32_t* err, stq_stream_t stream);

/* codes/scales -> float32 [rows, K] = e2m1(code) * 2^(e-127) rounded to binary32
 * (overflow -> +-inf; e = 255 -> NaN).  Bit-exact. */
stq_status mxfp4_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                        int64_t K, float* w, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Activation quantisation BF16 -> MXFP8 (E4M3 g32, UE8M0).  Source: the       */
/* "Hy4-preview-SF-WFP4AFP8" recipe (weight_fp4_activation_fp8, group 32,      */
/* ue8m0 / e4m3); scale rule: smallest power of two putting the group amax     */
/* <= 448.                                                                      */
/* ------------------------------------------------------------------------- */

/* x: bf16 bits [rows, K] -> codes [rows, K], scales [rows, K/32].  e as for MXFP4
 * with 448 in place of 6; codes = E4M3 RNE of x * 2^-k including subnormals, sign
 * kept (negative values that round to zero give 0x80).  A group holding NaN/Inf
 * gets e = 255 and codes 0x7F.  Bit-exact.  K % 32 == 0. */
stq_status mxfp8_quantize_bf16(const uint16_t* x, int64_t rows, int64_t K,
                               uint8_t* codes, uint8_t* scales, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Single-matrix products (the two single-matrix workloads).                  */
/* ------------------------------------------------------------------------- */

/* y[n, r] = sum_k W[r, k] x[n, k] (FP32 accumulate) for an STQ1_0 matrix W
 * [rows, K] and bf16 activations x [n, K]; y float32 [n, rows].  Tolerance
 * |y - y_ref| <= 1e-3 * sum_k |W x| + 1e-5.  rows % 16 == 0, K % 256 == 0.
 * n == 0 or rows == 0 is a no-op (pointers may then be NULL). */
stq_status stq1_gemv(const uint8_t* W, int64_t rows, int64_t K, const uint16_t* x,
                     int64_t n, float* y, stq_stream_t stream);

/* y[m, n] = sum_k a[m, k] w[n, k] for MXFP4 weights w [N, K] and MXFP8
 * activations a [M, K] (tcgen05 block-scaled MMA, FP32 accumulate); y float32
 * [M, N].  `err` (device int32, may be NULL) records STQ_ERR_TIMEOUT if a
 * pipeline wait ran out.  N % 128 == 0, K % 128 == 0. */
stq_status w4a8_gemm(const uint8_t* w_codes, const uint8_t* w_scales, int64_t N,
                     int64_t K, const uint8_t* a_codes, const uint8_t* a_scales,
                     int64_t M, float* y, int32_t* err, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* MoE layer.  Shapes: "Hy4-preview-FlashMoE-STQ1_0", "Package details"        */
/* (hidden 6144, MoE intermediate 2048, 256 routed experts, top-8, 1 shared).  */
/* ------------------------------------------------------------------------- */

enum { STQ_FMT_STQ1_0 = 0, STQ_FMT_MXFP4 = 1 };

/* Router: logits = x Wr^T (FP32 accumulate), softmax over E, top-k by
 * probability (ties -> lower id), weights renormalised over the k chosen.
 * x bf16 [T, H], w_router bf16 [E, H] -> topk_ids int32 [T, k], topk_w f32 [T, k].
 * logits: caller-owned f32 scratch of stq_router_ksplit(H) * T * E floats (the
 * logits are summed over that many slices of H); on return its first T*E floats
 * hold the logits [T, E].  A non-finite logit counts as probability 0 (a token whose
 * chosen probabilities are all 0 gets weights 1/k).  E <= 1024, k <= 32, k <= E,
 * H % 256 == 0.  T == 0 is a no-op (pointers may then be NULL). */
int32_t stq_router_ksplit(int32_t H);
stq_status moe_router_topk(const uint16_t* x, const uint16_t* w_router, int32_t T,
                           int32_t H, int32_t E, int32_t k, float* logits,
                           int32_t* topk_ids, float* topk_w, stq_stream_t stream);

/* Token-to-expert grouping (the step every expert launch reads).  Pairs are
 * p = t*k + slot.  counts [E]; offsets [E+1] = exclusive scan of counts;
 * perm [P] = pair at each sorted position, sorted by expert and stably by p;
 * inv [P] = sorted position of each pair (-1 for an id outside [0, E), which
 * also sets STQ_ERR_DEVICE in *err); tlist [E] = touched experts in ascending
 * order, ntouched [1] their number.  Integer, exact.  E <= 1024, T*k < 2^30
 * (else STQ_ERR_INVALID_ARG). */
stq_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E,
                       int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                       int32_t* tlist, int32_t* ntouched, int32_t* err,
                       stq_stream_t stream);

/* Router without a scratch argument (no counterpart on the pages; a convenience of
 * this library).  Same result as moe_router_topk, for callers that cannot allocate
 * device memory for scratch: code that must not call cudaMalloc (for instance a
 * host program whose device memory is all owned by its own pool, or one that runs
 * where allocation is not allowed) and so has no buffer to pass as `logits`.
 * The logits' partial sums go to a fixed 2 MiB array inside the library instead,
 * one per GPU that loads the library, held until the process exits.  Limit:
 * stq_router_ksplit(H) * T * E <= 524288 (e.g. T <= 256 for H = 6144, E = 256);
 * larger requests return STQ_ERR_WORKSPACE before any launch.  Every call looks up
 * the array's device address on the current device (cudaGetSymbolAddress); the first
 * call on a device may also load the library's module there, so make that first call
 * before any stream capture.
 * Every call shares the array and leaves its last contents there (each call
 * writes every entry it reads, so nothing needs clearing); calls whose kernels
 * overlap on the GPU (other streams, other host threads) race on it.  Allocates
 * nothing.  Outputs: topk_ids int32 [T, k], topk_w f32 [T, k].  T == 0 is a no-op
 * (pointers may then be NULL). */
stq_status moe_router_topk_static(const uint16_t* x, const uint16_t* w_router,
                                  int32_t T, int32_t H, int32_t E, int32_t k,
                                  int32_t* topk_ids, float* topk_w, stq_stream_t stream);

/* Format of the shared expert (moe_weights.sh_fmt).
 *   STQ_SHARED_BF16   sh_gate / sh_up / sh_down are bf16 matrices; h is rounded to bf16.
 *                     In the STQ1_0 decode regime its tiles are extra work items of the
 *                     routed GEMV kernels; otherwise (MXFP4 experts, STQ1_0 prefill regime)
 *                     it runs on the library-owned side stream described below.
 *   STQ_SHARED_MXFP8  "Hy4-preview-SF-WFP4AFP8", "Quant Diff": the shared experts'
 *                     gate/up/down are MXFP8 W8A8 g32.  sh_* are E4M3 codes (one byte
 *                     per weight, row-major) and sh_*_sc their UE8M0 scales [rows][K/32]
 *                     (as written by mxfp8_quantize_bf16); x and h are quantised to
 *                     MXFP8 g32 (the activation rule of mxfp8_quantize_bf16) and the
 *                     products accumulate in FP32.  The shared expert depends on x alone, so
 *                     moe_expert_forward runs it on a library-owned stream of the
 *                     current device (created with two events on first use, then
 *                     reused; not device memory), forked from `stream` after the
 *                     call's argument checks and joined back before the combine; the
 *                     call stays ordered on `stream` and can be captured into a graph.
 *                     Calls on one device share that stream: a lock keeps one call's
 *                     launches on it from interleaving with another's, each host thread
 *                     forks and joins through its own pair of events (so a call waits
 *                     for its own shared expert only), and calls from several host
 *                     threads run their shared experts one after another.  A call while
 *                     another thread is capturing such a call into a graph is not
 *                     supported. */
enum { STQ_SHARED_BF16 = 0, STQ_SHARED_MXFP8 = 1 };

typedef struct {
  int32_t fmt;              /* STQ_FMT_STQ1_0 or STQ_FMT_MXFP4 (routed experts) */
  const uint8_t* gate;      /* E matrices [I, H], expert-major, contiguous      */
  const uint8_t* up;        /* E matrices [I, H]                                 */
  const uint8_t* down;      /* E matrices [H, I]                                 */
  const uint8_t* gate_sc;   /* MXFP4 scales, E x [I, H/32]; NULL for STQ1_0      */
  const uint8_t* up_sc;     /* E x [I, H/32]                                     */
  const uint8_t* down_sc;   /* E x [H, I/32]                                     */
  const void* sh_gate;      /* shared expert [I, H] (sh_fmt); NULL = no shared   */
  const void* sh_up;        /* [I, H]                                            */
  const void* sh_down;      /* [H, I]                                            */
  int32_t sh_fmt;           /* STQ_SHARED_BF16 (0) or STQ_SHARED_MXFP8           */
  const uint8_t* sh_gate_sc;  /* MXFP8 scales [I, H/32]; NULL for BF16           */
  const uint8_t* sh_up_sc;    /* [I, H/32]                                       */
  const uint8_t* sh_down_sc;  /* [H, I/32]                                       */
} moe_weights;

/* Kernels for STQ1_0 routed experts (moe_desc.regime; MXFP4 experts have one path).
 *   STQ_REGIME_AUTO     prefill when T*k >= 32 * min(E, T*k) (32 or more routed tokens
 *                       per expert on average), else decode;
 *   STQ_REGIME_DECODE   the decode GEMV: BF16 activations times the ternary patterns,
 *                       FP32 accumulation, d per 256-block, h rounded to BF16;
 *   STQ_REGIME_PREFILL  the tensor-core GEMM ("Hy4-preview-SF-WFP4AFP8": activations
 *                       FP8 E4M3 g32 with UE8M0 scales): x quantised to MXFP8 g32, the
 *                       patterns as E4M3 +-1/0 with a unit scale (kind::mxf8f6f4), each
 *                       256-block's FP32 partial times d, h re-quantised to MXFP8 g32. */
enum { STQ_REGIME_AUTO = 0, STQ_REGIME_DECODE = 1, STQ_REGIME_PREFILL = 2 };

typedef struct {
  int32_t T, H, I, E, k;    /* tokens, hidden, intermediate, experts, top-k;
                               T >= 0, E <= 1024, 1 <= k <= min(32, E), T*k < 2^30 */
  int32_t out_fp32;         /* 1: y is float32 [T, H]; 0: y is bf16 [T, H]      */
  int32_t add_residual;     /* 1: y += x                                         */
  int32_t regime;           /* STQ_REGIME_* (STQ1_0 experts)                     */
  int32_t norm_out;         /* 1: y = RMSNorm(y) after the residual: unit gain,
                               y / sqrt(mean(y^2) + norm_eps) per token row over the
                               bf16-rounded y, the same bits as stq_rmsnorm_bf16 on
                               the unnormalised output; requires out_fp32 = 0      */
  float norm_eps;           /* eps of norm_out, finite and >= 0                  */
} moe_desc;

/* Bytes of device workspace moe_expert_forward needs for `d` (256-byte aligned
 * regions; the first int32 is the error word). 0 on an invalid descriptor. */
size_t moe_workspace_bytes(const moe_desc* d);

/* y[t] = sum_s topk_w[t,s] * FFN_{topk_ids[t,s]}(x[t]) + FFN_shared(x[t]) (+ x[t])
 * with FFN_e(x) = W_down,e (silu(W_gate,e x) * (W_up,e x)).  The intermediate h is
 * rounded to bf16 (STQ1_0 decode regime and the BF16 shared expert) or re-quantised
 * to MXFP8 (MXFP4 experts, the STQ1_0 prefill regime and the MXFP8 shared expert,
 * whose input x is quantised to MXFP8 first).  In the STQ1_0 decode regime an expert
 * with at most two routed tokens (when the layer averages at most two per expert)
 * multiplies its activations (x, then h) as a fixed-point value per 256-k block, 22 bits
 * below the block's largest bf16 exponent: exact for every element within 2^14 of the
 * block's largest magnitude, an error of at most 2^-22 of it otherwise; its sums are
 * exact integers per block, scaled in FP32.  Slots are summed in order
 * s = 0..k-1, without atomics.  Duplicate ids in a token are separate slots; an
 * id outside [0, E) sets STQ_ERR_DEVICE in the workspace error word and its slot
 * contributes 0.  workspace: >= moe_workspace_bytes(d) bytes, 256-B aligned. */
stq_status moe_expert_forward(const moe_desc* d, const uint16_t* x,
                              const int32_t* topk_ids, const float* topk_w,
                              const moe_weights* w, void* y, void* workspace,
                              size_t ws_bytes, stq_stream_t stream);

/* Byte offset, inside the workspace of `d`, of one intermediate region, so that
 * callers (and the parity tests) can inspect each stage:
 *   STQ_WS_COUNTS, _OFFSETS, _PERM, _INV, _TLIST, _NTOUCHED: as moe_permute;
 *   STQ_WS_H   bf16 [(P+T), I]: h of routed pairs (sorted order), then shared tokens;
 *   STQ_WS_Y   f32  [(P+T), H]: expert outputs, same row order (unweighted);
 *   STQ_WS_XQ/_XS  MXFP8 of x [(P+T), H] / [(P+T), H/32]: routed pairs in sorted
 *                  order (MXFP4 layers, STQ1_0 prefill regime), then the T tokens
 *                  (MXFP8 shared expert);
 *   STQ_WS_HQ/_HS  MXFP8 of h [(P+T), I] / [(P+T), I/32], same row order.
 * P = T*k.  Returns (size_t)-1 for an invalid descriptor or region. */
enum { STQ_WS_COUNTS = 0, STQ_WS_OFFSETS, STQ_WS_PERM, STQ_WS_INV, STQ_WS_TLIST,
       STQ_WS_NTOUCHED, STQ_WS_H, STQ_WS_Y, STQ_WS_XQ, STQ_WS_XS, STQ_WS_HQ, STQ_WS_HS };
size_t moe_workspace_offset(const moe_desc* d, int32_t region);

/* Synchronise `stream`, return the workspace's error word (0 = none) and clear it. */
stq_status moe_get_device_error(void* workspace, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Layer stacking                                                            */
/* ------------------------------------------------------------------------- */

/* RMS normalisation of bf16 rows with unit gain:
 *   y[t, :] = bf16_RNE( x[t, :] * 1 / sqrt(mean_j x[t, j]^2 + eps) ).
 * The pages' stacked decode ("Hy4-preview-FlashMoE-STQ1_0", "Package details":
 * consecutive MoE layers with a residual add between them) names no normalisation;
 * without one, eight layers of random SwiGLU experts grow the residual stream past
 * the FP32 range.  This library's reading puts one RMS normalisation after each
 * layer's residual add (the next layer's input is stq_rmsnorm_bf16 of the previous
 * layer's output).  Sum of squares, mean, scale and product in FP64 (fixed
 * summation order: deterministic), rounded to FP32 and then to bf16; x, y bf16 [T, H] row-major, device, 16-byte aligned, caller-owned;
 * y == x (in place) allowed.  H % 8 == 0; T == 0 is a no-op; eps >= 0 finite.  A row
 * with a non-finite element gives non-finite outputs.  One kernel launch. */
stq_status stq_rmsnorm_bf16(const uint16_t* x, int64_t T, int64_t H, float eps,
                            uint16_t* y, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Expert slot bank ("Hy4-preview-FlashMoE-STQ1_0", running with a slot bank:   */
/* routed experts stay outside HBM and are read on demand into a fixed number   */
/* of slots; a miss reads its expert in; at least top-k slots).  Host side.     */
/* ------------------------------------------------------------------------- */

/* Opaque host object: which expert each of n_slots slots holds, and when each slot was last
 * used.  Replacement (not stated on the pages): the least recently used slot among those
 * the current call does not need, ties to the lowest slot index. */
typedef struct stq_slot_bank stq_slot_bank;

/* New empty bank for experts [0, n_experts) in n_slots slots (1 <= n_slots <= n_experts);
 * NULL on invalid arguments or allocation failure.  Host memory only; not thread-safe. */
stq_slot_bank* stq_slot_bank_create(int32_t n_experts, int32_t n_slots);
void stq_slot_bank_destroy(stq_slot_bank* bank);

/* Map the routed expert ids of one call (host int32 [n], e.g. topk_ids of T tokens x k) to
 * slots: slot_ids (host int32 [n]) gets the slot that holds ids[i] after the call; the
 * experts that were not resident are listed in first-use order in load_expert / load_slot
 * (host int32, capacity n_slots), *n_loads of them: the caller copies those experts into
 * those slots (stq_slot_bank_copy) before running moe_expert_forward with E = n_slots and
 * the slot ids as topk_ids.  Errors (bank unchanged): STQ_ERR_INVALID_ARG for an id outside
 * [0, n_experts) or a call touching more distinct experts than there are slots. */
stq_status stq_slot_bank_map(stq_slot_bank* bank, const int32_t* ids, int64_t n, int32_t* slot_ids,
                             int32_t* load_expert, int32_t* load_slot, int32_t* n_loads);

/* The expert held by each slot (host int32 [n_slots], -1 = empty). */
stq_status stq_slot_bank_resident(const stq_slot_bank* bank, int32_t* slot_expert);

/* Copy the listed experts' matrices into their slots: for load i and matrix m,
 * mat_bytes[m] bytes from src[m] + load_expert[i] * mat_bytes[m] (the full expert-major
 * array of the bank's n_experts matrices, normally pinned host memory so the copy is
 * asynchronous) to dst[m] + load_slot[i] * mat_bytes[m] (the slot array of its n_slots
 * matrices, device memory).  One cudaMemcpyAsync per load and matrix on `stream`;
 * asynchronous.  STQ_ERR_INVALID_ARG (nothing enqueued) for null pointers or an expert or
 * slot index outside the bank's sizes; STQ_ERR_CUDA if a copy cannot be enqueued. */
stq_status stq_slot_bank_copy(const stq_slot_bank* bank, const int32_t* load_expert, const int32_t* load_slot,
                              int32_t n_loads, int32_t n_mats, const void* const* src, void* const* dst,
                              const size_t* mat_bytes, stq_stream_t stream);

/* ------------------------------------------------------------------------- */
/* Instrumentation (no counterpart on the pages).                             */
/* ------------------------------------------------------------------------- */

/* Self-test of the bounded waits: one CTA waits, through the same bounded mbarrier
 * wait the tensor-core kernels use, on a barrier that nothing arrives at.  After the
 * limit (about two seconds of GPU clock) the wait gives up, STQ_ERR_TIMEOUT is recorded
 * in *err (device int32, caller-owned; first error wins) and the kernel returns, so the
 * context stays usable.  Asynchronous on `stream`. */
stq_status stq_wait_selftest(int32_t* err, stq_stream_t stream);

/* Kernel kinds reported by the timing hook. */
enum { STQ_K_ROUTER_LOGITS = 0, STQ_K_ROUTER_TOPK, STQ_K_PERMUTE, STQ_K_QUANT_X,
       STQ_K_GATE_UP, STQ_K_DOWN, STQ_K_COMBINE, STQ_K_GEMV, STQ_K_GEMM,
       STQ_K_GATE_UP_MX, STQ_K_DOWN_MX, STQ_K_PLAN, STQ_K_SHARED_GATE_UP, STQ_K_SHARED_DOWN,
       STQ_K_RMSNORM, STQ_K_PACK_LS, STQ_K_GATE_UP_STQ_TC, STQ_K_DOWN_STQ_TC, STQ_K_ACT_LIMBS, STQ_K_COUNT };

/* Caller-owned host struct.  While installed, every kernel launched by
 * moe_router_topk, moe_router_topk_static, moe_expert_forward, stq1_gemv, w4a8_gemm,
 * stq_rmsnorm_bf16 and stq1_pack_ls is bracketed by event records of events[2n] / events[2n+1] on the
 * stream it runs on (inside stream capture as external event-record nodes of the
 * graph), kinds[n] is set to its STQ_K_* kind and n = count++ (until capacity pairs
 * are used).  events: cudaEvent_t[2*capacity] created with timing.  Process-wide, not
 * thread-safe; NULL uninstalls.  Used by the benchmark to time each kernel on its own
 * stream. */
typedef struct {
  void* const* events;
  int32_t capacity;
  int32_t* kinds;
  int32_t count;
} stq_timing;
stq_status stq_set_timing(stq_timing* t);

/* 1 for the checked build (libstqmoe_checked.so, compiled with -DSTQ_CHECKED=1), 0 otherwise.
 * The checked build has the same ABI; its kernels re-check every index they take from data
 * (expert ids of the touched list, token indices from the permutation, sorted positions from
 * the inverse map, gathered source rows) and, instead of using a bad one, record
 * STQ_ERR_DEVICE in the error word and skip the access. */
int32_t stq_checked_build(void);

/* Name of an STQ_K_* kind ("gate_up", "down_mx", ...; "unknown" outside the enum).  Static
 * storage.  Every kernel launch of the calls listed above is also wrapped in an NVTX range
 * of this name (host side, whether or not timing is installed), so a profiler can select
 * kernels by it (ncu --nvtx --nvtx-include "gate_up/"). */
const char* stq_kernel_kind_name(int32_t kind);

#ifdef __cplusplus
}
#endif

#endif /* STQMOE_H */
