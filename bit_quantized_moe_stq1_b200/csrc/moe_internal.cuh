// Internal structures shared by the MoE translation units (not part of the ABI).
#pragma once

#include "common.cuh"

struct MoeWsLayout {
  size_t err, counts, offsets, tlist, ntouched, perm, inv, h, Y, xq, xs, hq, hs, xl, xls, hl, hls, ntiles, n_ntiles,
      sched, chist, total;
};

// Device pointers into the caller's workspace.
struct MoeWs {
  int32_t* err;
  int32_t* counts;
  int32_t* offsets;
  int32_t* tlist;
  int32_t* ntouched;
  int32_t* perm;
  int32_t* inv;
  uint16_t* h;   // [(P+T), I] bf16: routed pairs (sorted order) then shared-expert tokens
  float* Y;      // [(P+T), H] fp32
  uint8_t* xq;   // [(P+T), H] MXFP8 codes of x: routed pairs in sorted order, then the tokens
  uint8_t* xs;   // [(P+T), H/32]
  uint8_t* hq;   // [(P+T), I] MXFP8 codes of h, same rows
  uint8_t* hs;   // [(P+T), I/32]
  int8_t* xl;    // [T][3][H] activation limbs of x (integer decode GEMV)
  float* xls;    // [T][stq_limb_scale_pitch(H/256)] their block scales, one row per limb
  int8_t* hl;    // [P][3][I] limbs of the routed rows of h
  float* hls;    // [P][stq_limb_scale_pitch(I/256)]
  int2* ntiles;  // [P/16 + E] (expert, first token) of each GEMM N tile
  int32_t* n_ntiles;
  int32_t* sched;  // [4] work counters of the persistent GEMV kernels: 0-2 zeroed by the permute
                   // kernel, 3 (the shared expert's down launch) by the shared gate/up kernel
  int32_t* chist;  // [ceil(P/1024)][E] per-chunk expert counts of the many-CTA grouping (nullptr: one CTA)
};

// Kernel arguments (by value).
struct MoeArgs {
  int T, H, I, E, k, P;
  const uint16_t* x;
  const uint8_t *wg, *wu, *wd;     // routed experts (STQ1_0 bytes or MXFP4 codes)
  const uint8_t *gsc, *usc, *dsc;  // MXFP4 scales
  const uint16_t *sg, *su, *sd;    // shared expert, bf16
  const uint8_t *sgq, *suq, *sdq;  // shared expert, MXFP8 codes
  const uint8_t *sgs, *sus, *sds;  // and scales
  const int32_t *counts, *offsets, *perm, *inv, *tlist, *ntouched;
  uint16_t* h;
  float* Y;
  uint8_t *xq, *xs, *hq, *hs;
  const int8_t* xl;  // limbs of x / of the routed h rows for the integer decode GEMV
  const float* xls;  // (nullptr: every item takes the BF16 path)
  const int8_t* hl;
  const float* hls;
  int2* ntiles;
  int32_t* n_ntiles;
  int32_t* err;
  int32_t* sched;   // work counter of this launch
  int n_shared_cta; // work items of the shared expert (first)
  int routed;       // 1: routed STQ1_0 items follow the shared ones
};

MoeWsLayout moe_ws_layout(const moe_desc& d);

// Grid of a persistent launch: min(items, per_sm x SMs), at least 1.
int stq_persistent_grid(int items, int per_sm = 4);

// N tiles of nt tokens of every expert with tokens: tiles[i] = (expert, first token),
// *n_tiles = their number (one CTA, E <= 1024).
stq_status stq_tile_plan_launch(const int32_t* counts, int E, int nt, int2* tiles, int32_t* n_tiles, cudaStream_t s);

// The BF16 shared expert on its own (gate/up, SwiGLU, down into the rows P.. of h and Y).
stq_status moe_shared_expert_bf16(const MoeArgs& a, cudaStream_t s);

// The MXFP8 shared expert (gemm_mx.cu): x -> MXFP8 rows P.. of xq/xs, gate/up + SwiGLU
// into MXFP8 rows P.. of hq/hs, down into rows P.. of Y.
stq_status moe_shared_expert_mx8(const MoeArgs& a, cudaStream_t s);

// Routed STQ1_0 experts in the prefill regime (gemm_stq.cu): activations quantised to
// MXFP8 in sorted pair order, gate/up + SwiGLU into MXFP8 h, down into Y.
stq_status moe_stq_prefill_experts(const MoeArgs& a, int slots, cudaStream_t s);
MoeWs moe_ws_pointers(void* workspace, const MoeWsLayout& L);

// Routed MXFP4 experts: activations quantised to MXFP8 in sorted pair order, gate/up,
// SwiGLU, down.
stq_status moe_mx_experts(const MoeArgs& a, int slots, cudaStream_t s);
// Their prefill regime on CTA pairs (gemm_mx2.cu), activations already quantised.
stq_status moe_mx_experts_pair(const MoeArgs& a, int slots, cudaStream_t s);
// Their prefill regime with the tokens on M (gemm_mx_tm.cu), activations already quantised:
// the gate/up launch (with its 128-token tile plan) and the down launch on the same plan.
stq_status moe_mx_gate_up_tm(const MoeArgs& a, int slots, cudaStream_t s);
stq_status moe_mx_down_tm(const MoeArgs& a, int slots, cudaStream_t s);
// Whether the down launch's 192-row weight tiles divide H.
bool moe_mx_down_tm_fits(const MoeArgs& a);

// BF16 -> MXFP8 quantisation launch (pack.cu).
stq_status stq_mxfp8_quantize_launch(const uint16_t* x, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales,
                                     cudaStream_t s);
// Same into sorted pair order: each of the T token rows is quantised once and written to
// the k output rows inv[t*k + s] (-1 = none; positions below out_rows); err: the error word
// of the checked build's position check.
stq_status stq_mxfp8_quantize_scatter_launch(const uint16_t* x, int64_t T, int64_t K, const int32_t* inv, int k,
                                             int64_t out_rows, int32_t* err, uint8_t* codes, uint8_t* scales,
                                             cudaStream_t s);
