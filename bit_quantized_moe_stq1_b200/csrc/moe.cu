// MoE layer: router, token-to-expert grouping, expert GEMVs with fused SwiGLU,
// shared expert, and the top-k combine.
//
// Shapes: "Hy4-preview-FlashMoE-STQ1_0", "Package details" (hidden 6144, MoE
// intermediate 2048, 256 routed experts, top-8, one shared expert).  The router
// (softmax, top-k, renormalise), the shared BF16 expert and the SwiGLU between
// gate/up and down are this library's reading of "run the experts"; the pages give
// the shapes and formats only.
//
// Data flow of moe_expert_forward, launches in this order on the caller's stream:
//   permute   ids [T,k] -> counts, offsets, perm (pair at each sorted position),
//             inv (sorted position of each pair), list of touched experts
//   experts, by format and regime:
//     STQ1_0, decode regime (this file): gate/up per touched expert and 128-feature
//             tile, g, u (FP32) -> h = silu(g)u as bf16 h[pos, I]; down per touched
//             expert and 256-row tile -> Y[pos, H] (FP32).  The BF16 shared expert's
//             16-row tiles are the first work items of both kernels (h, Y rows P + t).
//     STQ1_0, prefill regime (gemm_stq.cu) and MXFP4 (gemm_mx.cu): x -> MXFP8 in
//             sorted pair order, then the tensor-core GEMMs (gate/up with SwiGLU and
//             the MXFP8 h, then down); the BF16 shared expert as separate launches.
//   combine   y[t] = sum_s w[t,s] Y[inv[t,s]] (+ Y[P+t]) (+ x[t]) in slot order
// The MXFP8 shared expert (quantise x, gate/up, down into rows P + t) depends on x
// alone: it runs on a library-owned side stream, forked after the argument checks and
// joined before the combine.

#include <mutex>

#include "gemv.cuh"
#include "moe_internal.cuh"

namespace {

using namespace stq;

// ----------------------------------------------------------------------------- block scan

// Exclusive scan of one value per thread over a 1024-thread block; returns the
// exclusive prefix and writes the total to *total (shared).
__device__ __forceinline__ int block_excl_scan_1024(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int s = wsum[lane];
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(kFull, si, o);
      if (lane >= o) si += n;
    }
    wsum[lane] = si - s;
    if (lane == 31) *total = si;
  }
  __syncthreads();
  const int r = incl - v + wsum[warp];
  __syncthreads();
  return r;
}

// ----------------------------------------------------------------------------- permute

// The grouping by one CTA of 1024 threads; sm: 34 E ints of shared memory.
__device__ __forceinline__ void permute_cta(const int32_t* __restrict__ ids, int P, int E, const MoeWs& ws,
                                            int32_t* sm) {
  int32_t* cnt = sm;             // [E]
  int32_t* cursor = sm + E;      // [E]
  int32_t* whist = sm + 2 * E;   // [32][E]
  __shared__ int wsum[32];
  __shared__ int total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += 1024) cnt[e] = 0;
  // counters 0-2 (the STQ1_0 decode kernels); counter 3 belongs to the shared expert, which
  // may run on another stream and is zeroed there (shared_gateup_wide_kernel)
  if (ws.sched != nullptr && tid < 3) ws.sched[tid] = 0;
  __syncthreads();
  bool bad = false;
  for (int p = tid; p < P; p += 1024) {
    const int e = ids[p];
    if (e >= 0 && e < E) atomicAdd(&cnt[e], 1); else bad = true;
  }
  if (__syncthreads_or(bad) && tid == 0) stq_set_error(ws.err, STQ_ERR_DEVICE);
  // offsets (exclusive scan of counts) and the touched-expert list; E <= 1024
  const int v = tid < E ? cnt[tid] : 0;
  const int ex = block_excl_scan_1024(v, wsum, &total);
  if (tid < E) {
    cursor[tid] = ex;
    ws.offsets[tid] = ex;
    ws.counts[tid] = v;
  }
  if (tid == 0) ws.offsets[E] = total;
  const int flag = (tid < E && v > 0) ? 1 : 0;
  const int fx = block_excl_scan_1024(flag, wsum, &total);
  if (flag) ws.tlist[fx] = tid;
  if (tid == 0) *ws.ntouched = total;
  __syncthreads();
  // stable placement: chunks of 1024 pairs in pair order
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0; base < P; base += 1024) {
    const int p = base + tid;
    const bool valid = p < P;
    const int e = valid ? ids[p] : -1;
    const bool ok = valid && e >= 0 && e < E;
    for (int i = tid; i < 32 * E; i += 1024) whist[i] = 0;
    __syncthreads();
    const int key = ok ? e : -1 - lane;
    const unsigned peers = __match_any_sync(kFull, key);
    const int rank = __popc(peers & lt);
    if (ok && rank == 0) whist[warp * E + e] = __popc(peers);
    __syncthreads();
    for (int e2 = tid; e2 < E; e2 += 1024) {
      int run = cursor[e2];
#pragma unroll 4
      for (int w = 0; w < 32; ++w) {
        const int c = whist[w * E + e2];
        whist[w * E + e2] = run;
        run += c;
      }
      cursor[e2] = run;
    }
    __syncthreads();
    if (ok) {
      const int pos = whist[warp * E + e] + rank;
      ws.perm[pos] = p;
      ws.inv[p] = pos;
    } else if (valid) {
      ws.inv[p] = -1;
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(1024) moe_permute_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                           MoeWs ws) {
  extern __shared__ int32_t sm[];
  stq_pdl_begin();
  permute_cta(ids, P, E, ws, sm);
}

// The same grouping over many CTAs (large P): chunks of 1024 pairs.
//   hist   CTA c: histogram of chunk c's expert ids -> chist[c][e];
//   scan   one CTA: counts, offsets, touched list, and chist[c][e] turned into the sorted
//          position of chunk c's first pair of expert e (offsets[e] + the counts of e in
//          chunks before c);
//   place  CTA c: stable ranks inside the chunk (as above) from those positions.
// The result equals the one-CTA kernel's exactly.
__global__ void __launch_bounds__(1024) moe_permute_hist_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                int32_t* __restrict__ chist, int32_t* err) {
  extern __shared__ int32_t sm[];  // [E]
  const int tid = threadIdx.x, c = blockIdx.x;
  stq_pdl_begin();
  for (int e = tid; e < E; e += 1024) sm[e] = 0;
  __syncthreads();
  const int p = c * 1024 + tid;
  bool bad = false;
  if (p < P) {
    const int e = ids[p];
    if (e >= 0 && e < E) atomicAdd(&sm[e], 1); else bad = true;
  }
  if (__syncthreads_or(bad) && tid == 0) stq_set_error(err, STQ_ERR_DEVICE);
  for (int e = tid; e < E; e += 1024) chist[size_t(c) * E + e] = sm[e];
}

__global__ void __launch_bounds__(1024) moe_permute_scan_kernel(int E, int C, int32_t* __restrict__ chist, MoeWs ws) {
  __shared__ int wsum[32];
  __shared__ int total;
  const int tid = threadIdx.x;
  stq_pdl_begin();
  if (ws.sched != nullptr && tid < 3) ws.sched[tid] = 0;   // as the one-CTA kernel
  int v = 0;
  if (tid < E) {
    for (int c = 0; c < C; ++c) {
      const int h = chist[size_t(c) * E + tid];
      chist[size_t(c) * E + tid] = v;
      v += h;
    }
  }
  const int ex = block_excl_scan_1024(v, wsum, &total);
  if (tid < E) {
    ws.offsets[tid] = ex;
    ws.counts[tid] = v;
    for (int c = 0; c < C; ++c) chist[size_t(c) * E + tid] += ex;
  }
  if (tid == 0) ws.offsets[E] = total;
  const int flag = (tid < E && v > 0) ? 1 : 0;
  const int fx = block_excl_scan_1024(flag, wsum, &total);
  if (flag) ws.tlist[fx] = tid;
  if (tid == 0) *ws.ntouched = total;
}

__global__ void __launch_bounds__(1024) moe_permute_place_kernel(const int32_t* __restrict__ ids, int P, int E,
                                                                 const int32_t* __restrict__ chist, MoeWs ws) {
  extern __shared__ int32_t sm[];
  int32_t* cursor = sm;          // [E]
  int32_t* whist = sm + E;       // [32][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, c = blockIdx.x;
  stq_pdl_begin();
  for (int e = tid; e < E; e += 1024) cursor[e] = chist[size_t(c) * E + e];
  for (int i = tid; i < 32 * E; i += 1024) whist[i] = 0;
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  const int p = c * 1024 + tid;
  const bool valid = p < P;
  const int e = valid ? ids[p] : -1;
  const bool ok = valid && e >= 0 && e < E;
  const int key = ok ? e : -1 - lane;
  const unsigned peers = __match_any_sync(kFull, key);
  const int rank = __popc(peers & lt);
  if (ok && rank == 0) whist[warp * E + e] = __popc(peers);
  __syncthreads();
  for (int e2 = tid; e2 < E; e2 += 1024) {
    int run = cursor[e2];
#pragma unroll 4
    for (int w = 0; w < 32; ++w) {
      const int cw = whist[w * E + e2];
      whist[w * E + e2] = run;
      run += cw;
    }
  }
  __syncthreads();
  if (ok) {
    const int pos = whist[warp * E + e] + rank;
    ws.perm[pos] = p;
    ws.inv[p] = pos;
  } else if (valid) {
    ws.inv[p] = -1;
  }
}

// ----------------------------------------------------------------------------- router

// Router logits, split over K: part[ks][t][e] = sum over the ks-th slice of H of
// x[t, h] wr[e, h] (bf16 mma.sync, FP32 accumulate).  CTA = 16 experts x one K slice;
// its eight warps split the slice and are summed in a fixed order.
__global__ void __launch_bounds__(256) router_logits_kernel(const uint16_t* __restrict__ x,
                                                            const uint16_t* __restrict__ wr, int T, int H, int E,
                                                            int KS, float* __restrict__ part) {
  __shared__ float red[8][4][4][32];
  stq_pdl_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int e0 = (blockIdx.x / KS) * 16, ks = blockIdx.x % KS;
  const int slice = H / KS, kq = slice / 8;
  const int k0 = ks * slice + warp * kq, k1 = k0 + kq;
  const int er = min(e0 + g, E - 1);                // rows past E read a valid row; results dropped
  const uint16_t* rowg[1] = {wr + size_t(er) * H};
  const int er8 = min(e0 + g + 8, E - 1);
  for (int t0 = 0; t0 < T; t0 += 32) {
    const uint16_t* xr[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int tok = t0 + 8 * c + g;
      xr[c] = tok < T ? x + size_t(tok) * H : nullptr;
    }
    float acc[1][4][4] = {};
    // rows g+8 come from 8*ld further; a ragged last expert tile (warp-uniform test)
    // takes rows g and g+8 through two single-row passes over clamped rows
    if (e0 + 16 <= E) {
      bf16_warp_gemv<1, 4>(rowg, H, k0, k1, xr, acc);
    } else {
      // ragged expert tile: process rows g and g+8 through separate single-row passes
      const uint16_t* r0[1] = {wr + size_t(er) * H};
      float a0[1][4][4] = {}, a1[1][4][4] = {};
      bf16_warp_gemv<1, 4>(r0, 0, k0, k1, xr, a0);
      const uint16_t* r1[1] = {wr + size_t(er8) * H};
      bf16_warp_gemv<1, 4>(r1, 0, k0, k1, xr, a1);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        acc[0][c][0] = a0[0][c][0];
        acc[0][c][1] = a0[0][c][1];
        acc[0][c][2] = a1[0][c][2];
        acc[0][c][3] = a1[0][c][3];
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) red[warp][c][j][lane] = acc[0][c][j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v = red[0][c][j][lane];
#pragma unroll
          for (int w = 1; w < 8; ++w) v += red[w][c][j][lane];
          const int tok = t0 + 8 * c + 2 * t + (j & 1);
          const int e = e0 + g + 8 * (j >> 1);
          if (tok < T && e < E) part[(size_t(ks) * T + tok) * E + e] = v;
        }
    }
    __syncthreads();
  }
}

// One warp per token: softmax over E (max-shifted exp), top-k by probability with
// ties to the lower id, weights renormalised over the chosen k.  Each lane holds
// kMaxPer candidates (E <= 32 * kMaxPer): 8 for up to 256 experts, else 32.
template <int kMaxPer>
__global__ void router_topk_kernel(float* __restrict__ logits, int T, int E, int KS, int k,
                                   int32_t* __restrict__ ids, float* __restrict__ w) {
  stq_pdl_begin();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  constexpr int kMaxKs = 8;
  float p[kMaxPer];
  const int per = (E + 31) / 32;
  float m = -INFINITY;
  // Logits = sum of the KS partial slices, in slice order; all loads of a chunk of 8
  // experts are issued before any add.
#pragma unroll
  for (int j0 = 0; j0 < kMaxPer; j0 += 8) {
    if (j0 >= per) break;
    float part[kMaxKs][8];
#pragma unroll
    for (int ks = 0; ks < kMaxKs; ++ks)
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int e = lane + 32 * (j0 + jj);
        part[ks][jj] = (ks < KS && j0 + jj < per && e < E) ? logits[(size_t(ks) * T + t) * E + e] : 0.f;
      }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int e = lane + 32 * (j0 + jj);
      float v = part[0][jj];
#pragma unroll
      for (int ks = 1; ks < kMaxKs; ++ks) v += part[ks][jj];
      const bool valid = j0 + jj < per && e < E;
      if (valid) logits[size_t(t) * E + e] = v;
      p[j0 + jj] = valid ? v : -INFINITY;
      m = fmaxf(m, p[j0 + jj]);
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j)
    if (j >= ((per + 7) / 8) * 8) p[j] = -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  // Padding lanes get -1 (never chosen); a non-finite logit (or an infinite maximum)
  // counts as probability 0, so a valid expert id is chosen in every round.
#pragma unroll
  for (int j = 0; j < kMaxPer; ++j) {
    const float pv = expf(p[j] - m);
    p[j] = (p[j] == -INFINITY && !(j < per && lane + 32 * j < E)) ? -1.f : (pv >= 0.f ? pv : 0.f);
  }
  float sel_sum = 0.f;
  for (int r = 0; r < k; ++r) {
    float bp = -1.f;
    int bid = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kMaxPer; ++j) {
      const int e = lane + 32 * j;
      if (p[j] > bp) { bp = p[j]; bid = e; }   // ascending e within a lane: ties keep the lower id
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float op = __shfl_xor_sync(kFull, bp, o);
      const int oid = __shfl_xor_sync(kFull, bid, o);
      if (op > bp || (op == bp && oid < bid)) { bp = op; bid = oid; }
    }
    if (bid >= 0 && bid < E && (bid & 31) == lane) p[bid >> 5] = -1.f;  // remove the chosen expert
    sel_sum += bp;
    if (lane == 0) {
      ids[size_t(t) * k + r] = bid;
      w[size_t(t) * k + r] = bp;
    }
  }
  __syncwarp();
  if (lane < k) w[size_t(t) * k + lane] = sel_sum > 0.f ? w[size_t(t) * k + lane] / sel_sum : 1.f / float(k);
}

// ----------------------------------------------------------------------------- expert GEMVs

// Shared expert, gate/up: CTA = 16 features; the CTA's four warps split H.
__device__ __forceinline__ void shared_gateup(const MoeArgs& a, int bid, float (*red)[2][4][4][32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int f0 = bid * 16;
  const int kq = a.H / 4, k0 = warp * kq, k1 = k0 + kq;
  const uint16_t* rowg[2] = {a.sg + size_t(f0 + g) * a.H, a.su + size_t(f0 + g) * a.H};
  for (int t0 = 0; t0 < a.T; t0 += 32) {
    const uint16_t* xr[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int tok = t0 + 8 * c + g;
      xr[c] = tok < a.T ? a.x + size_t(tok) * a.H : nullptr;
    }
    float acc[2][4][4] = {};
    bf16_warp_gemv<2, 4>(rowg, a.H, k0, k1, xr, acc);
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[warp][i][c][j][lane] = acc[i][c][j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float gs = ((red[0][0][c][j][lane] + red[1][0][c][j][lane]) + red[2][0][c][j][lane]) + red[3][0][c][j][lane];
          const float us = ((red[0][1][c][j][lane] + red[1][1][c][j][lane]) + red[2][1][c][j][lane]) + red[3][1][c][j][lane];
          const int tok = t0 + 8 * c + 2 * t + (j & 1);
          const int f = f0 + g + 8 * (j >> 1);
          if (tok < a.T) a.h[size_t(a.P + tok) * a.I + f] = float_to_bf16_bits(silu_f32(gs) * us);
        }
    }
    __syncthreads();
  }
}

// Shared expert, down: CTA = 16 rows of H; the four warps split I.
__device__ __forceinline__ void shared_down(const MoeArgs& a, int bid, float (*red)[2][4][4][32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int r0 = bid * 16;
  const int kq = a.I / 4, k0 = warp * kq, k1 = k0 + kq;
  const uint16_t* rowg[1] = {a.sd + size_t(r0 + g) * a.I};
  for (int t0 = 0; t0 < a.T; t0 += 32) {
    const uint16_t* xr[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int tok = t0 + 8 * c + g;
      xr[c] = tok < a.T ? a.h + size_t(a.P + tok) * a.I : nullptr;
    }
    float acc[1][4][4] = {};
    bf16_warp_gemv<1, 4>(rowg, a.I, k0, k1, xr, acc);
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) red[warp][0][c][j][lane] = acc[0][c][j];
    __syncthreads();
    if (warp == 0) {
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float ys = ((red[0][0][c][j][lane] + red[1][0][c][j][lane]) + red[2][0][c][j][lane]) + red[3][0][c][j][lane];
          const int tok = t0 + 8 * c + 2 * t + (j & 1);
          const int r = r0 + g + 8 * (j >> 1);
          if (tok < a.T) a.Y[size_t(a.P + tok) * a.H + r] = ys;
        }
    }
    __syncthreads();
  }
}

// Shared expert gate/up on its own (the MXFP4 layers, whose routed experts run on the
// tensor-core GEMM): CTA = 16 features of h with 16 warps splitting K in 32-wide chunks,
// so that each SM keeps enough loads in flight; the warps' partial sums are added in warp
// order through shared memory (deterministic), warp w finishing token-chunk/fragment slot
// w.  NCH token chunks of 8 per pass.  (The down projection, K = I, keeps the 4-warp CTAs
// of the persistent STQ1_0 kernel: there the 16-way split left too little work per warp.)
constexpr int kWideWarps = 16;

template <int NCH>
__global__ void __launch_bounds__(kWideWarps * 32) shared_gateup_wide_kernel(MoeArgs a) {
  extern __shared__ float red[];  // [warp][2][NCH][4][32]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  stq_pdl_begin();
  // the work counter of the shared down launch that follows on this stream
  if (blockIdx.x == 0 && threadIdx.x == 0) a.sched[3] = 0;
  const int f0 = blockIdx.x * 16;
  const int nch = a.H / 32;
  const int k0 = 32 * (warp * nch / kWideWarps), k1 = 32 * ((warp + 1) * nch / kWideWarps);
  const uint16_t* rowg[2] = {a.sg + size_t(f0 + g) * a.H, a.su + size_t(f0 + g) * a.H};
  for (int t0 = 0; t0 < a.T; t0 += 8 * NCH) {
    const uint16_t* xr[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int tok = t0 + 8 * c + g;
      xr[c] = tok < a.T ? a.x + size_t(tok) * a.H : nullptr;
    }
    float acc[2][NCH][4] = {};
    bf16_warp_gemv<2, NCH>(rowg, a.H, k0, k1, xr, acc);
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) red[(((warp * 2 + i) * NCH + c) * 4 + j) * 32 + lane] = acc[i][c][j];
    __syncthreads();
    if (warp < NCH * 4) {
      const int c = warp >> 2, j = warp & 3;
      float gs = 0.f, us = 0.f;
      for (int w = 0; w < kWideWarps; ++w) {
        gs += red[(((w * 2 + 0) * NCH + c) * 4 + j) * 32 + lane];
        us += red[(((w * 2 + 1) * NCH + c) * 4 + j) * 32 + lane];
      }
      const int tok = t0 + 8 * c + 2 * t + (j & 1);
      const int f = f0 + g + 8 * (j >> 1);
      if (tok < a.T) a.h[size_t(a.P + tok) * a.I + f] = float_to_bf16_bits(silu_f32(gs) * us);
    }
    __syncthreads();
  }
}

// Next work item of a persistent CTA (one atomic per item, broadcast through smem).
__device__ __forceinline__ int next_item(int32_t* counter, int* slot) {
  if (threadIdx.x == 0) *slot = atomicAdd(counter, 1);
  __syncthreads();
  const int item = *slot;
  __syncthreads();
  return item;
}

// Activation rows src [rows, K] (bf16, K a multiple of 256) -> the integer decode GEMV's
// operand: three signed 8-bit limbs per element, limbs[row][l][K] (l = 0: hi, 1: mid,
// 2: lo), and per 256-k block b the scale of each limb, scales[row * pitch + l * nb + b] =
// 2^(Eb - 148 + 8*(2 - l)) (pitch = stq_limb_scale_pitch(nb)), Eb = the largest exponent
// field of the block's elements (1 for subnormals and zeros).  Inside each 256-byte block
// the limb of k = 64t + 16q + i sits at byte 16*(4q + t) + i, so that the four lanes of a
// GEMV quad read consecutive 16-byte chunks (conflict-free shared-memory loads).  An element
// with significand m (implicit bit included) and exponent field e' = max(e, 1) is
// q = m * 2^(e' - Eb + 14), rounded to nearest, ties to even, when e' < Eb - 14; |q| < 2^22,
// and q = hi*2^16 + mid*2^8 + lo with every limb in [-128, 127].  A block holding an Inf or
// NaN gets a NaN scale.  One warp per block; lane l takes elements 8l..8l+7.
__device__ __forceinline__ void act_limbs_warp(const uint16_t* __restrict__ src, int K, int8_t* __restrict__ limbs,
                                               float* __restrict__ scales, int64_t wid) {
  const int nb = K / 256, lane = threadIdx.x & 31;
  const int64_t row = wid / nb;
  const int b = int(wid - row * nb);
  const uint4 v = *reinterpret_cast<const uint4*>(src + row * K + 256 * b + 8 * lane);
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  uint32_t emax = 1;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t e = (u[i >> 1] >> (16 * (i & 1) + 7)) & 0xFFu;
    emax = e > emax ? e : emax;
  }
  const uint32_t eb = __reduce_max_sync(kFull, emax);
  const int pitch = stq_limb_scale_pitch(nb);
  uint32_t lb[3][2] = {};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t x = (u[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
    const uint32_t e = (x >> 7) & 0xFFu, ep = e > 1u ? e : 1u;
    const uint32_t m = (x & 0x7Fu) | (e != 0u ? 0x80u : 0u);
    uint32_t q;
    if (ep + 14u >= eb) {
      q = m << (ep + 14u - eb);
    } else {
      const uint32_t r = eb - ep - 14u < 9u ? eb - ep - 14u : 9u;
      q = (m + (1u << (r - 1u)) - 1u + ((m >> r) & 1u)) >> r;
    }
    const int32_t vq = (x & 0x8000u) ? -int32_t(q) : int32_t(q);
    const int32_t lo = int32_t(int8_t(vq & 0xFF));
    const int32_t v1 = (vq - lo) >> 8;
    const int32_t mid = int32_t(int8_t(v1 & 0xFF));
    const int32_t hi = (v1 - mid) >> 8;
    const int sh = 8 * (i & 3);
    lb[0][i >> 2] |= (uint32_t(hi) & 0xFFu) << sh;
    lb[1][i >> 2] |= (uint32_t(mid) & 0xFFu) << sh;
    lb[2][i >> 2] |= (uint32_t(lo) & 0xFFu) << sh;
  }
  // this lane's elements k = 8*lane .. 8*lane + 7: t = lane / 8, q = (lane % 8) / 2, i from 8 * (lane % 2)
  const int off = 16 * (4 * ((lane & 7) >> 1) + (lane >> 3)) + 8 * (lane & 1);
#pragma unroll
  for (int l = 0; l < 3; ++l)
    *reinterpret_cast<uint2*>(limbs + (row * 3 + l) * K + 256 * b + off) = make_uint2(lb[l][0], lb[l][1]);
  if (lane < 3)
    scales[row * pitch + lane * nb + b] = eb == 255u ? __int_as_float(0x7FC00000) : ldexpf(1.f, int(eb) - 132 - 8 * lane);
}

__global__ void __launch_bounds__(256) stq_act_limbs_kernel(const uint16_t* __restrict__ src, int64_t rows, int K,
                                                           int8_t* __restrict__ limbs, float* __restrict__ scales) {
  stq_pdl_begin();
  const int64_t wid = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (wid < rows * (K / 256)) act_limbs_warp(src, K, limbs, scales, wid);  // whole warps
}

// The grouping (CTA 0, as moe_permute_kernel) and the limbs of x (the other CTAs, one warp
// per 256-k block, as stq_act_limbs_kernel) in one launch: the two depend on separate
// inputs.
__global__ void __launch_bounds__(1024) moe_permute_limbs_kernel(const int32_t* __restrict__ ids, int P, int E, MoeWs ws,
                                                                 const uint16_t* __restrict__ x, int T, int H,
                                                                 int8_t* __restrict__ xl, float* __restrict__ xls) {
  extern __shared__ int32_t sm[];
  stq_pdl_begin();
  if (blockIdx.x == 0) {
    permute_cta(ids, P, E, ws, sm);
    return;
  }
  const int64_t wid = int64_t(blockIdx.x - 1) * 32 + (threadIdx.x >> 5);
  if (wid < int64_t(T) * (H / 256)) act_limbs_warp(x, H, xl, xls, wid);
}

// Items with at most this many tokens take the integer GEMV (two tokens per mma).
constexpr int kI8MaxTokens = 2;

// Resident CTAs per SM of the two persistent GEMV kernels: with the integer path three
// (168 registers a thread: its weights, operands and sums without spills; measured faster
// than four CTAs at 128 registers), without it four (128 registers, the BF16 path's best).
template <bool I8>
constexpr int gemv_ctas_per_sm() { return I8 ? 3 : 4; }

// The shared expert's partial sums (float[4][2][4][4][32]): all the shared memory a launch
// without the integer path takes.
constexpr int kGemvRedBytes = int(sizeof(float)) * 4 * 2 * 4 * 4 * 32;

// Shared memory of the two persistent GEMV kernels for K = H (gate/up) or I (down), when
// the integer path is on (otherwise a launch takes kGemvRedBytes): the item's activation
// stage (limb rows of its <= 2 tokens, pitch K + 64 so that the two token-limb rows a
// quarter-warp reads fall in different banks, then their scale rows) and the stage's
// barrier.  The shared expert's partial sums alias the stage: every copy into the stage has
// been waited on by the whole CTA before its item ends, and the copies of a routed item are
// issued after the barrier that ends the previous item.  Kept below 48 KB (no opt-in): in the
// stacked decode step, launches that opted in to more measured about 30 us each slower to
// overlap with the kernel before them.
struct GemvSmem {
  int xst, sst, xbar, total, pitch_x, pitch_s;
};
__host__ __device__ inline GemvSmem gemv_smem_layout(int K) {
  GemvSmem L;
  L.pitch_x = K + 64;
  L.pitch_s = stq_limb_scale_pitch(K / 256);
  L.xst = 0;
  L.sst = L.xst + 2 * 3 * L.pitch_x;
  const int end = L.sst + 2 * L.pitch_s * 4;
  L.xbar = (end > kGemvRedBytes ? end : kGemvRedBytes);
  L.total = L.xbar + 8;
  return L;
}
constexpr int kGemvSmemLimit = 47 * 1024;  // below the 48 KB default with the static shared memory

// The integer-path operand rows of a lane in the activation stage (row c = limb c % 3 of
// token c / 3; v0, v1: tokens 0 and 1 present).  Absent columns read row 0 with a zero scale.
__device__ __forceinline__ StqI8Cols i8_cols(const uint8_t* smem, const GemvSmem& L, int nb, bool v0, bool v1) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  auto present = [&](int c) { return c < 6 && (c < 3 ? v0 : v1); };
  const int8_t* xst = reinterpret_cast<const int8_t*>(smem + L.xst);
  const float* sst = reinterpret_cast<const float*>(smem + L.sst);
  auto scale_row = [&](int c) { return present(c) ? sst + (c / 3) * L.pitch_s + (c % 3) * nb : nullptr; };
  StqI8Cols cols;
  cols.xl = xst + (present(g) ? g : 0) * L.pitch_x;
  cols.s0 = scale_row(2 * t);
  cols.s1 = scale_row(2 * t + 1);
  return cols;
}

// Thread 0: bulk copies of the limb rows (3 x K bytes) and scale row of each present token
// (source rows r0, r1; -1 = absent) into the activation stage, completing on its barrier.
__device__ __forceinline__ void i8_stage_fill(uint8_t* smem, const GemvSmem& L, const int8_t* limbs,
                                              const float* scales, int K, int r0, int r1) {
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + L.xbar);
  const uint32_t per_token = uint32_t(3 * K + 4 * L.pitch_s);
  tc::fence_proxy_async_smem();  // earlier generic accesses of the stage before the copies
  tc::mbar_arrive_expect_tx(bar, (r0 >= 0 ? per_token : 0u) + (r1 >= 0 ? per_token : 0u));
  const int rows[2] = {r0, r1};
  for (int j = 0; j < 2; ++j) {
    if (rows[j] < 0) continue;
    for (int l = 0; l < 3; ++l)
      bulk_load(smem + L.xst + (3 * j + l) * L.pitch_x, limbs + (size_t(rows[j]) * 3 + l) * K, uint32_t(K), bar);
    bulk_load(smem + L.sst + j * L.pitch_s * 4, scales + size_t(rows[j]) * L.pitch_s, uint32_t(4 * L.pitch_s), bar);
  }
}

// Routed STQ1_0 gate/up + SwiGLU, persistent.  Items: the shared expert's 16-feature tiles
// (BF16, K split over the four warps) and, per touched expert, 128-feature tiles (warp = 32
// features = 2 gate tiles + 2 up tiles over all of H); the shared ones first on the BF16
// path, last on the integer path.
template <bool I8>
__global__ void __launch_bounds__(128, gemv_ctas_per_sm<I8>()) moe_gateup_stq_kernel(MoeArgs a) {
  extern __shared__ __align__(128) uint8_t gemv_smem[];
  __shared__ int s_item;
  auto red = reinterpret_cast<float (*)[2][4][4][32]>(gemv_smem);
  // the stage and its barrier exist only on the integer path (the launch's shared memory)
  const GemvSmem L = gemv_smem_layout(a.H);
  if (I8 && threadIdx.x == 0 && a.xl != nullptr) {
    tc::mbar_init(reinterpret_cast<uint64_t*>(gemv_smem + L.xbar), 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  bool live = true;    // false after a wait of this warp gave up
  uint32_t xphase = 0; // phase of the activation stage's barrier
  stq_pdl_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int per_expert = a.I / 128;
  const int n_items = a.n_shared_cta + (a.routed ? *a.ntouched * per_expert : 0);
  const int nb = a.H / 256;
  const size_t mat = size_t(a.I) * nb * 42;
  const size_t tstride = size_t(nb) * kTileBlockBytes;
  const uint32_t lut = lut_entry(lane), lut8 = lut_entry_i8(lane);
  for (;;) {
    const int item = next_item(a.sched, &s_item);
    if (item >= n_items) break;
    // the integer path takes the routed items first and the shared expert's smaller ones
    // last, where they fill the tail of the launch; the BF16 path the other way round
    const int n_shared = a.n_shared_cta, n_routed = n_items - n_shared;
    const bool shared_item = I8 ? item >= n_routed : item < n_shared;
    if (shared_item) {
      shared_gateup(a, I8 ? item - n_routed : item, red);
      continue;
    }
    const int bid = I8 ? item : item - n_shared;
    const int slot = bid / per_expert, ct = bid % per_expert;
    const int e = a.tlist[slot];
    if (!STQ_DCHECK(e >= 0 && e < a.E, a.err)) continue;
    const int pos0 = a.offsets[e], cnt = a.offsets[e + 1] - pos0;
    if (!STQ_DCHECK(pos0 >= 0 && cnt >= 0 && pos0 + cnt <= a.P, a.err)) continue;
    const int f0 = ct * 128 + warp * 32;
    const uint8_t* gb = a.wg + size_t(e) * mat;
    const uint8_t* ub = a.wu + size_t(e) * mat;
    const uint8_t* tb[4] = {gb + size_t(f0 / 16) * tstride, gb + size_t(f0 / 16 + 1) * tstride,
                            ub + size_t(f0 / 16) * tstride, ub + size_t(f0 / 16 + 1) * tstride};
    if (I8 && cnt <= kI8MaxTokens && a.xl != nullptr) {
      int tk[2] = {-1, -1};
      for (int j = 0; j < cnt; ++j) {
        const int tok = a.perm[pos0 + j] / a.k;
        tk[j] = STQ_DCHECK(tok >= 0 && tok < a.T, a.err) ? tok : -1;
      }
      if (threadIdx.x == 0 && live) i8_stage_fill(gemv_smem, L, a.xl, a.xls, a.H, tk[0], tk[1]);
      float acc[4][4] = {};
      if (!live) continue;
      live = stq_warp_gemv_i8<4>(tb, nb, i8_cols(gemv_smem, L, nb, tk[0] >= 0, tk[1] >= 0),
                                 reinterpret_cast<uint64_t*>(gemv_smem + L.xbar), xphase, lut8, acc, a.err);
      xphase ^= 1u;
      if (!live) continue;
      float y[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) stq_i8_tokens(acc[i], y[i]);
      const int j = t == 0 ? 0 : (t == 2 ? 1 : kI8MaxTokens);
      if (j < cnt) {
#pragma unroll
        for (int tp = 0; tp < 2; ++tp)
#pragma unroll
          for (int r = 0; r < 2; ++r)
            a.h[size_t(pos0 + j) * a.I + f0 + 16 * tp + g + 8 * r] = float_to_bf16_bits(silu_f32(y[tp][r]) * y[tp + 2][r]);
      }
      continue;
    }
    for (int c0 = 0; c0 < cnt; c0 += 8) {
      const int j = c0 + g;
      const int tok = j < cnt ? a.perm[pos0 + j] / a.k : -1;
      const uint16_t* xrow =
          (j < cnt && STQ_DCHECK(tok >= 0 && tok < a.T, a.err)) ? a.x + size_t(tok) * a.H : nullptr;
      float acc[4][4] = {};
      stq_warp_gemv<4>(tb, 0, nb, xrow, lut, acc);
#pragma unroll
      for (int tp = 0; tp < 2; ++tp)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c0 + 2 * t + (q & 1);
          const int f = f0 + 16 * tp + g + 8 * (q >> 1);
          if (col < cnt) a.h[size_t(pos0 + col) * a.I + f] = float_to_bf16_bits(silu_f32(acc[tp][q]) * acc[tp + 2][q]);
        }
    }
  }
}

// Routed STQ1_0 down, persistent.  Items: the shared expert's 16-row tiles and, per touched
// expert, 256-row tiles of H (warp = 4 tiles); the shared ones first on the BF16 path, last
// on the integer path.
template <bool I8>
__global__ void __launch_bounds__(128, gemv_ctas_per_sm<I8>()) moe_down_stq_kernel(MoeArgs a) {
  extern __shared__ __align__(128) uint8_t gemv_smem[];
  __shared__ int s_item;
  auto red = reinterpret_cast<float (*)[2][4][4][32]>(gemv_smem);
  // the stage and its barrier exist only on the integer path (the launch's shared memory)
  const GemvSmem L = gemv_smem_layout(a.I);
  if (I8 && threadIdx.x == 0 && a.hl != nullptr) {
    tc::mbar_init(reinterpret_cast<uint64_t*>(gemv_smem + L.xbar), 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  bool live = true;    // false after a wait of this warp gave up
  uint32_t xphase = 0; // phase of the activation stage's barrier
  stq_pdl_begin();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
  const int per_expert = a.H / 256;
  const int n_items = a.n_shared_cta + (a.routed ? *a.ntouched * per_expert : 0);
  const int nb = a.I / 256;
  const size_t mat = size_t(a.H) * nb * 42;
  const size_t tstride = size_t(nb) * kTileBlockBytes;
  const uint32_t lut = lut_entry(lane), lut8 = lut_entry_i8(lane);
  for (;;) {
    const int item = next_item(a.sched, &s_item);
    if (item >= n_items) break;
    // the integer path takes the routed items first and the shared expert's smaller ones
    // last, where they fill the tail of the launch; the BF16 path the other way round
    const int n_shared = a.n_shared_cta, n_routed = n_items - n_shared;
    const bool shared_item = I8 ? item >= n_routed : item < n_shared;
    if (shared_item) {
      shared_down(a, I8 ? item - n_routed : item, red);
      continue;
    }
    const int bid = I8 ? item : item - n_shared;
    const int slot = bid / per_expert, ct = bid % per_expert;
    const int e = a.tlist[slot];
    if (!STQ_DCHECK(e >= 0 && e < a.E, a.err)) continue;
    const int pos0 = a.offsets[e], cnt = a.offsets[e + 1] - pos0;
    if (!STQ_DCHECK(pos0 >= 0 && cnt >= 0 && pos0 + cnt <= a.P, a.err)) continue;
    const int r0 = ct * 256 + warp * 64;
    const uint8_t* db = a.wd + size_t(e) * mat;
    const uint8_t* tb[4] = {db + size_t(r0 / 16) * tstride, db + size_t(r0 / 16 + 1) * tstride,
                            db + size_t(r0 / 16 + 2) * tstride, db + size_t(r0 / 16 + 3) * tstride};
    if (I8 && cnt <= kI8MaxTokens && a.hl != nullptr) {
      if (threadIdx.x == 0 && live) i8_stage_fill(gemv_smem, L, a.hl, a.hls, a.I, pos0, cnt > 1 ? pos0 + 1 : -1);
      float acc[4][4] = {};
      if (!live) continue;
      live = stq_warp_gemv_i8<4, true, true>(tb, nb, i8_cols(gemv_smem, L, nb, true, cnt > 1),
                                       reinterpret_cast<uint64_t*>(gemv_smem + L.xbar), xphase, lut8, acc, a.err);
      xphase ^= 1u;
      if (!live) continue;
      float y[4][2];
#pragma unroll
      for (int i = 0; i < 4; ++i) stq_i8_tokens(acc[i], y[i]);
      const int j = t == 0 ? 0 : (t == 2 ? 1 : kI8MaxTokens);
      if (j < cnt) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int r = 0; r < 2; ++r) a.Y[size_t(pos0 + j) * a.H + r0 + 16 * i + g + 8 * r] = y[i][r];
      }
      continue;
    }
    for (int c0 = 0; c0 < cnt; c0 += 8) {
      const int j = c0 + g;
      const uint16_t* xrow = j < cnt ? a.h + size_t(pos0 + j) * a.I : nullptr;
      float acc[4][4] = {};
      stq_warp_gemv<4, true>(tb, 0, nb, xrow, lut, acc);   // the L2 prefetch measured faster here
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = c0 + 2 * t + (q & 1);
          const int r = r0 + 16 * i + g + 8 * (q >> 1);
          if (col < cnt) a.Y[size_t(pos0 + col) * a.H + r] = acc[i][q];
        }
    }
  }
}

// ----------------------------------------------------------------------------- combine

__global__ void moe_combine_kernel(int T, int H, int k, int P, const float* __restrict__ Y,
                                   const int32_t* __restrict__ inv, const float* __restrict__ topk_w, int has_shared,
                                   const uint16_t* __restrict__ resid, void* __restrict__ y, int out_fp32,
                                   int32_t* err) {
  stq_pdl_begin();
  const int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int h4 = H / 4;
  if (idx >= int64_t(T) * h4) return;
  const int t = int(idx / h4), c = int(idx % h4);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < k; ++s) {
    const int pos = inv[size_t(t) * k + s];
    if (pos < 0 || !STQ_DCHECK(pos < P, err)) continue;
    const float w = topk_w[size_t(t) * k + s];
    const float4 v = reinterpret_cast<const float4*>(Y + size_t(pos) * H)[c];
    acc.x = fmaf(w, v.x, acc.x);
    acc.y = fmaf(w, v.y, acc.y);
    acc.z = fmaf(w, v.z, acc.z);
    acc.w = fmaf(w, v.w, acc.w);
  }
  if (has_shared) {
    const float4 v = reinterpret_cast<const float4*>(Y + size_t(P + t) * H)[c];
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  if (resid != nullptr) {
    const uint2 r = reinterpret_cast<const uint2*>(resid + size_t(t) * H)[c];
    acc.x += bf16_bits_to_float(r.x & 0xFFFFu);
    acc.y += bf16_bits_to_float(r.x >> 16);
    acc.z += bf16_bits_to_float(r.y & 0xFFFFu);
    acc.w += bf16_bits_to_float(r.y >> 16);
  }
  if (out_fp32) {
    reinterpret_cast<float4*>(static_cast<float*>(y) + size_t(t) * H)[c] = acc;
  } else {
    const uint32_t lo = uint32_t(float_to_bf16_bits(acc.x)) | (uint32_t(float_to_bf16_bits(acc.y)) << 16);
    const uint32_t hi = uint32_t(float_to_bf16_bits(acc.z)) | (uint32_t(float_to_bf16_bits(acc.w)) << 16);
    reinterpret_cast<uint2*>(static_cast<uint16_t*>(y) + size_t(t) * H)[c] = make_uint2(lo, hi);
  }
}

// The combine and the stacked layers' RMS normalisation in one launch: one CTA of 1024
// threads per token row.  Phase 1 forms every element exactly as moe_combine_kernel does
// (slot-ordered FMAs, then the shared expert, then the residual, rounded to bf16) into
// shared memory; phase 2 sums the squares of the bf16 row in rmsnorm_bf16_kernel's FP64
// order (threads 0..255, uint4 chunks tid, tid + 256, ... ascending, an xor tree per warp,
// the eight warp partials in warp order); phase 3 writes x * (1 / sqrt(ms + eps)) rounded
// through FP32 to bf16.  The result has the bits of the two kernels run in sequence.  The
// residual may alias y: a row's reads all come before its writes.
__global__ void __launch_bounds__(1024) moe_combine_norm_kernel(int T, int H, int k, int P, const float* __restrict__ Y,
                                                                const int32_t* __restrict__ inv,
                                                                const float* __restrict__ topk_w, int has_shared,
                                                                const uint16_t* resid, uint16_t* y, float eps,
                                                                int32_t* err) {
  extern __shared__ uint4 srow[];  // the bf16 row, H / 8 chunks
  __shared__ double part[8];
  __shared__ double s_scale;
  __shared__ int s_pos[32];        // the row's k slots (k <= 32): sorted position, -1 = none
  __shared__ float s_w[32];
  stq_pdl_begin();
  const int t = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h4 = H / 4, n8 = H / 8;
  if (tid < k) {
    const int pos = inv[size_t(t) * k + tid];
    s_pos[tid] = (pos < 0 || !STQ_DCHECK(pos < P, err)) ? -1 : pos;
    s_w[tid] = topk_w[size_t(t) * k + tid];
  }
  __syncthreads();
  uint2* row2 = reinterpret_cast<uint2*>(srow);
  for (int c = tid; c < h4; c += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // eight slots' loads at a time, then their FMAs in slot order
    for (int s0 = 0; s0 < k; s0 += 8) {
      float4 v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int pos = s0 + j < k ? s_pos[s0 + j] : -1;
        v[j] = pos >= 0 ? reinterpret_cast<const float4*>(Y + size_t(pos) * H)[c] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (s0 + j >= k || s_pos[s0 + j] < 0) continue;
        const float w = s_w[s0 + j];
        acc.x = fmaf(w, v[j].x, acc.x);
        acc.y = fmaf(w, v[j].y, acc.y);
        acc.z = fmaf(w, v[j].z, acc.z);
        acc.w = fmaf(w, v[j].w, acc.w);
      }
    }
    if (has_shared) {
      const float4 v = reinterpret_cast<const float4*>(Y + size_t(P + t) * H)[c];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (resid != nullptr) {
      const uint2 r = reinterpret_cast<const uint2*>(resid + size_t(t) * H)[c];
      acc.x += bf16_bits_to_float(r.x & 0xFFFFu);
      acc.y += bf16_bits_to_float(r.x >> 16);
      acc.z += bf16_bits_to_float(r.y & 0xFFFFu);
      acc.w += bf16_bits_to_float(r.y >> 16);
    }
    row2[c] = make_uint2(uint32_t(float_to_bf16_bits(acc.x)) | (uint32_t(float_to_bf16_bits(acc.y)) << 16),
                         uint32_t(float_to_bf16_bits(acc.z)) | (uint32_t(float_to_bf16_bits(acc.w)) << 16));
  }
  __syncthreads();
  if (tid < 256) {
    double ss = 0.0;
    for (int i = tid; i < n8; i += 256) {
      const uint4 v = srow[i];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const double a = bf16_bits_to_float(w4[j] & 0xFFFFu), b = bf16_bits_to_float(w4[j] >> 16);
        ss = fma(a, a, ss);
        ss = fma(b, b, ss);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(kFull, ss, o);
    if (lane == 0) part[warp] = ss;
  }
  __syncthreads();
  if (tid == 0) {
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += part[w];
    s_scale = 1.0 / sqrt(tot / double(H) + double(eps));
  }
  __syncthreads();
  const double r = s_scale;
  uint4* yr = reinterpret_cast<uint4*>(y + size_t(t) * H);
  for (int i = tid; i < n8; i += blockDim.x) {
    const uint4 v = srow[i];
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __double2float_rn(double(bf16_bits_to_float(w4[j] & 0xFFFFu)) * r);
      const float b = __double2float_rn(double(bf16_bits_to_float(w4[j] >> 16)) * r);
      o[j] = uint32_t(float_to_bf16_bits(a)) | (uint32_t(float_to_bf16_bits(b)) << 16);
    }
    yr[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

// ----------------------------------------------------------------------------- host side

// CTAs of a persistent launch: per_sm per SM (the register-limited occupancy), never
// more than the work items.  The SM count is read once, from the first device that
// launches (the GPUs of one process are assumed alike).
int stq_persistent_grid(int items, int per_sm) {
  static const int sms = [] {
    int dev = 0, n = 0;
    return cudaGetDevice(&dev) == cudaSuccess &&
                   cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0
               ? n
               : 148;
  }();
  const int cap = per_sm * sms;
  return items < 1 ? 1 : (items < cap ? items : cap);
}

MoeWsLayout moe_ws_layout(const moe_desc& d) {
  MoeWsLayout L{};
  const size_t T = size_t(d.T), H = size_t(d.H), I = size_t(d.I), E = size_t(d.E), P = T * size_t(d.k);
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
  L.err = take(sizeof(int32_t));
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.tlist = take(E * 4);
  L.ntouched = take(4);
  L.perm = take(P * 4);
  L.inv = take(P * 4);
  L.h = take((P + T) * I * 2);
  L.Y = take((P + T) * H * 4);
  L.xq = take((P + T) * H);
  L.xs = take((P + T) * (H / 32));
  L.hq = take((P + T) * I);
  L.hs = take((P + T) * (I / 32));
  L.xl = take(T * 3 * H);
  L.xls = take(T * size_t(stq_limb_scale_pitch(int(H / 256))) * 4);
  L.hl = take(P * 3 * I);
  L.hls = take(P * size_t(stq_limb_scale_pitch(int(I / 256))) * 4);
  L.ntiles = take((P / 16 + E + 1) * 8);
  L.n_ntiles = take(4);
  L.sched = take(16);
  L.chist = take(size_t((P + 1023) / 1024) * E * 4);
  L.total = o;
  return L;
}

MoeWs moe_ws_pointers(void* workspace, const MoeWsLayout& L) {
  uint8_t* b = static_cast<uint8_t*>(workspace);
  MoeWs w;
  w.err = reinterpret_cast<int32_t*>(b + L.err);
  w.counts = reinterpret_cast<int32_t*>(b + L.counts);
  w.offsets = reinterpret_cast<int32_t*>(b + L.offsets);
  w.tlist = reinterpret_cast<int32_t*>(b + L.tlist);
  w.ntouched = reinterpret_cast<int32_t*>(b + L.ntouched);
  w.perm = reinterpret_cast<int32_t*>(b + L.perm);
  w.inv = reinterpret_cast<int32_t*>(b + L.inv);
  w.h = reinterpret_cast<uint16_t*>(b + L.h);
  w.Y = reinterpret_cast<float*>(b + L.Y);
  w.xq = b + L.xq;
  w.xs = b + L.xs;
  w.hq = b + L.hq;
  w.hs = b + L.hs;
  w.xl = reinterpret_cast<int8_t*>(b + L.xl);
  w.xls = reinterpret_cast<float*>(b + L.xls);
  w.hl = reinterpret_cast<int8_t*>(b + L.hl);
  w.hls = reinterpret_cast<float*>(b + L.hls);
  w.ntiles = reinterpret_cast<int2*>(b + L.ntiles);
  w.n_ntiles = reinterpret_cast<int32_t*>(b + L.n_ntiles);
  w.sched = reinterpret_cast<int32_t*>(b + L.sched);
  w.chist = reinterpret_cast<int32_t*>(b + L.chist);
  return w;
}

static bool desc_ok(const moe_desc* d) {
  // P = T*k below 2^30 (as moe_permute): pair and row indices, P + T included, stay in int32
  return d && d->T >= 0 && d->H > 0 && d->I > 0 && d->E > 0 && d->E <= 1024 && d->k > 0 && d->k <= 32 &&
         d->k <= d->E && int64_t(d->T) * d->k < (int64_t(1) << 30) && d->regime >= STQ_REGIME_AUTO &&
         d->regime <= STQ_REGIME_PREFILL &&
         (d->norm_out == 0 || (d->norm_out == 1 && d->out_fp32 == 0 && d->norm_eps >= 0.f && d->norm_eps < 3.0e38f));
}

extern "C" size_t moe_workspace_bytes(const moe_desc* d) {
  if (!desc_ok(d)) return 0;
  return moe_ws_layout(*d).total;
}

// The BF16 shared expert alone (used by MXFP4 layers): the shared CTAs of the two
// STQ1_0 kernels.
template <int NCH>
stq_status launch_shared_gateup_wide(const MoeArgs& a, cudaStream_t s) {
  const int smem = kWideWarps * 2 * NCH * 4 * 32 * 4;
  static StqSmemOptIn optin;
  const stq_status st = optin.ensure(shared_gateup_wide_kernel<NCH>, smem);
  if (st != STQ_OK) return st;
  StqTimed tm(STQ_K_SHARED_GATE_UP, s);
  return stq_launch(shared_gateup_wide_kernel<NCH>, dim3(unsigned(a.I / 16)), dim3(kWideWarps * 32), smem, s, a);
}

stq_status moe_shared_expert_bf16(const MoeArgs& a0, cudaStream_t s) {
  stq_status st = a0.T <= 8    ? launch_shared_gateup_wide<1>(a0, s)
                  : a0.T <= 16 ? launch_shared_gateup_wide<2>(a0, s)
                               : launch_shared_gateup_wide<4>(a0, s);
  if (st != STQ_OK) return st;
  MoeArgs a = a0;
  a.routed = 0;
  a.n_shared_cta = a.H / 16;
  a.sched = a0.sched + 3;
  StqTimed tm(STQ_K_SHARED_DOWN, s);
  return stq_launch(moe_down_stq_kernel<false>, dim3(unsigned(stq_persistent_grid(a.n_shared_cta, gemv_ctas_per_sm<false>()))),
                    dim3(128), kGemvRedBytes, s, a);
}

extern "C" size_t moe_workspace_offset(const moe_desc* d, int32_t region) {
  if (!desc_ok(d)) return ~size_t(0);
  const MoeWsLayout L = moe_ws_layout(*d);
  switch (region) {
    case STQ_WS_COUNTS: return L.counts;
    case STQ_WS_OFFSETS: return L.offsets;
    case STQ_WS_PERM: return L.perm;
    case STQ_WS_INV: return L.inv;
    case STQ_WS_TLIST: return L.tlist;
    case STQ_WS_NTOUCHED: return L.ntouched;
    case STQ_WS_H: return L.h;
    case STQ_WS_Y: return L.Y;
    case STQ_WS_XQ: return L.xq;
    case STQ_WS_XS: return L.xs;
    case STQ_WS_HQ: return L.hq;
    case STQ_WS_HS: return L.hs;
    default: return ~size_t(0);
  }
}

// From this many pairs (and with the workspace's chunk histograms) the grouping runs over
// many CTAs.
constexpr int kPermuteMultiCta = 8192;

stq_status moe_launch_permute(const int32_t* ids, int P, int E, const MoeWs& ws, cudaStream_t s) {
  if (P >= kPermuteMultiCta && ws.chist != nullptr) {
    const int C = (P + 1023) / 1024;
    const size_t smem = size_t(33) * E * sizeof(int32_t);
    static StqSmemOptIn optin;
    stq_status st = optin.ensure(moe_permute_place_kernel, int(smem));
    if (st != STQ_OK) return st;
    {
      StqTimed tm(STQ_K_PERMUTE, s);
      st = stq_launch(moe_permute_hist_kernel, dim3(unsigned(C)), dim3(1024), size_t(E) * sizeof(int32_t), s, ids, P, E,
                      ws.chist, ws.err);
    }
    if (st != STQ_OK) return st;
    {
      StqTimed tm(STQ_K_PERMUTE, s);
      st = stq_launch(moe_permute_scan_kernel, dim3(1), dim3(1024), 0, s, E, C, ws.chist, ws);
    }
    if (st != STQ_OK) return st;
    StqTimed tm(STQ_K_PERMUTE, s);
    return stq_launch(moe_permute_place_kernel, dim3(unsigned(C)), dim3(1024), smem, s, ids, P, E,
                      static_cast<const int32_t*>(ws.chist), ws);
  }
  const size_t smem = size_t(34) * E * sizeof(int32_t);
  static StqSmemOptIn optin;
  const stq_status st = optin.ensure(moe_permute_kernel, int(smem));
  if (st != STQ_OK) return st;
  StqTimed tm(STQ_K_PERMUTE, s);
  return stq_launch(moe_permute_kernel, dim3(1), dim3(1024), smem, s, ids, P, E, ws);
}

// Rows up to this many elements take the fused combine + RMS normalisation (the row's
// bf16 values in shared memory, below the 48 KB default).
constexpr int kCombineNormMaxH = 23 * 1024;

stq_status moe_launch_combine(const moe_desc& d, int P, const MoeWs& ws, const float* topk_w, bool has_shared,
                              const uint16_t* x, void* y, cudaStream_t s) {
  const int64_t n = int64_t(d.T) * (d.H / 4);
  if (n == 0) return STQ_OK;
  if (d.norm_out && d.H <= kCombineNormMaxH) {
    StqTimed tm(STQ_K_COMBINE, s);
    return stq_launch(moe_combine_norm_kernel, dim3(unsigned(d.T)), dim3(1024), size_t(d.H) * 2, s, d.T, d.H, d.k, P,
                      static_cast<const float*>(ws.Y), static_cast<const int32_t*>(ws.inv), topk_w,
                      has_shared ? 1 : 0, d.add_residual ? x : nullptr, static_cast<uint16_t*>(y), d.norm_eps,
                      ws.err);
  }
  stq_status st;
  {
    StqTimed tm(STQ_K_COMBINE, s);
    st = stq_launch(moe_combine_kernel, dim3(unsigned(ceil_div<int64_t>(n, 256))), dim3(256), 0, s, d.T, d.H, d.k, P,
                    static_cast<const float*>(ws.Y), static_cast<const int32_t*>(ws.inv), topk_w, has_shared ? 1 : 0,
                    d.add_residual ? x : nullptr, y, d.out_fp32, ws.err);
  }
  if (st != STQ_OK || !d.norm_out) return st;
  // rows too wide for the fused kernel: the normalisation as its own launch
  return stq_rmsnorm_bf16(static_cast<const uint16_t*>(y), d.T, d.H, d.norm_eps, static_cast<uint16_t*>(y),
                          reinterpret_cast<stq_stream_t>(s));
}

// A library-owned stream per device, created on first use: the MXFP8 shared expert
// depends on x alone, so it runs beside the routing, permutation and routed experts
// instead of after them.  Calls from several host threads share the stream; `mu` is held
// from the fork to the join record, so one call's launches on it never interleave with
// another's.
struct SideStream {
  cudaStream_t stream = nullptr;
  std::mutex mu;
};

// Fork and join events of the calling host thread on one device: a call waits on its own
// records only, whatever other threads record meanwhile.  Created on first use, kept for
// the thread's lifetime.
struct ForkJoin {
  cudaEvent_t fork = nullptr, join = nullptr;
};

static stq_status side_stream(SideStream** out, ForkJoin** fj) {
  static SideStream side[kStqMaxDevices];
  static std::mutex create_mu;
  thread_local ForkJoin events[kStqMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kStqMaxDevices) return STQ_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lock(create_mu);
    if (side[dev].stream == nullptr &&
        cudaStreamCreateWithFlags(&side[dev].stream, cudaStreamNonBlocking) != cudaSuccess)
      return STQ_ERR_CUDA;
  }
  ForkJoin& ev = events[dev];
  if (ev.fork == nullptr) {
    if (cudaEventCreateWithFlags(&ev.fork, cudaEventDisableTiming) != cudaSuccess) return STQ_ERR_CUDA;
    if (cudaEventCreateWithFlags(&ev.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaEventDestroy(ev.fork);
      ev.fork = nullptr;
      return STQ_ERR_CUDA;
    }
  }
  *out = &side[dev];
  *fj = &ev;
  return STQ_OK;
}

// Largest average of routed tokens per expert for which the STQ1_0 decode regime makes
// the activation limbs of the integer GEMV.
constexpr int kI8LimbsAvgTokens = 2;

stq_status moe_launch_act_limbs(const uint16_t* src, int64_t rows, int K, int8_t* limbs, float* scales,
                                cudaStream_t s) {
  const int64_t warps = rows * (K / 256);
  if (warps == 0) return STQ_OK;
  StqTimed tm(STQ_K_ACT_LIMBS, s);
  return stq_launch(stq_act_limbs_kernel, dim3(unsigned(ceil_div<int64_t>(warps, 8))), dim3(256), 0, s, src, rows, K,
                    limbs, scales);
}

// The routed STQ1_0 experts in the decode regime: the two persistent GEMV kernels (the BF16
// shared expert's tiles as their first items), with the integer path (I8: the activation
// limbs of x made before gate/up, those of h between gate/up and down) or without it.
template <bool I8>
stq_status launch_stq_decode(MoeArgs a, const moe_desc& d, const MoeWs& ws, const uint16_t* x, int P, int slots,
                             bool shared_bf16, bool x_limbs_done, cudaStream_t s) {
  stq_status st;
  const int smem_gu = I8 ? gemv_smem_layout(d.H).total : kGemvRedBytes;
  const int smem_dn = I8 ? gemv_smem_layout(d.I).total : kGemvRedBytes;
  if (I8) {
    if (!x_limbs_done && (st = moe_launch_act_limbs(x, d.T, d.H, ws.xl, ws.xls, s)) != STQ_OK) return st;
    a.xl = ws.xl;
    a.xls = ws.xls;
  }
  a.routed = 1;
  a.n_shared_cta = shared_bf16 ? d.I / 16 : 0;
  a.sched = ws.sched;
  {
    StqTimed tm(STQ_K_GATE_UP, s);
    st = stq_launch(moe_gateup_stq_kernel<I8>,
                    dim3(unsigned(stq_persistent_grid(a.n_shared_cta + slots * (d.I / 128), gemv_ctas_per_sm<I8>()))),
                    dim3(128), smem_gu, s, a);
  }
  if (st != STQ_OK) return st;
  if (I8) {
    if ((st = moe_launch_act_limbs(ws.h, P, d.I, ws.hl, ws.hls, s)) != STQ_OK) return st;
    a.hl = ws.hl;
    a.hls = ws.hls;
  }
  a.n_shared_cta = shared_bf16 ? d.H / 16 : 0;
  a.sched = ws.sched + 1;
  StqTimed tm(STQ_K_DOWN, s);
  return stq_launch(moe_down_stq_kernel<I8>,
                    dim3(unsigned(stq_persistent_grid(a.n_shared_cta + slots * (d.H / 256), gemv_ctas_per_sm<I8>()))),
                    dim3(128), smem_dn, s, a);
}

// Average routed tokens per expert from which STQ_REGIME_AUTO runs the STQ1_0 experts
// on the tensor-core GEMM instead of the decode GEMV.
constexpr int kStqPrefillTokensPerExpert = 32;

extern "C" stq_status moe_expert_forward(const moe_desc* d, const uint16_t* x, const int32_t* topk_ids,
                                         const float* topk_w, const moe_weights* w, void* y, void* workspace,
                                         size_t ws_bytes, stq_stream_t stream) {
  STQ_HOST_CHECK(desc_ok(d) && w && x && topk_ids && topk_w && y && workspace, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(w->fmt == STQ_FMT_STQ1_0 || w->fmt == STQ_FMT_MXFP4, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(w->gate && w->up && w->down, STQ_ERR_INVALID_ARG);
  const bool has_shared = w->sh_gate != nullptr;
  STQ_HOST_CHECK(!has_shared || (w->sh_up && w->sh_down), STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(!has_shared || w->sh_fmt == STQ_SHARED_BF16 || w->sh_fmt == STQ_SHARED_MXFP8, STQ_ERR_INVALID_ARG);
  const bool shared_bf16 = has_shared && w->sh_fmt == STQ_SHARED_BF16;
  const bool shared_mx8 = has_shared && w->sh_fmt == STQ_SHARED_MXFP8;
  if (shared_mx8) {
    STQ_HOST_CHECK(w->sh_gate_sc && w->sh_up_sc && w->sh_down_sc, STQ_ERR_INVALID_ARG);
    STQ_HOST_CHECK(((reinterpret_cast<uintptr_t>(w->sh_gate_sc) | reinterpret_cast<uintptr_t>(w->sh_up_sc) |
                     reinterpret_cast<uintptr_t>(w->sh_down_sc)) & 3u) == 0,
                   STQ_ERR_ALIGN);
  }
  STQ_HOST_CHECK(d->H % 256 == 0 && d->I % 256 == 0, STQ_ERR_SHAPE);
  if (w->fmt == STQ_FMT_MXFP4) STQ_HOST_CHECK(w->gate_sc && w->up_sc && w->down_sc, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(stq_aligned16(x) && stq_aligned16(y) && stq_aligned16(w->gate) && stq_aligned16(w->up) &&
                     stq_aligned16(w->down) && stq_aligned16(topk_ids) && stq_aligned16(topk_w),
                 STQ_ERR_ALIGN);
  STQ_HOST_CHECK((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, STQ_ERR_ALIGN);
  if (has_shared)
    STQ_HOST_CHECK(stq_aligned16(w->sh_gate) && stq_aligned16(w->sh_up) && stq_aligned16(w->sh_down), STQ_ERR_ALIGN);
  const MoeWsLayout L = moe_ws_layout(*d);
  STQ_HOST_CHECK(ws_bytes >= L.total, STQ_ERR_WORKSPACE);
  if (d->T == 0) return STQ_OK;
  cudaStream_t s = stq_cuda_stream(stream);
  const MoeWs ws = moe_ws_pointers(workspace, L);
  const int P = d->T * d->k;
  stq_status st = STQ_OK;

  MoeArgs a{};
  a.T = d->T; a.H = d->H; a.I = d->I; a.E = d->E; a.k = d->k; a.P = P;
  a.x = x;
  a.wg = w->gate; a.wu = w->up; a.wd = w->down;
  a.gsc = w->gate_sc; a.usc = w->up_sc; a.dsc = w->down_sc;
  if (shared_bf16) {
    a.sg = static_cast<const uint16_t*>(w->sh_gate);
    a.su = static_cast<const uint16_t*>(w->sh_up);
    a.sd = static_cast<const uint16_t*>(w->sh_down);
  } else if (shared_mx8) {
    a.sgq = static_cast<const uint8_t*>(w->sh_gate);
    a.suq = static_cast<const uint8_t*>(w->sh_up);
    a.sdq = static_cast<const uint8_t*>(w->sh_down);
    a.sgs = w->sh_gate_sc; a.sus = w->sh_up_sc; a.sds = w->sh_down_sc;
  }
  a.counts = ws.counts; a.offsets = ws.offsets; a.perm = ws.perm; a.inv = ws.inv; a.tlist = ws.tlist;
  a.ntouched = ws.ntouched;
  a.h = ws.h; a.Y = ws.Y;
  a.xq = ws.xq; a.xs = ws.xs; a.hq = ws.hq; a.hs = ws.hs;
  a.ntiles = ws.ntiles; a.n_ntiles = ws.n_ntiles;
  a.sched = ws.sched;
  a.err = ws.err;
  const int slots = d->E < P ? d->E : P;

  const bool prefill = d->regime == STQ_REGIME_PREFILL ||
                       (d->regime == STQ_REGIME_AUTO && P >= kStqPrefillTokensPerExpert * slots);
  const bool stq_decode = w->fmt == STQ_FMT_STQ1_0 && !prefill;
  // The shared expert depends on x alone.  Except in the STQ1_0 decode regime (whose
  // persistent GEMV kernels take its BF16 tiles as extra work items) it runs on the side
  // stream, beside the grouping, quantisation and routed experts: its workspace rows P..,
  // its work counter (sched[3], zeroed on that stream) and the sticky error word are all it
  // writes, and nothing on the routed path reads them.  Joined before the combine.
  SideStream* side = nullptr;
  ForkJoin* fj = nullptr;
  const bool on_side = shared_mx8 || (shared_bf16 && !stq_decode);
  if (on_side) {
    if ((st = side_stream(&side, &fj)) != STQ_OK) return st;
    std::lock_guard<std::mutex> lock(side->mu);
    if (cudaEventRecord(fj->fork, s) != cudaSuccess || cudaStreamWaitEvent(side->stream, fj->fork, 0) != cudaSuccess)
      return STQ_ERR_CUDA;
    st = shared_mx8 ? moe_shared_expert_mx8(a, side->stream) : moe_shared_expert_bf16(a, side->stream);
    if (st != STQ_OK) return st;
    if (cudaEventRecord(fj->join, side->stream) != cudaSuccess) return STQ_ERR_CUDA;
  }
  // The STQ1_0 decode regime's integer GEMV serves items of at most two tokens; its limbs
  // are made when the average expert has at most two and the activation stages fit in
  // kGemvSmemLimit.  With the one-CTA grouping, x's limbs come from the same launch.
  const bool i8 = stq_decode && int64_t(P) <= kI8LimbsAvgTokens * int64_t(slots) &&
                  gemv_smem_layout(d->H).total <= kGemvSmemLimit && gemv_smem_layout(d->I).total <= kGemvSmemLimit;
  const bool fused_limbs = i8 && !(P >= kPermuteMultiCta && ws.chist != nullptr);
  if (fused_limbs) {
    const size_t smem = size_t(34) * d->E * sizeof(int32_t);
    static StqSmemOptIn optin;
    if ((st = optin.ensure(moe_permute_limbs_kernel, int(smem))) != STQ_OK) return st;
    const int64_t warps = int64_t(d->T) * (d->H / 256);
    StqTimed tm(STQ_K_PERMUTE, s);
    st = stq_launch(moe_permute_limbs_kernel, dim3(unsigned(1 + ceil_div<int64_t>(warps, 32))), dim3(1024), smem, s,
                    topk_ids, P, d->E, ws, x, d->T, d->H, ws.xl, ws.xls);
  } else {
    st = moe_launch_permute(topk_ids, P, d->E, ws, s);
  }
  if (st != STQ_OK) return st;

  if (w->fmt == STQ_FMT_STQ1_0 && prefill) {
    if ((st = moe_stq_prefill_experts(a, slots, s)) != STQ_OK) return st;
  } else if (w->fmt == STQ_FMT_STQ1_0) {
    st = i8 ? launch_stq_decode<true>(a, *d, ws, x, P, slots, shared_bf16, fused_limbs, s)
            : launch_stq_decode<false>(a, *d, ws, x, P, slots, shared_bf16, false, s);
    if (st != STQ_OK) return st;
  } else {
    st = moe_mx_experts(a, slots, s);
    if (st != STQ_OK) return st;
  }
  if (on_side && cudaStreamWaitEvent(s, fj->join, 0) != cudaSuccess) return STQ_ERR_CUDA;
  return moe_launch_combine(*d, P, ws, topk_w, has_shared, x, y, s);
}

extern "C" int32_t stq_router_ksplit(int32_t H) {
  for (int ks = 8; ks > 1; ks >>= 1)
    if (H % (256 * ks) == 0) return ks;
  return 1;
}

extern "C" stq_status moe_router_topk(const uint16_t* x, const uint16_t* w_router, int32_t T, int32_t H, int32_t E,
                                      int32_t k, float* logits, int32_t* topk_ids, float* topk_w,
                                      stq_stream_t stream) {
  STQ_HOST_CHECK(T >= 0 && H > 0 && E > 0 && E <= 1024 && k > 0 && k <= 32 && k <= E, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(H % 256 == 0, STQ_ERR_SHAPE);
  if (T == 0) return STQ_OK;  // nothing to do; the pointers may then be NULL
  STQ_HOST_CHECK(x && w_router && logits && topk_ids && topk_w, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(stq_aligned16(x) && stq_aligned16(w_router), STQ_ERR_ALIGN);
  cudaStream_t s = stq_cuda_stream(stream);
  const int KS = stq_router_ksplit(H);
  stq_status st;
  {
    StqTimed tm(STQ_K_ROUTER_LOGITS, s);
    st = stq_launch(router_logits_kernel, dim3(unsigned(ceil_div(E, 16) * KS)), dim3(256), 0, s, x, w_router, T, H, E,
                    KS, logits);
  }
  if (st != STQ_OK) return st;
  StqTimed tm(STQ_K_ROUTER_TOPK, s);
  return E <= 256 ? stq_launch(router_topk_kernel<8>, dim3(unsigned(ceil_div(T, 4))), dim3(128), 0, s, logits, T, E, KS, k,
                               topk_ids, topk_w)
                  : stq_launch(router_topk_kernel<32>, dim3(unsigned(ceil_div(T, 4))), dim3(128), 0, s, logits, T, E, KS,
                               k, topk_ids, topk_w);
}

extern "C" stq_status moe_permute(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E, int32_t* counts,
                                  int32_t* offsets, int32_t* perm, int32_t* inv, int32_t* tlist, int32_t* ntouched,
                                  int32_t* err, stq_stream_t stream) {
  STQ_HOST_CHECK(counts && offsets && tlist && ntouched, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(T >= 0 && k > 0 && E > 0 && E <= 1024, STQ_ERR_INVALID_ARG);
  const int64_t P64 = int64_t(T) * k;
  STQ_HOST_CHECK(P64 < (int64_t(1) << 30), STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(P64 == 0 || (topk_ids && perm && inv), STQ_ERR_INVALID_ARG);
  MoeWs ws{};
  ws.err = err; ws.counts = counts; ws.offsets = offsets; ws.perm = perm; ws.inv = inv;
  ws.tlist = tlist; ws.ntouched = ntouched;
  return moe_launch_permute(topk_ids, int(P64), E, ws, stq_cuda_stream(stream));
}

// ----------------------------------------------------------------------------- router, no allocation
//
// The same two router kernels as moe_router_topk, for callers that cannot hand the
// library a scratch buffer: the logits partial sums live in a fixed array compiled
// into this module, one copy on every GPU that loads the library, kept until the
// process exits.  Host code may not pass the array's name to a kernel (on the host
// it is only a stand-in for the symbol), so every call looks up its device address
// with cudaGetSymbolAddress, with the call's device current.  Looking it up per call
// (not caching it) keeps the address right after a cudaDeviceReset, which reloads the
// module at another address in a new context.

constexpr size_t kRouterStaticFloats = size_t(1) << 19;  // 524,288 floats = 2 MiB per GPU

static __device__ __align__(256) float g_router_scratch[kRouterStaticFloats];

extern "C" stq_status moe_router_topk_static(const uint16_t* x, const uint16_t* w_router, int32_t T, int32_t H,
                                             int32_t E, int32_t k, int32_t* topk_ids, float* topk_w,
                                             stq_stream_t stream) {
  STQ_HOST_CHECK(T >= 0 && H > 0 && E > 0 && E <= 1024 && k > 0 && k <= 32 && k <= E, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(H % 256 == 0, STQ_ERR_SHAPE);
  const int KS = stq_router_ksplit(H);
  STQ_HOST_CHECK(size_t(KS) * size_t(T) * size_t(E) <= kRouterStaticFloats, STQ_ERR_WORKSPACE);
  if (T == 0) return STQ_OK;  // nothing to do; the pointers may then be NULL
  STQ_HOST_CHECK(x && w_router && topk_ids && topk_w, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(stq_aligned16(x) && stq_aligned16(w_router), STQ_ERR_ALIGN);
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_router_scratch) != cudaSuccess || addr == nullptr) return STQ_ERR_CUDA;
  float* scratch = static_cast<float*>(addr);
  cudaStream_t s = stq_cuda_stream(stream);
  // Every entry the top-k step reads is written first by the logits step, so the
  // array needs no clearing between calls.
  stq_status st;
  {
    StqTimed tm(STQ_K_ROUTER_LOGITS, s);
    st = stq_launch(router_logits_kernel, dim3(unsigned(ceil_div(E, 16) * KS)), dim3(256), 0, s, x, w_router, T, H, E,
                    KS, scratch);
  }
  if (st != STQ_OK) return st;
  StqTimed tm(STQ_K_ROUTER_TOPK, s);
  return E <= 256 ? stq_launch(router_topk_kernel<8>, dim3(unsigned(ceil_div(T, 4))), dim3(128), 0, s, scratch, T, E, KS, k,
                               topk_ids, topk_w)
                  : stq_launch(router_topk_kernel<32>, dim3(unsigned(ceil_div(T, 4))), dim3(128), 0, s, scratch, T, E, KS,
                               k, topk_ids, topk_w);
}
