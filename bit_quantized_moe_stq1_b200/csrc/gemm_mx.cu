// W4A8 grouped GEMM on the sm_100a tensor cores: MXFP4 (E2M1, UE8M0 per 32 along K)
// weights x MXFP8 (E4M3, UE8M0 per 32) activations, FP32 accumulators in TMEM.
// "Hy4-preview-SF-WFP4AFP8", "Quant Diff": routed experts are FP4 E2M1 weights with
// FP8 E4M3 activations, group 32, UE8M0 scales; the page notes that FP4 GEMMs need
// Blackwell.
//
// A work item is a 128 (weight rows) x NT (tokens of one expert) tile over all of K:
//   warps 0, 6 producers (alternate stages): per 128-k stage, TMA tile loads of the weights (E2M1 expanded
//              to one 16-element group per 16 bytes by the TMA, 128-byte swizzle) and of
//              the token activations (E4M3), and the UE8M0 scales of both, re-laid by the
//              warp into the scale-factor atom the MMA reads (row m of a 128-row block at
//              byte (m % 32) * 16 + (m / 32) * 4 + kb);
//   warp 1     TMEM allocation and, from one thread, tcgen05.cp of the scales into TMEM
//              and four tcgen05.mma.kind::mxf8f6f4.block_scale (K = 32 each) per stage;
//   warps 2-5  epilogue from TMEM: FP32 expert outputs, or (gate/up pair) SwiGLU and the
//              MXFP8 re-quantisation of h along the intermediate dimension.
// All mbarrier waits are bounded (STQ_ERR_TIMEOUT in the error word, then a clean exit
// that waits for in-flight copies and frees TMEM).

#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "gemm_common.cuh"
#include "tma.cuh"

namespace {

using gemm::Item;
using gemm::load_sf;
using gemm::store_sf;

constexpr int kKT = 128;                          // k per stage
constexpr int kATile = 128 * 128;                 // smem bytes of one 128 x 128 E2M1 tile (expanded)
constexpr uint32_t kATx = 128 * 128 / 2;          // bytes the TMA delivers for it
constexpr int kSf = 512;                          // one scale-factor atom: 128 rows x 4 k-blocks
// Two CTAs share an SM (half the shared memory each) unless the two accumulator buffers
// of a wider N tile need more than half of the SM's 512 TMEM columns.  The 240-wide tile
// (prefill) takes 4 stages of 48 KB.
constexpr int ctas_per_sm(int nt) { return nt <= 64 ? 2 : 1; }
constexpr int smem_budget(int nt) {
  return ctas_per_sm(nt) == 2 ? 112 * 1024 : nt > 128 ? 226 * 1024 : 200 * 1024;
}

// PAIR = the gate/up pair of one expert: the 128-row A tile holds 64 gate rows (TMEM
// lanes 0-63) and the same 64 rows of the up projection (lanes 64-127), so one MMA per
// k-block produces both and the epilogue pairs lane r with lane r + 64.
// A8: the weights are E4M3 (MXFP8, one byte per weight) instead of E2M1.
template <int NT, bool PAIR, bool A8 = false>
struct Cfg {
  static constexpr int kB = NT * 128;
  static constexpr int kSfbAtoms = NT > 128 ? 2 : 1;   // activation scale factors: 128 rows per atom
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kATile;
  static constexpr int kOffSfa = kOffB + kB;
  static constexpr int kOffSfb = kOffSfa + kSf;
  static constexpr int kStageRaw = kOffSfb + kSfbAtoms * kSf;
  static constexpr int kStage = (kStageRaw + 1023) / 1024 * 1024;
  static constexpr int kCtasPerSm = ctas_per_sm(NT);
  static constexpr int kUBuf = PAIR ? 4 * 32 * 9 * 4 : 0;   // gate/up exchange of the epilogue (pitch 9 words)
  static constexpr int kStagesRaw = (smem_budget(NT) - 2048 - kUBuf) / kStage;
  // even: the two producer warps own alternate stages (producer p fills stages 2i + p);
  // an odd count (one producer with a stage more than the other) measured slower
  static constexpr int kStages = (kStagesRaw > 8 ? 8 : kStagesRaw) & ~1;
  static constexpr int stages_of(int) { return kStages / 2; }
  static constexpr int kSmem = kStages * kStage + kUBuf + 1024 /* barriers */ + 1024 /* alignment */;
  static constexpr int kRowsPerTile = PAIR ? 64 : 128;   // output features per CTA
  // TMEM: accumulator buffers at columns 0 and kAccStride (tile i uses buffer i & 1), and
  // the scale factors of the current k-block (after both buffers, or between them for the
  // 240-wide tile: 240..243 weights, 244..251 the two activation atoms).
  static constexpr int kAccStride = NT > 128 ? 256 : NT;
  static constexpr int kColSfa = NT > 128 ? NT : 2 * NT;
  static constexpr int kColSfb = kColSfa + 4;
  static constexpr int kColsUsed = NT > 128 ? 256 + NT : 2 * NT + 4 + 4 * kSfbAtoms;
  static constexpr uint32_t kCols = kColsUsed <= 32 ? 32 : kColsUsed <= 64 ? 64 : kColsUsed <= 128 ? 128
                                   : kColsUsed <= 256 ? 256 : 512;
  static constexpr uint32_t kTx = (A8 ? uint32_t(kATile) : kATx) + uint32_t(kB);
  static_assert(kStages >= 2, "shared memory budget (one stage per producer at least)");
  static_assert(NT % 16 == 0 && NT >= 16 && (NT <= 128 || NT == 240), "tile N");
  static_assert(NT <= 128 || kColSfb + 8 <= 256, "scale factors between the accumulators");
  static_assert(kCtasPerSm * kCols <= 512, "TMEM columns");
};

struct GemmProblem {
  gemm::Tiling tiles;           // tiles.R = weight rows per expert
  int K, Ptot;                  // reduction length, activation rows
  const uint8_t* sa;            // weight scales [E*R][K/32] (gate scales for a pair)
  const uint8_t* sa2;           // up-projection scales (gate/up pair)
  const uint8_t* sb;            // activation scales [Ptot][K/32]
  gemm::EpiOut out;             // out.R = tiles.R
  int32_t* err;
};

// Pair tile: slices m1 = 0, 1 are gate rows row0 + lane + 32*m1, slices 2, 3 the same
// rows of the up projection.
__device__ __forceinline__ void load_sf_pair(uint32_t (&v)[4], const uint8_t* gsrc, const uint8_t* usrc, int row0,
                                             int k32, int kt, int nk, int lane) {
#pragma unroll
  for (int m1 = 0; m1 < 4; ++m1) {
    const uint8_t* src = m1 < 2 ? gsrc : usrc;
    const int r = row0 + lane + 32 * (m1 & 1);
    v[m1] = kt < nk ? __ldg(reinterpret_cast<const uint32_t*>(src + size_t(r) * k32 + size_t(kt) * 4)) : 0u;
  }
}

// Persistent: CTA b takes items b, b + gridDim.x, ...  Warp roles: warps 0 and 6 load
// (TMA for the operands, a register ring kPf of their stages ahead for the scale
// factors), warp 1 issues the MMAs (one elected thread), warps 2-5 drain the
// accumulators.  The smem
// ring and its barrier phases run on across items; the accumulator is double-buffered
// in TMEM (tfull / tempty), so the epilogue of one item overlaps the MMAs of the next.
constexpr int kGemmThreads = 224;  // producer, MMA, 4 epilogue warps, second producer
constexpr int kProducer2 = 6;

template <int NT, bool PAIR, bool A8>
__global__ void __launch_bounds__(kGemmThreads, Cfg<NT, PAIR, A8>::kCtasPerSm)
    w4a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                     const __grid_constant__ CUtensorMap tmB, GemmProblem p) {
  using C = Cfg<NT, PAIR, A8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ubuf = reinterpret_cast<float*>(smem + C::kStages * C::kStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage + C::kUBuf);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;   // [2]
  uint64_t* tempty = tfull + 2;           // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = p.tiles.R / C::kRowsPerTile;
  const int G = gridDim.x;
  const int nk = p.K / kKT;
  const int k32 = p.K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 4);
    }
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&tmA);
    if (PAIR) tc::prefetch_tensormap(&tmA2);
    tc::prefetch_tensormap(&tmB);
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, C::kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  stq_pdl_begin();   // barriers and TMEM are set up; from here on global memory is read

  if (warp == 0 || warp == kProducer2) {
    // ---------------------------------------------------------------- producers
    // Two producer warps take alternate k-steps (global step g = item * nk + kt, producer
    // g & 1), so the scale-factor stores and proxy fences of one stage overlap the other's.
    // Producer p's j-th step uses stage 2 (j % n_p) + p, round j / n_p, with n_p the number
    // of stages of parity p: no stage is shared, so each warp's final wait for its own
    // loads is exact.
    constexpr int kPf = 8;
    const int pid = warp == 0 ? 0 : 1;
    int last_round[C::kStages];
#pragma unroll
    for (int s = 0; s < C::kStages; ++s) last_round[s] = -1;
    // When nk is a multiple of the ring (2 kPf steps), the last steps of an item read the
    // next item's first scale factors into the ring, so an item boundary costs no wait.
    const bool cross = nk % (2 * kPf) == 0;
    bool ok = true;
    constexpr int kAt = C::kSfbAtoms;
    uint32_t ra[kPf][4], rb[kPf][kAt][4];
    for (int it = 0; ok; ++it) {
      const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, C::kRowsPerTile, NT);
      if (!I.valid) break;
      Item In{};
      if (cross) In = gemm::get_item(p.tiles, blockIdx.x + (it + 1) * G, MT, C::kRowsPerTile, NT);
      const int kt0 = ((pid - it * nk) % 2 + 2) % 2;  // first k-step of this item for this producer
      if (!cross || it == 0) {
#pragma unroll
        for (int d = 0; d < kPf; ++d) {
          if (PAIR) load_sf_pair(ra[d], p.sa, p.sa2, I.arow, k32, kt0 + 2 * d, nk, lane);
          else load_sf(ra[d], p.sa, I.arow, 128, 0x7fffffff, k32, kt0 + 2 * d, nk, lane);
#pragma unroll
          for (int at = 0; at < kAt; ++at)
            load_sf(rb[d][at], p.sb, I.brow + 128 * at, NT - 128 * at, p.Ptot, k32, kt0 + 2 * d, nk, lane);
        }
      }
      for (int k0 = kt0; k0 < nk && ok; k0 += 2 * kPf) {
#pragma unroll
        for (int d = 0; d < kPf; ++d) {
          const int kt = k0 + 2 * d;
          if (kt >= nk) break;
          const int j = (it * nk + kt) >> 1, np = C::stages_of(pid);
          const int s = 2 * (j % np) + pid, r = j / np;
          if (r > 0 && !tc::mbar_wait(&empty[s], (r - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * C::kStage;
          store_sf(st + C::kOffSfa, ra[d], lane);
#pragma unroll
          for (int at = 0; at < kAt; ++at) store_sf(st + C::kOffSfb + at * kSf, rb[d][at], lane);
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tc::mbar_arrive_expect_tx(&full[s], C::kTx);
            if (PAIR) {
              tc::tma_load_2d(st + C::kOffA, &tmA, kt * kKT, I.arow, &full[s]);              // gate rows: lanes 0-63
              tc::tma_load_2d(st + C::kOffA + kATile / 2, &tmA2, kt * kKT, I.arow, &full[s]);  // up rows: 64-127
            } else {
              tc::tma_load_2d(st + C::kOffA, &tmA, kt * kKT, I.arow, &full[s]);
            }
            tc::tma_load_2d(st + C::kOffB, &tmB, kt * kKT, I.brow, &full[s]);
          }
          last_round[s] = r;
          const int kn = kt + 2 * kPf;
          const Item& J = (cross && kn >= nk) ? In : I;  // In.valid is false past the last item
          const int kj = (cross && kn >= nk) ? kn - nk : kn;
          const int nkj = J.valid ? nk : 0;               // an invalid item reads zeros
          if (PAIR) load_sf_pair(ra[d], p.sa, p.sa2, J.arow, k32, kj, nkj, lane);
          else load_sf(ra[d], p.sa, J.arow, 128, 0x7fffffff, k32, kj, nkj, lane);
#pragma unroll
          for (int at = 0; at < kAt; ++at)
            load_sf(rb[d][at], p.sb, J.brow + 128 * at, NT - 128 * at, p.Ptot, k32, kj, nkj, lane);
        }
      }
    }
    // every load this warp issued has landed before the CTA may exit
    for (int q = 0; q < C::kStages; ++q)
      if (last_round[q] >= 0) tc::mbar_wait(&full[q], last_round[q] & 1, p.err);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      int g = 0;  // global k-step
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, C::kRowsPerTile, NT);
        if (!I.valid) break;
        const int ncols = gemm::item_cols(I, NT);
        const int buf = it & 1;
        if (it >= 2 && !tc::mbar_wait(&tempty[buf], ((it >> 1) - 1) & 1, p.err)) break;
        tc::fence_after_sync();
        const uint32_t acc_col = tmem + uint32_t(buf * C::kAccStride);
        for (int kt = 0; kt < nk; ++kt, ++g) {
          const int j = g >> 1, np = C::stages_of(g & 1);
          const int s = 2 * (j % np) + (g & 1), r = j / np;
          if (!tc::mbar_wait(&full[s], r & 1, p.err)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          uint8_t* st = smem + s * C::kStage;
          tc::cp_sf_32x128b_x4(tmem + C::kColSfa, tc::smem_desc_sf(tc::smem_u32(st + C::kOffSfa)));
#pragma unroll
          for (int at = 0; at < C::kSfbAtoms; ++at)
            tc::cp_sf_32x128b_x4(tmem + C::kColSfb + 4 * at, tc::smem_desc_sf(tc::smem_u32(st + C::kOffSfb + at * kSf)));
          const uint64_t da = tc::smem_desc_sw128(tc::smem_u32(st + C::kOffA));
          const uint64_t db = tc::smem_desc_sw128(tc::smem_u32(st + C::kOffB));
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t idesc = tc::idesc_mxf8f6f4_ab(ncols, A8 ? tc::kFmtE4M3 : tc::kFmtE2M1, tc::kFmtE4M3,
                                                         uint32_t(kb), uint32_t(kb));
            const uint32_t acc = (kt > 0 || kb > 0) ? 1u : 0u;
            tc::mma_mxf8f6f4(acc_col, da + 2 * kb, db + 2 * kb, idesc, (tmem + C::kColSfa) | (uint32_t(kb) << 30),
                             (tmem + C::kColSfb) | (uint32_t(kb) << 30), acc);
          }
          tc::commit(&empty[s]);
        }
        tc::commit(&tfull[buf]);  // also after an aborted item, so the epilogue never waits for ever
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    for (int it = 0;; ++it) {
      const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, C::kRowsPerTile, NT);
      if (!I.valid) break;
      const int buf = it & 1;
      bool ok = tc::mbar_wait(&tfull[buf], (it >> 1) & 1, p.err);
      // the four epilogue warps meet at named barriers, so they agree on ok first
      if constexpr (PAIR) ok = gemm::all_of_epilogue(ok);
      if (!ok) break;
      tc::fence_after_sync();
      gemm::epilogue_tile<NT, PAIR>(tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * C::kAccStride), I, p.out, ubuf,
                                    q, lane);
      // this warp's reads of the buffer are complete: hand it back to the MMA warp
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[buf]);
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, C::kCols);
  }
}

// A barrier nothing arrives at, waited on through the kernels' bounded wait.
__global__ void wait_selftest_kernel(int32_t* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    tc::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) tc::mbar_wait(&bar, 0, err);
  __syncthreads();
}

// N tiles of every touched expert: (expert, first token of the tile); one CTA.
__global__ void __launch_bounds__(1024) mx_plan_kernel(const int32_t* __restrict__ counts, int E, int nt,
                                                       int2* __restrict__ tiles, int32_t* __restrict__ n_tiles) {
  stq_pdl_begin();
  __shared__ int wsum[32];
  __shared__ int total;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = tid < E ? counts[tid] : 0;
  const int v = (c + nt - 1) / nt;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int s = wsum[lane];
    int si = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, si, o);
      if (lane >= o) si += n;
    }
    wsum[lane] = si - s;
    if (lane == 31) total = si;
  }
  __syncthreads();
  const int base = incl - v + wsum[warp];
  for (int j = 0; j < v; ++j) tiles[base + j] = make_int2(tid, j * nt);
  if (tid == 0) *n_tiles = total;
}

// ----------------------------------------------------------------------------- host side



// Persistent launch over p.tiles.max_items work items: at most kCtasPerSm CTAs per SM.
template <int NT, bool PAIR, bool A8>
stq_status launch_gemm(const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b, const GemmProblem& p,
                       cudaStream_t s) {
  using C = Cfg<NT, PAIR, A8>;
  static StqSmemOptIn optin;
  const stq_status st = optin.ensure(w4a8_gemm_kernel<NT, PAIR, A8>, C::kSmem);
  if (st != STQ_OK) return st;
  if (p.tiles.max_items <= 0) return STQ_OK;
  const unsigned grid = unsigned(stq_persistent_grid(p.tiles.max_items, C::kCtasPerSm));
  return stq_launch(w4a8_gemm_kernel<NT, PAIR, A8>, dim3(grid), dim3(kGemmThreads), C::kSmem, s, a, a2, b, p);
}

template <bool PAIR, bool A8 = false>
stq_status launch_nt(int nt, const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b, const GemmProblem& p,
                     cudaStream_t s) {
  switch (nt) {
    case 16: return launch_gemm<16, PAIR, A8>(a, a2, b, p, s);
    case 32: return launch_gemm<32, PAIR, A8>(a, a2, b, p, s);
    case 64: return launch_gemm<64, PAIR, A8>(a, a2, b, p, s);
    case 240: return launch_gemm<240, PAIR, A8>(a, a2, b, p, s);
    default: return launch_gemm<128, PAIR, A8>(a, a2, b, p, s);
  }
}

int pick_nt(int64_t tokens_per_expert) {
  return tokens_per_expert <= 16 ? 16 : tokens_per_expert <= 32 ? 32 : tokens_per_expert <= 64 ? 64
         : tokens_per_expert < 128 ? 128 : 240;
}

// The next narrower N tile.
int narrower_nt(int nt) { return nt > 128 ? 128 : nt / 2; }

}  // namespace

stq_status stq_tile_plan_launch(const int32_t* counts, int E, int nt, int2* tiles, int32_t* n_tiles, cudaStream_t s) {
  StqTimed tm(STQ_K_PLAN, s);
  return stq_launch(mx_plan_kernel, dim3(1), dim3(1024), 0, s, counts, E, nt, tiles, n_tiles);
}

stq_status moe_mx_experts(const MoeArgs& a, int slots, cudaStream_t s) {
  (void)slots;
  const int P = a.P;
  // 1. activations -> MXFP8 in sorted (expert-grouped) order
  stq_status st = stq_mxfp8_quantize_scatter_launch(a.x, a.T, a.H, a.inv, a.k, P, a.err, a.xq, a.xs, s);
  if (st != STQ_OK) return st;
  // 2. N tiles of the touched experts: the down projection takes the 240-wide tile from
  // 128 tokens per expert on average, the gate/up pair (whose SwiGLU/MXFP8 epilogue and
  // item balance measured slower there) at most 128
  const int slots_ = a.E < P ? a.E : P;
  // the CTA-pair GEMM from this many routed tokens per expert on average (0: not used; it
  // measured slower than the one-CTA kernels on the 4096-token prefill layer)
  constexpr int64_t kPairFromTokensPerExpert = 0;
  if (kPairFromTokensPerExpert > 0 && int64_t(P) / slots_ >= kPairFromTokensPerExpert)
    return moe_mx_experts_pair(a, slots_, s);
  // The gate/up pair with the tokens on M (gemm_mx_tm.cu) from this many routed tokens per
  // expert on average.  The down projection stays on this file's 240-token N tile unless
  // kDownTokensOnM: its token-major launch (N = 192, two accumulators) measured 0.99 ms
  // against 0.82 ms on the 4096-token prefill layer.
  constexpr int64_t kTokensOnMFrom = 32;
  constexpr bool kDownTokensOnM = false;
  const bool down_tokens_on_m = kDownTokensOnM && moe_mx_down_tm_fits(a);
  const bool tokens_on_m = int64_t(P) / slots_ >= kTokensOnMFrom;
  const int nt_dn = pick_nt(int64_t(P) / slots_);
  const int nt = nt_dn > 128 ? 128 : nt_dn;
  if (tokens_on_m) {
    if ((st = moe_mx_gate_up_tm(a, slots_, s)) != STQ_OK) return st;
    if (down_tokens_on_m) return moe_mx_down_tm(a, slots_, s);
  } else if ((st = stq_tile_plan_launch(a.counts, a.E, nt, a.ntiles, a.n_ntiles, s)) != STQ_OK) {
    return st;
  }
  const int max_tiles = P / nt + slots_;
  // 3. gate/up pair with SwiGLU and MXFP8 h
  CUtensorMap mg, mu, mx, md, mh;
  if (!tma::map_e2m1(&mg, a.wg, uint64_t(a.H), uint64_t(a.E) * a.I, 64) ||
      !tma::map_e2m1(&mu, a.wu, uint64_t(a.H), uint64_t(a.E) * a.I, 64) || !tma::map_u8(&mx, a.xq, a.H, P, nt) ||
      !tma::map_e2m1(&md, a.wd, uint64_t(a.I), uint64_t(a.E) * a.H) || !tma::map_u8(&mh, a.hq, a.I, P, nt_dn))
    return STQ_ERR_CUDA;
  GemmProblem gp{};
  gp.tiles.R = a.I;
  gp.tiles.offsets = a.offsets;
  gp.tiles.ntiles = a.ntiles;
  gp.tiles.n_ntiles = a.n_ntiles;
  gp.tiles.max_items = max_tiles * (a.I / 64);
  gp.K = a.H;
  gp.Ptot = P;
  gp.sa = a.gsc;
  gp.sa2 = a.usc;
  gp.sb = a.xs;
  gp.out.R = a.I;
  gp.out.hq = a.hq;
  gp.out.hs = a.hs;
  gp.err = a.err;
  if (!tokens_on_m) {
    StqTimed tm(STQ_K_GATE_UP_MX, s);
    st = launch_nt<true>(nt, mg, mu, mx, gp, s);
  }
  if (st != STQ_OK) return st;
  // 4. down (the N-tile plan is redone for its tile width once the gate/up launch is done with it)
  if ((tokens_on_m || nt_dn != nt) && (st = stq_tile_plan_launch(a.counts, a.E, nt_dn, a.ntiles, a.n_ntiles, s)) != STQ_OK)
    return st;
  GemmProblem dp = gp;
  dp.tiles.R = a.H;
  dp.tiles.max_items = (P / nt_dn + slots_) * (a.H / 128);
  dp.K = a.I;
  dp.sa = a.dsc;
  dp.sa2 = nullptr;
  dp.sb = a.hs;
  dp.out = gemm::EpiOut{a.H, a.Y, nullptr, nullptr};
  {
    StqTimed tm(STQ_K_DOWN_MX, s);
    st = launch_nt<false>(nt_dn, md, md, mh, dp, s);
  }
  return st;
}

// The MXFP8 shared expert ("Hy4-preview-SF-WFP4AFP8", "Quant Diff": shared experts are
// MXFP8 W8A8 g32): the same GEMM with E4M3 weights, over the T tokens as one dense
// expert.  Its activations and h take the rows P.. of the MXFP8 workspace regions, its
// outputs the rows P.. of Y.  N tile from the token count, halved while the gate/up
// launch would leave SMs idle.
stq_status moe_shared_expert_mx8(const MoeArgs& a, cudaStream_t s) {
  const int T = a.T, P = a.P;
  uint8_t* xq = a.xq + size_t(P) * a.H;
  uint8_t* xs = a.xs + size_t(P) * (a.H / 32);
  uint8_t* hq = a.hq + size_t(P) * a.I;
  uint8_t* hs = a.hs + size_t(P) * (a.I / 32);
  stq_status st = stq_mxfp8_quantize_launch(a.x, T, a.H, xq, xs, s);
  if (st != STQ_OK) return st;
  int nt = pick_nt(T);
  if (nt > 128) nt = 128;  // the 240-wide tile measured slower for the gate/up pair
  while (nt > 16 && (a.I / 64) * ((T + nt - 1) / nt) < 148) nt = narrower_nt(nt);
  const int ntile = (T + nt - 1) / nt;
  CUtensorMap mg, mu, mx, md, mh;
  if (!tma::map_u8(&mg, a.sgq, uint64_t(a.H), uint64_t(a.I), 64) ||
      !tma::map_u8(&mu, a.suq, uint64_t(a.H), uint64_t(a.I), 64) ||
      !tma::map_u8(&md, a.sdq, uint64_t(a.I), uint64_t(a.H), 128) || !tma::map_u8(&mx, xq, a.H, T, nt) ||
      !tma::map_u8(&mh, hq, a.I, T, nt))
    return STQ_ERR_CUDA;
  GemmProblem gp{};
  gp.tiles.R = a.I;
  gp.tiles.dense_M = T;
  gp.tiles.max_items = ntile * (a.I / 64);
  gp.K = a.H;
  gp.Ptot = T;
  gp.sa = a.sgs;
  gp.sa2 = a.sus;
  gp.sb = xs;
  gp.out = gemm::EpiOut{a.I, nullptr, hq, hs};
  gp.err = a.err;
  {
    StqTimed tm(STQ_K_SHARED_GATE_UP, s);
    st = launch_nt<true, true>(nt, mg, mu, mx, gp, s);
  }
  if (st != STQ_OK) return st;
  GemmProblem dp = gp;
  dp.tiles.R = a.H;
  dp.tiles.max_items = ntile * (a.H / 128);
  dp.K = a.I;
  dp.sa = a.sds;
  dp.sa2 = nullptr;
  dp.sb = hs;
  dp.out = gemm::EpiOut{a.H, a.Y + size_t(P) * a.H, nullptr, nullptr};
  StqTimed tm(STQ_K_SHARED_DOWN, s);
  return launch_nt<false, true>(nt, md, md, mh, dp, s);
}

extern "C" stq_status w4a8_gemm(const uint8_t* w_codes, const uint8_t* w_scales, int64_t N, int64_t K,
                                const uint8_t* a_codes, const uint8_t* a_scales, int64_t M, float* y, int32_t* err,
                                stq_stream_t stream) {
  STQ_HOST_CHECK(N >= 0 && K >= 0 && M >= 0, STQ_ERR_INVALID_ARG);
  if (N == 0 || M == 0) return STQ_OK;
  STQ_HOST_CHECK(w_codes && w_scales && a_codes && a_scales && y, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(N % 128 == 0 && K % 128 == 0 && K > 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(N < (int64_t(1) << 31) && M < (int64_t(1) << 31) && K < (int64_t(1) << 31), STQ_ERR_SHAPE);
  STQ_HOST_CHECK((reinterpret_cast<uintptr_t>(w_codes) & 31u) == 0 && stq_aligned16(a_codes) && stq_aligned16(y) &&
                     (reinterpret_cast<uintptr_t>(w_scales) & 3u) == 0 &&
                     (reinterpret_cast<uintptr_t>(a_scales) & 3u) == 0,
                 STQ_ERR_ALIGN);
  cudaStream_t s = stq_cuda_stream(stream);
  int nt = pick_nt(M);
  while (nt > 16 && (N / 128) * ((M + nt - 1) / nt) < 148) nt = narrower_nt(nt);  // fill the SMs
  CUtensorMap ma, mb;
  if (!tma::map_e2m1(&ma, w_codes, uint64_t(K), uint64_t(N)) || !tma::map_u8(&mb, a_codes, uint64_t(K), uint64_t(M), nt))
    return STQ_ERR_CUDA;
  GemmProblem p{};
  p.tiles.R = int(N);
  p.tiles.dense_M = int(M);
  p.K = int(K);
  p.Ptot = int(M);
  p.sa = w_scales;
  p.sb = a_scales;
  p.out = gemm::EpiOut{int(N), y, nullptr, nullptr};
  p.err = err;
  const int64_t items = (N / 128) * ((M + nt - 1) / nt);
  STQ_HOST_CHECK(items < (int64_t(1) << 31), STQ_ERR_SHAPE);
  p.tiles.max_items = int(items);
  StqTimed tm(STQ_K_GEMM, s);
  return launch_nt<false>(nt, ma, ma, mb, p, s);
}

extern "C" stq_status stq_wait_selftest(int32_t* err, stq_stream_t stream) {
  STQ_HOST_CHECK(err != nullptr, STQ_ERR_INVALID_ARG);
  wait_selftest_kernel<<<1, 32, 0, stq_cuda_stream(stream)>>>(err);
  return stq_launch_status();
}
