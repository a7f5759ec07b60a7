// W4A8 grouped GEMM of the prefill regime on CTA pairs: the same product as gemm_mx.cu
// (MXFP4 E2M1 weights x MXFP8 E4M3 activations, UE8M0 scales per 32 along K, FP32
// accumulators in TMEM; "Hy4-preview-SF-WFP4AFP8", "Quant Diff"), with one M = 256
// tcgen05.mma.cta_group::2 per k-block over two CTAs of a cluster.
//
// Why pairs: at M = 128 one k-block's MMA reads 4 KB of weights and N x 32 bytes of
// activations from shared memory while the TMA writes the next stages into it, and the
// two together exceed the SM's shared-memory bandwidth.  With a pair each SM holds only
// its 128 weight rows and half of the N activation rows, the MMA covers 256 x N outputs,
// and per SM the reads and writes of one k-block fit the bandwidth at N = 240.
//
// A work item is 256 weight rows (gate/up: 128 features, each CTA 64 gate + the same 64 up
// rows) x up to 240 tokens of one expert over all of K.  Per item both CTAs:
//   warps 5-8 (producers, 128-k stages in turn): TMA of the CTA's 128 weight rows and of
//      its half of the N token rows (rows n0 + rank * N/2 ..), whose completion bytes count
//      on the rank-0 CTA's barrier; the UE8M0 scales re-laid into the scale-factor atoms
//      (the CTA's own 128 weight rows, and the activations of all N tokens), which rank 1's
//      producer releases to rank 0 with an arrival on rank 0's barrier;
//   warp 0: TMEM (both CTAs, cta_group::2); in the rank-0 CTA one thread issues the scale
//      copies and four M = 256 MMAs per stage, and commits to both CTAs' barriers;
//   warps 1-4: the CTA's epilogue from its own TMEM (its 128 rows x N tokens).
// Barriers: full[s] (rank 0; both CTAs' producers and loads), empty[s] (both; one commit),
// tfull[b] (both; one commit), tempty[b] (rank 0; the eight epilogue warps).
// Every wait is bounded; after a timeout each role records STQ_ERR_TIMEOUT, keeps going to
// the end, and both CTAs meet at a final cluster barrier before TMEM is freed, so no CTA
// exits while the pair's copies or MMAs can still touch its memory.  No load multicasts.

#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "gemm_common.cuh"
#include "tma.cuh"

namespace {

using gemm::Item;
using gemm::load_sf;
using gemm::store_sf;

constexpr int kKT = 128;                      // k per stage
constexpr int kATile = 128 * 128;             // one CTA's 128 x 128 E2M1 weight tile (expanded)
constexpr uint32_t kATx = 128 * 128 / 2;      // bytes the TMA delivers for it
constexpr int kSf = 512;                      // scale-factor atom: 128 rows x 4 k-blocks
constexpr int kUBuf = 4 * 32 * 9 * 4;         // gate/up exchange of the epilogue
// Warps: 0 MMA (rank 0 issues; TMEM in both), 1-4 epilogue (TMEM lane quarters 1, 2, 3, 0),
// 5-8 producers.  Rank 0's producers lay out both CTAs' scale factors (about 2,000 cycles per
// stage, measured), so four of them take the stages in turn and keep ahead of the MMAs.
constexpr int kProducers = 4;
constexpr int kProducer0 = 5;
constexpr int kThreads = 32 * (kProducer0 + kProducers);
constexpr uint32_t kCols = 512;

// NT tokens per item (both CTAs; each holds NT/2 token rows): shared-memory stages and the
// TMEM columns of one CTA: two accumulators (at 0 and NT, or 0 and 256 for NT > 128) and
// the scale factors of the current stage (after them, or between them for NT > 128).
template <int NT>
struct PairCfg {
  static constexpr int kNHalf = NT / 2;
  static constexpr int kBTile = kNHalf * 128;
  static constexpr int kSfbAtoms = (NT + 127) / 128;
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kATile;
  static constexpr int kOffSfa = kOffB + kBTile;
  static constexpr int kOffSfb = kOffSfa + kSf;
  static constexpr int kStage = (kOffSfb + kSfbAtoms * kSf + 1023) / 1024 * 1024;
  static constexpr int kStagesRaw = ((226 * 1024 - 2048 - kUBuf) / kStage) & ~(kProducers - 1);
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  static constexpr int kSmem = kStages * kStage + kUBuf + 1024 /* barriers */ + 1024 /* alignment */;
  static constexpr uint32_t kTxPair = 2 * (kATx + uint32_t(kBTile));   // both CTAs' bytes per stage
  static constexpr int kAccStride = NT > 128 ? 256 : NT;
  static constexpr int kColSfa = NT > 128 ? NT : 2 * NT;
  static constexpr int kColSfb = kColSfa + 4;
  static_assert(NT % 16 == 0 && NT <= 240, "tile N");
  static_assert(kStages >= kProducers, "stages");
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kBTile % 1024 == 0 && kStage % 1024 == 0, "128-byte swizzle atoms");
  static_assert(kColSfb + 4 * kSfbAtoms <= (NT > 128 ? 256 : 512), "TMEM columns");
};

struct PairProblem {
  gemm::Tiling tiles;           // tiles.R = weight rows per expert; tile plan of NT tokens
  int K, Ptot;
  const uint8_t* sa;            // weight scales [E*R][K/32] (gate scales for a pair)
  const uint8_t* sa2;           // up-projection scales (gate/up pair)
  const uint8_t* sb;            // activation scales [Ptot][K/32]
  gemm::EpiOut out;
  int32_t* err;
};

// Scales of a gate/up CTA half: slices 0, 1 = gate rows row0 + lane + 32*m1, 2, 3 = up rows.
__device__ __forceinline__ void load_sf_gu(uint32_t (&v)[4], const uint8_t* gsrc, const uint8_t* usrc, int row0,
                                           int k32, int kt, int nk, int lane) {
#pragma unroll
  for (int m1 = 0; m1 < 4; ++m1) {
    const uint8_t* src = m1 < 2 ? gsrc : usrc;
    const int r = row0 + lane + 32 * (m1 & 1);
    v[m1] = kt < nk ? __ldg(reinterpret_cast<const uint32_t*>(src + size_t(r) * k32 + size_t(kt) * 4)) : 0u;
  }
}

// Cluster item -> this CTA's view: rows_per_cta weight rows starting at the CTA's half
// (the epilogue's M tile index is 2 * mt + rank).
template <int NT>
__device__ __forceinline__ Item cta_item(const gemm::Tiling& t, int item, int MT2, int rows_per_cta, int rank) {
  Item I = gemm::get_item(t, item, MT2, 2 * rows_per_cta, NT);
  if (!I.valid) return I;
  I.mt = 2 * I.mt + rank;
  I.arow = I.e * t.R + I.mt * rows_per_cta;
  return I;
}

template <int NT, bool PAIR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    w4a8_pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA2,
                          const __grid_constant__ CUtensorMap tmB, PairProblem p) {
  using C = PairCfg<NT>;
  constexpr int kStages = C::kStages, kStage = C::kStage, kOffA = C::kOffA, kOffB = C::kOffB, kOffSfa = C::kOffSfa,
                kOffSfb = C::kOffSfb, kAccStride = C::kAccStride, kColSfa = C::kColSfa, kColSfb = C::kColSfb;
  constexpr uint32_t kTxPair = C::kTxPair;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ubuf = reinterpret_cast<float*>(smem + kStages * kStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStage + kUBuf);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;   // [2]
  uint64_t* tempty = tfull + 2;        // [2]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = int(tc::cluster_ctarank());
  constexpr int kRowsPerCta = PAIR ? 64 : 128;   // output features of one CTA per item
  const int MT2 = p.tiles.R / (2 * kRowsPerCta);
  const int NC = gridDim.x / 2;                   // clusters
  const int cid = blockIdx.x / 2;
  const int nk = p.K / kKT;
  const int k32 = p.K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 2);                 // both CTAs' producers (rank 0's with the bytes)
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], 8);               // four epilogue warps of each CTA
    }
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&tmA);
    if (PAIR) tc::prefetch_tensormap(&tmA2);
    tc::prefetch_tensormap(&tmB);
  }
  if (warp == 0) tc::tmem_alloc_pair(tmem_holder, kCols);
  tc::fence_before_sync();
  tc::cluster_sync();   // both CTAs' barriers are initialised before any peer signals them
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  stq_pdl_begin();   // barriers and TMEM are set up; from here on global memory is read

  if (warp >= kProducer0) {
    // ---------------------------------------------------------------- producers
    // Global k-step g = item * nk + kt; producer pid takes the steps of its parity, its j-th
    // step (j = g / kProducers) at stage kProducers (j % np) + pid, round j / np
    // (np = kStages / kProducers).  The
    // scale factors, which the warp re-lays through registers, are read kLook of its steps
    // ahead (a second cursor over the same steps), so their latency hides behind earlier
    // stages, across item boundaries too.
    const int pid = warp - kProducer0;
    constexpr int np = kStages / kProducers;
    constexpr int kLook = 4;
    int last_round[kStages];
#pragma unroll
    for (int q = 0; q < kStages; ++q) last_round[q] = -1;
    int cg = pid, cit = -1, cncols = 0;   // look-ahead cursor
    Item CI{};
    // each CTA lays out its own scale factors: its 128 weight rows, and the activations of
    // all N tokens (both CTAs need those)
    auto sf_load = [&](uint32_t (&va)[4], uint32_t (&vb0)[4], uint32_t (&vb1)[4]) {
      const int it = cg / nk, kt = cg % nk;
      if (it != cit) {
        cit = it;
        CI = cta_item<NT>(p.tiles, cid + it * NC, MT2, kRowsPerCta, rank);
        cncols = CI.valid ? gemm::item_cols(CI, NT) : 0;
      }
      const int nkj = CI.valid ? nk : 0;   // past the last item: zeros, no loads
      if (PAIR) load_sf_gu(va, p.sa, p.sa2, CI.arow, k32, kt, nkj, lane);
      else load_sf(va, p.sa, CI.arow, 128, 0x7fffffff, k32, kt, nkj, lane);
      load_sf(vb0, p.sb, CI.brow, cncols, p.Ptot, k32, kt, nkj, lane);
      if (C::kSfbAtoms > 1) load_sf(vb1, p.sb, CI.brow + 128, cncols - 128, p.Ptot, k32, kt, nkj, lane);
      cg += kProducers;
    };
    uint32_t ra[kLook][4], rb0[kLook][4], rb1[kLook][4];
#pragma unroll
    for (int d = 0; d < kLook; ++d) sf_load(ra[d], rb0[d], rb1[d]);
    int g = pid, cur_it = -1, ncols = 0;
    Item I{};
    // the next item's descriptor is read one item ahead (its loads are in flight meanwhile)
    Item In = cta_item<NT>(p.tiles, cid + (g / nk) * NC, MT2, kRowsPerCta, rank);
    bool more = true;
    while (more) {
#pragma unroll
      for (int d = 0; d < kLook; ++d) {
        const int it = g / nk, kt = g % nk;
        if (it != cur_it) {
          I = (cur_it < 0 || it == cur_it + 1) ? In : cta_item<NT>(p.tiles, cid + it * NC, MT2, kRowsPerCta, rank);
          cur_it = it;
          In = cta_item<NT>(p.tiles, cid + (it + 1) * NC, MT2, kRowsPerCta, rank);
          ncols = I.valid ? gemm::item_cols(I, NT) : 0;
        }
        if (!I.valid) {
          more = false;
          break;
        }
        const int j = g / kProducers;
        const int s = kProducers * (j % np) + pid, r = j / np;
        if (r > 0 && !tc::mbar_wait(&empty[s], (r - 1) & 1, p.err)) {
          more = false;
          break;
        }
        uint8_t* st = smem + s * kStage;
        store_sf(st + kOffSfa, ra[d], lane);
        store_sf(st + kOffSfb, rb0[d], lane);
        if (C::kSfbAtoms > 1) store_sf(st + kOffSfb + kSf, rb1[d], lane);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const uint32_t bar0 = tc::mapa_shared(tc::smem_u32(&full[s]), 0);
          const int bhalf = I.brow + rank * (ncols / 2);   // this CTA's first token row
          if (rank == 0) tc::mbar_arrive_expect_tx(&full[s], kTxPair);
          if (PAIR) {
            tc::tma_load_2d_pair(st + kOffA, &tmA, kt * kKT, I.arow, bar0);                // gate rows: lanes 0-63
            tc::tma_load_2d_pair(st + kOffA + kATile / 2, &tmA2, kt * kKT, I.arow, bar0);  // up rows: 64-127
          } else {
            tc::tma_load_2d_pair(st + kOffA, &tmA, kt * kKT, I.arow, bar0);
          }
          tc::tma_load_2d_pair(st + kOffB, &tmB, kt * kKT, bhalf, bar0);
          // rank 1's scale-factor stores are released to rank 0's MMA thread by this arrival
          if (rank != 0) tc::mbar_arrive_remote(bar0);
        }
        last_round[s] = r;
        sf_load(ra[d], rb0[d], rb1[d]);   // the step kLook ahead
        g += kProducers;
      }
    }
    // rank 0: every load of both CTAs has landed (they count on its barriers) before the
    // pair passes the final cluster barrier
    if (rank == 0)
      for (int q = 0; q < kStages; ++q)
        if (last_round[q] >= 0) tc::mbar_wait(&full[q], last_round[q] & 1, p.err);
  } else if (warp == 0) {
    // ---------------------------------------------------------------- MMA issue (rank 0)
    if (rank == 0 && lane == 0) {
      int g = 0;
      bool ok = true;
      Item In = cta_item<NT>(p.tiles, cid, MT2, kRowsPerCta, 0);
      for (int it = 0; ok; ++it) {
        const Item I = In;
        if (!I.valid) break;
        In = cta_item<NT>(p.tiles, cid + (it + 1) * NC, MT2, kRowsPerCta, 0);   // read one item ahead
        const int ncols = gemm::item_cols(I, NT);
        const int buf = it & 1;
        if (it >= 2 && !tc::mbar_wait(&tempty[buf], ((it >> 1) - 1) & 1, p.err)) ok = false;
        tc::fence_after_sync();
        const uint32_t acc_col = tmem + uint32_t(buf * kAccStride);
        for (int kt = 0; kt < nk && ok; ++kt, ++g) {
          const int j = g / kProducers, np = kStages / kProducers;
          const int s = kProducers * (j % np) + g % kProducers, r = j / np;
          if (!tc::mbar_wait_cluster(&full[s], r & 1, p.err)) {   // rank 1's arrival releases at cluster scope
            ok = false;
            break;
          }
          tc::fence_after_sync();
          uint8_t* st = smem + s * kStage;
          tc::cp_sf_32x128b_x4_pair(tmem + kColSfa, tc::smem_desc_sf(tc::smem_u32(st + kOffSfa)));
          tc::cp_sf_32x128b_x4_pair(tmem + kColSfb, tc::smem_desc_sf(tc::smem_u32(st + kOffSfb)));
          if (C::kSfbAtoms > 1)
            tc::cp_sf_32x128b_x4_pair(tmem + kColSfb + 4, tc::smem_desc_sf(tc::smem_u32(st + kOffSfb + kSf)));
          const uint64_t da = tc::smem_desc_sw128(tc::smem_u32(st + kOffA));
          const uint64_t db = tc::smem_desc_sw128(tc::smem_u32(st + kOffB));
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t idesc = tc::idesc_mxf8f6f4_m256(ncols, tc::kFmtE2M1, tc::kFmtE4M3, uint32_t(kb), uint32_t(kb));
            tc::mma_mxf8f6f4_pair(acc_col, da + 2 * kb, db + 2 * kb, idesc, (tmem + kColSfa) | (uint32_t(kb) << 30),
                                  (tmem + kColSfb) | (uint32_t(kb) << 30), (kt > 0 || kb > 0) ? 1u : 0u);
          }
          tc::commit_pair(&empty[s], 0x3);
        }
        // also after an aborted item, so neither epilogue waits for ever
        tc::commit_pair(&tfull[buf], 0x3);
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;  // TMEM lanes 32q .. 32q+31
    for (int it = 0;; ++it) {
      const Item I = cta_item<NT>(p.tiles, cid + it * NC, MT2, kRowsPerCta, rank);
      if (!I.valid) break;
      const int buf = it & 1;
      bool ok = tc::mbar_wait(&tfull[buf], (it >> 1) & 1, p.err);
      if constexpr (PAIR) ok = gemm::all_of_epilogue(ok);
      if (!ok) break;
      tc::fence_after_sync();
      gemm::epilogue_tile<NT, PAIR>(tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * kAccStride), I, p.out, ubuf, q,
                                     lane);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive_peer(tc::mapa_shared(tc::smem_u32(&tempty[buf]), 0));
    }
  }
  // both CTAs: every role is done (or gave up) before TMEM is freed and the CTAs exit
  tc::fence_before_sync();
  __syncwarp();
  tc::cluster_sync();
  if (warp == 0) {
    tc::fence_after_sync();
    tc::tmem_dealloc_pair(tmem, kCols);
  }
}

// Clusters that can be resident at once (one CTA per SM), per device and kernel.
template <int NT, bool PAIR>
int max_pairs() {
  static int cached[kStqMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kStqMaxDevices) return 0;
  if (cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = PairCfg<NT>::kSmem;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, w4a8_pair_gemm_kernel<NT, PAIR>, &cfg) != cudaSuccess || n <= 0) return 0;
  cached[dev] = n;
  return n;
}

template <int NT, bool PAIR>
stq_status launch_pair_gemm(const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b, const PairProblem& p,
                            cudaStream_t s) {
  static StqSmemOptIn optin;
  const stq_status st = optin.ensure(w4a8_pair_gemm_kernel<NT, PAIR>, PairCfg<NT>::kSmem);
  if (st != STQ_OK) return st;
  if (p.tiles.max_items <= 0) return STQ_OK;
  const int pairs = max_pairs<NT, PAIR>();
  if (pairs <= 0) return STQ_ERR_CUDA;
  const int n = p.tiles.max_items < pairs ? p.tiles.max_items : pairs;
  return stq_launch(w4a8_pair_gemm_kernel<NT, PAIR>, dim3(unsigned(2 * n)), dim3(kThreads), PairCfg<NT>::kSmem, s, a,
                    a2, b, p);
}

// N tile of the pair GEMMs: gate/up (SwiGLU + MXFP8 epilogue) and down (FP32 outputs).
constexpr int kNtGateUp = 128;
constexpr int kNtDown = 240;

}  // namespace

// Routed MXFP4 experts of the prefill regime on CTA pairs (activations already quantised
// into xq/xs in sorted pair order): N-tile plans, gate/up with SwiGLU and MXFP8 h, down
// into Y.
stq_status moe_mx_experts_pair(const MoeArgs& a, int slots, cudaStream_t s) {
  const int P = a.P;
  stq_status st = stq_tile_plan_launch(a.counts, a.E, kNtGateUp, a.ntiles, a.n_ntiles, s);
  if (st != STQ_OK) return st;
  CUtensorMap mg, mu, mx, md, mh;
  if (!tma::map_e2m1(&mg, a.wg, uint64_t(a.H), uint64_t(a.E) * a.I, 64) ||
      !tma::map_e2m1(&mu, a.wu, uint64_t(a.H), uint64_t(a.E) * a.I, 64) ||
      !tma::map_u8(&mx, a.xq, a.H, P, kNtGateUp / 2) ||
      !tma::map_e2m1(&md, a.wd, uint64_t(a.I), uint64_t(a.E) * a.H) || !tma::map_u8(&mh, a.hq, a.I, P, kNtDown / 2))
    return STQ_ERR_CUDA;
  PairProblem gp{};
  gp.tiles.R = a.I;
  gp.tiles.offsets = a.offsets;
  gp.tiles.ntiles = a.ntiles;
  gp.tiles.n_ntiles = a.n_ntiles;
  gp.tiles.max_items = (P / kNtGateUp + slots) * (a.I / 128);
  gp.K = a.H;
  gp.Ptot = P;
  gp.sa = a.gsc;
  gp.sa2 = a.usc;
  gp.sb = a.xs;
  gp.out = gemm::EpiOut{a.I, nullptr, a.hq, a.hs};
  gp.err = a.err;
  {
    StqTimed tm(STQ_K_GATE_UP_MX, s);
    st = launch_pair_gemm<kNtGateUp, true>(mg, mu, mx, gp, s);
  }
  if (st != STQ_OK) return st;
  // the down projection's tiles (planned again once the gate/up launch is done with the plan)
  if (kNtDown != kNtGateUp && (st = stq_tile_plan_launch(a.counts, a.E, kNtDown, a.ntiles, a.n_ntiles, s)) != STQ_OK)
    return st;
  PairProblem dp = gp;
  dp.tiles.R = a.H;
  dp.tiles.max_items = (P / kNtDown + slots) * (a.H / 256);
  dp.K = a.I;
  dp.sa = a.dsc;
  dp.sa2 = nullptr;
  dp.sb = a.hs;
  dp.out = gemm::EpiOut{a.H, a.Y, nullptr, nullptr};
  StqTimed tm(STQ_K_DOWN_MX, s);
  return launch_pair_gemm<kNtDown, false>(md, md, mh, dp, s);
}
