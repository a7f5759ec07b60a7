// W4A8 grouped GEMM of the prefill regime with the tokens on M: the same product as
// gemm_mx.cu (MXFP4 E2M1 weights x MXFP8 E4M3 activations, UE8M0 scales per 32 along K,
// FP32 accumulators in TMEM; "Hy4-preview-SF-WFP4AFP8", "Quant Diff"), with the operand
// roles swapped: A = 128 token rows of one expert, B = 256 weight rows.
//
// Why: one tcgen05.mma of K = 32 costs the issuing thread about the same whatever its N,
// and so do the scale-factor copies, the commit and the stage-barrier wait of each 128-k
// stage.  With the weights on M and tokens on N, a 4096-token prefill layer (128 routed
// tokens per expert on average) gets N <= 128 and the tensor pipe idles most of each stage.
// With the tokens on M every MMA is N = 256 wide (the weight rows are always there), twice
// the work per issued instruction; the price is the unused token rows of an expert's last
// 128-token tile, which the MMA computes and the epilogue drops.
//
// A work item is 128 tokens of one expert (an N tile of the tile plan) x 256 weight rows
// over all of K.  Gate/up (PAIR): the 256 rows are 128 gate features and the same 128 up
// features, so TMEM lane t (token) holds g in columns 0-127 and u in 128-255 and SwiGLU
// and the MXFP8 re-quantisation of h along the features need no exchange between threads.
// Down: 256 output features, FP32 rows of Y.
//   warps 0, 10  producers (alternate stages): TMA of the activation tile (E4M3, 128 x 128 B)
//                and of two 128-row weight tiles (E2M1, expanded to one 16-element group per
//                16 bytes), 128-byte swizzle; the UE8M0 scales, read 8 stages ahead into a
//                register ring, re-laid into the scale-factor atoms (one for the tokens, two
//                for the weight rows);
//   warp 1       TMEM; one thread issues three tcgen05.cp and four M = 128, N = 256
//                kind::mxf8f6f4.block_scale MMAs per stage;
//   warps 2-9    epilogue: two warps per TMEM lane quarter, each loads its half of the
//                columns into registers, hands the accumulator back, then computes and
//                stores (one accumulator of 256 columns: two would not leave room in the
//                512 TMEM columns for the scale factors).
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

constexpr int kKT = 128;                       // k per stage
constexpr int kMT = 128;                       // tokens per item (M)
constexpr int kSf = 512;                       // scale-factor atom: 128 rows x 4 k-blocks
constexpr int kStages = 4;                     // the two producers own alternate stages
constexpr int kSfCols = 12;                    // TMEM columns of one stage's scale factors
constexpr uint32_t kCols = 512;
constexpr int kEpiWarps = 8;
constexpr int kEpi0 = 2;
constexpr int kProducer2 = kEpi0 + kEpiWarps;  // 10
constexpr int kThreads = 32 * (kProducer2 + 1);

// Gate/up (PAIR): N = 256 weight rows (128 features of each matrix) and one 256-column
// accumulator (two would leave no TMEM columns for the scale factors).  Down: N = 192
// output features and two accumulators at columns 0 and 256, so the FP32 epilogue of one
// item overlaps the MMAs of the next; the stages' scale factors sit after the first.
template <bool PAIR>
struct TmCfg {
  static constexpr int kNW = PAIR ? 256 : 192;         // weight rows per item (N)
  static constexpr int kAccBufs = PAIR ? 1 : 2;
  static constexpr int kAccStride = 256;
  static constexpr int kColSf = kNW;                   // stage s: columns kColSf + 12 s ..
  static constexpr int kRowsPerItem = PAIR ? 128 : kNW;  // rows of one weight matrix per item
  static constexpr int kOffA = 0;                      // activations: 128 rows x 128 B
  static constexpr int kOffB = kOffA + kMT * kKT;      // weights: kNW rows x 128 B (expanded E2M1)
  static constexpr int kOffSfa = kOffB + kNW * kKT;    // token scales
  static constexpr int kOffSfb = kOffSfa + kSf;        // weight-row scales, rows 0-127 then 128..
  static constexpr int kStage = (kOffSfb + 2 * kSf + 1023) / 1024 * 1024;
  static constexpr int kSmem = kStages * kStage + 1024 /* barriers */ + 1024 /* alignment */;
  static constexpr uint32_t kTx = uint32_t(kMT * kKT) + uint32_t(kNW * kKT / 2);  // TMA bytes per stage
  static_assert(kSmem <= 227 * 1024, "shared memory");
  static_assert(kColSf + kStages * kSfCols <= (kAccBufs == 2 ? kAccStride : int(kCols)), "TMEM columns");
  static_assert(kAccBufs == 1 || kAccStride + kNW <= int(kCols), "TMEM columns");
};

struct TmProblem {
  gemm::Tiling tiles;           // tiles.R = weight rows per expert
  int K, Ptot;                  // reduction length, activation rows
  const uint8_t* sa;            // weight scales [E*R][K/32] (gate scales for the pair)
  const uint8_t* sa2;           // up-projection scales (pair)
  const uint8_t* sb;            // activation scales [Ptot][K/32]
  gemm::EpiOut out;             // out.R = tiles.R
  int32_t* err;
};

// Scales of one stage: the 128 token rows of the item, and its weight rows (pair: 128 gate
// rows, then the same 128 rows of the up projection; down: rows 0-127, then 128..kNW-1).
template <bool PAIR>
__device__ __forceinline__ void load_stage_sf(uint32_t (&ra)[4], uint32_t (&rb)[2][4], const TmProblem& p,
                                              const Item& J, int k32, int kt, int nk, int lane) {
  load_sf(ra, p.sb, J.brow, kMT, p.Ptot, k32, kt, nk, lane);
  load_sf(rb[0], p.sa, J.arow, 128, 0x7fffffff, k32, kt, nk, lane);
  if (PAIR) load_sf(rb[1], p.sa2, J.arow, 128, 0x7fffffff, k32, kt, nk, lane);
  else load_sf(rb[1], p.sa, J.arow + 128, TmCfg<PAIR>::kNW - 128, 0x7fffffff, k32, kt, nk, lane);
}

// SwiGLU and MXFP8 of 32 features of one token: g, u are the FP32 accumulators; the
// group's E4M3 codes go to dst (32 bytes, 16-byte aligned) and its UE8M0 exponent is
// returned.  Same arithmetic as the gate/up epilogue of gemm_mx.cu.
__device__ __forceinline__ uint32_t swiglu_mx8_group(const uint32_t (&g)[32], const uint32_t (&u)[32], uint8_t* dst) {
  float h[32];
  bool anybad = false;
  uint32_t amax_bits = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const float gv = __uint_as_float(g[j]);
    h[j] = gv / (1.0f + __expf(-gv)) * __uint_as_float(u[j]);  // silu(g) * u
    const bool bad = !isfinite(h[j]);
    anybad |= bad;
    amax_bits = max(amax_bits, bad ? 0u : (__float_as_uint(h[j]) & 0x7FFFFFFFu));
  }
  const int ex = anybad ? 255 : mx_scale_exponent(__uint_as_float(amax_bits), 0x600000u, 8);
  const float f = pow2_float(127 - ex);
  uint32_t w[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    uint32_t v = 0u;
#pragma unroll
    for (int b = 0; b < 4; ++b) v |= (anybad ? 0x7Fu : e4m3_code(h[4 * q + b], f)) << (8 * b);
    w[q] = v;
  }
  reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
  reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  return uint32_t(ex);
}

// Persistent: CTA b takes items b, b + gridDim.x, ...  The smem ring and its barrier phases
// run on across items.
// tmW2: the up projection (pair), or the down matrix with 64-row boxes (rows 128-191 of an item).
template <bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    w4a8_tm_gemm_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                        const __grid_constant__ CUtensorMap tmW2, TmProblem p) {
  using C = TmCfg<PAIR>;
  constexpr int kNW = C::kNW, kStage = C::kStage, kRowsPerItem = C::kRowsPerItem;
  constexpr int kOffA = C::kOffA, kOffB = C::kOffB, kOffSfa = C::kOffSfa, kOffSfb = C::kOffSfb;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStage);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;         // [kAccBufs]
  uint64_t* tempty = tfull + C::kAccBufs;    // [kAccBufs]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + C::kAccBufs);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MT = p.tiles.R / kRowsPerItem;
  const int G = gridDim.x;
  const int nk = p.K / kKT;
  const int k32 = p.K / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 2);   // expect_tx arrival + the scale copies' commit
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < C::kAccBufs; ++b) {
      tc::mbar_init(&tfull[b], 1);
      tc::mbar_init(&tempty[b], kEpiWarps);
    }
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&tmX);
    tc::prefetch_tensormap(&tmW);
    if (PAIR) tc::prefetch_tensormap(&tmW2);
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  stq_pdl_begin();   // barriers and TMEM are set up; from here on global memory is read

  if (warp == 0 || warp == kProducer2) {
    // ---------------------------------------------------------------- producers
    // Global k-step g = item * nk + kt belongs to producer g & 1; its j-th step (j = g >> 1)
    // uses stage 2 (j % 2) + pid in round j / 2, so no stage is shared between the two.
    constexpr int kPf = 8;
    constexpr int kPerProducer = kStages / 2;
    const int pid = warp == 0 ? 0 : 1;
    int last_round[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_round[s] = -1;
    // When nk is a multiple of the ring (2 kPf steps), the last steps of an item read the
    // next item's first scale factors into the ring, so an item boundary costs no wait.
    const bool cross = nk % (2 * kPf) == 0;
    bool ok = true;
    uint32_t ra[kPf][4], rb[kPf][2][4];
    for (int it = 0; ok; ++it) {
      const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRowsPerItem, kMT);
      if (!I.valid) break;
      Item In{};
      if (cross) In = gemm::get_item(p.tiles, blockIdx.x + (it + 1) * G, MT, kRowsPerItem, kMT);
      const int kt0 = ((pid - it * nk) % 2 + 2) % 2;  // first k-step of this item for this producer
      if (!cross || it == 0) {
#pragma unroll
        for (int d = 0; d < kPf; ++d) load_stage_sf<PAIR>(ra[d], rb[d], p, I, k32, kt0 + 2 * d, nk, lane);
      }
      for (int k0 = kt0; k0 < nk && ok; k0 += 2 * kPf) {
#pragma unroll
        for (int d = 0; d < kPf; ++d) {
          const int kt = k0 + 2 * d;
          if (kt >= nk) break;
          const int j = (it * nk + kt) >> 1;
          const int s = 2 * (j % kPerProducer) + pid, r = j / kPerProducer;
          if (r > 0 && !tc::mbar_wait(&empty[s], (r - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStage;
          store_sf(st + kOffSfa, ra[d], lane);
          store_sf(st + kOffSfb, rb[d][0], lane);
          store_sf(st + kOffSfb + kSf, rb[d][1], lane);
          tc::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const uint32_t sf = tmem + uint32_t(C::kColSf + kSfCols * s);
            tc::fence_after_sync();
            tc::cp_sf_32x128b_x4(sf, tc::smem_desc_sf(tc::smem_u32(st + kOffSfa)));
            tc::cp_sf_32x128b_x4(sf + 4, tc::smem_desc_sf(tc::smem_u32(st + kOffSfb)));
            tc::cp_sf_32x128b_x4(sf + 8, tc::smem_desc_sf(tc::smem_u32(st + kOffSfb + kSf)));
            tc::commit(&full[s]);
            tc::mbar_arrive_expect_tx(&full[s], C::kTx);
            tc::tma_load_2d(st + kOffA, &tmX, kt * kKT, I.brow, &full[s]);
            if (PAIR) {
              tc::tma_load_2d(st + kOffB, &tmW, kt * kKT, I.arow, &full[s]);                // gate rows
              tc::tma_load_2d(st + kOffB + 128 * kKT, &tmW2, kt * kKT, I.arow, &full[s]);   // up rows
            } else {
              tc::tma_load_2d(st + kOffB, &tmW, kt * kKT, I.arow, &full[s]);                // rows 0-127
              tc::tma_load_2d(st + kOffB + 128 * kKT, &tmW2, kt * kKT, I.arow + 128, &full[s]);  // 128-191
            }
          }
          last_round[s] = r;
          const int kn = kt + 2 * kPf;
          const Item& J = (cross && kn >= nk) ? In : I;  // In.valid is false past the last item
          const int kj = (cross && kn >= nk) ? kn - nk : kn;
          const int nkj = J.valid ? nk : 0;               // an invalid item reads zeros
          load_stage_sf<PAIR>(ra[d], rb[d], p, J, k32, kj, nkj, lane);
        }
      }
    }
    // every load this warp issued has landed before the CTA may exit
    for (int q = 0; q < kStages; ++q)
      if (last_round[q] >= 0) tc::mbar_wait(&full[q], last_round[q] & 1, p.err);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t kIdescBase = tc::idesc_mxf8f6f4_ab(kNW, tc::kFmtE4M3, tc::kFmtE2M1, 0u, 0u);
      int g = 0;  // global k-step
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRowsPerItem, kMT);
        if (!I.valid) break;
        // the epilogue warps have taken this buffer's previous accumulator into registers
        const int buf = it % C::kAccBufs, round = it / C::kAccBufs;
        if (round >= 1 && !tc::mbar_wait(&tempty[buf], (round - 1) & 1, p.err)) break;
        tc::fence_after_sync();
        const uint32_t acc_col = tmem + uint32_t(buf * C::kAccStride);
        for (int kt = 0; kt < nk; ++kt, ++g) {
          const int j = g >> 1;
          const int s = 2 * (j % (kStages / 2)) + (g & 1), r = j / (kStages / 2);
          if (!tc::mbar_wait(&full[s], r & 1, p.err)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          uint8_t* st = smem + s * kStage;
          const uint32_t sf = tmem + uint32_t(C::kColSf + kSfCols * s);
          const uint64_t da = tc::smem_desc_sw128(tc::smem_u32(st + kOffA));
          const uint64_t db = tc::smem_desc_sw128(tc::smem_u32(st + kOffB));
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            const uint32_t idesc = kIdescBase | (uint32_t(kb) << 4) | (uint32_t(kb) << 29);
            tc::mma_mxf8f6f4(acc_col, da + 2 * kb, db + 2 * kb, idesc, sf | (uint32_t(kb) << 30),
                             (sf + 4) | (uint32_t(kb) << 30), (kt > 0 || kb > 0) ? 1u : 0u);
          }
          tc::commit(&empty[s]);
        }
        tc::commit(&tfull[buf]);  // also after an aborted item, so the epilogue never waits for ever
      }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                  // TMEM lanes 32q .. 32q+31: tokens of the tile
    const int h = (warp - kEpi0) >> 2;       // which half of the columns
    for (int it = 0;; ++it) {
      const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRowsPerItem, kMT);
      if (!I.valid) break;
      const int buf = it % C::kAccBufs, round = it / C::kAccBufs;
      if (!tc::mbar_wait(&tfull[buf], round & 1, p.err)) break;
      tc::fence_after_sync();
      const uint32_t tl = tmem + (uint32_t(32 * q) << 16) + uint32_t(buf * C::kAccStride);
      const int row = 32 * q + lane;
      const bool valid = I.n0 + row < I.cnt;
      const size_t pos = size_t(I.brow + row);
      if constexpr (PAIR) {
        // features f0 .. f0+63 of this half: g in columns 64h.., u in 128 + 64h..
        uint32_t g0[32], g1[32], u0[32], u1[32];
        tc::tmem_ld_x32(tl + 64 * h, g0);
        tc::tmem_ld_x32(tl + 64 * h + 32, g1);
        tc::tmem_ld_x32(tl + 128 + 64 * h, u0);
        tc::tmem_ld_x32(tl + 128 + 64 * h + 32, u1);
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty[buf]);
        if (valid) {
          const int f0 = I.mt * 128 + 64 * h;
          uint8_t* dst = p.out.hq + pos * p.out.R + f0;
          const uint32_t e0 = swiglu_mx8_group(g0, u0, dst);
          const uint32_t e1 = swiglu_mx8_group(g1, u1, dst + 32);
          *reinterpret_cast<uint16_t*>(p.out.hs + pos * (p.out.R / 32) + (f0 >> 5)) = uint16_t(e0 | (e1 << 8));
        }
      } else {
        // output features f0 .. f0+95 of this half: columns 96h ..
        uint32_t v0[32], v1[32], v2[32];
        tc::tmem_ld_x32(tl + 96 * h, v0);
        tc::tmem_ld_x32(tl + 96 * h + 32, v1);
        tc::tmem_ld_x32(tl + 96 * h + 64, v2);
        tc::tmem_ld_wait();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty[buf]);
        if (valid) {
          uint4* y = reinterpret_cast<uint4*>(p.out.Y + pos * p.out.R + I.mt * kNW + 96 * h);
#pragma unroll
          for (int c = 0; c < 8; ++c) y[c] = make_uint4(v0[4 * c], v0[4 * c + 1], v0[4 * c + 2], v0[4 * c + 3]);
#pragma unroll
          for (int c = 0; c < 8; ++c) y[8 + c] = make_uint4(v1[4 * c], v1[4 * c + 1], v1[4 * c + 2], v1[4 * c + 3]);
#pragma unroll
          for (int c = 0; c < 8; ++c) y[16 + c] = make_uint4(v2[4 * c], v2[4 * c + 1], v2[4 * c + 2], v2[4 * c + 3]);
        }
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kCols);
  }
}

template <bool PAIR>
stq_status launch_tm(const CUtensorMap& x, const CUtensorMap& w, const CUtensorMap& w2, const TmProblem& p,
                     cudaStream_t s) {
  static StqSmemOptIn optin;
  const stq_status st = optin.ensure(w4a8_tm_gemm_kernel<PAIR>, TmCfg<PAIR>::kSmem);
  if (st != STQ_OK) return st;
  if (p.tiles.max_items <= 0) return STQ_OK;
  const unsigned grid = unsigned(stq_persistent_grid(p.tiles.max_items, 1));
  return stq_launch(w4a8_tm_gemm_kernel<PAIR>, dim3(grid), dim3(kThreads), TmCfg<PAIR>::kSmem, s, x, w, w2, p);
}

}  // namespace

// Routed experts of an MXFP4 layer in the prefill regime, tokens on M; the activations are
// already MXFP8 in sorted order (a.xq, a.xs).  The gate/up launch plans 128-token tiles; the
// down launch reuses that plan.
namespace {

bool tm_maps(const MoeArgs& a, CUtensorMap* mg, CUtensorMap* mu, CUtensorMap* mx, CUtensorMap* md, CUtensorMap* mh) {
  return tma::map_e2m1(mg, a.wg, uint64_t(a.H), uint64_t(a.E) * a.I) &&
         tma::map_e2m1(mu, a.wu, uint64_t(a.H), uint64_t(a.E) * a.I) && tma::map_u8(mx, a.xq, a.H, a.P, kMT) &&
         tma::map_e2m1(md, a.wd, uint64_t(a.I), uint64_t(a.E) * a.H) && tma::map_u8(mh, a.hq, a.I, a.P, kMT);
}

TmProblem tm_problem(const MoeArgs& a, int slots) {
  TmProblem gp{};
  gp.tiles.R = a.I;
  gp.tiles.offsets = a.offsets;
  gp.tiles.ntiles = a.ntiles;
  gp.tiles.n_ntiles = a.n_ntiles;
  gp.tiles.max_items = (a.P / kMT + slots) * (a.I / 128);
  gp.K = a.H;
  gp.Ptot = a.P;
  gp.sa = a.gsc;
  gp.sa2 = a.usc;
  gp.sb = a.xs;
  gp.out.R = a.I;
  gp.out.hq = a.hq;
  gp.out.hs = a.hs;
  gp.err = a.err;
  return gp;
}

}  // namespace

stq_status moe_mx_gate_up_tm(const MoeArgs& a, int slots, cudaStream_t s) {
  stq_status st = stq_tile_plan_launch(a.counts, a.E, kMT, a.ntiles, a.n_ntiles, s);
  if (st != STQ_OK) return st;
  CUtensorMap mg, mu, mx, md, mh;
  if (!tm_maps(a, &mg, &mu, &mx, &md, &mh)) return STQ_ERR_CUDA;
  StqTimed tm(STQ_K_GATE_UP_MX, s);
  return launch_tm<true>(mx, mg, mu, tm_problem(a, slots), s);
}

bool moe_mx_down_tm_fits(const MoeArgs& a) { return a.H % TmCfg<false>::kNW == 0; }

stq_status moe_mx_down_tm(const MoeArgs& a, int slots, cudaStream_t s) {
  if (!moe_mx_down_tm_fits(a)) return STQ_ERR_SHAPE;
  CUtensorMap mg, mu, mx, md, mh, md64;
  if (!tm_maps(a, &mg, &mu, &mx, &md, &mh) || !tma::map_e2m1(&md64, a.wd, uint64_t(a.I), uint64_t(a.E) * a.H, 64))
    return STQ_ERR_CUDA;
  TmProblem dp = tm_problem(a, slots);
  dp.tiles.R = a.H;
  dp.tiles.max_items = (a.P / kMT + slots) * (a.H / TmCfg<false>::kNW);
  dp.K = a.I;
  dp.sa = a.dsc;
  dp.sa2 = nullptr;
  dp.sb = a.hs;
  dp.out = gemm::EpiOut{a.H, a.Y, nullptr, nullptr};
  StqTimed tm(STQ_K_DOWN_MX, s);
  return launch_tm<false>(mh, md, md64, dp, s);
}
