// Prefill-regime grouped GEMM of STQ1_0 weights x MXFP8 activations on the sm_100a
// tensor cores.
//
// STQ1_0 ("Hy4-preview-GGUF", section 3; "Hy4-preview-FlashMoE-STQ1_0", "How the STQ1_0
// packing works"): w = d * t with t in {-1, 0, +1}, one zero per four weights, d FP16
// per 256 weights of a row.  The ternary t is exact in E4M3 (+-1 = 0x38 / 0xB8), so a
// 256-k block of weights is decoded in shared memory to E4M3 and multiplied with the
// MXFP8 activations by tcgen05.mma kind::mxf8f6f4 with a unit weight scale (UE8M0 127);
// the activations keep their UE8M0 scale per 32 k.  d, FP16 with 11 significant bits,
// fits neither operand format, so each block's product lands in its own TMEM partial
// buffer and is promoted in FP32: acc += d[row] * partial, with acc in registers.
//
// Tile: 128 weight rows (M; for gate/up the 64 gate rows of 64 features and the same
// up rows) x 112 tokens of one expert (N), over all of K, one 256-k block per stage.
// TMEM (512 columns): partial buffers at 0 and 128, finished accumulators at 256 and 384
// (112 columns each); the weights' unit scale atom at 112 and the three stages' activation
// scale factors at 116, 240 and 248 (columns the 112-wide partials leave free).
//
// Warp roles (576 threads, one CTA per SM, persistent over work items):
//   warp 0       TMA of the activation tile (two 128-k boxes, 128-byte swizzle) and its
//                scale factors (loaded four stages ahead into a register ring), re-laid
//                into the scale-factor atoms and copied into the stage's TMEM slot;
//   warp 1       TMEM allocation and, from one thread, the eight K = 32 MMAs of a stage
//                into the partial buffer of the block;
//   warps 2-9    promotion: two warps per TMEM lane quarter (weight row), each holding 56
//                of the tile's token columns in registers; per block one TMEM load of the
//                partial, which frees the buffer, and acc += d * partial; after the item's
//                last block one TMEM store of the accumulator into a finished-accumulator
//                buffer;
//   warps 14-17  epilogue of a finished accumulator (FP32 outputs, or SwiGLU and the
//                MXFP8 re-quantisation of h);
//   warps 10-13  decode: each warp turns two 16-row STQ1_0 tile-blocks into E4M3 rows of
//                the A tile (a shuffle of a 32-entry pattern table per 5-bit code gives
//                the four bytes of one group).
// Every hand-off is an mbarrier with a bounded wait (STQ_ERR_TIMEOUT, then exit).

#include "gemm_common.cuh"
#include "gemv.cuh"
#include "tma.cuh"

namespace {

using gemm::Item;

constexpr int kNT = 112;                 // tokens per N tile
constexpr int kSubA = 128 * 128;         // one 128-row x 128-k E4M3 sub-tile (128-byte swizzle)
constexpr int kSubB = kNT * 128;         // one 112-row x 128-k activation sub-tile
constexpr int kSf = 512;                 // scale-factor atom: 128 rows x 4 k-blocks of 32
constexpr int kOffA = 0;                 // two sub-tiles: k 0..127, 128..255 of the block
constexpr int kOffB = 2 * kSubA;
constexpr int kOffSfb = kOffB + 2 * kSubB;
constexpr int kStage = (kOffSfb + 2 * kSf + 1023) / 1024 * 1024;
constexpr int kStages = 3;
constexpr int kHalf = kNT / 2;           // token columns per promotion warp
constexpr int kUBuf = 4 * 32 * 9 * 4;    // gate/up exchange of the epilogue
constexpr int kSmem = kStages * kStage + kUBuf + kSf /* unit weight scales */ + 1024 /* barriers */ +
                      1024 /* alignment */;
constexpr uint32_t kTxB = 2 * kSubB;     // bytes the TMA delivers per stage
constexpr int kThreads = 576;
constexpr int kDecodeWarp0 = 10;
constexpr int kEpiWarp0 = 14;
constexpr int kDecodeWarps = 4;
constexpr int kColP = 0;                 // partial buffers: kColP + 128 * i
constexpr int kPBufs = 2;
constexpr int kColAcc = 256;             // finished accumulators on their way out: kColAcc + 128 * i
constexpr int kPromoWarps = 8;
constexpr int kColSfa = 112;
// Stage s's two activation scale-factor atoms (8 columns), in columns the partials leave free.
__host__ __device__ constexpr int col_sfb(int s) { return s == 0 ? 116 : s == 1 ? 240 : 248; }
constexpr uint32_t kCols = 512;
static_assert(kSubB % 1024 == 0 && kStage % 1024 == 0, "128-byte swizzle atoms");
static_assert(kSmem <= 227 * 1024, "shared memory");
static_assert(kStages == 3 && kNT <= 112, "scale-factor slots in the partial buffers' free columns");

struct StqGemm {
  gemm::Tiling tiles;          // tiles.R = weight rows per expert
  int K, Ptot;                 // reduction length, activation rows
  const uint8_t* w0;           // STQ1_0 matrices, expert-major (gate, or down)
  const uint8_t* w1;           // up projection (gate/up pair)
  const uint8_t* sb;           // activation scales [Ptot][K/32]
  gemm::EpiOut out;
  int32_t* err;
};

// Pattern table entry of code c: byte l = E4M3 of t at lane l of the group.
__device__ __forceinline__ uint32_t e4m3_lut_entry(uint32_t c) {
  const uint32_t z = (c >> 3) & 3u, s = c & 7u;
  uint32_t e = 0, n = 0;
#pragma unroll
  for (uint32_t l = 0; l < 4; ++l) {
    if (l != z) {
      e |= (((s >> n) & 1u) ? 0xB8u : 0x38u) << (8 * l);
      ++n;
    }
  }
  return e;
}

// A-tile row m (0..127) -> (matrix, row within the expert matrix).
template <bool PAIR>
__device__ __forceinline__ const uint8_t* row_matrix(const StqGemm& p, int m, int mt, int& row) {
  if constexpr (PAIR) {
    row = mt * 64 + (m & 63);
    return m < 64 ? p.w0 : p.w1;
  } else {
    row = mt * 128 + m;
    return p.w0;
  }
}

// Tile-block (16 rows x 256 k) of block kb holding A-tile rows 16j..16j+15 of item I.
template <bool PAIR>
__device__ __forceinline__ const uint8_t* tile_block(const StqGemm& p, const Item& I, int j, int kb) {
  int row;
  const uint8_t* w = row_matrix<PAIR>(p, 16 * j, I.mt, row);
  const int nb = p.K / 256;
  const size_t mat = size_t(p.tiles.R) * nb * 42;
  return w + size_t(I.e) * mat + size_t(row >> 4) * nb * stq::kTileBlockBytes + size_t(kb) * stq::kTileBlockBytes;
}

// FP16 d of A-tile row m in block kb (the d-pair word of row m % 8, half m / 8 % 2).
template <bool PAIR>
__device__ __forceinline__ const uint16_t* d_ptr(const StqGemm& p, const Item& I, int m, int kb) {
  int row;
  const uint8_t* w = row_matrix<PAIR>(p, m, I.mt, row);
  const int nb = p.K / 256;
  const size_t mat = size_t(p.tiles.R) * nb * 42;
  const uint8_t* tb = w + size_t(I.e) * mat + size_t(row >> 4) * nb * stq::kTileBlockBytes +
                      size_t(kb) * stq::kTileBlockBytes;
  return reinterpret_cast<const uint16_t*>(tb + 4 * (row & 7) + 2 * ((row >> 3) & 1));
}

struct TileWords {
  uint32_t w[5];
};

__device__ __forceinline__ void load_tile_words(TileWords& t, const uint8_t* tb, int lane) {
  const uint4 a = stq::ldg_stream16(tb + 32 + 16 * lane);
  t.w[0] = a.x;
  t.w[1] = a.y;
  t.w[2] = a.z;
  t.w[3] = a.w;
  t.w[4] = stq::ldg_stream4(tb + 544 + 4 * lane);
}

// Groups 4c4..4c4+3 of this lane's row g + 8h as one 16-byte chunk.
template <int H, int C4>
__device__ __forceinline__ uint4 decode_chunk(const TileWords& t, uint32_t lut) {
  uint4 r;
  r.x = __shfl_sync(stq::kFull, lut, stq::code_at<2 * (4 * C4 + 0) + H>(t.w));
  r.y = __shfl_sync(stq::kFull, lut, stq::code_at<2 * (4 * C4 + 1) + H>(t.w));
  r.z = __shfl_sync(stq::kFull, lut, stq::code_at<2 * (4 * C4 + 2) + H>(t.w));
  r.w = __shfl_sync(stq::kFull, lut, stq::code_at<2 * (4 * C4 + 3) + H>(t.w));
  return r;
}

// Write the tile-block of A-tile rows 16j.. into the stage's A sub-tiles.  Lane (g, t)
// holds rows 16j + g and 16j + g + 8, k = 64t .. 64t + 63 of the block: sub-tile t / 2,
// 16-byte chunks 4 (t % 2) + c of the 128-byte row, stored at chunk (chunk ^ row % 8).
// Lanes t and t + 2 would hit the same banks (the sub-tiles are 16 KB apart), so lanes
// t >= 2 rotate their 160-bit code stream by 80 bits: their c-th store then holds chunk
// c ^ 2, and the eight lanes of each store phase cover eight distinct 16-byte bank groups.
template <int H, int C4>
__device__ __forceinline__ void put_chunk(uint8_t* row_base, const TileWords& t, uint32_t lut, int cbase, int sw,
                                          int g) {
  const int chunk = cbase + (C4 ^ sw);
  *reinterpret_cast<uint4*>(row_base + H * 1024 + ((chunk ^ g) << 4)) = decode_chunk<H, C4>(t, lut);
}

__device__ __forceinline__ void put_tile_block(uint8_t* a_stage, const TileWords& in, uint32_t lut, int j, int lane) {
  const int g = lane >> 2, tq = lane & 3;
  const bool up = tq >= 2;
  TileWords t;
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    // bits [32k + 80, 32k + 112) mod 160 of the stream
    const uint32_t rot = __funnelshift_r(in.w[(k + 2) % 5], in.w[(k + 3) % 5], 16);
    t.w[k] = up ? rot : in.w[k];
  }
  const int sw = up ? 2 : 0;
  const int cbase = 4 * (tq & 1);
  // rows 16j + g (H = 0) and 16j + g + 8 (H = 1: one 1024-byte 8-row group further)
  uint8_t* row_base = a_stage + (up ? kSubA : 0) + (2 * j) * 1024 + g * 128;
  put_chunk<0, 0>(row_base, t, lut, cbase, sw, g);
  put_chunk<0, 1>(row_base, t, lut, cbase, sw, g);
  put_chunk<0, 2>(row_base, t, lut, cbase, sw, g);
  put_chunk<0, 3>(row_base, t, lut, cbase, sw, g);
  put_chunk<1, 0>(row_base, t, lut, cbase, sw, g);
  put_chunk<1, 1>(row_base, t, lut, cbase, sw, g);
  put_chunk<1, 2>(row_base, t, lut, cbase, sw, g);
  put_chunk<1, 3>(row_base, t, lut, cbase, sw, g);
}

}  // namespace

namespace {

// Persistent over work items b, b + gridDim.x, ...; all roles walk the same item list,
// and a per-CTA block counter g (items x K blocks) drives every ring: stage g % 3, partial
// buffer g % 2; finished-accumulator buffer item % 2.
template <bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    stq_gemm_kernel(const __grid_constant__ CUtensorMap tmB, StqGemm p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* ubuf = reinterpret_cast<float*>(smem + kStages * kStage);
  uint8_t* sfa_unit = smem + kStages * kStage + kUBuf;
  uint64_t* full = reinterpret_cast<uint64_t*>(sfa_unit + kSf);  // [kStages]: TMA bytes + 3 arrivals
  uint64_t* empty = full + kStages;                              // [kStages]: MMAs of the stage done
  uint64_t* pfull = empty + kStages;                             // [kPBufs]: partial written
  uint64_t* pempty = pfull + kPBufs;                             // [kPBufs]: partial read (8 warps)
  uint64_t* afull = pempty + kPBufs;                             // [2]: accumulator staged (8 warps)
  uint64_t* aempty = afull + 2;                                  // [2]: accumulator drained (4 warps)
  uint64_t* mdone = aempty + 2;                                  // every MMA of this CTA completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(mdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kRows = PAIR ? 64 : 128;  // output features per item
  const int MT = p.tiles.R / kRows;
  const int G = gridDim.x;
  const int nb = p.K / 256;

  // unit weight scales (UE8M0 127 = 2^0) for every row and k-block
  for (int i = threadIdx.x; i < kSf / 4; i += kThreads) reinterpret_cast<uint32_t*>(sfa_unit)[i] = 0x7F7F7F7Fu;
  tc::fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      tc::mbar_init(&full[s], 2 + kDecodeWarps);   // TMA bytes, the scale copies, the decoders
      tc::mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < kPBufs; ++b) {
      tc::mbar_init(&pfull[b], 1);
      tc::mbar_init(&pempty[b], kPromoWarps);
    }
    for (int b = 0; b < 2; ++b) {
      tc::mbar_init(&afull[b], kPromoWarps);
      tc::mbar_init(&aempty[b], 4);
    }
    tc::mbar_init(mdone, 1);
    tc::fence_barrier_init();
    tc::prefetch_tensormap(&tmB);
  }
  if (warp == 1) tc::tmem_alloc(tmem_holder, kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_holder;
  stq_pdl_begin();   // barriers and TMEM are set up; from here on global memory is read

  if (warp == 0) {
    // ---------------------------------------------------------------- activation loads
    // The scale factors of a stage are global loads that the warp must re-lay before the
    // stage can start; a register ring holds them kLook stages ahead (a second cursor
    // walks the same item/block sequence), so their latency overlaps earlier stages.
    constexpr int kLook = 4;
    const int k32 = p.K / 32, nk = p.K / 128;
    int last_round[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_round[s] = -1;
    Item J = gemm::get_item(p.tiles, blockIdx.x, MT, kRows, kNT);
    int itJ = 0, kbJ = 0;
    uint32_t ring[kLook][2][4];
    auto load_next = [&](uint32_t (&v)[2][4]) {
      const int nkj = J.valid ? nk : 0;  // past the last item: zeros, no loads
      gemm::load_sf(v[0], p.sb, J.brow, kNT, p.Ptot, k32, 2 * kbJ, nkj, lane);
      gemm::load_sf(v[1], p.sb, J.brow, kNT, p.Ptot, k32, 2 * kbJ + 1, nkj, lane);
      if (J.valid && ++kbJ == nb) {
        kbJ = 0;
        ++itJ;
        J = gemm::get_item(p.tiles, blockIdx.x + itJ * G, MT, kRows, kNT);
      }
    };
#pragma unroll
    for (int d = 0; d < kLook; ++d) load_next(ring[d]);
    Item I = gemm::get_item(p.tiles, blockIdx.x, MT, kRows, kNT);
    int it = 0, kb = 0, g = 0;
    bool ok = true;
    while (ok && I.valid) {
#pragma unroll
      for (int d = 0; d < kLook; ++d) {
        if (!ok || !I.valid) break;
        const int s = g % kStages, r = g / kStages;
        if (r > 0 && !tc::mbar_wait(&empty[s], (r - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * kStage;
        gemm::store_sf(st + kOffSfb, ring[d][0], lane);
        gemm::store_sf(st + kOffSfb + kSf, ring[d][1], lane);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          // the scale factors go to this stage's TMEM slot from here, so the MMA thread only
          // issues MMAs (the MMAs of the slot's previous round are done: empty[s] above)
          tc::fence_after_sync();
          tc::cp_sf_32x128b_x4(tmem + uint32_t(col_sfb(s)), tc::smem_desc_sf(tc::smem_u32(st + kOffSfb)));
          tc::cp_sf_32x128b_x4(tmem + uint32_t(col_sfb(s) + 4), tc::smem_desc_sf(tc::smem_u32(st + kOffSfb + kSf)));
          tc::commit(&full[s]);
          tc::mbar_arrive_expect_tx(&full[s], kTxB);
          tc::tma_load_2d(st + kOffB, &tmB, kb * 256, I.brow, &full[s]);
          tc::tma_load_2d(st + kOffB + kSubB, &tmB, kb * 256 + 128, I.brow, &full[s]);
        }
        last_round[s] = r;
        load_next(ring[d]);  // the stage kLook steps ahead
        ++g;
        if (++kb == nb) {
          kb = 0;
          ++it;
          I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRows, kNT);
        }
      }
    }
    // every load this warp issued has landed before the CTA may exit
    for (int q = 0; q < kStages; ++q)
      if (last_round[q] >= 0) tc::mbar_wait(&full[q], last_round[q] & 1, p.err);
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      tc::cp_sf_32x128b_x4(tmem + kColSfa, tc::smem_desc_sf(tc::smem_u32(sfa_unit)));
      int g = 0;
      bool ok = true;
      for (int it = 0; ok; ++it) {
        const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRows, kNT);
        if (!I.valid) break;
        const uint32_t idesc_n = uint32_t(gemm::item_cols(I, kNT));
        for (int kb = 0; kb < nb; ++kb, ++g) {
          const int s = g % kStages, r = g / kStages, pb = g % kPBufs, pr = g / kPBufs;
          if (pr > 0 && !tc::mbar_wait(&pempty[pb], (pr - 1) & 1, p.err)) {
            ok = false;
            break;
          }
          if (!tc::mbar_wait(&full[s], r & 1, p.err)) {
            ok = false;
            break;
          }
          tc::fence_after_sync();
          uint8_t* st = smem + s * kStage;
          const uint32_t sfb = tmem + uint32_t(col_sfb(s));
          const uint32_t d_col = tmem + uint32_t(kColP + 128 * pb);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const int h = kk >> 2, j = kk & 3;
            const uint64_t da = tc::smem_desc_sw128(tc::smem_u32(st + kOffA + h * kSubA)) + 2 * j;
            const uint64_t db = tc::smem_desc_sw128(tc::smem_u32(st + kOffB + h * kSubB)) + 2 * j;
            const uint32_t idesc = tc::idesc_mxf8f6f4_ab(int(idesc_n), tc::kFmtE4M3, tc::kFmtE4M3, 0u, uint32_t(j));
            tc::mma_mxf8f6f4(d_col, da, db, idesc, tmem + kColSfa, (sfb + uint32_t(4 * h)) | (uint32_t(j) << 30),
                             kk > 0 ? 1u : 0u);
          }
          tc::commit(&empty[s]);
          tc::commit(&pfull[pb]);
        }
      }
      tc::commit(mdone);
      tc::mbar_wait(mdone, 0, p.err);
    }
    __syncwarp();
  } else if (warp <= 9) {
    // ---------------------------------------------------------------- promotion
    // Warp w: TMEM lane quarter q = w % 4 (A-tile rows 32q..32q+31), token columns
    // 56c..56c+55 of the tile (c = 0 for warps 2-5, 1 for 6-9), accumulated in registers.
    const int q = warp & 3, c = (warp - 2) >> 2;
    const int m = 32 * q + lane;  // A-tile row = TMEM lane
    const uint32_t lane_base = tmem + (uint32_t(32 * q) << 16) + uint32_t(kHalf * c);
    int g = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRows, kNT);
      if (!I.valid) break;
      float acc[kHalf];
#pragma unroll
      for (int j = 0; j < kHalf; ++j) acc[j] = 0.f;
      const uint16_t* dp = d_ptr<PAIR>(p, I, m, 0);
      uint16_t dnext = __ldg(dp);
      for (int kb = 0; kb < nb; ++kb, ++g) {
        const int pb = g % kPBufs, pr = g / kPBufs;
        const float d = __half2float(__ushort_as_half(dnext));
        if (kb + 1 < nb) dnext = __ldg(dp + (kb + 1) * (stq::kTileBlockBytes / 2));
        if (!tc::mbar_wait(&pfull[pb], pr & 1, p.err)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        const uint32_t tp = lane_base + uint32_t(kColP + 128 * pb);
        // 16 columns per TMEM round trip: 18 warps leave 96 registers per thread (five warps
        // share a sub-partition's 16K registers), and the accumulator takes 56 of them
#pragma unroll
        for (int c0 = 0; c0 < 48; c0 += 16) {
          uint32_t v[16];
          tc::tmem_ld_x16(tp + c0, v);
          tc::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[c0 + j] = fmaf(d, __uint_as_float(v[j]), acc[c0 + j]);
        }
        {
          uint32_t x[8];
          tc::tmem_ld_x8(tp + 48, x);
          tc::tmem_ld_wait();
          // the partial is in registers: hand the buffer back to the MMA warp
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&pempty[pb]);
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[48 + j] = fmaf(d, __uint_as_float(x[j]), acc[48 + j]);
        }
      }
      if (!ok) break;
      // hand the finished accumulator to the epilogue warps through TMEM buffer it % 2
      const int abuf = it & 1, ar = it >> 1;
      if (ar > 0 && !tc::mbar_wait(&aempty[abuf], (ar - 1) & 1, p.err)) break;
      tc::fence_after_sync();
      const uint32_t stg = lane_base + uint32_t(kColAcc + 128 * abuf);
#pragma unroll
      for (int c0 = 0; c0 < 48; c0 += 16) {
        uint32_t a16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) a16[j] = __float_as_uint(acc[c0 + j]);
        tc::tmem_st_x16(stg + c0, a16);
      }
      {
        uint32_t a8[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) a8[j] = __float_as_uint(acc[48 + j]);
        tc::tmem_st_x8(stg + 48, a8);
      }
      tc::tmem_st_wait();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&afull[abuf]);
    }
  } else if (warp >= kEpiWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;
    for (int it = 0;; ++it) {
      const Item I = gemm::get_item(p.tiles, blockIdx.x + it * G, MT, kRows, kNT);
      if (!I.valid) break;
      const int abuf = it & 1, ar = it >> 1;
      bool ok = tc::mbar_wait(&afull[abuf], ar & 1, p.err);
      // the four epilogue warps meet at named barriers, so they agree on ok first
      if constexpr (PAIR) ok = gemm::all_of_epilogue(ok);
      if (!ok) break;
      tc::fence_after_sync();
      gemm::epilogue_tile<kNT, PAIR>(tmem + (uint32_t(32 * q) << 16) + uint32_t(kColAcc + 128 * abuf), I, p.out,
                                     ubuf, q, lane);
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aempty[abuf]);
    }
  } else {
    // ---------------------------------------------------------------- decode
    constexpr int kTb = 8 / kDecodeWarps;  // tile-blocks per decoder warp
    const int j0 = (warp - kDecodeWarp0) * kTb;
    const uint32_t lut = e4m3_lut_entry(uint32_t(lane));
    Item I = gemm::get_item(p.tiles, blockIdx.x, MT, kRows, kNT);
    TileWords cur[kTb] = {}, nxt[kTb] = {};
    if (I.valid) {
#pragma unroll
      for (int i = 0; i < kTb; ++i) load_tile_words(cur[i], tile_block<PAIR>(p, I, j0 + i, 0), lane);
    }
    int g = 0;
    bool ok = true;
    for (int it = 0; ok && I.valid; ++it) {
      const Item In = gemm::get_item(p.tiles, blockIdx.x + (it + 1) * G, MT, kRows, kNT);
      for (int kb = 0; kb < nb; ++kb, ++g) {
        const int s = g % kStages, r = g / kStages;
        if (kb + 1 < nb) {
#pragma unroll
          for (int i = 0; i < kTb; ++i) load_tile_words(nxt[i], tile_block<PAIR>(p, I, j0 + i, kb + 1), lane);
        } else if (In.valid) {
#pragma unroll
          for (int i = 0; i < kTb; ++i) load_tile_words(nxt[i], tile_block<PAIR>(p, In, j0 + i, 0), lane);
        }
        if (r > 0 && !tc::mbar_wait(&empty[s], (r - 1) & 1, p.err)) {
          ok = false;
          break;
        }
        uint8_t* a_stage = smem + s * kStage + kOffA;
#pragma unroll
        for (int i = 0; i < kTb; ++i) put_tile_block(a_stage, cur[i], lut, j0 + i, lane);
        tc::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&full[s]);
#pragma unroll
        for (int i = 0; i < kTb; ++i) cur[i] = nxt[i];
      }
      I = In;
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
stq_status launch_stq_gemm(const CUtensorMap& b, const StqGemm& p, cudaStream_t s) {
  static StqSmemOptIn optin;
  const stq_status st = optin.ensure(stq_gemm_kernel<PAIR>, kSmem);
  if (st != STQ_OK) return st;
  if (p.tiles.max_items <= 0) return STQ_OK;
  return stq_launch(stq_gemm_kernel<PAIR>, dim3(unsigned(stq_persistent_grid(p.tiles.max_items, 1))), dim3(kThreads),
                    kSmem, s, b, p);
}

}  // namespace

stq_status moe_stq_prefill_experts(const MoeArgs& a, int slots, cudaStream_t s) {
  const int P = a.P;
  // 1. activations -> MXFP8 g32 in sorted (expert-grouped) order
  stq_status st = stq_mxfp8_quantize_scatter_launch(a.x, a.T, a.H, a.inv, a.k, P, a.err, a.xq, a.xs, s);
  if (st != STQ_OK) return st;
  // 2. N tiles of 112 tokens of the touched experts
  if ((st = stq_tile_plan_launch(a.counts, a.E, kNT, a.ntiles, a.n_ntiles, s)) != STQ_OK) return st;
  const int max_tiles = P / kNT + slots;  // sum over experts of ceil(count / 112)
  CUtensorMap mx, mh;
  if (!tma::map_u8(&mx, a.xq, uint64_t(a.H), uint64_t(P), kNT) || !tma::map_u8(&mh, a.hq, uint64_t(a.I), uint64_t(P), kNT))
    return STQ_ERR_CUDA;
  // 3. gate/up pair, SwiGLU, MXFP8 h
  StqGemm gp{};
  gp.tiles.R = a.I;
  gp.tiles.offsets = a.offsets;
  gp.tiles.ntiles = a.ntiles;
  gp.tiles.n_ntiles = a.n_ntiles;
  gp.tiles.max_items = max_tiles * (a.I / 64);
  gp.K = a.H;
  gp.Ptot = P;
  gp.w0 = a.wg;
  gp.w1 = a.wu;
  gp.sb = a.xs;
  gp.out = gemm::EpiOut{a.I, nullptr, a.hq, a.hs};
  gp.err = a.err;
  {
    StqTimed tm(STQ_K_GATE_UP_STQ_TC, s);
    st = launch_stq_gemm<true>(mx, gp, s);
  }
  if (st != STQ_OK) return st;
  // 4. down, FP32 expert outputs
  StqGemm dp = gp;
  dp.tiles.R = a.H;
  dp.tiles.max_items = max_tiles * (a.H / 128);
  dp.K = a.I;
  dp.w0 = dp.w1 = a.wd;
  dp.sb = a.hs;
  dp.out = gemm::EpiOut{a.H, a.Y, nullptr, nullptr};
  StqTimed tm(STQ_K_DOWN_STQ_TC, s);
  return launch_stq_gemm<false>(mh, dp, s);
}
