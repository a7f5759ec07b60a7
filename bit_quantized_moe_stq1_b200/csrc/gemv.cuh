// Warp-level building blocks of the decode-regime grouped GEMV (sm_100a).
//
// One warp computes D[16*NT rows, 8 tokens] with mma.sync m16n8k16 (bf16 in,
// FP32 accumulate): weights on M, the expert's tokens on N.
//
// STQ1_0 operand ("Hy4-preview-GGUF", section 3; "Hy4-preview-FlashMoE-STQ1_0",
// "How the STQ1_0 packing works"): each 5-bit pattern is decoded in registers.
// Lane c of the warp holds the 4-byte pattern table entry of code c (byte l =
// high byte of the bf16 value of lane l: 0x00 for 0, 0x40 for +2, 0xC0 for -2),
// so a decode is: funnel-shift the code to the bottom of a register (the shuffle
// only reads bits 4..0), shuffle the table entry from lane `code`, and two byte
// permutes that place the bytes into the two bf16x2 A-fragment registers.  The
// +-2 weights are exact in bf16; d/2 (FP16 -> FP32, exact) scales each 256-block
// partial sum in FP32.
//
// K order inside one mma: thread t of a quad holds k = 64t + 4s + {0,1} in its
// first A/B register and k = 64t + 4s + {2,3} in its second (step s of the
// block), for A and B alike, so every product pairs the right weight and
// activation and thread t reads one contiguous 128-byte activation slice per
// block.
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"

namespace stq {

constexpr int kTileBlockBytes = 672;  // 16 rows x 256 k of STQ1_0 (16 x 42 bytes)
constexpr unsigned kFull = 0xffffffffu;

// Pattern table entry of code c (see above); computed once per lane.
__device__ __forceinline__ uint32_t lut_entry(uint32_t c) {
  const uint32_t z = (c >> 3) & 3u, s = c & 7u;
  uint32_t e = 0, n = 0;
#pragma unroll
  for (uint32_t l = 0; l < 4; ++l) {
    if (l != z) {
      e |= (((s >> n) & 1u) ? 0xC0u : 0x40u) << (8 * l);
      ++n;
    }
  }
  return e;
}

// Code i (compile-time after unrolling) of a lane's 160-bit stream, with the code
// in bits 4..0 and junk above (ignored by the shuffle).
template <int I>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[5]) {
  constexpr int sh = 5 * I, w0 = sh >> 5, off = sh & 31;
  if constexpr (off > 27) {
    return __funnelshift_r(w[w0], w[w0 + 1], off);
  } else if constexpr (off == 0) {
    return w[w0];
  } else {
    return w[w0] >> off;
  }
}

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint32_t ldg_stream4(const void* p) {
  uint32_t r;
  asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
  return r;
}

template <int NT>
struct StqBlockRegs {
  uint32_t w[NT][5];
  uint32_t d[NT];
};

// Load one 256-k block of NT tiles.  tb[i] points at tile-block 0 of tile i.
template <int NT>
__device__ __forceinline__ void stq_load(StqBlockRegs<NT>& r, const uint8_t* const (&tb)[NT], int b, int lane) {
  const int g = lane >> 2;
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const uint8_t* p = tb[i] + size_t(b) * kTileBlockBytes;
    const uint4 a = ldg_stream16(p + 32 + 16 * lane);
    r.w[i][0] = a.x;
    r.w[i][1] = a.y;
    r.w[i][2] = a.z;
    r.w[i][3] = a.w;
    r.w[i][4] = ldg_stream4(p + 544 + 4 * lane);
    r.d[i] = ldg_stream4(p + 4 * g);
  }
}

template <int I, int NT>
__device__ __forceinline__ void stq_step(const StqBlockRegs<NT>& r, uint32_t lut, uint32_t b0, uint32_t b1,
                                         float (&part)[NT][4]) {
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const uint32_t e0 = __shfl_sync(kFull, lut, code_at<2 * I>(r.w[i]));
    const uint32_t e1 = __shfl_sync(kFull, lut, code_at<2 * I + 1>(r.w[i]));
    mma_bf16_16816(part[i], prmt(e0, 0u, 0x1404u), prmt(e1, 0u, 0x1404u), prmt(e0, 0u, 0x3424u),
                   prmt(e1, 0u, 0x3424u), b0, b1);
  }
}

template <int I, int NT>
struct StqSteps {
  __device__ __forceinline__ static void run(const StqBlockRegs<NT>& r, const uint4 (&xv)[8], uint32_t lut,
                                             float (&part)[NT][4]) {
    const uint4 q = xv[I >> 1];
    if constexpr (I & 1)
      stq_step<I, NT>(r, lut, q.z, q.w, part);
    else
      stq_step<I, NT>(r, lut, q.x, q.y, part);
    StqSteps<I + 1, NT>::run(r, xv, lut, part);
  }
};
template <int NT>
struct StqSteps<16, NT> {
  __device__ __forceinline__ static void run(const StqBlockRegs<NT>&, const uint4 (&)[8], uint32_t, float (&)[NT][4]) {}
};

// acc[i][*] += (d/2) * sum over one 256-k block, for NT tiles.
template <int NT>
__device__ __forceinline__ void stq_block(const StqBlockRegs<NT>& r, const uint4 (&xv)[8], uint32_t lut,
                                          float (&acc)[NT][4]) {
  float part[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) part[i][0] = part[i][1] = part[i][2] = part[i][3] = 0.f;
  StqSteps<0, NT>::run(r, xv, lut, part);
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const float dg = __half2float(__ushort_as_half((unsigned short)(r.d[i] & 0xFFFFu))) * 0.5f;
    const float dg8 = __half2float(__ushort_as_half((unsigned short)(r.d[i] >> 16))) * 0.5f;
    acc[i][0] = fmaf(dg, part[i][0], acc[i][0]);
    acc[i][1] = fmaf(dg, part[i][1], acc[i][1]);
    acc[i][2] = fmaf(dg8, part[i][2], acc[i][2]);
    acc[i][3] = fmaf(dg8, part[i][3], acc[i][3]);
  }
}

__device__ __forceinline__ void load_x_block(uint4 (&xv)[8], const uint16_t* xrow, int b, int t) {
  if (xrow != nullptr) {
    const uint4* p = reinterpret_cast<const uint4*>(xrow + 256 * b + 64 * t);
#pragma unroll
    for (int q = 0; q < 8; ++q) xv[q] = p[q];
  } else {
#pragma unroll
    for (int q = 0; q < 8; ++q) xv[q] = make_uint4(0u, 0u, 0u, 0u);
  }
}

// Whole-warp STQ1_0 GEMV over blocks [b0, b1) of NT tiles, token column g of this
// lane's quad taken from xrow (nullptr = padding column).  Weight loads for block
// b+1 are in flight while block b is multiplied; with L2_AHEAD the tile-blocks of block
// b+2 are also prefetched into L2 (six lanes, one 128-byte line each).
template <int NT, bool L2_AHEAD = false>
__device__ __forceinline__ void stq_warp_gemv(const uint8_t* const (&tb)[NT], int b0, int b1, const uint16_t* xrow,
                                              uint32_t lut, float (&acc)[NT][4]) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  if (b0 >= b1) return;
  StqBlockRegs<NT> cur, nxt;
  stq_load<NT>(cur, tb, b0, lane);
  for (int b = b0; b < b1; ++b) {
    if (L2_AHEAD && b + 2 < b1 && lane < 6) {
#pragma unroll
      for (int i = 0; i < NT; ++i)
        asm volatile("prefetch.global.L2 [%0];" ::"l"(tb[i] + size_t(b + 2) * kTileBlockBytes + 128 * lane));
    }
    if (b + 1 < b1) stq_load<NT>(nxt, tb, b + 1, lane);
    uint4 xv[8];
    load_x_block(xv, xrow, b, t);
    stq_block<NT>(cur, xv, lut, acc);
    cur = nxt;
  }
}

// ----------------------------------------------------------------------------- integer variant
//
// The same decode into int8 weights (+1 = 0x01, -1 = 0xFF, 0 = 0x00): the shuffled table
// entry is then a finished A-fragment register of mma.sync m16n8k32 s8 (four consecutive k
// of one row), so a 5-bit code costs one shift and one shuffle and no byte permutes.  The
// activations enter as three signed 8-bit limbs of a fixed-point value per 256-k block
// (written by stq_act_limbs_kernel, x's by the grouping's launch when it can take them):
// v = q * 2^(Eb - 148), q = hi*2^16 + mid*2^8 + lo, with
// Eb the largest bf16 exponent field of the block.  Every element within 2^14 of the
// block's largest magnitude is exact; smaller ones are rounded to the nearest multiple of
// 2^(Eb - 148), an absolute error of at most 2^-22 of the block's largest magnitude.  The
// s32 sums of one block are exact (|sum| <= 256 * 128).
//
// The eight B columns are (token, limb) pairs: column c = 3j + l is limb l of the item's
// token j (j = 0, 1; columns 6 and 7 are zero), so one mma serves two tokens.  K order:
// in mma m of a block, thread t's a0/a1 (rows g, g+8) hold the codes of k = 64t + 8m + 0..3
// (stream codes 4m, 4m+1) and a2/a3 those of k = 64t + 8m + 4..7 (codes 4m+2, 4m+3); its
// b0/b1 hold the activations of the same k: in the limb rows' block layout (k = 64t + 16q + i
// at byte 16*(4q + t) + i) the 16-byte chunk 4*(m/2) + t, bytes 8*(m%2) .. 8*(m%2) + 7.

// Table entry of code c for the integer decode.
__device__ __forceinline__ uint32_t lut_entry_i8(uint32_t c) {
  const uint32_t z = (c >> 3) & 3u, s = c & 7u;
  uint32_t e = 0, n = 0;
#pragma unroll
  for (uint32_t l = 0; l < 4; ++l) {
    if (l != z) {
      e |= (((s >> n) & 1u) ? 0xFFu : 0x01u) << (8 * l);
      ++n;
    }
  }
  return e;
}

// D = A * B + D for one m16n8k32 s8 tile with s32 accumulators.
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int M, int NT>
struct StqStepsI8 {
  __device__ __forceinline__ static void run(const StqBlockRegs<NT>& r, const uint4 (&xv)[4], uint32_t lut,
                                             int (&part)[NT][4]) {
    const uint4 q = xv[M >> 1];
    const uint32_t b0 = (M & 1) ? q.z : q.x, b1 = (M & 1) ? q.w : q.y;
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      const uint32_t a0 = __shfl_sync(kFull, lut, code_at<4 * M>(r.w[i]));
      const uint32_t a1 = __shfl_sync(kFull, lut, code_at<4 * M + 1>(r.w[i]));
      const uint32_t a2 = __shfl_sync(kFull, lut, code_at<4 * M + 2>(r.w[i]));
      const uint32_t a3 = __shfl_sync(kFull, lut, code_at<4 * M + 3>(r.w[i]));
      mma_s8_16832(part[i], a0, a1, a2, a3, b0, b1);
    }
    StqStepsI8<M + 1, NT>::run(r, xv, lut, part);
  }
};
template <int NT>
struct StqStepsI8<8, NT> {
  __device__ __forceinline__ static void run(const StqBlockRegs<NT>&, const uint4 (&)[4], uint32_t, int (&)[NT][4]) {}
};

// Floats per row of the limb scales of K = 256 nb: three rows of nb (one per limb), padded
// to a multiple of four so that a row copies as whole 16-byte units.
__host__ __device__ constexpr int stq_limb_scale_pitch(int nb) { return (3 * nb + 3) & ~3; }

// The operand rows of one lane for the integer GEMV of an item with one or two tokens, in
// shared memory.
struct StqI8Cols {
  const int8_t* xl;  // this lane's B column: one limb row of one token (any row for an empty column)
  const float* s0;   // per-block scales (limb weight included) of output column 2t (nullptr = zero)
  const float* s1;   // ... of output column 2t+1
};

// One 1-D bulk copy global -> this CTA's shared memory (no multicast); `bytes` and both
// addresses multiples of 16; completes on `bar`'s transaction count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   tc::smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(tc::smem_u32(bar))
               : "memory");
}

// Whole-warp STQ1_0 GEMV over the nb blocks of NT tiles on the integer path: the weights in
// registers, the loads of block b+1 in flight while block b is multiplied (with L2_AHEAD,
// block b+2 also prefetched into L2); the activation limbs and scales read from the item's
// shared-memory stage once its barrier `xbar` completes phase `xphase`, so that no global
// load sits between two blocks.  acc[i][q] accumulates, in FP32, d * scale * (s32 block
// sum) of output column 2t + (q & 1) (rows g, g+8 for q < 2, q >= 2); stq_i8_tokens folds
// the columns into tokens.  Returns false if the wait gave up (STQ_ERR_TIMEOUT recorded).
// One 256-k block of the integer path: activations and scales of block b from the stage,
// weights from r.
template <int NT>
__device__ __forceinline__ void stq_block_i8(const StqBlockRegs<NT>& r, int b, const StqI8Cols& c, uint32_t lut,
                                             float (&acc)[NT][4]) {
  const int t = threadIdx.x & 3;
  uint4 xv[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) xv[q] = *reinterpret_cast<const uint4*>(c.xl + 256 * b + 16 * (4 * q + t));
  const float sc0 = c.s0 != nullptr ? c.s0[b] : 0.f;
  const float sc1 = c.s1 != nullptr ? c.s1[b] : 0.f;
  int part[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i) part[i][0] = part[i][1] = part[i][2] = part[i][3] = 0;
  StqStepsI8<0, NT>::run(r, xv, lut, part);
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const float dg = __half2float(__ushort_as_half((unsigned short)(r.d[i] & 0xFFFFu)));
    const float dg8 = __half2float(__ushort_as_half((unsigned short)(r.d[i] >> 16)));
    acc[i][0] = fmaf(dg * sc0, __int2float_rn(part[i][0]), acc[i][0]);
    acc[i][1] = fmaf(dg * sc1, __int2float_rn(part[i][1]), acc[i][1]);
    acc[i][2] = fmaf(dg8 * sc0, __int2float_rn(part[i][2]), acc[i][2]);
    acc[i][3] = fmaf(dg8 * sc1, __int2float_rn(part[i][3]), acc[i][3]);
  }
}

template <int NT, bool L2_AHEAD>
__device__ __forceinline__ void stq_prefetch_l2(const uint8_t* const (&tb)[NT], int b, int nb) {
  const int lane = threadIdx.x & 31;
  if (L2_AHEAD && b < nb && lane < 6) {
#pragma unroll
    for (int i = 0; i < NT; ++i)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(tb[i] + size_t(b) * kTileBlockBytes + 128 * lane));
  }
}

// Whole-warp STQ1_0 GEMV over the nb blocks of NT tiles on the integer path: the weights in
// registers, the loads of block b+1 in flight while block b is multiplied (with L2_AHEAD
// block b+2 also prefetched into L2; with PINGPONG two buffers used in turn instead of a
// copy per block, measured faster for the down projection's short items and slower for
// gate/up); the activation limbs and scales read from the item's shared-memory stage once
// its barrier `xbar` completes phase `xphase`, so that no global load sits between two
// blocks.  acc[i][q] accumulates, in FP32, d * scale * (s32 block sum) of output column
// 2t + (q & 1) (rows g, g+8 for q < 2, q >= 2); stq_i8_tokens folds the columns into
// tokens.  Returns false if the wait gave up (STQ_ERR_TIMEOUT recorded).
template <int NT, bool L2_AHEAD = false, bool PINGPONG = false>
__device__ __forceinline__ bool stq_warp_gemv_i8(const uint8_t* const (&tb)[NT], int nb, const StqI8Cols& c,
                                                 uint64_t* xbar, uint32_t xphase, uint32_t lut, float (&acc)[NT][4],
                                                 int32_t* err) {
  const int lane = threadIdx.x & 31;
  if (nb <= 0) return true;
  StqBlockRegs<NT> r0, r1;
  stq_load<NT>(r0, tb, 0, lane);
  if (!__all_sync(kFull, tc::mbar_wait(xbar, xphase, err))) return false;
  if (!PINGPONG) {
    for (int b = 0; b < nb; ++b) {
      stq_prefetch_l2<NT, L2_AHEAD>(tb, b + 2, nb);
      if (b + 1 < nb) stq_load<NT>(r1, tb, b + 1, lane);
      stq_block_i8<NT>(r0, b, c, lut, acc);
      r0 = r1;
    }
    return true;
  }
  for (int b = 0; b < nb; b += 2) {
    stq_prefetch_l2<NT, L2_AHEAD>(tb, b + 2, nb);
    if (b + 1 < nb) stq_load<NT>(r1, tb, b + 1, lane);
    stq_block_i8<NT>(r0, b, c, lut, acc);
    if (b + 1 >= nb) break;
    stq_prefetch_l2<NT, L2_AHEAD>(tb, b + 3, nb);
    if (b + 2 < nb) stq_load<NT>(r0, tb, b + 2, lane);
    stq_block_i8<NT>(r1, b + 1, c, lut, acc);
  }
  return true;
}

// Sum the limb columns of the two tokens: y[j][r] = row g + 8r of token j, valid in lane
// t = 0 (token 0) and t = 2 (token 1) of each quad.  Token 0 is (column 0 + column 1) +
// column 2, token 1 is (column 4 + column 5) + column 3: a fixed order.  Whole warp.
__device__ __forceinline__ void stq_i8_tokens(const float (&acc)[4], float (&y)[2]) {
  const int t = threadIdx.x & 3;
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const float ce = acc[2 * r], co = acc[2 * r + 1];  // columns 2t, 2t+1
    const float v0 = t == 0 ? ce + co : (t == 1 ? ce : 0.f);
    const float v1 = t == 2 ? ce + co : (t == 1 ? co : 0.f);
    const float o0 = __shfl_xor_sync(kFull, v0, 1);  // t=0 <-> t=1
    const float o1 = __shfl_xor_sync(kFull, v1, 3);  // t=1 <-> t=2
    y[r] = t == 0 ? v0 + o0 : v1 + o1;
  }
}

// Whole-warp BF16 GEMV: NT tiles whose row g starts at rowg[i] (row g+8 is 8*ld
// elements further), k in [k0, k1) (multiples of 32), NCH token chunks of 8.
// Within each 32-k chunk thread t holds k = 8t..8t+7: {0,1},{2,3} in the first
// mma step and {4,5},{6,7} in the second, for A and B alike.
template <int NT, int NCH>
__device__ __forceinline__ void bf16_warp_gemv(const uint16_t* const (&rowg)[NT], int64_t ld, int k0, int k1,
                                               const uint16_t* const (&xrow)[NCH], float (&acc)[NT][NCH][4]) {
  const int t = threadIdx.x & 3;
#pragma unroll 2
  for (int k = k0; k < k1; k += 32) {
    uint4 A0[NT], A8[NT], X[NCH];
#pragma unroll
    for (int i = 0; i < NT; ++i) {
      A0[i] = ldg_stream16(rowg[i] + k + 8 * t);
      A8[i] = ldg_stream16(rowg[i] + 8 * ld + k + 8 * t);
    }
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      X[c] = xrow[c] ? *reinterpret_cast<const uint4*>(xrow[c] + k + 8 * t) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        mma_bf16_16816(acc[i][c], A0[i].x, A8[i].x, A0[i].y, A8[i].y, X[c].x, X[c].y);
        mma_bf16_16816(acc[i][c], A0[i].z, A8[i].z, A0[i].w, A8[i].w, X[c].z, X[c].w);
      }
    }
  }
}

}  // namespace stq
