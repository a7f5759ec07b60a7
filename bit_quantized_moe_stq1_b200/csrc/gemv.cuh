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
