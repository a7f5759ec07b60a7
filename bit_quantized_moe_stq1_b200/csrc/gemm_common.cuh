// Pieces shared by the grouped tensor-core GEMMs (W4A8 and STQ1_0 x MXFP8): activation
// scale-factor staging, the work-item map over (N tile, M tile), and the TMEM epilogue
// (FP32 expert outputs, or SwiGLU with the MXFP8 re-quantisation of h).
#pragma once

#include "moe_internal.cuh"
#include "tcgen05.cuh"

namespace gemm {

// Scales of 128-k stage kt for the four 32-row slices m1 of a 128-row block: lane m0
// reads the 4 bytes (4 k-blocks) of rows m0 + 32*m1.  Rows at or past `limit`
// (absolute) or `nvalid` (relative), and stages past nk, read as zero.
__device__ __forceinline__ void load_sf(uint32_t (&v)[4], const uint8_t* src, int row0, int nvalid, int limit,
                                        int k32, int kt, int nk, int lane) {
#pragma unroll
  for (int m1 = 0; m1 < 4; ++m1) {
    const int r = lane + 32 * m1;
    v[m1] = (kt < nk && r < nvalid && row0 + r < limit)
                ? __ldg(reinterpret_cast<const uint32_t*>(src + size_t(row0 + r) * k32 + size_t(kt) * 4))
                : 0u;
  }
}

// Store them into the scale-factor atom: row m = m0 + 32*m1 at byte m0*16 + m1*4 + kb.
__device__ __forceinline__ void store_sf(uint8_t* dst, const uint32_t (&v)[4], int lane) {
  *reinterpret_cast<uint4*>(dst + lane * 16) = make_uint4(v[0], v[1], v[2], v[3]);
}

// Grouped tiling: N tiles of NT tokens of one expert (from the tile plan), M tiles of
// rows_per_tile weight rows; work item i covers N tile i / MT and M tile i % MT.
struct Tiling {
  int R;                     // weight rows per expert
  const int32_t* offsets;    // grouped: [E+1]; nullptr = one dense expert of dense_M tokens
  const int2* ntiles;        // grouped: (expert, first token) per N tile
  const int32_t* n_ntiles;   // grouped: number of N tiles (device)
  int dense_M;
  int max_items;             // upper bound of the work items (N tiles x M tiles)
};

struct Item {
  bool valid;
  int e, mt, n0, pos0, cnt, arow, brow;
};

__device__ __forceinline__ Item get_item(const Tiling& p, int item, int MT, int rows_per_tile, int NT) {
  Item t{};
  const int nti = item / MT;
  t.mt = item - nti * MT;
  if (p.offsets != nullptr) {
    t.valid = item < p.max_items && nti < *p.n_ntiles;
    if (!t.valid) return t;
    const int2 w = p.ntiles[nti];
    t.e = w.x;
    t.n0 = w.y;
    t.pos0 = p.offsets[t.e];
    t.cnt = p.offsets[t.e + 1] - t.pos0;
  } else {
    t.valid = item < p.max_items;
    if (!t.valid) return t;
    t.e = 0;
    t.n0 = nti * NT;
    t.pos0 = 0;
    t.cnt = p.dense_M;
  }
  t.arow = t.e * p.R + t.mt * rows_per_tile;
  t.brow = t.pos0 + t.n0;
  return t;
}

// MMA width for an item: its tokens in the N tile, rounded up to the 16-column step of
// an M = 128 MMA (columns past it are neither computed nor read).
__device__ __forceinline__ int item_cols(const Item& I, int NT) {
  const int n = min(NT, I.cnt - I.n0);
  return (n + 15) & ~15;
}

// Outputs of the epilogue.
struct EpiOut {
  int R;          // weight rows per expert (output features)
  float* Y;       // single: [Ptot][R]
  uint8_t* hq;    // pair: MXFP8 codes of h [Ptot][R]
  uint8_t* hs;    // pair: scales [Ptot][R/32]
};

// Drain one NT-column accumulator tile (TMEM lanes 32q..32q+31 of this warp, columns
// from `tl`) into the outputs.  PAIR: lanes 0-63 are gate rows and 64-127 the same up
// rows; warps q and q+2 exchange halves of each 16-column chunk through `ubuf` and meet
// at named barrier 1 (all four epilogue warps, 128 threads).
template <int NT, bool PAIR>
__device__ __forceinline__ void epilogue_tile(uint32_t tl, const Item& I, const EpiOut& o, float* ubuf, int q,
                                              int lane) {
  for (int c0 = 0; c0 < NT; c0 += 16) {
    if (I.n0 + c0 >= I.cnt) break;
    uint32_t v[16];
    tc::tmem_ld_x16(tl + c0, v);
    tc::tmem_ld_wait();
    if constexpr (PAIR) {
      // Warps q and q+2 hold the gate and up values of the same 32 features; the gate
      // warp takes columns 0-7 of the chunk and the up warp columns 8-15, each handing
      // the other its half through shared memory.
      const int pr = q & 1;
      const bool gate = q < 2;
      float* mine = ubuf + (2 * pr + (gate ? 0 : 1)) * (32 * 9);
      const float* other = ubuf + (2 * pr + (gate ? 1 : 0)) * (32 * 9);
      if (gate) {
#pragma unroll
        for (int j = 0; j < 8; ++j) mine[lane * 9 + j] = __uint_as_float(v[8 + j]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) mine[lane * 9 + j] = __uint_as_float(v[j]);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const int f = I.mt * 64 + 32 * pr + lane;  // output feature of this lane
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int col = I.n0 + c0 + (gate ? j : 8 + j);
        if (col >= I.cnt) break;
        const float g = gate ? __uint_as_float(v[j]) : other[lane * 9 + j];
        const float u = gate ? other[lane * 9 + j] : __uint_as_float(v[8 + j]);
        const float h = g / (1.0f + __expf(-g)) * u;  // silu(g) * u
        const bool bad = !isfinite(h);
        // amax over the 32 features of this column: the bits of a non-negative float
        // order like the float, so one integer max reduction suffices
        const uint32_t amax_bits = __reduce_max_sync(0xffffffffu, bad ? 0u : (__float_as_uint(h) & 0x7FFFFFFFu));
        const bool anybad = __any_sync(0xffffffffu, bad);
        const int ex = anybad ? 255 : mx_scale_exponent(__uint_as_float(amax_bits), 0x600000u, 8);
        const uint32_t code = anybad ? 0x7Fu : e4m3_code(h, pow2_float(127 - ex));
        const size_t pos = size_t(I.pos0 + col);
        o.hq[pos * o.R + f] = uint8_t(code);
        if (lane == 0) o.hs[pos * (o.R / 32) + (f >> 5)] = uint8_t(ex);
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    } else {
      const int f = I.mt * 128 + 32 * q + lane;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int col = I.n0 + c0 + j;
        if (col >= I.cnt) break;
        o.Y[size_t(I.pos0 + col) * o.R + f] = __uint_as_float(v[j]);
      }
    }
  }
}

// The four epilogue warps agree on a flag (named barrier 1, 128 threads).
__device__ __forceinline__ bool all_of_epilogue(bool ok) {
  uint32_t all;
  asm volatile(
      "{\n .reg .pred p, r;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred r, 1, 128, p;\n"
      " selp.u32 %0, 1, 0, r;\n}"
      : "=r"(all)
      : "r"(ok ? 1u : 0u)
      : "memory");
  return all != 0u;
}

}  // namespace gemm
