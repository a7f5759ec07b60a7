// Format kernels: STQ1_0 pack/unpack, MXFP4 pack/unpack, BF16 -> MXFP8 quantisation.
//
// STQ1_0 ("Hy4-preview-GGUF", section 3; "Hy4-preview-FlashMoE-STQ1_0", "How the
// STQ1_0 packing works"): one warp owns one 672-byte tile-block (16 rows x 256 k)
// and produces exactly the layout documented in include/stqmoe.h.
// MXFP4 / MXFP8 ("Hy4-preview-SF-WFP4AFP8", "Quant Diff": E2M1 / E4M3, group 32,
// UE8M0).  All outputs are bit-exact functions of the inputs.

#include <cuda_fp8.h>

#include "common.cuh"

namespace {

constexpr int kTileBlockBytes = 672;

// ----------------------------------------------------------------------------- STQ1_0

// Pattern code of one group: zero at the first lane of smallest |w|, sign bits of
// the other lanes in ascending lane order (1 = negative).
__device__ __forceinline__ uint32_t stq_group_code(float4 v) {
  float m[4] = {fabsf(v.x), fabsf(v.y), fabsf(v.z), fabsf(v.w)};
  uint32_t neg[4] = {__float_as_uint(v.x) >> 31, __float_as_uint(v.y) >> 31, __float_as_uint(v.z) >> 31,
                     __float_as_uint(v.w) >> 31};
  uint32_t z = 0;
  float best = m[0];
#pragma unroll
  for (int l = 1; l < 4; ++l)
    if (m[l] < best) { best = m[l]; z = l; }
  uint32_t s = 0, n = 0;
#pragma unroll
  for (int l = 0; l < 4; ++l)
    if ((uint32_t)l != z) { s |= neg[l] << n; ++n; }
  return 8u * z + s;
}

__global__ void stq1_pack_kernel(const float* __restrict__ w, int64_t rows, int64_t K, uint8_t* __restrict__ out,
                                 int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nb = K / 256;
  if (warp >= (rows / 16) * nb) return;
  const int64_t tile = warp / nb, b = warp % nb;
  const float* base = w + tile * 16 * K + b * 256;

  // Block amax of row (lane & 15); each half-warp covers 128 of the 256 weights.
  const int r = lane & 15, half = lane >> 4;
  const float4* p = reinterpret_cast<const float4*>(base + r * K + half * 128);
  float amax = 0.f;
  bool bad = false;
#pragma unroll 8
  for (int i = 0; i < 32; ++i) {
    float4 v = p[i];
    bad |= !isfinite(v.x) || !isfinite(v.y) || !isfinite(v.z) || !isfinite(v.w);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
  bad = __any_sync(0xffffffffu, bad || amax > 65504.f);
  if (bad && lane == 0) stq_set_error(err, STQ_ERR_NONFINITE);
  __half dh = __float2half_rn(amax);
  const uint32_t dbits = __half_as_ushort(dh);  // lane r (and r + 16) holds d of tile row r

  const int g = lane >> 2, t = lane & 3;
  const uint32_t d_lo = __shfl_sync(0xffffffffu, dbits, g);
  const uint32_t d_hi = __shfl_sync(0xffffffffu, dbits, g + 8);
  uint32_t words[5] = {0u, 0u, 0u, 0u, 0u};
#pragma unroll
  for (int s = 0; s < 16; ++s) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = g + 8 * h;
      const float4 v = *reinterpret_cast<const float4*>(base + row * K + 4 * (16 * t + s));
      uint32_t code = stq_group_code(v);
      if ((h ? d_hi : d_lo) == 0u) code = 0u;
      const int i = 2 * s + h, sh = 5 * i, w0 = sh >> 5, off = sh & 31;
      words[w0] |= code << off;
      if (off > 27) words[w0 + 1] |= code >> (32 - off);
    }
  }
  uint8_t* ob = out + warp * kTileBlockBytes;
  const uint32_t dpair = dbits | (__shfl_sync(0xffffffffu, dbits, (lane + 8) & 31) << 16);
  if (lane < 8) reinterpret_cast<uint32_t*>(ob)[lane] = dpair;
  reinterpret_cast<uint4*>(ob + 32)[lane] = make_uint4(words[0], words[1], words[2], words[3]);
  reinterpret_cast<uint32_t*>(ob + 544)[lane] = words[4];
}

// ----------------------------------------------------------------------------- STQ1_0, least squares

// Incremental cost of zeroing a lane, v * (x*x - (|x| - d)^2), in FP64 in that order
// (explicit roundings: no fused multiply-adds, so every decision is reproducible).
__device__ __forceinline__ double ls_cost(float x, float v, double d) {
  const double ax = fabs(double(x));
  const double e = __dsub_rn(ax, d);
  return __dmul_rn(double(v), __dsub_rn(__dmul_rn(double(x), double(x)), __dmul_rn(e, e)));
}

// Lane of least cost in a group (first on ties).
__device__ __forceinline__ uint32_t ls_zero_lane(float4 x, float4 v, double d) {
  const double c[4] = {ls_cost(x.x, v.x, d), ls_cost(x.y, v.y, d), ls_cost(x.z, v.z, d), ls_cost(x.w, v.w, d)};
  uint32_t z = 0;
#pragma unroll
  for (int l = 1; l < 4; ++l)
    if (c[l] < c[z]) z = uint32_t(l);
  return z;
}

// Least-squares encoder ("Hy4-preview-GGUF", section 3, "Our encoder"): from the upstream
// scale d = amax, three rounds of (zero placement by least incremental cost at the
// current d, then d = sum(v |x|) / sum(v) over the kept lanes).  One warp per tile-block
// as stq1_pack_kernel.  Decisions: lane (row r = lane & 15, half = lane >> 4) owns 32
// groups of row r; the row's sums are FP64, its two halves added by one shuffle.
// Codes: lane (g, t) places its groups again with the scale of the last round's
// placement (the same decision, same arithmetic) and writes the layout.
__global__ void stq1_pack_ls_kernel(const float* __restrict__ w, const float* __restrict__ imp, int64_t rows,
                                    int64_t K, uint8_t* __restrict__ out, int32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nb = K / 256;
  if (warp >= (rows / 16) * nb) return;
  const int64_t tile = warp / nb, b = warp % nb;
  const float* base = w + tile * 16 * K + b * 256;
  const float4 one4 = make_float4(1.f, 1.f, 1.f, 1.f);
  const float4* ib = imp != nullptr ? reinterpret_cast<const float4*>(imp + b * 256) : nullptr;

  const int r = lane & 15, half = lane >> 4;
  const float4* p = reinterpret_cast<const float4*>(base + r * K + half * 128);
  float amax = 0.f;
  bool bad = false, badv = false;
  for (int i = 0; i < 32; ++i) {
    const float4 x = p[i];
    const float4 v = ib != nullptr ? ib[half * 32 + i] : one4;
    bad |= !isfinite(x.x) || !isfinite(x.y) || !isfinite(x.z) || !isfinite(x.w);
    badv |= !(v.x >= 0.f && v.y >= 0.f && v.z >= 0.f && v.w >= 0.f) || !isfinite(v.x) || !isfinite(v.y) ||
            !isfinite(v.z) || !isfinite(v.w);
    amax = fmaxf(amax, fmaxf(fmaxf(fabsf(x.x), fabsf(x.y)), fmaxf(fabsf(x.z), fabsf(x.w))));
  }
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 16));
  bad = __any_sync(0xffffffffu, bad || amax > 65504.f);
  badv = __any_sync(0xffffffffu, badv);
  if (lane == 0) {
    if (bad) stq_set_error(err, STQ_ERR_NONFINITE);
    if (badv) stq_set_error(err, STQ_ERR_INVALID_ARG);
  }
  double d = double(amax), d_place = d;
  for (int round = 0; round < 3; ++round) {
    d_place = d;
    double num = 0.0, den = 0.0;
    for (int i = 0; i < 32; ++i) {
      const float4 x = p[i];
      const float4 v = ib != nullptr ? ib[half * 32 + i] : one4;
      const uint32_t z = ls_zero_lane(x, v, d_place);
      const float xs[4] = {x.x, x.y, x.z, x.w}, vs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int l = 0; l < 4; ++l)
        if (uint32_t(l) != z) {
          num = __dadd_rn(num, __dmul_rn(double(vs[l]), fabs(double(xs[l]))));
          den = __dadd_rn(den, double(vs[l]));
        }
    }
    num = __dadd_rn(num, __shfl_xor_sync(0xffffffffu, num, 16));
    den = __dadd_rn(den, __shfl_xor_sync(0xffffffffu, den, 16));
    d = den > 0.0 ? __ddiv_rn(num, den) : 0.0;
  }
  const uint32_t dbits = __half_as_ushort(__double2half(d));  // lanes r and r + 16 hold row r's scale

  const int g = lane >> 2, t = lane & 3;
  const uint32_t d_lo = __shfl_sync(0xffffffffu, dbits, g);
  const uint32_t d_hi = __shfl_sync(0xffffffffu, dbits, g + 8);
  const double dp_lo = __shfl_sync(0xffffffffu, d_place, g);
  const double dp_hi = __shfl_sync(0xffffffffu, d_place, g + 8);
  uint32_t words[5] = {0u, 0u, 0u, 0u, 0u};
  for (int s = 0; s < 16; ++s) {
    const float4 v = ib != nullptr ? ib[16 * t + s] : one4;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = g + 8 * h;
      const float4 x = *reinterpret_cast<const float4*>(base + row * K + 4 * (16 * t + s));
      const uint32_t z = ls_zero_lane(x, v, h ? dp_hi : dp_lo);
      const uint32_t neg[4] = {__float_as_uint(x.x) >> 31, __float_as_uint(x.y) >> 31, __float_as_uint(x.z) >> 31,
                               __float_as_uint(x.w) >> 31};
      uint32_t sb = 0, n = 0;
#pragma unroll
      for (int l = 0; l < 4; ++l)
        if (uint32_t(l) != z) { sb |= neg[l] << n; ++n; }
      uint32_t code = 8u * z + sb;
      if ((h ? d_hi : d_lo) == 0u) code = 0u;
      const int i = 2 * s + h, sh = 5 * i, w0 = sh >> 5, off = sh & 31;
      words[w0] |= code << off;
      if (off > 27) words[w0 + 1] |= code >> (32 - off);
    }
  }
  uint8_t* ob = out + warp * kTileBlockBytes;
  const uint32_t dpair = dbits | (__shfl_sync(0xffffffffu, dbits, (lane + 8) & 31) << 16);
  if (lane < 8) reinterpret_cast<uint32_t*>(ob)[lane] = dpair;
  reinterpret_cast<uint4*>(ob + 32)[lane] = make_uint4(words[0], words[1], words[2], words[3]);
  reinterpret_cast<uint32_t*>(ob + 544)[lane] = words[4];
}

__global__ void stq1_unpack_kernel(const uint8_t* __restrict__ in, int64_t rows, int64_t K, float* __restrict__ w) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nb = K / 256;
  if (warp >= (rows / 16) * nb) return;
  const int64_t tile = warp / nb, b = warp % nb;
  const uint8_t* ib = in + warp * kTileBlockBytes;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t dpair = reinterpret_cast<const uint32_t*>(ib)[g];
  const uint4 a = reinterpret_cast<const uint4*>(ib + 32)[lane];
  const uint32_t words[5] = {a.x, a.y, a.z, a.w, reinterpret_cast<const uint32_t*>(ib + 544)[lane]};
  const float dv[2] = {__half2float(__ushort_as_half((unsigned short)(dpair & 0xFFFFu))),
                       __half2float(__ushort_as_half((unsigned short)(dpair >> 16)))};
  float* base = w + tile * 16 * K + b * 256;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int s = i >> 1, h = i & 1, sh = 5 * i, w0 = sh >> 5, off = sh & 31;
    uint32_t c = words[w0] >> off;
    if (off > 27) c |= words[w0 + 1] << (32 - off);
    c &= 31u;
    const uint32_t z = c >> 3;
    float vals[4];
    uint32_t n = 0;
#pragma unroll
    for (int l = 0; l < 4; ++l) {
      if ((uint32_t)l == z) {
        vals[l] = 0.f;
      } else {
        vals[l] = ((c >> n) & 1u) ? -dv[h] : dv[h];
        ++n;
      }
    }
    *reinterpret_cast<float4*>(base + (g + 8 * h) * K + 4 * (16 * t + s)) = make_float4(vals[0], vals[1], vals[2], vals[3]);
  }
}

// ----------------------------------------------------------------------------- MXFP4

// E2M1 round to nearest, ties to the even code, of y in [0, 6].
__device__ __forceinline__ uint32_t e2m1_rne_mag(float y) {
  return uint32_t(y > 0.25f) + uint32_t(y >= 0.75f) + uint32_t(y > 1.25f) + uint32_t(y >= 1.75f) +
         uint32_t(y > 2.5f) + uint32_t(y >= 3.5f) + uint32_t(y > 5.0f);
}

__global__ void mxfp4_pack_kernel(const float* __restrict__ w, int64_t rows, int64_t K, uint8_t* __restrict__ codes,
                                  uint8_t* __restrict__ scales, int32_t* err) {
  const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t ng = rows * (K / 32);
  if (gi >= ng) return;
  const float4* p = reinterpret_cast<const float4*>(w + gi * 32);
  float v[32];
  float amax = 0.f;
  bool bad = false;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    float4 q = p[i];
    v[4 * i] = q.x; v[4 * i + 1] = q.y; v[4 * i + 2] = q.z; v[4 * i + 3] = q.w;
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    bad |= !isfinite(v[i]);
    amax = fmaxf(amax, fabsf(v[i]));
  }
  if (bad) stq_set_error(err, STQ_ERR_NONFINITE);
  const int e = mx_scale_exponent(amax, 0x400000u, 2);  // limit 6 = 1.5 * 2^2
  const float f = pow2_float(127 - e);
  uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint32_t c = e2m1_rne_mag(fabsf(v[i]) * f) | ((__float_as_uint(v[i]) >> 31) << 3);
    out[i >> 3] |= c << (4 * (i & 7));
  }
  *reinterpret_cast<uint4*>(codes + gi * 16) = make_uint4(out[0], out[1], out[2], out[3]);
  scales[gi] = uint8_t(e);
}

__global__ void mxfp4_unpack_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                    int64_t rows, int64_t K, float* __restrict__ w) {
  const int64_t gi = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gi >= rows * (K / 32)) return;
  const uint4 c = *reinterpret_cast<const uint4*>(codes + gi * 16);
  const int e = scales[gi];
  const float sc = e == 255 ? __uint_as_float(0x7FC00000u) : pow2_float(e - 127);
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
  float4* out = reinterpret_cast<float4*>(w + gi * 32);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float r[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t code = (cw[q >> 1] >> (4 * (4 * (q & 1) + j))) & 15u;
      const uint32_t ef = (code >> 1) & 3u, m = code & 1u;
      const float mag = ef == 0 ? 0.5f * float(m) : (1.0f + 0.5f * float(m)) * float(1u << (ef - 1));
      const float val = (code & 8u) ? -mag : mag;
      r[j] = val * sc;
    }
    out[q] = make_float4(r[0], r[1], r[2], r[3]);
  }
}

// ----------------------------------------------------------------------------- MXFP8

// Four lanes per 32-element group, eight elements per lane.
// Grid (column chunks of 2048 elements, rows; rows beyond 65535 loop): thread = 8
// consecutive elements, 4 threads = one 32-element group, no 64-bit division per thread.
// RPB rows per CTA (rows RPB*blockIdx.y .. +RPB, then strided by the grid): every row's
// activation load is issued before the first row is quantised, so the load latency is paid
// once per RPB rows.
// Scatter (dst != nullptr): source row r (a token) is quantised once and its codes and
// scales are written to the k output rows dst[r*k + s], s = 0..k-1 (the sorted position of
// each of its (token, slot) pairs; -1 = none); out_rows bounds those positions.  Otherwise
// output row r is source row r.
template <int RPB>
__global__ void __launch_bounds__(256) mxfp8_quant_bf16_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                               int64_t K, uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ scales,
                                                               const int32_t* __restrict__ dst, int k,
                                                               int64_t out_rows, int32_t* err) {
  stq_pdl_begin();
  const int part = int(threadIdx.x & 3);
  const int64_t col8 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;  // 8-element chunk of the row
  const bool active = col8 < K / 8;                                     // whole 4-thread groups
  for (int64_t r0 = int64_t(blockIdx.y) * RPB; r0 < rows; r0 += int64_t(gridDim.y) * RPB) {
    uint4 raw[RPB];
#pragma unroll
    for (int j = 0; j < RPB; ++j) {
      raw[j] = make_uint4(0u, 0u, 0u, 0u);
      const int64_t row = r0 + j;
      if (active && row < rows) raw[j] = *reinterpret_cast<const uint4*>(x + row * K + col8 * 8);
    }
#pragma unroll
    for (int j = 0; j < RPB; ++j) {
      const int64_t row = r0 + j;
      if (row >= rows) break;  // the same for every thread of the CTA
      float v[8];
      float amax = 0.f;
      bool bad = false;
      if (active) {
        const uint32_t rw[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          v[2 * i] = bf16_bits_to_float(rw[i] & 0xFFFFu);
          v[2 * i + 1] = bf16_bits_to_float(rw[i] >> 16);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          bad |= !isfinite(v[i]);
          amax = fmaxf(amax, isfinite(v[i]) ? fabsf(v[i]) : 0.f);
        }
      }
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
      amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
      const unsigned badmask = __ballot_sync(0xffffffffu, bad);
      if (!active) continue;
      const bool gbad = (badmask >> (threadIdx.x & 28)) & 0xFu;
      int e = mx_scale_exponent(amax, 0x600000u, 8);  // limit 448 = 1.75 * 2^8
      uint32_t lo = 0u, hi = 0u;
      if (gbad) {
        e = 255;
        lo = hi = 0x7F7F7F7Fu;
      } else {
        const float f = pow2_float(127 - e);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const __nv_fp8x2_storage_t pr =
              __nv_cvt_float2_to_fp8x2(make_float2(v[i] * f, v[i + 1] * f), __NV_SATFINITE, __NV_E4M3);
          uint32_t c0 = pr & 0xFFu, c1 = (pr >> 8) & 0xFFu;
          // zero results carry the sign of the input
          if ((c0 & 0x7Fu) == 0u) c0 = (__float_as_uint(v[i]) >> 31) << 7;
          if ((c1 & 0x7Fu) == 0u) c1 = (__float_as_uint(v[i + 1]) >> 31) << 7;
          const uint32_t pair = c0 | (c1 << 8);
          if (i < 4) lo |= pair << (8 * i); else hi |= pair << (8 * (i - 4));
        }
      }
      const int64_t g32 = col8 >> 2;  // 32-element group of the row
      if (dst == nullptr) {
        *reinterpret_cast<uint2*>(codes + row * K + col8 * 8) = make_uint2(lo, hi);
        if (part == 0) scales[row * (K / 32) + g32] = uint8_t(e);
      } else {
        for (int s = 0; s < k; ++s) {
          const int64_t pos = dst[row * k + s];
          if (pos < 0 || !STQ_DCHECK(pos < out_rows, err)) continue;
          *reinterpret_cast<uint2*>(codes + pos * K + col8 * 8) = make_uint2(lo, hi);
          if (part == 0) scales[pos * (K / 32) + g32] = uint8_t(e);
        }
      }
    }
  }
}

// From 4096 rows a CTA takes 8 rows (enough CTAs remain to fill the SMs), below it one.
constexpr int64_t kQuantMultiRow = 4096;

dim3 quant_grid(int64_t rows, int64_t K) {
  const int64_t ry = rows >= kQuantMultiRow ? ceil_div<int64_t>(rows, 8) : rows;
  return dim3(unsigned(ceil_div<int64_t>(K / 8, 256)), unsigned(ry < 65535 ? ry : 65535));
}

}  // namespace

// ----------------------------------------------------------------------------- C ABI

extern "C" stq_status stq1_pack(const float* w, int64_t rows, int64_t K, uint8_t* out, int32_t* err,
                                stq_stream_t stream) {
  STQ_HOST_CHECK(w && out, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows >= 0 && K >= 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows % 16 == 0 && K % 256 == 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(stq_aligned16(w) && stq_aligned16(out), STQ_ERR_ALIGN);
  const int64_t warps = (rows / 16) * (K / 256);
  if (warps == 0) return STQ_OK;
  stq1_pack_kernel<<<unsigned(ceil_div<int64_t>(warps, 4)), 128, 0, stq_cuda_stream(stream)>>>(w, rows, K, out, err);
  return stq_launch_status();
}

extern "C" stq_status stq1_pack_ls(const float* w, const float* importance, int64_t rows, int64_t K, uint8_t* out,
                                   int32_t* err, stq_stream_t stream) {
  STQ_HOST_CHECK(rows >= 0 && K >= 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows % 16 == 0 && K % 256 == 0, STQ_ERR_SHAPE);
  if (rows == 0 || K == 0) return STQ_OK;  // nothing to read or write: pointers may be NULL
  STQ_HOST_CHECK(w && out, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(stq_aligned16(w) && stq_aligned16(out) && (importance == nullptr || stq_aligned16(importance)),
                 STQ_ERR_ALIGN);
  const int64_t warps = (rows / 16) * (K / 256);
  if (warps == 0) return STQ_OK;
  {
    StqTimed tm(STQ_K_PACK_LS, stq_cuda_stream(stream));
    stq1_pack_ls_kernel<<<unsigned(ceil_div<int64_t>(warps, 4)), 128, 0, stq_cuda_stream(stream)>>>(
        w, importance, rows, K, out, err);
  }
  return stq_launch_status();
}

extern "C" stq_status stq1_unpack(const uint8_t* in, int64_t rows, int64_t K, float* w, stq_stream_t stream) {
  STQ_HOST_CHECK(in && w, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows >= 0 && K >= 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows % 16 == 0 && K % 256 == 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(stq_aligned16(w) && stq_aligned16(in), STQ_ERR_ALIGN);
  const int64_t warps = (rows / 16) * (K / 256);
  if (warps == 0) return STQ_OK;
  stq1_unpack_kernel<<<unsigned(ceil_div<int64_t>(warps, 4)), 128, 0, stq_cuda_stream(stream)>>>(in, rows, K, w);
  return stq_launch_status();
}

extern "C" stq_status mxfp4_pack(const float* w, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales,
                                 int32_t* err, stq_stream_t stream) {
  STQ_HOST_CHECK(w && codes && scales, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows >= 0 && K >= 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(K % 32 == 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(stq_aligned16(w) && stq_aligned16(codes), STQ_ERR_ALIGN);
  const int64_t ng = rows * (K / 32);
  if (ng == 0) return STQ_OK;
  mxfp4_pack_kernel<<<unsigned(ceil_div<int64_t>(ng, 256)), 256, 0, stq_cuda_stream(stream)>>>(w, rows, K, codes,
                                                                                               scales, err);
  return stq_launch_status();
}

extern "C" stq_status mxfp4_unpack(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, float* w,
                                   stq_stream_t stream) {
  STQ_HOST_CHECK(w && codes && scales, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows >= 0 && K >= 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(K % 32 == 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(stq_aligned16(w) && stq_aligned16(codes), STQ_ERR_ALIGN);
  const int64_t ng = rows * (K / 32);
  if (ng == 0) return STQ_OK;
  mxfp4_unpack_kernel<<<unsigned(ceil_div<int64_t>(ng, 256)), 256, 0, stq_cuda_stream(stream)>>>(codes, scales, rows,
                                                                                                 K, w);
  return stq_launch_status();
}

stq_status stq_mxfp8_quantize_launch(const uint16_t* x, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales,
                                     cudaStream_t s) {
  const int64_t threads = rows * (K / 32) * 4;
  if (threads == 0) return STQ_OK;
  StqTimed tm(STQ_K_QUANT_X, s);
  const int32_t* no_map = nullptr;
  int32_t* no_err = nullptr;
  if (rows >= kQuantMultiRow)
    return stq_launch(mxfp8_quant_bf16_kernel<8>, quant_grid(rows, K), dim3(256), 0, s, x, rows, K, codes, scales, no_map,
                      1, rows, no_err);
  return stq_launch(mxfp8_quant_bf16_kernel<1>, quant_grid(rows, K), dim3(256), 0, s, x, rows, K, codes, scales, no_map,
                    1, rows, no_err);
}

stq_status stq_mxfp8_quantize_scatter_launch(const uint16_t* x, int64_t T, int64_t K, const int32_t* inv, int k,
                                             int64_t out_rows, int32_t* err, uint8_t* codes, uint8_t* scales,
                                             cudaStream_t s) {
  const int64_t threads = T * (K / 32) * 4;
  if (threads == 0) return STQ_OK;
  StqTimed tm(STQ_K_QUANT_X, s);
  if (T >= kQuantMultiRow)
    return stq_launch(mxfp8_quant_bf16_kernel<8>, quant_grid(T, K), dim3(256), 0, s, x, T, K, codes, scales, inv, k,
                      out_rows, err);
  return stq_launch(mxfp8_quant_bf16_kernel<1>, quant_grid(T, K), dim3(256), 0, s, x, T, K, codes, scales, inv, k,
                    out_rows, err);
}

extern "C" stq_status mxfp8_quantize_bf16(const uint16_t* x, int64_t rows, int64_t K, uint8_t* codes,
                                          uint8_t* scales, stq_stream_t stream) {
  STQ_HOST_CHECK(x && codes && scales, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(rows >= 0 && K >= 0, STQ_ERR_INVALID_ARG);
  STQ_HOST_CHECK(K % 32 == 0, STQ_ERR_SHAPE);
  STQ_HOST_CHECK(stq_aligned16(x) && stq_aligned16(codes), STQ_ERR_ALIGN);
  return stq_mxfp8_quantize_launch(x, rows, K, codes, scales, stq_cuda_stream(stream));
}
