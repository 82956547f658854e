// Producer side of the layer (the step before the hot path): a dense weight
// matrix W [N, K] is folded with the block rotation and rounded to ternary
// g128 (openbonsai.org, "How it works", steps 1 "Rotate" and 2 "Round"; the
// pages round with sequential GPTQ on calibration data, this is the plain
// stand-in).  Fold: W' = W R, i.e. every row gets the transform the run time
// applies to activations, w'_b = H (d_b * w_b) / 32.  Round: per 128-group
// s = fp16(mean |w'|), t = clip(rint(w' / s), -1, 1), t = 0 where s = 0.  The
// codes go out packed (2-bit slots or base-3) with the scales beside them.
//
// Arithmetic is fp64 throughout (the fold's sums, the group's sum of |w'|, the
// division w'/s) and the scale is rounded from fp64 to fp16 once, to nearest
// even.  For bf16 and fp16 input (and fp32 input whose values span fewer than
// about 40 binary orders inside a block) every one of those fp64 sums is
// exact, so the codes and scales do not depend on summation order and equal
// an exact-arithmetic rounding bit for bit.
//
// One warp per (row, 1024-block): lane c loads w[32 r + c] (r = 0..31, one
// load instruction reads 32 consecutive elements), transforms over r in
// registers; a transpose through 4 KB of shared memory (two halves of 16 rows
// of 32 doubles, 16-byte chunks XOR-swizzled by the row) gives lane a the
// elements 32 a .. 32 a + 31, transformed over the low five index bits in
// registers.  Lanes 4g .. 4g + 3 then hold group g of the block.
#pragma once
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kPwWarps = 8;

__device__ __forceinline__ void pw_fwht32(double (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & h) == 0) {
        const double a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// Nearest fp16 value (ties to even) of a non-negative double, by scaling to the
// fp16 unit in the last place of a's binade (a power of two, so exact) and
// rounding to an integer there; then converted to half exactly (the result is
// representable).  Values at or above 65520 round to infinity.
__device__ __forceinline__ __half pw_double_to_half_rn(double a) {
  if (!(a > 0.0)) return __float2half_rn(0.f);
  if (a >= 65520.0) return __ushort_as_half(static_cast<unsigned short>(0x7C00u));
  int e = ilogb(a);              // 2^e <= a < 2^(e+1)
  if (e < -14) e = -14;          // subnormal range: unit 2^-24
  const double unit = ldexp(1.0, e - 10);
  const double r = rint(a / unit) * unit;  // a / unit and the product are exact
  return __float2half_rn(static_cast<float>(r));
}

// kFmt: 0 = 2-bit slots, 1 = base-3.  grid (K / 1024, ceil(N / kPwWarps)).
template <typename TIn, int kFmt>
__global__ void __launch_bounds__(32 * kPwWarps)
    prepare_weights_kernel(const TIn* __restrict__ w, const int8_t* __restrict__ signs,
                           uint8_t* __restrict__ packed, uint16_t* __restrict__ scales, int64_t N, int K) {
  __shared__ __align__(16) double xbuf[kPwWarps][512];
  __shared__ __align__(16) uint8_t cbuf[kPwWarps][kHB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int blk = blockIdx.x;
  const int64_t row = static_cast<int64_t>(blockIdx.y) * kPwWarps + warp;
  if (row >= N) return;  // a whole warp; nothing below synchronises beyond the warp
  const int G = K >> 7;
  const TIn* src = w + row * K + static_cast<int64_t>(blk) * kHB;
  double v[32];
  if (signs != nullptr) {
    const int8_t* sg = signs + static_cast<int64_t>(blk) * kHB;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const double f = static_cast<double>(to_f32<TIn>(src[32 * i + lane]));
      v[i] = sg[32 * i + lane] < 0 ? -f : f;
    }
    pw_fwht32(v);  // over the high five index bits (r)
    double u[32];
    double* xb = xbuf[warp];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      // row r of this half, element c = lane: 16-byte chunk lane/2 stored at
      // chunk (lane/2) ^ r
#pragma unroll
      for (int r = 0; r < 16; ++r) xb[32 * r + ((((lane >> 1) ^ r) & 15) << 1) + (lane & 1)] = v[16 * hf + r];
      __syncwarp();
      if ((lane >> 4) == hf) {
        const int r = lane & 15;
        const double2* rowp = reinterpret_cast<const double2*>(xb + 32 * r);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const double2 t = rowp[q ^ r];
          u[2 * q] = t.x;
          u[2 * q + 1] = t.y;
        }
      }
      __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = u[i];
    pw_fwht32(v);  // over the low five index bits (c)
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= 0.03125;  // 1/32: exact
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = static_cast<double>(to_f32<TIn>(src[32 * lane + i]));
  }
  // group g = lane >> 2 of the block: scale and codes
  double sa = 0.0;
#pragma unroll
  for (int i = 0; i < 32; ++i) sa += fabs(v[i]);
  sa += __shfl_xor_sync(0xffffffffu, sa, 1);
  sa += __shfl_xor_sync(0xffffffffu, sa, 2);
  const __half s16 = pw_double_to_half_rn(sa * (1.0 / 128.0));  // exact division by 128
  const double s = static_cast<double>(__half2float(s16));
  const int g = lane >> 2;
  uint32_t c[32];  // biased codes t + 1
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const double q = s > 0.0 ? rint(__ddiv_rn(v[i], s)) : 0.0;
    c[i] = static_cast<uint32_t>(static_cast<int>(fmin(fmax(q, -1.0), 1.0)) + 1);
  }
  if ((lane & 3) == 0) scales[row * G + blk * 8 + g] = __half_as_ushort(s16);
  if constexpr (kFmt == 0) {
    // 2-bit slots: byte i of the row holds codes 4i .. 4i + 3 at bits 2j
    uint32_t wd[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      uint32_t acc = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) acc |= c[4 * h + j] << (2 * j);
      wd[h] = acc;
    }
    uint8_t* dst = packed + row * (K >> 2) + static_cast<int64_t>(blk) * (kHB / 4) + 8 * lane;
    *reinterpret_cast<uint2*>(dst) = make_uint2(wd[0] | (wd[1] << 8) | (wd[2] << 16) | (wd[3] << 24),
                                                wd[4] | (wd[5] << 8) | (wd[6] << 16) | (wd[7] << 24));
  } else {
    // base-3: per group 26 bytes; byte i < 25 = sum_j c[5i + j] 3^j, byte 25 =
    // c[125] + 3 c[126] + 9 c[127] + 27 + 81 (padding digits 1)
    uint8_t* cb = cbuf[warp];
#pragma unroll
    for (int i = 0; i < 32; ++i) cb[32 * lane + i] = static_cast<uint8_t>(c[i]);
    __syncwarp();
    uint8_t* dst = packed + row * (static_cast<int64_t>(G) * 26) + static_cast<int64_t>(blk) * 208;
    for (int idx = lane; idx < 208; idx += 32) {
      const int gg = idx / 26, i = idx - 26 * gg;
      const uint8_t* cg = cb + 128 * gg;
      uint32_t byte;
      if (i < 25)
        byte = cg[5 * i] + 3u * cg[5 * i + 1] + 9u * cg[5 * i + 2] + 27u * cg[5 * i + 3] + 81u * cg[5 * i + 4];
      else
        byte = cg[125] + 3u * cg[126] + 9u * cg[127] + 27u + 81u;
      dst[idx] = static_cast<uint8_t>(byte);
    }
  }
}

}  // namespace tb
