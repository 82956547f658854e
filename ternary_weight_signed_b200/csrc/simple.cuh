// Plain per-row kernel for the ternary g128 product: one warp per output row,
// lanes over 128-groups, codes decoded straight from the packed bytes with
// byte loads.  It takes every shape, alignment and packed format the API
// allows (K % 128 == 0) and both modes:
//   float  : y[m,n] = sum_g s[n,g] sum_{k in g} t[n,k] x'[m,k]   (x' fp32)
//   integer: y[m,n] = sum_k t[n,k] x[m,k]                          (exact int32)
// It is the path for shapes the fast kernels do not take, not a tuned kernel.
#pragma once
#include "tb_device.cuh"

namespace tb {

constexpr int kSimpleWarps = 8;
constexpr int kSimpleMC = 8;  // tokens per pass

// Decodes the 128 codes of group g of row n into t[0..127] (invalid -> 0).
template <int FMT>
__device__ __forceinline__ int8_t group_code(const uint8_t* __restrict__ grp, int k);

template <>
__device__ __forceinline__ int8_t group_code<0>(const uint8_t* __restrict__ grp, int k) {
  const uint32_t c = (grp[k >> 2] >> (2 * (k & 3))) & 3u;
  return c == 3u ? int8_t(0) : static_cast<int8_t>(static_cast<int>(c) - 1);
}

template <>
__device__ __forceinline__ int8_t group_code<1>(const uint8_t* __restrict__ grp, int k) {
  const int b = k / 5, j = k - 5 * (k / 5);
  const uint32_t v = grp[b];
  uint32_t d = v;
  uint32_t dig[5];
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    dig[i] = d % 3u;
    d /= 3u;
  }
  bool invalid = v >= 243u;
  if (b == 25) invalid = invalid || dig[3] != 1u || dig[4] != 1u;
  return invalid ? int8_t(0) : static_cast<int8_t>(static_cast<int>(dig[j]) - 1);
}

// 1-bit: bit k % 8 of byte k / 8, bit 1 = +1, bit 0 = -1.
template <>
__device__ __forceinline__ int8_t group_code<2>(const uint8_t* __restrict__ grp, int k) {
  return ((grp[k >> 3] >> (k & 7)) & 1u) ? int8_t(1) : int8_t(-1);
}

// Packed bytes of one 128-group and of one row of K codes, per format
// (0 = 2-bit slots, 1 = base-3, 2 = 1-bit).
__host__ __device__ constexpr int simple_group_bytes(int fmt) { return fmt == 0 ? 32 : (fmt == 1 ? 26 : 16); }

template <int FMT, bool INT_MODE, typename TX, typename TOut>
__global__ void __launch_bounds__(32 * kSimpleWarps)
    simple_linear_kernel(const TX* __restrict__ x, const uint8_t* __restrict__ packed,
                         const __half* __restrict__ scales, TOut* __restrict__ y, int M, int N,
                         int K) {
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = blockIdx.x * kSimpleWarps + warp;
  if (n >= N) return;
  const int G = K / 128;
  constexpr int grp_bytes = simple_group_bytes(FMT);
  const int64_t row_bytes = static_cast<int64_t>(G) * grp_bytes;
  const uint8_t* prow = packed + static_cast<int64_t>(n) * row_bytes;
  for (int m0 = 0; m0 < M; m0 += kSimpleMC) {
    const int mc = min(kSimpleMC, M - m0);
    float facc[kSimpleMC];
    int iacc[kSimpleMC];
#pragma unroll
    for (int i = 0; i < kSimpleMC; ++i) {
      facc[i] = 0.f;
      iacc[i] = 0;
    }
    for (int g = lane; g < G; g += 32) {
      const uint8_t* grp = prow + static_cast<int64_t>(g) * grp_bytes;
      float gf[kSimpleMC];
#pragma unroll
      for (int i = 0; i < kSimpleMC; ++i) gf[i] = 0.f;
      for (int k = 0; k < 128; ++k) {
        const int t = group_code<FMT>(grp, k);
        if (t == 0) continue;
        const int64_t kk = static_cast<int64_t>(g) * 128 + k;
#pragma unroll
        for (int i = 0; i < kSimpleMC; ++i) {
          if (i < mc) {
            if constexpr (INT_MODE) {
              iacc[i] += t * static_cast<int>(x[static_cast<int64_t>(m0 + i) * K + kk]);
            } else {
              const float xv = to_f32<TX>(x[static_cast<int64_t>(m0 + i) * K + kk]);
              gf[i] += t > 0 ? xv : -xv;
            }
          }
        }
      }
      if constexpr (!INT_MODE) {
        const float s = __half2float(scales[static_cast<int64_t>(n) * G + g]);
#pragma unroll
        for (int i = 0; i < kSimpleMC; ++i) facc[i] = fmaf(s, gf[i], facc[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < kSimpleMC; ++i) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        facc[i] += __shfl_xor_sync(0xffffffffu, facc[i], o);
        iacc[i] += __shfl_xor_sync(0xffffffffu, iacc[i], o);
      }
    }
    if (lane < mc) {
      float fv = 0.f;
      int iv = 0;
#pragma unroll
      for (int i = 0; i < kSimpleMC; ++i)
        if (i == lane) {
          fv = facc[i];
          iv = iacc[i];
        }
      TOut* out = y + static_cast<int64_t>(m0 + lane) * N + n;
      if constexpr (INT_MODE) {
        *out = iv;
      } else {
        *out = from_f32<TOut>(fv);
      }
    }
  }
}

}  // namespace tb
