// Signed block-Hadamard rotation of activations (fast Walsh-Hadamard
// transform on 1024-blocks) and the activation-prep kernels of the linear
// paths, which fuse the rotation with what each path reads:
//   * prep_gemv: rotate, then per 128-group 16-bit fixed point split into two
//     int8 planes (hi, lo) laid out for dp4a against the packed 2-bit words;
//   * prep_f32 / prep_f16: rotate, then store fp32 (plain kernel) or fp16
//     (tensor-core kernel).
//
// Rotation (news.ditty.ir, Bonsai 2 27B, second and third paragraphs): the
// weights carry W' = W R, R = blockdiag(diag(d_b) H / 32); the run time applies
// x'_b = H (d_b * x_b) / 32.  H is the Sylvester matrix in natural order, which
// is exactly what the in-place radix-2 butterfly below produces.
//
// One CTA of 128 threads per (row, 1024-block): each thread holds 8
// consecutive elements; butterfly distances 1..4 run in registers, 8..128 over
// warp shuffles, 256 and 512 through shared memory.
#pragma once
#include "tb_device.cuh"

namespace tb {

constexpr int kHB = 1024;        // Hadamard block
constexpr int kHThreads = 128;   // threads per block transform
constexpr float kHNorm = 0.03125f;  // 1 / sqrt(1024), exact

template <typename T>
__device__ __forceinline__ void load8(const T* p, float v[8]);
template <>
__device__ __forceinline__ void load8<float>(const float* p, float v[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__half>(const __half* p, float v[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __half22float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float v[8]) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float v[8]);
template <>
__device__ __forceinline__ void store8<float>(float* p, const float v[8]) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
template <>
__device__ __forceinline__ void store8<__half>(__half* p, const float v[8]) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float v[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// load8 for a pointer of unknown alignment: vector load when 16-byte aligned,
// element loads otherwise (the plain kernel accepts any naturally aligned x).
template <typename T>
__device__ __forceinline__ void load8_any(const T* p, float v[8]) {
  if ((reinterpret_cast<uintptr_t>(p) & 15u) == 0) {
    load8<T>(p, v);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = to_f32<T>(p[i]);
  }
}

__device__ __forceinline__ void load_signs8(const int8_t* s, float d[8]) {
  const uint2 u = *reinterpret_cast<const uint2*>(s);
  const int8_t* c = reinterpret_cast<const int8_t*>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) d[i] = static_cast<float>(c[i]);
}

// Unnormalised Walsh-Hadamard transform of one 1024-block held as v[8] per
// thread (thread t owns elements 8t..8t+7) by a group of 128 threads.  Result:
// each thread again owns elements 8t..8t+7 of the transform.  `t` is the
// thread's index in the group (0..127), `bar` a named barrier id private to the
// group (0 when the group is the whole 128-thread block), `sm` 1024 floats of
// shared memory private to the group, free for reuse on return.
__device__ __forceinline__ void fwht1024_group(float v[8], float* sm, int t, int bar) {
  // distances 1, 2, 4: inside the thread
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
  // distances 8 .. 128: partner thread t ^ (h / 8), inside the warp
#pragma unroll
  for (int lm = 1; lm < 32; lm <<= 1) {
    const bool upper = (t & lm) != 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], lm);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
  // distances 256 and 512: across the 4 warps, through shared memory
#pragma unroll
  for (int i = 0; i < 8; ++i) sm[8 * t + i] = v[i];
  asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int j = t + 128 * r;
    const float a = sm[j], b = sm[j + 256], c = sm[j + 512], d = sm[j + 768];
    const float a1 = a + b, b1 = a - b, c1 = c + d, d1 = c - d;
    sm[j] = a1 + c1;
    sm[j + 512] = a1 - c1;
    sm[j + 256] = b1 + d1;
    sm[j + 768] = b1 - d1;
  }
  asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = sm[8 * t + i];
  asm volatile("bar.sync %0, 128;" ::"r"(bar) : "memory");  // sm may be reused after this
}

// fwht1024_group over a whole 128-thread block.
__device__ __forceinline__ void fwht1024(float v[8], float* sm) { fwht1024_group(v, sm, threadIdx.x, 0); }

// Loads the thread's 8 elements of block `blk` of row `row`, applies the
// forward rotation (signs, transform, 1/32) when `signs` is non-null, else
// only converts to fp32.  Called by all 128 threads of a group: `t` is the
// thread's index in the group, `bar` the group's named barrier (see
// fwht1024_group).
template <typename TIn>
__device__ __forceinline__ void load_rotated8_group(const TIn* __restrict__ x, const int8_t* __restrict__ signs,
                                                    int64_t row, int blk, int64_t K, float v[8], float* sm,
                                                    int t, int bar) {
  const int64_t k0 = static_cast<int64_t>(blk) * kHB + 8 * t;
  load8_any<TIn>(x + row * K + k0, v);
  if (signs != nullptr) {
    float d[8];
    load_signs8(signs + k0, d);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= d[i];
    fwht1024_group(v, sm, t, bar);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= kHNorm;
  }
}

// load_rotated8_group over a whole 128-thread block.
template <typename TIn>
__device__ __forceinline__ void load_rotated8(const TIn* __restrict__ x, const int8_t* __restrict__ signs,
                                              int64_t row, int blk, int64_t K, float v[8],
                                              float* sm) {
  load_rotated8_group<TIn>(x, signs, row, blk, K, v, sm, threadIdx.x, 0);
}

// ---------------------------------------------------------------------------
// tb_hadamard_rotate: grid (M, K/1024), 128 threads.
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kHThreads) rotate_kernel(const TIn* x, TOut* y,
                                                           const int8_t* __restrict__ signs,
                                                           int64_t K, int inverse) {
  __shared__ float sm[kHB];
  const int64_t row = blockIdx.x;
  const int blk = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(blk) * kHB + 8 * threadIdx.x;
  float v[8], d[8];
  load8<TIn>(x + row * K + k0, v);
  load_signs8(signs + k0, d);
  if (!inverse) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= d[i];
  }
  fwht1024(v, sm);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] *= kHNorm;
  if (inverse) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= d[i];
  }
  store8<TOut>(y + row * K + k0, v);
}

// ---------------------------------------------------------------------------
// 16-bit fixed point of the rotated activations used by the decode kernels:
// per 128-group e_g = max|x'_g| / kQMax, q = rint(x' / e_g) in [-32512, 32512],
// q = 256 hi + lo with hi = (q + 128) >> 8 in [-127, 127], lo in [-128, 127].
constexpr float kQMax = 32512.0f;

// Rotated (or converted) activations in fp32 / fp16 for the plain and the
// tensor-core kernels: grid (M, K/1024).
template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kHThreads) prep_store_kernel(const TIn* __restrict__ x,
                                                               const int8_t* __restrict__ signs,
                                                               TOut* __restrict__ out, int64_t K) {
  __shared__ float sm[kHB];
  pdl_launch_dependents();
  const int64_t row = blockIdx.x;
  const int blk = blockIdx.y;
  float v[8];
  load_rotated8<TIn>(x, signs, row, blk, K, v, sm);
  store8<TOut>(out + row * K + static_cast<int64_t>(blk) * kHB + 8 * threadIdx.x, v);
}

// Conversion only (no rotation), for K % 1024 != 0: one thread per element.
template <typename TIn, typename TOut>
__global__ void convert_kernel(const TIn* __restrict__ x, TOut* __restrict__ out, int64_t n) {
  pdl_launch_dependents();
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i < n) out[i] = from_f32<TOut>(to_f32<TIn>(x[i]));
}

}  // namespace tb
