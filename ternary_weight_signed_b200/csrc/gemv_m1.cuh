// Decode GEMV for one token (M = 1) on the 2-bit slot format, sized so that
// two CTAs share an SM.
//
// y[n] = sum_g s[n, g] * sum_{k in g} t[n, k] x'[k]   (ternary g128;
// news.ditty.ir, "Bonsai 2 27B", second paragraph; ai4coding.ru, "What is a
// ternary model": the ternary product is an add, a subtract or nothing).
//
// Arithmetic.  x' is held per 128-group as 16-bit fixed point
// q = rint(x' / e_g), e_g = max|x'_g| / 32512.  A packed word w holds 16 codes
// (code 4b + j of the word in bits 8b + 2j); masking it with 0x03030303 << 2j
// leaves the biased codes c = t + 1 of slot j, times 4^j, one per byte.
// dp2a multiplies two of those bytes by two int16 values of q, so
//   T_j = sum over the group's words of 4^j c q   (exact in int32),
//   sum_k t q = T_0 + T_1 / 4 + T_2 / 16 + T_3 / 64 - sum_k q,
// and the group adds s[n, g] * e_g * (that) to row n's fp32 sum.
//
// Activation words of a group (256 bytes, 64 words): word 8 i + 2 j + h holds
// the int16 values of codes 16 i + 8 h + j (low half) and 16 i + 8 h + 4 + j
// (high half): what dp2a.lo (h = 0) and dp2a.hi (h = 1) pair with bytes 0, 1
// and 2, 3 of the slot-j mask of packed word i.  Then per group {e_g, sum q}.
//
// Rotation (news.ditty.ir, second and third paragraphs; openbonsai.org, "How
// it works", "Rotate"): x'_b = H (d_b * x_b) / 32 on each 1024-block, H the
// Sylvester matrix.  One warp rotates one block: lane c first holds elements
// 32 r + c (r = 0..31) and transforms over the high five index bits inside
// the lane; a transpose through shared memory gives lane a the elements
// 32 a .. 32 a + 31, transformed over the low five bits inside the lane, so
// lane a ends with x'[32 a .. 32 a + 31], a quarter of group a / 4.  The 1/32
// is exact and is folded into the fixed-point scale.
//
// Overlap of consecutive calls.  A CTA has 8 warps, at most 128 registers a
// thread and at most 113 KB of shared memory, so the next call's CTA fits on
// the SM beside it.  Every CTA lets its dependents launch at once
// (programmatic dependent launch): the next call's CTA fills its own ring
// with weights while this one computes, and only its activation work waits
// (griddepcontrol.wait) for this call to end.  HBM therefore keeps streaming
// across call boundaries, and a call waits on exactly one kernel boundary.
// Packed weights, scales and signs are read before that wait: they must not
// be written by a kernel that itself lets its dependents launch early.
//
// With `kFused` the CTA rotates x itself (one or two warps per 1024-block): no
// workspace.  Otherwise prep_gemv1_kernel writes the activation words to the
// workspace and one bulk copy brings them.
//
// Work split.  A CTA owns R consecutive rows; a 512-code chunk is 128 bytes of
// each (one TMA box, 128-byte swizzle); stages of NB chunks go through a ring
// of slots (usually all of them at once).  Rows come in tiles of 8: lane l
// works on row 8 t + (l & 7) of a tile and group slot l >> 3 of a chunk, so
// each quarter-warp holds one group's activation words (broadcast loads) and
// its eight lanes read eight rows whose swizzled 16-byte pieces fall in eight
// different bank groups.  Warp w < Wt * Wk owns row-tile group w / Wk (at most
// TPW tiles) and the chunks c = w % Wk (mod Wk), keeps one fp32 sum per tile
// in registers over all of its chunks, and runs two tiles at a time.  At the
// end the four group slots of a row are added by shuffles and the Wk warps of
// a tile group in order of w: the result does not depend on timing (bitwise
// reproducible).
#pragma once
#include "gemv.cuh"
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

// Packed formats this kernel reads (the library's format numbers): 2-bit slots
// (128 bytes of a row per 512-code chunk, 128-byte swizzle) and 1-bit (64
// bytes per chunk, 64-byte swizzle).
constexpr int kG1Fmt2Bit = 0;
constexpr int kG1Fmt1Bit = 2;
__host__ __device__ constexpr uint32_t g1_box_bytes(int fmt) { return fmt == kG1Fmt1Bit ? 64u : 128u; }

constexpr int kG1Warps = 8;
constexpr int kG1Threads = 32 * kG1Warps;
// Shared memory per CTA for two CTAs per SM (228 KB per SM, 1 KB reserved per CTA).
constexpr int kG1SmemMax = 115 * 1024 - 2048;
constexpr int kG1MaxRows = 256;  // TMA box height limit
// The CTA rotates x itself for K up to this many 1024-blocks (one per warp);
// longer K goes through prep_gemv1_kernel.
constexpr int kG1FusedMaxBlocks = kG1Warps;
constexpr int kG1GroupBytes = 256;
// Groups sit 272 bytes apart in shared memory: the four groups of a chunk,
// read together by the four quarter-warps, then start in four different
// 16-byte bank groups and one load serves all four in a single pass.
constexpr int kG1GroupStride = kG1GroupBytes + 16;
// A block's 8 groups of words double as its warp's 2 KB transpose buffer.
static_assert(8 * kG1GroupStride >= 512 * 4, "transpose buffer");

// d = c + a.lo16 * b.byte0 + a.hi16 * b.byte1 (lo) or * bytes 2, 3 (hi);
// a signed 16-bit, b unsigned 8-bit.
__device__ __forceinline__ int dp2a_lo(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ int dp2a_hi(uint32_t a, uint32_t b, int c) {
  int d;
  asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

struct Gemv1Params {
  const void* x;           // [K] activations (fused) or nullptr
  const int8_t* signs;     // [K] or nullptr (x already rotated)
  const uint8_t* act;      // prep_gemv1_kernel output (not fused)
  const uint16_t* scales;  // [N, K/128] fp16 bits
  void* y;                 // [N]
  int N, K;
  int R;                   // rows per CTA (TMA box height)
  int RT;                  // row tiles of 8 covering R
  int Wt, Wk;              // row-tile groups x chunk classes <= kG1Warps
  int NB, nb_log2;         // chunks (boxes) per stage, a power of two
  int nstage, nslots;
  int box_stride;          // bytes between boxes (R * 128 rounded up to 1 KB)
  int slot_bytes;          // NB * box_stride
  int off_act, off_sc, off_red, off_bar;  // shared-memory offsets from the 1 KB-aligned base
};

// Shared memory (offsets from the 1 KB-aligned base; 1 KB of slack in front):
//   ring  nslots x slot_bytes
//   act   G x 272 bytes (256 of activation words, 16 of padding), then G x
//         {float e_g, int sum q}
//   sc    R x G fp16 scales of the CTA's rows
//   red   Wk x R fp32 row sums of the warps (before that, the exchange
//         buffer of the two-warp rotation: 4 KB per 1024-block)
//   bar   full[nstage], pre_bar; counters done[nstage], issued[nstage], fault
struct Gemv1Layout {
  int off_act, off_sc, off_red, off_bar;
  int64_t bytes;
};
__host__ __device__ inline int64_t g1_act_bytes(int64_t K) { return (K / 128) * (kG1GroupStride + 8); }
// Two warps rotate each 1024-block when there are warps enough for that.
__host__ __device__ constexpr bool g1_half_blocks(int64_t K) { return 2 * (K / 1024) <= kG1Warps; }
__host__ __device__ inline Gemv1Layout gemv1_layout(int64_t K, int R, int Wk, int nstage, int64_t ring_bytes) {
  const int64_t G = K / 128;
  Gemv1Layout l;
  l.off_act = static_cast<int>(ring_bytes);
  l.off_sc = static_cast<int>(l.off_act + align128(g1_act_bytes(K)));
  l.off_red = static_cast<int>(l.off_sc + align128(static_cast<int64_t>(R) * G * 2));
  int64_t red = static_cast<int64_t>(Wk) * R * 4;
  if (g1_half_blocks(K) && red < (K / 1024) * 4096) red = (K / 1024) * 4096;
  l.off_bar = static_cast<int>(l.off_red + align128(red));
  l.bytes = 1024 + l.off_bar + 8 * (nstage + 1) + 4 * (2 * nstage + 1);
  return l;
}

// ---------------------------------------------------------------- rotation
template <typename T>
__device__ __forceinline__ void g1_load32(const T* p, float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) load8<T>(p + 8 * i, v + 8 * i);
}

// Radix-2 butterflies over the five index bits held in the lane (v[i], i the
// bits): after it v holds the 32-point Sylvester transform of the input.
__device__ __forceinline__ void g1_fwht32(float (&v)[32]) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
  }
}

// One warp: rotate 1024-block `blk` (with the block's 1024 signs `sgn`, in
// shared or global memory, when not null; else x is taken as already rotated)
// and write its 8 groups' activation words and info into `act` (G groups of
// words, then G infos).  When `sbar` is not null the signs arrive by a bulk
// copy completing on it.  `xbuf` is 2 KB of shared memory of this warp's own
// (16 rows of 32 floats); it may overlap the signs.  False if the wait for
// the signs gave up.
//
// With index k = 32 r + c, H_1024 = H_32 (x) H_32: lane c loads x[32 r + c]
// for r = 0..31 (each load instruction reads 32 consecutive elements) and
// transforms over r inside the lane; the 32 x 32 tile is transposed through
// xbuf (two halves of 16 rows; the 16-byte column chunks XOR-swizzled by the
// row, so neither the 4-byte stores of a row nor the 16-byte loads of a
// quarter-warp meet a bank twice); lane r then holds the 32 values of row r
// and transforms over c.  Lane a ends with x'[32 a .. 32 a + 31].
template <typename TIn, int kFmt>
__device__ __forceinline__ bool g1_rotate_block(const TIn* __restrict__ x, const int8_t* sgn, uint64_t* sbar,
                                                int blk, int G, uint8_t* act, float* xbuf, int lane) {
  const TIn* xb = x + static_cast<int64_t>(blk) * kHB;
  float v[32];
  float scale = 1.f;
  if (sgn != nullptr) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = to_f32<TIn>(xb[32 * i + lane]);
    // signs staged in shared memory by a bulk copy: wait for it while the
    // loads of x are in flight
    if (sbar != nullptr && !__all_sync(0xffffffffu, mbar_wait(sbar, 0, FAULT_WAIT_ACT))) return false;
    // sign byte -1 (0xFF) flips the float's sign bit
#pragma unroll
    for (int i = 0; i < 32; ++i)
      v[i] = __int_as_float(__float_as_int(v[i]) ^ (static_cast<int32_t>(sgn[32 * i + lane]) & INT32_MIN));
    __syncwarp();  // the signs may share memory with xbuf
    g1_fwht32(v);
    float u[32];
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int r = 0; r < 16; ++r) xbuf[32 * r + ((((lane >> 2) ^ r) & 7) << 2) + (lane & 3)] = v[16 * hf + r];
      __syncwarp();
      if ((lane >> 4) == hf) {
        const float4* row = reinterpret_cast<const float4*>(xbuf + 32 * (lane & 15));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 t = row[q ^ (lane & 7)];
          u[4 * q] = t.x;
          u[4 * q + 1] = t.y;
          u[4 * q + 2] = t.z;
          u[4 * q + 3] = t.w;
        }
      }
      __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = u[i];
    g1_fwht32(v);
    scale = kHNorm;
  } else {
    g1_load32<TIn>(xb + 32 * lane, v);
  }
  // 16-bit fixed point of the group (4 lanes): e = max|x'| / kQMax with x' = scale * v
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(v[i]));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  mx *= scale;  // exact (a power of two)
  const float e = mx / kQMax;
  // inv * scale is exact too, so q = rint(x' * kQMax / max|x'|) as in
  // prep_gemv_kernel.  The rounding adds 1.5 * 2^23: for |f| <= kQMax the sum's
  // bits are 0x4B400000 + rint(f) (round to nearest even), so their low 16
  // bits are q as int16.
  const float inv = mx > 0.f ? (kQMax / mx) * scale : 0.f;
  uint32_t qb[32];
  uint32_t qsb = 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float f = fminf(fmaxf(__fmul_rn(v[i], inv), -kQMax), kQMax);
    qb[i] = __float_as_uint(__fadd_rn(f, 12582912.0f));
    qsb += qb[i];
  }
  int qs = static_cast<int>(qsb - 32u * 0x4B400000u);
  qs += __shfl_xor_sync(0xffffffffu, qs, 1);
  qs += __shfl_xor_sync(0xffffffffu, qs, 2);
  uint32_t wv[16];
  if constexpr (kFmt == kG1Fmt2Bit) {
    // lane a holds codes 32 (a & 3) .. + 31 of group a >> 2, i.e. packed
    // words i = 2 (a & 3) + i2 (i2 = 0, 1); word 8 i + 2 j + h pairs codes
    // 16 i + 8 h + j and 16 i + 8 h + 4 + j
#pragma unroll
    for (int i2 = 0; i2 < 2; ++i2)
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int u = 16 * i2 + 8 * h + j;
          wv[8 * i2 + 2 * j + h] = __byte_perm(qb[u], qb[u + 4], 0x5410);
        }
  } else {
    // 1-bit: lane a holds the 32 codes of packed word i = a & 3 of group
    // a >> 2; word 16 i + 2 j + h pairs codes 32 i + 16 h + j and
    // 32 i + 16 h + 8 + j
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int u = 16 * h + j;
        wv[2 * j + h] = __byte_perm(qb[u], qb[u + 8], 0x5410);
      }
  }
  const int g = blk * 8 + (lane >> 2);
  uint4* dst = reinterpret_cast<uint4*>(act + g * kG1GroupStride + 64 * (lane & 3));
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(wv[4 * i], wv[4 * i + 1], wv[4 * i + 2], wv[4 * i + 3]);
  if ((lane & 3) == 0) {
    int2 inf;
    inf.x = __float_as_int(e);
    inf.y = qs;
    reinterpret_cast<int2*>(act + G * kG1GroupStride)[g] = inf;
  }
  return true;
}

// Two warps, halves hf = 0, 1 of 1024-block `blk`: lane l of half hf holds
// elements 512 hf + 16 l .. + 15.  Index bits 0-3 are transformed inside the
// lane, bits 4-8 across lanes, bit 9 across the two warps through `xch` (1024
// floats of the pair's own; named barrier `bar`, 64 threads).  Then each
// lane's 16 codes are word (l & 7) of group 8 blk + 4 hf + l / 8.
template <typename TIn, int kFmt>
__device__ __forceinline__ void g1_rotate_half(const TIn* __restrict__ x, const int8_t* __restrict__ signs,
                                               int blk, int hf, int G, uint8_t* act, float* xch, int bar, int lane) {
  const int64_t e0 = static_cast<int64_t>(blk) * kHB + 512 * hf + 16 * lane;
  float v[16];
  load8<TIn>(x + e0, v);
  load8<TIn>(x + e0 + 8, v + 8);
  float scale = 1.f;
  if (signs != nullptr) {
    const uint4 sg = *reinterpret_cast<const uint4*>(signs + e0);
    const uint32_t sw[4] = {sg.x, sg.y, sg.z, sg.w};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t sbit = (sw[i >> 2] << (24 - 8 * (i & 3))) & 0x80000000u;
      v[i] = __int_as_float(__float_as_int(v[i]) ^ static_cast<int>(sbit));
    }
#pragma unroll
    for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], b = v[i + h];
          v[i] = a + b;
          v[i + h] = a - b;
        }
      }
    }
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
      const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] = fmaf(sgn, v[i], __shfl_xor_sync(0xffffffffu, v[i], m));
    }
    float4* mine = reinterpret_cast<float4*>(xch + 512 * hf + 16 * lane);
#pragma unroll
    for (int i = 0; i < 4; ++i) mine[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
    const float4* other = reinterpret_cast<const float4*>(xch + 512 * (1 - hf) + 16 * lane);
    const float sgn = hf ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 o = other[i];
      v[4 * i] = fmaf(sgn, v[4 * i], o.x);
      v[4 * i + 1] = fmaf(sgn, v[4 * i + 1], o.y);
      v[4 * i + 2] = fmaf(sgn, v[4 * i + 2], o.z);
      v[4 * i + 3] = fmaf(sgn, v[4 * i + 3], o.w);
    }
    scale = kHNorm;
  }
  // 16-bit fixed point of the group (8 lanes)
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  mx *= scale;
  const float e = mx / kQMax;
  const float inv = mx > 0.f ? (kQMax / mx) * scale : 0.f;
  int q[16];
  int qs = 0;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    q[i] = max(-32512, min(32512, __float2int_rn(v[i] * inv)));
    qs += q[i];
  }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
  const int g = blk * 8 + 4 * hf + (lane >> 3);
  if constexpr (kFmt == kG1Fmt2Bit) {
    // the lane's 16 codes are packed word l & 7 of the group
    uint32_t wv[8];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h)
        wv[2 * j + h] =
            __byte_perm(static_cast<uint32_t>(q[8 * h + j]), static_cast<uint32_t>(q[8 * h + j + 4]), 0x5410);
    uint4* dst = reinterpret_cast<uint4*>(act + g * kG1GroupStride + 32 * (lane & 7));
    dst[0] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
    dst[1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
  } else {
    // 1-bit: the lane's 16 codes are half hh = l & 1 of packed word
    // i = (l & 7) / 2, i.e. the words 16 i + 2 j + hh (j = 0..7)
    const int i = (lane & 7) >> 1, hh = lane & 1;
    uint32_t* dst = reinterpret_cast<uint32_t*>(act + g * kG1GroupStride) + 16 * i + hh;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      dst[2 * j] = __byte_perm(static_cast<uint32_t>(q[j]), static_cast<uint32_t>(q[j + 8]), 0x5410);
  }
  if ((lane & 7) == 0) {
    int2 inf;
    inf.x = __float_as_int(e);
    inf.y = qs;
    reinterpret_cast<int2*>(act + G * kG1GroupStride)[g] = inf;
  }
}

// Activation words for long K: one warp per 1024-block, 4 warps per CTA,
// written to `ws` in the layout above.  Waits for the previous kernel on the
// stream (which may have produced x, or may still read ws) before touching
// either.
template <typename TIn, int kFmt>
__global__ void __launch_bounds__(128) prep_gemv1_kernel(const TIn* __restrict__ x, const int8_t* __restrict__ signs,
                                                         uint8_t* __restrict__ ws, int K) {
  __shared__ __align__(16) float xbuf[4][512];
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int blk = blockIdx.x * 4 + (threadIdx.x >> 5);
  const bool live = blk < (K >> 10);
  pdl_wait();
  if (live)
    g1_rotate_block<TIn, kFmt>(x, signs != nullptr ? signs + static_cast<int64_t>(blk) * kHB : nullptr, nullptr,
                               blk, K >> 7, ws, xbuf[threadIdx.x >> 5], lane);
}

// ---------------------------------------------------------------- decode
// Stage s: its chunks' weight boxes into slot `slot`, completing on `bar`.
template <int kFmt>
__device__ __forceinline__ void gemv1_issue(const CUtensorMap* tm, const Gemv1Params& p, uint8_t* ring,
                                            uint64_t* bar, int s, int slot, int r0) {
  constexpr uint32_t kBox = g1_box_bytes(kFmt);
  const int C = p.K >> 9;
  const int nb = min(p.NB, C - s * p.NB);
  uint8_t* dst = ring + static_cast<int64_t>(slot) * p.slot_bytes;
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nb) * static_cast<uint32_t>(p.R) * kBox);
  const uint64_t pol = l2_policy_evict_first();  // weights are read once per call
  for (int b = 0; b < nb; ++b)
    tma_load_2d_hint(dst + b * p.box_stride, tm, (s * p.NB + b) * static_cast<int>(kBox), r0, bar, pol);
}

// sum_k c_k q_k of one row's group: 8 packed words against the group's 64
// activation words (the four T_j combined exactly).
// One accumulator per slot j (words i = 0..3 and 4..7 in two halves so that
// each chain is 8 deep); |T_j| <= 16 * 2 * 32512 * 128 < 2^31.
__device__ __forceinline__ int g1_group_dot(const uint4& wa, const uint4& wb, const uint32_t (&A)[64]) {
  const uint32_t w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
  int t[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = w[i] & (0x03030303u << (2 * j));
      int& acc = t[i >> 2][j];
      acc = dp2a_lo(A[8 * i + 2 * j], c, acc);
      acc = dp2a_hi(A[8 * i + 2 * j + 1], c, acc);
    }
  }
  return (t[0][0] + t[1][0]) + ((t[0][1] + t[1][1]) >> 2) + ((t[0][2] + t[1][2]) >> 4) +
         ((t[0][3] + t[1][3]) >> 6);
}

// 1-bit: sum_k (t_k + 1) q_k = 2 sum_k b_k q_k of one row's group, b the bit
// of code k: 4 packed words of 32 codes against the group's 64 activation
// words.  Masking a word with 0x01010101 << j leaves bit j of each byte, i.e.
// 2^j b of codes 8 c + j (c = 0..3), so dp2a.lo / dp2a.hi pair bytes 0, 1 /
// 2, 3 with the words 16 i + 2 j + h; T_j is exact in int32 and
// 2 sum b q = sum_j T_j / 2^(j - 1).  |T_j| <= 8 * 2 * 128 * 32512 < 2^31.
__device__ __forceinline__ int g1_group_dot_1bit(const uint4& w4, const uint32_t (&A)[64]) {
  const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
  int t[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t c = w[i] & (0x01010101u << j);
      t[j] = dp2a_lo(A[16 * i + 2 * j], c, t[j]);
      t[j] = dp2a_hi(A[16 * i + 2 * j + 1], c, t[j]);
    }
  }
  return (t[0] << 1) + t[1] + (t[2] >> 1) + (t[3] >> 2) + (t[4] >> 3) + (t[5] >> 4) + (t[6] >> 5) + (t[7] >> 6);
}

// sum_k (t_k + 1) q_k of one row's group from the lane's piece of the box.
template <int kFmt>
__device__ __forceinline__ int g1_dot(const uint8_t* box, int pa, const uint32_t (&A)[64]) {
  if constexpr (kFmt == kG1Fmt2Bit) {
    const uint4 w0 = *reinterpret_cast<const uint4*>(box + pa);
    const uint4 w1 = *reinterpret_cast<const uint4*>(box + (pa ^ 16));
    return g1_group_dot(w0, w1, A);
  } else {
    return g1_group_dot_1bit(*reinterpret_cast<const uint4*>(box + pa), A);
  }
}

// TPW: row tiles per warp at most (1, 2 or 4).
template <typename TIn, typename TOut, bool kFused, int TPW, int kFmt>
__global__ void __launch_bounds__(kG1Threads, 2)
    gemv1_kernel(const __grid_constant__ CUtensorMap tm_w, const Gemv1Params p) {
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* ring = base;
  uint8_t* act = base + p.off_act;
  const __half* sc = reinterpret_cast<const __half*>(base + p.off_sc);
  float* red = reinterpret_cast<float*>(base + p.off_red);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + p.off_bar);
  uint64_t* pre_bar = full + p.nstage;  // scales (+ activation words when not fused)
  uint32_t* done = reinterpret_cast<uint32_t*>(pre_bar + 1);  // warps finished with stage s
  uint32_t* issued = done + p.nstage;                          // 1 once stage s was issued
  uint32_t* cta_fault = issued + p.nstage;

  const int G = p.K >> 7, C = p.K >> 9;
  const int r0 = blockIdx.x * p.R;
  const int nrows = min(p.R, p.N - r0);
  const int pre = min(p.nslots, p.nstage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const bool stall = test_stall_copies();  // failure-detection test: no weight copies
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_w);
    for (int s = 0; s < p.nstage; ++s) {
      mbar_init(&full[s], 1);
      done[s] = 0;
      issued[s] = s < pre && !stall ? 1u : 0u;
    }
    *cta_fault = 0;
    mbar_init(pre_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  // The weights do not depend on earlier work on the stream.  Issuing a TMA
  // copy takes a while, so the stages are spread over the warps' lane 0 (the
  // last warps first: the first warps rotate x).
  if (lane == 0) {
    if (warp == kG1Warps - 1) {
      const uint32_t sbytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(G * 2);
      const uint32_t abytes = kFused ? 0u : static_cast<uint32_t>(g1_act_bytes(p.K));
      // one warp per block: the block's signs go to the start of its slice of
      // the activation words
      const bool stage_signs = kFused && p.signs != nullptr && !g1_half_blocks(p.K);
      const uint32_t gbytes = stage_signs ? static_cast<uint32_t>(p.K) : 0u;
      mbar_arrive_expect_tx(pre_bar, sbytes + abytes + gbytes);
      bulk_load(base + p.off_sc, p.scales + static_cast<int64_t>(r0) * G, sbytes, pre_bar);
      if (stage_signs)
        for (int b = 0; b < (p.K >> 10); ++b)
          bulk_load(act + b * 8 * kG1GroupStride, p.signs + static_cast<int64_t>(b) * kHB, kHB, pre_bar);
    }
    for (int s = kG1Warps - 1 - warp; s < pre && !stall; s += kG1Warps)
      gemv1_issue<kFmt>(&tm_w, p, ring, &full[s], s, s, r0);
    if constexpr (!kFused) {
      if (warp == kG1Warps - 1) {
        pdl_wait();  // the prep kernel's activation words
        bulk_load(act, p.act, static_cast<uint32_t>(g1_act_bytes(p.K)), pre_bar);
      }
    }
  }
  if constexpr (kFused) {
    const int nblk = p.K >> 10;
    const TIn* x = static_cast<const TIn*>(p.x);
    if (g1_half_blocks(p.K)) {
      pdl_wait();  // x may be the previous kernel's output
      if (warp < 2 * nblk)
        g1_rotate_half<TIn, kFmt>(x, p.signs, warp >> 1, warp & 1, G, act, red + (warp >> 1) * kHB, 1 + (warp >> 1),
                                  lane);
    } else {
      // block `warp` (K <= kG1FusedMaxBlocks blocks); its signs were staged
      // in shared memory before the wait
      const bool live = warp < nblk;
      pdl_wait();  // x may be the previous kernel's output
      // the transpose buffer is this block's own slice of the activation words
      // (8 x 272 bytes, written only after the transpose)
      uint8_t* slice = act + warp * 8 * kG1GroupStride;
      if (live &&
          !g1_rotate_block<TIn, kFmt>(x, p.signs != nullptr ? reinterpret_cast<const int8_t*>(slice) : nullptr,
                                      pre_bar, warp, G, act, reinterpret_cast<float*>(slice), lane) &&
          lane == 0)
        atomicExch(cta_fault, 1u);
    }
  }
  __syncthreads();

  const int rsub = lane & 7, gslot = lane >> 3;
  const int tg = warp / p.Wk, wk = warp - tg * p.Wk;
  const bool active = tg < p.Wt;
  const int t0 = tg * p.RT / p.Wt, nt = active ? (tg + 1) * p.RT / p.Wt - t0 : 0;  // this warp's row tiles
  const int2* info = reinterpret_cast<const int2*>(act + G * kG1GroupStride);
  // byte offsets in a box of the lane's 16-byte pieces and of the rows'
  // scales.  2-bit: pieces 2 gslot and 2 gslot + 1 of the row's 128 bytes,
  // 128-byte swizzle (piece index XOR row mod 8 = rsub).  1-bit: piece gslot
  // of the row's 64 bytes, 64-byte swizzle (piece index XOR (row / 2) mod 4 =
  // rsub / 2).  Either way the eight rows of a quarter-warp land in eight
  // different 16-byte bank groups.  Rows past the CTA's end read valid rows
  // and their sums are dropped.
  constexpr int kBox = static_cast<int>(g1_box_bytes(kFmt));
  const int u0 = kFmt == kG1Fmt2Bit ? ((2 * gslot) ^ rsub) << 4 : (gslot ^ (rsub >> 1)) << 4;
  int pa[TPW], soff[TPW];
  float acc[TPW];
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const int r = 8 * (t0 + i) + rsub;
    pa[i] = min(r, p.R - 1) * kBox + u0;
    soff[i] = min(r, nrows - 1) * G;
    acc[i] = 0.f;
  }
  const bool refill = p.nslots < p.nstage;

  bool ok = __all_sync(0xffffffffu, mbar_wait_backoff(pre_bar, 0, FAULT_WAIT_ACT));
  int cur_s = -1;
  const uint8_t* sbase = ring;  // slot of the current stage
  for (int c = active && ok ? wk : C; c < C; c += p.Wk) {
    const int s = c >> p.nb_log2;
    if (s != cur_s) {
      ok = __all_sync(0xffffffffu, mbar_wait_backoff(&full[s], 0, FAULT_WAIT_FULL)) &&
           *reinterpret_cast<volatile uint32_t*>(cta_fault) == 0u;
      if (!ok) break;
      cur_s = s;
      sbase = ring + static_cast<int64_t>(s % p.nslots) * p.slot_bytes;
    }
    const uint8_t* box = sbase + (c - (s << p.nb_log2)) * p.box_stride;
    const int g = 4 * c + gslot;
    uint32_t A[64];
    const uint4* src = reinterpret_cast<const uint4*>(act + g * kG1GroupStride);
#pragma unroll
    for (int v = 0; v < 16; ++v) {
      const uint4 u4 = src[v];
      A[4 * v] = u4.x;
      A[4 * v + 1] = u4.y;
      A[4 * v + 2] = u4.z;
      A[4 * v + 3] = u4.w;
    }
    const int2 inf = info[g];
    const float e = __int_as_float(inf.x);
    if constexpr (TPW == 1) {
      const float sa = __half2float(sc[soff[0] + g]) * e;
      acc[0] = fmaf(__int2float_rn(g1_dot<kFmt>(box, pa[0], A) - inf.y), sa, acc[0]);
    } else {
#pragma unroll
      for (int tp = 0; tp < TPW; tp += 2) {
        // tiles beyond nt compute on valid rows and are dropped at the end
        const float sa = __half2float(sc[soff[tp] + g]) * e;
        const float sb = __half2float(sc[soff[tp + 1] + g]) * e;
        const int da = g1_dot<kFmt>(box, pa[tp], A) - inf.y;
        const int db = g1_dot<kFmt>(box, pa[tp + 1], A) - inf.y;
        acc[tp] = fmaf(__int2float_rn(da), sa, acc[tp]);
        acc[tp + 1] = fmaf(__int2float_rn(db), sb, acc[tp + 1]);
      }
    }
    if (refill) {
      // a stage's chunks are each used by Wt warps; the last use refills the
      // slot with the stage nslots ahead
      __syncwarp();
      if (lane == 0) {
        __threadfence_block();
        const int nch = min(p.NB, C - (s << p.nb_log2));
        if (atomicAdd(&done[s], 1u) == static_cast<uint32_t>(nch * p.Wt - 1) && s + p.nslots < p.nstage) {
          __threadfence_block();
          issued[s + p.nslots] = 1u;
          gemv1_issue<kFmt>(&tm_w, p, ring, &full[s + p.nslots], s + p.nslots, s % p.nslots, r0);
        }
      }
    }
  }
  if (!ok && lane == 0) atomicExch(cta_fault, 1u);  // the other warps stop at their next stage
  // row sums of this warp: the chunk's four group slots (lanes rsub + 8 k)
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    float v = acc[i];
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    const int r = 8 * (t0 + i) + rsub;
    if (i < nt && gslot == 0 && r < p.R) red[wk * p.R + r] = v;
  }
  __syncthreads();
  // After a wait that gave up, copies may still be in flight into the ring:
  // wait (bounded) for every issued stage before the CTA exits.
  if (threadIdx.x == 0 && *cta_fault != 0) {
    for (int s = 0; s < p.nstage; ++s)
      if (issued[s] && !mbar_wait(&full[s], 0, FAULT_WAIT_FULL)) break;
  }
  TOut* y = reinterpret_cast<TOut*>(p.y);
  for (int r = threadIdx.x; r < nrows; r += kG1Threads) {
    float sum = 0.f;
    for (int k = 0; k < p.Wk; ++k) sum += red[k * p.R + r];
    y[r0 + r] = from_f32<TOut>(sum);
  }
}

}  // namespace tb
