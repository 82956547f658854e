// Pack / unpack kernels for the packed formats (byte layouts in
// include/ternary_b200.h).  Elementwise, memory-bound, one thread per output
// word (2-bit) or per 128-group (base-3).  Bit-exact by construction; invalid
// input is counted, never trapped.
#pragma once
#include "tb_device.cuh"

namespace tb {

__device__ __forceinline__ void count_invalid(uint32_t bad, uint32_t* counter) {
  if (counter == nullptr) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) bad += __shfl_xor_sync(0xffffffffu, bad, o);
  if ((threadIdx.x & 31) == 0 && bad) atomicAdd(counter, bad);
}

// Biased code c = t + 1 for a valid t, else 1 (t = 0); *bad counts invalids.
__device__ __forceinline__ uint32_t biased_code(int t, uint32_t* bad) {
  const bool ok = (t >= -1) && (t <= 1);
  *bad += ok ? 0u : 1u;
  return ok ? static_cast<uint32_t>(t + 1) : 1u;
}

// One thread per 16 codes -> one 32-bit word (4 packed bytes).
__global__ void pack_2bit_kernel(const int4* __restrict__ codes, uint32_t* __restrict__ out,
                                 int64_t nwords, uint32_t* counter) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t bad = 0;
  if (i < nwords) {
    const int4 v = codes[i];
    const int8_t* c = reinterpret_cast<const int8_t*>(&v);
    uint32_t w = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) w |= biased_code(c[j], &bad) << (2 * j);
    out[i] = w;
  }
  count_invalid(bad, counter);
}

__global__ void unpack_2bit_kernel(const uint32_t* __restrict__ in, int4* __restrict__ codes,
                                   int64_t nwords, uint32_t* counter) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t bad = 0;
  if (i < nwords) {
    const uint32_t w = in[i];
    int4 v;
    int8_t* c = reinterpret_cast<int8_t*>(&v);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const uint32_t s = (w >> (2 * j)) & 3u;
      bad += (s == 3u);
      c[j] = (s == 3u) ? int8_t(0) : static_cast<int8_t>(static_cast<int>(s) - 1);
    }
    codes[i] = v;
  }
  count_invalid(bad, counter);
}

// One thread per 128-group: 128 codes in, 26 bytes out (13 16-bit stores; a
// group starts at an even byte offset).
__global__ void pack_base3_kernel(const int4* __restrict__ codes, uint16_t* __restrict__ out,
                                  int64_t ngroups, uint32_t* counter) {
  const int64_t gi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t bad = 0;
  if (gi < ngroups) {
    uint32_t c[130];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int4 v = codes[gi * 8 + q];
      const int8_t* t = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
      for (int j = 0; j < 16; ++j) c[16 * q + j] = biased_code(t[j], &bad);
    }
    c[128] = 1u;  // padding digits of the last byte
    c[129] = 1u;
    uint16_t* o = out + gi * 13;
#pragma unroll
    for (int h = 0; h < 13; ++h) {
      uint32_t b[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t* d = c + 5 * (2 * h + e);
        b[e] = d[0] + 3u * d[1] + 9u * d[2] + 27u * d[3] + 81u * d[4];
      }
      o[h] = static_cast<uint16_t>(b[0] | (b[1] << 8));
    }
  }
  count_invalid(bad, counter);
}

__global__ void unpack_base3_kernel(const uint16_t* __restrict__ in, int4* __restrict__ codes,
                                    int64_t ngroups, uint32_t* counter) {
  const int64_t gi = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t bad = 0;
  if (gi < ngroups) {
    int8_t t[130];
    const uint16_t* p = in + gi * 13;
#pragma unroll
    for (int h = 0; h < 13; ++h) {
      const uint32_t pair = p[h];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int byte_idx = 2 * h + e;
        uint32_t v = (pair >> (8 * e)) & 0xffu;
        uint32_t dig[5];
#pragma unroll
        for (int j = 0; j < 5; ++j) {
          dig[j] = v % 3u;
          v /= 3u;
        }
        const uint32_t raw = (pair >> (8 * e)) & 0xffu;
        bool invalid = raw >= 243u;
        if (byte_idx == 25) invalid = invalid || dig[3] != 1u || dig[4] != 1u;
        bad += invalid ? 1u : 0u;
#pragma unroll
        for (int j = 0; j < 5; ++j)
          t[5 * byte_idx + j] = invalid ? int8_t(0) : static_cast<int8_t>(static_cast<int>(dig[j]) - 1);
      }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      int4 v;
      int8_t* o = reinterpret_cast<int8_t*>(&v);
#pragma unroll
      for (int j = 0; j < 16; ++j) o[j] = t[16 * q + j];
      codes[gi * 8 + q] = v;
    }
  }
  count_invalid(bad, counter);
}

// 1-bit g128 (each weight -1 or +1; dev.to, "How Prism ML Squeezed a 27B
// Model Into 3.9 GB", the two formats that ship): weight k of a row in bit
// k % 8 of byte k / 8, bit 1 = +1.  One thread per 32 codes -> one 32-bit word
// (code u of the word in bit u).  Any code other than -1 and +1 (0 included)
// is packed as -1 and counted.
__global__ void pack_1bit_kernel(const int4* __restrict__ codes, uint32_t* __restrict__ out, int64_t nwords,
                                 uint32_t* counter) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  uint32_t bad = 0;
  if (i < nwords) {
    uint32_t w = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int4 v = codes[2 * i + h];
      const int8_t* c = reinterpret_cast<const int8_t*>(&v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        bad += (c[j] != 1 && c[j] != -1) ? 1u : 0u;
        w |= (c[j] == 1 ? 1u : 0u) << (16 * h + j);
      }
    }
    out[i] = w;
  }
  count_invalid(bad, counter);
}

// Every bit pattern is valid: bit 1 -> +1, bit 0 -> -1.
__global__ void unpack_1bit_kernel(const uint32_t* __restrict__ in, int4* __restrict__ codes, int64_t nwords) {
  const int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (i < nwords) {
    const uint32_t w = in[i];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int4 v;
      int8_t* c = reinterpret_cast<int8_t*>(&v);
#pragma unroll
      for (int j = 0; j < 16; ++j) c[j] = ((w >> (16 * h + j)) & 1u) ? int8_t(1) : int8_t(-1);
      codes[2 * i + h] = v;
    }
  }
}

// Base-3 groups (26 bytes) -> 2-bit slot groups (32 bytes): the 2-bit paths
// (prefill GEMM, tensor-core decode) consume the 2-bit layout, so a base-3
// matrix is re-encoded into the caller's workspace first.  A warp copies its
// 32 groups' bytes into shared memory with coalesced loads; then each lane
// decodes one group through a 243-entry table (byte value -> its five digits,
// which are the biased codes, as five 2-bit fields) and places each byte's ten
// bits at bit 10 i of the group's 256-bit slot string.  Invalid bytes decode
// as t = 0 (as tb_unpack_ternary does; the linear paths leave their output
// unspecified).  256 threads per block, 256 groups per block.
__global__ void __launch_bounds__(256) transcode_b3_to_2bit_kernel(const uint8_t* __restrict__ in,
                                                                   uint4* __restrict__ out, int64_t ngroups) {
  __shared__ uint16_t lut[256];
  __shared__ __align__(16) uint8_t buf[8][32 * 26];
  {
    const uint32_t i = threadIdx.x;
    uint32_t code = 0x155u;  // five codes 1 (t = 0)
    if (i < 243u) {
      uint32_t v = i;
      code = 0;
#pragma unroll
      for (int j = 0; j < 5; ++j) {
        code |= (v % 3u) << (2 * j);
        v /= 3u;
      }
    }
    lut[i] = static_cast<uint16_t>(code);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g0 = (static_cast<int64_t>(blockIdx.x) * 8 + warp) * 32;
  const int64_t left = ngroups - g0;
  const int ng = left <= 0 ? 0 : (left < 32 ? static_cast<int>(left) : 32);
  // even; the source is 4-byte aligned: the paths that re-encode need 16-byte
  // aligned packed weights, and a warp starts at byte 26 * 32 * k
  const int nbytes = 26 * ng;
  const uint8_t* src = in + 26 * g0;
  uint8_t* b = buf[warp];
  for (int w = lane; w < nbytes / 4; w += 32)
    reinterpret_cast<uint32_t*>(b)[w] = reinterpret_cast<const uint32_t*>(src)[w];
  if ((nbytes & 3) != 0 && lane == 0)
    *reinterpret_cast<uint16_t*>(b + nbytes - 2) = *reinterpret_cast<const uint16_t*>(src + nbytes - 2);
  __syncwarp();
  if (lane < ng) {
    const uint8_t* gb = b + 26 * lane;
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 26; ++i) {
      const uint32_t v = gb[i];
      uint32_t code;
      if (i < 25) {
        code = lut[v];
      } else {
        // k = 125..127 in digits 0-2; digits 3 and 4 must be the padding value 1
        code = (v >= 108u && v < 135u) ? (lut[v] & 0x3Fu) : 0x15u;
      }
      const int pos = 10 * i;
      w[pos >> 5] |= code << (pos & 31);
      if (i < 25 && (pos & 31) > 22) w[(pos >> 5) + 1] |= code >> (32 - (pos & 31));
    }
    out[2 * (g0 + lane)] = make_uint4(w[0], w[1], w[2], w[3]);
    out[2 * (g0 + lane) + 1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

}  // namespace tb
