// Decode GEMV for small M (1 to 4 tokens) on the base-3 format (5 trits per
// byte; every 128-group is its own 26-byte run: bytes 0..24 hold codes
// 5i..5i+4 as sum_j c_j 3^j, byte 25 holds codes 125..127 and two padding
// digits 1).  The pages name a dense trit packing for the CUDA GGUF files
// (news.ditty.ir, paragraph on the CUDA files); this layout is the library's
// own definition of it.
//
// Same arithmetic as the 2-bit kernel (gemv.cuh): x' as 16-bit fixed point
// per 128-group in two int8 planes, biased codes c = t + 1 as bytes, exact
// int32 dot products with dp4a, one fp32 scale multiply per group and row.
// What changes is how a packed byte b becomes dp4a operands:
//   * codes c_0..c_3 of b come from a lookup table, one 32-bit word per byte
//     value, replicated per lane (entry b of lane l at 4 (32 b + l)), so the
//     32 lanes of a warp always read 32 different banks;
//   * the fifth code c_4 = b / 81 is computed for the four bytes of a packed
//     word at once: the bytes go to 16-bit lanes, times 203, and bits 14-15 of
//     each lane are the quotient (exact for b < 243), gathered back into bytes.
// So the activation words of a group are 26 "main" words (byte n: codes 5n ..
// 5n+3; for byte 25 codes 125..127 and a zero) and 7 "fifth-digit" words
// (word k: codes 5(4k+j)+4, j = 0..3, zero past code 124), padded to 36 words
// per plane.
//
// Geometry: a box is one 1024-block of K, 208 bytes, of each of the CTA's R
// rows (no swizzle; a row pitch of 13 16-byte chunks makes lane = row loads of
// one chunk conflict-free).  A group starts at byte 26 g of the block, which
// is 16-byte aligned only for g = 0: three chunk loads cover it, and its words
// are aligned with warp-uniform selects and a 2-byte funnel shift.
// Pipeline, slots, refill and the final fixed-order reduction are those of the
// 2-bit kernel.
#pragma once
#include "gemv.cuh"

namespace tb {

constexpr int kB3BlockBytes = 208;           // one 1024-block of a row
constexpr int kB3GroupBytes = 26;
constexpr int kB3PlaneWords = 36;            // 26 main + 7 fifth-digit words, padded
constexpr int kB3ActGroupBytes = 2 * kB3PlaneWords * 4;  // 288
constexpr int kB3LutBytes = 256 * 32 * 4;    // 32 KB

__host__ __device__ constexpr int64_t b3_act_stage_bytes(int M, int NB) {
  return static_cast<int64_t>(M) * NB * 8 * (kB3ActGroupBytes + 8);
}
__host__ __device__ constexpr int64_t b3_nstage(int64_t K, int NB) { return (K / 1024 + NB - 1) / NB; }
// Workspace bound valid for every NB <= kGemvMaxNB.
__host__ __device__ constexpr int64_t b3_ws_bytes(int64_t M, int64_t K) {
  return (K / 1024 + kGemvMaxNB) * M * 8 * (kB3ActGroupBytes + 8);
}

// Position of code c (0..127) of a group in a plane's 144 bytes of words.
__device__ __forceinline__ int b3_code_pos(int c) {
  const int i = c / 5, r = c - 5 * (c / 5);
  return r < 4 ? 4 * i + r : 4 * (26 + (i >> 2)) + (i & 3);
}

// Activation prep for base-3: grid (K/1024, M), 128 threads; writes the stage
// blocks [stage][M][8 NB groups][288 B] + info [M][8 NB] {e, qsum}.  Launched
// with programmatic dependent launch (waits for the previous kernel first).
template <typename TIn>
__global__ void __launch_bounds__(kHThreads) prep_b3_kernel(const TIn* __restrict__ x,
                                                            const int8_t* __restrict__ signs,
                                                            uint8_t* __restrict__ ws, int K, int NB) {
  __shared__ float sm[kHB];
  __shared__ __align__(16) uint8_t grp[8 * kB3ActGroupBytes];
  pdl_launch_dependents();
  pdl_wait();
  const int blk = blockIdx.x, m = blockIdx.y, M = gridDim.y, t = threadIdx.x;
  for (int i = t; i < 8 * kB3ActGroupBytes / 16; i += kHThreads) reinterpret_cast<uint4*>(grp)[i] = make_uint4(0, 0, 0, 0);
  float v[8];
  load_rotated8<TIn>(x, signs, m, blk, K, v, sm);  // synchronises the block (transform)
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float e = mx / kQMax;
  const float inv = mx > 0.f ? kQMax / mx : 0.f;
  const int gb = t >> 4, u = t & 15;  // group of the block, thread within the group
  uint8_t* gw = grp + gb * kB3ActGroupBytes;
  int qs = 0;
  if (signs == nullptr) __syncthreads();  // the zero fill above must precede the byte stores
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = max(-32512, min(32512, __float2int_rn(v[i] * inv)));
    qs += q;
    const int hi = (q + 128) >> 8, lo = q - (hi << 8);
    const int pos = b3_code_pos(8 * u + i);
    gw[pos] = static_cast<uint8_t>(hi);
    gw[4 * kB3PlaneWords + pos] = static_cast<uint8_t>(lo);
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
  __syncthreads();
  const int g = blk * 8;  // first global group of the block
  const int s = g / (8 * NB), gs0 = g % (8 * NB);
  uint8_t* blkbase = ws + static_cast<int64_t>(s) * b3_act_stage_bytes(M, NB);
  uint4* dst = reinterpret_cast<uint4*>(blkbase + (static_cast<int64_t>(m) * 8 * NB + gs0) * kB3ActGroupBytes);
  for (int i = t; i < 8 * kB3ActGroupBytes / 16; i += kHThreads) dst[i] = reinterpret_cast<const uint4*>(grp)[i];
  if (u == 0) {
    int2 inf;
    inf.x = __float_as_int(e);
    inf.y = qs;
    reinterpret_cast<int2*>(blkbase + static_cast<int64_t>(M) * 8 * NB * kB3ActGroupBytes)[m * 8 * NB + gs0 + gb] = inf;
  }
}

// Fifth digits (b / 81) of the four bytes of w, as bytes.
__device__ __forceinline__ uint32_t b3_fifth(uint32_t w) {
  const uint32_t ev = __byte_perm(w, 0u, 0x4240) * 203u;  // bytes 0, 2 in 16-bit lanes
  const uint32_t od = __byte_perm(w, 0u, 0x4341) * 203u;  // bytes 1, 3
  const uint32_t t = __byte_perm(ev, od, 0x7351);         // bits 8..15 / 24..31 of each lane
  return (t >> 6) & 0x03030303u;
}

// The 7 words of group gp (0..7) of a 208-byte block row at `row` (16-byte
// aligned): bytes 0..25 of the group, then 2 more bytes (of the next group, or
// past the row: only the fifth-digit lanes with zero activations see them).
// Three 16-byte loads cover the group wherever it starts; the word offset
// (0..3) and the 2-byte shift are uniform across the warp and applied with
// selects and a funnel shift, so one code path serves all eight positions.
__device__ __forceinline__ void b3_group_words(const uint8_t* row, int gp, uint32_t (&G)[7]) {
  const int o = 26 * gp, c0 = o >> 4, q = (o & 15) >> 2;
  const uint32_t sh = (o & 2) ? 16u : 0u;
  uint32_t u[12];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const uint4 v = reinterpret_cast<const uint4*>(row)[c0 + c];
    u[4 * c] = v.x;
    u[4 * c + 1] = v.y;
    u[4 * c + 2] = v.z;
    u[4 * c + 3] = v.w;
  }
  uint32_t v[10], w[8];
#pragma unroll
  for (int i = 0; i < 10; ++i) v[i] = (q & 2) ? u[i + 2] : u[i];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = (q & 1) ? v[i + 1] : v[i];
#pragma unroll
  for (int k = 0; k < 7; ++k) G[k] = __funnelshift_r(w[k], w[k + 1], sh);
}

// Entry b of this lane's copy of the table: shared address lut_lane + 128 b.
__device__ __forceinline__ uint32_t b3_lut(uint32_t lut_lane, uint32_t b) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(lut_lane + (b << 7)));
  return v;
}

// Integer sums  sum_k c_k hi_k  and  sum_k c_k lo_k  of one group of one row:
// codes from the words G, activation planes A (hi at 0, lo at kB3PlaneWords).
__device__ __forceinline__ void b3_dot(const uint32_t (&G)[7], const uint32_t* A, uint32_t lut_lane, int& h,
                                       int& l) {
  int hh[4] = {0, 0, 0, 0}, ll[4] = {0, 0, 0, 0};
#pragma unroll
  for (int n = 0; n < 26; ++n) {
    const uint32_t b = __byte_perm(G[n >> 2], 0u, 0x4440u + (n & 3));
    const uint32_t c = b3_lut(lut_lane, b);
    hh[n & 3] = dp4a_us(c, A[n], hh[n & 3]);
    ll[n & 3] = dp4a_us(c, A[kB3PlaneWords + n], ll[n & 3]);
  }
#pragma unroll
  for (int k = 0; k < 7; ++k) {
    const uint32_t c = b3_fifth(G[k]);
    hh[k & 3] = dp4a_us(c, A[26 + k], hh[k & 3]);
    ll[k & 3] = dp4a_us(c, A[kB3PlaneWords + 26 + k], ll[k & 3]);
  }
  h = (hh[0] + hh[1]) + (hh[2] + hh[3]);
  l = (ll[0] + ll[1]) + (ll[2] + ll[3]);
}

struct GemvB3Params {
  const uint8_t* act;      // prep_b3_kernel output, stage blocks
  const uint16_t* scales;  // [N, K/128] fp16 bits
  void* y;                 // [M, N]
  int N, K;
  int R, RT, NB, nstage, nslots;
  int box_stride;          // bytes between the boxes of a slot (1 KB multiple)
  int slot_bytes;          // boxes + activation block
  int sc_bytes;            // shared-memory bytes for the CTA's scales
};

// Shared memory: [1 KB alignment slack] lookup table | scales | ring of slots |
// barriers and per-slot counters.
__host__ __device__ inline int64_t b3_smem_bytes(int64_t sc_bytes, int64_t slot_bytes, int nslots) {
  return 1024 + kB3LutBytes + sc_bytes + slot_bytes * nslots + 8 * (kGemvMaxSlots + 1) + 4 * kGemvMaxSlots;
}

// Copies stage s into slot slot_i: NB weight boxes and the activation block.
__device__ __forceinline__ void b3_issue_stage(const CUtensorMap* tm, const GemvB3Params& p, uint8_t* ring,
                                               uint64_t* full, int s, int slot_i, int r0, uint32_t wbytes,
                                               uint32_t abytes, bool weights, bool act) {
  uint8_t* slot = ring + static_cast<int64_t>(slot_i) * p.slot_bytes;
  if (weights) {
    mbar_arrive_expect_tx(&full[slot_i], wbytes + abytes);
    for (int b = 0; b < p.NB; ++b)
      tma_load_2d(slot + b * p.box_stride, tm, (s * p.NB + b) * kB3BlockBytes, r0, &full[slot_i]);
  }
  if (act) bulk_load(slot + p.NB * p.box_stride, p.act + static_cast<int64_t>(s) * abytes, abytes, &full[slot_i]);
}

// One item: group gs & 7 of box `box`, for up to kGemvRowTiles tiles of 32 rows.
template <int M>
__device__ __forceinline__ void b3_item(const uint8_t* box, const uint8_t* act, const __half* sc, const int (&roff)[4],
                                        const int (&soff)[4], int RT, int NB, int gs, int g, uint32_t lut_lane,
                                        float (&acc)[M][4]) {
  float e[M];
  int qs[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int2 inf = reinterpret_cast<const int2*>(act + M * 8 * NB * kB3ActGroupBytes)[m * 8 * NB + gs];
    e[m] = __int_as_float(inf.x);
    qs[m] = inf.y;
  }
  uint32_t A[2 * kB3PlaneWords];
  if constexpr (M == 1) {
    const uint4* src = reinterpret_cast<const uint4*>(act + gs * kB3ActGroupBytes);
#pragma unroll
    for (int v = 0; v < 2 * kB3PlaneWords / 4; ++v) {
      const uint4 u4 = src[v];
      A[4 * v] = u4.x; A[4 * v + 1] = u4.y; A[4 * v + 2] = u4.z; A[4 * v + 3] = u4.w;
    }
  }
#pragma unroll
  for (int t = 0; t < kGemvRowTiles; ++t) {
    if (t < RT) {
      uint32_t G[7];
      b3_group_words(box + roff[t], gs & 7, G);
      const float s_rg = __half2float(sc[soff[t] + g]);
#pragma unroll
      for (int m = 0; m < M; ++m) {
        if constexpr (M > 1) {
          const uint4* src = reinterpret_cast<const uint4*>(act + (m * 8 * NB + gs) * kB3ActGroupBytes);
#pragma unroll
          for (int v = 0; v < 2 * kB3PlaneWords / 4; ++v) {
            const uint4 u4 = src[v];
            A[4 * v] = u4.x; A[4 * v + 1] = u4.y; A[4 * v + 2] = u4.z; A[4 * v + 3] = u4.w;
          }
        }
        int h, l;
        b3_dot(G, A, lut_lane, h, l);
        acc[m][t] = fmaf(__int2float_rn(h * 256 + l - qs[m]), s_rg * e[m], acc[m][t]);
      }
    }
  }
}

// One CTA: rows [blockIdx.x * R, +R), all of K; the 16-warp pipeline of the
// 2-bit kernel with one item per group.
template <int M, typename TOut>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_b3_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvB3Params p) {
  constexpr int NW = kGemvWarps;
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint32_t* lut = reinterpret_cast<uint32_t*>(base);
  const __half* sc = reinterpret_cast<const __half*>(base + kB3LutBytes);
  uint8_t* ring = base + kB3LutBytes + p.sc_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + p.nslots * p.slot_bytes);
  uint64_t* sc_bar = full + kGemvMaxSlots;
  uint32_t* done = reinterpret_cast<uint32_t*>(sc_bar + 1);

  const int G = p.K / 128;
  const int r0 = blockIdx.x * p.R;
  const int nrows = min(p.R, p.N - r0);
  const int IPS = p.NB * 8;                // items (groups) per stage
  const int Q = IPS >= NW ? 1 : NW / IPS;  // stages worked on at once
  const int WPS = IPS >= NW ? NW : IPS;    // warps per stage
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t wbytes = static_cast<uint32_t>(p.NB) * static_cast<uint32_t>(p.R) * kB3BlockBytes;
  const uint32_t abytes = static_cast<uint32_t>(b3_act_stage_bytes(M, p.NB));
  const int act_off = p.NB * p.box_stride;
  const int pre = min(p.nslots, p.nstage);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemvMaxSlots; ++s) {
      mbar_init(&full[s], 1);
      done[s] = 0;
    }
    mbar_init(sc_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_w);
    const uint32_t sbytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(G * 2);
    mbar_arrive_expect_tx(sc_bar, sbytes);
    bulk_load(base + kB3LutBytes, p.scales + static_cast<int64_t>(r0) * G, sbytes, sc_bar);
    for (int s = 0; s < pre; ++s) b3_issue_stage(&tm_w, p, ring, full, s, s, r0, wbytes, abytes, true, false);
    pdl_wait();  // the prep kernel's activation blocks
    for (int s = 0; s < pre; ++s) b3_issue_stage(&tm_w, p, ring, full, s, s, r0, wbytes, abytes, false, true);
  }
  // lookup table: entry b = codes c_0..c_3 of byte b (digits of b in base 3),
  // bytes >= 243 (invalid) decode as c = 1; replicated for the 32 lanes
  for (int i = threadIdx.x; i < 256 * 32; i += kGemvThreads) {
    const int b = i >> 5;
    uint32_t v = 0x01010101u;
    if (b < 243) v = static_cast<uint32_t>(b % 3) | static_cast<uint32_t>((b / 3) % 3) << 8 |
                     static_cast<uint32_t>((b / 9) % 3) << 16 | static_cast<uint32_t>((b / 27) % 3) << 24;
    lut[i] = v;
  }
  __syncthreads();

  float acc[M][4];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int t = 0; t < 4; ++t) acc[m][t] = 0.f;
  int roff[4], soff[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    roff[t] = min(32 * t + lane, p.R - 1) * kB3BlockBytes;
    soff[t] = min(32 * t + lane, nrows - 1) * G;
  }
  const uint32_t lut_lane = smem_u32(lut) + 4u * static_cast<uint32_t>(lane);  // shared address

  const int it0 = IPS >= NW ? warp : warp % IPS;
  const int q = IPS >= NW ? 0 : warp / IPS;
  bool ok = mbar_wait_backoff(sc_bar, 0, FAULT_WAIT_ACT);
  int slot_i = q;
  uint32_t phase = 0;
  for (int s = q; s < p.nstage && ok; s += Q) {
    if (!mbar_wait_backoff(&full[slot_i], phase, FAULT_WAIT_FULL)) {
      ok = false;
      break;
    }
    const uint8_t* slot = ring + slot_i * p.slot_bytes;
    const uint8_t* act = slot + act_off;
    for (int it = it0; it < IPS; it += NW) {
      const int g = s * 8 * p.NB + it;  // global group
      if (g >= G) continue;
      const uint8_t* box = slot + (it >> 3) * p.box_stride;
      b3_item<M>(box, act, sc, roff, soff, p.RT, p.NB, it, g, lut_lane, acc);
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&done[slot_i], 1u) == static_cast<uint32_t>(WPS - 1)) {
        __threadfence_block();
        done[slot_i] = 0;
        if (s + p.nslots < p.nstage)
          b3_issue_stage(&tm_w, p, ring, full, s + p.nslots, slot_i, r0, wbytes, abytes, true, true);
      }
    }
    __syncwarp();
    slot_i += Q;
    if (slot_i >= p.nslots) {
      slot_i -= p.nslots;
      phase ^= 1u;
    }
  }
  if (threadIdx.x == 0) {
    for (int s = max(0, p.nstage - p.nslots); s < p.nstage; ++s)
      if (!mbar_wait(&full[s % p.nslots], (s / p.nslots) & 1, FAULT_WAIT_FULL)) break;
  }
  __syncthreads();
  float* part = reinterpret_cast<float*>(ring);
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int t = 0; t < 4; ++t)
      if (t < p.RT) part[((m * p.RT + t) * 32 + lane) * NW + warp] = acc[m][t];
  __syncthreads();
  TOut* y = reinterpret_cast<TOut*>(p.y);
  for (int idx = threadIdx.x; idx < M * nrows; idx += kGemvThreads) {
    const int m = idx / nrows, r = idx - m * nrows;
    const float* src = part + (m * p.RT * 32 + r) * NW;
    float sum = 0.f;
    for (int i = 0; i < NW; ++i) sum += src[i];
    y[static_cast<int64_t>(m) * p.N + r0 + r] = from_f32<TOut>(sum);
  }
}

}  // namespace tb
