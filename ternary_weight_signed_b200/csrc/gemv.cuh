// Decode GEMV for small M (1 to 4 tokens) on the 2-bit slot format.
//
// y[m, n] = sum_g s[n, g] * sum_{k in g} t[n, k] x'[m, k]   (ternary g128;
// news.ditty.ir second paragraph, ai4coding.ru "What is a ternary model").
//
// The ternary multiply is an add/subtract (ai4coding.ru, same section); here
// it is carried out on integers.  x' is held per 128-group as 16-bit fixed
// point q = rint(x' / e_g) split into two int8 planes (q = 256 hi + lo), and
// the packed 2-bit word gives the biased codes c = t + 1 as bytes, so
//   sum_k t q = 256 * sum c hi + sum c lo - sum q,
// four codes per dp4a instruction, exact in int32.  The group scale s * e_g
// is applied in fp32 once per group (per item, see below).
//
// Two ways to turn a packed word w (16 codes; code 4b + j of the word in bits
// 8b + 2j of it) into dp4a operands:
//   shift mode (M >= 2): c_j = (w >> 2j) & 0x03030303, shared by all tokens;
//   mask mode  (M == 1): w & (0x03030303 << 2j) = 4^j c_j, one instruction;
//     the four partial sums T_j are 4^j times the true ones, so they are
//     combined exactly as T_0 + (T_1 >> 2) + (T_2 >> 4) + (T_3 >> 6).
//
// Work split.  One CTA of 16 warps per SM; the CTAs own consecutive ranges of
// R <= 128 weight rows.  K is walked in stages of NB boxes; a box is 128 bytes
// (512 codes) of each of the CTA's rows, brought by one 2-D TMA copy with the
// 128-byte swizzle, so a warp whose lanes read the same 16-byte chunk of 32
// different rows hits every bank group once.  One lane = one weight row, so a
// row's sum never crosses lanes.  An item is one group (M = 1), half a group
// (M = 2) or a quarter group (M >= 3) of one stage; a warp takes an item,
// loads its activation words once into registers (broadcast shared-memory
// loads: every lane reads the same words) and runs it over all of the CTA's
// rows, 32 at a time, accumulating each row's fp32 sum in a register.  At the
// end the warps' per-row partials go through shared memory and are added in a
// fixed order (bitwise reproducible).
//
// The rotated fixed-point activations are made by prep_gemv_kernel (one
// 128-thread CTA per token and 1024-block) launched just before.  The decode
// kernel is launched with programmatic dependent launch: thread 0 issues the
// weight copies of the first stages (up to the whole ring, which is sized to
// the SM's shared memory) at once, and only the activation copies wait for the
// prep kernel.
#pragma once
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGemvMaxM = 4;
constexpr int kGemvWarps = 16;                       // warps per CTA, all consumers
constexpr int kGemvThreads = 32 * kGemvWarps;
constexpr int kGemvBoxCodes = 512;                  // K per box: 128 bytes of a row
constexpr int kGemvMaxNB = 8;                       // boxes per stage at most
constexpr int kGemvMaxSlots = 12;
constexpr int kGemvSmemTarget = 227 * 1024;         // one CTA per SM

constexpr int kGemvRowTiles = 4;  // rows per CTA <= 32 * kGemvRowTiles
// rows per CTA at most: 32 * gemv_max_row_tiles(M)
__host__ __device__ constexpr int gemv_max_row_tiles(int) { return kGemvRowTiles; }
// codes per item
__host__ __device__ constexpr int gemv_cpi(int M) { return M == 1 ? 128 : (M == 2 ? 64 : 32); }

// Activation block of one stage (what one bulk copy brings):
//   words[M][4 NB groups][256 B], then info[M][4 NB groups] {float e, int qsum}.
// Group words: [plane (hi, lo)][i = which 16 codes, 0..7][j = slot, 0..3],
// 4 bytes each; byte b of word (p, i, j) holds plane p of code 16 i + 4 b + j.
constexpr int kGemvGroupBytes = 256;
__host__ __device__ constexpr int64_t gemv_act_stage_bytes(int M, int NB) {
  return static_cast<int64_t>(M) * NB * 4 * (kGemvGroupBytes + 8);
}
__host__ __device__ constexpr int64_t gemv_nstage(int64_t K, int NB) {
  return (K / kGemvBoxCodes + NB - 1) / NB;
}
// Workspace bound valid for every NB <= kGemvMaxNB.
__host__ __device__ constexpr int64_t gemv_ws_bytes(int64_t M, int64_t K) {
  return (K / kGemvBoxCodes + kGemvMaxNB) * M * 4 * (kGemvGroupBytes + 8);
}

struct GemvParams {
  const uint8_t* act;      // prep_gemv_kernel output, stage blocks
  const uint16_t* scales;  // [N, K/128] fp16 bits
  void* y;                 // [M, N]
  int N, K;
  int R;                   // rows per CTA (box height)
  int RT;                  // row tiles of 32 covering R
  int NB;                  // boxes per stage
  int nstage;
  int nslots;
  int box_stride;          // bytes between the boxes of a slot (1 KB multiple)
  int slot_bytes;          // boxes + activation block
  int sc_bytes;            // shared-memory bytes for the CTA's scales
};

__host__ __device__ constexpr int64_t align_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }
__host__ __device__ constexpr int64_t align128(int64_t v) { return align_up(v, 128); }

// Shared memory: [1 KB alignment slack] scales | ring of slots | barriers and
// per-slot counters.
__host__ __device__ inline int64_t gemv_smem_bytes(int64_t sc_bytes, int64_t slot_bytes, int nslots) {
  return 1024 + sc_bytes + slot_bytes * nslots + 8 * (kGemvMaxSlots + 1) + 4 * kGemvMaxSlots;
}

// 16-bit fixed point of one 128-group whose values are spread over 16
// consecutive lanes of a warp, 8 each (lane u = t & 15 holds codes 8u .. 8u+7
// of the group, the layout of the 128-thread block transform).  Writes the
// group's 256 bytes of activation words to `gw` and, from lane u = 0, its
// {e_g, sum of q} to `*inf`.  Word (plane p, i, j) sits at byte 128 p + 16 i +
// 4 j, and its byte b holds plane p of code 16 i + 4 b + j: lane pair
// (2i, 2i + 1) holds word i's codes.
__device__ __forceinline__ void gemv_quantize_group8(const float v[8], int t, uint8_t* gw, int2* inf) {
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float e = mx / kQMax;
  const float inv = mx > 0.f ? kQMax / mx : 0.f;
  int hi[8], lo[8];
  int qs = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int q = max(-32512, min(32512, __float2int_rn(v[i] * inv)));
    qs += q;
    hi[i] = (q + 128) >> 8;
    lo[i] = q - (hi[i] << 8);
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
  // Byte b of word (plane, i, j) is code 16 i + 4 b + j: the even thread of the
  // pair supplies bytes 0, 1 (its elements j and 4 + j), the odd one bytes 2, 3.
  // The even thread writes the hi plane's four words, the odd one the lo plane's.
  const int u = t & 15, h = u & 1, wi = u >> 1;
  uint32_t word[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t hh = (static_cast<uint32_t>(hi[j]) & 0xFFu) | ((static_cast<uint32_t>(hi[4 + j]) & 0xFFu) << 8);
    const uint32_t hl = (static_cast<uint32_t>(lo[j]) & 0xFFu) | ((static_cast<uint32_t>(lo[4 + j]) & 0xFFu) << 8);
    const uint32_t recv = __shfl_xor_sync(0xffffffffu, h ? hh : hl, 1);
    word[j] = h ? (recv | (hl << 16)) : (hh | (recv << 16));
  }
  *reinterpret_cast<uint4*>(gw + h * 128 + wi * 16) = make_uint4(word[0], word[1], word[2], word[3]);
  if (u == 0) {
    int2 i2;
    i2.x = __float_as_int(e);
    i2.y = qs;
    *inf = i2;
  }
}

// Activation prep: grid (K/1024, M), 128 threads per (1024-block, token);
// thread t holds elements 8t .. 8t+7 of the block (the 128-thread block
// transform of hadamard.cuh), so a 128-group is 16 threads and thread pair
// (2i, 2i+1) of a group holds its 16-code word i.  Launched with programmatic
// dependent launch: it waits for the previous kernel on the stream (which may
// have produced x, or may still be reading this workspace) before touching
// either.
template <typename TIn>
__global__ void __launch_bounds__(kHThreads) prep_gemv_kernel(const TIn* __restrict__ x,
                                                              const int8_t* __restrict__ signs,
                                                              uint8_t* __restrict__ ws, int K, int NB) {
  __shared__ float sm[kHB];
  pdl_launch_dependents();
  pdl_wait();
  const int blk = blockIdx.x, m = blockIdx.y, M = gridDim.y, t = threadIdx.x;
  float v[8];
  load_rotated8<TIn>(x, signs, m, blk, K, v, sm);
  const int g = blk * 8 + (t >> 4);  // global group index
  const int s = g / (4 * NB), gs = g % (4 * NB);
  uint8_t* blkbase = ws + static_cast<int64_t>(s) * gemv_act_stage_bytes(M, NB);
  uint8_t* gw = blkbase + (static_cast<int64_t>(m) * 4 * NB + gs) * kGemvGroupBytes;
  int2* inf = reinterpret_cast<int2*>(blkbase + static_cast<int64_t>(M) * 4 * NB * kGemvGroupBytes) + m * 4 * NB + gs;
  gemv_quantize_group8(v, t, gw, inf);
}

// Integer group sum  sum_k c_k q_k  of one item for one token, mask mode (a
// whole group: 8 packed words, 64 activation words A[p][i][j] at 32 p + 4 i + j).
__device__ __forceinline__ int gemv_item_mask(const uint32_t (&w)[8], const uint32_t (&A)[64]) {
  int th[4] = {0, 0, 0, 0}, tl[4] = {0, 0, 0, 0};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t c = w[i] & (0x03030303u << (2 * j));
      th[j] = dp4a_us(c, A[4 * i + j], th[j]);
      tl[j] = dp4a_us(c, A[32 + 4 * i + j], tl[j]);
    }
  }
  int t[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) t[j] = th[j] * 256 + tl[j];
  return t[0] + (t[1] >> 2) + (t[2] >> 4) + (t[3] >> 6);
}

// Copies stage s into slot slot_i (= s % nslots): the NB weight boxes and the activation
// block, all completing on the slot's full barrier.  With act == false the
// activation copy is left for later (it waits for the prep kernel).
__device__ __forceinline__ void gemv_issue_stage(const CUtensorMap* tm, const GemvParams& p, uint8_t* ring,
                                                 uint64_t* full, int s, int slot_i, int r0, uint32_t wbytes,
                                                 uint32_t abytes, bool weights, bool act) {
  uint8_t* slot = ring + static_cast<int64_t>(slot_i) * p.slot_bytes;
  if (weights) {
    mbar_arrive_expect_tx(&full[slot_i], wbytes + abytes);
    for (int b = 0; b < p.NB; ++b) tma_load_2d(slot + b * p.box_stride, tm, (s * p.NB + b) * 128, r0, &full[slot_i]);
  }
  if (act)
    bulk_load(slot + p.NB * p.box_stride, p.act + static_cast<int64_t>(s) * abytes, abytes, &full[slot_i]);
}

// One CTA: rows [blockIdx.x * R, +R), all of K.  Sixteen warps, no dedicated
// producer: thread 0 issues the first nslots stages, and afterwards the last
// warp to finish with a stage refills its slot with the stage nslots later.
template <int M, typename TOut>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_2bit_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvParams p) {
  constexpr int CPI = gemv_cpi(M);  // codes per item
  constexpr int PPG = 128 / CPI;    // items per group
  constexpr int WPI = CPI / 16;     // packed 32-bit words per row and item
  constexpr int AW = 2 * WPI * 4;   // activation words per token and item
  constexpr int RTM = gemv_max_row_tiles(M);
  constexpr int NW = kGemvWarps;

  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const __half* sc = reinterpret_cast<const __half*>(base);
  uint8_t* ring = base + p.sc_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<int64_t>(p.nslots) * p.slot_bytes);
  uint64_t* sc_bar = full + kGemvMaxSlots;
  uint32_t* done = reinterpret_cast<uint32_t*>(sc_bar + 1);  // warps finished per slot

  const int G = p.K / 128;
  const int r0 = blockIdx.x * p.R;
  const int nrows = min(p.R, p.N - r0);
  const int IPS = p.NB * 4 * PPG;          // items per stage
  const int Q = IPS >= NW ? 1 : NW / IPS;  // stages worked on at once
  const int WPS = IPS >= NW ? NW : IPS;    // warps per stage
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t wbytes = static_cast<uint32_t>(p.NB) * static_cast<uint32_t>(p.R) * 128u;
  const uint32_t abytes = static_cast<uint32_t>(gemv_act_stage_bytes(M, p.NB));
  const int act_off = p.NB * p.box_stride;  // activation block inside a slot
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
    bulk_load(base, p.scales + static_cast<int64_t>(r0) * G, sbytes, sc_bar);
    // weights do not depend on the prep kernel; its activation blocks do
    for (int s = 0; s < pre; ++s) gemv_issue_stage(&tm_w, p, ring, full, s, s, r0, wbytes, abytes, true, false);
    pdl_wait();
    for (int s = 0; s < pre; ++s) gemv_issue_stage(&tm_w, p, ring, full, s, s, r0, wbytes, abytes, false, true);
  }
  // The other threads wait here (a hardware barrier, no issue slots taken)
  // while thread 0 waits for the prep kernel: a CTA that starts early, next to
  // one of the previous call still computing on the same SM, stays idle.
  __syncthreads();

  float acc[M][RTM];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int t = 0; t < RTM; ++t) acc[m][t] = 0.f;
  // This lane's rows are 32 t + lane (rows past R repeat row R - 1; their sums
  // are discarded): byte offsets of the rows in a box and of their scales.  The
  // 128-byte swizzle XORs the 16-byte chunk index with the row index mod 8,
  // which is lane & 7 for every tile.
  int roff[RTM], soff[RTM];
#pragma unroll
  for (int t = 0; t < RTM; ++t) {
    roff[t] = min(32 * t + lane, p.R - 1) * 128;
    soff[t] = min(32 * t + lane, nrows - 1) * G;
  }
  const int sw = lane & 7;

  const int it0 = IPS >= NW ? warp : warp % IPS;
  const int q = IPS >= NW ? 0 : warp / IPS;
  bool ok = mbar_wait_backoff(sc_bar, 0, FAULT_WAIT_ACT);
  // stage s lives in slot s % nslots with barrier phase (s / nslots) & 1;
  // nslots is a multiple of Q, so stepping s by Q wraps the slot exactly
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
      const int gs = it / PPG, pt = it % PPG;  // group within the stage, part of the group
      const int g = s * 4 * p.NB + gs;          // global group
      if (g >= G) continue;                     // past K in the last stage
      const int b = gs >> 2, gl = gs & 3;       // box, group within the box
      // activation words and {e, qsum} of this item for every token (broadcast loads)
      uint32_t A[M][AW];
      float e[M];
      int qs[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const uint8_t* gw = act + (m * 4 * p.NB + gs) * kGemvGroupBytes;
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
          const uint4* src = reinterpret_cast<const uint4*>(gw + pl * 128 + pt * CPI);
#pragma unroll
          for (int v = 0; v < AW / 8; ++v) {
            const uint4 u4 = src[v];
            A[m][pl * (AW / 2) + 4 * v] = u4.x;
            A[m][pl * (AW / 2) + 4 * v + 1] = u4.y;
            A[m][pl * (AW / 2) + 4 * v + 2] = u4.z;
            A[m][pl * (AW / 2) + 4 * v + 3] = u4.w;
          }
        }
        const int2 inf = reinterpret_cast<const int2*>(act + M * 4 * p.NB * kGemvGroupBytes)[m * 4 * p.NB + gs];
        e[m] = __int_as_float(inf.x);
        qs[m] = pt == 0 ? inf.y : 0;
      }
      const uint8_t* box = slot + b * p.box_stride;
      // the item's packed words of one row: chunk(s) of the row's 128 bytes
      int c0, c1 = 0, h8 = 0;
      if constexpr (WPI == 8) {
        c0 = ((2 * gl) ^ sw) << 4;
        c1 = ((2 * gl + 1) ^ sw) << 4;
      } else if constexpr (WPI == 4) {
        c0 = ((2 * gl + pt) ^ sw) << 4;
      } else {
        c0 = ((2 * gl + (pt >> 1)) ^ sw) << 4;
        h8 = 8 * (pt & 1);
      }
      uint32_t nx[WPI];  // next tile's words, loaded one tile ahead
      auto load_words = [&](int t, uint32_t (&w)[WPI]) {
        const uint8_t* rp = box + roff[t];
        if constexpr (WPI == 8) {
          const uint4 u0 = *reinterpret_cast<const uint4*>(rp + c0);
          const uint4 u1 = *reinterpret_cast<const uint4*>(rp + c1);
          w[0] = u0.x; w[1] = u0.y; w[2] = u0.z; w[3] = u0.w;
          w[4] = u1.x; w[5] = u1.y; w[6] = u1.z; w[7] = u1.w;
        } else if constexpr (WPI == 4) {
          const uint4 u0 = *reinterpret_cast<const uint4*>(rp + c0);
          w[0] = u0.x; w[1] = u0.y; w[2] = u0.z; w[3] = u0.w;
        } else {
          const uint2 u0 = *reinterpret_cast<const uint2*>(rp + c0 + h8);
          w[0] = u0.x; w[1] = u0.y;
        }
      };
      load_words(0, nx);
#pragma unroll
      for (int t = 0; t < RTM; ++t) {
        if (t < p.RT) {
          uint32_t w[WPI];
#pragma unroll
          for (int i = 0; i < WPI; ++i) w[i] = nx[i];
          if (t + 1 < RTM && t + 1 < p.RT) load_words(t + 1, nx);
          const float s_rg = __half2float(sc[soff[t] + g]);
          if constexpr (M == 1) {
            const int tot = gemv_item_mask(w, A[0]) - qs[0];
            acc[0][t] = fmaf(__int2float_rn(tot), s_rg * e[0], acc[0][t]);
          } else {
            int h[M], l[M];
#pragma unroll
            for (int m = 0; m < M; ++m) {
              h[m] = 0;
              l[m] = 0;
            }
#pragma unroll
            for (int i = 0; i < WPI; ++i) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint32_t c = (w[i] >> (2 * j)) & 0x03030303u;
#pragma unroll
                for (int m = 0; m < M; ++m) {
                  h[m] = dp4a_us(c, A[m][4 * i + j], h[m]);
                  l[m] = dp4a_us(c, A[m][AW / 2 + 4 * i + j], l[m]);
                }
              }
            }
#pragma unroll
            for (int m = 0; m < M; ++m)
              acc[m][t] = fmaf(__int2float_rn(h[m] * 256 + l[m] - qs[m]), s_rg * e[m], acc[m][t]);
          }
        }
      }
    }
    // the last warp out of this stage refills the slot
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&done[slot_i], 1u) == static_cast<uint32_t>(WPS - 1)) {
        __threadfence_block();
        done[slot_i] = 0;
        if (s + p.nslots < p.nstage)
          gemv_issue_stage(&tm_w, p, ring, full, s + p.nslots, slot_i, r0, wbytes, abytes, true, true);
      }
    }
    __syncwarp();
    slot_i += Q;
    if (slot_i >= p.nslots) {
      slot_i -= p.nslots;
      phase ^= 1u;
    }
  }
  // every copy must have landed before the ring is reused: wait for the last
  // stage of every slot (already complete unless a wait above gave up)
  if (threadIdx.x == 0) {
    for (int s = max(0, p.nstage - p.nslots); s < p.nstage; ++s)
      if (!mbar_wait(&full[s % p.nslots], (s / p.nslots) & 1, FAULT_WAIT_FULL)) break;
  }
  // park the per-warp row partials in the ring and add them in a fixed order
  __syncthreads();
  float* part = reinterpret_cast<float*>(ring);
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int t = 0; t < RTM; ++t)
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

// ---------------------------------------------------------------------------
// Decode at M = 1 with dynamic item distribution.  Same data path as
// gemv_2bit_kernel<1> (boxes, slots, activation blocks, mask-mode dp4a), but
// the warps take items (stage, group) in order from a CTA-wide counter, so a
// warp that the issue scheduler serves more often simply takes more items and
// all warps finish together.  Each item's row sums go to a partial buffer
// indexed by the item, and the final sum over items runs in item order, so the
// result does not depend on which warp took which item (bitwise
// reproducible).  Every stage has its own full barrier (used once), so a warp
// may wait for any stage; the warp completing the last item of stage s refills
// its slot with stage s + nslots.
__host__ __device__ inline int64_t gemv_dyn_part_bytes(int nstage, int NB, int RT) {
  return align128(static_cast<int64_t>(nstage) * NB * 4 * RT * 32 * 4);
}
__host__ __device__ inline int64_t gemv_dyn_smem_bytes(int64_t sc_bytes, int64_t slot_bytes, int nslots, int nstage,
                                                       int NB, int RT) {
  return 1024 + sc_bytes + slot_bytes * nslots + gemv_dyn_part_bytes(nstage, NB, RT) + 8 * (nstage + 1) +
         4 * (nstage + 2);
}

__device__ __forceinline__ void gemv_issue_stage_bar(const CUtensorMap* tm, const GemvParams& p, uint8_t* ring,
                                                     uint64_t* bar, int s, int slot_i, int r0, uint32_t wbytes,
                                                     uint32_t abytes, bool weights, bool act) {
  uint8_t* slot = ring + static_cast<int64_t>(slot_i) * p.slot_bytes;
  if (weights) {
    mbar_arrive_expect_tx(bar, wbytes + abytes);
    for (int b = 0; b < p.NB; ++b) tma_load_2d(slot + b * p.box_stride, tm, (s * p.NB + b) * 128, r0, bar);
  }
  if (act) bulk_load(slot + p.NB * p.box_stride, p.act + static_cast<int64_t>(s) * abytes, abytes, bar);
}

template <typename TOut>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_2bit_dyn_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvParams p) {
  constexpr int RTM = kGemvRowTiles;
  pdl_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const __half* sc = reinterpret_cast<const __half*>(base);
  uint8_t* ring = base + p.sc_bytes;
  float* part = reinterpret_cast<float*>(ring + p.nslots * p.slot_bytes);
  const int IPS = p.NB * 4;  // items (groups) per stage
  const int nitems = p.nstage * IPS;
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(part) +
                                               gemv_dyn_part_bytes(p.nstage, p.NB, p.RT));
  uint64_t* sc_bar = full + p.nstage;
  uint32_t* cnt = reinterpret_cast<uint32_t*>(sc_bar + 1);  // [0] next item, [1 + s] items done of stage s

  const int G = p.K / 128;
  const int r0 = blockIdx.x * p.R;
  const int nrows = min(p.R, p.N - r0);
  const int lane = threadIdx.x & 31;
  const uint32_t wbytes = static_cast<uint32_t>(p.NB) * static_cast<uint32_t>(p.R) * 128u;
  const uint32_t abytes = static_cast<uint32_t>(gemv_act_stage_bytes(1, p.NB));
  const int act_off = p.NB * p.box_stride;
  const int pre = min(p.nslots, p.nstage);
  const int RS = p.RT * 32;  // partial floats per item

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstage; ++s) {
      mbar_init(&full[s], 1);
      cnt[1 + s] = 0;
    }
    cnt[0] = 0;
    mbar_init(sc_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tm_w);
    const uint32_t sbytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(G * 2);
    mbar_arrive_expect_tx(sc_bar, sbytes);
    bulk_load(base, p.scales + static_cast<int64_t>(r0) * G, sbytes, sc_bar);
    for (int s = 0; s < pre; ++s) gemv_issue_stage_bar(&tm_w, p, ring, &full[s], s, s, r0, wbytes, abytes, true, false);
    pdl_wait();  // the prep kernel's activation blocks
    for (int s = 0; s < pre; ++s) gemv_issue_stage_bar(&tm_w, p, ring, &full[s], s, s, r0, wbytes, abytes, false, true);
  }
  __syncthreads();

  int roff[RTM], soff[RTM];
#pragma unroll
  for (int t = 0; t < RTM; ++t) {
    roff[t] = min(32 * t + lane, p.R - 1) * 128;
    soff[t] = min(32 * t + lane, nrows - 1) * G;
  }
  const int sw = lane & 7;
  bool ok = mbar_wait_backoff(sc_bar, 0, FAULT_WAIT_ACT);
  while (ok) {
    int i = 0;
    if (lane == 0) i = static_cast<int>(atomicAdd(&cnt[0], 1u));
    i = __shfl_sync(0xffffffffu, i, 0);
    if (i >= nitems) break;
    const int s = i / IPS, it = i - s * IPS;
    const int slot_i = s % p.nslots;
    if (!mbar_wait_backoff(&full[s], 0, FAULT_WAIT_FULL)) {
      ok = false;
      break;
    }
    const uint8_t* slot = ring + slot_i * p.slot_bytes;
    const int g = s * 4 * p.NB + it;
    float a[RTM];
#pragma unroll
    for (int t = 0; t < RTM; ++t) a[t] = 0.f;
    if (g < G) {
      const uint8_t* act = slot + act_off;
      uint32_t A[64];
      const uint4* src = reinterpret_cast<const uint4*>(act + it * kGemvGroupBytes);
#pragma unroll
      for (int v = 0; v < 16; ++v) {
        const uint4 u4 = src[v];
        A[4 * v] = u4.x; A[4 * v + 1] = u4.y; A[4 * v + 2] = u4.z; A[4 * v + 3] = u4.w;
      }
      const int2 inf = reinterpret_cast<const int2*>(act + 4 * p.NB * kGemvGroupBytes)[it];
      const float e = __int_as_float(inf.x);
      const uint8_t* box = slot + (it >> 2) * p.box_stride;
      const int gl = it & 3;
      const int c0 = ((2 * gl) ^ sw) << 4, c1 = ((2 * gl + 1) ^ sw) << 4;
#pragma unroll
      for (int t = 0; t < RTM; ++t) {
        if (t < p.RT) {
          const uint8_t* rp = box + roff[t];
          const uint4 u0 = *reinterpret_cast<const uint4*>(rp + c0);
          const uint4 u1 = *reinterpret_cast<const uint4*>(rp + c1);
          const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
          const float s_rg = __half2float(sc[soff[t] + g]);
          a[t] = __int2float_rn(gemv_item_mask(w, A) - inf.y) * (s_rg * e);
        }
      }
    }
    float* pp = part + static_cast<int64_t>(i) * RS;
#pragma unroll
    for (int t = 0; t < RTM; ++t)
      if (t < p.RT) pp[32 * t + lane] = a[t];
    // the warp finishing the last item of stage s refills its slot
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&cnt[1 + s], 1u) == static_cast<uint32_t>(IPS - 1) && s + p.nslots < p.nstage) {
        __threadfence_block();
        gemv_issue_stage_bar(&tm_w, p, ring, &full[s + p.nslots], s + p.nslots, slot_i, r0, wbytes, abytes, true,
                             true);
      }
    }
  }
  // every copy must have landed before the CTA exits
  if (threadIdx.x == 0) {
    for (int s = max(0, p.nstage - p.nslots); s < p.nstage; ++s)
      if (!mbar_wait(&full[s], 0, FAULT_WAIT_FULL)) break;
  }
  __syncthreads();
  // row r: four threads take the items i = 4 j + u (u = 0..3) and add them in
  // order of j; their four sums are then added in order of u
  TOut* y = reinterpret_cast<TOut*>(p.y);
  for (int base_r = 0; base_r < nrows; base_r += kGemvThreads / 4) {
    const int r = base_r + (threadIdx.x >> 2), u = threadIdx.x & 3;
    float sum = 0.f;
    if (r < nrows)
      for (int it = u; it < nitems; it += 4) sum += part[static_cast<int64_t>(it) * RS + r];
    const float s1 = __shfl_down_sync(0xffffffffu, sum, 1);
    const float s2 = __shfl_down_sync(0xffffffffu, sum, 2);
    const float s3 = __shfl_down_sync(0xffffffffu, sum, 3);
    if (u == 0 && r < nrows) y[r0 + r] = from_f32<TOut>(((sum + s1) + s2) + s3);
  }
}

}  // namespace tb
