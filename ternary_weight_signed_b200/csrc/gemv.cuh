// Decode GEMV for small M on the 2-bit slot format.
//
// y[m, n] = sum_g s[n, g] * sum_{k in g} t[n, k] x'[m, k]   (ternary g128;
// news.ditty.ir second paragraph, ai4coding.ru "What is a ternary model").
//
// The ternary multiply is an add/subtract (ai4coding.ru, same section).  Here
// it is carried out on integers: x' is held per 128-group as 16-bit fixed point
// q = rint(x' / e_g) split into two int8 planes (hi, lo), and the packed 2-bit
// word gives the biased codes c = t + 1 directly as bytes, so
//   sum_k t q = 256 * sum c hi + sum c lo - sum q
// with four codes per dp4a instruction and exact int32 sums; the group scale
// s * e_g is applied once per quarter-group in fp32.
//
// Memory side: a persistent grid, one CTA per SM.  CTA c owns a contiguous
// range of rows, whose packed codes are one contiguous byte range; it streams
// them as a few large 1-D bulk copies ("segments" of whole rows, up to
// kSegBytes) into a ring of shared-memory slots, after one copy of all of its
// scales.  Few, large copies matter: the copy engine's cost is per operation,
// and small boxes capped the stream far below HBM speed.
//
// Activations: for small M * K the consumer warps compute them in the
// kernel's prologue (rotation + fixed point, four groups of 128 threads, one
// 1024-block each at a time) while the first weight segments stream in, so a
// decode step is one kernel.  Otherwise a prep kernel writes them to the
// workspace and the consumers load them with plain loads (not through the copy
// engine, where they would queue behind the weights).
//
// Compute side: the work of a segment is split into items of (4 R rows, one
// 1024-code chunk of K), R = 2 rows per lane for M <= 2 and 1 otherwise.  Items
// are numbered across segments and consumer warp w takes items w, w + W, ...
// (W consumer warps), so the split is even for any N and K and every warp
// starts on the first segment to arrive.  Inside an item lane l owns 128-group
// l & 7 of the chunk for rows (l >> 3) + 4 i, i < R: the group scale is applied
// once per 128 codes, the activation words it loads serve R rows, and four
// independent dp4a chains keep the pipes busy.  The 8 lanes of a row reduce
// with 3 shuffles and one of them stores the item's sum in a per-(row, chunk)
// slot in shared memory.  At the end each row's chunk slots are summed in a
// fixed order, so results are bitwise reproducible.
#pragma once
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGemvConsumerWarps = 16;
constexpr int kGemvThreads = 32 * (kGemvConsumerWarps + 1);
constexpr int kGemvQuadRows = 4;
constexpr int kGemvMaxM = 4;
constexpr int kChunkCodes = 1024;        // K per item
constexpr int kSegBytes = 32 * 1024;     // target bytes of one weight segment
constexpr int kGemvMinSlots = 2;
constexpr int kGemvMaxSlots = 6;
constexpr int kGemvFwhtBytes = 4 * 1024 * 4;
constexpr int kGemvFusedMaxBlocks = 16;  // fuse the prologue when M * K/1024 <= this

struct GemvParams {
  const uint8_t* act;     // prep_gemv output, M rows of gemv_act_row_bytes(K) (when not fused)
  const void* x;          // [M, K] activations (fused prologue)
  const int8_t* signs;    // [K] or null (fused prologue)
  int xt;                 // dtype of x: 0 bf16, 1 fp16, 2 fp32
  int fused;              // 1: compute the activations in the prologue
  const uint8_t* packed;  // [N, K/4]
  const uint16_t* scales; // [N, K/128] fp16 bits
  void* y;                // [M, N]
  int N;
  int K;
  int seg_rows;           // rows per segment (a multiple of the item height)
  int nslots;             // ring depth
  int max_rows;           // largest row range of any CTA (sizes the shared buffers)
};

// Shared-memory layout, in order, each part 128-byte aligned:
//   act     M * gemv_act_row_bytes(K)
//   scales  max_rows * K/64 bytes
//   part    max_rows * (K/1024) * M floats
//   fwht    4 x 1024 floats (the fused prologue's transforms)
//   ring    nslots * seg_rows * K/4 bytes
//   barriers
__host__ __device__ constexpr int64_t align128(int64_t v) { return (v + 127) & ~int64_t(127); }

__host__ __device__ inline int64_t gemv_smem_bytes(int M, int64_t K, int max_rows, int seg_rows, int nslots) {
  return 1024 + align128(M * gemv_act_row_bytes(K)) + align128(static_cast<int64_t>(max_rows) * (K / 64)) +
         align128(static_cast<int64_t>(max_rows) * (K / 1024) * M * 4) + kGemvFwhtBytes +
         static_cast<int64_t>(nslots) * seg_rows * (K / 4) + 8 * (2 * nslots + 2);
}

template <int M, typename TOut>
__global__ void __launch_bounds__(kGemvThreads, 1) gemv_2bit_kernel(const GemvParams p) {
  extern __shared__ uint8_t smem_raw[];
  const int K = p.K;
  const int C = K / kChunkCodes;     // chunks per row
  const int64_t RB = K / 4;          // packed bytes per row
  const int G = K / 128;
  const int64_t act_bytes = static_cast<int64_t>(M) * gemv_act_row_bytes(K);

  // this CTA's rows
  const int r0 = static_cast<int>((static_cast<int64_t>(p.N) * blockIdx.x) / gridDim.x);
  const int r1 = static_cast<int>((static_cast<int64_t>(p.N) * (blockIdx.x + 1)) / gridDim.x);
  const int nrows = r1 - r0;
  const int nseg = (nrows + p.seg_rows - 1) / p.seg_rows;

  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* act = base;
  __half* sc = reinterpret_cast<__half*>(act + align128(act_bytes));
  float* acc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(sc) +
                                        align128(static_cast<int64_t>(p.max_rows) * (K / 64)));
  float* fsm = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(acc) +
                                        align128(static_cast<int64_t>(p.max_rows) * C * M * 4));
  uint8_t* ring = reinterpret_cast<uint8_t*>(fsm) + kGemvFwhtBytes;
  const int64_t slot_bytes = static_cast<int64_t>(p.seg_rows) * RB;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + p.nslots * slot_bytes);
  uint64_t* empty = full + p.nslots;
  uint64_t* sc_bar = empty + p.nslots;  // this CTA's scales

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nslots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvConsumerWarps);
    }
    mbar_init(sc_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint8_t* src = p.packed + static_cast<int64_t>(r0) * RB;
      const uint32_t sbytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(K / 64);
      mbar_arrive_expect_tx(sc_bar, sbytes);
      bulk_load(sc, p.scales + static_cast<int64_t>(r0) * G, sbytes, sc_bar);
      for (int s = 0; s < nseg; ++s) {
        const int slot = s % p.nslots;
        if (s >= p.nslots && !mbar_wait(&empty[slot], ((s / p.nslots) & 1) ^ 1, FAULT_WAIT_EMPTY)) break;
        const int rows = min(p.seg_rows, nrows - s * p.seg_rows);
        const uint32_t bytes = static_cast<uint32_t>(rows * RB);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_load(ring + slot * slot_bytes, src + static_cast<int64_t>(s) * p.seg_rows * RB, bytes, &full[slot]);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  constexpr int R = M <= 2 ? 2 : 1;           // rows per lane
  constexpr int IR = 4 * R;                   // rows per item
  const int g = lane & 7;                     // 128-group of the chunk this lane owns
  const int rl = lane >> 3;                   // row within each 4-row slice
  pdl_wait();  // x (fused) or the prep kernel's output must be complete
  if (p.fused) {
    // activations of all M tokens: rotation, 16-bit fixed point per 128-group,
    // planes laid out exactly as prep_gemv_kernel writes them
    const int cg = warp >> 2, t = threadIdx.x & 127;
    float* gsm = fsm + cg * 1024;
    const int nblk = K / kHB;
    for (int pi = cg; pi < M * nblk; pi += 4) {
      const int m = pi / nblk, blk = pi - m * nblk;
      const int64_t k0 = static_cast<int64_t>(blk) * kHB + 8 * t;
      float v[8];
      if (p.xt == 0)
        load8<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(p.x) + static_cast<int64_t>(m) * K + k0, v);
      else if (p.xt == 1)
        load8<__half>(static_cast<const __half*>(p.x) + static_cast<int64_t>(m) * K + k0, v);
      else
        load8<float>(static_cast<const float*>(p.x) + static_cast<int64_t>(m) * K + k0, v);
      if (p.signs != nullptr) {
        float dsg[8];
        load_signs8(p.signs + k0, dsg);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= dsg[i];
        fwht1024_group(v, gsm, t, 2 + cg);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] *= kHNorm;
      }
      float mx = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float e = mx / kQMax;
      const float inv = mx > 0.f ? kQMax / mx : 0.f;
      int qs = 0;
      uint8_t* hrow = act + static_cast<int64_t>(m) * gemv_act_row_bytes(K) + static_cast<int64_t>(blk) * kHB;
      const int c = t >> 1, h = t & 1;
      const int wbase = 128 * (c & 7) + 16 * (c >> 3);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int qi = max(-32512, min(32512, __float2int_rn(v[i] * inv)));
        qs += qi;
        const int hi = (qi + 128) >> 8;
        const int lo = qi - (hi << 8);
        const int b = 2 * h + (i >> 2), j = i & 3;
        hrow[wbase + 4 * j + b] = static_cast<uint8_t>(static_cast<int8_t>(hi));
        hrow[K + wbase + 4 * j + b] = static_cast<uint8_t>(static_cast<int8_t>(lo));
      }
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
      if ((t & 15) == 0) {
        int2 inf;
        inf.x = __float_as_int(e);
        inf.y = qs;
        reinterpret_cast<int2*>(act + static_cast<int64_t>(m) * gemv_act_row_bytes(K) + 2 * K)[blk * 8 + (t >> 4)] = inf;
      }
    }
  } else {
    const int64_t n16 = act_bytes / 16;
    for (int64_t i = threadIdx.x; i < n16; i += 32 * kGemvConsumerWarps)
      reinterpret_cast<uint4*>(act)[i] = reinterpret_cast<const uint4*>(p.act)[i];
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kGemvConsumerWarps) : "memory");
  bool ok = mbar_wait(sc_bar, 0, FAULT_WAIT_ACT);
  int item_base = 0;  // number of the first item of the current segment
  for (int s = 0; s < nseg && ok; ++s) {
    const int slot = s % p.nslots;
    const int srow0 = s * p.seg_rows;  // first row of the segment, relative to r0
    const int rows = min(p.seg_rows, nrows - srow0);
    const int nsl = (rows + IR - 1) / IR;  // row slices of IR rows
    const int nitems = nsl * C;
    int first = (warp - item_base) % kGemvConsumerWarps;
    if (first < 0) first += kGemvConsumerWarps;
    // Every warp waits for every segment, even one with no items in it: its
    // release of the slot must count toward this fill of the slot, not a later one.
    if (!mbar_wait(&full[slot], (s / p.nslots) & 1, FAULT_WAIT_FULL)) {
      ok = false;
      break;
    }
    const uint8_t* seg = ring + slot * slot_bytes;
    int sl = first / C;
    int kc = first - sl * C;
    for (int it = first; it < nitems; it += kGemvConsumerWarps) {
      const int grp = kc * 8 + g;  // group index within the row
      const uint8_t* ga = act + kc * kChunkCodes + g * 16;  // word 0 of this group, hi plane, token 0
      int qsum[M];
      float e[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const int2 inf = *reinterpret_cast<const int2*>(act + static_cast<int64_t>(m) * gemv_act_row_bytes(K) +
                                                        2 * K + 8 * grp);
        e[m] = __int_as_float(inf.x);
        qsum[m] = inf.y;
      }
      // rows of this lane (relative to the segment) and their packed words
      int srow[R];
      bool live[R];
      uint4 wv[R][2];
#pragma unroll
      for (int i = 0; i < R; ++i) {
        srow[i] = sl * IR + 4 * i + rl;
        live[i] = srow[i] < rows;
        const uint8_t* wp = seg + static_cast<int64_t>(live[i] ? srow[i] : 0) * RB + kc * 256 + g * 32;
        wv[i][0] = *reinterpret_cast<const uint4*>(wp);
        wv[i][1] = *reinterpret_cast<const uint4*>(wp + 16);
      }
      int dh[R][M][4], dl[R][M][4];
#pragma unroll
      for (int i = 0; i < R; ++i)
#pragma unroll
        for (int m = 0; m < M; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            dh[i][m][j] = 0;
            dl[i][m][j] = 0;
          }
#pragma unroll
      for (int wd = 0; wd < 8; ++wd) {  // 16-code word of the group
        uint4 ahi[M], alo[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const uint8_t* am = ga + static_cast<int64_t>(m) * gemv_act_row_bytes(K);
          ahi[m] = *reinterpret_cast<const uint4*>(am + 128 * wd);
          alo[m] = *reinterpret_cast<const uint4*>(am + K + 128 * wd);
        }
#pragma unroll
        for (int i = 0; i < R; ++i) {
          const uint32_t w = (&wv[i][wd >> 2].x)[wd & 3];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t c = (w >> (2 * j)) & 0x03030303u;
#pragma unroll
            for (int m = 0; m < M; ++m) {
              dh[i][m][j] = dp4a_us(c, (&ahi[m].x)[j], dh[i][m][j]);
              dl[i][m][j] = dp4a_us(c, (&alo[m].x)[j], dl[i][m][j]);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < R; ++i) {
        const float s_rg = live[i] ? __half2float(sc[static_cast<int64_t>(srow0 + srow[i]) * G + grp]) : 0.f;
        float v[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const int hi = (dh[i][m][0] + dh[i][m][1]) + (dh[i][m][2] + dh[i][m][3]);
          const int lo = (dl[i][m][0] + dl[i][m][1]) + (dl[i][m][2] + dl[i][m][3]);
          v[m] = __int2float_rn(hi * 256 + lo - qsum[m]) * (s_rg * e[m]);
          v[m] += __shfl_xor_sync(0xffffffffu, v[m], 1);
          v[m] += __shfl_xor_sync(0xffffffffu, v[m], 2);
          v[m] += __shfl_xor_sync(0xffffffffu, v[m], 4);
        }
        if (live[i] && g < M) {
          float o = v[0];
#pragma unroll
          for (int m = 1; m < M; ++m)
            if (g == m) o = v[m];
          acc[((srow0 + srow[i]) * C + kc) * M + g] = o;
        }
      }
      kc += kGemvConsumerWarps;
      while (kc >= C) {
        kc -= C;
        ++sl;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
    item_base += nitems;
  }
  // all consumer warps done: write this CTA's rows
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kGemvConsumerWarps) : "memory");
  TOut* y = reinterpret_cast<TOut*>(p.y);
  for (int i = threadIdx.x; i < nrows * M; i += 32 * kGemvConsumerWarps) {
    const int lr = i / M, m = i - lr * M;
    float v = 0.f;
    for (int kc = 0; kc < C; ++kc) v += acc[(lr * C + kc) * M + m];
    y[static_cast<int64_t>(m) * p.N + r0 + lr] = from_f32<TOut>(v);
  }
}

}  // namespace tb
