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
// kSegBytes) into a ring of shared-memory slots, and copies all of its scales
// once at the start.  Few, large copies matter: the copy engine's cost is per
// operation, and small boxes capped the stream far below HBM speed.
//
// Compute side: the work of a segment is split into items of (4 rows, one
// 1024-code chunk of K).  Items are numbered across segments and consumer warp
// w takes items w, w + W, ... (W consumer warps), so the split is even for any
// N and K.  Inside an item lane l owns quarter-group l (codes 32l..32l+31) of
// the chunk for all 4 rows, so every activation word it loads serves 4 rows.
// An item's 4 x M partial sums are reduced across the warp with shuffles and
// stored in a per-(row, chunk) slot in shared memory; at the end the chunks of
// each row are summed in a fixed order, so results are bitwise reproducible.
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

struct GemvParams {
  const uint8_t* act;     // prep_gemv output, M rows of gemv_act_row_bytes(K)
  const uint8_t* packed;  // [N, K/4]
  const uint16_t* scales; // [N, K/128] fp16 bits
  void* y;                // [M, N]
  int N;
  int K;
  int seg_rows;           // rows per segment (multiple of 4)
  int nslots;             // ring depth
  int max_rows;           // largest row range of any CTA (sizes the shared buffers)
};

// Shared-memory layout, in order, each part 128-byte aligned:
//   act     M * gemv_act_row_bytes(K)
//   scales  max_rows * K/64 bytes
//   part    max_rows * (K/1024) * M floats
//   ring    nslots * seg_rows * K/4 bytes
//   barriers
__host__ __device__ constexpr int64_t align128(int64_t v) { return (v + 127) & ~int64_t(127); }

__host__ __device__ inline int64_t gemv_smem_bytes(int M, int64_t K, int max_rows, int seg_rows, int nslots) {
  return 1024 + align128(M * gemv_act_row_bytes(K)) + align128(static_cast<int64_t>(max_rows) * (K / 64)) +
         align128(static_cast<int64_t>(max_rows) * (K / 1024) * M * 4) +
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
  uint8_t* ring = reinterpret_cast<uint8_t*>(acc) + align128(static_cast<int64_t>(p.max_rows) * C * M * 4);
  const int64_t slot_bytes = static_cast<int64_t>(p.seg_rows) * RB;
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + p.nslots * slot_bytes);
  uint64_t* empty = full + p.nslots;
  uint64_t* act_bar = empty + p.nslots;  // activations + this CTA's scales

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nslots; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvConsumerWarps);
    }
    mbar_init(act_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kGemvConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint8_t* src = p.packed + static_cast<int64_t>(r0) * RB;
      const uint32_t sbytes = static_cast<uint32_t>(nrows) * static_cast<uint32_t>(K / 64);
      bool act_issued = false;
      for (int s = 0; s < nseg; ++s) {
        const int slot = s % p.nslots;
        if (!act_issued && s == p.nslots) {
          // The first weight segments are in flight; now the activations
          // (written by the previous kernel, hence the grid-dependency wait)
          // and the scales.  Must precede the first wait for a free slot: the
          // consumers need both before they free any slot.
          pdl_wait();
          mbar_arrive_expect_tx(act_bar, static_cast<uint32_t>(act_bytes) + sbytes);
          bulk_load(act, p.act, static_cast<uint32_t>(act_bytes), act_bar);
          bulk_load(sc, p.scales + static_cast<int64_t>(r0) * G, sbytes, act_bar);
          act_issued = true;
        }
        if (s >= p.nslots && !mbar_wait(&empty[slot], ((s / p.nslots) & 1) ^ 1, FAULT_WAIT_EMPTY)) break;
        const int rows = min(p.seg_rows, nrows - s * p.seg_rows);
        const uint32_t bytes = static_cast<uint32_t>(rows * RB);
        mbar_arrive_expect_tx(&full[slot], bytes);
        bulk_load(ring + slot * slot_bytes, src + static_cast<int64_t>(s) * p.seg_rows * RB, bytes, &full[slot]);
      }
      if (!act_issued) {  // fewer segments than slots (or a fault)
        pdl_wait();
        mbar_arrive_expect_tx(act_bar, static_cast<uint32_t>(act_bytes) + sbytes);
        bulk_load(act, p.act, static_cast<uint32_t>(act_bytes), act_bar);
        bulk_load(sc, p.scales + static_cast<int64_t>(r0) * G, sbytes, act_bar);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  bool ok = mbar_wait(act_bar, 0, FAULT_WAIT_ACT);
  int item_base = 0;  // number of the first item of the current segment
  for (int s = 0; s < nseg && ok; ++s) {
    const int slot = s % p.nslots;
    const int srow0 = s * p.seg_rows;  // first row of the segment, relative to r0
    const int rows = min(p.seg_rows, nrows - srow0);
    const int nquads = (rows + kGemvQuadRows - 1) / kGemvQuadRows;
    const int nitems = nquads * C;
    int first = (warp - item_base) % kGemvConsumerWarps;
    if (first < 0) first += kGemvConsumerWarps;
    // Every warp waits for the segment, even one with no items in it: its
    // release of the slot must count toward this fill of the slot, not a later one.
    if (!mbar_wait(&full[slot], (s / p.nslots) & 1, FAULT_WAIT_FULL)) {
      ok = false;
      break;
    }
    if (first < nitems) {
      const uint8_t* seg = ring + slot * slot_bytes;
      for (int it = first; it < nitems; it += kGemvConsumerWarps) {
        const int qd = it / C, kc = it - qd * C;
        const int kq = kc * kChunkCodes + 32 * lane;  // first code of this lane's quarter
        const int lrow0 = srow0 + qd * kGemvQuadRows;  // quad's first row, relative to r0
        const int live = min(kGemvQuadRows, rows - qd * kGemvQuadRows);
        const uint8_t* wq = seg + static_cast<int64_t>(qd * kGemvQuadRows) * RB + kc * 256 + 8 * lane;
        int dhi[kGemvQuadRows][M], dlo[kGemvQuadRows][M];
        float e[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const int2 inf = *reinterpret_cast<const int2*>(act + static_cast<int64_t>(m) * gemv_act_row_bytes(K) +
                                                          2 * K + 8 * (kq >> 5));
          e[m] = __int_as_float(inf.x);
#pragma unroll
          for (int r = 0; r < kGemvQuadRows; ++r) {
            dhi[r][m] = 0;
            dlo[r][m] = -inf.y;
          }
        }
        // two 16-code halves of the quarter; one half's activation words live at a time
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 ahi[M], alo[M];
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const uint8_t* ar = act + static_cast<int64_t>(m) * gemv_act_row_bytes(K);
            ahi[m] = *reinterpret_cast<const uint4*>(ar + kq + 16 * h);
            alo[m] = *reinterpret_cast<const uint4*>(ar + K + kq + 16 * h);
          }
#pragma unroll
          for (int r = 0; r < kGemvQuadRows; ++r) {
            const uint32_t w = r < live ? *reinterpret_cast<const uint32_t*>(wq + r * RB + 4 * h) : 0x55555555u;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t c = (w >> (2 * j)) & 0x03030303u;
#pragma unroll
              for (int m = 0; m < M; ++m) {
                dhi[r][m] = dp4a_us(c, (&ahi[m].x)[j], dhi[r][m]);
                dlo[r][m] = dp4a_us(c, (&alo[m].x)[j], dlo[r][m]);
              }
            }
          }
        }
        float part[kGemvQuadRows][M];
#pragma unroll
        for (int r = 0; r < kGemvQuadRows; ++r) {
          const float s_rg = r < live ? __half2float(sc[static_cast<int64_t>(lrow0 + r) * G + kc * 8 + (lane >> 2)])
                                      : 0.f;
#pragma unroll
          for (int m = 0; m < M; ++m) part[r][m] = __int2float_rn(dhi[r][m] * 256 + dlo[r][m]) * (s_rg * e[m]);
        }
        // reduce the item's partials across the warp; lane r*M + m adds (row r, token m)
        float mine = 0.f;
#pragma unroll
        for (int r = 0; r < kGemvQuadRows; ++r) {
#pragma unroll
          for (int m = 0; m < M; ++m) {
            float v = part[r][m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == r * M + m) mine = v;
          }
        }
        if (lane < kGemvQuadRows * M && qd * kGemvQuadRows + lane / M < rows)
          acc[((lrow0 + lane / M) * C + kc) * M + (lane % M)] = mine;
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
