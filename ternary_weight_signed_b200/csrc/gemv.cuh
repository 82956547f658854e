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
// Layout of work: a persistent grid, one CTA per SM.  CTA c takes a contiguous
// range of row quads (4 rows).  A stage is up to 8 quads x one 1024-code chunk
// of K (1 KB of packed codes + 64 B of scales per quad), brought in by two 2-D
// TMA boxes per quad into a ring of shared-memory stages.  Warp 8 is the
// producer; warps 0..7 each own one quad of the stage, and lane l owns
// quarter-group l (codes 32l..32l+31) of the chunk, for all 4 rows of the quad,
// so each activation word it loads serves 4 rows.  At the end of a quad's K
// the 4 x M partial sums are reduced across the warp with shuffles.
#pragma once
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGemvConsumerWarps = 8;
constexpr int kGemvThreads = 32 * (kGemvConsumerWarps + 1);
constexpr int kGemvQuadRows = 4;
constexpr int kGemvMaxM = 4;
constexpr int kChunkCodes = 1024;                 // K per stage
constexpr int kQuadWBytes = kGemvQuadRows * 256;  // 2-bit codes of 4 rows x 1024
constexpr int kQuadSBytes = kGemvQuadRows * 16;   // 8 fp16 scales x 4 rows
// A tiled TMA box must land on a 128-byte aligned shared-memory address, so
// every quad's 64 bytes of scales get a 128-byte slot.
constexpr int kQuadSSlot = 128;
constexpr int kStageBytes = kGemvConsumerWarps * (kQuadWBytes + kQuadSSlot);  // 9216

struct GemvParams {
  const uint8_t* act;  // prep_gemv output, M rows of gemv_act_row_bytes(K)
  void* y;             // [M, N]
  int N;
  int K;
  int nquads;          // ceil(N / 4)
  int nstages;         // ring depth
};

template <int M>
struct ActWords {
  uint4 hi[M][2];
  uint4 lo[M][2];
  float e[M];
  int qs[M];
};

template <int M, typename TOut>
__global__ void __launch_bounds__(kGemvThreads, 1)
    gemv_2bit_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                     const GemvParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const int K = p.K;
  const int kchunks = K / kChunkCodes;
  const int64_t act_bytes = static_cast<int64_t>(M) * gemv_act_row_bytes(K);
  // 1024-byte aligned base (the launch reserves 1 KB of slack for this)
  uint8_t* act = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
  uint8_t* ring = act + ((act_bytes + 1023) & ~int64_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + static_cast<int64_t>(p.nstages) * kStageBytes);
  uint64_t* empty = full + p.nstages;
  uint64_t* act_bar = empty + p.nstages;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // contiguous quad range of this CTA
  const int q_begin = static_cast<int>((static_cast<int64_t>(p.nquads) * blockIdx.x) / gridDim.x);
  const int q_end = static_cast<int>((static_cast<int64_t>(p.nquads) * (blockIdx.x + 1)) / gridDim.x);
  const int nblocks = (q_end - q_begin + kGemvConsumerWarps - 1) / kGemvConsumerWarps;
  const int total_stages = nblocks * kchunks;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
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
      prefetch_tensormap(&tm_w);
      prefetch_tensormap(&tm_s);
      bool act_issued = false;
      for (int i = 0; i < total_stages; ++i) {
        const int slot = i % p.nstages;
        if (!act_issued && i == p.nstages) {
          // The weights of the first stages are in flight; now the
          // activations, which the previous kernel (prep) writes.  This must
          // come before the first wait on a free slot: the consumers need the
          // activations before they free any slot.
          pdl_wait();
          mbar_arrive_expect_tx(act_bar, static_cast<uint32_t>(act_bytes));
          bulk_load(act, p.act, static_cast<uint32_t>(act_bytes), act_bar);
          act_issued = true;
        }
        if (i >= p.nstages) {
          if (!mbar_wait(&empty[slot], ((i / p.nstages) & 1) ^ 1, FAULT_WAIT_EMPTY)) break;
        }
        const int blk = i / kchunks, kc = i % kchunks;
        const int q0 = q_begin + blk * kGemvConsumerWarps;
        const int nq = min(kGemvConsumerWarps, q_end - q0);
        uint8_t* st = ring + static_cast<int64_t>(slot) * kStageBytes;
        mbar_arrive_expect_tx(&full[slot], static_cast<uint32_t>(nq * (kQuadWBytes + kQuadSBytes)));
        for (int q = 0; q < nq; ++q) {
          const int row0 = (q0 + q) * kGemvQuadRows;
          tma_load_2d(st + q * kQuadWBytes, &tm_w, kc * 64, row0, &full[slot]);
          tma_load_2d(st + kGemvConsumerWarps * kQuadWBytes + q * kQuadSSlot, &tm_s, kc * 8, row0,
                      &full[slot]);
        }
      }
      if (!act_issued) {  // fewer stages than the ring holds (or a fault)
        pdl_wait();
        mbar_arrive_expect_tx(act_bar, static_cast<uint32_t>(act_bytes));
        bulk_load(act, p.act, static_cast<uint32_t>(act_bytes), act_bar);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  if (!mbar_wait(act_bar, 0, FAULT_WAIT_ACT)) return;
  float acc[kGemvQuadRows][M];
#pragma unroll
  for (int r = 0; r < kGemvQuadRows; ++r)
#pragma unroll
    for (int m = 0; m < M; ++m) acc[r][m] = 0.f;

  for (int i = 0; i < total_stages; ++i) {
    const int slot = i % p.nstages;
    const int blk = i / kchunks, kc = i % kchunks;
    const int q0 = q_begin + blk * kGemvConsumerWarps;
    const int nq = min(kGemvConsumerWarps, q_end - q0);
    if (!mbar_wait(&full[slot], (i / p.nstages) & 1, FAULT_WAIT_FULL)) return;
    const uint8_t* st = ring + static_cast<int64_t>(slot) * kStageBytes;
    if (warp < nq) {
      // activations of this lane's quarter-group for every token
      ActWords<M> a;
      const int kq = kc * kChunkCodes + 32 * lane;  // first code of the quarter
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const uint8_t* ar = act + static_cast<int64_t>(m) * gemv_act_row_bytes(K);
        a.hi[m][0] = *reinterpret_cast<const uint4*>(ar + kq);
        a.hi[m][1] = *reinterpret_cast<const uint4*>(ar + kq + 16);
        a.lo[m][0] = *reinterpret_cast<const uint4*>(ar + K + kq);
        a.lo[m][1] = *reinterpret_cast<const uint4*>(ar + K + kq + 16);
        const int2 inf = *reinterpret_cast<const int2*>(ar + 2 * K + 8 * (kq >> 5));
        a.e[m] = __int_as_float(inf.x);
        a.qs[m] = inf.y;
      }
      const uint8_t* wq = st + warp * kQuadWBytes;
      const __half* sq = reinterpret_cast<const __half*>(st + kGemvConsumerWarps * kQuadWBytes +
                                                         warp * kQuadSSlot);
#pragma unroll
      for (int r = 0; r < kGemvQuadRows; ++r) {
        const uint2 w2 = *reinterpret_cast<const uint2*>(wq + r * 256 + 8 * lane);
        const float sc = __half2float(sq[r * 8 + (lane >> 2)]);
        int dhi[M], dlo[M];
#pragma unroll
        for (int m = 0; m < M; ++m) {
          dhi[m] = 0;
          dlo[m] = -a.qs[m];
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t w = h ? w2.y : w2.x;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t c = (w >> (2 * j)) & 0x03030303u;
#pragma unroll
            for (int m = 0; m < M; ++m) {
              const uint32_t ah = (&a.hi[m][h].x)[j];
              const uint32_t al = (&a.lo[m][h].x)[j];
              dhi[m] = dp4a_us(c, ah, dhi[m]);
              dlo[m] = dp4a_us(c, al, dlo[m]);
            }
          }
        }
#pragma unroll
        for (int m = 0; m < M; ++m) {
          const int pq = dhi[m] * 256 + dlo[m];
          acc[r][m] = fmaf(__int2float_rn(pq), sc * a.e[m], acc[r][m]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);

    if (kc == kchunks - 1) {
      if (warp < nq) {
        // reduce across the warp; lane r*M + m writes (row r, token m)
        float out = 0.f;
#pragma unroll
        for (int r = 0; r < kGemvQuadRows; ++r) {
#pragma unroll
          for (int m = 0; m < M; ++m) {
            float v = acc[r][m];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == r * M + m) out = v;
            acc[r][m] = 0.f;
          }
        }
        const int row = (q0 + warp) * kGemvQuadRows + lane / M;
        const int m = lane % M;
        if (lane < kGemvQuadRows * M && row < p.N) {
          TOut* y = reinterpret_cast<TOut*>(p.y);
          y[static_cast<int64_t>(m) * p.N + row] = from_f32<TOut>(out);
        }
      }
    }
  }
}

}  // namespace tb
