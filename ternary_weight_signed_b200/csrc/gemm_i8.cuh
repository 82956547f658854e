// Integer-mode GEMM on the 5th-generation tensor cores (tcgen05 kind::i8,
// int32 accumulators in TMEM): y[m, n] = sum_k t[n, k] x[m, k] for int8 x,
// exact (a ternary product is an add, a subtract or nothing: ai4coding.ru,
// "What is a ternary model", last paragraph; no rotation, no scales).
//
// The weights enter the MMA as their biased codes, so no per-byte subtract is
// needed in the unpack:
//   2-bit : c = t + 1 in {0, 1, 2}, sum_k t x = sum_k c x - X[m];
//   1-bit : b in {0, 1} with t = 2 b - 1, sum_k t x = 2 sum_k b x - X[m];
// X[m] = sum_k x[m, k] is summed by the unpack threads from the x tiles as
// they arrive (one token row per thread, dp4a against 0x01010101) and applied
// in the epilogue.  |sum c x| <= 2 * 127 * K < 2^31 for K < 8.4 M.
//
// Tile: BM tokens x BN weight rows (BM = 256 or 128; BN = 128, 192 or 256),
// K in stages of 128 (one 128-byte swizzle atom of int8).  A = x straight from
// the caller's buffer by TMA (128-byte swizzle); B = the codes of the stage as
// bytes in natural k order, written by the unpack threads in the UMMA K-major
// 128-byte swizzled layout; four MMAs of K = 32 per stage.
// Warp roles as in the fp16 GEMM: warp 0 TMA, warp 1 TMEM allocation and the
// MMA-issuing thread, warps 2-9 unpack + x sums + epilogue.
//
// Every wait is bounded; after a timeout a role stops waiting, records a fault
// word and still reaches the final barrier so TMEM is always freed.
#pragma once
#include "gemm_tc.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGi8BK = 128;  // codes (bytes of x) per stage
__host__ __device__ constexpr int gi8_a_bytes(int bm) { return bm * kGi8BK; }
__host__ __device__ constexpr int gi8_b_bytes(int bn) { return bn * kGi8BK; }
// packed bytes of a weight row per stage: 32 (2-bit), 16 (1-bit)
__host__ __device__ constexpr int gi8_w_row_bytes(int fmt) { return fmt == 2 ? 16 : 32; }
__host__ __device__ constexpr int gi8_stage_bytes(int bm, int bn, int fmt) {
  return gi8_a_bytes(bm) + gi8_b_bytes(bn) + bn * gi8_w_row_bytes(fmt);
}
__host__ __device__ constexpr int gi8_stages(int bm, int bn, int fmt) {
  return (kGemmSmemCap - 1024 - 2048) / gi8_stage_bytes(bm, bn, fmt) < 8
             ? (kGemmSmemCap - 1024 - 2048) / gi8_stage_bytes(bm, bn, fmt)
             : 8;
}
// stages, 1 KB alignment slack, 1 KB of x sums, barriers
__host__ __device__ constexpr int gi8_smem_bytes(int bm, int bn, int fmt) {
  return gi8_stages(bm, bn, fmt) * gi8_stage_bytes(bm, bn, fmt) + 1024 + 1024 + 1024;
}

// kind::i8: D s32 (bits 4-5 = 2), A s8 (bits 7-9 = 1), B u8 (bits 10-12 = 0),
// both K-major, N >> 3 at bits 17-22, M = 128 (M >> 4 at bits 24-28).
__host__ __device__ constexpr uint32_t gi8_idesc(int bn) {
  return (2u << 4) | (1u << 7) | (static_cast<uint32_t>(bn >> 3) << 17) | (static_cast<uint32_t>(kGemmUM >> 4) << 24);
}

__device__ __forceinline__ void umma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 codes of a 2-bit word (code u in bits 2u) as 16 bytes c_u = t_u + 1 in
// natural order: the masks m_j = (w >> 2j) & 0x03030303 hold c_{4b+j} in byte
// b; a 4 x 4 byte transpose (eight byte permutes) gives (c_{4b}, .., c_{4b+3}).
__device__ __forceinline__ uint4 gi8_codes16(uint32_t w) {
  const uint32_t m0 = w & 0x03030303u, m1 = (w >> 2) & 0x03030303u, m2 = (w >> 4) & 0x03030303u,
                 m3 = (w >> 6) & 0x03030303u;
  const uint32_t a_lo = __byte_perm(m0, m1, 0x5140), a_hi = __byte_perm(m0, m1, 0x7362);  // c0 c1 c4 c5 | c8 ..
  const uint32_t b_lo = __byte_perm(m2, m3, 0x5140), b_hi = __byte_perm(m2, m3, 0x7362);  // c2 c3 c6 c7 | c10 ..
  return make_uint4(__byte_perm(a_lo, b_lo, 0x5410), __byte_perm(a_lo, b_lo, 0x7632), __byte_perm(a_hi, b_hi, 0x5410),
                    __byte_perm(a_hi, b_hi, 0x7632));
}

// Four 1-bit codes (bits 4r .. 4r + 3 of w) as four bytes b in {0, 1}: the
// product with 0x00204081 places bit i of the nibble at bit 8 i (the four
// shifted copies occupy disjoint bit ranges, so nothing carries).
__device__ __forceinline__ uint32_t gi8_bits4(uint32_t w, int r) {
  return (((w >> (4 * r)) & 0xFu) * 0x00204081u) & 0x01010101u;
}

struct GemmI8Params {
  int M, N, K;
  int32_t* y;  // [M, N]
};

template <int BM, int BN, int kFmt>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_i8_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const GemmI8Params p) {
  static_assert(BN % 32 == 0 && BN >= 128 && BN <= kGemmBN, "weight tile width");
  static_assert(BM == 128 || BM == 256, "token tile");
  static_assert(kFmt == 0 || kFmt == 2, "2-bit or 1-bit codes");
  constexpr int kA = gi8_a_bytes(BM), kB = gi8_b_bytes(BN), kWr = gi8_w_row_bytes(kFmt);
  constexpr int kW = BN * kWr, kStage = gi8_stage_bytes(BM, BN, kFmt), kStages = gi8_stages(BM, BN, kFmt);
  static_assert(kStages >= 2, "two stages at least");
  constexpr uint32_t kIdesc = gi8_idesc(BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int* xsum = reinterpret_cast<int*>(smem + kStages * kStage);  // [256] token sums
  uint64_t* full = reinterpret_cast<uint64_t*>(xsum + 256);
  uint64_t* bready = full + kStages;
  uint64_t* empty = bready + kStages;
  uint64_t* accum = empty + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = p.K / kGi8BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&bready[s], kGemmUnpackWarps);
      mbar_init(&empty[s], 1);
    }
    mbar_init(accum, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kGemmTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_w);
      pdl_wait();  // x may be the previous kernel's output
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kStages;
        if (kb >= kStages && !mbar_wait(&empty[s], ((kb / kStages) & 1) ^ 1, FAULT_WAIT_EMPTY)) break;
        uint8_t* st = smem + s * kStage;
        mbar_arrive_expect_tx(&full[s], kA + kW);
        tma_load_2d(st, &tm_x, kb * kGi8BK, m0, &full[s]);
        tma_load_2d(st + kA + kB, &tm_w, kb * (kWr / 4), n0, &full[s]);  // x in 32-bit words
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kStages;
        const uint32_t par = (kb / kStages) & 1;
        ok = mbar_wait(&full[s], par, FAULT_WAIT_FULL) && mbar_wait(&bready[s], par, FAULT_WAIT_FULL);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * kStage);
        const uint32_t b = a + kA;
#pragma unroll
        for (int kk = 0; kk < kGi8BK / 32; ++kk) {
          const uint64_t bd = umma_desc_sw128(b + 32 * kk);
          const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
          umma_i8(tmem, umma_desc_sw128(a + 32 * kk), bd, kIdesc, acc);
          if constexpr (BM == 256) umma_i8(tmem + BN, umma_desc_sw128(a + kGemmUM * 128 + 32 * kk), bd, kIdesc, acc);
        }
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
    }
  } else {
    // ------------------------------------------------- unpack + token sums
    const int r = threadIdx.x - 64;  // weight row (unpack) and token row (x sum) of the tile, 0..255
    const bool in_tile = r < BN;
    const bool x_row = r < BM;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    int xs = 0;
    bool ok = true;
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kStages;
      if (!mbar_wait(&full[s], (kb / kStages) & 1, FAULT_WAIT_FULL)) {
        ok = false;
        break;
      }
      uint8_t* st = smem + s * kStage;
      if (in_tile) {
        uint8_t* row = st + kA + r * 128;
        const uint8_t* wrow = st + kA + kB + r * kWr;
        if constexpr (kFmt == 0) {
          // 128 codes = 8 words of 16; word q -> 16-byte chunk q
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint4 w4 = *reinterpret_cast<const uint4*>(wrow + 16 * h);
            const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<uint4*>(row + 16 * ((4 * h + q) ^ sw)) = gi8_codes16(w[q]);
          }
        } else {
          // 128 codes = 4 words of 32; chunk q holds codes 16 q .. 16 q + 15
          const uint4 w4 = *reinterpret_cast<const uint4*>(wrow);
          const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t wd = w[q >> 1];
            const int r0 = 4 * (q & 1);
            *reinterpret_cast<uint4*>(row + 16 * (q ^ sw)) =
                make_uint4(gi8_bits4(wd, r0), gi8_bits4(wd, r0 + 1), gi8_bits4(wd, r0 + 2), gi8_bits4(wd, r0 + 3));
          }
        }
      }
      if (x_row) {
        // token row r of the x tile: 128 bytes (swizzled chunks; the sum does
        // not care).  Chunk q ^ (r & 7) at step q: the eight rows of a
        // quarter-warp read eight different 16-byte bank groups.
        const uint4* xr = reinterpret_cast<const uint4*>(st + r * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const uint4 v = xr[q ^ (r & 7)];
          xs = __dp4a(static_cast<int>(v.x), 0x01010101, xs);
          xs = __dp4a(static_cast<int>(v.y), 0x01010101, xs);
          xs = __dp4a(static_cast<int>(v.z), 0x01010101, xs);
          xs = __dp4a(static_cast<int>(v.w), 0x01010101, xs);
        }
      }
      fence_proxy_async_shared();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&bready[s]);
    }
    if (x_row) xsum[r] = xs;
    asm volatile("bar.sync 1, 256;" ::: "memory");  // the 8 unpack warps: token sums visible
    // ---------------------------------------------------------------- epilogue
    // wait for the accumulator even after a failed stage wait: the MMAs
    // issued so far must be complete before TMEM is freed
    if (mbar_wait(accum, 0, FAULT_WAIT_EPILOGUE) && ok) {
      tc_fence_after();
      const int q = warp & 3;
      const int h = (warp - 2) >> 2;
      const int ml = (BM == 256 ? kGemmUM * h : 0) + 32 * q + lane;  // token row in the tile
      const int m = m0 + ml;
      const int xm = ml < BM ? xsum[ml] : 0;
      const bool vec = (p.N % 4) == 0;
      constexpr int kCols = BM == 256 ? BN / 32 : BN / 64;
#pragma unroll 1
      for (int cc = 0; cc < kCols; ++cc) {
        const int c = BM == 256 ? cc : h * kCols + cc;
        uint32_t v32[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) +
                      static_cast<uint32_t>((BM == 256 ? BN * h : 0) + 32 * c),
                  v32);
        tmem_ld_wait();
        const int nb = n0 + 32 * c;
        if (m < p.M && nb < p.N) {
          const int valid = min(32, p.N - nb);
          int32_t* dst = p.y + static_cast<int64_t>(m) * p.N + nb;
          int32_t o[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            o[j] = (kFmt == 0 ? static_cast<int32_t>(v32[j]) : 2 * static_cast<int32_t>(v32[j])) - xm;
          if (vec && valid == 32) {
#pragma unroll
            for (int j = 0; j < 8; ++j)
              reinterpret_cast<int4*>(dst)[j] = make_int4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j < valid) dst[j] = o[j];
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGemmTmemCols);
  }
}

}  // namespace tb
