// Prefill GEMM on the 5th-generation tensor cores (tcgen05 + TMEM), 2-bit
// slot format (and 1-bit g128, unpacked the same way to exact fp16 s*t with
// t = -1 or +1).
//
// y[m, n] = sum_k x'[m, k] * w[n, k],  w = s[n, k/128] * t[n, k]  (ternary
// g128: news.ditty.ir, second paragraph).  Once unpacked the product is a dense
// contraction, so it runs as kind::f16 MMAs with fp32 accumulators in TMEM:
//   A = x' in fp16 (rotated activations, written by the prep kernel), and
//   B = fp16(s * t), which is exact because t is -1, 0 or +1 and s is an fp16
//       value, so no per-group rescaling of the accumulator is needed.
//
// Tile: BM tokens x BN weight rows (BM = 256 or 128; BN = 128, 192 or 256,
// chosen per shape), K in stages of 64 (one 128-byte swizzle atom of fp16).
// With BM = 256 the tokens are two M=128 MMAs that share the unpacked B tile,
// each with its own 128 x BN fp32 accumulator in TMEM; BM = 128 (few tokens)
// is one MMA and one accumulator.
// Warp roles:
//   warp 0    : TMA producer (x' tile with 128B swizzle, packed 2-bit codes);
//   warp 1    : TMEM allocation and the single thread issuing tcgen05.mma;
//   warps 2-9 : unpack the codes of the stage into fp16 s*t (one weight row
//               per thread), written straight into the UMMA K-major
//               128B-swizzled layout, then the epilogue (tcgen05.ld of the
//               accumulators, convert, store).
//
// Unpacking: the 2-bit word of 16 codes holds codes j and j+8 at bits 2j and
// 2j+16.  For j < 4, ((w >> 2j) & 0x00030003) | 0x64006400 is the fp16 pair
// (1024 + c_j, 1024 + c_{j+8}); for j >= 4 the same shifted word with mask
// 0x03000300 gives 1024 + 256 c.  One fma (v - 1024 or v/256 - 4) gives c
// exactly and one more gives s*c - s = s*t (exact).  That pairs k = j with
// k = j+8 in each half2, so the prep kernel
// stores x' with the same order inside every 16-element chunk
// (k = 0, 8, 1, 9, ..., 7, 15); the contraction over k does not depend on the
// order as long as both operands share it.
//
// Every wait is bounded; after a timeout a role stops waiting, records a fault
// word and still reaches the final barrier so TMEM is always freed.
#pragma once
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGemmBM = 256;      // tokens per tile at most: two MMAs of M = 128
constexpr int kGemmUM = 128;      // M of one MMA (TMEM lanes)
constexpr int kGemmBN = 256;     // widest weight tile
constexpr int kGemmBK = 64;
constexpr int kGemmSmemCap = 227 * 1024;  // dynamic shared memory of one CTA at most
constexpr int kGemmUnpackWarps = 8;
constexpr int kGemmThreads = 32 * (2 + kGemmUnpackWarps);
constexpr int kGemmTmemCols = 512;
// per tile (BM tokens, BN weight rows): A (fp16 x') and the packed codes of a
// stage come by TMA into a ring of stages; B (fp16 s*t, written by the unpack
// warps) has a ring of its own of kGemmBSlots buffers, so the copies run as
// far ahead as the stage ring allows while the unpack works one stage ahead of
// the MMAs.
constexpr int kGemmBSlots = 2;
__host__ __device__ constexpr int gemm_a_bytes(int bm) { return bm * kGemmBK * 2; }
__host__ __device__ constexpr int gemm_b_bytes(int bn) { return bn * kGemmBK * 2; }
__host__ __device__ constexpr int gemm_w_bytes(int bn) { return bn * kGemmBK / 4; }
__host__ __device__ constexpr int gemm_stage_bytes(int bm, int bn) {
  return gemm_a_bytes(bm) + gemm_w_bytes(bn);
}
// As many stages as fit (at most 8): small tiles have little MMA work per
// stage, so more stages are in flight to cover the copies' latency.
__host__ __device__ constexpr int gemm_stages(int bm, int bn) {
  return (kGemmSmemCap - 1024 - 256 - kGemmBSlots * gemm_b_bytes(bn)) / gemm_stage_bytes(bm, bn) < 8
             ? (kGemmSmemCap - 1024 - 256 - kGemmBSlots * gemm_b_bytes(bn)) / gemm_stage_bytes(bm, bn)
             : 8;
}
__host__ __device__ constexpr int gemm_smem_bytes(int bm, int bn) {
  return gemm_stages(bm, bn) * gemm_stage_bytes(bm, bn) + kGemmBSlots * gemm_b_bytes(bn) + 1024 /*align*/ +
         256 /*barriers*/;
}

// Instruction descriptor, kind::f16: D fp32 (bits 4-5 = 1), A and B fp16
// (bits 7-9, 10-12 = 0), both K-major (bits 15, 16 = 0), N >> 3 at bits 17-22,
// M >> 4 at bits 24-28.
__host__ __device__ constexpr uint32_t gemm_idesc(int bn) {
  return (1u << 4) | (static_cast<uint32_t>(bn >> 3) << 17) | (static_cast<uint32_t>(kGemmUM >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major operand in the canonical
// 128-byte swizzled layout: rows of 128 bytes, 8-row groups 1024 bytes apart
// (stride byte offset), start address >> 4 in bits 0-13, leading byte offset
// 16 (unused for this layout), version 1 at bit 46, swizzle mode 2 (128B) at
// bits 61-63.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on `bar` once all tcgen05 operations issued so far by this thread complete.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Activation prep for this kernel: rotation (when signs is non-null) and fp16
// store in the paired order above.  grid (M, K/1024), 128 threads.
template <typename TIn>
__global__ void __launch_bounds__(kHThreads) prep_gemm_kernel(const TIn* __restrict__ x,
                                                              const int8_t* __restrict__ signs,
                                                              __half* __restrict__ out, int64_t K) {
  __shared__ float sm[kHB];
  pdl_launch_dependents();
  const int64_t row = blockIdx.x;
  const int blk = blockIdx.y;
  float v[8];
  load_rotated8<TIn>(x, signs, row, blk, K, v, sm);
  // thread pair (2c, 2c+1) holds the 16-element chunk c; exchange halves
  const bool upper = (threadIdx.x & 1) != 0;
  float u[4], p[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) u[i] = upper ? v[i] : v[4 + i];
#pragma unroll
  for (int i = 0; i < 4; ++i) p[i] = __shfl_xor_sync(0xffffffffu, u[i], 1);
  float o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    o[2 * i] = upper ? p[i] : v[i];
    o[2 * i + 1] = upper ? v[4 + i] : p[i];
  }
  store8<__half>(out + row * K + static_cast<int64_t>(blk) * kHB + 8 * threadIdx.x, o);
}

struct GemmParams {
  int M, N, K;
  void* y;
  const uint16_t* scales;  // [N, K/128] fp16 bits
};

template <typename TOut>
__device__ __forceinline__ void store_row32(TOut* dst, const uint32_t (&r)[32], int valid, bool vec);

template <>
__device__ __forceinline__ void store_row32<float>(float* dst, const uint32_t (&r)[32], int valid, bool vec) {
  if (vec && valid == 32) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      reinterpret_cast<float4*>(dst)[j] =
          make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]), __uint_as_float(r[4 * j + 2]),
                      __uint_as_float(r[4 * j + 3]));
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < valid) dst[j] = __uint_as_float(r[j]);
  }
}

template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16* dst, const uint32_t (&r)[32], int valid,
                                                           bool vec) {
  if (vec && valid == 32) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint4 u;
      __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        h[e] = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 2 * e]), __uint_as_float(r[8 * j + 2 * e + 1]));
      reinterpret_cast<uint4*>(dst)[j] = u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < valid) dst[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
  }
}

// kFmt: 0 = 2-bit slots (16 bytes of a row per 64-code stage), 2 = 1-bit (16
// bytes per 128 codes: the box of an even stage also carries the codes of the
// odd stage after it, which the unpack threads keep in registers).
template <int BM, int BN, typename TOut, int kFmt>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                   const GemmParams p) {
  static_assert(kFmt == 0 || kFmt == 2, "2-bit or 1-bit codes");
  static_assert(BN % 32 == 0 && BN >= 128 && BN <= kGemmBN, "weight tile width");
  static_assert(BM == 128 || BM == 256, "token tile");
  constexpr int kA = gemm_a_bytes(BM), kStage = gemm_stage_bytes(BM, BN), kB = gemm_b_bytes(BN),
                kW = gemm_w_bytes(BN), kGemmStages = gemm_stages(BM, BN);
  static_assert(kGemmStages >= 2, "two stages at least");
  constexpr uint32_t kIdesc = gemm_idesc(BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* bring = smem + kGemmStages * kStage;  // kGemmBSlots x kB, 1 KB aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(bring + kGemmBSlots * kB);
  uint64_t* empty = full + kGemmStages;
  uint64_t* bfull = empty + kGemmStages;
  uint64_t* bempty = bfull + kGemmBSlots;
  uint64_t* accum = bempty + kGemmBSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM;
  const int nk = p.K / kGemmBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kGemmUnpackWarps);  // the MMAs read A, the unpack warps read the codes
    }
    for (int b = 0; b < kGemmBSlots; ++b) {
      mbar_init(&bfull[b], kGemmUnpackWarps);
      mbar_init(&bempty[b], 1);
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
      pdl_wait();  // x' comes from the prep kernel
      const bool stall = test_stall_copies();  // failure-detection test: no copies
      for (int kb = 0; kb < nk && !stall; ++kb) {
        const int s = kb % kGemmStages;
        if (kb >= kGemmStages &&
            !mbar_wait(&empty[s], ((kb / kGemmStages) & 1) ^ 1, FAULT_WAIT_EMPTY))
          break;
        uint8_t* st = smem + s * kStage;
        const bool wload = kFmt == 0 || (kb & 1) == 0;
        mbar_arrive_expect_tx(&full[s], kA + (wload ? kW : 0));
        tma_load_2d(st, &tm_x, kb * kGemmBK, m0, &full[s]);
        // x in 32-bit words: 2-bit, 4 words per stage; 1-bit, 4 words per two stages
        if (wload) tma_load_2d(st + kA, &tm_w, kFmt == 0 ? kb * 4 : (kb >> 1) * 4, n0, &full[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % kGemmStages, bs = kb % kGemmBSlots;
        const uint32_t par = (kb / kGemmStages) & 1;
        ok = mbar_wait(&full[s], par, FAULT_WAIT_FULL) &&
             mbar_wait(&bfull[bs], (kb / kGemmBSlots) & 1, FAULT_WAIT_FULL);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * kStage);
        const uint32_t b = smem_u32(bring + bs * kB);
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 16; ++kk) {
          const uint64_t bd = umma_desc_sw128(b + 32 * kk);
          const uint32_t acc = (kb | kk) != 0 ? 1u : 0u;
          umma_f16(tmem, umma_desc_sw128(a + 32 * kk), bd, kIdesc, acc);
          if constexpr (BM == 256)
            umma_f16(tmem + BN, umma_desc_sw128(a + kGemmUM * 128 + 32 * kk), bd, kIdesc, acc);
        }
        umma_commit(&empty[s]);
        umma_commit(&bempty[bs]);
      }
      umma_commit(accum);
    }
  } else {
    // ---------------------------------------------------------------- unpack
    const int r = threadIdx.x - 64;  // weight row of the tile this thread unpacks (0..255)
    const bool in_tile = r < BN;     // threads past the tile width only take part in the barriers
    const int G = p.K / 128;
    const int n = n0 + r;
    const bool row_ok = in_tile && n < p.N;
    const uint16_t* srow = p.scales + static_cast<int64_t>(row_ok ? n : 0) * G;
    __half s_next = __ushort_as_half(row_ok ? srow[0] : uint16_t(0));
    __half s_cur = s_next;
    const uint32_t sw = static_cast<uint32_t>(r & 7);
    const __half2 k1024 = __float2half2_rn(1024.f);
    const __half2 k1 = __float2half2_rn(1.f);
    const __half2 kinv256 = __float2half2_rn(1.f / 256.f);
    const __half2 km4 = __float2half2_rn(-4.f);
    uint32_t wcur[2] = {0u, 0u}, wnext[2] = {0u, 0u};  // 1-bit codes of this and the next stage
    bool ok = true;
    for (int kb = 0; kb < nk && ok; ++kb) {
      const int s = kb % kGemmStages, bs = kb % kGemmBSlots;
      if (!mbar_wait(&full[s], (kb / kGemmStages) & 1, FAULT_WAIT_FULL)) {
        ok = false;
        break;
      }
      if ((kb & 1) == 0) {  // a new 128-group starts: take its scale, prefetch the next
        const int g = kb >> 1;
        s_cur = s_next;
        if (g + 1 < G) s_next = __ushort_as_half(row_ok ? srow[g + 1] : uint16_t(0));
      }
      uint8_t* st = smem + s * kStage;
      // this stage's codes into registers; then the stage's slot is free as
      // far as the unpack is concerned
      uint4 w4 = make_uint4(0, 0, 0, 0);
      if (in_tile && (kFmt == 0 || (kb & 1) == 0)) w4 = *reinterpret_cast<const uint4*>(st + kA + r * 16);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      // the MMAs of stage kb - kGemmBSlots are done with this B buffer
      if (kb >= kGemmBSlots && !mbar_wait(&bempty[bs], ((kb / kGemmBSlots) & 1) ^ 1, FAULT_WAIT_EMPTY)) {
        ok = false;
        break;
      }
      const __half2 s2 = __halves2half2(s_cur, s_cur);
      const __half2 ns2 = __hneg2(s2);
      uint8_t* row = bring + bs * kB + r * 128;
      if constexpr (kFmt == 2) {
        // 1-bit: 16-code chunk c of the stage (c = 0..3) is half c & 1 of
        // word c >> 1.  z holds its low 8 codes in bits 0-7 and its high 8 in
        // bits 16-23; (z << (15 - j)) & 0x80008000 puts codes j and j + 8 on
        // the sign bits of a half2, and XOR with (-s, -s) gives (s t_j, s t_{j+8}).
        if ((kb & 1) == 0 && in_tile) {
          wcur[0] = w4.x;
          wcur[1] = w4.y;
          wnext[0] = w4.z;
          wnext[1] = w4.w;
        } else if (in_tile) {
          wcur[0] = wnext[0];
          wcur[1] = wnext[1];
        }
        const uint32_t nb = *reinterpret_cast<const uint32_t*>(&ns2);
#pragma unroll
        for (int c = 0; c < 4 && in_tile; ++c) {
          const uint32_t z = __byte_perm(wcur[c >> 1], 0u, (c & 1) ? 0x4342u : 0x4140u);
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) o[j] = ((z << (15 - j)) & 0x80008000u) ^ nb;
          *reinterpret_cast<uint4*>(row + 16 * ((2 * c) ^ sw)) = make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(row + 16 * ((2 * c + 1) ^ sw)) = make_uint4(o[4], o[5], o[6], o[7]);
        }
      }
#pragma unroll
      for (int wd = 0; wd < 4 && in_tile && kFmt == 0; ++wd) {
        const uint32_t w = (&w4.x)[wd];
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint32_t ws = w >> (2 * j);
          const uint32_t lo = (ws & 0x00030003u) | 0x64006400u;  // 1024 + c_j, 1024 + c_{j+8}
          const uint32_t hi = (ws & 0x03000300u) | 0x64006400u;  // 1024 + 256 c_{j+4}, ...
          const __half2 clo = __hfma2(*reinterpret_cast<const __half2*>(&lo), k1, __hneg2(k1024));
          const __half2 chi = __hfma2(*reinterpret_cast<const __half2*>(&hi), kinv256, km4);
          const __half2 vlo = __hfma2(clo, s2, ns2);
          const __half2 vhi = __hfma2(chi, s2, ns2);
          o[j] = *reinterpret_cast<const uint32_t*>(&vlo);
          o[j + 4] = *reinterpret_cast<const uint32_t*>(&vhi);
        }
        *reinterpret_cast<uint4*>(row + 16 * ((2 * wd) ^ sw)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(row + 16 * ((2 * wd + 1) ^ sw)) = make_uint4(o[4], o[5], o[6], o[7]);
      }
      fence_proxy_async_shared();  // generic-proxy stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) mbar_arrive(&bfull[bs]);
    }
    // ---------------------------------------------------------------- epilogue
    if (mbar_wait(accum, 0, FAULT_WAIT_EPILOGUE)) {
      tc_fence_after();
      const int q = warp & 3;             // TMEM lane quarter this warp may access
      const int h = (warp - 2) >> 2;      // BM = 256: which accumulator; BM = 128: which half of the columns
      const int m = m0 + (BM == 256 ? kGemmUM * h : 0) + 32 * q + lane;
      TOut* y = reinterpret_cast<TOut*>(p.y);
      const bool vec = (p.N % static_cast<int>(16 / sizeof(TOut))) == 0;  // 16-byte row alignment
      constexpr int kCols = BM == 256 ? BN / 32 : BN / 64;  // 32-column chunks per warp
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
          store_row32<TOut>(y + static_cast<int64_t>(m) * p.N + nb, v32, valid, vec);
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
