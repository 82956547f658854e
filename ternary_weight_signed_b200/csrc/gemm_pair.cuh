// Prefill GEMM on a pair of CTAs (tcgen05 cta_group::2), 2-bit slot format
// and 1-bit g128, with the unpacked weights in tensor memory.
//
// y[m, n] = sum_k x'[m, k] * w[n, k],  w = s[n, k/128] * t[n, k]  (ternary
// g128: news.ditty.ir, second paragraph).  The weights are the MMA's M side:
// each thread unpacks its weight row into exact fp16 s*t (t is -1, 0 or +1 and
// s an fp16 value) and writes it straight into tensor memory with tcgen05.st,
// where the MMA reads it as operand A.  The tokens are the N side: x' tiles
// come by TMA into shared memory as operand B.  So shared memory carries only
// the x' tiles and the packed codes; the fp16 weights never touch it.
//
// One pair tile is 256 weight rows x BT tokens (BT = 256, or 128 up to 128
// tokens).  CTA r of the cluster owns weight rows 128 r .. 128 r + 127 of the
// tile (its TMEM lanes) and loads tokens BT/2 r .. BT/2 r + BT/2 - 1 of the x'
// tile; one M = 256 MMA issued by CTA 0 multiplies both CTAs' A (TMEM) by the
// B halves of both CTAs, and each CTA's TMEM receives D for its own 128 weight
// rows and all BT tokens.  Per K step a CTA's shared memory is read for BT/2
// tokens only, half of what a one-CTA MMA of the same width reads.
//
// The kernel is persistent: one cluster per SM pair at most, each walking its
// tiles with one continuous stage sequence, so the copies and the unpack of a
// tile's first stages overlap the previous tile's last MMAs, and its MMAs wait
// only until every warp has read the previous tile's D into registers.
//
// Warp roles in each CTA:
//   warp 0     : TMA producer (x' half tile with 128B swizzle; packed codes);
//   warp 1     : TMEM allocation for the pair; in CTA 0, the thread issuing
//                the MMAs;
//   warps 2-17 : unpack, four sets of four warps: warp w takes TMEM lanes
//                32 (w % 4) .. + 31 and the stages g = j, j + 4, ... of its
//                set j = (w - 2) / 4 (A slot j), so each warp has four stages
//                of MMA time for the fixed cost of one (barrier waits, the
//                hand-off).  Right after its first stage of a tile, a warp
//                reads its quarter of the previous tile's D (its 32 lanes, BT/4
//                columns), releases D and stores y, the weight rows along the
//                warp's lanes.
// Hand-offs:
//   full[s]  (each CTA, shared-memory slot): x' half and codes landed (TMA);
//   sfree[s] (each CTA): the slot's MMAs are done (commit multicast to both
//            CTAs) and the unpack warps hold its codes in registers;
//   ready[a] (CTA 0, TMEM A slot): the 8 warps of the set, 4 per CTA, wrote the
//            slot and saw their x' half land (the other CTA's warps arrive
//            through the cluster's shared window);
//   afree[a] (each CTA): the MMAs reading the A slot are done (multicast);
//   accum    (each CTA): the tile's MMAs are done; dfree (CTA 0): all 32
//            unpack warps read D out.
// The code order inside a 16-code chunk is the one the prep kernel writes x'
// in (k = 0, 8, 1, 9, ..., 7, 15): the TMEM column j of a chunk holds the fp16
// pair (w_j, w_{j+8}).
//
// Every wait is bounded; after a timeout a role stops waiting, records a fault
// word and still reaches the final cluster barrier, so no CTA leaves while its
// peer may touch its memory, and TMEM is always freed.
#pragma once
#include "gemv.cuh"
#include "gemv_tc.cuh"
#include "hadamard.cuh"
#include "tcgen05.cuh"

namespace tb {

// ---------------------------------------------------------------------------
// Activation prep of the fp16 GEMM: rotation (when signs is non-null) and an
// fp16 store in the paired order inside every 16-element chunk (k = 0, 8, 1,
// 9, ..., 7, 15), the order the unpack writes the weights in.  grid (M,
// K/1024), 128 threads.
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


constexpr int kGpSets = 4;  // unpack warp sets (stage kb goes to set kb % 4)
constexpr int kGpThreads = 32 * (2 + 4 * kGpSets);
constexpr int kGpRows = 128;          // weight rows per CTA (TMEM lanes); 256 per pair
constexpr int kGpPairRows = 2 * kGpRows;
// A stage is two 128-byte swizzle atoms of x along K: 128 fp16 values (one
// scale group) or 256 int8 values; either way 64 TMEM columns of A and eight
// MMAs (K = 16 for kind::f16, 32 for kind::i8).
__host__ __device__ constexpr int gp_bk(bool integer) { return integer ? 256 : 128; }
__host__ __device__ constexpr int gp_atom_k(bool integer) { return gp_bk(integer) / 2; }
constexpr int kGpAtomBytes = 128;
constexpr int kGpASlots = kGpSets;    // TMEM A ring: set j owns slot j
constexpr int kGpACols = 64;          // TMEM columns of a stage's A slice
constexpr int kGpDCols = 256;         // D columns (tokens) at most; the A ring follows
constexpr int kGpTmemCols = 512;
constexpr int kGpSmemCap = 227 * 1024;
static_assert(kGpDCols + kGpASlots * kGpACols <= kGpTmemCols, "TMEM budget");

// x half tile of a stage: two atoms of BT/2 rows x 128 bytes
__host__ __device__ constexpr int gp_x_bytes(int bt) { return bt / 2 * 2 * kGpAtomBytes; }
// codes of a stage per row: 2 bits (fmt 0) or 1 bit (fmt 2) a code
__host__ __device__ constexpr int gp_w_row_bytes(int fmt, bool integer) {
  return fmt == 0 ? gp_bk(integer) / 4 : gp_bk(integer) / 8;
}
__host__ __device__ constexpr int gp_stage_bytes(int bt, int fmt, bool integer) {
  return gp_x_bytes(bt) + kGpRows * gp_w_row_bytes(fmt, integer);
}
// The shared-memory ring is deeper than the TMEM ring (copies run further
// ahead than the unpack): as many stages as fit, at most 8.
__host__ __device__ constexpr int gp_stages(int bt, int fmt, bool integer) {
  return (kGpSmemCap - 1024 - 256) / gp_stage_bytes(bt, fmt, integer) < 8
             ? (kGpSmemCap - 1024 - 256) / gp_stage_bytes(bt, fmt, integer)
             : 8;
}
__host__ __device__ constexpr int gp_smem_bytes(int bt, int fmt, bool integer) {
  return gp_stages(bt, fmt, integer) * gp_stage_bytes(bt, fmt, integer) + 1024 /*align*/ + 256 /*barriers*/;
}
// Instruction descriptor, M = 256 (pair), N = bt tokens, both operands
// K-major.  kind::f16: D fp32 (bits 4-5 = 1), A and B fp16.  kind::i8: D s32
// (bits 4-5 = 2), A and B signed 8-bit (bits 7 and 10).
__host__ __device__ constexpr uint32_t gp_idesc(int bt, bool integer) {
  return (integer ? (2u << 4) | (1u << 7) | (1u << 10) : (1u << 4)) | (static_cast<uint32_t>(bt >> 3) << 17) |
         (static_cast<uint32_t>(kGpPairRows >> 4) << 24);
}

// ---------------------------------------------------------------- cluster
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of both CTAs.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}
// Address of this CTA's shared variable at `saddr` in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
// Arrive on a barrier of either CTA of the cluster.  Default semantics
// (release at CTA scope): measured on B200, the cluster-scope release form
// held the arriving warp about 1600 cycles per arrival, once per stage.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// ---------------------------------------------------------------- tcgen05, pair forms
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D (both CTAs' TMEM) += A (both CTAs' TMEM) x B (both CTAs' shared memory).
template <bool kInt>
__device__ __forceinline__ void umma_pair_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  if constexpr (kInt)
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrives on the barrier at this offset in both CTAs once the MMAs issued so
// far complete.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}
// Tiles of one launch: tiles_n weight-row pairs x tiles_m token tiles, taken
// in order t = tn + tiles_n * tm by the clusters in turn (cluster c: t = c,
// c + C, ...), so that the clusters running at one time share token tiles.
struct GemmPairTiles {
  int tiles_n, tiles_m;
};

// kFmt: 0 = 2-bit slots, 2 = 1-bit g128.  kInt: integer mode (int8 x, no
// rotation, no scales, exact int32 y; A = t as signed bytes), else fp16 x' and
// A = fp16(s t).
template <int BT, typename TOut, int kFmt, bool kInt>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGpThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const GemmParams p, const GemmPairTiles tl) {
  static_assert(kFmt == 0 || kFmt == 2, "2-bit or 1-bit codes");
  static_assert(BT % 64 == 0 && BT >= 128 && BT <= kGpDCols, "token tile");
  constexpr int kBK = gp_bk(kInt), kAtomK = gp_atom_k(kInt), kWr = gp_w_row_bytes(kFmt, kInt);
  constexpr int kX = gp_x_bytes(BT), kAtom = kX / 2, kW = kGpRows * kWr;
  constexpr int kStage = gp_stage_bytes(BT, kFmt, kInt), S = gp_stages(BT, kFmt, kInt), SA = kGpASlots;
  static_assert(kAtom % 1024 == 0 && kStage % 1024 == 0, "128B-swizzle atoms stay 1024-byte aligned");
  static_assert(S >= SA, "the copies run at least as far ahead as the unpack");
  constexpr uint32_t kIdesc = gp_idesc(BT, kInt);
  constexpr int kCols = BT / kGpSets;  // D columns (tokens) one unpack warp reads out
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kStage);  // copies landed
  uint64_t* sfree = full + S;    // stage slot read: by the MMAs (x) and the unpack warps (codes)
  uint64_t* ready = sfree + S;   // (CTA 0) A slot written and x landed, in both CTAs
  uint64_t* afree = ready + SA;  // the MMAs reading an A slot are done
  uint64_t* accum = afree + SA;  // a tile's MMAs are done (D complete)
  uint64_t* dfree = accum + 1;   // (CTA 0) D read out by every unpack warp of both CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(dfree + 1);

  const uint32_t rank = cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cluster = static_cast<int>(blockIdx.x >> 1), nclusters = static_cast<int>(gridDim.x >> 1);
  const int ntiles = tl.tiles_n * tl.tiles_m;
  const int mine = (ntiles - cluster + nclusters - 1) / nclusters;  // tiles of this cluster
  // integer mode: K a multiple of 128; a last half stage reads zeros past K
  const int nk = (p.K + kBK - 1) / kBK;
  auto tile_n0 = [&](int i) {  // this CTA's first weight row in its i-th tile
    return ((cluster + i * nclusters) % tl.tiles_n) * kGpPairRows + static_cast<int>(rank) * kGpRows;
  };
  auto tile_m0 = [&](int i) { return ((cluster + i * nclusters) / tl.tiles_n) * BT; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&sfree[s], 1 + 4);  // the MMAs' commit and the 4 warps of the stage's set
    }
    for (int a = 0; a < SA; ++a) {
      mbar_init(&ready[a], 2 * 4);  // the 4 warps of the stage's set in each CTA
      mbar_init(&afree[a], 1);
    }
    mbar_init(accum, 1);
    mbar_init(dfree, 2 * 4 * kGpSets);  // every unpack warp of both CTAs
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kGpTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;
  const uint32_t tmem_a = tmem_d + kGpDCols;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_w);
      pdl_wait();  // x comes from the previous kernel (the prep kernel, in float mode)
      const bool stall = test_stall_copies();  // failure-detection test: no copies
      int g = 0;     // stage counter over all tiles of this cluster
      bool ok = !stall;
      for (int i = 0; i < mine && ok; ++i) {
        const int n0 = tile_n0(i), my = tile_m0(i) + static_cast<int>(rank) * (BT / 2);
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % S;
          if (g >= S && !mbar_wait(&sfree[s], ((g / S) & 1) ^ 1, FAULT_WAIT_EMPTY)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kStage;
          mbar_arrive_expect_tx(&full[s], kX + kW);
          tma_load_2d(st, &tm_x, kb * kBK, my, &full[s]);
          tma_load_2d(st + kAtom, &tm_x, kb * kBK + kAtomK, my, &full[s]);
          // x in 32-bit words: the codes of a stage are kWr bytes of each row
          tma_load_2d(st + kX, &tm_w, kb * (kWr / 4), n0, &full[s]);
        }
      }
      // the last copies issued land before the CTA may leave
      for (int h = g > S ? g - S : 0; h < g; ++h)
        if (!mbar_wait(&full[h % S], (h / S) & 1, FAULT_WAIT_FULL)) break;
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA (CTA 0)
    if (rank == 0 && lane == 0) {
      int g = 0;
      bool ok = true;
      for (int i = 0; i < mine && ok; ++i) {
        for (int kb = 0; kb < nk; ++kb, ++g) {
          const int s = g % S, a = g % SA;
          if (!mbar_wait(&ready[a], (g / SA) & 1, FAULT_WAIT_FULL)) {
            ok = false;
            break;
          }
          // the first MMA of a tile overwrites D: every warp has read out the last tile's
          if (kb == 0 && i > 0 && !mbar_wait(dfree, (i - 1) & 1, FAULT_WAIT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b = smem_u32(smem + s * kStage);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_pair_ts<kInt>(tmem_d, tmem_a + static_cast<uint32_t>(a * kGpACols + 8 * kk),
                               umma_desc_sw128(b + (kk >> 2) * kAtom + 32 * (kk & 3)), kIdesc,
                               (kb | kk) != 0 ? 1u : 0u);
          umma_commit_pair(&sfree[s]);
          umma_commit_pair(&afree[a]);
        }
        umma_commit_pair(accum);
      }
      if (!ok) umma_commit_pair(accum);  // whoever waits for the tile stops waiting
    }
  } else {
    // ---------------------------------------------------------------- unpack + read-out
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int set = (warp - 2) >> 2;   // stages g = set, set + 4, ... (A slot set)
    const int r = 32 * q + lane;       // weight row of this CTA = TMEM lane
    const int G = p.K / 128;
    const __half2 k1024 = __float2half2_rn(1024.f);
    const __half2 k1 = __float2half2_rn(1.f);
    const __half2 kinv256 = __float2half2_rn(1.f / 256.f);
    const __half2 km4 = __float2half2_rn(-4.f);
    const uint32_t lane_addr = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t ta = tmem_a + lane_addr + static_cast<uint32_t>(set * kGpACols);
    const uint32_t ready0 = cluster_map(smem_u32(&ready[set]), 0);  // CTA 0's ready barrier of this set
    const uint32_t dfree0 = cluster_map(smem_u32(dfree), 0);
    bool ok = true;
    int done = 0;  // tiles whose D this warp has read out and stored
    // D of tile `done` -> registers (then D is released) -> y
    auto read_out = [&]() {
      const bool got = __all_sync(0xffffffffu, mbar_wait(accum, done & 1, FAULT_WAIT_EPILOGUE));
      if (!got) {
        ok = false;
        return;
      }
      tc_fence_after();
      // 16-bit outputs are converted as they come (pairs of tokens in one
      // register), so the warp holds half as many registers until D is free
      constexpr bool kPack = sizeof(TOut) == 2;
      uint32_t h[kPack ? kCols / 2 : kCols];
#pragma unroll
      for (int c = 0; c < kCols; c += 32) {
        uint32_t v[32];
        tmem_ld_cols<32>(tmem_d + lane_addr + static_cast<uint32_t>(set * kCols + c), v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          if constexpr (kPack) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            h[(c + j) / 2] = *reinterpret_cast<const uint32_t*>(&b2);
          } else {
            h[c + j] = v[j];
            h[c + j + 1] = v[j + 1];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(dfree0);
      const int n = tile_n0(done) + r, mb = tile_m0(done) + set * kCols;
      if (n < p.N) {
        TOut* y = reinterpret_cast<TOut*>(p.y) + n;
#pragma unroll
        for (int j = 0; j < kCols; ++j) {
          if (mb + j >= p.M) break;
          TOut* dst = y + static_cast<int64_t>(mb + j) * p.N;
          if constexpr (kPack)
            *reinterpret_cast<uint16_t*>(dst) = static_cast<uint16_t>(h[j / 2] >> (16 * (j & 1)));
          else
            *reinterpret_cast<uint32_t*>(dst) = h[j];
        }
      }
      ++done;
    };
    const int total = mine * nk;
    for (int g = set; g < total && ok; g += kGpSets) {
      const int i = g / nk, kb = g - i * nk, s = g % S;
      // read out every tile before the last one first (a set may have no stage in a tile)
      while (ok && done < i - 1) read_out();
      if (!ok) break;
      const int n = tile_n0(i) + r;
      const bool row_ok = n < p.N;
      // this stage's scale (fp16 mode: stage kb is scale group kb)
      const uint16_t s_bits = (!kInt && row_ok) ? p.scales[static_cast<int64_t>(n) * G + kb] : uint16_t(0);
      // every lane waits (each reads the stage); the warp leaves together
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], (g / S) & 1, FAULT_WAIT_FULL))) {
        ok = false;
        break;
      }
      const uint8_t* wrow = smem + s * kStage + kX + r * kWr;
      uint4 wv[kWr / 16];
#pragma unroll
      for (int u = 0; u < kWr / 16; ++u) wv[u] = *reinterpret_cast<const uint4*>(wrow + 16 * u);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sfree[s]);  // the codes are in registers
      // the MMAs of stage g - 4 are done with this A slot
      if (g >= SA && !__all_sync(0xffffffffu, mbar_wait(&afree[set], ((g / SA) & 1) ^ 1, FAULT_WAIT_MMA))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const __half sc = __ushort_as_half(s_bits);
      const __half2 s2 = __halves2half2(sc, sc);
      const __half2 ns2 = __hneg2(s2);
#pragma unroll
      for (int half = 0; half < 2; ++half) {  // codes of half the stage -> 32 TMEM columns
        uint32_t o[32];
        if constexpr (kInt && kFmt == 0) {
          // codes 128 half .. + 127: packed words 8 half .. + 7, each as 16
          // bytes c = t + 1 in natural order, then t = c - 1 bytewise:
          // (c + 0x7F) ^ 0x80 never carries out of a byte (c <= 2)
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const uint4 c4 = gi8_codes16((&wv[0].x)[8 * half + u]);
#pragma unroll
            for (int b = 0; b < 4; ++b) o[4 * u + b] = ((&c4.x)[b] + 0x7F7F7F7Fu) ^ 0x80808080u;
          }
        } else if constexpr (kInt) {
          // 1-bit: codes 128 half .. + 127 are words 4 half .. + 3, 32 codes a
          // word; t = 2 b - 1 bytewise as (2 b + 0x7F) ^ 0x80
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t w = (&wv[0].x)[4 * half + u];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) o[8 * u + rr] = ((gi8_bits4(w, rr) << 1) + 0x7F7F7F7Fu) ^ 0x80808080u;
          }
        } else if constexpr (kFmt == 2) {
          // chunk c of the 128 codes (16 codes) is half c & 1 of word c >> 1.
          // z holds the chunk's low 8 codes in bits 0-7 and its high 8 in bits
          // 16-23; (z << (15 - j)) & 0x80008000 puts codes j and j + 8 on the
          // sign bits of a half2, and XOR with (-s, -s) gives (s t_j, s t_{j+8}).
          const uint32_t nb = *reinterpret_cast<const uint32_t*>(&ns2);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t w = (&wv[0].x)[2 * half + (c >> 1)];
            const uint32_t z = __byte_perm(w, 0u, (c & 1) ? 0x4342u : 0x4140u);
#pragma unroll
            for (int j = 0; j < 8; ++j) o[8 * c + j] = ((z << (15 - j)) & 0x80008000u) ^ nb;
          }
        } else {
#pragma unroll
          for (int wd = 0; wd < 4; ++wd) {
            const uint32_t w = (&wv[half].x)[wd];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t ws = w >> (2 * j);
              const uint32_t lo = (ws & 0x00030003u) | 0x64006400u;  // 1024 + c_j, 1024 + c_{j+8}
              const uint32_t hi = (ws & 0x03000300u) | 0x64006400u;  // 1024 + 256 c_{j+4}, ...
              const __half2 clo = __hfma2(*reinterpret_cast<const __half2*>(&lo), k1, __hneg2(k1024));
              const __half2 chi = __hfma2(*reinterpret_cast<const __half2*>(&hi), kinv256, km4);
              const __half2 vlo = __hfma2(clo, s2, ns2);
              const __half2 vhi = __hfma2(chi, s2, ns2);
              o[8 * wd + j] = *reinterpret_cast<const uint32_t*>(&vlo);
              o[8 * wd + j + 4] = *reinterpret_cast<const uint32_t*>(&vhi);
            }
          }
        }
        tmem_st32(ta + static_cast<uint32_t>(32 * half), o);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(ready0);
      // right after this warp's first stage of a tile, the previous tile's D
      while (ok && done < i) read_out();
    }
    while (ok && done < mine) read_out();
  }
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();  // neither CTA leaves while its peer may still touch its memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_d, kGpTmemCols);
  }
}

}  // namespace tb
