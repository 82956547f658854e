// Decode GEMV (M <= 16 tokens) on the tensor cores, 2-bit slot format (base-3
// weights reach it after re-encoding to 2-bit slots).
//
// y[m, n] = sum_g s[n, g] * sum_{k in g} t[n, k] x'[m, k]   (ternary g128;
// news.ditty.ir second paragraph; ai4coding.ru "What is a ternary model").
//
// The ternary products are exact integer sums.  Per 128-group, x' is held as
// 16-bit fixed point q = rint(x' / e_g) split into two int8 planes (hi, lo),
// and the packed 2-bit word gives the biased codes c = t + 1 as bytes, so
//   sum_k t q = 256 * sum c hi + sum c lo - sum q.
// Those sums are tcgen05 kind::i8 MMAs: A = the codes c (u8) of up to 128
// weight rows (one row per TMEM lane), written by unpacking warps straight
// into tensor memory; B = the activation planes of one group, 16 rows (up to
// 8 tokens) or 32 rows (up to 16) x 128 bytes in shared memory (row 2m = hi
// and 2m + 1 = lo of token m, the rest zero); D = int32 per-group sums in
// TMEM.  A group's scale s[n, g] multiplies its sum, so every group's D is
// read back and added to fp32 accumulators (one per token, in registers).
//
// Warp-specialised so that the per-group round trip (TMEM store, MMA, commit,
// read-back) is pipelined instead of run step by step:
//   warp 0    : producer: TMA of the weight boxes and bulk copies of the
//               activation atoms into a ring of shared-memory stages;
//   warp 1    : TMEM allocation and the one thread that issues the MMAs;
//   warps 2-5 : unpack: codes of a group -> a ring of A slots in TMEM;
//   warps 6-9 : read-back: a ring of D slots in TMEM -> scale -> fp32 sums.
// Each ring slot has a full and an empty barrier, so every role runs ahead
// of the next by up to the ring depth (8 groups).
//
// Work split over the CTAs: a CTA owns T tiles of up to 128 consecutive
// weight rows and a range of K (whole 1024-code blocks).  When there are few
// rows (N < 148 * 128) K is split over S CTAs per tile so that every SM has
// work while each tile's activations are still read once; the S partial sums
// go to the workspace and the last CTA of a tile to finish (a counter) adds
// them in a fixed order, so the result does not depend on timing.  With more
// rows than 148 * 128, a CTA runs T = 2 or more tiles in turn.
#pragma once
#include "tcgen05.cuh"
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGtcThreads = 32 * 14;  // producer, MMA, 4 unpack and 8 read-back warps
constexpr int kGtcMaxM = 16;
constexpr int kGtcMaxRows = 128;  // rows of a tile: one per TMEM lane
constexpr int kGtcGps = 4;        // groups per stage and per D ring slot (512 codes)
constexpr int kGtcSlots = 2;      // D ring slots in TMEM (4 groups each)
constexpr int kGtcAGroups = 4;    // groups per A ring slot
constexpr int kGtcASlots = 2;     // A ring slots in TMEM (4 groups each)
constexpr int kGtcMaxSplits = 32;
// Activation rows of the B operand (hi and lo plane of each token, padded):
// 16 up to 8 tokens, 32 up to 16; the MMA's N and the D columns per step.
__host__ __device__ constexpr int gtc_atom_rows(int M) { return M <= 8 ? 16 : 32; }
__host__ __device__ constexpr int gtc_atom_bytes(int M) { return gtc_atom_rows(M) * 128; }
// Token capacity of the kernel instance that serves M tokens.
__host__ __device__ constexpr int gtc_capacity(int M) { return M <= 4 ? 4 : (M <= 8 ? 8 : 16); }
// kind::i8: D s32 (bits 4-5 = 2), A u8 (bits 7-9 = 0), B s8 (bits 10-12 = 1),
// both K-major, N (N >> 3 at bits 17-22), M = 128 (M >> 4 at bits 24-28).
__host__ __device__ constexpr uint32_t gtc_idesc(int n) {
  return (2u << 4) | (1u << 10) | ((static_cast<uint32_t>(n) >> 3) << 17) | ((128u >> 4) << 24);
}

// Activation workspace of this path: G atoms of gtc_atom_rows(M) rows x 128
// bytes (row 2m = hi plane of token m, 2m + 1 = lo plane; rows >= 2M zero), each atom in the
// UMMA K-major 128-byte-swizzled layout (16-byte chunk c of row r at
// 16 (c ^ (r & 7)), 8-row groups 1 KB apart); inside each 16-code chunk byte
// 4j + b holds code k = 4b + j, the order in which ((w >> 2j) & 0x03030303)
// delivers the packed codes.  Then info[M][G] = {float e_g, int sum of q}.
__host__ __device__ constexpr int64_t gtc_atoms_bytes(int64_t M, int64_t K) {
  return (K / 128) * gtc_atom_bytes(static_cast<int>(M));
}
__host__ __device__ constexpr int64_t gtc_ws_bytes(int64_t M, int64_t K) {
  return gtc_atoms_bytes(M, K) + M * (K / 128) * 8;
}

// Also zeroes the decode kernel's ncnt tile counters (block (0, 0)).
template <typename TIn>
__global__ void __launch_bounds__(kHThreads) prep_gemv_tc_kernel(const TIn* __restrict__ x,
                                                                  const int8_t* __restrict__ signs,
                                                                  uint8_t* __restrict__ ws, int64_t K, int M,
                                                                  uint32_t* __restrict__ cnt, int ncnt) {
  __shared__ float sm[kHB];
  pdl_launch_dependents();
  if (blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < ncnt; i += kHThreads) cnt[i] = 0u;
  const int64_t m = blockIdx.x;
  const int blk = blockIdx.y;
  const int t = threadIdx.x;
  float v[8];
  load_rotated8<TIn>(x, signs, m, blk, K, v, sm);
  float mx = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(v[i]));
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const float e = mx / kQMax;
  const float inv = mx > 0.f ? kQMax / mx : 0.f;
  int q[8];
  int qs = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    q[i] = max(-32512, min(32512, __float2int_rn(v[i] * inv)));
    qs += q[i];
  }
#pragma unroll
  for (int o = 1; o < 16; o <<= 1) qs += __shfl_xor_sync(0xffffffffu, qs, o);
  // thread t holds codes 8t..8t+7 of the block: group gl = t / 16, 16-code
  // chunk c = (t / 2) % 8 of the group, half h = t % 2 of the chunk
  const int gl = t >> 4, c = (t >> 1) & 7, h = t & 1;
  const int64_t g = static_cast<int64_t>(blk) * 8 + gl;
  const int AR = gtc_atom_rows(M);
  uint8_t* atom = ws + g * gtc_atom_bytes(M);
  uint8_t hb[16], lb[16];  // this thread's 8 bytes land in half of a 16-byte chunk
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int hi = (q[i] + 128) >> 8;
    const int lo = q[i] - (hi << 8);
    const int b = 2 * h + (i >> 2), j = i & 3;  // code 8h + i = 4b + j -> byte 4j + b
    hb[4 * j + b] = static_cast<uint8_t>(static_cast<int8_t>(hi));
    lb[4 * j + b] = static_cast<uint8_t>(static_cast<int8_t>(lo));
  }
  // Bytes 4j + b with b in {2h, 2h + 1}: combine the two halves of the chunk
  // across the thread pair, then the even thread stores the hi row chunk and
  // the odd thread the lo row chunk.
  uint32_t mine_h[4], mine_l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    mine_h[j] = h ? (static_cast<uint32_t>(hb[4 * j + 2]) << 16) | (static_cast<uint32_t>(hb[4 * j + 3]) << 24)
                  : static_cast<uint32_t>(hb[4 * j]) | (static_cast<uint32_t>(hb[4 * j + 1]) << 8);
    mine_l[j] = h ? (static_cast<uint32_t>(lb[4 * j + 2]) << 16) | (static_cast<uint32_t>(lb[4 * j + 3]) << 24)
                  : static_cast<uint32_t>(lb[4 * j]) | (static_cast<uint32_t>(lb[4 * j + 1]) << 8);
  }
  uint32_t wh[4], wl[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    wh[j] = mine_h[j] | __shfl_xor_sync(0xffffffffu, mine_h[j], 1);
    wl[j] = mine_l[j] | __shfl_xor_sync(0xffffffffu, mine_l[j], 1);
  }
  const int row = 2 * static_cast<int>(m) + h;  // h = 0 stores hi, h = 1 stores lo
  const uint4 val = h ? make_uint4(wl[0], wl[1], wl[2], wl[3]) : make_uint4(wh[0], wh[1], wh[2], wh[3]);
  *reinterpret_cast<uint4*>(atom + row * 128 + 16 * (c ^ (row & 7))) = val;
  if (m == 0) {  // rows of tokens >= M are zero
    for (int r = 2 * M + h; r < AR; r += 2)
      *reinterpret_cast<uint4*>(atom + r * 128 + 16 * (c ^ (r & 7))) = make_uint4(0, 0, 0, 0);
  }
  if ((t & 15) == 0) {
    int2 inf;
    inf.x = __float_as_int(e);
    inf.y = qs;
    reinterpret_cast<int2*>(ws + gtc_atoms_bytes(M, K))[m * (K / 128) + g] = inf;
  }
}

struct GemvTcParams {
  const uint8_t* act;   // prep_gemv_tc_kernel output: atoms, then info [M][G]
  void* y;              // [M, N]
  float* part;          // [S][M][N] partial sums (S > 1)
  uint32_t* cnt;        // one counter per tile (S > 1), zeroed by the prep kernel
  int M, N, K, G;
  int R;                // rows per tile (<= 128)
  int T;                // tiles per CTA
  int S;                // K splits per tile
  int nblk;             // 1024-code blocks of K
  int gbox;             // groups of the scale box (the largest K range of a split)
  int sc_tile;          // fp16 elements between the tiles' scale blocks (128-byte multiple)
  int nstages;
  uint32_t box_stride;  // R x 128 bytes rounded up to 1024
  uint32_t stage_bytes; // one weight box, then 4 activation atoms
  uint32_t off_sc, off_info, off_red, off_bar;  // shared-memory offsets from the 1 KB-aligned base
};

// A operand from TMEM, B from shared memory, D in TMEM.
__device__ __forceinline__ void umma_i8_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

template <int NC>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[NC]);
template <>
__device__ __forceinline__ void tmem_ld_cols<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<32>(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld32(taddr, r);
}
template <>
__device__ __forceinline__ void tmem_ld_cols<64>(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
      "%32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, "
      "%48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

// Shared memory of the decode kernel (offsets from the 1 KB-aligned base):
//   stages  nstages x stage_bytes: a weight box (R rows x 128 bytes = 512
//           codes, 128-byte swizzle), then the 4 groups' activation atoms
//   sc      T x [R][gbox] fp16 scales of the CTA's tiles and K range
//   info    [MT][gbox] {e_g, sum q} of the CTA's K range (zero past M)
//   red     [2][128][MT] fp32: the read-back teams' sums at a tile end
//   bar     full/empty per stage, full/empty per A slot and per D slot,
//           the scales barrier, the MMA-done barrier, the TMEM address and
//           the last-CTA flag
struct GtcLayout {
  uint32_t off_sc, off_info, off_red, off_bar;
  int64_t bytes;
};
__host__ __device__ inline int64_t gtc_sc_tile_bytes(int R, int gbox) {
  return align128(static_cast<int64_t>(R) * gbox * 2);
}
__host__ __device__ inline GtcLayout gtc_layout(int M, int R, int T, int gbox, int nstages, uint32_t stage_bytes) {
  GtcLayout l;
  l.off_sc = static_cast<uint32_t>(nstages) * stage_bytes;
  l.off_info = l.off_sc + static_cast<uint32_t>(T * gtc_sc_tile_bytes(R, gbox));
  l.off_red = l.off_info + static_cast<uint32_t>(align128(static_cast<int64_t>(M) * gbox * 8));
  l.off_bar = l.off_red + static_cast<uint32_t>(2 * 128 * M * 4);
  l.bytes = 1024 + l.off_bar + 8 * (2 * nstages + 2 * kGtcASlots + 2 * kGtcSlots + 2) + 16;
  return l;
}

__device__ __forceinline__ bool elect_one() {
  uint32_t pred = 0;
  asm volatile(
      "{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(pred));
  return pred != 0;
}

// Read-back of one group's D columns (2 MT int32 per lane) into the token sums.
// One group's D columns (hi, lo sums of token m at dv[off + 2m], dv[off + 2m
// + 1]) into the token sums.  inf points at the group's info of token 0;
// token m's is inf[m * stride].  Tokens past M have zero activations and zero
// info, so they add zero and need no test.
template <int MT, int NV>
__device__ __forceinline__ void gtc_accumulate(const uint32_t (&dv)[NV], int off, float s, const int2* inf,
                                               int stride, float (&acc)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const int2 f = inf[m * stride];
    const int v = static_cast<int>(dv[off + 2 * m]) * 256 + static_cast<int>(dv[off + 2 * m + 1]) - f.y;
    acc[m] = fmaf(__int2float_rn(v), s * __int_as_float(f.x), acc[m]);
  }
}

// One step of the rings is one stage: kGtcGps = 4 groups (512 codes), so a
// slot holds 4 groups' A (4 x 32 columns) or D (4 x AR columns), and every
// wait, arrive and commit covers four groups.
template <int MT, typename TOut>
__global__ void __launch_bounds__(kGtcThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_s,
                   const GemvTcParams p) {
  constexpr int AR = gtc_atom_rows(MT);   // activation rows = MMA N = D columns per group
  constexpr int ATOM = gtc_atom_bytes(MT);
  constexpr uint32_t IDESC = gtc_idesc(AR);
  constexpr int G4 = kGtcGps;
  constexpr uint32_t A_COLS = 32u * kGtcAGroups;  // A columns of an A slot
  constexpr uint32_t D_COLS = static_cast<uint32_t>(AR) * G4;  // D columns of a slot
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int M = p.M;
  uint8_t* stages = base;
  const __half* sc = reinterpret_cast<const __half*>(base + p.off_sc);
  const int2* info = reinterpret_cast<const int2*>(base + p.off_info);
  float* red = reinterpret_cast<float*>(base + p.off_red);  // [2 teams][128 lanes][MT]
  uint64_t* full = reinterpret_cast<uint64_t*>(base + p.off_bar);
  uint64_t* empty = full + p.nstages;
  uint64_t* a_full = empty + p.nstages;
  uint64_t* a_empty = a_full + kGtcASlots;
  uint64_t* d_full = a_empty + kGtcASlots;
  uint64_t* d_empty = d_full + kGtcSlots;
  uint64_t* sb_bar = d_empty + kGtcSlots;
  uint64_t* mma_done = sb_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile uint32_t* last_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this CTA: tile group tg (T tiles of R rows) and K split sidx
  const int tg = blockIdx.x / p.S, sidx = blockIdx.x - tg * p.S;
  const int b0 = static_cast<int>((static_cast<int64_t>(p.nblk) * sidx) / p.S);
  const int b1 = static_cast<int>((static_cast<int64_t>(p.nblk) * (sidx + 1)) / p.S);
  const int g0 = 8 * b0, Gc = 8 * (b1 - b0);  // groups of this CTA's K range (a multiple of 8)
  const int row_base = tg * p.T * p.R;
  int nt = 0;  // tiles with rows
  while (nt < p.T && row_base + nt * p.R < p.N) ++nt;
  const int spt = Gc / G4;     // steps (stages) per tile
  const int nst = nt * spt;    // steps of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4 + 1);  // four unpack warps have read the codes, the MMAs are done
    }
    for (int d = 0; d < kGtcASlots; ++d) {
      mbar_init(&a_full[d], 4);
      mbar_init(&a_empty[d], 1);
    }
    for (int d = 0; d < kGtcSlots; ++d) {
      mbar_init(&d_full[d], 1);
      mbar_init(&d_empty[d], 4);
    }
    mbar_init(sb_bar, 1);
    mbar_init(mma_done, 1);
    fence_mbar_init();
  }
  // tokens past M: zero info (their activation rows are zero too)
  for (int i = threadIdx.x; i < (MT - M) * Gc; i += kGtcThreads)
    reinterpret_cast<int2*>(base + p.off_info)[M * Gc + i] = make_int2(0, 0);
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_a0 = tmem;                               // A ring: kGtcASlots x A_COLS columns
  const uint32_t tmem_d0 = tmem + A_COLS * kGtcASlots;         // D ring: kGtcSlots x D_COLS columns

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&tm_w);
      prefetch_tensormap(&tm_s);
      const uint32_t sc_box = static_cast<uint32_t>(p.R) * p.gbox * 2;  // bytes one scale box brings
      mbar_arrive_expect_tx(sb_bar, static_cast<uint32_t>(nt) * sc_box + static_cast<uint32_t>(M * Gc * 8));
      // scales and weights are layer constants: fetched before the wait for
      // the previous kernel (programmatic dependent launch)
      for (int t = 0; t < nt; ++t)
        tma_load_2d(base + p.off_sc + t * p.sc_tile * 2, &tm_s, g0, row_base + t * p.R, sb_bar);
      const uint64_t pol = l2_policy_evict_first();  // weights are read once per call
      const uint32_t stage_tx = static_cast<uint32_t>(p.R) * 128u + G4 * ATOM;
      const int pre = min(p.nstages, nst);
      {
        int t = 0, gl = 0;
        for (int q = 0; q < pre; ++q) {
          mbar_arrive_expect_tx(&full[q], stage_tx);
          tma_load_2d_hint(stages + static_cast<int64_t>(q) * p.stage_bytes, &tm_w, (g0 + gl) * 8,
                           row_base + t * p.R, &full[q], pol);
          gl += G4;
          if (gl == Gc) { gl = 0; ++t; }
        }
      }
      pdl_wait();  // activations come from the prep kernel
      // info [M][G] follows the G activation atoms
      const uint8_t* info_src = p.act + static_cast<int64_t>(p.G) * ATOM;
      for (int m = 0; m < M; ++m)
        bulk_load(base + p.off_info + m * Gc * 8, info_src + (static_cast<int64_t>(m) * p.G + g0) * 8,
                  static_cast<uint32_t>(Gc * 8), sb_bar);
      int issued = nst;  // stages whose copies went out
      int t = 0, gl = 0, slot = 0, phase = 0;
      for (int q = 0; q < nst; ++q) {
        uint8_t* st = stages + static_cast<int64_t>(slot) * p.stage_bytes;
        if (q >= pre) {
          if (!mbar_wait_backoff(&empty[slot], phase ^ 1, FAULT_WAIT_EMPTY)) {
            issued = q;
            break;
          }
          mbar_arrive_expect_tx(&full[slot], stage_tx);
          tma_load_2d_hint(st, &tm_w, (g0 + gl) * 8, row_base + t * p.R, &full[slot], pol);
        }
        bulk_load(st + p.box_stride, p.act + static_cast<int64_t>(g0 + gl) * ATOM, G4 * ATOM, &full[slot]);
        gl += G4;
        if (gl == Gc) { gl = 0; ++t; }
        if (++slot == p.nstages) { slot = 0; phase ^= 1; }
      }
      pdl_launch_dependents();  // the next kernel may start its prologue
      // Before the CTA exits every copy issued must have landed, also when a
      // consumer gave up waiting (bounded; immediate when all went well).
      for (int s = 0; s < min(p.nstages, issued); ++s) {
        const int qlast = s + ((issued - 1 - s) / p.nstages) * p.nstages;
        if (!mbar_wait(&full[s], (qlast / p.nstages) & 1, FAULT_WAIT_FULL)) break;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issue
    // The whole warp runs the loop (uniform control); one elected lane issues.
    int slot = 0, sphase = 0, d = 0, dphase = 0, as = 0, asphase = 0;
    bool ok = true;
    for (int q = 0; q < nst && ok; ++q) {
      ok = mbar_wait(&full[slot], sphase, FAULT_WAIT_FULL);
      if (ok && q >= kGtcSlots) ok = mbar_wait(&d_empty[d], dphase ^ 1, FAULT_WAIT_MMA);
      const uint32_t b_atom = smem_u32(stages + static_cast<int64_t>(slot) * p.stage_bytes + p.box_stride);
      const uint64_t bd0 = umma_desc_sw128(b_atom);
#pragma unroll
      for (int h = 0; h < G4 / kGtcAGroups; ++h) {
        ok = __all_sync(0xffffffffu, ok && mbar_wait(&a_full[as], asphase, FAULT_WAIT_MMA));
        if (!ok) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int gg = 0; gg < kGtcAGroups; ++gg) {
            const int g = h * kGtcAGroups + gg;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_i8_ts(tmem_d0 + D_COLS * d + static_cast<uint32_t>(AR * g),
                         tmem_a0 + A_COLS * as + 32u * gg + 8u * kk,
                         bd0 + static_cast<uint64_t>((g * ATOM + 32 * kk) >> 4), IDESC, kk > 0 ? 1u : 0u);
          }
          umma_commit(&a_empty[as]);
        }
        __syncwarp();
        if (++as == kGtcASlots) { as = 0; asphase ^= 1; }
      }
      if (!ok) break;
      if (elect_one()) {
        umma_commit(&d_full[d]);
        umma_commit(&empty[slot]);
      }
      __syncwarp();
      if (++slot == p.nstages) { slot = 0; sphase ^= 1; }
      if (++d == kGtcSlots) { d = 0; dphase ^= 1; }
    }
    if (elect_one()) umma_commit(mma_done);  // arrives once every MMA issued above is complete
    __syncwarp();
  } else if (warp < 6) {
    // ---------------------------------------------------------------- unpack
    const int qd = warp & 3;  // TMEM lane quarter
    const int L = 32 * qd + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * qd) << 16;
    const bool row_in_box = L < p.R;  // lanes past the tile's rows store zero codes
    const uint32_t x7 = static_cast<uint32_t>(L & 7);  // box stride and stage bytes are multiples of 1 KB
    int slot = 0, sphase = 0, as = 0, asphase = 0, half = 0;
    for (int q = 0; q < nst; ++q) {
      if (!__all_sync(0xffffffffu, mbar_wait_backoff(&full[slot], sphase, FAULT_WAIT_FULL))) break;
      // row L of the box: 128 bytes = 4 groups of 32; group g is the 16-byte
      // chunks 2 g and 2 g + 1, stored with the 128-byte swizzle
      const uint8_t* rowp = stages + static_cast<int64_t>(slot) * p.stage_bytes + L * 128;
      bool ok = true;
#pragma unroll
      for (int h = 0; h < G4 / kGtcAGroups; ++h) {
        if (half >= kGtcASlots &&
            !__all_sync(0xffffffffu, mbar_wait_backoff(&a_empty[as], asphase ^ 1, FAULT_WAIT_MMA))) {
          ok = false;
          break;
        }
#pragma unroll
        for (int gg = 0; gg < kGtcAGroups; ++gg) {
          const uint32_t c0 = 2u * static_cast<uint32_t>(h * kGtcAGroups + gg);
          const uint4 w0 =
              row_in_box ? *reinterpret_cast<const uint4*>(rowp + 16 * (c0 ^ x7)) : make_uint4(0, 0, 0, 0);
          const uint4 w1 =
              row_in_box ? *reinterpret_cast<const uint4*>(rowp + 16 * ((c0 + 1) ^ x7)) : make_uint4(0, 0, 0, 0);
          const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          uint32_t av[32];
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) av[4 * i + jb] = (wd[i] >> (2 * jb)) & 0x03030303u;
          tmem_st32(tmem_a0 + A_COLS * as + 32u * gg + lane_off, av);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&a_full[as]);
          if (h == G4 / kGtcAGroups - 1) mbar_arrive(&empty[slot]);  // this warp is done with the stage's codes
        }
        ++half;
        if (++as == kGtcASlots) { as = 0; asphase ^= 1; }
      }
      if (!ok) break;
      if (++slot == p.nstages) { slot = 0; sphase ^= 1; }
    }
  } else {
    // ---------------------------------------------------------------- read-back
    // Two teams of four warps (one per TMEM lane quarter) take alternate
    // steps, so one team's TMEM loads are in flight while the other adds.
    const int qd = warp & 3;
    const int team = (warp - 6) >> 2;
    const int L = 32 * qd + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * qd) << 16;
    pdl_wait();  // y (and the counters) follow the previous kernels on the stream
    bool ok = __all_sync(0xffffffffu, mbar_wait_backoff(sb_bar, 0, FAULT_WAIT_ACT));
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    TOut* y = reinterpret_cast<TOut*>(p.y);
    const int Lr = min(L, p.R - 1);
    // The loop never exits early: the eight read-back warps meet at named
    // barriers at tile ends.  After a wait that gave up (ok false) the work
    // of the remaining steps is skipped.
    int a = 0, aphase = 0, t = 0, gl = 0;
    for (int q = 0; q < nst; ++q) {
      const bool mine = (q & 1) == team;
      if (mine && ok) ok = __all_sync(0xffffffffu, mbar_wait_backoff(&d_full[a], aphase, FAULT_WAIT_MMA));
      if (mine && ok) {
        tc_fence_after();
        const uint32_t dslot = tmem_d0 + D_COLS * a + lane_off;
        const __half* srow = sc + t * p.sc_tile + Lr * p.gbox + gl;
        if constexpr (AR == 16) {
          // the step's 4 groups x 16 columns in one load
          uint32_t dv[64];
          tmem_ld_cols<64>(dslot, dv);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&d_empty[a]);
#pragma unroll
          for (int g = 0; g < G4; ++g) gtc_accumulate<MT, 64>(dv, 16 * g, __half2float(srow[g]), info + gl + g, Gc, acc);
        } else {
          // 4 groups x 32 columns: two loads of two groups
          uint32_t dv[64];
          tmem_ld_cols<64>(dslot, dv);
          tmem_ld_wait();
          gtc_accumulate<MT, 64>(dv, 0, __half2float(srow[0]), info + gl, Gc, acc);
          gtc_accumulate<MT, 64>(dv, 32, __half2float(srow[1]), info + gl + 1, Gc, acc);
          tmem_ld_cols<64>(dslot + 64, dv);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&d_empty[a]);
          gtc_accumulate<MT, 64>(dv, 0, __half2float(srow[2]), info + gl + 2, Gc, acc);
          gtc_accumulate<MT, 64>(dv, 32, __half2float(srow[3]), info + gl + 3, Gc, acc);
        }
      }
      gl += G4;
      if (gl == Gc) {
        // tile t done: the two teams' sums of this lane's row, added in team order
        const int n = row_base + t * p.R + L;
        const bool live = ok && L < p.R && n < p.N;
        float* xch = red + (team * 128 + L) * MT;
#pragma unroll
        for (int m = 0; m < MT; ++m) xch[m] = acc[m];
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight read-back warps
        if (team == 0) {
#pragma unroll
          for (int m = 0; m < MT; ++m) acc[m] += red[(128 + L) * MT + m];
        }
        if (p.S == 1) {
          if (live && team == 0)
#pragma unroll
            for (int m = 0; m < MT; ++m)
              if (m < M) y[static_cast<int64_t>(m) * p.N + n] = from_f32<TOut>(acc[m]);
        } else {
          if (live && team == 0)
#pragma unroll
            for (int m = 0; m < MT; ++m)
              if (m < M) p.part[(static_cast<int64_t>(sidx) * M + m) * p.N + n] = acc[m];
          __threadfence();
          asm volatile("bar.sync 1, 256;" ::: "memory");
          if (threadIdx.x == 192) {
            const uint32_t prev = atomicAdd(&p.cnt[tg * p.T + t], 1u);
            __threadfence();
            *last_flag = prev == static_cast<uint32_t>(p.S - 1) ? 1u : 0u;
          }
          asm volatile("bar.sync 1, 256;" ::: "memory");
          if (*last_flag != 0u && live && team == 0) {
            // The last CTA of the tile adds the S partial sums in split order.
            // Every split's MT loads are independent and issued together (a
            // dependent load per split and token measured 10 us per tile).
            float v[MT];
#pragma unroll
            for (int m = 0; m < MT; ++m) v[m] = 0.f;
#pragma unroll 4
            for (int s2 = 0; s2 < p.S; ++s2) {
              const float* src = p.part + static_cast<int64_t>(s2) * M * p.N + n;
              float pv[MT];
#pragma unroll
              for (int m = 0; m < MT; ++m) pv[m] = m < M ? __ldcg(src + static_cast<int64_t>(m) * p.N) : 0.f;
#pragma unroll
              for (int m = 0; m < MT; ++m) v[m] += pv[m];
            }
#pragma unroll
            for (int m = 0; m < MT; ++m)
              if (m < M) y[static_cast<int64_t>(m) * p.N + n] = from_f32<TOut>(v[m]);
          }
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");  // the exchange buffer is free again
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] = 0.f;
        gl = 0;
        ++t;
      }
      if (++a == kGtcSlots) { a = 0; aphase ^= 1; }
    }
  }
  // every MMA issued must be complete before TMEM is freed
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_wait(mma_done, 0, FAULT_WAIT_MMA);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tb
