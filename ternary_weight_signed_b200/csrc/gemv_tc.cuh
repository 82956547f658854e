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
// Those sums are tcgen05 kind::i8 MMAs: A = the codes c (u8) of 128 weight
// rows, written by the unpacking threads straight into tensor memory (A from
// TMEM: no shared-memory round trip for the big operand); B = the activation
// planes (s8) of one group, 16 rows (up to 8 tokens) or 32 rows (up to 16) x
// 128 bytes in shared memory (row 2m = hi and 2m + 1 = lo of token m, the rest
// zero); D = int32 in TMEM.  One group per MMA chain, so
// each D holds exact per-group sums that the same threads read back and scale
// by s[n, g] * e_g in fp32.
//
// Work split: one CTA per SM owns a contiguous range of rows; the CTA's K is
// split into `parts` ranges so that rows x parts fills up to the 128 TMEM
// lanes (lane = part * rows_box + row, rows_box a multiple of 32 so that every
// warp serves one part).  For a step j, lane (p, r) unpacks group p * gpp + j
// of row r into A columns [32 p, 32 p + 32) (its other parts' columns were
// zeroed once at the start), and the MMA chain runs over all parts with B = the
// matching groups' activations, so each lane's D is its own part's sum.
//
// Memory: per stage and part, nb 2-D TMA boxes each bring one 128-byte block
// of K (512 codes) for all of the CTA's rows with the 128-byte swizzle (so the
// threads reading one row each hit distinct banks), and one bulk copy brings
// the matching activation tiles.  Warp roles:
//   warp 0    : producer (TMA);
//   warp 1    : TMEM allocation and the thread issuing the MMAs;
//   warps 2-9 : unpack + read-back; warps w and w + 4 share a TMEM lane
//               quarter and take alternate steps.
#pragma once
#include "gemm_tc.cuh"
#include "hadamard.cuh"
#include "tb_device.cuh"

namespace tb {

constexpr int kGtcGroups = 4;  // step parities (groups of four unpack warps)
constexpr int kGtcUnpackWarps = 4 * kGtcGroups;
constexpr int kGtcThreads = 32 * (2 + kGtcUnpackWarps);
constexpr int kGtcMaxParts = 7;
constexpr int kGtcMaxM = 16;
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

template <typename TIn>
__global__ void __launch_bounds__(kHThreads) prep_gemv_tc_kernel(const TIn* __restrict__ x,
                                                                  const int8_t* __restrict__ signs,
                                                                  uint8_t* __restrict__ ws, int64_t K, int M) {
  __shared__ float sm[kHB];
  pdl_launch_dependents();
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
  const uint8_t* act;      // prep_gemv_tc output
  const uint16_t* scales;  // [N, G] fp16 bits
  void* y;                 // [M, N]
  int M;                   // tokens (<= the kernel's capacity MT)
  int N, K;
  int box_rows;            // rows of every TMA box (max rows of any CTA)
  int rows_box;            // TMEM lanes per part (box_rows rounded up to 32)
  int parts;               // K ranges per CTA (TMEM lane = part * rows_box + row)
  int gpp;                 // groups per part (multiple of 4)
  int nb;                  // 512-code blocks per stage per part
  int nstages;
  int depth;               // A / D ring depth in TMEM (a power of two, multiple of 4)
  int depth_log2;
  int gps_log2;            // log2 of the groups per stage and part (4 nb, a power of two)
  uint32_t w_box_bytes;    // bytes of one weight box (box_rows x 128)
  uint32_t box_stride;     // w_box_bytes rounded up to 1024
  uint32_t part_bytes;     // shared bytes of one part of a stage: nb boxes + 4 nb atoms
  uint32_t stage_bytes;    // whole stage (all parts)
  uint32_t tmem_cols;
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
__device__ __forceinline__ void tmem_ld_cols<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr));
}
template <>
__device__ __forceinline__ void tmem_ld_cols<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
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
__device__ __forceinline__ void tmem_ld_cols<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7])
               : "r"(taddr));
}

// Shared memory (1024-aligned base):
//   stages  nstages x stage_bytes: for each part, nb weight boxes (box_rows x
//           128 B, swizzled, 1024-aligned) then activation atoms (4 nb x 2 KB)
//   scales  box_rows x G x 2 bytes
//   info    M x G x 8 bytes
//   red     4 x 128 x M floats (partial sums of the four groups of a lane)
//   barriers and the TMEM address
__host__ __device__ inline int64_t gtc_smem_bytes(int M, int64_t K, int box_rows, uint32_t stage_bytes,
                                                  int nstages, int depth) {
  const int64_t G = K / 128;
  return 1024 + static_cast<int64_t>(nstages) * stage_bytes + align128(box_rows * G * 2) + align128(M * G * 8) +
         align128(kGtcGroups * 128 * gtc_capacity(M) * 4) + 8 * (2 * nstages + depth + 2) + 16;
}

template <int MT, typename TOut>
__global__ void __launch_bounds__(kGtcThreads, 1)
    gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const GemvTcParams p) {
  constexpr int AR = gtc_atom_rows(MT);      // activation rows, MMA N, D columns per step
  constexpr int ATOM = gtc_atom_bytes(MT);
  constexpr uint32_t IDESC = gtc_idesc(AR);
  const int M = p.M;
  // tm_w: the packed codes as uint32 [N rows][K/16], box 32 x box_rows, 128B swizzle
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int K = p.K;
  const int G = K / 128;
  const int r0 = static_cast<int>((static_cast<int64_t>(p.N) * blockIdx.x) / gridDim.x);
  const int r1 = static_cast<int>((static_cast<int64_t>(p.N) * (blockIdx.x + 1)) / gridDim.x);
  const int nrows = r1 - r0;
  const int steps = p.gpp;          // MMA chains per lane (groups per part)
  const int gps = 4 * p.nb;         // groups per stage per part (a power of two)
  const int gmask = gps - 1, dmask = p.depth - 1;
  const int nst = (steps + gps - 1) / gps;

  uint8_t* stages = base;
  __half* sc = reinterpret_cast<__half*>(stages + static_cast<int64_t>(p.nstages) * p.stage_bytes);
  int2* info = reinterpret_cast<int2*>(reinterpret_cast<uint8_t*>(sc) + align128(p.box_rows * G * 2));
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(info) + align128(M * G * 8));
  uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(red) + align128(kGtcGroups * 128 * MT * 4));
  uint64_t* empty = full + p.nstages;
  uint64_t* d_ready = empty + p.nstages;
  uint64_t* sb_bar = d_ready + p.depth;  // scales + info
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sb_bar + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t a_cols = 32u * p.parts;  // TMEM columns of one A slot

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGtcGroups);  // one commit per group of unpack warps
    }
    for (int d = 0; d < p.depth; ++d) mbar_init(&d_ready[d], 1);
    mbar_init(sb_bar, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_d0 = tmem + static_cast<uint32_t>(p.depth) * a_cols;  // D ring after the A ring

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tensormap(&tm_w);
      pdl_wait();  // the activation tiles come from the prep kernel
      const uint32_t sbytes = static_cast<uint32_t>(nrows) * G * 2;
      mbar_arrive_expect_tx(sb_bar, sbytes + static_cast<uint32_t>(M * G * 8));
      bulk_load(sc, p.scales + static_cast<int64_t>(r0) * G, sbytes, sb_bar);
      bulk_load(info, p.act + gtc_atoms_bytes(M, K), static_cast<uint32_t>(M * G * 8), sb_bar);
      const int bpp = p.gpp / 4;  // 512-code blocks per part
      for (int s = 0; s < nst; ++s) {
        const int slot = s % p.nstages;
        if (s >= p.nstages && !mbar_wait(&empty[slot], ((s / p.nstages) & 1) ^ 1, FAULT_WAIT_EMPTY)) break;
        uint8_t* st = stages + static_cast<int64_t>(slot) * p.stage_bytes;
        uint32_t bytes = 0;
        int nat[kGtcMaxParts];
        for (int pt = 0; pt < p.parts; ++pt) {
          const int g0 = pt * p.gpp + s * gps;  // first group of this stage and part
          nat[pt] = max(0, min(gps, min(G - g0, p.gpp - s * gps)));
          bytes += p.nb * p.w_box_bytes + static_cast<uint32_t>(nat[pt]) * ATOM;
        }
        mbar_arrive_expect_tx(&full[slot], bytes);
        for (int pt = 0; pt < p.parts; ++pt) {
          uint8_t* pw = st + static_cast<int64_t>(pt) * p.part_bytes;
          for (int b = 0; b < p.nb; ++b)
            tma_load_2d(pw + b * p.box_stride, &tm_w, (pt * bpp + s * p.nb + b) * 32, r0, &full[slot]);
          if (nat[pt] > 0)
            bulk_load(pw + (p.part_bytes - gps * ATOM),
                      p.act + static_cast<int64_t>(pt * p.gpp + s * gps) * ATOM,
                      static_cast<uint32_t>(nat[pt]) * ATOM, &full[slot]);
        }
      }
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------------- unpack, MMA, read-back
    const int q = warp & 3;                    // TMEM lane quarter
    const int sub = (warp - 2) >> 2;           // this group takes steps j with j % 4 == sub
    const bool issuer = (warp == 2 + 4 * sub) && lane == 0;
    const int L = 32 * q + lane;               // TMEM lane
    const int pt = L / p.rows_box;             // part of this lane (uniform across the warp)
    const int r = L - pt * p.rows_box;         // row (within the CTA) of this lane
    const bool live = pt < p.parts && r < nrows;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.f;
    // The other parts' columns of this lane stay zero for the whole kernel.
    if (p.parts > 1) {
      uint32_t z[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) z[i] = 0u;
      for (int d = 0; d < p.depth; ++d)
        for (int pp = 0; pp < p.parts; ++pp)
          if (pp != pt) tmem_st32(tmem + static_cast<uint32_t>(d) * a_cols + 32u * pp + lane_off, z);
      tmem_st_wait();
    }
    bool ok = mbar_wait(sb_bar, 0, FAULT_WAIT_ACT);
    // read back D of step jj and add its contribution
    auto readback = [&](int jj) {
      const int d = jj & dmask;
      ok = ok && mbar_wait(&d_ready[d], (jj >> p.depth_log2) & 1, FAULT_WAIT_MMA);
      tc_fence_after();
      uint32_t dv[2 * MT];
      tmem_ld_cols(tmem_d0 + static_cast<uint32_t>(AR) * d + lane_off, dv);
      tmem_ld_wait();
      const int g = pt * p.gpp + jj;
      if (live && g < G) {
        const float s = __half2float(sc[r * G + g]);
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          if (m < M) {
            const int2 inf = info[m * G + g];
            const int v = static_cast<int>(dv[2 * m]) * 256 + static_cast<int>(dv[2 * m + 1]) - inf.y;
            acc[m] = fmaf(__int2float_rn(v), s * __int_as_float(inf.x), acc[m]);
          }
        }
      }
    };
    // The loops never exit early: every warp of a group must reach the same
    // named barriers.  After a timed-out wait (ok == false) the work is skipped.
    for (int s = 0; s < nst; ++s) {
      const int slot = s % p.nstages;
      const int j0 = s * gps, j1 = min(steps, j0 + gps);
      const int first = j0 + ((sub - j0) % kGtcGroups + kGtcGroups) % kGtcGroups;
      const uint8_t* st = stages + static_cast<int64_t>(slot) * p.stage_bytes;
      if (first < j1) ok = ok && mbar_wait(&full[slot], (s / p.nstages) & 1, FAULT_WAIT_FULL);
      for (int j = first; j < j1; j += kGtcGroups) {
        const int d = j & dmask;
        if (j >= p.depth) readback(j - p.depth);
        uint32_t a[32];
        const int g = pt * p.gpp + j;
        if (ok && live && g < G) {
          // 32 bytes of row r, group g: box (j % gps) / 4 of this stage and part,
          // bytes 32 (g % 4) of the row, stored with the 128-byte swizzle
          // (16-byte chunk c at c ^ ((address >> 7) & 7))
          const uint8_t* rowp = st + static_cast<int64_t>(pt) * p.part_bytes +
                                static_cast<int64_t>((j & gmask) >> 2) * p.box_stride + r * 128;
          const uint32_t x7 = (smem_u32(rowp) >> 7) & 7u;
          const uint32_t c0 = 2u * static_cast<uint32_t>(j & 3);
          const uint4 w0 = *reinterpret_cast<const uint4*>(rowp + 16 * (c0 ^ x7));
          const uint4 w1 = *reinterpret_cast<const uint4*>(rowp + 16 * ((c0 + 1) ^ x7));
          const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) a[4 * i + jb] = (wd[i] >> (2 * jb)) & 0x03030303u;
          }
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) a[i] = 0u;
        }
        tmem_st32(tmem + static_cast<uint32_t>(d) * a_cols + 32u * pt + lane_off, a);
        tmem_st_wait();
        tc_fence_before();
        // the four warps of this group meet; one thread issues the step's MMAs
        asm volatile("bar.sync %0, %1;" ::"r"(2 + sub), "n"(128) : "memory");
        if (issuer && ok) {
          tc_fence_after();
          bool first_mma = true;
          for (int pp = 0; pp < p.parts; ++pp) {
            if (pp * p.gpp + j >= G) continue;  // this part has no group j
            const uint32_t b_atom = smem_u32(st + static_cast<int64_t>(pp) * p.part_bytes +
                                             (p.part_bytes - gps * ATOM) + (j & gmask) * ATOM);
            const uint32_t a_col = tmem + static_cast<uint32_t>(d) * a_cols + 32u * pp;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_i8_ts(tmem_d0 + static_cast<uint32_t>(AR) * d, a_col + 8u * kk, umma_desc_sw128(b_atom + 32u * kk), IDESC,
                         first_mma ? 0u : 1u);
              first_mma = false;
            }
          }
          umma_commit(&d_ready[d]);
        }
      }
      // this group's MMAs of stage s are all issued: release the stage when they finish
      if (issuer) umma_commit(&empty[slot]);
    }
    // drain: the last `depth` steps of this group
    for (int j = sub; j < steps; j += kGtcGroups)
      if (j + p.depth >= steps) readback(j);
    // partial sums of the four groups of this lane, then the parts of each row
    float* rs = red + (sub * 128 + L) * M;
#pragma unroll
    for (int m = 0; m < MT; ++m)
      if (m < M) rs[m] = live ? acc[m] : 0.f;
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kGtcUnpackWarps) : "memory");
    TOut* y = reinterpret_cast<TOut*>(p.y);
    for (int i = threadIdx.x - 64; i < nrows * M; i += 32 * kGtcUnpackWarps) {
      const int rr = i / M, m = i - rr * M;
      float v = 0.f;
      for (int pp = 0; pp < p.parts; ++pp) {
        const int l = pp * p.rows_box + rr;
#pragma unroll
        for (int u = 0; u < kGtcGroups; ++u) v += red[(u * 128 + l) * M + m];
      }
      y[static_cast<int64_t>(m) * p.N + r0 + rr] = from_f32<TOut>(v);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace tb
