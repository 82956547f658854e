// libternary_b200.so: the C ABI declared in include/ternary_b200.h.
//
// One translation unit: the kernels live in the included .cuh files.  Host
// code here validates arguments (before anything is enqueued), picks a kernel
// path, builds TMA descriptors and launches on the caller's stream.  Nothing
// here allocates device memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <unordered_set>

#include "ternary_b200.h"
#include "tb_device.cuh"

#include "gemm_pair.cuh"
#include "gemv.cuh"
#include "gemv_m1.cuh"
#include "prepare.cuh"
#include "gemv_b3.cuh"
#include "gemv_tc.cuh"
#include "hadamard.cuh"
#include "pack.cuh"
#include "simple.cuh"

namespace {

using namespace tb;

constexpr int kVersion = 1 * 10000 + 0 * 100 + 0;

// ------------------------------------------------------------------ device
struct DevInfo {
  bool valid = false;
  int sm_count = 0;
  int max_smem_optin = 0;
  int cc_major = 0;
};

std::mutex g_mu;
DevInfo g_dev[64];
std::unordered_set<uint64_t> g_smem_set;  // (function, device) pairs with the attribute set

tb_status current_device(const DevInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DevInfo& d = g_dev[dev];
  if (!d.valid) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
      cudaGetLastError();
      return TB_ERR_CUDA;
    }
    d.sm_count = prop.multiProcessorCount;
    d.max_smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
    d.cc_major = prop.major;
    d.valid = true;
  }
  if (d.cc_major != 10) return TB_ERR_DEVICE;
  *out = &d;
  return TB_OK;
}

// Raises a kernel's dynamic shared-memory limit to the device maximum, once
// per (kernel, device).
template <typename F>
tb_status allow_smem(F* fn, const DevInfo* d) {
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t key = reinterpret_cast<uint64_t>(reinterpret_cast<const void*>(fn)) ^
                       (static_cast<uint64_t>(dev) << 56);
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_smem_set.count(key)) return TB_OK;
  // all of these kernels stage through shared memory: ask for the largest carveout
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, fn) != cudaSuccess) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  const int dyn_max = d->max_smem_optin - static_cast<int>(fa.sharedSizeBytes);
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn_max) != cudaSuccess ||
      cudaFuncSetAttribute(fn, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  g_smem_set.insert(key);
  return TB_OK;
}

tb_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? TB_OK : TB_ERR_CUDA;
}

// ------------------------------------------------------------------ TMA maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

tb_status get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return TB_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return TB_OK;
}

// Row-major 2-D tensor [rows, cols] of `dtype` elements, box [box_rows, box_cols].
tb_status make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, int esize, const void* base,
                      uint64_t cols, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_cols,
                      uint32_t box_rows, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_NONE) {
  (void)esize;
  if (get_encoder() != TB_OK) return TB_ERR_CUDA;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? TB_OK : TB_ERR_CUDA;
}

// ------------------------------------------------------------------ helpers
bool is_float_dtype(int t) { return t == TB_BF16 || t == TB_FP16 || t == TB_FP32; }
int dtype_size(int t) {
  switch (t) {
    case TB_BF16:
    case TB_FP16: return 2;
    case TB_FP32:
    case TB_INT32: return 4;
    case TB_INT8: return 1;
    default: return 0;
  }
}
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

template <typename Kern, typename... Args>
tb_status launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, args...) != cudaSuccess) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  return TB_OK;
}

// ------------------------------------------------------------------ rotate dispatch
template <typename TIn, typename TOut>
void launch_rotate(const void* x, void* y, const int8_t* signs, int64_t M, int64_t K, int inverse,
                   cudaStream_t st) {
  dim3 grid(static_cast<unsigned>(M), static_cast<unsigned>(K / kHB));
  rotate_kernel<TIn, TOut><<<grid, kHThreads, 0, st>>>(static_cast<const TIn*>(x),
                                                       static_cast<TOut*>(y), signs, K, inverse);
}

template <typename TIn>
void launch_rotate_out(int yt, const void* x, void* y, const int8_t* signs, int64_t M, int64_t K,
                       int inverse, cudaStream_t st) {
  switch (yt) {
    case TB_BF16: launch_rotate<TIn, __nv_bfloat16>(x, y, signs, M, K, inverse, st); break;
    case TB_FP16: launch_rotate<TIn, __half>(x, y, signs, M, K, inverse, st); break;
    default: launch_rotate<TIn, float>(x, y, signs, M, K, inverse, st); break;
  }
}

// ------------------------------------------------------------------ linear: validation
struct LinearArgs {
  const void* x;
  int xt;
  const uint8_t* packed;
  const uint16_t* scales;
  int f;
  int64_t M, N, K;
  const int8_t* signs;
  void* y;
  int yt;
  void* ws;
  size_t ws_bytes;
  cudaStream_t st;
};

// Base-3 with 8 or more tokens re-encodes the weights to 2-bit slots in the
// workspace, in front of the activations of the 2-bit path that follows (the
// tensor-core decode up to 16 tokens, the GEMM beyond): one pass over the
// base-3 bytes beats a base-3 decode pass per chunk of 4 tokens.
constexpr int kB3TranscodeMinM = 8;
size_t b3_transcode_bytes(int f, int64_t M, int64_t N, int64_t K) {
  if (f != TB_FMT_BASE3 || M < kB3TranscodeMinM) return 0;
  return (static_cast<size_t>(N) * static_cast<size_t>(K / 4) + 255) & ~static_cast<size_t>(255);
}

size_t workspace_bytes(int64_t M, int64_t K) {
  size_t b = static_cast<size_t>(4) * static_cast<size_t>(M) * static_cast<size_t>(K);
  const size_t g = static_cast<size_t>(gtc_ws_bytes(M, K));  // tensor-core decode activations
  if (g > b) b = g;
  const size_t v = static_cast<size_t>(gemv_ws_bytes(M, K));  // decode activation words
  if (v > b) b = v;
  const size_t v3 = static_cast<size_t>(b3_ws_bytes(M, K));  // base-3 decode activation words
  if (v3 > b) b = v3;
  return (b + 255) & ~static_cast<size_t>(255);
}

size_t gtc_extra_bytes(int f, int64_t M, int64_t N, int64_t K);

// Everything a call may use: the activations of any path, the base-3
// re-encoding, the tensor-core decode's partial sums and counters.
size_t required_ws(int f, int64_t M, int64_t N, int64_t K) {
  return workspace_bytes(M, K) + b3_transcode_bytes(f, M, N, K) + gtc_extra_bytes(f, M, N, K);
}

bool fast_aligned(const LinearArgs& a) {
  return aligned(a.packed, 16) && aligned(a.scales, 16) && aligned(a.x, 16) && aligned(a.y, 16) &&
         aligned(a.ws, 16) && (a.signs == nullptr || aligned(a.signs, 16));
}

struct GemvPlan {
  int grid, R, RT, NB, nstage, nslots, box_stride, slot_bytes, sc_bytes;
  size_t smem;
};

// Geometry of the decode kernel for these sizes on a device with `sm_count`
// SMs and `max_smem` bytes of shared memory per block; false if it does not fit.
bool gemv_plan(int64_t M, int64_t N, int64_t K, int sm_count, int max_smem, GemvPlan* out) {
  if (M < 1 || M > kGemvMaxM || K % 1024 != 0 || K < 1024 || N < 1 || sm_count < 1) return false;
  GemvPlan pl;
  const int64_t rmax = 32 * gemv_max_row_tiles(static_cast<int>(M));
  int64_t R = (N + sm_count - 1) / sm_count;
  if (R > rmax) R = rmax;
  pl.R = static_cast<int>(R);
  pl.RT = static_cast<int>((R + 31) / 32);
  pl.grid = static_cast<int>((N + R - 1) / R);
  const int64_t G = K / 128;
  // boxes per stage: enough that one stage moves >= 12 KB of weights
  const int64_t boxes = K / kGemvBoxCodes;
  int NB = 1;
  while (NB < kGemvMaxNB && NB < boxes && static_cast<int64_t>(NB) * R * 128 < 12 * 1024) NB *= 2;
  pl.NB = NB;
  pl.nstage = static_cast<int>(gemv_nstage(K, NB));
  pl.box_stride = static_cast<int>(align_up(R * 128, 1024));
  pl.slot_bytes = static_cast<int>(align_up(static_cast<int64_t>(NB) * pl.box_stride +
                                                gemv_act_stage_bytes(static_cast<int>(M), NB), 1024));
  pl.sc_bytes = static_cast<int>(align_up(R * G * 2, 1024));
  // the scales of the CTA arrive on one barrier: < 2^20 bytes
  if (R * G * 2 >= (int64_t(1) << 20)) return false;
  const int64_t part = M * pl.RT * 32 * kGemvWarps * 4;  // row partials, parked in the ring at the end
  const int64_t budget = std::min<int64_t>(max_smem, kGemvSmemTarget);
  int64_t ns = (budget - gemv_smem_bytes(pl.sc_bytes, 0, 0)) / pl.slot_bytes;
  if (ns > kGemvMaxSlots) ns = kGemvMaxSlots;
  if (ns >= pl.nstage) {
    ns = pl.nstage;  // every stage has a slot of its own: no slot is reused
  } else {
    // When the warps split into Q groups that take alternate stages, each slot
    // must belong to one group (nslots a multiple of Q): a warp may then wait
    // on a slot's barrier at most one phase ahead of it.
    const int ips = NB * 4 * (128 / gemv_cpi(static_cast<int>(M)));
    const int qg = ips >= kGemvWarps ? 1 : kGemvWarps / ips;
    ns -= ns % qg;
    if (ns < qg || ns < 2) return false;
  }
  // the row partials are parked in the ring at the end
  while (ns * pl.slot_bytes < part && ns < kGemvMaxSlots) ++ns;
  if (ns * pl.slot_bytes < part) return false;
  pl.nslots = static_cast<int>(ns);
  const int64_t smem = gemv_smem_bytes(pl.sc_bytes, pl.slot_bytes, pl.nslots);
  if (smem > max_smem) return false;
  pl.smem = static_cast<size_t>(smem);
  *out = pl;
  return true;
}

struct G1Plan {
  int grid, R, RT, Wt, Wk, TPW, NB, nb_log2, nstage, nslots, box_stride, slot_bytes;
  bool fused;
  Gemv1Layout lay;
};

// Geometry of the one-token decode kernel (gemv_m1.cuh) for packed format
// `fmt` (2-bit or 1-bit); false if it does not fit.
bool g1_plan(int64_t N, int64_t K, int sm_count, int max_smem, bool fused, G1Plan* out, int fmt = TB_FMT_2BIT) {
  const int64_t box = g1_box_bytes(fmt);
  if (K % 1024 != 0 || K < 1024 || N < 1 || sm_count < 1) return false;
  if (fused && K / kHB > kG1FusedMaxBlocks) return false;
  G1Plan pl;
  int64_t R = (N + sm_count - 1) / sm_count;
  if (R > kG1MaxRows) R = kG1MaxRows;
  pl.R = static_cast<int>(R);
  pl.RT = static_cast<int>((R + 7) / 8);
  pl.grid = static_cast<int>((N + R - 1) / R);
  const int64_t C = K / 512;
  // Wt row-tile groups x Wk chunk classes (<= kG1Warps warps): the least
  // issue work for the busiest warp; a warp's tiles run two at a time and its
  // activation words are loaded once per chunk
  int64_t best_cost = -1;
  for (int wt = 1; wt <= kG1Warps; ++wt) {
    for (int wk = 1; wt * wk <= kG1Warps; ++wk) {
      const int64_t tpw = (pl.RT + wt - 1) / wt;
      if (tpw > 4) continue;
      const int tpl = tpw == 1 ? 1 : (tpw == 2 ? 2 : 4);  // kernel instance
      const int64_t cost = ((C + wk - 1) / wk) * (tpl * 110 + 20);
      if (best_cost < 0 || cost < best_cost) {
        best_cost = cost;
        pl.Wt = wt;
        pl.Wk = wk;
        pl.TPW = tpl;
      }
    }
  }
  if (best_cost < 0) return false;
  pl.box_stride = static_cast<int>(align_up(R * box, 1024));
  // stages of at least 8 KB of weights, a power of two of chunks
  int64_t want = (8192 + R * box - 1) / (R * box);
  if (want > C) want = C;
  int64_t nb = 1;
  pl.nb_log2 = 0;
  while (nb < want) {
    nb *= 2;
    ++pl.nb_log2;
  }
  pl.NB = static_cast<int>(nb);
  pl.nstage = static_cast<int>((C + nb - 1) / nb);
  pl.slot_bytes = static_cast<int>(nb) * pl.box_stride;
  pl.fused = fused;
  const int64_t budget = std::min<int64_t>(kG1SmemMax, max_smem);
  const Gemv1Layout l0 = gemv1_layout(K, pl.R, pl.Wk, pl.nstage, 0);
  int64_t ns = (budget - l0.bytes) / pl.slot_bytes;
  if (ns > pl.nstage) ns = pl.nstage;
  if (ns < 1 || ns < std::min<int64_t>(2, pl.nstage)) return false;
  pl.nslots = static_cast<int>(ns);
  pl.lay = gemv1_layout(K, pl.R, pl.Wk, pl.nstage, ns * pl.slot_bytes);
  if (pl.lay.bytes > budget) return false;
  *out = pl;
  return true;
}

bool g1_fused(int64_t K) { return K / kHB <= kG1FusedMaxBlocks; }

// The two-CTA one-token kernel wins when it rotates x itself or has at least
// eight row tiles per CTA; with few rows and long K (a down projection,
// 5120 x 17408: 19.3 against 23.3 us per call on B200) the 16-warp kernel with
// dynamic item distribution is faster.
bool g1_preferred(int64_t N, int64_t K, int sm_count) {
  return g1_fused(K) || (N + sm_count - 1) / sm_count >= 64;
}

struct B3Plan {
  int grid, R, RT, NB, nstage, nslots, box_stride, slot_bytes, sc_bytes;
  size_t smem;
};

// Geometry of the base-3 decode kernel; false if these sizes do not fit it.
bool b3_plan(int64_t M, int64_t N, int64_t K, int sm_count, int max_smem, B3Plan* out) {
  if (M < 1 || M > kGemvMaxM || K % 1024 != 0 || K < 1024 || N < 1 || sm_count < 1) return false;
  B3Plan pl;
  int64_t R = (N + sm_count - 1) / sm_count;
  if (R > 32 * kGemvRowTiles) R = 32 * kGemvRowTiles;
  pl.R = static_cast<int>(R);
  pl.RT = static_cast<int>((R + 31) / 32);
  pl.grid = static_cast<int>((N + R - 1) / R);
  const int64_t G = K / 128, C = K / 1024;
  int NB = 1;
  while (NB < kGemvMaxNB && NB < C && static_cast<int64_t>(NB) * R * kB3BlockBytes < 12 * 1024) NB *= 2;
  pl.NB = NB;
  pl.nstage = static_cast<int>(b3_nstage(K, NB));
  // + 16: the group-word loads of the last row may read one chunk past it
  pl.box_stride = static_cast<int>(align_up(R * kB3BlockBytes + 16, 1024));
  pl.slot_bytes = static_cast<int>(align_up(static_cast<int64_t>(NB) * pl.box_stride +
                                                b3_act_stage_bytes(static_cast<int>(M), NB), 1024));
  pl.sc_bytes = static_cast<int>(align_up(R * G * 2, 1024));
  if (R * G * 2 >= (int64_t(1) << 20)) return false;
  const int64_t part = M * pl.RT * 32 * kGemvWarps * 4;
  int64_t ns = (max_smem - b3_smem_bytes(pl.sc_bytes, 0, 0)) / pl.slot_bytes;
  if (ns > kGemvMaxSlots) ns = kGemvMaxSlots;
  if (ns >= pl.nstage) {
    ns = pl.nstage;
  } else {
    // slots reused by warp groups taking alternate stages: nslots a multiple of Q
    const int ips = NB * 8;
    const int qg = ips >= kGemvWarps ? 1 : kGemvWarps / ips;
    ns -= ns % qg;
    if (ns < qg || ns < 2) return false;
  }
  while (ns * pl.slot_bytes < part && ns < kGemvMaxSlots) ++ns;
  if (ns * pl.slot_bytes < part) return false;
  pl.nslots = static_cast<int>(ns);
  const int64_t smem = b3_smem_bytes(pl.sc_bytes, pl.slot_bytes, pl.nslots);
  if (smem > max_smem) return false;
  pl.smem = static_cast<size_t>(smem);
  *out = pl;
  return true;
}

struct GtcPlan {
  int grid, R, T, S, nblk, gbox, nstages, ntiles;
  uint32_t box_stride, stage_bytes;
  GtcLayout lay;
};

// Geometry of the tensor-core decode kernel; false if these sizes do not fit it.
// Tiles of up to 128 rows (one per TMEM lane, at least 16).  With no more
// than sm_count tiles of 128 rows, K is split over S CTAs per tile so that
// tiles x S fills the SMs (each tile's activations are still read once); with
// more, a CTA runs T tiles in turn.
bool gtc_plan(int64_t M, int64_t N, int64_t K, int sm_count, int max_smem, GtcPlan* out) {
  if (M < 1 || M > kGtcMaxM || K % 1024 != 0 || K < 1024 || N < 1 || sm_count < 1) return false;
  GtcPlan pl;
  pl.nblk = static_cast<int>(K / 1024);
  const int64_t tiles128 = (N + kGtcMaxRows - 1) / kGtcMaxRows;
  int64_t tiles;
  if (tiles128 <= sm_count) {
    pl.T = 1;
    pl.S = static_cast<int>(std::max<int64_t>(
        1, std::min<int64_t>(std::min<int64_t>(pl.nblk, kGtcMaxSplits), sm_count / tiles128)));
    tiles = std::min<int64_t>(sm_count / pl.S, (N + 15) / 16);
    pl.R = static_cast<int>((N + tiles - 1) / tiles);
  } else {
    pl.S = 1;
    const int64_t per_cta = (N + sm_count - 1) / sm_count;
    pl.T = static_cast<int>((per_cta + kGtcMaxRows - 1) / kGtcMaxRows);
    pl.R = static_cast<int>((per_cta + pl.T - 1) / pl.T);
  }
  tiles = (N + pl.R - 1) / pl.R;
  pl.ntiles = static_cast<int>(tiles);
  const int64_t groups = (tiles + pl.T - 1) / pl.T;
  if (groups * pl.S > 2147483647LL) return false;
  pl.grid = static_cast<int>(groups * pl.S);
  pl.gbox = 8 * ((pl.nblk + pl.S - 1) / pl.S);
  if (pl.gbox > 256 || pl.R > kGtcMaxRows) return false;  // TMA box limits
  pl.box_stride = static_cast<uint32_t>(align_up(static_cast<int64_t>(pl.R) * 128, 1024));
  pl.stage_bytes = pl.box_stride + 4u * static_cast<uint32_t>(gtc_atom_bytes(static_cast<int>(M)));
  const int MT = gtc_capacity(static_cast<int>(M));  // info and sums sized for the kernel's token capacity
  const GtcLayout l0 = gtc_layout(MT, pl.R, pl.T, pl.gbox, 0, pl.stage_bytes);
  int64_t ns = (max_smem - l0.bytes - 64) / pl.stage_bytes;
  if (ns > 8) ns = 8;
  if (ns < 2) return false;
  pl.nstages = static_cast<int>(ns);
  pl.lay = gtc_layout(MT, pl.R, pl.T, pl.gbox, pl.nstages, pl.stage_bytes);
  if (pl.lay.bytes > max_smem) return false;
  *out = pl;
  return true;
}

// Workspace of the tensor-core decode beyond its activations: the K splits'
// partial sums [S][M][N] fp32 and one counter per tile.  A bound over every
// plan (S <= min(K / 1024, kGtcMaxSplits); tiles of 16 rows or more).
size_t gtc_extra_bytes(int f, int64_t M, int64_t N, int64_t K) {
  if (M > kGtcMaxM || K % 1024 != 0 || (f != TB_FMT_2BIT && f != TB_FMT_BASE3)) return 0;
  const int64_t smax = std::min<int64_t>(K / 1024, kGtcMaxSplits);
  const size_t part = static_cast<size_t>(smax * M * N * 4);
  const size_t cnt = static_cast<size_t>(4 * ((N + 15) / 16));
  return ((part + 255) & ~static_cast<size_t>(255)) + ((cnt + 255) & ~static_cast<size_t>(255));
}

constexpr int kB200Sms = 148;
constexpr int kB200SmemOptin = 232448;

// Base-3 decode serves up to kB3MaxM tokens, in chunks of kGemvMaxM.
constexpr int kB3MaxM = kB3TranscodeMinM - 1;

bool gemv_ok(const LinearArgs& a) {
  const int64_t maxm = a.f == TB_FMT_BASE3 ? kB3MaxM : (a.f == TB_FMT_1BIT ? 1 : kGemvMaxM);
  if (!(is_float_dtype(a.xt) && a.M >= 1 && a.M <= maxm && a.K % 1024 == 0 && fast_aligned(a) &&
        a.N < (int64_t(1) << 30)))
    return false;
  if (a.f == TB_FMT_1BIT) {
    // one token only, on the one-token kernel
    G1Plan p1;
    return g1_plan(a.N, a.K, kB200Sms, kB200SmemOptin, g1_fused(a.K), &p1, TB_FMT_1BIT);
  }
  if (a.f == TB_FMT_BASE3) {
    B3Plan pl;
    return b3_plan(std::min<int64_t>(a.M, kGemvMaxM), a.N, a.K, kB200Sms, kB200SmemOptin, &pl);
  }
  if (a.M == 1 && g1_preferred(a.N, a.K, kB200Sms)) {
    G1Plan p1;
    if (g1_plan(a.N, a.K, kB200Sms, kB200SmemOptin, g1_fused(a.K), &p1)) return true;
  }
  GemvPlan pl;
  return gemv_plan(a.M, a.N, a.K, kB200Sms, kB200SmemOptin, &pl);
}

bool gemv_tc_ok(const LinearArgs& a) {
  GtcPlan pl;
  // base-3: after re-encoding to 2-bit slots (8 tokens and more)
  const bool fmt_ok = a.f == TB_FMT_2BIT || (a.f == TB_FMT_BASE3 && a.M >= kB3TranscodeMinM);
  return is_float_dtype(a.xt) && fmt_ok && a.M >= 1 && a.M <= kGtcMaxM &&
         a.K % 1024 == 0 && fast_aligned(a) && a.N < (int64_t(1) << 30) &&
         gtc_plan(a.M, a.N, a.K, kB200Sms, kB200SmemOptin, &pl);
}

bool gemm_ok(const LinearArgs& a) {
  // base-3 is served by re-encoding to 2-bit slots first, which the workspace
  // holds from kB3TranscodeMinM tokens on (up to 16 tokens the tensor-core
  // decode comes first where its row limit allows)
  if (a.f == TB_FMT_BASE3 && a.M < kB3TranscodeMinM) return false;
  return is_float_dtype(a.xt) && a.K % 1024 == 0 && fast_aligned(a) &&
         (a.M + 127) / 128 <= 65535 && a.N < (int64_t(1) << 30) &&
         ((a.N + 255) / 256) * ((a.M + 127) / 128) < (int64_t(1) << 31);  // tile indices fit an int
}

bool gemm_i8_ok(const LinearArgs& a);

int auto_path(const LinearArgs& a) {
  if (a.xt == TB_INT8) return gemm_i8_ok(a) ? TB_PATH_GEMM : TB_PATH_SIMPLE;
  if (a.f == TB_FMT_1BIT) {
    // 1-bit: the one-token decode, else the GEMM
    if (gemv_ok(a)) return TB_PATH_GEMV;
    return gemm_ok(a) ? TB_PATH_GEMM : TB_PATH_SIMPLE;
  }
  // 2-bit: the one-token kernel where it is preferred (it rotates x itself
  // and overlaps consecutive calls), else the tensor-core decode, whose cost
  // hardly grows with M.  Measured on B200: 2 tokens 13.9 against 17.6 us
  // (17408 x 5120) and 17.8 against 24.9 us (5120 x 17408); one token on the
  // long-K down shape 16.5 against 18.7 us.
  if (a.f == TB_FMT_2BIT && !(a.M == 1 && g1_preferred(a.N, a.K, kB200Sms)) && gemv_tc_ok(a))
    return TB_PATH_GEMV_TC;
  if (gemv_ok(a)) return TB_PATH_GEMV;       // M <= 4 (2-bit), M <= 7 (base-3)
  if (gemv_tc_ok(a)) return TB_PATH_GEMV_TC;  // up to 16 tokens (base-3 re-encoded)
  if (gemm_ok(a)) return TB_PATH_GEMM;
  return TB_PATH_SIMPLE;
}

// ------------------------------------------------------------------ linear: GEMV
// Both kernels go out with programmatic dependent launch: the prep kernel
// waits inside for the previous kernel on the stream, the decode kernel's
// producer for the prep kernel (see gemv.cuh).
template <int M>
tb_status launch_gemv(const LinearArgs& a, const DevInfo* d, const GemvPlan& pl, const CUtensorMap& tm,
                      const GemvParams& p) {
  auto k = a.yt == TB_FP32 ? gemv_2bit_kernel<M, float> : gemv_2bit_kernel<M, __nv_bfloat16>;
  if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;
  return launch_pdl(k, dim3(pl.grid), dim3(kGemvThreads), pl.smem, a.st, tm, p);
}

// One token: gemv1_2bit_kernel, with the rotation inside it for K up to
// kG1FusedMaxBlocks 1024-blocks, else after prep_gemv1_kernel.
template <typename TIn, typename TOut, bool kFused, int kFmt>
tb_status launch_gemv1(const LinearArgs& a, const DevInfo* d, const G1Plan& pl, const CUtensorMap& tm,
                       const Gemv1Params& p) {
  auto pick = [&]() {
    switch (pl.TPW) {
      case 1: return gemv1_kernel<TIn, TOut, kFused, 1, kFmt>;
      case 2: return gemv1_kernel<TIn, TOut, kFused, 2, kFmt>;
      default: return gemv1_kernel<TIn, TOut, kFused, 4, kFmt>;
    }
  };
  auto k = pick();
  if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;
  return launch_pdl(k, dim3(pl.grid), dim3(kG1Threads), static_cast<size_t>(pl.lay.bytes), a.st, tm, p);
}

template <typename TIn, int kFmt>
tb_status run_gemv1_typed(const LinearArgs& a, const DevInfo* d, const G1Plan& pl) {
  CUtensorMap tm;
  // 2-bit: 128 bytes of a row per chunk, 128-byte swizzle; 1-bit: 64 bytes, 64-byte swizzle
  const uint64_t row_bytes = kFmt == kG1Fmt1Bit ? a.K / 8 : a.K / 4;
  if (make_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.packed, row_bytes, a.N, row_bytes, g1_box_bytes(kFmt),
                  static_cast<uint32_t>(pl.R),
                  kFmt == kG1Fmt1Bit ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B) != TB_OK)
    return TB_ERR_CUDA;
  Gemv1Params p;
  p.x = pl.fused ? a.x : nullptr;
  p.signs = a.signs;
  p.act = static_cast<const uint8_t*>(a.ws);
  p.scales = a.scales;
  p.y = a.y;
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.R = pl.R;
  p.RT = pl.RT;
  p.Wt = pl.Wt;
  p.Wk = pl.Wk;
  p.NB = pl.NB;
  p.nb_log2 = pl.nb_log2;
  p.nstage = pl.nstage;
  p.nslots = pl.nslots;
  p.box_stride = pl.box_stride;
  p.slot_bytes = pl.slot_bytes;
  p.off_act = pl.lay.off_act;
  p.off_sc = pl.lay.off_sc;
  p.off_red = pl.lay.off_red;
  p.off_bar = pl.lay.off_bar;
  if (!pl.fused) {
    const dim3 pgrid(static_cast<unsigned>((a.K / kHB + 3) / 4));
    if (launch_pdl(prep_gemv1_kernel<TIn, kFmt>, pgrid, dim3(128), 0, a.st, static_cast<const TIn*>(a.x),
                   a.signs, static_cast<uint8_t*>(a.ws), static_cast<int>(a.K)) != TB_OK)
      return TB_ERR_CUDA;
    return a.yt == TB_FP32 ? launch_gemv1<TIn, float, false, kFmt>(a, d, pl, tm, p)
                           : launch_gemv1<TIn, __nv_bfloat16, false, kFmt>(a, d, pl, tm, p);
  }
  return a.yt == TB_FP32 ? launch_gemv1<TIn, float, true, kFmt>(a, d, pl, tm, p)
                         : launch_gemv1<TIn, __nv_bfloat16, true, kFmt>(a, d, pl, tm, p);
}

template <typename TIn>
tb_status run_gemv_typed(const LinearArgs& a, const DevInfo* d) {
  if (a.f == TB_FMT_1BIT) {
    G1Plan p1;
    if (a.M != 1 || !g1_plan(a.N, a.K, d->sm_count, d->max_smem_optin, g1_fused(a.K), &p1, TB_FMT_1BIT))
      return TB_ERR_SHAPE;
    return run_gemv1_typed<TIn, kG1Fmt1Bit>(a, d, p1);
  }
  if (a.M == 1 && g1_preferred(a.N, a.K, d->sm_count)) {
    G1Plan p1;
    if (g1_plan(a.N, a.K, d->sm_count, d->max_smem_optin, g1_fused(a.K), &p1))
      return run_gemv1_typed<TIn, kG1Fmt2Bit>(a, d, p1);
  }
  GemvPlan pl;
  if (!gemv_plan(a.M, a.N, a.K, d->sm_count, d->max_smem_optin, &pl)) return TB_ERR_SHAPE;
  uint8_t* act = static_cast<uint8_t*>(a.ws);
  CUtensorMap tm;
  if (make_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.packed, a.K / 4, a.N, a.K / 4, 128,
                  static_cast<uint32_t>(pl.R), CU_TENSOR_MAP_SWIZZLE_128B) != TB_OK)
    return TB_ERR_CUDA;
  const dim3 pgrid(static_cast<unsigned>(a.K / kHB), static_cast<unsigned>(a.M));
  if (launch_pdl(prep_gemv_kernel<TIn>, pgrid, dim3(kHThreads), 0, a.st, static_cast<const TIn*>(a.x), a.signs, act,
                 static_cast<int>(a.K), pl.NB) != TB_OK)
    return TB_ERR_CUDA;
  GemvParams p;
  p.act = act;
  p.scales = a.scales;
  p.y = a.y;
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.R = pl.R;
  p.RT = pl.RT;
  p.NB = pl.NB;
  p.nstage = pl.nstage;
  p.nslots = pl.nslots;
  p.box_stride = pl.box_stride;
  p.slot_bytes = pl.slot_bytes;
  p.sc_bytes = pl.sc_bytes;
  if (a.M == 1) {
    // dynamic item distribution: its own slot count (no warp-group constraint)
    // and a partial-sum buffer of one float per item and row
    const int64_t fixed = gemv_dyn_smem_bytes(pl.sc_bytes, 0, 0, pl.nstage, pl.NB, pl.RT);
    int64_t ns = (d->max_smem_optin - fixed) / pl.slot_bytes;
    if (ns > kGemvMaxSlots) ns = kGemvMaxSlots;
    if (ns > pl.nstage) ns = pl.nstage;
    if (ns >= 2 || (ns >= 1 && pl.nstage == 1)) {
      p.nslots = static_cast<int>(ns);
      const size_t smem = static_cast<size_t>(
          gemv_dyn_smem_bytes(pl.sc_bytes, pl.slot_bytes, p.nslots, pl.nstage, pl.NB, pl.RT));
      auto k = a.yt == TB_FP32 ? gemv_2bit_dyn_kernel<float> : gemv_2bit_dyn_kernel<__nv_bfloat16>;
      if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;
      return launch_pdl(k, dim3(pl.grid), dim3(kGemvThreads), smem, a.st, tm, p);
    }
  }
  switch (static_cast<int>(a.M)) {
    case 1: return launch_gemv<1>(a, d, pl, tm, p);
    case 2: return launch_gemv<2>(a, d, pl, tm, p);
    case 3: return launch_gemv<3>(a, d, pl, tm, p);
    case 4: return launch_gemv<4>(a, d, pl, tm, p);
    default: return TB_ERR_SHAPE;
  }
}

template <typename TIn>
tb_status run_gemv_tc_typed(const LinearArgs& a, const DevInfo* d, const GtcPlan& pl) {
  uint8_t* act = static_cast<uint8_t*>(a.ws);
  const size_t act_bytes = (static_cast<size_t>(gtc_ws_bytes(a.M, a.K)) + 255) & ~static_cast<size_t>(255);
  float* part = reinterpret_cast<float*>(act + act_bytes);
  const size_t part_bytes =
      (static_cast<size_t>(pl.S) * a.M * a.N * 4 + 255) & ~static_cast<size_t>(255);
  uint32_t* cnt = reinterpret_cast<uint32_t*>(act + act_bytes + part_bytes);
  if (act_bytes + part_bytes + 4 * static_cast<size_t>(pl.ntiles) > a.ws_bytes) return TB_ERR_WORKSPACE;
  const dim3 pgrid(static_cast<unsigned>(a.M), static_cast<unsigned>(a.K / kHB));
  // a plain launch: measured on B200, letting it start early under the
  // previous decode kernel cost 2-4 us per call
  prep_gemv_tc_kernel<TIn><<<pgrid, kHThreads, 0, a.st>>>(static_cast<const TIn*>(a.x), a.signs, act, a.K,
                                                          static_cast<int>(a.M), cnt, pl.S > 1 ? pl.ntiles : 0);
  if (launch_status() != TB_OK) return TB_ERR_CUDA;
  CUtensorMap tm_w, tm_s;
  if (make_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, a.K / 16, a.N, a.K / 4, 32,
                  static_cast<uint32_t>(pl.R), CU_TENSOR_MAP_SWIZZLE_128B) != TB_OK)
    return TB_ERR_CUDA;
  if (make_map_2d(&tm_s, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.scales, a.K / 128, a.N, (a.K / 128) * 2,
                  static_cast<uint32_t>(pl.gbox), static_cast<uint32_t>(pl.R)) != TB_OK)
    return TB_ERR_CUDA;
  GemvTcParams p;
  p.act = act;
  p.y = a.y;
  p.part = part;
  p.cnt = cnt;
  p.M = static_cast<int>(a.M);
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.G = static_cast<int>(a.K / 128);
  p.R = pl.R;
  p.T = pl.T;
  p.S = pl.S;
  p.nblk = pl.nblk;
  p.gbox = pl.gbox;
  p.sc_tile = static_cast<int>(gtc_sc_tile_bytes(pl.R, pl.gbox) / 2);
  p.nstages = pl.nstages;
  p.box_stride = pl.box_stride;
  p.stage_bytes = pl.stage_bytes;
  p.off_sc = pl.lay.off_sc;
  p.off_info = pl.lay.off_info;
  p.off_red = pl.lay.off_red;
  p.off_bar = pl.lay.off_bar;
  const size_t smem = static_cast<size_t>(pl.lay.bytes);
#define TB_GTC_CASE(MM)                                                                          \
  case MM:                                                                                       \
    if (a.yt == TB_FP32) {                                                                       \
      auto k = gemv_tc_kernel<MM, float>;                                                        \
      if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;                                         \
      return launch_pdl(k, dim3(pl.grid), dim3(kGtcThreads), smem, a.st, tm_w, tm_s, p);         \
    } else {                                                                                     \
      auto k = gemv_tc_kernel<MM, __nv_bfloat16>;                                                \
      if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;                                         \
      return launch_pdl(k, dim3(pl.grid), dim3(kGtcThreads), smem, a.st, tm_w, tm_s, p);         \
    }
  switch (gtc_capacity(static_cast<int>(a.M))) {
    TB_GTC_CASE(4)
    TB_GTC_CASE(8)
    TB_GTC_CASE(16)
    default: return TB_ERR_SHAPE;
  }
#undef TB_GTC_CASE
}

tb_status run_gemv_tc(const LinearArgs& a, const DevInfo* d) {
  if (a.f == TB_FMT_BASE3) {
    const size_t tb = b3_transcode_bytes(a.f, a.M, a.N, a.K);
    const int64_t ngroups = a.N * (a.K / 128);
    transcode_b3_to_2bit_kernel<<<static_cast<unsigned>((ngroups + 255) / 256), 256, 0, a.st>>>(
        a.packed, static_cast<uint4*>(a.ws), ngroups);
    if (launch_status() != TB_OK) return TB_ERR_CUDA;
    LinearArgs c = a;
    c.f = TB_FMT_2BIT;
    c.packed = static_cast<const uint8_t*>(a.ws);
    c.ws = static_cast<uint8_t*>(a.ws) + tb;
    c.ws_bytes = a.ws_bytes - tb;
    return run_gemv_tc(c, d);
  }
  GtcPlan pl;
  if (!gtc_plan(a.M, a.N, a.K, d->sm_count, d->max_smem_optin, &pl)) return TB_ERR_SHAPE;
  switch (a.xt) {
    case TB_BF16: return run_gemv_tc_typed<__nv_bfloat16>(a, d, pl);
    case TB_FP16: return run_gemv_tc_typed<__half>(a, d, pl);
    default: return run_gemv_tc_typed<float>(a, d, pl);
  }
}

template <int M>
tb_status launch_b3(const LinearArgs& a, const DevInfo* d, const B3Plan& pl, const CUtensorMap& tm,
                    const GemvB3Params& p) {
  auto k = a.yt == TB_FP32 ? gemv_b3_kernel<M, float> : gemv_b3_kernel<M, __nv_bfloat16>;
  if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;
  return launch_pdl(k, dim3(pl.grid), dim3(kGemvThreads), pl.smem, a.st, tm, p);
}

template <typename TIn>
tb_status run_b3_typed(const LinearArgs& a, const DevInfo* d) {
  B3Plan pl;
  if (!b3_plan(a.M, a.N, a.K, d->sm_count, d->max_smem_optin, &pl)) return TB_ERR_SHAPE;
  uint8_t* act = static_cast<uint8_t*>(a.ws);
  const int64_t row_bytes = (a.K / 128) * kB3GroupBytes;
  CUtensorMap tm;
  if (make_map_2d(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.packed, row_bytes, a.N, row_bytes, kB3BlockBytes,
                  static_cast<uint32_t>(pl.R)) != TB_OK)
    return TB_ERR_CUDA;
  const dim3 pgrid(static_cast<unsigned>(a.K / kHB), static_cast<unsigned>(a.M));
  if (launch_pdl(prep_b3_kernel<TIn>, pgrid, dim3(kHThreads), 0, a.st, static_cast<const TIn*>(a.x), a.signs, act,
                 static_cast<int>(a.K), pl.NB) != TB_OK)
    return TB_ERR_CUDA;
  GemvB3Params p;
  p.act = act;
  p.scales = a.scales;
  p.y = a.y;
  p.N = static_cast<int>(a.N);
  p.K = static_cast<int>(a.K);
  p.R = pl.R;
  p.RT = pl.RT;
  p.NB = pl.NB;
  p.nstage = pl.nstage;
  p.nslots = pl.nslots;
  p.box_stride = pl.box_stride;
  p.slot_bytes = pl.slot_bytes;
  p.sc_bytes = pl.sc_bytes;
  switch (static_cast<int>(a.M)) {
    case 1: return launch_b3<1>(a, d, pl, tm, p);
    case 2: return launch_b3<2>(a, d, pl, tm, p);
    case 3: return launch_b3<3>(a, d, pl, tm, p);
    case 4: return launch_b3<4>(a, d, pl, tm, p);
    default: return TB_ERR_SHAPE;
  }
}

tb_status run_gemv(const LinearArgs& a, const DevInfo* d) {
  if (a.f == TB_FMT_BASE3) {
    // more than kGemvMaxM tokens: one pass over the weights per chunk of tokens
    for (int64_t m0 = 0; m0 < a.M; m0 += kGemvMaxM) {
      LinearArgs c = a;
      c.M = std::min<int64_t>(kGemvMaxM, a.M - m0);
      c.x = static_cast<const uint8_t*>(a.x) + m0 * a.K * dtype_size(a.xt);
      c.y = static_cast<uint8_t*>(a.y) + m0 * a.N * dtype_size(a.yt);
      tb_status st;
      switch (a.xt) {
        case TB_BF16: st = run_b3_typed<__nv_bfloat16>(c, d); break;
        case TB_FP16: st = run_b3_typed<__half>(c, d); break;
        default: st = run_b3_typed<float>(c, d); break;
      }
      if (st != TB_OK) return st;
    }
    return TB_OK;
  }
  switch (a.xt) {
    case TB_BF16: return run_gemv_typed<__nv_bfloat16>(a, d);
    case TB_FP16: return run_gemv_typed<__half>(a, d);
    default: return run_gemv_typed<float>(a, d);
  }
}

// ------------------------------------------------------------------ linear: plain kernel
template <int FMT>
tb_status run_simple_fmt(const LinearArgs& a) {
  const dim3 grid(static_cast<unsigned>((a.N + kSimpleWarps - 1) / kSimpleWarps));
  const dim3 block(32 * kSimpleWarps);
  const int M = static_cast<int>(a.M), N = static_cast<int>(a.N), K = static_cast<int>(a.K);
  const __half* sc = reinterpret_cast<const __half*>(a.scales);
  if (a.xt == TB_INT8) {
    simple_linear_kernel<FMT, true, int8_t, int32_t><<<grid, block, 0, a.st>>>(
        static_cast<const int8_t*>(a.x), a.packed, sc, static_cast<int32_t*>(a.y), M, N, K);
    return launch_status();
  }
  float* xf = static_cast<float*>(a.ws);
  if (a.signs != nullptr) {
    const dim3 pg(static_cast<unsigned>(a.M), static_cast<unsigned>(a.K / kHB));
    switch (a.xt) {
      case TB_BF16:
        prep_store_kernel<__nv_bfloat16, float><<<pg, kHThreads, 0, a.st>>>(
            static_cast<const __nv_bfloat16*>(a.x), a.signs, xf, a.K);
        break;
      case TB_FP16:
        prep_store_kernel<__half, float><<<pg, kHThreads, 0, a.st>>>(static_cast<const __half*>(a.x),
                                                                      a.signs, xf, a.K);
        break;
      default:
        prep_store_kernel<float, float><<<pg, kHThreads, 0, a.st>>>(static_cast<const float*>(a.x),
                                                                     a.signs, xf, a.K);
        break;
    }
  } else {
    const int64_t n = a.M * a.K;
    const unsigned g = static_cast<unsigned>((n + 255) / 256);
    switch (a.xt) {
      case TB_BF16:
        convert_kernel<__nv_bfloat16, float><<<g, 256, 0, a.st>>>(static_cast<const __nv_bfloat16*>(a.x),
                                                                  xf, n);
        break;
      case TB_FP16:
        convert_kernel<__half, float><<<g, 256, 0, a.st>>>(static_cast<const __half*>(a.x), xf, n);
        break;
      default:
        convert_kernel<float, float><<<g, 256, 0, a.st>>>(static_cast<const float*>(a.x), xf, n);
        break;
    }
  }
  if (launch_status() != TB_OK) return TB_ERR_CUDA;
  if (a.yt == TB_FP32)
    return launch_pdl(simple_linear_kernel<FMT, false, float, float>, grid, block, 0, a.st,
                      static_cast<const float*>(xf), a.packed, sc, static_cast<float*>(a.y), M, N, K);
  return launch_pdl(simple_linear_kernel<FMT, false, float, __nv_bfloat16>, grid, block, 0, a.st,
                    static_cast<const float*>(xf), a.packed, sc, static_cast<__nv_bfloat16*>(a.y), M,
                    N, K);
}

tb_status run_simple(const LinearArgs& a) {
  switch (a.f) {
    case TB_FMT_2BIT: return run_simple_fmt<0>(a);
    case TB_FMT_BASE3: return run_simple_fmt<1>(a);
    default: return run_simple_fmt<2>(a);
  }
}

// ------------------------------------------------------------------ linear: tensor-core kernel
template <typename TIn>
void launch_prep_gemm(const LinearArgs& a, __half* xh) {
  const dim3 pg(static_cast<unsigned>(a.M), static_cast<unsigned>(a.K / kHB));
  prep_gemm_kernel<TIn><<<pg, kHThreads, 0, a.st>>>(static_cast<const TIn*>(a.x), a.signs, xh, a.K);
}

tb_status run_gemm_2bit(const LinearArgs& a, const DevInfo* d);

tb_status run_gemm(const LinearArgs& a, const DevInfo* d) {
  if (a.f != TB_FMT_BASE3) return run_gemm_2bit(a, d);
  const size_t tb = b3_transcode_bytes(a.f, a.M, a.N, a.K);
  const int64_t ngroups = a.N * (a.K / 128);
  transcode_b3_to_2bit_kernel<<<static_cast<unsigned>((ngroups + 255) / 256), 256, 0, a.st>>>(
      a.packed, static_cast<uint4*>(a.ws), ngroups);
  if (launch_status() != TB_OK) return TB_ERR_CUDA;
  LinearArgs c = a;
  c.f = TB_FMT_2BIT;
  c.packed = static_cast<const uint8_t*>(a.ws);
  c.ws = static_cast<uint8_t*>(a.ws) + tb;
  c.ws_bytes = a.ws_bytes - tb;
  return run_gemm_2bit(c, d);
}

// 2-bit slots or 1-bit codes (base-3 arrives re-encoded to 2-bit slots).
tb_status run_gemm_2bit(const LinearArgs& a, const DevInfo* d) {
  const bool one_bit = a.f == TB_FMT_1BIT;
  __half* xh = static_cast<__half*>(a.ws);
  switch (a.xt) {
    case TB_BF16: launch_prep_gemm<__nv_bfloat16>(a, xh); break;
    case TB_FP16: launch_prep_gemm<__half>(a, xh); break;
    default: launch_prep_gemm<float>(a, xh); break;
  }
  if (launch_status() != TB_OK) return TB_ERR_CUDA;
  // token tile: 256, or 128 up to 128 tokens.  Measured on B200, a pair
  // MMA with A in TMEM takes about 130 cycles at N = 128 and at N = 256 alike
  // (148 at N = 192), so narrower tiles only pay where the tokens are few.
  const int64_t pairs_n = (a.N + kGpPairRows - 1) / kGpPairRows;
  const int bt = a.M <= 128 ? 128 : 256;
  CUtensorMap tm_x, tm_w;
  if (make_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, xh, a.K, a.M, a.K * 2, gp_atom_k(false),
                  static_cast<uint32_t>(bt / 2), CU_TENSOR_MAP_SWIZZLE_128B) != TB_OK)
    return TB_ERR_CUDA;
  // the 128 codes of a stage: 32 bytes of a row (2-bit) or 16 (1-bit)
  const uint64_t wrow = one_bit ? a.K / 8 : a.K / 4;
  if (make_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, wrow / 4, a.N, wrow,
                  static_cast<uint32_t>(gp_w_row_bytes(one_bit ? 2 : 0, false) / 4), static_cast<uint32_t>(kGpRows)) !=
          TB_OK)
    return TB_ERR_CUDA;
  GemmParams gp;
  gp.M = static_cast<int>(a.M);
  gp.N = static_cast<int>(a.N);
  gp.K = static_cast<int>(a.K);
  gp.y = a.y;
  gp.scales = a.scales;
  GemmPairTiles tl;
  tl.tiles_n = static_cast<int>(pairs_n);
  tl.tiles_m = static_cast<int>((a.M + bt - 1) / bt);
  // persistent: one cluster per SM pair at most, each walking its tiles
  const int64_t ntiles = pairs_n * tl.tiles_m;
  const dim3 grid(static_cast<unsigned>(2 * std::min<int64_t>(ntiles, std::max(1, d->sm_count / 2))));
#define TB_GP_LAUNCH(BT, F)                                                                                   \
  {                                                                                                           \
    if (a.yt == TB_FP32) {                                                                                    \
      auto k = gemm_pair_kernel<BT, float, F, false>;                                                         \
      if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;                                                      \
      return launch_pdl(k, grid, dim3(kGpThreads), static_cast<size_t>(gp_smem_bytes(BT, F, false)), a.st,    \
                        tm_x, tm_w, gp, tl);                                                                  \
    }                                                                                                         \
    auto k = gemm_pair_kernel<BT, __nv_bfloat16, F, false>;                                                   \
    if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;                                                        \
    return launch_pdl(k, grid, dim3(kGpThreads), static_cast<size_t>(gp_smem_bytes(BT, F, false)), a.st, tm_x, \
                      tm_w, gp, tl);                                                                          \
  }
  if (bt == 128) {
    if (one_bit) TB_GP_LAUNCH(128, 2)
    TB_GP_LAUNCH(128, 0)
  }
  if (one_bit) TB_GP_LAUNCH(256, 2)
  TB_GP_LAUNCH(256, 0)
#undef TB_GP_LAUNCH
}

// ------------------------------------------------------------------ linear: integer-mode GEMM
// Integer mode on the tensor cores from this many tokens (fewer: the plain
// kernel, exact as well).
constexpr int kGi8MinM = 16;

bool gemm_i8_ok(const LinearArgs& a) {
  if (a.xt != TB_INT8 || a.M < kGi8MinM || a.K % 128 != 0 || (a.M + 127) / 128 > 65535 ||
      a.N >= (int64_t(1) << 30) || ((a.N + 255) / 256) * ((a.M + 127) / 128) >= (int64_t(1) << 31))
    return false;
  if (!(aligned(a.x, 16) && aligned(a.packed, 16) && aligned(a.y, 16))) return false;
  // base-3: re-encoded to 2-bit slots first, in a workspace the caller passed
  if (a.f == TB_FMT_BASE3)
    return a.ws != nullptr && aligned(a.ws, 16) && a.ws_bytes >= b3_transcode_bytes(a.f, a.M, a.N, a.K);
  return true;
}

tb_status run_gemm_i8(const LinearArgs& a, const DevInfo* d) {
  if (a.f == TB_FMT_BASE3) {
    const int64_t ngroups = a.N * (a.K / 128);
    transcode_b3_to_2bit_kernel<<<static_cast<unsigned>((ngroups + 255) / 256), 256, 0, a.st>>>(
        a.packed, static_cast<uint4*>(a.ws), ngroups);
    if (launch_status() != TB_OK) return TB_ERR_CUDA;
    LinearArgs c = a;
    c.f = TB_FMT_2BIT;
    c.packed = static_cast<const uint8_t*>(a.ws);
    return run_gemm_i8(c, d);
  }
  const bool one_bit = a.f == TB_FMT_1BIT;
  // the CTA-pair kernel of the fp16 GEMM in integer mode (kind::i8)
  const int64_t pairs_n = (a.N + kGpPairRows - 1) / kGpPairRows;
  const int bt = a.M <= 128 ? 128 : 256;
  CUtensorMap tm_x, tm_w;
  if (make_map_2d(&tm_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.x, a.K, a.M, a.K, gp_atom_k(true),
                  static_cast<uint32_t>(bt / 2), CU_TENSOR_MAP_SWIZZLE_128B) != TB_OK)
    return TB_ERR_CUDA;
  const uint64_t wrow = one_bit ? a.K / 8 : a.K / 4;
  if (make_map_2d(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.packed, wrow / 4, a.N, wrow,
                  static_cast<uint32_t>(gp_w_row_bytes(one_bit ? 2 : 0, true) / 4), static_cast<uint32_t>(kGpRows)) !=
      TB_OK)
    return TB_ERR_CUDA;
  GemmParams gp;
  gp.M = static_cast<int>(a.M);
  gp.N = static_cast<int>(a.N);
  gp.K = static_cast<int>(a.K);
  gp.y = a.y;
  gp.scales = nullptr;
  GemmPairTiles tl;
  tl.tiles_n = static_cast<int>(pairs_n);
  tl.tiles_m = static_cast<int>((a.M + bt - 1) / bt);
  const int64_t ntiles = pairs_n * tl.tiles_m;
  const dim3 grid(static_cast<unsigned>(2 * std::min<int64_t>(ntiles, std::max(1, d->sm_count / 2))));
#define TB_GI8_LAUNCH(BT, F)                                                                                  \
  {                                                                                                           \
    auto k = gemm_pair_kernel<BT, int32_t, F, true>;                                                          \
    if (allow_smem(k, d) != TB_OK) return TB_ERR_CUDA;                                                        \
    return launch_pdl(k, grid, dim3(kGpThreads), static_cast<size_t>(gp_smem_bytes(BT, F, true)), a.st, tm_x, \
                      tm_w, gp, tl);                                                                          \
  }
  if (bt == 128) {
    if (one_bit) TB_GI8_LAUNCH(128, 2)
    TB_GI8_LAUNCH(128, 0)
  }
  if (one_bit) TB_GI8_LAUNCH(256, 2)
  TB_GI8_LAUNCH(256, 0)
#undef TB_GI8_LAUNCH
}

bool known_format(int f) { return f == TB_FMT_2BIT || f == TB_FMT_BASE3 || f == TB_FMT_1BIT; }

tb_status validate_linear(const LinearArgs& a) {
  if (!known_format(a.f)) return TB_ERR_FORMAT;
  const bool int_mode = a.xt == TB_INT8;
  if (a.x == nullptr || a.packed == nullptr || a.y == nullptr) return TB_ERR_NULL;
  if (!int_mode && a.scales == nullptr) return TB_ERR_NULL;
  if (a.M < 1 || a.N < 1 || a.K < 128 || a.K % 128 != 0) return TB_ERR_SHAPE;
  if (a.M > kMaxDim || a.N > kMaxDim || a.K > kMaxDim) return TB_ERR_SHAPE;
  if (a.M * a.K > (int64_t(1) << 40) || a.N * a.K > (int64_t(1) << 44)) return TB_ERR_SHAPE;
  if (int_mode) {
    if (a.yt != TB_INT32) return TB_ERR_DTYPE;
    if (a.signs != nullptr) return TB_ERR_DTYPE;
  } else {
    if (!is_float_dtype(a.xt)) return TB_ERR_DTYPE;
    if (a.yt != TB_FP32 && a.yt != TB_BF16) return TB_ERR_DTYPE;
    if (a.signs != nullptr && a.K % 1024 != 0) return TB_ERR_SHAPE;
  }
  if (!aligned(a.x, dtype_size(a.xt)) || !aligned(a.y, dtype_size(a.yt)) ||
      (!int_mode && !aligned(a.scales, 2)))
    return TB_ERR_ALIGN;
  if (a.signs != nullptr && !aligned(a.signs, 8)) return TB_ERR_ALIGN;
  if (a.f == TB_FMT_BASE3 && !aligned(a.packed, 2)) return TB_ERR_ALIGN;
  if (!int_mode) {
    if (a.ws == nullptr || a.ws_bytes < required_ws(a.f, a.M, a.N, a.K)) return TB_ERR_WORKSPACE;
    if (!aligned(a.ws, 16)) return TB_ERR_ALIGN;
  }
  return TB_OK;
}

tb_status linear_impl(const LinearArgs& a, int path) {
  tb_status st = validate_linear(a);
  if (st != TB_OK) return st;
  if (path == TB_PATH_AUTO) path = auto_path(a);
  if (path == TB_PATH_GEMV && !gemv_ok(a)) return TB_ERR_SHAPE;
  if (path == TB_PATH_GEMM && !(a.xt == TB_INT8 ? gemm_i8_ok(a) : gemm_ok(a))) return TB_ERR_SHAPE;
  if (path == TB_PATH_GEMV_TC && !gemv_tc_ok(a)) return TB_ERR_SHAPE;
  if (path != TB_PATH_GEMV && path != TB_PATH_GEMM && path != TB_PATH_SIMPLE && path != TB_PATH_GEMV_TC)
    return TB_ERR_SHAPE;
  const DevInfo* d = nullptr;
  st = current_device(&d);
  if (st != TB_OK) return st;
  switch (path) {
    case TB_PATH_GEMV: return run_gemv(a, d);
    case TB_PATH_GEMM: return a.xt == TB_INT8 ? run_gemm_i8(a, d) : run_gemm(a, d);
    case TB_PATH_GEMV_TC: return run_gemv_tc(a, d);
    default: return run_simple(a);
  }
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char* tb_status_string(tb_status st) {
  switch (st) {
    case TB_OK: return "ok";
    case TB_ERR_NULL: return "null pointer";
    case TB_ERR_SHAPE: return "bad shape";
    case TB_ERR_DTYPE: return "bad dtype";
    case TB_ERR_FORMAT: return "bad format";
    case TB_ERR_ALIGN: return "bad alignment";
    case TB_ERR_CUDA: return "cuda error";
    case TB_ERR_WORKSPACE: return "workspace missing or too small";
    case TB_ERR_DEVICE: return "device is not sm_100";
    default: return "unknown status";
  }
}

int tb_version(void) { return kVersion; }

size_t tb_packed_bytes(tb_format f, int64_t N, int64_t K) {
  if (N <= 0 || K <= 0 || K % 128 != 0) return 0;
  if (f == TB_FMT_2BIT) return static_cast<size_t>(N) * static_cast<size_t>(K / 4);
  if (f == TB_FMT_BASE3) return static_cast<size_t>(N) * static_cast<size_t>(K / 128) * 26;
  if (f == TB_FMT_1BIT) return static_cast<size_t>(N) * static_cast<size_t>(K / 8);
  return 0;
}

tb_status tb_pack_ternary(tb_format f, const int8_t* codes, int64_t N, int64_t K, uint8_t* packed,
                          uint32_t* d_invalid_count, void* stream) {
  if (!known_format(f)) return TB_ERR_FORMAT;
  if (codes == nullptr || packed == nullptr) return TB_ERR_NULL;
  if (N <= 0 || K <= 0 || K % 128 != 0 || N > kMaxDim || K > kMaxDim) return TB_ERR_SHAPE;
  if (!aligned(codes, 16) || !aligned(packed, 16) ||
      (d_invalid_count != nullptr && !aligned(d_invalid_count, 4)))
    return TB_ERR_ALIGN;
  const DevInfo* d = nullptr;
  const tb_status st = current_device(&d);
  if (st != TB_OK) return st;
  const cudaStream_t s = as_stream(stream);
  if (f == TB_FMT_2BIT) {
    const int64_t nw = N * K / 16;
    pack_2bit_kernel<<<static_cast<unsigned>((nw + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const int4*>(codes), reinterpret_cast<uint32_t*>(packed), nw, d_invalid_count);
  } else if (f == TB_FMT_1BIT) {
    const int64_t nw = N * K / 32;
    pack_1bit_kernel<<<static_cast<unsigned>((nw + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const int4*>(codes), reinterpret_cast<uint32_t*>(packed), nw, d_invalid_count);
  } else {
    const int64_t ng = N * K / 128;
    pack_base3_kernel<<<static_cast<unsigned>((ng + 127) / 128), 128, 0, s>>>(
        reinterpret_cast<const int4*>(codes), reinterpret_cast<uint16_t*>(packed), ng, d_invalid_count);
  }
  return launch_status();
}

tb_status tb_unpack_ternary(tb_format f, const uint8_t* packed, int64_t N, int64_t K, int8_t* codes,
                            uint32_t* d_invalid_count, void* stream) {
  if (!known_format(f)) return TB_ERR_FORMAT;
  if (codes == nullptr || packed == nullptr) return TB_ERR_NULL;
  if (N <= 0 || K <= 0 || K % 128 != 0 || N > kMaxDim || K > kMaxDim) return TB_ERR_SHAPE;
  if (!aligned(codes, 16) || !aligned(packed, 16) ||
      (d_invalid_count != nullptr && !aligned(d_invalid_count, 4)))
    return TB_ERR_ALIGN;
  const DevInfo* d = nullptr;
  const tb_status st = current_device(&d);
  if (st != TB_OK) return st;
  const cudaStream_t s = as_stream(stream);
  if (f == TB_FMT_2BIT) {
    const int64_t nw = N * K / 16;
    unpack_2bit_kernel<<<static_cast<unsigned>((nw + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint32_t*>(packed), reinterpret_cast<int4*>(codes), nw, d_invalid_count);
  } else if (f == TB_FMT_1BIT) {
    const int64_t nw = N * K / 32;
    unpack_1bit_kernel<<<static_cast<unsigned>((nw + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const uint32_t*>(packed), reinterpret_cast<int4*>(codes), nw);
  } else {
    const int64_t ng = N * K / 128;
    unpack_base3_kernel<<<static_cast<unsigned>((ng + 127) / 128), 128, 0, s>>>(
        reinterpret_cast<const uint16_t*>(packed), reinterpret_cast<int4*>(codes), ng, d_invalid_count);
  }
  return launch_status();
}

tb_status tb_hadamard_rotate(const void* x, tb_dtype xt, void* y, tb_dtype yt, const int8_t* signs,
                             int64_t M, int64_t K, int inverse, void* stream) {
  if (x == nullptr || y == nullptr || signs == nullptr) return TB_ERR_NULL;
  if (!is_float_dtype(xt) || !is_float_dtype(yt)) return TB_ERR_DTYPE;
  if (M < 1 || K < 1024 || K % 1024 != 0 || M > kMaxDim || K / 1024 > 65535) return TB_ERR_SHAPE;
  if (x == y && xt != yt) return TB_ERR_DTYPE;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(signs, 8)) return TB_ERR_ALIGN;
  const DevInfo* d = nullptr;
  const tb_status st = current_device(&d);
  if (st != TB_OK) return st;
  const cudaStream_t s = as_stream(stream);
  switch (xt) {
    case TB_BF16: launch_rotate_out<__nv_bfloat16>(yt, x, y, signs, M, K, inverse != 0, s); break;
    case TB_FP16: launch_rotate_out<__half>(yt, x, y, signs, M, K, inverse != 0, s); break;
    default: launch_rotate_out<float>(yt, x, y, signs, M, K, inverse != 0, s); break;
  }
  return launch_status();
}

tb_status tb_prepare_weights(const void* w, tb_dtype wt, const int8_t* signs, int64_t N, int64_t K, tb_format f,
                             uint8_t* packed, uint16_t* scales, void* stream) {
  if (f != TB_FMT_2BIT && f != TB_FMT_BASE3) return TB_ERR_FORMAT;
  if (w == nullptr || packed == nullptr || scales == nullptr) return TB_ERR_NULL;
  if (!is_float_dtype(wt)) return TB_ERR_DTYPE;
  if (N < 1 || K < 1024 || K % 1024 != 0 || K > kMaxDim || K / 1024 > 65535 ||
      (N + kPwWarps - 1) / kPwWarps > 65535)
    return TB_ERR_SHAPE;
  if (!aligned(w, 4) || !aligned(packed, 16) || !aligned(scales, 2) || (signs != nullptr && !aligned(signs, 8)))
    return TB_ERR_ALIGN;
  const DevInfo* d = nullptr;
  const tb_status st = current_device(&d);
  if (st != TB_OK) return st;
  const cudaStream_t s = as_stream(stream);
  const dim3 grid(static_cast<unsigned>(K / 1024), static_cast<unsigned>((N + kPwWarps - 1) / kPwWarps));
  const dim3 block(32 * kPwWarps);
  const int k = static_cast<int>(K);
#define TB_PW(T)                                                                                                  \
  do {                                                                                                          \
    if (f == TB_FMT_2BIT)                                                                                       \
      prepare_weights_kernel<T, 0><<<grid, block, 0, s>>>(static_cast<const T*>(w), signs, packed, scales, N, k); \
    else                                                                                                        \
      prepare_weights_kernel<T, 1><<<grid, block, 0, s>>>(static_cast<const T*>(w), signs, packed, scales, N, k); \
  } while (0)
  switch (wt) {
    case TB_BF16: TB_PW(__nv_bfloat16); break;
    case TB_FP16: TB_PW(__half); break;
    default: TB_PW(float); break;
  }
#undef TB_PW
  return launch_status();
}

size_t tb_ternary_linear_workspace(tb_format f, int64_t M, int64_t N, int64_t K) {
  if (!known_format(f) || M < 1 || N < 1 || K < 128 || K % 128 != 0) return 0;
  return required_ws(f, M, N, K);
}

tb_status tb_ternary_linear_ex(const void* x, tb_dtype xt, const uint8_t* packed, const uint16_t* scales,
                               tb_format f, int64_t M, int64_t N, int64_t K, const int8_t* signs,
                               void* y, tb_dtype yt, void* workspace, size_t ws_bytes, tb_path path,
                               void* stream) {
  LinearArgs a{x, xt, packed, scales, f, M, N, K, signs, y, yt, workspace, ws_bytes, as_stream(stream)};
  return linear_impl(a, path);
}

tb_status tb_ternary_linear(const void* x, tb_dtype xt, const uint8_t* packed, const uint16_t* scales,
                            tb_format f, int64_t M, int64_t N, int64_t K, const int8_t* signs, void* y,
                            tb_dtype yt, void* workspace, size_t ws_bytes, void* stream) {
  return tb_ternary_linear_ex(x, xt, packed, scales, f, M, N, K, signs, y, yt, workspace, ws_bytes,
                              TB_PATH_AUTO, stream);
}

int tb_ternary_linear_path(tb_dtype xt, tb_format f, int64_t M, int64_t N, int64_t K, int has_signs,
                           int aligned16) {
  // A stand-in argument set with the requested alignment decides the path.
  const uintptr_t base = aligned16 ? 0x1000 : 0x1004;
  LinearArgs a{reinterpret_cast<const void*>(base), xt, reinterpret_cast<const uint8_t*>(base),
               reinterpret_cast<const uint16_t*>(base), f, M, N, K,
               has_signs ? reinterpret_cast<const int8_t*>(0x2000) : nullptr,
               reinterpret_cast<void*>(0x3000), xt == TB_INT8 ? TB_INT32 : TB_FP32,
               reinterpret_cast<void*>(0x4000),
               required_ws(f, M > 0 ? M : 1, N > 0 ? N : 1, K > 0 ? K : 128), nullptr};
  if (validate_linear(a) != TB_OK) return -1;
  return auto_path(a);
}

// ---------------------------------------------------------------------------
// Fixed scratch for callers that cannot allocate (tb_ternary_linear_noalloc).
// In host code g_noalloc_scratch is only a host-side stand-in for the device
// array: the kernels get its device address from cudaGetSymbolAddress, looked
// up once per device with that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[TB_NOALLOC_SCRATCH_BYTES];
static std::mutex g_noalloc_mu;
static void* g_noalloc_ptr[64] = {};

// Scratch the decode path can write for M tokens of width K: the activation
// stages of the CUDA-core decode (every M) and, for one token with K past the
// fused-rotation limit, the prep kernel's output for the one-token kernel.
// The larger of the two, whichever kernel the shape then selects.
static int64_t noalloc_need(int64_t M, int64_t K) {
  const int64_t v = gemv_ws_bytes(M, K);
  const int64_t g1 = M == 1 ? g1_act_bytes(K) : 0;
  return v > g1 ? v : g1;
}

static tb_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return TB_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return TB_OK;
}

tb_status tb_ternary_linear_noalloc(const void* x, tb_dtype xt, const uint8_t* packed,
                                    const uint16_t* scales, int64_t M, int64_t N, int64_t K,
                                    const int8_t* signs, void* y, tb_dtype yt, void* stream) {
  // Validate as tb_ternary_linear would with an ample aligned workspace, then
  // check the fixed scratch's limit and the GEMV path's own rules.
  LinearArgs a{x, xt, packed, scales, TB_FMT_2BIT, M, N, K, signs, y, yt,
               reinterpret_cast<void*>(static_cast<uintptr_t>(256)),
               required_ws(TB_FMT_2BIT, M > 0 ? M : 1, N > 0 ? N : 1, K > 0 ? K : 128), as_stream(stream)};
  tb_status st = validate_linear(a);
  if (st != TB_OK) return st;
  if (xt == TB_INT8) return TB_ERR_DTYPE;
  if (M > kGemvMaxM || K % 1024 != 0) return TB_ERR_SHAPE;
  if (noalloc_need(M, K) > static_cast<int64_t>(TB_NOALLOC_SCRATCH_BYTES)) return TB_ERR_WORKSPACE;
  if (!aligned(packed, 16) || !aligned(scales, 16) || !aligned(x, 16) || !aligned(y, 16) ||
      (signs != nullptr && !aligned(signs, 16)))
    return TB_ERR_ALIGN;
  const DevInfo* d = nullptr;
  st = current_device(&d);
  if (st != TB_OK) return st;
  void* scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != TB_OK) return st;
  a.ws = scratch;
  a.ws_bytes = TB_NOALLOC_SCRATCH_BYTES;
  if (!gemv_ok(a)) return TB_ERR_SHAPE;
  return run_gemv(a, d);
}

tb_status tb_test_stall_copies(uint32_t stall, uint64_t wait_limit_ns) {
  const uint32_t v = stall ? 1u : 0u;
  const unsigned long long lim = wait_limit_ns != 0 ? wait_limit_ns : tb::kWaitLimitNs;
  if (cudaMemcpyToSymbol(tb::g_test_stall, &v, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(tb::g_wait_limit_ns, &lim, sizeof(lim)) != cudaSuccess) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  return TB_OK;
}

tb_status tb_get_device_fault(uint32_t* code, int clear) {
  if (code == nullptr) return TB_ERR_NULL;
  if (cudaMemcpyFromSymbol(code, tb::g_fault, sizeof(uint32_t)) != cudaSuccess) {
    cudaGetLastError();
    return TB_ERR_CUDA;
  }
  if (clear) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(tb::g_fault, &zero, sizeof(uint32_t)) != cudaSuccess) {
      cudaGetLastError();
      return TB_ERR_CUDA;
    }
  }
  return TB_OK;
}

}  // extern "C"
