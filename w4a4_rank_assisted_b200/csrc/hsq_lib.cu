// hsq_lib.cu -- the C ABI of libhsq (declared in include/hsq.h): argument
// validation, launch planning, tensor-map construction and kernel launches.
//
// Everything numeric happens in the kernels of hsq_quant.cuh, hsq_gemm.cuh,
// hsq_gemv.cuh and hsq_lowrank.cuh (and, for the pack-time truncated-SVD
// helper only, plain fp32/fp64 cuBLAS GEMMs); this file checks arguments
// (synchronously, before any launch), plans and launches.  It allocates no
// device memory, except the helper's one cuBLAS handle per device.
#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include "../../include/hsq.h"
#include "hsq_device.cuh"
#include "hsq_fp4.cuh"
#include "hsq_gemm.cuh"
#include "hsq_gemv.cuh"
#include "hsq_lowrank.cuh"
#include "hsq_quant.cuh"

namespace {

constexpr int kMaxDim = 1 << 20;
constexpr int kMaxRank = 32;

// Kernel configurations (hsq_gemm.cuh), for scale groups of 64 and of 128 along K.
//   GemmCfg<BN, DH, STAGES, SWAP, GPS, NI8, NTM, UNPACK/helper warps, SSLOTS, E4M3, PIPE, PRE, CHB, BPG, PAIR>
// M > 64: 128 tokens x 256 outputs per tile, both operands pre-expanded to E4M3
// tiles, 8 drain warps in two column slices, 2 warps building the low-rank step.
// HSQ_PAIR=1 builds CTA-pair tiles instead (clusters of 2 sharing 256 tokens x
// 256 outputs, cta_group::2 MMAs, each CTA loading half of the outputs' operand
// rows): a third less operand traffic per CTA, but measured slower on B200, since
// every 64-group ends its accumulator chain and the pair adds a cross-CTA
// hand-off to each of those chain ends.
#ifndef HSQ_PAIR
#define HSQ_PAIR 0
#endif
// Drain layout of the large tiles: HSQ_LARGE_DH column slices of 4 warps each,
// HSQ_LARGE_CHB 8-column blocks per Tensor Memory load, HSQ_LARGE_PIPE (-1: by
// register budget) for the next load in flight during the current chunk's math.
#ifndef HSQ_LARGE_DH
#define HSQ_LARGE_DH 2
#endif
#ifndef HSQ_LARGE_STAGES
#define HSQ_LARGE_STAGES 6
#endif
#ifndef HSQ_LARGE128_STAGES
#define HSQ_LARGE128_STAGES 3
#endif
#ifndef HSQ_LARGE_CHB
#define HSQ_LARGE_CHB 2
#endif
#ifndef HSQ_LARGE_PIPE
#define HSQ_LARGE_PIPE -1
#endif
#ifndef HSQ_LARGE_BN
#define HSQ_LARGE_BN 256
#endif
#ifndef HSQ_LARGE_NTM
#define HSQ_LARGE_NTM 2
#endif
using CfgLarge64 = hsq::GemmCfg<HSQ_LARGE_BN, HSQ_LARGE_DH, HSQ_PAIR ? 8 : HSQ_LARGE_STAGES, false, 1, 3,
                                HSQ_LARGE_NTM, 2, HSQ_PAIR ? 12 : HSQ_LARGE_STAGES + 4, true, HSQ_LARGE_PIPE, true,
                                HSQ_LARGE_CHB, 1, HSQ_PAIR != 0>;
using CfgLarge128 = hsq::GemmCfg<HSQ_LARGE_BN, HSQ_LARGE_DH, HSQ_PAIR ? 4 : HSQ_LARGE128_STAGES, false, 1, 3,
                                 HSQ_LARGE_NTM, 2, HSQ_PAIR ? 8 : HSQ_LARGE128_STAGES + 4, true,
                                 HSQ_LARGE_PIPE, true, HSQ_LARGE_CHB, 2, HSQ_PAIR != 0>;
// 64 < M <= 256, groups of 64 ("mid"): tokens x outputs tiles of 128 x 256 that
// unpack both packed operands in shared memory (6 warps) instead of expanding
// them in HBM first -- with one or two token tiles each weight tile is read about
// once, so the per-call expansion of the whole weight matrix would only add traffic.
#ifndef HSQ_MID_MAX_M
#define HSQ_MID_MAX_M 256
#endif
using CfgMid64 = hsq::GemmCfg<256, 2, 6, false, 1, 3, 2, 6, 10, true, -1, false, 2, 1>;
// The same tiles for ranks above one low-rank step (LR_MAX_RANK): the steps after
// a tile's first are built on the MMA issuer's path, by the many-rank builder.
using CfgLarge64R = hsq::GemmCfg<HSQ_LARGE_BN, HSQ_LARGE_DH, HSQ_PAIR ? 8 : HSQ_LARGE_STAGES, false, 1, 3,
                                 HSQ_LARGE_NTM, 2, HSQ_PAIR ? 12 : HSQ_LARGE_STAGES + 4, true, HSQ_LARGE_PIPE, true,
                                 HSQ_LARGE_CHB, 1, HSQ_PAIR != 0, false, true>;
using CfgLarge128R = hsq::GemmCfg<HSQ_LARGE_BN, HSQ_LARGE_DH, HSQ_PAIR ? 4 : HSQ_LARGE128_STAGES, false, 1, 3,
                                  HSQ_LARGE_NTM, 2, HSQ_PAIR ? 8 : HSQ_LARGE128_STAGES + 4, true,
                                  HSQ_LARGE_PIPE, true, HSQ_LARGE_CHB, 2, HSQ_PAIR != 0, false, true>;
using CfgMid64R = hsq::GemmCfg<256, 2, 6, false, 1, 3, 2, 6, 10, true, -1, false, 2, 1, false, false, true>;
// Which kernels a rank takes.  The many-rank builder pays for itself once the
// second low-rank step holds two ranks or more.  Measured on FLUX MLP up
// (M = 4608, K = 3072, N = 12288): 463 vs 468 us at r = 16 (one rank in the
// second step: the previous builder is faster), 779 vs 528 us at r = 32.
static bool many_rank_kernel(int r) { return r > CfgLarge64::LR_MAX_RANK + 1; }
static_assert(CfgLarge64R::SMEM_BYTES == CfgLarge64::SMEM_BYTES && CfgLarge128R::SMEM_BYTES == CfgLarge128::SMEM_BYTES &&
                  CfgMid64R::SMEM_BYTES == CfgMid64::SMEM_BYTES && CfgLarge64R::THREADS == CfgLarge64::THREADS,
              "many-rank kernels: the same tiles");
// M <= 64: roles swapped, 128 weight rows x 16/32/64 tokens; packed codes
// unpacked in shared memory (the drain is light, so more warps unpack); four
// 64-blocks per stage either way
#ifndef HSQ_DEC16_STAGES
#define HSQ_DEC16_STAGES 6
#endif
#ifndef HSQ_DEC16_GPS
#define HSQ_DEC16_GPS 4
#endif
#ifndef HSQ_DEC16_UNPACK
#define HSQ_DEC16_UNPACK 6
#endif
#ifndef HSQ_DEC16_NI8
#define HSQ_DEC16_NI8 2
#endif
#ifndef HSQ_DEC16_NTM
#define HSQ_DEC16_NTM 4
#endif
using CfgDec16_64 = hsq::GemmCfg<16, 1, HSQ_DEC16_STAGES, true, HSQ_DEC16_GPS, HSQ_DEC16_NI8, HSQ_DEC16_NTM,
                                 HSQ_DEC16_UNPACK>;
using CfgDec32_64 = hsq::GemmCfg<32, 1, 5, true, 4, 2, 2, 10>;
using CfgDec64_64 = hsq::GemmCfg<64, 1, 8, true, 2, 2, 2, 6>;  // 64 accumulators: keep registers
using CfgDec16_128 = hsq::GemmCfg<16, 1, 6, true, 2, 2, 4, 10, 10, false, -1, false, 2, 2>;
using CfgDec32_128 = hsq::GemmCfg<32, 1, 5, true, 2, 2, 2, 10, 9, false, -1, false, 2, 2>;
using CfgDec64_128 = hsq::GemmCfg<64, 1, 8, true, 1, 2, 2, 6, 12, false, -1, false, 2, 2>;
// ... and the single-launch forward for up to 16 tokens: the 16-token decode
// tiles with the activation step inside (cooperative launch)
using CfgDec16F_64 = hsq::GemmCfg<16, 1, 6, true, 4, 2, 4, 10, 10, false, -1, false, 2, 1, false, true>;
using CfgDec16F_128 = hsq::GemmCfg<16, 1, 6, true, 2, 2, 4, 10, 10, false, -1, false, 2, 2, false, true>;

#ifndef HSQ_LR_MMA
#define HSQ_LR_MMA 1  // U L2 + b as a tensor-core step where the kernel supports it
#endif

// Scratch of hsq_linear_forward_noalloc (split-K counters, then partial tiles),
// for callers that cannot provide a workspace.  In host code this name only
// stands in for the device array: its device address comes from
// cudaGetSymbolAddress, looked up once per device.
constexpr size_t kNoallocScratchBytes = HSQ_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
struct NoallocSlot {
  std::once_flag once;
  void* ptr = nullptr;
  cudaError_t err = cudaSuccess;
};
NoallocSlot g_noalloc_slots[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (set-up on first use).
hsq_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSQ_ERR_UNSUPPORTED;
  NoallocSlot& slot = g_noalloc_slots[dev];
  std::call_once(slot.once, [&slot] { slot.err = cudaGetSymbolAddress(&slot.ptr, g_noalloc_scratch); });
  if (slot.err != cudaSuccess || !slot.ptr) return HSQ_ERR_CUDA;
  *out = slot.ptr;
  return HSQ_OK;
}

// Scratch of the single-launch forward's decode-tile form: the grid barrier's
// counters (the first 256 bytes, zero between launches; nothing else uses them),
// then per call the stream-K counters and partial tiles, the activation step's
// codes, scales and U partials, and one copy of U per CTA.
#ifndef HSQ_FUSED_SCRATCH_BYTES
#define HSQ_FUSED_SCRATCH_BYTES (8u << 20)
#endif
constexpr size_t kFusedScratchBytes = HSQ_FUSED_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_fused_scratch[kFusedScratchBytes];
NoallocSlot g_fused_slots[kMaxDevices];

hsq_status fused_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return HSQ_ERR_UNSUPPORTED;
  NoallocSlot& slot = g_fused_slots[dev];
  std::call_once(slot.once, [&slot] { slot.err = cudaGetSymbolAddress(&slot.ptr, g_fused_scratch); });
  if (slot.err != cudaSuccess || !slot.ptr) return HSQ_ERR_CUDA;
  *out = slot.ptr;
  return HSQ_OK;
}

#ifndef HSQ_PDL
#define HSQ_PDL 1  // launch with programmatic stream serialization (see grid_dep_wait)
#endif
#ifndef HSQ_FUSED_PDL
#define HSQ_FUSED_PDL 1  // ... the cooperative decode tiles too, where the driver accepts it
#endif

// Launch `kernel` so that it may start while the preceding kernel in the stream
// is still running; the kernel itself waits (grid_dep_wait) before touching
// memory that kernel may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(bool allow, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = (HSQ_PDL && allow) ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The row-owning activation kernel for many rows (0: always the sub-block kernel).
#ifndef HSQ_ACT_ROWS
#define HSQ_ACT_ROWS 1
#endif
// ... from this many rows per SM on
#ifndef HSQ_ACT_ROWS16_MIN
#define HSQ_ACT_ROWS16_MIN 24
#endif
// ... with this many rows per warp (8 warps per block)
#ifndef HSQ_ACT_ROWS_SUB
#define HSQ_ACT_ROWS_SUB 2
#endif

thread_local int t_debug_flags = 0;
thread_local int t_debug_limit_ms = 0;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int groups_of(int K, int group) { return (K + group - 1) / group; }
int scales_ld(int rows) { return (rows + 3) & ~3; }

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* e = std::getenv("HSQ_WAIT_LIMIT_MS");
    long ms = e ? std::strtol(e, nullptr, 10) : 4000;
    if (ms <= 0) ms = 4000;
    return static_cast<uint64_t>(ms) * 1000000ull;
  }();
  return v;
}

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  static int cache[64] = {0};
  if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cache[dev] = n;
  return n;
}

// ------------------------------------------------------------------ planning
enum Kind { kLarge = 0, kDec16, kDec32, kDec64, kGemv, kMid };

// M <= 8: the weight stream on the CUDA cores (hsq_gemv.cuh) when its shared
// memory (the block's widened activation codes and weight scales, and a ring of
// at least two stages of weight rows) fits; otherwise the decode tiles.
constexpr int kGemvMaxM = 8;
constexpr size_t kGemvSmemMax = 227 * 1024;
int gemv_mt(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : 8; }
// Rows per block of the weight stream: N spread evenly over the SMs, rounded up
// to a multiple of 4 (so that each group's run of block scales is 16-byte aligned).
int gemv_rows_per_block(int N, int nsm) { return ((N + nsm - 1) / nsm + 3) / 4 * 4; }
hsq::GemvLayout gemv_plan_layout(int M, int N, int Kp, int G, int nsm) {
  return hsq::gemv_layout(gemv_mt(M), Kp, G, gemv_rows_per_block(N, nsm), kGemvSmemMax);
}

struct Plan {
  Kind kind;
  int group;      // 64 or 128
  int BN;
  bool swap;
  int drain_warps;
  int gps_stage;  // scale groups per pipeline stage of the chosen kernel
  int bps_stage;  // 64-blocks per pipeline stage (the TMA box width / 32 bytes)
  int tiles_r, tiles_c, stages_per_tile, stream_len, grid;
  int pm = 1;     // CTAs per tile (2: CTA pairs)
  size_t counters_bytes, partial_bytes;
  // pre-expanded operands (large tiles): 8-row groups and bytes
  int rg_r, rg_c;
  size_t pre_x_bytes, pre_w_bytes;
  size_t split_bytes() const { return stream_len > 0 ? counters_bytes + partial_bytes : 0; }
  // workspace: [stream-K counters][stream-K partials][expanded row operand][expanded col operand]
  size_t pre_x_offset() const { return (split_bytes() + 255) / 256 * 256; }
  size_t pre_w_offset() const { return pre_x_offset() + pre_x_bytes; }
  size_t ws_bytes() const { return pre_x_bytes + pre_w_bytes > 0 ? pre_w_offset() + pre_w_bytes : split_bytes(); }
};

template <class C>
void plan_from(Plan& p) {
  p.BN = C::BN;
  p.gps_stage = C::GPS;
  p.bps_stage = C::BPS;
  p.drain_warps = C::NUM_DRAIN_WARPS;
}

// Workers of the large-tile kernel: CTAs, or CTA pairs that the device can hold
// at once (asked of the occupancy calculator once per device; half the SMs when
// no device answers, as on a machine without a GPU).
int large_workers(int nsm) {
  if (!CfgLarge64::PAIR) return nsm;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return nsm / 2;
  }
  static int cache[64] = {0};
  if (cache[dev]) return cache[dev];
  int n = nsm / 2;
  auto* kern = hsq::w4a4_gemm_kernel<CfgLarge64>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, CfgLarge64::SMEM_BYTES) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * n);
    cfg.blockDim = dim3(CfgLarge64::THREADS);
    cfg.dynamicSmemBytes = CfgLarge64::SMEM_BYTES;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, kern, &cfg) == cudaSuccess && c > 0) n = std::min(n, c);
  }
  cudaGetLastError();
  cache[dev] = n;
  return n;
}

void finish_plan(Plan& p, int G, int group, int nsm);

Plan make_plan(int M, int N, int K, int group, int nsm) {
  Plan p{};
  p.group = group;
  const bool g128 = group == 128;
  const int G = groups_of(K, group);
  if (M <= kGemvMaxM && gemv_plan_layout(M, N, G * group, G, nsm).stages > 0) {
    // one block per SM at most, a contiguous run of weight rows per block; no workspace
    p.kind = kGemv;
    p.swap = true;
    p.tiles_r = gemv_rows_per_block(N, nsm);  // rows per block
    p.grid = (N + p.tiles_r - 1) / p.tiles_r;
    p.tiles_c = 1;
    p.stream_len = 0;
    return p;
  }
  if (M <= 64) {
    p.swap = true;
    p.kind = M <= 16 ? kDec16 : M <= 32 ? kDec32 : kDec64;
    if (p.kind == kDec16) g128 ? plan_from<CfgDec16_128>(p) : plan_from<CfgDec16_64>(p);
    if (p.kind == kDec32) g128 ? plan_from<CfgDec32_128>(p) : plan_from<CfgDec32_64>(p);
    if (p.kind == kDec64) g128 ? plan_from<CfgDec64_128>(p) : plan_from<CfgDec64_64>(p);
    p.tiles_r = (N + 127) / 128;
    p.tiles_c = (M + p.BN - 1) / p.BN;
  } else if (M <= HSQ_MID_MAX_M && !g128) {
    p.swap = false;
    p.kind = kMid;
    plan_from<CfgMid64>(p);
    p.tiles_r = (M + 127) / 128;
    p.tiles_c = (N + p.BN - 1) / p.BN;
  } else {
    p.swap = false;
    p.kind = kLarge;
    g128 ? plan_from<CfgLarge128>(p) : plan_from<CfgLarge64>(p);
    p.pm = CfgLarge64::PM;
    p.tiles_r = (M + CfgLarge64::TILE_M - 1) / CfgLarge64::TILE_M;
    p.tiles_c = (N + p.BN - 1) / p.BN;
  }
  finish_plan(p, G, group, nsm);
  return p;
}

// Work decomposition and workspace sizes of a plan whose kernel and tiles are set.
void finish_plan(Plan& p, int G, int group, int nsm) {
  const long tiles = static_cast<long>(p.tiles_r) * p.tiles_c;
  p.stages_per_tile = (G + p.gps_stage - 1) / p.gps_stage;
  // Whole tiles per worker (a CTA, or a CTA pair) when they fill the device in
  // nearly full waves; otherwise stream-K: equal runs of stages per worker
  // across tile boundaries.
  const long nw = p.kind == kLarge ? large_workers(nsm) : nsm;
  const long waves = (tiles + nw - 1) / nw;
  const double fill = static_cast<double>(tiles) / static_cast<double>(waves * nw);
  const long total = tiles * p.stages_per_tile;
  if ((tiles >= nw && fill >= 0.9) || total <= nw || total >= (1l << 30)) {
    p.stream_len = 0;
    p.grid = p.pm * static_cast<int>(std::min<long>(tiles, nw));
  } else {
    p.stream_len = static_cast<int>((total + nw - 1) / nw);
    p.grid = p.pm * static_cast<int>((total + p.stream_len - 1) / p.stream_len);
  }
  p.counters_bytes = ((static_cast<size_t>(tiles) * p.pm * p.drain_warps * 4 + 255) / 256) * 256;
  p.partial_bytes = static_cast<size_t>(p.grid) * 2 * p.BN * 128 * 4;
  if (p.kind == kLarge) {  // both large configurations pre-expand their operands
    const size_t blocks = static_cast<size_t>(G) * (group / 64);  // 64-wide K blocks
    p.rg_r = p.tiles_r * (CfgLarge64::TILE_M / 8);
    p.rg_c = p.tiles_c * (p.BN / 8);
    p.pre_x_bytes = blocks * p.rg_r * CfgLarge64::E8_SBO;
    p.pre_w_bytes = blocks * p.rg_c * CfgLarge64::E8_SBO;
  }
}

// The 16-token decode tiles for any M <= 16 (the single-launch forward).
Plan make_dec16_plan(int M, int N, int K, int group, int nsm) {
  Plan p{};
  p.group = group;
  p.swap = true;
  p.kind = kDec16;
  group == 128 ? plan_from<CfgDec16F_128>(p) : plan_from<CfgDec16F_64>(p);
  p.tiles_r = (N + 127) / 128;
  p.tiles_c = (M + p.BN - 1) / p.BN;
  finish_plan(p, groups_of(K, group), group, nsm);
  return p;
}
static_assert(CfgLarge64::PRE && CfgLarge128::PRE && CfgLarge64::BN == CfgLarge128::BN &&
                  CfgLarge64::PAIR == CfgLarge128::PAIR,
              "large configurations");

// ------------------------------------------------------------------ tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(f);
  }();
  return fn;
}

// 2-D map over packed codes [rows][Kp/2] bytes, box = `groups` 64-groups (32 bytes each) x box_rows.
bool make_codes_map(CUtensorMap* map, const uint8_t* codes, int rows, int Kp, int box_rows, int groups) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Kp / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Kp / 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(32 * groups), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over NVFP4 codes [rows][Kq/2] bytes for the block-scaled kernel: box =
// 128 bytes (a stage's K = 256) x box_rows rows (the tile's), 128-byte swizzle
// (the layout its MMA descriptors read).
bool make_fp4_codes_map(CUtensorMap* map, const uint8_t* codes, int rows, int Kq, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(Kq / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(Kq / 2)};
  const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over a group-major scale matrix [G][ld] fp32 for the weight stream: box
// = box_rows rows x G groups (one block's scales in one copy).
bool make_scales_map(CUtensorMap* map, const float* scales, int ld, int G, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(ld), static_cast<cuuint64_t>(G)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(G)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(scales), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pre-expanded E4M3 tiles (large tiles with CTA pairs) viewed as rows of 256
// bytes; one box of 32 rows is one 8 KB block of 128 rows x 64 codes.
bool make_e8_map(CUtensorMap* map, const uint8_t* base, size_t bytes) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || bytes % 256 != 0) return false;
  const cuuint64_t dims[2] = {256u, static_cast<cuuint64_t>(bytes / 256)};
  const cuuint64_t strides[1] = {256u};
  const cuuint32_t box[2] = {256u, 32u};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Y [M][N] (bf16 or fp32) for the epilogue's TMA stores: boxes of 32 rows x
// 128 bytes, 128-byte swizzle.
bool make_y_map(CUtensorMap* map, void* Y, int M, int N, bool f32) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const int es = f32 ? 4 : 2;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * es};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / es), 32u};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <class Cfg>
hsq_status launch_gemm(const Plan& p, const CUtensorMap& tr, const CUtensorMap& tc, const CUtensorMap& ty,
                       const hsq::GemmArgs& a, cudaStream_t st) {
  static std::mutex mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      if (cudaFuncSetAttribute(hsq::w4a4_gemm_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::SMEM_BYTES) != cudaSuccess)
        return HSQ_ERR_CUDA;
      if (Cfg::REALLOC) {
        // the warpgroup register split assumes the block launches with exactly
        // LAUNCH_REGS registers per thread; refuse to launch otherwise
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, hsq::w4a4_gemm_kernel<Cfg>) != cudaSuccess) return HSQ_ERR_CUDA;
        if (fa.numRegs != Cfg::LAUNCH_REGS) return HSQ_ERR_UNSUPPORTED;
      }
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  cudaError_t e;
  if constexpr (Cfg::PAIR) {
    // CTA pairs: clusters of two, no early start
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (p.grid % 2 != 0) return HSQ_ERR_INVALID_ARG;
    e = cudaLaunchKernelEx(&cfg, hsq::w4a4_gemm_kernel<Cfg>, tr, tc, ty, a);
  } else {
    // decode tiles start early (their weight prefetch overlaps the activation
    // step); the GPU-filling large tiles measured faster without an early start
    e = launch_pdl(p.swap, hsq::w4a4_gemm_kernel<Cfg>, dim3(p.grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, st, tr,
                   tc, ty, a);
  }
  if (e != cudaSuccess) return HSQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

// The single-launch forward on 16-token decode tiles: the kernel runs the
// activation step itself, spread over its CTAs, and then waits at a grid
// barrier, so every CTA must be resident at once -- a cooperative launch, after
// the occupancy check.
template <class Cfg>
hsq_status launch_gemm_fused(const Plan& p, const CUtensorMap& tr, const CUtensorMap& tc, const hsq::GemmArgs& a,
                             cudaStream_t st) {
  static_assert(Cfg::FUSED && !Cfg::REALLOC, "fused decode tiles");
  static std::mutex mu;
  static int max_blocks[64] = {0};  // resident CTAs per SM, per device (0: not asked yet)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return HSQ_ERR_UNSUPPORTED;
  int nb = 0;
  {
    std::lock_guard<std::mutex> lk(mu);
    if (max_blocks[dev] == 0) {
      if (cudaFuncSetAttribute(hsq::w4a4_gemm_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::SMEM_BYTES) != cudaSuccess)
        return HSQ_ERR_CUDA;
      int b = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, hsq::w4a4_gemm_kernel<Cfg>, Cfg::THREADS,
                                                        Cfg::SMEM_BYTES) != cudaSuccess)
        return HSQ_ERR_CUDA;
      max_blocks[dev] = b > 0 ? b : -1;
    }
    nb = max_blocks[dev];
  }
  if (nb <= 0 || p.grid > nb * device_sm_count()) return HSQ_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(p.grid);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  // with an early start where the driver takes one (the kernel requests only
  // weight tiles before its grid_dep_wait), else without
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  static int pdl_ok[64] = {0};  // 0: untried, 1: accepted, -1: refused
  if (HSQ_PDL && HSQ_FUSED_PDL && pdl_ok[dev] >= 0) {
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, hsq::w4a4_gemm_kernel<Cfg>, tr, tc, tr, a);
    if (e == cudaSuccess) {
      pdl_ok[dev] = 1;
      return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
    }
    if (pdl_ok[dev] == 1) return HSQ_ERR_CUDA;
    (void)cudaGetLastError();  // refused at the first try: launch without the early start from now on
    pdl_ok[dev] = -1;
  }
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, hsq::w4a4_gemm_kernel<Cfg>, tr, tc, tr, a) != cudaSuccess) return HSQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

// `a` has the shape, rows_per_block and pointers set; the ring layout and the
// wait limit are filled in here.
template <int MT, int LPG, int RF = -1>
hsq_status launch_gemv(const Plan& p, hsq::GemvArgs a, cudaStream_t st) {
  static std::mutex mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      if (cudaFuncSetAttribute(hsq::w4a4_gemv_kernel<MT, LPG, RF>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kGemvSmemMax)) != cudaSuccess)
        return HSQ_ERR_CUDA;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  const hsq::GemvLayout L = hsq::gemv_layout(MT, a.Kp, a.G, a.rows_per_block, kGemvSmemMax);
  if (L.stages < 1 || L.bytes > kGemvSmemMax) return HSQ_ERR_UNSUPPORTED;
  a.rs = L.rs; a.stages = L.stages;
  a.off_sws = L.off_sws; a.off_x = L.off_x; a.off_sxs = L.off_sxs; a.off_us = L.off_us; a.off_bars = L.off_bars;
  a.limit_ns = wait_limit_ns();
  CUtensorMap tm_sw;
  if (!make_scales_map(&tm_sw, a.w_scales, a.ldw, a.G, a.rows_per_block)) return HSQ_ERR_CUDA;
  // starts early: its weight copies do not depend on the preceding kernel, and
  // it waits for the activation step before reading its codes
  if (launch_pdl(true, hsq::w4a4_gemv_kernel<MT, LPG, RF>, dim3(p.grid), dim3(hsq::kGemvThreads), L.bytes, st,
                 tm_sw, a) != cudaSuccess)
    return HSQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

// ------------------------------------------------------------------ truncated-SVD helper
// Workspace carve-up of hsq_lowrank_init (each part 256-byte aligned).
struct LrLayout {
  int p;
  size_t A, Q, Y, Z, Z64, Q64, Y64, G, Rinv, V, L1c, C, end;
};

LrLayout lr_layout(int N, int K, int r) {
  LrLayout L{};
  L.p = std::min(r + hsq::kLrOversample, std::min(N, K));
  const size_t p = static_cast<size_t>(L.p);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = (off + bytes + 255) / 256 * 256;
    return at;
  };
  L.A = take(4ull * N * K);
  L.Q = take(4 * K * p);
  L.Y = take(4 * N * p);
  L.Z = take(4 * K * p);
  L.Z64 = take(8 * K * p);
  L.Q64 = take(8 * K * p);
  L.Y64 = take(8 * N * p);
  L.G = take(8 * p * p);
  L.Rinv = take(8 * p * p);
  L.V = take(4 * p * p);
  L.L1c = take(4ull * K * r);
  L.C = take(4ull * N * r);
  L.end = off;
  return L;
}

// One cuBLAS handle per device, created on first use (creating one costs
// milliseconds); calls on it are serialised.
struct BlasSlot {
  std::mutex mu;
  cublasHandle_t h = nullptr;
};
BlasSlot g_blas[kMaxDevices];

}  // namespace

// The many-row activation kernel: its X ring is dynamic shared memory (set once
// per device and instantiation).
template <int R, int GL, int NW, int SUB, bool FP4 = false>
cudaError_t launch_act_rows(const __nv_bfloat16* X, const float* s, const __nv_bfloat16* L1, int M, int K, int Kp,
                            int ld, uint8_t* codes, float* scales, float* U, cudaStream_t st, float* gs = nullptr,
                            uint8_t* xe = nullptr, int xe_rg = 0, unsigned* zc = nullptr, int zc_words = 0) {
  using C = hsq::ActRowsCfg<NW, SUB>;
  constexpr int kSmem = C::STAGES * C::STAGE_BYTES;
  static std::mutex mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      const cudaError_t e = cudaFuncSetAttribute(hsq::quantize_act_rows_kernel<R, GL, NW, SUB, FP4>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
      if (e != cudaSuccess) return e;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  return launch_pdl(!FP4, hsq::quantize_act_rows_kernel<R, GL, NW, SUB, FP4>, dim3((M + C::RB - 1) / C::RB),
                    dim3(NW * 32), static_cast<size_t>(kSmem), st, X, s, L1, M, K, Kp, ld, codes, scales, U,
                    wait_limit_ns(), gs, xe, xe_rg, zc, zc_words);
}

// hsq_linear_forward_fused for the shapes the weight stream's fused form does
// not take (5..16 tokens, or ranks other than 0, 1, 2, 4): 16-token decode
// tiles with the activation step inside, scratch from g_fused_scratch.
// Scratch layout of the decode-tile form (byte offsets into g_fused_scratch).
struct FusedLayout {
  Plan p;
  size_t o_cnt, o_part, o_codes, o_sc, o_up, o_u, total;
};
FusedLayout fused_dec16_layout(int M, int N, int K, int r, int group, int nsm) {
  FusedLayout L{};
  const int G = groups_of(K, group), Kp = G * group;
  L.p = make_dec16_plan(M, N, K, group, nsm);
  const int ldx = scales_ld(M), nchk = (Kp + 255) / 256, rr = std::max(r, 1);
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t off = 256;  // [0, 256): the grid barrier's counters
  L.o_cnt = off;
  off = up(off + L.p.counters_bytes);
  L.o_part = off;
  off = up(off + L.p.partial_bytes);
  L.o_codes = off;
  off = up(off + static_cast<size_t>(M) * (Kp / 2));
  L.o_sc = off;
  off = up(off + static_cast<size_t>(G) * ldx * 4);
  L.o_up = off;
  off = up(off + static_cast<size_t>(M) * nchk * rr * 4);
  L.o_u = off;
  off = up(off + static_cast<size_t>(L.p.grid) * M * rr * 4);
  L.total = off;
  return L;
}

// Which form hsq_linear_forward_fused takes (0: none), from the shape alone.
int fused_form(int M, int N, int K, int r, int group, int nsm) {
  if (group != 64 && group != 128) return 0;
  if (M < 1 || N < 1 || K < 1 || M > kMaxDim || N > kMaxDim || K > kMaxDim || r < 0 || r > kMaxRank) return 0;
  if (K % 8 != 0 || N % 8 != 0) return 0;
  const int G = groups_of(K, group), Kp = G * group;
  if (M <= 4 && (r == 0 || r == 1 || r == 2 || r == 4) && gemv_plan_layout(M, N, Kp, G, nsm).stages >= 1) return 1;
  if (M <= 16 && fused_dec16_layout(M, N, K, r, group, nsm).total <= kFusedScratchBytes) return 2;
  return 0;
}

hsq_status forward_fused_dec16(const void* X_bf16, const float* s, const void* L1_bf16, const uint8_t* w_codes,
                               const float* w_scales, const void* L2_bf16, const void* bias_bf16, int M, int N, int K,
                               int r, int group, void* Y, hsq_out_dtype out, cudaStream_t stream) {
  const int G = groups_of(K, group), Kp = G * group, nsm = device_sm_count();
  const FusedLayout FL = fused_dec16_layout(M, N, K, r, group, nsm);
  const Plan& p = FL.p;
  const int ldx = scales_ld(M), ldw = scales_ld(N);
  const size_t o_cnt = FL.o_cnt, o_part = FL.o_part, o_codes = FL.o_codes, o_sc = FL.o_sc, o_up = FL.o_up,
               o_u = FL.o_u;
  if (FL.total > kFusedScratchBytes) return HSQ_ERR_UNSUPPORTED;
  void* scr = nullptr;
  hsq_status st = fused_scratch(&scr);
  if (st != HSQ_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(scr);

  hsq::GemmArgs a{};
  CUtensorMap tm_row, tm_col;
  a.scales_r = w_scales; a.ld_r = ldw; a.rows_r = N;
  a.scales_c = reinterpret_cast<float*>(base + o_sc); a.ld_c = ldx; a.rows_c = M;
  if (!make_codes_map(&tm_row, w_codes, N, Kp, 128, p.bps_stage) ||
      !make_codes_map(&tm_col, base + o_codes, M, Kp, p.BN, p.bps_stage))
    return HSQ_ERR_CUDA;
  a.U = nullptr;  // the kernel's own
  a.L2 = static_cast<const __nv_bfloat16*>(L2_bf16);
  a.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
  a.Y = Y;
  a.out_f32 = out == HSQ_OUT_F32 ? 1 : 0;
  a.M = M; a.N = N; a.G = G; a.r = r;
  a.tiles_r = p.tiles_r; a.tiles_c = p.tiles_c;
  a.stages_per_tile = p.stages_per_tile; a.stream_len = p.stream_len;
  if (p.stream_len > 0) {
    a.ws_counters = reinterpret_cast<unsigned*>(base + o_cnt);
    a.ws_partials = reinterpret_cast<float*>(base + o_part);
    a.fx_zero_words = static_cast<int>(p.counters_bytes / 4);
  }
  a.fx_X = static_cast<const __nv_bfloat16*>(X_bf16);
  a.fx_s = s;
  a.fx_L1 = static_cast<const __nv_bfloat16*>(L1_bf16);
  a.fx_K = K; a.fx_Kp = Kp; a.fx_group = group;
  a.fx_codes = base + o_codes;
  a.fx_scales = reinterpret_cast<float*>(base + o_sc);
  a.fx_upart = reinterpret_cast<float*>(base + o_up);
  a.fx_U = reinterpret_cast<float*>(base + o_u);
  a.fx_bar = reinterpret_cast<unsigned*>(base);
  a.lr_mma = 0;
  a.limit_ns = wait_limit_ns();
  if (t_debug_flags) {
    a.debug_flags = t_debug_flags;
    a.limit_ns = static_cast<uint64_t>(t_debug_limit_ms > 0 ? t_debug_limit_ms : 50) * 1000000ull;
    t_debug_flags = 0;
  }
  return group == 128 ? launch_gemm_fused<CfgDec16F_128>(p, tm_row, tm_col, a, stream)
                      : launch_gemm_fused<CfgDec16F_64>(p, tm_row, tm_col, a, stream);
}

extern "C" {

size_t hsq_lowrank_workspace_bytes(int N, int K, int r) {
  if (N < 1 || K < 1 || r < 1 || r > kMaxRank || r > std::min(N, K)) return 0;
  return lr_layout(N, K, r).end;
}

hsq_status hsq_lowrank_init(const void* W_bf16, const float* s, int N, int K, int r, int iters,
                            unsigned long long seed, void* L1_bf16, void* L2_bf16, void* workspace,
                            size_t ws_bytes, cudaStream_t stream) {
  if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim) return HSQ_ERR_INVALID_ARG;
  if (r < 1 || r > kMaxRank || r > std::min(N, K)) return HSQ_ERR_UNSUPPORTED;
  if (iters < 0 || iters > 64) return HSQ_ERR_INVALID_ARG;
  if (!W_bf16 || !s || !L1_bf16 || !L2_bf16 || !workspace) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(W_bf16) || !aligned16(s) || !aligned16(L1_bf16) || !aligned16(L2_bf16) || !aligned16(workspace))
    return HSQ_ERR_ALIGNMENT;
  const LrLayout L = lr_layout(N, K, r);
  if (ws_bytes < L.end) return HSQ_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HSQ_ERR_CUDA;
  BlasSlot& slot = g_blas[dev];
  std::lock_guard<std::mutex> lk(slot.mu);
  if (!slot.h && cublasCreate(&slot.h) != CUBLAS_STATUS_SUCCESS) {
    slot.h = nullptr;
    return HSQ_ERR_CUDA;
  }
  cublasHandle_t h = slot.h;
  if (cublasSetStream(h, stream) != CUBLAS_STATUS_SUCCESS ||
      cublasSetMathMode(h, CUBLAS_DEFAULT_MATH) != CUBLAS_STATUS_SUCCESS)  // plain fp32, no TF32
    return HSQ_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* A = reinterpret_cast<float*>(ws + L.A);
  float* Q = reinterpret_cast<float*>(ws + L.Q);
  float* Y = reinterpret_cast<float*>(ws + L.Y);
  float* Z = reinterpret_cast<float*>(ws + L.Z);
  double* Z64 = reinterpret_cast<double*>(ws + L.Z64);
  double* Q64 = reinterpret_cast<double*>(ws + L.Q64);
  double* Y64 = reinterpret_cast<double*>(ws + L.Y64);
  double* G = reinterpret_cast<double*>(ws + L.G);
  double* Rinv = reinterpret_cast<double*>(ws + L.Rinv);
  float* V = reinterpret_cast<float*>(ws + L.V);
  float* L1c = reinterpret_cast<float*>(ws + L.L1c);
  float* C = reinterpret_cast<float*>(ws + L.C);
  const int p = L.p;
  const int blocks = 4 * device_sm_count();
  const float one = 1.f, zero = 0.f;
  const double done = 1.0, dzero = 0.0;
  bool ok = true;
  auto blas = [&](cublasStatus_t st) { ok = ok && st == CUBLAS_STATUS_SUCCESS; };
  // orthonormalise the K x p matrix Z (fp32) into Q (fp32): CholeskyQR twice, in fp64
  auto orth = [&]() {
    hsq::lr_to_f64_kernel<<<blocks, 256, 0, stream>>>(Z, Z64, static_cast<size_t>(K) * p);
    double* src = Z64;
    double* dst = Q64;
    for (int pass = 0; pass < 2; ++pass) {
      blas(cublasDgemm(h, CUBLAS_OP_T, CUBLAS_OP_N, p, p, K, &done, src, K, src, K, &dzero, G, p));
      hsq::lr_chol_inv_kernel<<<1, hsq::kLrMaxP, 0, stream>>>(G, p, Rinv);
      blas(cublasDgemm(h, CUBLAS_OP_N, CUBLAS_OP_N, K, p, p, &done, src, K, Rinv, p, &dzero, dst, K));
      std::swap(src, dst);
    }
    hsq::lr_to_f32_kernel<<<blocks, 256, 0, stream>>>(src, Q, static_cast<size_t>(K) * p);
  };
  hsq::lr_smooth_kernel<<<blocks, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(W_bf16), s, N, K, A);
  hsq::lr_random_kernel<<<blocks, 256, 0, stream>>>(Z, static_cast<size_t>(K) * p, seed);
  orth();
  for (int it = 0; it < iters && ok; ++it) {
    // Z = W_hat^T (W_hat Q): Y = A^T Q (N x p), Z = A Y (K x p)
    blas(cublasSgemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, p, K, &one, A, K, Q, K, &zero, Y, N));
    blas(cublasSgemm(h, CUBLAS_OP_N, CUBLAS_OP_N, K, p, N, &one, A, K, Y, N, &zero, Z, K));
    orth();
  }
  // Rayleigh-Ritz: T = (W_hat Q)^T (W_hat Q) in fp64, its eigenvectors V
  blas(cublasSgemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, p, K, &one, A, K, Q, K, &zero, Y, N));
  hsq::lr_to_f64_kernel<<<blocks, 256, 0, stream>>>(Y, Y64, static_cast<size_t>(N) * p);
  blas(cublasDgemm(h, CUBLAS_OP_T, CUBLAS_OP_N, p, p, N, &done, Y64, N, Y64, N, &dzero, G, p));
  hsq::lr_jacobi_kernel<<<1, hsq::kLrMaxP, 0, stream>>>(G, p, V);
  // L1 = Q V[:, :r] (K x r), C = W_hat L1 (N x r) = L2^T
  blas(cublasSgemm(h, CUBLAS_OP_N, CUBLAS_OP_N, K, r, p, &one, Q, K, V, p, &zero, L1c, K));
  blas(cublasSgemm(h, CUBLAS_OP_T, CUBLAS_OP_N, N, r, K, &one, A, K, L1c, K, &zero, C, N));
  hsq::lr_sign_out_kernel<<<r, 256, 0, stream>>>(L1c, C, K, N, r, static_cast<__nv_bfloat16*>(L1_bf16),
                                                   static_cast<__nv_bfloat16*>(L2_bf16));
  if (!ok) return HSQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}


int hsq_num_groups(int K, int group) {
  if (group <= 0 || K < 0) return 0;
  return (K + group - 1) / group;
}

size_t hsq_codes_bytes(int rows, int K, int group) {
  if (rows < 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(hsq_num_groups(K, group)) * group / 2;
}

int hsq_scales_ld(int rows) { return rows < 0 ? 0 : scales_ld(rows); }

size_t hsq_scales_bytes(int rows, int K, int group) {
  return static_cast<size_t>(hsq_num_groups(K, group)) * hsq_scales_ld(rows) * 4;
}

size_t hsq_workspace_bytes(int M, int N, int K, int r) {
  (void)r;
  if (M < 1 || N < 1 || K < 1) return 0;
  // enough for either supported group size
  const int nsm = device_sm_count();
  return std::max(make_plan(M, N, K, 64, nsm).ws_bytes(), make_plan(M, N, K, 128, nsm).ws_bytes());
}

const char* hsq_status_string(hsq_status s) {
  switch (s) {
    case HSQ_OK: return "HSQ_OK";
    case HSQ_ERR_INVALID_ARG: return "HSQ_ERR_INVALID_ARG";
    case HSQ_ERR_ALIGNMENT: return "HSQ_ERR_ALIGNMENT";
    case HSQ_ERR_UNSUPPORTED: return "HSQ_ERR_UNSUPPORTED";
    case HSQ_ERR_CUDA: return "HSQ_ERR_CUDA";
    case HSQ_ERR_TIMEOUT: return "HSQ_ERR_TIMEOUT";
    case HSQ_ERR_SCRATCH_LIMIT: return "HSQ_ERR_SCRATCH_LIMIT";
  }
  return "HSQ_UNKNOWN_STATUS";
}

void hsq_debug_force_timeout(int flags, int limit_ms) {
  t_debug_flags = flags;
  t_debug_limit_ms = limit_ms;
}

hsq_status hsq_get_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return HSQ_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, hsq::g_status, sizeof(v)) != cudaSuccess) return HSQ_ERR_CUDA;
  if (v) {
    const unsigned zero = 0;
    if (cudaMemcpyToSymbol(hsq::g_status, &zero, sizeof(zero)) != cudaSuccess) return HSQ_ERR_CUDA;
    return HSQ_ERR_TIMEOUT;
  }
  return HSQ_OK;
}

static hsq_status check_common(int rows, int K, int r, int group) {
  if (group != 64 && group != 128) return HSQ_ERR_UNSUPPORTED;
  if (rows < 1 || K < 1 || rows > kMaxDim || K > kMaxDim || r < 0) return HSQ_ERR_INVALID_ARG;
  if (r > kMaxRank || (K % 8) != 0) return HSQ_ERR_UNSUPPORTED;
  return HSQ_OK;
}

hsq_status hsq_pack_weights(const void* W_bf16, const float* s, const void* L1_bf16, const void* L2_bf16, int N,
                            int K, int r, int group, uint8_t* w_codes, float* w_scales, cudaStream_t stream) {
  hsq_status st = check_common(N, K, r, group);
  if (st != HSQ_OK) return st;
  if (!W_bf16 || !s || !w_codes || !w_scales) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1_bf16 != nullptr) || (r > 0) != (L2_bf16 != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(W_bf16) || !aligned16(s) || !aligned16(w_codes) || !aligned16(w_scales) ||
      (L1_bf16 && !aligned16(L1_bf16)) || (L2_bf16 && !aligned16(L2_bf16)))
    return HSQ_ERR_ALIGNMENT;
  const int G = groups_of(K, group), Kp = G * group, ld = scales_ld(N);
  const int blocks = (N + 7) / 8;
  if (group == 128)
    hsq::pack_weights_kernel<16><<<blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(W_bf16), s, static_cast<const __nv_bfloat16*>(L1_bf16),
        static_cast<const __nv_bfloat16*>(L2_bf16), N, K, r, Kp, ld, w_codes, w_scales);
  else
    hsq::pack_weights_kernel<8><<<blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(W_bf16), s, static_cast<const __nv_bfloat16*>(L1_bf16),
        static_cast<const __nv_bfloat16*>(L2_bf16), N, K, r, Kp, ld, w_codes, w_scales);
  if (cudaGetLastError() != cudaSuccess) return HSQ_ERR_CUDA;
  if (ld > N) {
    const int n = (ld - N) * G;
    hsq::zero_scale_pad_kernel<<<(n + 255) / 256, 256, 0, stream>>>(w_scales, N, ld, G);
    if (cudaGetLastError() != cudaSuccess) return HSQ_ERR_CUDA;
  }
  return HSQ_OK;
}

// hsq_quantize_act, optionally also clearing zc_words words at zc (the split-K
// counters of the GEMM that follows, for hsq_linear_forward_x).
static hsq_status quantize_act_impl(const void* X_bf16, const float* s, const void* L1_bf16, int M, int K, int r,
                                    int group, uint8_t* x_codes, float* x_scales, float* U, cudaStream_t stream,
                                    unsigned* zc, int zc_words);

hsq_status hsq_quantize_act(const void* X_bf16, const float* s, const void* L1_bf16, int M, int K, int r,
                            int group, uint8_t* x_codes, float* x_scales, float* U, cudaStream_t stream) {
  return quantize_act_impl(X_bf16, s, L1_bf16, M, K, r, group, x_codes, x_scales, U, stream, nullptr, 0);
}

static hsq_status quantize_act_impl(const void* X_bf16, const float* s, const void* L1_bf16, int M, int K, int r,
                                    int group, uint8_t* x_codes, float* x_scales, float* U, cudaStream_t stream,
                                    unsigned* zc, int zc_words) {
  hsq_status st = check_common(M, K, r, group);
  if (st != HSQ_OK) return st;
  if (!X_bf16 || !s || !x_codes || !x_scales) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1_bf16 != nullptr) || (r > 0 && !U)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(s) || !aligned16(x_codes) || !aligned16(x_scales) ||
      (L1_bf16 && !aligned16(L1_bf16)) || (U && !aligned16(U)))
    return HSQ_ERR_ALIGNMENT;
  const int G = groups_of(K, group), Kp = G * group, ld = scales_ld(M);
  const auto* X = static_cast<const __nv_bfloat16*>(X_bf16);
  const auto* L1 = static_cast<const __nv_bfloat16*>(L1_bf16);
#define HSQ_ACT_LAUNCH(RV, SM)                                                                              \
  lerr = (group == 128 ? launch_pdl(true, hsq::quantize_act_kernel<RV, SM, 16>,                             \
                                    dim3((M + hsq::ActCfg<RV, SM>::RB - 1) / hsq::ActCfg<RV, SM>::RB),     \
                                    dim3(hsq::ActCfg<RV, SM>::NW * 32), 0, stream, X, s, L1, M, K, r, Kp, ld, \
                                    x_codes, x_scales, U, static_cast<float*>(nullptr), zc, zc_words)      \
                       : launch_pdl(true, hsq::quantize_act_kernel<RV, SM, 8>,                              \
                                    dim3((M + hsq::ActCfg<RV, SM>::RB - 1) / hsq::ActCfg<RV, SM>::RB),     \
                                    dim3(hsq::ActCfg<RV, SM>::NW * 32), 0, stream, X, s, L1, M, K, r, Kp, ld, \
                                    x_codes, x_scales, U, static_cast<float*>(nullptr), zc, zc_words))
#define HSQ_ACT_RANKS(SM)                   \
  switch (r) {                              \
    case 0: HSQ_ACT_LAUNCH(0, SM); break;   \
    case 1: HSQ_ACT_LAUNCH(1, SM); break;   \
    case 2: HSQ_ACT_LAUNCH(2, SM); break;   \
    case 4: HSQ_ACT_LAUNCH(4, SM); break;   \
    case 8: HSQ_ACT_LAUNCH(8, SM); break;   \
    case 16: HSQ_ACT_LAUNCH(16, SM); break; \
    case 32: HSQ_ACT_LAUNCH(32, SM); break; \
    default: HSQ_ACT_LAUNCH(-1, SM); break; \
  }
#define HSQ_ACT_ROWS_LAUNCH(RV, NW, SUB)                                                                  \
  lerr = (group == 128 ? launch_act_rows<RV, 16, NW, SUB>(X, s, L1, M, K, Kp, ld, x_codes, x_scales, U, stream,    \
                                                          nullptr, nullptr, 0, zc, zc_words)                   \
                       : launch_act_rows<RV, 8, NW, SUB>(X, s, L1, M, K, Kp, ld, x_codes, x_scales, U, stream,     \
                                                         nullptr, nullptr, 0, zc, zc_words))
#define HSQ_ACT_ROWS_RANKS(NW, SUB)               \
  switch (r) {                                    \
    case 0: HSQ_ACT_ROWS_LAUNCH(0, NW, SUB); break; \
    case 1: HSQ_ACT_ROWS_LAUNCH(1, NW, SUB); break; \
    case 2: HSQ_ACT_ROWS_LAUNCH(2, NW, SUB); break; \
    default: HSQ_ACT_ROWS_LAUNCH(4, NW, SUB); break; \
  }
  cudaError_t lerr = cudaSuccess;
  // few rows: one block per sub-block with 32 warps spread over K; many rows
  // (from 24 per SM: one and a half 16-row blocks per SM) and ranks 0, 1, 2, 4: the
  // row-owning kernel; else 8 warps x 2 sub-blocks
  const bool rows_kernel = HSQ_ACT_ROWS && (r <= 2 || r == 4) && M >= HSQ_ACT_ROWS16_MIN * device_sm_count();
  if (M <= 64) {
    HSQ_ACT_RANKS(true)
  } else if (rows_kernel) {
    HSQ_ACT_ROWS_RANKS(8, HSQ_ACT_ROWS_SUB)
  } else {
    HSQ_ACT_RANKS(false)
  }
#undef HSQ_ACT_ROWS_RANKS
#undef HSQ_ACT_ROWS_LAUNCH
#undef HSQ_ACT_RANKS
#undef HSQ_ACT_LAUNCH
  return (lerr == cudaSuccess && cudaGetLastError() == cudaSuccess) ? HSQ_OK : HSQ_ERR_CUDA;
}

// hsq_linear_forward and hsq_linear_forward_pre: w_e4m3, when not null, is the
// weights' expanded copy (hsq_expand_weights), used where the GEMM reads
// pre-expanded operands instead of expanding w_codes into the workspace.
// x_expanded: the activations' E4M3 tiles are already in the workspace (written
// by the activation kernel of hsq_linear_forward_x); x_codes is then unused.
static hsq_status forward_impl(const uint8_t* x_codes, const float* x_scales, const float* U, const uint8_t* w_codes,
                               const float* w_scales, const uint8_t* w_e4m3, const void* L2_bf16,
                               const void* bias_bf16, int M, int N, int K, int r, int group, void* Y,
                               hsq_out_dtype out, void* workspace, size_t ws_bytes, cudaStream_t stream,
                               bool x_expanded = false) {
  hsq_status st = check_common(M, K, r, group);
  if (st != HSQ_OK) return st;
  if (N < 1 || N > kMaxDim) return HSQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return HSQ_ERR_UNSUPPORTED;
  if (out != HSQ_OUT_BF16 && out != HSQ_OUT_F32) return HSQ_ERR_INVALID_ARG;
  if (!x_codes || !x_scales || !w_codes || !w_scales || !Y) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L2_bf16 != nullptr) || (r > 0) != (U != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(Y) || (U && !aligned16(U)) || (L2_bf16 && !aligned16(L2_bf16)) ||
      (bias_bf16 && !aligned16(bias_bf16)) || (workspace && !aligned16(workspace)) ||
      (w_e4m3 && !aligned16(w_e4m3)))
    return HSQ_ERR_ALIGNMENT;

  const int G = groups_of(K, group), Kp = G * group;
  const Plan p = make_plan(M, N, K, group, device_sm_count());
  // with the weights' expanded copy the workspace ends before the expanded weights
  const bool w_pre = w_e4m3 && p.pre_w_bytes > 0;
  const size_t ws_need = w_pre ? p.pre_w_offset() : p.ws_bytes();
  if (ws_need > 0 && (!workspace || ws_bytes < ws_need)) return HSQ_ERR_INVALID_ARG;
  if (p.kind == kGemv) {
    hsq::GemvArgs ga{};
    ga.x_codes = x_codes; ga.x_scales = x_scales; ga.ldx = scales_ld(M);
    ga.w_codes = w_codes; ga.w_scales = w_scales; ga.ldw = scales_ld(N);
    ga.U = U; ga.r = r;
    ga.L2 = static_cast<const __nv_bfloat16*>(L2_bf16);
    ga.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
    ga.Y = Y;
    ga.out_f32 = out == HSQ_OUT_F32 ? 1 : 0;
    ga.M = M; ga.N = N; ga.Kp = Kp; ga.G = G;
    ga.rows_per_block = p.tiles_r;
    const int mt = gemv_mt(M);
    const bool g128 = group == 128;
    if (mt == 1) return g128 ? launch_gemv<1, 4>(p, ga, stream) : launch_gemv<1, 2>(p, ga, stream);
    if (mt == 2) return g128 ? launch_gemv<2, 4>(p, ga, stream) : launch_gemv<2, 2>(p, ga, stream);
    if (mt == 4) return g128 ? launch_gemv<4, 4>(p, ga, stream) : launch_gemv<4, 2>(p, ga, stream);
    return g128 ? launch_gemv<8, 4>(p, ga, stream) : launch_gemv<8, 2>(p, ga, stream);
  }

  hsq::GemmArgs a{};
  const int ldx = scales_ld(M), ldw = scales_ld(N);
  CUtensorMap tm_row, tm_col;
  bool ok;
  if (!p.swap) {
    a.scales_r = x_scales; a.ld_r = ldx; a.rows_r = M;
    a.scales_c = w_scales; a.ld_c = ldw; a.rows_c = N;
    ok = make_codes_map(&tm_row, x_codes, M, Kp, 128, p.bps_stage) &&
         make_codes_map(&tm_col, w_codes, N, Kp, p.BN, p.bps_stage);
  } else {
    a.scales_r = w_scales; a.ld_r = ldw; a.rows_r = N;
    a.scales_c = x_scales; a.ld_c = ldx; a.rows_c = M;
    ok = make_codes_map(&tm_row, w_codes, N, Kp, 128, p.bps_stage) &&
         make_codes_map(&tm_col, x_codes, M, Kp, p.BN, p.bps_stage);
  }
  CUtensorMap tm_y = tm_row;  // only the tokens x outputs kernel stores through a map
  if (!p.swap) ok = make_y_map(&tm_y, Y, M, N, out == HSQ_OUT_F32);
  if (!ok) return HSQ_ERR_CUDA;
  a.U = U;
  a.L2 = static_cast<const __nv_bfloat16*>(L2_bf16);
  a.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
  a.Y = Y;
  a.out_f32 = out == HSQ_OUT_F32 ? 1 : 0;
  a.M = M; a.N = N; a.G = G; a.r = r;
  a.tiles_r = p.tiles_r; a.tiles_c = p.tiles_c;
  a.stages_per_tile = p.stages_per_tile; a.stream_len = p.stream_len;
  if (p.stream_len > 0) {
    a.ws_counters = static_cast<unsigned*>(workspace);
    a.ws_partials = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + p.counters_bytes);
  }
  if (p.pre_x_bytes > 0) {
    // expand both code matrices into MMA-ready E4M3 tiles (rows padded to whole tiles)
    uint8_t* xe = static_cast<uint8_t*>(workspace) + p.pre_x_offset();
    uint8_t* we = w_pre ? const_cast<uint8_t*>(w_e4m3) : static_cast<uint8_t*>(workspace) + p.pre_w_offset();
    const int blocks = 4 * device_sm_count();
    if ((!x_expanded && launch_pdl(false, hsq::expand_e4m3_kernel, dim3(blocks), dim3(256), 0, stream, x_codes, M,
                                   Kp, p.rg_r * 8, xe) != cudaSuccess) ||
        (!w_pre && launch_pdl(false, hsq::expand_e4m3_kernel, dim3(blocks), dim3(256), 0, stream, w_codes, N, Kp,
                              p.rg_c * 8, we) != cudaSuccess))
      return HSQ_ERR_CUDA;
    a.xe = xe;
    a.we = we;
    a.rg_r = p.rg_r;
    a.rg_c = p.rg_c;
    // CTA pairs read the expanded tiles with tiled loads (the row and col maps
    // of the pre-expanded kernel)
    if (CfgLarge64::PAIR && !(make_e8_map(&tm_row, xe, p.pre_x_bytes) && make_e8_map(&tm_col, we, p.pre_w_bytes)))
      return HSQ_ERR_CUDA;
  }
  // U L2 + b as a bf16 MMA step when the kernel has one and the rank fits its K
  // U L2 + b as tensor-core steps of LR_MAX_RANK ranks each (at least one: the bias)
  static_assert(CfgLarge64::LR_MAX_RANK == CfgLarge128::LR_MAX_RANK, "low-rank chunk");
  // (at most three steps: r <= 32 < 3 * LR_MAX_RANK; the kernel builds chunks 0..2)
  static_assert(kMaxRank <= 3 * CfgLarge64::LR_MAX_RANK, "low-rank steps");
  static_assert(CfgMid64::LR_MMA && CfgMid64::LR_MAX_RANK == CfgLarge64::LR_MAX_RANK, "mid tiles: low-rank steps");
  a.lr_mma = (HSQ_LR_MMA && (p.kind == kLarge || p.kind == kMid) && CfgLarge64::LR_MMA && CfgLarge128::LR_MMA)
                 ? std::max(1, (r + CfgLarge64::LR_MAX_RANK - 1) / CfgLarge64::LR_MAX_RANK)
                 : 0;
  a.limit_ns = wait_limit_ns();
  if (t_debug_flags) {
    a.debug_flags = t_debug_flags;
    a.limit_ns = static_cast<uint64_t>(t_debug_limit_ms > 0 ? t_debug_limit_ms : 50) * 1000000ull;
    t_debug_flags = 0;
  }
  const bool g128 = group == 128;
  switch (p.kind) {
    case kLarge:
      if (many_rank_kernel(r))
        return g128 ? launch_gemm<CfgLarge128R>(p, tm_row, tm_col, tm_y, a, stream)
                    : launch_gemm<CfgLarge64R>(p, tm_row, tm_col, tm_y, a, stream);
      return g128 ? launch_gemm<CfgLarge128>(p, tm_row, tm_col, tm_y, a, stream)
                  : launch_gemm<CfgLarge64>(p, tm_row, tm_col, tm_y, a, stream);
    case kMid:
      if (many_rank_kernel(r)) return launch_gemm<CfgMid64R>(p, tm_row, tm_col, tm_y, a, stream);
      return launch_gemm<CfgMid64>(p, tm_row, tm_col, tm_y, a, stream);
    case kDec16:
      return g128 ? launch_gemm<CfgDec16_128>(p, tm_row, tm_col, tm_y, a, stream)
                  : launch_gemm<CfgDec16_64>(p, tm_row, tm_col, tm_y, a, stream);
    case kDec32:
      return g128 ? launch_gemm<CfgDec32_128>(p, tm_row, tm_col, tm_y, a, stream)
                  : launch_gemm<CfgDec32_64>(p, tm_row, tm_col, tm_y, a, stream);
    case kDec64:
      return g128 ? launch_gemm<CfgDec64_128>(p, tm_row, tm_col, tm_y, a, stream)
                  : launch_gemm<CfgDec64_64>(p, tm_row, tm_col, tm_y, a, stream);
  }
  return HSQ_ERR_INVALID_ARG;
}

hsq_status hsq_linear_forward(const uint8_t* x_codes, const float* x_scales, const float* U, const uint8_t* w_codes,
                              const float* w_scales, const void* L2_bf16, const void* bias_bf16, int M, int N, int K,
                              int r, int group, void* Y, hsq_out_dtype out, void* workspace, size_t ws_bytes,
                              cudaStream_t stream) {
  return forward_impl(x_codes, x_scales, U, w_codes, w_scales, nullptr, L2_bf16, bias_bf16, M, N, K, r, group, Y, out,
                      workspace, ws_bytes, stream);
}

hsq_status hsq_linear_forward_pre(const uint8_t* x_codes, const float* x_scales, const float* U,
                                  const uint8_t* w_codes, const float* w_scales, const uint8_t* w_e4m3,
                                  const void* L2_bf16, const void* bias_bf16, int M, int N, int K, int r, int group,
                                  void* Y, hsq_out_dtype out, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  if (!w_e4m3) return HSQ_ERR_INVALID_ARG;
  return forward_impl(x_codes, x_scales, U, w_codes, w_scales, w_e4m3, L2_bf16, bias_bf16, M, N, K, r, group, Y, out,
                      workspace, ws_bytes, stream);
}

// hsq_linear_forward_x's workspace: the GEMM's part first, then the activation
// step's outputs (packed codes only where the GEMM does not take expanded tiles
// from the activation kernel), scales and U.
struct XLayout {
  Plan p;
  bool expanded;  // the activation kernel writes the GEMM's E4M3 tiles itself
  size_t gemm, o_codes, o_scales, o_u, total;
};
static XLayout x_layout(int M, int N, int K, int r, int group, int nsm, bool w_pre) {
  XLayout L{};
  L.p = make_plan(M, N, K, group, nsm);
  const int G = groups_of(K, group), Kp = G * group;
  L.expanded = L.p.pre_x_bytes > 0 && HSQ_ACT_ROWS && (r <= 2 || r == 4) && M >= HSQ_ACT_ROWS16_MIN * nsm;
  L.gemm = (w_pre && L.p.pre_w_bytes > 0) ? L.p.pre_w_offset() : L.p.ws_bytes();
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t off = up(L.gemm);
  L.o_codes = off;
  if (!L.expanded) off = up(off + static_cast<size_t>(M) * (Kp / 2));
  L.o_scales = off;
  off = up(off + static_cast<size_t>(G) * scales_ld(M) * 4);
  L.o_u = off;
  off = up(off + static_cast<size_t>(M) * std::max(r, 1) * 4);
  L.total = off;
  return L;
}

size_t hsq_workspace_bytes_x(int M, int N, int K, int r, int group, int with_w_e4m3) {
  if (check_common(M, K, r, group) != HSQ_OK || N < 1 || N > kMaxDim) return 0;
  return x_layout(M, N, K, r, group, device_sm_count(), with_w_e4m3 != 0).total;
}

hsq_status hsq_linear_forward_x(const void* X_bf16, const float* s, const void* L1_bf16, const uint8_t* w_codes,
                                const float* w_scales, const uint8_t* w_e4m3, const void* L2_bf16,
                                const void* bias_bf16, int M, int N, int K, int r, int group, void* Y,
                                hsq_out_dtype out, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  hsq_status st = check_common(M, K, r, group);
  if (st != HSQ_OK) return st;
  if (N < 1 || N > kMaxDim) return HSQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return HSQ_ERR_UNSUPPORTED;
  if (out != HSQ_OUT_BF16 && out != HSQ_OUT_F32) return HSQ_ERR_INVALID_ARG;
  if (!X_bf16 || !s || !w_codes || !w_scales || !Y || !workspace) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1_bf16 != nullptr) || (r > 0) != (L2_bf16 != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(s) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(Y) ||
      !aligned16(workspace) || (w_e4m3 && !aligned16(w_e4m3)) || (L1_bf16 && !aligned16(L1_bf16)) ||
      (L2_bf16 && !aligned16(L2_bf16)) || (bias_bf16 && !aligned16(bias_bf16)))
    return HSQ_ERR_ALIGNMENT;
  const int nsm = device_sm_count();
  const XLayout L = x_layout(M, N, K, r, group, nsm, w_e4m3 != nullptr);
  if (ws_bytes < L.total) return HSQ_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  float* xs = reinterpret_cast<float*>(base + L.o_scales);
  float* U = r > 0 ? reinterpret_cast<float*>(base + L.o_u) : nullptr;
  // the split-K counters start at zero whatever the workspace held: the
  // activation kernel clears them (after the preceding kernel, before the GEMM)
  unsigned* zc = (L.p.kind != kGemv && L.p.stream_len > 0) ? static_cast<unsigned*>(workspace) : nullptr;
  const int zc_words = zc ? static_cast<int>(L.p.counters_bytes / 4) : 0;
  if (!L.expanded) {
    st = quantize_act_impl(X_bf16, s, L1_bf16, M, K, r, group, base + L.o_codes, xs, U, stream, zc, zc_words);
    if (st != HSQ_OK) return st;
    return forward_impl(base + L.o_codes, xs, U, w_codes, w_scales, w_e4m3, L2_bf16, bias_bf16, M, N, K, r, group,
                        Y, out, workspace, L.gemm, stream);
  }
  // the activation kernel writes the GEMM's E4M3 tiles (padding rows zeroed first)
  const int G = groups_of(K, group), Kp = G * group, ld = scales_ld(M);
  const int rows_pad = L.p.rg_r * 8;
  uint8_t* xe = base + L.p.pre_x_offset();
  if (rows_pad > M) {
    const size_t n = static_cast<size_t>(Kp / 64) * (rows_pad - M) * 4;
    const int blocks = static_cast<int>(std::min<size_t>(4 * nsm, (n + 255) / 256));
    if (launch_pdl(true, hsq::zero_e4m3_rows_kernel, dim3(blocks), dim3(256), 0, stream, xe, M, rows_pad, Kp) !=
        cudaSuccess)
      return HSQ_ERR_CUDA;
  }
  const auto* X = static_cast<const __nv_bfloat16*>(X_bf16);
  const auto* L1 = static_cast<const __nv_bfloat16*>(L1_bf16);
  cudaError_t lerr = cudaSuccess;
#define HSQ_X_ACT(RV)                                                                                          \
  lerr = group == 128 ? launch_act_rows<RV, 16, 8, HSQ_ACT_ROWS_SUB>(X, s, L1, M, K, Kp, ld, nullptr, xs, U, stream, \
                                                                    nullptr, xe, L.p.rg_r, zc, zc_words)        \
                      : launch_act_rows<RV, 8, 8, HSQ_ACT_ROWS_SUB>(X, s, L1, M, K, Kp, ld, nullptr, xs, U, stream,  \
                                                                   nullptr, xe, L.p.rg_r, zc, zc_words)
  switch (r) {
    case 0: HSQ_X_ACT(0); break;
    case 1: HSQ_X_ACT(1); break;
    case 2: HSQ_X_ACT(2); break;
    default: HSQ_X_ACT(4); break;
  }
#undef HSQ_X_ACT
  if (lerr != cudaSuccess || cudaGetLastError() != cudaSuccess) return HSQ_ERR_CUDA;
  return forward_impl(xe, xs, U, w_codes, w_scales, w_e4m3, L2_bf16, bias_bf16, M, N, K, r, group, Y, out, workspace,
                      L.gemm, stream, true);
}

size_t hsq_weights_e4m3_bytes(int N, int K, int group) {
  if (N < 1 || K < 1 || N > kMaxDim || K > kMaxDim || (group != 64 && group != 128)) return 0;
  const size_t rows_pad = static_cast<size_t>((N + CfgLarge64::BN - 1) / CfgLarge64::BN) * CfgLarge64::BN;
  return rows_pad * static_cast<size_t>(groups_of(K, group) * group);
}

hsq_status hsq_expand_weights(const uint8_t* w_codes, int N, int K, int group, uint8_t* w_e4m3,
                              cudaStream_t stream) {
  hsq_status st = check_common(N, K, 0, group);
  if (st != HSQ_OK) return st;
  if (!w_codes || !w_e4m3) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(w_codes) || !aligned16(w_e4m3)) return HSQ_ERR_ALIGNMENT;
  const int Kp = groups_of(K, group) * group;
  const int rows_pad = (N + CfgLarge64::BN - 1) / CfgLarge64::BN * CfgLarge64::BN;
  const int blocks = 4 * device_sm_count();
  if (launch_pdl(false, hsq::expand_e4m3_kernel, dim3(blocks), dim3(256), 0, stream, w_codes, N, Kp, rows_pad,
                 w_e4m3) != cudaSuccess)
    return HSQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

size_t hsq_workspace_bytes_pre(int M, int N, int K, int r) {
  (void)r;
  if (M < 1 || N < 1 || K < 1) return 0;
  const int nsm = device_sm_count();
  size_t need = 0;
  for (int group : {64, 128}) {
    const Plan p = make_plan(M, N, K, group, nsm);
    need = std::max(need, p.pre_w_bytes > 0 ? p.pre_w_offset() : p.ws_bytes());
  }
  return need;
}

hsq_status hsq_linear_forward_noalloc(const uint8_t* x_codes, const float* x_scales, const float* U,
                                      const uint8_t* w_codes, const float* w_scales, const void* L2_bf16,
                                      const void* bias_bf16, int M, int N, int K, int r, int group, void* Y,
                                      hsq_out_dtype out, cudaStream_t stream) {
  // The same argument checks as hsq_linear_forward, made before the scratch is touched,
  // so that a rejected call launches nothing.
  hsq_status st = check_common(M, K, r, group);
  if (st != HSQ_OK) return st;
  if (N < 1 || N > kMaxDim) return HSQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return HSQ_ERR_UNSUPPORTED;
  if (out != HSQ_OUT_BF16 && out != HSQ_OUT_F32) return HSQ_ERR_INVALID_ARG;
  if (!x_codes || !x_scales || !w_codes || !w_scales || !Y) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L2_bf16 != nullptr) || (r > 0) != (U != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_scales) || !aligned16(w_codes) || !aligned16(w_scales) ||
      !aligned16(Y) || (U && !aligned16(U)) || (L2_bf16 && !aligned16(L2_bf16)) ||
      (bias_bf16 && !aligned16(bias_bf16)))
    return HSQ_ERR_ALIGNMENT;
  const Plan p = make_plan(M, N, K, group, device_sm_count());
  void* scratch = nullptr;
  if (p.ws_bytes() > 0) {
    if (p.ws_bytes() > kNoallocScratchBytes) return HSQ_ERR_SCRATCH_LIMIT;
    st = noalloc_scratch(&scratch);
    if (st != HSQ_OK) return st;
    // the split-K counters must start at zero; the partial tiles are written before they are read
    if (cudaMemsetAsync(scratch, 0, p.counters_bytes, stream) != cudaSuccess) return HSQ_ERR_CUDA;
  }
  return hsq_linear_forward(x_codes, x_scales, U, w_codes, w_scales, L2_bf16, bias_bf16, M, N, K, r, group, Y, out,
                            scratch, scratch ? kNoallocScratchBytes : 0, stream);
}

hsq_status hsq_linear_forward_fused(const void* X_bf16, const float* s, const void* L1_bf16, const uint8_t* w_codes,
                                    const float* w_scales, const void* L2_bf16, const void* bias_bf16, int M, int N,
                                    int K, int r, int group, void* Y, hsq_out_dtype out, cudaStream_t stream) {
  hsq_status st = check_common(M, K, r, group);
  if (st != HSQ_OK) return st;
  if (N < 1 || N > kMaxDim) return HSQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return HSQ_ERR_UNSUPPORTED;
  if (out != HSQ_OUT_BF16 && out != HSQ_OUT_F32) return HSQ_ERR_INVALID_ARG;
  if (!X_bf16 || !s || !w_codes || !w_scales || !Y) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1_bf16 != nullptr) || (r > 0) != (L2_bf16 != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(s) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(Y) ||
      (L1_bf16 && !aligned16(L1_bf16)) || (L2_bf16 && !aligned16(L2_bf16)) || (bias_bf16 && !aligned16(bias_bf16)))
    return HSQ_ERR_ALIGNMENT;
  const int G = groups_of(K, group), Kp = G * group;
  const int mt = gemv_mt(M);
  const int nsm = device_sm_count();
  // up to 4 tokens at ranks 0, 1, 2, 4 with the block's rows in shared memory:
  // the weight stream, each block repeating the activation step; else up to 16
  // tokens: the decode tiles, the step spread over the grid
  const int form = fused_form(M, N, K, r, group, nsm);
  if (form == 0) return HSQ_ERR_UNSUPPORTED;
  if (form == 2)
    return forward_fused_dec16(X_bf16, s, L1_bf16, w_codes, w_scales, L2_bf16, bias_bf16, M, N, K, r, group, Y, out,
                               stream);
  Plan p{};
  p.kind = kGemv;
  p.tiles_r = gemv_rows_per_block(N, nsm);
  p.grid = (N + p.tiles_r - 1) / p.tiles_r;
  hsq::GemvArgs ga{};
  ga.w_codes = w_codes; ga.w_scales = w_scales; ga.ldw = scales_ld(N);
  ga.r = r;
  ga.L2 = static_cast<const __nv_bfloat16*>(L2_bf16);
  ga.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
  ga.Y = Y;
  ga.out_f32 = out == HSQ_OUT_F32 ? 1 : 0;
  ga.M = M; ga.N = N; ga.Kp = Kp; ga.G = G;
  ga.rows_per_block = p.tiles_r;
  ga.X = static_cast<const __nv_bfloat16*>(X_bf16);
  ga.s = s;
  ga.L1 = static_cast<const __nv_bfloat16*>(L1_bf16);
  ga.K = K; ga.group = group;
  const bool g128 = group == 128;
#define HSQ_FUSED(MTV, RV) \
  return g128 ? launch_gemv<MTV, 4, RV>(p, ga, stream) : launch_gemv<MTV, 2, RV>(p, ga, stream)
#define HSQ_FUSED_R(MTV)          \
  switch (r) {                    \
    case 0: HSQ_FUSED(MTV, 0);    \
    case 1: HSQ_FUSED(MTV, 1);    \
    case 2: HSQ_FUSED(MTV, 2);    \
    default: HSQ_FUSED(MTV, 4);   \
  }
  if (mt == 1) HSQ_FUSED_R(1);
  if (mt == 2) HSQ_FUSED_R(2);
  HSQ_FUSED_R(4);
#undef HSQ_FUSED_R
#undef HSQ_FUSED
}

int hsq_fused_form(int M, int N, int K, int r, int group) { return fused_form(M, N, K, r, group, device_sm_count()); }

// ------------------------------------------------------------------ NVFP4 variant
// Block-scaled GEMM tile: 128 tokens x HSQ_FP4_BN outputs (hsq_fp4.cuh).
#ifndef HSQ_FP4_BN
#define HSQ_FP4_BN 256
#endif
using CfgFp4 = hsq::Fp4Cfg<HSQ_FP4_BN, HSQ_FP4_BN == 256 ? 1 : 2, HSQ_FP4_BN == 256 ? 3 : 5>;
static int fp4_kq(int K) { return (K + 63) / 64 * 64; }

size_t hsq_fp4_codes_bytes(int rows, int K) {
  if (rows < 0 || K < 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(fp4_kq(K)) / 2;
}

size_t hsq_fp4_scales_bytes(int rows, int K) {
  if (rows < 0 || K < 0) return 0;
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>(fp4_kq(K) / 64) * 512;
}

static hsq_status fp4_check(int rows, int K, int r) {
  if (rows < 1 || K < 1 || rows > kMaxDim || K > kMaxDim || r < 0) return HSQ_ERR_INVALID_ARG;
  if (r > kMaxRank || (K % 8) != 0) return HSQ_ERR_UNSUPPORTED;
  return HSQ_OK;
}

hsq_status hsq_fp4_pack_weights(const void* W_bf16, const float* s, const void* L1_bf16, const void* L2_bf16, int N,
                                int K, int r, uint8_t* w_codes, uint8_t* w_sf, float* w_gs, cudaStream_t stream) {
  hsq_status st = fp4_check(N, K, r);
  if (st != HSQ_OK) return st;
  if (!W_bf16 || !s || !w_codes || !w_sf || !w_gs) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1_bf16 != nullptr) || (r > 0) != (L2_bf16 != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(W_bf16) || !aligned16(s) || !aligned16(w_codes) || !aligned16(w_sf) || !aligned16(w_gs) ||
      (L1_bf16 && !aligned16(L1_bf16)) || (L2_bf16 && !aligned16(L2_bf16)))
    return HSQ_ERR_ALIGNMENT;
  const int Kq = fp4_kq(K), KC = Kq / 64;
  const auto* W = static_cast<const __nv_bfloat16*>(W_bf16);
  const auto* L1 = static_cast<const __nv_bfloat16*>(L1_bf16);
  const auto* L2 = static_cast<const __nv_bfloat16*>(L2_bf16);
  const int blocks = (N + 7) / 8;
  if (cudaMemsetAsync(w_gs, 0, 2 * sizeof(float), stream) != cudaSuccess) return HSQ_ERR_CUDA;
  // first pass: absmax of the residual; second pass: codes and block scales
  hsq::pack_weights_kernel<2, 1><<<blocks, 256, 0, stream>>>(W, s, L1, L2, N, K, r, Kq, 0, w_codes, nullptr, w_gs);
  hsq::pack_weights_kernel<2, 2><<<blocks, 256, 0, stream>>>(W, s, L1, L2, N, K, r, Kq, 0, w_codes,
                                                             reinterpret_cast<float*>(w_sf), w_gs);
  const int pad = (N + 127) / 128 * 128 - N;
  if (pad > 0) hsq::nvfp4_zero_sf_pad_kernel<<<(pad * KC + 255) / 256, 256, 0, stream>>>(w_sf, N, KC);
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

hsq_status hsq_fp4_quantize_act(const void* X_bf16, const float* s, const void* L1_bf16, int M, int K, int r,
                                uint8_t* x_codes, uint8_t* x_sf, float* x_gs, float* U, cudaStream_t stream) {
  hsq_status st = fp4_check(M, K, r);
  if (st != HSQ_OK) return st;
  if (!X_bf16 || !s || !x_codes || !x_sf || !x_gs) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L1_bf16 != nullptr) || (r > 0 && !U)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(X_bf16) || !aligned16(s) || !aligned16(x_codes) || !aligned16(x_sf) || !aligned16(x_gs) ||
      (L1_bf16 && !aligned16(L1_bf16)) || (U && !aligned16(U)))
    return HSQ_ERR_ALIGNMENT;
  const int Kq = fp4_kq(K), KC = Kq / 64;
  const auto* X = static_cast<const __nv_bfloat16*>(X_bf16);
  const auto* L1 = static_cast<const __nv_bfloat16*>(L1_bf16);
  float* sf = reinterpret_cast<float*>(x_sf);
  if (cudaMemsetAsync(x_gs, 0, 2 * sizeof(float), stream) != cudaSuccess) return HSQ_ERR_CUDA;
  // the tensor absmax from column maxima: about four blocks of rows per SM,
  // rows per block a multiple of 8 once there are enough (eight loads in flight)
  const int nsm = device_sm_count();
  int rpb = std::max(1, (M + 4 * nsm - 1) / (4 * nsm));
  if (rpb > 4) rpb = (rpb + 7) / 8 * 8;
  if (launch_pdl(false, hsq::nvfp4_act_colmax_kernel, dim3((M + rpb - 1) / rpb), dim3(128), 0, stream, X, s, M, K,
                 rpb, x_gs) != cudaSuccess)
    return HSQ_ERR_CUDA;
  cudaError_t lerr = cudaSuccess;
#define HSQ_FP4_ACT(RV, SM)                                                                                \
  lerr = launch_pdl(false, hsq::quantize_act_kernel<RV, SM, 2, true>,                                      \
                    dim3((M + hsq::ActCfg<RV, SM>::RB - 1) / hsq::ActCfg<RV, SM>::RB),                     \
                    dim3(hsq::ActCfg<RV, SM>::NW * 32), 0, stream, X, s, L1, M, K, r, Kq, 0, x_codes, sf, U, \
                    x_gs, static_cast<unsigned*>(nullptr), 0)
#define HSQ_FP4_RANKS(SM)                  \
  switch (r) {                             \
    case 0: HSQ_FP4_ACT(0, SM); break;     \
    case 1: HSQ_FP4_ACT(1, SM); break;     \
    case 2: HSQ_FP4_ACT(2, SM); break;     \
    case 4: HSQ_FP4_ACT(4, SM); break;     \
    case 8: HSQ_FP4_ACT(8, SM); break;     \
    case 16: HSQ_FP4_ACT(16, SM); break;   \
    case 32: HSQ_FP4_ACT(32, SM); break;   \
    default: HSQ_FP4_ACT(-1, SM); break;   \
  }
  if (M <= 64) {
    HSQ_FP4_RANKS(true)
  } else if (HSQ_ACT_ROWS && (r <= 2 || r == 4) && M >= HSQ_ACT_ROWS16_MIN * nsm) {
    // many rows: the row-owning kernel in its NVFP4 form
    switch (r) {
      case 0: lerr = launch_act_rows<0, 2, 8, 2, true>(X, s, L1, M, K, Kq, 0, x_codes, sf, U, stream, x_gs); break;
      case 1: lerr = launch_act_rows<1, 2, 8, 2, true>(X, s, L1, M, K, Kq, 0, x_codes, sf, U, stream, x_gs); break;
      case 2: lerr = launch_act_rows<2, 2, 8, 2, true>(X, s, L1, M, K, Kq, 0, x_codes, sf, U, stream, x_gs); break;
      default: lerr = launch_act_rows<4, 2, 8, 2, true>(X, s, L1, M, K, Kq, 0, x_codes, sf, U, stream, x_gs); break;
    }
  } else {
    HSQ_FP4_RANKS(false)
  }
#undef HSQ_FP4_RANKS
#undef HSQ_FP4_ACT
  if (lerr != cudaSuccess) return HSQ_ERR_CUDA;
  const int pad = (M + 127) / 128 * 128 - M;
  if (pad > 0) hsq::nvfp4_zero_sf_pad_kernel<<<(pad * KC + 255) / 256, 256, 0, stream>>>(x_sf, M, KC);
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

hsq_status hsq_fp4_linear_forward(const uint8_t* x_codes, const uint8_t* x_sf, const float* x_gs, const float* U,
                                  const uint8_t* w_codes, const uint8_t* w_sf, const float* w_gs,
                                  const void* L2_bf16, const void* bias_bf16, int M, int N, int K, int r, void* Y,
                                  hsq_out_dtype out, cudaStream_t stream) {
  hsq_status st = fp4_check(M, K, r);
  if (st != HSQ_OK) return st;
  if (N < 1 || N > kMaxDim) return HSQ_ERR_INVALID_ARG;
  if (N % 8 != 0) return HSQ_ERR_UNSUPPORTED;
  if (out != HSQ_OUT_BF16 && out != HSQ_OUT_F32) return HSQ_ERR_INVALID_ARG;
  if (!x_codes || !x_sf || !x_gs || !w_codes || !w_sf || !w_gs || !Y) return HSQ_ERR_INVALID_ARG;
  if ((r > 0) != (L2_bf16 != nullptr) || (r > 0) != (U != nullptr)) return HSQ_ERR_INVALID_ARG;
  if (!aligned16(x_codes) || !aligned16(x_sf) || !aligned16(x_gs) || !aligned16(w_codes) || !aligned16(w_sf) ||
      !aligned16(w_gs) || !aligned16(Y) || (U && !aligned16(U)) || (L2_bf16 && !aligned16(L2_bf16)) ||
      (bias_bf16 && !aligned16(bias_bf16)))
    return HSQ_ERR_ALIGNMENT;
  using Cfg = CfgFp4;
  const int Kq = fp4_kq(K);
  CUtensorMap tm_a, tm_b, tm_y;
  if (!make_fp4_codes_map(&tm_a, x_codes, M, Kq, Cfg::BM) || !make_fp4_codes_map(&tm_b, w_codes, N, Kq, Cfg::BN) ||
      !make_y_map(&tm_y, Y, M, N, out == HSQ_OUT_F32))
    return HSQ_ERR_CUDA;
  hsq::Fp4Args a{};
  a.x_sf = x_sf; a.w_sf = w_sf; a.x_gs = x_gs; a.w_gs = w_gs;
  a.U = U;
  a.L2 = static_cast<const __nv_bfloat16*>(L2_bf16);
  a.bias = static_cast<const __nv_bfloat16*>(bias_bf16);
  a.M = M; a.N = N; a.KC = Kq / 64; a.r = r;
  a.tiles_m = (M + Cfg::BM - 1) / Cfg::BM;
  a.tiles_n = (N + Cfg::BN - 1) / Cfg::BN;
  a.out_f32 = out == HSQ_OUT_F32 ? 1 : 0;
  a.limit_ns = wait_limit_ns();
  static std::mutex mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  {
    std::lock_guard<std::mutex> lk(mu);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
      if (cudaFuncSetAttribute(hsq::fp4_gemm_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::SMEM_BYTES) != cudaSuccess)
        return HSQ_ERR_CUDA;
      if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
  }
  const int tiles = a.tiles_m * a.tiles_n;
  const int grid = std::min(tiles, device_sm_count());
  if (launch_pdl(false, hsq::fp4_gemm_kernel<Cfg>, dim3(grid), dim3(Cfg::THREADS), Cfg::SMEM_BYTES, stream, tm_a,
                 tm_b, tm_y, a) != cudaSuccess)
    return HSQ_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? HSQ_OK : HSQ_ERR_CUDA;
}

}  // extern "C"
