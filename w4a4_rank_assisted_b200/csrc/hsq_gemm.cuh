// hsq_gemm.cuh -- packed INT4 x INT4 GEMM on tcgen05 (kind::i8) with a per-group
// fp32 rescale and a fused low-rank + bias epilogue.
//
// Computes (Deflating the Hessian, Abstract: 4-bit residual product plus the
// high-precision low-rank branch)
//     Y[m,n] = sum_g sx[g][m] sw[g][n] P_g[m,n] + sum_j U[m,j] L2[j,n] + b[n],
//     P_g[m,n] = sum_{k in group g} qx[m,k] qw[n,k]   (exact, int32)
//
// Blackwell has no INT4 tensor-core mode, so each 64-wide group is unpacked in
// shared memory to INT8 and multiplied with two tcgen05.mma.kind::i8 (K = 32
// each) into a Tensor Memory buffer; drain warps read the int32 partial with
// tcgen05.ld and fold it into fp32 register accumulators with its two scales.
//
// Operands are named by their role in the MMA:
//   "row" operand  -> MMA A, 128 rows per tile, one TMEM lane per row;
//   "col" operand  -> MMA B, BN rows per tile, one TMEM column per row.
// For large M the row operand is the activations (tile 128 tokens x BN=256
// outputs); for decode-sized M the roles swap (128 weight rows x BN tokens), so
// the MMA's M=128 side is always filled.
//
// Unpack: a packed byte holds two 4-bit two's-complement codes.  Masking a code
// into the HIGH nibble of a byte gives the int8 value 16*q, so one AND (odd
// codes) or one shift+AND (even codes) unpacks four codes; the MMA then sums
// 256*q_x*q_w, and the drain folds 1/256 into the per-row scale (a power-of-two,
// so the fp32 result is unchanged).  The even/odd split permutes K inside a
// group identically for both operands, which leaves every P_g unchanged.
//
// Warp roles (one CTA per SM, persistent over work units):
//   warp 0      TMA producer: packed row/col tiles + the col scales of one group
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2-7   unpack packed -> INT8 canonical K-major smem layout
//   warps 8..   drain / epilogue; warp w reads TMEM lanes 32*(w%4)..+31
// Pipelines: packed ring (STAGES) -> int8 double buffer -> TMEM double buffer.
#pragma once

#include "hsq_device.cuh"

namespace hsq {

// Canonical no-swizzle K-major layout of an operand with `rows` rows and one
// 64-wide group: core matrix (row/8, kc) (kc = 16-byte K chunk 0..3) at
// (row/8)*SBO + kc*LBO bytes, its 8 rows 16 bytes apart; the second K=32 MMA
// starts 2*LBO bytes in.  LBO = 160 (not 128) staggers the four K chunks of a
// row block across shared-memory banks, so that the unpack warps' 16-byte
// stores of 8 consecutive threads (4 rows x 2 halves) hit 8 distinct bank groups;
// SBO = 3*LBO + 128.
#ifndef HSQ_PAD_LAYOUT
#define HSQ_PAD_LAYOUT 1
#endif
constexpr uint32_t kLBO = HSQ_PAD_LAYOUT ? 160 : 128;
constexpr uint32_t kSBO = 3 * kLBO + 128;

struct GemmArgs {
  const float* scales_r;  // row operand scales   [G][ld_r]
  const float* scales_c;  // col operand scales   [G][ld_c]
  int ld_r, ld_c;
  int rows_r, rows_c;     // valid rows of each operand
  const float* U;         // [M][r]
  const __nv_bfloat16* L2;    // [r][N]
  const __nv_bfloat16* bias;  // [N] or nullptr
  void* Y;                // [M][N]
  int out_f32;
  int M, N, G, r;
  int tiles_r, tiles_c, splits, groups_per_split;
  float* ws_partials;     // split-K partial tiles
  unsigned* ws_counters;  // split-K arrival counters (zero between calls)
  uint64_t limit_ns;      // wait limit
  int debug_flags;        // 1: producer issues nothing (forces the timeout path)
};

// DRAIN_ selects how a group's int32 partial becomes fp32 in the drain; all
// three give bit-identical results:
//   0: cvt.rn.f32.s32 per value, scalar fmul/fma
//   1: cvt.rn.f32.s32 per value, packed f32x2 mul/fma
//   2: the TMEM partial starts each group at the bit pattern of 1.5*2^23, so the
//      MMA leaves 1.5*2^23 + P (exact, |P| < 2^22) as an fp32 bit pattern; one
//      packed f32x2 subtract recovers P exactly (no int->float conversion), and
//      the drain re-fills the buffer with the pattern after reading it.
#ifndef HSQ_DRAIN_MODE
#define HSQ_DRAIN_MODE 1
#endif
template <int BN_, int DH_, int STAGES_, bool SWAP_, int DRAIN_ = HSQ_DRAIN_MODE>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int DH = DH_;               // column slices handled by separate drain warps
  static constexpr int CW = BN / DH;           // columns per drain thread
  static constexpr int STAGES = STAGES_;
  static constexpr bool SWAP = SWAP_;
  static constexpr int DRAIN = DRAIN_;
  static constexpr int NUM_UNPACK_WARPS = 6;
  static constexpr int NUM_DRAIN_WARPS = 4 * DH;
  static constexpr int THREADS = 32 * (2 + NUM_UNPACK_WARPS + NUM_DRAIN_WARPS);
  // Register split (setmaxnreg): producer/MMA/unpack warpgroups give registers
  // to the drain warpgroups, which hold CW fp32 accumulators per thread.
  static constexpr bool REALLOC = CW >= 64;
#ifndef HSQ_REGS_LOW
#define HSQ_REGS_LOW 64
#endif
  static constexpr int REGS_LOW = HSQ_REGS_LOW;
  static constexpr int REGS_HIGH_RAW = ((65536 - 256 * REGS_LOW) / (32 * NUM_DRAIN_WARPS)) / 8 * 8;
  static constexpr int REGS_HIGH = REGS_HIGH_RAW > 232 ? 232 : REGS_HIGH_RAW;
  static constexpr int A_PACK = BM * 32;       // packed bytes per group
  static constexpr int B_PACK = BN * 32;
  static constexpr int CS_BYTES = BN * 4;
  static constexpr int STAGE_BYTES = ((A_PACK + B_PACK + CS_BYTES + 1023) / 1024) * 1024;
  static constexpr int A_I8 = (BM / 8) * kSBO;  // int8 operand bytes per group
  static constexpr int B_I8 = (BN / 8) * kSBO;
  static constexpr int I8_BYTES = ((A_I8 + B_I8 + 1023) / 1024) * 1024;
  static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128
                                 : (2 * BN <= 256) ? 256 : 512;
  static constexpr int NUM_BARS = 2 * STAGES + 2 + 2 + 2 + 2 + 1;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 2 * I8_BYTES + NUM_BARS * 8 + 64;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(CW % 16 == 0, "drain chunks of 16 columns");
  static_assert(2 * BN <= 512, "TMEM");
};


constexpr uint32_t kMagicBits = 0x4B400000u;  // 1.5 * 2^23
constexpr float kMagic = 12582912.0f;

// One unpack task: 16 packed bytes (32 codes) of one row -> two 16-byte core
// matrix rows (even codes, odd codes).  Task t reads row t/2, half t%2, so 8
// consecutive threads read 128 contiguous bytes.
__device__ __forceinline__ void unpack_task(const uint8_t* src_stage, uint8_t* dst, int t) {
  const int row = t >> 1;
  const int half = t & 1;  // which 16 packed bytes (K 0-31 or 32-63)
  const uint4 p = *reinterpret_cast<const uint4*>(src_stage + t * 16);
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
  uint4 lo, hi;
  uint32_t* lo_w = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* hi_w = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    lo_w[i] = (w[i] << 4) & 0xF0F0F0F0u;  // even codes, 16*q as int8
    hi_w[i] = w[i] & 0xF0F0F0F0u;         // odd codes,  16*q as int8
  }
  uint8_t* base = dst + (row >> 3) * kSBO + (2 * half) * kLBO + (row & 7) * 16;
  *reinterpret_cast<uint4*>(base) = lo;
  *reinterpret_cast<uint4*>(base + kLBO) = hi;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_row, const __grid_constant__ CUtensorMap tm_col,
                     const GemmArgs args) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, CW = Cfg::CW, STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* i8_base = smem + STAGES * Cfg::STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(i8_base + 2 * Cfg::I8_BYTES);
  uint64_t* full = bars;                 // [STAGES] packed stage landed
  uint64_t* empty = bars + STAGES;       // [STAGES] packed stage free
  uint64_t* full8 = bars + 2 * STAGES;   // [2] int8 operands ready
  uint64_t* empty8 = full8 + 2;          // [2] int8 operands consumed by the MMA
  uint64_t* tfull = empty8 + 2;          // [2] TMEM partial ready
  uint64_t* tempty = tfull + 2;          // [2] TMEM partial drained
  uint64_t* final_bar = tempty + 2;      // teardown: all MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tail_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const WaitPolicy wp{args.limit_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::NUM_UNPACK_WARPS + Cfg::NUM_DRAIN_WARPS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full8[b], Cfg::NUM_UNPACK_WARPS);
      mbar_init(&empty8[b], 1);
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], Cfg::NUM_DRAIN_WARPS);
    }
    mbar_init(final_bar, 1);
    *abort_flag = 0;
    *tail_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_row);
    prefetch_tensormap(&tm_col);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int units = args.tiles_r * args.tiles_c * args.splits;
  uint32_t issued = 0;  // producer: loads issued (for the teardown drain)

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (Cfg::REALLOC) regs_dealloc<Cfg::REGS_LOW>();
    if (lane == 0 && !(args.debug_flags & 1)) {
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const int split = u % args.splits;
        const int tile = u / args.splits;
        const int tr = tile % args.tiles_r, tc = tile / args.tiles_r;
        const int g0 = split * args.groups_per_split;
        const int g1 = min(args.G, g0 + args.groups_per_split);
        const int c0 = tc * BN;
        const uint32_t cs_bytes = static_cast<uint32_t>(min(BN, args.ld_c - c0)) * 4u;
        for (int g = g0; g < g1; ++g, ++it) {
          const int s = it % STAGES;
          if (!wait_one(&empty[s], ((it / STAGES) & 1) ^ 1, wp)) { ok = false; break; }
          uint8_t* st = stage_base + s * Cfg::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[s], Cfg::A_PACK + Cfg::B_PACK + cs_bytes);
          tma_load_2d(st, &tm_row, &full[s], g * 32, tr * BM);
          tma_load_2d(st + Cfg::A_PACK, &tm_col, &full[s], g * 32, c0);
          bulk_load(st + Cfg::A_PACK + Cfg::B_PACK, args.scales_c + static_cast<size_t>(g) * args.ld_c + c0,
                    cs_bytes, &full[s]);
          issued = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (Cfg::REALLOC) regs_dealloc<Cfg::REGS_LOW>();
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_i8(BM, BN);
      uint32_t it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
        const int split = u % args.splits;
        const int g0 = split * args.groups_per_split;
        const int g1 = min(args.G, g0 + args.groups_per_split);
        for (int g = g0; g < g1; ++g, ++it) {
          const int b = it & 1;
          const uint32_t ph = (it >> 1) & 1;
          if (!wait_one(&full8[b], ph, wp)) { ok = false; break; }
          // DRAIN 2: the drain pre-fills both buffers once and so completes phase 0 itself
          if (!wait_one(&tempty[b], Cfg::DRAIN == 2 ? ph : ph ^ 1, wp)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(i8_base + b * Cfg::I8_BYTES);
          const uint32_t b_addr = a_addr + Cfg::A_I8;
          const uint32_t d = tmem_base + static_cast<uint32_t>(b * BN);
          mma_i8(d, smem_desc_kmajor(a_addr, kLBO, kSBO), smem_desc_kmajor(b_addr, kLBO, kSBO), idesc,
                 Cfg::DRAIN == 2 ? 1u : 0u);
          mma_i8(d, smem_desc_kmajor(a_addr + 2 * kLBO, kLBO, kSBO), smem_desc_kmajor(b_addr + 2 * kLBO, kLBO, kSBO),
                 idesc, 1u);
          mma_commit(&empty8[b]);
          mma_commit(&tfull[b]);
        }
      }
    }
  } else if (warp < 2 + Cfg::NUM_UNPACK_WARPS) {
    // ------------------------------------------------------------ unpack
    if (Cfg::REALLOC) regs_dealloc<Cfg::REGS_LOW>();
    const int ut = (warp - 2) * 32 + lane;
    constexpr int NT = 32 * Cfg::NUM_UNPACK_WARPS;
    uint32_t it = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
      const int split = u % args.splits;
      const int g0 = split * args.groups_per_split;
      const int g1 = min(args.G, g0 + args.groups_per_split);
      for (int g = g0; g < g1; ++g, ++it) {
        const int s = it % STAGES;
        const int b = it & 1;
        if (!wait_warp(&full[s], (it / STAGES) & 1, wp)) { ok = false; break; }
        if (!wait_warp(&empty8[b], ((it >> 1) & 1) ^ 1, wp)) { ok = false; break; }
        const uint8_t* st = stage_base + s * Cfg::STAGE_BYTES;
        uint8_t* dst = i8_base + b * Cfg::I8_BYTES;
        for (int t = ut; t < 2 * BM; t += NT) unpack_task(st, dst, t);
        for (int t = ut; t < 2 * BN; t += NT) unpack_task(st + Cfg::A_PACK, dst + Cfg::A_I8, t);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&full8[b]);
          mbar_arrive(&empty[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ drain + epilogue
    if (Cfg::REALLOC) regs_alloc<Cfg::REGS_HIGH>();
    const int dw = warp - (2 + Cfg::NUM_UNPACK_WARPS);
    const int q = warp & 3;            // TMEM lane quadrant
    const int h = dw >> 2;             // column slice
    const int row_local = q * 32 + lane;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t it = 0;
    bool ok = true;
    if (Cfg::DRAIN == 2) {
      // pre-fill this warp's lanes/columns of both TMEM buffers with the pattern
#pragma unroll
      for (int b = 0; b < 2; ++b)
#pragma unroll
        for (int c = 0; c < CW / 16; ++c) tmem_st16_fill(t_lane + static_cast<uint32_t>(b * BN + h * CW + c * 16), kMagicBits);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[0]);
        mbar_arrive(&tempty[1]);
      }
    }
    for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
      const int split = u % args.splits;
      const int tile = u / args.splits;
      const int tr = tile % args.tiles_r, tc = tile / args.tiles_r;
      const int g0 = split * args.groups_per_split;
      const int g1 = min(args.G, g0 + args.groups_per_split);
      const int row = tr * BM + row_local;
      const bool row_ok = row < args.rows_r;
      float acc[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = 0.f;
      float s_next = row_ok ? __ldg(args.scales_r + static_cast<size_t>(g0) * args.ld_r + row) : 0.f;
      for (int g = g0; g < g1; ++g, ++it) {
        const int s = it % STAGES;
        const int b = it & 1;
        const float s_row = s_next * (1.0f / 256.0f);
        if (g + 1 < g1 && row_ok) s_next = __ldg(args.scales_r + static_cast<size_t>(g + 1) * args.ld_r + row);
        if (!wait_warp(&tfull[b], (it >> 1) & 1, wp)) { ok = false; break; }
        if (!wait_warp(&full[s], (it / STAGES) & 1, wp)) { ok = false; break; }
        tc_fence_after();
        const float* cs = reinterpret_cast<const float*>(stage_base + s * Cfg::STAGE_BYTES + Cfg::A_PACK +
                                                         Cfg::B_PACK) + h * CW;
#pragma unroll
        for (int c = 0; c < CW / 16; ++c) {
          uint32_t v[16];
          const uint32_t taddr = t_lane + static_cast<uint32_t>(b * BN + h * CW + c * 16);
          tmem_ld16(taddr, v);
          tmem_ld_wait();
          if (Cfg::DRAIN == 2) tmem_st16_fill(taddr, kMagicBits);
#pragma unroll
          for (int j4 = 0; j4 < 4; ++j4) {
            const float4 sc = *reinterpret_cast<const float4*>(cs + c * 16 + j4 * 4);
            const float scv[4] = {sc.x, sc.y, sc.z, sc.w};
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int j = j4 * 4 + e;
              float& a0 = acc[c * 16 + j];
              float& a1 = acc[c * 16 + j + 1];
              if (Cfg::DRAIN == 0) {
                a0 = fmaf(s_row, scv[e] * __int2float_rn(static_cast<int>(v[j])), a0);
                a1 = fmaf(s_row, scv[e + 1] * __int2float_rn(static_cast<int>(v[j + 1])), a1);
              } else {
                float p0, p1, t0, t1;
                if (Cfg::DRAIN == 1) {
                  p0 = __int2float_rn(static_cast<int>(v[j]));
                  p1 = __int2float_rn(static_cast<int>(v[j + 1]));
                } else {
                  fadd2(p0, p1, __uint_as_float(v[j]), __uint_as_float(v[j + 1]), -kMagic, -kMagic);
                }
                fmul2(t0, t1, p0, p1, scv[e], scv[e + 1]);
                ffma2(a0, a1, s_row, s_row, t0, t1, a0, a1);
              }
            }
          }
        }
        if (Cfg::DRAIN == 2) tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&tempty[b]);
          mbar_arrive(&empty[s]);
        }
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      const int col0 = tc * BN + h * CW;
      if (args.splits > 1) {
        // Split-K: every drain warp owns a 32-row x CW-column sub-tile.  It
        // writes its fp32 partial, and the warp that arrives last for that
        // sub-tile sums all splits in split order (deterministic), runs the
        // epilogue and re-zeroes the counter.  No cross-warp barrier is used.
        const size_t tile_base = static_cast<size_t>(tile) * args.splits;
        float* part = args.ws_partials + ((tile_base + split) * BN + h * CW) * BM + row_local;
#pragma unroll
        for (int j = 0; j < CW; ++j) part[static_cast<size_t>(j) * BM] = acc[j];
        __threadfence();
        __syncwarp();
        unsigned* counter = args.ws_counters + static_cast<size_t>(tile) * Cfg::NUM_DRAIN_WARPS + dw;
        int last = 0;
        if (lane == 0) last = (atomicAdd(counter, 1u) == static_cast<unsigned>(args.splits - 1)) ? 1 : 0;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
#pragma unroll
        for (int j = 0; j < CW; ++j) acc[j] = 0.f;
        for (int sp = 0; sp < args.splits; ++sp) {
          const float* p = args.ws_partials + ((tile_base + sp) * BN + h * CW) * BM + row_local;
#pragma unroll
          for (int j = 0; j < CW; ++j) acc[j] += __ldcg(p + static_cast<size_t>(j) * BM);
        }
        if (lane == 0) *counter = 0u;
      }
      if (!row_ok) continue;
      if (!Cfg::SWAP) {
        // rows are tokens m, columns are output features n
        const int m = row;
        for (int i = 0; i < args.r; ++i) {
          const float um = __ldg(args.U + static_cast<size_t>(m) * args.r + i);
          const __nv_bfloat16* l2 = args.L2 + static_cast<size_t>(i) * args.N;
#pragma unroll
          for (int j8 = 0; j8 < CW / 8; ++j8) {
            const int n = col0 + j8 * 8;
            if (n < args.N) {
              float l[8];
              bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(l2 + n)), l);
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[j8 * 8 + e] = fmaf(um, l[e], acc[j8 * 8 + e]);
            }
          }
        }
#pragma unroll
        for (int j8 = 0; j8 < CW / 8; ++j8) {
          const int n = col0 + j8 * 8;
          if (n < args.N) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = acc[j8 * 8 + e];
            if (args.bias) {
              float bb[8];
              bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(args.bias + n)), bb);
#pragma unroll
              for (int e = 0; e < 8; ++e) y[e] += bb[e];
            }
            const size_t off = static_cast<size_t>(m) * args.N + n;
            if (args.out_f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(args.Y) + off);
              dst[0] = make_float4(y[0], y[1], y[2], y[3]);
              dst[1] = make_float4(y[4], y[5], y[6], y[7]);
            } else {
              uint4 o;
              __nv_bfloat162* ob = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
              for (int e = 0; e < 4; ++e) ob[e] = __floats2bfloat162_rn(y[2 * e], y[2 * e + 1]);
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(args.Y) + off) = o;
            }
          }
        }
      } else {
        // rows are output features n, columns are tokens m
        const int n = row;
        const float bn = args.bias ? __bfloat162float(args.bias[n]) : 0.f;
        for (int i = 0; i < args.r; ++i) {
          const float l2 = __bfloat162float(args.L2[static_cast<size_t>(i) * args.N + n]);
#pragma unroll
          for (int j = 0; j < CW; ++j) {
            const int m = col0 + j;
            if (m < args.M) acc[j] = fmaf(__ldg(args.U + static_cast<size_t>(m) * args.r + i), l2, acc[j]);
          }
        }
#pragma unroll
        for (int j = 0; j < CW; ++j) {
          const int m = col0 + j;
          if (m < args.M) {
            const float y = acc[j] + bn;
            const size_t off = static_cast<size_t>(m) * args.N + n;
            if (args.out_f32) static_cast<float*>(args.Y)[off] = y;
            else static_cast<__nv_bfloat16*>(args.Y)[off] = __float2bfloat16_rn(y);
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    const WaitPolicy tail{args.limit_ns, tail_flag};
    if (warp == 0 && lane == 0) {
      // let every load still in flight land before the CTA's shared memory goes away
      const uint32_t first = issued > static_cast<uint32_t>(STAGES) ? issued - STAGES : 0u;
      for (uint32_t i = first; i < issued; ++i) wait_one(&full[i % STAGES], (i / STAGES) & 1, tail);
    }
    if (warp == 1 && lane == 0) {
      mma_commit(final_bar);  // arrives once every MMA issued above has completed
      wait_one(final_bar, 0, tail);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace hsq
