// hsq_fp4.cuh -- the NVFP4 variant of the layer's forward on tcgen05
// block-scaled tensor-core MMAs.
//
// The DiRotQ page (papernotes.org, quantization settings) names, besides INT4
// W4A4 with groups of 64, the 4-bit floating-point setting of Blackwell: the
// standard NVFP4 format, E2M1 values with one FP8 (E4M3) scale per 16 values,
// here with the usual second-level fp32 scale g per tensor.  The layer is the
// same as the INT4 one,
//     Y = gx gw sum_k (ex[m,k] bx[m,k/16]) (ew[n,k] bw[n,k/16]) + U L2 + b,
// with ex, ew the E2M1 codes of X_hat and of the residual R.  Blackwell's
// kind::mxf4nvf4 MMA multiplies the block scales inside the instruction, so one
// accumulator chain runs over the whole of K for a tile and the drain runs once
// per tile (the INT4 kernel instead ends a chain at every 64-wide group).
//
// Tile 128 tokens x 128 outputs, a stage is K = 256 (four K = 64 MMAs):
//   warp 0      TMA producer: both operands (128-byte rows, 128-byte swizzle)
//               and their E4M3 scale atoms (bulk copies) into a STAGES ring
//   warp 1      TMEM allocator and MMA issuer: per stage, tcgen05.cp of the
//               scale atoms into Tensor Memory, then the block-scaled MMAs
//   warps 2..5  epilogue: Y = acc * gx gw + U L2 + b from the tile's TMEM
//               accumulator (two accumulators, so the next tile's MMAs run
//               while this one drains), stored with TMA.
// Persistent: one CTA per SM walks tiles b, b + grid, ...  Every wait is bounded.
#pragma once

#include "hsq_device.cuh"

namespace hsq {

struct Fp4Args {
  const uint8_t* x_sf;   // activation block scales, [tiles_m][KC][512] E4M3 atoms
  const uint8_t* w_sf;   // weight block scales, [tiles_n][KC][512]
  const float* x_gs;     // x_gs[0] = activation tensor scale
  const float* w_gs;     // w_gs[0] = weight tensor scale
  const float* U;        // [M][r]
  const __nv_bfloat16* L2;    // [r][N]
  const __nv_bfloat16* bias;  // [N] or nullptr
  int M, N, KC, r;       // KC: 64-wide K chunks (K rounded up to 64)
  int tiles_m, tiles_n;
  int out_f32;
  uint64_t limit_ns;
};

// Tile 128 tokens x BN outputs; a stage is K = 256 (KCS = 4 chunks of K = 64).
// BN = 256 halves the activation reads per output against BN = 128 (the kernel is
// bound by reading its operands from L2), but its accumulator then fills half of
// Tensor Memory, so there is one (NTM = 1) and the epilogue's reads of it are not
// overlapped with the next tile's MMAs.
template <int BN_, int NTM_, int STAGES_>
struct Fp4Cfg {
  static constexpr int BM = 128, BN = BN_;
  static constexpr int KCS = 4;                        // 64-wide K chunks per stage (128 bytes per row)
  static constexpr int STAGES = STAGES_;
  static constexpr int BATOMS = BN / 128;              // 128-row scale atoms of the B tile
  static constexpr int A_BYTES = BM * 128;             // 16 KB
  static constexpr int B_BYTES = BN * 128;
  static constexpr int SF_ATOM = 512;                  // 128 rows x 4 scales
  static constexpr int SFA_OFF = A_BYTES + B_BYTES;
  static constexpr int SFB_OFF = SFA_OFF + KCS * SF_ATOM;  // [BATOMS][KCS] atoms
  static constexpr int STAGE_BYTES = SFB_OFF + BATOMS * KCS * SF_ATOM;  // a multiple of 1024
  // epilogue: four warps (one per TMEM lane quadrant) for each 128 columns of the tile
  static constexpr int EPI_PARTS = BN / 128;
  static constexpr int NUM_EPI_WARPS = 4 * EPI_PARTS;
  static constexpr int THREADS = 32 * (2 + NUM_EPI_WARPS);
  static constexpr int NTM = NTM_;                     // TMEM accumulators
  static constexpr int SFC = 4 + 4 * BATOMS;           // TMEM scale columns per K = 64 chunk (A, then B)
  static constexpr int SF_COL0 = NTM * BN;             // scale columns follow the accumulators
  static constexpr int SF_COLS = KCS * SFC;            // per stage
  static constexpr int TMEM_COLS = 512;
  static constexpr int YST_BYTES = NUM_EPI_WARPS * 4096;
  // the epilogue's bias and L2 columns of a tile, [1 + 32][BN] bf16 (row 0 the
  // bias, rows 1.. the ranks), two buffers
  static constexpr int LR_ROWS = 33;
  static constexpr int LR_BYTES = LR_ROWS * BN * 2;
  static constexpr int LR_BUFS = NTM;  // a tile's copy is issued LR_BUFS tiles ahead
  static constexpr int NUM_BARS = 2 * STAGES + 2 * NTM + 1 + 2 * LR_BUFS;
  static constexpr int SMEM_BYTES =
      1024 + STAGES * STAGE_BYTES + YST_BYTES + LR_BUFS * LR_BYTES + NUM_BARS * 8 + 64;
  static_assert(BN == 128 || BN == 256, "B tile");
  static_assert(STAGE_BYTES % 1024 == 0, "128-byte-swizzled tiles start on 1024-byte boundaries");
  static_assert(SF_COL0 + 2 * SF_COLS <= TMEM_COLS, "TMEM");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    fp4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                    const __grid_constant__ CUtensorMap tm_y, const Fp4Args args) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, STAGES = Cfg::STAGES, KCS = Cfg::KCS, NTM = Cfg::NTM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* ystage = smem + STAGES * Cfg::STAGE_BYTES;
  __nv_bfloat16* lrs = reinterpret_cast<__nv_bfloat16*>(ystage + Cfg::YST_BYTES);  // [2][LR_ROWS][BN]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ystage + Cfg::YST_BYTES + Cfg::LR_BUFS * Cfg::LR_BYTES);
  uint64_t* full = bars;                 // [STAGES] stage landed
  uint64_t* empty = bars + STAGES;       // [STAGES] stage consumed by the MMAs
  uint64_t* tfull = empty + STAGES;      // [NTM] accumulator complete
  uint64_t* tempty = tfull + NTM;        // [NTM] accumulator drained
  uint64_t* final_bar = tempty + NTM;    // teardown: all MMAs done
  uint64_t* lrfull = final_bar + 1;      // [LR_BUFS] a tile's bias and L2 columns landed
  uint64_t* lrempty = lrfull + Cfg::LR_BUFS;  // [LR_BUFS] ... and read by every epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tail_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const WaitPolicy wp{args.limit_ns, abort_flag};
  const int tiles = args.tiles_m * args.tiles_n;
  const int kstages = (args.KC + KCS - 1) / KCS;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < NTM; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], Cfg::NUM_EPI_WARPS);
    }
    mbar_init(final_bar, 1);
    for (int b = 0; b < Cfg::LR_BUFS; ++b) {
      mbar_init(&lrfull[b], 1);
      mbar_init(&lrempty[b], Cfg::NUM_EPI_WARPS);
    }
    *abort_flag = 0;
    *tail_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dep_wait();  // codes, scales, U come from the preceding kernels

  uint32_t issued = 0;  // producer: stages issued (for the teardown)
  uint32_t lr_issued[2] = {0u, 0u}, lr_done[2] = {0u, 0u};  // epilogue: bias/L2 copies issued / waited per buffer

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int tm = t % args.tiles_m, tn = t / args.tiles_m;
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % STAGES;
          if (!wait_one(&empty[s], ((it / STAGES) & 1) ^ 1, wp)) { ok = false; break; }
          const int kc0 = ks * KCS;
          const int nc = min(KCS, args.KC - kc0);
          uint8_t* st = stage_base + s * Cfg::STAGE_BYTES;
          // the boxes are counted whole, rows and K beyond the tensors included (zero-filled)
          const int batoms = min(Cfg::BATOMS, (args.N - tn * BN + 127) / 128);  // atoms holding weight rows
          mbar_arrive_expect_tx(&full[s], Cfg::A_BYTES + Cfg::B_BYTES + (1 + batoms) * nc * Cfg::SF_ATOM);
          tma_load_2d(st, &tm_a, &full[s], kc0 * 32, tm * BM);
          tma_load_2d(st + Cfg::A_BYTES, &tm_b, &full[s], kc0 * 32, tn * BN);
          bulk_load(st + Cfg::SFA_OFF, args.x_sf + (static_cast<size_t>(tm) * args.KC + kc0) * Cfg::SF_ATOM,
                    nc * Cfg::SF_ATOM, &full[s]);
          // (an atom past the last weight row is not loaded: its scales only reach
          // accumulator columns past N, which are never stored)
          for (int j = 0; j < batoms; ++j)
              bulk_load(st + Cfg::SFB_OFF + j * KCS * Cfg::SF_ATOM,
                        args.w_sf + (static_cast<size_t>(tn * Cfg::BATOMS + j) * args.KC + kc0) * Cfg::SF_ATOM,
                        nc * Cfg::SF_ATOM, &full[s]);
          issued = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_fp4_block16(BM, BN);
      uint32_t it = 0, nt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++nt) {
        const int tb = nt % NTM;
        if (!wait_one(&tempty[tb], ((nt / NTM) & 1) ^ 1, wp)) break;
        const uint32_t d = tmem_base + static_cast<uint32_t>(tb * BN);
        for (int ks = 0; ks < kstages; ++ks, ++it) {
          const int s = it % STAGES;
          if (!wait_one(&full[s], (it / STAGES) & 1, wp)) { ok = false; break; }
          tc_fence_after();
          const int nc = min(KCS, args.KC - ks * KCS);
          const uint32_t st = smem_u32(stage_base + s * Cfg::STAGE_BYTES);
          // chunk i's scales: A at columns SFC i .. +3, B's atoms j at SFC i + 4 + 4 j .. +3
          // (B row n at column SFC i + 4 + n / 32)
          const uint32_t sfc = tmem_base + static_cast<uint32_t>(Cfg::SF_COL0 + (it & 1) * Cfg::SF_COLS);
          for (int i = 0; i < nc; ++i) {
            tmem_cp_sf_atom(sfc + Cfg::SFC * i, smem_desc_kmajor(st + Cfg::SFA_OFF + i * Cfg::SF_ATOM, 128, 128));
#pragma unroll
            for (int j = 0; j < Cfg::BATOMS; ++j)
              tmem_cp_sf_atom(sfc + Cfg::SFC * i + 4 + 4 * j,
                              smem_desc_kmajor(st + Cfg::SFB_OFF + (j * KCS + i) * Cfg::SF_ATOM, 128, 128));
          }
          for (int i = 0; i < nc; ++i) {
            // chunk i is 32 bytes into each 128-byte swizzled row
            mma_fp4_block16(d, smem_desc_kmajor_sw128(st + 32 * i, 1024),
                            smem_desc_kmajor_sw128(st + Cfg::A_BYTES + 32 * i, 1024), idesc, sfc + Cfg::SFC * i,
                            sfc + Cfg::SFC * i + 4, (ks > 0 || i > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&tfull[tb]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant of this warp
    const int ew = warp - 2;
    const int part = ew >> 2;  // the tile's 128-column part this warp drains
    const uint32_t t_q = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const float gg = __fmul_rn(__ldg(args.x_gs), __ldg(args.w_gs));
    uint8_t* stg = ystage + ew * 4096;
    // A tile's bias and L2 columns are bulk-copied into shared memory LR_BUFS
    // tiles ahead (buffer nt % LR_BUFS), so the epilogue's math reads no global memory.
    const bool lr_issuer = ew == 0 && lane == 0;
    auto issue_lr = [&](int t, int b) {
      const int n0 = (t / args.tiles_m) * BN;
      const uint32_t cb = static_cast<uint32_t>(min(BN, args.N - n0)) * 2u;  // N % 8 == 0: a multiple of 16
      mbar_arrive_expect_tx(&lrfull[b], cb * static_cast<uint32_t>(args.r + (args.bias ? 1 : 0)));
      __nv_bfloat16* dst = lrs + b * Cfg::LR_ROWS * BN;
      if (args.bias) bulk_load(dst, args.bias + n0, cb, &lrfull[b]);
      for (int j = 0; j < args.r; ++j)
        bulk_load(dst + (1 + j) * BN, args.L2 + static_cast<size_t>(j) * args.N + n0, cb, &lrfull[b]);
      ++lr_issued[b];
    };
    if (lr_issuer)
      for (int b = 0; b < Cfg::LR_BUFS; ++b)
        if (blockIdx.x + b * static_cast<int>(gridDim.x) < tiles) issue_lr(blockIdx.x + b * gridDim.x, b);
    uint32_t nt = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++nt) {
      const int tm = t % args.tiles_m, tn = t / args.tiles_m;
      const int tb = nt % NTM;
      if (!wait_warp(&tfull[tb], (nt / NTM) & 1, wp)) break;
      const int lb = nt % Cfg::LR_BUFS;
      if (!wait_warp(&lrfull[lb], (nt / Cfg::LR_BUFS) & 1, wp)) break;
      ++lr_done[lb];
      const __nv_bfloat16* lrb = lrs + lb * Cfg::LR_ROWS * BN;
      tc_fence_after();
      const int m = tm * BM + q * 32 + lane;
      const int y0 = tm * BM + q * 32;
      // this warp's 128 columns (thread = row); once every epilogue warp has its
      // part in registers the accumulator is free for the next tile's MMAs
      {
        const int n0 = tn * BN + part * 128;
        uint32_t v[8][16];
#pragma unroll
        for (int c = 0; c < 8; ++c) tmem_ld16(t_q + static_cast<uint32_t>(tb * BN + part * 128 + 16 * c), v[c]);
        // wait for the loads; every destination register passes through a wait, so
        // that no read of them is scheduled before it (later waits return at once)
#pragma unroll
        for (int c = 0; c < 8; c += 2) tmem_ld_wait(v[c], v[c + 1]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[tb]);
        if (n0 < args.N) {  // warp-uniform
        // Y = acc * gx gw + b, then + U[m][j] L2[j][:] rank by rank, in place in
        // the accumulator registers (an 8-column block is all in or all out: N % 8 == 0)
        // (the columns of the shared bias / L2 rows past N hold stale values: they
        // only reach outputs past N, which are never stored)
        auto vf = [&](int c) -> float& { return *reinterpret_cast<float*>(&v[c >> 4][c & 15]); };
        const __nv_bfloat16* lrp = lrb + part * 128;
#pragma unroll
        for (int c8 = 0; c8 < 16; ++c8) {
          float b[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) b[e] = 0.f;
          if (args.bias) bf16x8_to_f32(*reinterpret_cast<const uint4*>(lrp + 8 * c8), b);
#pragma unroll
          for (int e = 0; e < 8; ++e) vf(8 * c8 + e) = __fadd_rn(__fmul_rn(vf(8 * c8 + e), gg), b[e]);
        }
#pragma unroll 1
        for (int j = 0; j < args.r; ++j) {
          const float uj = m < args.M ? __ldg(args.U + static_cast<size_t>(m) * args.r + j) : 0.f;
          const __nv_bfloat16* l2 = lrp + (1 + j) * BN;
#pragma unroll
          for (int c8 = 0; c8 < 16; ++c8) {
            float l[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(l2 + 8 * c8), l);
#pragma unroll
            for (int e = 0; e < 8; ++e) vf(8 * c8 + e) = __fmaf_rn(uj, l[e], vf(8 * c8 + e));
          }
        }
        auto y = [&](int c) { return __uint_as_float(v[c >> 4][c & 15]); };
        // store: 32 rows x 128 bytes per TMA box, 128-byte swizzled staging
        if (!args.out_f32) {
#pragma unroll
          for (int pz = 0; pz < 2; ++pz) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              uint4 w;
              __nv_bfloat162* wb = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                wb[e] = __floats2bfloat162_rn(y(64 * pz + 8 * c + 2 * e), y(64 * pz + 8 * c + 2 * e + 1));
              *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) = w;
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && n0 + 64 * pz < args.N && y0 < args.M) {
              tma_store_2d(&tm_y, stg, n0 + 64 * pz, y0);
              bulk_commit_group();
            }
          }
        } else {
#pragma unroll
          for (int pz = 0; pz < 4; ++pz) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<float4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                  make_float4(y(32 * pz + 4 * c), y(32 * pz + 4 * c + 1), y(32 * pz + 4 * c + 2),
                              y(32 * pz + 4 * c + 3));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && n0 + 32 * pz < args.N && y0 < args.M) {
              tma_store_2d(&tm_y, stg, n0 + 32 * pz, y0);
              bulk_commit_group();
            }
          }
        }
        }  // n0 < N
      }
      // this warp is done with the tile's bias / L2 buffer; once all are, it is
      // refilled for the tile LR_BUFS ahead
      __syncwarp();
      if (lane == 0) mbar_arrive(&lrempty[lb]);
      if (lr_issuer && t + Cfg::LR_BUFS * static_cast<int>(gridDim.x) < tiles) {
        if (!wait_one(&lrempty[lb], (nt / Cfg::LR_BUFS) & 1, wp)) break;
        issue_lr(t + Cfg::LR_BUFS * gridDim.x, lb);
      }
    }
    if (lane == 0) bulk_wait_all();
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
    if (warp == 2 && lane == 0) {
      // and the bias / L2 copies not yet waited for
      for (int b = 0; b < Cfg::LR_BUFS; ++b)
        if (lr_issued[b] > lr_done[b]) wait_one(&lrfull[b], (lr_issued[b] - 1) & 1, tail);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace hsq
