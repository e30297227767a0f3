// hsq_gemm.cuh -- packed INT4 x INT4 GEMM on tcgen05 with a per-group fp32
// rescale and a fused low-rank + bias epilogue.
//
// Computes (Deflating the Hessian, Abstract: 4-bit residual product plus the
// high-precision low-rank branch)
//     Y[m,n] = sum_g sx[g][m] sw[g][n] P_g[m,n] + sum_j U[m,j] L2[j,n] + b[n],
//     P_g[m,n] = sum_{k in group g} qx[m,k] qw[n,k]   (exact integers)
//
// Blackwell has no INT4 tensor-core mode.  Each 64-wide block of codes is fed
// to the tensor cores in an 8-bit form whose products and 64-term sums are
// exact, two K = 32 MMAs per block into a group's own Tensor Memory partial;
// drain warps read that partial with tcgen05.ld and fold it into fp32 register
// accumulators with the group's two scales.  The 8-bit forms:
//   kind::i8      int8 16*q (decode tiles): the MMA sums 256*q_x*q_w in int32,
//                 the drain folds 1/256 into the row scale (a power of two);
//   kind::f8f6f4  E4M3 subnormals q*2^-9 (tokens x outputs tiles): every product
//                 and partial is exact in fp32, so the drain needs no int->fp32
//                 conversion and folds 2^18 into the row scale instead.
// Either way the group partial is the same number.
//
// Operands are named by their role in the MMA:
//   "row" operand  -> MMA A, 128 rows per tile, one TMEM lane per row;
//   "col" operand  -> MMA B, BN rows per tile, one TMEM column per row.
// For large M the row operand is the activations (tile 128 tokens x BN=256
// outputs); for decode-sized M the roles swap (128 weight rows x BN tokens), so
// the MMA's M=128 side is always filled.
//
// Where the 8-bit operands come from (GemmCfg):
//   packed codes staged by TMA and widened in shared memory by unpack warps
//     (decode tiles; tokens x outputs tiles for up to 256 tokens): a packed
//     byte holds two 4-bit two's-complement codes; masking a code into the
//     HIGH nibble of a byte gives 16*q (one AND or shift+AND per four codes),
//     or the E4M3 byte sign<<7 | |q|.  The even/odd split permutes K inside a
//     block identically for both operands, which leaves every P_g unchanged;
//   pre-expanded (PRE; more tokens): expand_e4m3_kernel writes both code
//     matrices once per call as MMA-ready E4M3 tiles, and a stage is two bulk
//     copies.
// The low-rank branch U L2 + b enters the same accumulators as bf16 MMA steps
// ahead of a tile's first group (tokens x outputs tiles) or is added by the
// drain at the tile's start (decode tiles).
//
// Pipeline (one CTA per SM, persistent over work units).  One pipeline step
// ("stage") carries GPS consecutive scale groups, so that the fixed cost of each
// hand-off is shared by GPS groups:
//   warp 0      TMA producer: row/col tiles + the row and col scales of each
//               group, into a STAGES-deep ring (scales in a deeper ring of their own)
//   warp 1      TMEM allocator and MMA issuer (one elected lane)
//   warps 2..   unpack (packed -> 8-bit K-major layout, NI8 buffers) or, with
//               PRE, the builders of the low-rank step's operands
//   last warps  drain / epilogue; warp w reads TMEM lanes 32*(w%4)..+31; NTM
//               TMEM buffers of GPS x BN columns
// Work is whole tiles per CTA, or stream-K runs of stages with a deterministic
// last-arriver reduction when the tiles do not fill the SMs.
#pragma once

#include "hsq_device.cuh"
#include "hsq_quant.cuh"

#ifndef HSQ_ONE_PHASE
#define HSQ_ONE_PHASE 0
#endif

// Drain: hand a TMEM partial buffer back to the MMA warp right after its last
// load (1) or after the stage's math (0).
#ifndef HSQ_EARLY_RELEASE
#define HSQ_EARLY_RELEASE 0
#endif

// Registers per thread left to the producer / MMA / helper warpgroups of
// blocks of up to 512 threads (the rest go to the drain warpgroups).
#ifndef HSQ_REGS_LOW_SMALL
#define HSQ_REGS_LOW_SMALL 64
#endif

namespace hsq {

// Canonical no-swizzle K-major layout of one operand and one 64-wide group:
// core matrix (row/8, kc) (kc = 16-byte K chunk 0..3) at (row/8)*SBO + kc*LBO
// bytes, its 8 rows 16 bytes apart; the second K=32 MMA starts 2*LBO bytes in.
// LBO = 160 (not 128) staggers the four K chunks of a row block across shared-
// memory banks so the unpack's 16-byte stores are conflict free; SBO = 3*LBO+128.
constexpr uint32_t kLBO = 160;
constexpr uint32_t kSBO = 3 * kLBO + 128;

// Bytes of one group's int8 operand with `rows` rows, padded so that
// consecutive groups start 16 bytes apart modulo 128 (another bank stagger).
__host__ __device__ constexpr int i8_group_stride(int rows) {
  return (rows / 8) * static_cast<int>(kSBO) + ((16 - ((rows / 8) * static_cast<int>(kSBO)) % 128) + 128) % 128;
}

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
  int tiles_r, tiles_c;   // output tiles along the row / col operand
  int stages_per_tile;    // ceil(G / GPS)
  int stream_len;         // 0: whole tiles per CTA; else stages per CTA (stream-K)
  float* ws_partials;     // stream-K partial tiles, [CTA][2][BN][128]
  unsigned* ws_counters;  // stream-K arrival counters per (tile, drain warp), zero between calls
  uint64_t limit_ns;      // wait limit
  int debug_flags;        // 1: producer issues nothing (forces the timeout path)
  int lr_mma;             // low-rank steps that start a tile's first unit (kernels with LR_MMA; 0: none)
  const uint8_t* xe;      // pre-expanded row operand (kernels with PRE): [G][rg_r][4][8][16] E4M3
  const uint8_t* we;      // pre-expanded col operand: [G][rg_c][4][8][16]
  int rg_r, rg_c;         // 8-row groups of each (rows padded to whole tiles)
  // Kernels with FUSED (decode tiles): the activation step runs inside the
  // kernel.  Its input, and scratch for its codes [M][Kp/2] (which tm_col maps),
  // its scales [G][ld_c] (= scales_c), the per-chunk U partials [M][nchunks][r],
  // one copy of U per CTA [grid][M][r] and the grid barrier's two counters; the
  // stream-K counters (fx_zero_words words) are cleared before the barrier.
  const __nv_bfloat16* fx_X;   // [M][fx_K]
  const float* fx_s;           // [fx_K]
  const __nv_bfloat16* fx_L1;  // [fx_K][r]
  int fx_K, fx_Kp, fx_group;
  uint8_t* fx_codes;
  float* fx_scales;
  float* fx_upart;
  float* fx_U;
  unsigned* fx_bar;
  int fx_zero_words;
};

template <int BN_, int DH_, int STAGES_, bool SWAP_, int GPS_, int NI8_, int NTM_, int UNPACK_WARPS_ = 6,
          int SSLOTS_ = STAGES_ + 4, bool F8_ = false, int PIPE_ = -1, bool PRE_ = false, int CHB_ = 2,
          int BPG_ = 1, bool PAIR_ = false, bool FUSED_ = false, bool LRFAST_ = false>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int DH = DH_;               // column slices handled by separate drain warps
  static constexpr int CW = BN / DH;           // columns per drain thread
  static constexpr int STAGES = STAGES_;
  static constexpr bool SWAP = SWAP_;
  static constexpr int GPS = GPS_;             // scale groups per pipeline stage
  // 64-wide K blocks per scale group: 1 for groups of 64, 2 for groups of 128.
  // Codes move and multiply in 64-blocks (a block is two K = 32 MMAs); a group's
  // blocks accumulate into one TMEM partial, which the drain rescales once.
  static constexpr int BPG = BPG_;
  static constexpr int BPS = GPS * BPG;        // 64-blocks per stage
  static constexpr int NI8 = NI8_;             // int8 operand buffers
  static constexpr int NTM = NTM_;             // TMEM partial buffers
  static constexpr int SSLOTS = SSLOTS_;       // scale ring slots (released by the drain)
  // Operand encoding of the unpacked codes.  false: int8 16*q, kind::i8, int32
  // group partials in TMEM (converted to fp32 by the drain).  true: E4M3
  // subnormals q * 2^-9, kind::f8f6f4, fp32 group partials in TMEM; every
  // product and every partial sum (|P| <= 64 * 49) is exact in both, so both
  // give the same per-group partial P_g.
  static constexpr bool F8 = F8_;
  // Pre-expanded operands (tokens x outputs tiles): both code matrices are
  // expanded once per call (expand_e4m3_kernel) into E4M3 tiles laid out the
  // way the MMA reads them, so a stage is two contiguous bulk copies and no
  // warp unpacks in the main loop; the NUM_UNPACK_WARPS warps then only build
  // the low-rank step's operands.
  static constexpr bool PRE = PRE_;
  static constexpr int E8_SBO = 512;  // pre-expanded tile: bytes per 8-row group (4 K-chunks of 8 rows x 16 B)
  // CTA pairs (pre-expanded tokens x outputs tiles only): the two CTAs of a
  // cluster share one tile of 2 x 128 tokens x BN outputs; the even CTA issues
  // cta_group::2 MMAs that read each CTA's 128 token rows and BN/2 output rows
  // from that CTA's own shared memory and leave each CTA's 128 x BN partial in
  // its own Tensor Memory.  Per CTA and step the operand bytes drop from
  // (128 + BN) to (128 + BN/2) rows' worth, the drain work stays the same.
  static constexpr bool PAIR = PAIR_;
  // The activation step inside the kernel (decode tiles; launched cooperatively):
  // see fused_act_phase.
  static constexpr bool FUSED = FUSED_;
  static_assert(!FUSED || (SWAP && !PRE && !PAIR), "fused activation step: decode tiles");
  static constexpr int PM = PAIR ? 2 : 1;      // CTAs per tile
  static constexpr int TILE_M = BM * PM;       // tokens per tile
  static constexpr int B_ROWS = BN / PM;       // col-operand rows held by one CTA
  static constexpr int A_E8_BLK = BM / 8 * E8_SBO;  // one 64-block of a tile
  static constexpr int B_E8_BLK = B_ROWS / 8 * E8_SBO;
  static constexpr int A_E8 = BPG * A_E8_BLK;
  static constexpr int B_E8 = BPG * B_E8_BLK;
  static constexpr int NUM_UNPACK_WARPS = UNPACK_WARPS_;
  static constexpr int NUM_DRAIN_WARPS = 4 * DH;
  static constexpr int THREADS = 32 * (2 + NUM_UNPACK_WARPS + NUM_DRAIN_WARPS);
  // Register split (setmaxnreg): producer/MMA/unpack warpgroups give registers
  // to the drain warpgroups, which hold CW fp32 accumulators per thread.
  // setmaxnreg.inc draws only on the registers the block was launched with
  // (THREADS x LAUNCH_REGS, LAUNCH_REGS being the __launch_bounds__ cap that
  // ptxas allocates for kernels that reallocate), so the split is sized
  // against that total; the host checks the kernel's actual register count
  // against LAUNCH_REGS before the first launch.
  static constexpr bool REALLOC = CW >= 128 || THREADS >= 768;
  static constexpr int LAUNCH_REGS = ((65536 / THREADS) / 8 * 8) > 255 ? 248 : (65536 / THREADS) / 8 * 8;
  static constexpr int LOW_THREADS = THREADS - 32 * NUM_DRAIN_WARPS;  // producer, MMA, unpack warpgroups
  static constexpr int REGS_LOW = (THREADS <= 512 || LOW_THREADS <= 128) ? HSQ_REGS_LOW_SMALL : 40;
  static constexpr int REGS_HIGH_RAW =
      ((THREADS * LAUNCH_REGS - LOW_THREADS * REGS_LOW) / (32 * NUM_DRAIN_WARPS)) / 8 * 8;
  static constexpr int REGS_HIGH = REGS_HIGH_RAW > 232 ? 232 : REGS_HIGH_RAW;
  static_assert(!REALLOC || LOW_THREADS * REGS_LOW + 32 * NUM_DRAIN_WARPS * REGS_HIGH <= THREADS * LAUNCH_REGS,
                "register split exceeds the block's launch allocation");
  static_assert(LOW_THREADS % 128 == 0, "whole low warpgroups");
  static_assert((2 + NUM_UNPACK_WARPS) % 4 == 0, "drain warps start on a warpgroup boundary");
  static constexpr int A_PACK = BM * 32 * BPS;  // packed bytes per stage (row operand)
  static constexpr int B_PACK = BN * 32 * BPS;  // packed bytes per stage (col operand)
  static constexpr int CS_BYTES = BN * 4;       // col scales of one group
  static constexpr int RS_BYTES = BM * 4;       // row scales of one group
  // Packed stage: row tile then col tile (released by the unpack warps).  The
  // scales of the same stage go to a separate, deeper ring (released by the
  // drain), so a packed stage is free again as soon as it is unpacked.
  static constexpr int STAGE_BYTES = PRE ? ((A_E8 + B_E8 + 1023) / 1024) * 1024 : ((A_PACK + B_PACK + 1023) / 1024) * 1024;
  static constexpr int CS_OFF = 0;                        // scale slot: col scales,
  static constexpr int RS_OFF = GPS * CS_BYTES;           // then row scales
  static constexpr int SSLOT_BYTES = ((RS_OFF + GPS * RS_BYTES + 127) / 128) * 128;
  static constexpr int SA = i8_group_stride(BM);  // int8 bytes of one group, row operand
  static constexpr int SB = i8_group_stride(BN);  // int8 bytes of one group, col operand
  static constexpr int I8_BYTES = ((BPS * (SA + SB) + 1023) / 1024) * 1024;
  static constexpr int NI8E = PRE ? 0 : NI8;   // int8 buffers actually laid out
  static constexpr int TMEM_NEED = NTM * GPS * BN;
  static constexpr int TMEM_COLS = TMEM_NEED <= 32 ? 32 : TMEM_NEED <= 64 ? 64 : TMEM_NEED <= 128 ? 128
                                 : TMEM_NEED <= 256 ? 256 : 512;
  // Low-rank steps (tokens x outputs tiles with E4M3 operands): U L2 + b enters
  // a tile's accumulators as extra pipeline steps ahead of its groups, each a
  // bf16 MMA over an augmented K of LR_K = 32 covering LR_MAX_RANK ranks (hi and
  // lo bf16 parts of U against L2 twice) and, in the first step, ones against
  // the bias.
  static constexpr bool LR_MMA = F8 && !SWAP && GPS == 1;
  static constexpr int LR_K = 32;
  static constexpr int LR_MAX_RANK = (LR_K - 2) / 2;
  static constexpr int LR_SBO = LR_K / 8 * 128;  // bytes per 8-row group (4 K-chunks of 16 B)
  static_assert(!LR_MMA || PRE || (BM + BN) / 8 * LR_SBO <= I8_BYTES, "low-rank operands fit an int8 buffer");
  // with pre-expanded operands the low-rank operands get a buffer of their own
  static constexpr int LR_BYTES = (PRE && LR_MMA) ? (BM + B_ROWS) / 8 * LR_SBO : 0;
  // Build the low-rank steps with build_lr_operands_mlp (the host takes these
  // kernels for ranks above LR_MAX_RANK; a separate instantiation, so that the
  // kernels for lower ranks keep their code unchanged)
  static constexpr bool LRFAST = LRFAST_;
  static_assert(!LRFAST || LR_MMA, "many-rank builder: kernels with low-rank steps");
  static_assert(!PAIR || (PRE && LR_MMA), "CTA pairs: pre-expanded tokens x outputs tiles");
  static_assert(!PAIR || A_E8_BLK == 8192 && B_E8_BLK == 8192, "CTA pairs: one 32 x 256-byte TMA box per block");
  static_assert(!PRE || (F8 && !SWAP && GPS == 1), "pre-expanded operands: E4M3, tokens x outputs, one group a stage");
  // One barrier phase per pipeline step (pre-expanded, single-CTA tiles): the
  // group's scales are copied on the operand stage's barrier, and the MMA's one
  // commit per step both frees the stage and tells the drain the partial is
  // ready.  (Each phase that asynchronous copies or tcgen05.commit complete costs
  // a CTA a fixed ~800 cycles on B200, whatever the bytes; two phases per step
  // instead of four halve that.)  Safe for STAGES >= 3: the drain, which waits on
  // the step's stage barriers, can lag the producer by at most STAGES - 1 + NTM
  // steps, so no stage barrier runs a phase ahead of it.
  static constexpr bool ONE_PHASE = HSQ_ONE_PHASE && PRE && !PAIR;
  static_assert(!ONE_PHASE || (STAGES >= 3 && NTM <= STAGES - 1), "one phase per step: ring depth");
  // Tokens x outputs tiles write Y with TMA stores: each drain warp stages a
  // 32-row x 128-byte box (128-byte swizzle) in its own 4 KB buffer.
  static constexpr bool TMA_STORE = !SWAP;
  static constexpr int YST_BYTES = TMA_STORE ? NUM_DRAIN_WARPS * 4096 : 0;
  static constexpr int NUM_BARS = 2 * STAGES + 2 * SSLOTS + 2 * NI8E + 2 * NTM + 1 + 2;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + YST_BYTES + NI8E * I8_BYTES +
                                    LR_BYTES + SSLOTS * SSLOT_BYTES + NUM_BARS * 8 + 64;
  // unpack tasks (16 packed bytes each) per stage, and per unpack thread
  static constexpr int TASKS = PRE ? 1 : 2 * BPS * (BM + BN);
  static constexpr int TPT = (TASKS + 32 * NUM_UNPACK_WARPS - 1) / (32 * NUM_UNPACK_WARPS);
  // Drain software pipeline (next chunk's TMEM load in flight during the current
  // chunk) when registers allow; with 4 drain warps per scheduler the warps
  // themselves hide the load latency.
  static constexpr bool PIPE = PIPE_ >= 0 ? PIPE_ != 0 : NUM_DRAIN_WARPS <= 8;
  // 8-column blocks per TMEM load of the drain (2 or 4): one load and one wait
  // cover 16 * CHB columns of both half quadrants
  static constexpr int CHB = CHB_;
  static_assert(CHB == 2 || CHB == 4 || CHB == 8, "drain chunk");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N");
  static_assert(CW % (8 * CHB_) == 0, "drain chunks");
  static_assert(TMEM_NEED <= 512, "TMEM");
  static_assert(32 * BPS <= 256, "TMA box width");
  static_assert(!PRE || GPS == 1, "pre-expanded operands: one group a stage");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

// Unpack 16 packed bytes (32 codes) into two 16-byte int8 core-matrix rows
// (even codes, odd codes).
template <bool F8, int HI_OFF = static_cast<int>(kLBO)>
__device__ __forceinline__ void unpack16(const uint4& p, uint8_t* dst) {
  const uint32_t w[4] = {p.x, p.y, p.z, p.w};
  uint4 lo, hi;
  uint32_t* lo_w = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* hi_w = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (!F8) {
      lo_w[i] = (w[i] << 4) & 0xF0F0F0F0u;  // even codes, 16*q as int8
      hi_w[i] = w[i] & 0xF0F0F0F0u;         // odd codes,  16*q as int8
    } else {
      // Two's complement nibbles -> sign-magnitude nibbles (codes are never -8):
      // for a negative nibble 8+j, (8+j) ^ 7 + 1 = 8 | (8-j) = sign | |q|.
      const uint32_t sg = w[i] & 0x88888888u;
      const uint32_t one = sg >> 3;
      const uint32_t sm = (w[i] ^ (sg - one)) + one;
      // E4M3 subnormal bytes: sign in bit 7, |q| in the mantissa, value q * 2^-9
      lo_w[i] = (sm & 0x07070707u) | ((sm << 4) & 0x80808080u);  // even codes
      hi_w[i] = ((sm >> 4) & 0x07070707u) | (sm & 0x80808080u);  // odd codes
    }
  }
  *reinterpret_cast<uint4*>(dst) = lo;
  *reinterpret_cast<uint4*>(dst + HI_OFF) = hi;
}

// Expands a packed INT4 code matrix [rows][Kp/2] into the layout in which the
// pre-expanded large-tile kernel's MMA reads its operands: E4M3 bytes
// [G][rows_pad/8][4 K-chunks][8 rows][16 B], chunk 2h+p of group g holding the
// codes 32h + 2e + p (e = 0..15), the same even/odd order as the shared-memory
// unpack (any order works if both operands share it).  Rows >= rows are zero,
// so whole tiles can be copied.  One thread per (group, 8-row group, half,
// row); the eight threads of a row group write 128 contiguous bytes.
__global__ void __launch_bounds__(256) expand_e4m3_kernel(const uint8_t* __restrict__ codes, int rows, int Kp,
                                                          int rows_pad, uint8_t* __restrict__ out) {
  grid_dep_wait();  // the codes may come from the preceding kernel
  const size_t RG = static_cast<size_t>(rows_pad / 8);
  const size_t total = static_cast<size_t>(Kp / 64) * RG * 16;
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r8 = static_cast<int>(t & 7);
    const int half = static_cast<int>((t >> 3) & 1);
    const size_t gr = t >> 4;  // g * RG + rg
    const int g = static_cast<int>(gr / RG);
    const int row = static_cast<int>(gr % RG) * 8 + r8;
    uint4 p = make_uint4(0u, 0u, 0u, 0u);
    if (row < rows)
      p = __ldg(reinterpret_cast<const uint4*>(codes + static_cast<size_t>(row) * (Kp / 2) + g * 32 + half * 16));
    unpack16<true, 128>(p, out + (gr * 4 + 2 * half) * 128 + r8 * 16);
  }
  // the next kernel (the GEMM, one CTA per SM) may launch once the blocks are done
  if (threadIdx.x == 0) grid_dep_launch();
}

// Operands of the low-rank step for one tile (BM rows r0.. of tokens, B_ROWS
// columns c0.. of outputs: this CTA's share of a pair tile), written as bf16
// K-major core matrices (8 rows x 16 bytes,
// K-chunks 128 bytes apart, 8-row groups LR_SBO apart) into an int8 buffer:
//   A[m][2i] = bf16(U[m][i]),  A[m][2i+1] = bf16(U[m][i] - A[m][2i]),  A[m][LR_K-2] = 1
//   B[n][2i] = B[n][2i+1] = L2[i][n],                               B[n][LR_K-2] = bias[n]
// so that A B^T = U L2 + b with U carried to about 16 significant bits.  Rows
// outside the matrices and unused K are zero.  Threads t0, t0 + nt, ... each
// build whole rows.
template <class Cfg>
__device__ __forceinline__ void build_lr_operands(const GemmArgs& a, int r0, int c0, int chunk, uint8_t* dst, int t0,
                                                  int nt) {
  constexpr int BM = Cfg::BM, BNR = Cfg::B_ROWS, K = Cfg::LR_K;
  for (int t = t0; t < BM + BNR; t += nt) {
    const bool rowop = t < BM;
    const int row = rowop ? t : t - BM;
    const int idx = rowop ? r0 + row : c0 + row;  // token m or output n
    const bool valid = idx < (rowop ? a.M : a.N);
    uint8_t* base = dst + (rowop ? 0 : (BM / 8) * Cfg::LR_SBO) + (row >> 3) * Cfg::LR_SBO + (row & 7) * 16;
#pragma unroll
    for (int c = 0; c < K / 8; ++c) {  // one 16-byte K-chunk: ranks 4c .. 4c+3
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = 0.f;
      if (valid) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = Cfg::LR_MAX_RANK * chunk + 4 * c + e;  // rank
          if (4 * c + e < Cfg::LR_MAX_RANK && i < a.r) {
            if (rowop) {
              const float v = __ldg(a.U + static_cast<size_t>(idx) * a.r + i);
              f[2 * e] = __bfloat162float(__float2bfloat16_rn(v));
              f[2 * e + 1] = v - f[2 * e];  // exact; rounded to bf16 below
            } else {
              const float l = __bfloat162float(a.L2[static_cast<size_t>(i) * a.N + idx]);
              f[2 * e] = l;
              f[2 * e + 1] = l;
            }
          }
        }
        if (c == K / 8 - 1 && chunk == 0)  // element K-2 of the first chunk: ones against the bias
          f[6] = rowop ? 1.f : (a.bias ? __bfloat162float(a.bias[idx]) : 0.f);
      }
      uint4 w;
      __nv_bfloat162* wb = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) wb[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
      *reinterpret_cast<uint4*>(base + c * 128) = w;
    }
  }
}

// The same operands, built for ranks above LR_MAX_RANK (kernels with LRFAST).
// Those take two or three low-rank steps per tile, and every step after the
// first is built while the MMA issuer waits for it (one operand buffer), so
// the build's latency is paid per tile.  Here a row's loads (its ranks of U or
// of L2, and its bias) are all issued before any is used, at clamped in-range
// addresses, so they are in flight together: a step takes a few memory round
// trips instead of one per rank.  The bits are those of build_lr_operands.
template <class Cfg>
__device__ __forceinline__ void build_lr_operands_mlp(const GemmArgs& a, int r0, int c0, int chunk, uint8_t* dst, int t0,
                                                  int nt) {
  constexpr int BM = Cfg::BM, BNR = Cfg::B_ROWS, K = Cfg::LR_K, R = Cfg::LR_MAX_RANK;
  static_assert(K == 32 && R <= 15, "one step: four 16-byte K-chunks of four ranks each, the last with the bias");
  const int rk0 = R * chunk;                               // first rank of this step
  const int nr = a.r > rk0 ? min(R, a.r - rk0) : 0;        // ranks in this step
  auto store_chunk = [](uint8_t* p, const float (&f)[8]) {
    uint4 w;
    __nv_bfloat162* wb = reinterpret_cast<__nv_bfloat162*>(&w);
#pragma unroll
    for (int e = 0; e < 4; ++e) wb[e] = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    *reinterpret_cast<uint4*>(p) = w;
  };
  // token rows: [hi lo] pairs of U
  for (int t = t0; t < BM; t += nt) {
    const int m = r0 + t;
    const bool valid = m < a.M;
    float u[R];
#pragma unroll
    for (int j = 0; j < R; ++j) u[j] = 0.f;
    if (nr > 0) {
      const float* up = a.U + static_cast<size_t>(min(m, a.M - 1)) * a.r + rk0;
#pragma unroll
      for (int j = 0; j < R; ++j) u[j] = __ldg(up + min(j, nr - 1));
    }
    uint8_t* base = dst + (t >> 3) * Cfg::LR_SBO + (t & 7) * 16;
#pragma unroll
    for (int c = 0; c < K / 8; ++c) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) f[e] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = 4 * c + e;
        if (j < R && j < nr && valid) {
          f[2 * e] = __bfloat162float(__float2bfloat16_rn(u[j]));
          f[2 * e + 1] = u[j] - f[2 * e];  // exact; rounded to bf16 in the store
        }
      }
      if (c == K / 8 - 1 && chunk == 0 && valid) f[6] = 1.f;  // ones against the bias
      store_chunk(base + c * 128, f);
    }
  }
  // output rows: L2 twice, and the bias; two rows per pass where few warps build
  // (more would spill under the builders' register budget)
  constexpr int P = Cfg::NUM_UNPACK_WARPS <= 2 ? 2 : 1;
  for (int t = t0; t < BNR; t += P * nt) {
    unsigned short l[P][R], bb[P];
    bool valid[P];
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const int row = t + p * nt;
      const int n = c0 + row;
      valid[p] = row < BNR && n < a.N;
      const int nc = min(n, a.N - 1);
#pragma unroll
      for (int j = 0; j < R; ++j) l[p][j] = 0;
      if (nr > 0) {
#pragma unroll
        for (int j = 0; j < R; ++j)
          l[p][j] = __ldg(reinterpret_cast<const unsigned short*>(a.L2) + static_cast<size_t>(rk0 + min(j, nr - 1)) * a.N + nc);
      }
      bb[p] = (chunk == 0 && a.bias) ? __ldg(reinterpret_cast<const unsigned short*>(a.bias) + nc) : 0;
    }
#pragma unroll
    for (int p = 0; p < P; ++p) {
      const int row = t + p * nt;
      if (!(row < BNR)) continue;
      uint8_t* base = dst + (BM / 8) * Cfg::LR_SBO + (row >> 3) * Cfg::LR_SBO + (row & 7) * 16;
#pragma unroll
      for (int c = 0; c < K / 8; ++c) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 4 * c + e;
          if (j < R && j < nr && valid[p]) {
            const float v = __bfloat162float(__ushort_as_bfloat16(l[p][j]));
            f[2 * e] = v;
            f[2 * e + 1] = v;
          }
        }
        if (c == K / 8 - 1 && chunk == 0 && valid[p]) f[6] = __bfloat162float(__ushort_as_bfloat16(bb[p]));
        store_chunk(base + c * 128, f);
      }
    }
  }
}

// One unit of a CTA's work: groups [g0, g1) of one output tile.
struct Unit {
  int tile, g0, g1;
  int nslots;  // CTAs contributing to this tile (1: this CTA owns it whole)
  int slot;    // 0 if this is the CTA's first unit, 1 if its last (stream-K partials)
  int first;   // first contributing CTA
};

// Work decomposition.  Whole-tile mode: CTA b takes tiles b, b + grid, ...
// Stream-K mode: the tiles' pipeline stages, laid end to end, are cut into
// equal ranges of stream_len stages, one per CTA, so every CTA streams the same
// amount of operand data; a range splits at tile boundaries into units, and a
// tile cut between CTAs is finished by whichever of them arrives last.
// All stage arithmetic is 32-bit: the host uses stream-K only when the total
// stage count is below 2^30 (64-bit division would expand into a long call-like
// sequence inside warps running with a reduced register budget).
// With CTA pairs the workers are the pairs (both CTAs of a pair take the same units).
template <int GPS, bool PAIR = false>
__device__ __forceinline__ bool next_unit(const GemmArgs& a, int k, Unit& u) {
  const int tiles = a.tiles_r * a.tiles_c;
  const unsigned wid = PAIR ? blockIdx.x >> 1 : blockIdx.x;
  const int nwk = static_cast<int>(PAIR ? gridDim.x >> 1 : gridDim.x);
  if (a.stream_len == 0) {
    const int t = static_cast<int>(wid) + k * nwk;
    if (t >= tiles) return false;
    u.tile = t; u.g0 = 0; u.g1 = a.G; u.nslots = 1; u.slot = 0; u.first = static_cast<int>(wid);
    return true;
  }
  const unsigned S = static_cast<unsigned>(a.stages_per_tile), L = static_cast<unsigned>(a.stream_len);
  const unsigned begin = wid * L;
  const unsigned end = min(begin + L, static_cast<unsigned>(tiles) * S);
  unsigned pos = begin;
  for (int i = 0; i < k && pos < end; ++i) pos = (pos / S + 1) * S;
  if (pos >= end) return false;
  const unsigned t = pos / S;
  const unsigned uend = min(end, (t + 1) * S);
  u.tile = static_cast<int>(t);
  u.g0 = static_cast<int>((pos - t * S) * GPS);
  u.g1 = min(a.G, static_cast<int>((uend - t * S) * GPS));
  u.first = static_cast<int>((t * S) / L);
  const int last = static_cast<int>(((t + 1) * S - 1) / L);
  u.nslots = last - u.first + 1;
  u.slot = (begin >= t * S) ? 0 : 1;
  return true;
}

// The activation step inside a decode-tile launch (kernels with FUSED).  Every
// warp of the grid takes (token, 256-channel chunk) items gw, gw + W, ... and
// computes them as the activation kernel does -- X_hat = X/s, the group absmax,
// codes and scales, with the same helpers, so the same bits -- writing codes
// and scales to the scratch and the chunk's U partial, summed over the warp's
// lanes, to fx_upart.  The stream-K counters are cleared on the way.  Every
// thread calls it.
template <int GL>
__device__ __forceinline__ void fused_act_phase(const GemmArgs& a) {
  const int lane = lane_id();
  const int nw = static_cast<int>(blockDim.x >> 5);
  // items spread over the CTAs first (warp w of CTA b is global warp w * grid + b)
  const int gw = static_cast<int>(threadIdx.x >> 5) * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
  const int W = static_cast<int>(gridDim.x) * nw;
  for (int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x); i < a.fx_zero_words;
       i += static_cast<int>(gridDim.x * blockDim.x))
    a.ws_counters[i] = 0u;
  const int M = a.M, K = a.fx_K, Kp = a.fx_Kp, r = a.r;
  const int nchk = (Kp + 255) >> 8;
  for (int item = gw; item < M * nchk; item += W) {
    const int m = item / nchk, c = item - m * nchk;  // warp-uniform
    const int k0 = c * 256 + lane * 8;
    const bool real = k0 < K, in_k = k0 < Kp;  // K % 8 == 0: a lane's 8 channels are all real or all padding
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    float sv[8], sz[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sv[e] = 1.f;
    if (real) {
      raw = __ldg(reinterpret_cast<const uint4*>(a.fx_X + static_cast<size_t>(m) * K + k0));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(a.fx_s + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(a.fx_s + k0 + 4));
      sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
      sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sz[e] = __frcp_rn(sv[e]);
    float xh[8];
    smooth8(raw, sv, sz, real, xh);
    float sc;
    const uint32_t packed = quantize8_fast<GL>(xh, sc);
    if (in_k) {
      *reinterpret_cast<uint32_t*>(a.fx_codes + static_cast<size_t>(m) * (Kp / 2) + k0 / 2) = packed;
      if ((lane & (GL - 1)) == 0) {
        float* srow = a.fx_scales + static_cast<size_t>(k0 / (8 * GL)) * a.ld_c;
        srow[m] = sc;
        if (m == M - 1)
          for (int p = M; p < a.ld_c; ++p) srow[p] = 0.f;  // padding of the group-major layout
      }
    }
    for (int j0 = 0; j0 < r; j0 += 8) {  // the chunk's U partial, 8 ranks at a time
      float u[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) u[jj] = 0.f;
      if (real) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const __nv_bfloat16* row = a.fx_L1 + static_cast<size_t>(k0 + e) * r + j0;
          if (r % 8 == 0) {  // ranks j0 .. j0+7 of channel k0+e: one 16-byte load
            float f[8];
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(row)), f);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) u[jj] = fmaf(xh[e], f[jj], u[jj]);
          } else {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
              if (j0 + jj < r) u[jj] = fmaf(xh[e], __bfloat162float(__ldg(row + jj)), u[jj]);
          }
        }
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) u[jj] += __shfl_xor_sync(0xffffffffu, u[jj], o);
      if (lane == 0)
#pragma unroll
        for (int jj = 0; jj < 8; ++jj)
          if (j0 + jj < r) a.fx_upart[(static_cast<size_t>(m) * nchk + c) * r + j0 + jj] = u[jj];
    }
  }
}

// Grid-wide barrier of a cooperative launch (every CTA resident), with a time
// limit.  Counters bar[0] (arrivals) and bar[1] (departures) are zero between
// launches: the last CTA to leave clears both, after a timeout too.  Every
// thread calls it; it returns false, with the timeout status raised and the
// CTA's abort flag set, if the grid did not gather in time.  Writes made before
// it are visible after it to every CTA, to the async proxy (TMA and bulk copies
// issued by thread 0) as well.
__device__ __forceinline__ bool grid_barrier(unsigned* bar, uint64_t limit_ns, volatile int* abort, int* s_ok) {
  asm volatile("fence.proxy.async.global;" ::: "memory");  // this thread's writes, for async-proxy readers
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    __threadfence();
    atomicAdd(&bar[0], 1u);
    const uint64_t t0 = global_timer_ns();
    for (;;) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= gridDim.x) break;
      __nanosleep(128);
      if (global_timer_ns() - t0 > limit_ns) {
        ok = 0;
        *abort = 1;
        atomicOr(&g_status, kStatusTimeout);
        break;
      }
    }
    asm volatile("fence.proxy.async.global;" ::: "memory");
    if (atomicAdd(&bar[1], 1u) == gridDim.x - 1) {  // every CTA has left the wait
      atomicExch(&bar[0], 0u);
      atomicExch(&bar[1], 0u);
    }
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_row, const __grid_constant__ CUtensorMap tm_col,
                     const __grid_constant__ CUtensorMap tm_y, const GemmArgs args) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, CW = Cfg::CW, STAGES = Cfg::STAGES, GPS = Cfg::GPS;
  constexpr int NI8 = Cfg::NI8E, NTM = Cfg::NTM;
  constexpr bool PAIR = Cfg::PAIR;
  constexpr int TILE_M = Cfg::TILE_M;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* ystage = smem + STAGES * Cfg::STAGE_BYTES;  // 1024-aligned (stage sizes are)
  uint8_t* i8_base = ystage + Cfg::YST_BYTES;
  uint8_t* lr_buf = i8_base + NI8 * Cfg::I8_BYTES;  // low-rank operands (pre-expanded mode)
  uint8_t* sc_base = lr_buf + Cfg::LR_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sc_base + Cfg::SSLOTS * Cfg::SSLOT_BYTES);
  uint64_t* full = bars;                   // [STAGES] packed stage landed
  uint64_t* empty = bars + STAGES;         // [STAGES] packed stage unpacked
  uint64_t* sfull = bars + 2 * STAGES;     // [SSLOTS] scales landed
  uint64_t* sempty = sfull + Cfg::SSLOTS;  // [SSLOTS] scales drained
  uint64_t* full8 = sempty + Cfg::SSLOTS;  // [NI8] int8 operands ready
  uint64_t* empty8 = full8 + NI8;          // [NI8] int8 operands consumed by the MMA
  uint64_t* tfull = empty8 + NI8;          // [NTM] TMEM partials ready
  uint64_t* tempty = tfull + NTM;          // [NTM] TMEM partials drained
  uint64_t* final_bar = tempty + NTM;      // teardown: all MMAs done
  uint64_t* lrfull = final_bar + 1;        // low-rank operands built (pre-expanded mode)
  uint64_t* lrempty = lrfull + 1;          // low-rank operands consumed by the MMA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Cfg::NUM_BARS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tail_flag = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const WaitPolicy wp{args.limit_ns, abort_flag};
  // CTA pairs: rank 0 (the even CTA) issues the MMAs; each CTA owns tile rows
  // crank*128 .. +127 and output rows crank*B_ROWS .. of the col operand
  const uint32_t crank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = crank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], Cfg::PRE ? 1 : Cfg::NUM_UNPACK_WARPS);  // PRE: released by the MMA's commit
    }
    for (int s = 0; s < Cfg::SSLOTS; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], Cfg::NUM_DRAIN_WARPS);
    }
    for (int b = 0; b < NI8; ++b) {
      mbar_init(&full8[b], Cfg::NUM_UNPACK_WARPS);
      mbar_init(&empty8[b], 1);
    }
    for (int b = 0; b < NTM; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], Cfg::NUM_DRAIN_WARPS * Cfg::PM);  // pairs: both CTAs' drain warps
    }
    mbar_init(final_bar, 1);
    mbar_init(lrfull, Cfg::NUM_UNPACK_WARPS * Cfg::PM);
    mbar_init(lrempty, 1);
    *abort_flag = 0;
    *tail_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_row);
    prefetch_tensormap(&tm_col);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);  // the same warp of both CTAs
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync();  // the peer's barriers are initialised before any remote arrive
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // every warp but the producer reads or writes global memory only after the
  // preceding kernel is complete (U, L2, bias, Y, the workspace)
  if (!Cfg::FUSED && warp != 0) grid_dep_wait();

  uint32_t issued = 0;  // producer: stages issued (for the teardown drain)
  uint32_t npre = 0;    // producer: weight tiles requested before the preceding kernel completed
  // Weights x tokens tiles: the weight tiles of the first STAGES steps are
  // requested before waiting for the preceding kernel (the packed weights are
  // never written by the kernel just before this one: the packing kernel does
  // not let its successor start early).  Their token halves follow once the
  // tokens' codes exist.
  auto prefetch_weights = [&]() {
    if constexpr (Cfg::SWAP) {
      Unit pu;
      for (int k = 0; npre < static_cast<uint32_t>(STAGES) && next_unit<GPS, PAIR>(args, k, pu); ++k) {
        const int r0p = (pu.tile % args.tiles_r) * BM;
        for (int g = pu.g0; g < pu.g1 && npre < static_cast<uint32_t>(STAGES); g += GPS, ++npre) {
          mbar_arrive_expect_tx(&full[npre], Cfg::A_PACK + Cfg::B_PACK);
          tma_load_2d(stage_base + npre * Cfg::STAGE_BYTES, &tm_row, &full[npre], g * Cfg::BPG * 32, r0p);
        }
      }
    }
  };
  // FUSED: the activation step, distributed over the grid, then a grid barrier;
  // the drain warps then sum U (fixed chunk order) into the CTA's own copy while
  // the pipeline fills.
  bool fused_ok = true;
  const float* Uv = args.U;
  // U: the preceding kernel's (read-only here), or this CTA's own copy (written above)
  auto load_u = [](const float* p) -> float {
    if constexpr (Cfg::FUSED) return *p;
    else return __ldg(p);
  };
  if constexpr (Cfg::FUSED) {
    if (warp == 0 && lane == 0 && !(args.debug_flags & 1)) prefetch_weights();
    issued = npre;
    grid_dep_wait();
    fused_act_phase<(Cfg::BPG == 2 ? 16 : 8)>(args);
    fused_ok = grid_barrier(args.fx_bar, args.limit_ns, abort_flag, reinterpret_cast<int*>(tmem_slot + 3));
    Uv = args.fx_U + static_cast<size_t>(blockIdx.x) * args.M * args.r;  // summed by the drain warps
  }

  if (!fused_ok) {
    // the grid did not gather: no work unit runs; the teardown lets the weight
    // tiles already requested land
  } else if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (Cfg::REALLOC) regs_dealloc<Cfg::REGS_LOW>();
    if (lane == 0 && !(args.debug_flags & 1)) {
      // (weight tiles first; the token halves follow right after the wait,
      // before anything that can give up)
      if constexpr (!Cfg::FUSED) {
        prefetch_weights();
        grid_dep_wait();
      }
      grid_dep_launch();
      uint32_t it = 0;
      bool ok = true;
      Unit un;
      for (int k = 0; ok && next_unit<GPS, PAIR>(args, k, un); ++k) {
        const int tr = un.tile % args.tiles_r, tc = un.tile / args.tiles_r;
        const int g0 = un.g0, g1 = un.g1;
        const int c0 = tc * BN;
        const int r0 = tr * TILE_M + static_cast<int>(crank) * BM;  // this CTA's first row
        const uint32_t cs_bytes = static_cast<uint32_t>(min(BN, args.ld_c - c0)) * 4u;
        // (the odd CTA of a pair tile past the last row has no row scales to load)
        const uint32_t rs_bytes = static_cast<uint32_t>(max(0, min(BM, args.ld_r - r0))) * 4u;
        const bool lr_unit = Cfg::LR_MMA && args.lr_mma && g0 == 0;
        for (int g = lr_unit ? g0 - GPS * args.lr_mma : g0; g < g1; g += GPS, ++it) {
          const int ng = min(GPS, g1 - g);
          const int s = it % STAGES;
          const int ss = it % Cfg::SSLOTS;
          if (!wait_one(&empty[s], ((it / STAGES) & 1) ^ 1, wp)) { ok = false; break; }
          if (!wait_one(&sempty[ss], ((it / Cfg::SSLOTS) & 1) ^ 1, wp)) { ok = false; break; }
          if (g < g0) {
            // low-rank step: its operands are built by the unpack warps; its
            // scales are 1 (columns) and 2^-18 (rows, undone by the drain's
            // E4M3 factor), so the drain folds it in like any group
            float4* scw = reinterpret_cast<float4*>(sc_base + ss * Cfg::SSLOT_BYTES);
            for (int i = 0; i < BN / 4; ++i) scw[(Cfg::CS_OFF / 16) + i] = make_float4(1.f, 1.f, 1.f, 1.f);
            const float lo = 1.0f / 262144.0f;
            for (int i = 0; i < BM / 4; ++i) scw[(Cfg::RS_OFF / 16) + i] = make_float4(lo, lo, lo, lo);
            if (!Cfg::ONE_PHASE) mbar_arrive(&sfull[ss]);  // (ONE_PHASE: released with the stage's arrival below)
            if (leader) mbar_arrive(&full[s]);  // pairs: only the MMA issuer's barrier counts
            issued = it + 1;
            continue;
          }
          uint8_t* st = stage_base + s * Cfg::STAGE_BYTES;
          uint8_t* sc = sc_base + ss * Cfg::SSLOT_BYTES;
          if constexpr (PAIR) {
            // MMA-ready E4M3 tiles, this CTA's share: 128 token rows and B_ROWS
            // output rows per 64-block, one 32 x 256-byte box each.  Both CTAs'
            // bytes are counted on the even CTA's barrier, which the even CTA
            // arms with the pair's total (the odd CTA's bytes may land first:
            // the phase cannot complete before that arrival).
            if (leader) mbar_arrive_expect_tx(&full[s], Cfg::PM * (Cfg::A_E8 + Cfg::B_E8));
            const uint32_t fb = mapa_shared(smem_u32(&full[s]), 0u);
#pragma unroll
            for (int b = 0; b < Cfg::BPG; ++b) {
              const int blk = g * Cfg::BPG + b;
              tma_load_2d_pair(st + b * Cfg::A_E8_BLK, &tm_row, fb, 0, 2 * (blk * args.rg_r + r0 / 8));
              tma_load_2d_pair(st + Cfg::A_E8 + b * Cfg::B_E8_BLK, &tm_col, fb, 0,
                               2 * (blk * args.rg_c + (c0 + static_cast<int>(crank) * Cfg::B_ROWS) / 8));
            }
          } else if constexpr (Cfg::PRE) {
            // MMA-ready E4M3 tiles: one contiguous block per operand (and, with
            // ONE_PHASE, the group's scales on the same barrier)
            mbar_arrive_expect_tx(&full[s], Cfg::A_E8 + Cfg::B_E8 + (Cfg::ONE_PHASE ? ng * (cs_bytes + rs_bytes) : 0u));
#pragma unroll
            for (int b = 0; b < Cfg::BPG; ++b) {
              const size_t blk = static_cast<size_t>(g) * Cfg::BPG + b;
              bulk_load(st + b * Cfg::A_E8_BLK, args.xe + (blk * args.rg_r + tr * (BM / 8)) * Cfg::E8_SBO,
                        Cfg::A_E8_BLK, &full[s]);
              bulk_load(st + Cfg::A_E8 + b * Cfg::B_E8_BLK, args.we + (blk * args.rg_c + tc * (BN / 8)) * Cfg::E8_SBO,
                        Cfg::B_E8_BLK, &full[s]);
            }
          } else {
            if (it >= npre) {
              mbar_arrive_expect_tx(&full[s], Cfg::A_PACK + Cfg::B_PACK);
              tma_load_2d(st, &tm_row, &full[s], g * Cfg::BPG * 32, r0);
            }
            tma_load_2d(st + Cfg::A_PACK, &tm_col, &full[s], g * Cfg::BPG * 32, c0);
          }
          uint64_t* sbar = Cfg::ONE_PHASE ? &full[s] : &sfull[ss];
          if (!Cfg::ONE_PHASE) mbar_arrive_expect_tx(&sfull[ss], ng * (cs_bytes + rs_bytes));
          for (int j = 0; j < ng; ++j) {
            bulk_load(sc + Cfg::CS_OFF + j * Cfg::CS_BYTES,
                      args.scales_c + static_cast<size_t>(g + j) * args.ld_c + c0, cs_bytes, sbar);
            if (rs_bytes)
              bulk_load(sc + Cfg::RS_OFF + j * Cfg::RS_BYTES,
                        args.scales_r + static_cast<size_t>(g + j) * args.ld_r + r0, rs_bytes, sbar);
          }
          issued = it + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (Cfg::REALLOC) regs_dealloc<Cfg::REGS_LOW>();
    if (Cfg::PRE && lane == 0 && leader) {
      // pre-expanded operands: the MMAs read the stage itself and release it.
      // Pairs: one cta_group::2 MMA covers both CTAs' rows; its completion is
      // signalled to the same barrier in both CTAs.
      constexpr uint32_t idesc = idesc_f8(TILE_M, BN);
      constexpr uint32_t idesc_lr = idesc_bf16(TILE_M, BN);
      auto commit_both = [&](uint64_t* bar) {
        if constexpr (PAIR) {
          mma_commit_pair(mapa_shared(smem_u32(bar), 0u));
          mma_commit_pair(mapa_shared(smem_u32(bar), 1u));
        } else {
          mma_commit(bar);
        }
      };
      uint32_t it = 0, nlr = 0;
      bool ok = true;
      Unit un;
      for (int k = 0; ok && next_unit<GPS, PAIR>(args, k, un); ++k) {
        const int g0 = un.g0, g1 = un.g1;
        const bool lr_unit = Cfg::LR_MMA && args.lr_mma && g0 == 0;
        for (int g = lr_unit ? g0 - GPS * args.lr_mma : g0; g < g1; g += GPS, ++it) {
          const int s = it % STAGES;
          const int tb = it % NTM;
          if (!wait_one(&full[s], (it / STAGES) & 1, wp)) { ok = false; break; }
          if (!(PAIR ? wait_one_cluster(&tempty[tb], ((it / NTM) & 1) ^ 1, wp)
                     : wait_one(&tempty[tb], ((it / NTM) & 1) ^ 1, wp))) { ok = false; break; }
          const uint32_t d = tmem_base + static_cast<uint32_t>(tb * BN);
          if (Cfg::LR_MMA && g < g0) {
            // low-rank step: [U_hi U_lo 1] x [L2 L2 b] over K = LR_K, from the low-rank buffer
            if (!(PAIR ? wait_one_cluster(lrfull, nlr & 1, wp) : wait_one(lrfull, nlr & 1, wp))) { ok = false; break; }
            tc_fence_after();
            const uint32_t abuf = smem_u32(lr_buf), bbuf = abuf + (BM / 8) * Cfg::LR_SBO;
#pragma unroll
            for (int q = 0; q < Cfg::LR_K / 16; ++q) {
              const uint64_t da = smem_desc_kmajor(abuf + q * 256, 128, Cfg::LR_SBO);
              const uint64_t db = smem_desc_kmajor(bbuf + q * 256, 128, Cfg::LR_SBO);
              if constexpr (PAIR) mma_bf16_pair(d, da, db, idesc_lr, q > 0 ? 1u : 0u);
              else mma_bf16(d, da, db, idesc_lr, q > 0 ? 1u : 0u);
            }
            commit_both(lrempty);
            ++nlr;
          } else {
            tc_fence_after();
            const uint32_t stg = smem_u32(stage_base + s * Cfg::STAGE_BYTES);
#pragma unroll
            for (int b = 0; b < Cfg::BPG; ++b) {
              const uint32_t abuf = stg + b * Cfg::A_E8_BLK, bbuf = stg + Cfg::A_E8 + b * Cfg::B_E8_BLK;
#pragma unroll
              for (int kh = 0; kh < 2; ++kh) {  // two K = 32 MMAs per 64-block
                const uint64_t da = smem_desc_kmajor(abuf + 256 * kh, 128, Cfg::E8_SBO);
                const uint64_t db = smem_desc_kmajor(bbuf + 256 * kh, 128, Cfg::E8_SBO);
                const uint32_t acc = (b > 0 || kh > 0) ? 1u : 0u;
                if constexpr (PAIR) mma_f8_pair(d, da, db, idesc, acc);
                else mma_f8(d, da, db, idesc, acc);
              }
            }
          }
          commit_both(&empty[s]);
          if (!Cfg::ONE_PHASE) commit_both(&tfull[tb]);
        }
      }
    } else if (!Cfg::PRE && lane == 0) {
      constexpr uint32_t idesc = Cfg::F8 ? idesc_f8(BM, BN) : idesc_i8(BM, BN);
      constexpr int NI8D = NI8 > 0 ? NI8 : 1;  // (unused when PRE)
      uint32_t it = 0;
      bool ok = true;
      Unit un;
      for (int k = 0; ok && next_unit<GPS, PAIR>(args, k, un); ++k) {
        const int g0 = un.g0, g1 = un.g1;
        const bool lr_unit = Cfg::LR_MMA && args.lr_mma && g0 == 0;
        for (int g = lr_unit ? g0 - GPS * args.lr_mma : g0; g < g1; g += GPS, ++it) {
          const int ng = min(GPS, g1 - g);
          const int b = it % NI8D;
          const int tb = it % NTM;
          if (!wait_one(&full8[b], (it / NI8D) & 1, wp)) { ok = false; break; }
          if (!wait_one(&tempty[tb], ((it / NTM) & 1) ^ 1, wp)) { ok = false; break; }
          tc_fence_after();
          const uint32_t buf = smem_u32(i8_base + b * Cfg::I8_BYTES);
          if (Cfg::LR_MMA && g < g0) {
            // low-rank step: [U_hi U_lo 1] x [L2 L2 b] over K = LR_K, two K=16 bf16 MMAs
            constexpr uint32_t idesc_lr = idesc_bf16(BM, BN);
            const uint32_t d = tmem_base + static_cast<uint32_t>(tb * GPS * BN);
            const uint32_t b_addr = buf + (BM / 8) * Cfg::LR_SBO;
#pragma unroll
            for (int q = 0; q < Cfg::LR_K / 16; ++q)
              mma_bf16(d, smem_desc_kmajor(buf + q * 256, 128, Cfg::LR_SBO),
                       smem_desc_kmajor(b_addr + q * 256, 128, Cfg::LR_SBO), idesc_lr, q > 0 ? 1u : 0u);
            mma_commit(&empty8[b]);
            mma_commit(&tfull[tb]);
            continue;
          }
          for (int j = 0; j < ng; ++j) {
            const uint32_t d = tmem_base + static_cast<uint32_t>((tb * GPS + j) * BN);
#pragma unroll
            for (int bb = 0; bb < Cfg::BPG; ++bb) {
              const int jb = j * Cfg::BPG + bb;  // 64-block within the stage
              const uint32_t a_addr = buf + jb * Cfg::SA;
              const uint32_t b_addr = buf + Cfg::BPS * Cfg::SA + jb * Cfg::SB;
              const uint32_t acc0 = bb > 0 ? 1u : 0u;
              if constexpr (Cfg::F8) {
                mma_f8(d, smem_desc_kmajor(a_addr, kLBO, kSBO), smem_desc_kmajor(b_addr, kLBO, kSBO), idesc, acc0);
                mma_f8(d, smem_desc_kmajor(a_addr + 2 * kLBO, kLBO, kSBO),
                       smem_desc_kmajor(b_addr + 2 * kLBO, kLBO, kSBO), idesc, 1u);
              } else {
                mma_i8(d, smem_desc_kmajor(a_addr, kLBO, kSBO), smem_desc_kmajor(b_addr, kLBO, kSBO), idesc, acc0);
                mma_i8(d, smem_desc_kmajor(a_addr + 2 * kLBO, kLBO, kSBO),
                       smem_desc_kmajor(b_addr + 2 * kLBO, kLBO, kSBO), idesc, 1u);
              }
            }
          }
          mma_commit(&empty8[b]);
          mma_commit(&tfull[tb]);
        }
      }
    }
  } else if (warp < 2 + Cfg::NUM_UNPACK_WARPS) {
    // ------------------------------------------------------------ unpack
    if (Cfg::REALLOC) regs_dealloc<Cfg::REGS_LOW>();
    if constexpr (Cfg::PRE) {
      // pre-expanded mode: these warps only build the low-rank step's operands,
      // one tile ahead at most (single buffer)
      const int ut = (warp - 2) * 32 + lane;
      uint32_t nlr = 0;
      bool ok = true;
      Unit un;
      for (int k = 0; ok && next_unit<GPS, PAIR>(args, k, un); ++k) {
        if (!(Cfg::LR_MMA && args.lr_mma && un.g0 == 0)) continue;
        const int tr = un.tile % args.tiles_r, tc = un.tile / args.tiles_r;
        const int lr0 = tr * TILE_M + static_cast<int>(crank) * BM;        // this CTA's token rows
        const int lc0 = tc * BN + static_cast<int>(crank) * Cfg::B_ROWS;  // and output rows
        for (int chunk = 0; chunk < args.lr_mma; ++chunk) {
          if (!wait_warp(lrempty, (nlr & 1) ^ 1, wp)) { ok = false; break; }
          // chunks as constants, so that each build unrolls over a fixed rank range
          constexpr int LT = 32 * Cfg::NUM_UNPACK_WARPS;
          if constexpr (Cfg::LRFAST) {
            if (chunk == 0) build_lr_operands_mlp<Cfg>(args, lr0, lc0, 0, lr_buf, ut, LT);
            else if (chunk == 1) build_lr_operands_mlp<Cfg>(args, lr0, lc0, 1, lr_buf, ut, LT);
            else build_lr_operands_mlp<Cfg>(args, lr0, lc0, 2, lr_buf, ut, LT);
          } else {
            if (chunk == 0) build_lr_operands<Cfg>(args, lr0, lc0, 0, lr_buf, ut, LT);
            else if (chunk == 1) build_lr_operands<Cfg>(args, lr0, lc0, 1, lr_buf, ut, LT);
            else build_lr_operands<Cfg>(args, lr0, lc0, 2, lr_buf, ut, LT);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (leader) mbar_arrive(lrfull);
            else mbar_arrive_cluster(mapa_shared(smem_u32(lrfull), 0u));  // the MMA issuer's barrier
          }
          ++nlr;
        }
      }
    } else {
      constexpr int NT = 32 * Cfg::NUM_UNPACK_WARPS;
      // This thread's tasks are the same at every stage: precompute their offsets.
      // Task t -> operand (row tasks first), row, 16-byte chunk c of the row's
      // 32*BPS packed bytes (c fastest, so 8 consecutive threads read 128
      // contiguous bytes); 64-block jb = c/2, half = c%2, scale group jb/BPG.
      uint32_t src_off[Cfg::TPT], dst_off[Cfg::TPT];
      int grp[Cfg::TPT];
      const int ut = (warp - 2) * 32 + lane;
  #pragma unroll
      for (int i = 0; i < Cfg::TPT; ++i) {
        int t = ut + i * NT;
        grp[i] = GPS;  // GPS = no task
        src_off[i] = dst_off[i] = 0;
        if (t < Cfg::TASKS) {
          const bool colop = t >= 2 * Cfg::BPS * BM;
          if (colop) t -= 2 * Cfg::BPS * BM;
          const int row = t / (2 * Cfg::BPS), c = t % (2 * Cfg::BPS);
          const int jb = c >> 1, half = c & 1;
          grp[i] = jb / Cfg::BPG;
          src_off[i] = (colop ? Cfg::A_PACK : 0) + row * 32 * Cfg::BPS + c * 16;
          dst_off[i] = (colop ? Cfg::BPS * Cfg::SA + jb * Cfg::SB : jb * Cfg::SA) + (row >> 3) * kSBO +
                       2 * half * kLBO + (row & 7) * 16;
        }
      }
      uint32_t it = 0;
      bool ok = true;
      Unit un;
      for (int k = 0; ok && next_unit<GPS, PAIR>(args, k, un); ++k) {
        const int g0 = un.g0, g1 = un.g1;
        const bool lr_unit = Cfg::LR_MMA && args.lr_mma && g0 == 0;
        for (int g = lr_unit ? g0 - GPS * args.lr_mma : g0; g < g1; g += GPS, ++it) {
          const int ng = min(GPS, g1 - g);
          const int s = it % STAGES;
          const int b = it % NI8;
          if (!wait2_warp(&full[s], (it / STAGES) & 1, &empty8[b], ((it / NI8) & 1) ^ 1, wp)) { ok = false; break; }
          const uint8_t* st = stage_base + s * Cfg::STAGE_BYTES;
          uint8_t* dst = i8_base + b * Cfg::I8_BYTES;
          if (Cfg::LR_MMA && g < g0) {
            const int tr = un.tile % args.tiles_r, tc = un.tile / args.tiles_r;
            const int chunk = (g - (g0 - GPS * args.lr_mma)) / GPS;
            if constexpr (Cfg::LRFAST) {
              if (chunk == 0) build_lr_operands_mlp<Cfg>(args, tr * BM, tc * BN, 0, dst, ut, NT);
              else if (chunk == 1) build_lr_operands_mlp<Cfg>(args, tr * BM, tc * BN, 1, dst, ut, NT);
              else build_lr_operands_mlp<Cfg>(args, tr * BM, tc * BN, 2, dst, ut, NT);
            } else {
              if (chunk == 0) build_lr_operands<Cfg>(args, tr * BM, tc * BN, 0, dst, ut, NT);
              else if (chunk == 1) build_lr_operands<Cfg>(args, tr * BM, tc * BN, 1, dst, ut, NT);
              else build_lr_operands<Cfg>(args, tr * BM, tc * BN, 2, dst, ut, NT);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(&full8[b]);
              mbar_arrive(&empty[s]);
            }
            continue;
          }
          uint4 pk[Cfg::TPT];
  #pragma unroll
          for (int i = 0; i < Cfg::TPT; ++i)  // all loads first (always inside the stage)
            pk[i] = *reinterpret_cast<const uint4*>(st + src_off[i]);
          // with one group per stage and tasks filling every thread, no task test is needed
          constexpr bool ALL_TASKS = GPS == 1 && Cfg::TASKS % NT == 0;
  #pragma unroll
          for (int i = 0; i < Cfg::TPT; ++i)
            if (ALL_TASKS || grp[i] < ng) unpack16<Cfg::F8>(pk[i], dst + dst_off[i]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&full8[b]);
            mbar_arrive(&empty[s]);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ drain + epilogue
    if (Cfg::REALLOC) regs_alloc<Cfg::REGS_HIGH>();
    const int dw = warp - (2 + Cfg::NUM_UNPACK_WARPS);
    if constexpr (Cfg::FUSED) {
      // this CTA's copy of U: the chunks' partials in a fixed order; the drain
      // warps alone read it (named barrier 1 over them)
      const int nchk = (args.fx_Kp + 255) >> 8;
      float* Uc = const_cast<float*>(Uv);
      for (int t = dw * 32 + lane; t < args.M * args.r; t += 32 * Cfg::NUM_DRAIN_WARPS) {
        const int m = t / args.r, j = t - (t / args.r) * args.r;
        float v = 0.f;
        for (int c = 0; c < nchk; ++c) v += __ldcg(args.fx_upart + (static_cast<size_t>(m) * nchk + c) * args.r + j);
        Uc[t] = v;
      }
      named_bar_sync(1, 32 * Cfg::NUM_DRAIN_WARPS);
    }
    const int q = warp & 3;            // TMEM lane quadrant
    const int h = dw >> 2;             // column slice
    const int qd = lane >> 2, qc = lane & 3;
    // Thread <-> accumulator layout, that of tcgen05.ld.16x256b: the thread holds
    // rows q*32 + qd + 8i (i = 0..3) of the tile and, in each 8-column block b of
    // its slice, columns h*CW + 8b + 2qc + {0, 1}, as the pair acc2[i*NBLK + b].
    // A column-scale pair then serves four rows, and the four threads of a quad
    // read four different pairs, so the per-group scale loads stay few.
    constexpr int NBLK = CW / 8;   // 8-column blocks of the slice
    constexpr int CHB = Cfg::CHB;  // blocks per chunk (one TMEM load per half quadrant)
    constexpr int NCC = NBLK / CHB;  // chunks per group
    const uint32_t t_q = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    uint32_t it = 0;
    bool ok = true;
    Unit un;
    for (int k = 0; ok && next_unit<GPS, PAIR>(args, k, un); ++k) {
      const int tile = un.tile;
      const int tr = tile % args.tiles_r, tc = tile / args.tiles_r;
      const int g0 = un.g0, g1 = un.g1;
      const int rbase = tr * TILE_M + static_cast<int>(crank) * BM + q * 32 + qd;  // row of i = 0 (row i adds 8i)
      const int col0 = tc * BN + h * CW + 2 * qc;  // column of block 0, first of the pair
      const bool lr_unit = Cfg::LR_MMA && args.lr_mma && g0 == 0;
      float2 acc2[4 * NBLK];
#pragma unroll
      for (int j = 0; j < 4 * NBLK; ++j) acc2[j] = make_float2(0.f, 0.f);
      // The unit that holds the tile's first stage starts its accumulators at
      // U L2 + b (when no low-rank MMA step carries it).
      if (g0 == 0 && !lr_unit) {
        if constexpr (!Cfg::SWAP) {
          // rows are tokens m, columns are output features n
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int m = rbase + 8 * i;
            if (m >= args.rows_r) continue;
            if (args.bias) {
#pragma unroll
              for (int b = 0; b < NBLK; ++b) {
                const int n = col0 + 8 * b;
                if (n < args.N) acc2[i * NBLK + b] = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(args.bias + n));
              }
            }
            const float* urow = args.U + static_cast<size_t>(m) * args.r;
            for (int kk = 0; kk < args.r; ++kk) {
              const float um = __ldg(urow + kk);
              const float2 um2 = make_float2(um, um);
              const __nv_bfloat16* l2 = args.L2 + static_cast<size_t>(kk) * args.N;
#pragma unroll
              for (int b = 0; b < NBLK; ++b) {
                const int n = col0 + 8 * b;
                if (n < args.N)
                  acc2[i * NBLK + b] = __ffma2_rn(um2, __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(l2 + n)),
                                                  acc2[i * NBLK + b]);
              }
            }
          }
        } else {
          // rows are output features n, columns are tokens m
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int n = rbase + 8 * i;
            if (n >= args.rows_r) continue;
            const float bn = args.bias ? __bfloat162float(args.bias[n]) : 0.f;
#pragma unroll
            for (int b = 0; b < NBLK; ++b) acc2[i * NBLK + b] = make_float2(bn, bn);
            for (int kk = 0; kk < args.r; ++kk) {
              const float l2 = __bfloat162float(args.L2[static_cast<size_t>(kk) * args.N + n]);
#pragma unroll
              for (int b = 0; b < NBLK; ++b) {
                const int m = col0 + 8 * b;
                if (m < args.M) acc2[i * NBLK + b].x = fmaf(load_u(Uv + static_cast<size_t>(m) * args.r + kk), l2, acc2[i * NBLK + b].x);
                if (m + 1 < args.M) acc2[i * NBLK + b].y = fmaf(load_u(Uv + static_cast<size_t>(m + 1) * args.r + kk), l2, acc2[i * NBLK + b].y);
              }
            }
          }
        }
      }
      for (int g = lr_unit ? g0 - GPS * args.lr_mma : g0; g < g1; g += GPS, ++it) {
        const int ng = GPS == 1 ? 1 : min(GPS, g1 - g);
        const int ss = it % Cfg::SSLOTS;
        const int tb = it % NTM;
        if (Cfg::ONE_PHASE) {
          // the step's MMAs are complete (so its stage, scales included, had landed)
          if (!wait_warp(&empty[it % STAGES], (it / STAGES) & 1, wp)) { ok = false; break; }
        } else if (!wait2_warp(&tfull[tb], (it / NTM) & 1, &sfull[ss], (it / Cfg::SSLOTS) & 1, wp)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float* cs_stage = reinterpret_cast<const float*>(sc_base + ss * Cfg::SSLOT_BYTES + Cfg::CS_OFF);
        const float* rs_stage = reinterpret_cast<const float*>(sc_base + ss * Cfg::SSLOT_BYTES + Cfg::RS_OFF);
        // The stage's partials are read from TMEM one 16-column chunk (both
        // half quadrants) at a time.  tcgen05.wait::ld waits for every load the
        // thread has issued, so the pipeline is one chunk deep: the loads of
        // chunk i+1 are in flight while chunk i is folded into the accumulators.
        const int nbt = ng * NCC;  // chunks in this stage
        uint32_t vbuf[Cfg::PIPE ? 2 : 1][2][4 * CHB];
        auto issue = [&](int bi, uint32_t (&dst)[2][4 * CHB]) {
          const int j = bi / NCC, cc = bi % NCC;
          const uint32_t col = static_cast<uint32_t>((tb * GPS + j) * BN + h * CW + 8 * CHB * cc);
          if constexpr (CHB == 2) {
            tmem_ld_q8(t_q + col, dst[0]);
            tmem_ld_q8(t_q + (16u << 16) + col, dst[1]);
          } else if constexpr (CHB == 4) {
            tmem_ld_q16(t_q + col, dst[0]);
            tmem_ld_q16(t_q + (16u << 16) + col, dst[1]);
          } else {
            tmem_ld_q32(t_q + col, dst[0]);
            tmem_ld_q32(t_q + (16u << 16) + col, dst[1]);
          }
        };
        auto wait_chunk = [&](uint32_t (&dst)[2][4 * CHB]) {
          if constexpr (CHB == 8) {
            tmem_ld_wait(dst[0]);  // (one wait covers both loads; the second passes its registers through)
            tmem_ld_wait(dst[1]);
          } else {
            tmem_ld_wait(dst[0], dst[1]);
          }
        };
        // With HSQ_EARLY_RELEASE the TMEM buffer is handed back to the MMA warp as
        // soon as the stage's last load has landed, before that chunk's math.
        auto release_tmem = [&]() {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader) mbar_arrive(&tempty[tb]);
            else mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[tb]), 0u));  // the MMA issuer's barrier
          }
        };
        if constexpr (Cfg::PIPE) {
          issue(0, vbuf[0]);
          wait_chunk(vbuf[0]);
          if (HSQ_EARLY_RELEASE && nbt == 1) release_tmem();
        }
        float2 rs2[4];
#pragma unroll
        for (int bi = 0; bi < GPS * NCC; ++bi) {
          if (bi >= nbt) break;  // warp-uniform
          const int j = bi / NCC, cc = bi % NCC;
          uint32_t(&cur)[2][4 * CHB] = vbuf[Cfg::PIPE ? (bi & 1) : 0];
          if constexpr (Cfg::PIPE) {
            if (bi + 1 < nbt) issue(bi + 1, vbuf[(bi + 1) & 1]);
          } else {
            issue(bi, cur);
            wait_chunk(cur);
            if (HSQ_EARLY_RELEASE && bi + 1 == nbt) release_tmem();
          }
          if (cc == 0) {
            // the four rows' scales of group g+j, times the factor that undoes the
            // operand encoding: 1/256 for 16*q (int8), 2^18 for q * 2^-9 (E4M3)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float rs = rs_stage[j * BM + q * 32 + qd + 8 * i] * (Cfg::F8 ? 262144.0f : (1.0f / 256.0f));
              rs2[i] = make_float2(rs, rs);
            }
          }
          const float* cs = cs_stage + j * BN + h * CW + 8 * CHB * cc + 2 * qc;
#pragma unroll
          for (int kb = 0; kb < CHB; ++kb) {
            const float2 c2 = *reinterpret_cast<const float2*>(cs + 8 * kb);
            const int b = CHB * cc + kb;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t u0 = cur[i >> 1][4 * kb + 2 * (i & 1)], u1 = cur[i >> 1][4 * kb + 2 * (i & 1) + 1];
              const float2 pp = Cfg::F8 ? make_float2(__uint_as_float(u0), __uint_as_float(u1))
                                        : make_float2(__int2float_rn(static_cast<int>(u0)),
                                                      __int2float_rn(static_cast<int>(u1)));
              acc2[i * NBLK + b] = __ffma2_rn(rs2[i], __fmul2_rn(pp, c2), acc2[i * NBLK + b]);
            }
          }
          if constexpr (Cfg::PIPE) {
            if (bi + 1 < nbt) {
              wait_chunk(vbuf[(bi + 1) & 1]);
              if (HSQ_EARLY_RELEASE && bi + 2 == nbt) release_tmem();
            }
          }
        }
        if (!HSQ_EARLY_RELEASE) release_tmem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[ss]);
      }
      if (!ok) break;

      // ---------------------------------------------------------- epilogue
      if (un.nslots > 1) {
        // Stream-K: every drain warp owns a 32-row x CW-column sub-tile.  It
        // writes its fp32 partial to this CTA's slot (in the threads' own
        // layout, so each store is 32 consecutive pairs), and the warp that
        // arrives last for that sub-tile sums the contributing CTAs' partials
        // in CTA order (deterministic), runs the epilogue and re-zeroes the
        // counter.  No cross-warp or cross-CTA waiting.
        constexpr int SLOT2 = BN * BM / 2;  // float2 per CTA slot
        float2* part = reinterpret_cast<float2*>(args.ws_partials) +
                       (static_cast<size_t>(blockIdx.x) * 2 + un.slot) * SLOT2 + dw * (4 * NBLK * 32) + lane;
        // (pairs: a tile's sub-tiles are counted per CTA rank; worker c's CTA of this rank is 2c + crank)
#pragma unroll
        for (int j = 0; j < 4 * NBLK; ++j) part[j * 32] = acc2[j];
        __threadfence();
        __syncwarp();
        unsigned* counter =
            args.ws_counters + (static_cast<size_t>(tile) * Cfg::PM + crank) * Cfg::NUM_DRAIN_WARPS + dw;
        int last = 0;
        if (lane == 0) last = (atomicAdd(counter, 1u) == static_cast<unsigned>(un.nslots - 1)) ? 1 : 0;
        last = __shfl_sync(0xffffffffu, last, 0);
        if (!last) continue;
        __threadfence();
#pragma unroll
        for (int j = 0; j < 4 * NBLK; ++j) acc2[j] = make_float2(0.f, 0.f);
        const unsigned S = static_cast<unsigned>(args.stages_per_tile);
        const unsigned L = static_cast<unsigned>(args.stream_len);
#pragma unroll 1
        for (int c = un.first; c < un.first + un.nslots; ++c) {
          const int cslot = (static_cast<unsigned>(c) * L >= static_cast<unsigned>(tile) * S) ? 0 : 1;
          const size_t cta = static_cast<size_t>(c) * Cfg::PM + crank;
          const float2* p = reinterpret_cast<const float2*>(args.ws_partials) +
                            (cta * 2 + cslot) * SLOT2 + dw * (4 * NBLK * 32) + lane;
          // 16 pairs in flight at a time (the accumulators already use most registers)
#pragma unroll
          for (int j0 = 0; j0 < 4 * NBLK; j0 += 16) {
            float2 v[16];
#pragma unroll
            for (int e = 0; e < 16 && j0 + e < 4 * NBLK; ++e) v[e] = __ldcg(p + (j0 + e) * 32);
#pragma unroll
            for (int e = 0; e < 16 && j0 + e < 4 * NBLK; ++e) {
              acc2[j0 + e].x += v[e].x;
              acc2[j0 + e].y += v[e].y;
            }
            asm volatile("" ::: "memory");
          }
        }
        if (lane == 0) *counter = 0u;
      }
      // the accumulators already hold U L2 + b (added by the tile's first unit)
      if constexpr (Cfg::TMA_STORE) {
        // Stage 32 rows x 128 bytes at a time in this warp's buffer, in the
        // 128-byte swizzled layout (16-byte chunk c of row r at chunk c ^ (r % 8),
        // so the quad-layout writes hit distinct banks), then one TMA store of
        // that box; rows and columns outside Y are clipped by the TMA unit.
        uint8_t* stg = ystage + dw * 4096;
        const int y0 = tr * TILE_M + static_cast<int>(crank) * BM + q * 32;
        const int x0 = tc * BN + h * CW;
        if (!args.out_f32) {
#pragma unroll
          for (int pz = 0; pz < CW / 64; ++pz) {  // 8 blocks = 64 bf16 columns per box
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rl = qd + 8 * i;
#pragma unroll
              for (int kb = 0; kb < 8; ++kb) {
                const __nv_bfloat162 v = __float22bfloat162_rn(acc2[i * NBLK + 8 * pz + kb]);
                *reinterpret_cast<__nv_bfloat162*>(stg + rl * 128 + ((kb ^ (rl & 7)) << 4) + qc * 4) = v;
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && x0 + 64 * pz < args.N && y0 < args.M) {  // skip boxes wholly outside Y
              tma_store_2d(&tm_y, stg, x0 + 64 * pz, y0);
              bulk_commit_group();
            }
          }
        } else {
#pragma unroll
          for (int pz = 0; pz < CW / 32; ++pz) {  // 4 blocks = 32 fp32 columns per box
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rl = qd + 8 * i;
#pragma unroll
              for (int kb = 0; kb < 4; ++kb) {
                const int c16 = 2 * kb + (qc >> 1);  // 16-byte chunk of the row
                *reinterpret_cast<float2*>(stg + rl * 128 + ((c16 ^ (rl & 7)) << 4) + (qc & 1) * 8) =
                    acc2[i * NBLK + 4 * pz + kb];
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && x0 + 32 * pz < args.N && y0 < args.M) {
              tma_store_2d(&tm_y, stg, x0 + 32 * pz, y0);
              bulk_commit_group();
            }
          }
        }
      } else if (!Cfg::SWAP) {
        // rows are tokens m, columns are output features n
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = rbase + 8 * i;
          if (m >= args.rows_r) continue;
          const size_t rowoff = static_cast<size_t>(m) * args.N;
#pragma unroll
          for (int b = 0; b < NBLK; ++b) {
            const int n = col0 + 8 * b;
            if (n < args.N) {
              if (args.out_f32) *reinterpret_cast<float2*>(static_cast<float*>(args.Y) + rowoff + n) = acc2[i * NBLK + b];
              else *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(args.Y) + rowoff + n) =
                  __float22bfloat162_rn(acc2[i * NBLK + b]);
            }
          }
        }
      } else {
        // rows are output features n, columns are tokens m
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int n = rbase + 8 * i;
          if (n >= args.rows_r) continue;
#pragma unroll
          for (int b = 0; b < NBLK; ++b) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int m = col0 + 8 * b + e;
              if (m < args.M) {
                const float v = e ? acc2[i * NBLK + b].y : acc2[i * NBLK + b].x;
                const size_t off = static_cast<size_t>(m) * args.N + n;
                if (args.out_f32) static_cast<float*>(args.Y)[off] = v;
                else static_cast<__nv_bfloat16*>(args.Y)[off] = __float2bfloat16_rn(v);
              }
            }
          }
        }
      }
    }
    // the warp's TMA stores must be complete before the CTA's shared memory goes away
    if (Cfg::TMA_STORE && lane == 0) bulk_wait_all();
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    const WaitPolicy tail{args.limit_ns, tail_flag};
    if (warp == 0 && lane == 0) {
      // let every load still in flight land before the CTA's shared memory goes away
      // (pairs: operand bytes are counted on the even CTA's barriers only)
      const uint32_t first = issued > static_cast<uint32_t>(STAGES) ? issued - STAGES : 0u;
      if (leader)
        for (uint32_t i = first; i < issued; ++i) wait_one(&full[i % STAGES], (i / STAGES) & 1, tail);
      const uint32_t sfirst = issued > static_cast<uint32_t>(Cfg::SSLOTS) ? issued - Cfg::SSLOTS : 0u;
      if (!Cfg::ONE_PHASE)  // (with ONE_PHASE the scales land on the stage barriers waited above)
        for (uint32_t i = sfirst; i < issued; ++i)
          wait_one(&sfull[i % Cfg::SSLOTS], (i / Cfg::SSLOTS) & 1, tail);
    }
    if (warp == 1 && lane == 0 && leader) {
      // arrives once every MMA issued above has completed (pairs: the even CTA issues them)
      if constexpr (PAIR) mma_commit_pair(mapa_shared(smem_u32(final_bar), 0u));
      else mma_commit(final_bar);
      wait_one(final_bar, 0, tail);
    }
    __syncthreads();
  }
  if constexpr (PAIR) {
    // the pair's MMA completions are signalled to both CTAs' stage barriers:
    // let the last of them land before this CTA's shared memory goes away
    if (warp == 0 && lane == 0 && !*abort_flag) {
      const WaitPolicy tail{args.limit_ns, tail_flag};
      const uint32_t first = issued > static_cast<uint32_t>(STAGES) ? issued - STAGES : 0u;
      for (uint32_t i = first; i < issued; ++i) wait_one(&empty[i % STAGES], (i / STAGES) & 1, tail);
    }
    tc_fence_before();
    cluster_sync();  // both CTAs are done with the pair's Tensor Memory and barriers
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  } else if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

}  // namespace hsq
