// hsq_gemv.cuh -- the forward for a few tokens (M <= 8) as a weight stream on
// the CUDA cores.
//
// Computes the same layer as hsq_gemm.cuh (Deflating the Hessian, Abstract:
// 4-bit residual product plus the high-precision low-rank branch)
//     Y[m,n] = sum_g sx[g][m] sw[g][n] P_g[m,n] + sum_j U[m,j] L2[j,n] + b[n],
//     P_g[m,n] = sum_{k in group g} qx[m,k] qw[n,k]   (exact, int32)
// for M <= 8 tokens.  There the product is a matrix-vector stream: every weight
// byte is used for at most 16 multiply-adds, so the work is bound by reading the
// packed weights once, and a tensor-core tile (128 rows, its TMA/unpack/MMA/drain
// hand-offs per stage) only adds latency.  Here every warp streams whole weight
// rows with 16-byte loads (a warp reads 512 contiguous bytes per instruction);
// codes are widened in registers to int8 16*q (one AND or shift+AND per four
// codes, the same trick as the tensor-core unpack), and __dp4a forms the exact
// group partial 256*P_g in int32 (|256 P_g| <= 256 * 128 * 49 < 2^24, so its fp32
// conversion is exact).  The block's activation codes are widened the same way
// once into shared memory.  Each group partial is scaled by sx*sw in fp32, the
// low-rank branch and the bias are added, and the warp's sum is written.
//
// Fused form (RF >= 0, up to 4 tokens and rank 0, 1, 2 or 4): the block runs the
// activation step itself in its prologue -- X_hat = X/s, the group codes and
// scales, U = X_hat L1, with the same arithmetic as quantize_act_kernel, so the
// codes are the same bits -- straight into shared memory, so that a layer is one
// launch and nothing of the activation step goes through HBM.  Every block
// repeats that small step (M*K elements and K*r L1 values, from L2).
#pragma once

#include "hsq_device.cuh"
#include "hsq_quant.cuh"

namespace hsq {

struct GemvArgs {
  const uint8_t* x_codes;  // [M][Kp/2]
  const float* x_scales;   // [G][ldx]
  const float* U;          // [M][r]
  const uint8_t* w_codes;  // [N][Kp/2]
  const float* w_scales;   // [G][ldw]
  const __nv_bfloat16* L2;    // [r][N]
  const __nv_bfloat16* bias;  // [N] or nullptr
  void* Y;                    // [M][N]
  int ldx, ldw, r, out_f32;
  int M, N, Kp, G;
  int rows_per_block;  // a multiple of 4: the block's rows are n0 = block * rows_per_block ..
  // weight ring (GemvLayout): stages of rs whole rows, their byte offsets in shared memory
  int rs, stages;
  uint32_t off_sws, off_x, off_sxs, off_us, off_bars;
  uint64_t limit_ns;
  // fused form: the layer's input instead of x_codes / x_scales / U
  const __nv_bfloat16* X;   // [M][K]
  const float* s;           // [K]
  const __nv_bfloat16* L1;  // [K][r]
  int K, group;
};

// Block: warp 0 streams the weights (one elected lane issues bulk copies),
// warps 1..15 compute.
constexpr int kGemvThreads = 512;
constexpr int kGemvComputeWarps = kGemvThreads / 32 - 1;
// 16-byte weight chunks a lane reads from the ring per batch
constexpr int kGemvBatch = 4;
// smallest ring stage (whole rows; at least one row)
constexpr int kGemvStageBytes = 16384;
// most shared memory the ring may take, and into how many stages a block's rows
// are cut at most (before the ring's size limits them)
#ifndef HSQ_GEMV_RING_KB
#define HSQ_GEMV_RING_KB 224
#endif
#ifndef HSQ_GEMV_SPLIT
#define HSQ_GEMV_SPLIT 2
#endif

// Shared-memory layout of the weight stream for MT tokens, Kp codes per row, G
// scale groups and rows_per_block rows: the weight ring (stages of rs rows),
// the block's weight scales [G][rows_per_block], the widened activation codes
// (even and odd codes of every packed word, MT*Kp bytes), the activation scales
// [G][MT], U [MT][4], the per-warp U partials [16][MT][4] and the barriers.
struct GemvLayout {
  int rs, stages;
  uint32_t off_sws, off_x, off_sxs, off_us, off_bars, bytes;
};

__host__ __device__ constexpr uint32_t gemv_align16(size_t v) { return static_cast<uint32_t>((v + 15) / 16 * 16); }

// smem_max: the block's shared-memory limit; returns stages = 0 when not even
// two stages fit (one, if the block's rows fill only one), and the caller then
// takes another path.
inline GemvLayout gemv_layout(int MT, int Kp, int G, int rows_per_block, size_t smem_max) {
  GemvLayout L{};
  const int rowbytes = Kp / 2;
  const size_t fixed = gemv_align16(static_cast<size_t>(G) * rows_per_block * 4) +
                       gemv_align16(static_cast<size_t>(MT) * Kp) + gemv_align16(static_cast<size_t>(G) * MT * 4) +
                       gemv_align16(MT * 4 * 4) + gemv_align16((kGemvThreads / 32) * MT * 4 * 4);
  // the block's scales are one TMA box: at most 256 along each dimension
  if (rows_per_block > 256 || G > 256) return L;
  // Few, large stages: every stage is one bulk copy whose completion costs the
  // block a fixed ~800 cycles whatever its size, so the block's rows come in
  // about two copies (half of them each, or half the ring when that is smaller).
  size_t budget = smem_max > fixed + 1024 ? smem_max - fixed - 1024 : 0;  // 1024: barriers, rounding
  if (budget > static_cast<size_t>(HSQ_GEMV_RING_KB) * 1024) budget = static_cast<size_t>(HSQ_GEMV_RING_KB) * 1024;
  size_t target = static_cast<size_t>(rows_per_block) * rowbytes / HSQ_GEMV_SPLIT;
  if (target > budget / 2) target = budget / 2;
  if (target < static_cast<size_t>(kGemvStageBytes)) target = kGemvStageBytes;
  L.rs = static_cast<int>(target / rowbytes);
  if (L.rs < 1) L.rs = 1;
  if (L.rs > rows_per_block) L.rs = rows_per_block;
  const size_t stage = static_cast<size_t>(L.rs) * rowbytes;
  const int need = (rows_per_block + L.rs - 1) / L.rs;  // stages the block's rows fill
  int st = static_cast<int>(budget / stage);
  if (st > need) st = need;
  if (st > 32) st = 32;
  L.stages = (st >= 2 || (st >= 1 && need == 1)) ? st : 0;
  size_t off = gemv_align16(static_cast<size_t>(L.stages) * stage);
  L.off_sws = static_cast<uint32_t>(off);
  off += gemv_align16(static_cast<size_t>(G) * rows_per_block * 4);
  L.off_x = static_cast<uint32_t>(off);
  off += gemv_align16(static_cast<size_t>(MT) * Kp);
  L.off_sxs = static_cast<uint32_t>(off);
  off += gemv_align16(static_cast<size_t>(G) * MT * 4);
  L.off_us = static_cast<uint32_t>(off);
  off += gemv_align16(MT * 4 * 4) + gemv_align16((kGemvThreads / 32) * MT * 4 * 4);
  L.off_bars = static_cast<uint32_t>(off);
  off += (2 * 32 + 2) * 8;
  L.bytes = static_cast<uint32_t>(off);
  return L;
}

// Named barrier of the compute warps (the producer warp does not take part).
__device__ __forceinline__ void gemv_compute_sync() { named_bar_sync(1, kGemvComputeWarps * 32); }

// MT: tokens the kernel is built for (M <= MT); LPG: lanes per scale group (a
// lane holds 32 codes, so 2 for groups of 64 and 4 for groups of 128); RF: -1
// reads the activation step's outputs, 0/1/2/4 is the fused form of that rank.
template <int MT, int LPG, int RF = -1>
__global__ void __launch_bounds__(kGemvThreads, 1)
    w4a4_gemv_kernel(const __grid_constant__ CUtensorMap tm_sw, const GemvArgs a) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  const int W4 = a.Kp / 8;  // packed 32-bit words per row
  const int rowbytes = a.Kp / 2;
  const int RB = a.rows_per_block;
  uint8_t* ring = gemv_smem;
  float* sws = reinterpret_cast<float*>(gemv_smem + a.off_sws);            // [G][RB]
  uint32_t* xlo = reinterpret_cast<uint32_t*>(gemv_smem + a.off_x);        // [MT][W4] even codes, int8 16*q
  uint32_t* xhi = xlo + MT * W4;                                           // [MT][W4] odd codes
  float* sxs = reinterpret_cast<float*>(gemv_smem + a.off_sxs);            // [G][MT]
  float* Us = reinterpret_cast<float*>(gemv_smem + a.off_us);              // fused: U [MT][4]
  float* upart = Us + MT * 4;                                              // fused: [warp][MT][4]
  uint64_t* full = reinterpret_cast<uint64_t*>(gemv_smem + a.off_bars);    // [stages] rows landed
  uint64_t* empty = full + 32;                                             // [stages] rows consumed
  uint64_t* sfull = empty + 32;                                            // the block's weight scales landed
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sfull + 1);
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int nch = a.Kp / 32;  // 16-byte chunks per row (a multiple of LPG)
  const int n0 = blockIdx.x * RB;
  const int nrows = min(a.N, n0 + RB) - n0;
  const int nst = (nrows + a.rs - 1) / a.rs;  // stages of this block
  const WaitPolicy wp{a.limit_ns, abort_flag};

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kGemvComputeWarps);  // every compute warp arrives once per stage
    }
    mbar_init(sfull, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  uint32_t issued = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ weight stream
    // The packed weights and their scales are never written by the kernel just
    // before this one, so they are requested before waiting for it: the block's
    // scales as one 2-D box of [G][RB] floats (rows past the matrix read as 0),
    // then its rows, a stage of rs contiguous rows per bulk copy, as far ahead as
    // the ring allows.
    if (lane == 0) {
      prefetch_tensormap(&tm_sw);
      mbar_arrive_expect_tx(sfull, static_cast<uint32_t>(RB) * a.G * 4u);
      tma_load_2d(sws, &tm_sw, sfull, n0, 0);
      for (int it = 0; it < nst; ++it) {
        const int s = it % a.stages;
        if (it >= a.stages && !wait_one(&empty[s], ((it / a.stages) & 1) ^ 1, wp)) break;
        const int rows = min(a.rs, nrows - it * a.rs);
        const uint32_t bytes = static_cast<uint32_t>(rows) * rowbytes;
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_load(ring + static_cast<size_t>(s) * a.rs * rowbytes,
                  a.w_codes + static_cast<size_t>(n0 + it * a.rs) * rowbytes, bytes, &full[s]);
        issued = it + 1;
      }
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int cw = warp - 1;
    const int ct = threadIdx.x - 32;
    grid_dep_wait();  // the activation codes (or X) come from the preceding kernel
    const float* Uv = a.U;  // U [M][r]: the activation step's, or this block's own (fused)
    if constexpr (RF < 0) {
      for (int i = ct; i < MT * W4; i += kGemvComputeWarps * 32) {
        const int m = i / W4, j = i - m * W4;
        uint32_t w = 0u;
        if (m < a.M) w = __ldg(reinterpret_cast<const unsigned int*>(a.x_codes + static_cast<size_t>(m) * (a.Kp / 2)) + j);
        xlo[i] = (w << 4) & 0xF0F0F0F0u;
        xhi[i] = w & 0xF0F0F0F0u;
      }
      for (int i = ct; i < a.G * MT; i += kGemvComputeWarps * 32) {
        const int g = i / MT, m = i - g * MT;
        sxs[i] = m < a.M ? __ldg(a.x_scales + static_cast<size_t>(g) * a.ldx + m) : 0.f;
      }
    } else {
      // the activation step: compute warp cw takes (token, 256-channel chunk)
      // pairs cw, cw + 15, ...; a lane handles 8 channels, as in quantize_act_kernel
      constexpr int RA = RF > 0 ? RF : 1;
      const int nchk = (a.Kp + 255) / 256;
      float u[MT][RA];
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < RA; ++j) u[m][j] = 0.f;
      // a chunk's X row, smoothing factors and L1 rows are requested one chunk ahead
      constexpr int RL = RF > 0 ? RF : 1;
      auto ld = [&](int pc, uint4& raw, float4& s0, float4& s1, uint4 (&l1)[RL]) {
        const bool live = pc < MT * nchk;
        const int m = live ? pc / nchk : 0;
        const int k0 = (live ? pc - m * nchk : 0) * 256 + lane * 8;
        const bool real = live && m < a.M && k0 < a.K;
        s0 = real ? __ldg(reinterpret_cast<const float4*>(a.s + k0)) : make_float4(1.f, 1.f, 1.f, 1.f);
        s1 = real ? __ldg(reinterpret_cast<const float4*>(a.s + k0 + 4)) : make_float4(1.f, 1.f, 1.f, 1.f);
        raw = real ? __ldg(reinterpret_cast<const uint4*>(a.X + static_cast<size_t>(m) * a.K + k0))
                   : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int v = 0; v < RF; ++v)
          l1[v] = real ? __ldg(reinterpret_cast<const uint4*>(a.L1 + static_cast<size_t>(k0) * RF) + v)
                       : make_uint4(0u, 0u, 0u, 0u);
      };
      uint4 rawn, l1n[RL];
      float4 s0n, s1n;
      ld(cw, rawn, s0n, s1n, l1n);
      for (int pc = cw; pc < MT * nchk; pc += kGemvComputeWarps) {
        const uint4 raw = rawn;
        const float4 s0 = s0n, s1 = s1n;
        uint4 l1c[RL];
#pragma unroll
        for (int v = 0; v < RL; ++v) l1c[v] = l1n[v];
        ld(pc + kGemvComputeWarps, rawn, s0n, s1n, l1n);
        const int m = pc / nchk, c = pc - (pc / nchk) * nchk;  // warp-uniform
        const int k0 = c * 256 + lane * 8;
        const bool real = m < a.M && k0 < a.K;  // K % 8 == 0: all 8 channels real or all padding
        const bool in_k = k0 < a.Kp;
        const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
        float sz[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) sz[e] = __frcp_rn(sv[e]);
        float xh[8];
        smooth8(raw, sv, sz, real, xh);
        float sc;
        const uint32_t packed = LPG == 2 ? quantize8_fast<8>(xh, sc) : quantize8_fast<16>(xh, sc);
        if (in_k) {
          const int j = k0 / 8;  // the lane's packed word
          xlo[m * W4 + j] = (packed << 4) & 0xF0F0F0F0u;
          xhi[m * W4 + j] = packed & 0xF0F0F0F0u;
          if ((lane & (4 * LPG - 1)) == 0) sxs[(k0 / a.group) * MT + m] = sc;  // (0 for padding rows)
        }
        if constexpr (RF > 0) {
          // the 8 channels' L1 rows (8*RF bf16, contiguous; zero for padding)
#pragma unroll
          for (int v = 0; v < RF; ++v) {
            float f[8];
            bf16x8_to_f32(l1c[v], f);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const int e = (v * 8 + t) / RF, jr = (v * 8 + t) % RF;
#pragma unroll
              for (int mm = 0; mm < MT; ++mm)
                if (mm == m) u[mm][jr] = fmaf(xh[e], f[t], u[mm][jr]);
            }
          }
        }
      }
      if constexpr (RF > 0) {
        // U: lanes, then warps in a fixed order
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
          for (int j = 0; j < RF; ++j) {
            float v = u[m][j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) upart[(cw * MT + m) * 4 + j] = v;
          }
        gemv_compute_sync();
        if (ct < MT * RF) {
          const int m = ct / RF, j = ct - (ct / RF) * RF;
          float v = 0.f;
          for (int w = 0; w < kGemvComputeWarps; ++w) v += upart[(w * MT + m) * 4 + j];
          Us[m * RF + j] = v;
        }
      }
      Uv = Us;
    }
    gemv_compute_sync();
    if (ct == 0) grid_dep_launch();

    // the block's weight scales
    bool ok = wait_warp(sfull, 0, wp);
    // Rows cw, cw + 15, ... of the block, each read from the ring: its chunks'
    // group partials (dp4a of int8 16*q, exact), scaled, into acc; at the row's
    // end the low-rank branch (lane j adds U[m][j] L2[j][n]), the warp's sum, the
    // bias, Y.  Every warp waits for every stage in order and arrives on its
    // release once, also for stages that hold none of its rows: a parity wait is
    // only sound if the waiter has seen the slot's previous use land and the
    // slot cannot be refilled twice before the waiter looks (with the ring
    // reusing slots, a warp that skipped a phase could pass a wait one use early,
    // or miss a use and wait for one two ahead).
    for (int it = 0; ok && it < nst; ++it) {
      const int s = it % a.stages;
      if (!wait_warp(&full[s], (it / a.stages) & 1, wp)) { ok = false; break; }
      const int r0 = it * a.rs, r1 = min(nrows, r0 + a.rs);
      for (int i = r0 + (cw - r0 % kGemvComputeWarps + kGemvComputeWarps) % kGemvComputeWarps; i < r1;
           i += kGemvComputeWarps) {
      const uint4* wrow = reinterpret_cast<const uint4*>(ring + (static_cast<size_t>(s) * a.rs + (i - it * a.rs)) * rowbytes);
      const int n = n0 + i;
      float acc[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.f;
      for (int c0 = 0; c0 < nch; c0 += 32 * kGemvBatch) {
        uint4 wv[kGemvBatch];
        float swv[kGemvBatch];
#pragma unroll
        for (int b = 0; b < kGemvBatch; ++b) {
          const int c = c0 + 32 * b + lane;
          wv[b] = c < nch ? wrow[c] : make_uint4(0u, 0u, 0u, 0u);
          swv[b] = c < nch ? sws[(c / LPG) * RB + i] : 0.f;
        }
#pragma unroll
        for (int b = 0; b < kGemvBatch; ++b) {
          if (c0 + 32 * b >= nch) break;  // warp-uniform
          const int c = c0 + 32 * b + lane;
          const bool valid = c < nch;  // the LPG lanes of a group agree
          const int g = c / LPG;
          const uint32_t w[4] = {wv[b].x, wv[b].y, wv[b].z, wv[b].w};
          int wl[4], wh[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            wl[j] = static_cast<int>((w[j] << 4) & 0xF0F0F0F0u);  // even codes, 16*q
            wh[j] = static_cast<int>(w[j] & 0xF0F0F0F0u);         // odd codes, 16*q
          }
          const int cc = valid ? c : 0;
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            const uint4 l = *reinterpret_cast<const uint4*>(xlo + m * W4 + 4 * cc);
            const uint4 h = *reinterpret_cast<const uint4*>(xhi + m * W4 + 4 * cc);
            int p = __dp4a(wl[0], static_cast<int>(l.x), 0);
            p = __dp4a(wl[1], static_cast<int>(l.y), p);
            p = __dp4a(wl[2], static_cast<int>(l.z), p);
            p = __dp4a(wl[3], static_cast<int>(l.w), p);
            p = __dp4a(wh[0], static_cast<int>(h.x), p);
            p = __dp4a(wh[1], static_cast<int>(h.y), p);
            p = __dp4a(wh[2], static_cast<int>(h.z), p);
            p = __dp4a(wh[3], static_cast<int>(h.w), p);
#pragma unroll
            for (int o = 1; o < LPG; o <<= 1) p += __shfl_xor_sync(0xffffffffu, p, o);  // 256 * P_g
            if (valid && (lane & (LPG - 1)) == 0)
              acc[m] = fmaf(static_cast<float>(p) * (1.0f / 256.0f), sxs[g * MT + m] * swv[b], acc[m]);
          }
        }
      }
      if (lane < a.r) {
        const float l2 = __bfloat162float(a.L2[static_cast<size_t>(lane) * a.N + n]);
#pragma unroll
        for (int m = 0; m < MT; ++m)
          if (m < a.M) acc[m] = fmaf(Uv[m * a.r + lane], l2, acc[m]);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], o);
      const float bn = a.bias ? __bfloat162float(a.bias[n]) : 0.f;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (lane == m && m < a.M) {
          const float y = acc[m] + bn;
          const size_t off = static_cast<size_t>(m) * a.N + n;
          if (a.out_f32) static_cast<float*>(a.Y)[off] = y;
          else static_cast<__nv_bfloat16*>(a.Y)[off] = __float2bfloat16_rn(y);
        }
      }
      }  // rows of this stage
      __syncwarp();  // every lane's ring reads of the stage are done
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag && warp == 0 && lane == 0) {
    // let the copies still in flight land before the block's shared memory goes away
    volatile int tail = 0;
    const WaitPolicy tp{a.limit_ns, &tail};
    wait_one(sfull, 0, tp);
    const uint32_t first = issued > static_cast<uint32_t>(a.stages) ? issued - a.stages : 0u;
    for (uint32_t i = first; i < issued; ++i) wait_one(&full[i % a.stages], (i / a.stages) & 1, tp);
  }
}

}  // namespace hsq
