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
  int rows_per_block;
  // fused form: the layer's input instead of x_codes / x_scales / U
  const __nv_bfloat16* X;   // [M][K]
  const float* s;           // [K]
  const __nv_bfloat16* L1;  // [K][r]
  int K, group;
};

constexpr int kGemvThreads = 512;
// 16-byte weight chunks per lane per batch (4 measured better than 8, which
// half-fills a batch when a row has 4 chunks per lane), and batches in flight
// (3 measured no better than 2)
constexpr int kGemvBatch = 4;
constexpr int kGemvDepth = 2;

// Shared memory of one block: widened activation codes (even and odd codes of
// every packed word, MT*Kp bytes), the activation scales [G][MT] and, fused, U
// [MT][4] with its per-warp partials [16][MT][4].
__host__ __device__ constexpr size_t gemv_smem_bytes(int MT, int Kp, int G) {
  return static_cast<size_t>(MT) * Kp + static_cast<size_t>(G) * MT * 4 + (kGemvThreads / 32 + 1) * MT * 4 * 4;
}

// MT: tokens the kernel is built for (M <= MT); LPG: lanes per scale group (a
// lane holds 32 codes, so 2 for groups of 64 and 4 for groups of 128); RF: -1
// reads the activation step's outputs, 0/1/2/4 is the fused form of that rank.
template <int MT, int LPG, int RF = -1>
__global__ void __launch_bounds__(kGemvThreads, 1) w4a4_gemv_kernel(const GemvArgs a) {
  extern __shared__ __align__(16) uint8_t gemv_smem[];
  const int W4 = a.Kp / 8;  // packed 32-bit words per row
  uint32_t* xlo = reinterpret_cast<uint32_t*>(gemv_smem);  // [MT][W4] even codes, int8 16*q
  uint32_t* xhi = xlo + MT * W4;                           // [MT][W4] odd codes
  float* sxs = reinterpret_cast<float*>(xhi + MT * W4);     // [G][MT]
  float* Us = sxs + a.G * MT;                               // fused: U [MT][4]
  float* upart = Us + MT * 4;                               // fused: [warp][MT][4]
  const int warp = threadIdx.x >> 5, lane = lane_id();
  const int nwarps = blockDim.x >> 5;
  const int nch = a.Kp / 32;  // 16-byte chunks per row (a multiple of LPG)
  const int n0 = blockIdx.x * a.rows_per_block;
  const int n1 = min(a.N, n0 + a.rows_per_block);
  // The warp's rows n0 + warp, + nwarps, ... are streamed as one sequence of
  // batches (kGemvBatch chunks per lane), kGemvDepth - 1 batches ahead of the
  // one in use, across row ends too.
  const int nrows = n1 > n0 + warp ? (n1 - n0 - warp + nwarps - 1) / nwarps : 0;
  const int bpr = (nch + 32 * kGemvBatch - 1) / (32 * kGemvBatch);  // batches per row
  const int total = nrows * bpr;
  // (a batch's weight scales are loaded with its codes: they are as far away)
  auto load = [&](int t, uint4 (&dst)[kGemvBatch], float (&dsw)[kGemvBatch]) {
    const int n = n0 + warp + (t / bpr) * nwarps;
    const int c0 = (t % bpr) * 32 * kGemvBatch;
    const uint4* wrow = reinterpret_cast<const uint4*>(a.w_codes + static_cast<size_t>(n) * (a.Kp / 2));
#pragma unroll
    for (int b = 0; b < kGemvBatch; ++b) {
      const int c = c0 + 32 * b + lane;
      dst[b] = c < nch ? __ldg(wrow + c) : make_uint4(0u, 0u, 0u, 0u);
      dsw[b] = c < nch ? __ldg(a.w_scales + static_cast<size_t>(c / LPG) * a.ldw + n) : 0.f;
    }
  };
  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.f;
  uint4 wb[kGemvDepth][kGemvBatch];
  float sb[kGemvDepth][kGemvBatch];
  // the packed weights are never written by the kernel just before this one (the
  // activation step), so the first batches are requested before waiting for it
#pragma unroll
  for (int d = 0; d + 1 < kGemvDepth; ++d)
    if (d < total) load(d, wb[d], sb[d]);
  grid_dep_wait();  // the activation codes (or X) come from the preceding kernel
  const float* Uv = a.U;  // U [M][r]: the activation step's, or this block's own (fused)
  if constexpr (RF < 0) {
    for (int i = threadIdx.x; i < MT * W4; i += blockDim.x) {
      const int m = i / W4, j = i - m * W4;
      uint32_t w = 0u;
      if (m < a.M) w = __ldg(reinterpret_cast<const unsigned int*>(a.x_codes + static_cast<size_t>(m) * (a.Kp / 2)) + j);
      xlo[i] = (w << 4) & 0xF0F0F0F0u;
      xhi[i] = w & 0xF0F0F0F0u;
    }
    for (int i = threadIdx.x; i < a.G * MT; i += blockDim.x) {
      const int g = i / MT, m = i - g * MT;
      sxs[i] = m < a.M ? __ldg(a.x_scales + static_cast<size_t>(g) * a.ldx + m) : 0.f;
    }
  } else {
    // the activation step: warp w takes (token, 256-channel chunk) pairs w, w + 16, ...;
    // a lane handles 8 channels, as in quantize_act_kernel
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
    ld(warp, rawn, s0n, s1n, l1n);
    for (int pc = warp; pc < MT * nchk; pc += nwarps) {
      const uint4 raw = rawn;
      const float4 s0 = s0n, s1 = s1n;
      uint4 l1c[RL];
#pragma unroll
      for (int v = 0; v < RL; ++v) l1c[v] = l1n[v];
      ld(pc + nwarps, rawn, s0n, s1n, l1n);
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
          if (lane == 0) upart[(warp * MT + m) * 4 + j] = v;
        }
      __syncthreads();
      if (threadIdx.x < MT * RF) {
        const int m = threadIdx.x / RF, j = threadIdx.x - (threadIdx.x / RF) * RF;
        float v = 0.f;
        for (int w = 0; w < nwarps; ++w) v += upart[(w * MT + m) * 4 + j];
        Us[m * RF + j] = v;
      }
    }
    Uv = Us;
  }
  __syncthreads();
  if (threadIdx.x == 0) grid_dep_launch();

  // one batch: its chunks' group partials, scaled, into acc; at a row's end the
  // low-rank branch (lane j adds U[m][j] L2[j][n]), the warp's sum, the bias, Y
  auto consume = [&](int t, const uint4 (&wv)[kGemvBatch], const float (&swv)[kGemvBatch]) {
    const int n = n0 + warp + (t / bpr) * nwarps;
    const int c0 = (t % bpr) * 32 * kGemvBatch;
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
    if ((t + 1) % bpr != 0) return;
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
      acc[m] = 0.f;
    }
  };
  // a ring of kGemvDepth batches: batch t + kGemvDepth - 1 is requested before batch t is used
  constexpr int kAhead = kGemvDepth - 1;
  for (int t0 = 0; t0 < total; t0 += kGemvDepth) {
#pragma unroll
    for (int d = 0; d < kGemvDepth; ++d) {
      const int t = t0 + d;
      if (t >= total) break;
      if (t + kAhead < total) load(t + kAhead, wb[(d + kAhead) % kGemvDepth], sb[(d + kAhead) % kGemvDepth]);
      consume(t, wb[d], sb[d]);
    }
  }
}

}  // namespace hsq
