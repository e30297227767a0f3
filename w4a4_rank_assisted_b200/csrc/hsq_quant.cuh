// hsq_quant.cuh -- the two quantizing kernels: offline weight packing and the
// fused per-forward activation step.
//
// Quantizer (Deflating the Hessian, Abstract: 4-bit weights and activations;
// Table 1 caption: groups of 64 along K; Table 3 and Table 4 captions: groups of
// 128 for the Qwen3-8B results): symmetric signed INT4 with one fp32 scale per
// group, scale = absmax / 7 (IEEE division), code = round-half-even(v / scale)
// clamped to [-7, 7].  Both kernels give every lane 8 consecutive K-elements, so
// a group spans GL = group/8 adjacent lanes (8 or 16) and its absmax is a
// log2(GL)-step xor-shuffle reduction.
#pragma once

#include "hsq_device.cuh"

namespace hsq {

// Absmax of a group spread over GL adjacent lanes (8 values each): GL = 8 for
// groups of 64, 16 for groups of 128.  Every lane of the warp must call it.
template <int GL>
__device__ __forceinline__ float group_absmax(const float (&v)[8]) {
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
#pragma unroll
  for (int o = 1; o < GL; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  return amax;
}

// Quantize one lane's 8 values of a group spread over GL adjacent lanes.
// Every lane of the warp must call this (it shuffles).  Returns the 8 codes
// packed as 4 bytes (code e in bits 4e..4e+3) and the group's scale.
template <int GL>
__device__ __forceinline__ uint32_t quantize8(const float (&v)[8], float& scale) {
  const float amax = group_absmax<GL>(v);
  scale = __fdiv_rn(amax, 7.0f);
  uint32_t packed = 0;
  if (scale != 0.f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int q = __float2int_rn(__fdiv_rn(v[e], scale));
      q = max(-7, min(7, q));
      packed |= static_cast<uint32_t>(q & 0xF) << (4 * e);
    }
  }
  return packed;
}

// x / y rounded to nearest-even, given z = RN(1/y): one product and Markstein's
// fused-multiply-add correction, q1 = RN(q + z (x - q y)) with the remainder
// x - q y exact (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990).  The result
// equals the IEEE quotient for normal x, y and a normal, finite quotient; very
// small or very large inputs take the ordinary division.  The tests compare every code and scale it
// decides against the oracle's IEEE division.
__device__ __forceinline__ float div_by_recip(float x, float y, float z) {
  const float ax = fabsf(x);
  if (ax < 0x1p-100f || ax > 0x1p100f) return __fdiv_rn(x, y);
  const float q = __fmul_rn(x, z);
  const float r = __fmaf_rn(-q, y, x);
  return __fmaf_rn(r, z, q);
}

// X_hat = x / s for a lane's 8 channels (bf16 x, fp32 s and its reciprocal z):
// product and correction, exact for normal operands and quotients and for
// x = 0; the warp takes the guarded division only if some lane holds an element
// outside [2^-100, 2^100].  Padding channels (real = false) give 0.  Every lane
// of the warp must call it (it votes).
__device__ __forceinline__ void smooth8(const uint4& raw, const float (&sv)[8], const float (&sz)[8], bool real,
                                        float (&xh)[8]) {
  float x[8];
  bf16x8_to_f32(raw, x);
  bool odd = false;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float ax = fabsf(x[e]);
    odd |= (ax != 0.f) & ((ax < 0x1p-100f) | (ax > 0x1p100f));
    const float q0 = __fmul_rn(x[e], sz[e]);
    xh[e] = __fmaf_rn(__fmaf_rn(-q0, sv[e], x[e]), sz[e], q0);
  }
  if (__any_sync(0xffffffffu, odd)) {
#pragma unroll
    for (int e = 0; e < 8; ++e) xh[e] = div_by_recip(x[e], sv[e], sz[e]);
  }
  if (!real) {
#pragma unroll
    for (int e = 0; e < 8; ++e) xh[e] = 0.f;
  }
}

// Round-half-even of |t| < 2^22 to an integer: add 1.5*2^23 (the sum's last
// mantissa bit is then the units place) and read the integer from the bits.
__device__ __forceinline__ int rint_small(float t) {
  return __float_as_int(__fadd_rn(t, 12582912.0f)) - 0x4B400000;
}

// Same result as quantize8, with the per-element divisions by the group scale
// done as one product and Markstein's correction against one reciprocal per
// group.  With the scale in [2^-100, 2^100] no element needs the guarded
// division: |v| <= 7 scale keeps the quotient and the remainder normal, and an
// element below 2^-126 has a quotient below 2^-26, which rounds to code 0 either
// way.  Nor does a code need clamping: scale = RN(absmax / 7) makes |v / scale|
// at most 7 (1 + 2^-24), which rounds to 7.  The code's 4-bit two's complement
// is read straight from the bits of t + 1.5 * 2^23 (its offset 0x4B400000 is a
// multiple of 16).
template <int GL>
__device__ __forceinline__ uint32_t quantize8_fast(const float (&v)[8], float& scale) {
  const float amax = group_absmax<GL>(v);
  scale = __fdiv_rn(amax, 7.0f);
  uint32_t packed = 0;
  if (scale >= 0x1p-100f && scale <= 0x1p100f) {
    const float z = __frcp_rn(scale);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float q0 = __fmul_rn(v[e], z);
      const float t = __fmaf_rn(__fmaf_rn(-q0, scale, v[e]), z, q0);
      packed |= (static_cast<uint32_t>(__float_as_int(__fadd_rn(t, 12582912.0f))) & 0xFu) << (4 * e);
    }
  } else if (scale != 0.f) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      int q = __float2int_rn(__fdiv_rn(v[e], scale));
      q = max(-7, min(7, q));
      packed |= static_cast<uint32_t>(q & 0xF) << (4 * e);
    }
  }
  return packed;
}

// NVFP4 (the DiRotQ page's FP4 setting: E2M1 values, one E4M3 scale per 16
// values, and one fp32 scale g per tensor).  One lane's 8 values of a 16-value
// block that spans two adjacent lanes: the block scale is the E4M3 byte
// b = RN_sat(fp32(blockmax / sixg)), sixg = fp32(6 g); each code is the E2M1
// rounding of fp32(v / fp32(b g)).  A zero g or a zero block scale gives codes
// 0.  Returns the 8 codes (code e in bits 4e..4e+3) and sets `sf` to b.  Every
// lane of the warp must call it (it shuffles).
__device__ __forceinline__ uint32_t quantize8_nvfp4(const float (&v)[8], float g, float sixg, uint32_t& sf) {
  float bmax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) bmax = fmaxf(bmax, fabsf(v[e]));
  bmax = fmaxf(bmax, __shfl_xor_sync(0xffffffffu, bmax, 1));
  sf = 0u;
  if (g == 0.f) return 0u;
  sf = f32_to_e4m3_rn_sat(__fdiv_rn(bmax, sixg));
  const float denom = __fmul_rn(e4m3_to_f32(sf), g);
  if (denom == 0.f) return 0u;
  float t[8];
  if (denom >= 0x1p-100f && denom <= 0x1p100f) {
    const float z = __frcp_rn(denom);
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = div_by_recip(v[e], denom, z);
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) t[e] = __fdiv_rn(v[e], denom);
  }
  return f32x8_to_e2m1(t);
}

// The per-tensor NVFP4 scale from the tensor's absmax: g = fp32(amax / 2688)
// (2688 = 6 * 448: the largest E2M1 magnitude times the largest E4M3 scale).
__device__ __forceinline__ float nvfp4_tensor_scale(float amax) { return __fdiv_rn(amax, 2688.0f); }

// Byte offset of the scale word of matrix row `row` and 64-wide K chunk `kc` in
// the NVFP4 scale layout: atoms of 128 rows x 64 K (512 bytes) ordered
// [row tile][K chunk]; inside an atom, row i's four block scales form the
// 32-bit word at 16 (i % 32) + 4 (i / 32).
__device__ __forceinline__ size_t nvfp4_sf_word_offset(int row, int kc, int kchunks) {
  return (static_cast<size_t>(row >> 7) * kchunks + kc) * 512 + 16 * (row & 31) + 4 * ((row & 127) >> 5);
}

// Gather the block-scale bytes of lanes 8p, 8p+2, 8p+4, 8p+6 (the four 16-value
// blocks of a 64-wide K chunk) into one word on lane 8p.  Every lane calls it.
__device__ __forceinline__ uint32_t gather_sf_word(uint32_t sf) {
  const uint32_t b1 = __shfl_down_sync(0xffffffffu, sf, 2);
  const uint32_t b2 = __shfl_down_sync(0xffffffffu, sf, 4);
  const uint32_t b3 = __shfl_down_sync(0xffffffffu, sf, 6);
  return sf | (b1 << 8) | (b2 << 16) | (b3 << 24);
}

// Zero the scale words of rows [rows, rows_pad) (rows_pad: rows rounded up to
// 128) in every K chunk of an NVFP4 scale matrix.
__global__ void nvfp4_zero_sf_pad_kernel(uint8_t* sf, int rows, int kchunks) {
  const int pad = ((rows + 127) & ~127) - rows;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < pad * kchunks) {
    const int row = rows + i / kchunks, kc = i % kchunks;
    *reinterpret_cast<uint32_t*>(sf + nvfp4_sf_word_offset(row, kc, kchunks)) = 0u;
  }
}

// Absmax of the smoothed activations X_hat = fp32(X)/s over the whole tensor
// (the NVFP4 tensor scale's input), as the same quotients the quantizer forms;
// folded into gs[1] (zeroed before the launch) with an integer atomicMax on the
// float's bits (valid for values >= 0).  Warps stride over 8-element groups.
__global__ void __launch_bounds__(256) nvfp4_act_amax_kernel(const __nv_bfloat16* __restrict__ X,
                                                             const float* __restrict__ s, int M, int K,
                                                             float* gs) {
  grid_dep_wait();  // X may come from the preceding kernel
  const int lane = lane_id();
  const size_t groups = static_cast<size_t>(M) * (K / 8);
  // block b takes a contiguous run of 8-element groups
  const size_t per_block = (groups + gridDim.x - 1) / gridDim.x;
  const size_t g0 = static_cast<size_t>(blockIdx.x) * per_block;
  const size_t g1 = min(groups, g0 + per_block);
  float amax = 0.f;
  for (size_t base = g0 + (threadIdx.x >> 5) * 32; base < g1; base += (blockDim.x / 32) * 32) {
    const size_t i = base + lane;
    const bool valid = i < g1;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    float sv[8], sz[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sv[e] = 1.f;
    if (valid) {
      const int m = static_cast<int>(i / (K / 8)), k0 = static_cast<int>(i % (K / 8)) * 8;
      raw = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k0));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
      sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
      sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sz[e] = __frcp_rn(sv[e]);
    float xh[8];
    smooth8(raw, sv, sz, valid, xh);
#pragma unroll
    for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(xh[e]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0 && amax > 0.f) atomicMax(reinterpret_cast<unsigned int*>(gs + 1), __float_as_uint(amax));
}

// The same absmax from column maxima: max over (m, k) of RN(|x[m,k]| / s[k]) is
// max over k of RN(max_m |x[m,k]| / s[k]), because a correctly rounded quotient
// does not decrease as its dividend grows (s > 0).  Block b takes a run of rows;
// each thread keeps the packed bf16 maxima of |x| over those rows for its 8
// channels at a time, then divides them by s (IEEE) and folds the block's
// maximum into gs[1] as nvfp4_act_amax_kernel does.
__global__ void __launch_bounds__(128) nvfp4_act_colmax_kernel(const __nv_bfloat16* __restrict__ X,
                                                               const float* __restrict__ s, int M, int K,
                                                               int rows_per_block, float* gs) {
  grid_dep_wait();  // X may come from the preceding kernel
  const int m0 = blockIdx.x * rows_per_block, m1 = min(M, m0 + rows_per_block);
  float amax = 0.f;
  for (int cg = threadIdx.x; cg < K / 8; cg += blockDim.x) {
    __nv_bfloat162 mx[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) mx[i] = __floats2bfloat162_rn(0.f, 0.f);
    const uint4* col = reinterpret_cast<const uint4*>(X + static_cast<size_t>(m0) * K) + cg;
    const size_t stride = K / 8;
    int m = m0;
    for (; m + 8 <= m1; m += 8, col += 8 * stride) {  // eight independent loads in flight
      uint4 raw[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) raw[j] = __ldg(col + j * stride);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = __hmax2(mx[i], __habs2(h[i]));
      }
    }
    for (; m < m1; ++m, col += stride) {
      const uint4 raw = __ldg(col);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = __hmax2(mx[i], __habs2(h[i]));
    }
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + cg * 8));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + cg * 8 + 4));
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(mx[i]);
      amax = fmaxf(amax, __fdiv_rn(f.x, sv[2 * i]));
      amax = fmaxf(amax, __fdiv_rn(f.y, sv[2 * i + 1]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0 && amax > 0.f) atomicMax(reinterpret_cast<unsigned int*>(gs + 1), __float_as_uint(amax));
}

// Rows [rows, rows_pad) of an E4M3 tile layout (that of expand_e4m3_kernel:
// [Kp/64][rows_pad/8][4 chunks][8 rows][16 B]) set to zero codes: one thread per
// (64-block, padding row, chunk), 16 bytes each.
__global__ void zero_e4m3_rows_kernel(uint8_t* __restrict__ xe, int rows, int rows_pad, int Kp) {
  grid_dep_wait();
  const int pad = rows_pad - rows;
  const size_t total = static_cast<size_t>(Kp / 64) * pad * 4;
  for (size_t t = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < total;
       t += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int chunk = static_cast<int>(t & 3);
    const int row = rows + static_cast<int>((t >> 2) % pad);
    const size_t blk = (t >> 2) / pad;
    *reinterpret_cast<uint4*>(xe + ((blk * (rows_pad / 8) + (row >> 3)) * 4 + chunk) * 128 + (row & 7) * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  if (threadIdx.x == 0) grid_dep_launch();
}

// ---------------------------------------------------------------------------
// Weight packing (offline): R[n,k] = fp32(W[n,k]*s[k] - sum_j L1[k,j]*L2[j,n]),
// the sum in fp64 for j = 0..r-1 with every multiply and add rounded on its own
// (no fused multiply-add), then quantized.  One warp per output row n.
// ---------------------------------------------------------------------------
// MODE 0: INT4 codes and fp32 group scales (GL lanes per group).
// MODE 1 (NVFP4, first pass): only the absmax of R, folded into gs[1].
// MODE 2 (NVFP4, second pass): E2M1 codes and E4M3 block scales (scale layout of
//   nvfp4_sf_word_offset, `scales` taken as its bytes) with g from gs[1]; the
//   first warp writes g to gs[0].
template <int GL, int MODE = 0>
__global__ void __launch_bounds__(256) pack_weights_kernel(const __nv_bfloat16* __restrict__ W,
                                                           const float* __restrict__ s,
                                                           const __nv_bfloat16* __restrict__ L1,
                                                           const __nv_bfloat16* __restrict__ L2, int N,
                                                           int K, int r, int Kp, int ld,
                                                           uint8_t* __restrict__ codes,
                                                           float* __restrict__ scales, float* gs = nullptr) {
  const int n = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = lane_id();
  if (n >= N) return;  // warp-uniform
  float g = 0.f, sixg = 0.f, amax = 0.f;
  if constexpr (MODE == 2) {
    g = nvfp4_tensor_scale(gs[1]);
    sixg = __fmul_rn(6.0f, g);
    if (n == 0 && lane == 0) gs[0] = g;
  }
  for (int c0 = 0; c0 < Kp; c0 += 256) {
    const int k0 = c0 + lane * 8;
    float R[8];
    if (k0 < K) {  // K % 8 == 0: all 8 elements are real
      const uint4 wraw = __ldg(reinterpret_cast<const uint4*>(W + static_cast<size_t>(n) * K + k0));
      float w[8];
      bf16x8_to_f32(wraw, w);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int k = k0 + e;
        double lr = 0.0;
        for (int j = 0; j < r; ++j) {
          const double a = static_cast<double>(__bfloat162float(L1[static_cast<size_t>(k) * r + j]));
          const double b = static_cast<double>(__bfloat162float(L2[static_cast<size_t>(j) * N + n]));
          lr = __dadd_rn(lr, __dmul_rn(a, b));
        }
        const double what = __dmul_rn(static_cast<double>(w[e]), static_cast<double>(__ldg(s + k)));
        R[e] = __double2float_rn(__dsub_rn(what, lr));
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) R[e] = 0.f;
    }
    if constexpr (MODE == 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(R[e]));
    } else if constexpr (MODE == 2) {
      uint32_t sf;
      const uint32_t packed = quantize8_nvfp4(R, g, sixg, sf);
      const uint32_t word = gather_sf_word(sf);
      if (k0 < Kp) {
        *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(n) * (Kp / 2) + k0 / 2) = packed;
        if ((lane & 7) == 0)
          *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(scales) +
                                       nvfp4_sf_word_offset(n, k0 / 64, Kp / 64)) = word;
      }
    } else {
      float sc;
      const uint32_t packed = quantize8<GL>(R, sc);
      if (k0 < Kp) {
        *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(n) * (Kp / 2) + k0 / 2) = packed;
        if ((lane & (GL - 1)) == 0) scales[static_cast<size_t>(k0 / (8 * GL)) * ld + n] = sc;
      }
    }
  }
  if constexpr (MODE == 1) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0 && amax > 0.f) atomicMax(reinterpret_cast<unsigned int*>(gs + 1), __float_as_uint(amax));
  }
}

// Zero the padding entries [rows, ld) of every group row of a scale matrix.
__global__ void zero_scale_pad_kernel(float* scales, int rows, int ld, int G) {
  const int pad = ld - rows;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < pad * G) scales[static_cast<size_t>(i / pad) * ld + rows + (i % pad)] = 0.f;
}

// ---------------------------------------------------------------------------
// Fused activation step: X_hat = fp32(X)/s (IEEE division), its group codes and
// scales, and U = X_hat L1 accumulated in fp32.
//
// A block of NW warps owns RB consecutive token rows, split into sub-blocks of
// SUB rows.  Warp w works on sub-block w % (RB/SUB) and on the 256-wide K chunks
// w / (RB/SUB), + NW/(RB/SUB), ...  Per chunk a lane loads the smoothing factors
// of its 8 channels once and reuses them for the SUB rows, whose X loads are
// issued together (one chunk ahead).
//
// U = X_hat L1 takes one of two forms.  Ranks up to 4: a lane keeps the L1 rows
// of its 8 channels in registers and accumulates all r columns.  Ranks of 8 and
// more: the warp parks its SUB rows of X_hat in shared memory, and the lanes are
// regrouped so that lane (kq, p) owns the rank pair (2p, 2p+1) of the channels
// kq, kq + KP, kq + 2 KP, ... of the chunk; each L1 load of the warp is then one
// contiguous run of KP rows of L1, applied to the SUB rows with packed fp32 FMAs.
// U is reduced across lanes with shuffles and across warps through shared
// memory in a fixed order, so the result does not depend on scheduling.  Small
// M uses NW = 16 warps on one sub-block so that K is spread over the whole block.
//
// R is the rank as a compile-time constant (1, 2, 4, 8, 16, 32, or 0 for no
// branch); R = -1 is the generic path for any other r <= 32 (two 2-byte L1 loads
// per rank pair).
// ---------------------------------------------------------------------------
template <int R, bool SMALL>
struct ActCfg {
  static constexpr int RMAX = R < 0 ? 32 : R;  // accumulator width
  static constexpr int SUB = SMALL ? 2 : 4;
  static constexpr int NW = SMALL ? 16 : 8;
  static constexpr int RB = SMALL ? SUB : 2 * SUB;
  static constexpr int NSUB = RB / SUB;
  // ranks of 8 and more: X_hat through shared memory, lanes over rank pairs
  static constexpr bool PAIRS = R >= 8 || R < 0;
  static constexpr int LPR = PAIRS ? RMAX / 2 : 1;  // lanes on one L1 row (one rank pair each)
  static constexpr int KP = PAIRS ? 32 / LPR : 1;  // L1 rows per warp load
  static constexpr int KS = 256 / KP;        // channels of one residue class in a chunk
  static constexpr int KSP = KS + 4;         // padded: the KP classes start on different banks
  static constexpr int XS_FLOATS = PAIRS ? NW * SUB * KP * KSP : 1;
};

// FP4 = true: the NVFP4 form (quantize8_nvfp4; `scales` is taken as the bytes of
// the NVFP4 scale layout, `ld` is unused, g comes from the absmax in gs[1] and
// the first block writes it to gs[0]).
template <int R, bool SMALL, int GL, bool FP4 = false>
__global__ void __launch_bounds__(ActCfg<R, SMALL>::NW * 32)
    quantize_act_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ s,
                        const __nv_bfloat16* __restrict__ L1, int M, int K, int r, int Kp, int ld,
                        uint8_t* __restrict__ codes, float* __restrict__ scales, float* __restrict__ U,
                        float* gs = nullptr, unsigned* zc = nullptr, int zc_words = 0) {
  using C = ActCfg<R, SMALL>;
  constexpr int SUB = C::SUB, NW = C::NW, RB = C::RB, NSUB = C::NSUB;
  grid_dep_wait();  // X (and for FP4 the absmax) may come from the preceding kernel
  // the next GEMM's split-K counters, when asked (the preceding kernel is done with them)
  for (int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x); i < zc_words;
       i += static_cast<int>(gridDim.x * blockDim.x))
    zc[i] = 0u;
  float g = 0.f, sixg = 0.f;
  if constexpr (FP4) {
    g = nvfp4_tensor_scale(gs[1]);
    sixg = __fmul_rn(6.0f, g);
    if (blockIdx.x == 0 && threadIdx.x == 0) gs[0] = g;
  }
  // a grid of a few blocks lets the next kernel start right away (it runs on the
  // idle SMs); a grid that fills the GPU lets it start only as blocks finish, so
  // that early arrivals do not take SMs from this kernel's later blocks
  const bool early = gridDim.x <= 64;
  if (early && threadIdx.x == 0) grid_dep_launch();
  constexpr int RA = C::RMAX > 0 ? C::RMAX : 1;
  constexpr bool PAIRS = C::PAIRS;
  constexpr int KP = C::KP, KS = C::KS, KSP = C::KSP, LPR = C::LPR;
  __shared__ float upart[R != 0 ? NW : 1][SUB][RA];
  __shared__ __align__(16) float xs_all[C::XS_FLOATS];
  const int warp = threadIdx.x >> 5;
  const int lane = lane_id();
  const int sb = warp % NSUB;
  const int mb = blockIdx.x * RB + sb * SUB;  // first row of this warp's sub-block
  const int nchunks = (Kp + 255) / 256;

  float u[SUB][PAIRS ? 1 : RA];
  float2 u2[PAIRS ? SUB : 1];
#pragma unroll
  for (int i = 0; i < SUB; ++i) {
#pragma unroll
    for (int j = 0; j < (PAIRS ? 1 : RA); ++j) u[i][j] = 0.f;
    if constexpr (PAIRS) u2[i] = make_float2(0.f, 0.f);
  }
  float* xw = xs_all + (PAIRS ? warp * SUB * KP * KSP : 0);  // this warp's X_hat rows
  const int kq = lane / LPR, pr = lane % LPR;                // L1 row class, rank pair

  // X rows of a chunk are loaded one chunk ahead, so their HBM latency overlaps
  // the previous chunk's arithmetic
  auto load_x = [&](int c, uint4 (&xr)[SUB]) {
    const int k0 = c * 256 + lane * 8;
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      const int m = mb + i;
      xr[i] = (c < nchunks && k0 < K && m < M)
                  ? __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k0))
                  : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 xnext[SUB];
  load_x(warp / NSUB, xnext);
  for (int c = warp / NSUB; c < nchunks; c += NW / NSUB) {
    const int k0 = c * 256 + lane * 8;
    uint4 xr[SUB];
#pragma unroll
    for (int i = 0; i < SUB; ++i) xr[i] = xnext[i];
    load_x(c + NW / NSUB, xnext);
    const bool real = k0 < K;  // K % 8 == 0: a lane's 8 channels are all real or all padding
    const bool in_k = k0 < Kp;
    float sv[8], sz[8];
    if (real) {
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
      sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
      sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) sv[e] = 1.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) sz[e] = __frcp_rn(sv[e]);  // reused by the SUB rows
    // small ranks: the 8 channels' L1 rows (8*R bf16, contiguous) stay in registers
    float l1s[8][(R > 0 && R <= 4) ? R : 1];
    if constexpr (R > 0 && R <= 4) {
      const uint4* src = reinterpret_cast<const uint4*>(L1 + static_cast<size_t>(k0) * R);
#pragma unroll
      for (int v = 0; v < R; ++v) {
        float f[8];
        bf16x8_to_f32(real ? __ldg(src + v) : make_uint4(0u, 0u, 0u, 0u), f);
#pragma unroll
        for (int t = 0; t < 8; ++t) l1s[(v * 8 + t) / R][(v * 8 + t) % R] = f[t];
      }
    }
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      const int m = mb + i;
      if (m >= M) break;  // warp-uniform
      float xh[8];
      smooth8(xr[i], sv, sz, real, xh);
      if constexpr (R > 0 && R <= 4) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
#pragma unroll
          for (int j = 0; j < R; ++j) u[i][j] = fmaf(xh[e], l1s[e][j], u[i][j]);
      } else if constexpr (PAIRS) {
        // park X_hat by residue class: channel lane*8+e goes to class (lane*8+e) % KP,
        // slot (lane*8+e) / KP
        float* xrow = xw + i * KP * KSP;
        if constexpr (KP == 2) {
          *reinterpret_cast<float4*>(xrow + lane * 4) = make_float4(xh[0], xh[2], xh[4], xh[6]);
          *reinterpret_cast<float4*>(xrow + KSP + lane * 4) = make_float4(xh[1], xh[3], xh[5], xh[7]);
        } else if constexpr (KP == 4) {
#pragma unroll
          for (int e = 0; e < 4; ++e)
            *reinterpret_cast<float2*>(xrow + e * KSP + lane * 2) = make_float2(xh[e], xh[e + 4]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) xrow[e * KSP + lane] = xh[e];
        }
      }
      if constexpr (FP4) {
        uint32_t sf;
        const uint32_t packed = quantize8_nvfp4(xh, g, sixg, sf);
        const uint32_t word = gather_sf_word(sf);
        if (in_k) {
          *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(m) * (Kp / 2) + k0 / 2) = packed;
          if ((lane & 7) == 0)
            *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(scales) +
                                         nvfp4_sf_word_offset(m, k0 / 64, Kp / 64)) = word;
        }
      } else {
        float sc;
        const uint32_t packed = quantize8_fast<GL>(xh, sc);
        if (in_k) {
          *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(m) * (Kp / 2) + k0 / 2) = packed;
          if ((lane & (GL - 1)) == 0) {
            float* srow = scales + static_cast<size_t>(k0 / (8 * GL)) * ld;
            srow[m] = sc;
            if (m == M - 1)
              for (int p = M; p < ld; ++p) srow[p] = 0.f;  // padding of the group-major layout
          }
        }
      }
    }
    if constexpr (PAIRS) {
      // U[i][2pr..2pr+1] += sum over this lane's channels k of X_hat[i][k] L1[k][2pr..2pr+1]
      const int kv = min(256, K - c * 256);  // real channels of the chunk
      const int nrows = min(SUB, M - mb);    // rows parked by this warp
      __syncwarp();
      if (nrows > 0) {
        const __nv_bfloat16* l1c = L1 + static_cast<size_t>(c) * 256 * r;
        const float* xq = xw + kq * KSP;
        for (int t = 0; t < KS && kq + KP * t < kv; t += 4) {
          float2 l[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int k = kq + KP * (t + q);
            if constexpr (R > 0) {
              uint32_t raw = 0u;
              if (k < kv) raw = __ldg(reinterpret_cast<const unsigned int*>(l1c + static_cast<size_t>(k) * R) + pr);
              l[q] = make_float2(__uint_as_float(raw << 16), __uint_as_float(raw & 0xffff0000u));
            } else {
              const __nv_bfloat16* row = l1c + static_cast<size_t>(k) * r + 2 * pr;
              const bool k_ok = k < kv;
              l[q].x = (k_ok && 2 * pr < r) ? __bfloat162float(__ldg(row)) : 0.f;
              l[q].y = (k_ok && 2 * pr + 1 < r) ? __bfloat162float(__ldg(row + 1)) : 0.f;
            }
          }
#pragma unroll
          for (int i = 0; i < SUB; ++i) {
            const float4 xv = *reinterpret_cast<const float4*>(xq + i * KP * KSP + t);
            u2[i] = __ffma2_rn(make_float2(xv.x, xv.x), l[0], u2[i]);
            u2[i] = __ffma2_rn(make_float2(xv.y, xv.y), l[1], u2[i]);
            u2[i] = __ffma2_rn(make_float2(xv.z, xv.z), l[2], u2[i]);
            u2[i] = __ffma2_rn(make_float2(xv.w, xv.w), l[3], u2[i]);
          }
        }
      }
      __syncwarp();  // the next chunk's rows overwrite the parked ones
    }
  }
  if (!early && threadIdx.x == 0) grid_dep_launch();
  if constexpr (PAIRS) {
#pragma unroll
    for (int i = 0; i < SUB; ++i) {
      float2 v = u2[i];
#pragma unroll
      for (int o = LPR; o < 32; o <<= 1) {  // the KP lanes of one rank pair
        v.x += __shfl_xor_sync(0xffffffffu, v.x, o);
        v.y += __shfl_xor_sync(0xffffffffu, v.y, o);
      }
      if (kq == 0) {
        upart[warp][i][2 * pr] = v.x;
        upart[warp][i][2 * pr + 1] = v.y;
      }
    }
    __syncthreads();
  } else if constexpr (R != 0) {
#pragma unroll
    for (int i = 0; i < SUB; ++i)
#pragma unroll
      for (int j = 0; j < RA; ++j) {
        float v = u[i][j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) upart[warp][i][j] = v;
      }
    __syncthreads();
  }
  if constexpr (R != 0) {
    const int rows = min(RB, M - static_cast<int>(blockIdx.x) * RB);
    for (int t = threadIdx.x; t < rows * r; t += blockDim.x) {
      const int row = t / r, j = t - (t / r) * r;
      const int tsb = row / SUB, i = row - tsb * SUB;
      float v = 0.f;
      for (int w = tsb; w < NW; w += NSUB) v += upart[w][i][j];  // fixed order
      U[(static_cast<size_t>(blockIdx.x) * RB + row) * r + j] = v;
    }
  }
}

// ---------------------------------------------------------------------------
// The activation step for many rows and ranks 0..4 (the same outputs as
// quantize_act_kernel, fewer instructions per element).
//
// A block of NW warps owns RB = NW * SUB consecutive rows; warp w owns rows
// w*SUB .. w*SUB+SUB-1 of them across all of K, so U needs no reduction across
// warps.  K is walked in chunks of 256 channels:
//   * each warp streams its own row pieces (512 bytes per row and chunk) into a
//     ring of STAGES shared-memory stages with 16-byte asynchronous copies, one
//     per lane, STAGES chunks ahead of its compute (the copies zero-fill past K
//     and past the last row);
//   * the chunk's per-channel tables -- RN(1/s), -s and the L1 rows as fp32 --
//     sit in a ring of TS slots; every warp builds its 256/NW channels of chunk
//     c + TD while it computes chunk c (the global loads issued two chunks
//     earlier) and arrives on the slot's `tfull` mbarrier; a warp done with a
//     chunk arrives on the slot's `tempty` mbarrier, which the builders of the
//     slot's next chunk wait for.  Warps are never held in lockstep: a warp
//     may run up to TS - TD chunks ahead of the slowest one.
// Lane l handles channels 8l .. 8l+7 of a row; the SUB rows of a warp are
// processed side by side.  Arithmetic on channel pairs uses the packed fp32x2
// instructions: X_hat = x / s as a product with RN(1/s) and Markstein's
// correction, the rank products accumulated per channel parity, the codes as a
// product with RN(1/scale), its correction and the round-to-integer addition.
// The correction gives the IEEE quotient when the dividend, divisor and
// quotient are normal; instead of testing every element, a group takes it only
// when s lies in [2^-24, 2^24] for the chunk and the group's absmax (a
// NaN-propagating maximum) lies in [2^-60, 2^75]:
//   * such a group's elements with 2^-100 <= |x| <= 2^100 are exact;
//   * smaller elements have |X_hat| < 2^-75, far below half a code step
//     (scale >= 2^-63), so code 0 on both sides and no effect on the absmax;
//   * larger elements make the absmax exceed 2^75 (or NaN), so the group is
//     not taken;
// otherwise the warp redoes the chunk's rows with IEEE divisions (quantize8).
// ---------------------------------------------------------------------------
template <int NW, int SUB>
struct ActRowsCfg {
  static constexpr int RB = NW * SUB;
  static constexpr int STAGES = 4;  // X ring depth (chunks)
  static constexpr int TS = 4;      // table slots
  static constexpr int TD = 2;      // tables are built this many chunks ahead
  static constexpr int STAGE_BYTES = RB * 512;
};

// Shared-memory float4 slot of logical slot q in a lane's block of S slots
// (S = 1, 2, 4 or 8), XOR-swizzled so that the 8 lanes of each quarter-warp
// phase of a 128-bit load hit 8 different 16-byte bank groups.
template <int S>
__device__ __forceinline__ int swz_slot(int lane, int q) {
  return q ^ ((lane / (8 / S)) & (S - 1));
}

// max that propagates NaN (PTX max.NaN.f32).
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// NaN-propagating absmax of a lane's 8 values (a depth-3 tree).
__device__ __forceinline__ float absmax8_nan(const float (&v)[8]) {
  const float a = fmax_nan(fmax_nan(fabsf(v[0]), fabsf(v[1])), fmax_nan(fabsf(v[2]), fabsf(v[3])));
  const float b = fmax_nan(fmax_nan(fabsf(v[4]), fabsf(v[5])), fmax_nan(fabsf(v[6]), fabsf(v[7])));
  return fmax_nan(a, b);
}

// 16-byte asynchronous global -> shared copy; bytes past `src_bytes` (0 or 16)
// are zero-filled.
__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Sum over e of (0x4B400000 << 4e) modulo 2^32: the exponent bits that the
// round-to-integer additions leave in the nibble-packing sum below.
__host__ __device__ constexpr uint32_t int4_pack_bias() {
  uint32_t b = 0;
  for (int e = 0; e < 8; ++e) b += 0x4B400000u << (4 * e);
  return b;
}

// Codes of 8 values of a group whose absmax `amax` lies in [2^-60, 2^75]
// (every lane of the group passes the same amax): scale = RN(amax / 7) by
// Markstein's correction against RN(1/7); each code RN(v / scale) by the
// correction against RN(1/scale), then rounded to an integer by adding
// 1.5 * 2^23 + 8, which leaves code + 8 (in 1..15) in the low mantissa bits.
// The 8 sums are packed by shifts and adds; the exponent bits they drag along
// add up to one constant (int4_pack_bias), and XOR 8 per nibble turns code + 8
// into the code's 4-bit two's complement.
__device__ __forceinline__ uint32_t quantize8_int4_ranged(const float (&v)[8], float amax, float& scale) {
  constexpr float kInv7 = 1.0f / 7.0f;
  const float q = __fmul_rn(amax, kInv7);
  scale = __fmaf_rn(__fmaf_rn(-q, 7.0f, amax), kInv7, q);
  const float z = __frcp_rn(scale);
  const float ns = -scale;
  constexpr float kRound = 12582920.0f;  // 1.5 * 2^23 + 8
  uint32_t b[8];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    float q0, q1, r0, r1, t0, t1;
    fmul2(q0, q1, v[2 * p], v[2 * p + 1], z, z);
    ffma2(r0, r1, q0, q1, ns, ns, v[2 * p], v[2 * p + 1]);
    ffma2(t0, t1, r0, r1, z, z, q0, q1);
    fadd2(t0, t1, t0, t1, kRound, kRound);
    b[2 * p] = __float_as_uint(t0);
    b[2 * p + 1] = __float_as_uint(t1);
  }
  const uint32_t p01 = (b[1] << 4) + b[0], p23 = (b[3] << 4) + b[2];
  const uint32_t p45 = (b[5] << 4) + b[4], p67 = (b[7] << 4) + b[6];
  const uint32_t acc = (((p67 << 8) + p45) << 16) + ((p23 << 8) + p01);
  return (acc - int4_pack_bias()) ^ 0x88888888u;
}

// NVFP4 codes of a lane's 8 values (half of a 16-value block; both lanes of the
// block pass the same bmax, which lies in [2^-60, 2^75]), g > 0, z6 = RN(1/sixg):
// sf = E4M3(RN(bmax / sixg)), the quotient by Markstein's correction; the codes
// E2M1(RN(v / fp32(b g))) by the correction against RN(1 / fp32(b g)).
__device__ __forceinline__ uint32_t quantize8_nvfp4_ranged(const float (&v)[8], float bmax, float g, float sixg,
                                                           float z6, uint32_t& sf) {
  const float q = __fmul_rn(bmax, z6);
  sf = f32_to_e4m3_rn_sat(__fmaf_rn(__fmaf_rn(-q, sixg, bmax), z6, q));
  const float denom = __fmul_rn(e4m3_to_f32(sf), g);
  if (denom == 0.f) return 0u;
  const float z = __frcp_rn(denom);
  const float nd = -denom;
  float t[8];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    float q0, q1, r0, r1;
    fmul2(q0, q1, v[2 * p], v[2 * p + 1], z, z);
    ffma2(r0, r1, q0, q1, nd, nd, v[2 * p], v[2 * p + 1]);
    ffma2(t[2 * p], t[2 * p + 1], r0, r1, z, z, q0, q1);
  }
  return f32x8_to_e2m1(t);
}

// FP4 = true: the NVFP4 form (GL = 2 lanes per 16-value block; `scales` taken
// as the bytes of the NVFP4 scale layout, `ld` unused; g from the absmax in
// gs[1], written to gs[0] by the first block).  A block takes the fast path when
// its absmax lies in [2^-60, 2^75]: the block scale is then E4M3(RN(bmax / 6g))
// with the quotient by Markstein's correction against RN(1/(6g)) (a quotient
// too small to be normal rounds to E4M3 zero either way), the divisor
// fp32(b g) is 0 or at least bmax / 12, so elements below 2^-100 give
// quotients far below 1/4 (E2M1 code 0 on both sides), and the codes are the
// E2M1 rounding of the corrected quotients.
template <int R, int GL, int NW, int SUB, bool FP4 = false>
__global__ void __launch_bounds__(NW * 32, 16 / NW)
    quantize_act_rows_kernel(const __nv_bfloat16* __restrict__ X, const float* __restrict__ s,
                             const __nv_bfloat16* __restrict__ L1, int M, int K, int Kp, int ld,
                             uint8_t* __restrict__ codes, float* __restrict__ scales, float* __restrict__ U,
                             uint64_t limit_ns, float* gs = nullptr, uint8_t* __restrict__ xe = nullptr,
                             int xe_rg = 0, unsigned* zc = nullptr, int zc_words = 0) {
  static_assert(R >= 0 && R <= 4 && R != 3, "ranks 0, 1, 2 and 4");
  static_assert(NW <= 8, "one byte per warp in an 8-byte flag word");
  using C = ActRowsCfg<NW, SUB>;
  constexpr int RB = C::RB, STAGES = C::STAGES, TS = C::TS, TD = C::TD, NT = NW * 32;
  constexpr int CPT = 256 / NT;          // table channels built per thread
  constexpr int RT = R > 0 ? R : 1;
  constexpr int LS = 2 * RT;             // float4 slots of a lane's L1 block (8 channels x R)
  constexpr int PW = RT > 1 ? RT / 2 : 1;
  extern __shared__ __align__(128) uint8_t ring[];  // STAGES x STAGE_BYTES (dynamic)
  // per lane (8 channels): 4 slots (z_2p, z_2p+1, -s_2p, -s_2p+1), swizzled
  __shared__ __align__(16) float tzs[TS][32 * 16];
  // per lane: slot data L1[2p][j], L1[2p+1][j] at ((p R + j) 2 + h), swizzled
  __shared__ __align__(16) float tl1[R > 0 ? TS : 1][R > 0 ? 32 * 8 * RT : 4];
  __shared__ __align__(8) uint8_t tbad[TS][8];  // per warp: some s of its channels out of range
  __shared__ __align__(8) uint64_t tfull[TS], tempty[TS];
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = lane_id();
  const int mw = blockIdx.x * RB + warp * SUB;  // this warp's first row
  const int nchunks = (Kp + 255) >> 8;
  if (tid == 0) {
#pragma unroll
    for (int t = 0; t < TS; ++t) {
      mbar_init(&tfull[t], NW);
      mbar_init(&tempty[t], NW);
      *reinterpret_cast<uint2*>(tbad[t]) = make_uint2(0u, 0u);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();  // X (and for FP4 the absmax) may come from the preceding kernel
  // the next GEMM's split-K counters, when asked (the preceding kernel is done with them)
  for (int i = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x); i < zc_words;
       i += static_cast<int>(gridDim.x * blockDim.x))
    zc[i] = 0u;
  float g = 0.f, sixg = 0.f, z6 = 0.f;
  if constexpr (FP4) {
    g = nvfp4_tensor_scale(gs[1]);
    sixg = __fmul_rn(6.0f, g);
    z6 = sixg > 0.f ? __frcp_rn(sixg) : 0.f;
    if (blockIdx.x == 0 && tid == 0) gs[0] = g;
  }
  const bool early = gridDim.x <= 64;
  if (early && tid == 0) grid_dep_launch();
  const WaitPolicy wp{limit_ns, &abort_flag};

  // this warp's row pieces of chunk c into stage c % STAGES (one commit group
  // per chunk, empty past the last chunk, so that group counts stay uniform)
  auto issue = [&](int c) {
    if (c < nchunks) {
      const int k0 = c * 256 + lane * 8;
#pragma unroll
      for (int i = 0; i < SUB; ++i) {
        const int m = mw + i;
        const bool in = m < M && k0 < K;
        cp_async16(ring + (c % STAGES) * C::STAGE_BYTES + (warp * SUB + i) * 512 + lane * 16,
                   in ? static_cast<const void*>(X + static_cast<size_t>(m) * K + k0) : static_cast<const void*>(X),
                   in ? 16u : 0u);
      }
    }
    cp_async_commit();
  };

  // the table inputs of this thread's channels; queue slot d holds chunk c+TD+d
  // during iteration c
  float ps[2][CPT];
  uint32_t pl[2][CPT][PW];
  auto fetch = [&](int c, float (&fs)[CPT], uint32_t (&fl)[CPT][PW]) {
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const int k = c * 256 + tid + q * NT;
      const bool in = c < nchunks && k < K;
      fs[q] = in ? __ldg(s + k) : 1.f;
      if constexpr (R == 4) {
        const uint2 v = in ? __ldg(reinterpret_cast<const uint2*>(L1 + static_cast<size_t>(k) * 4))
                           : make_uint2(0u, 0u);
        fl[q][0] = v.x;
        fl[q][1] = v.y;
      } else if constexpr (R == 2) {
        fl[q][0] = in ? __ldg(reinterpret_cast<const unsigned int*>(L1 + static_cast<size_t>(k) * 2)) : 0u;
      } else if constexpr (R == 1) {
        fl[q][0] = in ? static_cast<uint32_t>(__ldg(reinterpret_cast<const unsigned short*>(L1 + k))) : 0u;
      } else {
        fl[q][0] = 0u;
      }
    }
  };
  // this warp's channels of chunk cb's tables into slot cb % TS (after the
  // slot's previous chunk is released); returns false on a timeout
  auto build = [&](int cb) -> bool {
    const int t = cb % TS;
    if (cb >= TS && !wait_warp(&tempty[t], ((cb / TS) - 1) & 1, wp)) return false;
    bool bad = false;
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const int ch = tid + q * NT;          // channel within the chunk
      const int ln = ch >> 3, e = ch & 7;   // consuming lane, its channel
      const float sv = ps[0][q];
      bad |= !(sv >= 0x1p-24f && sv <= 0x1p24f);
      float* zb = &tzs[t][ln * 16];
      const int p = e >> 1, h = e & 1;
      zb[swz_slot<4>(ln, p) * 4 + h] = __frcp_rn(sv);
      zb[swz_slot<4>(ln, p) * 4 + 2 + h] = -sv;
      if constexpr (R > 0) {
        float* lb = &tl1[t][ln * 8 * RT];
#pragma unroll
        for (int j = 0; j < R; ++j) {
          const uint32_t w = pl[0][q][j >> 1];
          const float f = __uint_as_float((j & 1) ? (w & 0xffff0000u) : (w << 16));
          const int idx = (p * R + j) * 2 + h;
          lb[swz_slot<LS>(ln, idx >> 2) * 4 + (idx & 3)] = f;
        }
      }
    }
    const bool anybad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      tbad[t][warp] = anybad ? 1 : 0;
      mbar_arrive(&tfull[t]);  // release: this warp's table writes
    }
    return true;
  };
  auto advance = [&](int cnext) {  // shift the queue, fetch chunk cnext into its tail
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      ps[0][q] = ps[1][q];
#pragma unroll
      for (int h = 0; h < PW; ++h) pl[0][q][h] = pl[1][q][h];
    }
    fetch(cnext, ps[1], pl[1]);
  };

  // prologue: X chunks 0..STAGES-1 in flight, tables of chunks 0..TD-1 built,
  // the queue holding chunks TD and TD+1
  bool ok = true;
#pragma unroll
  for (int c = 0; c < STAGES; ++c) issue(c);
  fetch(0, ps[0], pl[0]);
  fetch(1, ps[1], pl[1]);
#pragma unroll
  for (int c = 0; c < TD; ++c) {
    if (c < nchunks) ok = ok && build(c);
    advance(c + 2);
  }

  float2 acc[SUB][RT];
#pragma unroll
  for (int i = 0; i < SUB; ++i)
#pragma unroll
    for (int j = 0; j < RT; ++j) acc[i][j] = make_float2(0.f, 0.f);

  for (int c = 0; ok && c < nchunks; ++c) {
    const int t = c % TS;
    if (c + TD < nchunks) {
      if (!build(c + TD)) { ok = false; break; }
    }
    advance(c + TD + 2);
    if (!wait_warp(&tfull[t], (c / TS) & 1, wp)) { ok = false; break; }
    cp_async_wait<STAGES - 1>();  // this lane's copies of chunk c have landed
    __syncwarp();                 // ... and every other lane's
    if (mw < M) {
      const uint2 bw = *reinterpret_cast<const uint2*>(tbad[t]);
      const bool sbad = (bw.x | bw.y) != 0u;
      const int k0 = c * 256 + lane * 8;
      const bool real = k0 < K, in_k = k0 < Kp;
      float zz[8], ns[8];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const float4 v = *reinterpret_cast<const float4*>(&tzs[t][lane * 16 + swz_slot<4>(lane, p) * 4]);
        zz[2 * p] = v.x; zz[2 * p + 1] = v.y; ns[2 * p] = v.z; ns[2 * p + 1] = v.w;
      }
      const uint8_t* stage = ring + (c % STAGES) * C::STAGE_BYTES + warp * SUB * 512 + lane * 16;
      float xh[SUB][8], amax[SUB];
#pragma unroll
      for (int i = 0; i < SUB; ++i) {
        const uint4 raw = *reinterpret_cast<const uint4*>(stage + i * 512);
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float x0 = __uint_as_float(w[p] << 16), x1 = __uint_as_float(w[p] & 0xffff0000u);
          float q0, q1, r0, r1;
          fmul2(q0, q1, x0, x1, zz[2 * p], zz[2 * p + 1]);
          ffma2(r0, r1, q0, q1, ns[2 * p], ns[2 * p + 1], x0, x1);
          ffma2(xh[i][2 * p], xh[i][2 * p + 1], r0, r1, zz[2 * p], zz[2 * p + 1], q0, q1);
        }
        amax[i] = absmax8_nan(xh[i]);
      }
#pragma unroll
      for (int o = 1; o < GL; o <<= 1)
#pragma unroll
        for (int i = 0; i < SUB; ++i) amax[i] = fmax_nan(amax[i], __shfl_xor_sync(0xffffffffu, amax[i], o));
      bool bad = false;
#pragma unroll
      for (int i = 0; i < SUB; ++i)
        bad |= (mw + i < M) && in_k && (sbad || !(amax[i] >= 0x1p-60f && amax[i] <= 0x1p75f));
      uint32_t packed[SUB];
      float sc[SUB];      // INT4: the group scales
      uint32_t sfb[SUB];  // FP4: the E4M3 block scales
      if (__any_sync(0xffffffffu, bad)) {
        // the exact path: IEEE quotients (-ns = s; padding lanes read zeros)
#pragma unroll
        for (int i = 0; i < SUB; ++i) {
          float x[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(stage + i * 512), x);
#pragma unroll
          for (int e = 0; e < 8; ++e) xh[i][e] = real ? __fdiv_rn(x[e], -ns[e]) : 0.f;
          if constexpr (FP4) packed[i] = quantize8_nvfp4(xh[i], g, sixg, sfb[i]);
          else packed[i] = quantize8<GL>(xh[i], sc[i]);
        }
      } else {
#pragma unroll
        for (int i = 0; i < SUB; ++i) {
          if constexpr (FP4) packed[i] = quantize8_nvfp4_ranged(xh[i], amax[i], g, sixg, z6, sfb[i]);
          else packed[i] = quantize8_int4_ranged(xh[i], amax[i], sc[i]);
        }
      }
      if constexpr (R > 0) {
        float lp[8 * RT];
#pragma unroll
        for (int q = 0; q < LS; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(&tl1[t][lane * 8 * RT + swz_slot<LS>(lane, q) * 4]);
          lp[4 * q] = v.x; lp[4 * q + 1] = v.y; lp[4 * q + 2] = v.z; lp[4 * q + 3] = v.w;
        }
#pragma unroll
        for (int i = 0; i < SUB; ++i)
#pragma unroll
          for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int j = 0; j < R; ++j)
              ffma2(acc[i][j].x, acc[i][j].y, xh[i][2 * p], xh[i][2 * p + 1], lp[(p * R + j) * 2],
                    lp[(p * R + j) * 2 + 1], acc[i][j].x, acc[i][j].y);
      }
      if constexpr (FP4) {
        // the four block scales of each 64-wide chunk: one word on lane 8p
#pragma unroll
        for (int i = 0; i < SUB; ++i) {
          const uint32_t word = gather_sf_word(sfb[i]);
          if (in_k && mw + i < M) {
            *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(mw + i) * (Kp / 2) + k0 / 2) = packed[i];
            if ((lane & 7) == 0)
              *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(scales) +
                                           nvfp4_sf_word_offset(mw + i, k0 / 64, Kp / 64)) = word;
          }
        }
      } else if (in_k) {
        if (xe) {
          // the GEMM's E4M3 tile layout instead of packed codes: lane l's 8 codes
          // are codes 8(l % 8) .. +7 of 64-block k0/64; even codes go to chunk
          // 2h, odd ones to chunk 2h+1 (h = (l % 8) / 4), bytes 4(l % 4) .. +3
          // of the row's 16-byte slot (the layout of expand_e4m3_kernel)
          const int h = (lane & 7) >> 2;
          const size_t blk = static_cast<size_t>(k0 >> 6);
#pragma unroll
          for (int i = 0; i < SUB; ++i) {
            const int m = mw + i;
            if (m >= M) break;
            const uint32_t w = packed[i];
            const uint32_t sg = w & 0x88888888u, one = sg >> 3;
            const uint32_t sm = (w ^ (sg - one)) + one;  // sign-magnitude nibbles (codes are never -8)
            const uint32_t lo = (sm & 0x07070707u) | ((sm << 4) & 0x80808080u);
            const uint32_t hi = ((sm >> 4) & 0x07070707u) | (sm & 0x80808080u);
            uint8_t* dst = xe + ((blk * xe_rg + (m >> 3)) * 4 + 2 * h) * 128 + (m & 7) * 16 + 4 * (lane & 3);
            *reinterpret_cast<uint32_t*>(dst) = lo;
            *reinterpret_cast<uint32_t*>(dst + 128) = hi;
          }
        } else {
#pragma unroll
          for (int i = 0; i < SUB; ++i)
            if (mw + i < M)
              *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(mw + i) * (Kp / 2) + k0 / 2) = packed[i];
        }
        if ((lane & (GL - 1)) == 0) {
          float* srow = scales + static_cast<size_t>(k0 / (8 * GL)) * ld;
          if (SUB == 2 && mw + 1 < M) {
            *reinterpret_cast<float2*>(srow + mw) = make_float2(sc[0], sc[SUB - 1]);
          } else {
#pragma unroll
            for (int i = 0; i < SUB; ++i)
              if (mw + i < M) srow[mw + i] = sc[i];
          }
          if (M - 1 < mw + SUB)
            for (int p = M; p < ld; ++p) srow[p] = 0.f;  // padding of the group-major layout
        }
      }
    }
    __syncwarp();  // every lane is done with stage c % STAGES and table slot t
    if (lane == 0) mbar_arrive(&tempty[t]);
    issue(c + STAGES);
  }
  cp_async_wait<0>();  // no copy outlives the block
  if (!early && tid == 0) grid_dep_launch();

  if constexpr (R > 0) {
#pragma unroll
    for (int i = 0; i < SUB; ++i)
#pragma unroll
      for (int j = 0; j < R; ++j) {
        float v = acc[i][j].x + acc[i][j].y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && ok && mw + i < M) U[static_cast<size_t>(mw + i) * R + j] = v;
      }
  }
}

}  // namespace hsq
