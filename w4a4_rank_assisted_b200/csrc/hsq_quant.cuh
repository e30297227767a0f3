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
                        float* gs = nullptr) {
  using C = ActCfg<R, SMALL>;
  constexpr int SUB = C::SUB, NW = C::NW, RB = C::RB, NSUB = C::NSUB;
  grid_dep_wait();  // X (and for FP4 the absmax) may come from the preceding kernel
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

}  // namespace hsq
