// hsq_quant.cuh -- the two quantizing kernels: offline weight packing and the
// fused per-forward activation step.
//
// Quantizer (Deflating the Hessian, Abstract: 4-bit weights and activations;
// Table 1 caption: groups of 64 along K): symmetric signed INT4 with one fp32
// scale per 64 values, scale = absmax / 7 (IEEE division), code =
// round-half-even(v / scale) clamped to [-7, 7].  Both kernels give every lane
// 8 consecutive K-elements, so one 64-group spans 8 adjacent lanes and its
// absmax is a 3-step xor-shuffle reduction.
#pragma once

#include "hsq_device.cuh"

namespace hsq {

// Quantize one lane's 8 values of a 64-group spread over 8 adjacent lanes.
// Every lane of the warp must call this (it shuffles).  Returns the 8 codes
// packed as 4 bytes (code e in bits 4e..4e+3) and the group's scale.
__device__ __forceinline__ uint32_t quantize8(const float (&v)[8], float& scale) {
  float amax = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[e]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
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

// ---------------------------------------------------------------------------
// Weight packing (offline): R[n,k] = fp32(W[n,k]*s[k] - sum_j L1[k,j]*L2[j,n]),
// the sum in fp64 for j = 0..r-1 with every multiply and add rounded on its own
// (no fused multiply-add), then quantized.  One warp per output row n.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) pack_weights_kernel(const __nv_bfloat16* __restrict__ W,
                                                           const float* __restrict__ s,
                                                           const __nv_bfloat16* __restrict__ L1,
                                                           const __nv_bfloat16* __restrict__ L2, int N,
                                                           int K, int r, int Kp, int ld,
                                                           uint8_t* __restrict__ codes,
                                                           float* __restrict__ scales) {
  const int n = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = lane_id();
  if (n >= N) return;  // warp-uniform
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
    float sc;
    const uint32_t packed = quantize8(R, sc);
    if (k0 < Kp) {
      *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(n) * (Kp / 2) + k0 / 2) = packed;
      if ((lane & 7) == 0) scales[static_cast<size_t>(k0 / 64) * ld + n] = sc;
    }
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
// scales, and U = X_hat L1 in fp32.  One warp per token row, 8 rows per block;
// each lane loads 8 bf16 (one 16-byte load) per 256-wide chunk of K.
// RT is a compile-time upper bound on r (the loops are unrolled and predicated).
// ---------------------------------------------------------------------------
template <int RT>
__global__ void __launch_bounds__(256) quantize_act_kernel(const __nv_bfloat16* __restrict__ X,
                                                           const float* __restrict__ s,
                                                           const __nv_bfloat16* __restrict__ L1, int M,
                                                           int K, int r, int Kp, int ld,
                                                           uint8_t* __restrict__ codes,
                                                           float* __restrict__ scales,
                                                           float* __restrict__ U) {
  const int m = static_cast<int>(blockIdx.x * 8 + (threadIdx.x >> 5));
  const int lane = lane_id();
  if (m >= M) return;  // warp-uniform
  float u[RT > 0 ? RT : 1];
#pragma unroll
  for (int j = 0; j < (RT > 0 ? RT : 1); ++j) u[j] = 0.f;

  for (int c0 = 0; c0 < Kp; c0 += 256) {
    const int k0 = c0 + lane * 8;
    float xh[8];
    if (k0 < K) {
      const uint4 xraw = __ldg(reinterpret_cast<const uint4*>(X + static_cast<size_t>(m) * K + k0));
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
      float x[8];
      bf16x8_to_f32(xraw, x);
      const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) xh[e] = __fdiv_rn(x[e], sv[e]);
      if (RT > 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const __nv_bfloat16* l1row = L1 + static_cast<size_t>(k0 + e) * r;
#pragma unroll
          for (int j = 0; j < RT; ++j)
            if (j < r) u[j] = fmaf(xh[e], __bfloat162float(__ldg(l1row + j)), u[j]);
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) xh[e] = 0.f;
    }
    float sc;
    const uint32_t packed = quantize8(xh, sc);
    if (k0 < Kp) {
      *reinterpret_cast<uint32_t*>(codes + static_cast<size_t>(m) * (Kp / 2) + k0 / 2) = packed;
      if ((lane & 7) == 0) {
        float* srow = scales + static_cast<size_t>(k0 / 64) * ld;
        srow[m] = sc;
        if (m == M - 1)
          for (int p = M; p < ld; ++p) srow[p] = 0.f;  // padding of the group-major layout
      }
    }
  }
  if (RT > 0) {
#pragma unroll
    for (int j = 0; j < RT; ++j) {
      float v = u[j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && j < r) U[static_cast<size_t>(m) * r + j] = v;
    }
  }
}

}  // namespace hsq
