// hsq_lowrank.cuh -- pack-time helper: plain truncated-SVD initialisation of
// the low-rank pair (Deflating the Hessian, Table 6: the "Plain SVD" row of the
// L1-initialisation ablation).
//
// L1 [K, r] = the top-r right singular vectors of W_hat = W diag(s) (orthonormal
// columns: the protected subspace of Figure 1's caption), L2 [r, N] =
// L1^T W_hat^T, so that (L1 L2)^T approximates the best rank-r approximation of
// W_hat.  Computed by subspace iteration with p = r + 8 columns: Q <- orth(W_hat^T
// (W_hat Q)) `iters` times from a seeded random start, then Rayleigh-Ritz on
// T = (W_hat Q)^T (W_hat Q).  The large products are plain fp32 GEMMs (cuBLAS);
// the kernels here do the rest: the smoothed fp32 copy of W, the random start,
// fp64 CholeskyQR factors, the p x p symmetric eigenproblem (cyclic Jacobi) and
// the sign convention plus bf16 output.  Matrices are column-major unless named
// otherwise: the row-major [N][K] W_hat is the column-major K x N matrix A.
#pragma once

#include "hsq_device.cuh"

namespace hsq {

constexpr int kLrOversample = 8;
constexpr int kLrMaxP = 40;  // r <= 32 plus the oversampling

// A[k + K n] = fp32(W[n][k]) * s[k]  (W_hat, row-major [N][K] = column-major K x N)
__global__ void lr_smooth_kernel(const __nv_bfloat16* __restrict__ W, const float* __restrict__ s, int N, int K,
                                 float* __restrict__ A) {
  const size_t total = static_cast<size_t>(N) * K;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int k = static_cast<int>(i % K);
    A[i] = __bfloat162float(W[i]) * s[k];
  }
}

// Uniform values in [-1, 1) from a counter-based hash of (seed, index):
// SplitMix64 (Steele, Lea, Flood: "Fast splittable pseudorandom number
// generators", OOPSLA 2014) of seed + index * golden gamma.
__global__ void lr_random_kernel(float* __restrict__ Q, size_t n, unsigned long long seed) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    unsigned long long z = seed + (static_cast<unsigned long long>(i) + 1ull) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    Q[i] = static_cast<float>(static_cast<double>(z >> 11) * (1.0 / 4503599627370496.0) - 1.0);
  }
}

__global__ void lr_to_f64_kernel(const float* __restrict__ a, double* __restrict__ b, size_t n) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    b[i] = static_cast<double>(a[i]);
}

__global__ void lr_to_f32_kernel(const double* __restrict__ a, float* __restrict__ b, size_t n) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    b[i] = static_cast<float>(a[i]);
}

// CholeskyQR factor (one block of kLrMaxP threads): G (p x p, the Gram matrix
// Z^T Z) = R^T R with R upper triangular; writes R^-1 (upper triangular) so that
// Z R^-1 has orthonormal columns.  A relative shift of 1e-14 * trace(G) / p
// keeps the factorisation defined when Z's columns are nearly dependent (the
// repeated pass then restores orthonormality).
__global__ void lr_chol_inv_kernel(const double* __restrict__ G, int p, double* __restrict__ Rinv) {
  __shared__ double R[kLrMaxP][kLrMaxP];
  __shared__ double Ri[kLrMaxP][kLrMaxP];
  __shared__ double shift;
  const int t = threadIdx.x;
  if (t == 0) {
    double tr = 0.0;
    for (int i = 0; i < p; ++i) tr += G[i + i * p];
    shift = 1e-14 * tr / p + 1e-300;
  }
  __syncthreads();
  for (int i = t; i < p * p; i += blockDim.x) {
    const int r = i % p, c = i / p;
    R[r][c] = G[r + c * p] + (r == c ? shift : 0.0);
    Ri[r][c] = 0.0;
  }
  __syncthreads();
  // right-looking Cholesky on the upper triangle (row j of R is finished at step j)
  for (int j = 0; j < p; ++j) {
    if (t == 0) R[j][j] = sqrt(fmax(R[j][j], shift));
    __syncthreads();
    if (t > j && t < p) R[j][t] /= R[j][j];
    __syncthreads();
    for (int c = j + 1 + t; c < p; c += blockDim.x)
      for (int r = j + 1; r <= c; ++r) R[r][c] -= R[j][r] * R[j][c];
    __syncthreads();
  }
  // R^-1 by back substitution, one column per thread
  if (t < p) {
    const int c = t;
    for (int r = c; r >= 0; --r) {
      double v = (r == c) ? 1.0 : 0.0;
      for (int k = r + 1; k <= c; ++k) v -= R[r][k] * Ri[k][c];
      Ri[r][c] = v / R[r][r];
    }
  }
  __syncthreads();
  for (int i = t; i < p * p; i += blockDim.x) Rinv[i] = Ri[i % p][i / p];
}

// Symmetric eigenproblem of T (p x p) by cyclic Jacobi rotations (one block of
// kLrMaxP threads; threads update the two rows/columns of a rotation in
// parallel).  Writes the eigenvectors as the columns of V (p x p, fp32), in order
// of decreasing eigenvalue.
__global__ void lr_jacobi_kernel(const double* __restrict__ Tin, int p, float* __restrict__ V) {
  __shared__ double T[kLrMaxP][kLrMaxP];
  __shared__ double E[kLrMaxP][kLrMaxP];
  __shared__ double cs[2];
  __shared__ int order[kLrMaxP];
  __shared__ int done;
  const int t = threadIdx.x;
  for (int i = t; i < p * p; i += blockDim.x) {
    const int r = i % p, c = i / p;
    T[r][c] = 0.5 * (Tin[r + c * p] + Tin[c + r * p]);
    E[r][c] = (r == c) ? 1.0 : 0.0;
  }
  __syncthreads();
  for (int sweep = 0; sweep < 60; ++sweep) {
    if (t == 0) {
      double off = 0.0, tot = 0.0;
      for (int r = 0; r < p; ++r)
        for (int c = 0; c < p; ++c) {
          tot += T[r][c] * T[r][c];
          if (r != c) off += T[r][c] * T[r][c];
        }
      done = off <= 1e-30 * tot;
    }
    __syncthreads();
    if (done) break;
    for (int a = 0; a < p - 1; ++a)
      for (int b = a + 1; b < p; ++b) {
        if (t == 0) {
          const double apq = T[a][b];
          double c = 1.0, s = 0.0;
          if (fabs(apq) > 1e-300) {
            const double th = (T[b][b] - T[a][a]) / (2.0 * apq);
            const double tn = (th >= 0.0 ? 1.0 : -1.0) / (fabs(th) + sqrt(th * th + 1.0));
            c = 1.0 / sqrt(tn * tn + 1.0);
            s = tn * c;
          }
          cs[0] = c;
          cs[1] = s;
        }
        __syncthreads();
        const double c = cs[0], s = cs[1];
        if (s != 0.0) {
          if (t < p) {  // columns a, b of T and of E
            const double ta = T[t][a], tb = T[t][b];
            T[t][a] = c * ta - s * tb;
            T[t][b] = s * ta + c * tb;
            const double ea = E[t][a], eb = E[t][b];
            E[t][a] = c * ea - s * eb;
            E[t][b] = s * ea + c * eb;
          }
          __syncthreads();
          if (t < p) {  // rows a, b of T
            const double ta = T[a][t], tb = T[b][t];
            T[a][t] = c * ta - s * tb;
            T[b][t] = s * ta + c * tb;
          }
        }
        __syncthreads();
      }
  }
  if (t == 0) {  // order by decreasing eigenvalue (selection; ties keep the lower index first)
    for (int i = 0; i < p; ++i) order[i] = i;
    for (int i = 0; i < p; ++i) {
      int best = i;
      for (int j = i + 1; j < p; ++j)
        if (T[order[j]][order[j]] > T[order[best]][order[best]]) best = j;
      const int tmp = order[i];
      order[i] = order[best];
      order[best] = tmp;
    }
  }
  __syncthreads();
  for (int i = t; i < p * p; i += blockDim.x) {
    const int r = i % p, c = i / p;
    V[r + c * p] = static_cast<float>(E[r][order[c]]);
  }
}

// Sign convention and output (one block per column j of L1): the entry of
// largest magnitude of L1[:, j] (lowest index on ties) is made positive, and L2's
// row j follows; L1 is written row-major [K][r] and L2 row-major [r][N] in bf16.
// L1c: column-major K x r; C = W_hat L1, column-major N x r (= row-major [r][N]).
__global__ void lr_sign_out_kernel(const float* __restrict__ L1c, const float* __restrict__ C, int K, int N, int r,
                                   __nv_bfloat16* __restrict__ L1, __nv_bfloat16* __restrict__ L2) {
  __shared__ float bv[1024];
  __shared__ int bi[1024];
  const int j = blockIdx.x;
  const int t = threadIdx.x;
  float best = -1.f;
  int bidx = K;
  for (int k = t; k < K; k += blockDim.x) {
    const float v = fabsf(L1c[k + static_cast<size_t>(K) * j]);
    if (v > best) {  // k increases: the first maximum of this thread's stride
      best = v;
      bidx = k;
    }
  }
  bv[t] = best;
  bi[t] = bidx;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (t < o) {
      const float v2 = bv[t + o];
      const int i2 = bi[t + o];
      if (v2 > bv[t] || (v2 == bv[t] && i2 < bi[t])) {
        bv[t] = v2;
        bi[t] = i2;
      }
    }
    __syncthreads();
  }
  const float sg = L1c[bi[0] + static_cast<size_t>(K) * j] < 0.f ? -1.f : 1.f;
  for (int k = t; k < K; k += blockDim.x)
    L1[static_cast<size_t>(k) * r + j] = __float2bfloat16_rn(sg * L1c[k + static_cast<size_t>(K) * j]);
  for (int n = t; n < N; n += blockDim.x)
    L2[static_cast<size_t>(j) * N + n] = __float2bfloat16_rn(sg * C[n + static_cast<size_t>(N) * j]);
}

}  // namespace hsq
