/*
 * hsq.h -- C ABI of libhsq, a B200 (sm_100a) implementation of the
 * low-rank-assisted W4A4 linear layer
 *
 *     Y = Q4(X_hat) Q4(R)^T + (X_hat L1) L2 + b,
 *     X_hat = X diag(s)^-1,     R = W diag(s) - (L1 L2)^T,
 *
 * from "Deflating the Hessian: Rank-4 W4A4 Quantization for Multimodal
 * Diffusion Transformers" (H-SVDQuant, arXiv 2610.11315):
 *   - Abstract: every weight is a low-bit residual plus a high-precision
 *     low-rank component; weights and activations are both 4-bit (W4A4).
 *   - Table 1 and Table 8 captions: quantization groups of 64 along K;
 *     Table 3 and Table 4 captions: groups of 128 for the Qwen3-8B results.
 *   - rit.work blog, diagonal-scaling paragraph: the smoothing vector s moves
 *     range between activations and weights without changing the layer's
 *     full-precision map (X_hat R^T + X_hat L1 L2 = X W^T before quantizing).
 *
 * Quantizer (symmetric signed INT4, one fp32 scale per group of `group` values along K):
 *   scale = fp32(absmax / 7); code = clamp(round_half_even(fp32(v / scale)), -7, 7);
 *   an all-zero group has scale 0 and codes 0.  K is zero-padded to
 *   Kp = group * ceil(K / group).
 *
 * Conventions shared by every call
 *   - Every data pointer is a DEVICE pointer owned by the caller; the library
 *     allocates no device memory.  Every pointer must be 16-byte aligned.
 *   - bf16 tensors are row-major __nv_bfloat16 (passed as void*).
 *   - Packed codes: row-major [rows][Kp/2] bytes; byte j of a row holds code
 *     2j in bits 0-3 and code 2j+1 in bits 4-7, 4-bit two's complement.
 *     Padded codes (k >= K) are 0.
 *   - Scales: group-major fp32 [G][ld] with G = ceil(K/group) and
 *     ld = hsq_scales_ld(rows) = rows rounded up to a multiple of 4; entry
 *     [g][i] is the scale of group g of row i; entries i >= rows are written 0.
 *   - Calls are asynchronous on `stream`.  Arguments are validated on the host
 *     before anything is launched; a rejected call launches nothing.
 *   - Every wait inside a kernel is bounded; a kernel that gives up records
 *     HSQ_ERR_TIMEOUT in a device status word, which hsq_get_device_status()
 *     reports.
 *   - Supported: group == 64 or 128, 0 <= r <= 32, K % 8 == 0, N % 8 == 0,
 *     1 <= M, N, K <= 2^20.
 */
#ifndef HSQ_H_
#define HSQ_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSQ_OK = 0,
  HSQ_ERR_INVALID_ARG = 1,   /* null pointer, bad size, L1/L2 null with r > 0, ws too small */
  HSQ_ERR_ALIGNMENT = 2,     /* a pointer is not 16-byte aligned */
  HSQ_ERR_UNSUPPORTED = 3,   /* group not 64 or 128, r > 32, K or N not a multiple of 8 */
  HSQ_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed (launch, tensor map) */
  HSQ_ERR_TIMEOUT = 5,       /* a kernel gave up waiting (reported by hsq_get_device_status) */
  HSQ_ERR_SCRATCH_LIMIT = 6  /* hsq_linear_forward_noalloc: shape needs more than HSQ_NOALLOC_SCRATCH_BYTES */
} hsq_status;

typedef enum { HSQ_OUT_BF16 = 0, HSQ_OUT_F32 = 1 } hsq_out_dtype;

/* Number of groups along K: ceil(K / group).  Returns 0 if group <= 0. */
int hsq_num_groups(int K, int group);

/* Bytes of a packed code matrix with `rows` rows: rows * Kp / 2. */
size_t hsq_codes_bytes(int rows, int K, int group);

/* Leading dimension (in floats) of a group-major scale matrix: rows rounded up to 4. */
int hsq_scales_ld(int rows);

/* Bytes of a scale matrix: ceil(K/group) * hsq_scales_ld(rows) * 4. */
size_t hsq_scales_bytes(int rows, int K, int group);

/*
 * Bytes of scratch that hsq_linear_forward needs for this shape on the current
 * device, for either group size: split-K counters and partial tiles, and for
 * M > 64 (groups of 128; M > 256 for groups of 64) the two code matrices
 * expanded to E4M3 bytes (0 when nothing is needed, as for M <= 8 whenever the
 * weight stream takes the shape).  The caller zero-fills the workspace once before its first use;
 * every completed call leaves the split-K counters zero again.
 */
size_t hsq_workspace_bytes(int M, int N, int K, int r);

/*
 * Offline weight packing (Abstract: low-bit residual + high-precision
 * low-rank part).  R[n,k] = fp32(W[n,k]*s[k] - sum_{j<r} L1[k,j]*L2[j,n]),
 * formed in fp64 with the sum taken for j = 0..r-1, each multiply and add
 * rounded separately; R is then quantized per group of each row.
 *   W_bf16   [N][K] bf16        s   [K] fp32 (all > 0)
 *   L1_bf16  [K][r] bf16        L2_bf16 [r][N] bf16   (both NULL iff r == 0)
 *   w_codes  out [N][Kp/2] u8   w_scales out [G][hsq_scales_ld(N)] fp32
 */
hsq_status hsq_pack_weights(const void* W_bf16, const float* s, const void* L1_bf16,
                            const void* L2_bf16, int N, int K, int r, int group,
                            uint8_t* w_codes, float* w_scales, cudaStream_t stream);

/*
 * Per-forward activation step (one fused kernel): X_hat = fp32(fp32(X)/s_k)
 * (rit.work blog: smoothing), its group-wise INT4 codes and scales, and the
 * low-rank down-projection U = X_hat L1 accumulated in fp32.
 *   X_bf16  [M][K] bf16          s [K] fp32        L1_bf16 [K][r] bf16 (NULL iff r == 0)
 *   x_codes out [M][Kp/2] u8     x_scales out [G][hsq_scales_ld(M)] fp32
 *   U       out [M][r] fp32 (may be NULL iff r == 0)
 */
hsq_status hsq_quantize_act(const void* X_bf16, const float* s, const void* L1_bf16,
                            int M, int K, int r, int group, uint8_t* x_codes,
                            float* x_scales, float* U, cudaStream_t stream);

/*
 * The layer's forward (Abstract: 4-bit residual product plus the 16-bit
 * low-rank branch):
 *   Y[m,n] = sum_g sx[g][m] * sw[g][n] * P_g[m,n] + sum_j U[m,j] * L2[j,n] + b[n],
 * with P_g the exact integer dot product of group g's codes.  For M > 8 the
 * INT4 codes are multiplied on the tensor cores (tcgen05) one group at a time
 * into Tensor Memory and each group's exact partial is rescaled into an fp32
 * accumulator, which also receives the low-rank branch and the bias before
 * the single rounding to the output type.  For M <= 8 the same sums run as a
 * weight stream on the CUDA cores (integer dot products of the codes), which
 * needs no workspace.
 *   x_codes/x_scales/U   as written by hsq_quantize_act (U NULL iff r == 0)
 *   w_codes/w_scales     as written by hsq_pack_weights
 *   L2_bf16 [r][N] (NULL iff r == 0), bias_bf16 [N] or NULL for no bias
 *   Y out [M][N], bf16 (HSQ_OUT_BF16, round-to-nearest-even) or fp32 (HSQ_OUT_F32)
 *   workspace / ws_bytes: scratch of at least hsq_workspace_bytes(M,N,K,r) bytes
 *     (may be NULL when that is 0); calls that share a workspace must not run
 *     concurrently.  Before its first use the workspace must hold zeros (its
 *     split-K counters); every call leaves them at zero again, so one
 *     zero-filled buffer serves any number of calls.
 */
hsq_status hsq_linear_forward(const uint8_t* x_codes, const float* x_scales, const float* U,
                              const uint8_t* w_codes, const float* w_scales,
                              const void* L2_bf16, const void* bias_bf16,
                              int M, int N, int K, int r, int group,
                              void* Y, hsq_out_dtype out,
                              void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * The weights' expanded copy, for hsq_linear_forward_pre.  Where the GEMM reads
 * pre-expanded operands -- M > 256, or M > 64 with groups of 128 -- a forward
 * first rewrites both code matrices into E4M3 tiles (one byte per code, the
 * layout the tensor cores read).  The weights' part of that never changes
 * between calls, so it can be done once, after hsq_pack_weights:
 *   hsq_weights_e4m3_bytes(N, K, group): bytes of the copy, Kp x (N rounded up
 *     to 256); 0 for an invalid shape;
 *   hsq_expand_weights: writes the copy from w_codes (asynchronous on stream).
 * A memory-for-speed trade of the library (Kp N bytes more per layer); the
 * method's stored format stays the packed INT4 codes.
 */
size_t hsq_weights_e4m3_bytes(int N, int K, int group);
hsq_status hsq_expand_weights(const uint8_t* w_codes, int N, int K, int group, uint8_t* w_e4m3,
                              cudaStream_t stream);

/*
 * hsq_linear_forward with the weights' expanded copy w_e4m3 (required): where
 * the GEMM reads pre-expanded operands it takes the weights from w_e4m3
 * instead of expanding w_codes again, and the workspace needs only
 * hsq_workspace_bytes_pre(M, N, K, r) bytes; elsewhere w_e4m3 is unused.  The
 * results are the same bits as hsq_linear_forward's.
 */
size_t hsq_workspace_bytes_pre(int M, int N, int K, int r);
hsq_status hsq_linear_forward_pre(const uint8_t* x_codes, const float* x_scales, const float* U,
                                  const uint8_t* w_codes, const float* w_scales, const uint8_t* w_e4m3,
                                  const void* L2_bf16, const void* bias_bf16,
                                  int M, int N, int K, int r, int group,
                                  void* Y, hsq_out_dtype out,
                                  void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * The activation step and the forward in one call (X in, Y out), for callers
 * that do not need the activation codes themselves: the same Y, bit for bit,
 * as hsq_quantize_act followed by hsq_linear_forward (w_e4m3 NULL) or
 * hsq_linear_forward_pre (w_e4m3 from hsq_expand_weights).  Where the GEMM
 * reads expanded operands and the many-row activation kernel applies (M at
 * least 24 per SM, r in {0, 1, 2, 4}), that kernel writes the activations'
 * E4M3 tiles itself, so no packed codes are written and no expansion runs;
 * elsewhere the call is those two steps.  The activation step's scales and U
 * live in the workspace:
 *   hsq_workspace_bytes_x(M, N, K, r, group, with_w_e4m3): its bytes (0 for an
 *     invalid shape); with_w_e4m3 != 0 when w_e4m3 will be passed.
 *   X_bf16, s, L1_bf16 as for hsq_quantize_act; the rest as for
 *   hsq_linear_forward; workspace is required, and need not hold zeros (the
 *   call clears its split-K counters itself).
 */
size_t hsq_workspace_bytes_x(int M, int N, int K, int r, int group, int with_w_e4m3);
hsq_status hsq_linear_forward_x(const void* X_bf16, const float* s, const void* L1_bf16,
                                const uint8_t* w_codes, const float* w_scales, const uint8_t* w_e4m3,
                                const void* L2_bf16, const void* bias_bf16,
                                int M, int N, int K, int r, int group,
                                void* Y, hsq_out_dtype out,
                                void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Bytes of the library's built-in scratch array used by
 * hsq_linear_forward_noalloc (16 MiB).  Every GPU on which the library is
 * loaded holds this array for the life of the process.
 */
#define HSQ_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * hsq_linear_forward without a caller-provided workspace.  The paper has no
 * counterpart: this is a convenience of the library, not a step of the method.
 *
 * Some callers cannot hand the library scratch memory: a plain C host program
 * that links only this library and has no device allocator of its own, or a
 * serving loop that must not allocate once it is running (cudaMalloc and
 * cudaFree synchronize the device and may fail under memory pressure).  For
 * them this call takes the same arguments as hsq_linear_forward minus
 * workspace/ws_bytes, and uses a file-scope device array of
 * HSQ_NOALLOC_SCRATCH_BYTES bytes for the scratch hsq_linear_forward would
 * take from the workspace (split-K counters and partial tiles, expanded codes).
 * It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *
 *   - Inputs and outputs are still caller-owned device pointers, exactly as
 *     for hsq_linear_forward; the results are the same.
 *   - Shapes whose scratch need for the given group exceeds
 *     HSQ_NOALLOC_SCRATCH_BYTES are rejected with HSQ_ERR_SCRATCH_LIMIT before
 *     anything is launched (M > 256, or M > 64 with groups of 128, needs
 *     (M + N) * Kp bytes of expanded codes, rows rounded up to whole tiles, plus
 *     any split-K scratch; smaller M needs only split-K scratch, at most about
 *     40 MB, and none up to 8 tokens).
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current); make that first call before any
 *     stream capture.
 *   - Each call first clears, on `stream`, the part of the array that must
 *     start at zero (the split-K counters).  All calls share the one array and
 *     it keeps the last call's contents, so calls whose kernels overlap on the
 *     GPU (different streams, no ordering between them) race and give wrong
 *     results; order them on one stream or with events.
 */
hsq_status hsq_linear_forward_noalloc(const uint8_t* x_codes, const float* x_scales, const float* U,
                                      const uint8_t* w_codes, const float* w_scales,
                                      const void* L2_bf16, const void* bias_bf16,
                                      int M, int N, int K, int r, int group,
                                      void* Y, hsq_out_dtype out, cudaStream_t stream);

/*
 * Activation step and forward in one launch, for decode-sized inputs: the
 * same results as hsq_quantize_act followed by hsq_linear_forward (the same
 * codes and scales; U up to its fp32 summation order), for up to 16 tokens and
 * any rank r <= 32.  Two forms, chosen from the shape (hsq_fused_form tells
 * which without launching anything):
 *   1. the weight stream, each block repeating the activation step with the
 *      codes kept on chip (nothing of the step goes through HBM), for
 *      M <= 4 tokens, rank r in {0, 1, 2, 4}, and K small enough that one
 *      block's shared memory holds the rows' widened codes, the block's weight
 *      scales and a ring of weight rows: T (Kp + 4 G + 272) + 4 G RB +
 *      S rs Kp/2 + 1024 bytes <= 227 KiB, T = M rounded up to 1, 2 or 4,
 *      RB = ceil(N / SMs) rounded up to 4 (the rows of one block), rs rows per
 *      ring stage (about half the block's rows, at least 16 KiB of them, at
 *      most half of what the ring can hold) and S = 2 stages (1 when one stage
 *      holds all RB rows), with RB <= 256 and G <= 256; e.g. K <= 16384 for
 *      groups of 64 and K <= 29696 for groups of 128 at M = 4, N = 12288 on
 *      148 SMs;
 *   2. otherwise, for M <= 16: the 16-token tensor-core decode tiles, launched
 *      cooperatively (every CTA resident at once), whose CTAs first share out
 *      the activation step -- (token, 256-channel) pieces, written to a
 *      library-owned device array -- then meet at a grid barrier (time-limited:
 *      a barrier that does not gather sets HSQ_ERR_TIMEOUT in the device status
 *      and the launch does no GEMM work), sum U per CTA in a fixed order and
 *      run the decode-tile GEMM on those codes.  The array is 8 MiB: the
 *      shape's stream-K partials (about 16 KiB per SM), its codes M Kp/2, its
 *      scales, U partials and copies must fit it (K up to about 500000 at
 *      M = 16).  As with hsq_linear_forward_noalloc, all calls share that one
 *      array: calls whose kernels overlap on the GPU (different streams, no
 *      ordering between them) race; the first call on a device looks up the
 *      array's address (once per device), so make it before any stream capture.
 * Other shapes return HSQ_ERR_UNSUPPORTED before anything is launched (use the
 * two calls).  The pages do not name this fusion; it is the step before the
 * path (activations quantized online) moved into the path's first kernel.
 *   X_bf16 [M][K] bf16, s [K] fp32, L1_bf16 [K][r] bf16 (NULL iff r == 0)
 *   w_codes/w_scales as written by hsq_pack_weights; L2_bf16, bias_bf16, Y, out
 *   as for hsq_linear_forward.  No workspace.
 */
hsq_status hsq_linear_forward_fused(const void* X_bf16, const float* s, const void* L1_bf16,
                                    const uint8_t* w_codes, const float* w_scales,
                                    const void* L2_bf16, const void* bias_bf16,
                                    int M, int N, int K, int r, int group,
                                    void* Y, hsq_out_dtype out, cudaStream_t stream);

/*
 * The form hsq_linear_forward_fused takes for this shape on the current device:
 * 0 = none (the call returns HSQ_ERR_UNSUPPORTED, or INVALID_ARG for an invalid
 * shape), 1 = the weight stream, 2 = the cooperative decode tiles.  Host
 * arithmetic only: launches nothing, and with no device present assumes 148 SMs.
 */
int hsq_fused_form(int M, int N, int K, int r, int group);

/*
 * Pack-time helper: plain truncated-SVD initialisation of the low-rank pair
 * (Table 6 of the paper, "Plain SVD" row of the L1-initialisation ablation), so
 * that weights without a calibrated pair can be packed.  Not on the forward path.
 *   L1 out [K][r] bf16: the top-r right singular vectors of W_hat = W diag(s)
 *     (orthonormal columns; each column's entry of largest magnitude positive)
 *   L2 out [r][N] bf16: L1^T W_hat^T, so that (L1 L2)^T approximates the best
 *     rank-r approximation of W_hat
 * by subspace iteration with r + 8 columns from a random start drawn from
 * `seed` (the same seed gives the same result), `iters` iterations (0..64;
 * more sharpen the subspace when W_hat's singular values r and r+1 are close),
 * then Rayleigh-Ritz.  W_bf16 [N][K], s [K] as for hsq_pack_weights; 1 <= r <=
 * min(32, N, K) (else HSQ_ERR_UNSUPPORTED).  workspace: at least
 * hsq_lowrank_workspace_bytes(N, K, r) bytes (about 4 N K).  The large products
 * are fp32 cuBLAS GEMMs; the library keeps one cuBLAS handle per device (which
 * holds device memory of its own) and serialises these calls.
 */
size_t hsq_lowrank_workspace_bytes(int N, int K, int r);
hsq_status hsq_lowrank_init(const void* W_bf16, const float* s, int N, int K, int r, int iters,
                            unsigned long long seed, void* L1_bf16, void* L2_bf16,
                            void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ------------------------------------------------------------------------
 * NVFP4 variant.  The DiRotQ page (papernotes.org, quantization settings)
 * names, next to INT4 W4A4 with groups of 64, the 4-bit floating-point W4A4
 * setting of Blackwell: the standard NVFP4 format, E2M1 values sharing one FP8
 * scale per 16 values.  The same layer (smoothed X_hat, residual R, the 16-bit
 * low-rank branch and the bias as above) with both 4-bit operands in NVFP4:
 *
 *   g  = fp32(amax(|V|) / 2688) per tensor (2688 = 6 * 448)
 *   b  = E4M3(fp32(blockmax / fp32(6 g))) per 16 values along K: round to
 *        nearest, ties to even, saturating at 448
 *   code = E2M1(fp32(v / fp32(b g))): nearest of {0, .5, 1, 1.5, 2, 3, 4, 6},
 *        ties to the even mantissa, saturating at 6; sign in bit 3; a value
 *        that rounds to 0 has code 0
 *   g = 0 gives scales 0 and codes 0; a block whose scale is 0 has codes 0.
 *   Y = gx gw sum_k (ex bx)(ew bw) + U L2 + b   (the tensor-core MMA applies
 *       the block scales; fp32 accumulation)
 *
 * Layouts (K rounded up to Kq = 64 * ceil(K/64); padding codes and scales 0):
 *   codes   [rows][Kq/2] bytes, code 2j in bits 0-3 and 2j+1 in bits 4-7
 *   scales  E4M3 bytes in atoms of 128 rows x 64 K, [ceil(rows/128)][Kq/64][512]:
 *           in atom (t, c) the byte at 16 (i % 32) + 4 (i / 32) + j is the
 *           scale of row 128 t + i, values 64 c + 16 j .. + 15 (rows past
 *           `rows` are written 0)
 *   gs      device float[2]: gs[0] receives g; gs[1] is the call's scratch
 * Supported: K % 8 == 0, N % 8 == 0, 0 <= r <= 32, 1 <= M, N, K <= 2^20;
 * pointers 16-byte aligned; calls asynchronous on `stream`.
 */
size_t hsq_fp4_codes_bytes(int rows, int K);   /* rows * Kq / 2 */
size_t hsq_fp4_scales_bytes(int rows, int K);  /* ceil(rows/128) * Kq/64 * 512 */

/* Offline: R as in hsq_pack_weights (fp64, fixed order, one fp32 rounding),
 * then NVFP4 codes, block scales and the tensor scale (two passes over W). */
hsq_status hsq_fp4_pack_weights(const void* W_bf16, const float* s, const void* L1_bf16,
                                const void* L2_bf16, int N, int K, int r, uint8_t* w_codes,
                                uint8_t* w_sf, float* w_gs, cudaStream_t stream);

/* Per forward: X_hat = fp32(fp32(X)/s), its NVFP4 codes, block scales and
 * tensor scale (a first kernel takes the tensor's absmax), and U = X_hat L1 in
 * fp32 exactly as hsq_quantize_act computes it. */
hsq_status hsq_fp4_quantize_act(const void* X_bf16, const float* s, const void* L1_bf16, int M, int K,
                                int r, uint8_t* x_codes, uint8_t* x_sf, float* x_gs, float* U,
                                cudaStream_t stream);

/* The forward on tcgen05 block-scaled MMAs (kind::mxf4nvf4, E4M3 scales per
 * 16 values applied inside the instruction, one accumulator chain per tile),
 * then Y = acc * fp32(gx gw) + U L2 + b rounded once to the output type.  No
 * workspace.  Arguments as written by the two calls above; L2, bias, Y, out as
 * for hsq_linear_forward. */
hsq_status hsq_fp4_linear_forward(const uint8_t* x_codes, const uint8_t* x_sf, const float* x_gs,
                                  const float* U, const uint8_t* w_codes, const uint8_t* w_sf,
                                  const float* w_gs, const void* L2_bf16, const void* bias_bf16,
                                  int M, int N, int K, int r, void* Y, hsq_out_dtype out,
                                  cudaStream_t stream);

/* Human-readable name of a status code (static storage). */
const char* hsq_status_string(hsq_status status);

/*
 * Synchronizes `stream`, then reads and clears the device status word of the
 * current device: HSQ_ERR_TIMEOUT if any kernel since the last read gave up
 * waiting, HSQ_ERR_CUDA if the synchronization itself failed, else HSQ_OK.
 */
hsq_status hsq_get_device_status(cudaStream_t stream);

/*
 * Test hook: when `flags` is nonzero, the next hsq_linear_forward call on this
 * host thread runs with a deliberately unreachable wait and a wait limit of
 * about `limit_ms` milliseconds, so that its kernel exits through the timeout
 * path (no data movement is issued).  Used to check that a kernel that gives
 * up returns cleanly and reports HSQ_ERR_TIMEOUT.
 */
void hsq_debug_force_timeout(int flags, int limit_ms);

#ifdef __cplusplus
}
#endif

#endif /* HSQ_H_ */
