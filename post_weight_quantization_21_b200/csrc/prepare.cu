// A2 + A3: dampening and U = upper Cholesky factor of Hd^-1 (FDE Interviews breakdown of GPTQ,
// figure "THE IDEA, VISUALLY" step 2, "U = chol(H^-1)"; nubint.ai review, "Proposed method":
// Cholesky reformulation and dampening; zhiliyouxian blog, 算法流程 "H = H + lambda * I").
//
// Route.  With J the index-reversal permutation, factor P = J Hd J = L L^T (ordinary lower
// Cholesky) and invert Y = L^-1.  Then Hd = R R^T with R = J L J upper, and U = R^-1 = J Y J is upper
// with U^T U = Hd^-1, so by uniqueness of the Cholesky factor U = chol(Hd^-1).  This needs one
// factorisation and one triangular inversion (2/3 d^3 flops) instead of the pages' factorise /
// invert / multiply / factorise route (4/3 d^3 flops); the oracle computes the pages' route.
//
// Everything runs in place in the caller's U buffer:
//   1. diag_mean      lambda = damp * mean(diag H)                              (1 CTA)
//   2. reverse_damp   lower(P) = J (H + lambda I) J                              (from H's upper part)
//   3. chol_step x D  right-looking blocked Cholesky, one launch per 64-column panel.  Launch j
//                     applies panel j-1's rank-64 update to every tile right of it, and factors
//                     panel j: every CTA of the panel recomputes the 64x64 diagonal block, so the
//                     CTAs of a launch never wait on one another.  The diagonal blocks' inverses
//                     go to the workspace.
//   4. leaf_copy      diagonal blocks of P <- their inverses
//   5. trtri levels   Y = L^-1 by doubling: [[A,0],[C,B]]^-1 = [[A^-1,0],[-B^-1 C A^-1, B^-1]].
//                     T = C A^-1 is parked transposed in P's unused upper triangle.
//   6. rotate         U = J Y J (lower of the buffer -> upper), strict lower part zeroed.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int NB = 64;
constexpr int LDS = NB + 1;
constexpr int kThreads = 256;

struct PrepPlan {
  int D;  // 64-blocks per dimension
};

PrepPlan prep_plan(int64_t d) { return PrepPlan{(int)((d + NB - 1) / NB)}; }

// workspace layout: [0,256) lambda (float); [256, ...) D inverse diagonal blocks of 64x64 fp32
size_t side_offset() { return 256; }

__global__ void diag_mean_kernel(const float* __restrict__ H, int d, float damp, float* __restrict__ lam) {
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += (double)H[(size_t)i * d + i];
  __shared__ double red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) *lam = (float)((double)damp * s / (double)d);
  }
}

// lower(P)[i][j] = H[d-1-i][d-1-j] (+lambda on the diagonal); 32x32 tiles, block (32, 8).
__global__ void reverse_damp_kernel(const float* __restrict__ H, int d, const float* __restrict__ lam,
                                    float* __restrict__ P) {
  if (blockIdx.x > blockIdx.y) return;
  const float l = *lam;
  const int j = blockIdx.x * 32 + threadIdx.x;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = blockIdx.y * 32 + r;
    if (i >= d || j >= d || j > i) continue;
    float v = H[(size_t)(d - 1 - i) * d + (d - 1 - j)];
    if (i == j) v += l;
    P[(size_t)i * d + j] = v;
  }
}

__device__ __forceinline__ void load_tile(float (*s)[LDS], const float* __restrict__ P, int d, int r0,
                                          int c0, bool identity_pad) {
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    const int gr = r0 + r, gc = c0 + c;
    float v;
    if (gr < d && gc < d)
      v = P[(size_t)gr * d + gc];
    else
      v = (identity_pad && r == c) ? 1.0f : 0.0f;
    s[r][c] = v;
  }
}

// acc[p][q] += sum_m A[ty*4+p][m] * B[tx*4+q][m]      (A B^T)
__device__ __forceinline__ void tile_nt(float acc[4][4], const float (*A)[LDS], const float (*B)[LDS],
                                        int ty, int tx, int m_lo = 0, int m_hi = NB) {
  for (int m = m_lo; m < m_hi; ++m) {
    float a[4], b[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) a[p] = A[ty * 4 + p][m];
#pragma unroll
    for (int q = 0; q < 4; ++q) b[q] = B[tx * 4 + q][m];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
  }
}

// acc[p][q] += sum_m A[ty*4+p][m] * B[m][tx*4+q]      (A B)
__device__ __forceinline__ void tile_nn(float acc[4][4], const float (*A)[LDS], const float (*B)[LDS],
                                        int ty, int tx) {
  for (int m = 0; m < NB; ++m) {
    float a[4], b[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) a[p] = A[ty * 4 + p][m];
#pragma unroll
    for (int q = 0; q < 4; ++q) b[q] = B[m][tx * 4 + q];
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[p][q] = fmaf(a[p], b[q], acc[p][q]);
  }
}

__device__ __forceinline__ void zero_acc(float acc[4][4]) {
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[p][q] = 0.f;
}

// In-smem Cholesky of the 64x64 block A (lower part) followed by its inverse Li (lower).
// pivot_base: reversed-order index of A's first column (for the failure report).
__device__ void factor_and_invert(float (*A)[LDS], float (*Li)[LDS], int d, int pivot_base,
                                  int32_t* status) {
  const int tid = threadIdx.x;
  // right-looking with an unscaled pivot column: A[i][c] -= A[i][k] A[c][k] / A[k][k]
  for (int k = 0; k < NB; ++k) {
    const float piv = A[k][k];
    if (tid == 0 && !(piv > 0.0f && isfinite(piv)))
      report_status(status, GPTQ_ERR_NOT_PD, d - 1 - (pivot_base + k));
    const float inv = 1.0f / piv;
    for (int e = tid; e < NB * NB; e += kThreads) {
      const int i = e / NB, c = e % NB;
      if (c > k && c <= i) A[i][c] = fmaf(-A[i][k] * inv, A[c][k], A[i][c]);
    }
    __syncthreads();
  }
  // scale: L[i][c] = A[i][c] / sqrt(A[c][c]) for i >= c; zero above the diagonal
  for (int e = tid; e < NB * NB; e += kThreads) {
    const int i = e / NB, c = e % NB;
    Li[i][c] = (c <= i) ? A[i][c] / sqrtf(A[c][c]) : 0.0f;
  }
  __syncthreads();
  for (int e = tid; e < NB * NB; e += kThreads) {
    const int i = e / NB, c = e % NB;
    A[i][c] = Li[i][c];
    Li[i][c] = (i == c) ? 1.0f : 0.0f;  // right-hand sides R = I
  }
  __syncthreads();
  // forward substitution on all 64 right-hand sides: R[i][c] -= L[i][k] R[k][c] / L[k][k]
  for (int k = 0; k < NB; ++k) {
    const float inv = 1.0f / A[k][k];
    for (int e = tid; e < NB * NB; e += kThreads) {
      const int i = e / NB, c = e % NB;
      if (i > k && c <= k) Li[i][c] = fmaf(-A[i][k] * inv, Li[k][c], Li[i][c]);
    }
    __syncthreads();
  }
  for (int e = tid; e < NB * NB; e += kThreads) {
    const int i = e / NB, c = e % NB;
    Li[i][c] = (c <= i) ? Li[i][c] / A[i][i] : 0.0f;
  }
  __syncthreads();
}

__device__ __forceinline__ void tri_index(int t, int& rr, int& cc) {
  // t -> (rr, cc) with 0 <= cc <= rr, row-major over the lower triangle
  int r = (int)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while ((r + 1) * (r + 2) / 2 <= t) ++r;
  while (r * (r + 1) / 2 > t) --r;
  rr = r;
  cc = t - r * (r + 1) / 2;
}

// One launch per panel j (see the file comment).  Blocks [0, D-j) factor the panel's row blocks;
// the rest update the trailing lower tiles (r, c), j+1 <= c <= r < D, with panel j-1.
__global__ void __launch_bounds__(kThreads) chol_step_kernel(float* __restrict__ P, int d, int D, int j,
                                                              float* __restrict__ side,
                                                              int32_t* __restrict__ status) {
  extern __shared__ float smem[];
  float(*S0)[LDS] = reinterpret_cast<float(*)[LDS]>(smem);
  float(*S1)[LDS] = S0 + NB;
  float(*S2)[LDS] = S1 + NB;
  float(*S3)[LDS] = S2 + NB;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int n_panel = D - j;
  float acc[4][4];
  if ((int)blockIdx.x < n_panel) {
    const int r = j + blockIdx.x;
    // S0: diagonal block (j, j) ; S1: L(j, j-1) ; S2: tile (r, j) ; S3: L(r, j-1)
    load_tile(S0, P, d, j * NB, j * NB, true);
    if (r > j) load_tile(S2, P, d, r * NB, j * NB, false);
    if (j > 0) {
      load_tile(S1, P, d, j * NB, (j - 1) * NB, false);
      if (r > j) load_tile(S3, P, d, r * NB, (j - 1) * NB, false);
    }
    __syncthreads();
    if (j > 0) {
      zero_acc(acc);
      tile_nt(acc, S1, S1, ty, tx);
      float acc2[4][4];
      zero_acc(acc2);
      if (r > j) tile_nt(acc2, S3, S1, ty, tx);
      __syncthreads();
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          S0[ty * 4 + p][tx * 4 + q] -= acc[p][q];
          if (r > j) S2[ty * 4 + p][tx * 4 + q] -= acc2[p][q];
        }
      __syncthreads();
    }
    // S1 <- inverse of the factored diagonal block (S0 becomes L_jj)
    factor_and_invert(S0, S1, d, j * NB, status);
    if (r == j) {
      float* out = side + (size_t)j * NB * NB;
      for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) out[e] = S1[e / NB][e % NB];
    } else {
      // L(r, j) = tile(r, j) * Li^T
      zero_acc(acc);
      tile_nt(acc, S2, S1, ty, tx);
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int gr = r * NB + ty * 4 + p, gc = j * NB + tx * 4 + q;
          if (gr < d && gc < d) P[(size_t)gr * d + gc] = acc[p][q];
        }
    }
    return;
  }
  // trailing update with panel j-1
  int rr, cc;
  tri_index(blockIdx.x - n_panel, rr, cc);
  const int r = j + 1 + rr, c = j + 1 + cc;
  load_tile(S0, P, d, r * NB, (j - 1) * NB, false);
  load_tile(S1, P, d, c * NB, (j - 1) * NB, false);
  __syncthreads();
  zero_acc(acc);
  tile_nt(acc, S0, S1, ty, tx);
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int gr = r * NB + ty * 4 + p, gc = c * NB + tx * 4 + q;
      if (gr < d && gc < d && gc <= gr) P[(size_t)gr * d + gc] -= acc[p][q];
    }
}

__global__ void leaf_copy_kernel(float* __restrict__ P, int d, const float* __restrict__ side) {
  const int j = blockIdx.x;
  const float* src = side + (size_t)j * NB * NB;
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    const int gr = j * NB + r, gc = j * NB + c;
    if (gr < d && gc < d) P[(size_t)gr * d + gc] = (c <= r) ? src[e] : 0.0f;
  }
}

// Level with g-block halves.  Pair p: A = blocks [a0, a0+g), B = [a0+g, min(a0+2g, D)).
// T tile (r, c) (r in B, c in A) = sum_{k=c}^{a0+g-1} C(r, k) * Ainv(k, c), stored transposed at
// block (c, r) of the upper triangle.
__global__ void __launch_bounds__(kThreads) trtri_t_kernel(float* __restrict__ P, int d, int D, int g) {
  extern __shared__ float smem[];
  float(*Cs)[LDS] = reinterpret_cast<float(*)[LDS]>(smem);
  float(*As)[LDS] = Cs + NB;
  const int per_pair = g * g;  // upper bound of tiles per pair (B may be shorter)
  const int p = blockIdx.x / per_pair, t = blockIdx.x % per_pair;
  const int a0 = p * 2 * g, b0 = a0 + g;
  const int b1 = min(a0 + 2 * g, D);
  const int r = b0 + t / g, c = a0 + t % g;
  if (r >= b1) return;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4];
  zero_acc(acc);
  for (int k = c; k < a0 + g; ++k) {
    load_tile(Cs, P, d, r * NB, k * NB, false);
    load_tile(As, P, d, k * NB, c * NB, false);
    __syncthreads();
    tile_nn(acc, Cs, As, ty, tx);
    __syncthreads();
  }
#pragma unroll
  for (int pp = 0; pp < 4; ++pp)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int x = ty * 4 + pp, y = tx * 4 + q;  // T[x][y] -> P[c*NB + y][r*NB + x]
      const int gr = c * NB + y, gc = r * NB + x;
      if (gr < d && gc < d) P[(size_t)gr * d + gc] = acc[pp][q];
    }
}

// Y tile (r, c) = - sum_{k=b0}^{r} Binv(r, k) * T(k, c), written over C(r, c).
__global__ void __launch_bounds__(kThreads) trtri_y_kernel(float* __restrict__ P, int d, int D, int g) {
  extern __shared__ float smem[];
  float(*Bs)[LDS] = reinterpret_cast<float(*)[LDS]>(smem);
  float(*Ts)[LDS] = Bs + NB;
  const int per_pair = g * g;
  const int p = blockIdx.x / per_pair, t = blockIdx.x % per_pair;
  const int a0 = p * 2 * g, b0 = a0 + g;
  const int b1 = min(a0 + 2 * g, D);
  const int r = b0 + t / g, c = a0 + t % g;
  if (r >= b1) return;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4];
  zero_acc(acc);
  for (int k = b0; k <= r; ++k) {
    load_tile(Bs, P, d, r * NB, k * NB, false);
    load_tile(Ts, P, d, c * NB, k * NB, false);  // holds T(k, c) transposed
    __syncthreads();
    tile_nt(acc, Bs, Ts, ty, tx);
    __syncthreads();
  }
#pragma unroll
  for (int pp = 0; pp < 4; ++pp)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int gr = r * NB + ty * 4 + pp, gc = c * NB + tx * 4 + q;
      if (gr < d && gc < d) P[(size_t)gr * d + gc] = -acc[pp][q];
    }
}

// U = J Y J: buffer[d-1-i][d-1-j] <- buffer[i][j] for i > j, buffer[i][j] <- 0; diagonal reversed.
__global__ void rotate_kernel(float* __restrict__ P, int d) {
  if (blockIdx.x > blockIdx.y) return;
  const int j = blockIdx.x * 32 + threadIdx.x;
  for (int r = threadIdx.y; r < 32; r += blockDim.y) {
    const int i = blockIdx.y * 32 + r;
    if (i >= d || j >= d || j > i) continue;
    if (i > j) {
      const float v = P[(size_t)i * d + j];
      P[(size_t)(d - 1 - i) * d + (d - 1 - j)] = v;
      P[(size_t)i * d + j] = 0.0f;
    } else if (i < d - 1 - i) {
      const size_t a = (size_t)i * d + i, b = (size_t)(d - 1 - i) * d + (d - 1 - i);
      const float va = P[a], vb = P[b];
      P[a] = vb;
      P[b] = va;
    }
  }
}

}  // namespace

size_t prepare_workspace(int64_t d) {
  PrepPlan p = prep_plan(d);
  return side_offset() + (size_t)p.D * NB * NB * sizeof(float);
}

gptq_status prepare_launch(const float* H, int64_t d64, float damp, float* U, int32_t* status,
                           void* workspace, cudaStream_t stream) {
  const int d = (int)d64;
  PrepPlan pl = prep_plan(d);
  const int D = pl.D;
  char* ws = static_cast<char*>(workspace);
  float* lam = reinterpret_cast<float*>(ws);
  float* side = reinterpret_cast<float*>(ws + side_offset());
  static bool attr_done = false;
  const int smem4 = 4 * NB * LDS * sizeof(float);
  const int smem2 = 2 * NB * LDS * sizeof(float);
  if (!attr_done) {
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(chol_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem4));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(trtri_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2));
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(trtri_y_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2));
    attr_done = true;
  }
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), stream));
  diag_mean_kernel<<<1, 1024, 0, stream>>>(H, d, damp, lam);
  GPTQ_LAUNCH_CHECK();
  const int D32 = (d + 31) / 32;
  reverse_damp_kernel<<<dim3(D32, D32), dim3(32, 8), 0, stream>>>(H, d, lam, U);
  GPTQ_LAUNCH_CHECK();
  for (int j = 0; j < D; ++j) {
    int n = D - j;
    if (j > 0) n += (D - j - 1) * (D - j) / 2;
    chol_step_kernel<<<n, kThreads, smem4, stream>>>(U, d, D, j, side, status);
    GPTQ_LAUNCH_CHECK();
  }
  leaf_copy_kernel<<<D, kThreads, 0, stream>>>(U, d, side);
  GPTQ_LAUNCH_CHECK();
  for (int g = 1; g < D; g *= 2) {
    const int pairs = (D + 2 * g - 1) / (2 * g);
    const int n = pairs * g * g;
    trtri_t_kernel<<<n, kThreads, smem2, stream>>>(U, d, D, g);
    GPTQ_LAUNCH_CHECK();
    trtri_y_kernel<<<n, kThreads, smem2, stream>>>(U, d, D, g);
    GPTQ_LAUNCH_CHECK();
  }
  rotate_kernel<<<dim3(D32, D32), dim3(32, 8), 0, stream>>>(U, d);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
