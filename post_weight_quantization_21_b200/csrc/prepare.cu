// A2 + A3: dampening and U = upper Cholesky factor of Hd^-1 (FDE Interviews breakdown of GPTQ,
// figure "THE IDEA, VISUALLY" step 2, "U = chol(H^-1)"; nubint.ai review, "Proposed method":
// Cholesky reformulation and dampening; zhiliyouxian blog, 算法流程 "H = H + lambda * I").
//
// Route.  With J the index-reversal permutation, factor P = J Hd J = L L^T (ordinary lower
// Cholesky) and invert Y = L^-1.  Then Hd = R R^T with R = J L J upper, and U = R^-1 = J Y J is upper
// with U^T U = Hd^-1, so by uniqueness of the Cholesky factor U = chol(Hd^-1).  One factorisation and
// one triangular inversion (2/3 d^3 flops) replace the pages' factorise / invert / multiply /
// factorise route (4/3 d^3 flops); the oracle computes the pages' route.
//
// One cooperative launch, one CTA (128 threads) per work item at a time, grid-wide barriers between
// phases (bounded waits).  32x32 blocks, D = ceil(d / 32) block rows.  Everything lives in the
// caller's U buffer ("P"): L (then Y) in the lower block triangle, the running right-hand sides R of
// the inversion transposed in the upper block triangle.
//   phase A   lambda = damp * mean(diag H)
//   phase B   lower(P) = J (H + lambda I) J, upper(P) = 0
//   phase j = 0..D  (each item independent of the others in its phase)
//     panel     r = j..D-1: update P(r, j) and the diagonal block P(j, j) with panel j-1, factor the
//               diagonal block and invert it (one warp, registers), L(r, j) = P(r, j) L(j,j)^-T.
//               Every panel item refactors the 32x32 diagonal block, so no barrier separates the
//               factorisation from the triangular solve.
//     trailing  P(r, c) -= L(r, j-1) L(c, j-1)^T for j+1 <= c <= r
//     inverse   Y(j-1, c) = L(j-1,j-1)^-1 R(j-1, c) (final row block of Y, written over L(j-1, c));
//               R(i, c) -= L(i, j-1) Y(j-1, c) for i >= j.  (Right-looking block forward
//               substitution of L Y = I, one block row behind the factorisation.)
//   phase R   U = J Y J: lower block triangle -> upper, strict lower part zeroed.
#include <math.h>

#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int NB = 32;
constexpr int TS = 36;  // shared tile row stride (floats): rows stay 16-byte aligned
constexpr int kThreads = 128;
constexpr int kYChunk = 4;  // R updates per inverse item
constexpr long long kWaitCycles = 4000000000LL;

struct PrepArgs {
  const float* H;
  float* P;
  float* side;     // D inverse diagonal blocks, 32x32 row-major
  float* lam;
  unsigned* bar;   // [0] arrivals, [32] generation (separate 128-byte lines)
  int* abort_flag;
  int32_t* status;
  float damp;
  int d, D;
};

// ------------------------------------------------------------------ grid barrier (bounded)
__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Grid barrier over a monotonically increasing arrival count (zeroed before the launch): barrier
// number g is complete once the count reaches g * gridDim.x, so arriving is one atomic and waiting
// is polling that word; no reset or separate release word is needed.  The wait is bounded.
__device__ bool grid_barrier(const PrepArgs& a, unsigned& gen) {
  __shared__ int s_ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    int ok = 1;
    const unsigned target = (gen + 1) * gridDim.x;
    unsigned* count = a.bar;
    __threadfence();
    const unsigned arrived = atomicAdd(count, 1u) + 1u;
    if (arrived != target) {
      const long long t0 = clock64();
      unsigned ns = 16;
      while (ld_acquire(count) < target) {
        if (*(volatile int*)a.abort_flag) {
          ok = 0;
          break;
        }
        if (clock64() - t0 > kWaitCycles) {
          *(volatile int*)a.abort_flag = 1;
          report_status(a.status, GPTQ_ERR_TIMEOUT, -1);
          ok = 0;
          break;
        }
        __nanosleep(ns);
        if (ns < 64) ns *= 2;
      }
    }
    __threadfence();
    gen += 1;
    s_ok = ok;
  }
  __syncthreads();
  return s_ok != 0;
}

// ------------------------------------------------------------------ 32x32 tile helpers
// Loads read through L2 (__ldcg): P is written by other CTAs during the launch.
__device__ __forceinline__ float ldp(const float* p) { return __ldcg(p); }

// A 32x32 block held in registers, 8 values per thread: element e = tid + 128 k sits at row e / 32,
// column e % 32 (each warp reads whole rows, coalesced).  fetch() issues all 8 loads before any is
// used, so a tile costs one L2 round trip; put_*() store it to shared memory.
struct TileRegs {
  float v[8];
};

__device__ __forceinline__ TileRegs fetch(const float* P, int d, int br, int bc, bool identity_pad = false) {
  TileRegs t;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = threadIdx.x + kThreads * k;
    const int r = e >> 5, c = e & 31;
    const int gr = br * NB + r, gc = bc * NB + c;
    t.v[k] = (gr < d && gc < d) ? ldp(P + (size_t)gr * d + gc) : ((identity_pad && r == c) ? 1.0f : 0.0f);
  }
  return t;
}

// A 32x32 row-major block M in global memory (the inverse diagonal blocks)
__device__ __forceinline__ TileRegs fetch_block(const float* M) {
  TileRegs t;
#pragma unroll
  for (int k = 0; k < 8; ++k) t.v[k] = ldp(M + threadIdx.x + kThreads * k);
  return t;
}

__device__ __forceinline__ void put_nat(float (*S)[TS], const TileRegs& t) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = threadIdx.x + kThreads * k;
    S[e >> 5][e & 31] = t.v[k];
  }
}

__device__ __forceinline__ void put_tr(float (*S)[TS], const TileRegs& t) {
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int e = threadIdx.x + kThreads * k;
    S[e & 31][e >> 5] = t.v[k];
  }
}

// Thread (ty, tx) owns rows 2ty, 2ty+1 and columns 4tx..4tx+3 of a 32x32 output.
// acc[p][q] += sum_m Ak[m][2ty+p] * Bk[m][4tx+q]   (operands stored k-major)
__device__ __forceinline__ void mma32(float acc[2][4], const float (*Ak)[TS], const float (*Bk)[TS], int ty,
                                      int tx) {
#pragma unroll 8
  for (int m = 0; m < NB; ++m) {
    const float2 av = *reinterpret_cast<const float2*>(&Ak[m][2 * ty]);
    const float4 bv = *reinterpret_cast<const float4*>(&Bk[m][4 * tx]);
    acc[0][0] = fmaf(av.x, bv.x, acc[0][0]);
    acc[0][1] = fmaf(av.x, bv.y, acc[0][1]);
    acc[0][2] = fmaf(av.x, bv.z, acc[0][2]);
    acc[0][3] = fmaf(av.x, bv.w, acc[0][3]);
    acc[1][0] = fmaf(av.y, bv.x, acc[1][0]);
    acc[1][1] = fmaf(av.y, bv.y, acc[1][1]);
    acc[1][2] = fmaf(av.y, bv.z, acc[1][2]);
    acc[1][3] = fmaf(av.y, bv.w, acc[1][3]);
  }
}

__device__ __forceinline__ void zero(float acc[2][4]) {
#pragma unroll
  for (int p = 0; p < 2; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[p][q] = 0.0f;
}

// Warp 0: factor the 32x32 block A (lower part, natural layout) and write its inverse transposed:
// LiT[m][y] = L^-1[y][m].  Lane i keeps row i of A; lane c keeps column c of the right-hand sides
// of L Y = I.  Right-looking with an unscaled pivot column:
//   A[i][x] -= A[i][k] A[x][k] / A[k][k],   R[x][c] -= A[x][k] R[k][c] / A[k][k]   (x > k)
// then L^-1[i][c] = R[i][c] / sqrt(pivot_i).  Entry A[x][k] of the pivot column reaches every lane by
// a shuffle from lane x.  pivot_base: reversed-order index of the block's first column, for the
// failure report.
__device__ void warp_factor_invert(const float (*A)[TS], float (*LiT)[TS], int d, int pivot_base, int32_t* status) {
  const int lane = threadIdx.x & 31;
  float a[NB], rr[NB], rs[NB];
#pragma unroll
  for (int c = 0; c < NB; ++c) {
    a[c] = A[lane][c];
    rr[c] = (c == lane) ? 1.0f : 0.0f;
  }
  int bad = -1;  // first non-positive pivot (the pivot is the same on every lane)
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    const float p = __shfl_sync(0xffffffffu, a[k], k);
    const float inv = __fdividef(1.0f, p);
    rs[k] = rsqrtf(p);
    if (bad < 0 && !(p > 0.0f && isfinite(p)) && pivot_base + k < d) bad = k;
    const float li = a[k] * inv;
    const float t = rr[k] * inv;
#pragma unroll
    for (int x = k + 1; x < NB; ++x) {
      const float v = __shfl_sync(0xffffffffu, a[k], x);  // A[x][k]
      a[x] = fmaf(-li, v, a[x]);
      rr[x] = fmaf(-v, t, rr[x]);
    }
  }
  if (lane == 0 && bad >= 0) report_status(status, GPTQ_ERR_NOT_PD, d - 1 - (pivot_base + bad));
  // column `lane` of L^-1 is row `lane` of LiT
#pragma unroll
  for (int i = 0; i < NB; ++i) LiT[lane][i] = (i >= lane) ? rr[i] * rs[i] : 0.0f;
  __syncwarp();
}

__global__ void __launch_bounds__(kThreads) prepare_kernel(const PrepArgs a) {
  __shared__ __align__(16) float S0[NB][TS];
  __shared__ __align__(16) float S1[NB][TS];
  __shared__ __align__(16) float S2[NB][TS];
  __shared__ __align__(16) float S3[NB][TS];
  __shared__ __align__(16) float S4[NB][TS];
  const int tid = threadIdx.x;
  const int ty = tid >> 3, tx = tid & 7;
  const int d = a.d, D = a.D;
  float* P = a.P;
  unsigned gen = 0;

  // ---------------------------------------------------------------- phase A: lambda
  if (blockIdx.x == 0) {
    double s = 0.0;
    for (int i = tid; i < d; i += kThreads) s += (double)a.H[(size_t)i * d + i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    __shared__ double red[kThreads / 32];
    if ((tid & 31) == 0) red[tid >> 5] = s;
    __syncthreads();
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < kThreads / 32; ++w) t += red[w];
      *a.lam = (float)((double)a.damp * t / (double)d);
    }
  }
  if (!grid_barrier(a, gen)) return;

  // ---------------------------------------------------------------- phase B: reversed, damped copy
  {
    const float lam = __ldcg(a.lam);
    for (int i = blockIdx.x; i < d; i += gridDim.x) {
      const float* src = a.H + (size_t)(d - 1 - i) * d + (d - 1);
      float* dst = P + (size_t)i * d;
      for (int j = tid; j < d; j += kThreads) {
        float v = 0.0f;
        if (j <= i) {
          v = src[-j];
          if (i == j) v += lam;
        }
        dst[j] = v;
      }
    }
  }
  if (!grid_barrier(a, gen)) return;

  // ---------------------------------------------------------------- phases 0..D
  for (int j = 0; j <= D; ++j) {
    const int n_panel = (j < D) ? D - j : 0;
    const int n_trail = (j >= 1 && j < D) ? (D - j - 1) * (D - j) / 2 : 0;
    const int rows_left = (j < D) ? D - j : 0;
    const int chunks = (rows_left + kYChunk - 1) / kYChunk;
    const int per_c = chunks > 0 ? chunks : 1;
    const int n_inv = (j >= 1) ? j * per_c : 0;
    const int n_items = n_panel + n_trail + n_inv;
    // Item assignment.  A panel item (~6 us: its 32x32 factorisation) or an inverse item (~5 us)
    // gets a CTA of its own; the short trailing items share the remaining CTAs.  Handing a second
    // item to a panel CTA would stretch the phase, and every CTA waits for the longest one.
    const int G = gridDim.x;
    const bool by_role = n_panel + n_inv < G;
    for (int k = 0;; ++k) {
      int it;
      if (!by_role) {
        it = blockIdx.x + k * G;
        if (it >= n_items) break;
      } else if ((int)blockIdx.x < n_panel) {
        if (k > 0) break;
        it = blockIdx.x;
      } else if ((int)blockIdx.x < n_panel + n_inv) {
        if (k > 0) break;
        it = n_panel + n_trail + ((int)blockIdx.x - n_panel);
      } else {
        const int t = ((int)blockIdx.x - n_panel - n_inv) + k * (G - n_panel - n_inv);
        if (t >= n_trail) break;
        it = n_panel + t;
      }
      float acc[2][4], acc2[2][4];
      if (it < n_panel) {
        // ------------------------------------------------ panel item
        const int r = j + it;
        {
          const TileRegs t0 = fetch(P, d, j, j, true);                    // diagonal block
          const TileRegs t1 = fetch(P, d, r > j ? r : D, j);              // own block (none when r == j)
          const TileRegs t2 = fetch(P, d, j > 0 ? j : D, j - 1);          // L(j, j-1)
          const TileRegs t3 = fetch(P, d, (j > 0 && r > j) ? r : D, j - 1);  // L(r, j-1)
          put_nat(S0, t0);
          put_nat(S1, t1);
          put_tr(S2, t2);
          put_tr(S3, t3);
        }
        __syncthreads();
        if (j > 0) {
          zero(acc);
          mma32(acc, S2, S2, ty, tx);
          zero(acc2);
          if (r > j) mma32(acc2, S3, S2, ty, tx);
          __syncthreads();
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              S0[2 * ty + p][4 * tx + q] -= acc[p][q];
              if (r > j) S1[2 * ty + p][4 * tx + q] -= acc2[p][q];
            }
        }
        __syncthreads();  // the transposition below reads elements other warps just updated
        // S3 <- tile(r, j) transposed, for the triangular solve
        if (r > j) {
          for (int e = tid; e < NB * NB; e += kThreads) S3[e & 31][e >> 5] = S1[e >> 5][e & 31];
        }
        __syncthreads();
        if (tid < 32) warp_factor_invert(S0, S4, d, j * NB, a.status);
        __syncthreads();
        if (r == j) {
          float* out = a.side + (size_t)j * NB * NB;  // natural layout: out[y][m] = S4[m][y]
          for (int e = tid; e < NB * NB; e += kThreads) out[e] = S4[e & 31][e >> 5];
        } else {
          zero(acc);
          mma32(acc, S3, S4, ty, tx);  // L(r, j) = tile(r, j) * Linv^T
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int gr = r * NB + 2 * ty + p, gc = j * NB + 4 * tx + q;
              if (gr < d && gc < d) P[(size_t)gr * d + gc] = acc[p][q];
            }
        }
      } else if (it < n_panel + n_trail) {
        // ------------------------------------------------ trailing item
        const int t = it - n_panel;
        int rr = (int)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
        while ((rr + 1) * (rr + 2) / 2 <= t) ++rr;
        while (rr * (rr + 1) / 2 > t) --rr;
        const int cc = t - rr * (rr + 1) / 2;
        const int r = j + 1 + rr, c = j + 1 + cc;
        float old[2][4];
        {
          const TileRegs t0 = fetch(P, d, r, j - 1);
          const TileRegs t1 = fetch(P, d, c, j - 1);
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int gr = r * NB + 2 * ty + p, gc = c * NB + 4 * tx + q;
              old[p][q] = (gr < d && gc < d) ? ldp(P + (size_t)gr * d + gc) : 0.0f;
            }
          put_tr(S0, t0);
          put_tr(S1, t1);
        }
        __syncthreads();
        zero(acc);
        mma32(acc, S0, S1, ty, tx);
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int gr = r * NB + 2 * ty + p, gc = c * NB + 4 * tx + q;
            if (gr < d && gc < d) P[(size_t)gr * d + gc] = old[p][q] - acc[p][q];
          }
      } else {
        // ------------------------------------------------ inverse item: column block c, rows chunk
        const int t = it - n_panel - n_trail;
        const int c = t / per_c, ch = t % per_c;
        // Y(j-1, c) = Linv_{j-1} R(j-1, c);  R(j-1, j-1) = I, else R(j-1, c) sits transposed at P(c, j-1)
        {
          const TileRegs t0 = fetch_block(a.side + (size_t)(j - 1) * NB * NB);
          const TileRegs t1 = fetch(P, d, c < j - 1 ? c : D, j - 1);
          put_tr(S0, t0);  // S0[m][x] = Linv[x][m]
          put_tr(S1, t1);  // S1[m][y] = R(j-1, c)[m][y]  (R(j-1, c) is stored transposed at P(c, j-1))
        }
        __syncthreads();
        if (c < j - 1) {
          zero(acc);
          mma32(acc, S0, S1, ty, tx);
        } else {
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[p][q] = S0[4 * tx + q][2 * ty + p];
        }
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int q = 0; q < 4; ++q) S2[2 * ty + p][4 * tx + q] = acc[p][q];  // Y natural
        if (ch == 0) {
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int gr = (j - 1) * NB + 2 * ty + p, gc = c * NB + 4 * tx + q;
              if (gr < d && gc < d) P[(size_t)gr * d + gc] = acc[p][q];
            }
        }
        const int i0 = j + ch * kYChunk;
        const int i1 = min(i0 + kYChunk, D);
        for (int i = i0; i < i1; ++i) {
          float old[2][4];
          const TileRegs t3 = fetch(P, d, i, j - 1);
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // R(i, c) is stored transposed at P(c, i)
              const int gr = c * NB + 4 * tx + q, gc = i * NB + 2 * ty + p;
              old[p][q] = (gr < d && gc < d) ? ldp(P + (size_t)gr * d + gc) : 0.0f;
            }
          __syncthreads();
          put_tr(S3, t3);  // S3[m][x] = L(i, j-1)[x][m]
          __syncthreads();
          zero(acc);
          mma32(acc, S3, S2, ty, tx);
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int gr = c * NB + 4 * tx + q, gc = i * NB + 2 * ty + p;
              if (gr < d && gc < d) P[(size_t)gr * d + gc] = old[p][q] - acc[p][q];
            }
        }
      }
      __syncthreads();
    }
    if (!grid_barrier(a, gen)) return;
  }

  // ---------------------------------------------------------------- phase R: U = J Y J in place
  for (int i = blockIdx.x; i < d; i += gridDim.x) {
    float* row = P + (size_t)i * d;
    float* mirror = P + (size_t)(d - 1 - i) * d + (d - 1);
    for (int j = tid; j <= i; j += kThreads) {
      if (j < i) {
        mirror[-j] = ldp(row + j);
        row[j] = 0.0f;
      } else if (i < d - 1 - i) {  // diagonal pair (i, i) <-> (d-1-i, d-1-i)
        const float va = ldp(row + i), vb = ldp(mirror - i);
        row[i] = vb;
        mirror[-i] = va;
      }
    }
  }
}

constexpr size_t kSideOffset = 1024;

}  // namespace

// Orders up to kSmallOrder run as the one-launch kernel above (the panel chain dominates); larger
// orders are dominated by dense block products and take the 128-block path (prepare_blocked.cu).
constexpr int64_t kSmallOrder = 1024;

// the blocked path's tile products go to the tensor cores when rows are 16-byte aligned
bool prepare_uses_tensor_cores(int64_t d) { return d > kSmallOrder && d % 4 == 0; }

size_t prepare_workspace(int64_t d) {
  if (d > kSmallOrder) return prepare_blocked_workspace(d);
  const int64_t D = (d + NB - 1) / NB;
  return kSideOffset + (size_t)D * NB * NB * sizeof(float);
}

gptq_status prepare_launch(const float* H, int64_t d64, float damp, float* U, int32_t* status, void* workspace,
                           cudaStream_t stream, bool lookahead, bool pair) {
  if (d64 > kSmallOrder) return prepare_blocked_launch(H, d64, damp, U, status, workspace, stream, lookahead, pair);
  const int d = (int)d64;
  char* ws = static_cast<char*>(workspace);
  PrepArgs a;
  a.H = H;
  a.P = U;
  a.lam = reinterpret_cast<float*>(ws);
  a.bar = reinterpret_cast<unsigned*>(ws + 256);
  a.abort_flag = reinterpret_cast<int*>(ws + 512);
  a.side = reinterpret_cast<float*>(ws + kSideOffset);
  a.status = status;
  a.damp = damp;
  a.d = d;
  a.D = (d + NB - 1) / NB;
  int dev = 0, sms = 0, occ = 0, coop = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
  if (!coop) return GPTQ_ERR_CUDA;
  GPTQ_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prepare_kernel, kThreads, 0));
  if (occ < 1) return GPTQ_ERR_CUDA;
  // one CTA per SM: the orders served here have few items per phase, and more CTAs only slow the
  // grid barrier
  const int grid = sms;
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), stream));
  GPTQ_CUDA_TRY(cudaMemsetAsync(ws + 256, 0, 512, stream));  // barrier words and abort flag
  void* args[] = {&a};
  GPTQ_CUDA_TRY(cudaLaunchCooperativeKernel(reinterpret_cast<void*>(prepare_kernel), dim3(grid), dim3(kThreads),
                                            args, 0, stream));
  count_launch();
  return GPTQ_OK;
}

}  // namespace gptq

namespace gptq {
// ------------------------------------------------------------------------------------------------
// Allocation-free variant.  The prepare step's scratch (damping value, barrier words, the inverse
// diagonal blocks: at most 1 KiB + d/128 * 64 KiB, about 4 MiB at d = 8192) lives in this file-scope
// device array instead of a caller workspace, sized for d <= GPTQ_PREPARE_STATIC_MAX_D.  Every GPU that loads the library keeps it for
// the life of the process.
namespace {
// the 128-block path's need at the largest accepted order (larger than the one-launch kernel's)
constexpr size_t kStaticScratchBytes = 1024 + (size_t)(GPTQ_PREPARE_STATIC_MAX_D / 128) * 128 * 128 * sizeof(float);
static __device__ __align__(256) unsigned char g_prepare_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchAddress {
  unsigned long long ctx_id;  // the context the address belongs to
  void* addr;
};
ScratchAddress g_scratch_address[kMaxDevices] = {};

// Unique id of the calling thread's current CUDA context (through the runtime's driver entry points,
// no link against libcuda); false when no context is current or the driver lacks the calls.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_prepare_scratch in the current device's context.  Host code must not use the
// symbol itself: it is a host-side stand-in.  The address is looked up with that device current and
// cached per device together with the context's id; when the context changes (the device was reset,
// or its primary context released and made again, which reloads the module) it is looked up again.
gptq_status static_scratch(void** out) {
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPTQ_ERR_CUDA;
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchAddress& c = g_scratch_address[dev];
  if (have_id && c.addr != nullptr && c.ctx_id == id) {
    *out = c.addr;
    return GPTQ_OK;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_prepare_scratch) != cudaSuccess || p == nullptr) return GPTQ_ERR_CUDA;
  if (!have_id) have_id = current_context_id(&id);  // the lookup makes the device's context current
  c.ctx_id = have_id ? id : 0;
  c.addr = have_id ? p : nullptr;  // without a context id nothing is cached: the next call looks up again
  *out = p;
  return GPTQ_OK;
}
}  // namespace

gptq_status prepare_launch_static(const float* H, int64_t d, float damp, float* U, int32_t* status,
                                  cudaStream_t stream) {
  static_assert(kStaticScratchBytes >= kSideOffset + (kSmallOrder / NB) * NB * NB * sizeof(float), "scratch too small");
  void* scratch = nullptr;
  gptq_status st = static_scratch(&scratch);
  if (st != GPTQ_OK) return st;
  const size_t need = d > kSmallOrder ? prepare_blocked_workspace(d, false) : prepare_workspace(d);
  if (need > kStaticScratchBytes) return GPTQ_ERR_WORKSPACE;
  // no look-ahead stream here: this variant creates no CUDA objects, so every launch stays on `stream`;
  // its scratch holds no split panel, so the trailing updates take the single-CTA tiles
  return prepare_launch(H, d, damp, U, status, scratch, stream, false, false);
}

}  // namespace gptq
