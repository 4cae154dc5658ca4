// A2 + A3 for large orders: dampening and U = upper Cholesky factor of Hd^-1 with 128-wide blocks
// and host-ordered launches (FDE Interviews breakdown of GPTQ, figure "THE IDEA, VISUALLY" step 2,
// "U = chol(H^-1)"; zhiliyouxian blog, 算法流程 "H = H + lambda * I").
//
// Same route as the one-launch kernel (prepare.cu): factor P = J Hd J = L L^T, invert Y = L^-1, and
// U = J Y J.  Here the work of large orders is dominated by dense block products, so it is spelled
// as a right-looking blocked Cholesky over 128-column panels followed by a recursive-doubling
// triangular inverse, each step a launch:
//   diag_mean, reverse_damp                        lambda, lower(P) = J (H + lambda I) J
//   factor(0)
//   for each panel p:
//     trsm(p)           L(r, p) = P(r, p) L(p,p)^-T for every row block r > p
//     syrk(p)           P(r, c) -= L(r, p) L(c, p)^T for p < c <= r
//     factor(p+1)       one CTA: the diagonal block (p+1, p+1) factored in four 32-wide steps (each a
//                       one-warp factorisation, the rest overlapped by the other warps) and inverted
//                       -> side[p+1] = L(p+1,p+1)^-1
//   leaf_copy           diagonal blocks of P <- side
//   for g = 1, 2, 4, ...: T = C A^-1, Y21 = -B^-1 T for [[A,0],[C,B]] pairs of g blocks
//   rotate              U = J Y J
// factor(p+1) depends only on trsm(p) and the update of block (p+1, p+1), so that tile and the
// factorisation run on a second stream alongside the rest of syrk(p) (look-ahead): the serial chain
// per panel is trsm + max(syrk, diagonal tile + factor) instead of their sum.  The block products
// run on the tensor cores as 3xTF32 (gemm_tf32x3.cu) when rows are 16-byte aligned (d % 4 == 0),
// else on an fp32 FMA tile kernel below (128x128x128 tiles, 8x8 outputs per thread), where the
// factorisation does the diagonal block's last update itself.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int BB = 128;   // block order
constexpr int LDS = BB + 4;
constexpr int kSideOff = 1024;
constexpr int kSub = 32;  // sub-block of the diagonal factorisation

// ------------------------------------------------------------------ lambda and reversed copy
__global__ void diag_mean_kernel(const float* __restrict__ H, int d, float damp, float* __restrict__ lam) {
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s += (double)H[(size_t)i * d + i];
  __shared__ double red[32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    *lam = (float)((double)damp * t / (double)d);
  }
}

__global__ void reverse_damp_kernel(const float* __restrict__ H, int d, const float* __restrict__ lam,
                                    float* __restrict__ P) {
  const float l = *lam;
  for (int i = blockIdx.x; i < d; i += gridDim.x) {
    const float* src = H + (size_t)(d - 1 - i) * d + (d - 1);
    float* dst = P + (size_t)i * d;
    for (int j = threadIdx.x; j <= i; j += blockDim.x) dst[j] = src[-j] + (i == j ? l : 0.0f);
  }
}

// ------------------------------------------------------------------ panel factorisation
// One warp factors a 32x32 block (lower part, stride LDS) and writes its inverse, natural layout,
// into Li (stride LDS): lane i keeps row i of A and column i of the right-hand sides of L Y = I;
// right-looking with an unscaled pivot column, column k reaching every lane by shuffles.
__device__ void warp_factor_invert_128(const float* A, float* Li, int d, int pivot_base, int32_t* status) {
  const int lane = threadIdx.x & 31;
  float a[kSub], rr[kSub], rs[kSub];
#pragma unroll
  for (int c = 0; c < kSub; ++c) {
    a[c] = A[lane * LDS + c];
    rr[c] = (c == lane) ? 1.0f : 0.0f;
  }
  int bad = -1;  // first non-positive pivot (the pivot is the same on every lane)
#pragma unroll
  for (int k = 0; k < kSub; ++k) {
    const float p = __shfl_sync(0xffffffffu, a[k], k);
    const float inv = __fdividef(1.0f, p);
    rs[k] = rsqrtf(p);
    if (bad < 0 && !(p > 0.0f && isfinite(p)) && pivot_base + k < d) bad = k;
    const float li = a[k] * inv;
    const float t = rr[k] * inv;
#pragma unroll
    for (int x = k + 1; x < kSub; ++x) {
      const float v = __shfl_sync(0xffffffffu, a[k], x);  // A[x][k]
      a[x] = fmaf(-li, v, a[x]);
      rr[x] = fmaf(-v, t, rr[x]);
    }
  }
  if (lane == 0 && bad >= 0) report_status(status, GPTQ_ERR_NOT_PD, d - 1 - (pivot_base + bad));
  // lane holds column `lane` of the right-hand sides: Linv[i][lane] = rr[i] / sqrt(pivot_i)
#pragma unroll
  for (int i = 0; i < kSub; ++i) Li[i * LDS + lane] = (i >= lane) ? rr[i] * rs[i] : 0.0f;
  __syncwarp();
}

// out (M x N, stride LDS) = beta * out + alpha * sum_{k<K} A[m][k] * B(k, n), by all 256 threads;
// M, N multiples of 16 (at most 128), K a multiple of 4; out must not overlap A or B.
// B(k, n) = B[n][k] (TB) or B[k][n] (!TB).  The output is cut into 16x16 warp tiles dealt
// round-robin to the 8 warps, so small products still use every warp; lane (mi, ni) = (lane / 4,
// lane % 4) owns rows mi + 8i and columns ni + 4j of its tile.  A (and B when TB) is read as float4
// along k; with the row stride LDS = 132 the rows of one load fall in distinct bank groups.  The
// pass loop stays rolled: these products run once each per launch, so a compact body keeps the
// kernel inside the instruction cache.  Ends with a barrier.  beta is 0 or 1.
template <bool TB>
__device__ void block_mm_w(float* out, const float* A, const float* B, int M, int N, int K, float alpha, float beta,
                           int w0, int nw) {
  const int warp = (threadIdx.x >> 5) - w0, lane = threadIdx.x & 31;
  const int mi = lane >> 2, ni = lane & 3;
  const int wn = N / 16, n_wt = (M / 16) * wn;
#pragma unroll 1
  for (int wt = warp; wt < n_wt; wt += nw) {
    float r[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) r[i][j] = 0.0f;
    const float* a = A + ((wt / wn) * 16 + mi) * LDS;
    const int n0 = (wt % wn) * 16 + ni;
#pragma unroll 2
    for (int k = 0; k < K; k += 4) {
      float4 av[2], bv[4];
#pragma unroll
      for (int i = 0; i < 2; ++i) av[i] = *reinterpret_cast<const float4*>(a + 8 * i * LDS + k);
      if (TB) {
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = *reinterpret_cast<const float4*>(B + (n0 + 4 * j) * LDS + k);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          bv[j] = make_float4(B[k * LDS + n0 + 4 * j], B[(k + 1) * LDS + n0 + 4 * j], B[(k + 2) * LDS + n0 + 4 * j],
                              B[(k + 3) * LDS + n0 + 4 * j]);
      }
#pragma unroll
      for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float acc = r[i][j];
          acc = fmaf(av[i].x, bv[j].x, acc);
          acc = fmaf(av[i].y, bv[j].y, acc);
          acc = fmaf(av[i].z, bv[j].z, acc);
          acc = fmaf(av[i].w, bv[j].w, acc);
          r[i][j] = acc;
        }
    }
    float* o = out + ((wt / wn) * 16 + mi) * LDS + (wt % wn) * 16 + ni;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float* e = o + 8 * i * LDS + 4 * j;
        *e = (beta != 0.0f ? *e : 0.0f) + alpha * r[i][j];
      }
  }
}

template <bool TB>
__device__ void block_mm(float* out, const float* A, const float* B, int M, int N, int K, float alpha, float beta) {
  block_mm_w<TB>(out, A, B, M, N, K, alpha, beta, 0, 8);
  __syncthreads();
}

// barrier of warps 1-7 (the helpers of the diagonal-block factorisation)
__device__ __forceinline__ void helpers_sync() { asm volatile("bar.sync 1, 224;" ::: "memory"); }

// Factors the 128x128 diagonal block p and writes side[p] = L(p,p)^-1 (row-major, zeros above the
// diagonal).  With `update` (p > 0) the block first receives its last update,
// P(p,p) - L(p,p-1) L(p,p-1)^T, here (the trailing update of panel p-1 then leaves this block out, so
// the factorisation can run alongside it); otherwise the block arrives fully updated.
// One CTA of 256 threads, dynamic shared memory.
__device__ void factor_block(const float* P, int d, int p, bool update, float* side, int32_t* status, float* sm) {
  float* A = sm;                  // [128][LDS]
  float* Li = sm + BB * LDS;      // [128][LDS]
  float* S = Li + BB * LDS;       // [128][LDS]: L(p, p-1), then scratch
  const int p0 = p * BB;
  if (!update && d % 4 == 0) {
    // 16-byte rows: one batch of 16 float4 loads per thread; the upper part and rows / columns past
    // the order read as the identity
    float4 va[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = threadIdx.x + q * 256;
      const int i = e / (BB / 4), c = (e % (BB / 4)) * 4;
      const int gi = p0 + i, gc = p0 + c;
      va[q] = (gi < d && gc < d) ? *reinterpret_cast<const float4*>(P + (size_t)gi * d + gc) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = threadIdx.x + q * 256;
      const int i = e / (BB / 4), c = (e % (BB / 4)) * 4;
      const bool in = p0 + i < d;
      float x[4] = {va[q].x, va[q].y, va[q].z, va[q].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const bool col_in = in && p0 + c + u < d;
        A[i * LDS + c + u] = col_in ? ((c + u <= i) ? x[u] : 0.0f) : ((i == c + u) ? 1.0f : 0.0f);
      }
      *reinterpret_cast<float4*>(Li + i * LDS + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  } else
  // batched loads: every thread issues its 16 loads before storing
  for (int base = 0; base < BB * BB; base += 16 * 256) {
    float va[16], vs[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = base + threadIdx.x + q * 256;
      const int i = e / BB, c = e % BB;
      const int gi = p0 + i, gc = p0 + c;
      va[q] = (gi < d && gc < d) ? ((c <= i) ? P[(size_t)gi * d + gc] : 0.0f) : ((i == c) ? 1.0f : 0.0f);
      vs[q] = (update && gi < d && gc - BB < d) ? P[(size_t)gi * d + gc - BB] : 0.0f;
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = base + threadIdx.x + q * 256;
      A[(e / BB) * LDS + e % BB] = va[q];
      S[(e / BB) * LDS + e % BB] = vs[q];
      Li[(e / BB) * LDS + e % BB] = 0.0f;
    }
  }
  __syncthreads();
  if (update) block_mm<true>(A, S, S, BB, BB, BB, -1.0f, 1.0f);  // A -= L(p,p-1) L(p,p-1)^T (S is free after)
  // Four 32-wide steps.  Warp 0 factors diagonal block s (the chain); meanwhile warps 1-7 finish what
  // step s-1 left that block s does not need: the panel solves of rows below s+1, the trailing
  // update, and row band s-1 of the inverse.  Only the next row band's solve and the next diagonal
  // block's update stay on the chain.  L blocks go to S (row band t, column band s), the inverse
  // Y = L^-1 builds up in Li (zeros above the diagonal), and the band products' scratch Z uses the
  // strictly upper part of A's first row band, which nothing else writes.
  auto blk = [](float* M, int t, int c) { return M + t * kSub * LDS + c * kSub; };
  float* Z = A + kSub;  // rows 0..31, columns 32..127 of A
  constexpr int NSUB = BB / kSub;
#pragma unroll 1
  for (int st = 0; st < NSUB; ++st) {
    const int warp = threadIdx.x >> 5;
    if (warp == 0) {
      warp_factor_invert_128(blk(A, st, st), blk(Li, st, st), d, p0 + st * kSub, status);
    } else if (st >= 1) {
      const int q = st - 1;  // the previous step
      const int below = NSUB - 1 - st;  // row bands after st
      if (below > 0)  // L(t, q) for t > st
        block_mm_w<true>(blk(S, st + 1, q), blk(A, st + 1, q), blk(Li, q, q), below * kSub, kSub, kSub, 1.0f, 0.0f, 1, 7);
      helpers_sync();
      if (below > 0)  // A(t, c) -= L(t, q) L(c, q)^T for t > st, c >= st (upper tiles included, unused)
        block_mm_w<true>(blk(A, st + 1, st), blk(S, st + 1, q), blk(S, st, q), below * kSub, (below + 1) * kSub, kSub,
                         -1.0f, 1.0f, 1, 7);
      if (q >= 1) {  // inverse row band q: Y(q, 0..q-1) = -Li(q,q) L(q, 0..q-1) Y(0..q-1, 0..q-1)
        block_mm_w<false>(Z, blk(S, q, 0), Li, kSub, q * kSub, q * kSub, 1.0f, 0.0f, 1, 7);
        helpers_sync();
        block_mm_w<false>(blk(Li, q, 0), blk(Li, q, q), Z, kSub, q * kSub, kSub, -1.0f, 0.0f, 1, 7);
      }
    }
    __syncthreads();
    if (st + 1 < NSUB) {
      // the chain: L(st+1, st), then the last update of diagonal block st+1
      block_mm<true>(blk(S, st + 1, st), blk(A, st + 1, st), blk(Li, st, st), kSub, kSub, kSub, 1.0f, 0.0f);
      block_mm<true>(blk(A, st + 1, st + 1), blk(S, st + 1, st), blk(S, st + 1, st), kSub, kSub, kSub, -1.0f, 1.0f);
    }
  }
  // inverse row band NSUB-1
  block_mm<false>(Z, blk(S, NSUB - 1, 0), Li, kSub, (NSUB - 1) * kSub, (NSUB - 1) * kSub, 1.0f, 0.0f);
  block_mm<false>(blk(Li, NSUB - 1, 0), blk(Li, NSUB - 1, NSUB - 1), Z, kSub, (NSUB - 1) * kSub, kSub, -1.0f, 0.0f);
  float4* out = reinterpret_cast<float4*>(side + (size_t)p * BB * BB);
  for (int e = threadIdx.x; e < BB * BB / 4; e += blockDim.x) {
    const int i = e / (BB / 4), c = (e % (BB / 4)) * 4;
    const float4 l = *reinterpret_cast<const float4*>(Li + i * LDS + c);
    out[e] = make_float4(c <= i ? l.x : 0.f, c + 1 <= i ? l.y : 0.f, c + 2 <= i ? l.z : 0.f, c + 3 <= i ? l.w : 0.f);
  }
}

constexpr int kFactorSmem = 3 * BB * LDS * sizeof(float);

__global__ void __launch_bounds__(256, 1) factor_kernel(const float* __restrict__ P, int d, int p, int update,
                                                     float* __restrict__ side, int32_t* status) {
  extern __shared__ __align__(16) float fsm[];
  factor_block(P, d, p, update != 0, side, status, fsm);
}

// ------------------------------------------------------------------ 128x128x128 tile products
enum TileMode { kTrsm = 0, kSyrk = 1, kTrtriT = 2, kTrtriY = 3 };

struct TileArgs {
  float* P;
  const float* side;
  int d, D;   // order, 128-blocks
  int p;      // panel (trsm, syrk)
  int g;      // half size in blocks (trtri levels)
  int skip;   // syrk: leading output tiles left out (the next diagonal block, factored alongside)
};

__device__ __forceinline__ float ld_or0(const float* base, int64_t r, int64_t c, int d) {
  return (r < d && c < d) ? base[r * d + c] : 0.0f;
}

// Output tile C (128x128 at block (ri, ci)) = sum over K blocks of A(ri, k) B(k, ci):
//   trsm:    A = P(r, p),  B(k, n) = side[p][n][k]            -> P(r, p) = acc
//   syrk:    A = P(r, p),  B(k, n) = P(c, p)[n][k]            -> P(r, c) -= acc
//   trtriT:  A = P(r, k),  B = P(k, c) (k from c to a1-1)     -> P(c, r) = acc^T   (T parked transposed)
//   trtriY:  A = P(r, k),  B(k, n) = P(c, k)[n][k] (k <= r)   -> P(r, c) = -acc
template <int MODE>
__global__ void __launch_bounds__(256) tile_gemm_kernel(const TileArgs a) {
  constexpr int KC = 32;
  __shared__ __align__(16) float As[KC][BB + 4];  // As[k][m]
  __shared__ __align__(16) float Bs[KC][BB + 4];  // Bs[k][n]
  const int d = a.d;
  int ri = 0, ci = 0, kb0 = 0, kb1 = 1;
  const int bid = blockIdx.x + (MODE == kSyrk ? a.skip : 0);
  if (MODE == kTrsm) {
    ri = a.p + 1 + bid;
    ci = a.p;
  } else if (MODE == kSyrk) {
    int rr = (int)((sqrt(8.0 * (double)bid + 1.0) - 1.0) * 0.5);
    while ((rr + 1) * (rr + 2) / 2 <= bid) ++rr;
    while (rr * (rr + 1) / 2 > bid) --rr;
    ri = a.p + 1 + rr;
    ci = a.p + 1 + (bid - rr * (rr + 1) / 2);
  } else {
    const int per_pair = a.g * a.g;
    const int q = bid / per_pair, t = bid % per_pair;
    const int a0 = q * 2 * a.g, b0 = a0 + a.g, b1 = min(a0 + 2 * a.g, a.D);
    ri = b0 + t / a.g;
    ci = a0 + t % a.g;
    if (ri >= b1) return;
    if (MODE == kTrtriT) {
      kb0 = ci;
      kb1 = b0;  // A^-1 (k, c) is zero for k < c
    } else {
      kb0 = b0;
      kb1 = ri + 1;  // B^-1 (r, k) is zero for k > r
    }
  }
  const int64_t r0 = (int64_t)ri * BB, c0 = (int64_t)ci * BB;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  float ra[16], rb[16];
  // slice s of the K range: block kb = kb0 + s / 4, columns (s % 4) * 32 .. +32 of that block
  auto fetch = [&](int s) {
    const int kb = kb0 + s / (BB / KC);
    const int64_t k0 = (int64_t)kb * BB + (s % (BB / KC)) * KC;
#pragma unroll
    for (int q = 0; q < 16; ++q) {  // A: 128 rows (m) x 32 k, read along k
      const int e = tid + 256 * q;
      const int m = e / KC, k = e % KC;
      const int64_t acol = (MODE == kTrsm || MODE == kSyrk) ? (int64_t)a.p * BB + (k0 - (int64_t)kb * BB) + k : k0 + k;
      ra[q] = ld_or0(a.P, r0 + m, acol, d);
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = tid + 256 * q;
      if (MODE == kTrtriT) {  // B natural: rows k, columns n
        const int k = e / BB, n = e % BB;
        rb[q] = ld_or0(a.P, k0 + k, c0 + n, d);
      } else {                // B stored [n][k]
        const int n = e / KC, k = e % KC;
        if (MODE == kTrsm) {
          const int64_t kk = k0 - (int64_t)kb * BB + k;
          rb[q] = a.side[((size_t)a.p * BB + n) * BB + kk];
        } else if (MODE == kSyrk) {
          rb[q] = ld_or0(a.P, c0 + n, (int64_t)a.p * BB + (k0 - (int64_t)kb * BB) + k, d);
        } else {  // trtriY: T(k, c) stored at P(c, k)
          rb[q] = ld_or0(a.P, c0 + n, k0 + k, d);
        }
      }
    }
  };
  auto store = [&]() {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = tid + 256 * q;
      As[e % KC][e / KC] = ra[q];
    }
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int e = tid + 256 * q;
      if (MODE == kTrtriT)
        Bs[e / BB][e % BB] = rb[q];
      else
        Bs[e % KC][e / KC] = rb[q];
    }
  };
  const int n_slices = (kb1 - kb0) * (BB / KC);
  fetch(0);
  for (int s = 0; s < n_slices; ++s) {
    __syncthreads();
    store();
    __syncthreads();
    if (s + 1 < n_slices) fetch(s + 1);
#pragma unroll 4
    for (int k = 0; k < KC; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[k][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t gr = r0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t gc = c0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (gr >= d || gc >= d) continue;
      if (MODE == kTrsm) {
        a.P[gr * d + gc] = acc[i][j];
      } else if (MODE == kSyrk) {
        a.P[gr * d + gc] -= acc[i][j];
      } else if (MODE == kTrtriT) {
        a.P[gc * d + gr] = acc[i][j];
      } else {
        a.P[gr * d + gc] = -acc[i][j];
      }
    }
  }
}

// diagonal 128-blocks of P <- their inverses (zeros above the diagonal)
__global__ void leaf_copy_kernel(float* __restrict__ P, int d, const float* __restrict__ side) {
  const int p = blockIdx.x;
  const float* src = side + (size_t)p * BB * BB;
  for (int e = threadIdx.x; e < BB * BB; e += blockDim.x) {
    const int i = e / BB, c = e % BB;
    const int64_t gi = (int64_t)p * BB + i, gc = (int64_t)p * BB + c;
    if (gi < d && gc < d) P[gi * d + gc] = src[e];
  }
}

// U = J Y J in place: lower block triangle -> upper, strict lower part zeroed, diagonal reversed
__global__ void rotate_kernel(float* __restrict__ P, int d) {
  for (int i = blockIdx.x; i < d; i += gridDim.x) {
    float* row = P + (size_t)i * d;
    float* mirror = P + (size_t)(d - 1 - i) * d + (d - 1);
    for (int j = threadIdx.x; j <= i; j += blockDim.x) {
      if (j < i) {
        mirror[-j] = row[j];
        row[j] = 0.0f;
      } else if (i < d - 1 - i) {
        const float va = row[i], vb = mirror[-i];
        row[i] = vb;
        mirror[-i] = va;
      }
    }
  }
}

}  // namespace

// Two-level trailing update on the pair path: panels are grouped in outer blocks of kOuterPanels.
// After panel p, the update reaches only the columns of p's outer block (K = 128); after an outer
// block's last panel, its L columns (K = 1024) update everything to its right at once.  In exact
// arithmetic every block P(r, c) still receives every earlier panel's term before it is used; the
// trailing matrix is read and written once per outer block instead of once per panel.
constexpr int kOuterPanels = 8;

// header (1 KiB), the inverse diagonal blocks (side), and with_pair: the tf32 hi / lo split of an
// outer block's L columns ([d, 1024] each) for the pair-GEMM trailing updates
size_t prepare_blocked_workspace(int64_t d, bool with_pair) {
  const int64_t D = (d + BB - 1) / BB;
  size_t n = kSideOff + (size_t)D * BB * BB * sizeof(float);
  if (with_pair) n = align_up(n, 256) + 2 * align_up((size_t)d * kOuterPanels * BB * sizeof(float), 256);
  return n;
}

namespace {

// The look-ahead stream and its two events, one set per device, made on first use.
struct LookAhead {
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

std::mutex g_lookahead_mu;
LookAhead g_lookahead[64];

}  // namespace

namespace {
// The 3xTF32 tensor-core path needs 16-byte aligned rows (d % 4 == 0) and bases; other orders run
// the fp32 FMA tile kernel.
struct TcMaps {
  CUtensorMap p128, p32, p32mn, side128;
};

bool tc_maps(TcMaps& m, const float* P, const float* side, int d, int D) {
  return tf32x3_map(&m.p128, P, d, d, d, 128) && tf32x3_map(&m.p32, P, d, d, d, 32) &&
         tf32x3_map(&m.p32mn, P, d, d, d, 32, true) && tf32x3_map(&m.side128, side, (int64_t)D * BB, BB, BB, 128);
}
}  // namespace

gptq_status prepare_blocked_launch(const float* H, int64_t d64, float damp, float* U, int32_t* status, void* workspace,
                                   cudaStream_t s, bool lookahead, bool pair) {
  const int d = (int)d64;
  const int D = (d + BB - 1) / BB;
  char* ws = static_cast<char*>(workspace);
  float* lam = reinterpret_cast<float*>(ws);
  float* side = reinterpret_cast<float*>(ws + kSideOff);
  int dev = 0, sms = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(factor_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kFactorSmem));
  TcMaps maps;
  const bool tc = prepare_uses_tensor_cores(d);
  // U is 16-byte aligned (checked by the entry points), the scratch 256-byte aligned and d % 4 == 0 on
  // this path, so the maps encode unless the driver call itself fails
  if (tc && !tc_maps(maps, U, side, d, D)) return GPTQ_ERR_CUDA;
  // the trailing updates on CTA pairs from the split L panel (workspace entry point, tensor-core path)
  const bool use_pair = tc && pair;
  constexpr int KO = kOuterPanels * BB;  // row stride of the split L columns
  float* Lh = nullptr;
  float* Ll = nullptr;
  CUtensorMap mLh, mLl, mP;
  if (use_pair) {
    const size_t off = align_up(kSideOff + (size_t)D * BB * BB * sizeof(float), 256);
    Lh = reinterpret_cast<float*>(ws + off);
    Ll = reinterpret_cast<float*>(ws + off + align_up((size_t)d * KO * sizeof(float), 256));
    if (!split_map(&mLh, Lh, d, KO, KO) || !split_map(&mLl, Ll, d, KO, KO) || !tf32x3_map(&mP, U, d, d, d, 32))
      return GPTQ_ERR_CUDA;
  }
  std::unique_lock<std::mutex> hold(g_lookahead_mu, std::defer_lock);
  LookAhead* la = nullptr;
  if (lookahead && dev < 64) {
    hold.lock();  // the events are shared: one enqueue sequence at a time
    la = &g_lookahead[dev];
    if (la->side == nullptr) {
      GPTQ_CUDA_TRY(cudaStreamCreateWithFlags(&la->side, cudaStreamNonBlocking));
      GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&la->fork, cudaEventDisableTiming));
      GPTQ_CUDA_TRY(cudaEventCreateWithFlags(&la->join, cudaEventDisableTiming));
    }
  }
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), s));
  diag_mean_kernel<<<1, 1024, 0, s>>>(H, d, damp, lam);
  GPTQ_LAUNCH_CHECK();
  reverse_damp_kernel<<<sms * 4, 256, 0, s>>>(H, d, lam, U);
  GPTQ_LAUNCH_CHECK();
  factor_kernel<<<1, 256, kFactorSmem, s>>>(U, d, 0, 0, side, status);
  GPTQ_LAUNCH_CHECK();
  TileArgs ta{U, side, d, D, 0, 0, 1};
  Tf32x3Args g{};
  g.D = D;
  g.o_w = d;
  g.o_h = d;
  g.status = status;
  gptq_status st = GPTQ_OK;
  for (int p = 0; p + 1 < D; ++p) {
    const int below = D - p - 1;
    const int tri = below * (below + 1) / 2;
    // trsm(p)
    if (tc) {
      g.kind = kGemmTrsm, g.epi = kEpiStore, g.b_mn = 0, g.tiles = below, g.p = p, g.skip = 0;
      if ((st = tf32x3_gemm_launch(maps.p128, maps.side128, maps.p32, g, s)) != GPTQ_OK) return st;
    } else {
      ta.p = p;
      tile_gemm_kernel<kTrsm><<<below, 256, 0, s>>>(ta);
      GPTQ_LAUNCH_CHECK();
    }
    // factor(p+1) and the trailing update of panel p.  On the tensor-core path the next diagonal
    // block gets its update as a one-tile product first, and the trailing update leaves one SM free
    // for that chain; on the fp32 path the factorisation does the diagonal update itself.
    cudaStream_t fs = (la != nullptr) ? la->side : s;
    if (la != nullptr) {
      GPTQ_CUDA_TRY(cudaEventRecord(la->fork, s));
      GPTQ_CUDA_TRY(cudaStreamWaitEvent(la->side, la->fork, 0));
    }
    if (tc && use_pair) {
      // L(r, p) of the trailing rows, split into tf32 hi / lo into the outer block's slot p % 8 (rows
      // keep their absolute index); then the pair-GEMM updates of the two levels
      const int o0 = p / kOuterPanels * kOuterPanels, pend = std::min(o0 + kOuterPanels, D);
      const int j = p - o0;
      const int64_t rows = d - (int64_t)(p + 1) * BB;
      const size_t roff = (size_t)(p + 1) * BB * KO + (size_t)j * BB;
      if ((st = split_rows_launch(U + (size_t)(p + 1) * BB * d + (size_t)p * BB, d, rows, Lh + roff, Ll + roff, KO,
                                  s)) != GPTQ_OK)
        return st;
      const bool boundary = p + 1 == pend;  // p closes its outer block
      PairGemmArgs pg{};
      pg.kind = kPairSyrk;
      pg.o_w = d;
      pg.o_h = d;
      pg.out_y0 = pg.out_x0 = pg.row0 = (p + 1) * BB;
      pg.status = status;
      if (!boundary) {
        // inner: rows below p, the columns of p's outer block after p; K = 128 (panel p)
        CUtensorMap mSh, mSl;
        if (!split_map(&mSh, Lh + (size_t)j * BB, d, BB, KO) || !split_map(&mSl, Ll + (size_t)j * BB, d, BB, KO))
          return GPTQ_ERR_CUDA;
        pg.cols_blk = pend - p - 1;
        pg.super_r = (below + 1) / 2;
        pg.super_c = (pg.cols_blk + 1) / 2;
        pg.tiles = pg.super_c * pg.super_r - pg.super_c * (pg.super_c - 1) / 2;
        pg.nk = BB / 32;
        if (la != nullptr) {
          g.kind = kGemmSyrk, g.epi = kEpiSub, g.b_mn = 0, g.tiles = 1, g.p = p, g.skip = 0;
          if ((st = tf32x3_gemm_launch(maps.p128, maps.p128, maps.p32, g, fs)) != GPTQ_OK) return st;
          factor_kernel<<<1, 256, kFactorSmem, fs>>>(U, d, p + 1, 0, side, status);
          GPTQ_LAUNCH_CHECK();
          GPTQ_CUDA_TRY(cudaEventRecord(la->join, fs));
          pg.skip_diag = 1;
          if ((st = tf32x3_pair_launch(mSh, mSl, mSh, mSl, mP, pg, s, 1)) != GPTQ_OK) return st;
          GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, la->join, 0));
        } else {
          pg.skip_diag = 0;
          if ((st = tf32x3_pair_launch(mSh, mSl, mSh, mSl, mP, pg, s)) != GPTQ_OK) return st;
          factor_kernel<<<1, 256, kFactorSmem, s>>>(U, d, p + 1, 0, side, status);
          GPTQ_LAUNCH_CHECK();
        }
      } else {
        // outer: everything right of the outer block, K = the outer block's columns; the next diagonal
        // block needs all of them, so it is factored after this update (no look-ahead here)
        const int kcols = (pend - o0) * BB;
        CUtensorMap mOh, mOl;
        if (!split_map(&mOh, Lh, d, kcols, KO) || !split_map(&mOl, Ll, d, kcols, KO)) return GPTQ_ERR_CUDA;
        pg.cols_blk = below;
        pg.super_r = pg.super_c = (below + 1) / 2;
        pg.tiles = pg.super_r * (pg.super_r + 1) / 2;
        pg.nk = kcols / 32;
        pg.skip_diag = 0;
        if ((st = tf32x3_pair_launch(mOh, mOl, mOh, mOl, mP, pg, s)) != GPTQ_OK) return st;
        factor_kernel<<<1, 256, kFactorSmem, s>>>(U, d, p + 1, 0, side, status);
        GPTQ_LAUNCH_CHECK();
      }
    } else if (tc) {
      if (la != nullptr) {
        g.kind = kGemmSyrk, g.epi = kEpiSub, g.b_mn = 0, g.tiles = 1, g.p = p, g.skip = 0;
        if ((st = tf32x3_gemm_launch(maps.p128, maps.p128, maps.p32, g, fs)) != GPTQ_OK) return st;
        factor_kernel<<<1, 256, kFactorSmem, fs>>>(U, d, p + 1, 0, side, status);
        GPTQ_LAUNCH_CHECK();
        GPTQ_CUDA_TRY(cudaEventRecord(la->join, fs));
        g.kind = kGemmSyrk, g.epi = kEpiSub, g.b_mn = 0, g.tiles = tri - 1, g.p = p, g.skip = 1;
        if ((st = tf32x3_gemm_launch(maps.p128, maps.p128, maps.p32, g, s, 1)) != GPTQ_OK) return st;
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, la->join, 0));
      } else {
        g.kind = kGemmSyrk, g.epi = kEpiSub, g.b_mn = 0, g.tiles = tri, g.p = p, g.skip = 0;
        if ((st = tf32x3_gemm_launch(maps.p128, maps.p128, maps.p32, g, s)) != GPTQ_OK) return st;
        factor_kernel<<<1, 256, kFactorSmem, s>>>(U, d, p + 1, 0, side, status);
        GPTQ_LAUNCH_CHECK();
      }
    } else {
      if (la != nullptr) {
        factor_kernel<<<1, 256, kFactorSmem, fs>>>(U, d, p + 1, 1, side, status);
        GPTQ_LAUNCH_CHECK();
        GPTQ_CUDA_TRY(cudaEventRecord(la->join, fs));
      }
      if (tri > 1) {
        ta.p = p;
        tile_gemm_kernel<kSyrk><<<tri - 1, 256, 0, s>>>(ta);
        GPTQ_LAUNCH_CHECK();
      }
      if (la != nullptr) {
        GPTQ_CUDA_TRY(cudaStreamWaitEvent(s, la->join, 0));
      } else {
        factor_kernel<<<1, 256, kFactorSmem, s>>>(U, d, p + 1, 1, side, status);
        GPTQ_LAUNCH_CHECK();
      }
    }
  }
  leaf_copy_kernel<<<D, 256, 0, s>>>(U, d, side);
  GPTQ_LAUNCH_CHECK();
  for (int gl = 1; gl < D; gl *= 2) {
    const int pairs = (D + 2 * gl - 1) / (2 * gl);
    if (tc) {
      g.g = gl, g.tiles = pairs * gl * gl, g.skip = 0, g.p = 0;
      g.kind = kGemmTrtriT, g.epi = kEpiStoreT, g.b_mn = 1;
      if ((st = tf32x3_gemm_launch(maps.p128, maps.p32mn, maps.p32, g, s)) != GPTQ_OK) return st;
      g.kind = kGemmTrtriY, g.epi = kEpiStoreNeg, g.b_mn = 0;
      if ((st = tf32x3_gemm_launch(maps.p128, maps.p128, maps.p32, g, s)) != GPTQ_OK) return st;
    } else {
      ta.g = gl;
      tile_gemm_kernel<kTrtriT><<<pairs * gl * gl, 256, 0, s>>>(ta);
      GPTQ_LAUNCH_CHECK();
      tile_gemm_kernel<kTrtriY><<<pairs * gl * gl, 256, 0, s>>>(ta);
      GPTQ_LAUNCH_CHECK();
    }
  }
  rotate_kernel<<<sms * 4, 256, 0, s>>>(U, d);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
