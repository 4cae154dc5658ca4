// A4 - A7: grid, column loop with error compensation, lazy block updates, packing.
//
// GPTQ's column loop (FDE Interviews breakdown of GPTQ, figure "THE IDEA, VISUALLY"):
//   1. round column i to the b-bit grid;  2. err = (w_i - q_i) / U_ii;
//   3. W[:, i+1:] -= err * U[i, i+1:];   4. apply in blocks of 128 columns.
// Rows are independent once U is known (section 01: one column order shared by every row), so rows
// are spread over lanes and the block's corner of U sits in shared memory; the block never leaves
// the SM.  Two forms:
//   - quantize_rows_kernel (layers whose U stays in L2, few rows): one warp per row, lane l holding
//     NS consecutive columns of the block; after each block the CTA applies step 4 to its own rows,
//     streaming U through shared memory.  One launch per layer.
//   - colloop_kernel + a per-block lazy update (other layers): 4 or 8 lanes per row, so one warp
//     instruction advances several rows; step 4 for all rows is a tensor-core 3xTF32 product
//     W[:, i2:] -= Err[:, i1:i2] U[i1:i2, i2:] (gemm_tf32x3.cu), or lazy_gemm_kernel on the fp32 FMA
//     units with GPTQ_FLAG_FP32_FMA.
#include "common.cuh"
#include "kernels.h"

namespace gptq {
namespace {

constexpr int kRowsPerCta = 8;  // one warp per row

// w_work = float(W); per-row grid from the original row when group_size == 0.
template <typename T>
__global__ void __launch_bounds__(256) convert_rowgrid_kernel(const T* __restrict__ W, int64_t m, int d,
                                                              int bits, int group_size,
                                                              float* __restrict__ w_work,
                                                              float* __restrict__ scales,
                                                              int32_t* __restrict__ zeros) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kRowsPerCta + warp;
  if (row >= m) return;
  const T* src = W + row * d;
  float* dst = w_work + row * d;
  float mn = INFINITY, mx = -INFINITY;
  for (int c = lane; c < d; c += 32) {
    const float v = to_f32(src[c]);
    dst[c] = v;
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  if (group_size == 0) {
    mn = warp_min(mn);
    mx = warp_max(mx);
    if (lane == 0) {
      float s, z, rs;
      grid_from_range(mn, mx, (float)((1 << bits) - 1), s, z, rs);
      scales[row] = s;
      zeros[row] = (int32_t)z;
    }
  }
}

// Column loop of one row over block [i1, i1 + 32*NS), run by one warp.  Lane L holds the NS
// consecutive columns i1 + NS*L .. i1 + NS*L + NS-1 in v[0..NS-1] (current values).  Us is the
// block's corner of U (strict upper part, row-major B x B) and invd the reciprocals of its diagonal.
//
// Step i (owner lane L = i / NS, slot s = i % NS): every lane rounds its own v[s] (only the owner's
// result is kept), the owner's error is broadcast, and every lane applies err * U[i, j] to its
// columns after i.  The owner updates its next column from its own error before the broadcast lands,
// so the dependency chain leaves the lane only once every NS steps; the U row of the next step is
// read one step ahead.
template <int NS>
__device__ __forceinline__ void column_loop(float (&v)[NS], const float* __restrict__ Us,
                                            const float* __restrict__ invd, int i1, int group_size,
                                            int n_groups, float maxq, float& scale, float& zero,
                                            float& rscale, const float* wrow, int64_t row,
                                            float* __restrict__ scales, int32_t* __restrict__ zeros,
                                            uint32_t (&code_reg)[NS], float (&err_reg)[NS]) {
  constexpr int B = 32 * NS;
  const int lane = threadIdx.x & 31;
  // this lane's NS entries of the current U row, the next row loaded one step ahead
  // one vector load per lane (NS consecutive floats, 4 * NS-byte aligned)
  auto load_row = [&](float (&dst)[NS], const float* src) {
    if constexpr (NS == 4) {
      const float4 x = *reinterpret_cast<const float4*>(src);
      dst[0] = x.x, dst[1] = x.y, dst[2] = x.z, dst[3] = x.w;
    } else if constexpr (NS == 2) {
      const float2 x = *reinterpret_cast<const float2*>(src);
      dst[0] = x.x, dst[1] = x.y;
    } else {
      dst[0] = src[0];
    }
  };
  float un[NS];
  load_row(un, Us + lane * NS);
  float inv_next = invd[0];
#pragma unroll 1
  for (int L = 0; L < 32; ++L) {
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int i = L * NS + s;
      float u[NS];
#pragma unroll
      for (int t = 0; t < NS; ++t) u[t] = un[t];
      const float inv_i = inv_next;
      if (i + 1 < B) {
        load_row(un, Us + (i + 1) * B + lane * NS);
        inv_next = invd[i + 1];
      }
      if (group_size != 0 && s == 0 && ((i1 + i) % group_size) == 0) {
        // grid of the group starting here, from the current values of its columns
        const int c_end = i + group_size;  // block-local end (may pass the block)
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int t = 0; t < NS; ++t) {
          const int c = lane * NS + t;
          if (c >= i && c < c_end) {
            mn = fminf(mn, v[t]);
            mx = fmaxf(mx, v[t]);
          }
        }
        for (int c = i1 + B + lane; c < i1 + c_end; c += 32) {  // group wider than the block
          const float x = wrow[c];
          mn = fminf(mn, x);
          mx = fmaxf(mx, x);
        }
        mn = warp_min(mn);
        mx = warp_max(mx);
        grid_from_range(mn, mx, maxq, scale, zero, rscale);
        if (lane == 0) {
          const int g = (i1 + i) / group_size;
          scales[row * n_groups + g] = scale;
          zeros[row * n_groups + g] = (int32_t)zero;
        }
      }
      const bool owner = (lane == L);
      const float wi = owner ? v[s] : 0.0f;  // only the owner's value matters
      // code - zero, clamped to the grid; the quotient as an IEEE fp32 product with 1/scale
      const float qz = fminf(fmaxf(round_even(__fmul_rn(wi, rscale)), -zero), maxq - zero);
      const float delta = fmaf(-scale, qz, wi);  // w_i - dequantized value
      const float err = delta * inv_i;
      // selects rather than branches: every lane runs the same instructions
      code_reg[s] = owner ? (uint32_t)(qz + zero) : code_reg[s];
      err_reg[s] = owner ? err : err_reg[s];
      // Us rows are pre-divided by U_ii: err * U[i][j] = delta * Us[i][j]
      if (s + 1 < NS) v[s + 1] = owner ? fmaf(-delta, u[s + 1], v[s + 1]) : v[s + 1];  // owner's next column first
      const float e = __shfl_sync(0xffffffffu, delta, L);
      // columns after i: every column of a lane past the owner, the owner's columns after s + 1
      const float f_near = (lane > L) ? e : 0.0f;
      const float f_far = (lane >= L) ? e : 0.0f;
#pragma unroll
      for (int t = 0; t < NS; ++t) v[t] = fmaf(t <= s + 1 ? -f_near : -f_far, u[t], v[t]);
    }
  }
}

// Grid state of a row at the start of block i1.
__device__ __forceinline__ void grid_at_block(int64_t row, int i1, int group_size, int n_groups,
                                              const float* scales, const int32_t* zeros, float& scale,
                                              float& zero) {
  if (group_size == 0) {
    scale = scales[row];
    zero = (float)zeros[row];
  } else if (i1 % group_size != 0) {  // block inside a group that started in an earlier block
    scale = scales[row * n_groups + i1 / group_size];
    zero = (float)zeros[row * n_groups + i1 / group_size];
  } else {
    scale = 1.0f;
    zero = 0.0f;
  }
}

// Loads the block's corner of U, strict upper part, each row divided by its diagonal entry
// (Us[r][c] = U[i1+r][i1+c] / U[i1+r][i1+r]), and the reciprocals of the diagonal.  All of a thread's
// float4 loads are issued before the first store (one L2 round trip per call).
template <int B>
__device__ __forceinline__ void load_u_block(float* Us, float* invd, const float* __restrict__ U, int d, int i1) {
  constexpr int PER = B * B / 4 / 256;  // float4 per thread (blockDim.x == 256)
  float4 v[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + 256 * k;
    const int r = e / (B / 4), c = (e % (B / 4)) * 4;
    v[k] = *reinterpret_cast<const float4*>(U + (size_t)(i1 + r) * d + i1 + c);
  }
  if (threadIdx.x < B) invd[threadIdx.x] = 1.0f / U[(size_t)(i1 + threadIdx.x) * d + i1 + threadIdx.x];
  __syncthreads();
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + 256 * k;
    const int r = e / (B / 4), c = (e % (B / 4)) * 4;
    const float ir = invd[r];
    float4 u = v[k];
    u.x = (c + 0 > r) ? u.x * ir : 0.0f;
    u.y = (c + 1 > r) ? u.y * ir : 0.0f;
    u.z = (c + 2 > r) ? u.z * ir : 0.0f;
    u.w = (c + 3 > r) ? u.w * ir : 0.0f;
    *reinterpret_cast<float4*>(Us + r * B + c) = u;
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}

// Column loop over block [i1, i1 + B) on the per-block launch path, CTAs of 4 warps.  LPR lanes
// share a row (32 / LPR rows per warp): lane `sub` of the row's group holds the C = B/LPR
// consecutive columns i1 + sub*C .. i1 + sub*C + C-1 in registers.  At block column i the owner lane
// (sub = i / C) rounds its column, updates its own next column straight away (its chain stays in its
// registers for C steps), and the error reaches the group with one shuffle; each lane then applies
// it to its columns after i.  The rounding runs once per warp instruction for 32 / LPR rows, so a
// row-step costs a few warp instructions instead of a whole warp's; LPR = 8 gives layers with fewer
// rows twice the warps (the step latency needs several warps per scheduler to hide).  The raw U
// block (B x B) sits in shared memory with each row's C-column chunks padded apart so the group's
// float4 reads of a row fall in distinct bank groups; err * U[i, j] with err = delta / U_ii is the
// page's update.  The block's errors leave as fp32 (err_out), or, for the updates on CTA pairs,
// already split into tf32 hi = tf32(err) rounded to nearest and lo = tf32(err - hi) (e_hi / e_lo
// non-null; the same layout, row stride err_ld), which saves a split launch per block.
__device__ __forceinline__ float tf32_rna(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

template <int C, int LPR>
__global__ void __launch_bounds__(128, 3) colloop_kernel(float* __restrict__ w, int64_t m, int d, int i1,
                                                      const float* __restrict__ U, int bits,
                                                      int group_size, uint8_t* __restrict__ codes,
                                                      float* __restrict__ scales,
                                                      int32_t* __restrict__ zeros,
                                                      float* __restrict__ err_out, int err_ld,
                                                      float* __restrict__ e_hi, float* __restrict__ e_lo) {
  constexpr int B = LPR * C;
  constexpr int CS = ((C + 4) / 4) % 2 == 1 ? C + 4 : C + 8;  // chunk stride: an odd number of 16-byte granules
  constexpr int RS = LPR * CS;                                  // row stride
  extern __shared__ __align__(16) float sm[];
  float* Ub = sm;             // U[i1 + r][i1 + q*C + t] at Ub[r*RS + q*CS + t]
  float* invd = sm + B * RS;  // 1 / U_ii
  for (int e = threadIdx.x; e < B * B / 4; e += blockDim.x) {
    const int r = e / (B / 4), c = (e % (B / 4)) * 4;
    cp_async16(Ub + r * RS + (c / C) * CS + c % C, U + (size_t)(i1 + r) * d + i1 + c);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (threadIdx.x < B) invd[threadIdx.x] = 1.0f / U[(size_t)(i1 + threadIdx.x) * d + i1 + threadIdx.x];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane & (LPR - 1);
  const int qbase = lane & ~(LPR - 1);
  const int64_t row = ((int64_t)blockIdx.x * (blockDim.x / 32) + warp) * (32 / LPR) + lane / LPR;
  const bool valid = row < m;  // lanes past the last row keep shuffling with zeros
  const int n_groups = group_size ? d / group_size : 1;
  float* wrow = w + (valid ? row : 0) * d;
  float v[C];
#pragma unroll
  for (int q = 0; q < C / 4; ++q) {
    const float4 x = valid ? *reinterpret_cast<const float4*>(wrow + i1 + sub * C + 4 * q) : make_float4(0.f, 0.f, 0.f, 0.f);
    v[4 * q] = x.x;
    v[4 * q + 1] = x.y;
    v[4 * q + 2] = x.z;
    v[4 * q + 3] = x.w;
  }
  const float maxq = (float)((1 << bits) - 1);
  float scale = 1.0f, zero = 0.0f;
  if (valid) grid_at_block(row, i1, group_size, n_groups, scales, zeros, scale, zero);
  float rscale = __frcp_rn(scale);
  uint32_t cw[C / 4];
  float er[C];
#pragma unroll
  for (int q = 0; q < C / 4; ++q) cw[q] = 0u;
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // U row of the current step in registers, the next step's row loaded one step ahead (issue is in
  // program order: loads made just before their FMAs would put the shared-memory latency on every step)
  float4 un[C / 4];
#pragma unroll
  for (int q = 0; q < C / 4; ++q) un[q] = reinterpret_cast<const float4*>(Ub + sub * CS)[q];
  float inv_next = invd[0];
#pragma unroll 1
  for (int o = 0; o < LPR; ++o) {
    const bool owner = (sub == o);
#pragma unroll
    for (int s = 0; s < C; ++s) {
      const int i = o * C + s;  // block column
      float4 u[C / 4];
#pragma unroll
      for (int q = 0; q < C / 4; ++q) u[q] = un[q];
      const float inv_i = inv_next;
      if (i + 1 < B) {
        const float* unext = Ub + (i + 1) * RS + sub * CS;
#pragma unroll
        for (int q = 0; q < C / 4; ++q) un[q] = reinterpret_cast<const float4*>(unext)[q];
        inv_next = invd[i + 1];
      }
      if (s == 0 && group_size != 0 && ((i1 + i) % group_size) == 0) {
        // grid of the group starting here, from the current values of its columns
        const int gend = i + group_size;  // block-local end (may pass the block)
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int t = 0; t < C; ++t) {
          const int c = sub * C + t;
          if (c >= i && c < gend) {
            mn = fminf(mn, v[t]);
            mx = fmaxf(mx, v[t]);
          }
        }
        if (valid)
          for (int c = i1 + B + sub; c < i1 + gend; c += LPR) {  // group wider than the rest of the block
            const float x = wrow[c];
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
          }
#pragma unroll
        for (int x = 1; x < LPR; x <<= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, x));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
        }
        grid_from_range(mn, mx, maxq, scale, zero, rscale);
        if (sub == 0 && valid) {
          const int g = (i1 + i) / group_size;
          scales[row * n_groups + g] = scale;
          zeros[row * n_groups + g] = (int32_t)zero;
        }
      }
      const float wi = v[s];  // the owner's column (other lanes compute and discard)
      // code - zero, clamped to the grid; the quotient as an IEEE fp32 product with 1/scale
      const float qz = fminf(fmaxf(round_even(__fmul_rn(wi, rscale)), -zero), maxq - zero);
      const float delta = fmaf(-scale, qz, wi);  // w_i - dequantized value
      const float err = delta * inv_i;
      // the owner keeps its code and error and updates its own next column straight away
      // (selects rather than a branch: every lane runs the same instructions)
      const float* ur = reinterpret_cast<const float*>(u);
      cw[s >> 2] |= owner ? ((uint32_t)(qz + zero) << (8 * (s & 3))) : 0u;
      er[s] = owner ? err : er[s];
      if (s + 1 < C) v[s + 1] = owner ? fmaf(-err, ur[s + 1], v[s + 1]) : v[s + 1];
      const float e = __shfl_sync(0xffffffffu, err, qbase | o);
      // columns after i: every column of a lane past the owner, the owner's columns after s + 1
      const float f_near = (sub > o) ? e : 0.0f;
      const float f_far = (sub >= o) ? e : 0.0f;
#pragma unroll
      for (int t = 0; t < C; ++t) v[t] = fmaf(t <= s + 1 ? -f_near : -f_far, ur[t], v[t]);
    }
  }
  if (!valid) return;
  uint8_t* crow = codes + row * d + i1 + sub * C;
#pragma unroll
  for (int q = 0; q < C / 4; ++q) reinterpret_cast<uint32_t*>(crow)[q] = cw[q];
  const int64_t eo = row * err_ld + sub * C;
  if (e_hi != nullptr) {
#pragma unroll
    for (int q = 0; q < C / 4; ++q) {
      float h[4], l[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) h[t] = tf32_rna(er[4 * q + t]), l[t] = tf32_rna(er[4 * q + t] - h[t]);
      *reinterpret_cast<float4*>(e_hi + eo + 4 * q) = make_float4(h[0], h[1], h[2], h[3]);
      *reinterpret_cast<float4*>(e_lo + eo + 4 * q) = make_float4(l[0], l[1], l[2], l[3]);
    }
  } else {
#pragma unroll
    for (int q = 0; q < C / 4; ++q)
      *reinterpret_cast<float4*>(err_out + eo + 4 * q) = make_float4(er[4 * q], er[4 * q + 1], er[4 * q + 2], er[4 * q + 3]);
  }
}

// Whole quantization of 8 rows per CTA in one launch (layers whose U stays in L2): for every block,
// the column loop (one warp per row, U corner in shared memory), then the lazy update of the CTA's
// rows, W[rows, i2:] -= Err[rows, :] U[i1:i2, i2:], with U streamed through two shared-memory
// buffers of 128 columns by cp.async (the next chunk lands while the current one is used).  Rows are
// independent given U, so CTAs never wait on one another.
template <typename T, int NS>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const T* __restrict__ W, int64_t m, int d,
                                                            const float* __restrict__ U, int bits,
                                                            int group_size, float* __restrict__ w,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales,
                                                            int32_t* __restrict__ zeros) {
  constexpr int B = 32 * NS;
  constexpr int CW = 128;  // lazy-update chunk width (columns)
  extern __shared__ __align__(16) float sm[];
  float* Us = sm;                // [B][B] corner of U, then [B][CW] chunks of the U panel (buffer 0)
  float* invd = sm + B * CW;     // [B]
  float* errs = invd + B;        // [8][B]
  float* Us2 = errs + kRowsPerCta * B;  // [B][CW] chunk buffer 1
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kRowsPerCta + warp;
  const bool valid = row < m;
  const float maxq = (float)((1 << bits) - 1);
  const int n_groups = group_size ? d / group_size : 1;
  float* wr = w + (valid ? row : 0) * d;
  if (valid) {
    const T* src = W + row * d;
    float mn = INFINITY, mx = -INFINITY;
    for (int c = lane; c < d; c += 32) {
      const float x = to_f32(src[c]);
      wr[c] = x;
      mn = fminf(mn, x);
      mx = fmaxf(mx, x);
    }
    if (group_size == 0) {
      mn = warp_min(mn);
      mx = warp_max(mx);
      if (lane == 0) {
        float s, z, rs;
        grid_from_range(mn, mx, maxq, s, z, rs);
        scales[row] = s;
        zeros[row] = (int32_t)z;
      }
    }
  }
  float scale = 1.0f, zero = 0.0f, rscale = 1.0f;
  for (int i1 = 0; i1 < d; i1 += B) {
    __syncthreads();
    load_u_block<B>(Us, invd, U, d, i1);
    __syncthreads();
    if (valid) {
      __syncwarp();
      if (i1 == 0 || group_size == 0) {
        grid_at_block(row, i1, group_size, n_groups, scales, zeros, scale, zero);
        rscale = __frcp_rn(scale);
      }
      float v[NS];
#pragma unroll
      for (int s = 0; s < NS; ++s) v[s] = wr[i1 + lane * NS + s];
      uint32_t code_reg[NS];
      float err_reg[NS];
      column_loop<NS>(v, Us, invd, i1, group_size, n_groups, maxq, scale, zero, rscale, wr, row, scales,
                      zeros, code_reg, err_reg);
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        codes[row * d + i1 + lane * NS + s] = (uint8_t)code_reg[s];
        errs[warp * B + lane * NS + s] = err_reg[s];
      }
    }
    // lazy update of this CTA's rows over the columns after the block, chunk by chunk; columns past
    // d are not copied (no lane reads them)
    const int n_chunks = (d - (i1 + B) + CW - 1) / CW;
    auto issue_chunk = [&](int c, float* dst) {
      const int c0 = i1 + B + c * CW;
      for (int e = threadIdx.x; e < B * CW / 4; e += blockDim.x) {
        const int r = e / (CW / 4), cc = (e % (CW / 4)) * 4;
        if (c0 + cc < d) cp_async16(dst + r * CW + cc, U + (size_t)(i1 + r) * d + c0 + cc);
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    __syncthreads();  // the column loop is done with the U corner in buffer 0
    if (n_chunks > 0) issue_chunk(0, Us);
    for (int c = 0; c < n_chunks; ++c) {
      float* cur = (c & 1) ? Us2 : Us;
      if (c + 1 < n_chunks) {
        issue_chunk(c + 1, (c & 1) ? Us : Us2);
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        asm volatile("cp.async.wait_group 0;" ::: "memory");
      }
      __syncthreads();  // chunk c has landed for every thread
      const int c0 = i1 + B + c * CW;
      if (valid && c0 + 4 * lane < d) {
        float4 o = *reinterpret_cast<const float4*>(wr + c0 + 4 * lane);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const float* er = errs + warp * B;
#pragma unroll 8
        for (int k = 0; k < B; ++k) {
          const float e = er[k];
          const float4 u = *reinterpret_cast<const float4*>(cur + k * CW + 4 * lane);
          acc.x = fmaf(e, u.x, acc.x);
          acc.y = fmaf(e, u.y, acc.y);
          acc.z = fmaf(e, u.z, acc.z);
          acc.w = fmaf(e, u.w, acc.w);
        }
        o.x -= acc.x;
        o.y -= acc.y;
        o.z -= acc.z;
        o.w -= acc.w;
        *reinterpret_cast<float4*>(wr + c0 + 4 * lane) = o;
      }
      __syncthreads();  // every thread is done with `cur` before chunk c + 2 is copied into it
    }
  }
}

// w[:, i2:] -= Err[:, 0:B] * U[i1:i1+B, i2:] (lazy update of all rows for one block).
// 128x128 output tile per CTA, 256 threads with 8x8 outputs each (rows ty*4+{0..3} and 64+ty*4+{0..3},
// likewise columns), K = B staged 32 at a time through shared memory; the next K slice is loaded
// into registers while the current one is used.
template <int B>
__global__ void __launch_bounds__(256) lazy_gemm_kernel(float* __restrict__ w, int64_t m, int d, int i1,
                                                        const float* __restrict__ U,
                                                        const float* __restrict__ err) {
  constexpr int KC = 32, TM = 128, TN = 128, LDA = TM + 4, LDB = TN + 4;
  __shared__ __align__(16) float As[KC][LDA];  // As[k][row] = err[row][k0 + k]
  __shared__ __align__(16) float Bs[KC][LDB];  // Bs[k][col] = U[i1 + k0 + k][c0 + col]
  const int i2 = i1 + B;
  const int64_t r0 = (int64_t)blockIdx.x * TM;
  const int c0 = i2 + blockIdx.y * TN;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  float4 ra[4], rb[4];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // A slice: 128 rows x 32 k, float4 along k
      const int e = tid + 256 * q;
      const int r = e / (KC / 4), k = (e % (KC / 4)) * 4;
      const int64_t gr = r0 + r;
      ra[q] = (gr < m) ? *reinterpret_cast<const float4*>(err + gr * B + k0 + k) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // B slice: 32 k x 128 columns, float4 along columns
      const int e = tid + 256 * q;
      const int k = e / (TN / 4), c = (e % (TN / 4)) * 4;
      rb[q] = (c0 + c < d) ? *reinterpret_cast<const float4*>(U + (size_t)(i1 + k0 + k) * d + c0 + c)
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store = [&]() {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + 256 * q;
      const int r = e / (KC / 4), k = (e % (KC / 4)) * 4;
      As[k + 0][r] = ra[q].x;
      As[k + 1][r] = ra[q].y;
      As[k + 2][r] = ra[q].z;
      As[k + 3][r] = ra[q].w;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + 256 * q;
      const int k = e / (TN / 4), c = (e % (TN / 4)) * 4;
      *reinterpret_cast<float4*>(&Bs[k][c]) = rb[q];
    }
  };
  float acc[8][8];
#pragma unroll
  for (int p = 0; p < 8; ++p)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[p][q] = 0.0f;
  fetch(0);
  for (int k0 = 0; k0 < B; k0 += KC) {
    __syncthreads();
    store();
    __syncthreads();
    if (k0 + KC < B) fetch(k0 + KC);
#pragma unroll 4
    for (int k = 0; k < KC; ++k) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[k][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[k][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[k][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[k][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int p = 0; p < 8; ++p)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[p][q] = fmaf(av[p], bv[q], acc[p][q]);
    }
  }
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int64_t gr = r0 + (p < 4 ? ty * 4 + p : 64 + ty * 4 + (p - 4));
    if (gr >= m) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int gc = c0 + h * 64 + tx * 4;
      if (gc < d) {
        float4* dst = reinterpret_cast<float4*>(w + gr * d + gc);
        float4 o = *dst;
        o.x -= acc[p][4 * h + 0];
        o.y -= acc[p][4 * h + 1];
        o.z -= acc[p][4 * h + 2];
        o.w -= acc[p][4 * h + 3];
        *dst = o;
      }
    }
  }
}

// One thread per 32-code unit: the unit's 32 code bytes come in as two 16-byte loads (eight 4-byte
// loads when the codes are only 4-byte aligned, single bytes otherwise) and leave as exactly BITS
// words, so a warp reads 1 KB and writes 128 * BITS bytes, both contiguous.  HBM-bound: m d (1 + b/8)
// bytes.  `align`: 16, 4 or 1, the alignment every unit's first code byte has.
template <int BITS>
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t* __restrict__ codes, int64_t m, int d, int align,
                                                   int32_t* __restrict__ packed) {
  const int upr = d / 32, wpr = upr * BITS;
  constexpr uint32_t mask = (1u << BITS) - 1u;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < m * upr; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / upr;
    const int u = (int)(e % upr);
    const uint8_t* src = codes + row * d + (int64_t)u * 32;
    uint32_t c[8];
    if (align == 16) {
      const uint4 lo = __ldg(reinterpret_cast<const uint4*>(src)), hi = __ldg(reinterpret_cast<const uint4*>(src) + 1);
      c[0] = lo.x, c[1] = lo.y, c[2] = lo.z, c[3] = lo.w, c[4] = hi.x, c[5] = hi.y, c[6] = hi.z, c[7] = hi.w;
    } else if (align == 4) {
#pragma unroll
      for (int k = 0; k < 8; ++k) c[k] = __ldg(reinterpret_cast<const uint32_t*>(src) + k);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        c[k] = (uint32_t)src[4 * k] | ((uint32_t)src[4 * k + 1] << 8) | ((uint32_t)src[4 * k + 2] << 16) |
               ((uint32_t)src[4 * k + 3] << 24);
    }
    uint32_t w[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = 0u;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t q = (c[j / 4] >> (8 * (j % 4))) & mask;
      const int bit = BITS * j, k = bit / 32, sh = bit % 32;
      w[k] |= q << sh;
      if (sh + BITS > 32) w[k + 1] |= q >> (32 - sh);
    }
    int32_t* dst = packed + row * wpr + (int64_t)u * BITS;
#pragma unroll
    for (int k = 0; k < BITS; ++k) dst[k] = (int32_t)w[k];
  }
}

template <typename T>
void launch_convert(const void* W, int64_t m, int d, int bits, int gs, float* ww, float* sc, int32_t* z,
                    cudaStream_t s) {
  const int grid = (int)((m + kRowsPerCta - 1) / kRowsPerCta);
  convert_rowgrid_kernel<T><<<grid, 256, 0, s>>>(static_cast<const T*>(W), m, d, bits, gs, ww, sc, z);
}

// Per-block launches: the column loop of block [i1, i1 + B) for all rows, then the lazy update of the
// trailing columns, on the tensor cores (3xTF32) unless `fma` asks for the fp32 FMA tile kernel or the
// buffers are not 16-byte aligned for TMA.
// The lazy update of 128-column blocks on CTA pairs (gemm_tf32x3_pair.cu), in two levels.  Columns
// are grouped in outer blocks of kOuter = 1024 (eight blocks).  After each block's column loop its
// errors update the remaining columns of the same outer block (K = 128); after the outer block's last
// block, the outer block's errors (Err [m, 1024]) update all later columns at once (K = 1024).  In
// exact arithmetic this is the same sum as one update per block (each column still receives every
// earlier block's term before its own block runs); it reads and writes the trailing W once per outer
// block instead of once per block.  Errors and U panels are split into tf32 hi / lo first:
// err/e_hi/e_lo [m, 1024], u_hi/u_lo [d, 1024] (or [n, 128] for the inner updates).
constexpr int kOuter = 1024;
struct PairBuffers {
  float *e_hi, *e_lo, *u_hi, *u_lo;
};

template <int NS>
gptq_status run_blocks(float* ww, int64_t m, int d, const float* U, int bits, int gs, uint8_t* codes,
                       float* scales, int32_t* zeros, float* err, bool fma, int32_t* status, cudaStream_t s,
                       const PairBuffers* pb) {
  constexpr int B = 32 * NS;
  // lanes per row of the column loop: 8 while that still leaves about 7 warps per SM, else 4
  const bool lpr8 = m <= 6144;
  constexpr int C4 = B / 4, C8 = B / 8;
  constexpr int CS4 = ((C4 + 4) / 4) % 2 == 1 ? C4 + 4 : C4 + 8, CS8 = ((C8 + 4) / 4) % 2 == 1 ? C8 + 4 : C8 + 8;
  const int loop_rows = lpr8 ? 16 : 32;  // 4 warps of 32 / LPR rows
  const int smem = (B * (lpr8 ? 8 * CS8 : 4 * CS4) + B) * (int)sizeof(float);
  if (lpr8)
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(colloop_kernel<C8, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  else
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(colloop_kernel<C4, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int grid_rows = (int)((m + loop_rows - 1) / loop_rows);
  CUtensorMap mErr, mU, mW;
  const bool tc = quantize_lazy_on_tensor_cores(m, d, fma ? GPTQ_FLAG_FP32_FMA : 0u);
  // every base is 16-byte aligned and every row stride a multiple of 16 bytes here (d % 32 == 0), so
  // the maps encode unless the driver call itself fails
  if (tc && !(tf32x3_map(&mErr, err, m, B, B, 128) && tf32x3_map(&mU, U, d, d, d, 32, true) &&
              tf32x3_map(&mW, ww, m, d, d, 32)))
    return GPTQ_ERR_CUDA;
  const bool pair = tc && B == 128 && pb != nullptr;
  // outer blocks of 1024 columns when every group lies inside one (a group's grid reads its later
  // columns at the group start, so those must have received every earlier update), else 128
  const int outer = (pair && (gs == 0 || kOuter % gs == 0)) ? kOuter : B;
  const int err_ld = pair ? kOuter : B;  // the err buffer holds an outer block's errors on the pair path
  CUtensorMap mEh, mEl, mUh, mUl, mUin_h, mUin_l;
  if (pair && !(split_map(&mEh, pb->e_hi, m, kOuter, kOuter) && split_map(&mEl, pb->e_lo, m, kOuter, kOuter) &&
                split_map(&mUh, pb->u_hi, d, outer, outer) && split_map(&mUl, pb->u_lo, d, outer, outer) &&
                split_map(&mUin_h, pb->u_hi, d, B, B) && split_map(&mUin_l, pb->u_lo, d, B, B)))
    return GPTQ_ERR_CUDA;
  auto pair_update = [&](const CUtensorMap& a_hi, const CUtensorMap& a_lo, const CUtensorMap& b_hi,
                         const CUtensorMap& b_lo, int c0, int c1, int K) -> gptq_status {
    PairGemmArgs pg{};
    pg.kind = kPairLazy;
    pg.tiles_n = (c1 - c0 + 255) / 256;
    pg.tiles = (int)((m + 255) / 256) * pg.tiles_n;
    pg.nk = K / 32;
    pg.o_w = c1;
    pg.o_h = (int)m;
    pg.out_y0 = 0;
    pg.out_x0 = c0;
    pg.status = status;
    return tf32x3_pair_launch(a_hi, a_lo, b_hi, b_lo, mW, pg, s);
  };
  Tf32x3Args g{};
  g.kind = kGemmLazy;
  g.epi = kEpiSub;
  g.b_mn = 1;
  g.k = B;
  g.o_w = d;
  g.o_h = (int)m;
  g.status = status;
  const int tiles_m = (int)((m + 127) / 128);
  for (int i1 = 0; i1 < d; i1 += B) {
    const int o0 = pair ? i1 / outer * outer : i1;           // start of this block's outer block
    const int slot = i1 - o0;                                 // its column offset in the outer block
    float* err_b = err + slot;                                // this block's errors (row stride err_ld)
    // on the pair path the column loop writes the errors split into tf32 hi / lo (slot of the outer block)
    float* eh = pair ? pb->e_hi + slot : nullptr;
    float* el = pair ? pb->e_lo + slot : nullptr;
    if (lpr8)
      colloop_kernel<C8, 8><<<grid_rows, 128, smem, s>>>(ww, m, d, i1, U, bits, gs, codes, scales, zeros, err_b,
                                                        err_ld, eh, el);
    else
      colloop_kernel<C4, 4><<<grid_rows, 128, smem, s>>>(ww, m, d, i1, U, bits, gs, codes, scales, zeros, err_b,
                                                        err_ld, eh, el);
    GPTQ_LAUNCH_CHECK();
    const int rest = d - (i1 + B);
    if (rest > 0) {
      if (pair) {
        const int oend = std::min(o0 + outer, d);
        gptq_status st = GPTQ_OK;
        if (i1 + B < oend) {  // the rest of this outer block, K = 128 (this block's errors)
          CUtensorMap mEbh, mEbl;
          if (!split_map(&mEbh, pb->e_hi + slot, m, B, kOuter) || !split_map(&mEbl, pb->e_lo + slot, m, B, kOuter))
            return GPTQ_ERR_CUDA;
          st = split_transpose_launch(U + (size_t)i1 * d + i1 + B, d, oend - (i1 + B), B, pb->u_hi, pb->u_lo, s);
          if (st == GPTQ_OK) st = pair_update(mEbh, mEbl, mUin_h, mUin_l, i1 + B, oend, B);
          if (st != GPTQ_OK) return st;
        }
        if (i1 + B == oend && oend < d) {  // the outer block is done: every later column, K = outer
          st = split_transpose_launch(U + (size_t)o0 * d + oend, d, d - oend, outer, pb->u_hi, pb->u_lo, s);
          if (st == GPTQ_OK) {
            if (outer == kOuter) {
              st = pair_update(mEh, mEl, mUh, mUl, oend, d, kOuter);
            } else {  // one block per outer block: its errors sit at slot 0 with row stride kOuter
              CUtensorMap mEbh, mEbl;
              if (!split_map(&mEbh, pb->e_hi, m, B, kOuter) || !split_map(&mEbl, pb->e_lo, m, B, kOuter))
                return GPTQ_ERR_CUDA;
              st = pair_update(mEbh, mEbl, mUh, mUl, oend, d, B);
            }
          }
          if (st != GPTQ_OK) return st;
        }
      } else if (tc) {
        g.i1 = i1;
        g.i2 = i1 + B;
        g.tiles_n = (rest + 127) / 128;
        g.tiles = tiles_m * g.tiles_n;
        const gptq_status st = tf32x3_gemm_launch(mErr, mU, mW, g, s);
        if (st != GPTQ_OK) return st;
      } else {
        dim3 grid((unsigned)((m + 127) / 128), (rest + 127) / 128);
        lazy_gemm_kernel<B><<<grid, 256, 0, s>>>(ww, m, d, i1, U, err);
        GPTQ_LAUNCH_CHECK();
      }
    }
  }
  return GPTQ_OK;
}

template <typename T, int NS>
gptq_status launch_rows(const void* W, int64_t m, int d, const float* U, int bits, int gs, float* ww, uint8_t* codes,
                        float* scales, int32_t* zeros, cudaStream_t s) {
  constexpr int B = 32 * NS;
  const int smem = (2 * B * 128 + B + kRowsPerCta * B) * sizeof(float);
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(quantize_rows_kernel<T, NS>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int grid = (int)((m + kRowsPerCta - 1) / kRowsPerCta);
  quantize_rows_kernel<T, NS><<<grid, 256, smem, s>>>(static_cast<const T*>(W), m, d, U, bits, gs, ww, codes, scales,
                                                      zeros);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

template <typename T>
gptq_status launch_rows_b(const void* W, int64_t m, int d, const float* U, const gptq_quant_cfg& cfg, float* ww,
                          uint8_t* codes, float* scales, int32_t* zeros, cudaStream_t s) {
  switch (cfg.block_size) {
    case 32: return launch_rows<T, 1>(W, m, d, U, cfg.bits, cfg.group_size, ww, codes, scales, zeros, s);
    case 64: return launch_rows<T, 2>(W, m, d, U, cfg.bits, cfg.group_size, ww, codes, scales, zeros, s);
    case 128: return launch_rows<T, 4>(W, m, d, U, cfg.bits, cfg.group_size, ww, codes, scales, zeros, s);
    default: return GPTQ_ERR_ARG;
  }
}

}  // namespace

// fp32 working copy of W, the block's errors, and (128-column blocks on the per-block path) an outer
// block's errors with their tf32 hi / lo splits and the split U panels of the two-level lazy update
bool pair_lazy_layout(int64_t m, int64_t d, int block_size) { return block_size == 128 && !quantize_fused(m, d); }

size_t quantize_workspace(int64_t m, int64_t d, int block_size) {
  const int err_w = pair_lazy_layout(m, d, block_size) ? kOuter : block_size;
  size_t n = align_up((size_t)m * d * sizeof(float), 256) + align_up((size_t)m * err_w * sizeof(float), 256);
  if (pair_lazy_layout(m, d, block_size))
    n += 2 * align_up((size_t)m * kOuter * sizeof(float), 256) + 2 * align_up((size_t)d * kOuter * sizeof(float), 256);
  return n;
}

// One launch per layer with 8 rows per CTA pays off while rows are few (each CTA streams all of U
// from L2 for only 8 rows); with many rows the per-block launches run the lazy update as one large
// GEMM across all rows instead.
bool quantize_fused(int64_t m, int64_t d) { return d <= 4096 && m <= 2048; }

bool quantize_lazy_on_tensor_cores(int64_t m, int64_t d, uint32_t flags) {
  // the tensor-core update numbers its 128x128 tiles with 32-bit ints
  const bool tiles_fit = ((m + 127) / 128) * ((d + 127) / 128) <= 0x7fffffff;
  return !quantize_fused(m, d) && !(flags & GPTQ_FLAG_FP32_FMA) && tiles_fit;
}

gptq_status quantize_launch(const void* W, int32_t w_dtype, int64_t m, int64_t d64, const float* U,
                            const gptq_quant_cfg& cfg, uint8_t* codes, float* scales, int32_t* zeros,
                            int32_t* status, void* workspace, cudaStream_t s, bool clear_status) {
  const int d = (int)d64;
  if (clear_status) GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), s));
  char* ws = static_cast<char*>(workspace);
  float* ww = reinterpret_cast<float*>(ws);
  float* err = reinterpret_cast<float*>(ws + align_up((size_t)m * d * sizeof(float), 256));
  if (quantize_fused(m, d)) {
    switch (w_dtype) {
      case GPTQ_FP32: return launch_rows_b<float>(W, m, d, U, cfg, ww, codes, scales, zeros, s);
      case GPTQ_FP16: return launch_rows_b<__half>(W, m, d, U, cfg, ww, codes, scales, zeros, s);
      case GPTQ_BF16: return launch_rows_b<__nv_bfloat16>(W, m, d, U, cfg, ww, codes, scales, zeros, s);
      default: return GPTQ_ERR_ARG;
    }
  }
  switch (w_dtype) {
    case GPTQ_FP32: launch_convert<float>(W, m, d, cfg.bits, cfg.group_size, ww, scales, zeros, s); break;
    case GPTQ_FP16: launch_convert<__half>(W, m, d, cfg.bits, cfg.group_size, ww, scales, zeros, s); break;
    case GPTQ_BF16: launch_convert<__nv_bfloat16>(W, m, d, cfg.bits, cfg.group_size, ww, scales, zeros, s); break;
    default: return GPTQ_ERR_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  const bool fma = (cfg.flags & GPTQ_FLAG_FP32_FMA) != 0;
  PairBuffers pb;
  const bool pair_layout = pair_lazy_layout(m, d, cfg.block_size);
  if (pair_layout) {
    size_t off = align_up((size_t)m * d * sizeof(float), 256) + align_up((size_t)m * kOuter * sizeof(float), 256);
    pb.e_hi = reinterpret_cast<float*>(ws + off);
    off += align_up((size_t)m * kOuter * sizeof(float), 256);
    pb.e_lo = reinterpret_cast<float*>(ws + off);
    off += align_up((size_t)m * kOuter * sizeof(float), 256);
    pb.u_hi = reinterpret_cast<float*>(ws + off);
    off += align_up((size_t)d * kOuter * sizeof(float), 256);
    pb.u_lo = reinterpret_cast<float*>(ws + off);
  }
  switch (cfg.block_size) {
    case 32: return run_blocks<1>(ww, m, d, U, cfg.bits, cfg.group_size, codes, scales, zeros, err, fma, status, s,
                                  nullptr);
    case 64: return run_blocks<2>(ww, m, d, U, cfg.bits, cfg.group_size, codes, scales, zeros, err, fma, status, s,
                                  nullptr);
    case 128: return run_blocks<4>(ww, m, d, U, cfg.bits, cfg.group_size, codes, scales, zeros, err, fma, status, s,
                                   pair_layout ? &pb : nullptr);
    default: return GPTQ_ERR_ARG;
  }
}

gptq_status pack_launch(const uint8_t* codes, int64_t m, int64_t d, int32_t bits, int32_t* packed,
                        cudaStream_t s) {
  const int64_t n = m * (d * bits / 32);
  if (n == 0) return GPTQ_OK;
  const int64_t units = m * (d / 32);
  const int blocks = (int)std::min<int64_t>((units + 255) / 256, 148 * 16);
  // d % 32 == 0, so every unit starts as aligned as the codes' base
  const uintptr_t base = reinterpret_cast<uintptr_t>(codes);
  const int align = base % 16 == 0 ? 16 : (base % 4 == 0 ? 4 : 1);
  switch (bits) {
    case 2: pack_kernel<2><<<blocks, 256, 0, s>>>(codes, m, (int)d, align, packed); break;
    case 3: pack_kernel<3><<<blocks, 256, 0, s>>>(codes, m, (int)d, align, packed); break;
    case 4: pack_kernel<4><<<blocks, 256, 0, s>>>(codes, m, (int)d, align, packed); break;
    default: return GPTQ_ERR_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
