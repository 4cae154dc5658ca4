// Inference with the packed weights: Y = X_in @ What^T, What[r, j] = scale[r, g] (q[r, j] - zero[r, g]),
// the codes read straight from the packed words (FDE Interviews breakdown of GPTQ, section 01, last
// paragraph: kernels that read the 3-bit weights and dequantize them on the fly).
//
// Every packed word is read once, so for a handful of input rows the bound is HBM, and the work to keep
// under it is the integer work of taking the codes apart.  A unit of 32 codes is exactly `bits` words of
// a row's bit stream (code j in bits [b j, b j + b)).  Each word gets two copies carrying the exponent of
// 1.0 in bits [23, 32): its own bits [0, 23), and the word shifted down (joined with the next word where a
// code straddles the two) so that its upper codes sit below bit 23.  A code whose bits are [s, s + b) in
// one of the copies is then ONE AND with an immediate away from F = 1 + q 2^(s - 23), exact.  F - 1 =
// q 2^(s - 23) is exact too, and one fused F c - c with c the input pre-scaled by 2^(23 - s) (an exact
// power-of-two scaling shared by all rows) gives q x_j with a single rounding; it and the accumulation
// run as fp32x2 operations on two codes at a time.  A unit adds scale (sum_j q_j x_j - zero sum_j x_j) to
// its row (units never straddle a group: group sizes are multiples of 32); with a per-row grid the sums
// run over all of a thread's units first.  The pre-scaled inputs stay finite for |x| < 2^100.
//
// Two tilings of the same arithmetic, split-K over column tiles (a second kernel sums the tiles in
// order, so the result does not depend on scheduling):
//  * staged form (d % 128 == 0): each warp streams its rows through a ring of shared-memory stages
//    filled by bulk async copies (below);
//  * register form (any d % 32 == 0): a CTA takes 64 rows x 4096 columns; warp w owns 8 rows, lane l the
//    units l, l + 32, ... of the tile, loading the next unit's words while it decodes the current one.
#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

// Building with GPTQ_DQ_STAGED=0 keeps the register form for every order (for comparisons).
#ifndef GPTQ_DQ_STAGED
#define GPTQ_DQ_STAGED 1
#endif
constexpr int kWarps = 8;
// rows per warp: fewer rows for more input rows, so that a thread's sums stay in registers
__host__ __device__ constexpr int rows_per_warp(int nb) { return nb == 1 ? 8 : (nb == 2 ? 4 : 2); }
constexpr int kUnitsPerTile = 128;  // 32-column units per column tile of the register form

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// 1 + q_j / 2^BITS for code j (0..31) of a unit held in w[0..BITS-1].
template <int BITS>
__device__ __forceinline__ float decode(const uint32_t (&w)[BITS], const int j) {
  constexpr int P = 23 - BITS;  // mantissa position of the code
  const int bit = BITS * j, k = bit >> 5, s = bit & 31;
  uint32_t v;
  if (s >= P) {
    const uint32_t hi = (k + 1 < BITS) ? w[k + 1] : 0u;
    v = __funnelshift_r(w[k], hi, s - P);
  } else {
    const uint32_t lo = (k > 0) ? w[k - 1] : 0u;
    v = __funnelshift_l(lo, w[k], P - s);
  }
  return __uint_as_float((v & (((1u << BITS) - 1u) << P)) | 0x3F800000u);
}

// Where code j of a unit is decoded: its word, its bit offset inside the register it is masked from,
// and whether that register is the word itself or the word's shifted copy.
template <int BITS>
struct UnitLayout {
  __host__ __device__ static constexpr int word(int j) { return BITS * j / 32; }
  __host__ __device__ static constexpr int local(int j) { return BITS * j % 32; }
  __host__ __device__ static constexpr bool direct(int j) { return local(j) + BITS <= 23; }
  // end (exclusive, from the word's bit 0) of the last code that starts in word k: 32 or a little more
  __host__ __device__ static constexpr int last_end(int k) {
    return BITS * ((32 * k + 31) / BITS) + BITS - 32 * k;
  }
  // right shift of word k (joined with word k + 1) that puts its last code at bits [23 - b, 23)
  __host__ __device__ static constexpr int shift(int k) { return last_end(k) - 23; }
  __host__ __device__ static constexpr bool straddles(int k) { return last_end(k) > 32; }
  __host__ __device__ static constexpr int pos(int j) { return direct(j) ? local(j) : local(j) - shift(word(j)); }
};
// every code's bits lie in [0, 23) of its register (checked for each width at compile time)
template <int BITS>
__host__ __device__ constexpr bool layout_ok() {
  for (int j = 0; j < 32; ++j) {
    const int p = UnitLayout<BITS>::pos(j);
    if (p < 0 || p + BITS > 23) return false;
  }
  for (int k = 0; k < BITS; ++k)  // plain shifts clear bits [23, 32) of the shifted copy
    if (!UnitLayout<BITS>::straddles(k) && UnitLayout<BITS>::shift(k) < 9) return false;
  return UnitLayout<BITS>::last_end(BITS - 1) == 32;  // the unit's last word ends on a code boundary
}
static_assert(layout_ok<2>() && layout_ok<3>() && layout_ok<4>(), "code positions");

__host__ __device__ constexpr float pow2i(int e) { return (float)(1u << e); }
constexpr uint32_t kOneBits = 0x3F800000u;  // 1.0f

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// register pairs are formed and split with PTX vector moves, which cost no instructions
__device__ __forceinline__ uint64_t pack_u32(uint32_t lo, uint32_t hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
  return d;
}
__device__ __forceinline__ uint64_t pack2(float lo, float hi) { return pack_u32(__float_as_uint(lo), __float_as_uint(hi)); }
__device__ __forceinline__ void unpack_u32(uint64_t v, uint32_t& lo, uint32_t& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
}
__device__ __forceinline__ float lo_of(uint64_t v) {
  uint32_t lo, hi;
  unpack_u32(v, lo, hi);
  return __uint_as_float(lo);
}
__device__ __forceinline__ float hi_of(uint64_t v) {
  uint32_t lo, hi;
  unpack_u32(v, lo, hi);
  return __uint_as_float(hi);
}

template <typename T>
__device__ __forceinline__ void load_pairs8(const T* p, uint64_t (&v)[4]);  // 8 values as 4 (even, odd) pairs
template <>
__device__ __forceinline__ void load_pairs8<float>(const float* p, uint64_t (&v)[4]) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = pack2(a.x, a.y), v[1] = pack2(a.z, a.w), v[2] = pack2(b.x, b.y), v[3] = pack2(b.z, b.w);
}
template <>
__device__ __forceinline__ void load_pairs8<__half>(const __half* p, uint64_t (&v)[4]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[k]));
    v[k] = pack2(f.x, f.y);
  }
}
template <>
__device__ __forceinline__ void load_pairs8<__nv_bfloat16>(const __nv_bfloat16* p, uint64_t (&v)[4]) {
  const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
    v[k] = pack2(f.x, f.y);
  }
}

// One pair of codes (2P, 2P + 1) for every row: part[r][b] += (q_2P x_2P, q_2P+1 x_2P+1).  The code
// index is a template argument, so every position, mask and scale below is a compile-time constant.
template <int BITS, int RW, int NB, int P>
__device__ __forceinline__ void pair_step(const uint32_t (&wo)[RW][BITS], const uint32_t (&vo)[RW][BITS],
                                          const uint64_t (&c)[NB], const uint64_t (&nc)[NB],
                                          uint64_t (&part)[RW][NB]) {
  using L = UnitLayout<BITS>;
  constexpr int j = 2 * P;
  constexpr int k0 = L::word(j), k1 = L::word(j + 1);
  constexpr bool d0 = L::direct(j), d1 = L::direct(j + 1);
  // the code's bits and the exponent field: one AND with an immediate gives F
  constexpr uint32_t m0 = (((1u << BITS) - 1u) << L::pos(j)) | kOneBits;
  constexpr uint32_t m1 = (((1u << BITS) - 1u) << L::pos(j + 1)) | kOneBits;
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const uint32_t s0 = d0 ? wo[r][k0] : vo[r][k0];
    const uint32_t s1 = d1 ? wo[r][k1] : vo[r][k1];
    const uint64_t f = pack_u32(s0 & m0, s1 & m1);
    // F c - c = (F - 1) c = q x exactly before the one rounding
#pragma unroll
    for (int b = 0; b < NB; ++b) part[r][b] = add2(part[r][b], fma2(f, c[b], nc[b]));
  }
}

// Codes 8Q .. 8Q + 7: their inputs are loaded and pre-scaled once for all rows, then four pair steps.
template <int BITS, int RW, int NB, typename TX, int Q>
__device__ __forceinline__ void quad_step(const uint32_t (&wo)[RW][BITS], const uint32_t (&vo)[RW][BITS],
                                          const TX* __restrict__ xp, int64_t ldx, uint64_t (&part)[RW][NB],
                                          float (&xs)[NB]) {
  using L = UnitLayout<BITS>;
  uint64_t c[4][NB], nc[4][NB];  // (even, odd) input pairs scaled by 2^(23 - pos): c and -c
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    uint64_t xv[4];
    load_pairs8<TX>(xp + b * ldx + 8 * Q, xv);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const float lo = lo_of(xv[t]), hi = hi_of(xv[t]);
      xs[b] += lo + hi;
      const float s0 = pow2i(23 - L::pos(8 * Q + 2 * t)), s1 = pow2i(23 - L::pos(8 * Q + 2 * t + 1));
      c[t][b] = pack2(lo * s0, hi * s1);
      nc[t][b] = pack2(lo * -s0, hi * -s1);
    }
  }
  pair_step<BITS, RW, NB, 4 * Q + 0>(wo, vo, c[0], nc[0], part);
  pair_step<BITS, RW, NB, 4 * Q + 1>(wo, vo, c[1], nc[1], part);
  pair_step<BITS, RW, NB, 4 * Q + 2>(wo, vo, c[2], nc[2], part);
  pair_step<BITS, RW, NB, 4 * Q + 3>(wo, vo, c[3], nc[3], part);
}

// part[r][b] += (sum over the unit's even codes of q x, sum over its odd codes of q x) for the RW rows
// whose words are w[r] and input row b; xs[b] += the sum of the unit's inputs.  xp: the unit's first input.
// Each word gets two copies that carry the exponent of 1.0 in bits [23, 32): wo (the word's bits [0, 23))
// and vo (the word shifted down past its upper codes); a code is then one AND away from its F.
// one_bits holds the bits of 1.0f in a register (read from shared memory by the caller).
template <int BITS, int RW, int NB, typename TX>
__device__ __forceinline__ void unit_dot(const uint32_t (&w)[RW][BITS], const TX* __restrict__ xp, int64_t ldx,
                                         uint32_t one_bits, uint64_t (&part)[RW][NB], float (&xs)[NB]) {
  using L = UnitLayout<BITS>;
  uint32_t wo[RW][BITS], vo[RW][BITS];
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int k = 0; k < BITS; ++k) {
      wo[r][k] = (w[r][k] & 0x007FFFFFu) | one_bits;
      if (L::straddles(k))
        vo[r][k] = (__funnelshift_r(w[r][k], w[r][k + 1 < BITS ? k + 1 : k], L::shift(k)) & 0x007FFFFFu) | one_bits;
      else
        vo[r][k] = (w[r][k] >> L::shift(k)) | one_bits;  // a shift by >= 9 leaves bits [23, 32) clear
    }
  quad_step<BITS, RW, NB, TX, 0>(wo, vo, xp, ldx, part, xs);
  quad_step<BITS, RW, NB, TX, 1>(wo, vo, xp, ldx, part, xs);
  quad_step<BITS, RW, NB, TX, 2>(wo, vo, xp, ldx, part, xs);
  quad_step<BITS, RW, NB, TX, 3>(wo, vo, xp, ldx, part, xs);
}

// the grid (scale, zero) of rows row0 + r at grid column g (zeros for rows past m)
template <int RW>
__device__ __forceinline__ void load_grid(const float* __restrict__ scales, const int32_t* __restrict__ zeros, int row0,
                                          int m, int ng, int g, float (&sc)[RW], int32_t (&z)[RW]) {
#pragma unroll
  for (int r = 0; r < RW; ++r) {
    const int row = row0 + r;
    sc[r] = row < m ? __ldg(scales + (int64_t)row * ng + g) : 0.0f;
    z[r] = row < m ? __ldg(zeros + (int64_t)row * ng + g) : 0;
  }
}

// acc[r][b] += scale (sum q x - zero sum x); clears the sums
template <int RW, int NB>
__device__ __forceinline__ void unit_finish(uint64_t (&part)[RW][NB], float (&xs)[NB], const float (&sc)[RW],
                                            const int32_t (&z)[RW], float (&acc)[RW][NB]) {
#pragma unroll
  for (int r = 0; r < RW; ++r) {
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      acc[r][b] = fmaf(sc[r], fmaf(-(float)z[r], xs[b], lo_of(part[r][b]) + hi_of(part[r][b])), acc[r][b]);
      part[r][b] = 0ull;
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) xs[b] = 0.0f;
}

// the warp's row sums (over lanes) written as this column tile's partial sums
template <int RW, int NB>
__device__ __forceinline__ void write_partials(float (&acc)[RW][NB], int lane, int row0, int m, int batch,
                                               float* __restrict__ partial) {
#pragma unroll
  for (int r = 0; r < RW; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      float v = acc[r][b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      acc[r][b] = v;
    }
  if (lane == 0) {
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int row = row0 + r;
      if (row < m) {
#pragma unroll
        for (int b = 0; b < NB; ++b) partial[((int64_t)blockIdx.y * batch + b) * m + row] = acc[r][b];
      }
    }
  }
}

template <int BITS, int NB, typename TX>
__global__ void __launch_bounds__(kWarps * 32, 2) dequant_matmul_kernel(const uint32_t* __restrict__ packed,
                                                                     const float* __restrict__ scales,
                                                                     const int32_t* __restrict__ zeros, int m,
                                                                     int d, int group_size,
                                                                     const TX* __restrict__ X, int64_t ldx,
                                                                     float* __restrict__ partial, int batch) {
  constexpr int RW = rows_per_warp(NB);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row0 = (blockIdx.x * kWarps + warp) * RW;
  __shared__ uint32_t s_one;
  if (threadIdx.x == 0) s_one = 0x3F800000u;
  __syncthreads();
  const uint32_t one_bits = s_one;
  const int n_units = d >> 5;
  const int u_begin = blockIdx.y * kUnitsPerTile;
  const int u_end = min(n_units, u_begin + kUnitsPerTile);
  const int wpr = n_units * BITS;  // words per row
  const int ng = group_size ? d / group_size : 1;
  const int upg = group_size ? group_size >> 5 : n_units;
  float acc[RW][NB], xs[NB];
  uint64_t part[RW][NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    xs[b] = 0.0f;
#pragma unroll
    for (int r = 0; r < RW; ++r) acc[r][b] = 0.0f, part[r][b] = 0ull;
  }
  uint32_t w[RW][BITS], wn[RW][BITS];
  float sc[RW];
  int32_t z[RW];
  auto load_words = [&](uint32_t (&dst)[RW][BITS], int u) {
#pragma unroll
    for (int r = 0; r < RW; ++r) {
      const int row = row0 + r;
#pragma unroll
      for (int k = 0; k < BITS; ++k)
        dst[r][k] = (row < m && u < u_end) ? __ldg(packed + (int64_t)row * wpr + (int64_t)u * BITS + k) : 0u;
    }
  };
  // the next unit's words are loaded while the current one is decoded
  int u = u_begin + lane;
  load_words(wn, u);
  for (; u < u_end; u += 32) {
#pragma unroll
    for (int r = 0; r < RW; ++r)
#pragma unroll
      for (int k = 0; k < BITS; ++k) w[r][k] = wn[r][k];
    load_words(wn, u + 32);
    unit_dot<BITS, RW, NB, TX>(w, X + (int64_t)u * 32, ldx, one_bits, part, xs);
    if (group_size) {
      load_grid<RW>(scales, zeros, row0, m, ng, u / upg, sc, z);
      unit_finish<RW, NB>(part, xs, sc, z, acc);
    }
  }
  if (!group_size) {
    load_grid<RW>(scales, zeros, row0, m, ng, 0, sc, z);
    unit_finish<RW, NB>(part, xs, sc, z, acc);
  }
  write_partials<RW, NB>(acc, lane, row0, m, batch, partial);
}

// Staged form (d % 128 == 0): every warp streams its own RW rows through a ring of S stages in shared
// memory, one stage per 1024-column chunk (RW bulk async copies, one per row, completing on the stage's
// mbarrier).  A warp reads a landed stage into registers, refills it with the chunk S ahead and only
// then decodes, so S chunks of every warp are in flight while it computes; no warp waits for another.
constexpr int kChunkUnits = 32;  // one unit per lane per chunk

// stages per warp: about 96 KB of packed words per CTA (two CTAs per SM), at most 8
template <int BITS, int NB>
__host__ __device__ constexpr int staged_depth() {
  return 96 / (rows_per_warp(NB) * BITS) > 8 ? 8 : 96 / (rows_per_warp(NB) * BITS);
}
template <int BITS, int NB>
__host__ __device__ constexpr int staged_smem_bytes() {
  return kWarps * staged_depth<BITS, NB>() * rows_per_warp(NB) * kChunkUnits * BITS * 4;
}

// one lane's BITS words of a unit from shared memory: one 8- or 16-byte load at 2 and 4 bits (lanes
// 8 or 16 bytes apart, no bank conflicts), three 4-byte loads at 3 bits (stride 3 words, conflict-free)
template <int BITS>
__device__ __forceinline__ void load_unit_words(const uint32_t* p, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
  } else if constexpr (BITS == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x, w[1] = v.y;
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = p[k];
  }
}

template <int BITS, int NB, typename TX>
__global__ void __launch_bounds__(kWarps * 32, 2) dequant_matmul_staged_kernel(
    const uint32_t* __restrict__ packed, const float* __restrict__ scales, const int32_t* __restrict__ zeros, int m,
    int d, int group_size, const TX* __restrict__ X, int64_t ldx, float* __restrict__ partial, int batch,
    int chunks_per_tile, int32_t* status) {
  constexpr int RW = rows_per_warp(NB);
  constexpr int S = staged_depth<BITS, NB>();
  constexpr int CW = kChunkUnits * BITS;  // words of one row in one chunk
  extern __shared__ __align__(128) uint32_t sw[];  // [warp][stage][row][CW]
  __shared__ uint64_t bars[kWarps][S];
  __shared__ int abort_flag;
  __shared__ uint32_t s_one;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = d >> 5, wpr = n_units * BITS;
  const int n_chunks = (n_units + kChunkUnits - 1) / kChunkUnits;
  const int ng = group_size ? d / group_size : 1;
  const int upg = group_size ? group_size >> 5 : n_units;
  const int row0 = (blockIdx.x * kWarps + warp) * RW;
  const int rows = max(0, min(RW, m - row0));
  const int c0 = blockIdx.y * chunks_per_tile, c1 = min(n_chunks, c0 + chunks_per_tile);
  uint32_t* ring = sw + warp * S * RW * CW;
  if (threadIdx.x == 0) {
    for (int w = 0; w < kWarps; ++w)
      for (int st = 0; st < S; ++st) tc::mbar_init(&bars[w][st], 1);
    abort_flag = 0;
    s_one = kOneBits;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const uint32_t one_bits = s_one;
  // chunk c into stage st: lane 0 arrives with the byte count, lane r < rows copies row r
  auto issue = [&](int c, int st) {
    const int cu0 = c * kChunkUnits;
    const uint32_t bytes = (uint32_t)min(kChunkUnits, n_units - cu0) * BITS * 4;
    if (lane == 0) tc::mbar_expect_tx(&bars[warp][st], bytes * (uint32_t)rows);
    if (lane < rows)
      tc::bulk_load(ring + (st * RW + lane) * CW, packed + (int64_t)(row0 + lane) * wpr + (int64_t)cu0 * BITS, bytes,
                    &bars[warp][st]);
  };
  float acc[RW][NB], xs[NB], sc[RW];
  int32_t z[RW];
  uint64_t part[RW][NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    xs[b] = 0.0f;
#pragma unroll
    for (int r = 0; r < RW; ++r) acc[r][b] = 0.0f, part[r][b] = 0ull;
  }
  int issued = c0, consumed = c0;  // chunks issued into the ring / taken out of it
  if (rows > 0) {
    for (; issued < c1 && issued < c0 + S; ++issued) issue(issued, issued - c0);
    for (int c = c0; c < c1; ++c) {
      const int i = c - c0, st = i % S;
      const int u = c * kChunkUnits + lane;
      if (group_size) load_grid<RW>(scales, zeros, row0, m, ng, min(u, n_units - 1) / upg, sc, z);
      // bounded wait for the stage; on a timeout (or another warp's) the warp stops and drains below
      if (!tc::mbar_wait(&bars[warp][st], (uint32_t)(i / S) & 1u, &abort_flag, status, 42)) break;
      uint32_t w[RW][BITS];
#pragma unroll
      for (int r = 0; r < RW; ++r) load_unit_words<BITS>(ring + (st * RW + r) * CW + lane * BITS, w[r]);
      consumed = c + 1;
      // every lane's reads of the stage are ordered before the async copy that refills it
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (issued < c1) issue(issued++, st);
      if (u < n_units) {
        unit_dot<BITS, RW, NB, TX>(w, X + (int64_t)u * 32, ldx, one_bits, part, xs);
        if (group_size) unit_finish<RW, NB>(part, xs, sc, z, acc);
      }
    }
    // after an abort, the copies still in flight land (bounded waits) before the CTA ends
    if (abort_flag && lane == 0)
      for (int i = consumed - c0; i < issued - c0; ++i) tc::mbar_wait_drain(&bars[warp][i % S], (uint32_t)(i / S) & 1u);
  }
  if (!group_size) {
    load_grid<RW>(scales, zeros, row0, m, ng, 0, sc, z);
    unit_finish<RW, NB>(part, xs, sc, z, acc);
  }
  write_partials<RW, NB>(acc, lane, row0, m, batch, partial);
}

// Y[b][r] = sum over column tiles of the partial sums, in tile order.
__global__ void __launch_bounds__(256) dequant_reduce_kernel(const float* __restrict__ partial, int tiles,
                                                             int64_t n, float* __restrict__ Y, int64_t ldy, int m,
                                                             int b0) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int t = 0; t < tiles; ++t) s += partial[t * n + e];
    const int64_t b = e / m, r = e % m;
    Y[(b0 + b) * ldy + r] = s;
  }
}

// Column tiles of the staged form for an m x d product: the split of the row's chunks that minimises
// waves of CTAs (two per SM) x (chunks per CTA + 2), the 2 standing for a CTA's ring fill and drain;
// ties go to fewer tiles.
int staged_chunks_per_tile(int64_t m, int64_t d, int nb, int sms) {
  const int64_t row_blocks = (m + kWarps * rows_per_warp(nb) - 1) / (kWarps * rows_per_warp(nb));
  const int64_t n_chunks = (d / 32 + kChunkUnits - 1) / kChunkUnits;
  const int64_t slots = 2 * (int64_t)sms;
  int64_t best_cost = INT64_MAX, best = n_chunks;
  for (int64_t per = n_chunks; per >= 1; --per) {
    const int64_t tiles = (n_chunks + per - 1) / per;
    const int64_t cost = ((row_blocks * tiles + slots - 1) / slots) * (per + 2);
    if (cost < best_cost) best_cost = cost, best = per;
  }
  return (int)best;
}

int device_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

bool use_staged(int64_t d) { return GPTQ_DQ_STAGED && d % 128 == 0; }

template <int BITS, typename TX>
gptq_status launch_form(int nb, int m, int d, int gs, const uint32_t* packed, const float* scales,
                        const int32_t* zeros, const TX* X, int64_t ldx, float* partial, int32_t* status, int* tiles,
                        cudaStream_t s) {
  const int rows_per_cta = kWarps * rows_per_warp(nb);
  const int row_blocks = (m + rows_per_cta - 1) / rows_per_cta;
  if (use_staged(d)) {
    const int per = staged_chunks_per_tile(m, d, nb, device_sms());
    const int n_chunks = (d / 32 + kChunkUnits - 1) / kChunkUnits;
    *tiles = (n_chunks + per - 1) / per;
    const dim3 grid(row_blocks, *tiles);
    switch (nb) {
#define GPTQ_DQ_STAGED_CASE(NB)                                                                                 \
  case NB:                                                                                                       \
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(dequant_matmul_staged_kernel<BITS, NB, TX>,                               \
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,                              \
                                       staged_smem_bytes<BITS, NB>()));                                          \
    dequant_matmul_staged_kernel<BITS, NB, TX><<<grid, kWarps * 32, staged_smem_bytes<BITS, NB>(), s>>>(          \
        packed, scales, zeros, m, d, gs, X, ldx, partial, NB, per, status);                                      \
    break;
      GPTQ_DQ_STAGED_CASE(1)
      GPTQ_DQ_STAGED_CASE(2)
      GPTQ_DQ_STAGED_CASE(3)
      GPTQ_DQ_STAGED_CASE(4)
#undef GPTQ_DQ_STAGED_CASE
      default: return GPTQ_ERR_ARG;
    }
  } else {
    *tiles = (d / 32 + kUnitsPerTile - 1) / kUnitsPerTile;
    const dim3 grid(row_blocks, *tiles);
    switch (nb) {
      case 1: dequant_matmul_kernel<BITS, 1, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 1); break;
      case 2: dequant_matmul_kernel<BITS, 2, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 2); break;
      case 3: dequant_matmul_kernel<BITS, 3, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 3); break;
      case 4: dequant_matmul_kernel<BITS, 4, TX><<<grid, kWarps * 32, 0, s>>>(packed, scales, zeros, m, d, gs, X, ldx, partial, 4); break;
      default: return GPTQ_ERR_ARG;
    }
  }
  return GPTQ_OK;
}

// the most column tiles either form can use (sizes the partial sums): one per 1024-column chunk
int64_t max_tiles(int64_t d) { return std::max<int64_t>(1, (d / 32 + kChunkUnits - 1) / kChunkUnits); }

template <typename TX>
gptq_status launch_typed(const int32_t* packed, const float* scales, const int32_t* zeros, int m, int d, int bits,
                         int gs, const void* Xv, int64_t batch, float* Y, float* partial, int32_t* status,
                         cudaStream_t s) {
  const TX* X = static_cast<const TX*>(Xv);
  const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
  for (int64_t b0 = 0; b0 < batch; b0 += 4) {
    const int nb = (int)std::min<int64_t>(4, batch - b0);
    int tiles = 0;
    gptq_status st = GPTQ_ERR_ARG;
    switch (bits) {
      case 2: st = launch_form<2, TX>(nb, m, d, gs, pw, scales, zeros, X + b0 * d, d, partial, status, &tiles, s); break;
      case 3: st = launch_form<3, TX>(nb, m, d, gs, pw, scales, zeros, X + b0 * d, d, partial, status, &tiles, s); break;
      case 4: st = launch_form<4, TX>(nb, m, d, gs, pw, scales, zeros, X + b0 * d, d, partial, status, &tiles, s); break;
      default: return GPTQ_ERR_ARG;
    }
    if (st != GPTQ_OK) return st;
    GPTQ_LAUNCH_CHECK();
    const int64_t n = (int64_t)nb * m;
    const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 8);
    dequant_reduce_kernel<<<blocks, 256, 0, s>>>(partial, tiles, n, Y, m, m, (int)b0);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

// What[r][j] = scale[r][g(j)] * (q[r][j] - zero[r][g(j)]) from the packed words, 32 codes per thread
template <typename TO, int BITS>
__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t* __restrict__ packed,
                                                         const float* __restrict__ scales,
                                                         const int32_t* __restrict__ zeros, int64_t m, int d,
                                                         int group_size, TO* __restrict__ out) {
  const int units = d >> 5, ng = group_size ? d / group_size : 1, upg = group_size ? group_size >> 5 : units;
  const int wpr = units * BITS;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < m * units; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / units;
    const int u = (int)(e % units);
    uint32_t w[BITS];
#pragma unroll
    for (int k = 0; k < BITS; ++k) w[k] = packed[r * wpr + (int64_t)u * BITS + k];
    const float sc = scales[r * ng + u / upg], z = (float)zeros[r * ng + u / upg];
    TO* dst = out + r * d + (int64_t)u * 32;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float q = (decode<BITS>(w, j) - 1.0f) * (float)(1 << BITS);  // exact: q = 2^b (f - 1)
      dst[j] = from_f32<TO>(sc * (q - z));
    }
  }
}

}  // namespace

size_t dequant_matmul_workspace(int64_t m, int64_t d, int64_t batch) {
  return align_up((size_t)max_tiles(d) * (size_t)std::min<int64_t>(batch, 4) * m * sizeof(float), 256);
}

template <typename TO>
gptq_status dequantize_typed(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m, int64_t d,
                             int32_t bits, int32_t group_size, void* out, cudaStream_t s) {
  const uint32_t* pw = reinterpret_cast<const uint32_t*>(packed);
  const int64_t n = m * (d / 32);
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  TO* o = static_cast<TO*>(out);
  switch (bits) {
    case 2: dequantize_kernel<TO, 2><<<blocks, 256, 0, s>>>(pw, scales, zeros, m, (int)d, group_size, o); break;
    case 3: dequantize_kernel<TO, 3><<<blocks, 256, 0, s>>>(pw, scales, zeros, m, (int)d, group_size, o); break;
    case 4: dequantize_kernel<TO, 4><<<blocks, 256, 0, s>>>(pw, scales, zeros, m, (int)d, group_size, o); break;
    default: return GPTQ_ERR_ARG;
  }
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

gptq_status dequantize_launch(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m, int64_t d,
                              int32_t bits, int32_t group_size, void* out, int32_t out_dtype, cudaStream_t s) {
  switch (out_dtype) {
    case GPTQ_FP16: return dequantize_typed<__half>(packed, scales, zeros, m, d, bits, group_size, out, s);
    case GPTQ_BF16: return dequantize_typed<__nv_bfloat16>(packed, scales, zeros, m, d, bits, group_size, out, s);
    case GPTQ_FP32: return dequantize_typed<float>(packed, scales, zeros, m, d, bits, group_size, out, s);
    default: return GPTQ_ERR_ARG;
  }
}

gptq_status dequant_matmul_launch(const int32_t* packed, const float* scales, const int32_t* zeros, int64_t m,
                                  int64_t d, int32_t bits, int32_t group_size, const void* X, int32_t x_dtype,
                                  int64_t batch, float* Y, int32_t* status, void* workspace, cudaStream_t s) {
  float* partial = static_cast<float*>(workspace);
  GPTQ_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int32_t), s));
  switch (x_dtype) {
    case GPTQ_FP16:
      return launch_typed<__half>(packed, scales, zeros, (int)m, (int)d, bits, group_size, X, batch, Y, partial,
                                  status, s);
    case GPTQ_BF16:
      return launch_typed<__nv_bfloat16>(packed, scales, zeros, (int)m, (int)d, bits, group_size, X, batch, Y,
                                         partial, status, s);
    case GPTQ_FP32:
      return launch_typed<float>(packed, scales, zeros, (int)m, (int)d, bits, group_size, X, batch, Y, partial,
                                 status, s);
    default: return GPTQ_ERR_ARG;
  }
}

}  // namespace gptq
