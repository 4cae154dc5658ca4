// A1 on the 5th-generation tensor cores: H = scale * X^T X for 16-bit calibration inputs.
//
// GPTQ's curvature H = 2 X X^T (FDE Interviews breakdown of GPTQ, section 01; X there is
// [in, tokens]) is a symmetric rank-N product, so only tiles that touch the upper triangle are
// computed.  X is stored [tokens, d] with channels contiguous, so both operands are MN-major: a
// TMA box of 64 channels x 64 tokens lands in shared memory as 64 rows of 128 bytes with the
// 128-byte swizzle, which is the canonical MN-major SW128 layout tcgen05.mma reads directly.
//
// One CTA per SM (persistent).  A work unit is a 128 x 256 tile of H times a range of tokens
// (split-K when there are fewer tiles than SMs).  Warp roles:
//   warp 0      TMA producer: 4-stage ring of 48 KB stages (A: 128 ch, B: 256 ch, 64 tokens)
//   warp 1      tcgen05.mma issuer (one thread) + TMEM owner; 4 MMAs of K=16 per stage into one of
//               two 128x256 fp32 accumulators in TMEM (512 columns)
//   warps 2-9   epilogue: every `chunk` tokens the MMA switches accumulator and the epilogue adds
//               the finished one into fp32 registers (128 per thread), bounding the length of the
//               in-TMEM accumulation chain; at the end of a unit it writes the tile (or its split
//               partial) to global memory.
// Every mbarrier wait is bounded: on a timeout the kernel records GPTQ_ERR_TIMEOUT, lets the
// other roles leave, waits (bounded) for its own TMA copies and MMAs in flight, frees TMEM, returns.
//
// Orders 512..8192 run the CTA-pair form instead (hessian_pair_kernel, further down): 256 x 256
// tiles on two SMs with tcgen05.mma.cta_group::2, half the shared-memory traffic per product.
#include <atomic>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

constexpr int BM = 128;            // rows of the H tile (channels i)
constexpr int BN = 256;            // columns of the H tile (channels j)
constexpr int BK = 64;             // tokens per pipeline stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int CHUNK_BYTES = 64 * BK * 2;  // one TMA box: 64 channels x 64 tokens
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr uint32_t TMEM_COLS = 512;
constexpr int kPlanSMs = 148;
constexpr int kMinTokensPerSplit = 4096;
constexpr int kChunkTokens = 1024;  // flush period of the TMEM accumulator

struct TcPlan {
  int nbi, nbj, tiles, splits, units;
  int64_t tokens_per_split;
};

int tiles_for(int nbi, int nbj) {
  int t = 0;
  for (int bj = 0; bj < nbj; ++bj) t += (2 * bj + 2 < nbi) ? 2 * bj + 2 : nbi;
  return t;
}

// CTA-pair form: 256 x 256 tiles of the upper block triangle, one pair of SMs per unit
constexpr int PT = 256;            // pair tile (rows and columns)
// Orders [512, 8192] use the pair kernel.  Wider layers keep the single-CTA kernel: at d = 11008 and
// 49152 (units of all 262,144 tokens) it measured faster than the pair form (631 against 700 ms at
// 49152), while the pair form wins at 4096 (3.4 against 3.6 ms) and on short token ranges.
#ifndef GPTQ_HESSIAN_PAIR_MIN_ORDER
#define GPTQ_HESSIAN_PAIR_MIN_ORDER 512
#endif
#ifndef GPTQ_HESSIAN_PAIR_MAX_ORDER
#define GPTQ_HESSIAN_PAIR_MAX_ORDER 8192
#endif

bool use_pair(int64_t d) { return d >= GPTQ_HESSIAN_PAIR_MIN_ORDER && d <= GPTQ_HESSIAN_PAIR_MAX_ORDER; }

TcPlan tc_plan(int64_t n_tokens, int64_t d) {
  TcPlan p;
  const bool pairs = use_pair(d);
  if (pairs) {
    p.nbi = p.nbj = (int)((d + PT - 1) / PT);
    p.tiles = p.nbi * (p.nbi + 1) / 2;
  } else {
    p.nbi = (int)((d + BM - 1) / BM);
    p.nbj = (int)((d + BN - 1) / BN);
    p.tiles = tiles_for(p.nbi, p.nbj);
  }
  const int workers = pairs ? kPlanSMs / 2 : kPlanSMs;
  int64_t max_s = n_tokens / kMinTokensPerSplit;
  if (max_s < 1) max_s = 1;
  if (max_s > 16) max_s = 16;
  // Split the tokens only when one split leaves SMs idle: every split adds a write and a re-read of
  // all partial tiles (at d = 49152, 13 splits were 63 GB of partials for a 0.24 % shorter tail).
  auto efficiency = [&](int s) {
    const int units = p.tiles * s;
    const int waves = (units + workers - 1) / workers;
    return (double)units / ((double)waves * workers);
  };
  int best = 1;
  double best_eff = efficiency(1);
  if (best_eff < 0.97) {
    for (int s = 2; s <= max_s; ++s) {
      const double eff = efficiency(s);
      if (eff > best_eff + 1e-9) {
        best_eff = eff;
        best = s;
      }
    }
  }
  p.splits = best;
  p.units = p.tiles * best;
  int64_t tps = (n_tokens + best - 1) / best;
  p.tokens_per_split = (tps + BK - 1) / BK * BK;
  return p;
}

struct TcArgs {
  int d, nbi, tiles, splits, units;
  int64_t n_tokens, tokens_per_split;
  int chunk_stages;
  uint32_t idesc;
  float scale;
  int accumulate;
  float* H;
  float* partial;
  int32_t* status;
  long long test_wait;  // > 0: the failure-detection test (see gptq_test_hessian_timeout)
};

using namespace tc;

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// unit -> (tile row block bi, tile column block bj, split s)
__device__ __forceinline__ void unit_coords(int u, const TcArgs& a, int& bi, int& bj, int& s) {
  s = u / a.tiles;
  int t = u % a.tiles;
  int j = 0;
  for (;; ++j) {
    const int cnt = (2 * j + 2 < a.nbi) ? 2 * j + 2 : a.nbi;
    if (t < cnt) break;
    t -= cnt;
  }
  bi = t;
  bj = j;
}

__device__ __forceinline__ int unit_stages(int s, const TcArgs& a) {
  const int64_t t0 = (int64_t)s * a.tokens_per_split;
  int64_t t1 = t0 + a.tokens_per_split;
  if (t1 > a.n_tokens) t1 = a.n_tokens;
  if (t1 <= t0) return 0;
  return (int)((t1 - t0 + BK - 1) / BK);
}

__global__ void __launch_bounds__(THREADS, 1) hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                 const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
      uint32_t stage = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
        int bi, bj, s;
        unit_coords(u, a, bi, bj, s);
        const int n = unit_stages(s, a);
        const int64_t tok0 = (int64_t)s * a.tokens_per_split;
        for (int k = 0; k < n; ++k, ++stage) {
          const uint32_t slot = stage % STAGES, round = stage / STAGES;
          if (!mbar_wait(&empty[slot], (round & 1) ^ 1, abort_flag, a.status, 1)) {
            ok = false;
            break;
          }
          uint8_t* A = smem + slot * STAGE_BYTES;
          uint8_t* B = A + A_BYTES;
          const int y = (int)(tok0 + (int64_t)k * BK);
          mbar_expect_tx(&full[slot], STAGE_BYTES);
          tma_load_2d(A, &tmap, bi * BM, y, &full[slot]);
          tma_load_2d(A + CHUNK_BYTES, &tmap, bi * BM + 64, y, &full[slot]);
#pragma unroll
          for (int h = 0; h < 4; ++h) tma_load_2d(B + h * CHUNK_BYTES, &tmap, bj * BN + 64 * h, y, &full[slot]);
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA leaves
        const uint32_t first = stage > STAGES ? stage - STAGES : 0;
        for (uint32_t i = first; i < stage; ++i) mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t stage = 0, chunk = 0;
      bool ok = true;
      const uint32_t smem0 = smem_u32(smem);
      // failure-detection test only: wait, for at most test_wait cycles, on a barrier nothing arrives
      // on before this thread's own final commit, so the wait gives up and the timeout path runs
      if (a.test_wait > 0) ok = mbar_wait(drain, 0, abort_flag, a.status, 5, a.test_wait);
      for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
        int bi, bj, s;
        unit_coords(u, a, bi, bj, s);
        const int n = unit_stages(s, a);
        for (int k = 0; k < n && ok; ++chunk) {
          const uint32_t buf = chunk & 1, use = chunk >> 1;
          if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status, 2)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + buf * BN;
          const int in_chunk = (n - k < a.chunk_stages) ? n - k : a.chunk_stages;
          for (int c = 0; c < in_chunk; ++c, ++k, ++stage) {
            const uint32_t slot = stage % STAGES, round = stage / STAGES;
            if (!mbar_wait(&full[slot], round & 1, abort_flag, a.status, 3)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t A = smem0 + slot * STAGE_BYTES, B = A + A_BYTES;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              // 16 tokens = 2 swizzle atoms = 2048 bytes further along K
              const uint64_t ad = sdesc_sw128(A + kk * 2048, CHUNK_BYTES, 1024);
              const uint64_t bd = sdesc_sw128(B + kk * 2048, CHUNK_BYTES, 1024);
              umma_f16(d_tmem, ad, bd, a.idesc, (c > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&empty[slot]);
          }
          if (ok) umma_commit(&acc_full[buf]);
        }
      }
      // all MMAs issued by this thread are complete before TMEM is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2;
    const int quad = warp & 3;  // TMEM lanes this warp may access: 32*quad .. 32*quad+31
    const int half = ew >> 2;   // columns 128*half .. 128*half+127 of the tile
    const int r = 32 * quad + lane;
    uint32_t chunk = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < a.units && ok; u += gridDim.x) {
      int bi, bj, s;
      unit_coords(u, a, bi, bj, s);
      const int n = unit_stages(s, a);
      const int n_chunks = (n + a.chunk_stages - 1) / a.chunk_stages;
      float acc[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) acc[c] = 0.0f;
      for (int c = 0; c < n_chunks; ++c, ++chunk) {
        const uint32_t buf = chunk & 1, use = chunk >> 1;
        if (!mbar_wait(&acc_full[buf], use & 1, abort_flag, a.status, 4)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + buf * BN + 128 * half;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[32];
          tmem_ld32(taddr + 32 * q, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 * q + i] += v[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
      }
      if (!ok) break;
      if (a.splits == 1) {
        const int i = bi * BM + r;
        const int j0 = bj * BN + 128 * half;
        if (i < a.d) {
          float* row = a.H + (size_t)i * a.d;
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            const int j = j0 + c;
            if (j < a.d) {
              float4 v = make_float4(a.scale * acc[c], a.scale * acc[c + 1], a.scale * acc[c + 2],
                                     a.scale * acc[c + 3]);
              float4* dst = reinterpret_cast<float4*>(row + j);
              if (a.accumulate) {
                const float4 o = *dst;
                v.x += o.x;
                v.y += o.y;
                v.z += o.z;
                v.w += o.w;
              }
              *dst = v;
            }
          }
        }
      } else {
        const int t = u % a.tiles;
        float* dst = a.partial + (((size_t)s * a.tiles + t) * BM + r) * BN + 128 * half;
#pragma unroll
        for (int c = 0; c < 128; c += 4)
          *reinterpret_cast<float4*>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// H[tile] (+)= scale * sum over splits of the partial tiles, in split order.
__global__ void hessian_tc_reduce_kernel(const float* __restrict__ partial, int d, int nbi, int tiles, int splits,
                                         float scale, int accumulate, float* __restrict__ H) {
  const int t = blockIdx.y;
  int tt = t, bj = 0;
  for (;; ++bj) {
    const int cnt = (2 * bj + 2 < nbi) ? 2 * bj + 2 : nbi;
    if (tt < cnt) break;
    tt -= cnt;
  }
  const int bi = tt;
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= BM * BN) return;
  const int r = e / BN, c = e % BN;
  const int i = bi * BM + r, j = bj * BN + c;
  if (i >= d || j >= d) return;
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(partial + ((size_t)s * tiles + t) * (BM * BN) + e);
    sum.x += v.x;
    sum.y += v.y;
    sum.z += v.z;
    sum.w += v.w;
  }
  float4* dst = reinterpret_cast<float4*>(H + (size_t)i * d + j);
  float4 out = make_float4(scale * sum.x, scale * sum.y, scale * sum.z, scale * sum.w);
  if (accumulate) {
    const float4 o = *dst;
    out.x += o.x;
    out.y += o.y;
    out.z += o.z;
    out.w += o.w;
  }
  *dst = out;
}

// ------------------------------------------------------------------------------------------------
// CTA-pair form (orders >= 512).  The single-CTA kernel above is bound by shared-memory bandwidth:
// per 64-token stage its SM takes 48 KB of TMA writes and 48 KB of MMA operand reads for 128 x 256 x 64
// multiply-adds.  Here a cluster of two CTAs computes a 256 x 256 tile with tcgen05.mma.cta_group::2
// (M = 256, N = 256): each CTA holds 128 of the tile's rows of A and 128 of its columns of B, the even
// CTA's single MMA thread drives both tensor cores, and each SM moves 32 KB in and 32 KB out of shared
// memory per stage for the same 128 x 256 x 64 multiply-adds per SM.
//   warp 0      TMA producer of this CTA's halves (6-stage ring of 32 KB); both CTAs' copies of a stage
//               complete on the even CTA's stage barrier, which expects the bytes of both
//   warp 1      even CTA: MMA issuer
//   warps 2-9   epilogue of this CTA's 128 rows (TMEM of both CTAs is written by the pair's MMAs)
// Stage and accumulator releases come back to both CTAs through tcgen05.commit multicast; the odd
// CTA's epilogue releases an accumulator by arriving on the even CTA's acc_empty.  Both CTAs meet at a
// cluster barrier before TMEM is freed, so neither leaves while the pair's MMAs or copies may still
// touch the other CTA.
// Every mbarrier wait is bounded, as in the single-CTA kernel.
constexpr int P_HALF = PT / 2;
constexpr int P_STAGES = 7;
constexpr int P_STAGE_BYTES = 2 * P_HALF * BK * 2;  // A half + B half, 64 tokens: 32 KB

__device__ __forceinline__ void umma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// index of a triangle entry: t -> (i <= j), column-major (j-th column holds j + 1 entries)
__device__ __forceinline__ void tri_coords(int64_t t, int& i, int& j) {
  int jj = (int)((sqrt(8.0 * (double)t + 1.0) - 1.0) * 0.5);
  while ((int64_t)(jj + 1) * (jj + 2) / 2 <= t) ++jj;
  while ((int64_t)jj * (jj + 1) / 2 > t) --jj;
  j = jj;
  i = (int)(t - (int64_t)jj * (jj + 1) / 2);
}

// unit -> (tile row block bi <= tile column block bj, split s).  The upper block triangle is walked in
// patches of kPatch x kPatch tiles (patch columns left to right, patches top to bottom, tiles within a
// patch column by column), so the pairs that run at the same time share few 256-channel blocks of X:
// they stream the same token rows in step, and those rows come from L2 instead of HBM.
constexpr int kPatch = 8;

__device__ __forceinline__ int64_t patch_prefix(int J) {  // tiles in the first J (full-width) patch columns
  return (int64_t)kPatch * kPatch * J * (J - 1) / 2 + (int64_t)J * kPatch * (kPatch + 1) / 2;
}

__device__ __forceinline__ void pair_coords(int u, const TcArgs& a, int& bi, int& bj, int& s) {
  s = u / a.tiles;
  const int64_t t = u % a.tiles;
  const int nb = a.nbi;
  const int np = (nb + kPatch - 1) / kPatch;
  int lo = 0, hi = np - 1;  // the patch column J with patch_prefix(J) <= t < patch_prefix(J + 1)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (patch_prefix(mid) <= t) lo = mid; else hi = mid - 1;
  }
  const int J = lo;
  const int w = min(kPatch, nb - J * kPatch);  // width of patch column J (the last one may be narrower)
  const int64_t r = t - patch_prefix(J);
  if (r < (int64_t)J * kPatch * w) {  // an off-diagonal patch (I < J): kPatch x w tiles
    const int I = (int)(r / (kPatch * w));
    const int q = (int)(r % (kPatch * w));
    bi = I * kPatch + q % kPatch;
    bj = J * kPatch + q / kPatch;
  } else {  // the diagonal patch: its upper triangle
    int li, lj;
    tri_coords(r - (int64_t)J * kPatch * w, li, lj);
    bi = J * kPatch + li;
    bj = J * kPatch + lj;
  }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    hessian_pair_kernel(const __grid_constant__ CUtensorMap tmap, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  uint64_t* empty = full + P_STAGES;
  uint64_t* acc_full = empty + P_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0 leads the pair
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2 * EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) tmem_alloc_pair(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any arrival crosses the pair
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (this CTA's halves)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
      uint32_t stage = 0;
      bool ok = true;
      const uint32_t full0 = mapa_shared(full, 0);  // the even CTA's stage barriers
      for (int u = pair; u < a.units && ok; u += n_pairs) {
        int bi, bj, s;
        pair_coords(u, a, bi, bj, s);
        const int n = unit_stages(s, a);
        const int64_t tok0 = (int64_t)s * a.tokens_per_split;
        const int ra = bi * PT + P_HALF * (int)rank, rb = bj * PT + P_HALF * (int)rank;
        for (int k = 0; k < n; ++k, ++stage) {
          const uint32_t slot = stage % P_STAGES, round = stage / P_STAGES;
          if (!mbar_wait_cluster(&empty[slot], (round & 1) ^ 1, abort_flag, a.status, 21)) {
            ok = false;
            break;
          }
          uint8_t* A = smem + slot * P_STAGE_BYTES;
          uint8_t* B = A + P_HALF * BK * 2;
          const int y = (int)(tok0 + (int64_t)k * BK);
          const uint32_t bar = full0 + slot * 8;
          if (rank == 0) mbar_expect_tx(&full[slot], 2 * P_STAGE_BYTES);
          tma_load_2d_pair(A, &tmap, ra, y, bar);
          tma_load_2d_pair(A + CHUNK_BYTES, &tmap, ra + 64, y, bar);
          tma_load_2d_pair(B, &tmap, rb, y, bar);
          tma_load_2d_pair(B + CHUNK_BYTES, &tmap, rb + 64, y, bar);
        }
      }
      // let the copies already issued land before the CTA leaves: the even CTA watches them on its
      // stage barriers (its copies and the odd CTA's); the odd CTA cannot wait on those barriers, and
      // the cluster barrier at the end keeps it resident until the even CTA has drained
      if (!ok && rank == 0) {
        const uint32_t first = stage > P_STAGES ? stage - P_STAGES : 0;
        for (uint32_t i = first; i < stage; ++i) mbar_wait_drain_cluster(&full[i % P_STAGES], (i / P_STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // -------------------------------------------------------------- MMA issuer (even CTA)
      uint32_t stage = 0, chunk = 0;
      bool ok = a.test_wait > 0 ? mbar_wait(drain, 0, abort_flag, a.status, 5, a.test_wait) : true;
      const uint64_t adesc0 = sdesc_sw128(smem_u32(smem), CHUNK_BYTES, 1024);
      for (int u = pair; u < a.units && ok; u += n_pairs) {
        int bi, bj, s;
        pair_coords(u, a, bi, bj, s);
        const int n = unit_stages(s, a);
        for (int k = 0; k < n && ok; ++chunk) {
          const uint32_t buf = chunk & 1, use = chunk >> 1;
          if (!mbar_wait_cluster(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status, 22)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + buf * PT;
          const int in_chunk = (n - k < a.chunk_stages) ? n - k : a.chunk_stages;
          for (int c = 0; c < in_chunk; ++c, ++k, ++stage) {
            const uint32_t slot = stage % P_STAGES, round = stage / P_STAGES;
            if (!mbar_wait_cluster(&full[slot], round & 1, abort_flag, a.status, 23)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // descriptors of this slot: the start-address field (address / 16, 14 bits) of the slot-0
            // descriptors plus the offset; shared-memory offsets stay below 256 KB, so no carry leaves it
            const uint64_t ad0 = adesc0 + (uint64_t)((slot * P_STAGE_BYTES) >> 4);
            const uint64_t bd0 = ad0 + (uint64_t)((P_HALF * BK * 2) >> 4);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma_f16_pair(d_tmem, ad0 + (uint64_t)(kk * (2048 >> 4)), bd0 + (uint64_t)(kk * (2048 >> 4)), a.idesc,
                            (c > 0 || kk > 0) ? 1u : 0u);
            umma_commit_pair(&empty[slot]);
          }
          if (ok) umma_commit_pair(&acc_full[buf]);
        }
      }
      // every MMA of the pair is complete before either CTA frees TMEM or leaves
      umma_commit_pair(drain);
      mbar_wait_drain(drain, 0);
    } else if (lane == 0) {
      // odd CTA: the pair's last MMAs are complete before this CTA frees TMEM
      mbar_wait_drain_cluster(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (this CTA's rows)
    const int ew = warp - 2;
    const int quad = warp & 3;
    const int half = ew >> 2;  // columns 128*half .. 128*half+127 of the tile
    const int r = 32 * quad + lane;
    const uint32_t acc_empty0 = mapa_shared(acc_empty, 0);
    uint32_t chunk = 0;
    bool ok = true;
    for (int u = pair; u < a.units && ok; u += n_pairs) {
      int bi, bj, s;
      pair_coords(u, a, bi, bj, s);
      const int n = unit_stages(s, a);
      const int n_chunks = (n + a.chunk_stages - 1) / a.chunk_stages;
      float acc[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) acc[c] = 0.0f;
      for (int c = 0; c < n_chunks; ++c, ++chunk) {
        const uint32_t buf = chunk & 1, use = chunk >> 1;
        if (!mbar_wait_cluster(&acc_full[buf], use & 1, abort_flag, a.status, 26)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + buf * PT + 128 * half;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float v[32];
          tmem_ld32(taddr + 32 * q, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[32 * q + i] += v[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc_empty0 + buf * 8);
      }
      if (!ok) break;
      const int i = bi * PT + P_HALF * (int)rank + r;
      const int j0 = bj * PT + 128 * half;
      if (a.splits == 1) {
        if (i < a.d) {
          float* row = a.H + (size_t)i * a.d;
#pragma unroll
          for (int c = 0; c < 128; c += 4) {
            const int j = j0 + c;
            if (j < a.d) {
              float4 v = make_float4(a.scale * acc[c], a.scale * acc[c + 1], a.scale * acc[c + 2],
                                     a.scale * acc[c + 3]);
              float4* dst = reinterpret_cast<float4*>(row + j);
              if (a.accumulate) {
                const float4 o = *dst;
                v.x += o.x;
                v.y += o.y;
                v.z += o.z;
                v.w += o.w;
              }
              *dst = v;
            }
          }
        }
      } else {
        const int t = u % a.tiles;
        float* dst = a.partial + (((size_t)s * a.tiles + t) * PT + P_HALF * rank + r) * PT + 128 * half;
#pragma unroll
        for (int c = 0; c < 128; c += 4)
          *reinterpret_cast<float4*>(dst + c) = make_float4(acc[c], acc[c + 1], acc[c + 2], acc[c + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the pair's MMAs are done and no arrival is on its way to the other CTA
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// H[tile] (+)= scale * sum over splits of the pair kernel's 256 x 256 partial tiles, in split order.
__global__ void hessian_pair_reduce_kernel(const float* __restrict__ partial, int d, int nb, int tiles, int splits,
                                           float scale, int accumulate, float* __restrict__ H) {
  const int t = blockIdx.y;
  TcArgs tiles_of;
  tiles_of.tiles = tiles;
  tiles_of.nbi = nb;
  int bi, bj, s;
  pair_coords(t, tiles_of, bi, bj, s);
  const int e = (blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= PT * PT) return;
  const int r = e / PT, c = e % PT;
  const int i = bi * PT + r, jj = bj * PT + c;
  if (i >= d || jj >= d) return;
  float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < splits; ++s) {
    const float4 v = *reinterpret_cast<const float4*>(partial + ((size_t)s * tiles + t) * (PT * PT) + e);
    sum.x += v.x;
    sum.y += v.y;
    sum.z += v.z;
    sum.w += v.w;
  }
  float4* dst = reinterpret_cast<float4*>(H + (size_t)i * d + jj);
  float4 out = make_float4(scale * sum.x, scale * sum.y, scale * sum.z, scale * sum.w);
  if (accumulate) {
    const float4 o = *dst;
    out.x += o.x;
    out.y += o.y;
    out.z += o.z;
    out.w += o.w;
  }
  *dst = out;
}

constexpr int kPairSmemBytes = P_STAGES * P_STAGE_BYTES + 1024 + 512;

// Clusters of two that can be resident at once (cached per device).
int pair_slots(int dev, int sms) {
  static std::atomic<int> cached[64];
  if (dev < 0 || dev >= 64) return 0;
  int v = cached[dev].load();
  if (v > 0) return v;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sms);
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = kPairSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, hessian_pair_kernel, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 0;
  }
  cached[dev].store(n);
  return n;
}

constexpr int kSmemBytes = STAGES * STAGE_BYTES + 1024 + 256;

// One-shot request of the failure-detection test (gptq_test_hessian_timeout), taken by the next launch.
std::atomic<long long> g_test_wait{0};

}  // namespace

bool hessian_tc_supported(int64_t n_tokens, int64_t d, int32_t x_dtype) {
  return (x_dtype == GPTQ_BF16 || x_dtype == GPTQ_FP16) && d >= 256 && d % 8 == 0 && n_tokens >= BK &&
         n_tokens < (int64_t(1) << 31);
}

size_t hessian_tc_workspace(int64_t n_tokens, int64_t d) {
  TcPlan p = tc_plan(n_tokens, d);
  const size_t tile = use_pair(d) ? (size_t)PT * PT : (size_t)BM * BN;
  return p.splits > 1 ? (size_t)p.splits * p.tiles * tile * sizeof(float) : 0;
}

int hessian_tc_launches(int64_t n_tokens, int64_t d) { return tc_plan(n_tokens, d).splits > 1 ? 2 : 1; }

gptq_status hessian_tc_launch(const void* X, int32_t x_dtype, int64_t n_tokens, int64_t d, float* H, float scale,
                              int32_t accumulate, int32_t* status, void* workspace, cudaStream_t stream) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tc::encode_fn();
  if (encode == nullptr) return GPTQ_ERR_CUDA;
  TcPlan p = tc_plan(n_tokens, d);
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)n_tokens};
  const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)BK};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType dt =
      x_dtype == GPTQ_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  if (encode(&map, dt, 2, const_cast<void*>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GPTQ_ERR_ARG;
  int dev = 0, sms = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes));
  TcArgs a;
  a.d = (int)d;
  a.nbi = p.nbi;
  a.tiles = p.tiles;
  a.splits = p.splits;
  a.units = p.units;
  a.n_tokens = n_tokens;
  a.tokens_per_split = p.tokens_per_split;
  a.chunk_stages = kChunkTokens / BK;
  const uint32_t fmt = x_dtype == GPTQ_BF16 ? 1u : 0u;
  // kind::f16 instruction descriptor: D f32, A/B bf16 or f16, both MN-major, N = 256, M = 128
  a.idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(BN >> 3) << 17) |
            ((uint32_t)(BM >> 4) << 24);
  a.scale = scale;
  a.accumulate = accumulate;
  a.H = H;
  a.partial = static_cast<float*>(workspace);
  a.status = status;
  a.test_wait = g_test_wait.exchange(0);
  if (use_pair(d)) {
    // M = 256 (two CTAs), N = 256; both operands MN-major
    a.idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(PT >> 3) << 17) |
              ((uint32_t)(PT >> 4) << 24);
    GPTQ_CUDA_TRY(cudaFuncSetAttribute(hessian_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kPairSmemBytes));
    // the kernel is persistent: launch no more pairs than can be resident at once (clusters are placed
    // within a GPC, so fewer than sms / 2 may fit), or the extra pairs would run as a second wave
    const int resident = pair_slots(dev, sms);
    if (resident < 1) return GPTQ_ERR_CUDA;
    const int pairs = p.units < resident ? p.units : resident;
    hessian_pair_kernel<<<2 * pairs, THREADS, kPairSmemBytes, stream>>>(map, a);
    GPTQ_LAUNCH_CHECK();
    if (p.splits > 1) {
      dim3 g((PT * PT / 4 + 255) / 256, p.tiles);
      hessian_pair_reduce_kernel<<<g, 256, 0, stream>>>(a.partial, a.d, p.nbi, p.tiles, p.splits, scale, accumulate,
                                                        H);
      GPTQ_LAUNCH_CHECK();
    }
    return GPTQ_OK;
  }
  const int grid = p.units < sms ? p.units : sms;
  hessian_tc_kernel<<<grid, THREADS, kSmemBytes, stream>>>(map, a);
  GPTQ_LAUNCH_CHECK();
  if (p.splits > 1) {
    dim3 g((BM * BN / 4 + 255) / 256, p.tiles);
    hessian_tc_reduce_kernel<<<g, 256, 0, stream>>>(a.partial, a.d, p.nbi, p.tiles, p.splits, scale, accumulate, H);
    GPTQ_LAUNCH_CHECK();
  }
  return GPTQ_OK;
}

}  // namespace gptq

extern "C" void gptq_test_hessian_timeout(int64_t cycles) { gptq::g_test_wait.store(cycles > 0 ? cycles : 0); }
