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

TcPlan tc_plan(int64_t n_tokens, int64_t d) {
  TcPlan p;
  p.nbi = (int)((d + BM - 1) / BM);
  p.nbj = (int)((d + BN - 1) / BN);
  p.tiles = tiles_for(p.nbi, p.nbj);
  int64_t max_s = n_tokens / kMinTokensPerSplit;
  if (max_s < 1) max_s = 1;
  if (max_s > 16) max_s = 16;
  int best = 1;
  double best_eff = -1.0;
  for (int s = 1; s <= max_s; ++s) {
    const int units = p.tiles * s;
    const int waves = (units + kPlanSMs - 1) / kPlanSMs;
    const double eff = (double)units / ((double)waves * kPlanSMs);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = s;
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
  return p.splits > 1 ? (size_t)p.splits * p.tiles * BM * BN * sizeof(float) : 0;
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
