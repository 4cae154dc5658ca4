// fp32-accurate products C -= A B^T on CTA pairs (3xTF32 with tcgen05.mma.cta_group::2).
//
// The two dense block products of the path: the trailing update of the blocked Cholesky in the
// prepare step, P(r, c) -= L(r, p) L(c, p)^T, and the lazy block update of the column loop (FDE
// Interviews breakdown of GPTQ, figure "THE IDEA, VISUALLY" step 4), W[:, i2:] -= Err U[i1:i2, i2:].
//
// The single-CTA form (gemm_tf32x3.cu) splits each landed fp32 tile into tf32 hi and lo in shared
// memory and reads both operands three times per k-step; per 128 x 128 x 32 stage that is about
// 224 KB of shared-memory traffic against 96 KB of MMA reads, so it runs at about half the tensor
// rate.  Here:
//   - the operands are split once in global memory (split_rows_kernel, split_transpose_kernel): hi =
//     tf32(x) rounded to nearest, lo = tf32(x - hi), both K-major, so the kernel is TMA -> MMA only;
//   - a pair of SMs computes a 256 x 256 tile: each CTA loads 128 rows of A (hi and lo) and 128 rows of
//     B (hi and lo); the even CTA's thread issues M = 256, N = 256, K = 8 kind::tf32 MMAs, three per
//     k-step (lo_a hi_b, hi_a lo_b, hi_a hi_b, accumulated in fp32 in TMEM as in the single-CTA form).
// Per SM and 32-deep stage: 64 KB of TMA writes and 96 KB of MMA reads for twice the products of a
// single-CTA stage.
//
// Warps: 0 TMA producer (both CTAs; their copies complete on the even CTA's stage barrier), 1 MMA
// issuer (even CTA), 2-5 epilogue (both CTAs: TMEM -> registers -> 32 x 32 staging tiles -> TMA
// reduce-add of -A B^T into C).  Stage and accumulator releases return to both CTAs by multicast
// commits; the odd CTA's epilogue releases an accumulator on the even CTA's barrier; a cluster
// barrier precedes the paired TMEM free.  Every mbarrier wait is bounded.
#include <mutex>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

using namespace tc;

constexpr int PT = 256;            // output tile of a pair
constexpr int HALF = 128;          // rows of A and of B per CTA
constexpr int TK = 32;             // K per stage (one 128-byte row of fp32)
constexpr int STAGES = 3;
constexpr int OPND = HALF * TK * 4;  // 16 KB
constexpr int STAGE_BYTES = 4 * OPND;  // A hi, A lo, B hi, B lo
constexpr int EPI_WARPS = 4;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int STG = 32 * 32 * 4;
constexpr int kSmemBytes = STAGES * STAGE_BYTES + EPI_WARPS * 2 * STG + 1024 + 256;
constexpr uint32_t TMEM_COLS = 2 * PT;

struct Maps {
  CUtensorMap a_hi, a_lo, b_hi, b_lo, out;
};

// output tile t -> first A row and first B row of the pair's 256, output origin
__device__ __forceinline__ void tile_of(int t, const PairGemmArgs& g, int& a_row, int& b_row, int& oy, int& ox) {
  if (g.kind == kPairLazy) {
    const int tm = t / g.tiles_n, tn = t % g.tiles_n;
    a_row = tm * PT;
    b_row = tn * PT;
    oy = g.out_y0 + tm * PT;
    ox = g.out_x0 + tn * PT;
  } else {  // syrk: super-blocks (R, C), C < super_c, C <= R < super_r, column by column
    int lo = 0, hi = g.super_c - 1;  // the column C with prefix(C) <= t < prefix(C + 1)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)mid * g.super_r - (int64_t)mid * (mid - 1) / 2 <= t) lo = mid; else hi = mid - 1;
    }
    const int C = lo;
    const int R = C + (int)(t - ((int64_t)C * g.super_r - (int64_t)C * (C - 1) / 2));
    a_row = g.row0 + R * PT;
    b_row = g.row0 + C * PT;
    oy = g.out_y0 + R * PT;
    ox = g.out_x0 + C * PT;
  }
}

__device__ __forceinline__ void umma_tf32_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    tf32x3_pair_kernel(const __grid_constant__ Maps m, const PairGemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + EPI_WARPS * 2 * STG);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
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
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (this CTA's halves)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&m.a_hi)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&m.b_hi)) : "memory");
      uint32_t stage = 0;
      bool ok = true;
      const uint32_t full0 = mapa_shared(full, 0);
      for (int t = pair; t < g.tiles && ok; t += n_pairs) {
        int a_row, b_row, oy, ox;
        tile_of(t, g, a_row, b_row, oy, ox);
        a_row += HALF * (int)rank;
        b_row += HALF * (int)rank;
        for (int ks = 0; ks < g.nk; ++ks, ++stage) {
          const uint32_t slot = stage % STAGES, round = stage / STAGES;
          if (!mbar_wait_cluster(&empty[slot], (round & 1) ^ 1, abort_flag, g.status, 31)) {
            ok = false;
            break;
          }
          uint8_t* S = smem + slot * STAGE_BYTES;
          const uint32_t bar = full0 + slot * 8;
          if (rank == 0) mbar_expect_tx(&full[slot], 2 * STAGE_BYTES);
          tma_load_2d_pair(S, &m.a_hi, TK * ks, a_row, bar);
          tma_load_2d_pair(S + OPND, &m.a_lo, TK * ks, a_row, bar);
          tma_load_2d_pair(S + 2 * OPND, &m.b_hi, TK * ks, b_row, bar);
          tma_load_2d_pair(S + 3 * OPND, &m.b_lo, TK * ks, b_row, bar);
        }
      }
      if (!ok && rank == 0) {
        const uint32_t first = stage > STAGES ? stage - STAGES : 0;
        for (uint32_t i = first; i < stage; ++i) mbar_wait_drain_cluster(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // -------------------------------------------------------------- MMA issuer (even CTA)
      uint32_t stage = 0, tcount = 0;
      bool ok = true;
      const uint64_t d0 = sdesc_sw128(smem_u32(smem), 16, 1024);  // K-major, 128-byte rows
      for (int t = pair; t < g.tiles && ok; t += n_pairs) {
        const uint32_t buf = tcount & 1, use = tcount >> 1;
        if (!mbar_wait_cluster(&acc_empty[buf], (use & 1) ^ 1, abort_flag, g.status, 32)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * PT;
        for (int ks = 0; ks < g.nk; ++ks, ++stage) {
          const uint32_t slot = stage % STAGES, round = stage / STAGES;
          if (!mbar_wait_cluster(&full[slot], round & 1, abort_flag, g.status, 33)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors: start-address field (address / 16) of the stage's operands plus the offset
          // of k-step kk (8 fp32 = 32 bytes along the swizzled 128-byte row)
          const uint64_t ah = d0 + (uint64_t)((slot * STAGE_BYTES) >> 4);
          const uint64_t al = ah + (uint64_t)(OPND >> 4), bh = ah + (uint64_t)((2 * OPND) >> 4),
                         bl = ah + (uint64_t)((3 * OPND) >> 4);
#pragma unroll
          for (int kk = 0; kk < TK / 8; ++kk) {
            const uint64_t o = (uint64_t)kk * 2;  // 32 bytes
            umma_tf32_pair(d_tmem, al + o, bh + o, g.idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            umma_tf32_pair(d_tmem, ah + o, bl + o, g.idesc, 1u);
            umma_tf32_pair(d_tmem, ah + o, bh + o, g.idesc, 1u);
          }
          umma_commit_pair(&empty[slot]);
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[buf]);
        ++tcount;
      }
      umma_commit_pair(drain);
      mbar_wait_drain(drain, 0);
    } else if (lane == 0) {
      mbar_wait_drain_cluster(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue (this CTA's 128 rows)
    const int ew = warp - 2;
    const int quad = warp & 3;
    uint8_t* stg = staging + ew * 2 * STG;
    const uint32_t acc_empty0 = mapa_shared(acc_empty, 0);
    uint32_t tcount = 0, sb = 0;
    bool ok = true;
    for (int t = pair; t < g.tiles && ok; t += n_pairs) {
      int a_row, b_row, oy, ox;
      tile_of(t, g, a_row, b_row, oy, ox);
      const uint32_t buf = tcount & 1, use = tcount >> 1;
      if (!mbar_wait_cluster(&acc_full[buf], use & 1, abort_flag, g.status, 34)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + buf * PT;
      const int y = oy + HALF * (int)rank + 32 * quad;
#pragma unroll 1
      for (int ch = 0; ch < PT / 32; ++ch) {
        const int x = ox + 32 * ch;
        // syrk: only blocks on or below the diagonal, and not the look-ahead's diagonal block
        bool keep = x < g.o_w && y < g.o_h;
        if (g.kind == kPairSyrk) {
          const int rb = (y - g.out_y0) / HALF, cb = (x - g.out_x0) / HALF;  // 128-blocks of the region
          keep = keep && cb <= rb && cb < g.cols_blk && !(g.skip_diag && rb == 0 && cb == 0);
        }
        float v[32];
        tmem_ld32(taddr + 32 * ch, v);
        if (!keep) continue;  // (warp-uniform: x and y are the same for the whole warp)
        uint8_t* buf_s = stg + sb * STG;
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<float4*>(buf_s + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_float4(-v[4 * c], -v[4 * c + 1], -v[4 * c + 2], -v[4 * c + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_reduce_add_2d(&m.out, x, y, buf_s);
          bulk_commit();
        }
        sb ^= 1;  // the next kept chunk stages into the other buffer
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + buf * 8);
      ++tcount;
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

// hi[r * dld + k], lo[r * dld + k] of src[r * ld + k], k < 128 (rows of a 128-wide panel)
__global__ void __launch_bounds__(256) split_rows_kernel(const float* __restrict__ src, int64_t ld, int rows,
                                                         float* __restrict__ hi, float* __restrict__ lo,
                                                         int64_t dld) {
  const int64_t n = (int64_t)rows * (HALF / 4);
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = e / (HALF / 4);
    const int c = (int)(e % (HALF / 4)) * 4;
    const float4 x = *reinterpret_cast<const float4*>(src + r * ld + c);
    float4 h, l;
    h.x = tf32_rn(x.x), h.y = tf32_rn(x.y), h.z = tf32_rn(x.z), h.w = tf32_rn(x.w);
    l.x = tf32_rn(x.x - h.x), l.y = tf32_rn(x.y - h.y), l.z = tf32_rn(x.z - h.z), l.w = tf32_rn(x.w - h.w);
    *reinterpret_cast<float4*>(hi + r * dld + c) = h;
    *reinterpret_cast<float4*>(lo + r * dld + c) = l;
  }
}

// hi[n][k], lo[n][k] of src[k * ld + n], k < k_rows, n < cols: a panel of k_rows rows transposed to
// K-major ([cols, k_rows], k_rows a multiple of 32)
__global__ void __launch_bounds__(256) split_transpose_kernel(const float* __restrict__ src, int64_t ld, int cols,
                                                              int k_rows, float* __restrict__ hi,
                                                              float* __restrict__ lo) {
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  const int n_nb = (cols + 31) / 32, n_kb = k_rows / 32;
  for (int64_t w = blockIdx.x; w < (int64_t)n_nb * n_kb; w += gridDim.x) {
    const int nb = (int)(w / n_kb), kb = (int)(w % n_kb) * 32;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      const int k = kb + ty + j, n = nb * 32 + tx;
      tile[ty + j][tx] = (n < cols) ? src[(int64_t)k * ld + n] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 32; j += 8) {
      const int n = nb * 32 + ty + j, k = kb + tx;
      if (n < cols) {
        const float x = tile[tx][ty + j];
        const float h = tf32_rn(x);
        hi[(int64_t)n * k_rows + k] = h;
        lo[(int64_t)n * k_rows + k] = tf32_rn(x - h);
      }
    }
  }
}

std::mutex g_pair_mu;
int g_pair_slots[64] = {};

int pair_slots(int dev) {
  std::lock_guard<std::mutex> lock(g_pair_mu);
  if (dev < 0 || dev >= 64) return 0;
  if (g_pair_slots[dev] == 0) {
    if (cudaFuncSetAttribute(tf32x3_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) !=
        cudaSuccess)
      return 0;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)sms);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = kSmemBytes;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tf32x3_pair_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      return 0;
    }
    g_pair_slots[dev] = n;
  }
  return g_pair_slots[dev];
}

}  // namespace

bool split_map(CUtensorMap* map, const float* base, int64_t rows, int64_t cols, int64_t ld) {
  // [rows, cols] fp32 K-major operand: boxes of 32 k x 128 rows, 128-byte swizzle
  return tf32x3_map(map, base, rows, cols, ld, HALF);
}

gptq_status split_rows_launch(const float* src, int64_t ld, int64_t rows, float* hi, float* lo, int64_t dld,
                              cudaStream_t s) {
  if (rows <= 0) return GPTQ_OK;
  const int64_t n = rows * (HALF / 4);
  const int blocks = (int)std::min<int64_t>((n + 255) / 256, 148 * 16);
  split_rows_kernel<<<blocks, 256, 0, s>>>(src, ld, (int)rows, hi, lo, dld);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

gptq_status split_transpose_launch(const float* src, int64_t ld, int64_t cols, int k_rows, float* hi, float* lo,
                                   cudaStream_t s) {
  if (cols <= 0) return GPTQ_OK;
  const int64_t work = ((cols + 31) / 32) * (k_rows / 32);
  const int blocks = (int)std::min<int64_t>(work, 148 * 8);
  split_transpose_kernel<<<blocks, 256, 0, s>>>(src, ld, (int)cols, k_rows, hi, lo);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

gptq_status tf32x3_pair_launch(const CUtensorMap& a_hi, const CUtensorMap& a_lo, const CUtensorMap& b_hi,
                               const CUtensorMap& b_lo, const CUtensorMap& out, PairGemmArgs g, cudaStream_t s,
                               int reserve_pairs) {
  if (g.tiles <= 0) return GPTQ_OK;
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  int slots = pair_slots(dev);
  if (slots < 1) return GPTQ_ERR_CUDA;
  slots -= reserve_pairs;
  if (slots < 1) slots = 1;
  // kind::tf32 instruction descriptor: D f32, A/B tf32, both K-major, N = 256, M = 256 (two CTAs)
  g.idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(PT >> 3) << 17) | ((uint32_t)(PT >> 4) << 24);
  Maps m{a_hi, a_lo, b_hi, b_lo, out};
  const int pairs = g.tiles < slots ? g.tiles : slots;
  tf32x3_pair_kernel<<<2 * pairs, THREADS, kSmemBytes, s>>>(m, g);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
