// fp32-accurate block products on the 5th-generation tensor cores (3xTF32).
//
// The prepare step's blocked Cholesky and triangular inverse, and the column loop's lazy block
// update (FDE Interviews breakdown of GPTQ, figure "THE IDEA, VISUALLY" step 4: the trailing columns
// are updated once per 128-column block), are dense fp32 products of 128 x 128 tiles.  tcgen05.mma
// has no fp32 operand kind; kind::tf32 reads 10 explicit mantissa bits.  Each operand x is split into
// hi = tf32(x) (round to nearest) and lo = tf32(x - hi), and a*b is accumulated as
// lo_a*hi_b + hi_a*lo_b + hi_a*hi_b in fp32 in TMEM; the dropped lo*lo term and the rounding of lo
// are each below 2^-22 |a b|, so a product keeps about the accuracy of an fp32 FMA.
//
// Persistent kernel, one CTA per SM, one 128 x 128 output tile per work unit, K in stages of 32:
//   warp 0      TMA producer: A box 128 rows x 32 k (K-major); B box 128 x 32 (K-major) or four
//               32 n x 32 k boxes (MN-major, 128-byte swizzle with 32-byte granules); 3-stage ring
//   warp 1      TMEM owner (256 columns: two 128-column accumulators) and tcgen05.mma issuer: per
//               stage 4 k-steps of K = 8, three MMAs each
//   warps 2-5   converters: split the landed fp32 tiles into hi (in place) and lo (second buffer)
//   warps 6-9   epilogue: TMEM -> registers -> per-warp 32 x 32 staging tile -> TMA store, TMA
//               reduce-add (C -= A B is C += (-A B)), or a transposed TMA store
// Every mbarrier wait is bounded: on a timeout the kernel records GPTQ_ERR_TIMEOUT, lets the other
// roles leave, waits (bounded) for its own copies and MMAs in flight, frees TMEM and returns.
#include <mutex>

#include "kernels.h"
#include "tc_common.cuh"

namespace gptq {
namespace {

using namespace tc;

constexpr int TM = 128, TN = 128, TK = 32;
constexpr int STAGES = 3;
constexpr int OPND = TM * TK * 4;  // 16 KB: one operand tile of one stage
constexpr int STAGE_BYTES = 4 * OPND;  // A hi, B hi, A lo, B lo
constexpr int CONV_WARPS = 4, EPI_WARPS = 4;
constexpr int THREADS = 32 * (2 + CONV_WARPS + EPI_WARPS);
constexpr int STG = 32 * 32 * 4;  // one 32 x 32 staging tile
constexpr int kSmemBytes = STAGES * STAGE_BYTES + EPI_WARPS * 2 * STG + 1024 + 256;
constexpr uint32_t TMEM_COLS = 2 * TN;

struct Job {
  int ax, ay;  // A box origin (x = k, y = rows)
  int bx, by;  // B box origin (K-major: x = k, y = n; MN-major: x = n, y = k)
  int nk;      // K stages
  int ox, oy;  // output tile origin in the output map (transposed store: x runs along the tile's rows)
};

__device__ __forceinline__ bool job_of(int t, const Tf32x3Args& a, Job& j) {
  switch (a.kind) {
    case kGemmTrsm: {  // L(r, p) = P(r, p) L(p,p)^-T, r = p+1+t
      const int ri = a.p + 1 + t;
      j = {a.p * TM, ri * TM, 0, a.p * TM, TM / TK, a.p * TM, ri * TM};
      return true;
    }
    case kGemmSyrk: {  // P(r, c) -= L(r, p) L(c, p)^T, p < c <= r, lower-triangle order
      const int bid = t + a.skip;
      int rr = (int)((sqrt(8.0 * (double)bid + 1.0) - 1.0) * 0.5);
      while ((rr + 1) * (rr + 2) / 2 <= bid) ++rr;
      while (rr * (rr + 1) / 2 > bid) --rr;
      const int ri = a.p + 1 + rr, ci = a.p + 1 + (bid - rr * (rr + 1) / 2);
      j = {a.p * TM, ri * TM, a.p * TM, ci * TM, TM / TK, ci * TM, ri * TM};
      return true;
    }
    case kGemmTrtriT:
    case kGemmTrtriY: {  // pairs [[A, 0], [C, B]] of g blocks: T = C A^-1 (parked transposed), Y = -B^-1 T
      const int per_pair = a.g * a.g;
      const int q = t / per_pair, u = t % per_pair;
      const int a0 = q * 2 * a.g, b0 = a0 + a.g, b1 = min(a0 + 2 * a.g, a.D);
      const int ri = b0 + u / a.g, ci = a0 + u % a.g;
      if (ri >= b1) return false;
      if (a.kind == kGemmTrtriT)  // sum over k in [c, b0) of P(r, k) P(k, c); store into P(c, r) transposed
        j = {ci * TM, ri * TM, ci * TM, ci * TM, (b0 - ci) * (TM / TK), ri * TM, ci * TM};
      else  // sum over k in [b0, r] of P(r, k) T(k, c) with T(k, c) = P(c, k)^T
        j = {b0 * TM, ri * TM, b0 * TM, ci * TM, (ri + 1 - b0) * (TM / TK), ci * TM, ri * TM};
      return true;
    }
    default: {  // lazy update: W[r, c] -= Err[r, :] U[i1:i1+K, c], c >= i2
      const int tr = t / a.tiles_n, tcn = t % a.tiles_n;
      const int c0 = a.i2 + tcn * TN;
      j = {0, tr * TM, c0, a.i1, a.k / TK, c0, tr * TM};
      return true;
    }
  }
}

__device__ __forceinline__ void umma_tf32(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ float tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return __uint_as_float(r);
}

__global__ void __launch_bounds__(THREADS, 1)
    tf32x3_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                       const __grid_constant__ CUtensorMap mapO, const Tf32x3Args a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + EPI_WARPS * 2 * STG);
  uint64_t* conv = full + STAGES;
  uint64_t* empty = conv + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&conv[s], CONV_WARPS * 32);
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
  if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapA)) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&mapB)) : "memory");
      uint32_t stage = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < a.tiles && ok; t += gridDim.x) {
        Job j;
        if (!job_of(t, a, j)) continue;
        for (int ks = 0; ks < j.nk; ++ks, ++stage) {
          const uint32_t slot = stage % STAGES, round = stage / STAGES;
          if (!mbar_wait(&empty[slot], (round & 1) ^ 1, abort_flag, a.status, 11)) {
            ok = false;
            break;
          }
          uint8_t* A = smem + slot * STAGE_BYTES;
          uint8_t* B = A + OPND;
          mbar_expect_tx(&full[slot], 2 * OPND);
          tma_load_2d(A, &mapA, j.ax + TK * ks, j.ay, &full[slot]);
          if (a.b_mn) {
#pragma unroll
            for (int h = 0; h < TN / 32; ++h) tma_load_2d(B + h * 4096, &mapB, j.bx + 32 * h, j.by + TK * ks, &full[slot]);
          } else {
            tma_load_2d(B, &mapB, j.bx + TK * ks, j.by, &full[slot]);
          }
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
      uint32_t stage = 0, tcount = 0;
      bool ok = true;
      const uint32_t smem0 = smem_u32(smem);
      for (int t = blockIdx.x; t < a.tiles && ok; t += gridDim.x) {
        Job j;
        if (!job_of(t, a, j)) continue;
        const uint32_t buf = tcount & 1, use = tcount >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag, a.status, 12)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * TN;
        for (int ks = 0; ks < j.nk; ++ks, ++stage) {
          const uint32_t slot = stage % STAGES, round = stage / STAGES;
          if (!mbar_wait(&conv[slot], round & 1, abort_flag, a.status, 13)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t Ahi = smem0 + slot * STAGE_BYTES, Bhi = Ahi + OPND, Alo = Ahi + 2 * OPND, Blo = Ahi + 3 * OPND;
#pragma unroll
          for (int kk = 0; kk < TK / 8; ++kk) {
            // K-major: 8 k = 32 bytes further along the 128-byte row; MN-major: 8 rows of 128 bytes
            const uint64_t ah = sdesc_sw128(Ahi + kk * 32, 16, 1024), al = sdesc_sw128(Alo + kk * 32, 16, 1024);
            const uint64_t bh =
                a.b_mn ? sdesc_sw128_32b(Bhi + kk * 1024, 4096, 512) : sdesc_sw128(Bhi + kk * 32, 16, 1024);
            const uint64_t bl =
                a.b_mn ? sdesc_sw128_32b(Blo + kk * 1024, 4096, 512) : sdesc_sw128(Blo + kk * 32, 16, 1024);
            umma_tf32(d_tmem, al, bh, a.idesc, (ks > 0 || kk > 0) ? 1u : 0u);
            umma_tf32(d_tmem, ah, bl, a.idesc, 1u);
            umma_tf32(d_tmem, ah, bh, a.idesc, 1u);
          }
          umma_commit(&empty[slot]);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
        ++tcount;
      }
      // all MMAs issued by this thread are complete before TMEM is released
      umma_commit(drain);
      mbar_wait_drain(drain, 0);
    }
    __syncwarp();
  } else if (warp < 2 + CONV_WARPS) {
    // ---------------------------------------------------------------- hi / lo split
    const int ct = threadIdx.x - 64;
    uint32_t stage = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < a.tiles && ok; t += gridDim.x) {
      Job j;
      if (!job_of(t, a, j)) continue;
      for (int ks = 0; ks < j.nk; ++ks, ++stage) {
        const uint32_t slot = stage % STAGES, round = stage / STAGES;
        if (!mbar_wait(&full[slot], round & 1, abort_flag, a.status, 14)) {
          ok = false;
          break;
        }
        float4* hi = reinterpret_cast<float4*>(smem + slot * STAGE_BYTES);  // A then B, 2 x 16 KB
        float4* lo = hi + 2 * OPND / 16;
#pragma unroll 4
        for (int i = ct; i < 2 * OPND / 16; i += CONV_WARPS * 32) {
          const float4 x = hi[i];
          float4 h, l;
          h.x = tf32_rn(x.x);
          h.y = tf32_rn(x.y);
          h.z = tf32_rn(x.z);
          h.w = tf32_rn(x.w);
          l.x = tf32_rn(x.x - h.x);
          l.y = tf32_rn(x.y - h.y);
          l.z = tf32_rn(x.z - h.z);
          l.w = tf32_rn(x.w - h.w);
          hi[i] = h;
          lo[i] = l;
        }
        fence_proxy_async_smem();
        mbar_arrive(&conv[slot]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int ew = warp - 2 - CONV_WARPS;
    const int quad = warp & 3;  // TMEM lanes this warp may access: 32*quad .. 32*quad+31
    uint8_t* stg = staging + ew * 2 * STG;
    uint32_t tcount = 0, sb = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < a.tiles && ok; t += gridDim.x) {
      Job j;
      if (!job_of(t, a, j)) continue;
      const uint32_t buf = tcount & 1, use = tcount >> 1;
      if (!mbar_wait(&acc_full[buf], use & 1, abort_flag, a.status, 15)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + buf * TN;
#pragma unroll 1
      for (int ch = 0; ch < TN / 32; ++ch, sb ^= 1) {
        float v[32];
        tmem_ld32(taddr + 32 * ch, v);
        if (a.epi == kEpiStoreNeg || a.epi == kEpiSub) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = -v[i];
        }
        uint8_t* buf_s = stg + sb * STG;
        if (lane == 0) bulk_wait_read<1>();  // the store that last used this buffer has read it
        __syncwarp();
        if (a.epi != kEpiStoreT) {
          // row `lane` of the 32 x 32 box, 128-byte swizzle: 16-byte chunk c sits at c ^ (row & 7)
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<float4*>(buf_s + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        } else {
          // transposed: element (row n, column lane) of the box holds acc[lane][n]
#pragma unroll
          for (int n = 0; n < 32; ++n)
            *reinterpret_cast<float*>(buf_s + n * 128 + ((((lane >> 2) ^ (n & 7))) << 4) + (lane & 3) * 4) = v[n];
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          int x, y;
          if (a.epi != kEpiStoreT) {
            x = j.ox + 32 * ch;
            y = j.oy + 32 * quad;
          } else {
            x = j.ox + 32 * quad;
            y = j.oy + 32 * ch;
          }
          if (x < a.o_w && y < a.o_h) {  // boxes wholly outside the output are skipped
            if (a.epi == kEpiSub)
              tma_reduce_add_2d(&mapO, x, y, buf_s);
            else
              tma_store_2d(&mapO, x, y, buf_s);
          }
          bulk_commit();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      ++tcount;
    }
    if (lane == 0) bulk_wait<0>();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

// ------------------------------------------------------------------------------------------ host
bool tf32x3_map(CUtensorMap* map, const float* base, int64_t rows, int64_t cols, int64_t ld, int box_rows,
                bool mn_operand) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = tc::encode_fn();
  if (encode == nullptr) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) != 0 || (ld * 4) % 16 != 0 || rows < 1 || cols < 1) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
  const cuuint32_t box[2] = {32, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE,
                mn_operand ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
std::mutex g_setup_mu;
int g_sms[64] = {};
}  // namespace

// reserve_sms: SMs left free for work launched alongside on another stream
gptq_status tf32x3_gemm_launch(const CUtensorMap& mapA, const CUtensorMap& mapB, const CUtensorMap& mapO,
                               Tf32x3Args a, cudaStream_t stream, int reserve_sms) {
  if (a.tiles <= 0) return GPTQ_OK;
  int dev = 0;
  GPTQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return GPTQ_ERR_CUDA;
  int sms = 0;
  {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_sms[dev] == 0) {
      int n = 0;
      GPTQ_CUDA_TRY(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev));
      GPTQ_CUDA_TRY(cudaFuncSetAttribute(tf32x3_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes));
      g_sms[dev] = n;
    }
    sms = g_sms[dev];
  }
  sms -= reserve_sms;
  if (sms < 1) sms = 1;
  // kind::tf32 instruction descriptor: D f32, A/B tf32, A K-major, B K- or MN-major, N = 128, M = 128
  a.idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(a.b_mn ? 1 : 0) << 16) | ((uint32_t)(TN >> 3) << 17) |
            ((uint32_t)(TM >> 4) << 24);
  const int grid = a.tiles < sms ? a.tiles : sms;
  tf32x3_gemm_kernel<<<grid, THREADS, kSmemBytes, stream>>>(mapA, mapB, mapO, a);
  GPTQ_LAUNCH_CHECK();
  return GPTQ_OK;
}

}  // namespace gptq
