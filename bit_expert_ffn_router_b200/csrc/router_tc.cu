// Router logits of the prefill path on the tcgen05 tensor cores.
//
// The router turns each token into one logit per expert, l[t,e] = sum_i
// x[t,i] W_r[e,i] (news.blueqat.app/post/3262, section on the GPU / CPU / RAM
// / SSD split: the router runs on the GPU for every token); at a prefill
// chunk of 8,192 tokens that is a 17 GFLOP contraction.
//
// x is bf16, so it is exact as a bf16 operand. Each fp32 weight splits
// exactly into three bf16 parts, w = hi + mid + lo (hi = bf16(w), mid =
// bf16(w - hi), lo = bf16(w - hi - mid); each remainder is exact in fp32 and
// |w - (hi + mid + lo)| <= 2^-27 |w|). Every product x * part is exact in
// fp32, so three bf16 MMAs per K step give the fp32 dot product up to the
// accumulation's rounding, as the CUDA-core router does.
//
// One persistent CTA per SM, ten warps, tiles of 128 experts x 128 tokens:
//   warp 0     TMA producer: fp32 W_r tile (two 128B-swizzled boxes of 32
//              columns) and the bf16 x tile per 64-wide K stage;
//   warp 1     TMEM allocation and the tcgen05.mma issue (A from TMEM);
//   warps 2-5  split: each thread owns one expert row and writes its three
//              bf16 parts into tensor memory;
//   warps 6-9  epilogue: accumulators (+ bias) to the [T, E] logits.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace moe {

namespace {

constexpr int kRM = 128;              // experts per tile (MMA M)
constexpr int kRN = 128;              // tokens per tile (MMA N)
constexpr int kRK = 64;               // K per stage
constexpr int kRStages = 4;           // shared-memory stages
constexpr int kRTStages = 2;          // TMEM A stages (three bf16 parts each)
constexpr int kRPartCols = kRK / 2;   // one bf16 part of a stage: 64 values per lane = 32 columns
constexpr int kRAccCols = 2 * kRN;    // two accumulator buffers
constexpr int kRTmemCols = 512;
static_assert(kRAccCols + kRTStages * 3 * kRPartCols <= kRTmemCols, "tensor memory budget");
constexpr int kRThreads = 10 * 32;

struct RSmem {
  static constexpr int kAHalf = kRM * 32 * 4;                // 128 rows x 32 fp32 (one swizzled box): 16 KB
  static constexpr int kStageBytes = 2 * kAHalf + kRN * kRK * 2;  // A fp32 (32 KB) + B bf16 (16 KB)
  static constexpr int kBar = kRStages * kStageBytes;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;
};
static_assert(RSmem::kAlloc <= 227 * 1024, "shared memory budget");

struct RBars {
  uint64_t sm_full[kRStages];   // TMA -> split warps (A) and MMA (B)
  uint64_t sm_empty[kRStages];  // split warps (128) + MMA commit (1) -> producer
  uint64_t t_full[kRTStages];   // split warps -> MMA (count 128)
  uint64_t t_empty[kRTStages];  // MMA commit -> split warps
  uint64_t d_full[2];           // MMA commit -> epilogue
  uint64_t d_empty[2];          // epilogue -> MMA (count 128)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(RBars) <= 512, "barrier block");

struct RouterParams {
  const float* bias;  // [T, E] or null
  float* logits;      // [T, E]
  int T, E, d;
  int m_tiles, tiles;
  int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ bool r_aborted(const RBars* B) {
  return *reinterpret_cast<const volatile int*>(&B->abort_flag) != 0;
}

__device__ __forceinline__ bool r_wait(RBars* B, uint64_t* bar, uint32_t parity, const RouterParams& P, int where) {
  if (mbar_test(bar, parity)) return true;
  if (r_aborted(B)) return false;
  if (mbar_wait(bar, parity, global_timer_ns() + P.timeout_ns)) return true;
  report(P.status, kDevTimeout, 200 + where);
  *reinterpret_cast<volatile int*>(&B->abort_flag) = 1;
  return false;
}

// Warp-wide wait (lane 0 waits, the warp follows): the tcgen05.ld/st after it
// are warp-collective.
__device__ __forceinline__ bool r_wait_warp(RBars* B, uint64_t* bar, uint32_t parity, const RouterParams& P,
                                            int where) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = r_wait(B, bar, parity, P, where) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ uint32_t bf16_bits_rn(float v) {
  return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v)));
}

__global__ void __launch_bounds__(kRThreads, 1)
router_tc_kernel(const __grid_constant__ CUtensorMap tW, const __grid_constant__ CUtensorMap tX,
                 const RouterParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RBars* B = reinterpret_cast<RBars*>(smem + RSmem::kBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;
  const int ks = P.d / kRK;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRStages; ++i) {
      mbar_init(&B->sm_full[i], 1);
      mbar_init(&B->sm_empty[i], 128 + 1);
    }
    for (int i = 0; i < kRTStages; ++i) {
      mbar_init(&B->t_full[i], 128);
      mbar_init(&B->t_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B->d_full[i], 1);
      mbar_init(&B->d_empty[i], 128);
    }
    mbar_init(&B->mma_done, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&B->tmem_base, kRTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < P.tiles && ok && !r_aborted(B); w += G) {
        const int m0 = (w % P.m_tiles) * kRM, n0 = (w / P.m_tiles) * kRN;
        for (int k = 0; k < ks; ++k, ++g) {
          const int s = g % kRStages;
          if (g >= kRStages && !r_wait(B, &B->sm_empty[s], ((g / kRStages) - 1) & 1, P, 1)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * RSmem::kStageBytes;
          mbar_arrive_expect_tx(&B->sm_full[s], RSmem::kStageBytes);
          tma_load_2d(st, &tW, k * kRK, m0, &B->sm_full[s]);
          tma_load_2d(st + RSmem::kAHalf, &tW, k * kRK + 32, m0, &B->sm_full[s]);
          tma_load_2d(st + 2 * RSmem::kAHalf, &tX, k * kRK, n0, &B->sm_full[s]);
        }
      }
      const uint64_t drain = global_timer_ns() + P.timeout_ns;
      for (int n = max(0, g - kRStages); n < g; ++n) mbar_wait(&B->sm_full[n % kRStages], (n / kRStages) & 1, drain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = instr_desc_f16(kRN, true);
      int g = 0, it = 0;
      for (int w = blockIdx.x; w < P.tiles && !r_aborted(B); w += G, ++it) {
        const int acc = it & 1;
        if (it >= 2 && !r_wait(B, &B->d_empty[acc], ((it >> 1) - 1) & 1, P, 2)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kRN);
        bool ok = true;
        for (int k = 0; k < ks; ++k, ++g) {
          const int s = g % kRStages, t = g % kRTStages;
          if (!r_wait(B, &B->t_full[t], (g / kRTStages) & 1, P, 3) ||
              !r_wait(B, &B->sm_full[s], (g / kRStages) & 1, P, 4)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t db = smem_desc(smem + s * RSmem::kStageBytes + 2 * RSmem::kAHalf);
          const uint32_t ta = tmem + static_cast<uint32_t>(kRAccCols + t * 3 * kRPartCols);
#pragma unroll
          for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int kk = 0; kk < kRK / 16; ++kk)
              tc_mma_ts(d_tmem, ta + j * kRPartCols + 8 * kk, db + 2 * kk, idesc, (k > 0 || j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&B->t_empty[t]);
          tc_commit(&B->sm_empty[s]);
        }
        if (!ok) break;
        tc_commit(&B->d_full[acc]);
      }
      tc_commit(&B->mma_done);
      mbar_wait(&B->mma_done, 0, global_timer_ns() + P.timeout_ns);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ split into bf16 parts
    const int r = 32 * (warp & 3) + lane;  // expert row of the tile = this thread's TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    int g = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < P.tiles && ok; w += G) {
      if (__shfl_sync(0xffffffffu, r_aborted(B) ? 1 : 0, 0)) break;
      for (int k = 0; k < ks; ++k, ++g) {
        const int s = g % kRStages, t = g % kRTStages;
        if (!r_wait_warp(B, &B->sm_full[s], (g / kRStages) & 1, P, 5) ||
            (g >= kRTStages && !r_wait_warp(B, &B->t_empty[t], ((g / kRTStages) - 1) & 1, P, 6))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // Row r of the two swizzled fp32 boxes (16-byte chunk c at c ^ (r % 8)),
        // one box (32 values) at a time: part j of K values 32h + 2c, 32h + 2c + 1
        // goes to column j * 32 + 16h + c.
        const uint8_t* st = smem + s * RSmem::kStageBytes;
        const uint32_t ta = lane_addr + static_cast<uint32_t>(kRAccCols + t * 3 * kRPartCols);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          float wv[32];
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const float4 q = *reinterpret_cast<const float4*>(st + h * RSmem::kAHalf + r * 128 + ((c ^ (r & 7)) * 16));
            wv[4 * c] = q.x;
            wv[4 * c + 1] = q.y;
            wv[4 * c + 2] = q.z;
            wv[4 * c + 3] = q.w;
          }
          if (h == 1) mbar_arrive(&B->sm_empty[s]);  // the fp32 tile is in registers
#pragma unroll
          for (int j = 0; j < 3; ++j) {
            uint32_t part[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const uint32_t b0 = bf16_bits_rn(wv[2 * c]), b1 = bf16_bits_rn(wv[2 * c + 1]);
              part[c] = b0 | (b1 << 16);
              wv[2 * c] -= __uint_as_float(b0 << 16);  // exact remainder for the next part
              wv[2 * c + 1] -= __uint_as_float(b1 << 16);
            }
            tmem_st16_nowait(ta + j * kRPartCols + 16 * h, part);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&B->t_full[t]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int r = 32 * q + lane;
    int it = 0;
    for (int w = blockIdx.x; w < P.tiles; w += G, ++it) {
      if (__shfl_sync(0xffffffffu, r_aborted(B) ? 1 : 0, 0)) break;
      const int m0 = (w % P.m_tiles) * kRM, n0 = (w / P.m_tiles) * kRN;
      const int acc = it & 1;
      if (!r_wait_warp(B, &B->d_full[acc], (it >> 1) & 1, P, 7)) break;
      tc_fence_after();
      const uint32_t base = tmem + static_cast<uint32_t>(acc * kRN) + (static_cast<uint32_t>(q * 32) << 16);
      const int e = m0 + r, ec = min(e, P.E - 1);
      for (int c0 = 0; c0 < kRN && n0 + c0 < P.T; c0 += 16) {
        float bv[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {  // all loads issued before any is used (clamped, valid addresses)
          const int tc = min(n0 + c0 + i, P.T - 1);
          bv[i] = P.bias != nullptr ? __ldg(P.bias + static_cast<size_t>(tc) * P.E + ec) : 0.f;
        }
        float v[16];
        tmem_ld16(base + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int t = n0 + c0 + i;
          if (t < P.T && e < P.E) P.logits[static_cast<size_t>(t) * P.E + e] = v[i] + bv[i];
        }
      }
      tc_fence_before();
      mbar_arrive(&B->d_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kRTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode_r = nullptr;

bool encode_2d(CUtensorMap* m, CUtensorMapDataType type, int elem_bytes, const void* base, int cols, int rows,
               int box_cols, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t es[2] = {1u, 1u};
  return g_encode_r(m, type, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t router_tc_init(const Ctx& ctx) {
  (void)ctx;
  return cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RSmem::kAlloc);
}

bool router_tc_ok(const moe_layer_cfg& c) { return c.d % kRK == 0; }

cudaError_t launch_router_tc(const Ctx& ctx, const moe_layer_cfg& c, const uint16_t* x, const float* wr,
                             const float* bias, int T, float* logits, cudaStream_t s) {
  if (!router_tc_ok(c)) return cudaErrorNotSupported;
  if (g_encode_r == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
    g_encode_r = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  CUtensorMap tW, tX;
  if (!encode_2d(&tW, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, wr, c.d, c.E, 32, kRM) ||
      !encode_2d(&tX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, c.d, T, kRK, kRN))
    return cudaErrorInvalidValue;
  RouterParams P{};
  P.bias = bias;
  P.logits = logits;
  P.T = T;
  P.E = c.E;
  P.d = c.d;
  P.m_tiles = (c.E + kRM - 1) / kRM;
  P.tiles = P.m_tiles * ((T + kRN - 1) / kRN);
  P.status = ctx.d_status;
  P.timeout_ns = ctx.timeout_ns;
  const int grid = P.tiles < ctx.num_sms ? P.tiles : ctx.num_sms;
  router_tc_kernel<<<grid, kRThreads, RSmem::kAlloc, s>>>(tW, tX, P);
  return cudaGetLastError();
}

}  // namespace moe
