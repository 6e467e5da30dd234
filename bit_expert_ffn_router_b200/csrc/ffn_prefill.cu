// Prefill-path expert FFN: a grouped GEMM on the tcgen05 tensor cores with
// the 2/3-bit dequantisation fused in.
//
// The pages process long inputs in chunks of up to 8,192 tokens, layer by
// layer (news.blueqat.app/post/3262, section on the GPU / CPU / RAM / SSD
// split). With T*k = 81,920 token-expert pairs per chunk the expert FFN is a
// dense contraction: for every expert, its sorted pairs form the N side of a
// GEMM whose M side is the expert's weight rows.
//
//   gate/up: D[128 weight rows, N pairs] = W_gu[rows, d] * Xg[pairs, d]^T,
//            epilogue h = silu(g) * u (rows 2c, 2c+1 are neighbours) -> fp16
//   down:    D[128 output rows, N pairs] = W_d[rows, f] * H[pairs, f]^T,
//            epilogue z = gate * D -> fp32 rows in pair order
//
// One persistent CTA per SM, fifteen warps:
//   warp 0      activation producer: the 128B-swizzled K-major activation
//               tile by TMA, a box of 16 to 128 rows sized to the item's N;
//   warp 14     weight producer: packed codes (3-D tensor maps over the
//               whole expert pool) and fp16 scales (one bulk copy per work
//               item), running ahead of the activations as far as its own
//               ring allows;
//   warp 1      TMEM allocation and the single-thread tcgen05.mma issue;
//   warps 2-9   dequantisation, two teams of four warps taking alternate
//               128-wide K stages: each thread owns one weight row and writes
//               s * (q - 2^(b-1)) as fp16 straight into tensor memory (its
//               TMEM lane), where the MMA reads its A operand. The weights
//               never pass through shared memory, whose bandwidth the
//               activation tiles and codes already use;
//   warps 10-13 epilogue: tcgen05.ld of the fp32 accumulators (two TMEM
//               buffers, so the next item's MMAs overlap this item's stores).
//
// K order. A 32-bit word of 2-bit codes holds a 16-code group; shifting it by
// 2i and masking 0x00030003 yields codes i and i+8 in the two halves of one
// fp16x2 register. The dequantiser stores that pair as K positions 2i, 2i+1,
// i.e. inside every aligned group of 16 the K order is
//     position 2i <- index i,   position 2i+1 <- index i+8.
// A dot product does not depend on the order of its terms, so the activation
// operands are stored in the same order (the x gather and the gate/up
// epilogue's h writes permute within each group of 16) and the result is the
// plain contraction. Groups never straddle a 32-weight scale block.
//
// Operands are fp16 on both sides (A and B of one kind::f16 MMA share a
// type): 2-bit weights are exact in fp16, 3-bit ones round at 2^-12
// relative, bf16 activations convert exactly in fp16's normal range.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"
#include "ptx.cuh"
#include "tc.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;            // weight rows per tile (MMA M)
constexpr int kBN = kTileN;         // pairs per tile (MMA N, max)
constexpr int kBK = 128;            // K per pipeline stage: 8 MMAs of K = 16
constexpr int kSub = 64;            // K per 128-byte swizzle atom of fp16 (two per stage)
constexpr int kStages = 4;          // ring depth: A stages (TMEM), activation slots, code chunks
constexpr int kDqThreads = 128;     // threads per dequant team (one per weight row)
constexpr int kThreads = 15 * 32;
constexpr int kAccCols = 2 * kBN;   // two accumulator buffers (TMEM columns 0..255)
constexpr int kACols = kBK / 2;     // one A stage: 128 fp16 per lane = 64 columns
constexpr int kTmemCols = 512;      // accumulators + kStages A stages
static_assert(kAccCols + kStages * kACols <= kTmemCols, "tensor memory budget");
constexpr int kMaxKDim = 2048;      // largest reduction size (scale staging holds 128 x K/16 bytes)

struct PrefillSmem {
  // byte offsets from the 1024-aligned base of dynamic shared memory
  static constexpr int kSubBytes = kBN * kSub * 2;                 // one swizzled sub-tile: 16 KB
  static constexpr int kB = 0;                                     // kStages x 2 sub-tiles
  static constexpr int kCodeLo = kB + kStages * 2 * kSubBytes;     // kStages x (128 rows x 32 B)
  static constexpr int kCodeHi = kCodeLo + kStages * kBM * (kBK / 4);  // kStages x (128 x 16 B)
  static constexpr int kScale = kCodeHi + kStages * kBM * (kBK / 8);   // 2 x (128 rows x K/16 B)
  static constexpr int kScaleBuf = kBM * (kMaxKDim / kBlock) * 2;
  static constexpr int kStage = kScale + 2 * kScaleBuf;            // epilogue staging 16 KB
  static constexpr int kBar = kStage + 16384;
  static constexpr int kBytes = kBar + 1024;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base
};
static_assert(PrefillSmem::kAlloc <= 227 * 1024, "shared memory budget");

struct Bars {
  uint64_t a_full[kStages];     // dequant team -> MMA (count 128): A stage written to TMEM
  uint64_t b_full[kStages];     // TMA -> MMA (tx): activation slot landed
  uint64_t st_empty[kStages];   // MMA commit -> dequant team and activation producer: A stage and slot free
  uint64_t c_full[kStages];     // TMA -> dequant (tx): code chunk landed
  uint64_t c_empty[kStages];    // dequant team -> weight producer (count 128)
  uint64_t s_full[2];           // bulk copy -> dequant (tx)
  uint64_t s_empty[2];          // both dequant teams -> producer (count 256)
  uint64_t d_full[2];           // MMA commit -> epilogue
  uint64_t d_empty[2];          // epilogue -> MMA (count 128)
  uint64_t mma_done;            // final MMA commit, waited on before TMEM is freed
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

struct GemmParams {
  const int4* tile_info;        // per token tile: {expert (E = shared), first row, rows, slot}
  const int32_t* tile_offset;   // [E+2]; tile_offset[E+1] = number of token tiles
  const float* pair_gate;       // [n_pairs]
  const uint8_t* pool;          // scale sections are read with plain bulk copies
  const uint8_t* shared;        // shared-expert record (or null)
  size_t stride;
  size_t scale_off;             // section offset of this matrix's scales inside a record
  int E, n_pairs;
  int K, m_tiles;               // reduction size, weight-row tiles per expert
  int hi_col0;                  // byte column of the high plane in a code row (3-bit)
  int sc_row_bytes;             // fp16 scale bytes per weight row (K/16)
  void* out;                    // gate/up: h fp16 [n_rows, f]; down: z fp32 [n_rows, d]
  int ld_out;                   // elements per output row
  int* status;
  unsigned long long timeout_ns;
};

__device__ __forceinline__ bool aborted(const Bars* B) {
  return *reinterpret_cast<const volatile int*>(&B->abort_flag) != 0;
}

// Waits at most `limit` ns; on expiry records the place, raises the CTA's
// abort flag and returns false (every role then leaves its loop).
__device__ __forceinline__ bool wait_bar(Bars* B, uint64_t* bar, uint32_t parity, uint64_t limit, int* status,
                                         int where) {
  if (aborted(B)) return false;
  if (mbar_try_wait(bar, parity)) return true;
  if (mbar_wait(bar, parity, global_timer_ns() + limit)) return true;
  report(status, kDevTimeout, 100 + where);
  *reinterpret_cast<volatile int*>(&B->abort_flag) = 1;
  return false;
}

// For waits that are usually already satisfied (the MMA thread's): one
// non-blocking test, then the bounded wait.
__device__ __forceinline__ bool wait_fast(Bars* B, uint64_t* bar, uint32_t parity, uint64_t limit, int* status,
                                          int where) {
  return mbar_test(bar, parity) || wait_bar(B, bar, parity, limit, status, where);
}

// The abort flag as lane 0 sees it, the same for the whole warp.
__device__ __forceinline__ bool aborted_warp(const Bars* B) {
  return __shfl_sync(0xffffffffu, aborted(B) ? 1 : 0, 0) != 0;
}

// Warp-wide wait: lane 0 waits, the result is broadcast and the warp
// synchronises (ordering the other lanes' later accesses after lane 0's
// observation of the phase). Every lane then takes the same path, which the
// warp-collective tcgen05.ld / tcgen05.st that follow require.
__device__ __forceinline__ bool wait_bar_warp(Bars* B, uint64_t* bar, uint32_t parity, uint64_t limit, int* status,
                                              int where) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(B, bar, parity, limit, status, where) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

// ------------------------------------------------------------------ K-order permutation
// Position of index i inside its group of 16 (inverse of: position 2i <- i,
// position 2i+1 <- i+8).
__host__ __device__ __forceinline__ int k_position(int i) { return i < 8 ? 2 * i : 2 * i - 15; }

// ------------------------------------------------------------------ dequantisation of one K stage
// One weight row's 64 weights s * (q - 2^(BITS-1)) of a K stage as 32 fp16
// pairs, in the permuted K order: word 8q + i holds (index 16q+i, index
// 16q+i+8) of the stage.
template <int BITS>
__device__ __forceinline__ void dequant_stage(uint32_t* out, const uint8_t* lo, const uint8_t* hi, uint32_t s01) {
  const uint4 w = *reinterpret_cast<const uint4*>(lo);  // 64 two-bit codes: four groups of 16
  const uint32_t wl[4] = {w.x, w.y, w.z, w.w};
  uint32_t hq[4] = {0u, 0u, 0u, 0u};
  if (BITS == 3) {
    // the groups' high bits, spread so that index i lands at bit 2+i and
    // index i+8 at bit 18+i
    const uint2 hv = *reinterpret_cast<const uint2*>(hi);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t h16 = ((q < 2 ? hv.x : hv.y) >> (16 * (q & 1))) & 0xffffu;
      hq[q] = ((h16 & 0xffu) | ((h16 & 0xff00u) << 8)) << 2;
    }
  }
  const __half2 s0 = __half2half2(__ushort_as_half(static_cast<unsigned short>(s01 & 0xffffu)));
  const __half2 s1 = __half2half2(__ushort_as_half(static_cast<unsigned short>(s01 >> 16)));
  // 0x6400 | q is the fp16 number 1024 + q; subtracting 1024 + 2^(BITS-1) is exact
  const __half2 off = __float2half2_rn(1024.f + static_cast<float>(1 << (BITS - 1)));
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const __half2 s = q < 2 ? s0 : s1;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      uint32_t v = (wl[q] >> (2 * i)) & 0x00030003u;
      if (BITS == 3) v |= (hq[q] >> i) & 0x00040004u;
      v |= 0x64006400u;
      const __half2 y = __hmul2(__hsub2(*reinterpret_cast<const __half2*>(&v), off), s);
      out[8 * q + i] = *reinterpret_cast<const uint32_t*>(&y);
    }
  }
}

// ------------------------------------------------------------------ the kernel
template <int BITS, bool DOWN>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tB16, const __grid_constant__ CUtensorMap tB32,
                    const __grid_constant__ CUtensorMap tB64, const __grid_constant__ CUtensorMap tB128,
                    const __grid_constant__ CUtensorMap tLo, const __grid_constant__ CUtensorMap tHi,
                    const __grid_constant__ CUtensorMap tLoS, const __grid_constant__ CUtensorMap tHiS,
                    const GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* B = reinterpret_cast<Bars*>(smem + PrefillSmem::kBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&B->a_full[i], kDqThreads);
      mbar_init(&B->b_full[i], 1);
      mbar_init(&B->st_empty[i], 1);
      mbar_init(&B->c_full[i], 1);
      mbar_init(&B->c_empty[i], kDqThreads);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B->s_full[i], 1);
      mbar_init(&B->s_empty[i], 2 * kDqThreads);
      mbar_init(&B->d_full[i], 1);
      mbar_init(&B->d_empty[i], 128);
    }
    mbar_init(&B->mma_done, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {  // TMEM: accumulators and the A stages
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&B->tmem_base)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = B->tmem_base;

  // everything below reads the grouping (and, for the down pass, h) written
  // by the kernels before this one
  grid_dep_wait();
  const uint64_t limit = P.timeout_ns;  // limit of each wait
  const int total = __ldg(P.tile_offset + P.E + 1) * P.m_tiles;
  const int ks_per_item = P.K / kBK;
  const uint32_t code_tx = kBM * (kBK / 4) + (BITS == 3 ? kBM * (kBK / 8) : 0);
  const uint32_t scale_tx = kBM * P.sc_row_bytes;
  const int G = gridDim.x;

  if (warp == 0) {
    // ---------------------------------------------------------- activation producer
    if (lane == 0) {
      int g = 0;
      int4 next = blockIdx.x < total ? __ldg(P.tile_info + blockIdx.x / P.m_tiles) : make_int4(0, 0, 0, 0);
      bool ok = true;
      for (int w = blockIdx.x; w < total && ok && !aborted(B); w += G) {
        const int4 info = next;  // {expert, row0, rows, slot}
        if (w + G < total) next = __ldg(P.tile_info + (w + G) / P.m_tiles);
        const int box = info.z <= 16 ? 16 : info.z <= 32 ? 32 : info.z <= 64 ? 64 : 128;
        const CUtensorMap* mB = box == 16 ? &tB16 : box == 32 ? &tB32 : box == 64 ? &tB64 : &tB128;
        const uint32_t b_tx = static_cast<uint32_t>(box) * kBK * 2;
        for (int k = 0; k < ks_per_item; ++k, ++g) {
          const int st = g % kStages;
          if (g >= kStages && !wait_bar(B, &B->st_empty[st], ((g / kStages) - 1) & 1, limit, P.status, 3)) {
            ok = false;
            break;
          }
          uint8_t* slot = smem + PrefillSmem::kB + st * 2 * PrefillSmem::kSubBytes;
          mbar_arrive_expect_tx(&B->b_full[st], b_tx);
          tma_load_2d(slot, mB, k * kBK, info.y, &B->b_full[st]);
          tma_load_2d(slot + PrefillSmem::kSubBytes, mB, k * kBK + kSub, info.y, &B->b_full[st]);
        }
      }
      // every copy this thread issued lands before the CTA may exit (bounded wait)
      const uint64_t drain = global_timer_ns() + P.timeout_ns;
      for (int n = max(0, g - kStages); n < g; ++n) mbar_wait(&B->b_full[n % kStages], (n / kStages) & 1, drain);
    }
  } else if (warp == 14) {
    // ---------------------------------------------------------- weight producer
    if (lane == 0) {
      int g = 0, it = 0;
      int4 next = blockIdx.x < total ? __ldg(P.tile_info + blockIdx.x / P.m_tiles) : make_int4(0, 0, 0, 0);
      for (int w = blockIdx.x; w < total && !aborted(B); w += G, ++it) {
        const int4 info = next;
        if (w + G < total) next = __ldg(P.tile_info + (w + G) / P.m_tiles);
        const int m = w % P.m_tiles;
        const bool sh = info.x >= P.E;
        const CUtensorMap* mLo = sh ? &tLoS : &tLo;
        const CUtensorMap* mHi = sh ? &tHiS : &tHi;
        const int slot = sh ? 0 : info.w;
        const uint8_t* rec = sh ? P.shared : P.pool + static_cast<size_t>(slot) * P.stride;
        const int sb = it & 1;
        if (it >= 2 && !wait_bar(B, &B->s_empty[sb], ((it >> 1) - 1) & 1, limit, P.status, 1)) break;
        mbar_arrive_expect_tx(&B->s_full[sb], scale_tx);
        bulk_g2s(smem + PrefillSmem::kScale + sb * PrefillSmem::kScaleBuf,
                 rec + P.scale_off + static_cast<size_t>(m) * scale_tx, scale_tx, &B->s_full[sb]);
        bool ok = true;
        for (int k = 0; k < ks_per_item; ++k, ++g) {
          const int st = g % kStages;
          if (g >= kStages && !wait_bar(B, &B->c_empty[st], ((g / kStages) - 1) & 1, limit, P.status, 2)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&B->c_full[st], code_tx);
          tma_load_3d(smem + PrefillSmem::kCodeLo + st * kBM * (kBK / 4), mLo, k * (kBK / 4), m * kBM, slot,
                      &B->c_full[st]);
          if (BITS == 3)
            tma_load_3d(smem + PrefillSmem::kCodeHi + st * kBM * (kBK / 8), mHi, P.hi_col0 + k * (kBK / 8),
                        m * kBM, slot, &B->c_full[st]);
        }
        if (!ok) break;
      }
      const uint64_t drain = global_timer_ns() + P.timeout_ns;
      for (int n = max(0, g - kStages); n < g; ++n) mbar_wait(&B->c_full[n % kStages], (n / kStages) & 1, drain);
      for (int n = max(0, it - 2); n < it; ++n) mbar_wait(&B->s_full[n & 1], (n >> 1) & 1, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      int g = 0, it = 0;
      int4 next = blockIdx.x < total ? __ldg(P.tile_info + blockIdx.x / P.m_tiles) : make_int4(0, 0, 0, 0);
      for (int w = blockIdx.x; w < total && !aborted(B); w += G, ++it) {
        const int4 info = next;
        if (w + G < total) next = __ldg(P.tile_info + (w + G) / P.m_tiles);
        const int n = (info.z + 15) / 16 * 16;
        const uint32_t idesc = instr_desc_f16(n, false);
        const int acc = it & 1;
        if (it >= 2 && !wait_fast(B, &B->d_empty[acc], ((it >> 1) - 1) & 1, limit, P.status, 4)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int k = 0; k < ks_per_item; ++k, ++g) {
          const int st = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          if (!wait_fast(B, &B->a_full[st], ph, limit, P.status, 5) ||
              !wait_fast(B, &B->b_full[st], ph, limit, P.status, 6)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ta = tmem + static_cast<uint32_t>(kAccCols + st * kACols);
          const uint8_t* slot = smem + PrefillSmem::kB + st * 2 * PrefillSmem::kSubBytes;
          const uint64_t db0 = smem_desc(slot), db1 = smem_desc(slot + PrefillSmem::kSubBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)  // K = 16 per MMA: 8 TMEM columns of A, 32 bytes of B
            tc_mma_ts(d_tmem, ta + 8 * kk, (kk < 4 ? db0 : db1) + 2 * (kk & 3), idesc, (k > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&B->st_empty[st]);
        }
        if (!ok) break;
        tc_commit(&B->d_full[acc]);
      }
      // all MMAs issued above complete before the tensor memory is freed
      tc_commit(&B->mma_done);
      mbar_wait(&B->mma_done, 0, global_timer_ns() + P.timeout_ns);
    }
  } else if (warp >= 2 && warp < 10) {
    // ---------------------------------------------------------- dequantisation
    const int team = (warp - 2) >> 2;          // takes the stages g with g % 2 == team
    const int r = 32 * (warp & 3) + lane;      // weight row of the tile = this thread's TMEM lane
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    int g = 0, it = 0;
    for (int w = blockIdx.x; w < total && !aborted_warp(B); w += G, ++it) {
      const int sb = it & 1;
      if (!wait_bar_warp(B, &B->s_full[sb], (it >> 1) & 1, limit, P.status, 7)) break;
      const uint8_t* sc = smem + PrefillSmem::kScale + sb * PrefillSmem::kScaleBuf + r * P.sc_row_bytes;
      bool ok = true;
      for (int k = 0; k < ks_per_item; ++k, ++g) {
        if ((g & 1) != team) continue;
        const int st = g % kStages;
        if (!wait_bar_warp(B, &B->c_full[st], (g / kStages) & 1, limit, P.status, 8) ||
            (g >= kStages && !wait_bar_warp(B, &B->st_empty[st], ((g / kStages) - 1) & 1, limit, P.status, 9))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint2 s4 = *reinterpret_cast<const uint2*>(sc + 8 * k);  // scales of the stage's 4 blocks
        const uint8_t* lo = smem + PrefillSmem::kCodeLo + st * kBM * (kBK / 4) + r * (kBK / 4);
        const uint8_t* hi = smem + PrefillSmem::kCodeHi + st * kBM * (kBK / 8) + r * (kBK / 8);
        const uint32_t ta = lane_addr + static_cast<uint32_t>(kAccCols + st * kACols);
        uint32_t a_half[kACols / 2];
        dequant_stage<BITS>(a_half, lo, hi, s4.x);  // K 0..63 of the stage
        tmem_st32(ta, a_half);
        dequant_stage<BITS>(a_half, lo + 16, hi + 8, s4.y);  // K 64..127
        tmem_st32(ta + kACols / 2, a_half);
        tc_fence_before();  // the stores are complete; order them before the arrival
        mbar_arrive(&B->a_full[st]);
        mbar_arrive(&B->c_empty[st]);
      }
      if (!ok) break;
      mbar_arrive(&B->s_empty[sb]);
    }
  } else if (warp >= 10 && warp < 14) {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;       // accumulator lane = weight row of the tile
    const int et = threadIdx.x - 320;  // 0..127 among the epilogue threads
    int it = 0;
    int4 next = blockIdx.x < total ? __ldg(P.tile_info + blockIdx.x / P.m_tiles) : make_int4(0, 0, 0, 0);
    for (int w = blockIdx.x; w < total && !aborted_warp(B); w += G, ++it) {
      const int4 info = next;
      if (w + G < total) next = __ldg(P.tile_info + (w + G) / P.m_tiles);
      const int m = w % P.m_tiles, row0 = info.y, rows = info.z;
      const int acc = it & 1;
      if (!wait_bar_warp(B, &B->d_full[acc], (it >> 1) & 1, limit, P.status, 10)) break;
      tc_fence_after();
      const uint32_t base = tmem + static_cast<uint32_t>(acc * kBN) + (static_cast<uint32_t>(q * 32) << 16);
      if (!DOWN) {
        // channel m*64 + r/2 (gate on the even lane, up on the odd one),
        // stored at its permuted position inside its group of 16
        const int lc = r >> 1;
        const int lp = (lc & ~15) | k_position(lc & 15);
        __half* hs = reinterpret_cast<__half*>(smem + PrefillSmem::kStage);  // [kBN pairs][64 channels]
        // the lane pair (gate, up) shares the 16 columns of a chunk: the gate
        // lane takes columns 0..7, the up lane 8..15 (h is rounded to fp16, so
        // the fast exponential and division are well inside its precision)
        const bool up_lane = (lane & 1) != 0;
        for (int c0 = 0; c0 < rows; c0 += 16) {
          float v[16], o[16];
          tmem_ld16(base + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __shfl_xor_sync(0xffffffffu, v[i], 1);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float g = up_lane ? o[8 + i] : v[i];
            const float u = up_lane ? v[8 + i] : o[i];
            const int col = c0 + (up_lane ? 8 : 0) + i;
            if (col < rows) hs[col * 64 + lp] = __float2half_rn(__fdividef(g, 1.f + __expf(-g)) * u);
          }
        }
        tc_fence_before();
        mbar_arrive(&B->d_empty[acc]);
        named_sync(2, 128);
        __half* out = static_cast<__half*>(P.out);
        for (int e = et; e < rows * 8; e += 128) {  // 128 bytes (64 channels) per pair row
          const int row = e >> 3, ch = (e & 7) * 8;
          *reinterpret_cast<uint4*>(out + static_cast<size_t>(row0 + row) * P.ld_out + m * 64 + ch) =
              *reinterpret_cast<const uint4*>(hs + row * 64 + ch);
        }
        named_sync(2, 128);
      } else {
        // output dim m*128 + r, 32 pairs at a time through the staging tile
        float* zs = reinterpret_cast<float*>(smem + PrefillSmem::kStage);  // [32 pairs][128 dims]
        float* out = static_cast<float*>(P.out);
        for (int c0 = 0; c0 < rows; c0 += 32) {
          // lane i fetches the gate of pair c0 + i (one coalesced load; the
          // shared expert's rows and rows past the tile take gate 1)
          const int pl = row0 + c0 + lane;
          const float g_l = __ldg(P.pair_gate + min(pl, P.n_pairs - 1));
          const float gate_l = (c0 + lane < rows && pl < P.n_pairs) ? g_l : 1.f;
          float v[32];
          tmem_ld16(base + c0, v);
          tmem_ld16(base + c0 + 16, v + 16);
#pragma unroll
          for (int i = 0; i < 32; ++i) zs[i * 128 + r] = __shfl_sync(0xffffffffu, gate_l, i) * v[i];
          named_sync(2, 128);
          const int nrow = min(32, rows - c0);
          for (int e = et; e < nrow * 32; e += 128) {
            const int row = e >> 5, col = (e & 31) * 4;
            *reinterpret_cast<float4*>(out + static_cast<size_t>(row0 + c0 + row) * P.ld_out + m * kBM + col) =
                *reinterpret_cast<const float4*>(zs + row * 128 + col);
          }
          named_sync(2, 128);
        }
        tc_fence_before();
        mbar_arrive(&B->d_empty[acc]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// ------------------------------------------------------------------ x gather (bf16 -> fp16 rows in pair order)
// Row r < n_pairs is token pair_token[r]; rows n_pairs .. n_rows-1 are the
// shared expert's rows, token r - n_pairs. Inside every group of 16 columns
// the row is stored in the permuted K order: position 2i <- column i,
// position 2i+1 <- column i+8.
__global__ void __launch_bounds__(256) gather_x_kernel(const uint16_t* __restrict__ x,
                                                       const int32_t* __restrict__ pair_token, int n_pairs,
                                                       int n_rows, int T, int d, __half* __restrict__ xg) {
  const int r = blockIdx.x;
  if (r >= n_rows) return;
  // the token index is clamped into [0, T): a grouping that saw a bad expert
  // index (reported as MOE_EDEVICE) must still not steer a read out of x
  const int t = min(max(r < n_pairs ? __ldg(pair_token + r) : r - n_pairs, 0), T - 1);
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
  uint4* dst = reinterpret_cast<uint4*>(xg + static_cast<size_t>(r) * d);
  for (int gi = threadIdx.x; gi < d / 16; gi += blockDim.x) {
    const uint4 a = __ldg(src + 2 * gi), b = __ldg(src + 2 * gi + 1);  // columns 16gi .. +7, +8 .. +15
    const uint32_t lo[4] = {a.x, a.y, a.z, a.w}, hi[4] = {b.x, b.y, b.z, b.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // (column i, column i+8) as one fp16 pair
      const uint32_t xi = (i & 1) ? (lo[i >> 1] & 0xffff0000u) : (lo[i >> 1] << 16);
      const uint32_t xj = (i & 1) ? (hi[i >> 1] & 0xffff0000u) : (hi[i >> 1] << 16);
      const __half2 h = __floats2half2_rn(__uint_as_float(xi), __uint_as_float(xj));
      o[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    dst[2 * gi] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * gi + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Token-tile table: for every extended expert x (routed 0..E-1, shared = E)
// and each of its ceil(n_x / 128) token tiles, {x, first sorted row, rows,
// pool slot}, at index tile_offset[x] + i.
__global__ void __launch_bounds__(256) tile_table_kernel(const int32_t* __restrict__ tile_offset,
                                                         const int32_t* __restrict__ expert_offset,
                                                         const int32_t* __restrict__ expert_count,
                                                         const int32_t* __restrict__ pair_slot, int E, int T,
                                                         int n_pairs, int has_shared, int4* __restrict__ info) {
  const int x = blockIdx.x * blockDim.x + threadIdx.x;
  if (x > E) return;
  const int n = x < E ? expert_count[x] : (has_shared ? T : 0);
  const int base = x < E ? expert_offset[x] : n_pairs;
  const int slot = (x < E && n > 0) ? pair_slot[base] : 0;
  const int t0 = tile_offset[x];
  for (int i = 0; i * kBN < n; ++i) info[t0 + i] = make_int4(x, base + i * kBN, min(kBN, n - i * kBN), slot);
}

// ------------------------------------------------------------------ tensor maps (host)
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaError_t get_encoder() {
  if (g_encode != nullptr) return cudaSuccess;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) return cudaErrorNotSupported;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return cudaSuccess;
}

// Largest slot count a tensor map over the pool admits. The grouping only
// produces slots below the caller's n_slots, so no load goes past the pool.
constexpr cuuint64_t kMapSlots = 1ull << 24;

// 3-D byte tensor over one code section of every record: [slots][rows][row_bytes],
// boxes of box_bytes x 128 rows x 1 record.
bool map_codes(CUtensorMap* m, const uint8_t* base, size_t row_bytes, int rows, size_t slot_stride,
               cuuint64_t slots, int box_bytes) {
  const cuuint64_t dims[3] = {row_bytes, static_cast<cuuint64_t>(rows), slots};
  const cuuint64_t strides[2] = {row_bytes, slot_stride};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_bytes), static_cast<cuuint32_t>(kBM), 1u};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp16 activation tensor [rows][K], boxes of 64 x box_rows with the
// 128-byte swizzle; rows past the end read as zeros.
bool map_act(CUtensorMap* m, const __half* base, int K, int rows, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kSub), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t es[2] = {1u, 1u};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps and launch of one grouped GEMM pass over the matrix whose code
// section starts at `codes_off` (rows x K) and scales at `scales_off`.
template <int BITS, bool DOWN>
cudaError_t run_pass(const Ctx& ctx, const FfnArgs& a, GemmParams P, const __half* act, int n_rows, int K, int rows,
                     size_t codes_off, size_t scales_off, cudaStream_t s) {
  const size_t row_b = static_cast<size_t>(K) * BITS / 8;
  const uint8_t* shr = a.shared != nullptr ? a.shared : a.pool;  // keeps the shared maps well formed
  CUtensorMap maps[8];
  bool ok = true;
  for (int i = 0; i < 4; ++i) ok = ok && map_act(&maps[i], act, K, n_rows, 16 << i);  // 64-wide boxes
  ok = ok && map_codes(&maps[4], a.pool + codes_off, row_b, rows, a.stride, kMapSlots, kBK / 4);
  ok = ok && map_codes(&maps[5], a.pool + codes_off, row_b, rows, a.stride, kMapSlots, kBK / 8);
  ok = ok && map_codes(&maps[6], shr + codes_off, row_b, rows, a.stride, 1, kBK / 4);
  ok = ok && map_codes(&maps[7], shr + codes_off, row_b, rows, a.stride, 1, kBK / 8);
  if (!ok) return cudaErrorInvalidValue;
  P.K = K;
  P.m_tiles = rows / kBM;
  P.hi_col0 = K / 4;
  P.sc_row_bytes = K / kBlock * 2;
  P.scale_off = scales_off;

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctx.num_sms);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = PrefillSmem::kAlloc;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<BITS, DOWN>, maps[0], maps[1], maps[2], maps[3], maps[4],
                            maps[5], maps[6], maps[7], P);
}

template <int BITS>
cudaError_t run_ffn(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a, const int4* info, __half* xg,
                    __half* h16, float* z_rows, int n_pairs, int n_rows, cudaStream_t s) {
  GemmParams P{};
  P.tile_info = info;
  P.tile_offset = a.g->tile_offset;
  P.pair_gate = a.g->pair_gate;
  P.pool = a.pool;
  P.shared = a.shared;
  P.stride = a.stride;
  P.E = c.E;
  P.n_pairs = n_pairs;
  P.status = a.status;
  P.timeout_ns = ctx.timeout_ns;
  // gate/up: A = W_gu [2f, d], B = xg [n_rows, d] -> h16 [n_rows, f]
  P.out = h16;
  P.ld_out = c.f;
  cudaError_t e = run_pass<BITS, false>(ctx, a, P, xg, n_rows, c.d, 2 * c.f, a.lay.gu_codes, a.lay.gu_scales, s);
  if (e != cudaSuccess) return e;
  // down: A = W_d [d, f], B = h16 [n_rows, f] -> z_rows [n_rows, d]
  P.out = z_rows;
  P.ld_out = c.d;
  return run_pass<BITS, true>(ctx, a, P, h16, n_rows, c.f, c.d, a.lay.dn_codes, a.lay.dn_scales, s);
}

}  // namespace

bool prefill_geometry_ok(int d, int f) {
  return d % kBK == 0 && f % kBK == 0 && d % kBM == 0 && (2 * f) % kBM == 0 && d <= kMaxKDim && f <= kMaxKDim;
}

cudaError_t prefill_init(const Ctx& ctx) {
  (void)ctx;
  const void* fns[4] = {reinterpret_cast<const void*>(grouped_gemm_kernel<2, false>),
                        reinterpret_cast<const void*>(grouped_gemm_kernel<2, true>),
                        reinterpret_cast<const void*>(grouped_gemm_kernel<3, false>),
                        reinterpret_cast<const void*>(grouped_gemm_kernel<3, true>)};
  for (const void* fn : fns) {
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, PrefillSmem::kAlloc);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_ffn_prefill(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a, void* ws, float* z_rows,
                               cudaStream_t s) {
  if (!prefill_geometry_ok(c.d, c.f)) return cudaErrorNotSupported;
  cudaError_t e = get_encoder();
  if (e != cudaSuccess) return e;
  const WsLayout w = ws_layout(c, a.T);
  char* b = static_cast<char*>(ws);
  __half* xg = reinterpret_cast<__half*>(b + w.x16);
  __half* h16 = reinterpret_cast<__half*>(b + w.h);
  int4* info = reinterpret_cast<int4*>(b + w.tile_info);

  tile_table_kernel<<<(c.E + 1 + 255) / 256, 256, 0, s>>>(a.g->tile_offset, a.g->expert_offset, a.g->expert_count,
                                                           a.g->pair_slot, c.E, a.T, w.n_pairs, a.shared != nullptr,
                                                           info);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  gather_x_kernel<<<w.n_rows, 128, 0, s>>>(a.x, a.g->pair_token, w.n_pairs, w.n_rows, a.T, c.d, xg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return c.bits == 2 ? run_ffn<2>(ctx, c, a, info, xg, h16, z_rows, w.n_pairs, w.n_rows, s)
                     : run_ffn<3>(ctx, c, a, info, xg, h16, z_rows, w.n_pairs, w.n_rows, s);
}

}  // namespace moe
