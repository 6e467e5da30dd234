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
// One persistent CTA per SM, ten warps:
//   warp 0     TMA producer: packed codes (3-D tensor maps over the whole
//              expert pool), fp16 scales (one bulk copy per tile) and the
//              activation tile (128B-swizzled, K-major);
//   warp 1     TMEM allocation and the single-thread tcgen05.mma issue;
//   warps 2-5  dequantisation: each thread owns one weight row and writes
//              s * (q - 2^(b-1)) as fp16 straight into the 128B-swizzled
//              K-major layout the tensor core reads;
//   warps 6-9  epilogue: tcgen05.ld of the fp32 accumulators (two TMEM
//              buffers, so the next tile's MMAs overlap this tile's stores).
// Operands are fp16 on both sides (A and B of one kind::f16 MMA share a
// type): 2-bit weights are exact in fp16, 3-bit ones round at 2^-12
// relative, bf16 activations convert exactly in fp16's normal range.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "moe_internal.cuh"
#include "ptx.cuh"

namespace moe {

namespace {

constexpr int kBM = 128;            // weight rows per tile (MMA M)
constexpr int kBN = kTileN;         // pairs per tile (MMA N, max)
constexpr int kBK = 64;             // K per pipeline stage (one 128-byte swizzle row of fp16)
constexpr int kChunk = 128;         // codes per code-chunk load (two stages)
constexpr int kKPerChunk = kChunk / kBK;
constexpr int kStages = 4;          // A/B ring depth
constexpr int kCStages = 4;         // code-chunk ring depth
constexpr int kThreads = 320;
constexpr int kTmemCols = 2 * kBN;  // two accumulator buffers
constexpr int kMaxKDim = 2048;      // largest reduction size (scale staging holds 128 x K/16 bytes)

struct PrefillSmem {
  // byte offsets from the 1024-aligned base of dynamic shared memory
  static constexpr int kA = 0;                                     // kStages x 16 KB, 128B-swizzled
  static constexpr int kB = kA + kStages * kBM * kBK * 2;          // kStages x 16 KB, 128B-swizzled
  static constexpr int kCodeLo = kB + kStages * kBN * kBK * 2;     // kCStages x (128 rows x 32 B)
  static constexpr int kCodeHi = kCodeLo + kCStages * kBM * (kChunk / 4);  // kCStages x (128 x 16 B)
  static constexpr int kScale = kCodeHi + kCStages * kBM * (kChunk / 8);   // 2 x (128 rows x K/16 B)
  static constexpr int kScaleBuf = kBM * (kMaxKDim / kBlock) * 2;
  static constexpr int kStage = kScale + 2 * kScaleBuf;            // epilogue staging 16 KB
  static constexpr int kBar = kStage + 16384;
  static constexpr int kBytes = kBar + 1024;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base
};

struct Bars {
  uint64_t ab_full_a[kStages];   // dequant -> MMA (count 128)
  uint64_t ab_full_b[kStages];   // TMA -> MMA (tx)
  uint64_t ab_empty[kStages];    // MMA commit -> producer, dequant
  uint64_t c_full[kCStages];     // TMA -> dequant (tx)
  uint64_t c_empty[kCStages];    // dequant -> producer (count 128)
  uint64_t s_full[2];            // bulk copy -> dequant (tx)
  uint64_t s_empty[2];           // dequant -> producer (count 128)
  uint64_t d_full[2];            // MMA commit -> epilogue
  uint64_t d_empty[2];           // epilogue -> MMA (count 128)
  uint64_t mma_done;             // final MMA commit, waited on before TMEM is freed
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 1024, "barrier block");

struct GemmParams {
  const int32_t* tile_offset;    // [E+2]
  const int32_t* expert_offset;  // [E+1]
  const int32_t* expert_count;   // [E]
  const int32_t* pair_slot;      // [n_pairs]
  const float* pair_gate;        // [n_pairs]
  const uint8_t* pool;           // scale sections are read with plain bulk copies
  const uint8_t* shared;         // shared-expert record (or null)
  size_t stride;
  size_t scale_off;              // section offset of this matrix's scales inside a record
  int E, T, n_pairs;
  int K, m_tiles;                // reduction size, weight-row tiles per expert
  int hi_col0;                   // byte column of the high plane in a code row (3-bit)
  int sc_row_bytes;              // fp16 scale bytes per weight row (K/16)
  void* out;                     // gate/up: h fp16 [n_rows, f]; down: z fp32 [n_rows, d]
  int ld_out;                    // elements per output row
  int* status;
  unsigned long long timeout_ns;
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled operand
// tile: rows of 128 bytes, 8-row atoms of 1024 bytes.
__device__ __forceinline__ uint64_t smem_desc(const void* p) {
  const uint64_t addr = smem_u32(p);
  uint64_t d = 0;
  d |= (addr >> 4) & 0x3FFFull;                // start address
  d |= uint64_t(16 >> 4) << 16;                // leading byte offset (not used by swizzled K-major)
  d |= uint64_t(1024 >> 4) << 32;              // stride byte offset: next 8-row atom
  d |= uint64_t(1) << 46;                      // descriptor version
  d |= uint64_t(2) << 61;                      // layout: 128-byte swizzle
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulator, fp16 A and B, both
// K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t instr_desc(int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(kBM >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// 32 lanes x 16 consecutive fp32 columns of the warp's TMEM lane quarter.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

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

// ------------------------------------------------------------------ work decoding
struct Item {
  int expert;  // 0..E-1 routed, E shared
  int row0;    // first sorted row of the tile
  int rows;    // valid rows (1..kBN)
  int slot;    // pool slot (routed experts)
  int m;       // weight-row tile
};

// Work item w = token tile * m_tiles + weight-row tile; consecutive items
// share a token tile, so CTAs running side by side read the same activation
// rows from L2 and different weight tiles.
__device__ __forceinline__ Item decode_item(const GemmParams& P, int w) {
  const int tile = w / P.m_tiles;
  Item it;
  it.m = w - tile * P.m_tiles;
  int lo = 0, hi = P.E;  // last extended expert x with tile_offset[x] <= tile
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(P.tile_offset + mid) <= tile) lo = mid;
    else hi = mid - 1;
  }
  it.expert = lo;
  const int ti = tile - __ldg(P.tile_offset + lo);
  const int base = lo < P.E ? __ldg(P.expert_offset + lo) : P.n_pairs;
  const int cnt = lo < P.E ? __ldg(P.expert_count + lo) : P.T;
  it.row0 = base + ti * kBN;
  it.rows = min(kBN, cnt - ti * kBN);
  it.slot = lo < P.E ? __ldg(P.pair_slot + it.row0) : 0;
  return it;
}

// ------------------------------------------------------------------ dequantisation of one K stage
// Thread r writes row r of the A tile: 64 weights s * (q - 2^(BITS-1)) as
// fp16, 16-byte chunk j of the row at chunk position j ^ (r % 8) (the
// 128-byte swizzle the descriptor names).
template <int BITS>
__device__ __forceinline__ void dequant_stage(uint8_t* a_tile, const uint8_t* lo, const uint8_t* hi,
                                              const uint16_t* sc, int r) {
  const uint4 w = *reinterpret_cast<const uint4*>(lo);  // 64 two-bit codes
  const uint32_t wl[4] = {w.x, w.y, w.z, w.w};
  uint2 hw = make_uint2(0u, 0u);
  if (BITS == 3) hw = *reinterpret_cast<const uint2*>(hi);  // their 64 high bits
  const uint32_t hb[2] = {hw.x, hw.y};
  const __half2 s0 = __half2half2(__ushort_as_half(sc[0]));
  const __half2 s1 = __half2half2(__ushort_as_half(sc[1]));
  // 0x6400 | q is the fp16 number 1024 + q; subtracting 1024 + 2^(BITS-1) is exact
  const __half2 off = __float2half2_rn(1024.f + static_cast<float>(1 << (BITS - 1)));
  uint8_t* row = a_tile + r * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j) {  // weights 8j .. 8j+7
    const uint32_t wd = wl[j >> 1] >> (16 * (j & 1));
    uint32_t hbits = 0;
    if (BITS == 3) hbits = (hb[j >> 2] >> (8 * (j & 3))) & 0xffu;
    uint32_t out[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {  // weights 8j+2p (low half), 8j+2p+1 (high half)
      uint32_t q = ((wd >> (4 * p)) & 0x3u) | (((wd >> (4 * p + 2)) & 0x3u) << 16);
      if (BITS == 3) q |= (((hbits >> (2 * p)) & 1u) << 2) | (((hbits >> (2 * p + 1)) & 1u) << 18);
      q |= 0x64006400u;
      const __half2 v = __hsub2(*reinterpret_cast<const __half2*>(&q), off);
      const __half2 y = __hmul2(v, (j < 4) ? s0 : s1);
      out[p] = *reinterpret_cast<const uint32_t*>(&y);
    }
    *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) * 16)) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// ------------------------------------------------------------------ the kernel
template <int BITS, bool DOWN>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_kernel(const __grid_constant__ CUtensorMap tB, const __grid_constant__ CUtensorMap tLo,
                    const __grid_constant__ CUtensorMap tHi, const __grid_constant__ CUtensorMap tLoS,
                    const __grid_constant__ CUtensorMap tHiS, const GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* B = reinterpret_cast<Bars*>(smem + PrefillSmem::kBar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&B->ab_full_a[i], 128);
      mbar_init(&B->ab_full_b[i], 1);
      mbar_init(&B->ab_empty[i], 1);
    }
    for (int i = 0; i < kCStages; ++i) {
      mbar_init(&B->c_full[i], 1);
      mbar_init(&B->c_empty[i], 128);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&B->s_full[i], 1);
      mbar_init(&B->s_empty[i], 128);
      mbar_init(&B->d_full[i], 1);
      mbar_init(&B->d_empty[i], 128);
    }
    mbar_init(&B->mma_done, 1);
    B->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {  // TMEM: two accumulator buffers of kBN fp32 columns
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
  const uint64_t deadline = P.timeout_ns;  // limit of each wait
  const int total = __ldg(P.tile_offset + P.E + 1) * P.m_tiles;
  const int ks_per_item = P.K / kBK;
  const int chunks_per_item = P.K / kChunk;
  const uint32_t code_tx = kBM * (kChunk / 4) + (BITS == 3 ? kBM * (kChunk / 8) : 0);
  const uint32_t scale_tx = kBM * P.sc_row_bytes;

  if (warp == 0) {
    // ---------------------------------------------------------- producer
    if (lane == 0) {
      int g = 0, gc = 0, it = 0;
      for (int w = blockIdx.x; w < total && !aborted(B); w += gridDim.x, ++it) {
        const Item I = decode_item(P, w);
        const bool sh = I.expert >= P.E;
        const CUtensorMap* mLo = sh ? &tLoS : &tLo;
        const CUtensorMap* mHi = sh ? &tHiS : &tHi;
        const int slot = sh ? 0 : I.slot;
        const uint8_t* rec = sh ? P.shared : P.pool + static_cast<size_t>(slot) * P.stride;
        const int sb = it & 1;
        if (it >= 2 && !wait_bar(B, &B->s_empty[sb], ((it >> 1) - 1) & 1, deadline, P.status, 1)) break;
        mbar_arrive_expect_tx(&B->s_full[sb], scale_tx);
        bulk_g2s(smem + PrefillSmem::kScale + sb * PrefillSmem::kScaleBuf,
                 rec + P.scale_off + static_cast<size_t>(I.m) * scale_tx, scale_tx, &B->s_full[sb]);
        bool ok = true;
        for (int c = 0; c < chunks_per_item && ok; ++c, ++gc) {
          const int cs = gc % kCStages;
          if (gc >= kCStages && !wait_bar(B, &B->c_empty[cs], ((gc / kCStages) - 1) & 1, deadline, P.status, 2)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&B->c_full[cs], code_tx);
          tma_load_3d(smem + PrefillSmem::kCodeLo + cs * kBM * (kChunk / 4), mLo, c * (kChunk / 4), I.m * kBM, slot,
                      &B->c_full[cs]);
          if (BITS == 3)
            tma_load_3d(smem + PrefillSmem::kCodeHi + cs * kBM * (kChunk / 8), mHi, P.hi_col0 + c * (kChunk / 8),
                        I.m * kBM, slot, &B->c_full[cs]);
          for (int k = 0; k < kKPerChunk; ++k, ++g) {
            const int st = g % kStages;
            if (g >= kStages && !wait_bar(B, &B->ab_empty[st], ((g / kStages) - 1) & 1, deadline, P.status, 3)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&B->ab_full_b[st], kBN * kBK * 2);
            tma_load_2d(smem + PrefillSmem::kB + st * kBN * kBK * 2, &tB, (c * kKPerChunk + k) * kBK, I.row0,
                        &B->ab_full_b[st]);
          }
        }
        if (!ok) break;
      }
      // Every copy this thread issued lands before the CTA may exit: wait
      // (bounded) for the last phase armed on each ring slot.
      const uint64_t drain = global_timer_ns() + P.timeout_ns;
      for (int n = max(0, g - kStages); n < g; ++n) mbar_wait(&B->ab_full_b[n % kStages], (n / kStages) & 1, drain);
      for (int n = max(0, gc - kCStages); n < gc; ++n) mbar_wait(&B->c_full[n % kCStages], (n / kCStages) & 1, drain);
      for (int n = max(0, it - 2); n < it; ++n) mbar_wait(&B->s_full[n & 1], (n >> 1) & 1, drain);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issue
    if (lane == 0) {
      int g = 0, it = 0;
      for (int w = blockIdx.x; w < total && !aborted(B); w += gridDim.x, ++it) {
        const Item I = decode_item(P, w);
        const int n = (I.rows + 15) / 16 * 16;
        const uint32_t idesc = instr_desc(n);
        const int acc = it & 1;
        if (it >= 2 && !wait_bar(B, &B->d_empty[acc], ((it >> 1) - 1) & 1, deadline, P.status, 4)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * kBN);
        bool ok = true;
        for (int k = 0; k < ks_per_item; ++k, ++g) {
          const int st = g % kStages;
          const uint32_t ph = (g / kStages) & 1;
          if (!wait_bar(B, &B->ab_full_a[st], ph, deadline, P.status, 5) ||
              !wait_bar(B, &B->ab_full_b[st], ph, deadline, P.status, 6)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = smem_desc(smem + PrefillSmem::kA + st * kBM * kBK * 2);
          const uint64_t db = smem_desc(smem + PrefillSmem::kB + st * kBN * kBK * 2);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)  // K = 16 per MMA: 32 bytes = 2 descriptor units
            tc_mma(d_tmem, da + 2 * kk, db + 2 * kk, idesc, (k > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&B->ab_empty[st]);
        }
        if (!ok) break;
        tc_commit(&B->d_full[acc]);
      }
      // all MMAs issued above complete before the tensor memory is freed
      tc_commit(&B->mma_done);
      mbar_wait(&B->mma_done, 0, global_timer_ns() + P.timeout_ns);
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------- dequantisation
    const int r = threadIdx.x - 64;  // weight row of the tile
    int g = 0, gc = 0, it = 0;
    for (int w = blockIdx.x; w < total && !aborted(B); w += gridDim.x, ++it) {
      const int sb = it & 1;
      if (!wait_bar(B, &B->s_full[sb], (it >> 1) & 1, deadline, P.status, 7)) break;
      const uint16_t* sc = reinterpret_cast<const uint16_t*>(smem + PrefillSmem::kScale + sb * PrefillSmem::kScaleBuf) +
                           r * (P.sc_row_bytes / 2);
      bool ok = true;
      for (int c = 0; c < chunks_per_item && ok; ++c, ++gc) {
        const int cs = gc % kCStages;
        if (!wait_bar(B, &B->c_full[cs], (gc / kCStages) & 1, deadline, P.status, 8)) {
          ok = false;
          break;
        }
        const uint8_t* lo = smem + PrefillSmem::kCodeLo + cs * kBM * (kChunk / 4) + r * (kChunk / 4);
        const uint8_t* hi = smem + PrefillSmem::kCodeHi + cs * kBM * (kChunk / 8) + r * (kChunk / 8);
        for (int k = 0; k < kKPerChunk; ++k, ++g) {
          const int st = g % kStages;
          if (g >= kStages && !wait_bar(B, &B->ab_empty[st], ((g / kStages) - 1) & 1, deadline, P.status, 9)) {
            ok = false;
            break;
          }
          const int kb = (c * kKPerChunk + k) * (kBK / kBlock);  // first scale block of the stage
          dequant_stage<BITS>(smem + PrefillSmem::kA + st * kBM * kBK * 2, lo + k * (kBK / 4), hi + k * (kBK / 8),
                              sc + kb, r);
          fence_proxy_async();  // generic-proxy writes -> visible to the tensor core
          mbar_arrive(&B->ab_full_a[st]);
        }
        mbar_arrive(&B->c_empty[cs]);
      }
      if (!ok) break;
      mbar_arrive(&B->s_empty[sb]);
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;       // accumulator lane = weight row of the tile
    const int et = threadIdx.x - 192;  // 0..127 among the epilogue threads
    int it = 0;
    for (int w = blockIdx.x; w < total && !aborted(B); w += gridDim.x, ++it) {
      const Item I = decode_item(P, w);
      const int acc = it & 1;
      if (!wait_bar(B, &B->d_full[acc], (it >> 1) & 1, deadline, P.status, 10)) break;
      tc_fence_after();
      const uint32_t base = tmem + static_cast<uint32_t>(acc * kBN) + (static_cast<uint32_t>(q * 32) << 16);
      if (!DOWN) {
        // channel m*64 + r/2: gate on the even lane, up on the odd one
        __half* hs = reinterpret_cast<__half*>(smem + PrefillSmem::kStage);  // [kBN pairs][64 channels]
        for (int c0 = 0; c0 < I.rows; c0 += 16) {
          float v[16];
          tmem_ld16(base + c0, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float u = __shfl_xor_sync(0xffffffffu, v[i], 1);
            if ((lane & 1) == 0 && c0 + i < I.rows)
              hs[(c0 + i) * 64 + (r >> 1)] = __float2half_rn(v[i] / (1.f + expf(-v[i])) * u);
          }
        }
        tc_fence_before();
        mbar_arrive(&B->d_empty[acc]);
        named_sync(2, 128);
        __half* out = static_cast<__half*>(P.out);
        for (int e = et; e < I.rows * 8; e += 128) {  // 128 bytes (64 channels) per pair row
          const int row = e >> 3, ch = (e & 7) * 8;
          *reinterpret_cast<uint4*>(out + static_cast<size_t>(I.row0 + row) * P.ld_out + I.m * 64 + ch) =
              *reinterpret_cast<const uint4*>(hs + row * 64 + ch);
        }
        named_sync(2, 128);
      } else {
        // output dim m*128 + r, 32 pairs at a time through the staging tile
        float* zs = reinterpret_cast<float*>(smem + PrefillSmem::kStage);  // [32 pairs][128 dims]
        float* out = static_cast<float*>(P.out);
        for (int c0 = 0; c0 < I.rows; c0 += 32) {
          float v[32];
          tmem_ld16(base + c0, v);
          tmem_ld16(base + c0 + 16, v + 16);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int p = I.row0 + c0 + i;
            const float gt = (c0 + i < I.rows && p < P.n_pairs) ? __ldg(P.pair_gate + p) : 1.f;
            zs[i * 128 + r] = gt * v[i];
          }
          named_sync(2, 128);
          const int nrow = min(32, I.rows - c0);
          for (int e = et; e < nrow * 32; e += 128) {
            const int row = e >> 5, col = (e & 31) * 4;
            *reinterpret_cast<float4*>(out + static_cast<size_t>(I.row0 + c0 + row) * P.ld_out + I.m * kBM + col) =
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
// shared expert's rows, token r - n_pairs.
__global__ void __launch_bounds__(256) gather_x_kernel(const uint16_t* __restrict__ x,
                                                       const int32_t* __restrict__ pair_token, int n_pairs,
                                                       int n_rows, int d, __half* __restrict__ xg) {
  const int r = blockIdx.x;
  if (r >= n_rows) return;
  const int t = r < n_pairs ? __ldg(pair_token + r) : r - n_pairs;
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * d);
  uint4* dst = reinterpret_cast<uint4*>(xg + static_cast<size_t>(r) * d);
  for (int i = threadIdx.x; i < d / 8; i += blockDim.x) {
    const uint4 v = __ldg(src + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h = __floats2half2_rn(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xffff0000u));
      o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
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

// 2-D fp16 activation tensor [rows][K], boxes of 64 x 128 with the 128-byte
// swizzle; rows past the end read as zeros.
bool map_act(CUtensorMap* m, const __half* base, int K, int rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(kBN)};
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
  CUtensorMap maps[5];
  bool ok = map_act(&maps[0], act, K, n_rows);
  ok = ok && map_codes(&maps[1], a.pool + codes_off, row_b, rows, a.stride, kMapSlots, kChunk / 4);
  ok = ok && map_codes(&maps[2], a.pool + codes_off, row_b, rows, a.stride, kMapSlots, kChunk / 8);
  ok = ok && map_codes(&maps[3], shr + codes_off, row_b, rows, a.stride, 1, kChunk / 4);
  ok = ok && map_codes(&maps[4], shr + codes_off, row_b, rows, a.stride, 1, kChunk / 8);
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
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<BITS, DOWN>, maps[0], maps[1], maps[2], maps[3], maps[4], P);
}

template <int BITS>
cudaError_t run_ffn(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a, __half* xg, __half* h16,
                    float* z_rows, int n_pairs, int n_rows, cudaStream_t s) {
  GemmParams P{};
  P.tile_offset = a.g->tile_offset;
  P.expert_offset = a.g->expert_offset;
  P.expert_count = a.g->expert_count;
  P.pair_slot = a.g->pair_slot;
  P.pair_gate = a.g->pair_gate;
  P.pool = a.pool;
  P.shared = a.shared;
  P.stride = a.stride;
  P.E = c.E;
  P.T = a.T;
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
  return d % kChunk == 0 && f % kChunk == 0 && d % kBM == 0 && (2 * f) % kBM == 0 && d <= kMaxKDim &&
         f <= kMaxKDim;
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

  gather_x_kernel<<<w.n_rows, 256, 0, s>>>(a.x, a.g->pair_token, w.n_pairs, w.n_rows, c.d, xg);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return c.bits == 2 ? run_ffn<2>(ctx, c, a, xg, h16, z_rows, w.n_pairs, w.n_rows, s)
                     : run_ffn<3>(ctx, c, a, xg, h16, z_rows, w.n_pairs, w.n_rows, s);
}

}  // namespace moe
