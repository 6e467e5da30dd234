// Token -> expert grouping: a stable counting sort of the T*k (token, j)
// pairs by expert, with no atomics, plus the slot lookup through the expert
// slot table.
//
// The slot table is the indirection that stands for the pages' hot-expert
// cache: the engine keeps the most used ~4,500 experts of all layers in VRAM,
// chosen per expert rather than per layer (vramglass.com, section
// その1：よく使うエキスパートを選んでGPUに置く; bakeman.jp/archives/4749, section
// スパースMoEの局所性を活かすアプローチ). On one B200 every expert is in HBM and
// the table only maps an expert to its slot.
//
// Sorted order is (expert, token, j). Pairs are numbered p = t*k + j; within
// one expert they appear in ascending p, which is ascending token.
//
// slot_of[e] == kSlotAbsent marks an expert this device does not hold (expert
// parallelism): its pairs are left out of the sort (pair_pos = -1, count 0),
// so the sorted pairs, the unique experts and the tiles cover the held ones.
#include "moe_internal.cuh"

namespace moe {

constexpr int kSmallThreads = 1024;  // one thread per expert, E <= 1024
constexpr int kSmallMaxPairs = 512;  // the one-CTA path's limit on T*k

// Exclusive scan over the block (blockDim.x == 1024). Returns the exclusive
// prefix of v; *total receives the sum.
__device__ int block_exclusive_scan(int v, int* s_warp, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  __syncthreads();
  if (lane == 31) s_warp[w] = inc;
  __syncthreads();
  if (w == 0) {
    int x = s_warp[lane];
    int xi = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += n;
    }
    s_warp[lane] = xi - x;  // exclusive prefix of warp totals
    if (lane == 31) s_warp[32] = xi;
  }
  __syncthreads();
  const int r = s_warp[w] + inc - v;
  *total = s_warp[32];
  __syncthreads();
  return r;
}

// Fills the tile table of the prefill grouped GEMM: for every "extended"
// expert x (routed 0..E-1, shared = E), ceil(n_x / kTileN) token tiles;
// tile_offset[x] is the exclusive prefix, tile_offset[E+1] the total.
__device__ void write_tiles(int e, int count, int E, int T, int n_shared, int* s_warp,
                            int32_t* tile_offset) {
  int tiles = (e < E) ? (count + kTileN - 1) / kTileN : 0;
  int total;
  const int off = block_exclusive_scan(tiles, s_warp, &total);
  if (e < E) tile_offset[e] = off;
  if (threadIdx.x == 0) {
    const int sh = n_shared ? (T + kTileN - 1) / kTileN : 0;
    tile_offset[E] = total;
    tile_offset[E + 1] = total + sh;
  }
}

// Per-expert totals -> offsets, unique list, slot lookup, tiles. Thread e
// holds count (0 for e >= E); an absent expert's count becomes 0. Returns
// the expert's first sorted position.
__device__ int finish_counts(int e, int count, int E, int T, int n_shared, const int32_t* slot_of, int n_slots,
                             const GroupPtrs& g, int* s_warp, int* status, int* slot_out) {
  int slot = 0;
  if (e < E) {
    slot = slot_of[e];
    if (slot == kSlotAbsent) {
      count = 0;
    } else if (count > 0 && (slot < 0 || slot >= n_slots)) {
      report(status, kDevBadSlot, e);
      slot = 0;
    }
  }
  int total;
  const int off = block_exclusive_scan(count, s_warp, &total);
  int nu;
  const int u = block_exclusive_scan(count > 0 ? 1 : 0, s_warp, &nu);
  if (e < E) {
    g.expert_count[e] = count;
    g.expert_offset[e] = off;
    if (e == E - 1) g.expert_offset[E] = off + count;
    if (count > 0) {
      g.uniq_expert[u] = e;
      g.uniq_slot[u] = slot;
      g.uniq_offset[u] = off;
    }
  }
  if (threadIdx.x == 0) {
    *g.n_uniq = nu;
    g.uniq_offset[nu] = total;  // the sorted (held) pairs
  }
  write_tiles(e, count, E, T, n_shared, s_warp, g.tile_offset);
  *slot_out = slot;
  return off;
}

// The one mapping of an expert index every grouping pass applies: an index
// outside [0, E) is filed under expert 0 (and reported once, by the counting
// pass), so the counting and scatter passes agree on every pair's expert and
// the sorted positions stay a permutation of [0, T*k).
__device__ __forceinline__ int mapped_expert(int e, int E) { return (e < 0 || e >= E) ? 0 : e; }

__device__ __forceinline__ int checked_expert(int e, int E, int p, int* status) {
  if (e < 0 || e >= E) report(status, kDevBadExpert, p);
  return mapped_expert(e, E);
}

// ---------------------------------------------------------------- one CTA (small T*k)
__global__ void __launch_bounds__(kSmallThreads)
group_small_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, int T, int k,
                   int E, const int32_t* __restrict__ slot_of, int n_slots, int n_shared,
                   GroupPtrs g, int* status) {
  __shared__ int s_idx[kSmallMaxPairs];
  __shared__ int s_warp[33];
  const int n_pairs = T * k;
  const int e = threadIdx.x;
  for (int p = threadIdx.x; p < n_pairs; p += blockDim.x) s_idx[p] = checked_expert(idx[p], E, p, status);
  __syncthreads();
  int count = 0;
  if (e < E)
    for (int p = 0; p < n_pairs; ++p) count += (s_idx[p] == e);
  int slot;
  int r = finish_counts(e, count, E, T, n_shared, slot_of, n_slots, g, s_warp, status, &slot);
  const bool absent = e < E && slot_of[e] == kSlotAbsent;
  if (e < E && count > 0) {
    for (int p = 0; p < n_pairs; ++p) {
      if (s_idx[p] == e && absent) {
        g.pair_pos[p] = -1;
      } else if (s_idx[p] == e) {
        g.pair_token[r] = p / k;
        g.pair_j[r] = p % k;
        g.pair_gate[r] = gate[p];
        g.pair_slot[r] = slot;
        g.pair_pos[p] = r;
        ++r;
      }
    }
  }
}

// ---------------------------------------------------------------- many CTAs (large T*k)
// Phase 1 and 3 walk a chunk of kGroupChunk pairs with one warp, 32 pairs at a
// time in order. Lanes holding the same expert find each other with
// __match_any_sync; a pair's rank among equal experts in the chunk is the
// running count so far plus the number of matching lanes below it.
template <bool kScatter>
__global__ void __launch_bounds__(32)
group_chunk_kernel(const int32_t* __restrict__ idx, const float* __restrict__ gate, int n_pairs,
                   int k, int E, GroupPtrs g, const int32_t* __restrict__ slot_of, int n_slots,
                   int* status) {
  __shared__ int cnt[kMaxE];
  const int lane = threadIdx.x;
  const int c = blockIdx.x;
  for (int e = lane; e < E; e += 32) cnt[e] = 0;
  __syncwarp();
  const int p0 = c * kGroupChunk;
  const int p1 = min(p0 + kGroupChunk, n_pairs);
  const int32_t* base = g.chunk_hist + static_cast<size_t>(c) * E;
  for (int pb = p0; pb < p1; pb += 32) {
    const int p = pb + lane;
    const bool valid = p < p1;
    int e = -1;
    if (valid) e = kScatter ? mapped_expert(idx[p], E) : checked_expert(idx[p], E, p, status);
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    const int before = valid ? cnt[e] : 0;
    __syncwarp();
    if (valid && rank == 0) cnt[e] = before + __popc(peers);
    __syncwarp();
    if (kScatter && valid && slot_of[e] == kSlotAbsent) {
      g.pair_pos[p] = -1;
    } else if (kScatter && valid) {
      const int r = g.expert_offset[e] + base[e] + before + rank;
      int slot = slot_of[e];
      if (slot < 0 || slot >= n_slots) slot = 0;
      g.pair_token[r] = p / k;
      g.pair_j[r] = p % k;
      g.pair_gate[r] = gate[p];
      g.pair_slot[r] = slot;
      g.pair_pos[p] = r;
    }
  }
  if (!kScatter) {
    int32_t* out = g.chunk_hist + static_cast<size_t>(c) * E;
    for (int e = lane; e < E; e += 32) out[e] = cnt[e];
  }
}

// Phase 2: per expert, an exclusive scan over the chunks (in place: the
// histogram becomes each chunk's base inside the expert's segment), then the
// block-wide scan over experts.
__global__ void __launch_bounds__(kSmallThreads)
group_scan_kernel(int n_chunks, int T, int k, int E, const int32_t* __restrict__ slot_of,
                  int n_slots, int n_shared, GroupPtrs g, int* status) {
  __shared__ int s_warp[33];
  const int e = threadIdx.x;
  int running = 0;
  if (e < E) {
    for (int c = 0; c < n_chunks; ++c) {
      int32_t* h = g.chunk_hist + static_cast<size_t>(c) * E + e;
      const int v = *h;
      *h = running;
      running += v;
    }
  }
  int slot;
  finish_counts(e, running, E, T, n_shared, slot_of, n_slots, g, s_warp, status, &slot);
}

cudaError_t launch_group(const Ctx& ctx, const moe_layer_cfg& c, const int32_t* idx,
                         const float* gate, int T, const int32_t* slot_of, int n_slots,
                         const GroupPtrs& g, cudaStream_t s) {
  const int n_pairs = T * c.k;
  if (n_pairs <= kSmallMaxPairs) {
    group_small_kernel<<<1, kSmallThreads, 0, s>>>(idx, gate, T, c.k, c.E, slot_of, n_slots,
                                                   c.n_shared, g, ctx.d_status);
    return cudaGetLastError();
  }
  const int n_chunks = (n_pairs + kGroupChunk - 1) / kGroupChunk;
  group_chunk_kernel<false><<<n_chunks, 32, 0, s>>>(idx, gate, n_pairs, c.k, c.E, g, slot_of,
                                                    n_slots, ctx.d_status);
  group_scan_kernel<<<1, kSmallThreads, 0, s>>>(n_chunks, T, c.k, c.E, slot_of, n_slots,
                                                c.n_shared, g, ctx.d_status);
  group_chunk_kernel<true><<<n_chunks, 32, 0, s>>>(idx, gate, n_pairs, c.k, c.E, g, slot_of,
                                                   n_slots, ctx.d_status);
  return cudaGetLastError();
}

}  // namespace moe
