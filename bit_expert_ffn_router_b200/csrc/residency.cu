// Dynamic expert residency on one device: usage tallies from the routing the
// decode and prefill calls leave in their workspaces, and exchanges of expert
// records between pool slots with the matching slot-table update.
//
// The pages' engine keeps the experts it uses most in GPU memory, chosen from
// usage statistics and swapped as a conversation goes on (vramglass.com,
// section その1：よく使うエキスパートを選んでGPUに置く; news.blueqat.app/post/3262,
// section GPU・CPU・RAM・SSDの分担). On one B200 every record is in HBM; the
// first n_hot slots of the pool stand for the hot set, and an exchange is a
// device-side copy of two records plus two slot-table entries.
#include <cuda_runtime.h>

#include "moe_internal.cuh"

namespace moe {
namespace {

// counts[l * E + e] += expert_count of layer l (one routing record per layer,
// rec_bytes apart). Each element has one owner: integer adds, no atomics.
__global__ void usage_count_kernel(const char* __restrict__ ws, size_t rec_bytes, size_t count_off, int L, int E,
                                   int32_t* __restrict__ counts) {
  const int n = L * E;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int l = i / E, e = i - l * E;
    const int32_t* ec = reinterpret_cast<const int32_t*>(ws + static_cast<size_t>(l) * rec_bytes + count_off);
    counts[i] += ec[e];
  }
}

// Pair i exchanges the records at slots slot_of[a_i] and slot_of[b_i] in
// 16-byte units; blockIdx.y is the pair. A slot outside [0, n_slots) is
// reported and the pair left alone.
__global__ void swap_records_kernel(uint8_t* __restrict__ pool, size_t stride, size_t units,
                                    const int32_t* __restrict__ slot_of, SwapBatch batch, int n_slots,
                                    int* status) {
  const int p = blockIdx.y;
  const int sa = slot_of[batch.a[p]], sb = slot_of[batch.b[p]];
  if (sa < 0 || sa >= n_slots || sb < 0 || sb >= n_slots) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, kDevBadSlot, batch.a[p]);
    return;
  }
  uint4* ra = reinterpret_cast<uint4*>(pool + static_cast<size_t>(sa) * stride);
  uint4* rb = reinterpret_cast<uint4*>(pool + static_cast<size_t>(sb) * stride);
  for (size_t u = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 va = ra[u], vb = rb[u];
    ra[u] = vb;
    rb[u] = va;
  }
}

// After the records moved: slot_of[a_i] <-> slot_of[b_i] (one thread per
// pair, in-range slots only, as the copy kernel did).
__global__ void swap_entries_kernel(int32_t* __restrict__ slot_of, SwapBatch batch, int n, int n_slots) {
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= n) return;
  const int sa = slot_of[batch.a[p]], sb = slot_of[batch.b[p]];
  if (sa < 0 || sa >= n_slots || sb < 0 || sb >= n_slots) return;
  slot_of[batch.a[p]] = sb;
  slot_of[batch.b[p]] = sa;
}

}  // namespace

cudaError_t launch_usage_count(const Ctx& ctx, const char* ws, size_t rec_bytes, size_t count_off, int L, int E,
                               int32_t* counts, cudaStream_t s) {
  const int n = L * E;
  const int threads = 256;
  int blocks = (n + threads - 1) / threads;
  if (blocks > 4 * ctx.num_sms) blocks = 4 * ctx.num_sms;
  usage_count_kernel<<<blocks, threads, 0, s>>>(ws, rec_bytes, count_off, L, E, counts);
  return cudaGetLastError();
}

cudaError_t launch_slot_swaps(const Ctx& ctx, uint8_t* pool, size_t stride, size_t record_bytes, int32_t* slot_of,
                              int n_slots, const SwapBatch& batch, int n, cudaStream_t s) {
  const size_t units = record_bytes / 16;
  // enough CTAs to keep every SM busy for a batch of any size
  int per_pair = (ctx.num_sms * 4 + n - 1) / n;
  if (per_pair < 1) per_pair = 1;
  const int max_per_pair = static_cast<int>((units + 255) / 256);
  if (per_pair > max_per_pair) per_pair = max_per_pair;
  swap_records_kernel<<<dim3(per_pair, n), 256, 0, s>>>(pool, stride, units, slot_of, batch, n_slots, ctx.d_status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  swap_entries_kernel<<<(n + 63) / 64, 64, 0, s>>>(slot_of, batch, n, n_slots);
  return cudaGetLastError();
}

}  // namespace moe
