// Internal declarations shared by the libmoe translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/moe.h"

namespace moe {

// ---------------------------------------------------------------- constants

constexpr int kBlock = 32;            // weights per fp16 scale
constexpr int kMaxE = 1024;           // experts per layer
constexpr int kMaxK = 32;             // experts per token
constexpr int kSlotAbsent = -1;       // slot-table value of an expert this device does not hold
constexpr int kGroupChunk = 512;      // pairs per chunk in the multi-CTA grouping
constexpr int kTileN = 128;           // tokens per tile of the prefill grouped GEMM

// Device status word codes (word 0 holds the first error seen).
constexpr int kDevBadExpert = 1;
constexpr int kDevBadSlot = 2;
constexpr int kDevTimeout = 3;

struct Ctx {
  int device = 0;
  int num_sms = 0;
  int* d_status = nullptr;     // [4] ints: code, detail, spare, spare
  unsigned long long timeout_ns = 200ull * 1000 * 1000;  // limit of every device-side wait
  unsigned long long* d_trace = nullptr;  // phase timestamps (MOE_TRACE), kTraceSlots per CTA
  void* static_scratch = nullptr;  // device address of the static scratch (first static call)
  bool coop_pdl = false;
  int last_detail = 0;             // detail word of the last device error moe_check_device_status read           // a cooperative launch also takes programmatic serialization
};
constexpr int kTraceSlots = 64;
constexpr int kTraceCtas = 1024;

}  // namespace moe

// The opaque context handle of the C ABI.
struct moe_ctx {
  moe::Ctx c;
};

namespace moe {

// ---------------------------------------------------------------- workspace

// Workspace of one call: the routing record (what moe_layer_routing views)
// first, then the scratch of the path the call takes.
struct WsLayout {
  size_t logits, idx, gate;
  size_t expert_count, expert_offset, pair_token, pair_j, pair_gate, pair_slot, pair_pos;
  size_t uniq_expert, uniq_slot, uniq_offset, n_uniq;
  size_t rec_bytes;              // end of the routing record
  size_t chunk_hist, tile_offset;
  size_t exchange;               // decode path: the tagged-word exchange area
  size_t h, z, x16;              // prefill path
  size_t tile_info;              // prefill: int4 per token tile
  size_t total;
  int n_pairs, n_rows, n_chunks, n_uniq_max;
};

WsLayout ws_layout(const moe_layer_cfg& c, int T);

// Makes `device` current for the lifetime of the guard and then restores the
// caller's current device, so that no entry point leaves the host thread on
// another device than it found.
struct DeviceGuard {
  explicit DeviceGuard(int device);
  ~DeviceGuard();
  DeviceGuard(const DeviceGuard&) = delete;
  DeviceGuard& operator=(const DeviceGuard&) = delete;
  bool ok = false;
  bool switched = false;
  int prev = 0;
};

// Records a failed CUDA call as the host thread's last error (read by
// moe_last_cuda_error).
void record_cuda_error(cudaError_t e);

// ---------------------------------------------------------------- device helpers

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ void report(int* status, int code, int detail) {
  if (status != nullptr) {
    if (atomicCAS(status, 0, code) == 0) status[1] = detail;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sum over aligned groups of `width` lanes (width a power of two <= 32).
__device__ __forceinline__ float group_sum(float v, int width) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    if (o < width) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Four such sums at once (two float2), interleaved.
__device__ __forceinline__ void group_sum4(float2& a, float2& b, int width) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    if (o < width) {
      const float x0 = __shfl_xor_sync(0xffffffffu, a.x, o);
      const float x1 = __shfl_xor_sync(0xffffffffu, a.y, o);
      const float x2 = __shfl_xor_sync(0xffffffffu, b.x, o);
      const float x3 = __shfl_xor_sync(0xffffffffu, b.y, o);
      a.x += x0;
      a.y += x1;
      b.x += x2;
      b.y += x3;
    }
}

// Two such sums at once (interleaved, so their shuffle latencies overlap).
__device__ __forceinline__ float2 group_sum2(float2 v, int width) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    if (o < width) {
      const float a = __shfl_xor_sync(0xffffffffu, v.x, o);
      const float b = __shfl_xor_sync(0xffffffffu, v.y, o);
      v.x += a;
      v.y += b;
    }
  return v;
}

// Loads that bypass L1 (data written by an earlier kernel of the same stream).
__device__ __forceinline__ int ld_cg(const int* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }

// ---------------------------------------------------------------- launchers (host)

// router.cu
cudaError_t launch_router_logits(const Ctx& ctx, const moe_layer_cfg& c, const uint16_t* x,
                                 const float* wr, const float* bias, int T, float* logits,
                                 cudaStream_t s);
cudaError_t launch_topk(const Ctx& ctx, const moe_layer_cfg& c, const float* logits, int T,
                        int32_t* idx, float* gate, cudaStream_t s);

// group.cu
struct GroupPtrs {
  int32_t *expert_count, *expert_offset, *pair_token, *pair_j, *pair_slot, *pair_pos;
  float* pair_gate;
  int32_t *uniq_expert, *uniq_slot, *uniq_offset, *n_uniq;
  int32_t *chunk_hist, *tile_offset;
};
GroupPtrs group_ptrs(const moe_layer_cfg& c, int T, void* ws);
cudaError_t launch_group(const Ctx& ctx, const moe_layer_cfg& c, const int32_t* idx,
                         const float* gate, int T, const int32_t* slot_of, int n_slots,
                         const GroupPtrs& g, cudaStream_t s);

// decode_stack.cu
struct StackArgs {
  bool route;               // true: router + top-k + grouping run inside the kernel
  const uint16_t* x;        // [T, d] bf16: layer 0's input
  int T, L;                 // tokens, layers (L > 1 only with route)
  const float* wr;          // route: [L, E, d]
  const float* bias;        // route: [L, T, E] or null
  const int32_t* slot_of;   // route: [L, E]
  int n_slots;
  const uint8_t* pool;
  size_t stride;
  const uint8_t* shared;    // layer l's shared record at shared + l * stride, or null
  moe_expert_layout lay;
  void* y;                  // [L, T, d]
  char* rec;                // route: layer l's routing record at rec + l * rec_bytes
  size_t rec_bytes;
  int ro[14];               // offsets in a record: logits, idx, gate, expert_count, expert_offset,
                            // pair_token, pair_j, pair_gate, pair_slot, pair_pos, uniq_expert,
                            // uniq_slot, uniq_offset, n_uniq
  const GroupPtrs* g;       // not route: the given grouping
  char* exchange;           // decode_exchange_bytes(cfg, T) bytes, 256-byte aligned
};
cudaError_t launch_decode_stack(const Ctx& ctx, const moe_layer_cfg& c, const StackArgs& a, cudaStream_t s);
size_t decode_exchange_bytes(const moe_layer_cfg& c, int T);
// Moves the decode kernel's tag counter past an interrupted launch's tags.
cudaError_t decode_skip_tags(const Ctx& ctx, cudaStream_t s);
bool decode_geometry_ok(int d, int f);

// FFN arguments of the prefill path
struct FfnArgs {
  const uint16_t* x;        // [T, d] bf16
  int T;
  const GroupPtrs* g;
  const uint8_t* pool;
  size_t stride;
  const uint8_t* shared;    // record or null
  moe_expert_layout lay;
  void* h;
  void* y;
  int* status;
};

// ffn_prefill.cu
cudaError_t launch_ffn_prefill(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a,
                               void* ws, float* z_rows, cudaStream_t s);
cudaError_t prefill_init(const Ctx& ctx);
bool prefill_geometry_ok(int d, int f);

// combine.cu
cudaError_t launch_combine(const Ctx& ctx, const moe_layer_cfg& c, const int32_t* pair_pos,
                           int n_pairs, const float* z_rows, const uint16_t* x, int T, void* y,
                           cudaStream_t s);

// residency.cu: usage tallies and slot exchanges
constexpr int kSwapBatch = 64;  // exchanges per launch (passed by value)
struct SwapBatch {
  int32_t a[kSwapBatch], b[kSwapBatch];  // slot-table entries whose slots trade places
};
cudaError_t launch_usage_count(const Ctx& ctx, const char* ws, size_t rec_bytes, size_t count_off, int L, int E,
                               int32_t* counts, cudaStream_t s);
cudaError_t launch_slot_swaps(const Ctx& ctx, uint8_t* pool, size_t stride, size_t record_bytes, int32_t* slot_of,
                              int n_slots, const SwapBatch& batch, int n, cudaStream_t s);

// kernel attribute set-up, once per context
cudaError_t decode_init(Ctx& ctx);
cudaError_t router_init(const Ctx& ctx);

// router_tc.cu: prefill router logits on the tensor cores
bool router_tc_ok(const moe_layer_cfg& c);
cudaError_t launch_router_tc(const Ctx& ctx, const moe_layer_cfg& c, const uint16_t* x, const float* wr,
                             const float* bias, int T, float* logits, cudaStream_t s);
cudaError_t router_tc_init(const Ctx& ctx);

}  // namespace moe
