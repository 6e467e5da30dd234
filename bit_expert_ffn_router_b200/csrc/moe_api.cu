// C ABI of libmoe: argument checks, workspace carving and kernel launches.
// Every compute entry point is asynchronous on the caller's stream and
// allocates nothing; see include/moe.h for the contract of each call.
#include <algorithm>
#include <cstdlib>
#include <new>
#include <vector>

#include "moe_internal.cuh"

namespace moe {

static size_t align_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

WsLayout ws_layout(const moe_layer_cfg& c, int T) {
  WsLayout w{};
  const size_t Tz = static_cast<size_t>(T);
  w.n_pairs = T * c.k;
  w.n_rows = w.n_pairs + (c.n_shared ? T : 0);
  w.n_chunks = (w.n_pairs + kGroupChunk - 1) / kGroupChunk;
  w.n_uniq_max = w.n_pairs < c.E ? w.n_pairs : c.E;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  // routing record
  w.logits = take(Tz * c.E * 4);
  w.idx = take(Tz * c.k * 4);
  w.gate = take(Tz * c.k * 4);
  w.expert_count = take(static_cast<size_t>(c.E) * 4);
  w.expert_offset = take((static_cast<size_t>(c.E) + 1) * 4);
  w.pair_token = take(static_cast<size_t>(w.n_pairs) * 4);
  w.pair_j = take(static_cast<size_t>(w.n_pairs) * 4);
  w.pair_gate = take(static_cast<size_t>(w.n_pairs) * 4);
  w.pair_slot = take(static_cast<size_t>(w.n_pairs) * 4);
  w.pair_pos = take(static_cast<size_t>(w.n_pairs) * 4);
  w.uniq_expert = take(static_cast<size_t>(w.n_uniq_max) * 4);
  w.uniq_slot = take(static_cast<size_t>(w.n_uniq_max) * 4);
  w.uniq_offset = take((static_cast<size_t>(w.n_uniq_max) + 1) * 4);
  w.n_uniq = take(16);
  w.rec_bytes = o;
  // grouping kernels' scratch
  w.chunk_hist = take(static_cast<size_t>(w.n_chunks) * c.E * 4);
  w.tile_offset = take((static_cast<size_t>(c.E) + 2) * 4);
  if (T <= MOE_DECODE_MAX_T) {
    w.exchange = take(decode_exchange_bytes(c, T));
  } else {
    // h: fp16 rows padded by one tile; z: the fp32 pair buffer; x gathered
    // into pair order as fp16 (the grouped GEMM's operand)
    w.h = take((static_cast<size_t>(w.n_rows) + kTileN) * c.f * 2);
    w.z = take(static_cast<size_t>(w.n_rows) * c.d * 4);
    w.x16 = take(static_cast<size_t>(w.n_rows) * c.d * 2);
    w.tile_info = take((static_cast<size_t>(w.n_rows) / kTileN + c.E + 2) * 16);
  }
  w.total = o;
  return w;
}

GroupPtrs group_ptrs(const moe_layer_cfg& c, int T, void* ws) {
  const WsLayout w = ws_layout(c, T);
  char* b = static_cast<char*>(ws);
  GroupPtrs g;
  g.expert_count = reinterpret_cast<int32_t*>(b + w.expert_count);
  g.expert_offset = reinterpret_cast<int32_t*>(b + w.expert_offset);
  g.pair_token = reinterpret_cast<int32_t*>(b + w.pair_token);
  g.pair_j = reinterpret_cast<int32_t*>(b + w.pair_j);
  g.pair_gate = reinterpret_cast<float*>(b + w.pair_gate);
  g.pair_slot = reinterpret_cast<int32_t*>(b + w.pair_slot);
  g.pair_pos = reinterpret_cast<int32_t*>(b + w.pair_pos);
  g.uniq_expert = reinterpret_cast<int32_t*>(b + w.uniq_expert);
  g.uniq_slot = reinterpret_cast<int32_t*>(b + w.uniq_slot);
  g.uniq_offset = reinterpret_cast<int32_t*>(b + w.uniq_offset);
  g.n_uniq = reinterpret_cast<int32_t*>(b + w.n_uniq);
  g.chunk_hist = reinterpret_cast<int32_t*>(b + w.chunk_hist);
  g.tile_offset = reinterpret_cast<int32_t*>(b + w.tile_offset);
  return g;
}

static moe_status check_cfg(const moe_layer_cfg* c) {
  if (c == nullptr) return MOE_EINVAL;
  if (c->bits != 2 && c->bits != 3) return MOE_EUNSUPPORTED;
  if (c->block != kBlock) return MOE_EUNSUPPORTED;
  if (c->d <= 0 || c->f <= 0 || c->E <= 0 || c->k <= 0) return MOE_EINVAL;
  if (c->k > c->E || c->k > kMaxK) return MOE_EINVAL;
  if (c->E > kMaxE) return MOE_EUNSUPPORTED;
  if (c->n_shared != 0 && c->n_shared != 1) return MOE_EUNSUPPORTED;
  if (c->skip_from < 0 || c->skip_from > c->k || c->hot_slots < 0) return MOE_EINVAL;
  if (c->d % 128 != 0 || c->f % 64 != 0 || c->d > 4096 || c->f > 4096) return MOE_EUNSUPPORTED;
  if (!decode_geometry_ok(c->d, c->f)) return MOE_EUNSUPPORTED;
  return MOE_OK;
}

// The entry points outside the fused decode kernel do not skip experts.
static moe_status check_cfg_unskipped(const moe_layer_cfg* c) {
  const moe_status st = check_cfg(c);
  if (st != MOE_OK) return st;
  return c->skip_from != 0 ? MOE_EUNSUPPORTED : MOE_OK;
}

static bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

static thread_local cudaError_t g_last_cuda_error = cudaSuccess;

void record_cuda_error(cudaError_t e) {
  if (e != cudaSuccess) g_last_cuda_error = e;
}

static moe_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return MOE_OK;
  g_last_cuda_error = e;
  return MOE_ECUDA;
}

DeviceGuard::DeviceGuard(int device) {
  cudaError_t e = cudaGetDevice(&prev);
  if (e == cudaSuccess && prev != device) {
    e = cudaSetDevice(device);
    switched = e == cudaSuccess;
  }
  ok = e == cudaSuccess;
  record_cuda_error(e);
}

DeviceGuard::~DeviceGuard() {
  if (switched) cudaSetDevice(prev);
}

static moe_expert_layout layout_of(const moe_layer_cfg& c) {
  moe_expert_layout l;
  const size_t gu_row = static_cast<size_t>(c.d) * c.bits / 8;
  const size_t dn_row = static_cast<size_t>(c.f) * c.bits / 8;
  size_t o = 0;
  l.gu_codes = o;
  o = align_up(o + 2 * static_cast<size_t>(c.f) * gu_row, 256);
  l.dn_codes = o;
  o = align_up(o + static_cast<size_t>(c.d) * dn_row, 256);
  l.gu_scales = o;
  o = align_up(o + 2 * static_cast<size_t>(c.f) * (c.d / kBlock) * 2, 256);
  l.dn_scales = o;
  o = align_up(o + static_cast<size_t>(c.d) * (c.f / kBlock) * 2, 256);
  l.bytes = o;
  return l;
}

static moe_status check_pool(const moe_layer_cfg& c, const uint8_t* pool, size_t stride,
                             const uint8_t* shared) {
  const moe_expert_layout l = layout_of(c);
  if (pool == nullptr || !aligned(pool, 256) || stride % 256 != 0 || stride < l.bytes)
    return MOE_EINVAL;
  if (c.n_shared && (shared == nullptr || !aligned(shared, 256))) return MOE_EINVAL;
  return MOE_OK;
}

static moe_status fill_grouping(const moe_layer_cfg& c, int T, void* ws, moe_grouping* out) {
  const WsLayout w = ws_layout(c, T);
  const GroupPtrs g = group_ptrs(c, T, ws);
  out->T = T;
  out->k = c.k;
  out->E = c.E;
  out->n_pairs = w.n_pairs;
  out->n_rows = w.n_rows;
  out->expert_count = g.expert_count;
  out->expert_offset = g.expert_offset;
  out->pair_token = g.pair_token;
  out->pair_j = g.pair_j;
  out->pair_gate = g.pair_gate;
  out->pair_slot = g.pair_slot;
  out->pair_pos = g.pair_pos;
  out->uniq_expert = g.uniq_expert;
  out->uniq_slot = g.uniq_slot;
  out->uniq_offset = g.uniq_offset;
  out->n_uniq = g.n_uniq;
  out->internal = ws;
  return MOE_OK;
}

static moe_status run_ffn(moe_ctx* ctx, const moe_layer_cfg* cfg, int bits, const void* x,
                          const moe_grouping* grp, const uint8_t* pool, size_t stride,
                          const uint8_t* shared, void* ws, size_t ws_bytes, float* z_rows,
                          void* y, moe_stream stream) {
  if (ctx == nullptr || grp == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg_unskipped(cfg);
  if (st != MOE_OK) return st;
  if (cfg->bits != bits) return MOE_EINVAL;
  const int T = grp->T;
  if (T < 0 || grp->k != cfg->k || grp->E != cfg->E) return MOE_EINVAL;
  if (T == 0) return MOE_OK;
  if (ws == nullptr || grp->internal != ws) return MOE_EINVAL;
  if (ws_bytes < ws_layout(*cfg, T).total) return MOE_ENOSPACE;
  if ((st = check_pool(*cfg, pool, stride, shared)) != MOE_OK) return st;
  if (x == nullptr || !aligned(x, 16)) return MOE_EINVAL;
  const GroupPtrs g = group_ptrs(*cfg, T, ws);
  const WsLayout w = ws_layout(*cfg, T);
  FfnArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.T = T;
  a.g = &g;
  a.pool = pool;
  a.stride = stride;
  a.shared = cfg->n_shared ? shared : nullptr;
  a.lay = layout_of(*cfg);
  a.h = static_cast<char*>(ws) + w.h;
  a.y = y;
  a.status = ctx->c.d_status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (z_rows == nullptr) {
    if (T > MOE_DECODE_MAX_T || y == nullptr || !aligned(y, 16)) return MOE_EINVAL;
    StackArgs d{};
    d.route = false;
    d.x = a.x;
    d.T = T;
    d.L = 1;
    d.n_slots = 0x7fffffff;
    d.g = &g;
    d.pool = pool;
    d.stride = stride;
    d.shared = a.shared;
    d.lay = a.lay;
    d.y = y;
    d.exchange = static_cast<char*>(ws) + w.exchange;
    const cudaError_t e = launch_decode_stack(ctx->c, *cfg, d, s);
    if (e == cudaErrorNotSupported) return MOE_EUNSUPPORTED;
    return from_cuda(e);
  }
  if (!aligned(z_rows, 16)) return MOE_EINVAL;
  const cudaError_t e = launch_ffn_prefill(ctx->c, *cfg, a, ws, z_rows, s);
  if (e == cudaErrorNotSupported) return MOE_EUNSUPPORTED;
  return from_cuda(e);
}

// The fused decode kernel over L chained layers (L = 1: moe_layer_forward).
// Arguments are checked by the caller; ws holds L routing records followed
// by the rest of a one-layer workspace.
static moe_status run_stack(moe_ctx* ctx, const moe_layer_cfg& c, int L, const void* x, int T,
                            const float* w_router, const float* logit_bias, const int32_t* slot_of,
                            int n_slots, const uint8_t* pool, size_t stride, const uint8_t* shared, void* ws,
                            void* y, moe_stream stream) {
  const WsLayout w = ws_layout(c, T);
  char* b = static_cast<char*>(ws);
  StackArgs d{};
  d.route = true;
  d.x = static_cast<const uint16_t*>(x);
  d.T = T;
  d.L = L;
  d.wr = w_router;
  d.bias = logit_bias;
  d.slot_of = slot_of;
  d.n_slots = n_slots;
  d.pool = pool;
  d.stride = stride;
  d.shared = c.n_shared ? shared : nullptr;
  d.lay = layout_of(c);
  d.y = y;
  d.rec = b;
  d.rec_bytes = w.rec_bytes;
  const size_t offs[14] = {w.logits, w.idx, w.gate, w.expert_count, w.expert_offset, w.pair_token, w.pair_j,
                           w.pair_gate, w.pair_slot, w.pair_pos, w.uniq_expert, w.uniq_slot, w.uniq_offset,
                           w.n_uniq};
  for (int i = 0; i < 14; ++i) d.ro[i] = static_cast<int>(offs[i]);
  d.exchange = b + static_cast<size_t>(L - 1) * w.rec_bytes + w.exchange;
  const cudaError_t e = launch_decode_stack(ctx->c, c, d, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return MOE_EUNSUPPORTED;
  return from_cuda(e);
}

static moe_status fill_routing(const moe_layer_cfg& c, int T, void* rec, moe_routing* out) {
  const WsLayout w = ws_layout(c, T);
  char* b = static_cast<char*>(rec);
  out->T = T;
  out->k = c.k;
  out->E = c.E;
  out->logits = reinterpret_cast<float*>(b + w.logits);
  out->idx = reinterpret_cast<int32_t*>(b + w.idx);
  out->gate = reinterpret_cast<float*>(b + w.gate);
  return fill_grouping(c, T, rec, &out->grouping);
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_ctx_create(int device, moe_ctx** out) {
  if (out == nullptr || device < 0) return MOE_EINVAL;
  *out = nullptr;
  moe_ctx* ctx = new (std::nothrow) moe_ctx;
  if (ctx == nullptr) return MOE_EINVAL;
  ctx->c.device = device;
  DeviceGuard dg(device);
  if (!dg.ok ||
      cudaDeviceGetAttribute(&ctx->c.num_sms, cudaDevAttrMultiProcessorCount, ctx->c.device) !=
          cudaSuccess ||
      cudaMalloc(&ctx->c.d_status, 64) != cudaSuccess) {
    delete ctx;
    return MOE_ECUDA;
  }
  // limit of every device-side wait (default 200 ms): MOE_TIMEOUT_US overrides it
  if (const char* t = getenv("MOE_TIMEOUT_US")) {
    const long long us = atoll(t);
    if (us > 0) ctx->c.timeout_ns = static_cast<unsigned long long>(us) * 1000ull;
  }
  if (getenv("MOE_TRACE") != nullptr) {
    const size_t n = static_cast<size_t>(kTraceCtas) * kTraceSlots * sizeof(unsigned long long);
    if (cudaMalloc(&ctx->c.d_trace, n) != cudaSuccess || cudaMemset(ctx->c.d_trace, 0, n) != cudaSuccess) {
      cudaFree(ctx->c.d_status);
      delete ctx;
      return MOE_ECUDA;
    }
  }
  if (cudaMemset(ctx->c.d_status, 0, 64) != cudaSuccess || router_init(ctx->c) != cudaSuccess || router_tc_init(ctx->c) != cudaSuccess ||
      decode_init(ctx->c) != cudaSuccess || prefill_init(ctx->c) != cudaSuccess) {
    cudaFree(ctx->c.d_status);
    delete ctx;
    return MOE_ECUDA;
  }
  *out = ctx;
  return MOE_OK;
}

void moe_ctx_destroy(moe_ctx* ctx) {
  if (ctx == nullptr) return;
  DeviceGuard dg(ctx->c.device);
  if (ctx->c.d_trace != nullptr) cudaFree(ctx->c.d_trace);
  cudaFree(ctx->c.d_status);
  delete ctx;
}

const char* moe_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda_error); }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument";
    case MOE_EUNSUPPORTED: return "unsupported configuration";
    case MOE_ECUDA: return "CUDA error";
    case MOE_ETIMEOUT: return "device wait timed out";
    case MOE_EDEVICE: return "kernel saw an out-of-range expert or slot index";
    case MOE_ENOSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

moe_status moe_check_device_status(moe_ctx* ctx, moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  int h[4] = {0, 0, 0, 0};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(h, ctx->c.d_status, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ECUDA;
  if (h[0] == 0) return MOE_OK;
  ctx->c.last_detail = h[1];
  // clear the status word, and move the decode kernel's tag counter past any
  // tag an interrupted launch may have written
  if (cudaMemsetAsync(ctx->c.d_status, 0, 64, s) != cudaSuccess || decode_skip_tags(ctx->c, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ECUDA;
  return h[0] == kDevTimeout ? MOE_ETIMEOUT : MOE_EDEVICE;
}

int moe_last_device_error_detail(const moe_ctx* ctx) { return ctx == nullptr ? 0 : ctx->c.last_detail; }

moe_status moe_trace_fetch(moe_ctx* ctx, unsigned long long* host, int n, moe_stream stream) {
  if (ctx == nullptr || host == nullptr || n < 0) return MOE_EINVAL;
  if (ctx->c.d_trace == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  const int cap = kTraceCtas * kTraceSlots;
  const size_t bytes = static_cast<size_t>(n < cap ? n : cap) * sizeof(unsigned long long);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host, ctx->c.d_trace, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaMemsetAsync(ctx->c.d_trace, 0, static_cast<size_t>(cap) * sizeof(unsigned long long), s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return from_cuda(cudaGetLastError());
  return MOE_OK;
}

moe_status moe_layer_routing(const moe_layer_cfg* cfg, int T, void* ws, size_t ws_bytes, moe_routing* out) {
  if (out == nullptr) return MOE_EINVAL;
  const moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || ws == nullptr || !aligned(ws, 256)) return MOE_EINVAL;
  if (ws_bytes < ws_layout(*cfg, T).rec_bytes) return MOE_ENOSPACE;
  return fill_routing(*cfg, T, ws, out);
}

size_t moe_stack_workspace_bytes(const moe_layer_cfg* cfg, int L, int T) {
  if (check_cfg(cfg) != MOE_OK || L < 1 || T < 0 || T > MOE_DECODE_MAX_T) return 0;
  const WsLayout w = ws_layout(*cfg, T);
  return static_cast<size_t>(L - 1) * w.rec_bytes + w.total;
}

moe_status moe_stack_routing(const moe_layer_cfg* cfg, int L, int T, void* ws, size_t ws_bytes, int layer,
                             moe_routing* out) {
  if (out == nullptr) return MOE_EINVAL;
  const moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (L < 1 || layer < 0 || layer >= L || T < 0 || T > MOE_DECODE_MAX_T) return MOE_EINVAL;
  if (ws == nullptr || !aligned(ws, 256)) return MOE_EINVAL;
  if (ws_bytes < moe_stack_workspace_bytes(cfg, L, T)) return MOE_ENOSPACE;
  const WsLayout w = ws_layout(*cfg, T);
  return fill_routing(*cfg, T, static_cast<char*>(ws) + static_cast<size_t>(layer) * w.rec_bytes, out);
}

moe_status moe_stack_forward(moe_ctx* ctx, const moe_layer_cfg* cfg, int L, const void* x, int T,
                             const float* w_router, const float* logit_bias, const int32_t* slot_of, int n_slots,
                             const uint8_t* slot_pool, size_t slot_stride, const uint8_t* shared_experts,
                             void* ws, size_t ws_bytes, void* y, moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (L < 1 || T < 0 || T > MOE_DECODE_MAX_T || n_slots <= 0) return MOE_EINVAL;
  if (cfg->E > 512) return MOE_EUNSUPPORTED;
  if (L > 1 && cfg->out_fp32) return MOE_EINVAL;  // layer l + 1 reads layer l's bf16 output
  if (T == 0) return MOE_OK;
  if (x == nullptr || w_router == nullptr || slot_of == nullptr || y == nullptr) return MOE_EINVAL;
  if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(y, 16)) return MOE_EINVAL;
  if (ws == nullptr || !aligned(ws, 256)) return MOE_EINVAL;
  if (ws_bytes < moe_stack_workspace_bytes(cfg, L, T)) return MOE_ENOSPACE;
  if ((st = check_pool(*cfg, slot_pool, slot_stride, shared_experts)) != MOE_OK) return st;
  return run_stack(ctx, *cfg, L, x, T, w_router, logit_bias, slot_of, n_slots, slot_pool, slot_stride,
                   shared_experts, ws, y, stream);
}

moe_status moe_usage_count(moe_ctx* ctx, const moe_layer_cfg* cfg, int L, int T, const void* ws, size_t ws_bytes,
                           int32_t* counts, moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  const moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (L < 1 || T < 0 || (L > 1 && T > MOE_DECODE_MAX_T)) return MOE_EINVAL;
  if (ws == nullptr || !aligned(ws, 256) || counts == nullptr || !aligned(counts, 4)) return MOE_EINVAL;
  const WsLayout w = ws_layout(*cfg, T);
  if (ws_bytes < static_cast<size_t>(L - 1) * w.rec_bytes + w.rec_bytes) return MOE_ENOSPACE;
  if (T == 0) return MOE_OK;
  return from_cuda(launch_usage_count(ctx->c, static_cast<const char*>(ws), w.rec_bytes, w.expert_count, L,
                                      cfg->E, counts, static_cast<cudaStream_t>(stream)));
}

moe_status moe_slot_swap(moe_ctx* ctx, const moe_layer_cfg* cfg, uint8_t* slot_pool, size_t slot_stride,
                         int32_t* slot_of, int n_entries, int n_slots, const int32_t* a, const int32_t* b, int n,
                         moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  const moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (n < 0 || n_entries <= 0 || n_slots <= 0) return MOE_EINVAL;
  if (n == 0) return MOE_OK;
  if (slot_pool == nullptr || slot_of == nullptr || a == nullptr || b == nullptr) return MOE_EINVAL;
  const size_t rec = layout_of(*cfg).bytes;
  if (!aligned(slot_pool, 256) || !aligned(slot_of, 4) || slot_stride % 256 != 0 || slot_stride < rec)
    return MOE_EINVAL;
  // every entry in range, the 2n entries distinct (each exchange owns its two slots)
  std::vector<int32_t> all;
  all.reserve(2 * static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    if (a[i] < 0 || a[i] >= n_entries || b[i] < 0 || b[i] >= n_entries) return MOE_EINVAL;
    all.push_back(a[i]);
    all.push_back(b[i]);
  }
  std::sort(all.begin(), all.end());
  if (std::adjacent_find(all.begin(), all.end()) != all.end()) return MOE_EINVAL;
  for (int i0 = 0; i0 < n; i0 += kSwapBatch) {
    SwapBatch batch;
    const int m = std::min(kSwapBatch, n - i0);
    for (int i = 0; i < m; ++i) {
      batch.a[i] = a[i0 + i];
      batch.b[i] = b[i0 + i];
    }
    for (int i = m; i < kSwapBatch; ++i) batch.a[i] = batch.b[i] = 0;
    const cudaError_t e = launch_slot_swaps(ctx->c, slot_pool, slot_stride, rec, slot_of, n_slots, batch, m,
                                            static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return from_cuda(e);
  }
  return MOE_OK;
}

moe_status moe_expert_layout_get(const moe_layer_cfg* cfg, moe_expert_layout* out) {
  if (out == nullptr) return MOE_EINVAL;
  const moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  *out = layout_of(*cfg);
  return MOE_OK;
}

size_t moe_workspace_bytes(const moe_layer_cfg* cfg, int T) {
  if (check_cfg(cfg) != MOE_OK || T < 0) return 0;
  return ws_layout(*cfg, T).total;
}

moe_status moe_router_topk(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x,
                           const float* w_router, const float* logit_bias, int T, float* logits,
                           int32_t* idx, float* gate, moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg_unskipped(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_EINVAL;
  if (T == 0) return MOE_OK;
  if (x == nullptr || w_router == nullptr || logits == nullptr || idx == nullptr || gate == nullptr)
    return MOE_EINVAL;
  if (!aligned(x, 16) || !aligned(w_router, 16)) return MOE_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_router_logits(ctx->c, *cfg, static_cast<const uint16_t*>(x), w_router,
                                       logit_bias, T, logits, s);
  if (e != cudaSuccess) return MOE_ECUDA;
  return from_cuda(launch_topk(ctx->c, *cfg, logits, T, idx, gate, s));
}

moe_status moe_topk(moe_ctx* ctx, const moe_layer_cfg* cfg, const float* logits, int T,
                    int32_t* idx, float* gate, moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg_unskipped(cfg);
  if (st != MOE_OK) return st;
  if (T < 0) return MOE_EINVAL;
  if (T == 0) return MOE_OK;
  if (logits == nullptr || idx == nullptr || gate == nullptr) return MOE_EINVAL;
  return from_cuda(launch_topk(ctx->c, *cfg, logits, T, idx, gate, static_cast<cudaStream_t>(stream)));
}

moe_status moe_group_tokens(moe_ctx* ctx, const moe_layer_cfg* cfg, const int32_t* idx,
                            const float* gate, int T, const int32_t* slot_of, int n_slots,
                            void* ws, size_t ws_bytes, moe_grouping* out, moe_stream stream) {
  if (ctx == nullptr || out == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg_unskipped(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || n_slots <= 0) return MOE_EINVAL;
  if (ws == nullptr || !aligned(ws, 256)) return MOE_EINVAL;
  if (ws_bytes < ws_layout(*cfg, T).total) return MOE_ENOSPACE;
  fill_grouping(*cfg, T, ws, out);
  if (T == 0) return MOE_OK;
  if (idx == nullptr || gate == nullptr || slot_of == nullptr) return MOE_EINVAL;
  const GroupPtrs g = group_ptrs(*cfg, T, ws);
  return from_cuda(launch_group(ctx->c, *cfg, idx, gate, T, slot_of, n_slots, g,
                                static_cast<cudaStream_t>(stream)));
}

moe_status moe_expert_ffn_q2(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x,
                             const moe_grouping* grouping, const uint8_t* slot_pool,
                             size_t slot_stride, const uint8_t* shared_expert, void* ws,
                             size_t ws_bytes, float* z_rows, void* y, moe_stream stream) {
  return run_ffn(ctx, cfg, 2, x, grouping, slot_pool, slot_stride, shared_expert, ws, ws_bytes,
                 z_rows, y, stream);
}

moe_status moe_expert_ffn_q3(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x,
                             const moe_grouping* grouping, const uint8_t* slot_pool,
                             size_t slot_stride, const uint8_t* shared_expert, void* ws,
                             size_t ws_bytes, float* z_rows, void* y, moe_stream stream) {
  return run_ffn(ctx, cfg, 3, x, grouping, slot_pool, slot_stride, shared_expert, ws, ws_bytes,
                 z_rows, y, stream);
}

moe_status moe_combine(moe_ctx* ctx, const moe_layer_cfg* cfg, const moe_grouping* grouping,
                       const float* z_rows, const void* x, int T, void* y, moe_stream stream) {
  if (ctx == nullptr || grouping == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg_unskipped(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || grouping->T != T || grouping->k != cfg->k) return MOE_EINVAL;
  if (T == 0) return MOE_OK;
  if (z_rows == nullptr || y == nullptr || !aligned(z_rows, 16) || !aligned(y, 16)) return MOE_EINVAL;
  if (cfg->residual && (x == nullptr || !aligned(x, 16))) return MOE_EINVAL;
  return from_cuda(launch_combine(ctx->c, *cfg, grouping->pair_pos, grouping->n_pairs, z_rows,
                                  static_cast<const uint16_t*>(x), T, y,
                                  static_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_forward(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x, int T,
                             const float* w_router, const float* logit_bias,
                             const int32_t* slot_of, int n_slots, const uint8_t* slot_pool,
                             size_t slot_stride, const uint8_t* shared_expert, void* ws,
                             size_t ws_bytes, void* y, moe_stream stream) {
  if (ctx == nullptr) return MOE_EINVAL;
  DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  moe_status st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (T < 0 || n_slots <= 0) return MOE_EINVAL;
  if (T == 0) return MOE_OK;
  if (x == nullptr || w_router == nullptr || slot_of == nullptr || y == nullptr) return MOE_EINVAL;
  if (!aligned(x, 16) || !aligned(w_router, 16) || !aligned(y, 16)) return MOE_EINVAL;
  if (ws == nullptr || !aligned(ws, 256)) return MOE_EINVAL;
  const WsLayout w = ws_layout(*cfg, T);
  if (ws_bytes < w.total) return MOE_ENOSPACE;
  if ((st = check_pool(*cfg, slot_pool, slot_stride, shared_expert)) != MOE_OK) return st;
  char* b = static_cast<char*>(ws);
  float* logits = reinterpret_cast<float*>(b + w.logits);
  int32_t* idx = reinterpret_cast<int32_t*>(b + w.idx);
  float* gate = reinterpret_cast<float*>(b + w.gate);
  if (T <= MOE_DECODE_MAX_T && cfg->E <= 512)  // one fused kernel: router, top-k, grouping, experts, combine
    return run_stack(ctx, *cfg, 1, x, T, w_router, logit_bias, slot_of, n_slots, slot_pool, slot_stride,
                     shared_expert, ws, y, stream);
  if (cfg->skip_from != 0) return MOE_EUNSUPPORTED;  // skipping lives in the fused decode kernel only
  if ((st = moe_router_topk(ctx, cfg, x, w_router, logit_bias, T, logits, idx, gate, stream)) != MOE_OK)
    return st;
  moe_grouping g;
  if ((st = moe_group_tokens(ctx, cfg, idx, gate, T, slot_of, n_slots, ws, ws_bytes, &g, stream)) !=
      MOE_OK)
    return st;
  if (T <= MOE_DECODE_MAX_T)  // E > 512: separate router / grouping kernels, fused expert kernel
    return run_ffn(ctx, cfg, cfg->bits, x, &g, slot_pool, slot_stride, shared_expert, ws, ws_bytes, nullptr, y,
                   stream);
  float* z = reinterpret_cast<float*>(b + w.z);
  if ((st = run_ffn(ctx, cfg, cfg->bits, x, &g, slot_pool, slot_stride, shared_expert, ws, ws_bytes, z,
                    nullptr, stream)) != MOE_OK)
    return st;
  return moe_combine(ctx, cfg, &g, z, x, T, y, stream);
}

}  // extern "C"
