// moe_layer_forward_static: the whole-layer entry point with its scratch in a
// fixed static device array instead of a caller workspace.
//
// Which callers need it: a host that links only this library and owns no
// device allocator (plain C, no PyTorch), and a decode loop that must not
// call cudaMalloc, which can synchronise the whole device. Such a caller gets
// the full step without handing over any memory of its own.
//
// The array is part of the library's device image: the driver reserves it on
// each device when the module loads there, so no call allocates. The step
// itself is the unchanged moe_layer_forward, given the array as workspace.
#include "moe_internal.cuh"

namespace {

// Largest workspace the static variant serves (moe_workspace_bytes(cfg, T)):
// the full-size layer (d=2048, f=768, E=512, k=10) needs about 2.7 MB at
// T = 8.
constexpr size_t kStaticScratchBytes = MOE_STATIC_SCRATCH_BYTES;
static_assert(kStaticScratchBytes % 256 == 0, "scratch size");

// No byte of it needs to start at zero: every byte a call reads was written
// earlier in the same call.
static __device__ __align__(256) unsigned char g_scratch[kStaticScratchBytes];

// Device address of g_scratch on the context's device, looked up on the
// context's first call with that device current and kept in the context. A
// context lives on one device and does not outlive a reset of it, so the
// address it holds stays valid for as long as the context does.
cudaError_t scratch_of(moe::Ctx& c, void** out) {
  if (c.static_scratch == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess) return e;
    c.static_scratch = p;
  }
  *out = c.static_scratch;
  return cudaSuccess;
}

}  // namespace

extern "C" {

moe_status moe_layer_forward_static(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x, int T,
                                    const float* w_router, const float* logit_bias, const int32_t* slot_of,
                                    int n_slots, const uint8_t* slot_pool, size_t slot_stride,
                                    const uint8_t* shared_expert, void* y, moe_stream stream) {
  if (ctx == nullptr || cfg == nullptr || T < 0) return MOE_EINVAL;
  const size_t need = moe_workspace_bytes(cfg, T);
  if (need == 0) return MOE_EINVAL;  // invalid configuration
  if (need > kStaticScratchBytes) return MOE_ENOSPACE;
  moe::DeviceGuard dg(ctx->c.device);
  if (!dg.ok) return MOE_ECUDA;
  void* scratch = nullptr;
  const cudaError_t e = scratch_of(ctx->c, &scratch);
  if (e != cudaSuccess) {
    moe::record_cuda_error(e);
    return MOE_ECUDA;
  }
  return moe_layer_forward(ctx, cfg, x, T, w_router, logit_bias, slot_of, n_slots, slot_pool, slot_stride,
                           shared_expert, scratch, kStaticScratchBytes, y, stream);
}

}  // extern "C"
