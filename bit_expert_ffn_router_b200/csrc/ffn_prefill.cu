// Prefill-path expert FFN (tensor-core grouped GEMM). Placeholder until the
// tcgen05 kernels land: reports "not supported".
#include "moe_internal.cuh"

namespace moe {

cudaError_t launch_ffn_prefill(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a, void* ws,
                               float* z_rows, cudaStream_t s) {
  (void)ctx; (void)c; (void)a; (void)ws; (void)z_rows; (void)s;
  return cudaErrorNotSupported;
}

cudaError_t prefill_init(const Ctx& ctx) {
  (void)ctx;
  return cudaSuccess;
}

}  // namespace moe
