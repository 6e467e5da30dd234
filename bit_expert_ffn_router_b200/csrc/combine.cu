// Combine of the prefill path: y[t] = sum_j z_rows[pair_pos[t,j]] (j in top-k
// order, rows already multiplied by their gates) + z_rows[n_pairs + t] (the
// shared expert), plus x[t] when the layer adds its residual.
//
// A pair the grouping left out (pair_pos -1: its expert is not held on this
// device) adds nothing.
//
// The pages join each layer's routed experts (computed partly on the GPU and
// partly on the CPU) before moving to the next layer (vramglass.com, section
// その2：GPUとCPUで同時に計算する); here every expert runs on the GPU and the
// join is a fixed-order sum, so the result is deterministic.
#include "moe_internal.cuh"

namespace moe {

template <bool OUT_F32>
__global__ void __launch_bounds__(256)
combine_kernel(const int32_t* __restrict__ pair_pos, int n_pairs, int k, int has_shared,
               const float* __restrict__ z, const uint16_t* __restrict__ x, int d, void* y) {
  __shared__ int pos[kMaxK];
  const int t = blockIdx.x;
  if (threadIdx.x < k) pos[threadIdx.x] = pair_pos[t * k + threadIdx.x];
  __syncthreads();
  const int n4 = d / 4;
  for (int c4 = threadIdx.x; c4 < n4; c4 += blockDim.x) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; ++j) {
      if (pos[j] < 0) continue;
      const float4 v = __ldcs(reinterpret_cast<const float4*>(z + static_cast<size_t>(pos[j]) * d) + c4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    if (has_shared) {
      const float4 v = __ldcs(reinterpret_cast<const float4*>(z + static_cast<size_t>(n_pairs + t) * d) + c4);
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const size_t o = static_cast<size_t>(t) * d + 4 * c4;
    if (x != nullptr) {
      const uint2 xv = *reinterpret_cast<const uint2*>(x + o);
      acc.x += __uint_as_float(xv.x << 16);
      acc.y += __uint_as_float(xv.x & 0xffff0000u);
      acc.z += __uint_as_float(xv.y << 16);
      acc.w += __uint_as_float(xv.y & 0xffff0000u);
    }
    if (OUT_F32) {
      *reinterpret_cast<float4*>(static_cast<float*>(y) + o) = acc;
    } else {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
      __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 out;
      out.x = *reinterpret_cast<uint32_t*>(&lo);
      out.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(y) + o) = out;
    }
  }
}

cudaError_t launch_combine(const Ctx& ctx, const moe_layer_cfg& c, const int32_t* pair_pos,
                           int n_pairs, const float* z_rows, const uint16_t* x, int T, void* y,
                           cudaStream_t s) {
  (void)ctx;
  if (T == 0) return cudaSuccess;
  const uint16_t* xr = c.residual ? x : nullptr;
  if (c.out_fp32)
    combine_kernel<true><<<T, 256, 0, s>>>(pair_pos, n_pairs, c.k, c.n_shared, z_rows, xr, c.d, y);
  else
    combine_kernel<false><<<T, 256, 0, s>>>(pair_pos, n_pairs, c.k, c.n_shared, z_rows, xr, c.d, y);
  return cudaGetLastError();
}

}  // namespace moe
