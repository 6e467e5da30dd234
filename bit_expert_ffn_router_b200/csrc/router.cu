// Router logits and top-k selection.
//
// The router decides, for every token on the GPU, which of the layer's 512
// experts run (news.blueqat.app/post/3262, section GPU・CPU・RAM・SSDの分担:
// the router sits with attention on the GPU); each token takes 10 of them
// (same page, first section). The pages give no formula; this is the plain
// linear router l = x W_r^T followed by a top-k with ties to the lower expert
// index and a softmax over the chosen logits.
#include "moe_internal.cuh"

namespace moe {

// ------------------------------------------------------------ decode router
// One warp per expert row, every token of the (small) batch at once. W_r is
// streamed once with 16-byte loads; x sits in shared memory as fp32. The sum
// for a token does not depend on the other tokens in the batch: each lane
// accumulates its columns in ascending order, then a fixed butterfly.
constexpr int kRouterWarps = 4;

template <int MAXT>
__global__ void __launch_bounds__(kRouterWarps * 32)
router_rows_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                   const float* __restrict__ bias, int T, int d, int E,
                   float* __restrict__ logits) {
  extern __shared__ float xs[];  // [T][d]
  for (int i = threadIdx.x; i < T * d; i += blockDim.x) xs[i] = bf16_bits_to_float(x[i]);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * kRouterWarps + (threadIdx.x >> 5);
  if (e >= E) return;
  const float4* w4 = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * d);
  float acc[MAXT];
#pragma unroll
  for (int t = 0; t < MAXT; ++t) acc[t] = 0.f;
  const int n4 = d >> 2;
#pragma unroll 4
  for (int c4 = lane; c4 < n4; c4 += 32) {
    const float4 w = __ldg(w4 + c4);
#pragma unroll
    for (int t = 0; t < MAXT; ++t) {
      if (t < T) {
        const float4 xv = reinterpret_cast<const float4*>(xs + t * d)[c4];
        float a = acc[t];
        a = fmaf(w.x, xv.x, a);
        a = fmaf(w.y, xv.y, a);
        a = fmaf(w.z, xv.z, a);
        a = fmaf(w.w, xv.w, a);
        acc[t] = a;
      }
    }
  }
#pragma unroll
  for (int t = 0; t < MAXT; ++t) {
    if (t < T) {
      const float s = warp_sum(acc[t]);
      if (lane == 0) {
        const size_t o = static_cast<size_t>(t) * E + e;
        logits[o] = bias ? s + bias[o] : s;
      }
    }
  }
}

// ------------------------------------------------------------ prefill router
// logits[T, E] = x[T, d] (bf16) * W_r[E, d]^T (fp32) as a tiled fp32 GEMM on
// the CUDA cores: 128x128 tiles, 16-deep k steps, 8x8 outputs per thread,
// k accumulated in ascending order.
constexpr int kGM = 128, kGN = 128, kGK = 16;

__global__ void __launch_bounds__(256)
router_gemm_kernel(const uint16_t* __restrict__ x, const float* __restrict__ wr,
                   const float* __restrict__ bias, int T, int d, int E,
                   float* __restrict__ logits) {
  __shared__ __align__(16) float As[kGK][kGM];
  __shared__ __align__(16) float Bs[kGK][kGN];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * kGM, n0 = blockIdx.x * kGN;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  // loader mapping: row = tid / 2, 8 consecutive k per thread
  const int lr = tid >> 1, lk = (tid & 1) * 8;
  for (int k0 = 0; k0 < d; k0 += kGK) {
    {
      const int m = m0 + lr;
      uint4 raw = make_uint4(0, 0, 0, 0);
      if (m < T) raw = *reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * d + k0 + lk);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        As[lk + 2 * q][lr] = __uint_as_float(w[q] << 16);
        As[lk + 2 * q + 1][lr] = __uint_as_float(w[q] & 0xffff0000u);
      }
      const int n = n0 + lr;
      float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0;
      if (n < E) {
        const float4* p = reinterpret_cast<const float4*>(wr + static_cast<size_t>(n) * d + k0 + lk);
        b0 = __ldg(p);
        b1 = __ldg(p + 1);
      }
      Bs[lk + 0][lr] = b0.x; Bs[lk + 1][lr] = b0.y; Bs[lk + 2][lr] = b0.z; Bs[lk + 3][lr] = b0.w;
      Bs[lk + 4][lr] = b1.x; Bs[lk + 5][lr] = b1.y; Bs[lk + 6][lr] = b1.z; Bs[lk + 7][lr] = b1.w;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][64 + ty * 4]);
      const float4 c0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float4 c1 = *reinterpret_cast<const float4*>(&Bs[kk][64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (m >= T) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + (j - 4));
      if (n >= E) continue;
      const size_t o = static_cast<size_t>(m) * E + n;
      logits[o] = bias ? acc[i][j] + bias[o] : acc[i][j];
    }
  }
}

cudaError_t launch_router_logits(const Ctx& ctx, const moe_layer_cfg& c, const uint16_t* x,
                                 const float* wr, const float* bias, int T, float* logits,
                                 cudaStream_t s) {
  if (T <= MOE_DECODE_MAX_T) {
    const size_t smem = static_cast<size_t>(T) * c.d * sizeof(float);
    const dim3 grid((c.E + kRouterWarps - 1) / kRouterWarps);
    router_rows_kernel<MOE_DECODE_MAX_T><<<grid, kRouterWarps * 32, smem, s>>>(x, wr, bias, T, c.d,
                                                                              c.E, logits);
  } else if (router_tc_ok(c)) {
    return launch_router_tc(ctx, c, x, wr, bias, T, logits, s);  // tensor cores, bf16 three-part split
  } else {
    const dim3 grid((c.E + kGN - 1) / kGN, (T + kGM - 1) / kGM);
    router_gemm_kernel<<<grid, 256, 0, s>>>(x, wr, bias, T, c.d, c.E, logits);
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------ top-k
// One warp per token. A logit and its expert index form one 64-bit key
// (order-preserving float bits above the complemented index), so one max
// per round picks the largest logit and, among equal logits, the lowest
// index. NaN keys sort below -inf; -0.0 is folded into +0.0.
__device__ __forceinline__ uint32_t order_bits(float v) {
  if (v != v) return 0u;  // NaN: below every number
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float from_order_bits(uint32_t o) {
  if (o == 0u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

__device__ __forceinline__ unsigned long long umax64(unsigned long long a, unsigned long long b) {
  return a > b ? a : b;
}

template <int VPL>
__global__ void __launch_bounds__(256)
topk_kernel(const float* __restrict__ logits, int T, int E, int k, int renorm,
            int32_t* __restrict__ idx, float* __restrict__ gate) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + static_cast<size_t>(t) * E;
  unsigned long long key[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = v * 32 + lane;
    key[v] = 0ull;
    if (e < E) {
      const float l = row[e];
      key[v] = (static_cast<unsigned long long>(order_bits(l)) << 32) | static_cast<uint32_t>(~e);
    }
  }
  unsigned long long mine = 0ull;
  for (int j = 0; j < k; ++j) {
    unsigned long long m = 0ull;
#pragma unroll
    for (int v = 0; v < VPL; ++v) m = umax64(m, key[v]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = umax64(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int e = static_cast<int>(~static_cast<uint32_t>(m));
    if ((e & 31) == lane) {
#pragma unroll
      for (int v = 0; v < VPL; ++v)
        if (v == (e >> 5)) key[v] = 0ull;
    }
    if (lane == j) mine = m;
  }
  const bool sel = lane < k;
  const float lj = sel ? from_order_bits(static_cast<uint32_t>(mine >> 32)) : 0.f;
  const float l0 = __shfl_sync(0xffffffffu, lj, 0);
  const float ex = sel ? expf(lj - l0) : 0.f;
  float denom;
  if (renorm) {
    denom = warp_sum(ex);
  } else {
    float s = 0.f;
    for (int e = lane; e < E; e += 32) s += expf(row[e] - l0);
    denom = warp_sum(s);
  }
  if (sel) {
    const size_t o = static_cast<size_t>(t) * k + lane;
    idx[o] = static_cast<int32_t>(~static_cast<uint32_t>(mine));
    gate[o] = ex / denom;
  }
}

cudaError_t launch_topk(const Ctx& ctx, const moe_layer_cfg& c, const float* logits, int T,
                        int32_t* idx, float* gate, cudaStream_t s) {
  (void)ctx;
  const dim3 grid((T + 7) / 8);
  const int vpl = (c.E + 31) / 32;
  if (vpl <= 1) topk_kernel<1><<<grid, 256, 0, s>>>(logits, T, c.E, c.k, c.renorm, idx, gate);
  else if (vpl <= 2) topk_kernel<2><<<grid, 256, 0, s>>>(logits, T, c.E, c.k, c.renorm, idx, gate);
  else if (vpl <= 4) topk_kernel<4><<<grid, 256, 0, s>>>(logits, T, c.E, c.k, c.renorm, idx, gate);
  else if (vpl <= 8) topk_kernel<8><<<grid, 256, 0, s>>>(logits, T, c.E, c.k, c.renorm, idx, gate);
  else if (vpl <= 16) topk_kernel<16><<<grid, 256, 0, s>>>(logits, T, c.E, c.k, c.renorm, idx, gate);
  else topk_kernel<32><<<grid, 256, 0, s>>>(logits, T, c.E, c.k, c.renorm, idx, gate);
  return cudaGetLastError();
}

cudaError_t router_init(const Ctx& ctx) {
  (void)ctx;
  return cudaFuncSetAttribute(router_rows_kernel<MOE_DECODE_MAX_T>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              MOE_DECODE_MAX_T * 4096 * static_cast<int>(sizeof(float)));
}

}  // namespace moe
