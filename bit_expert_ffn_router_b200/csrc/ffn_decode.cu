// Decode-path expert FFN (T <= MOE_DECODE_MAX_T): stream each selected
// expert's packed 2/3-bit rows once, dequantise in registers, accumulate in
// fp32 on the CUDA cores.
//
// The pages read a token's 10 routed experts plus the shared one from memory
// every decode step and are bound by how fast those bytes arrive
// (vramglass.com, section その2：GPUとCPUで同時に計算する; news.blueqat.app/post/3262,
// section GPU・CPU・RAM・SSDの分担). On a B200 all experts sit in HBM, so this
// path is an HBM-bound streaming GEMV.
//
// Two kernels:
//   gateup: h[row, c] = silu(W_g[c] . x_t) * (W_u[c] . x_t) for every sorted
//           pair (routed) and every token (shared expert);
//   down:   each CTA owns a range of output rows, computes W_d[r] . h for every
//           pair, and combines them per token in top-k order with the gates,
//           so the combine needs no atomics and no second pass.
//
// Dot products: a row's blocks are split over LPR lanes, BPL blocks (32*BPL
// columns) per lane; RPW = 32/LPR rows share one warp step. Within a block
// sum(q_i * x_i) is accumulated in ascending i and the offset is applied as
// s * (sum(q x) - 2^(b-1) * sum(x)); blocks ascend, then a fixed butterfly.
// Nothing depends on which other tokens are in the batch, so a token's result
// is bit-identical at T=1 and inside a T=4 verify batch.
#include "moe_internal.cuh"

namespace moe {

constexpr int kDecWarps = 8;
constexpr int kChanGroup = 8;  // channels (16 gate/up rows) per gate/up work item

struct RowGeom {
  int lpr;  // lanes per row
  int bpl;  // blocks per lane
};

static RowGeom row_geom(int K) {
  const int nb = K / kBlock;
  int lpr = 1;
  while (lpr < 32 && nb % (lpr * 2) == 0) lpr *= 2;
  return RowGeom{lpr, nb / lpr};
}

template <int BITS, int BPL>
__device__ __forceinline__ float row_dot(const uint8_t* __restrict__ codes,
                                         const uint16_t* __restrict__ scales, int K, int g,
                                         const float* xr, const float* xb) {
  constexpr float kOff = static_cast<float>(1 << (BITS - 1));
  float total = 0.f;
  const uint2* lo = reinterpret_cast<const uint2*>(codes) + g * BPL;
#pragma unroll
  for (int b = 0; b < BPL; ++b) {
    const uint2 w = __ldg(lo + b);
    uint32_t hi = 0;
    if (BITS == 3) hi = __ldg(reinterpret_cast<const uint32_t*>(codes + K / 4) + g * BPL + b);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t word = (i < 16) ? w.x : w.y;
      uint32_t q = (word >> (2 * (i & 15))) & 3u;
      if (BITS == 3) q |= ((hi >> i) & 1u) << 2;
      acc = fmaf(static_cast<float>(q), xr[b * 32 + i], acc);
    }
    const float s = __half2float(__ushort_as_half(__ldg(scales + g * BPL + b)));
    total = fmaf(s, acc - kOff * xb[b], total);
  }
  return total;
}

template <int BPL>
__device__ __forceinline__ void load_vec(const float* __restrict__ src, int g, float* xr, float* xb) {
  const float4* p = reinterpret_cast<const float4*>(src + g * BPL * 32);
#pragma unroll
  for (int b = 0; b < BPL; ++b) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 v = p[b * 8 + i];
      xr[b * 32 + 4 * i + 0] = v.x;
      xr[b * 32 + 4 * i + 1] = v.y;
      xr[b * 32 + 4 * i + 2] = v.z;
      xr[b * 32 + 4 * i + 3] = v.w;
      s += v.x;
      s += v.y;
      s += v.z;
      s += v.w;
    }
    xb[b] = s;
  }
}

__device__ __forceinline__ float silu(float z) { return z / (1.f + expf(-z)); }

// ------------------------------------------------------------------ gate/up
template <int BITS, int BPL>
__global__ void __launch_bounds__(kDecWarps * 32)
gateup_decode_kernel(FfnArgs a, GroupPtrs g, int d, int f, int n_pairs, int lpr) {
  extern __shared__ float smem[];
  float* xs = smem;                                   // [T][d]
  float* res = smem + a.T * d;                        // [warps][2*kChanGroup]
  for (int i = threadIdx.x; i < a.T * d; i += blockDim.x) xs[i] = bf16_bits_to_float(a.x[i]);
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rpw = 32 / lpr;
  const int rl = lane / lpr, gl = lane % lpr;
  const int n_uniq = ld_cg(g.n_uniq);
  const int n_ext = n_uniq + (a.shared ? 1 : 0);
  const int groups = f / kChanGroup;
  const int n_items = n_ext * groups;
  const size_t row_b = static_cast<size_t>(d) * BITS / 8;
  const int sc_row = d / kBlock;
  float* wres = res + warp * 2 * kChanGroup;

  for (int item = blockIdx.x * kDecWarps + warp; item < n_items; item += gridDim.x * kDecWarps) {
    const int u = item / groups, cg = item % groups;
    const uint8_t* rec;
    int p_begin, p_end;
    if (u < n_uniq) {
      rec = a.pool + static_cast<size_t>(ld_cg(g.uniq_slot + u)) * a.stride;
      p_begin = ld_cg(g.uniq_offset + u);
      p_end = ld_cg(g.uniq_offset + u + 1);
    } else {
      rec = a.shared;
      p_begin = n_pairs;
      p_end = n_pairs + a.T;
    }
    const uint8_t* codes = rec + a.lay.gu_codes;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(rec + a.lay.gu_scales);
    for (int p = p_begin; p < p_end; ++p) {
      const int t = (u < n_uniq) ? ld_cg(g.pair_token + p) : p - n_pairs;
      float xr[BPL * 32], xb[BPL];
      load_vec<BPL>(xs + t * d, gl, xr, xb);
      for (int s0 = 0; s0 < 2 * kChanGroup; s0 += rpw) {
        const int rloc = s0 + rl;
        const int row = 2 * cg * kChanGroup + rloc;
        float v = 0.f;
        if (rloc < 2 * kChanGroup)
          v = row_dot<BITS, BPL>(codes + row * row_b, scales + static_cast<size_t>(row) * sc_row, d, gl,
                                 xr, xb);
        v = group_sum(v, lpr);
        if (gl == 0 && rloc < 2 * kChanGroup) wres[rloc] = v;
      }
      __syncwarp();
      if (lane < kChanGroup) {
        const float gv = wres[2 * lane], uv = wres[2 * lane + 1];
        a.h[static_cast<size_t>(p) * f + cg * kChanGroup + lane] = silu(gv) * uv;
      }
      __syncwarp();
    }
  }
}

// ------------------------------------------------------------------ down + combine
template <int BITS, int BPL, bool OUT_F32>
__global__ void __launch_bounds__(kDecWarps * 32)
down_decode_kernel(FfnArgs a, GroupPtrs g, int d, int f, int k, int n_pairs, int n_rows,
                   int lpr, int rows_per_cta, int residual) {
  extern __shared__ float zs[];  // [n_rows][rows_per_cta]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rpw = 32 / lpr;
  const int rl = lane / lpr, gl = lane % lpr;
  const int r0 = blockIdx.x * rows_per_cta;
  const int r1 = min(r0 + rows_per_cta, d);
  if (r0 >= d) return;
  const size_t row_b = static_cast<size_t>(f) * BITS / 8;
  const int sc_row = f / kBlock;

  for (int p = warp; p < n_rows; p += kDecWarps) {
    const uint8_t* rec =
        (p < n_pairs) ? a.pool + static_cast<size_t>(ld_cg(g.pair_slot + p)) * a.stride : a.shared;
    const uint8_t* codes = rec + a.lay.dn_codes;
    const uint16_t* scales = reinterpret_cast<const uint16_t*>(rec + a.lay.dn_scales);
    float hr[BPL * 32], hb[BPL];
    load_vec<BPL>(a.h + static_cast<size_t>(p) * f, gl, hr, hb);
    for (int r = r0; r < r1; r += rpw) {
      const int row = r + rl;
      float v = 0.f;
      if (row < r1)
        v = row_dot<BITS, BPL>(codes + row * row_b, scales + static_cast<size_t>(row) * sc_row, f, gl,
                               hr, hb);
      v = group_sum(v, lpr);
      if (gl == 0 && row < r1) zs[p * rows_per_cta + (row - r0)] = v;
    }
  }
  __syncthreads();

  const int nr = r1 - r0;
  for (int i = threadIdx.x; i < a.T * nr; i += blockDim.x) {
    const int t = i / nr, rr = i % nr;
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int p = ld_cg(g.pair_pos + t * k + j);
      acc = fmaf(ld_cg(g.pair_gate + p), zs[p * rows_per_cta + rr], acc);
    }
    if (a.shared) acc += zs[(n_pairs + t) * rows_per_cta + rr];
    const size_t o = static_cast<size_t>(t) * d + r0 + rr;
    if (residual) acc += bf16_bits_to_float(a.x[o]);
    if (OUT_F32) static_cast<float*>(a.y)[o] = acc;
    else static_cast<__nv_bfloat16*>(a.y)[o] = __float2bfloat16_rn(acc);
  }
}

// ------------------------------------------------------------------ launch
template <int BITS, int BPL>
static cudaError_t launch_gateup(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a,
                                 int lpr, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(a.T) * c.d + kDecWarps * 2 * kChanGroup) * sizeof(float);
  const int grid = ctx.num_sms * 2;
  gateup_decode_kernel<BITS, BPL><<<grid, kDecWarps * 32, smem, s>>>(a, *a.g, c.d, c.f, a.T * c.k,
                                                                     lpr);
  return cudaGetLastError();
}

template <int BITS, int BPL>
static cudaError_t launch_down(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a, int lpr,
                               cudaStream_t s) {
  const int rpw = 32 / lpr;
  const int n_pairs = a.T * c.k;
  const int n_rows = n_pairs + (a.shared ? a.T : 0);
  int groups = (c.d + rpw - 1) / rpw;
  int grid = groups < ctx.num_sms ? groups : ctx.num_sms;
  const int rows_per_cta = ((groups + grid - 1) / grid) * rpw;
  grid = (c.d + rows_per_cta - 1) / rows_per_cta;
  const size_t smem = static_cast<size_t>(n_rows) * rows_per_cta * sizeof(float);
  if (c.out_fp32)
    down_decode_kernel<BITS, BPL, true><<<grid, kDecWarps * 32, smem, s>>>(
        a, *a.g, c.d, c.f, c.k, n_pairs, n_rows, lpr, rows_per_cta, c.residual);
  else
    down_decode_kernel<BITS, BPL, false><<<grid, kDecWarps * 32, smem, s>>>(
        a, *a.g, c.d, c.f, c.k, n_pairs, n_rows, lpr, rows_per_cta, c.residual);
  return cudaGetLastError();
}

template <int BITS>
static cudaError_t launch_bits(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a,
                               cudaStream_t s) {
  const RowGeom gg = row_geom(c.d), gd = row_geom(c.f);
  cudaError_t e = cudaSuccess;
  switch (gg.bpl) {
    case 1: e = launch_gateup<BITS, 1>(ctx, c, a, gg.lpr, s); break;
    case 2: e = launch_gateup<BITS, 2>(ctx, c, a, gg.lpr, s); break;
    case 3: e = launch_gateup<BITS, 3>(ctx, c, a, gg.lpr, s); break;
    case 4: e = launch_gateup<BITS, 4>(ctx, c, a, gg.lpr, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  switch (gd.bpl) {
    case 1: return launch_down<BITS, 1>(ctx, c, a, gd.lpr, s);
    case 2: return launch_down<BITS, 2>(ctx, c, a, gd.lpr, s);
    case 3: return launch_down<BITS, 3>(ctx, c, a, gd.lpr, s);
    case 4: return launch_down<BITS, 4>(ctx, c, a, gd.lpr, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_ffn_decode(const Ctx& ctx, const moe_layer_cfg& c, const FfnArgs& a,
                              cudaStream_t s) {
  return c.bits == 2 ? launch_bits<2>(ctx, c, a, s) : launch_bits<3>(ctx, c, a, s);
}

template <int BITS, int BPL>
static cudaError_t set_attrs() {
  const int big = 200 * 1024;
  cudaError_t e = cudaFuncSetAttribute(gateup_decode_kernel<BITS, BPL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(down_decode_kernel<BITS, BPL, true>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, big);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(down_decode_kernel<BITS, BPL, false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, big);
}

cudaError_t decode_init(const Ctx& ctx) {
  (void)ctx;
  cudaError_t e;
#define MOE_SET(B, P) if ((e = set_attrs<B, P>()) != cudaSuccess) return e;
  MOE_SET(2, 1) MOE_SET(2, 2) MOE_SET(2, 3) MOE_SET(2, 4)
  MOE_SET(3, 1) MOE_SET(3, 2) MOE_SET(3, 3) MOE_SET(3, 4)
#undef MOE_SET
  return cudaSuccess;
}

// Host helper used by the API layer to check the geometry before launching.
bool decode_geometry_ok(int d, int f) {
  return row_geom(d).bpl <= 4 && row_geom(f).bpl <= 4;
}

}  // namespace moe
