// Decode path (T <= MOE_DECODE_MAX_T): one persistent kernel per layer.
//
// The pages' engine reads, per token and layer, the router, the shared expert
// and the 10 routed experts it picks, and its speed is set by how fast those
// bytes arrive (vramglass.com, sections なぜVRAM 12GBで足りるのか and
// その2：GPUとCPUで同時に計算する; news.blueqat.app/post/3262, section
// GPU・CPU・RAM・SSDの分担). On a B200 every expert sits in HBM, so the step is
// a chain of HBM-bound GEMVs whose cost is mostly latency: this kernel keeps
// the weight stream continuous across the whole layer.
//
// One CTA per SM, 15 consumer warps + 1 producer warp:
//   producer: cp.async.bulk copies of this CTA's weight rows into a
//             shared-memory byte ring, one mbarrier per stage; once routing
//             is known the rest of the stage list is laid out in one step and
//             issued in consumption order (the down-projection rows stream in
//             while gate/up is still computing);
//   consumers: [router rows -> grid barrier -> top-k + grouping (every CTA
//             computes it, CTA 0 publishes it)] -> gate/up + SwiGLU into h ->
//             grid barrier -> down rows of this CTA's output slice for every
//             (expert, token) -> combine in top-k order -> y.
// The shared expert's gate/up rows are fetched before routing is known; with
// routing in the kernel they are computed right after it, while the routed
// experts' rows are on their way.
//
// Grid barriers and every mbarrier wait are bounded by a global-timer limit;
// on expiry the kernel records MOE_ETIMEOUT in the context's status word,
// drains its own copies and returns.
#include "moe_internal.cuh"
#include "dequant.cuh"

namespace moe {

// Consumer warps per CTA (plus one producer warp): 15 for 2-bit rows (four
// warps per SM sub-partition, <= 128 registers each), 11 for 3-bit rows,
// whose high-plane operands need more registers.
__host__ __device__ constexpr int consumer_warps(int bits) { return bits == 2 ? 15 : 11; }
constexpr int kNB = 32;               // stage mbarrier ring
constexpr int kStageAlign = 128;

enum : int { kStGU = 0, kStDN = 1 };
constexpr int kShared = -1;  // expert id of the shared expert in stage records

struct StageRec {
  int type, u, a, b;  // GU: expert u, channels [a, b); DN: expert u, rows [a, b)
  int off, bytes, code_bytes, pad;
};

struct DLParams {
  const uint16_t* x;
  int T, d, f, E, k, renorm, residual, has_shared, out_f32;
  const float* wr;
  const float* bias;
  float* logits;
  int32_t* idx;
  float* gate;
  const int32_t* slot_of;
  int n_slots;
  GroupPtrs g;
  const uint8_t* pool;
  size_t stride;
  const uint8_t* shared;
  moe_expert_layout lay;
  float* h;                  // kRep copies of [n_rows, f], h_rep floats apart
  size_t h_rep;
  float* logits_rep;         // route: kRep copies of [T, E]
  void* y;
  int* status;
  unsigned long long* gbar;  // grid-barrier arrival counter
  unsigned long long timeout_ns;
  unsigned long long* trace;  // null, or kTraceSlots timestamps per CTA
  int rpc;         // down rows per CTA
  int gu_lpr, dn_lpr;
  int gu_row, gu_sc, dn_row, dn_sc;  // bytes per row: codes and scales
  int gu_chan;     // channels per gate/up stage (one per consumer warp)
  // shared-memory map (byte offsets), computed on the host
  int sm_stages, sm_route, sm_zs, sm_xq, sm_wr, sm_hq, sm_ring, ring_bytes, max_stages, wr_rows;
  int h_rows;      // quantised h rows the staging area holds
};

// ------------------------------------------------------------------ grid barrier
// A monotonic 64-bit arrival counter shared by all launches on a context:
// every CTA arrives exactly once per barrier episode and none arrives at the
// next episode before the current one completes, so an arrival that reads
// `old` belongs to the episode ending at (old / G + 1) * G.
__device__ __forceinline__ unsigned long long gbar_arrive(unsigned long long* gb, unsigned nctas) {
  __threadfence();
  const unsigned long long old = atomicAdd(gb, 1ull);
  return (old / nctas + 1) * nctas;
}

__device__ __forceinline__ bool gbar_wait(const unsigned long long* gb, unsigned long long target,
                                          uint64_t deadline) {
  while (ld_acquire_gpu_u64(gb) < target) {
    if (global_timer_ns() > deadline) return false;
    __nanosleep(32);
  }
  return true;
}

// ------------------------------------------------------------------ shared state
struct DLShared {
  uint64_t full[kNB];
  uint64_t empty[kNB];
  uint64_t wr_bar;
  uint64_t list_bar;
  int abort_flag;
  int n_sh, n_gu, n_st;  // shared-expert GU stages, all GU stages, all stages
  int n_uniq;
  unsigned long long bar_target;
};

struct RouteSmem {
  int32_t* idx;        // [T*k]
  float* gate;         // [T*k]
  int32_t* sorted_e;   // [np]
  int32_t* pair_token; // [np]
  float* pair_gate;    // [np]
  int32_t* pair_pos;   // [T*k]
  int32_t* uniq_e;     // [np]
  int32_t* uniq_slot;  // [np]
  int32_t* uniq_off;   // [np + 1]
  int32_t* slot_s;     // [E] this layer's slot table (routing path)
};

__device__ __forceinline__ RouteSmem route_smem(char* base, int np) {
  RouteSmem r;
  int32_t* p = reinterpret_cast<int32_t*>(base);
  r.idx = p;
  r.gate = reinterpret_cast<float*>(p + np);
  r.sorted_e = p + 2 * np;
  r.pair_token = p + 3 * np;
  r.pair_gate = reinterpret_cast<float*>(p + 4 * np);
  r.pair_pos = p + 5 * np;
  r.uniq_e = p + 6 * np;
  r.uniq_slot = p + 7 * np;
  r.uniq_off = p + 8 * np;
  r.slot_s = p + 9 * np + 1;
  return r;
}

__device__ __forceinline__ void set_abort(DLShared* S, int* status, int where) {
  report(status, kDevTimeout, where);
  *reinterpret_cast<volatile int*>(&S->abort_flag) = 1;
}

__device__ __forceinline__ bool aborted(DLShared* S) {
  return *reinterpret_cast<volatile int*>(&S->abort_flag) != 0;
}

// ------------------------------------------------------------------ stage list
// GU stages for channels [c0, c1) of expert u, at most gu_chan channels each.
__device__ int push_gu(StageRec* st, int n, int u, int c0, int c1, const DLParams& P) {
  const int gu_row = P.gu_row, gu_sc = P.gu_sc;
  for (int c = c0; c < c1; c += P.gu_chan) {
    const int e = min(c + P.gu_chan, c1);
    StageRec r;
    r.type = kStGU;
    r.u = u;
    r.a = c;
    r.b = e;
    r.code_bytes = 2 * (e - c) * gu_row;
    r.bytes = r.code_bytes + 2 * (e - c) * gu_sc;
    r.off = 0;
    r.pad = 0;
    st[n++] = r;
  }
  return n;
}

__device__ int push_dn(StageRec* st, int n, int u, int r0, int r1, const DLParams& P) {
  if (r1 <= r0) return n;
  const int dn_row = P.dn_row, dn_sc = P.dn_sc;
  StageRec r;
  r.type = kStDN;
  r.u = u;
  r.a = r0;
  r.b = r1;
  r.code_bytes = (r1 - r0) * dn_row;
  r.bytes = r.code_bytes + (r1 - r0) * dn_sc;
  r.off = 0;
  r.pad = 0;
  st[n++] = r;
  return n;
}

// Routed stage list: this CTA's share of the nu*f routed gate/up channels,
// then the down slices: routed experts in order, shared last, so that the h
// rows they read are one ascending range. Stages [0, n_sh) (the shared
// expert's gate/up) are already in place.
__device__ void build_routed_list(StageRec* st, DLShared* S, int n_sh, int nu, int b, int G, int r0, int r1,
                                  const DLParams& P) {
  // 32-bit arithmetic: the launch guarantees nu * f * G < 2^31
  int n = n_sh;
  const int tot = nu * P.f;
  int c = tot * b / G;
  const int c1 = tot * (b + 1) / G;
  while (c < c1) {
    const int u = c / P.f;
    const int ub = u * P.f;
    const int ce = min(c1, ub + P.f) - ub;
    n = push_gu(st, n, u, c - ub, ce, P);
    c = ub + ce;
  }
  S->n_gu = n;
  for (int u = 0; u < nu; ++u) n = push_dn(st, n, u, r0, r1, P);
  if (P.has_shared) n = push_dn(st, n, kShared, r0, r1, P);
  S->n_st = n;
  S->n_uniq = nu;
}

// ------------------------------------------------------------------ producer
struct Ring {
  int head;       // end of the newest live stage
  int tail;       // oldest live stage index
  int issued;     // stages issued so far
};

__device__ __forceinline__ const uint8_t* expert_record(const DLParams& P, const RouteSmem& R, int u) {
  return u == kShared ? P.shared : P.pool + static_cast<size_t>(R.uniq_slot[u]) * P.stride;
}

// Sorted rows (pairs) an expert's FFN runs for: routed u -> its pairs; shared -> np + t.
__device__ __forceinline__ void expert_rows(const RouteSmem& R, int u, int np, int T, int& p0, int& p1) {
  if (u == kShared) {
    p0 = np;
    p1 = np + T;
  } else {
    p0 = R.uniq_off[u];
    p1 = R.uniq_off[u + 1];
  }
}

// Frees the oldest live stage (waits for its consumer). False on timeout.
__device__ bool ring_pop(DLShared* S, StageRec* st, Ring& rg, uint64_t deadline) {
  const int j = rg.tail;
  if (!mbar_wait(&S->empty[j % kNB], (j / kNB) & 1, deadline)) return false;
  rg.tail++;
  if (rg.tail == rg.issued) rg.head = 0;
  return true;
}

// Reserves ring space for stage i (the producer's lane 0), freeing older
// stages as needed but never one at index >= pop_limit (reserved in the
// current batch, not issued yet). Returns 1 on success, 2 if the stage must
// wait for the next batch, 0 on timeout or abort.
__device__ int ring_alloc(DLShared* S, StageRec* st, Ring& rg, int i, int cap, int pop_limit, uint64_t deadline) {
  StageRec& s = st[i];
  const int need = (s.bytes + kStageAlign - 1) / kStageAlign * kStageAlign;
  int start = -1;
  while (true) {
    if (aborted(S)) return 0;
    if (rg.tail == rg.issued) {
      rg.head = 0;
      start = 0;
      break;
    }
    if (i - rg.tail < kNB) {
      const int toff = st[rg.tail].off;
      if (rg.head > toff) {  // live region does not wrap
        if (rg.head + need <= cap) { start = rg.head; break; }
        if (need <= toff) { start = 0; break; }
      } else if (rg.head + need <= toff) {
        start = rg.head;
        break;
      }
    }
    if (rg.tail >= pop_limit) return 2;
    if (!ring_pop(S, st, rg, deadline)) return 0;
  }
  s.off = start;
  rg.head = start + need;
  rg.issued = i + 1;
  return 1;
}

// Arms stage i's mbarrier and issues its two bulk copies (codes, scales).
// Any lane may issue any reserved stage: copies issued from several lanes
// at once overlap their issue latency.
__device__ void stage_issue(DLShared* S, const StageRec& s, int i, uint8_t* ring, const DLParams& P,
                            const RouteSmem& R) {
  const uint8_t* rec = expert_record(P, R, s.u);
  uint8_t* dst = ring + s.off;
  uint64_t* bar = &S->full[i % kNB];
  mbar_arrive_expect_tx(bar, static_cast<uint32_t>(s.bytes));
  const int rows = s.type == kStGU ? 2 * (s.b - s.a) : s.b - s.a;
  const int first = s.type == kStGU ? 2 * s.a : s.a;
  const int row_b = s.code_bytes / rows;
  const int sc_b = (s.bytes - s.code_bytes) / rows;
  const size_t oc = s.type == kStGU ? P.lay.gu_codes : P.lay.dn_codes;
  const size_t os = s.type == kStGU ? P.lay.gu_scales : P.lay.dn_scales;
  bulk_g2s(dst, rec + oc + static_cast<size_t>(first) * row_b, s.code_bytes, bar);
  bulk_g2s(dst + s.code_bytes, rec + os + static_cast<size_t>(first) * sc_b, s.bytes - s.code_bytes, bar);
}

// ------------------------------------------------------------------ consumers
// The quantisers below walk their jobs in warp-sized steps, kQD steps at a
// time: all loads of a group are issued before any value is used, so a group
// costs about one memory round trip (at T = 1 one group covers all h rows a
// CTA needs). A step past the end is skipped as a whole (the test is uniform
// across the warp); inside the last step, idle lanes read a clamped, valid
// address, so no single load carries a guard.
constexpr int kQD = 3;

// Quantises the T token rows of x (bf16, global) into the gate/up layout,
// four lanes per 32-value block, and keeps the raw rows in xs for the router.
template <int BITS>
__device__ void quantise_x(const DLParams& P, int* xq, uint16_t* xs, int nct) {
  const int nb = P.d / kBlock, bpl = nb / P.gu_lpr;
  const int words = QV<BITS>::kWords * nb;
  const int jobs = P.T * nb;
  const int q = threadIdx.x & 3;
  if constexpr (BITS == 2) {
    // thread q of a block takes its 8 consecutive values in one 16-byte load
#pragma unroll 1
    for (int base0 = threadIdx.x & ~31; base0 < jobs * 4; base0 += kQD * nct) {
      uint4 raw[kQD];
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        if (base0 + g * nct >= jobs * 4) break;
        const int job = min((base0 + g * nct + (threadIdx.x & 31)) >> 2, jobs - 1);
        const size_t a = static_cast<size_t>(job / nb) * P.d + (job % nb) * kBlock + 8 * q;
        raw[g] = __ldcg(reinterpret_cast<const uint4*>(P.x + a));
      }
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        const int base = base0 + g * nct;  // warp-uniform
        if (base >= jobs * 4) break;
        const int job = (base + (threadIdx.x & 31)) >> 2;
        const bool live = job < jobs;
        const int t = live ? job / nb : 0, blk = live ? job % nb : 0;
        const size_t at = static_cast<size_t>(t) * P.d + blk * kBlock + 8 * q;
        if (live) *reinterpret_cast<uint4*>(xs + at) = raw[g];
        const uint32_t w[4] = {raw[g].x, raw[g].y, raw[g].z, raw[g].w};
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint16_t h = static_cast<uint16_t>(w[k >> 1] >> (16 * (k & 1)));
          v[k] = live ? bf16_bits_to_float(h) : 0.f;
        }
        const int gl = blk / bpl, bb = blk % bpl;
        quant_quad_c2(v, xq + t * words, nb, bb * P.gu_lpr + gl, q, live);
      }
    }
  } else {
#pragma unroll 1
    for (int base0 = threadIdx.x & ~31; base0 < jobs * 4; base0 += kQD * nct) {
      uint16_t bits[kQD][8];
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        if (base0 + g * nct >= jobs * 4) break;
        const int job = min((base0 + g * nct + (threadIdx.x & 31)) >> 2, jobs - 1);
        const size_t a = static_cast<size_t>(job / nb) * P.d + (job % nb) * kBlock + q;
#pragma unroll
        for (int k = 0; k < 8; ++k) bits[g][k] = __ldcg(P.x + a + 4 * k);
      }
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        const int base = base0 + g * nct;  // warp-uniform
        if (base >= jobs * 4) break;
        const int job = (base + (threadIdx.x & 31)) >> 2;
        const bool live = job < jobs;
        const int t = live ? job / nb : 0, blk = live ? job % nb : 0;
        const size_t at = static_cast<size_t>(t) * P.d + blk * kBlock + q;
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (live) xs[at + 4 * k] = bits[g][k];
          v[k] = live ? bf16_bits_to_float(bits[g][k]) : 0.f;
        }
        const int gl = blk / bpl, bb = blk % bpl;
        quant_quad<BITS>(v, xq + t * words, nb, bb * P.gu_lpr + gl, q, live);
      }
    }
  }
}

// Quantises h rows [lo, hi) (fp32, global; this CTA's copy) into the down layout.
template <int BITS>
__device__ void quantise_h(const DLParams& P, int lo, int hi, int* hq, int nct, unsigned long long* tr) {
  const int nb = P.f / kBlock, bpl = nb / P.dn_lpr;
  const int words = QV<BITS>::kWords * nb;
  const int jobs = (hi - lo) * nb;
  const int q = threadIdx.x & 3;
  const float* hb = P.h + (blockIdx.x % kRep) * P.h_rep;
  if constexpr (BITS == 2) {
    // thread q of a block takes its 8 consecutive values in two 16-byte loads
#pragma unroll 1
    for (int base0 = threadIdx.x & ~31; base0 < jobs * 4; base0 += kQD * nct) {
      float4 raw[kQD][2];
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        if (base0 + g * nct >= jobs * 4) break;
        const int job = min((base0 + g * nct + (threadIdx.x & 31)) >> 2, jobs - 1);
        const float4* src =
            reinterpret_cast<const float4*>(hb + static_cast<size_t>(lo + job / nb) * P.f + (job % nb) * kBlock + 8 * q);
        raw[g][0] = __ldcg(src);
        raw[g][1] = __ldcg(src + 1);
      }
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        const int base = base0 + g * nct;  // warp-uniform
        if (base >= jobs * 4) break;
        const int job = (base + (threadIdx.x & 31)) >> 2;
        const bool live = job < jobs;
        const int r = live ? job / nb : 0, blk = live ? job % nb : 0;
        const float v[8] = {raw[g][0].x, raw[g][0].y, raw[g][0].z, raw[g][0].w,
                            raw[g][1].x, raw[g][1].y, raw[g][1].z, raw[g][1].w};
        if (tr != nullptr && g == 0 && threadIdx.x == 0) tr[30] = global_timer_ns() + (__float_as_uint(v[0]) & 0u);
        const int gl = blk / bpl, bb = blk % bpl;
        quant_quad_c2(v, hq + r * words, nb, bb * P.dn_lpr + gl, q, live);
      }
    }
  } else {
#pragma unroll 1
    for (int base0 = threadIdx.x & ~31; base0 < jobs * 4; base0 += kQD * nct) {
      float vals[kQD][8];
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        if (base0 + g * nct >= jobs * 4) break;
        const int job = min((base0 + g * nct + (threadIdx.x & 31)) >> 2, jobs - 1);
        const float* src = hb + static_cast<size_t>(lo + job / nb) * P.f + (job % nb) * kBlock + q;
#pragma unroll
        for (int k = 0; k < 8; ++k) vals[g][k] = __ldcg(src + 4 * k);
      }
#pragma unroll
      for (int g = 0; g < kQD; ++g) {
        const int base = base0 + g * nct;  // warp-uniform
        if (base >= jobs * 4) break;
        const int job = (base + (threadIdx.x & 31)) >> 2;
        const bool live = job < jobs;
        const int r = live ? job / nb : 0, blk = live ? job % nb : 0;
        float v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = live ? vals[g][k] : 0.f;
        if (tr != nullptr && g == 0 && threadIdx.x == 0) tr[30] = global_timer_ns() + (__float_as_uint(v[0]) & 0u);
        const int gl = blk / bpl, bb = blk % bpl;
        quant_quad<BITS>(v, hq + r * words, nb, bb * P.dn_lpr + gl, q, live);
      }
    }
  }
}

// Gate/up stage: warp w computes channel a + w (gate row and up row side by
// side) for every token of the stage's expert and writes h.
template <int BITS, int BPL>
__device__ __forceinline__ void process_gu(const StageRec& s, const uint8_t* ring, const DLParams& P,
                                           const RouteSmem& R, int np, const int* xq, int& cur_t, XR<BITS>* xr,
                                           unsigned long long* tr = nullptr) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c = s.a + warp;
  const int lpr = P.gu_lpr, gl = lane % lpr;
  const bool active = lane < lpr;  // lane group 0 holds the channel's two rows
  const int rows = 2 * (s.b - s.a);
  const int row_b = s.code_bytes / rows;
  const int nb = P.d / kBlock, sc_n = nb;
  const uint8_t* cg = ring + s.off + 2 * (c - s.a) * row_b;
  const uint16_t* sg = reinterpret_cast<const uint16_t*>(ring + s.off + s.code_bytes) + 2 * (c - s.a) * sc_n;
  int p0, p1;
  expert_rows(R, s.u, np, P.T, p0, p1);
#pragma unroll 1
  for (int p = p0; p < p1; ++p) {
    const int t = (s.u == kShared) ? p - np : R.pair_token[p];
    if (t != cur_t) {
      load_xr<BITS, BPL>(xq + t * QV<BITS>::kWords * nb, nb, lpr, gl, xr);
      cur_t = t;
    }
    if (tr != nullptr && lane == 0) tr[20] = clock64();
    float2 v = make_float2(0.f, 0.f);
    if (active) v = row_dot2<BITS, BPL>(cg, sg, cg + row_b, sg + sc_n, P.d, gl, xr);
    if (tr != nullptr && lane == 0) tr[21] = clock64() + (__float_as_uint(v.x) & 0u);
    v = group_sum2(v, lpr);
    if (tr != nullptr && lane == 0) tr[22] = clock64() + (__float_as_uint(v.y) & 0u);
    float hv = 0.f;
    // fast exponential and division: h is requantised to 16 bits for the
    // down rows, far coarser than their few-ulp error
    if (lane == 0) hv = __fdividef(v.x, 1.f + __expf(-v.x)) * v.y;
    hv = __shfl_sync(0xffffffffu, hv, 0);
    if (lane < kRep) P.h[lane * P.h_rep + static_cast<size_t>(p) * P.f + c] = hv;
    if (tr != nullptr && lane == 0) tr[23] = clock64();
  }
}

// Down stage (one expert, this CTA's output rows) by one warp: for every
// token of the expert, its quantised h row is held in registers and the
// rows are swept RPW at a time.
template <int BITS, int BPL>
__device__ __forceinline__ void process_dn(const StageRec& s, const uint8_t* ring, const DLParams& P,
                                           const RouteSmem& R, int np, const int* hq, int h_lo, float* zs) {
  const int lane = threadIdx.x & 31;
  const int lpr = P.dn_lpr, rpw = 32 / lpr;
  const int rl = lane / lpr, gl = lane % lpr;
  const int rows = s.b - s.a;
  const uint8_t* codes = ring + s.off;
  const uint16_t* scales = reinterpret_cast<const uint16_t*>(ring + s.off + s.code_bytes);
  const int row_b = s.code_bytes / rows;
  const int nb = P.f / kBlock, sc_n = nb;
  int p0, p1;
  expert_rows(R, s.u, np, P.T, p0, p1);
  XR<BITS> hr[BPL];
#pragma unroll 1
  for (int p = p0; p < p1; ++p) {
    load_xr<BITS, BPL>(hq + (p - h_lo) * QV<BITS>::kWords * nb, nb, lpr, gl, hr);
#pragma unroll 1
    for (int r0 = 0; r0 < rows; r0 += rpw) {
      const int r = r0 + rl;
      float v = 0.f;
      if (r < rows) v = row_dot<BITS, BPL>(codes + r * row_b, scales + r * sc_n, P.f, gl, hr);
      v = group_sum(v, lpr);
      if (gl == 0 && r < rows) zs[p * P.rpc + r] = v;
    }
  }
}

// Stable sort of the T*k pairs by expert inside the CTA, unique experts and
// slot lookup. Every consumer thread takes part.
__device__ void group_in_smem(const DLParams& P, const RouteSmem& R, DLShared* S, int np, int nct) {
  const int tid = threadIdx.x;
  for (int p = tid; p < np; p += nct) {
    const int e = min(max(R.idx[p], 0), P.E - 1);
    int pos = 0;
    for (int q = 0; q < np; ++q) {
      const int eq = min(max(R.idx[q], 0), P.E - 1);
      pos += (eq < e) || (eq == e && q < p);
    }
    R.sorted_e[pos] = e;
    R.pair_token[pos] = p / P.k;
    R.pair_gate[pos] = R.gate[p];
    R.pair_pos[p] = pos;
  }
  named_sync(1, nct);
  if (tid < 32) {
    int base = 0;
    for (int c = 0; c < np; c += 32) {
      const int i = c + tid;
      const bool first = i < np && (i == 0 || R.sorted_e[i - 1] != R.sorted_e[i]);
      const unsigned m = __ballot_sync(0xffffffffu, first);
      if (first) {
        const int u = base + __popc(m & ((1u << tid) - 1u));
        const int e = R.sorted_e[i];
        int slot = R.slot_s[e];
        if (slot < 0 || slot >= P.n_slots) {
          report(P.status, kDevBadSlot, e);
          slot = 0;
        }
        R.uniq_e[u] = e;
        R.uniq_slot[u] = slot;
        R.uniq_off[u] = i;
      }
      base += __popc(m);
    }
    if (tid == 0) {
      R.uniq_off[base] = np;
      S->n_uniq = base;
    }
  }
  named_sync(1, nct);
}

// CTA 0 publishes the grouping in the layout of moe_grouping.
__device__ void publish_grouping(const DLParams& P, const RouteSmem& R, int n_uniq, int np, int nct) {
  const int tid = threadIdx.x;
  for (int p = tid; p < np; p += nct) {
    P.g.pair_token[p] = R.pair_token[p];
    P.g.pair_gate[p] = R.pair_gate[p];
    P.g.pair_pos[p] = R.pair_pos[p];
    int j = 0;
    for (int q = 0; q < P.k; ++q) j = (R.pair_pos[R.pair_token[p] * P.k + q] == p) ? q : j;
    P.g.pair_j[p] = j;
    int u = 0;
    for (int v = 0; v < n_uniq; ++v) u = (R.uniq_off[v] <= p) ? v : u;
    P.g.pair_slot[p] = R.uniq_slot[u];
  }
  for (int u = tid; u < n_uniq; u += nct) {
    P.g.uniq_expert[u] = R.uniq_e[u];
    P.g.uniq_slot[u] = R.uniq_slot[u];
    P.g.uniq_offset[u] = R.uniq_off[u];
  }
  if (tid == 0) {
    P.g.uniq_offset[n_uniq] = np;
    *P.g.n_uniq = n_uniq;
  }
  for (int e = tid; e < P.E; e += nct) {
    int below = 0, cnt = 0;
    for (int q = 0; q < np; ++q) {
      below += R.sorted_e[q] < e;
      cnt += R.sorted_e[q] == e;
    }
    P.g.expert_count[e] = cnt;
    P.g.expert_offset[e] = below;
    if (e == P.E - 1) P.g.expert_offset[P.E] = below + cnt;
  }
}

// Top-k of token t by one warp over the fp32 logits in global memory, with
// the selection rule of the standalone top-k kernel: largest first, equal
// logits to the lower expert index, NaN below every number, -0 == +0.
// Key per value: order-preserving bits + 1 (NaN -> 1, taken/absent -> 0).
// Each round: warp max of the keys, then the lowest index holding it.
// E <= 512 (16 values per lane).
__device__ __forceinline__ uint32_t order_key(float v) {
  if (v != v) return 1u;
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return ((u & 0x80000000u) ? ~u : (u | 0x80000000u)) + 1u;
}

__device__ __forceinline__ float key_value(uint32_t k) {
  if (k <= 1u) return __uint_as_float(0x7fc00000u);
  const uint32_t o = k - 1u;
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

//
// Fast path: the k-th largest of the 32 lane maxima (a bitonic sort across
// the lanes) is a lower bound L of the k-th largest key, since those k lane
// maxima are k distinct values. When at most 32 keys reach L, they are
// compacted into `scratch` (32 words per warp) and each is ranked against the
// others in one pass; otherwise k rounds of warp max select them.
__device__ void topk_warp(const DLParams& P, const RouteSmem& R, int t, unsigned long long* scratch,
                          unsigned long long* tr) {
  constexpr int VPL = 16;
  const int lane = threadIdx.x & 31;
  const float* row = P.logits_rep + (static_cast<size_t>(blockIdx.x % kRep) * P.T + t) * P.E;
  // every load is issued before any is used: the index is clamped into the
  // row, so the loads need no guard and their latencies overlap
  float lv[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) lv[v] = __ldcg(row + min(v * 32 + lane, P.E - 1));
  uint32_t key[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) key[v] = v * 32 + lane < P.E ? order_key(lv[v]) : 0u;
  if (tr != nullptr && lane == 0) {
    uint32_t any = 0u;
#pragma unroll
    for (int v = 0; v < VPL; ++v) any |= key[v];
    tr[28] = global_timer_ns() + (any & 0u);
  }
  uint32_t mine_key = 0u;
  int mine_e = 0;
  uint32_t lmax = 0u;
#pragma unroll
  for (int v = 0; v < VPL; ++v) lmax = max(lmax, key[v]);
  uint32_t srt = lmax;  // bitonic sort of the lane maxima, descending
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint32_t o = __shfl_xor_sync(0xffffffffu, srt, stride);
      const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0 || size == 32);
      srt = keep_max ? max(srt, o) : min(srt, o);
    }
  }
  const uint32_t L = __shfl_sync(0xffffffffu, srt, P.k - 1);
  int cnt = 0;
#pragma unroll
  for (int v = 0; v < VPL; ++v) cnt += (L > 0u && key[v] >= L) ? 1 : 0;
  const int C = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
  if (L > 0u && C <= 32) {
    int pos = cnt;  // exclusive prefix of cnt over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, pos, o);
      if (lane >= o) pos += n;
    }
    pos -= cnt;
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (key[v] >= L)  // larger word = larger key, then lower expert index
        scratch[pos++] = (static_cast<unsigned long long>(key[v]) << 32) |
                         (0xffffffffu - static_cast<uint32_t>(v * 32 + lane));
    __syncwarp();
    const unsigned long long mine = lane < C ? scratch[lane] : 0ull;
    int rank = 0;
    for (int j = 0; j < C; ++j) rank += scratch[j] > mine ? 1 : 0;
    __syncwarp();
    if (lane < C && rank < P.k) scratch[rank] = mine;
    __syncwarp();
    if (lane < P.k) {
      const unsigned long long sel = scratch[lane];
      mine_key = static_cast<uint32_t>(sel >> 32);
      mine_e = static_cast<int>(0xffffffffu - static_cast<uint32_t>(sel & 0xffffffffu));
    }
    __syncwarp();
  } else {
#pragma unroll 1
  for (int j = 0; j < P.k; ++j) {
    uint32_t lm = 0u;
#pragma unroll
    for (int v = 0; v < VPL; ++v) lm = max(lm, key[v]);
    const uint32_t M = __reduce_max_sync(0xffffffffu, lm);
    uint32_t my = 0xffffffffu;
#pragma unroll
    for (int v = VPL - 1; v >= 0; --v)
      if (key[v] == M) my = static_cast<uint32_t>(v * 32 + lane);
    const int e = static_cast<int>(__reduce_min_sync(0xffffffffu, lm == M ? my : 0xffffffffu));
    // take the chosen value out (a select per element keeps key[] in registers)
#pragma unroll
    for (int v = 0; v < VPL; ++v) key[v] = (v * 32 + lane == e) ? 0u : key[v];
    if (lane == j) {
      mine_key = M;
      mine_e = e;
    }
  }
  }
  if (tr != nullptr && lane == 0) tr[29] = global_timer_ns() + (mine_key & 0u);
  const bool sel = lane < P.k;
  const float lj = sel ? key_value(mine_key) : 0.f;
  const float l0 = __shfl_sync(0xffffffffu, lj, 0);
  const float ex = sel ? expf(lj - l0) : 0.f;
  float denom;
  if (P.renorm) {
    denom = warp_sum(ex);
  } else {
    float s = 0.f;  // full-softmax denominator (re-read: keeps the logits out of registers above)
    for (int e = lane; e < P.E; e += 32) s += expf(__ldcg(row + e) - l0);
    denom = warp_sum(s);
  }
  if (sel) {
    R.idx[t * P.k + lane] = mine_e;
    R.gate[t * P.k + lane] = ex / denom;
  }
}

// Router rows [e0, e1) of this CTA for every token: lanes read W_r and x
// (both in shared memory) in interleaved 4-column groups. Every logit is
// written kRep times (one copy per group of readers).
__device__ void router_rows(const DLParams& P, const float* wrs, const uint16_t* xs, int e0, int e1, int cw) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n4 = P.d / 4;
  for (int t = 0; t < P.T; ++t) {
    const uint2* x2 = reinterpret_cast<const uint2*>(xs + static_cast<size_t>(t) * P.d);
#pragma unroll 1
    for (int e = e0 + warp; e < e1; e += cw) {
      const float4* w4 = reinterpret_cast<const float4*>(wrs + static_cast<size_t>(e - e0) * P.d);
      const size_t o = static_cast<size_t>(t) * P.E + e;
      const float bv = P.bias != nullptr ? __ldcg(P.bias + o) : 0.f;  // in flight during the dot product
      float acc = 0.f;
#pragma unroll 4
      for (int c4 = lane; c4 < n4; c4 += 32) {
        const float4 w = w4[c4];
        const uint2 xb = x2[c4];
        acc = fmaf(w.x, __uint_as_float(xb.x << 16), acc);
        acc = fmaf(w.y, __uint_as_float(xb.x & 0xffff0000u), acc);
        acc = fmaf(w.z, __uint_as_float(xb.y << 16), acc);
        acc = fmaf(w.w, __uint_as_float(xb.y & 0xffff0000u), acc);
      }
      acc = warp_sum(acc);
      if (lane < kRep) P.logits_rep[lane * static_cast<size_t>(P.T) * P.E + o] = acc + bv;
    }
  }
}

// ------------------------------------------------------------------ the kernel
// Control flow is the same for every consumer thread (all named barriers are
// reached by all of them); a timeout only turns the remaining work off.
template <int BITS, int GBPL, int DBPL, bool ROUTE>
__global__ void __launch_bounds__((consumer_warps(BITS) + 1) * 32, 1) decode_layer_kernel(const DLParams P) {
  constexpr int CW = consumer_warps(BITS);
  constexpr int CT = CW * 32;
  extern __shared__ __align__(128) char smem[];
  DLShared* S = reinterpret_cast<DLShared*>(smem);
  StageRec* st = reinterpret_cast<StageRec*>(smem + P.sm_stages);
  const int np = P.T * P.k;
  const RouteSmem R = route_smem(smem + P.sm_route, np);
  float* zs = reinterpret_cast<float*>(smem + P.sm_zs);
  int* xq = reinterpret_cast<int*>(smem + P.sm_xq);
  float* wrs = reinterpret_cast<float*>(smem + P.sm_wr);
  int* hq = reinterpret_cast<int*>(smem + P.sm_hq);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + P.sm_hq);  // raw x for the router (before hq is used)
  uint8_t* ring = reinterpret_cast<uint8_t*>(smem + P.sm_ring);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  const uint64_t t_start = global_timer_ns();
  const uint64_t deadline = t_start + P.timeout_ns;
  unsigned long long* trace = P.trace != nullptr && b < kTraceCtas ? P.trace + b * kTraceSlots : nullptr;
#define MOE_TRACE(slot) \
  if (trace != nullptr) trace[(slot)] = global_timer_ns();

  // static splits: router rows, shared-expert channels, output rows of this CTA
  const int e0 = static_cast<int>((static_cast<long long>(P.E) * b) / G);
  const int e1 = static_cast<int>((static_cast<long long>(P.E) * (b + 1)) / G);
  const int cs0 = static_cast<int>((static_cast<long long>(P.f) * b) / G);
  const int cs1 = static_cast<int>((static_cast<long long>(P.f) * (b + 1)) / G);
  const int r0 = min(b * P.rpc, P.d), r1 = min(r0 + P.rpc, P.d);

  if (warp == 0) {  // lane i initialises stage barrier pair i
    static_assert(kNB == 32, "one stage barrier pair per lane");
    mbar_init(&S->full[lane], 1);
    mbar_init(&S->empty[lane], CW);
    if (lane == 0) {
      if (trace != nullptr) {
        trace[0] = t_start;
        trace[14] = clock64();
      }
      mbar_init(&S->wr_bar, 1);
      mbar_init(&S->list_bar, 1);
      S->abort_flag = 0;
      S->n_sh = P.has_shared ? push_gu(st, 0, kShared, cs0, cs1, P) : 0;
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == CW) {
    // ------------------------------------------------------------ producer
    // lane 0 reserves ring space for up to 32 stages at a time, then every
    // lane issues one reserved stage
    Ring rg{0, 0, 0};
    bool ok = true, wr_issued = false;
    if (ROUTE && e1 > e0 && lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>((e1 - e0) * P.d * 4);
      mbar_arrive_expect_tx(&S->wr_bar, bytes);
      bulk_g2s(wrs, P.wr + static_cast<size_t>(e0) * P.d, bytes, &S->wr_bar);
      wr_issued = true;
    }
    const int n_sh = S->n_sh;
    int n_st = n_sh;
    if (!ROUTE) {
      // the grouping is already in global memory (written by an earlier
      // kernel): build the whole stage list now and stream every row at once
      grid_dep_wait();
      const int np = P.T * P.k;
      const int nu = min(max(__ldcg(P.g.n_uniq), 0), min(np, P.E));
      for (int u = lane; u < nu; u += 32) {
        int slot = __ldcg(P.g.uniq_slot + u);
        if (slot < 0 || slot >= P.n_slots) {
          report(P.status, kDevBadSlot, u);
          slot = 0;
        }
        R.uniq_slot[u] = slot;
      }
      __syncwarp();
      if (lane == 0) {
        build_routed_list(st, S, n_sh, nu, b, G, r0, r1, P);
        mbar_arrive(&S->list_bar);
      }
      __syncwarp();
    }
    bool listed = !ROUTE, planned = false;
    int i = 0;
    while (ok) {
      if (i == n_sh && !listed) {
        int got = 1;
        if (lane == 0) got = mbar_wait(&S->list_bar, 0, deadline) ? 1 : 0;
        got = __shfl_sync(0xffffffffu, got, 0);
        if (!got) {
          ok = false;
          break;
        }
        listed = true;
        if (lane == 0) MOE_TRACE(12)
      }
      if (listed) n_st = S->n_st;
      const int end = listed ? n_st : n_sh;
      if (i >= end) {
        if (listed) break;
        continue;
      }
      if (listed && !planned) {
        // Once the list is known, lay the rest of it out in the ring in one
        // step (a prefix sum over the stage sizes) if it fits the ring and the
        // stage mbarriers, and issue it in order. The stages before it (the
        // shared expert's gate/up, consumed after the routing step) stay
        // live: the layout goes after them, or, if it does not fit there,
        // they are waited for and freed first.
        planned = true;
        const int cnt = end - i;
        if (cnt <= 32) {
          const int need =
              lane < cnt ? (st[i + lane].bytes + kStageAlign - 1) / kStageAlign * kStageAlign : 0;
          int incl = need;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
          }
          const int tot = __shfl_sync(0xffffffffu, incl, 31);
          int base = -1, okp = 1;
          if (lane == 0) {
            // live stages stay if the layout fits after them and no stage of
            // it shares an mbarrier with one of them
            const bool live = rg.tail < rg.issued;
            if (live && rg.head > st[rg.tail].off && rg.head + tot <= P.ring_bytes && end - rg.tail <= kNB) {
              base = rg.head;
            } else if (tot <= P.ring_bytes) {
              while (rg.tail < rg.issued)
                if (!ring_pop(S, st, rg, deadline)) {
                  okp = 0;
                  break;
                }
              base = 0;
            }
          }
          okp = __shfl_sync(0xffffffffu, okp, 0);
          base = __shfl_sync(0xffffffffu, base, 0);
          if (!okp) {
            ok = false;
            break;
          }
          if (base >= 0) {
            if (lane < cnt) st[i + lane].off = base + incl - need;
            if (lane == 0) {
              rg.head = base + tot;
              rg.issued = end;
            }
            __syncwarp();
            if (lane == 0 && i == n_sh) MOE_TRACE(16)
            // at most two stages in flight: stage j is issued once stage j-2
            // has landed, so the copies arrive in the order they are consumed
            int okq = 1;
            if (lane == 0)
              for (int j = 0; j < cnt; ++j) {
                if (j >= 2 && !mbar_wait(&S->full[(i + j - 2) % kNB], ((i + j - 2) / kNB) & 1, deadline)) {
                  okq = 0;
                  rg.issued = i + j;
                  break;
                }
                stage_issue(S, st[i + j], i + j, ring, P, R);
              }
            okq = __shfl_sync(0xffffffffu, okq, 0);
            __syncwarp();
            if (lane == 0 && i == n_sh) MOE_TRACE(17)
            if (!okq) {
              ok = false;
              i = __shfl_sync(0xffffffffu, rg.issued, 0);
              break;
            }
            i = end;
            continue;
          }
        }
      }
      int batch = 0, okl = 1;
      if (lane == 0) {
        const int want = min(32, end - i);
        while (batch < want) {
          const int r = ring_alloc(S, st, rg, i + batch, P.ring_bytes, i, deadline);
          if (r == 0) okl = 0;
          if (r != 1) break;
          ++batch;
        }
      }
      okl = __shfl_sync(0xffffffffu, okl, 0);
      batch = __shfl_sync(0xffffffffu, batch, 0);
      if (lane == 0 && i == n_sh) MOE_TRACE(16)
      if (!okl) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane < batch) stage_issue(S, st[i + lane], i + lane, ring, P, R);
      __syncwarp();
      if (lane == 0 && i == n_sh) MOE_TRACE(17)
      i += batch;
    }
    if (lane == 0) MOE_TRACE(13)
    if (!ok) {
      // stages below i were issued (those reserved in a failed batch were not)
      rg.tail = __shfl_sync(0xffffffffu, rg.tail, 0);
      rg.issued = i;
      if (lane == 0) {
        if (!aborted(S)) set_abort(S, P.status, 10);
        // every issued copy must land before the CTA may exit; copies finish
        // in microseconds, the 100 ms bound only guards against the impossible
        const uint64_t d2 = global_timer_ns() + 100000000ull;
        for (int j = rg.tail; j < rg.issued; ++j) mbar_wait(&S->full[j % kNB], (j / kNB) & 1, d2);
        if (wr_issued) mbar_wait(&S->wr_bar, 0, d2);
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int tid = threadIdx.x;
  grid_dep_wait();  // x (and the workspace) may come from the previous kernel
  // this layer's slot table, fetched now and parked in shared memory after the
  // router, so that the slot lookup after top-k is a shared-memory read (the
  // routing path has E <= 2 * CT)
  int slot_v0 = 0, slot_v1 = 0;
  if (ROUTE) {
    if (tid < P.E) slot_v0 = __ldg(P.slot_of + tid);
    if (tid + CT < P.E) slot_v1 = __ldg(P.slot_of + tid + CT);
  }
  quantise_x<BITS>(P, xq, xs, CT);
  named_sync(1, CT);
  if (tid == 0) MOE_TRACE(1)

  if (ROUTE) {
    if (e1 > e0 && !mbar_wait_warp(&S->wr_bar, 0, deadline)) set_abort(S, P.status, 1);
    if (!aborted(S)) router_rows(P, wrs, xs, e0, e1, CW);
    if (tid < P.E) R.slot_s[tid] = slot_v0;
    if (tid + CT < P.E) R.slot_s[tid + CT] = slot_v1;
    named_sync(1, CT);
    if (tid == 0) MOE_TRACE(2)
    if (tid == 0 && !aborted(S)) S->bar_target = gbar_arrive(P.gbar, G);
  }

  // gate/up stages: the shared expert's [0, n_sh) need no routing and are
  // fetched from the start. With routing in the kernel it is resolved first
  // (loop index 0): the shared stages then run while the routed stages'
  // copies are on their way. Otherwise the list comes from the producer once
  // the loop reaches n_sh. The routed stages follow.
  XR<BITS> xr[GBPL];
  int cur_t = -1;
  const int n_sh = S->n_sh;
  int n_gu = n_sh;
#pragma unroll 1
  for (int i = 0;; ++i) {
    if (i == (ROUTE ? 0 : n_sh)) {
      // the cached x row (xr, cur_t) stays in registers across the routing
      // step: the routed stages of a token reuse it
      if (tid == 0) MOE_TRACE(3)
      if (ROUTE) {
        if (tid == 0 && !aborted(S) && !gbar_wait(P.gbar, S->bar_target, deadline)) set_abort(S, P.status, 3);
        named_sync(1, CT);
        if (tid == 0) MOE_TRACE(4)
        if (!aborted(S))
          for (int t = warp; t < P.T; t += CW)
            topk_warp(P, R, t, reinterpret_cast<unsigned long long*>(smem + P.sm_hq) + warp * 32,
                      t == 0 ? trace : nullptr);
        named_sync(1, CT);
        if (tid == 0) MOE_TRACE(10)
        if (b == 0)
          for (int q = tid; q < np; q += CT) {
            P.idx[q] = R.idx[q];
            P.gate[q] = R.gate[q];
          }
        group_in_smem(P, R, S, np, CT);
        if (b == 0) publish_grouping(P, R, S->n_uniq, np, CT);
      } else {
        // grouping written by moe_group_tokens; the producer has read the
        // slots and built the stage list
        const int nu_g = min(max(__ldcg(P.g.n_uniq), 0), min(np, P.E));
        for (int p = tid; p < np; p += CT) {
          R.pair_token[p] = min(max(__ldcg(P.g.pair_token + p), 0), P.T - 1);
          R.pair_gate[p] = __ldcg(P.g.pair_gate + p);
          R.pair_pos[p] = min(max(__ldcg(P.g.pair_pos + p), 0), np - 1);
        }
        for (int u = tid; u <= nu_g; u += CT) R.uniq_off[u] = min(max(__ldcg(P.g.uniq_offset + u), 0), np);
        if (!mbar_wait_warp(&S->list_bar, 0, deadline)) set_abort(S, P.status, 7);
      }
      if (ROUTE && tid == 0) {
        build_routed_list(st, S, n_sh, S->n_uniq, b, G, r0, r1, P);
        mbar_arrive(&S->list_bar);
      }
      named_sync(1, CT);
      if (tid == 0) MOE_TRACE(5)
      n_gu = S->n_gu;
    }
    if (i >= n_gu) break;
    if (!aborted(S) && warp < st[i].b - st[i].a) {
      if (mbar_wait_warp(&S->full[i % kNB], (i / kNB) & 1, deadline)) {
        if (tid == 0 && i == n_sh) MOE_TRACE(18)
        process_gu<BITS, GBPL>(st[i], ring, P, R, np, xq, cur_t, xr, (i == n_sh + 1 && warp == 0) ? trace : nullptr);
        if (tid == 0 && i == n_gu - 1) MOE_TRACE(19)
      } else {
        set_abort(S, P.status, 4);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S->empty[i % kNB]);
  }
  const int n_st = S->n_st;

  // every h row of every CTA must be written before any down row is computed
  named_sync(1, CT);
  if (tid == 0) MOE_TRACE(6)
  if (tid == 0 && !aborted(S)) {
    const unsigned long long target = gbar_arrive(P.gbar, G);
    if (!gbar_wait(P.gbar, target, deadline)) set_abort(S, P.status, 5);
  }
  named_sync(1, CT);
  if (tid == 0) MOE_TRACE(7)
  grid_dep_launch();
  if (tid == 0) MOE_TRACE(11)

  // down stages, in chunks whose h rows fit the quantised staging area
#pragma unroll 1
  for (int i0 = n_gu; i0 < n_st;) {
    int q0, q1;
    expert_rows(R, st[i0].u, np, P.T, q0, q1);
    const int h_lo = q0;
    int i1 = i0, h_hi = q0;
    while (i1 < n_st) {
      expert_rows(R, st[i1].u, np, P.T, q0, q1);
      if (q1 - h_lo > P.h_rows) break;
      h_hi = q1;
      ++i1;
    }
    quantise_h<BITS>(P, h_lo, h_hi, hq, CT, i0 == n_gu ? trace : nullptr);
    if (tid == 0 && i0 == n_gu) MOE_TRACE(31)
    named_sync(1, CT);
    if (tid == 0) MOE_TRACE(24)
#pragma unroll 1
    for (int i = i0; i < i1; ++i) {
      if (!aborted(S) && (i - n_gu) % CW == warp) {
        if (trace != nullptr && warp == 1 && lane == 0) trace[25] = global_timer_ns();
        const bool got = mbar_wait_warp(&S->full[i % kNB], (i / kNB) & 1, deadline);
        if (trace != nullptr && warp == 1 && lane == 0) trace[26] = global_timer_ns();
        if (got)
          process_dn<BITS, DBPL>(st[i], ring, P, R, np, hq, h_lo, zs);
        else
          set_abort(S, P.status, 6);
        if (trace != nullptr && warp == 1 && lane == 0) trace[27] = global_timer_ns();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S->empty[i % kNB]);
    }
    named_sync(1, CT);
    i0 = i1;
  }
  if (tid == 0) MOE_TRACE(8)
  if (aborted(S)) return;

  // combine: y[t, r] = sum_j gate[t,j] z[(t,j)][r] + z_shared[t][r] (+ x)
  const int nr = r1 - r0;
  for (int i = tid; i < P.T * nr; i += CT) {
    const int t = i / nr, rr = i % nr;
    float acc = 0.f;
    for (int j = 0; j < P.k; ++j) {
      const int p = R.pair_pos[t * P.k + j];
      acc = fmaf(R.pair_gate[p], zs[p * P.rpc + rr], acc);
    }
    if (P.has_shared) acc += zs[(np + t) * P.rpc + rr];
    const size_t o = static_cast<size_t>(t) * P.d + r0 + rr;
    if (P.residual) acc += bf16_bits_to_float(P.x[o]);
    if (P.out_f32) static_cast<float*>(P.y)[o] = acc;
    else static_cast<__nv_bfloat16*>(P.y)[o] = __float2bfloat16_rn(acc);
  }
  named_sync(1, CT);
  if (tid == 0) {
    MOE_TRACE(9)
    if (trace != nullptr) trace[15] = clock64();
  }
#undef MOE_TRACE
}

// ------------------------------------------------------------------ host side
namespace {

struct RowGeom {
  int lpr, bpl;
};

RowGeom row_geom(int K) {
  const int nb = K / kBlock;
  int lpr = 1;
  while (lpr < 32 && nb % (lpr * 2) == 0) lpr *= 2;
  return RowGeom{lpr, nb / lpr};
}

size_t align_up(size_t n, size_t a) { return (n + a - 1) / a * a; }

constexpr int kSmemMax = 227 * 1024;

typedef void (*DLKernel)(const DLParams);

template <int BITS, bool ROUTE>
DLKernel pick(int gbpl, int dbpl) {
  if (gbpl == 2 && dbpl == 3) return decode_layer_kernel<BITS, 2, 3, ROUTE>;
  if (gbpl == 1 && dbpl == 1) return decode_layer_kernel<BITS, 1, 1, ROUTE>;
  if (gbpl == 2 && dbpl == 2) return decode_layer_kernel<BITS, 2, 2, ROUTE>;
  if (gbpl == 2 && dbpl == 1) return decode_layer_kernel<BITS, 2, 1, ROUTE>;
  if (gbpl == 1 && dbpl == 3) return decode_layer_kernel<BITS, 1, 3, ROUTE>;
  if (gbpl == 4 && dbpl == 3) return decode_layer_kernel<BITS, 4, 3, ROUTE>;
  return nullptr;
}

DLKernel pick_kernel(int bits, bool route, int gbpl, int dbpl) {
  if (bits == 2) return route ? pick<2, true>(gbpl, dbpl) : pick<2, false>(gbpl, dbpl);
  return route ? pick<3, true>(gbpl, dbpl) : pick<3, false>(gbpl, dbpl);
}

}  // namespace

bool decode_geometry_ok(int d, int f) {
  return pick_kernel(2, true, row_geom(d).bpl, row_geom(f).bpl) != nullptr;
}

cudaError_t decode_init(const Ctx& ctx) {
  (void)ctx;
  const int combos[6][2] = {{2, 3}, {1, 1}, {2, 2}, {2, 1}, {1, 3}, {4, 3}};
  for (int bits = 2; bits <= 3; ++bits)
    for (int r = 0; r < 2; ++r)
      for (const auto& c : combos) {
        const cudaError_t e = cudaFuncSetAttribute(pick_kernel(bits, r != 0, c[0], c[1]),
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax);
        if (e != cudaSuccess) return e;
      }
  return cudaSuccess;
}

cudaError_t launch_decode_layer(const Ctx& ctx, const moe_layer_cfg& c, const DecodeArgs& a, cudaStream_t s) {
  const RowGeom gg = row_geom(c.d), gd = row_geom(c.f);
  if (a.route && c.E > 512) return cudaErrorNotSupported;  // fused top-k holds 16 logits per lane
  DLKernel kern = pick_kernel(c.bits, a.route, gg.bpl, gd.bpl);
  if (kern == nullptr) return cudaErrorNotSupported;
  const int G = ctx.num_sms;
  const int CW = consumer_warps(c.bits);
  const int T = a.T, np = T * c.k;
  DLParams P{};
  P.x = a.x;
  P.T = T;
  P.d = c.d;
  P.f = c.f;
  P.E = c.E;
  P.k = c.k;
  P.renorm = c.renorm;
  P.residual = c.residual;
  P.has_shared = a.shared != nullptr;
  P.out_f32 = c.out_fp32;
  P.wr = a.wr;
  P.bias = a.bias;
  P.logits = a.logits;
  P.idx = a.idx;
  P.gate = a.gate;
  P.slot_of = a.slot_of;
  P.n_slots = a.n_slots;
  P.g = *a.g;
  P.pool = a.pool;
  P.stride = a.stride;
  P.shared = a.shared;
  P.lay = a.lay;
  P.h = a.h;
  P.h_rep = static_cast<size_t>(np + (c.n_shared ? T : 0)) * c.f;
  P.logits_rep = a.logits_rep;
  P.y = a.y;
  P.status = ctx.d_status;
  P.gbar = ctx.d_gbar;
  P.timeout_ns = ctx.timeout_ns;
  P.trace = ctx.d_trace;
  P.gu_lpr = gg.lpr;
  P.dn_lpr = gd.lpr;
  P.gu_row = c.d * c.bits / 8;
  P.gu_sc = c.d / kBlock * 2;
  P.dn_row = c.f * c.bits / 8;
  P.dn_sc = c.f / kBlock * 2;
  P.gu_chan = CW;
  // output rows per CTA: a multiple of the smallest row count whose code and
  // scale bytes are both multiples of 16 (bulk-copy granularity)
  int gran = 1;
  while ((gran * P.dn_row) % 16 != 0 || (gran * P.dn_sc) % 16 != 0) gran *= 2;
  P.rpc = static_cast<int>(align_up((c.d + G - 1) / G, gran));
  P.wr_rows = (c.E + G - 1) / G;
  const int n_uniq_max = np < c.E ? np : c.E;
  // the device-side list arithmetic is 32-bit: nu * f * G must stay below 2^31
  if (static_cast<long long>(n_uniq_max) * c.f * G >= (1LL << 31)) return cudaErrorNotSupported;
  const int sh_ch = (c.f + G - 1) / G;
  P.max_stages = (sh_ch + CW - 1) / CW + 1 +
                 static_cast<int>((static_cast<long long>(n_uniq_max) * c.f + G - 1) / G + CW - 1) / CW +
                 n_uniq_max + 2 + n_uniq_max + 2;
  const size_t qw = c.bits == 3 ? 34 : 18;  // words per quantised block
  size_t o = align_up(sizeof(DLShared), 128);
  P.sm_stages = static_cast<int>(o);
  o = align_up(o + static_cast<size_t>(P.max_stages) * sizeof(StageRec), 128);
  P.sm_route = static_cast<int>(o);
  o = align_up(o + (9 * static_cast<size_t>(np) + 1 + (a.route ? c.E : 0)) * 4, 128);
  P.sm_zs = static_cast<int>(o);
  o = align_up(o + static_cast<size_t>(np + T) * P.rpc * 4, 128);  // z rows [np + T][rpc]
  P.sm_xq = static_cast<int>(o);
  o = align_up(o + static_cast<size_t>(T) * qw * (c.d / kBlock) * 4, 128);
  P.sm_wr = static_cast<int>(o);
  if (a.route) o = align_up(o + static_cast<size_t>(P.wr_rows) * c.d * 4, 128);
  // quantised h rows for the down phase: every row if they fit in 48 KB, else
  // as many as fit (at least the T rows one expert can have)
  const int n_rows_all = np + (P.has_shared ? T : 0);
  const size_t h_row_bytes = qw * (c.f / kBlock) * 4;
  const int h_cap = static_cast<int>((48 * 1024) / h_row_bytes);
  P.h_rows = n_rows_all < h_cap ? n_rows_all : (h_cap > T ? h_cap : T);
  P.sm_hq = static_cast<int>(o);  // also holds the raw x [T, d] bf16 before the down phase
  const size_t hq_bytes = static_cast<size_t>(P.h_rows) * h_row_bytes;
  const size_t xs_bytes = static_cast<size_t>(T) * c.d * 2;
  const size_t tk_bytes = static_cast<size_t>(CW) * 32 * 8;  // top-k scratch (after the router, before hq)
  size_t region = hq_bytes > xs_bytes ? hq_bytes : xs_bytes;
  region = region > tk_bytes ? region : tk_bytes;
  o = align_up(o + region, 128);
  P.sm_ring = static_cast<int>(o);
  const long long ring = static_cast<long long>(kSmemMax) - static_cast<long long>(o);
  const long long gu_stage = 2LL * CW * (P.gu_row + P.gu_sc);
  const long long dn_stage = static_cast<long long>(P.rpc) * (P.dn_row + P.dn_sc);
  if (ring < 2 * (gu_stage > dn_stage ? gu_stage : dn_stage)) return cudaErrorNotSupported;
  P.ring_bytes = static_cast<int>(ring / kStageAlign * kStageAlign);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3((CW + 1) * 32);
  cfg.dynamicSmemBytes = kSmemMax;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace moe
