// Decode path (T <= MOE_DECODE_MAX_T): one persistent kernel runs L
// consecutive layers, layer l + 1 taking layer l's output as its input.
//
// The pages' engine reads, per token and layer, the router, the shared expert
// and the 10 routed experts the router picks, and its speed is set by how fast
// those bytes arrive (vramglass.com, sections なぜVRAM 12GBで足りるのか and
// その2：GPUとCPUで同時に計算する; news.blueqat.app/post/3262, section
// GPU・CPU・RAM・SSDの分担); each layer waits for the previous one (the same
// page, section その2: the GPU and CPU halves join before the next layer). On a
// B200 every expert sits in HBM, so a layer is a short chain of dependent
// steps around ~16-50 MB of weight reads. This kernel keeps that chain short:
//
//  * One CTA per SM (a cooperative launch, so all CTAs are resident), one
//    producer warp issuing cp.async.bulk copies of down rows and 15 (2-bit)
//    or 11 (3-bit) consumer warps.
//  * Cross-CTA data (x, h) moves as 64-bit words that carry a 32-bit payload
//    and a 32-bit tag naming the layer; a reader polls the words themselves
//    until every tag matches. Tags come from a per-device counter that every
//    launch advances, so words left by earlier launches never match. Where
//    every CTA must have finished a step (the logits, h), each adds 1 to a
//    per-device completion counter and one thread per CTA waits for it.
//  * Per layer: the logits are already summed (below) -> top-k and grouping
//    in every CTA while the other warps read x -> each consumer warp streams
//    the gate/up rows of its own channel tasks with cp.async while the
//    producer streams this CTA's down rows into a ring -> gate/up + SwiGLU,
//    each 32-channel block of h requantised to int16 by the CTA that owns it
//    and published as words -> every CTA stages all of h and computes its
//    slice of output rows for every expert -> combine -> output words (the
//    next layer's x) -> this CTA's partial logits of the next layer from
//    those rows, added into exact fixed-point accumulators.
//  * Layer l + 1's router columns and shared expert do not depend on x: they
//    are fetched while layer l is still running.
//
// Every wait is bounded by a global-timer deadline; on expiry the kernel
// records MOE_ETIMEOUT in the context's status word, stops working and
// returns. A kernel that finds the status word already set does nothing.
#include <cstdio>
#include <cstdlib>
#include <random>

#include "moe_internal.cuh"
#include "dequant.cuh"

namespace moe {

__host__ __device__ constexpr int ds_consumer_warps(int bits) { return bits == 2 ? 15 : 11; }
constexpr int kDsNS = 12;       // weight ring slots (at most)
constexpr int kDsMaxBlk = 40;   // gate/up channel blocks of one CTA in one layer (at most)
constexpr int kDsArr = 16;      // arrivals that release a ring slot (one down group)
constexpr int kDsGuDepth = 4;   // gate/up tasks a consumer warp has in flight
constexpr int kDsGpd = 6;       // routed experts per down group (ring slot)
constexpr int kQW = 18;         // words per quantised 32-value block: 16 int16 pairs, scale, sum
constexpr int kDsMaxCtas = 256;  // grid size limit (done words per layer parity)
constexpr int kDsPollNs = 64;      // back-off between polls of words that were not there yet

// Tag source: every launch reads it and the last CTA to exit advances it by
// the number of layers; tags of a launch are base + 1 .. base + L.
__device__ unsigned int g_ds_epoch;
__device__ unsigned int g_ds_exit;
// Completion counters, one per 128-byte line: kCntOut (a layer's output rows
// and the next layer's partial logits) takes 1 from every CTA per layer, so
// after layer l of a launch with tag base `base` it holds (base + l + 1) * G
// (mod 2^32); kCntZero (the first two accumulator sets zeroed) and
// kCntLogits (layer 0's partial logits added) take L from every CTA in the
// prologue. All advance in step with the tag counter. (kCntH, once the count
// of a layer's h blocks, is no longer added to: the h words carry tags.)
constexpr int kCntLogits = 0, kCntH = 32, kCntOut = 64, kCntZero = 96;
__device__ unsigned int g_ds_cnt[128];

// Division by a runtime constant with one wide multiply: n / d for n < 2^31
// and n < 2^32 / d, with m = floor(2^32 / d) + 1 (the remainder term stays
// below one step of n / d in that range).
struct FastDiv {
  uint32_t d;
  unsigned long long m;
};

__host__ __device__ inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  f.m = 0x100000000ull / d + 1;
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv& f) {
  return static_cast<uint32_t>((static_cast<unsigned long long>(n) * f.m) >> 32);
}

__device__ __forceinline__ uint32_t fmod_(uint32_t n, const FastDiv& f) { return n - fdiv(n, f) * f.d; }

// Offsets (bytes) of the arrays of one layer's routing record.
struct RecOff {
  int logits, idx, gate, expert_count, expert_offset, pair_token, pair_j, pair_gate, pair_slot, pair_pos;
  int uniq_expert, uniq_slot, uniq_offset, n_uniq;
};

struct DSParams {
  const uint16_t* x;            // [T, d] bf16: layer 0's input
  int T, d, f, E, k, L, renorm, residual, has_shared, out_f32;
  int skip_from, hot_slots;  // pairs of rank >= skip_from on a slot >= hot_slots are left out (skip_from > 0)
  const float* wr;              // route: [L, E, d]
  const float* bias;            // route: null or [L, T, E]
  const int32_t* slot_of;       // route: [L, E]
  int n_slots;
  const uint8_t* pool;
  size_t stride;
  const uint8_t* shared;        // layer l's shared expert at shared + l * stride, or null
  moe_expert_layout lay;
  void* y;                      // [L, T, d]
  char* rec;                    // route: layer l's routing record at rec + l * rec_bytes
  size_t rec_bytes;
  RecOff ro;
  GroupPtrs g;                  // not route: the given grouping
  long long* lacc;                // [3, 3, T, E] router logits in fixed point: [part][layer % 3]; parts
                                  // in units of 2^-32, 2^22 and 2^76
  int* lbad;                      // [3, T, E] flags: 1 a partial was not finite, 2 / 4 part 1 / 2 used
  unsigned long long* h_ll;       // [n_rows, f/32, kQW]
  unsigned long long* y_ll;       // [2, T, d/2]
  int* status;
  unsigned long long timeout_ns;
  unsigned long long* trace;
  // geometry (host computed)
  int gu_lpr, dn_lpr, gran, n_units;
  int gu_lsh, dn_lsh;           // log2 of gu_lpr, dn_lpr (both powers of two)
  FastDiv fd_nb, fd_nbf, fd_ring, fd_gpd;  // d / 32, f / 32, ring slots, down stages per slot
  FastDiv fd_hrow, fd_hp;  // 16-byte units of a quantised h row; rpc / 2
  int gu_row, gu_sc, dn_row, dn_sc;  // bytes per row: codes, scales
  int rpc;                      // output rows per CTA (at most)
  int n_ring, slot_bytes;       // weight ring: slots and bytes per slot
  int dn_stride, gpd;           // bytes per down stage, down stages per ring slot
  int hq_rows;
  int sm_ws, sm_ysl, sm_x, sm_xq, sm_hs, sm_zs, sm_route, sm_xres, sm_ring, sm_shdn;
  int sm_gub, gu_task_bytes, gu_depth;  // per-warp gate/up buffers: gu_depth tasks of gu_task_bytes each
  int max_blk;                  // gate/up blocks of one CTA in one layer (h staging slots)
};

struct DSShared {
  uint64_t full[kDsNS], empty[kDsNS];   // weight ring
  uint64_t shdn_full[2], shdn_empty[2];  // the shared expert's down rows, by layer parity
  uint64_t route_bar;
  int abort_flag;
  unsigned base_tag;
  int n_uniq;
  int route_ok;  // this layer's routing in shared memory is complete (read behind route_bar)
  // A copy of the launch parameters for the out-of-line helpers: they read
  // it from shared memory instead of from a per-thread stack copy.
  DSParams prm;
};

// Start of part b of n items split into G near-equal parts (n * G < 2^31,
// which the launch checks).
__device__ __forceinline__ int split_at(int n, int b, int G) {
  return static_cast<int>(static_cast<unsigned>(n) * static_cast<unsigned>(b) / static_cast<unsigned>(G));
}

// The kernel's dynamic shared memory.
extern __shared__ __align__(128) char ds_smem[];

struct DSRoute {
  int32_t* idx;        // [np]  top-k of token t at t*k + j
  float* gate;         // [np]
  int32_t* sorted_e;   // [np]  expert of each sorted pair
  int32_t* pair_token; // [np]
  float* pair_gate;    // [np]
  int32_t* pair_pos;   // [np]  sorted position of pair t*k + j
  int32_t* uniq_e;     // [np]
  int32_t* uniq_slot;  // [np]
  int32_t* uniq_off;   // [np + 1]
  int32_t* slot_s;     // [E]   this layer's slot table
};

__device__ __forceinline__ DSRoute ds_route(char* base, int np) {
  DSRoute r;
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

// ------------------------------------------------------------------ tagged words
__device__ __forceinline__ unsigned long long ll_word(uint32_t v, uint32_t tag) {
  return (static_cast<unsigned long long>(tag) << 32) | v;
}

__device__ __forceinline__ void st_ll(unsigned long long* p, unsigned long long w) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}

__device__ __forceinline__ void st_ll2(unsigned long long* p, unsigned long long a, unsigned long long b) {
  asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(a), "l"(b) : "memory");
}

__device__ __forceinline__ unsigned long long ld_ll(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void ld_ll2(const unsigned long long* p, unsigned long long& a, unsigned long long& b) {
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

__device__ __forceinline__ bool tag_ok(unsigned long long w, uint32_t tag) {
  return static_cast<uint32_t>(w >> 32) == tag;
}

__device__ __forceinline__ bool mbar_test(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void ds_abort(DSShared* S, int* status, int where) {
  report(status, kDevTimeout, where);
  *reinterpret_cast<volatile int*>(&S->abort_flag) = 1;
}

__device__ __forceinline__ bool ds_aborted(const DSShared* S) {
  return *reinterpret_cast<const volatile int*>(&S->abort_flag) != 0;
}

// Counts this CTA's part of an exchange as written (the tagged words it
// stored before the last CTA barrier); relaxed, fire and forget.
__device__ __forceinline__ void cnt_add(int which, unsigned n = 1u) {
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(&g_ds_cnt[which]), "r"(n) : "memory");
}

// Polls an exchange counter (one thread) until it reaches `target`
// (wrap-safe); false on timeout or abort.
__device__ __forceinline__ bool cnt_wait(int which, unsigned target, DSShared* S, int* status, int where,
                                         uint64_t deadline) {
  while (true) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(&g_ds_cnt[which]) : "memory");
    if (static_cast<int>(v - target) >= 0) return true;
    if (*reinterpret_cast<volatile int*>(&S->abort_flag) != 0) return false;
    if (global_timer_ns() > deadline) {
      report(status, kDevTimeout, where);
      *reinterpret_cast<volatile int*>(&S->abort_flag) = 1;
      return false;
    }
    __nanosleep(32);
  }
}

// The same, agreed by the whole warp (call with the warp converged): code
// that follows it may use full-warp collectives.
__device__ __forceinline__ bool ds_aborted_warp(const DSShared* S) {
  return __any_sync(0xffffffffu, ds_aborted(S));
}

// Warp-wide bounded mbarrier wait by lane 0 (false on timeout or abort).
__device__ __forceinline__ bool ds_wait_warp(uint64_t* b, uint32_t parity, const DSShared* S, uint64_t deadline) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) {
    while (!mbar_try_wait(b, parity, 20000u)) {
      if (ds_aborted(S) || global_timer_ns() > deadline) {
        ok = 0;
        break;
      }
    }
  }
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ------------------------------------------------------------------ quantised vectors
// A vector block in shared memory holds kQW words in the column layout of
// dequant.cuh (word w of block column col at vec[w * nb + col]): 16 int16
// pairs, the scale and the integer sum. For 3-bit weights the high-plane
// pairs are rebuilt from the low-plane words when the block is loaded: pair
// (v_t, v_t+8) takes the halves of words t%4 and 4 + t%4 that hold v_t and
// v_t+8, and the same for the second 16 values.
template <int BITS, int BPL>
__device__ __forceinline__ void load_xq(const int* __restrict__ vec, int nb, int lpr, int gl, XR<BITS>* xr) {
#pragma unroll
  for (int bb = 0; bb < BPL; ++bb) {
    const int col = bb * lpr + gl;
#pragma unroll
    for (int w = 0; w < 16; ++w) xr[bb].p[w] = vec[w * nb + col];
    xr[bb].sx = __int_as_float(vec[16 * nb + col]);
    xr[bb].sum = vec[17 * nb + col];
    if (BITS == 3) {
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const uint32_t sel = (t < 4) ? 0x5410u : 0x7632u;
        xr[bb].ph[t] = static_cast<int>(__byte_perm(xr[bb].p[t & 3], xr[bb].p[4 + (t & 3)], sel));
        xr[bb].ph[8 + t] = static_cast<int>(__byte_perm(xr[bb].p[8 + (t & 3)], xr[bb].p[12 + (t & 3)], sel));
      }
    }
  }
}

// Quantises the 32 values of one block held one per lane (lane c holds value
// c) and returns the word this lane owns (lanes 0..17), in the layout above.
__device__ __forceinline__ uint32_t quant_block_warp(float v, int lane) {
  const float m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(v))));
  const float inv = m > 0.f ? __fdividef(32767.f, m) : 0.f;
  constexpr float kMagic = 12582912.f;  // 1.5 * 2^23: rint(v * inv) in the low bits
  const int r = __float_as_int(fmaf(v, inv, kMagic));
  const int sum = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(r - 0x4B400000)));
  // word k < 16 pairs values a_k and a_k + 4, a_k = 16(k/8) + k%4 + 8((k/4)%2)
  const int a = 16 * (lane >> 3) + (lane & 3) + 8 * ((lane >> 2) & 1);
  const int ra = __shfl_sync(0xffffffffu, r, a & 31);
  const int rb = __shfl_sync(0xffffffffu, r, (a + 4) & 31);
  if (lane < 16) return __byte_perm(ra, rb, 0x5410);
  if (lane == 16) return __float_as_uint(m * (1.f / 32767.f));
  return static_cast<uint32_t>(sum);
}

// ------------------------------------------------------------------ x of a layer
// Every consumer thread takes part. Layer 0 (or the given-grouping mode)
// reads the bf16 input; layer l > 0 reads the previous layer's output words
// and every CTA's done word. A thread issues the loads of up to kXB jobs
// (four words each) at once and re-polls, all together, only the words whose
// tag was not there yet, so a batch costs about one L2 round trip. Writes the
// raw bf16 rows (xs, for the router), the quantised gate/up operand (xq) and
// this CTA's residual rows (xres).
constexpr int kXB = 1;

template <int BITS, int GBPL>
__device__ void ds_read_x(const DSParams& P, int l, uint32_t tag, uint16_t* xs, int* xq, float* xres, int r0,
                          int r1, DSShared* S, uint64_t deadline, int tid0, int CT) {
  const int nb = P.d / kBlock;
  const int words = kQW * nb;
  const int jobs = P.T * nb * 4;  // four threads per 32-value block
  const int tid = threadIdx.x - tid0;  // the threads [tid0, tid0 + CT) take part (whole warps)
  const bool chained = l > 0;
  const unsigned long long* yl = P.y_ll + static_cast<size_t>((l - 1) & 1) * P.T * (P.d / 2);
  const int per_thread = (jobs + CT - 1) / CT;
#pragma unroll 1
  for (int k0 = 0; k0 < per_thread; k0 += kXB) {
    uint32_t w4[kXB][4];
    if (!chained) {
#pragma unroll
      for (int i = 0; i < kXB; ++i) {
        const int j = tid + (k0 + i) * CT;
        const int job = j < jobs ? j >> 2 : 0, q = j & 3;
        const int t = fdiv(job, P.fd_nb), blk = job - t * nb;
        const uint4 raw = j < jobs ? __ldcg(reinterpret_cast<const uint4*>(P.x + static_cast<size_t>(t) * P.d +
                                                                           blk * kBlock + 8 * q))
                                   : make_uint4(0u, 0u, 0u, 0u);
        w4[i][0] = raw.x;
        w4[i][1] = raw.y;
        w4[i][2] = raw.z;
        w4[i][3] = raw.w;
      }
    } else {
      unsigned long long v[kXB][4];
      const unsigned long long* src[kXB];
#pragma unroll
      for (int i = 0; i < kXB; ++i) {
        const int j = tid + (k0 + i) * CT;
        const int job = j < jobs ? j >> 2 : 0, q = j & 3;
        const int t = fdiv(job, P.fd_nb), blk = job - t * nb;
        src[i] = yl + static_cast<size_t>(t) * (P.d / 2) + blk * 16 + 4 * q;
        if (j < jobs) {
          ld_ll2(src[i], v[i][0], v[i][1]);
          ld_ll2(src[i] + 2, v[i][2], v[i][3]);
        } else {  // no load: a slot past the end counts as present
          v[i][0] = v[i][1] = v[i][2] = v[i][3] = ll_word(0u, tag - 1);
        }
      }
      while (true) {
        bool all = true;
#pragma unroll
        for (int i = 0; i < kXB; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c) all = all && tag_ok(v[i][c], tag - 1);
        if (all) break;
        if (ds_aborted(S) || global_timer_ns() > deadline) {
          if (!ds_aborted(S)) ds_abort(S, P.status, 21);
          break;
        }
        __nanosleep(kDsPollNs);
#pragma unroll
        for (int i = 0; i < kXB; ++i)
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (!tag_ok(v[i][c], tag - 1)) v[i][c] = ld_ll(src[i] + c);
      }
#pragma unroll
      for (int i = 0; i < kXB; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) w4[i][c] = static_cast<uint32_t>(v[i][c]);
    }
#pragma unroll
    for (int i = 0; i < kXB; ++i) {
      if (k0 + i >= per_thread) break;  // uniform across the warp
      const int j = tid + (k0 + i) * CT;
      const bool live = j < jobs;
      const int job = live ? j >> 2 : 0, q = j & 3;
      const int t = fdiv(job, P.fd_nb), blk = job - t * nb;
      float v8[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint16_t h = static_cast<uint16_t>(w4[i][e >> 1] >> (16 * (e & 1)));
        v8[e] = live ? bf16_bits_to_float(h) : 0.f;
      }
      if (live) {
        if (xs != nullptr)
          *reinterpret_cast<uint4*>(xs + static_cast<size_t>(t) * P.d + blk * kBlock + 8 * q) =
              make_uint4(w4[i][0], w4[i][1], w4[i][2], w4[i][3]);
        const int c0 = blk * kBlock + 8 * q;
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (c0 + e >= r0 && c0 + e < r1) xres[t * P.rpc + (c0 + e - r0)] = v8[e];
      }
      const int gl = blk / GBPL, bb = blk - gl * GBPL;
      quant_quad_c2(v8, xq + t * words, nb, (bb << P.gu_lsh) + gl, q, live);
    }
  }
}

// ------------------------------------------------------------------ top-k
// Selection rule (as the standalone top-k kernel): largest first, equal
// logits to the lower expert index, NaN below every number, -0 == +0.
// Key per value: order-preserving bits + 1 (NaN -> 1, taken/absent -> 0).
__device__ __forceinline__ uint32_t ds_order_key(float v) {
  if (v != v) return 1u;
  uint32_t u = __float_as_uint(v);
  if (u == 0x80000000u) u = 0u;
  return ((u & 0x80000000u) ? ~u : (u | 0x80000000u)) + 1u;
}

__device__ __forceinline__ float ds_key_value(uint32_t k) {
  if (k <= 1u) return __uint_as_float(0x7fc00000u);
  const uint32_t o = k - 1u;
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

constexpr int kDsMaxE = 512;  // experts a decode launch supports

// ---- router, split by rows: CTA b owns output rows [r0, r1) of every
// layer. With x_{l+1} = y_l, its rows of y_l (bf16, as the next layer reads
// them) against the same columns of layer l+1's router give a partial logit
// for every (token, expert); the partials of all CTAs add up to the logits.
// They are added as 64-bit integers, so the sum is exact and does not depend
// on the order the CTAs arrive in. A partial p is cut into three parts in
// units of 2^-32, 2^22 and 2^76: the multiple of 2^76 (p's bits at and above
// 2^76), the multiple of 2^22 in what remains, and the rest rounded to
// 2^-32. Every part is below 2^54 in magnitude, so up to 2^9 CTAs add without
// overflow. The cut is exact for |p| >= 2^22 (its unit is then at least 2^-1);
// below that, p is rounded to 2^-32 alone, the one rounding there is. A flag
// word per logit tells the reader which of the upper parts were used; a
// partial that is not finite sets flag 1 and the logit reads NaN.
constexpr double kLogitUlp = 1.0 / 4294967296.0;
constexpr double kLogitUnit1 = 4194304.0;                  // 2^22
constexpr double kLogitUnit2 = 75557863725914323419136.0;  // 2^76

__device__ __forceinline__ long long ld_relaxed_s64(const long long* p) {
  long long v;
  asm volatile("ld.relaxed.gpu.global.s64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ int ld_relaxed_s32(const int* p) {
  int v;
  asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Columns [r0, r1) of every row of layer l's router into ws (rpc floats per
// expert), 8-byte cp.async pieces spread over the given threads; one commit.
__device__ __forceinline__ void ds_wslice_load(const DSParams& P, int l, float* ws, int r0, int r1, int tid,
                                               int nthreads) {
  const int pairs = (r1 - r0) / 2, n = P.E * pairs;
  const float* src = P.wr + static_cast<size_t>(l) * P.E * P.d + r0;
#pragma unroll 1
  for (int i = tid; i < n; i += nthreads) {
    const int e = i / pairs, c = 2 * (i - e * pairs);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(smem_u32(ws + e * P.rpc + c)),
                 "l"(src + static_cast<size_t>(e) * P.d + c)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Warp t: reads token t's E <= 512 logits (all of a lane's 16 at once: the
// fixed-point sums every CTA added, plus the bias), turns them into order
// keys held in registers, selects its k experts and gates into R.
// Selection: k rounds of a warp maximum over the keys (ties go to the lower
// expert index through a second, minimum reduction over the indices that
// hold the maximum); lane j keeps the j-th pick. The publishing CTA also
// writes the plain logits.
__device__ __noinline__ void ds_topk(const DSParams& P, int l, int t, float* pub_logits, unsigned long long* td) {
  // the parameters this uses, in registers: P sits in shared memory, and the
  // ordered loads below would make the compiler read it again each time
  const int E = P.E, T = P.T, k = P.k, L = P.L;
  const DSRoute R = ds_route(ds_smem + P.sm_route, T * k);
  DSShared* S = reinterpret_cast<DSShared*>(ds_smem);
  constexpr int KPL = kDsMaxE / 32;  // keys a lane holds
  const int lane = threadIdx.x & 31;
  const size_t o = (static_cast<size_t>(l % 3) * T + t) * E;
  const long long* const acc = P.lacc + o;
  const int* const flg = P.lbad + o;
  const size_t part = 3 * static_cast<size_t>(T) * E;  // distance between the parts' accumulators
  const float* const bias = P.bias != nullptr ? P.bias + (static_cast<size_t>(l) * T + t) * E : nullptr;
  long long w[KPL];
  int fl[KPL];
  float bv[KPL];
#pragma unroll
  for (int v = 0; v < KPL; ++v) {  // every load in flight at once
    const int e = v * 32 + lane;
    w[v] = e < E ? ld_relaxed_s64(acc + e) : 0;
    fl[v] = e < E ? ld_relaxed_s32(flg + e) : 0;
    bv[v] = (bias != nullptr && e < E) ? __ldg(bias + e) : 0.f;
  }
  // the next layer's bias rows into L2 while this layer runs
  if (bias != nullptr && l + 1 < L && lane * 32 < E)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(bias + static_cast<size_t>(T) * E + lane * 32));
  // the logits: the 2^-32 part alone, rounded once to float (a power-of-two
  // scale is exact), unless an upper part was used; NaN where a partial was
  // not finite; then the bias
  float lv[KPL];
  bool upper = false;
#pragma unroll
  for (int v = 0; v < KPL; ++v) {
    float c = __ll2float_rn(w[v]) * 2.3283064365386963e-10f;  // 2^-32
    if (fl[v] & 1) c = __uint_as_float(0x7fc00000u);
    lv[v] = bias != nullptr ? c + bv[v] : c;
    upper = upper || (fl[v] & 6) != 0;
  }
  if (__any_sync(0xffffffffu, upper)) {  // seldom: upper parts first, then the 2^-32 part, in double
#pragma unroll 1
    for (int v = 0; v < KPL; ++v) {
      const int e = v * 32 + lane;
      if ((fl[v] & 6) == 0 || (fl[v] & 1) != 0 || e >= E) continue;
      double sum = 0.0;
      if (fl[v] & 4) sum = static_cast<double>(ld_relaxed_s64(acc + 2 * part + e)) * kLogitUnit2;
      if (fl[v] & 2) sum += static_cast<double>(ld_relaxed_s64(acc + part + e)) * kLogitUnit1;
      sum += static_cast<double>(w[v]) * kLogitUlp;
      const float c = static_cast<float>(sum);
      lv[v] = bias != nullptr ? c + __ldg(bias + e) : c;
    }
  }
  uint32_t kv[KPL];  // order keys; 0 = absent (e >= E) or taken
#pragma unroll
  for (int v = 0; v < KPL; ++v) kv[v] = v * 32 + lane < E ? ds_order_key(lv[v]) : 0u;
  if (pub_logits != nullptr) {  // the publishing CTA
    float* const pl = pub_logits + static_cast<size_t>(t) * E;
#pragma unroll
    for (int v = 0; v < KPL; ++v)
      if (v * 32 + lane < E) pl[v * 32 + lane] = lv[v];
  }
  if (td && lane == 0) td[29] = global_timer_ns();
  // lane best: its largest key, ties to its lowest register index (so the
  // lowest expert index), packed as key << 32 | (KPL - 1 - index)
  auto lane_best = [&kv]() {
    unsigned long long b[KPL];
#pragma unroll
    for (int i = 0; i < KPL; ++i) b[i] = (static_cast<unsigned long long>(kv[i]) << 32) | (KPL - 1 - i);
#pragma unroll
    for (int h = KPL / 2; h > 0; h >>= 1)
#pragma unroll
      for (int i = 0; i < h; ++i) b[i] = b[i] > b[i + h] ? b[i] : b[i + h];
    return b[0];
  };
  unsigned long long lb = lane_best();
  uint32_t mine_key = 0u;
  int mine_e = 0;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    // the warp maximum, then the lowest expert index holding it; only the
    // lane that held it looks at its keys again
    const uint32_t lk = static_cast<uint32_t>(lb >> 32);
    const uint32_t M = __reduce_max_sync(0xffffffffu, lk);
    const int li = KPL - 1 - static_cast<int>(lb & 0xffu);
    const unsigned le = lk == M ? static_cast<unsigned>(lane + 32 * li) : 0x7fffffffu;
    const int e = static_cast<int>(__reduce_min_sync(0xffffffffu, le));
    if (lane == (e & 31)) {
#pragma unroll
      for (int i = 0; i < KPL; ++i) kv[i] = (i == (e >> 5)) ? 0u : kv[i];
      lb = lane_best();
    }
    if (lane == j) {
      mine_key = M;
      mine_e = e;
    }
  }
  if (td && lane == 0) td[30] = global_timer_ns();
  const bool sel = lane < k;
  const float lj = sel ? ds_key_value(mine_key) : 0.f;
  const float l0 = __shfl_sync(0xffffffffu, lj, 0);
  const float ex = sel ? expf(lj - l0) : 0.f;
  float sum = ex;
  if (!P.renorm) {
    // full-softmax denominator over the whole row (lv, still in registers)
    float ev[KPL];
#pragma unroll
    for (int v = 0; v < KPL; ++v) ev[v] = expf(lv[v] - l0);
    sum = 0.f;
#pragma unroll
    for (int v = 0; v < KPL; ++v)
      if (v * 32 + lane < E) sum += ev[v];  // in order of e within the lane; NaN logits make the sum NaN
  }
  const float denom = warp_sum(sum);
  const float gate = ex / denom;
  if (sel) {
    R.idx[t * k + lane] = mine_e;
    R.gate[t * k + lane] = gate;
  }
  if (T == 1) {
    // one token: its k experts are distinct, so the grouping is the order of
    // the kept ones by expert index, found here by ranks instead of a
    // CTA-wide sort
    int slot = 0;
    bool held = true;
    if (sel) {
      slot = R.slot_s[min(max(mine_e, 0), E - 1)];
      held = slot != kSlotAbsent;
      if (held && (slot < 0 || slot >= P.n_slots)) {
        report(P.status, kDevBadSlot, mine_e);
        slot = 0;
      }
    }
    const int skip_from = P.skip_from, hot_slots = P.hot_slots;
    const bool keep = sel && held && !(skip_from > 0 && lane >= skip_from && slot >= hot_slots);
    const unsigned kept = __ballot_sync(0xffffffffu, keep);
    int pos = 0;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {  // lanes at and above k hold no pick
      const int ej = __shfl_sync(0xffffffffu, mine_e, j);
      pos += (((kept >> j) & 1u) != 0u && ej < mine_e) ? 1 : 0;
    }
    if (sel) R.pair_pos[lane] = keep ? pos : -1;
    if (keep) {
      R.sorted_e[pos] = mine_e;
      R.pair_token[pos] = 0;
      R.pair_gate[pos] = gate;
      R.uniq_e[pos] = mine_e;
      R.uniq_slot[pos] = slot;
      R.uniq_off[pos] = pos;
    }
    if (lane == 0) {
      const int n = __popc(kept);
      R.uniq_off[n] = n;
      S->n_uniq = n;
    }
  }
}

// Stable sort of the T*k pairs by expert in shared memory, the unique
// experts and their slots. Every consumer thread takes part.
// Pair p = t * k + j stays unless its expert is not held here (slot
// kSlotAbsent), or skipping is on, its rank j >= skip_from and its expert's
// slot is not resident.
__device__ __forceinline__ bool ds_keep_pair(const DSParams& P, const DSRoute& R, int p, int e) {
  const int slot = R.slot_s[e];
  return slot != kSlotAbsent && (P.skip_from == 0 || p % P.k < P.skip_from || slot < P.hot_slots);
}

__device__ __noinline__ void ds_group(const DSParams& P, DSShared* S, int np, int CT, int* sk) {
  const DSRoute R = ds_route(ds_smem + P.sm_route, np);
  const int tid = threadIdx.x;
  // a sort key per pair: expert, then pair index (np <= 1024) for a kept
  // pair; past every such key for one left out
  constexpr int kOut = 0x7fffffff;
#pragma unroll 1
  for (int p = tid; p < np; p += CT) {
    const int e = min(max(R.idx[p], 0), P.E - 1);
    sk[p] = ds_keep_pair(P, R, p, e) ? (e << 10) + p : kOut;
  }
  named_sync(1, CT);
  // a kept pair's place in the sorted order is the number of smaller keys
#pragma unroll 1
  for (int p = tid; p < np; p += CT) {
    const int kp = sk[p];
    if (kp == kOut) {
      R.pair_pos[p] = -1;
      continue;
    }
    int pos = 0;
#pragma unroll 8
    for (int q = 0; q < np; ++q) pos += sk[q] < kp ? 1 : 0;
    R.sorted_e[pos] = kp >> 10;
    R.pair_token[pos] = p / P.k;
    R.pair_gate[pos] = R.gate[p];
    R.pair_pos[p] = pos;
  }
  named_sync(1, CT);
  if (tid < 32) {
    int n_kept = 0;  // the sorted pairs
#pragma unroll 1
    for (int c = 0; c < np; c += 32) {
      const int q = c + tid;
      n_kept += __popc(__ballot_sync(0xffffffffu, q < np && sk[q] != kOut));
    }
    int base = 0;
#pragma unroll 1
    for (int c = 0; c < n_kept; c += 32) {
      const int i = c + tid;
      const bool first = i < n_kept && (i == 0 || R.sorted_e[i - 1] != R.sorted_e[i]);
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
      R.uniq_off[base] = n_kept;
      S->n_uniq = base;
    }
  }
  named_sync(1, CT);
}

// Writes layer l's routing record (the publishing CTA only).
__device__ __noinline__ void ds_publish(const DSParams& P, int l, int np, int nu, int CT) {
  const DSRoute R = ds_route(ds_smem + P.sm_route, np);
  char* rec = P.rec + static_cast<size_t>(l) * P.rec_bytes;
  int32_t* idx = reinterpret_cast<int32_t*>(rec + P.ro.idx);
  float* gate = reinterpret_cast<float*>(rec + P.ro.gate);
  int32_t* pt = reinterpret_cast<int32_t*>(rec + P.ro.pair_token);
  int32_t* pj = reinterpret_cast<int32_t*>(rec + P.ro.pair_j);
  float* pg = reinterpret_cast<float*>(rec + P.ro.pair_gate);
  int32_t* ps = reinterpret_cast<int32_t*>(rec + P.ro.pair_slot);
  int32_t* pp = reinterpret_cast<int32_t*>(rec + P.ro.pair_pos);
  int32_t* ue = reinterpret_cast<int32_t*>(rec + P.ro.uniq_expert);
  int32_t* us = reinterpret_cast<int32_t*>(rec + P.ro.uniq_slot);
  int32_t* uo = reinterpret_cast<int32_t*>(rec + P.ro.uniq_offset);
  int32_t* ec = reinterpret_cast<int32_t*>(rec + P.ro.expert_count);
  int32_t* eo = reinterpret_cast<int32_t*>(rec + P.ro.expert_offset);
  const int tid = threadIdx.x;
#pragma unroll 1
  for (int q = tid; q < np; q += CT) {
    const int pos = R.pair_pos[q];  // -1: a pair left out
    const int e = min(max(R.idx[q], 0), P.E - 1);
    int slot = R.slot_s[e];
    if (slot < 0 || slot >= P.n_slots) slot = 0;
    idx[q] = R.idx[q];
    gate[q] = R.gate[q];
    pp[q] = pos;
    if (pos < 0) continue;
    pt[pos] = q / P.k;
    pj[pos] = q % P.k;
    pg[pos] = R.gate[q];
    ps[pos] = slot;
  }
#pragma unroll 1
  for (int u = tid; u < nu; u += CT) {
    ue[u] = R.uniq_e[u];
    us[u] = R.uniq_slot[u];
    uo[u] = R.uniq_off[u];
  }
  const int n_kept = R.uniq_off[nu];  // the sorted pairs (all T * k unless some were left out)
  if (tid == 0) {
    uo[nu] = n_kept;
    *reinterpret_cast<int32_t*>(rec + P.ro.n_uniq) = nu;
  }
#pragma unroll 1
  for (int e = tid; e < P.E; e += CT) {  // counts by binary search in the sorted experts
    int lo = 0, hi = n_kept;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (R.sorted_e[mid] < e) lo = mid + 1; else hi = mid;
    }
    int lo2 = lo, hi2 = n_kept;
    while (lo2 < hi2) {
      const int mid = (lo2 + hi2) >> 1;
      if (R.sorted_e[mid] <= e) lo2 = mid + 1; else hi2 = mid;
    }
    ec[e] = lo2 - lo;
    eo[e] = lo;
    if (e == P.E - 1) eo[P.E] = n_kept;
  }
}

// Adds this CTA's partial logits of the next layer: ysl [T, rpc] holds its
// rows of that layer's input, ws the router's columns. buf: the layer's
// parity.
__device__ __noinline__ void ds_partial_logits(const DSParams& P, const float* ws, const float* ysl, int nr,
                                               int buf, int CT) {
  const int E = P.E, T = P.T, rpc = P.rpc;  // in registers (P is in shared memory)
  long long* const acc = P.lacc + static_cast<size_t>(buf) * T * E;
  const size_t part = 3 * static_cast<size_t>(T) * E;
  int* const badf = P.lbad + static_cast<size_t>(buf) * T * E;
#pragma unroll 1
  for (int e = threadIdx.x; e < E; e += CT) {
    const float* wrow = ws + e * rpc;
#pragma unroll 1
    for (int t = 0; t < T; ++t) {
      const float* yrow = ysl + t * rpc;
      float p = 0.f;
#pragma unroll 2
      for (int r = 0; r < nr; ++r) p = fmaf(yrow[r], wrow[r], p);
      const size_t o = static_cast<size_t>(t) * E + e;
      if (!isfinite(p)) {
        asm volatile("red.relaxed.gpu.global.or.b32 [%0], 1;" ::"l"(badf + o) : "memory");
        continue;
      }
      double rem = static_cast<double>(p);
      int used = 0;
      if (fabs(rem) >= kLogitUnit2) {  // the multiple of 2^76: below 2^52 for a finite float
        const long long a = static_cast<long long>(trunc(rem * (1.0 / kLogitUnit2)));
        rem -= static_cast<double>(a) * kLogitUnit2;
        asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(acc + 2 * part + o), "l"(a) : "memory");
        used |= 4;
      }
      if (fabs(rem) >= kLogitUnit1) {  // the multiple of 2^22 in a remainder below 2^76
        const long long a = static_cast<long long>(trunc(rem * (1.0 / kLogitUnit1)));
        rem -= static_cast<double>(a) * kLogitUnit1;
        asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(acc + part + o), "l"(a) : "memory");
        used |= 2;
      }
      const long long q = __double2ll_rn(rem * 4294967296.0);  // |rem| < 2^22
      if (q != 0) asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(acc + o), "l"(q) : "memory");
      if (used) asm volatile("red.relaxed.gpu.global.or.b32 [%0], %1;" ::"l"(badf + o), "r"(used) : "memory");
    }
  }
}


// ------------------------------------------------------------------ gate/up
// Rows of h: routed pair p at p (sorted order), shared token t at np + t.
struct GUBlock {
  const uint8_t* rec;  // not used by consumers (the ring holds the rows)
  int u;               // unique-expert index, or -1 for the shared expert
  int cb;              // channel block inside the expert
};

__device__ __forceinline__ void gu_block_of(int beta, int nsh, int sb0, int rb0, const FastDiv& fd_nbf, GUBlock& gb) {
  if (beta < nsh) {
    gb.u = -1;
    gb.cb = sb0 + beta;
  } else {
    const int g = rb0 + beta - nsh;
    gb.u = fdiv(g, fd_nbf);
    gb.cb = g - gb.u * fd_nbf.d;
  }
}

// Rows (token count and first h row) of expert u (-1: shared).
__device__ __forceinline__ void expert_h_rows(const DSRoute& R, int u, int np, int T, int& first, int& n) {
  if (u < 0) {
    first = np;
    n = T;
  } else {
    first = R.uniq_off[u];
    n = R.uniq_off[u + 1] - first;
  }
}

__device__ __forceinline__ int h_row_token(const DSRoute& R, int u, int first, int i) {
  return u < 0 ? i : R.pair_token[first + i];
}

// ---- gate/up data path: every consumer warp streams the rows of its own
// channel tasks (task j = channel j % 32 of block j / 32; blocks in order:
// this CTA's shared-expert blocks, then its routed blocks; warp w takes
// tasks w, w + CW, ...) into a private buffer of kDsGuDepth task slots with
// 16-byte cp.async, one commit group per task (gu_depth <= kDsGuDepth slots,
// chosen at launch to fit shared memory). Many warps issuing at once
// keep the copies' issue cost off one thread, and no slot is shared.

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// waits until at most n (clamped to 0..kDsGuDepth-1) of this thread's newest groups are pending
__device__ __forceinline__ void cp_async_wait_pending(int n) {
  if (n <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
  else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
  else if (n == 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
  else if (n == 3) asm volatile("cp.async.wait_group 3;" ::: "memory");
  else asm volatile("cp.async.wait_group 4;" ::: "memory");
}
static_assert(kDsGuDepth == 4, "cp_async_wait_pending covers depths up to 4");

// First routed gate/up block (index u * nbf + cb over the unique experts)
// whose work offset sh_w + nbf * uniq_off[u] + cb * n_u is at least x.
__device__ __forceinline__ int routed_block_at(const DSRoute& R, int nu, int nbf, int sh_w, int x) {
  if (nu <= 0) return 0;
  int lo = 0, hi = nu - 1;  // the last u whose first block starts at or before x
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sh_w + nbf * R.uniq_off[mid] <= x) lo = mid; else hi = mid - 1;
  }
  const int base = sh_w + nbf * R.uniq_off[lo];
  if (x <= base) return lo * nbf;
  const int n = max(R.uniq_off[lo + 1] - R.uniq_off[lo], 1);
  const int cb = (x - base + n - 1) / n;
  return cb >= nbf ? (lo + 1) * nbf : lo * nbf + cb;
}

// Record (byte address) and channel of task j of layer l, or false past the
// CTA's blocks.
__device__ __forceinline__ const uint8_t* gu_task_rec(const DSParams& P, const int32_t* uniq_slot, int l, int j,
                                                      int nsh, int sb0, int rb0, int& ch, int& u) {
  const int beta = j >> 5;
  if (beta < nsh) {
    u = -1;
    ch = (sb0 + beta) * 32 + (j & 31);
    return P.shared + static_cast<size_t>(l) * P.stride;
  }
  const int g = rb0 + beta - nsh;
  u = static_cast<int>(fdiv(g, P.fd_nbf));
  ch = (g - u * static_cast<int>(P.fd_nbf.d)) * 32 + (j & 31);
  return P.pool + static_cast<size_t>(uniq_slot[u]) * P.stride;
}

// One task's rows (gate and up of channel ch: codes, then scales) into a
// buffer slot; the warp's lanes split the 16-byte pieces. Commits one group
// (empty when there is no task) so that group counts stay per task.
__device__ __forceinline__ void gu_load(const DSParams& P, const uint8_t* rec, int ch, uint8_t* dst, bool valid) {
  const int lane = threadIdx.x & 31;
  if (valid) {
    const int cbytes = 2 * P.gu_row, sbytes = 2 * P.gu_sc;
    const uint8_t* cs = rec + P.lay.gu_codes + static_cast<size_t>(2 * ch) * P.gu_row;
    const uint8_t* ss = rec + P.lay.gu_scales + static_cast<size_t>(2 * ch) * P.gu_sc;
#pragma unroll 1
    for (int o = lane * 16; o < cbytes; o += 32 * 16) cp_async16(dst + o, cs + o);
#pragma unroll 1
    for (int o = lane * 16; o < sbytes; o += 32 * 16) cp_async16(dst + cbytes + o, ss + o);
  }
  cp_async_commit();
}

// Issues this warp's shared-expert tasks of layer l (the first ones of its
// list) before the layer's routing is known. Returns how many were issued.
template <int CW>
__device__ __noinline__ int gu_prefetch_shared(const DSParams& Q, int l, int nsh, int sb0) {
  const int warp = threadIdx.x >> 5;
  uint8_t* wbuf = reinterpret_cast<uint8_t*>(ds_smem + Q.sm_gub) +
                  static_cast<size_t>(warp) * Q.gu_depth * Q.gu_task_bytes;
  int n = 0;
#pragma unroll 1
  for (int j = warp; j < nsh * 32 && n < Q.gu_depth; j += CW, ++n) {
    int ch, u;
    const uint8_t* rec = gu_task_rec(Q, nullptr, l, j, nsh, sb0, 0, ch, u);
    gu_load(Q, rec, ch, wbuf + static_cast<size_t>(n) * Q.gu_task_bytes, true);
  }
  return n;
}

// The gate/up + SwiGLU phase of layer l for one consumer warp: streams and
// computes its tasks (the first n_pre of them were issued already), each for
// every token of the block's expert; h -> hs. Out of line on purpose: the
// loop gets the whole register budget instead of sharing it with the live
// state of the kernel around it. The launch parameters come from their
// shared-memory copy and are read into registers once. Returns false when
// the phase gave up (abort).
template <int BITS, int BPL, int CW>
__device__ __noinline__ bool gu_phase(const DSParams& Q, DSShared* S, int l, int nsh, int sb0, int rb0, int n_blk,
                                      int n_pre, unsigned long long* td) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int d = Q.d, T = Q.T, np = Q.T * Q.k, nb = Q.d / kBlock;
  const int lpr = Q.gu_lpr, gl = lane & (lpr - 1);
  const bool active = lane < lpr;
  const int gu_row = Q.gu_row, tb = Q.gu_task_bytes;
  float* hs = reinterpret_cast<float*>(ds_smem + Q.sm_hs);
  const int* xq = reinterpret_cast<const int*>(ds_smem + Q.sm_xq);
  const int depth = Q.gu_depth;
  uint8_t* wbuf = reinterpret_cast<uint8_t*>(ds_smem + Q.sm_gub) + static_cast<size_t>(warp) * depth * tb;
  const DSRoute R = ds_route(ds_smem + Q.sm_route, np);
  const int n_task = warp < n_blk * 32 ? (n_blk * 32 - warp + CW - 1) / CW : 0;
  int issued = n_pre;
  // fill the pipeline
#pragma unroll 1
  for (; issued < n_task && issued < depth; ++issued) {
    int ch, u;
    const uint8_t* rec = gu_task_rec(Q, R.uniq_slot, l, warp + issued * CW, nsh, sb0, rb0, ch, u);
    gu_load(Q, rec, ch, wbuf + static_cast<size_t>(issued) * tb, true);
  }
  XR<BITS> xr[BPL];
  int cur_t = -1, rs = 0;  // rs: the slot of task i (task i + depth refills it)
  bool ok = true;
#pragma unroll 1
  for (int i = 0; i < n_task; ++i) {
    if (ds_aborted_warp(S)) {
      ok = false;
      break;
    }
    const int task = warp + i * CW;
    const int beta = task >> 5, c = task & 31;
    const int u = beta < nsh ? -1 : static_cast<int>(fdiv(rb0 + beta - nsh, Q.fd_nbf));
    cp_async_wait_pending(issued - i - 1);
    __syncwarp();
    if (td && lane == 0) {
      if (i == 0) td[22] = global_timer_ns();  // first task's rows in
      if (i < 8) td[32 + i] = global_timer_ns();
    }
    const uint8_t* st = wbuf + static_cast<size_t>(rs) * tb;
    const uint8_t* cg = st;
    const uint16_t* sg = reinterpret_cast<const uint16_t*>(st + 2 * gu_row);
    float* hsl = hs + beta * T * 32;
    int first, n;
    expert_h_rows(R, u, np, T, first, n);
#pragma unroll 1
    for (int k = 0; k < n; ++k) {
      const int t = h_row_token(R, u, first, k);
      if (t != cur_t) {
        load_xq<BITS, BPL>(xq + t * kQW * nb, nb, lpr, gl, xr);
        cur_t = t;
      }
      float2 v = make_float2(0.f, 0.f);
      if (active) v = row_dot2<BITS, BPL>(cg, sg, cg + gu_row, sg + nb, d, gl, xr);
      v = group_sum2(v, lpr);
      // fast exponential and division: h is requantised to 16 bits for the
      // down rows, far coarser than their few-ulp error
      if (lane == 0) hsl[k * 32 + c] = __fdividef(v.x, 1.f + __expf(-v.x)) * v.y;
    }
    if (td && lane == 0 && i < 8) td[48 + i] = global_timer_ns();
    __syncwarp();  // the slot is read: refill it with task i + depth
    if (issued < n_task) {
      int ch, uu;
      const uint8_t* rec = gu_task_rec(Q, R.uniq_slot, l, warp + issued * CW, nsh, sb0, rb0, ch, uu);
      gu_load(Q, rec, ch, wbuf + static_cast<size_t>(rs) * tb, true);
      ++issued;
    }
    rs = rs + 1 == depth ? 0 : rs + 1;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");  // nothing of this layer stays in flight
  return ok;
}

// A gate/up block's 32 channels are in hs: requantise each token's 32
// values and publish them as tagged words (one warp).
__device__ __noinline__ void gu_publish(const DSParams& P, int u, int cb, int np, const float* hsl, uint32_t tag) {
  const DSRoute R = ds_route(ds_smem + P.sm_route, np);
  const int lane = threadIdx.x & 31;
  const int nbf = P.f / kBlock;
  int first, n;
  expert_h_rows(R, u, np, P.T, first, n);
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const uint32_t wq = quant_block_warp(hsl[i * 32 + lane], lane);
    if (lane < kQW) st_ll(P.h_ll + (static_cast<size_t>(first + i) * nbf + cb) * kQW + lane, ll_word(wq, tag));
  }
}

// ------------------------------------------------------------------ down
// Stages the quantised h rows of DN stages [i0, i1) into hq (every consumer
// thread takes part). The round's rows, in stage order, are the shared
// expert's T rows (when stage 0 is in the round) followed by the routed rows
// [uniq_off[ua], uniq_off[ub]), one contiguous range of h. A thread loads up
// to kHB 16-byte units at once and re-polls, together, only the words that
// were not there yet. kHB: 6 with the 15 consumer warps of the 2-bit kernel
// (one token's 11 rows in one round of loads), 4 with the 11 of the 3-bit one
// (fewer registers to spare).
template <int DBPL, int kHB>
__device__ void ds_stage_h(const DSParams& P, const DSRoute& R, int np, int i0, int i1, int sh, uint32_t tag,
                           int* hq, DSShared* S, uint64_t deadline, int CT) {
  const int nbf = P.f / kBlock;
  const int units_per_row = nbf * (kQW / 2);  // 16-byte units
  const FastDiv& fd_row = P.fd_hrow;
  const int n_sh = (sh && i0 == 0) ? P.T : 0;
  const int ua = max(i0 - sh, 0), ub = max(i1 - sh, 0);
  const int rfirst = R.uniq_off[ua];
  const int n_rows = n_sh + (ub > ua ? R.uniq_off[ub] - rfirst : 0);
  const int units = n_rows * units_per_row;
#pragma unroll 1
  for (int j0 = threadIdx.x; j0 < units; j0 += kHB * CT) {
    unsigned long long v[kHB][2];
    const unsigned long long* src[kHB];
#pragma unroll
    for (int k = 0; k < kHB; ++k) {
      const int j = min(j0 + k * CT, units - 1);
      const int r = fdiv(j, fd_row), rem = j - r * units_per_row;
      const int hrow = r < n_sh ? np + r : rfirst + (r - n_sh);
      const int blk = rem / (kQW / 2), w2 = rem % (kQW / 2);
      src[k] = P.h_ll + (static_cast<size_t>(hrow) * nbf + blk) * kQW + 2 * w2;
      if (j0 + k * CT < units) ld_ll2(src[k], v[k][0], v[k][1]);
      else v[k][0] = v[k][1] = ll_word(0u, tag);  // past the end: no load
    }
    while (true) {
      bool all = true;
#pragma unroll
      for (int k = 0; k < kHB; ++k) all = all && tag_ok(v[k][0], tag) && tag_ok(v[k][1], tag);
      if (all) break;
      if (ds_aborted(S) || global_timer_ns() > deadline) {
        if (!ds_aborted(S)) ds_abort(S, P.status, 23);
        break;
      }
      __nanosleep(kDsPollNs);
#pragma unroll
      for (int k = 0; k < kHB; ++k) {
        if (!tag_ok(v[k][0], tag)) v[k][0] = ld_ll(src[k]);
        if (!tag_ok(v[k][1], tag)) v[k][1] = ld_ll(src[k] + 1);
      }
    }
#pragma unroll
    for (int k = 0; k < kHB; ++k) {
      const int j = j0 + k * CT;
      if (j < units) {
        const int r = fdiv(j, fd_row), rem = j - r * units_per_row;
        const int blk = rem / (kQW / 2), w2 = rem % (kQW / 2);
        int* dst = hq + r * kQW * nbf + ((blk % DBPL) << P.dn_lsh) + blk / DBPL;
        dst[(2 * w2) * nbf] = static_cast<int>(static_cast<uint32_t>(v[k][0]));
        dst[(2 * w2 + 1) * nbf] = static_cast<int>(static_cast<uint32_t>(v[k][1]));
      }
    }
  }
}

// Down stage (one expert, this CTA's output rows) by one warp: every token
// row of the expert is loaded once and the rows are swept RPW at a time.
template <int BITS, int BPL>
__device__ __forceinline__ void dn_task(const DSParams& P, const DSRoute& R, const uint8_t* st, int u, int np,
                                        const int* hq, int hq_row0, int nrows_out, float* zs) {
  const int lane = threadIdx.x & 31;
  const int lpr = P.dn_lpr, rpw = 32 >> P.dn_lsh;
  const int rl = lane >> P.dn_lsh, gl = lane & (lpr - 1);
  const int nb = P.f / kBlock;
  const uint8_t* codes = st;
  const uint16_t* scales = reinterpret_cast<const uint16_t*>(st + nrows_out * P.dn_row);
  int first, n;
  expert_h_rows(R, u, np, P.T, first, n);
  XR<BITS> hr[BPL];
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    load_xq<BITS, BPL>(hq + (hq_row0 + i) * kQW * nb, nb, lpr, gl, hr);
#pragma unroll 1
    for (int r0 = 0; r0 < nrows_out; r0 += rpw) {
      const int r = r0 + rl;
      float v = 0.f;
      if (r < nrows_out) v = row_dot<BITS, BPL>(codes + r * P.dn_row, scales + r * nb, P.f, gl, hr);
      v = group_sum(v, lpr);
      if (gl == 0 && r < nrows_out) zs[(first + i) * P.rpc + r] = v;
    }
  }
}

// ------------------------------------------------------------------ producer
// One ring of fixed-size slots carries the down groups of a layer (the down
// rows, this CTA's output rows, of up to `gpd` routed experts each), issued
// as soon as the routing is known, so they stream in while gate/up computes;
// consumers free a slot with 16 arrivals.
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

// Down rows [r0, r1) of one record into dst (codes, then scales).
__device__ __noinline__ void copy_dn(const DSParams& P, uint8_t* dst, const uint8_t* rec, int r0, int r1,
                                        uint64_t* bar) {
  const uint32_t cb = (r1 - r0) * P.dn_row, sb = (r1 - r0) * P.dn_sc;
  bulk_g2s(dst, rec + P.lay.dn_codes + static_cast<size_t>(r0) * P.dn_row, cb, bar);
  bulk_g2s(dst + cb, rec + P.lay.dn_scales + static_cast<size_t>(r0) * P.dn_sc, sb, bar);
}

// ------------------------------------------------------------------ the kernel
template <int BITS, int GBPL, int DBPL, bool ROUTE>
__global__ void __launch_bounds__((ds_consumer_warps(BITS) + 1) * 32, 1) decode_stack_kernel(const DSParams P) {
  constexpr int CW = ds_consumer_warps(BITS);
  constexpr int CT = CW * 32;
  char* smem = ds_smem;
  DSShared* S = reinterpret_cast<DSShared*>(smem);
  const int np = P.T * P.k;
  const DSRoute R = ds_route(smem + P.sm_route, np);
  float* wsl = reinterpret_cast<float*>(smem + P.sm_ws);    // this CTA's columns of the next router
  float* ysl = reinterpret_cast<float*>(smem + P.sm_ysl);   // this CTA's rows of the next layer's input
  // quantised h rows of a round of down stages: the gate/up buffers and the
  // x staging area behind them (both idle during the down phase)
  int* hq = reinterpret_cast<int*>(smem + P.sm_gub);
  int* xq = reinterpret_cast<int*>(smem + P.sm_xq);
  float* hs = reinterpret_cast<float*>(smem + P.sm_hs);
  float* zs = reinterpret_cast<float*>(smem + P.sm_zs);
  float* xres = reinterpret_cast<float*>(smem + P.sm_xres);
  uint8_t* ring = reinterpret_cast<uint8_t*>(smem + P.sm_ring);
  uint8_t* shdn = reinterpret_cast<uint8_t*>(smem + P.sm_shdn);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  const int nbf = P.f / kBlock;

  // static splits: output rows (units of `gran` rows; the router columns
  // follow them) and the shared expert's channel blocks of this CTA
  const int r0 = P.gran * split_at(P.n_units, b, G);
  const int r1 = P.gran * split_at(P.n_units, b + 1, G);
  // gate/up blocks are split among the CTAs by work (h rows x channels):
  // the shared expert's blocks first (T rows each), then routed expert u's
  // (n_u rows each); CTA b takes the blocks whose work offset falls in
  // [W b / G, W (b + 1) / G). W does not depend on the routing, so the
  // shared-expert share is known before it.
  const int gu_w = nbf * P.T * (P.k + (P.has_shared ? 1 : 0));
  const int gu_lo = split_at(gu_w, b, G), gu_hi = split_at(gu_w, b + 1, G);
  const int sh_w = P.has_shared ? nbf * P.T : 0;
  const int sb0 = P.has_shared ? min(nbf, (gu_lo + P.T - 1) / P.T) : 0;
  const int sb1 = P.has_shared ? min(nbf, (gu_hi + P.T - 1) / P.T) : 0;
  const int nsh = sb1 - sb0;
  const bool has_rows = r1 > r0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDsNS; ++i) {
      mbar_init(&S->full[i], 1);
      mbar_init(&S->empty[i], kDsArr);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S->shdn_full[i], 1);
      mbar_init(&S->shdn_empty[i], 1);
    }
    mbar_init(&S->route_bar, 1);
    S->abort_flag = 0;
    S->n_uniq = 0;
    S->route_ok = 0;
    S->prm = P;
    fence_mbar_init();
  }
  __syncthreads();
  grid_dep_wait();  // x, the workspace and the tag counter come from earlier kernels
  if (threadIdx.x == 0) {
    S->base_tag = *reinterpret_cast<volatile unsigned*>(&g_ds_epoch);
    if (*reinterpret_cast<volatile int*>(P.status) != 0) S->abort_flag = 1;  // an earlier error is pending
  }
  __syncthreads();
  const uint32_t base = S->base_tag;
  const uint64_t t_start = global_timer_ns();
  const uint64_t deadline = t_start + P.timeout_ns;
  unsigned long long* trace = P.trace != nullptr && b < kTraceCtas ? P.trace + b * kTraceSlots : nullptr;
  const int dl = P.L > 1 ? 1 : 0;
  const DSParams& Q = S->prm;  // what the out-of-line helpers get

  if (warp == CW) {
    // ============================================================ producer
    // Lane i of the warp issues item i of each window of n_ring ring items (a
    // gate/up stage or a down group), after waiting, on its own, for its
    // slot's previous item to be consumed: copies issued from many lanes at
    // once overlap their issue latency. A window never holds two items of
    // one slot, so every wait is for the phase right after the one the
    // previous window saw complete (mbarrier parity cannot tell phase k
    // from phase k - 2).
    uint32_t seq = 0, shdn_count = 0;
    bool ok = true;
    // waits (lane-local, bounded) until ring slot `q` may be reused
    auto slot_ready = [&](uint32_t q) -> bool {
      if (q < static_cast<uint32_t>(P.n_ring)) return true;
      const uint32_t qd = fdiv(q, P.fd_ring);
      const uint32_t parity = (qd - 1) & 1;
      while (!mbar_try_wait(&S->empty[q - qd * P.n_ring], parity, 100000u)) {
        if (ds_aborted(S) || global_timer_ns() > deadline) return false;
      }
      return true;
    };
    // layer l's shared-expert down rows: buffer l & 1, its (l >> 1)-th use
    auto issue_shdn = [&](int l) -> bool {
      const int j = l & 1;
      if (l >= 2) {
        while (!mbar_try_wait(&S->shdn_empty[j], ((l >> 1) - 1) & 1, 100000u)) {
          if (ds_aborted(S) || global_timer_ns() > deadline) return false;
        }
      }
      const uint8_t* rec = P.shared + static_cast<size_t>(l) * P.stride;
      mbar_arrive_expect_tx(&S->shdn_full[j], (r1 - r0) * (P.dn_row + P.dn_sc));
      copy_dn(Q, shdn + j * P.dn_stride, rec, r0, r1, &S->shdn_full[j]);
      return true;
    };
    const bool sh_dn = P.has_shared && has_rows;
    // Iteration l issues layer l's routed items (l >= 0), then layer l + 1's
    // shared-expert down rows (they do not depend on its x). shdn_count
    // (lane 1) counts the copies the lane actually issued.
#pragma unroll 1
    for (int l = -1; l < P.L && ok; ++l) {
      if (ds_aborted_warp(S)) break;
      if (l >= 0) {
        // routing of layer l is in shared memory once route_bar completes
        int got = 1;
        if (lane == 0) {
          while (!mbar_try_wait(&S->route_bar, l & 1, 100000u)) {
            if (ds_aborted(S) || global_timer_ns() > deadline) {
              got = 0;
              break;
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, got, 0)) {
          ok = false;
          break;
        }
        if (S->route_ok == 0) {  // the consumers gave the layer up
          ok = false;
          break;
        }
        unsigned long long* td = (trace != nullptr && l == dl && lane == 0) ? trace : nullptr;
        if (td) td[16] = global_timer_ns();
        const int nu = min(max(S->n_uniq, 0), min(np, P.E));
        const int n_items = has_rows ? (nu + P.gpd - 1) / P.gpd : 0;  // down groups
#pragma unroll 1
        for (int w0 = 0; w0 < n_items && ok; w0 += P.n_ring) {
          const int it = w0 + lane;
          bool mine = true;
          if (lane < P.n_ring && it < n_items) {
            const uint32_t q = seq + it;
            mine = slot_ready(q);
            if (trace != nullptr && l == dl && w0 == 0 && lane < 8) trace[56 + lane] = global_timer_ns();
            if (mine) {
              const int u0 = it * P.gpd, u1 = min(nu, u0 + P.gpd);
              const int slot = fmod_(q, P.fd_ring);
              uint8_t* dst = ring + static_cast<size_t>(slot) * P.slot_bytes;
              mbar_arrive_expect_tx(&S->full[slot], (u1 - u0) * (r1 - r0) * (P.dn_row + P.dn_sc));
#pragma unroll 1
              for (int u = u0; u < u1; ++u)
                copy_dn(Q, dst + (u - u0) * P.dn_stride, P.pool + static_cast<size_t>(R.uniq_slot[u]) * P.stride,
                        r0, r1, &S->full[slot]);
            }
          }
          if (trace != nullptr && l == dl && w0 == 0 && lane < 8) trace[40 + lane] = global_timer_ns();
          ok = __all_sync(0xffffffffu, mine);
          if (td && w0 == 0) td[17] = global_timer_ns();
        }
        seq += n_items;
        if (td) td[18] = global_timer_ns();
        if (!ok) break;
      }
      if (l + 1 < P.L) {
        const int ln = l + 1;
        int okn = 1;
        if (sh_dn && lane == 1) {
          okn = issue_shdn(ln) ? 1 : 0;
          shdn_count += okn;
        }
        ok = __all_sync(0xffffffffu, okn != 0);
      }
    }
    if (lane == 0 && !ok && !ds_aborted(S)) ds_abort(S, P.status, 10);
    // every issued copy lands before the CTA may exit; copies take
    // microseconds, so after an abort (when a counted ring item may never
    // have been issued) the waits give up after 2 ms in all
    const uint64_t d2 = global_timer_ns() + 2000000ull;
    if (lane == 0) {
#pragma unroll 1
      for (uint32_t q = seq > static_cast<uint32_t>(P.n_ring) ? seq - P.n_ring : 0; q < seq; ++q)
        while (!mbar_try_wait(&S->full[q % P.n_ring], (q / P.n_ring) & 1, 20000u) && global_timer_ns() < d2) {
        }
    }
    if (lane == 1)
#pragma unroll 1
      for (uint32_t q = shdn_count > 2u ? shdn_count - 2u : 0u; q < shdn_count; ++q)
        while (!mbar_try_wait(&S->shdn_full[q & 1], (q >> 1) & 1, 20000u) && global_timer_ns() < d2) {
        }
    __syncwarp();
  } else {
    // ============================================================ consumers
    const int tid = threadIdx.x;
    const int nr_out = r1 - r0;
    uint32_t seq = 0;
    // this warp's shared-expert gate/up rows of the next layer, issued ahead
    int n_pre = (P.has_shared && !ds_aborted(S)) ? gu_prefetch_shared<CW>(Q, 0, nsh, sb0) : 0;
    if (ROUTE) {
      // ---- layer 0's logits: every CTA zeroes its share of the first two
      // accumulator sets (layers 0 and 1), waits for all, then adds its rows
      // of x against its columns of layer 0's router
      ds_wslice_load(P, 0, wsl, r0, r1, tid, CT);
      if (P.bias != nullptr && tid < P.T * 32 && (tid & 31) * 32 < P.E)  // layer 0's bias rows into L2
        asm volatile("prefetch.global.L2 [%0];" ::"l"(P.bias + static_cast<size_t>(tid >> 5) * P.E + (tid & 31) * 32));
      {
        const int n0 = split_at(2 * P.T * P.E, b, G), n1 = split_at(2 * P.T * P.E, b + 1, G);
        const size_t tp = 3 * static_cast<size_t>(P.T) * P.E;  // between the parts
#pragma unroll 1
        for (int i = n0 + tid; i < n1; i += CT) {
          P.lacc[i] = 0;
          P.lacc[tp + i] = 0;
          P.lacc[2 * tp + i] = 0;
          P.lbad[i] = 0;
        }
      }
#pragma unroll 1
      for (int i = tid; i < P.T * nr_out; i += CT) {
        const int t = i / nr_out, r = i - t * nr_out;
        ysl[t * P.rpc + r] = bf16_bits_to_float(P.x[static_cast<size_t>(t) * P.d + r0 + r]);
      }
      __threadfence();
      named_sync(1, CT);
      // the counters advance by L per CTA and launch, in step with the tags
      if (tid == 0) {
        cnt_add(kCntZero, static_cast<unsigned>(P.L));
        if (!ds_aborted(S)) cnt_wait(kCntZero, (base + P.L) * G, S, P.status, 19, deadline);
      }
      asm volatile("cp.async.wait_all;" ::: "memory");
      named_sync(1, CT);
      if (!ds_aborted(S)) ds_partial_logits(Q, wsl, ysl, nr_out, 0, CT);
      __threadfence();
      named_sync(1, CT);
      if (tid == 0) cnt_add(kCntLogits, static_cast<unsigned>(P.L));
    } else if (tid == 0) {
      cnt_add(kCntZero, static_cast<unsigned>(P.L));  // no logits here, but the counters advance in step
      cnt_add(kCntLogits, static_cast<unsigned>(P.L));
    }
#pragma unroll 1
    for (int l = 0; l < P.L; ++l) {
      const uint32_t tag = base + 1 + static_cast<uint32_t>(l);
      const bool publisher = ROUTE && b == l % G;
      // trace slots: 8 phase stamps for layers 0 and 1, then details of
      // layer dl (the second one when there is one)
      const bool traced = trace != nullptr && l < 2 && tid == 0;
      unsigned long long* tdet = (trace != nullptr && l == dl) ? trace : nullptr;
      if (traced) trace[8 * l] = global_timer_ns();
      int nu = 0;
      if (ROUTE) {
#pragma unroll 1
        for (int e = tid; e < P.E; e += CT) R.slot_s[e] = __ldg(P.slot_of + static_cast<size_t>(l) * P.E + e);
        // the logits of this layer are complete once every CTA has added its
        // partials: at the end of the previous layer (with its output rows),
        // or in the prologue for layer 0
        if (tid == 0 && !ds_aborted(S)) {
          if (l == 0) cnt_wait(kCntLogits, (base + P.L) * G, S, P.status, 22, deadline);
          else cnt_wait(kCntOut, (base + l) * G, S, P.status, 20, deadline);
          __threadfence();
        }
        named_sync(1, CT);
        if (tdet && tid == 0) tdet[31] = global_timer_ns();
        if (traced) trace[8 * l + 1] = global_timer_ns();
        // ---- top-k (warp t) while the other warps read x for gate/up
        float* pub = publisher ? reinterpret_cast<float*>(P.rec + static_cast<size_t>(l) * P.rec_bytes + P.ro.logits)
                               : nullptr;
        if (warp < P.T) {
          if (!ds_aborted_warp(S))
            ds_topk(Q, l, warp, pub,
                    (tdet && warp == 0) ? tdet : nullptr);
        } else {
          // the accumulator set of layer l + 2 (every CTA read it as layer
          // l - 1's), zeroed off the top-k's path; the fence before this
          // CTA's count at the end of the layer publishes it before any CTA
          // adds to it (at the end of layer l + 1)
          if (l + 2 < P.L) {
            const size_t n0 = split_at(P.T * P.E, b, G), n1 = split_at(P.T * P.E, b + 1, G);
            const size_t nb1 = static_cast<size_t>((l + 2) % 3) * P.T * P.E;
            const size_t tp = 3 * static_cast<size_t>(P.T) * P.E;  // between the parts
#pragma unroll 1
            for (size_t i = n0 + tid - P.T * 32; i < n1; i += CT - P.T * 32) {
              P.lacc[nb1 + i] = 0;
              P.lacc[tp + nb1 + i] = 0;
              P.lacc[2 * tp + nb1 + i] = 0;
              P.lbad[nb1 + i] = 0;
            }
          }
          if (!ds_aborted_warp(S))
            ds_read_x<BITS, GBPL>(P, l, tag, nullptr, xq, xres, r0, r1, S, deadline, P.T * 32, CT - P.T * 32);
          if (tdet && tid == P.T * 32) tdet[24] = global_timer_ns();
        }
        if (tdet && tid == 0) tdet[20] = global_timer_ns();
        named_sync(1, CT);
        if (traced) trace[8 * l + 2] = global_timer_ns();
        if (P.T > 1) {  // (one token: the top-k warp has grouped its pairs)
          if (!ds_aborted_warp(S)) ds_group(Q, S, np, CT, reinterpret_cast<int*>(smem + P.sm_x));
          else named_sync(1, CT), named_sync(1, CT), named_sync(1, CT);
        }
        // the routing is complete unless some thread gave up: one decision
        // for every consumer thread, which the producer reads behind route_bar
        const bool route_bad = named_sync_or(1, CT, ds_aborted(S));
        nu = route_bad ? 0 : min(max(S->n_uniq, 0), min(np, P.E));
        if (tdet && tid == 0) tdet[21] = global_timer_ns();
        if (tid == 0) {
          S->route_ok = route_bad ? 0 : 1;
          mbar_arrive(&S->route_bar);
        }
        if (route_bad) break;  // every consumer thread leaves the layer loop here
      } else {
        if (!ds_aborted_warp(S)) ds_read_x<BITS, GBPL>(P, 0, tag, nullptr, xq, xres, r0, r1, S, deadline, 0, CT);
        // the grouping was written by moe_group_tokens
        const int nug = min(max(__ldcg(P.g.n_uniq), 0), min(np, P.E));
#pragma unroll 1
        for (int p = tid; p < np; p += CT) {
          R.pair_token[p] = min(max(__ldcg(P.g.pair_token + p), 0), P.T - 1);
          R.pair_gate[p] = __ldcg(P.g.pair_gate + p);
          R.pair_pos[p] = min(max(__ldcg(P.g.pair_pos + p), -1), np - 1);  // -1: a pair left out
        }
#pragma unroll 1
        for (int u = tid; u <= nug; u += CT) R.uniq_off[u] = min(max(__ldcg(P.g.uniq_offset + u), 0), np);
#pragma unroll 1
        for (int u = tid; u < nug; u += CT) {
          int slot = __ldcg(P.g.uniq_slot + u);
          if (slot < 0 || slot >= P.n_slots) {
            report(P.status, kDevBadSlot, u);
            slot = 0;
          }
          R.uniq_slot[u] = slot;
        }
        if (tid == 0) S->n_uniq = nug;
        const bool route_bad = named_sync_or(1, CT, ds_aborted(S));
        nu = route_bad ? 0 : nug;
        if (tid == 0) {
          S->route_ok = route_bad ? 0 : 1;
          mbar_arrive(&S->route_bar);
        }
        if (route_bad) break;  // every consumer thread leaves the layer loop here
      }
      if (traced) trace[8 * l + 3] = global_timer_ns();

      // ---- gate/up + SwiGLU: 32 channel tasks per block, blocks in order
      const int rb0 = routed_block_at(R, nu, nbf, sh_w, max(gu_lo, sh_w));
      const int rb1 = routed_block_at(R, nu, nbf, sh_w, max(gu_hi, sh_w));
      const int n_blk = nsh + (rb1 - rb0);
      if (!ds_aborted_warp(S))
        gu_phase<BITS, GBPL, CW>(Q, S, l, nsh, sb0, rb0, n_blk, n_pre, (tdet && warp == 0) ? tdet : nullptr);
      else
        asm volatile("cp.async.wait_all;" ::: "memory");
      if (tdet && tid == 0) tdet[23] = global_timer_ns();
      named_sync(1, CT);
      // every block's 32 channels are in hs: requantise and publish them
      if (!ds_aborted(S)) {
#pragma unroll 1
        for (int beta = warp; beta < n_blk; beta += CW) {
          GUBlock gb;
          gu_block_of(beta, nsh, sb0, rb0, P.fd_nbf, gb);
          gu_publish(Q, gb.u, gb.cb, np, hs + beta * P.T * 32, tag);
        }
      }
      named_sync(1, CT);
      // the publishing CTA writes the layer's routing record; the h words
      // of the other CTAs are tagged, so the staging below waits for each
      // word itself (no count of the CTAs that have published)
      if (publisher) ds_publish(Q, l, np, nu, CT);
      named_sync(1, CT);
      if (traced) trace[8 * l + 4] = global_timer_ns();

      // ---- down rows of this CTA for every expert (shared first). Stage i:
      // the shared expert (i = 0, its own buffer) or routed expert u, whose
      // rows sit in ring group u / gpd. A round of stages never spans more
      // groups than the ring has slots, so no warp waits on a slot whose
      // previous use in this layer is still pending.
      const int sh = (P.has_shared && has_rows) ? 1 : 0;
      const int n_dn = has_rows ? nu + sh : 0;
      const uint32_t grp0 = seq;  // sequence number of this layer's first down group
      bool sliced = false;
#pragma unroll 1
      for (int i0 = 0; i0 < n_dn;) {
        int i1 = i0, rows = 0;
        while (i1 < n_dn) {
          const int u = i1 - sh;
          if (u >= 0 && i1 > i0) {
            const int ua = max(i0 - sh, 0);
            if (static_cast<int>(fdiv(u, P.fd_gpd) - fdiv(ua, P.fd_gpd)) >= P.n_ring) break;
          }
          int first, n;
          expert_h_rows(R, u, np, P.T, first, n);
          if (rows + n > P.hq_rows) break;
          rows += n;
          ++i1;
        }
        if (i1 == i0) {  // a stage larger than the staging area: cannot happen with valid routing
          if (tid == 0) ds_abort(S, P.status, 24);
          break;
        }
        if (!ds_aborted(S)) ds_stage_h<DBPL, BITS == 2 ? 6 : 4>(P, R, np, i0, i1, sh, tag, hq, S, deadline, CT);
        named_sync(1, CT);
        if (traced && i0 == 0) trace[8 * l + 5] = global_timer_ns();
        if (ROUTE && i0 == 0 && l + 1 < P.L && !ds_aborted(S)) {
          // the next router's columns, for the partial logits at the end of
          // this layer: issued once this CTA's reads of other CTAs' words
          // are done, so that its many small copies delay none of them
          ds_wslice_load(P, l + 1, wsl, r0, r1, tid, CT);
          sliced = true;
        }
        // each warp takes whole stages; the hq row of stage i is the rows of
        // the stages before it in this round
#pragma unroll 1
        for (int i = i0 + warp; i < i1; i += CW) {
          if (ds_aborted_warp(S)) break;
          const int u = i - sh;
          // hq row of the stage's first row: the round's shared rows, then
          // the routed rows before it
          const int n_sh = (sh && i0 == 0) ? P.T : 0;
          const int row0 = u < 0 ? 0 : n_sh + R.uniq_off[u] - R.uniq_off[max(i0 - sh, 0)];
          const uint8_t* st;
          uint64_t* full;
          uint32_t parity;
          int slot = 0;
          if (u < 0) {
            st = shdn + (l & 1) * P.dn_stride;
            full = &S->shdn_full[l & 1];
            parity = (l >> 1) & 1;
          } else {
            const int g = fdiv(u, P.fd_gpd);
            const uint32_t sq = grp0 + g;
            const uint32_t sqd = fdiv(sq, P.fd_ring);
            slot = sq - sqd * P.n_ring;
            st = ring + static_cast<size_t>(slot) * P.slot_bytes + (u - g * P.gpd) * P.dn_stride;
            full = &S->full[slot];
            parity = sqd & 1;
          }
          if (!ds_wait_warp(full, parity, S, deadline)) {
            if (lane == 0 && !ds_aborted(S)) ds_abort(S, P.status, 3);
            break;
          }
          dn_task<BITS, DBPL>(P, R, st, u, np, hq, row0, nr_out, zs);
          __syncwarp();
          if (lane == 0) {
            if (u < 0) {
              mbar_arrive(&S->shdn_empty[l & 1]);
            } else {
              // the group's 16 arrivals: its first expert brings the ones the
              // group has no expert for
              const int g0 = fdiv(u, P.fd_gpd) * P.gpd;
              const int m = min(nu - g0, P.gpd);
              mbar_arrive_cnt(&S->empty[slot], u == g0 ? kDsArr - (m - 1) : 1);
            }
          }
        }
        named_sync(1, CT);
        i0 = i1;
      }
      seq += has_rows ? (nu + P.gpd - 1) / P.gpd : 0;
      if (ROUTE && !sliced && has_rows && l + 1 < P.L && !ds_aborted(S)) ds_wslice_load(P, l + 1, wsl, r0, r1, tid, CT);
      if (traced) trace[8 * l + 6] = global_timer_ns();
      // the down phase is done with the buffers: this warp's shared-expert
      // gate/up rows of the next layer go in now
      n_pre = (l + 1 < P.L && P.has_shared && !ds_aborted_warp(S)) ? gu_prefetch_shared<CW>(Q, l + 1, nsh, sb0) : 0;

      // ---- combine: y[t, r] = sum_j gate[t,j] z[(t,j)][r] + z_shared[t][r] (+ x)
      if (!ds_aborted(S) && has_rows) {
        const int hp = P.rpc / 2;  // row pairs of the widest CTA
        char* yl = static_cast<char*>(P.y) + static_cast<size_t>(l) * P.T * P.d * (P.out_f32 ? 4 : 2);
        unsigned long long* yll = P.y_ll + static_cast<size_t>(l & 1) * P.T * (P.d / 2);
#pragma unroll 1
        for (int i = tid; i < P.T * hp; i += CT) {
          const int t = fdiv(i, P.fd_hp), rr = 2 * (i - t * hp);
          if (rr >= nr_out) continue;
          float a0 = 0.f, a1 = 0.f;
#pragma unroll 1
          for (int j = 0; j < P.k; ++j) {
            const int p = R.pair_pos[t * P.k + j];
            if (p < 0) continue;  // left out
            const float g = R.pair_gate[p];
            a0 = fmaf(g, zs[p * P.rpc + rr], a0);
            a1 = fmaf(g, zs[p * P.rpc + rr + 1], a1);
          }
          if (P.has_shared) {
            a0 += zs[(np + t) * P.rpc + rr];
            a1 += zs[(np + t) * P.rpc + rr + 1];
          }
          if (P.residual) {
            a0 += xres[t * P.rpc + rr];
            a1 += xres[t * P.rpc + rr + 1];
          }
          const size_t o = static_cast<size_t>(t) * P.d + r0 + rr;
          if (P.out_f32) {
            *reinterpret_cast<float2*>(yl + o * 4) = make_float2(a0, a1);
          } else {
            const __nv_bfloat162 hv = __floats2bfloat162_rn(a0, a1);
            *reinterpret_cast<__nv_bfloat162*>(yl + o * 2) = hv;
            if (ROUTE && l + 1 < P.L) {
              st_ll(yll + o / 2, ll_word(*reinterpret_cast<const uint32_t*>(&hv), tag));
              ysl[t * P.rpc + rr] = __low2float(hv);  // the next layer's input, as it will read it
              ysl[t * P.rpc + rr + 1] = __high2float(hv);
            }
          }
        }
      }
      if (l + 2 == P.L && tid == 0) grid_dep_launch();
      named_sync(1, CT);
      if (ROUTE && l + 1 < P.L) {
        // the next layer's logits: this CTA's rows of its input against its
        // columns of the next router (loaded during this layer's down phase;
        // the warp's shared-expert copies for the next layer, issued after
        // them, may stay in flight)
        cp_async_wait_pending(n_pre);
        named_sync(1, CT);
        if (!ds_aborted(S) && has_rows) ds_partial_logits(Q, wsl, ysl, nr_out, (l + 1) % 3, CT);
        __threadfence();
        named_sync(1, CT);
      }
      // this CTA's output rows and its partial logits are written, and it has
      // read everything of layer l that other CTAs wrote
      if (tid == 0) cnt_add(kCntOut);
      if (traced) trace[8 * l + 7] = global_timer_ns();
    }
    if (P.L == 1 && tid == 0) grid_dep_launch();
    asm volatile("cp.async.wait_all;" ::: "memory");  // a layer given up may leave copies in flight
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the last CTA to leave advances the tag counter past this launch's tags
    __threadfence();
    const unsigned old = atomicAdd(&g_ds_exit, 1u);
    if (old == static_cast<unsigned>(G - 1)) {
      atomicExch(&g_ds_exit, 0u);
      atomicExch(&g_ds_epoch, base + static_cast<unsigned>(P.L));
    }
  }
}

// Moves the tag counter far past every tag an interrupted launch may have
// written, so that none of its words can match a later launch.
__global__ void ds_skip_tags_kernel(int G) {
  const unsigned e = atomicAdd(&g_ds_epoch, 1u << 20) + (1u << 20);
  atomicExch(&g_ds_exit, 0u);
  // the exchange counters restart in step with the new tag counter
  atomicExch(&g_ds_cnt[kCntLogits], e * G);
  atomicExch(&g_ds_cnt[kCntH], e * G);
  atomicExch(&g_ds_cnt[kCntOut], e * G);
  atomicExch(&g_ds_cnt[kCntZero], e * G);
}

// ------------------------------------------------------------------ host side
namespace {

struct RowGeom {
  int lpr, bpl;
};

RowGeom ds_row_geom(int K) {
  const int nb = K / kBlock;
  int lpr = 1;
  while (lpr < 32 && nb % (lpr * 2) == 0) lpr *= 2;
  return RowGeom{lpr, nb / lpr};
}

size_t ds_align(size_t n, size_t a) { return (n + a - 1) / a * a; }

constexpr int kDsSmemMax = 227 * 1024;

typedef void (*DSKernel)(const DSParams);

template <int BITS, bool ROUTE>
DSKernel ds_pick(int gbpl, int dbpl) {
  if (gbpl == 2 && dbpl == 3) return decode_stack_kernel<BITS, 2, 3, ROUTE>;
  if (gbpl == 1 && dbpl == 1) return decode_stack_kernel<BITS, 1, 1, ROUTE>;
  if (gbpl == 2 && dbpl == 2) return decode_stack_kernel<BITS, 2, 2, ROUTE>;
  if (gbpl == 2 && dbpl == 1) return decode_stack_kernel<BITS, 2, 1, ROUTE>;
  if (gbpl == 1 && dbpl == 3) return decode_stack_kernel<BITS, 1, 3, ROUTE>;
  if (gbpl == 4 && dbpl == 3) return decode_stack_kernel<BITS, 4, 3, ROUTE>;
  return nullptr;
}

DSKernel ds_pick_kernel(int bits, bool route, int gbpl, int dbpl) {
  if (bits == 2) return route ? ds_pick<2, true>(gbpl, dbpl) : ds_pick<2, false>(gbpl, dbpl);
  return route ? ds_pick<3, true>(gbpl, dbpl) : ds_pick<3, false>(gbpl, dbpl);
}

}  // namespace

bool decode_geometry_ok(int d, int f) {
  return ds_pick_kernel(2, true, ds_row_geom(d).bpl, ds_row_geom(f).bpl) != nullptr;
}

size_t decode_exchange_bytes(const moe_layer_cfg& c, int T) {
  const size_t n_rows = static_cast<size_t>(T) * c.k + (c.n_shared ? T : 0);
  const size_t lg = ds_align(3 * static_cast<size_t>(T) * c.E * (3 * 8 + 4), 256);  // fixed-point logits + flags
  const size_t h = ds_align(n_rows * (c.f / kBlock) * kQW * 8, 256);
  const size_t y = ds_align(2 * static_cast<size_t>(T) * (c.d / 2) * 8, 256);
  return lg + h + y;
}

__global__ void ds_probe_kernel() {}

cudaError_t decode_init(Ctx& ctx) {
  const int combos[6][2] = {{2, 3}, {1, 1}, {2, 2}, {2, 1}, {1, 3}, {4, 3}};
  for (int bits = 2; bits <= 3; ++bits)
    for (int r = 0; r < 2; ++r)
      for (const auto& c : combos) {
        const cudaError_t e = cudaFuncSetAttribute(ds_pick_kernel(bits, r != 0, c[0], c[1]),
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kDsSmemMax);
        if (e != cudaSuccess) return e;
      }
  // a tag counter that starts where no earlier process's words are likely to
  // match (the first context on this device in the process picks it)
  unsigned cur = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&cur, g_ds_epoch, sizeof(cur));
  if (e != cudaSuccess) return e;
  if (cur == 0) {
    std::random_device rd;
    const unsigned start = (static_cast<unsigned>(rd()) & 0xfff00000u) | 0x00010000u;
    e = cudaMemcpyToSymbol(g_ds_epoch, &start, sizeof(start));
    if (e != cudaSuccess) return e;
    unsigned cnt[128] = {};
    cnt[kCntLogits] = cnt[kCntH] = cnt[kCntOut] = cnt[kCntZero] = start * static_cast<unsigned>(ctx.num_sms);
    e = cudaMemcpyToSymbol(g_ds_cnt, cnt, sizeof(cnt));
    if (e != cudaSuccess) return e;
  }
  // whether a cooperative launch also takes programmatic serialization here
  // (probed once, outside any stream capture, with an empty kernel)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1);
  cfg.blockDim = dim3(32);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  ctx.coop_pdl = cudaLaunchKernelEx(&cfg, ds_probe_kernel) == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess;
  (void)cudaGetLastError();
  return cudaSuccess;
}

cudaError_t decode_skip_tags(const Ctx& ctx, cudaStream_t s) {
  ds_skip_tags_kernel<<<1, 1, 0, s>>>(ctx.num_sms);
  return cudaGetLastError();
}

cudaError_t launch_decode_stack(const Ctx& ctx, const moe_layer_cfg& c, const StackArgs& a, cudaStream_t s) {
  const RowGeom gg = ds_row_geom(c.d), gd = ds_row_geom(c.f);
  if (a.route && c.E > 512) return cudaErrorNotSupported;  // the fused top-k holds 16 logits per lane
  DSKernel kern = ds_pick_kernel(c.bits, a.route, gg.bpl, gd.bpl);
  if (kern == nullptr) return cudaErrorNotSupported;
  const int G = ctx.num_sms;
  if (G > kDsMaxCtas) return cudaErrorNotSupported;
  const int CW = ds_consumer_warps(c.bits);
  const int T = a.T, np = T * c.k;
  const int n_rows = np + (c.n_shared ? T : 0);
  const int nbd = c.d / kBlock, nbf = c.f / kBlock;
  DSParams P{};
  P.x = a.x;
  P.T = T;
  P.d = c.d;
  P.f = c.f;
  P.E = c.E;
  P.k = c.k;
  P.L = a.L;
  P.renorm = c.renorm;
  P.residual = c.residual;
  P.has_shared = a.shared != nullptr;
  P.skip_from = c.skip_from;
  P.hot_slots = c.hot_slots;
  P.out_f32 = c.out_fp32;
  P.wr = a.wr;
  P.bias = a.bias;
  P.slot_of = a.slot_of;
  P.n_slots = a.n_slots;
  P.pool = a.pool;
  P.stride = a.stride;
  P.shared = a.shared;
  P.lay = a.lay;
  P.y = a.y;
  P.rec = a.rec;
  P.rec_bytes = a.rec_bytes;
  P.ro.logits = a.ro[0];
  P.ro.idx = a.ro[1];
  P.ro.gate = a.ro[2];
  P.ro.expert_count = a.ro[3];
  P.ro.expert_offset = a.ro[4];
  P.ro.pair_token = a.ro[5];
  P.ro.pair_j = a.ro[6];
  P.ro.pair_gate = a.ro[7];
  P.ro.pair_slot = a.ro[8];
  P.ro.pair_pos = a.ro[9];
  P.ro.uniq_expert = a.ro[10];
  P.ro.uniq_slot = a.ro[11];
  P.ro.uniq_offset = a.ro[12];
  P.ro.n_uniq = a.ro[13];
  if (a.g != nullptr) P.g = *a.g;
  {
    char* ex = a.exchange;
    const size_t lg = ds_align(3 * static_cast<size_t>(T) * c.E * (3 * 8 + 4), 256);
    const size_t h = ds_align(static_cast<size_t>(n_rows) * nbf * kQW * 8, 256);
    P.lacc = reinterpret_cast<long long*>(ex);
    P.lbad = reinterpret_cast<int*>(ex + 9 * static_cast<size_t>(T) * c.E * 8);
    P.h_ll = reinterpret_cast<unsigned long long*>(ex + lg);
    P.y_ll = reinterpret_cast<unsigned long long*>(ex + lg + h);
  }
  P.status = ctx.d_status;
  P.timeout_ns = ctx.timeout_ns;
  P.trace = ctx.d_trace;
  P.gu_lpr = gg.lpr;
  P.dn_lpr = gd.lpr;
  P.gu_lsh = __builtin_ctz(static_cast<unsigned>(gg.lpr));
  P.dn_lsh = __builtin_ctz(static_cast<unsigned>(gd.lpr));
  P.fd_nb = make_fastdiv(nbd);
  P.fd_nbf = make_fastdiv(nbf);
  P.gu_row = c.d * c.bits / 8;
  P.gu_sc = nbd * 2;
  P.dn_row = c.f * c.bits / 8;
  P.dn_sc = nbf * 2;
  // output rows come in units of `gran` rows: even (output words hold two
  // rows) and with code and scale bytes that are multiples of 16 (bulk copies)
  int gran = 2;
  while ((gran * P.dn_row) % 16 != 0 || (gran * P.dn_sc) % 16 != 0) gran *= 2;
  if (c.d % gran != 0) return cudaErrorNotSupported;
  P.gran = gran;
  P.n_units = c.d / gran;
  P.rpc = gran * ((P.n_units + G - 1) / G);
  // ring slots hold a group of down stages (this CTA's output rows of up to
  // kDsGpd experts); a gate/up task is the two rows of one channel
  P.dn_stride = static_cast<int>(ds_align(static_cast<size_t>(P.rpc) * (P.dn_row + P.dn_sc), 16));
  P.gu_task_bytes = static_cast<int>(ds_align(2 * static_cast<size_t>(P.gu_row + P.gu_sc), 128));
  if ((2 * P.gu_row) % 16 != 0 || (2 * P.gu_sc) % 16 != 0) return cudaErrorNotSupported;
  // shared-memory map
  size_t o = ds_align(sizeof(DSShared), 128);
  P.sm_route = static_cast<int>(o);
  o = ds_align(o + (9 * static_cast<size_t>(np) + 1 + (a.route ? c.E : 0)) * 4, 128);
  P.sm_zs = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(n_rows) * P.rpc * 4, 128);
  P.sm_xres = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(T) * P.rpc * 4, 128);
  P.sm_hs = static_cast<int>(o);
  const int nu_max0 = np < c.E ? np : c.E;
  // gate/up work (h rows x channel blocks) split among the CTAs in 32-bit
  // arithmetic; a CTA's blocks start at distinct work offsets of its share
  const long long gu_w = static_cast<long long>(nbf) * T * (c.k + (a.shared != nullptr ? 1 : 0));
  if (static_cast<long long>(nu_max0) * nbf * G >= (1ll << 31) || gu_w * G >= (1ll << 31) ||
      static_cast<long long>(c.E > P.n_units ? c.E : P.n_units) * G >= (1ll << 31))
    return cudaErrorNotSupported;
  P.max_blk = static_cast<int>((gu_w + G - 1) / G);
  if (P.max_blk > kDsMaxBlk) return cudaErrorNotSupported;
  const size_t hs_bytes = static_cast<size_t>(P.max_blk) * T * 32 * 4;
  o = ds_align(o + hs_bytes, 128);
  P.sm_xq = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(T) * kQW * nbd * 4, 128);
  // the next router's columns of this CTA's rows, and its rows of the next input
  P.sm_ws = static_cast<int>(o);
  o = ds_align(o + (a.route ? static_cast<size_t>(c.E) * P.rpc * 4 : 0), 128);
  P.sm_ysl = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(T) * P.rpc * 4, 128);
  P.sm_shdn = static_cast<int>(o);
  o = ds_align(o + 2 * static_cast<size_t>(P.dn_stride), 128);
  const size_t before_gub = o;
  // then the per-warp gate/up buffers, the staging area and the ring. The
  // staging area holds the top-k key rows; the gate/up buffers and the
  // staging area together hold the quantised h rows of a round of down
  // stages (at least T rows). The first of (gate/up depth, experts per down
  // group) from (4, 6) down to (2, 1) that leaves room for two ring slots
  // wins.
  const size_t hq_row = static_cast<size_t>(kQW) * nbf * 4;
  const size_t keys_bytes = static_cast<size_t>(T) * c.k * 4;  // the grouping's sort keys
  size_t x_min = keys_bytes;
  if (x_min < T * hq_row) x_min = T * hq_row;
  int n_ring = 0;
  size_t fixed = 0, x_bytes = 0;
  for (int depth = kDsGuDepth; depth >= 2 && n_ring < 2; --depth) {
    for (int gpd : {kDsGpd, 4, 2, 1}) {
      const int slot_bytes = static_cast<int>(ds_align(static_cast<size_t>(gpd) * P.dn_stride, 128));
      fixed = ds_align(before_gub + static_cast<size_t>(CW) * depth * P.gu_task_bytes, 128);
      auto ring_slots = [&](size_t xb) {
        const long long r = static_cast<long long>(kDsSmemMax) - static_cast<long long>(ds_align(fixed + xb, 128));
        return r > 0 ? static_cast<int>(r / slot_bytes) : 0;
      };
      x_bytes = ds_align(x_min, 128);
      n_ring = ring_slots(x_bytes);
      if (n_ring >= 2) {
        P.gu_depth = depth;
        P.slot_bytes = slot_bytes;
        P.gpd = slot_bytes / P.dn_stride;
        break;
      }
    }
  }
  if (n_ring < 2) return cudaErrorNotSupported;
  if (n_ring > kDsNS) n_ring = kDsNS;
  P.sm_gub = static_cast<int>(before_gub);
  P.sm_x = static_cast<int>(fixed);
  P.hq_rows = static_cast<int>((fixed - before_gub + x_bytes) / hq_row);
  if (P.hq_rows > n_rows) P.hq_rows = n_rows;
  o = ds_align(fixed + x_bytes, 128);
  P.n_ring = n_ring;
  P.fd_ring = make_fastdiv(n_ring);
  P.fd_hrow = make_fastdiv(nbf * (kQW / 2));
  P.fd_hp = make_fastdiv(P.rpc / 2);
  P.fd_gpd = make_fastdiv(P.gpd);
  P.sm_ring = static_cast<int>(o);
  o += static_cast<size_t>(n_ring) * P.slot_bytes;
  if (o > static_cast<size_t>(kDsSmemMax)) return cudaErrorNotSupported;

  if (getenv("MOE_DEBUG") != nullptr)
    fprintf(stderr,
            "decode_stack: bits=%d T=%d L=%d route=%d G=%d smem=%zu n_ring=%d slot=%d gpd=%d dn_stride=%d "
            "hq_rows=%d rpc=%d gran=%d coop_pdl=%d\n",
            c.bits, T, a.L, a.route ? 1 : 0, G, o, P.n_ring, P.slot_bytes, P.gpd, P.dn_stride, P.hq_rows, P.rpc,
            P.gran, ctx.coop_pdl ? 1 : 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3((CW + 1) * 32);
  cfg.dynamicSmemBytes = o;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  // programmatic serialization lets the next launch's prologue overlap this
  // one's tail, where the device takes it together with a cooperative launch
  cfg.numAttrs = ctx.coop_pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kern, P);
}

}  // namespace moe
