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
//    producer warp issuing cp.async.bulk copies and 15 (2-bit) or 11 (3-bit)
//    consumer warps.
//  * Cross-CTA data moves as 64-bit words that carry a 32-bit payload and a
//    32-bit tag naming the layer; a reader polls the words themselves until
//    every tag matches. There are no grid barriers, fences or atomics on the
//    critical path. Tags come from a per-device counter that every launch
//    advances, so words left by earlier launches never match.
//  * Per layer: x (every CTA reads all of it) -> router rows of this CTA ->
//    logits words -> top-k and grouping in every CTA -> the producer issues
//    ALL of this CTA's routed gate/up and down rows at once into two
//    fixed-slot rings -> gate/up + SwiGLU, each 32-channel block of h
//    requantised to int16 by the CTA that owns it and published as words ->
//    every CTA stages all of h and computes its slice of output rows for
//    every expert -> combine -> output words (the next layer's x).
//  * Layer l + 1's router rows and shared expert do not depend on x: the
//    producer fetches them while layer l is still running.
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
constexpr int kDsNHS = 4;       // h staging slots of the gate/up epilogue
constexpr int kDsCps = 16;      // gate/up channels per ring stage
constexpr int kQW = 18;         // words per quantised 32-value block: 16 int16 pairs, scale, sum
constexpr int kDsMaxCtas = 256;  // grid size limit (done words per layer parity)
constexpr int kDsLogitCopies = 4;  // copies of the logit words: CTA b reads copy b % 4
constexpr int kDsPollNs = 64;      // back-off between polls of words that were not there yet

// Tag source: every launch reads it and the last CTA to exit advances it by
// the number of layers; tags of a launch are base + 1 .. base + L.
__device__ unsigned int g_ds_epoch;
__device__ unsigned int g_ds_exit;

// Offsets (bytes) of the arrays of one layer's routing record.
struct RecOff {
  int logits, idx, gate, expert_count, expert_offset, pair_token, pair_j, pair_gate, pair_slot, pair_pos;
  int uniq_expert, uniq_slot, uniq_offset, n_uniq;
};

struct DSParams {
  const uint16_t* x;            // [T, d] bf16: layer 0's input
  int T, d, f, E, k, L, renorm, residual, has_shared, out_f32;
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
  unsigned long long* logits_ll;  // [kDsLogitCopies, T, E]
  unsigned long long* h_ll;       // [n_rows, f/32, kQW]
  unsigned long long* y_ll;       // [2, T, d/2]
  unsigned long long* done_ll;    // [2, kDsMaxCtas]
  int* status;
  unsigned long long timeout_ns;
  unsigned long long* trace;
  // geometry (host computed)
  int gu_lpr, dn_lpr, gran, n_units;
  int gu_row, gu_sc, dn_row, dn_sc;  // bytes per row: codes, scales
  int rpc;                      // output rows per CTA (at most)
  int n_ring, slot_bytes;       // weight ring: slots and bytes per slot
  int dn_stride, gpd;           // bytes per down stage, down stages per ring slot
  int hq_rows;
  int sm_wr, sm_x, sm_xq, sm_hs, sm_zs, sm_route, sm_xres, sm_ring, sm_shdn;
};

struct DSShared {
  uint64_t full[kDsNS], empty[kDsNS];   // weight ring
  uint64_t shdn_full[2], shdn_empty[2];  // the shared expert's down rows, by layer parity
  uint64_t wr_full, wr_empty, route_bar;
  int abort_flag;
  unsigned base_tag;
  int n_uniq;
  int hs_done[kDsNHS];  // channel tasks finished for the block staged in the slot
  int hs_gen[kDsNHS];   // epilogues finished in the slot
};

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
  const float inv = m > 0.f ? 32767.f / m : 0.f;
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
constexpr int kXB = 4;

template <int BITS>
__device__ void ds_read_x(const DSParams& P, int l, uint32_t tag, uint16_t* xs, int* xq, float* xres, int r0,
                          int r1, DSShared* S, uint64_t deadline, int CT) {
  const int nb = P.d / kBlock, bpl = nb / P.gu_lpr;
  const int words = kQW * nb;
  const int jobs = P.T * nb * 4;  // four threads per 32-value block
  const int tid = threadIdx.x;
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
        const int t = job / nb, blk = job % nb;
        const uint4 raw =
            __ldcg(reinterpret_cast<const uint4*>(P.x + static_cast<size_t>(t) * P.d + blk * kBlock + 8 * q));
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
        const int t = job / nb, blk = job % nb;
        src[i] = yl + static_cast<size_t>(t) * (P.d / 2) + blk * 16 + 4 * q;
        ld_ll2(src[i], v[i][0], v[i][1]);
        ld_ll2(src[i] + 2, v[i][2], v[i][3]);
      }
      // every CTA's done word rides along in the first batch
      const unsigned long long* dp = P.done_ll + static_cast<size_t>((l - 1) & 1) * kDsMaxCtas + tid;
      const bool has_done = k0 == 0 && tid < static_cast<int>(gridDim.x);
      unsigned long long dw = has_done ? ld_ll(dp) : ll_word(0u, tag - 1);
      while (true) {
        bool all = tag_ok(dw, tag - 1);
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
        if (!tag_ok(dw, tag - 1)) dw = ld_ll(dp);
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
      const int t = job / nb, blk = job % nb;
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
      const int gl = blk / bpl, bb = blk % bpl;
      quant_quad_c2(v8, xq + t * words, nb, bb * P.gu_lpr + gl, q, live);
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

// Warp t: polls token t's E <= 512 logit words (16 per lane), selects its k
// experts and gates into R. Fast path: the k-th largest of the 32 lane maxima
// bounds the k-th largest key from below; when at most 32 keys reach it they
// are ranked against each other in one pass, otherwise k rounds of warp
// maximum select them. The publishing CTA also writes the plain logits.
__device__ void ds_topk(const DSParams& P, const DSRoute& R, int t, uint32_t tag, float* pub_logits,
                        unsigned long long* scratch, DSShared* S, uint64_t deadline) {
  constexpr int VPL = 16;
  const int lane = threadIdx.x & 31;
  const unsigned long long* row =
      P.logits_ll + (static_cast<size_t>(blockIdx.x % kDsLogitCopies) * P.T + t) * P.E;
  unsigned long long w[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) w[v] = ld_ll(row + min(v * 32 + lane, P.E - 1));
  bool ok = true;
  while (true) {  // re-poll only the words not there yet, all at once
    bool all = true;
#pragma unroll
    for (int v = 0; v < VPL; ++v) all = all && tag_ok(w[v], tag);
    if (all) break;
    if (ds_aborted(S) || global_timer_ns() > deadline) {
      ok = false;
      break;
    }
    __nanosleep(kDsPollNs);
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (!tag_ok(w[v], tag)) w[v] = ld_ll(row + min(v * 32 + lane, P.E - 1));
  }
  if (!__all_sync(0xffffffffu, ok)) {
    if (lane == 0 && !ds_aborted(S)) ds_abort(S, P.status, 22);
    return;
  }
  float lv[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) lv[v] = __uint_as_float(static_cast<uint32_t>(w[v]));
  if (pub_logits != nullptr) {
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (v * 32 + lane < P.E) pub_logits[static_cast<size_t>(t) * P.E + v * 32 + lane] = lv[v];
  }
  uint32_t key[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) key[v] = v * 32 + lane < P.E ? ds_order_key(lv[v]) : 0u;
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
  const uint32_t Lk = __shfl_sync(0xffffffffu, srt, P.k - 1);
  int cnt = 0;
#pragma unroll
  for (int v = 0; v < VPL; ++v) cnt += (Lk > 0u && key[v] >= Lk) ? 1 : 0;
  const int C = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(cnt)));
  if (Lk > 0u && C <= 32) {
    int pos = cnt;  // exclusive prefix of cnt over the lanes
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, pos, o);
      if (lane >= o) pos += n;
    }
    pos -= cnt;
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (Lk > 0u && key[v] >= Lk)  // larger word = larger key, then lower expert index
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
#pragma unroll
      for (int v = 0; v < VPL; ++v) key[v] = (v * 32 + lane == e) ? 0u : key[v];
      if (lane == j) {
        mine_key = M;
        mine_e = e;
      }
    }
  }
  const bool sel = lane < P.k;
  const float lj = sel ? ds_key_value(mine_key) : 0.f;
  const float l0 = __shfl_sync(0xffffffffu, lj, 0);
  const float ex = sel ? expf(lj - l0) : 0.f;
  float denom;
  if (P.renorm) {
    denom = warp_sum(ex);
  } else {
    float s = 0.f;  // full-softmax denominator over every logit of the row
#pragma unroll
    for (int v = 0; v < VPL; ++v)
      if (v * 32 + lane < P.E) s += expf(lv[v] - l0);
    denom = warp_sum(s);
  }
  if (sel) {
    R.idx[t * P.k + lane] = mine_e;
    R.gate[t * P.k + lane] = ex / denom;
  }
}

// Stable sort of the T*k pairs by expert in shared memory, the unique
// experts and their slots. Every consumer thread takes part.
__device__ void ds_group(const DSParams& P, const DSRoute& R, DSShared* S, int np, int CT) {
  const int tid = threadIdx.x;
  for (int p = tid; p < np; p += CT) {
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
  named_sync(1, CT);
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
  named_sync(1, CT);
}

// Writes layer l's routing record (the publishing CTA only).
__device__ void ds_publish(const DSParams& P, const DSRoute& R, int l, int np, int nu, int CT) {
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
  for (int q = tid; q < np; q += CT) {
    const int pos = R.pair_pos[q];
    const int e = min(max(R.idx[q], 0), P.E - 1);
    int slot = R.slot_s[e];
    if (slot < 0 || slot >= P.n_slots) slot = 0;
    idx[q] = R.idx[q];
    gate[q] = R.gate[q];
    pp[q] = pos;
    pt[pos] = q / P.k;
    pj[pos] = q % P.k;
    pg[pos] = R.gate[q];
    ps[pos] = slot;
  }
  for (int u = tid; u < nu; u += CT) {
    ue[u] = R.uniq_e[u];
    us[u] = R.uniq_slot[u];
    uo[u] = R.uniq_off[u];
  }
  if (tid == 0) {
    uo[nu] = np;
    *reinterpret_cast<int32_t*>(rec + P.ro.n_uniq) = nu;
  }
  for (int e = tid; e < P.E; e += CT) {  // counts by binary search in the sorted experts
    int lo = 0, hi = np;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (R.sorted_e[mid] < e) lo = mid + 1; else hi = mid;
    }
    int lo2 = lo, hi2 = np;
    while (lo2 < hi2) {
      const int mid = (lo2 + hi2) >> 1;
      if (R.sorted_e[mid] <= e) lo2 = mid + 1; else hi2 = mid;
    }
    ec[e] = lo2 - lo;
    eo[e] = lo;
    if (e == P.E - 1) eo[P.E] = np;
  }
}

// ------------------------------------------------------------------ router
// Router rows [e0, e1) of this CTA for every token (W_r rows and x in shared
// memory); each logit goes out as a tagged word. Lanes take interleaved
// 4-column groups and the warp sum is a fixed butterfly, so a token's logit
// does not depend on the batch.
__device__ void ds_router(const DSParams& P, int l, uint32_t tag, const float* wrs, const uint16_t* xs, int e0,
                          int e1, int CW) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n4 = P.d / 4, nr = e1 - e0;
  const float* bias = P.bias != nullptr ? P.bias + static_cast<size_t>(l) * P.T * P.E : nullptr;
#pragma unroll 1
  for (int task = warp; task < nr * P.T; task += CW) {
    const int e = e0 + task % nr, t = task / nr;
    const float4* w4 = reinterpret_cast<const float4*>(wrs + static_cast<size_t>(e - e0) * P.d);
    const uint2* x2 = reinterpret_cast<const uint2*>(xs + static_cast<size_t>(t) * P.d);
    const size_t o = static_cast<size_t>(t) * P.E + e;
    const float bv = bias != nullptr ? __ldg(bias + o) : 0.f;
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
    if (lane < kDsLogitCopies)
      st_ll(P.logits_ll + static_cast<size_t>(lane) * P.T * P.E + o, ll_word(__float_as_uint(acc + bv), tag));
  }
}

// ------------------------------------------------------------------ gate/up
// Rows of h: routed pair p at p (sorted order), shared token t at np + t.
struct GUBlock {
  const uint8_t* rec;  // not used by consumers (the ring holds the rows)
  int u;               // unique-expert index, or -1 for the shared expert
  int cb;              // channel block inside the expert
};

__device__ __forceinline__ void gu_block_of(int beta, int nsh, int sb0, int rb0, int nbf, GUBlock& gb) {
  if (beta < nsh) {
    gb.u = -1;
    gb.cb = sb0 + beta;
  } else {
    const int g = rb0 + beta - nsh;
    gb.u = g / nbf;
    gb.cb = g % nbf;
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

// One gate/up channel task: channel c (of a 32-channel block) for every token
// of the block's expert, the weights in ring stage `st`; h values -> hs.
template <int BITS, int BPL>
__device__ __forceinline__ void gu_task(const DSParams& P, const DSRoute& R, const uint8_t* st, int cl,
                                        const int* xq, int u, int np, float* hs, int c, int& cur_t,
                                        XR<BITS>* xr) {
  const int lane = threadIdx.x & 31;
  const int lpr = P.gu_lpr, gl = lane % lpr;
  const bool active = lane < lpr;
  const int nb = P.d / kBlock;
  const uint8_t* cg = st + 2 * cl * P.gu_row;
  const uint16_t* sg = reinterpret_cast<const uint16_t*>(st + 2 * kDsCps * P.gu_row) + 2 * cl * nb;
  int first, n;
  expert_h_rows(R, u, np, P.T, first, n);
#pragma unroll 1
  for (int i = 0; i < n; ++i) {
    const int t = h_row_token(R, u, first, i);
    if (t != cur_t) {
      load_xq<BITS, BPL>(xq + t * kQW * nb, nb, lpr, gl, xr);
      cur_t = t;
    }
    float2 v = make_float2(0.f, 0.f);
    if (active) v = row_dot2<BITS, BPL>(cg, sg, cg + P.gu_row, sg + nb, P.d, gl, xr);
    v = group_sum2(v, lpr);
    // fast exponential and division: h is requantised to 16 bits for the
    // down rows, far coarser than their few-ulp error
    if (lane == 0) hs[i * 32 + c] = __fdividef(v.x, 1.f + __expf(-v.x)) * v.y;
  }
}

// ------------------------------------------------------------------ down
// Stages the quantised h rows of DN stages [i0, i1) into hq (every consumer
// thread takes part), in stage order. A thread loads up to kHB 16-byte units
// at once and re-polls, together, only the words not there yet.
constexpr int kHB = 8;

__device__ void ds_stage_h(const DSParams& P, const DSRoute& R, int np, int i0, int i1, bool sh_first, uint32_t tag,
                           int* hq, DSShared* S, uint64_t deadline, int CT) {
  const int nbf = P.f / kBlock, bpl = nbf / P.dn_lpr;
  const int units_per_row = nbf * (kQW / 2);  // 16-byte units
  // rows of the round: stage order, each stage's rows contiguous in h
  int n_rows = 0;
  for (int i = i0; i < i1; ++i) {
    const int u = (sh_first && i == 0) ? -1 : i - (sh_first ? 1 : 0);
    int first, n;
    expert_h_rows(R, u, np, P.T, first, n);
    n_rows += n;
  }
  const int units = n_rows * units_per_row;
#pragma unroll 1
  for (int j0 = threadIdx.x; j0 < units; j0 += kHB * CT) {
    unsigned long long v[kHB][2];
    const unsigned long long* src[kHB];
    int dst_row[kHB], dst_col[kHB], dst_w[kHB];
#pragma unroll
    for (int k = 0; k < kHB; ++k) {
      const int j = min(j0 + k * CT, units - 1);
      const int r = j / units_per_row, rem = j % units_per_row;
      // row r of the round -> its h row (walk the stages)
      int base = 0, hrow = 0;
      for (int i = i0; i < i1; ++i) {
        const int u = (sh_first && i == 0) ? -1 : i - (sh_first ? 1 : 0);
        int first, n;
        expert_h_rows(R, u, np, P.T, first, n);
        if (r < base + n) {
          hrow = first + (r - base);
          break;
        }
        base += n;
      }
      const int blk = rem / (kQW / 2), w2 = rem % (kQW / 2);
      src[k] = P.h_ll + (static_cast<size_t>(hrow) * nbf + blk) * kQW + 2 * w2;
      dst_row[k] = r;
      dst_col[k] = (blk % bpl) * P.dn_lpr + blk / bpl;
      dst_w[k] = 2 * w2;
      ld_ll2(src[k], v[k][0], v[k][1]);
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
      if (j0 + k * CT < units) {
        int* dst = hq + dst_row[k] * kQW * nbf;
        dst[dst_w[k] * nbf + dst_col[k]] = static_cast<int>(static_cast<uint32_t>(v[k][0]));
        dst[(dst_w[k] + 1) * nbf + dst_col[k]] = static_cast<int>(static_cast<uint32_t>(v[k][1]));
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
  const int lpr = P.dn_lpr, rpw = 32 / lpr;
  const int rl = lane / lpr, gl = lane % lpr;
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
// One ring of fixed-size slots carries, in order, every gate/up stage (16
// channels) and down group (the down rows of up to `gpd` routed experts) of
// a layer; consumers free a slot with 16 arrivals. Down groups follow the
// gate/up stages, so they stream in while gate/up is still computing.
__device__ __forceinline__ bool ring_slot_free(uint64_t* empty, uint32_t seq, int n) {
  return seq < static_cast<uint32_t>(n) || mbar_test(&empty[seq % n], ((seq / n) - 1) & 1);
}

__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}

__device__ __forceinline__ void issue_gu(const DSParams& P, DSShared* S, uint8_t* ring, uint32_t seq,
                                         const uint8_t* rec, int ch0) {
  const int slot = seq % P.n_ring;
  uint8_t* dst = ring + static_cast<size_t>(slot) * P.slot_bytes;
  const uint32_t cb = 2 * kDsCps * P.gu_row, sb = 2 * kDsCps * P.gu_sc;
  mbar_arrive_expect_tx(&S->full[slot], cb + sb);
  bulk_g2s(dst, rec + P.lay.gu_codes + static_cast<size_t>(2 * ch0) * P.gu_row, cb, &S->full[slot]);
  bulk_g2s(dst + cb, rec + P.lay.gu_scales + static_cast<size_t>(2 * ch0) * P.gu_sc, sb, &S->full[slot]);
}

// Down rows [r0, r1) of one record into dst (codes, then scales).
__device__ __forceinline__ void copy_dn(const DSParams& P, uint8_t* dst, const uint8_t* rec, int r0, int r1,
                                        uint64_t* bar) {
  const uint32_t cb = (r1 - r0) * P.dn_row, sb = (r1 - r0) * P.dn_sc;
  bulk_g2s(dst, rec + P.lay.dn_codes + static_cast<size_t>(r0) * P.dn_row, cb, bar);
  bulk_g2s(dst + cb, rec + P.lay.dn_scales + static_cast<size_t>(r0) * P.dn_sc, sb, bar);
}

// Waits (bounded) until ring slot `seq` may be reused.
__device__ __forceinline__ bool wait_slot(DSShared* S, uint64_t* empty, uint32_t seq, int n, uint64_t deadline) {
  while (!ring_slot_free(empty, seq, n)) {
    if (ds_aborted(S) || global_timer_ns() > deadline) return false;
    __nanosleep(32);
  }
  return true;
}

// ------------------------------------------------------------------ the kernel
template <int BITS, int GBPL, int DBPL, bool ROUTE>
__global__ void __launch_bounds__((ds_consumer_warps(BITS) + 1) * 32, 1) decode_stack_kernel(const DSParams P) {
  constexpr int CW = ds_consumer_warps(BITS);
  constexpr int CT = CW * 32;
  extern __shared__ __align__(128) char smem[];
  DSShared* S = reinterpret_cast<DSShared*>(smem);
  const int np = P.T * P.k;
  const DSRoute R = ds_route(smem + P.sm_route, np);
  float* wrs = reinterpret_cast<float*>(smem + P.sm_wr);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + P.sm_x);
  int* hq = reinterpret_cast<int*>(smem + P.sm_x);  // the same region after the router
  int* xq = reinterpret_cast<int*>(smem + P.sm_xq);
  float* hs = reinterpret_cast<float*>(smem + P.sm_hs);
  float* zs = reinterpret_cast<float*>(smem + P.sm_zs);
  float* xres = reinterpret_cast<float*>(smem + P.sm_xres);
  uint8_t* ring = reinterpret_cast<uint8_t*>(smem + P.sm_ring);
  uint8_t* shdn = reinterpret_cast<uint8_t*>(smem + P.sm_shdn);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, b = blockIdx.x;
  const int nbf = P.f / kBlock;

  // static splits: router rows, output rows (units of `gran` rows) and the
  // shared expert's channel blocks of this CTA
  const int e0 = static_cast<int>((static_cast<long long>(P.E) * b) / G);
  const int e1 = static_cast<int>((static_cast<long long>(P.E) * (b + 1)) / G);
  const int r0 = P.gran * static_cast<int>((static_cast<long long>(P.n_units) * b) / G);
  const int r1 = P.gran * static_cast<int>((static_cast<long long>(P.n_units) * (b + 1)) / G);
  const int sb0 = P.has_shared ? (b * nbf + G - 1) / G : 0;
  const int sb1 = P.has_shared ? ((b + 1) * nbf + G - 1) / G : 0;
  const int nsh = sb1 - sb0;
  const bool has_rows = r1 > r0;
  const bool wr_rows = ROUTE && e1 > e0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kDsNS; ++i) {
      mbar_init(&S->full[i], 1);
      mbar_init(&S->empty[i], kDsCps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S->shdn_full[i], 1);
      mbar_init(&S->shdn_empty[i], 1);
    }
    mbar_init(&S->wr_full, 1);
    mbar_init(&S->wr_empty, CW);
    mbar_init(&S->route_bar, 1);
    S->abort_flag = 0;
    for (int i = 0; i < kDsNHS; ++i) {
      S->hs_done[i] = 0;
      S->hs_gen[i] = 0;
    }
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

  if (warp == CW) {
    // ============================================================ producer
    if (lane == 0) {
      uint32_t seq = 0, wr_count = 0, shdn_count = 0;
      bool ok = true;
      auto issue_wr = [&](int l) {
        const uint32_t bytes = static_cast<uint32_t>((e1 - e0) * P.d * 4);
        mbar_arrive_expect_tx(&S->wr_full, bytes);
        bulk_g2s(wrs, P.wr + (static_cast<size_t>(l) * P.E + e0) * P.d, bytes, &S->wr_full);
        ++wr_count;
      };
      // layer l's shared-expert down rows: buffer l & 1, its (l >> 1)-th use
      auto issue_shdn = [&](int l) {
        const int j = l & 1;
        if (l >= 2) {
          while (!mbar_try_wait(&S->shdn_empty[j], ((l >> 1) - 1) & 1, 20000u)) {
            if (ds_aborted(S) || global_timer_ns() > deadline) {
              ok = false;
              return;
            }
          }
        }
        const uint8_t* rec = P.shared + static_cast<size_t>(l) * P.stride;
        mbar_arrive_expect_tx(&S->shdn_full[j], (r1 - r0) * (P.dn_row + P.dn_sc));
        copy_dn(P, shdn + j * P.dn_stride, rec, r0, r1, &S->shdn_full[j]);
        ++shdn_count;
      };
      auto issue_shgu = [&](int l) {
        const uint8_t* rec = P.shared + static_cast<size_t>(l) * P.stride;
        for (int blk = sb0; blk < sb1 && ok; ++blk)
          for (int q = 0; q < 32 / kDsCps && ok; ++q) {
            if (!(ok = wait_slot(S, S->empty, seq, P.n_ring, deadline))) break;
            issue_gu(P, S, ring, seq++, rec, blk * 32 + q * kDsCps);
          }
      };
      if (!ds_aborted(S)) {
        if (wr_rows) issue_wr(0);
        if (P.has_shared && has_rows) issue_shdn(0);
        if (P.has_shared) issue_shgu(0);
      }
      for (int l = 0; l < P.L && ok && !ds_aborted(S); ++l) {
        // routing of layer l is in shared memory once route_bar completes
        while (!mbar_try_wait(&S->route_bar, l & 1, 20000u)) {
          if (ds_aborted(S) || global_timer_ns() > deadline) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        unsigned long long* td = (trace != nullptr && l == dl) ? trace : nullptr;
        if (td) td[16] = global_timer_ns();
        const int nu = S->n_uniq;
        const int tot = nu * nbf;
        const int rb0 = static_cast<int>((static_cast<long long>(tot) * b) / G);
        const int rb1 = static_cast<int>((static_cast<long long>(tot) * (b + 1)) / G);
        for (int ig = 0; ig < (rb1 - rb0) * (32 / kDsCps) && ok; ++ig) {
          const int blk = rb0 + ig / (32 / kDsCps);
          const int u = blk / nbf, cb = blk % nbf;
          if (!(ok = wait_slot(S, S->empty, seq, P.n_ring, deadline))) break;
          issue_gu(P, S, ring, seq++, P.pool + static_cast<size_t>(R.uniq_slot[u]) * P.stride,
                   cb * 32 + (ig % (32 / kDsCps)) * kDsCps);
          if (td && ig == 0) td[17] = global_timer_ns();
        }
        if (td) td[18] = global_timer_ns();
        const int n_grp = has_rows ? (nu + P.gpd - 1) / P.gpd : 0;
        for (int g = 0; g < n_grp && ok; ++g) {
          if (!(ok = wait_slot(S, S->empty, seq, P.n_ring, deadline))) break;
          const int u0 = g * P.gpd, u1 = min(nu, u0 + P.gpd);
          const int slot = seq % P.n_ring;
          uint8_t* dst = ring + static_cast<size_t>(slot) * P.slot_bytes;
          mbar_arrive_expect_tx(&S->full[slot], (u1 - u0) * (r1 - r0) * (P.dn_row + P.dn_sc));
          for (int u = u0; u < u1; ++u)
            copy_dn(P, dst + (u - u0) * P.dn_stride, P.pool + static_cast<size_t>(R.uniq_slot[u]) * P.stride, r0, r1,
                    &S->full[slot]);
          ++seq;
        }
        if (td) td[19] = global_timer_ns();
        if (!ok) break;
        if (l + 1 < P.L) {
          // the next layer's inputs that do not depend on x
          if (wr_rows) {
            while (!mbar_try_wait(&S->wr_empty, l & 1, 20000u)) {
              if (ds_aborted(S) || global_timer_ns() > deadline) {
                ok = false;
                break;
              }
            }
            if (!ok) break;
            issue_wr(l + 1);
          }
          if (P.has_shared && has_rows) issue_shdn(l + 1);
          if (P.has_shared && ok) issue_shgu(l + 1);
        }
      }
      if (!ok && !ds_aborted(S)) ds_abort(S, P.status, 10);
      // every issued copy lands before the CTA may exit (they take
      // microseconds; the 100 ms bound only guards against the impossible)
      const uint64_t d2 = global_timer_ns() + 100000000ull;
      for (uint32_t q = seq > static_cast<uint32_t>(P.n_ring) ? seq - P.n_ring : 0; q < seq; ++q)
        while (!mbar_try_wait(&S->full[q % P.n_ring], (q / P.n_ring) & 1, 20000u) && global_timer_ns() < d2) {
        }
      for (uint32_t q = shdn_count > 2u ? shdn_count - 2u : 0u; q < shdn_count; ++q)
        while (!mbar_try_wait(&S->shdn_full[q & 1], (q >> 1) & 1, 20000u) && global_timer_ns() < d2) {
        }
      if (wr_count > 0)
        while (!mbar_try_wait(&S->wr_full, (wr_count - 1) & 1, 20000u) && global_timer_ns() < d2) {
        }
    }
    __syncwarp();
  } else {
    // ============================================================ consumers
    const int tid = threadIdx.x;
    uint32_t seq = 0, blk_seq = 0;
    XR<BITS> xr[GBPL];
#pragma unroll 1
    for (int l = 0; l < P.L; ++l) {
      const uint32_t tag = base + 1 + static_cast<uint32_t>(l);
      // trace slots: 8 phase stamps for layers 0 and 1, then details of
      // layer dl (the second one when there is one)
      const bool traced = trace != nullptr && l < 2 && tid == 0;
      unsigned long long* tdet = (trace != nullptr && l == dl) ? trace : nullptr;
      if (traced) trace[8 * l] = global_timer_ns();
      // ---- x of this layer
      if (!ds_aborted(S))
        ds_read_x<BITS>(P, ROUTE ? l : 0, tag, wr_rows ? xs : nullptr, xq, xres, r0, r1, S, deadline, CT);
      if (ROUTE) {
        for (int e = tid; e < P.E; e += CT) R.slot_s[e] = __ldg(P.slot_of + static_cast<size_t>(l) * P.E + e);
      }
      named_sync(1, CT);
      if (traced) trace[8 * l + 1] = global_timer_ns();
      int nu = 0;
      if (ROUTE) {
        // ---- router rows of this CTA
        if (wr_rows) {
          if (ds_wait_warp(&S->wr_full, l & 1, S, deadline)) {
            if (!ds_aborted(S)) ds_router(P, l, tag, wrs, xs, e0, e1, CW);
          } else if (lane == 0 && !ds_aborted(S)) {
            ds_abort(S, P.status, 1);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&S->wr_empty);
        }
        if (traced) trace[8 * l + 2] = global_timer_ns();
        // ---- top-k (warp t) and grouping (all)
        const bool publisher = b == l % G;
        float* pub = publisher ? reinterpret_cast<float*>(P.rec + static_cast<size_t>(l) * P.rec_bytes + P.ro.logits)
                               : nullptr;
        if (warp < P.T && !ds_aborted(S))
          ds_topk(P, R, warp, tag, pub, reinterpret_cast<unsigned long long*>(hs) + warp * 32, S, deadline);
        if (tdet && tid == 0) tdet[20] = global_timer_ns();
        named_sync(1, CT);
        if (!ds_aborted(S)) ds_group(P, R, S, np, CT);
        else named_sync(1, CT), named_sync(1, CT);
        nu = S->n_uniq;
        if (tdet && tid == 0) tdet[21] = global_timer_ns();
        if (tid == 0) mbar_arrive(&S->route_bar);
        if (publisher && !ds_aborted(S)) ds_publish(P, R, l, np, nu, CT);
      } else {
        // the grouping was written by moe_group_tokens
        const int nug = min(max(__ldcg(P.g.n_uniq), 0), min(np, P.E));
        for (int p = tid; p < np; p += CT) {
          R.pair_token[p] = min(max(__ldcg(P.g.pair_token + p), 0), P.T - 1);
          R.pair_gate[p] = __ldcg(P.g.pair_gate + p);
          R.pair_pos[p] = min(max(__ldcg(P.g.pair_pos + p), 0), np - 1);
        }
        for (int u = tid; u <= nug; u += CT) R.uniq_off[u] = min(max(__ldcg(P.g.uniq_offset + u), 0), np);
        for (int u = tid; u < nug; u += CT) {
          int slot = __ldcg(P.g.uniq_slot + u);
          if (slot < 0 || slot >= P.n_slots) {
            report(P.status, kDevBadSlot, u);
            slot = 0;
          }
          R.uniq_slot[u] = slot;
        }
        if (tid == 0) S->n_uniq = nug;
        named_sync(1, CT);
        nu = nug;
        if (tid == 0) mbar_arrive(&S->route_bar);
      }
      if (traced) trace[8 * l + 3] = global_timer_ns();

      // ---- gate/up + SwiGLU: 32 channel tasks per block, blocks in order
      const int tot = nu * nbf;
      const int rb0 = static_cast<int>((static_cast<long long>(tot) * b) / G);
      const int rb1 = static_cast<int>((static_cast<long long>(tot) * (b + 1)) / G);
      const int n_blk = nsh + (rb1 - rb0);
      int cur_t = -1;
#pragma unroll 1
      for (int task = warp; task < n_blk * 32; task += CW) {
        if (ds_aborted(S)) break;
        const int beta = task >> 5, c = task & 31;
        GUBlock gb;
        gu_block_of(beta, nsh, sb0, rb0, nbf, gb);
        const uint32_t sq = seq + beta * (32 / kDsCps) + c / kDsCps;
        const int slot = sq % P.n_ring;
        const uint32_t bid = blk_seq + beta;
        const int hslot = bid % kDsNHS;
        const int gen = bid / kDsNHS;
        // the slot's previous block must have been published
        bool ok = true;
        if (lane == 0) {
          while (*reinterpret_cast<volatile int*>(&S->hs_gen[hslot]) != gen) {
            if (ds_aborted(S) || global_timer_ns() > deadline) {
              ok = false;
              break;
            }
            __nanosleep(20);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (!ok || !ds_wait_warp(&S->full[slot], (sq / P.n_ring) & 1, S, deadline)) {
          if (lane == 0 && !ds_aborted(S)) ds_abort(S, P.status, 2);
          break;
        }
        if (tdet && tid == 0) {
          const int it = task / CW;
          if (it == 0) tdet[22] = global_timer_ns();
          if (it < 8) tdet[24 + it] = global_timer_ns();
        }
        float* hsl = hs + hslot * P.T * 32;
        gu_task<BITS, GBPL>(P, R, ring + static_cast<size_t>(slot) * P.slot_bytes, c % kDsCps, xq, gb.u, np, hsl,
                            c, cur_t, xr);
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          mbar_arrive(&S->empty[slot]);
          __threadfence_block();
          last = atomicAdd(&S->hs_done[hslot], 1) == 31;
        }
        last = __shfl_sync(0xffffffffu, last, 0);
        if (last) {
          // the block's 32 channels are in hs: requantise each token's 32
          // values and publish them as tagged words
          __threadfence_block();
          int first, n;
          expert_h_rows(R, gb.u, np, P.T, first, n);
          for (int i = 0; i < n; ++i) {
            const uint32_t wq = quant_block_warp(hsl[i * 32 + lane], lane);
            if (lane < kQW)
              st_ll(P.h_ll + (static_cast<size_t>(first + i) * nbf + gb.cb) * kQW + lane, ll_word(wq, tag));
          }
          __syncwarp();
          if (lane == 0) {
            S->hs_done[hslot] = 0;
            __threadfence_block();
            *reinterpret_cast<volatile int*>(&S->hs_gen[hslot]) = gen + 1;
          }
        }
      }
      if (tdet && tid == 0) tdet[23] = global_timer_ns();
      seq += n_blk * (32 / kDsCps);
      blk_seq += n_blk;
      named_sync(1, CT);
      if (traced) trace[8 * l + 4] = global_timer_ns();

      // ---- down rows of this CTA for every expert (shared first). Stage i:
      // the shared expert (i = 0, its own buffer) or routed expert u, whose
      // rows sit in ring group u / gpd. A round of stages never spans more
      // groups than the ring has slots, so no warp waits on a slot whose
      // previous use in this layer is still pending.
      const int sh = (P.has_shared && has_rows) ? 1 : 0;
      const int n_dn = has_rows ? nu + sh : 0;
      const int nr_out = r1 - r0;
      const uint32_t grp0 = seq;  // sequence number of this layer's first down group
#pragma unroll 1
      for (int i0 = 0; i0 < n_dn;) {
        int i1 = i0, rows = 0;
        while (i1 < n_dn) {
          const int u = i1 - sh;
          if (u >= 0 && i1 > i0) {
            const int ua = max(i0 - sh, 0);
            if (u / P.gpd - ua / P.gpd >= P.n_ring) break;
          }
          int first, n;
          expert_h_rows(R, u, np, P.T, first, n);
          if (rows + n > P.hq_rows) break;
          rows += n;
          ++i1;
        }
        if (!ds_aborted(S)) ds_stage_h(P, R, np, i0, i1, sh != 0, tag, hq, S, deadline, CT);
        named_sync(1, CT);
        if (traced && i0 == 0) trace[8 * l + 5] = global_timer_ns();
        // each warp takes whole stages; the hq row of stage i is the rows of
        // the stages before it in this round
#pragma unroll 1
        for (int i = i0 + warp; i < i1; i += CW) {
          if (ds_aborted(S)) break;
          int row0 = 0;
          for (int j = i0; j < i; ++j) {
            int fj, nj;
            expert_h_rows(R, j - sh, np, P.T, fj, nj);
            row0 += nj;
          }
          const int u = i - sh;
          const uint8_t* st;
          uint64_t* full;
          uint32_t parity;
          int slot = 0;
          if (u < 0) {
            st = shdn + (l & 1) * P.dn_stride;
            full = &S->shdn_full[l & 1];
            parity = (l >> 1) & 1;
          } else {
            const uint32_t sq = grp0 + u / P.gpd;
            slot = sq % P.n_ring;
            st = ring + static_cast<size_t>(slot) * P.slot_bytes + (u % P.gpd) * P.dn_stride;
            full = &S->full[slot];
            parity = (sq / P.n_ring) & 1;
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
              const int m = min(nu - (u / P.gpd) * P.gpd, P.gpd);
              mbar_arrive_cnt(&S->empty[slot], (u % P.gpd) == 0 ? kDsCps - (m - 1) : 1);
            }
          }
        }
        named_sync(1, CT);
        i0 = i1;
      }
      seq += has_rows ? (nu + P.gpd - 1) / P.gpd : 0;
      // this CTA has read everything of layer l that other CTAs wrote
      if (tid == 0 && ROUTE && l + 1 < P.L)
        st_ll(P.done_ll + static_cast<size_t>(l & 1) * kDsMaxCtas + b, ll_word(0u, tag));
      if (traced) trace[8 * l + 6] = global_timer_ns();

      // ---- combine: y[t, r] = sum_j gate[t,j] z[(t,j)][r] + z_shared[t][r] (+ x)
      if (!ds_aborted(S) && has_rows) {
        const int npairs = nr_out / 2;
        char* yl = static_cast<char*>(P.y) + static_cast<size_t>(l) * P.T * P.d * (P.out_f32 ? 4 : 2);
        unsigned long long* yll = P.y_ll + static_cast<size_t>(l & 1) * P.T * (P.d / 2);
        for (int i = tid; i < P.T * npairs; i += CT) {
          const int t = i / npairs, rr = 2 * (i % npairs);
          float a0 = 0.f, a1 = 0.f;
          for (int j = 0; j < P.k; ++j) {
            const int p = R.pair_pos[t * P.k + j];
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
            if (ROUTE && l + 1 < P.L)
              st_ll(yll + o / 2, ll_word(*reinterpret_cast<const uint32_t*>(&hv), tag));
          }
        }
      }
      if (l + 2 == P.L && tid == 0) grid_dep_launch();
      named_sync(1, CT);
      if (traced) trace[8 * l + 7] = global_timer_ns();
    }
    if (P.L == 1 && tid == 0) grid_dep_launch();
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
__global__ void ds_skip_tags_kernel() {
  atomicAdd(&g_ds_epoch, 1u << 20);
  atomicExch(&g_ds_exit, 0u);
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
  const size_t lg = ds_align(static_cast<size_t>(kDsLogitCopies) * T * c.E * 8, 256);
  const size_t h = ds_align(n_rows * (c.f / kBlock) * kQW * 8, 256);
  const size_t y = ds_align(2 * static_cast<size_t>(T) * (c.d / 2) * 8, 256);
  const size_t dn = 2 * kDsMaxCtas * 8;
  return lg + h + y + dn;
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

cudaError_t decode_skip_tags(cudaStream_t s) {
  ds_skip_tags_kernel<<<1, 1, 0, s>>>();
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
    const size_t lg = ds_align(static_cast<size_t>(kDsLogitCopies) * T * c.E * 8, 256);
    const size_t h = ds_align(static_cast<size_t>(n_rows) * nbf * kQW * 8, 256);
    const size_t y = ds_align(2 * static_cast<size_t>(T) * (c.d / 2) * 8, 256);
    P.logits_ll = reinterpret_cast<unsigned long long*>(ex);
    P.h_ll = reinterpret_cast<unsigned long long*>(ex + lg);
    P.y_ll = reinterpret_cast<unsigned long long*>(ex + lg + h);
    P.done_ll = reinterpret_cast<unsigned long long*>(ex + lg + h + y);
  }
  P.status = ctx.d_status;
  P.timeout_ns = ctx.timeout_ns;
  P.trace = ctx.d_trace;
  P.gu_lpr = gg.lpr;
  P.dn_lpr = gd.lpr;
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
  const int wr_rows = a.route ? (c.E + G - 1) / G : 0;
  // ring slots hold one gate/up stage (16 channels) or a group of down
  // stages (this CTA's output rows of up to gpd experts)
  const size_t gu_stage = static_cast<size_t>(2 * kDsCps) * (P.gu_row + P.gu_sc);
  P.dn_stride = static_cast<int>(ds_align(static_cast<size_t>(P.rpc) * (P.dn_row + P.dn_sc), 16));
  P.slot_bytes = static_cast<int>(ds_align(gu_stage > static_cast<size_t>(P.dn_stride) ? gu_stage : P.dn_stride, 128));
  P.gpd = P.slot_bytes / P.dn_stride;
  // shared-memory map
  size_t o = ds_align(sizeof(DSShared), 128);
  P.sm_route = static_cast<int>(o);
  o = ds_align(o + (9 * static_cast<size_t>(np) + 1 + (a.route ? c.E : 0)) * 4, 128);
  P.sm_zs = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(n_rows) * P.rpc * 4, 128);
  P.sm_xres = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(T) * P.rpc * 4, 128);
  P.sm_hs = static_cast<int>(o);
  const size_t hs_bytes = static_cast<size_t>(kDsNHS) * T * 32 * 4;
  const size_t tk_bytes = static_cast<size_t>(MOE_DECODE_MAX_T) * 32 * 8;  // top-k scratch (aliases hs)
  o = ds_align(o + (hs_bytes > tk_bytes ? hs_bytes : tk_bytes), 128);
  P.sm_xq = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(T) * kQW * nbd * 4, 128);
  P.sm_wr = static_cast<int>(o);
  o = ds_align(o + static_cast<size_t>(wr_rows) * c.d * 4, 128);
  P.sm_shdn = static_cast<int>(o);
  o = ds_align(o + 2 * static_cast<size_t>(P.dn_stride), 128);
  P.sm_x = static_cast<int>(o);
  const size_t fixed = o;
  // the staging area: raw x for the router, then the quantised h rows of a
  // round of down stages (all rows if they fit in 48 KB, else 48 KB worth,
  // at least T rows); at least three ring slots
  const size_t xs_bytes = a.route ? static_cast<size_t>(T) * c.d * 2 : 0;
  const size_t hq_row = static_cast<size_t>(kQW) * nbf * 4;
  size_t hq_bytes = static_cast<size_t>(n_rows) * hq_row;
  const size_t hq_cap = 48 * 1024 > T * hq_row ? 48 * 1024 : T * hq_row;
  if (hq_bytes > hq_cap) hq_bytes = hq_cap;
  const size_t x_bytes = ds_align(xs_bytes > hq_bytes ? xs_bytes : hq_bytes, 128);
  P.hq_rows = static_cast<int>(x_bytes / hq_row);
  if (P.hq_rows > n_rows) P.hq_rows = n_rows;
  o = ds_align(fixed + x_bytes, 128);
  const long long rem = static_cast<long long>(kDsSmemMax) - static_cast<long long>(o);
  int n_ring = static_cast<int>(rem / P.slot_bytes);
  if (n_ring > kDsNS) n_ring = kDsNS;
  if (n_ring < 3) return cudaErrorNotSupported;
  P.n_ring = n_ring;
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
