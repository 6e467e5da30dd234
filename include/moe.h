/*
 * moe.h -- C ABI of libmoe: the per-layer sparse Mixture-of-Experts FFN step
 * of a Qwen3.8-Flash-Next-shaped model on one NVIDIA B200 (sm_100a).
 *
 * The step (per layer, per token t):
 *   1. router logits  l[t,e] = sum_i x[t,i] * W_r[e,i]  (+ an optional bias)
 *   2. top-k          the k largest logits, ties to the lower expert index,
 *                     gates = softmax over the k chosen logits
 *   3. grouping       the T*k (token, j) pairs stably sorted by expert, each
 *                     expert mapped to its slot in an expert pool
 *   4. experts        h = silu(W_g x) * (W_u x), z = W_d h on 2- or 3-bit
 *                     block-quantised weights, dequantised inside the kernels
 *   5. combine        y[t] = sum_j gate[t,j] * z_(t,j) + z_shared[t]
 *
 * The pages this follows describe the model as 48 layers x 512 experts, of
 * which a token uses 10 plus one always-on shared expert (Strataとは,
 * news.blueqat.app/post/3262, first section; geekoyaji.com
 * "freetoken-vs-strata-moe-offload", section 共通の仕組み), expert weights at 2
 * to 3 bits (news.blueqat.app, section 量子化の種類とサイズ), a router and shared
 * expert that run on the GPU for every token (news.blueqat.app, section
 * GPU・CPU・RAM・SSDの分担), decode passes that verify up to 3 drafted tokens
 * at once, so T <= 4 (vramglass.com, section その3), and prefill chunks of up to
 * 8,192 tokens (news.blueqat.app, section GPU・CPU・RAM・SSDの分担). The pages
 * give no formulas and no bit layout; both are defined here.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller. The
 *     library allocates no device memory on any compute call; scratch comes
 *     from a caller workspace of moe_workspace_bytes() bytes.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream). Errors detected on the host are returned at once;
 *     errors detected by a kernel are recorded in the context's device status
 *     word and returned by moe_check_device_status().
 *   - No exception or abort crosses the ABI. A context may be used by one host
 *     thread and one stream at a time; it belongs to the device named at its
 *     creation, and every call made with it launches there (the caller's
 *     current device is restored before the call returns).
 *   - The decode path (T <= MOE_DECODE_MAX_T) is one cooperative launch of a
 *     CTA per SM: it starts once every SM is free, and decode calls on one
 *     device must not overlap in time (one stream, or calls ordered with
 *     events), since they share a per-device tag counter.
 *
 * Expert record (one routed or shared expert, `moe_expert_layout`):
 *   gu_codes  [2f rows, d cols] packed codes; row 2c is gate channel c,
 *             row 2c+1 is up channel c
 *   dn_codes  [d rows, f cols] packed codes
 *   gu_scales [2f rows, d/32] fp16 (raw bits), one scale per 32 weights
 *   dn_scales [d rows, f/32] fp16
 *   Each section starts on a 256-byte boundary. A weight is
 *   w = scale * (q - 2^(bits-1)), q in [0, 2^bits). Blocks of 32 run along the
 *   reduction (column) axis. 2-bit rows: code c in byte c/4 at bits 2*(c%4).
 *   3-bit rows: that 2-bit plane for the low bits (cols/4 bytes) followed by a
 *   1-bit plane (cols/8 bytes) with the high bit of code c at bit c%8 of byte
 *   c/8. The pages name Q2_0 and the IQ2/IQ3 formats but print none of their
 *   bits; this format costs 2.5 / 3.5 bits per weight, the IQ2_XS / IQ3_S rows
 *   of the pages' quantisation table.
 *
 * Expert pool: expert e of a layer lives at slot_pool + slot_of[e]*slot_stride
 * (the slot table stands for the pages' hot-expert cache; on one B200 every
 * expert is in HBM and the table is only an indirection). slot_of[e] = -1
 * (MOE_SLOT_ABSENT) marks an expert this device does not hold: its pairs are
 * left out of the grouping (pair_pos = -1) and add nothing to y. This is how
 * an expert-parallel step splits a layer over devices (each device holds a
 * subset of the experts and produces a partial y; the partials are summed).
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef int moe_status;
#define MOE_OK            0
#define MOE_EINVAL        1  /* bad shape, NULL pointer, misalignment, k > E, k > 32 */
#define MOE_EUNSUPPORTED  2  /* bits not in {2,3}, block != 32, shape outside the kernels' range */
#define MOE_ECUDA         3  /* a CUDA runtime call or kernel launch failed */
#define MOE_ETIMEOUT      4  /* a bounded device-side wait gave up (read by moe_check_device_status) */
#define MOE_EDEVICE       5  /* a kernel found a bad index (expert >= E, slot >= n_slots) */
#define MOE_ENOSPACE      6  /* workspace smaller than moe_workspace_bytes() */

typedef struct moe_ctx moe_ctx;
typedef void* moe_stream; /* cudaStream_t */

/* Slot-table value of an expert this device does not hold. */
#define MOE_SLOT_ABSENT (-1)

/* Largest T that takes the decode path (weight streaming, fused combine). */
#define MOE_DECODE_MAX_T 8

typedef struct {
  int d;         /* hidden size (multiple of 128) */
  int f;         /* expert intermediate size (multiple of 64) */
  int E;         /* routed experts per layer, 1..1024 */
  int k;         /* experts per token, 1..min(E, 32) */
  int n_shared;  /* 0 or 1 shared expert */
  int bits;      /* 2 or 3 */
  int block;     /* weights per scale; must be 32 */
  int renorm;    /* 1: gates = softmax over the k chosen logits; 0: full softmax read at them */
  int out_fp32;  /* 1: y is fp32; 0: y is bf16 (round to nearest even) */
  int residual;  /* 1: y = x + moe(x) */
  /* Skipping low-ranked experts that are not resident (the pages' engine, on
   * NVIDIA GPUs, by default leaves out low-ranked experts that are not in GPU
   * memory and documents the small output change: news.blueqat.app/post/3262,
   * section どう見るか). skip_from = 0: off. Else, in the fused decode calls
   * (moe_layer_forward with T <= MOE_DECODE_MAX_T and E <= 512,
   * moe_stack_forward), the pair of rank j >= skip_from of a token whose
   * expert's slot is >= hot_slots is left out: it adds nothing to y, the
   * other gates keep their values (no renormalisation), and an expert left
   * with no pair is not read at all. The routing views then group the kept
   * pairs only (uniq_offset[n_uniq] = their number; pair_pos = -1 for a pair
   * left out). Other paths reject skip_from != 0 with MOE_EUNSUPPORTED. */
  int skip_from; /* 0..k */
  int hot_slots; /* slots [0, hot_slots) count as resident */
} moe_layer_cfg;

typedef struct {
  size_t gu_codes, dn_codes, gu_scales, dn_scales; /* byte offsets inside a record */
  size_t bytes;                                    /* record size, a multiple of 256 */
} moe_expert_layout;

/* Token grouping: device pointers into the caller's workspace, filled by
 * moe_group_tokens. Sorted order is (expert, token, j); the shared expert's
 * rows follow the routed pairs, token t at row n_pairs + t. */
typedef struct {
  int T, k, E;
  int n_pairs;            /* T*k */
  int n_rows;             /* n_pairs + T*n_shared */
  int32_t* expert_count;  /* [E]    pairs per expert */
  int32_t* expert_offset; /* [E+1]  exclusive prefix sum of expert_count */
  int32_t* pair_token;    /* [n_pairs] token of each sorted pair */
  int32_t* pair_j;        /* [n_pairs] rank j of the pair in its token's top-k */
  float*   pair_gate;     /* [n_pairs] gate of the pair */
  int32_t* pair_slot;     /* [n_pairs] pool slot of the pair's expert */
  int32_t* pair_pos;      /* [T*k]  sorted position of pair (t, j) at t*k + j */
  int32_t* uniq_expert;   /* [min(E, n_pairs)] experts with >= 1 pair, ascending */
  int32_t* uniq_slot;     /* [min(E, n_pairs)] their pool slots */
  int32_t* uniq_offset;   /* [min(E, n_pairs) + 1] first sorted pair of each */
  int32_t* n_uniq;        /* [1] number of such experts */
  void*    internal;      /* library-private scratch (tile lists, histograms) */
} moe_grouping;

/* ---- context ------------------------------------------------------------ */

/* Creates a context on CUDA device `device`: queries the SM count, allocates
 * the 16-byte device status word (the only device allocation the library
 * makes) and sets kernel attributes. Every later call with this context
 * launches on that device. Call outside stream capture. */
MOE_API moe_status moe_ctx_create(int device, moe_ctx** out);
MOE_API void moe_ctx_destroy(moe_ctx* ctx);
MOE_API const char* moe_status_string(moe_status s);

/* Text of the last CUDA runtime error a call on this host thread turned into
 * MOE_ECUDA ("no error" if none). Diagnostic only. */
MOE_API const char* moe_last_cuda_error(void);

/* Synchronises `stream`, reads and clears the device status word. Returns
 * MOE_OK, MOE_EDEVICE (bad expert or slot index seen by a kernel) or
 * MOE_ETIMEOUT (a bounded wait ran out). */
MOE_API moe_status moe_check_device_status(moe_ctx* ctx, moe_stream stream);

/* Diagnostics: the detail word a kernel recorded with the last device error
 * that moe_check_device_status returned (for MOE_ETIMEOUT, the wait that gave
 * up; for MOE_EDEVICE, the pair or expert index), 0 if none. */
MOE_API int moe_last_device_error_detail(const moe_ctx* ctx);

/* Diagnostics: when the environment variable MOE_TRACE is set at context
 * creation, the decode kernel records the global-timer value (ns) at its
 * phase boundaries, 64 slots per CTA. This copies up to n values (CTA
 * major) into host memory, synchronising `stream`, and clears the record.
 * Returns MOE_EINVAL if tracing is off. */
MOE_API moe_status moe_trace_fetch(moe_ctx* ctx, unsigned long long* host, int n, moe_stream stream);

/* ---- sizes -------------------------------------------------------------- */

/* Layout of one expert record for cfg (see the header comment). */
MOE_API moe_status moe_expert_layout_get(const moe_layer_cfg* cfg, moe_expert_layout* out);

/* Bytes of workspace every call below needs for T tokens (0 if cfg is invalid). */
MOE_API size_t moe_workspace_bytes(const moe_layer_cfg* cfg, int T);

/* ---- steps -------------------------------------------------------------- */

/* Router + top-k. x: [T, d] bf16 row-major (16-byte aligned); w_router: [E, d]
 * fp32 row-major; logit_bias: NULL or [T, E] fp32 added to the logits;
 * logits (out): [T, E] fp32; idx (out): [T, k] int32 in descending-logit
 * order; gate (out): [T, k] fp32. The router runs for every token on the GPU
 * (news.blueqat.app/post/3262, section GPU・CPU・RAM・SSDの分担). T = 0 is a
 * no-op. */
MOE_API moe_status moe_router_topk(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x,
                           const float* w_router, const float* logit_bias, int T,
                           float* logits, int32_t* idx, float* gate, moe_stream stream);

/* Top-k and gates from given fp32 logits [T, E] (the selection step alone):
 * each token keeps the k largest of its E logits, 10 of 512 at full size
 * (news.blueqat.app/post/3262, first section Strataとは; geekoyaji.com
 * "freetoken-vs-strata-moe-offload", section 共通の仕組み). Ties go to the
 * lower expert index; NaN ranks below every number. idx [T, k] int32 in
 * descending-logit order, gate [T, k] fp32 (softmax over the k chosen, or the
 * full softmax when cfg->renorm == 0). T = 0 is a no-op. */
MOE_API moe_status moe_topk(moe_ctx* ctx, const moe_layer_cfg* cfg, const float* logits, int T,
                    int32_t* idx, float* gate, moe_stream stream);

/* Stable counting sort of the T*k pairs by expert, without atomics, and the
 * slot lookup slot = slot_of[e]. idx, gate: [T, k] from moe_topk; slot_of:
 * [E] int32 (this layer's slice of the slot table); n_slots bounds the slots
 * (a slot >= n_slots is reported as MOE_EDEVICE). Fills *out with views into
 * ws. The slot table stands for the pages' hot-expert cache (vramglass.com,
 * section その1：よく使うエキスパートを選んでGPUに置く). */
MOE_API moe_status moe_group_tokens(moe_ctx* ctx, const moe_layer_cfg* cfg, const int32_t* idx,
                            const float* gate, int T, const int32_t* slot_of, int n_slots,
                            void* ws, size_t ws_bytes, moe_grouping* out, moe_stream stream);

/* Expert FFN over 2-bit (q2) or 3-bit (q3) records: for every sorted pair and
 * every shared-expert row, h = silu(W_g x) * (W_u x) and z = W_d h, with the
 * weights dequantised inside the kernels. The pages put the experts at 2 to
 * 3 bits per weight (news.blueqat.app/post/3262, section 量子化の種類とサイズ)
 * and run the shared expert on the GPU for every token (same page, section
 * GPU・CPU・RAM・SSDの分担); the SwiGLU form is the one the pages' model family
 * uses and is not printed there.
 * slot_pool: base of the pool (256-byte aligned), slot_stride: bytes between
 * slots (a multiple of 256, >= the record size); shared_expert: one record or
 * NULL when cfg->n_shared == 0; ws: the workspace the grouping came from.
 *   z_rows == NULL: decode path (T <= MOE_DECODE_MAX_T). The combine is fused:
 *       y [T, d] (fp32 or bf16 per cfg->out_fp32) is written directly.
 *   z_rows != NULL: z_rows [n_rows, d] fp32 receives gate * z for each sorted
 *       pair and z for each shared row; y is not touched (pass NULL) and
 *       moe_combine finishes the step. Any T. */
MOE_API moe_status moe_expert_ffn_q2(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x,
                             const moe_grouping* grouping, const uint8_t* slot_pool,
                             size_t slot_stride, const uint8_t* shared_expert, void* ws,
                             size_t ws_bytes, float* z_rows, void* y, moe_stream stream);
MOE_API moe_status moe_expert_ffn_q3(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x,
                             const moe_grouping* grouping, const uint8_t* slot_pool,
                             size_t slot_stride, const uint8_t* shared_expert, void* ws,
                             size_t ws_bytes, float* z_rows, void* y, moe_stream stream);

/* y[t] = sum_j z_rows[pair_pos[t,j]] (j ascending) + z_rows[n_pairs + t]
 * (+ x[t] when cfg->residual), written as fp32 or bf16. x may be NULL unless
 * residual. This is the pages' per-layer join of the routed experts' results
 * (vramglass.com, section その2：GPUとCPUで同時に計算する). */
MOE_API moe_status moe_combine(moe_ctx* ctx, const moe_layer_cfg* cfg, const moe_grouping* grouping,
                       const float* z_rows, const void* x, int T, void* y, moe_stream stream);

/* The whole step: router -> top-k -> grouping -> experts -> combine, the
 * per-layer expert step of the pages' engine (news.blueqat.app/post/3262,
 * sections Strataとは and GPU・CPU・RAM・SSDの分担). Picks the decode path for
 * T <= MOE_DECODE_MAX_T (decode passes of up to 4 tokens: vramglass.com,
 * section その3) and the tensor-core grouped GEMM path otherwise (prefill
 * chunks of up to 8,192 tokens: news.blueqat.app, section
 * GPU・CPU・RAM・SSDの分担). Arguments as above; ws must hold
 * moe_workspace_bytes(cfg, T). */
MOE_API moe_status moe_layer_forward(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x, int T,
                             const float* w_router, const float* logit_bias,
                             const int32_t* slot_of, int n_slots, const uint8_t* slot_pool,
                             size_t slot_stride, const uint8_t* shared_expert, void* ws,
                             size_t ws_bytes, void* y, moe_stream stream);

/* The routing a whole-step call computed, as views into its workspace.
 * After moe_layer_forward(cfg, T, ws) has completed on its stream, the
 * workspace holds that step's router logits, top-k and grouping; this fills
 * *out with device pointers to them (no device work, no synchronisation):
 *   logits [T, E] fp32 (router output plus bias), idx [T, k] int32 and
 *   gate [T, k] fp32 (as moe_router_topk), grouping (as moe_group_tokens).
 * The same views serve moe_router_topk / moe_group_tokens callers that pass
 * this workspace. A later call with the same workspace overwrites them.
 * This is the per-token expert choice the pages' engine logs and tallies to
 * pick its hot experts (vramglass.com, section その1). */
typedef struct {
  int T, k, E;
  float* logits;
  int32_t* idx;
  float* gate;
  moe_grouping grouping;
} moe_routing;
MOE_API moe_status moe_layer_routing(const moe_layer_cfg* cfg, int T, void* ws, size_t ws_bytes,
                                     moe_routing* out);

/* ---- the decode stack ----------------------------------------------------- */

/* L consecutive layers of the decode path in one launch: layer 0 reads x,
 * layer l + 1 reads layer l's output y[l] (a model's MoE layers in a row, with
 * the per-layer join of the pages' engine between them: vramglass.com,
 * section その2). Per layer the same step as moe_layer_forward (router,
 * top-k, grouping, experts, combine; with cfg->residual, y[l] = x_l + moe(x_l)).
 * While layer l runs, layer l + 1's router columns and shared expert, which
 * do not depend on x, are already being fetched, and layer l + 1's logits are
 * summed from every CTA's rows of y[l] as they are written (exact fixed-point
 * partial sums, so the logits do not depend on the order of the adds).
 *   - T: 1..MOE_DECODE_MAX_T tokens; cfg->E <= 512; L >= 1.
 *   - w_router: [L, E, d] fp32; logit_bias: NULL or [L, T, E] fp32;
 *     slot_of: [L, E] int32 (the stack's slot table, one row per layer);
 *     slot_pool / slot_stride: the pool as for moe_layer_forward;
 *     shared_experts: layer l's shared expert record at
 *     shared_experts + l * slot_stride (NULL when cfg->n_shared == 0).
 *   - y: [L, T, d]; bf16 (cfg->out_fp32 must be 0 when L > 1, since the
 *     next layer reads it as its bf16 input).
 *   - ws: moe_stack_workspace_bytes(cfg, L, T) bytes, 256-byte aligned.
 *     After the call has completed, layer l's routing is readable through
 *     moe_stack_routing. Nothing in it needs to start at zero.
 * The kernel is a cooperative launch of one CTA per SM whose CTAs exchange
 * data while they run: the launch waits until every SM is free, and calls on
 * one device must not overlap in time (issue them on one stream, or order
 * them with events). Same status and error conventions as every call. */
MOE_API size_t moe_stack_workspace_bytes(const moe_layer_cfg* cfg, int L, int T);
MOE_API moe_status moe_stack_forward(moe_ctx* ctx, const moe_layer_cfg* cfg, int L, const void* x, int T,
                                     const float* w_router, const float* logit_bias, const int32_t* slot_of,
                                     int n_slots, const uint8_t* slot_pool, size_t slot_stride,
                                     const uint8_t* shared_experts, void* ws, size_t ws_bytes, void* y,
                                     moe_stream stream);
/* Views of layer `layer`'s routing inside a stack workspace (as
 * moe_layer_routing). */
MOE_API moe_status moe_stack_routing(const moe_layer_cfg* cfg, int L, int T, void* ws, size_t ws_bytes,
                                     int layer, moe_routing* out);

/* ---- expert residency --------------------------------------------------- */

/* The pages' engine keeps its most used experts in GPU memory, picked from
 * usage statistics and swapped as a conversation goes on (vramglass.com,
 * section その1：よく使うエキスパートを選んでGPUに置く; news.blueqat.app/post/3262,
 * section GPU・CPU・RAM・SSDの分担). Here the pool's first slots stand for that
 * hot set; these two calls tally usage and move records between slots.
 *
 * moe_usage_count: counts[l * E + e] += the number of (token, j) pairs routed
 * to expert e in layer l by the call whose workspace is ws, once that call
 * has completed on `stream`'s order: L = 1 for a moe_layer_forward (or
 * moe_router_topk + moe_group_tokens) workspace at T tokens, L layers for a
 * moe_stack_forward workspace (T <= MOE_DECODE_MAX_T). counts: [L, E] int32
 * device array; integer adds in a fixed owner per element, so the tallies are
 * exact and deterministic.
 *
 * moe_slot_swap: for i < n, the records at slots slot_of[a[i]] and
 * slot_of[b[i]] trade places in the pool and the two slot-table entries trade
 * values, so every entry still names its own expert's record and later calls
 * give the same results bit for bit. a, b: HOST arrays of n indices into the
 * device slot table slot_of (n_entries entries, e.g. L * E); the 2n indices
 * must be distinct and in range (MOE_EINVAL otherwise), and the slots they
 * name distinct as well (true when no two entries share a slot, as in a pool
 * with one record per layer and expert; not checked). A slot outside
 * [0, n_slots) found on the device is reported as MOE_EDEVICE and that pair is
 * left alone. Calls that read the pool or the table must be ordered after this
 * one (same stream). */
MOE_API moe_status moe_usage_count(moe_ctx* ctx, const moe_layer_cfg* cfg, int L, int T, const void* ws,
                                   size_t ws_bytes, int32_t* counts, moe_stream stream);
MOE_API moe_status moe_slot_swap(moe_ctx* ctx, const moe_layer_cfg* cfg, uint8_t* slot_pool, size_t slot_stride,
                                 int32_t* slot_of, int n_entries, int n_slots, const int32_t* a, const int32_t* b,
                                 int n, moe_stream stream);

/* moe_layer_forward without a workspace argument: the step's scratch is a
 * static device array of MOE_STATIC_SCRATCH_BYTES inside the library image,
 * reserved on each device when the library's module loads there, so the call
 * allocates nothing. The pages have no counterpart; this serves callers that
 * own no device allocator (a plain C host linking only this library) and
 * decode loops that must not call cudaMalloc, which can synchronise the
 * device.
 *   - Arguments and results as moe_layer_forward, minus ws / ws_bytes.
 *   - Limit: moe_workspace_bytes(cfg, T) must be <= MOE_STATIC_SCRATCH_BYTES,
 *     else MOE_ENOSPACE and nothing runs. The full-size layer (d=2048,
 *     f=768, E=512, k=10) needs about 2.7 MB at T = 8, so every decode
 *     batch fits; at that size prefill chunks above about two dozen tokens
 *     do not.
 *   - Nothing in the scratch needs to start at zero.
 *   - There is ONE scratch per device, shared by every context and stream:
 *     calls that overlap in time on one device (two streams, two host
 *     threads) race on it and give wrong results. Serialise them, e.g. on
 *     one stream.
 *   - The first call on a device does a one-time set-up (it looks up the
 *     array's device address with that device current); make that first
 *     call before any stream capture begins. */
#define MOE_STATIC_SCRATCH_BYTES (4u << 20)
MOE_API moe_status moe_layer_forward_static(moe_ctx* ctx, const moe_layer_cfg* cfg, const void* x, int T,
                                    const float* w_router, const float* logit_bias,
                                    const int32_t* slot_of, int n_slots, const uint8_t* slot_pool,
                                    size_t slot_stride, const uint8_t* shared_expert, void* y,
                                    moe_stream stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H_ */
