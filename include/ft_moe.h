/*
 * ft_moe.h — C ABI of a routed Mixture-of-Experts FFN layer that runs over an
 * HBM expert-slot cache in front of a pinned-host expert pool, on one B200.
 *
 * Sources. The method is described only by web pages about the FreeToken
 * edge-MoE serving system (arXiv 2608.16157). Citations below name the page by
 * its title and the section on it:
 *   [paperlens]  "論文解説: FreeToken — 手元のPCを「一台の推論基盤」として使い切る
 *                帯域適応型MoEサービング" (ta-paperlens digest of the paper)
 *   [techfeed]   techfeed recap of "Meet FreeToken: An Edge-Native MoE Serving
 *                Engine that Runs 753B GLM-5.2 on a Single Workstation GPU"
 *   [leadeas]    "FreeToken ― コンシューマGPUで大規模MoEモデルをローカル高速推論する
 *                エンジン" (leadeas.co.jp)
 *   [wiki]       "FreeToken：エッジネイティブMoEセットアップガイドと比較"
 *   [ainew]      "UC バークレーと MIT、MoE モデルを一般ハードウェアで動かす推論エンジン
 *                「FreeToken」公開"
 *
 * What one layer call computes (the result never depends on where a weight
 * was read from: [paperlens] 設計: 2階建てのエキスパート記憶, paper §3.3; the
 * partial sums are added with no change to routing, [techfeed]
 * 帯域適応型実行（q*ポリシー）):
 *   s[t,e]  = sum_i x[t,i] * W_r[e,i] + b[e]            router logits, fp32
 *   ids[t,:] = the k largest s[t,.], descending; equal scores -> lower e first
 *   w[t,j]  = exp(s[t,ids_j] - max) / sum_j' exp(...)    softmax over the k chosen
 *   for each chosen expert e of token t (rank j):
 *     g = W_gate[e] x_t, u = W_up[e] x_t                 [d_ff]
 *     h = g * sigmoid(g) * u                             SwiGLU
 *     Y_j = W_down[e] h                                  [d]
 *   y[t] = sum_{j=0..k-1} w[t,j] * Y_j                   fixed rank order, fp32
 * (E experts per layer, k << E per token: [paperlens] MoEは扉を開けると同時に、
 * 別の扉を閉める, paper §1.)
 *
 * Expert memory ([paperlens] 設計: 2階建てのエキスパート記憶, paper §3; [leadeas]
 * VRAMをキャッシュとして使う): every (layer, expert) weight blob lives in a pinned,
 * device-mapped host pool owned by the context (the source of truth). HBM holds
 * C slots, one blob per slot, shared by all layers under one LRU ([techfeed]
 * セマンティック認識キャッシング). On a decode step with m missed experts,
 * q* = round(m * B_P / B_H) of them are copied into slots by the copy engine
 * and the other m - q* are read by the expert kernel straight from the mapped
 * host pool ([techfeed] 帯域適応型実行（q*ポリシー）; on this GPU there is no CPU
 * compute leg). A prefill call loads every expert of the next layer while the
 * current one computes ([paperlens] プレフィル: 全層ダブルバッファと「意味の錨」,
 * paper §3.1).
 *
 * Conventions for every entry point:
 *   - Returns ft_status; nothing throws across the ABI.
 *   - "device pointer" arguments are CUDA device addresses on cfg.device, owned
 *     by the caller, which must keep them alive until the work on the compute
 *     stream that reads or writes them has finished.
 *   - Work is enqueued on the compute stream given to ft_moe_init. Calls that
 *     return host data (ft_cache_stats, ft_moe_last_*) synchronise both streams.
 *   - A device-side failure (a bounded wait that ran out, a bad index caught by
 *     a kernel) latches an error word; the next call returns FT_ETIMEOUT or
 *     FT_ESTATE and ft_cache_stats reports it in device_error.
 *   - One context per host thread; calls on one context are not thread safe.
 */
#ifndef FT_MOE_H
#define FT_MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ft_ctx ft_ctx; /* opaque; owned by the library */

typedef enum {
  FT_OK = 0,
  FT_EINVAL = 1,       /* an argument is out of range or a pointer is NULL */
  FT_ENOMEM = 2,       /* pinned-host or device allocation failed */
  FT_ECUDA = 3,        /* a CUDA runtime call failed */
  FT_ETIMEOUT = 4,     /* a bounded wait (host or device) gave up */
  FT_ESTATE = 5,       /* call out of order (e.g. no router set) or latched device error */
  FT_EUNSUPPORTED = 6  /* valid request this library does not implement */
} ft_status;

/* Expert weight format. F32 implies fp32 activations (x, y, W_r); BF16 and
 * NVFP4 imply bf16 activations. */
typedef enum { FT_W_F32 = 0, FT_W_BF16 = 1, FT_W_NVFP4 = 2 } ft_wtype;

/* Decode: look up the routed experts of this layer (hit / staged / streamed).
 * Prefill: the whole layer is resident before it computes and the next layer
 * is loaded behind it (needs cache_slots >= 2E; with fewer slots a prefill
 * call follows the decode rules for its routed experts, the on-demand
 * fallback of [paperlens] プレフィル: 全層ダブルバッファと「意味の錨」). */
typedef enum { FT_DECODE = 0, FT_PREFILL = 1 } ft_mode;

typedef struct {
  int32_t n_layers;    /* L >= 1 */
  int32_t n_experts;   /* E, 1..512 */
  int32_t top_k;       /* k, 1..min(E, 16) */
  int32_t d_model;     /* d, multiple of 64, <= 16384 */
  int32_t d_ff;        /* d_ff, multiple of 64, <= 16384 */
  int32_t wtype;       /* ft_wtype */
  int64_t cache_slots; /* C, 0..max(L*E, 2E) HBM slots of ft_moe_slot_bytes() each */
  int32_t max_tokens;  /* T upper bound of one forward, 1..65536 */
  int32_t device;      /* CUDA device ordinal */
} ft_config;

/* Slot blob layout: one contiguous blob per (layer, expert), the unit of every
 * cache slot and host-pool entry ("one slot holds every tensor one (layer,
 * expert) pair needs": [paperlens] 設計: 2階建てのエキスパート記憶).
 * Matrices are row-major, rows = output features, the reduction axis K
 * contiguous:
 *   W_gate [d_ff][d], W_up [d_ff][d], W_down [d][d_ff]
 * FT_W_F32 / FT_W_BF16: the three matrices back to back, fp32 / bf16 elements.
 *   bytes = 3*d*d_ff*elem
 * FT_W_NVFP4: all codes, then all block scales:
 *   [gate codes d_ff*d/2][up codes d_ff*d/2][down codes d*d_ff/2]
 *   [gate scales d_ff*d/16][up scales d_ff*d/16][down scales d*d_ff/16]
 *   Element (r, c) of a matrix with K columns is the 4-bit e2m1 code in byte
 *   r*K/2 + c/2: low nibble for even c, high nibble for odd c. Its scale is the
 *   e4m3 byte r*K/16 + c/16 of that matrix's scale array (16-element blocks
 *   along K). Value = e2m1(code) * e4m3(scale) * tensor_scale[matrix], the
 *   per-matrix fp32 tensor scale set with ft_moe_set_tensor_scales.
 *   e2m1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0:
 *         magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6.
 *   e4m3: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0,
 *         subnormals at exponent 0, code 0x7F/0xFF is NaN, max 448.
 *   bytes = 3*d*d_ff/2 + 3*d*d_ff/16
 */
ft_status ft_moe_slot_bytes(const ft_config* cfg, uint64_t* out_bytes);

/* Create a context: validates cfg, allocates the pinned mapped host pool
 * (L*E blobs, contents undefined until filled), C HBM slots, the device LRU
 * table (empty: every expert starts on the host, a cold cache as in
 * [techfeed] 弾性メモリ管理), scratch for max_tokens, and a mapped mailbox.
 * compute_stream / copy_stream are cudaStream_t handles owned by the caller
 * (0 for compute selects the legacy default stream; copy_stream must be a
 * distinct non-default stream). Bandwidths start at B_P = B_H (q* = m).
 * On failure *out is NULL and nothing is leaked. */
ft_status ft_moe_init(const ft_config* cfg, void* compute_stream, void* copy_stream, ft_ctx** out);

/* Free everything the context owns. Synchronises its streams first. NULL ok. */
void ft_moe_destroy(ft_ctx* ctx);

/* Host pointer to the pinned pool blob of (layer, expert), ft_moe_slot_bytes()
 * long, for the caller to fill in the layout above. The pool is the source of
 * truth: writing a blob after it was cached requires ft_moe_reset_cache. */
ft_status ft_moe_expert_ptr(ft_ctx* ctx, int32_t layer, int32_t expert, void** host_blob);

/* NVFP4 only: the fp32 tensor scales (gate, up, down) of (layer, expert).
 * scales is a host array of 3 floats, copied. */
ft_status ft_moe_set_tensor_scales(ft_ctx* ctx, int32_t layer, int32_t expert, const float* scales);

/* Router weights of a layer: device pointer to W_r [E][d] (fp32 for FT_W_F32,
 * else bf16), row-major. Caller-owned; the pointer is kept, not copied. */
ft_status ft_moe_set_router(ft_ctx* ctx, int32_t layer, const void* w_router_dev);

/* One MoE layer on T tokens, enqueued on the compute stream.
 *   x_dev   [T][d] activations (fp32 or bf16, see ft_wtype), device pointer,
 *             16-byte aligned
 *   bias_dev  NULL, or fp32 device pointer: [E] (bias_per_token = 0) or
 *             [T][E] (bias_per_token = 1), added to the router logits
 *   y_dev   [T][d] output, same type as x, 16-byte aligned; may not alias x
 *   ids_dev_opt [T][k] int32, w_dev_opt [T][k] fp32: optional outputs of the
 *             routing (rank order), NULL to skip
 * T may be 0 (no work, no lookups). In decode mode (or prefill with C < 2E)
 * the call blocks the host until the layer's lookup kernel has run (bounded
 * wait, FT_ETIMEOUT) because the copy engine needs the staged list. */
ft_status ft_moe_layer_forward(ft_ctx* ctx, int32_t layer, int32_t mode, const void* x_dev, int32_t T,
                               const float* bias_dev, int32_t bias_per_token, void* y_dev,
                               int32_t* ids_dev_opt, float* w_dev_opt);

/* ft_moe_layer_forward with the activations in host memory: x_host [T][d]
 * is copied into a device buffer the context owns, the layer runs, and its
 * output is copied back into y_host [T][d], all enqueued on the compute
 * stream in that order (the call returns once the work is enqueued; in
 * decode mode it also waits for the layer's lookup as ft_moe_layer_forward
 * does). Page-locked host buffers make both copies asynchronous; pageable
 * ones make the runtime copy through its own staging. The caller reads y_host
 * after synchronising the compute stream, and keeps x_host unchanged until
 * then. Types, sizes and the other arguments as ft_moe_layer_forward (bias
 * stays a device pointer: it is model data); x_host and y_host may not
 * overlap. T <= max_tokens. */
ft_status ft_moe_layer_forward_host(ft_ctx* ctx, int32_t layer, int32_t mode, const void* x_host, int32_t T,
                                    const float* bias_dev, int32_t bias_per_token, void* y_host);

/* Expert outputs of rows that are already routed: the owner's half of an
 * expert-parallel layer, where G devices split the E experts of every layer
 * in G contiguous blocks and each device runs only the experts it owns on the
 * rows other devices send it (see ft_ep_pack). The pages serve one GPU; in a
 * datacenter a fast interconnect hides the moves between devices ([ainew]
 * "UC バークレーと MIT、MoE モデルを一般ハードウェアで動かす推論エンジン
 * 「FreeToken」公開", opening paragraph), and here each device's misses go over
 * its own host link.
 *
 * The context is this device's: its n_experts are the experts it owns, local
 * ids 0..n_experts-1, with their pool, slots and LRU. Row i goes through expert
 * eids_dev[i] - expert_base with weight 1, exactly as a token routed to that
 * expert alone: the same lookup, q* split, staging and expert kernels as
 * ft_moe_layer_forward with top_k = 1 (mode FT_DECODE or FT_PREFILL), and no
 * router.
 *   rows_dev  [n][d] activations (fp32 for FT_W_F32, else bf16), 16-byte aligned
 *   eids_dev  [n] int32 global expert ids, device pointer
 *   expert_base  global id of local expert 0
 *   out_dev   [n][d] fp32 expert outputs in row order (unrounded, so that the
 *             source device's combine rounds once), 16-byte aligned
 * n may be 0; n <= max_tokens (FT_EINVAL otherwise). An id outside
 * [expert_base, expert_base + n_experts) latches a device error (FT_ESTATE
 * on the next call) and that row is computed with local expert 0. */
ft_status ft_moe_expert_rows(ft_ctx* ctx, int32_t layer, int32_t mode, const void* rows_dev,
                             const int32_t* eids_dev, int32_t expert_base, int32_t n, float* out_dev);

/* Counters since init (or the last ft_moe_reset_cache). Synchronises. */
typedef struct {
  uint64_t layer_calls;     /* forward calls with T > 0 */
  uint64_t lookups;         /* unique (layer, expert) lookups */
  uint64_t hits;
  uint64_t misses;
  uint64_t staged;          /* misses copied into a slot (copy engine) */
  uint64_t streamed;        /* misses read from the host pool by the kernel */
  uint64_t bytes_h2d;       /* copy-engine bytes */
  uint64_t bytes_zero_copy; /* weight bytes kernels read from host memory */
  int32_t last_m;           /* misses of the last lookup batch */
  int32_t last_qstar;       /* q* of the last decode batch (before the capacity clamp) */
  int32_t last_qstage;      /* misses actually staged in that batch */
  int32_t device_error;     /* 0, or the latched ft_status of a device failure */
  uint64_t kernel_launches; /* CUDA kernels this context launched */
  uint64_t prefetched;      /* blobs staged by the decode prefetch (ft_moe_set_prefetch) */
  /* Device time, from CUDA events the context records on its own streams
   * around every layer call: ms_compute sums each call's span on the compute
   * stream (first launch to the combine, the streamed class's side stream
   * joined in), ms_copy each call's span of copy-engine staging on the copy
   * stream (the staged misses and the prefill layer-ahead loads). Where
   * ms_copy is close to ms_compute the copies ran hidden behind compute. */
  double ms_compute;
  double ms_copy;
} ft_stats;
ft_status ft_cache_stats(ft_ctx* ctx, ft_stats* out);

/* The q* split inputs, in MB/s: B_P (host-to-GPU link share) and B_H (host
 * memory bandwidth), as profiled by `ft bench bw` in [techfeed]
 * 帯域適応型実行（q*ポリシー） (e.g. 52.7:77.3 GB/s). Used from the next forward.
 * 0 < bh; bp may be 0 (nothing staged) or >= bh (everything staged). */
ft_status ft_set_bandwidths(ft_ctx* ctx, uint32_t bp_mbps, uint32_t bh_mbps);

/* Empty the cache and zero the counters (cold start). Synchronises. */
ft_status ft_moe_reset_cache(ft_ctx* ctx);

/* Predictive prefetch for decode, off by default. When on, every decode call
 * of layer l, right after its lookup, stages into slots the experts that layer
 * (l+1) mod L was routed to in its own last decode call and that are not
 * resident: ascending expert id, each inserted like a staged miss (a fresh LRU
 * stamp), evicting nothing that layer l's lookup touched or inserted, and as
 * many as unpinned slots allow; resident ones are left untouched. The copies
 * go out on the copy stream behind layer l's staged copies, so they overlap
 * layer l's compute; the next call's experts read from those slots wait for
 * them. Lookup counters are unchanged (the next layer's lookup then sees hits);
 * ft_stats.prefetched counts the blobs. Only decode calls record their routing
 * and prefetch; ft_moe_reset_cache and ft_moe_resize_cache clear the record.
 * This extends the layer-ahead loading of prefill ([paperlens] プレフィル:
 * 全層ダブルバッファと「意味の錨」, paper §3.1) to decode, predicting the next
 * layer from its previous step; the pages give no decode prefetch policy.
 * enable: 0 off, non-zero on. Errors: FT_EINVAL (NULL ctx). */
ft_status ft_moe_set_prefetch(ft_ctx* ctx, int32_t enable);

/* Grow or shrink the HBM slot pool to new_slots at a safe point, without
 * touching the host pool: the elastic memory manager of [techfeed]
 * 弾性メモリ管理, which may hand expert-slot memory to the KV cache and take
 * it back because what the cache holds never changes a result.
 *   new_slots: 0 .. max(L*E, 2E), like ft_config.cache_slots.
 * Rule: the min(new_slots, resident) most recently used entries survive with
 * their stamps; a survivor whose slot index is below new_slots keeps its
 * slot, the others move, in ascending order of their old slot, to the lowest
 * free slots below new_slots; the LRU clock and the counters are kept; the
 * prefill layer-ahead state is cleared (the next prefill call looks its own
 * layer up again). Synchronises every stream of the context, allocates the
 * new pool, copies the survivors device-to-device, then frees the old pool,
 * so both pools exist for a moment.
 * Errors: FT_EINVAL (range), FT_ENOMEM (the new pool or tables could not be
 * allocated: the context is unchanged), FT_ESTATE / FT_ETIMEOUT (a device
 * error is latched: nothing is done). */
ft_status ft_moe_resize_cache(ft_ctx* ctx, int64_t new_slots);

/* Routing and lookup record of the last forward call, copied to host arrays
 * (synchronises). Any pointer may be NULL.
 *   counts [E], offsets [E+1]: tokens per expert and their exclusive scan
 *   perm [T*k]: sorted position -> flat index t*k+j, ordered by expert then
 *               token (stable); inv [T*k]: flat index -> sorted position
 *   lookup_e [E], lookup_kind [E]: the looked-up experts in lookup order and
 *               their outcome (0 hit, 1 staged, 2 streamed); n_lookup of them.
 *               A prefill call lists its prefetch of the next layer in the
 *               second part, with lookup_kind 0 / 1 and layer+1 implied.
 *   n_lookup_cur: how many of them belong to this layer (rest: next layer)
 *   m, qstar, qstage: of this layer's batch (qstar = -1 for prefill loads)
 */
ft_status ft_moe_last_route(ft_ctx* ctx, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                            int32_t* lookup_e, int32_t* lookup_kind, int32_t* n_lookup, int32_t* n_lookup_cur,
                            int32_t* m, int32_t* qstar, int32_t* qstage);

/* Cache contents (synchronises): key_of [C] = layer*E+expert or -1 for a free
 * slot, stamp [C] = last-use stamp (0 when free). Either may be NULL. */
ft_status ft_moe_cache_contents(ft_ctx* ctx, int32_t* key_of, uint64_t* stamp);

/* Host-link probe (the B200 stand-in for `ft bench bw`, [techfeed]
 * 帯域適応型実行（q*ポリシー）): copy-engine H2D GB/s of `bytes` from the pinned
 * pool into HBM, and GB/s of a kernel reading the same bytes zero-copy from
 * the mapped pool. Synchronises. bytes <= pool size, multiple of 4096. */
ft_status ft_moe_probe_link(ft_ctx* ctx, uint64_t bytes, double* h2d_gbs, double* zero_copy_gbs);

/* Per-kernel timing. While enabled, every kernel launch (and each group of
 * staging copies) is bracketed by CUDA events on the stream it runs on, and
 * tagged with its algorithmic bytes and flops (each weight read once plus
 * activations in and out). This adds two event records per launch. */
ft_status ft_moe_profile(ft_ctx* ctx, int32_t enable);

typedef struct {
  char name[32];        /* kernel, e.g. "gemv_gateup_hit" */
  uint64_t launches;
  double ms;            /* summed event time of those launches */
  double bytes;         /* summed algorithmic bytes */
  double flops;         /* summed algorithmic flops */
} ft_kernel_time;

/* Fold finished records into per-kernel totals (synchronises) and copy up to
 * cap of them to out; *n_out = number of kernels with records. reset != 0
 * clears the totals after copying. */
ft_status ft_moe_profile_read(ft_ctx* ctx, ft_kernel_time* out, int32_t cap, int32_t* n_out, int32_t reset);

/* Router logits, top-k and softmax weights of one layer WITHOUT allocating
 * anything: the same kernels as ft_moe_layer_forward's routing, with their
 * logits scratch in a fixed device array compiled into this library.
 *
 * The paper has no counterpart for this entry point. It exists for callers
 * that cannot call cudaMalloc at the point where they route: a serving loop
 * whose memory manager has already handed every free byte of HBM to the KV
 * cache and the expert slots (an allocation would fail or force an eviction),
 * code that must not take the implicit device synchronisation of cudaMalloc /
 * cudaFree in the middle of a decode step, or a host program that forbids
 * allocations outside its own allocator. No context is needed.
 *
 *   x_dev [T][d_model] activations (fp32 when wtype is FT_W_F32, else bf16),
 *   w_router_dev [n_experts][d_model] (same type), both 16-byte aligned;
 *   bias_dev NULL, [n_experts] or [T][n_experts] fp32 (bias_per_token);
 *   ids_dev [T][top_k] int32 and w_dev [T][top_k] fp32 receive the result in
 *   rank order, exactly as ft_moe_layer_forward's ids/weights outputs.
 *   stream: cudaStream_t to enqueue on (0 = legacy default stream).
 * Limits: T <= FT_ROUTE_STATIC_MAX_TOKENS (the scratch holds that many tokens
 * times 512 experts of fp32 logits, 2 MiB, resident on every GPU that loads
 * the library until the process exits); n_experts <= 512, top_k <= 16,
 * d_model a multiple of 64. Larger sizes return FT_EINVAL, nothing is launched.
 * The first call on a device looks up the scratch's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture. It calls no cudaMalloc, cudaFree or allocating routine.
 * All calls share the one scratch array: calls that may overlap on the GPU
 * (different streams without ordering between them) race on it; order them.
 * The scratch needs no clearing: every logit a call reads it wrote first. */
#define FT_ROUTE_STATIC_MAX_TOKENS 1024
ft_status ft_route_topk_static(const void* x_dev, const void* w_router_dev, const float* bias_dev,
                               int32_t bias_per_token, int32_t T, int32_t n_experts, int32_t d_model, int32_t top_k,
                               int32_t wtype, int32_t* ids_dev, float* w_dev, void* stream);

/* Expert parallelism, the two context-free steps around the exchange. G
 * devices split the E experts of every layer in G contiguous blocks (device o
 * owns [o E/G, (o+1) E/G)); each routes its own tokens (ft_route_topk_static),
 * sends every routed row (t, j) to the owner of its expert, gets the expert
 * output back and combines ([ainew] page as for ft_moe_expert_rows).
 *
 * ft_ep_pack orders the T*k routed rows of this device by expert, then by flat
 * index t*k + j (the stable permutation of ft_moe_last_route), so the rows for
 * owner o are one contiguous block and the blocks follow owner order:
 *   ids_dev   [T][top_k] int32 routing ids (rank order), device pointer
 *   x_dev     [T][d_model] activations (fp32 for FT_W_F32, else bf16)
 *   rows_dev  [T*top_k][d_model] out: x[t] for the row at each sorted position
 *   eids_dev  [T*top_k] int32 out: the row's expert
 *   owner_counts_dev [n_owners] int64 out: rows for each owner, in order
 *   inv_dev   [T*top_k] int32 out: flat index t*k+j -> its row's position
 *   bad_ids_dev  NULL, or int32 out: number of ids outside [0, n_experts)
 *             (such ids are treated as expert n_experts - 1)
 *   scratch_dev / scratch_bytes: device scratch of at least
 *             ft_ep_pack_scratch_bytes(T, top_k, n_experts) bytes, 256-byte
 *             aligned, not read before it is written
 *   stream: cudaStream_t to enqueue on (0 = legacy default stream)
 * x, rows 16-byte aligned; n_experts <= 512 and a multiple of n_owners;
 * top_k <= 16; d_model a multiple of 8. Nothing is allocated. */
ft_status ft_ep_pack_scratch_bytes(int32_t T, int32_t top_k, int32_t n_experts, uint64_t* out_bytes);
ft_status ft_ep_pack(const int32_t* ids_dev, int32_t T, int32_t top_k, int32_t n_experts, int32_t n_owners,
                     const void* x_dev, int32_t d_model, int32_t wtype, void* rows_dev, int32_t* eids_dev,
                     int64_t* owner_counts_dev, int32_t* inv_dev, int32_t* bad_ids_dev, void* scratch_dev,
                     uint64_t scratch_bytes, void* stream);

/* y[t] = sum_{j<k} w[t,j] * Y[inv[t*k+j]] in rank order, fp32, one rounding to
 * the activation type: the combine of ft_moe_layer_forward over the expert
 * outputs that came back from the owners, in the order ft_ep_pack sent them.
 *   y_rows_dev [T*top_k][d_model] fp32; w_dev [T][top_k] fp32; inv_dev from
 *   ft_ep_pack (a permutation of 0..T*k-1); y_dev [T][d_model] (fp32 for
 *   FT_W_F32, else bf16). 16-byte aligned; d_model a multiple of 4. */
ft_status ft_ep_combine(const float* y_rows_dev, const float* w_dev, const int32_t* inv_dev, int32_t T,
                        int32_t top_k, int32_t d_model, int32_t wtype, void* y_dev, void* stream);

/* Static string for a status code. */
const char* ft_status_str(ft_status s);

#ifdef __cplusplus
}
#endif
#endif /* FT_MOE_H */
