// Internal declarations shared by the library's translation units: the
// device-side state of a context, the expert work list written by the lookup
// kernel, the host mailbox, and the kernel launchers. Not part of the ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/ft_moe.h"

namespace ft {

// Outcome of one expert lookup. Hit and staged experts are read from their
// HBM slot; streamed experts are read by the expert kernels directly from the
// mapped host pool (the "compute where the weights are" leg of the q* split,
// done by the GPU here).
enum Kind : int32_t { KIND_HIT = 0, KIND_STAGED = 1, KIND_STREAMED = 2 };
constexpr int N_CLASSES = 3;  // work-list classes, indexed by Kind

// Device error codes latched in DevState::error (0 = none).
enum DevError : uint32_t { DERR_NONE = 0, DERR_NO_VICTIM = 1, DERR_BAD_INDEX = 2, DERR_TIMEOUT = 3 };

constexpr int MAX_E = 512;
constexpr int MAX_K = 16;
constexpr int TOK_CHUNK = 8;   // tokens one SIMT GEMV pass carries
constexpr int MMA_CHUNK = 16;  // tokens one tensor-core GEMV unit carries

// One routed expert of the current call, in ascending expert order inside
// its class. tok_off / n_tok index the sorted (perm) order.
struct WorkItem {
  int32_t e;
  int32_t slot;     // HBM slot (hit / staged), -1 when streamed
  int32_t tok_off;  // first sorted position of this expert's tokens
  int32_t n_tok;    // number of tokens routed to it (>= 1)
};

// Per-class compact work lists: items [cls][0..n_items) and, for the GEMV
// kernels, the number of (row block x token chunk) units.
struct WorkLists {
  int32_t n_items[N_CLASSES];
  int32_t pad;
  WorkItem items[N_CLASSES][MAX_E];
};

// Host-visible record of the last lookup batch, written by the lookup kernel
// into mapped pinned memory. The host copy thread reads it after the lookup
// kernel's event completed.
struct Mailbox {
  int32_t reserved;
  int32_t n_copy;     // slots to fill by H2D copy (staged + prefill loads)
  int32_t m, qstar, qstage;
  int32_t n_lookup, n_lookup_cur;
  int32_t n_hit_cls, n_staged_cls, n_streamed_cls;
  uint32_t pad_error;  // copy of the device error word at the end of the lookup
  int32_t n_tok_cls[3];  // tokens routed to the experts of each work class
  int32_t copy_key[2 * MAX_E];   // layer*E + e
  int32_t copy_slot[2 * MAX_E];
  int32_t lookup_e[2 * MAX_E];
  int32_t lookup_kind[2 * MAX_E];
};

// Counters (device), mirrored into ft_stats.
struct DevCounters {
  unsigned long long layer_calls, lookups, hits, misses, staged, streamed, bytes_h2d, bytes_zero_copy;
  int32_t last_m, last_qstar, last_qstage, pad;
  unsigned long long prefetched;  // blobs staged by the decode prefetch
};

// LRU clock state (device).
struct LruClock {
  unsigned long long clock;        // last stamp handed out
  unsigned long long batch_start;  // first stamp of the latest lookup batch
};

struct Shape {
  int L, E, k, d, d_ff, wtype;
  long long C;
  size_t slot_bytes;
};

// Arguments of the lookup kernel (one batch of keys of one layer).
struct LookupArgs {
  int layer;
  int use_counts;     // 1: routed experts (counts > 0); 0: all E experts (prefill load)
  int limit_q;        // 1: apply q* (decode rules); 0: stage every miss
  int pin_prev;       // 1: also pin the previous batch (prefill prefetch of layer+1)
  int append;         // 1: append to the mailbox lookup record (prefill second batch)
  int is_current;     // 1: this batch is the called layer's (m, q*, q_stage are reported)
  int build_work;     // 1: (re)build the work lists from this batch
  unsigned bp_mbps, bh_mbps;
  int prefetch;       // 1: decode prefetch batch: resident experts are not touched, missing ones staged
                      //    while victims last, no lookup record, only the prefetched counter moves
  const int32_t* counts_src;  // routing counts of the batch (null: this call's)
  int32_t* record_counts;     // fused decode routing: also store this call's routing counts here (null: no)
};

// Device pointers of a context.
struct DevState {
  int32_t* slot_of;          // [L*E] slot or -1
  int32_t* key_of;           // [C] key or -1
  unsigned long long* stamp; // [C]
  LruClock* clk;
  DevCounters* ctr;
  uint32_t* error;
  WorkLists* work;
  Mailbox* mbox;             // mapped host memory (device address)
  // routing scratch
  float* scores;             // [Tmax*E]
  int32_t* ids;              // [Tmax*k]
  float* wts;                // [Tmax*k]
  int32_t* counts;           // [E]
  int32_t* offsets;          // [E+1]
  int32_t* perm;             // [Tmax*k]
  int32_t* inv;              // [Tmax*k]
  int32_t* perm_chunks;      // [ceil(Tmax*k / 1024)][E] per-chunk counts, then offsets (large-T permutation)
  // expert scratch
  float* hbuf;               // [Tmax*k, d_ff] SwiGLU activations (fp32)
  float* ybuf;               // [Tmax*k, d] expert outputs (fp32)
  __nv_bfloat16* xs;         // [Tmax*k, d] gathered bf16 activations (prefill)
  __nv_bfloat16* hs;         // [Tmax*k, d_ff] bf16 SwiGLU activations (prefill)
  uint16_t* h16;             // [Tmax*k, d_ff] 16-bit SwiGLU activations (MMA decode path)
  uint16_t* h16lo;           // [Tmax*k, d_ff] bf16 residual of h16 (BF16), f16 rest h - 2^24 h16 (NVFP4)
  uint16_t* x16;             // [Tmax, d] f16 copy of the activations times 2^-s_t (NVFP4 MMA path)
  float* xscale;             // [Tmax] 2^s_t of each token's f16 copy (NVFP4 MMA path)
  float* tscale;             // [L*E*3] NVFP4 tensor scales
  void* xin;                 // [Tmax, d] activations copied in from host memory (ft_moe_layer_forward_host)
  void* yout;                // [Tmax, d] output copied back to host memory
  uint8_t* slots;            // HBM slot pool [C * slot_bytes]
  const uint8_t* pool_dev;   // device address of the called layer's blobs in the mapped host pool
  void* tc_plan;             // host: tensor maps of the prefill GEMM (owned, see prefill_tc_free)
  int32_t* sched;            // [N_CLASSES] unit tickets + [N_CLASSES][sched_chunks] chunk completion counters
  int sched_chunks;
  int32_t* route_ctr;        // last-CTA ticket of the fused decode routing kernel (0 between calls)
  int32_t* prev_counts;      // [L][E] routing counts of each layer's last decode call (prefetch)
  uint32_t* landed;          // [MAX_E] per staged blob of a decode call: the call's epoch once its copy landed
  uint32_t landed_epoch;     // epoch of the current call (0: staged experts wait for all copies on the host side)
};

// ---- launchers (all enqueue on `st`) ----
// router logits s = x W_r^T + b, fp32 [T, E]
void launch_router_scores(const Shape& sh, const void* x, const void* w_router, const float* bias, int bias_per_token,
                          int T, float* scores, cudaStream_t st);
// top-k + softmax weights (ids, wts)
void launch_topk(const Shape& sh, const float* scores, int T, DevState& ds, cudaStream_t st);
// stable permutation (counts, offsets, perm, inv)
int launch_permute(const Shape& sh, int T, DevState& ds, cudaStream_t st);  // returns kernels launched
size_t perm_chunks_ints(int max_entries, int E);
// decode routing in one launch (T <= 32): logits, top-k, permutation, lookup
void launch_route_decode(const Shape& sh, const void* x, const void* w_router, const float* bias, int bias_per_token,
                         int T, const LookupArgs& la, const LookupArgs& pf, DevState& ds, bool to_f16,
                         cudaStream_t st);
// one lookup batch; writes work lists, mailbox, counters
void launch_lookup(const Shape& sh, const LookupArgs& a, DevState& ds, cudaStream_t st);
// decode / fallback experts (SIMT grouped GEMV) for one work class;
// phase 0: gate/up + SwiGLU into hbuf, phase 1: down into ybuf
void launch_expert_gemv(const Shape& sh, int cls, int phase, int layer, const void* x, int T, DevState& ds,
                        int max_items, int max_tok, cudaStream_t st);
// y[t] = sum_j w[t,j] Y[inv[t*k+j]]
void launch_combine(const Shape& sh, int T, DevState& ds, void* y, cudaStream_t st);
// zero-copy read probe: reads `bytes` from src, returns nothing useful
void launch_read_probe(const uint8_t* src, size_t bytes, unsigned long long* sink, cudaStream_t st);

}  // namespace ft
