// Host runtime behind include/ft_moe.h: the context, the pinned expert pool,
// the HBM slot pool, streams and events, and the per-call orchestration of
// the routing, lookup, copy-engine staging, expert and combine kernels.
//
// Two-tier expert memory ([paperlens] "設計: 2階建てのエキスパート記憶", paper §3):
// the pinned host pool is the source of truth, the slot pool is a cache.
// Decode call: router -> top-k/permutation -> lookup (q* split, [techfeed]
// "帯域適応型実行（q*ポリシー）") on the compute stream; the streamed misses run
// on a side stream straight from the mapped pool while the hits run on the
// compute stream; the host waits for the lookup kernel (bounded), issues the
// copy-engine H2D copies of the staged misses on the copy stream, and the
// staged experts run once their copies land. Prefill call: the whole layer is
// resident before it computes and the next layer is copied in behind it
// ([paperlens] "プレフィル: 全層ダブルバッファと「意味の錨」", paper §3.1).
#include <algorithm>
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

#include <cuda.h>

#include "ft_internal.cuh"

namespace ft {
cudaError_t route_kernels_init();
cudaError_t expert_kernels_init(int device);
void launch_prefill_work(const Shape& sh, int layer, DevState& ds, cudaStream_t st);
bool prefill_tc_supported(const Shape& sh);
cudaError_t prefill_tc_init(const Shape& sh, DevState& ds, int max_rows);
void prefill_tc_free(DevState& ds);
void launch_prefill_gather(const Shape& sh, const void* x, int T, DevState& ds, cudaStream_t st);
bool gemv_mma_supported(const Shape& sh);
cudaError_t gemv_mma_init(int device);
void launch_to_f16(const void* x, int T, int d, void* y, float* xscale, cudaStream_t st);
void launch_gemv_mma(const Shape& sh, int cls, int layer, const void* x16, int T, DevState& ds, int max_items,
                     int max_tok, cudaStream_t st);
void launch_gemm_tc(const Shape& sh, int phase, int layer, int T, DevState& ds, cudaStream_t st);
void launch_rows_in(const int32_t* eids, int n, int base, int E, DevState& ds, cudaStream_t st);
void launch_combine_rows(const float* ybuf, const float* wts, const int32_t* inv, int T, int k, int d, bool out_f32,
                         void* y, cudaStream_t st);
}  // namespace ft

using namespace ft;

struct ft_ctx {
  ft_config cfg;
  Shape sh;
  cudaStream_t s_comp = nullptr, s_copy = nullptr, s_side = nullptr;
  std::vector<uint8_t*> pool_host;  // per layer, E blobs each (pinned, mapped)
  std::vector<uint8_t*> pool_dev;   // device addresses of the same
  std::vector<const void*> router;  // per layer W_r device pointer
  std::vector<float> tscale_host;   // [L*E*3]
  DevState ds{};
  Mailbox* mbox_host = nullptr;
  cudaEvent_t ev_look = nullptr, ev_side = nullptr, ev_copy = nullptr, ev_pf[2] = {nullptr, nullptr};
  cudaEvent_t ev_t0 = nullptr, ev_t1 = nullptr;
  unsigned bp = 1, bh = 1;
  int prefetched = -1;   // layer whose experts the previous prefill call loaded ahead
  int last_T = 0, last_k = 0;  // rows and top-k of the last call (k = 1 after ft_moe_expert_rows)
  unsigned long long layer_calls = 0;
  int last_m = 0, last_qstar = 0, last_qstage = 0;
  ft_status latched = FT_OK;
  bool use_tc = false;
  bool use_mma = false;  // tensor-core decode GEMV (BF16 / NVFP4), else SIMT
  unsigned long long* probe_sink = nullptr;
  // stream memory operation that marks a staged blob as landed (null: not available)
  CUresult (*write_value)(CUstream, CUdeviceptr, cuuint32_t, unsigned int) = nullptr;
  uint32_t epoch = 0;
  // decode prefetch (opt-in): after layer l's lookup, stage the experts layer
  // (l+1) mod L was routed to in its last decode call
  bool prefetch_on = false;
  std::vector<char> has_prev;           // per layer: prev_counts holds its last decode routing
  bool pf_pending = false;              // prefetch copies in flight; readers wait on ev_pfd
  cudaEvent_t ev_pfd = nullptr;
  // launch accounting and optional per-launch CUDA-event profiling
  unsigned long long kernel_launches = 0;
  bool profiling = false;
  struct ProfRec {
    int name;
    cudaEvent_t a, b;
    double bytes, flops;
  };
  std::vector<ProfRec> pend;
  std::vector<cudaEvent_t> evpool;
  // always-on spans of each call on the compute stream and of its staging
  // copies on the copy stream (ft_stats.ms_compute / ms_copy)
  struct Span {
    cudaEvent_t a, b;
    bool copy;
  };
  std::vector<Span> spans;
  double ms_compute = 0, ms_copy = 0;
  struct Agg {
    unsigned long long n = 0;
    double ms = 0, bytes = 0, flops = 0;
  };
  std::vector<Agg> agg;
};

namespace {

bool fault(const char* what) {
  const char* f = getenv("FT_FAULT");
  return f && strstr(f, what) != nullptr;
}

#define CK(call)                                                                      \
  do {                                                                                \
    cudaError_t e_ = (call);                                                          \
    if (e_ != cudaSuccess) {                                                          \
      fprintf(stderr, "ft_moe: %s failed: %s (%s:%d)\n", #call, cudaGetErrorString(e_), \
              __FILE__, __LINE__);                                                    \
      return e_ == cudaErrorMemoryAllocation ? FT_ENOMEM : FT_ECUDA;                  \
    }                                                                                 \
  } while (0)

ft_status validate(const ft_config* c) {
  if (!c) return FT_EINVAL;
  if (c->n_layers < 1 || c->n_experts < 1 || c->n_experts > MAX_E) return FT_EINVAL;
  if (c->top_k < 1 || c->top_k > MAX_K || c->top_k > c->n_experts) return FT_EINVAL;
  if (c->d_model < 64 || c->d_model % 64 || c->d_model > 16384) return FT_EINVAL;
  if (c->d_ff < 64 || c->d_ff % 64 || c->d_ff > 16384) return FT_EINVAL;
  if (c->wtype < FT_W_F32 || c->wtype > FT_W_NVFP4) return FT_EINVAL;
  // up to every expert of every layer, or two layers' worth (the prefill
  // double buffer) when that is more
  const long long le = (long long)c->n_layers * c->n_experts, two = 2ll * c->n_experts;
  if (c->cache_slots < 0 || c->cache_slots > (le > two ? le : two) || c->cache_slots >= (1ll << 20))
    return FT_EINVAL;
  if (c->max_tokens < 1 || c->max_tokens > 65536) return FT_EINVAL;
  if (c->device < 0) return FT_EINVAL;
  return FT_OK;
}

size_t slot_bytes_of(const ft_config* c) {
  const size_t n = 3ull * c->d_model * c->d_ff;
  return c->wtype == FT_W_F32 ? 4 * n : (c->wtype == FT_W_BF16 ? 2 * n : n / 2 + n / 16);
}

// Host wait for an event with a deadline; the compute stream keeps running.
ft_status wait_event(cudaEvent_t ev, double seconds) {
  if (fault("poll_timeout")) return FT_ETIMEOUT;  // injected: a wait that never completes
  const auto t0 = std::chrono::steady_clock::now();
  long spins = 0;
  for (;;) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e == cudaSuccess) return FT_OK;
    if (e != cudaErrorNotReady) return FT_ECUDA;
    if ((++spins & 1023) == 0) {
      const double dt = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
      if (dt > seconds) return FT_ETIMEOUT;
      std::this_thread::yield();
    }
  }
}

constexpr double WAIT_S = 30.0;

void free_all(ft_ctx* c) {
  if (!c) return;
  if (c->s_comp || c->s_side) cudaDeviceSynchronize();
  DevState& d = c->ds;
  void* dev_ptrs[] = {d.slot_of, d.key_of, d.stamp, d.clk, d.ctr, d.error, d.work, d.scores, d.ids, d.wts,
                      d.counts, d.offsets, d.perm, d.inv, d.perm_chunks, d.hbuf, d.ybuf, d.xs, d.hs, d.tscale, d.slots,
                      d.h16, d.h16lo, d.x16, d.xscale, d.xin, d.yout, d.sched, d.route_ctr, d.landed, d.prev_counts, c->probe_sink};
  for (void* p : dev_ptrs)
    if (p) cudaFree(p);
  for (uint8_t* p : c->pool_host)
    if (p) cudaFreeHost(p);
  prefill_tc_free(d);
  if (c->mbox_host) cudaFreeHost(c->mbox_host);
  cudaEvent_t evs[] = {c->ev_look, c->ev_side, c->ev_copy, c->ev_pf[0], c->ev_pf[1], c->ev_t0, c->ev_t1, c->ev_pfd};
  for (cudaEvent_t e : evs)
    if (e) cudaEventDestroy(e);
  for (auto& r : c->pend) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (auto& r : c->spans) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  for (cudaEvent_t e : c->evpool) cudaEventDestroy(e);
  if (c->s_side) cudaStreamDestroy(c->s_side);
  delete c;
}

void fold_spans(ft_ctx* c, bool wait);
cudaEvent_t pooled_event(ft_ctx* c);

ft_status reset_state(ft_ctx* c) {
  const Shape& sh = c->sh;
  DevState& d = c->ds;
  CK(cudaMemsetAsync(d.slot_of, 0xFF, sizeof(int32_t) * sh.L * sh.E, c->s_comp));
  if (sh.C > 0) {
    CK(cudaMemsetAsync(d.key_of, 0xFF, sizeof(int32_t) * sh.C, c->s_comp));
    CK(cudaMemsetAsync(d.stamp, 0, sizeof(unsigned long long) * sh.C, c->s_comp));
  }
  CK(cudaMemsetAsync(d.clk, 0, sizeof(LruClock), c->s_comp));
  CK(cudaMemsetAsync(d.ctr, 0, sizeof(DevCounters), c->s_comp));
  CK(cudaMemsetAsync(d.error, 0, sizeof(uint32_t), c->s_comp));
  CK(cudaStreamSynchronize(c->s_comp));
  memset(c->mbox_host, 0, sizeof(Mailbox));
  CK(cudaStreamSynchronize(c->s_copy));
  fold_spans(c, true);
  c->ms_compute = c->ms_copy = 0;
  c->prefetched = -1;
  c->has_prev.assign(sh.L, 0);
  c->pf_pending = false;
  c->latched = FT_OK;
  c->last_m = c->last_qstar = c->last_qstage = 0;
  c->layer_calls = 0;
  return FT_OK;
}

ft_status check_device_error(ft_ctx* c) {
  // the lookup kernel mirrors the device error word into the mailbox
  const uint32_t e = ((volatile Mailbox*)c->mbox_host)->pad_error;
  if (e) c->latched = e == DERR_TIMEOUT ? FT_ETIMEOUT : FT_ESTATE;
  return c->latched;
}


enum ProfName {
  P_ROUTER, P_TOPK, P_PERMUTE, P_LOOKUP, P_GU_HIT, P_DN_HIT, P_GU_STAGED, P_DN_STAGED, P_GU_STREAM, P_DN_STREAM,
  P_COMBINE, P_STAGE_COPY, P_PREFILL_WORK, P_GATHER, P_GEMM_GU, P_GEMM_DN, P_GEMV_HIT, P_GEMV_STAGED,
  P_GEMV_STREAM, P_TO_F16, P_ROUTE_FUSED, P_PF_COPY, P_COUNT
};
const char* const kProfNames[P_COUNT] = {
    "router_scores", "topk_softmax", "permute", "lookup", "gemv_gateup_hit", "gemv_down_hit",
    "gemv_gateup_staged", "gemv_down_staged", "gemv_gateup_streamed", "gemv_down_streamed", "combine",
    "h2d_stage_copies", "prefill_work", "prefill_gather", "gemm_tc_gateup", "gemm_tc_down", "gemv_hit",
    "gemv_staged", "gemv_streamed", "to_f16", "route_decode_fused", "h2d_prefetch_copies"};

cudaEvent_t pooled_event(ft_ctx* c) {
  if (!c->evpool.empty()) {
    cudaEvent_t e = c->evpool.back();
    c->evpool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Bracket one launch (or a group of copies) on its stream when profiling.
// Returns the record index, or -1.
int prof_begin(ft_ctx* c, int name, cudaStream_t s, double bytes = 0, double flops = 0) {
  if (!c->profiling) return -1;
  ft_ctx::ProfRec r{name, pooled_event(c), pooled_event(c), bytes, flops};
  cudaEventRecord(r.a, s);
  c->pend.push_back(r);
  return (int)c->pend.size() - 1;
}

void prof_end(ft_ctx* c, int idx, cudaStream_t s) {
  if (idx >= 0) cudaEventRecord(c->pend[idx].b, s);
}

void prof_bytes(ft_ctx* c, int idx, double bytes, double flops) {
  if (idx >= 0) {
    c->pend[idx].bytes = bytes;
    c->pend[idx].flops = flops;
  }
}

// Fold finished spans into ms_compute / ms_copy, oldest first; with wait,
// every span (the caller has synchronised the streams). A span whose end has
// not been reached stops the non-blocking fold, so the list stays short.
void fold_spans(ft_ctx* c, bool wait) {
  size_t n = 0;
  for (; n < c->spans.size(); ++n) {
    const ft_ctx::Span& r = c->spans[n];
    if (!wait && cudaEventQuery(r.b) != cudaSuccess) break;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) == cudaSuccess) (r.copy ? c->ms_copy : c->ms_compute) += ms;
    c->evpool.push_back(r.a);
    c->evpool.push_back(r.b);
  }
  c->spans.erase(c->spans.begin(), c->spans.begin() + n);
  cudaGetLastError();  // a not-ready query is not an error of the next call
}

// Weight bytes per element of the expert format (codes plus block scales for NVFP4).
double weight_bytes_per_elem(int wtype) {
  return wtype == FT_W_F32 ? 4.0 : (wtype == FT_W_BF16 ? 2.0 : 0.5 + 1.0 / 16.0);
}

// Algorithmic bytes / flops of one grouped-GEMV phase over n_items experts
// carrying n_tok tokens: each weight once, activations in, outputs out.
void gemv_cost(const Shape& sh, int phase, int n_items, int n_tok, double& bytes, double& flops) {
  const double wb = weight_bytes_per_elem(sh.wtype), ab = sh.wtype == FT_W_F32 ? 4.0 : 2.0;
  const double dd = (double)sh.d * sh.d_ff;
  if (phase == 0) {
    bytes = n_items * 2.0 * dd * wb + n_tok * (double)sh.d * ab + n_tok * (double)sh.d_ff * 4.0;
    flops = 2.0 * n_tok * 2.0 * dd;
  } else {
    bytes = n_items * dd * wb + n_tok * (double)sh.d_ff * 4.0 + n_tok * (double)sh.d * 4.0;
    flops = 2.0 * n_tok * dd;
  }
}

}  // namespace

extern "C" {

const char* ft_status_str(ft_status s) {
  switch (s) {
    case FT_OK: return "ok";
    case FT_EINVAL: return "invalid argument";
    case FT_ENOMEM: return "out of memory";
    case FT_ECUDA: return "CUDA error";
    case FT_ETIMEOUT: return "timed out";
    case FT_ESTATE: return "bad state";
    case FT_EUNSUPPORTED: return "unsupported";
  }
  return "unknown status";
}

ft_status ft_moe_slot_bytes(const ft_config* cfg, uint64_t* out) {
  if (!out) return FT_EINVAL;
  const ft_status v = validate(cfg);
  if (v != FT_OK) return v;
  *out = slot_bytes_of(cfg);
  return FT_OK;
}

ft_status ft_moe_init(const ft_config* cfg, void* compute_stream, void* copy_stream, ft_ctx** out) {
  if (!out) return FT_EINVAL;
  *out = nullptr;
  const ft_status v = validate(cfg);
  if (v != FT_OK) return v;
  if (!copy_stream || copy_stream == compute_stream) return FT_EINVAL;
  CK(cudaSetDevice(cfg->device));
  ft_ctx* c = new (std::nothrow) ft_ctx();
  if (!c) return FT_ENOMEM;
  c->cfg = *cfg;
  Shape& sh = c->sh;
  sh.L = cfg->n_layers;
  sh.E = cfg->n_experts;
  sh.k = cfg->top_k;
  sh.d = cfg->d_model;
  sh.d_ff = cfg->d_ff;
  sh.wtype = cfg->wtype;
  sh.C = cfg->cache_slots;
  sh.slot_bytes = slot_bytes_of(cfg);
  c->s_comp = (cudaStream_t)compute_stream;
  c->s_copy = (cudaStream_t)copy_stream;
  c->router.assign(sh.L, nullptr);
  c->tscale_host.assign((size_t)sh.L * sh.E * 3, 1.0f);
  c->agg.assign(P_COUNT, ft_ctx::Agg{});
  ft_status st = FT_OK;
#define TRY(call)                    \
  do {                               \
    st = (call);                     \
    if (st != FT_OK) {               \
      free_all(c);                   \
      return st;                     \
    }                                \
  } while (0)
  auto cuda_try = [&](cudaError_t e) -> ft_status {
    if (e == cudaSuccess) return FT_OK;
    fprintf(stderr, "ft_moe_init: %s\n", cudaGetErrorString(e));
    return e == cudaErrorMemoryAllocation ? FT_ENOMEM : FT_ECUDA;
  };
  TRY(cuda_try(cudaStreamCreateWithFlags(&c->s_side, cudaStreamNonBlocking)));
  // pinned, mapped host pool, one chunk per layer
  c->pool_host.assign(sh.L, nullptr);
  c->pool_dev.assign(sh.L, nullptr);
  for (int l = 0; l < sh.L; ++l) {
    if (fault("pool_alloc")) TRY(FT_ENOMEM);
    TRY(cuda_try(cudaHostAlloc((void**)&c->pool_host[l], sh.slot_bytes * sh.E,
                               cudaHostAllocMapped | cudaHostAllocPortable)));
    TRY(cuda_try(cudaHostGetDevicePointer((void**)&c->pool_dev[l], c->pool_host[l], 0)));
  }
  TRY(cuda_try(cudaHostAlloc((void**)&c->mbox_host, sizeof(Mailbox), cudaHostAllocMapped)));
  memset(c->mbox_host, 0, sizeof(Mailbox));
  DevState& d = c->ds;
  TRY(cuda_try(cudaHostGetDevicePointer((void**)&d.mbox, c->mbox_host, 0)));
  const size_t Tk = (size_t)cfg->max_tokens * sh.k;
  if (fault("slot_alloc")) TRY(FT_ENOMEM);
  if (sh.C > 0) TRY(cuda_try(cudaMalloc((void**)&d.slots, sh.slot_bytes * (size_t)sh.C)));
  TRY(cuda_try(cudaMalloc((void**)&d.slot_of, sizeof(int32_t) * sh.L * sh.E)));
  TRY(cuda_try(cudaMalloc((void**)&d.key_of, sizeof(int32_t) * (sh.C > 0 ? sh.C : 1))));
  TRY(cuda_try(cudaMalloc((void**)&d.stamp, sizeof(unsigned long long) * (sh.C > 0 ? sh.C : 1))));
  TRY(cuda_try(cudaMalloc((void**)&d.clk, sizeof(LruClock))));
  TRY(cuda_try(cudaMalloc((void**)&d.ctr, sizeof(DevCounters))));
  TRY(cuda_try(cudaMalloc((void**)&d.error, sizeof(uint32_t))));
  TRY(cuda_try(cudaMalloc((void**)&d.work, sizeof(WorkLists))));
  TRY(cuda_try(cudaMalloc((void**)&d.scores, sizeof(float) * cfg->max_tokens * sh.E)));
  TRY(cuda_try(cudaMalloc((void**)&d.ids, sizeof(int32_t) * Tk)));
  TRY(cuda_try(cudaMalloc((void**)&d.wts, sizeof(float) * Tk)));
  TRY(cuda_try(cudaMalloc((void**)&d.counts, sizeof(int32_t) * sh.E)));
  TRY(cuda_try(cudaMalloc((void**)&d.offsets, sizeof(int32_t) * (sh.E + 1))));
  TRY(cuda_try(cudaMalloc((void**)&d.perm, sizeof(int32_t) * Tk)));
  TRY(cuda_try(cudaMalloc((void**)&d.inv, sizeof(int32_t) * Tk)));
  TRY(cuda_try(cudaMalloc((void**)&d.perm_chunks, sizeof(int32_t) * perm_chunks_ints((int)Tk, sh.E))));
  TRY(cuda_try(cudaMalloc((void**)&d.hbuf, sizeof(float) * Tk * sh.d_ff)));
  TRY(cuda_try(cudaMalloc((void**)&d.ybuf, sizeof(float) * Tk * sh.d)));
  TRY(cuda_try(cudaMalloc((void**)&d.tscale, sizeof(float) * sh.L * sh.E * 3)));
  {
    const size_t act = (size_t)cfg->max_tokens * sh.d * (sh.wtype == FT_W_F32 ? 4 : 2);
    TRY(cuda_try(cudaMalloc(&d.xin, act)));
    TRY(cuda_try(cudaMalloc(&d.yout, act)));
  }
  TRY(cuda_try(cudaMalloc((void**)&c->probe_sink, sizeof(unsigned long long))));
  c->use_mma = gemv_mma_supported(sh);
  if (c->use_mma) {
    TRY(cuda_try(cudaMalloc((void**)&d.h16, sizeof(uint16_t) * Tk * sh.d_ff)));
    TRY(cuda_try(cudaMalloc((void**)&d.h16lo, sizeof(uint16_t) * Tk * sh.d_ff)));
    if (sh.wtype == FT_W_NVFP4) {
      TRY(cuda_try(cudaMalloc((void**)&d.x16, sizeof(uint16_t) * (size_t)cfg->max_tokens * sh.d)));
      TRY(cuda_try(cudaMalloc((void**)&d.xscale, sizeof(float) * (size_t)cfg->max_tokens)));
    }
    TRY(cuda_try(gemv_mma_init(cfg->device)));
  }
  d.sched_chunks = sh.E + (int)((Tk + MMA_CHUNK - 1) / MMA_CHUNK) + 1;
  TRY(cuda_try(cudaMalloc((void**)&d.sched, sizeof(int32_t) * (N_CLASSES + (size_t)N_CLASSES * d.sched_chunks))));
  TRY(cuda_try(cudaMemset(d.sched, 0, sizeof(int32_t) * (N_CLASSES + (size_t)N_CLASSES * d.sched_chunks))));
  TRY(cuda_try(cudaMalloc((void**)&d.route_ctr, sizeof(int32_t))));
  TRY(cuda_try(cudaMemset(d.route_ctr, 0, sizeof(int32_t))));
  TRY(cuda_try(cudaMalloc((void**)&d.prev_counts, sizeof(int32_t) * (size_t)sh.L * sh.E)));
  TRY(cuda_try(cudaMalloc((void**)&d.landed, sizeof(uint32_t) * MAX_E)));
  TRY(cuda_try(cudaMemset(d.landed, 0, sizeof(uint32_t) * MAX_E)));
  d.landed_epoch = 0;
  {
    // cuStreamWriteValue32 lets the copy stream mark each staged blob as it
    // lands, so the staged experts' GEMV can start before the last copy ends;
    // without it the staged GEMV waits for every copy (an event)
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuStreamWriteValue32", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess && fn) {
      c->write_value = reinterpret_cast<CUresult (*)(CUstream, CUdeviceptr, cuuint32_t, unsigned int)>(fn);
      if (c->write_value((CUstream)c->s_side, (CUdeviceptr)d.landed, 0u, 0) != CUDA_SUCCESS ||
          cudaStreamSynchronize(c->s_side) != cudaSuccess)
        c->write_value = nullptr;
    }
    cudaGetLastError();
  }
  c->use_tc = prefill_tc_supported(sh) && sh.C >= 2ll * sh.E;
  if (c->use_tc) {
    TRY(cuda_try(cudaMalloc((void**)&d.xs, sizeof(__nv_bfloat16) * (Tk + 256) * sh.d)));
    TRY(cuda_try(cudaMalloc((void**)&d.hs, sizeof(__nv_bfloat16) * (Tk + 256) * sh.d_ff)));
    TRY(cuda_try(prefill_tc_init(sh, d, (int)Tk)));
  }
  d.pool_dev = nullptr;
  TRY(cuda_try(cudaMemcpy(d.tscale, c->tscale_host.data(), sizeof(float) * c->tscale_host.size(),
                          cudaMemcpyHostToDevice)));
  TRY(cuda_try(cudaEventCreateWithFlags(&c->ev_look, cudaEventDisableTiming)));
  TRY(cuda_try(cudaEventCreateWithFlags(&c->ev_side, cudaEventDisableTiming)));
  TRY(cuda_try(cudaEventCreateWithFlags(&c->ev_copy, cudaEventDisableTiming)));
  TRY(cuda_try(cudaEventCreateWithFlags(&c->ev_pf[0], cudaEventDisableTiming)));
  TRY(cuda_try(cudaEventCreateWithFlags(&c->ev_pf[1], cudaEventDisableTiming)));
  TRY(cuda_try(cudaEventCreateWithFlags(&c->ev_pfd, cudaEventDisableTiming)));
  TRY(cuda_try(cudaEventCreate(&c->ev_t0)));
  TRY(cuda_try(cudaEventCreate(&c->ev_t1)));
  TRY(cuda_try(route_kernels_init()));
  TRY(cuda_try(expert_kernels_init(cfg->device)));
  TRY(reset_state(c));
#undef TRY
  *out = c;
  return FT_OK;
}

void ft_moe_destroy(ft_ctx* c) { free_all(c); }

ft_status ft_moe_expert_ptr(ft_ctx* c, int32_t layer, int32_t expert, void** host_blob) {
  if (!c || !host_blob || layer < 0 || layer >= c->sh.L || expert < 0 || expert >= c->sh.E) return FT_EINVAL;
  *host_blob = c->pool_host[layer] + (size_t)expert * c->sh.slot_bytes;
  return FT_OK;
}

ft_status ft_moe_set_tensor_scales(ft_ctx* c, int32_t layer, int32_t expert, const float* scales) {
  if (!c || !scales || layer < 0 || layer >= c->sh.L || expert < 0 || expert >= c->sh.E) return FT_EINVAL;
  if (c->sh.wtype != FT_W_NVFP4) return FT_EINVAL;
  const size_t o = ((size_t)layer * c->sh.E + expert) * 3;
  memcpy(&c->tscale_host[o], scales, 3 * sizeof(float));
  CK(cudaMemcpyAsync(c->ds.tscale + o, &c->tscale_host[o], 3 * sizeof(float), cudaMemcpyHostToDevice, c->s_comp));
  CK(cudaStreamSynchronize(c->s_comp));
  return FT_OK;
}

ft_status ft_moe_set_router(ft_ctx* c, int32_t layer, const void* w) {
  if (!c || !w || layer < 0 || layer >= c->sh.L) return FT_EINVAL;
  if ((uintptr_t)w & 15) return FT_EINVAL;
  c->router[layer] = w;
  return FT_OK;
}

ft_status ft_set_bandwidths(ft_ctx* c, uint32_t bp, uint32_t bh) {
  if (!c || bh == 0) return FT_EINVAL;
  c->bp = bp;
  c->bh = bh;
  return FT_OK;
}

ft_status ft_moe_reset_cache(ft_ctx* c) {
  if (!c) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_copy));
  CK(cudaStreamSynchronize(c->s_side));
  return reset_state(c);
}

// The experts of one work class: one fused tensor-core launch (BF16 /
// NVFP4), or the two SIMT phases (fp32). pr receives the profile records.
static void gemv_class(ft_ctx* c, int cls, int layer, const void* x, int T, int max_items, int Tk, cudaStream_t st,
                       int (&pr)[2]) {
  static const int fused[3] = {P_GEMV_HIT, P_GEMV_STAGED, P_GEMV_STREAM};
  static const int gu[3] = {P_GU_HIT, P_GU_STAGED, P_GU_STREAM};
  static const int dn[3] = {P_DN_HIT, P_DN_STAGED, P_DN_STREAM};
  if (c->use_mma) {
    pr[0] = prof_begin(c, fused[cls], st);
    launch_gemv_mma(c->sh, cls, layer, c->sh.wtype == FT_W_NVFP4 ? (const void*)c->ds.x16 : x, T, c->ds, max_items, Tk,
                    st);
    prof_end(c, pr[0], st);
    pr[1] = -1;
    c->kernel_launches += 1;
  } else {
    for (int ph = 0; ph < 2; ++ph) {
      pr[ph] = prof_begin(c, ph == 0 ? gu[cls] : dn[cls], st);
      launch_expert_gemv(c->sh, cls, ph, layer, x, T, c->ds, max_items, Tk, st);
      prof_end(c, pr[ph], st);
    }
    c->kernel_launches += 2;
  }
}

// Algorithmic bytes / flops of a class's launches, once its size is known.
static void gemv_class_cost(ft_ctx* c, const int (&pr)[2], int n_items, int n_tok) {
  if (!c->profiling) return;
  double b0, f0, b1, f1;
  gemv_cost(c->sh, 0, n_items, n_tok, b0, f0);
  gemv_cost(c->sh, 1, n_items, n_tok, b1, f1);
  if (pr[1] < 0) {
    prof_bytes(c, pr[0], b0 + b1, f0 + f1);
  } else {
    prof_bytes(c, pr[0], b0, f0);
    prof_bytes(c, pr[1], b1, f1);
  }
}

// One cudaMemcpyAsync per staged blob on the copy stream; with epoch != 0,
// each copy is followed by a stream write of the epoch into landed[i - from].
static ft_status issue_copies(ft_ctx* c, int from, int to, uint32_t epoch = 0) {
  const Mailbox* mb = c->mbox_host;
  const Shape& sh = c->sh;
  if (to <= from) return FT_OK;
  ft_ctx::Span sp{pooled_event(c), pooled_event(c), true};
  CK(cudaEventRecord(sp.a, c->s_copy));
  struct Close {  // the span ends behind whatever copies were issued
    ft_ctx* c;
    ft_ctx::Span sp;
    ~Close() {
      if (cudaEventRecord(sp.b, c->s_copy) == cudaSuccess)
        c->spans.push_back(sp);
      else
        c->evpool.push_back(sp.a), c->evpool.push_back(sp.b);
    }
  } close{c, sp};
  for (int i = from; i < to; ++i) {
    const int key = mb->copy_key[i], slot = mb->copy_slot[i];
    const int l = key / sh.E, e = key % sh.E;
    if (l < 0 || l >= sh.L || slot < 0 || slot >= sh.C) return FT_ESTATE;
    if (fault("memcpy")) return FT_ECUDA;
    CK(cudaMemcpyAsync(c->ds.slots + (size_t)slot * sh.slot_bytes, c->pool_host[l] + (size_t)e * sh.slot_bytes,
                       sh.slot_bytes, cudaMemcpyHostToDevice, c->s_copy));
    if (epoch && c->write_value((CUstream)c->s_copy, (CUdeviceptr)(c->ds.landed + (i - from)), epoch, 0) !=
                     CUDA_SUCCESS)
      return FT_ECUDA;
  }
  return FT_OK;
}

// One layer call. With rows_eids == null: routing of T tokens, then lookup,
// experts and combine (ft_moe_layer_forward). With rows_eids: T rows already
// routed, row i to expert rows_eids[i] - rows_base, weight 1, no router; the
// caller has set sh.k to 1, and y receives the fp32 expert outputs in row
// order (ft_moe_expert_rows).
static ft_status layer_call(ft_ctx* c, int32_t layer, int32_t mode, const void* x, int32_t T, const float* bias,
                            int32_t bias_per_token, void* y, int32_t* ids_opt, float* w_opt,
                            const int32_t* rows_eids, int32_t rows_base) {
  const Shape& sh = c->sh;
  if (layer < 0 || layer >= sh.L || (mode != FT_DECODE && mode != FT_PREFILL)) return FT_EINVAL;
  if (T < 0 || T > c->cfg.max_tokens) return FT_EINVAL;
  if (c->latched != FT_OK) return c->latched;
  if (T == 0) return FT_OK;
  if (!x || !y || x == y) return FT_EINVAL;
  if (((uintptr_t)x | (uintptr_t)y) & 15) return FT_EINVAL;  // 16-byte vector loads and stores
  if (bias && ((uintptr_t)bias & 3)) return FT_EINVAL;
  if (!rows_eids && !c->router[layer]) return FT_ESTATE;
  DevState& d = c->ds;
  cudaStream_t cs = c->s_comp;
  fold_spans(c, false);
  struct CallSpan {  // this call's span on the compute stream, recorded on every return path
    ft_ctx* c;
    ft_ctx::Span sp;
    ~CallSpan() {
      if (cudaEventRecord(sp.b, c->s_comp) == cudaSuccess)
        c->spans.push_back(sp);
      else
        c->evpool.push_back(sp.a), c->evpool.push_back(sp.b);
    }
  } call_span{c, {pooled_event(c), pooled_event(c), false}};
  CK(cudaEventRecord(call_span.sp.a, cs));
  c->last_T = T;
  c->last_k = sh.k;
  c->layer_calls += 1;
  const double ab = sh.wtype == FT_W_F32 ? 4.0 : 2.0;
  const int Tk = T * sh.k;
  const bool full_prefill = mode == FT_PREFILL && sh.C >= 2ll * sh.E;
  // decode (and the on-demand prefill fallback) at small T: router, top-k,
  // permutation and lookup in one launch
  const bool fused_route = !full_prefill && T <= 32 && !rows_eids;
  LookupArgs la{};
  la.layer = layer;
  la.use_counts = 1;
  la.limit_q = 1;
  la.is_current = 1;
  la.build_work = 1;
  la.bp_mbps = c->bp;
  la.bh_mbps = c->bh;
  d.pool_dev = c->pool_dev[layer];
  // NVFP4 experts read an f16 copy of x; the fused routing writes it itself
  const bool want_f16 = c->use_mma && sh.wtype == FT_W_NVFP4 && !(full_prefill && c->use_tc);
  if (want_f16 && !fused_route) {
    launch_to_f16(x, T, sh.d, d.x16, d.xscale, cs);
    c->kernel_launches += 1;
  }
  // decode prefetch: right behind this call's lookup, a batch for the next
  // layer from its last decode routing (pins this batch's slots); the fused
  // routing runs it in the same launch. Then this call's routing counts become
  // this layer's record (the fused routing stores them itself, after the
  // prefetch batch has read the old ones, which matters for one-layer models)
  const int nxt_layer = (layer + 1) % sh.L;
  const bool want_pf = mode == FT_DECODE && !full_prefill && c->prefetch_on && c->has_prev[nxt_layer];
  LookupArgs pa{};
  pa.layer = -1;  // none
  if (want_pf) {
    pa.layer = nxt_layer;
    pa.use_counts = 1;
    pa.pin_prev = 1;
    pa.append = 1;
    pa.prefetch = 1;
    pa.counts_src = d.prev_counts + (size_t)nxt_layer * sh.E;
  }
  const bool pf_in_route = fused_route && want_pf;
  const bool record_in_route = mode == FT_DECODE && fused_route && !full_prefill;
  if (record_in_route) la.record_counts = d.prev_counts + (size_t)layer * sh.E;
  int p = -1;
  if (rows_eids) {
    p = prof_begin(c, P_PERMUTE, cs, Tk * 16.0 + sh.E * 8.0);
    launch_rows_in(rows_eids, T, rows_base, sh.E, d, cs);
    const int n_perm = launch_permute(sh, T, d, cs);
    prof_end(c, p, cs);
    c->kernel_launches += 1 + n_perm;
  } else if (fused_route) {
    p = prof_begin(c, P_ROUTE_FUSED, cs, T * (double)sh.d * ab + sh.E * (double)sh.d * ab + sh.C * 8.0);
    LookupArgs none{};
    none.layer = -1;
    launch_route_decode(sh, x, c->router[layer], bias, bias_per_token, T, la, pf_in_route ? pa : none, d, want_f16,
                        cs);
    prof_end(c, p, cs);
    c->kernel_launches += 1;
  } else {
    p = prof_begin(c, P_ROUTER, cs, T * (double)sh.d * ab + sh.E * (double)sh.d * ab + T * (double)sh.E * 4.0,
                   2.0 * T * sh.E * (double)sh.d);
    launch_router_scores(sh, x, c->router[layer], bias, bias_per_token, T, d.scores, cs);
    prof_end(c, p, cs);
    p = prof_begin(c, P_TOPK, cs, T * (double)sh.E * 4.0 + Tk * 8.0);
    launch_topk(sh, d.scores, T, d, cs);
    prof_end(c, p, cs);
    p = prof_begin(c, P_PERMUTE, cs, Tk * 12.0 + sh.E * 8.0);
    const int n_perm = launch_permute(sh, T, d, cs);
    prof_end(c, p, cs);
    c->kernel_launches += 2 + n_perm;
  }
  if (ids_opt) CK(cudaMemcpyAsync(ids_opt, d.ids, sizeof(int32_t) * Tk, cudaMemcpyDeviceToDevice, cs));
  if (w_opt) CK(cudaMemcpyAsync(w_opt, d.wts, sizeof(float) * Tk, cudaMemcpyDeviceToDevice, cs));
  const int max_items = Tk < sh.E ? Tk : sh.E;
  ft_status st = FT_OK;
  if (!full_prefill) {
    if (!fused_route) {
      p = prof_begin(c, P_LOOKUP, cs, sh.C * 8.0 + sh.E * 16.0);
      launch_lookup(sh, la, d, cs);
      prof_end(c, p, cs);
      c->kernel_launches += 1;
    }
    if (mode == FT_DECODE) {
      if (want_pf && !pf_in_route) {
        p = prof_begin(c, P_LOOKUP, cs, sh.C * 8.0 + sh.E * 16.0);
        launch_lookup(sh, pa, d, cs);
        prof_end(c, p, cs);
        c->kernel_launches += 1;
      }
      if (!record_in_route)
        CK(cudaMemcpyAsync(d.prev_counts + (size_t)layer * sh.E, d.counts, sizeof(int32_t) * sh.E,
                           cudaMemcpyDeviceToDevice, cs));
      c->has_prev[layer] = 1;
    }
    CK(cudaEventRecord(c->ev_look, cs));
    CK(cudaStreamWaitEvent(c->s_side, c->ev_look, 0));
    int pr_stream[2], pr_hit[2], pr_staged[2];
    gemv_class(c, KIND_STREAMED, layer, x, T, max_items, Tk, c->s_side, pr_stream);
    CK(cudaEventRecord(c->ev_side, c->s_side));
    if (c->pf_pending) {  // slots the last call prefetched may be this call's hits
      CK(cudaStreamWaitEvent(cs, c->ev_pfd, 0));
      c->pf_pending = false;
    }
    gemv_class(c, KIND_HIT, layer, x, T, max_items, Tk, cs, pr_hit);
    st = wait_event(c->ev_look, WAIT_S);
    if (st != FT_OK) return c->latched = st;
    if (check_device_error(c) != FT_OK) return c->latched;
    const Mailbox* mb = c->mbox_host;
    const int n_copy = mb->qstage;       // this layer's staged blobs come first in the copy list
    const int n_copy_all = mb->n_copy;   // then the prefetched ones
    c->last_m = mb->m;
    c->last_qstar = mb->qstar;
    c->last_qstage = mb->qstage;
    gemv_class_cost(c, pr_stream, mb->n_streamed_cls, mb->n_tok_cls[KIND_STREAMED]);
    gemv_class_cost(c, pr_hit, mb->n_hit_cls, mb->n_tok_cls[KIND_HIT]);
    if (n_copy > 0) {
      // with landed flags the staged GEMV starts at once and each of its
      // experts waits (on the device) for its own copy; else it waits for all
      const bool flags = c->write_value != nullptr && c->use_mma && n_copy <= MAX_E;
      if (flags && ++c->epoch == 0) ++c->epoch;
      // the staged class's profile window opens with its first copy: its
      // bytes cross the host link inside that window, whatever the GEMV's
      // own launch time
      cudaEvent_t stage_open = nullptr;
      if (c->profiling) {
        stage_open = pooled_event(c);
        CK(cudaEventRecord(stage_open, c->s_copy));
      }
      p = prof_begin(c, P_STAGE_COPY, c->s_copy, n_copy * (double)sh.slot_bytes);
      st = issue_copies(c, 0, n_copy, flags ? c->epoch : 0);
      prof_end(c, p, c->s_copy);
      if (st != FT_OK) return c->latched = st;
      CK(cudaEventRecord(c->ev_copy, c->s_copy));
      if (flags)
        d.landed_epoch = c->epoch;
      else
        CK(cudaStreamWaitEvent(cs, c->ev_copy, 0));
      gemv_class(c, KIND_STAGED, layer, x, T, max_items, Tk, cs, pr_staged);
      if (stage_open) {
        if (pr_staged[0] >= 0 && pr_staged[1] < 0) {
          c->evpool.push_back(c->pend[pr_staged[0]].a);
          c->pend[pr_staged[0]].a = stage_open;
        } else {
          c->evpool.push_back(stage_open);
        }
      }
      d.landed_epoch = 0;
      gemv_class_cost(c, pr_staged, mb->n_staged_cls, mb->n_tok_cls[KIND_STAGED]);
    }
    if (n_copy_all > n_copy) {
      p = prof_begin(c, P_PF_COPY, c->s_copy, (n_copy_all - n_copy) * (double)sh.slot_bytes);
      st = issue_copies(c, n_copy, n_copy_all);
      prof_end(c, p, c->s_copy);
      if (st != FT_OK) return c->latched = st;
      CK(cudaEventRecord(c->ev_pfd, c->s_copy));
      c->pf_pending = true;
    }
    CK(cudaStreamWaitEvent(cs, c->ev_side, 0));
    c->prefetched = -1;
  } else {
    const bool load_cur = c->prefetched != layer;
    const bool load_next = layer + 1 < sh.L;
    if (load_cur) {
      LookupArgs a{};
      a.layer = layer;
      a.is_current = 1;
      launch_lookup(sh, a, d, cs);
      c->kernel_launches += 1;
    }
    if (load_next) {
      LookupArgs a{};
      a.layer = layer + 1;
      a.pin_prev = 1;
      a.append = load_cur ? 1 : 0;
      launch_lookup(sh, a, d, cs);
      c->kernel_launches += 1;
    }
    if (load_cur || load_next) {
      CK(cudaEventRecord(c->ev_look, cs));
      st = wait_event(c->ev_look, WAIT_S);
      if (st != FT_OK) return c->latched = st;
      if (check_device_error(c) != FT_OK) return c->latched;
      const Mailbox* mb = c->mbox_host;
      int split = 0;
      while (split < mb->n_copy && mb->copy_key[split] / sh.E == layer) ++split;
      if (load_cur) {
        c->last_m = mb->m;
        c->last_qstar = -1;
        c->last_qstage = mb->qstage;
        p = prof_begin(c, P_STAGE_COPY, c->s_copy, split * (double)sh.slot_bytes);
        st = issue_copies(c, 0, split);
        prof_end(c, p, c->s_copy);
        if (st != FT_OK) return c->latched = st;
        CK(cudaEventRecord(c->ev_pf[layer & 1], c->s_copy));
      } else {
        c->last_m = c->last_qstage = 0;
        c->last_qstar = -1;
      }
      if (load_next) {
        p = prof_begin(c, P_STAGE_COPY, c->s_copy, (mb->n_copy - split) * (double)sh.slot_bytes);
        st = issue_copies(c, split, mb->n_copy);
        prof_end(c, p, c->s_copy);
        if (st != FT_OK) return c->latched = st;
        CK(cudaEventRecord(c->ev_pf[(layer + 1) & 1], c->s_copy));
      }
    }
    if (!load_cur && !load_next) {
      // no lookup this call: clear the record (the last lookup kernel has
      // finished, the host waited for it)
      Mailbox* mb = c->mbox_host;
      mb->n_copy = mb->n_lookup = mb->n_lookup_cur = 0;
      mb->m = mb->qstage = 0;
      mb->qstar = -1;
      c->last_m = c->last_qstage = 0;
      c->last_qstar = -1;
    }
    c->prefetched = load_next ? layer + 1 : -1;
    p = prof_begin(c, P_PREFILL_WORK, cs);
    launch_prefill_work(sh, layer, d, cs);
    prof_end(c, p, cs);
    c->kernel_launches += 1;
    CK(cudaStreamWaitEvent(cs, c->ev_pf[layer & 1], 0));
    if (c->pf_pending) {  // slots a decode prefetch is still writing
      CK(cudaStreamWaitEvent(cs, c->ev_pfd, 0));
      c->pf_pending = false;
    }
    if (c->use_tc) {
      // algorithmic bytes with every routed expert read once; at prefill
      // sizes nearly all E experts are routed, so min(E, T*k) is used
      const double n_it = max_items, dd = (double)sh.d * sh.d_ff;
      p = prof_begin(c, P_GATHER, cs, Tk * (double)sh.d * 2.0 + T * (double)sh.d * ab);
      launch_prefill_gather(sh, x, T, d, cs);
      prof_end(c, p, cs);
      const double wb = weight_bytes_per_elem(sh.wtype);
      p = prof_begin(c, P_GEMM_GU, cs, n_it * 2.0 * dd * wb + Tk * (double)sh.d * 2.0 + Tk * (double)sh.d_ff * 2.0,
                     2.0 * Tk * 2.0 * dd);
      launch_gemm_tc(sh, 0, layer, T, d, cs);
      prof_end(c, p, cs);
      p = prof_begin(c, P_GEMM_DN, cs, n_it * dd * wb + Tk * (double)sh.d_ff * 2.0 + Tk * (double)sh.d * 4.0,
                     2.0 * Tk * dd);
      launch_gemm_tc(sh, 1, layer, T, d, cs);
      prof_end(c, p, cs);
      c->kernel_launches += 3;
    } else {
      d.pool_dev = c->pool_dev[layer];
      int pr[2];
      gemv_class(c, KIND_HIT, layer, x, T, max_items, Tk, cs, pr);
      gemv_class_cost(c, pr, max_items, Tk);  // upper bound: every routed expert
    }
  }
  if (rows_eids) {  // k = 1, weight 1: each row's fp32 output, back in row order
    p = prof_begin(c, P_COMBINE, cs, Tk * (double)sh.d * 8.0 + Tk * 8.0);
    launch_combine_rows(d.ybuf, d.wts, d.inv, T, 1, sh.d, true, y, cs);
  } else {
    p = prof_begin(c, P_COMBINE, cs, Tk * (double)sh.d * 4.0 + T * (double)sh.d * ab + Tk * 8.0);
    launch_combine(sh, T, d, y, cs);
  }
  prof_end(c, p, cs);
  c->kernel_launches += 1;
  CK(cudaGetLastError());
  return FT_OK;
}

ft_status ft_moe_layer_forward(ft_ctx* c, int32_t layer, int32_t mode, const void* x, int32_t T, const float* bias,
                               int32_t bias_per_token, void* y, int32_t* ids_opt, float* w_opt) {
  if (!c) return FT_EINVAL;
  return layer_call(c, layer, mode, x, T, bias, bias_per_token, y, ids_opt, w_opt, nullptr, 0);
}

ft_status ft_moe_layer_forward_host(ft_ctx* c, int32_t layer, int32_t mode, const void* x_host, int32_t T,
                                    const float* bias, int32_t bias_per_token, void* y_host) {
  if (!c) return FT_EINVAL;
  if (T < 0 || T > c->cfg.max_tokens) return FT_EINVAL;
  if (c->latched != FT_OK) return c->latched;
  if (T == 0) return FT_OK;
  if (!x_host || !y_host) return FT_EINVAL;
  const size_t bytes = (size_t)T * c->sh.d * (c->sh.wtype == FT_W_F32 ? 4 : 2);
  const uintptr_t xa = (uintptr_t)x_host, ya = (uintptr_t)y_host;
  if (xa < ya + bytes && ya < xa + bytes) return FT_EINVAL;  // overlapping host buffers
  CK(cudaMemcpyAsync(c->ds.xin, x_host, bytes, cudaMemcpyHostToDevice, c->s_comp));
  const ft_status st = layer_call(c, layer, mode, c->ds.xin, T, bias, bias_per_token, c->ds.yout, nullptr, nullptr,
                                  nullptr, 0);
  if (st != FT_OK) return st;
  CK(cudaMemcpyAsync(y_host, c->ds.yout, bytes, cudaMemcpyDeviceToHost, c->s_comp));
  return FT_OK;
}

ft_status ft_moe_expert_rows(ft_ctx* c, int32_t layer, int32_t mode, const void* rows, const int32_t* eids,
                             int32_t expert_base, int32_t n, float* out) {
  if (!c) return FT_EINVAL;
  if (n > 0 && !eids) return FT_EINVAL;
  // every row is its own "token" routed to one expert: the pipeline runs with
  // k = 1 for this call (launch arguments are taken by value when enqueued)
  struct KeepK {
    Shape& sh;
    int k;
    ~KeepK() { sh.k = k; }
  } keep{c->sh, c->sh.k};
  c->sh.k = 1;
  return layer_call(c, layer, mode, rows, n, nullptr, 0, out, nullptr, nullptr, eids, expert_base);
}

ft_status ft_cache_stats(ft_ctx* c, ft_stats* out) {
  if (!c || !out) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_copy));
  CK(cudaStreamSynchronize(c->s_side));
  CK(cudaStreamSynchronize(c->s_comp));
  DevCounters h{};
  uint32_t err = 0;
  CK(cudaMemcpy(&h, c->ds.ctr, sizeof(h), cudaMemcpyDeviceToHost));
  CK(cudaMemcpy(&err, c->ds.error, sizeof(err), cudaMemcpyDeviceToHost));
  out->layer_calls = c->layer_calls;
  out->lookups = h.lookups;
  out->hits = h.hits;
  out->misses = h.misses;
  out->staged = h.staged;
  out->streamed = h.streamed;
  out->bytes_h2d = h.bytes_h2d;
  out->bytes_zero_copy = h.bytes_zero_copy;
  out->last_m = c->last_m;
  out->last_qstar = c->last_qstar;
  out->last_qstage = c->last_qstage;
  out->device_error = err ? (err == DERR_TIMEOUT ? FT_ETIMEOUT : FT_ESTATE) : (int32_t)c->latched;
  out->kernel_launches = c->kernel_launches;
  out->prefetched = h.prefetched;
  fold_spans(c, true);
  out->ms_compute = c->ms_compute;
  out->ms_copy = c->ms_copy;
  return FT_OK;
}

ft_status ft_moe_set_prefetch(ft_ctx* c, int32_t enable) {
  if (!c) return FT_EINVAL;
  c->prefetch_on = enable != 0;
  return FT_OK;
}

ft_status ft_moe_last_route(ft_ctx* c, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv,
                            int32_t* lookup_e, int32_t* lookup_kind, int32_t* n_lookup, int32_t* n_lookup_cur,
                            int32_t* m, int32_t* qstar, int32_t* qstage) {
  if (!c) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_copy));
  CK(cudaStreamSynchronize(c->s_side));
  CK(cudaStreamSynchronize(c->s_comp));
  const Shape& sh = c->sh;
  const size_t Tk = (size_t)c->last_T * c->last_k;
  if (counts) CK(cudaMemcpy(counts, c->ds.counts, sizeof(int32_t) * sh.E, cudaMemcpyDeviceToHost));
  if (offsets) CK(cudaMemcpy(offsets, c->ds.offsets, sizeof(int32_t) * (sh.E + 1), cudaMemcpyDeviceToHost));
  if (perm && Tk) CK(cudaMemcpy(perm, c->ds.perm, sizeof(int32_t) * Tk, cudaMemcpyDeviceToHost));
  if (inv && Tk) CK(cudaMemcpy(inv, c->ds.inv, sizeof(int32_t) * Tk, cudaMemcpyDeviceToHost));
  const Mailbox* mb = c->mbox_host;
  if (lookup_e) memcpy(lookup_e, mb->lookup_e, sizeof(int32_t) * mb->n_lookup);
  if (lookup_kind) memcpy(lookup_kind, mb->lookup_kind, sizeof(int32_t) * mb->n_lookup);
  if (n_lookup) *n_lookup = mb->n_lookup;
  if (n_lookup_cur) *n_lookup_cur = mb->n_lookup_cur;
  if (m) *m = c->last_m;
  if (qstar) *qstar = c->last_qstar;
  if (qstage) *qstage = c->last_qstage;
  return FT_OK;
}

ft_status ft_moe_cache_contents(ft_ctx* c, int32_t* key_of, uint64_t* stamp) {
  if (!c) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_copy));
  CK(cudaStreamSynchronize(c->s_side));
  CK(cudaStreamSynchronize(c->s_comp));
  if (c->sh.C == 0) return FT_OK;
  if (key_of) CK(cudaMemcpy(key_of, c->ds.key_of, sizeof(int32_t) * c->sh.C, cudaMemcpyDeviceToHost));
  if (stamp) CK(cudaMemcpy(stamp, c->ds.stamp, sizeof(uint64_t) * c->sh.C, cudaMemcpyDeviceToHost));
  return FT_OK;
}

ft_status ft_moe_resize_cache(ft_ctx* c, int64_t new_slots) {
  if (!c) return FT_EINVAL;
  Shape& sh = c->sh;
  DevState& d = c->ds;
  const long long le = (long long)sh.L * sh.E, two = 2ll * sh.E;
  if (new_slots < 0 || new_slots > (le > two ? le : two) || new_slots >= (1ll << 20)) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_copy));
  CK(cudaStreamSynchronize(c->s_side));
  CK(cudaStreamSynchronize(c->s_comp));
  if (check_device_error(c) != FT_OK) return c->latched;
  const long long C = sh.C, Cn = new_slots;
  c->prefetched = -1;
  c->has_prev.assign(sh.L, 0);  // the prefetch record does not survive a resize
  c->pf_pending = false;
  if (Cn == C) return FT_OK;

  // 1. what is resident now
  std::vector<int32_t> key(C > 0 ? C : 1, -1);
  std::vector<unsigned long long> stamp(C > 0 ? C : 1, 0);
  if (C > 0) {
    CK(cudaMemcpy(key.data(), d.key_of, sizeof(int32_t) * C, cudaMemcpyDeviceToHost));
    CK(cudaMemcpy(stamp.data(), d.stamp, sizeof(unsigned long long) * C, cudaMemcpyDeviceToHost));
  }
  // 2. survivors: the Cn most recently used; they keep their slot when it
  // still exists, else take the lowest free ones (ascending old slot)
  std::vector<long long> res;
  for (long long s = 0; s < C; ++s)
    if (key[s] >= 0) res.push_back(s);
  std::sort(res.begin(), res.end(), [&](long long a, long long b) { return stamp[a] > stamp[b]; });
  if ((long long)res.size() > Cn) res.resize(Cn);
  std::sort(res.begin(), res.end());
  const size_t nC = Cn > 0 ? (size_t)Cn : 1;
  std::vector<int32_t> nkey(nC, -1), slot_of((size_t)sh.L * sh.E, -1);
  std::vector<unsigned long long> nstamp(nC, 0);
  std::vector<std::pair<long long, long long>> moves;  // (old slot, new slot)
  for (long long s : res)
    if (s < Cn) moves.push_back({s, s}), nkey[s] = key[s], nstamp[s] = stamp[s];
  long long t = 0;
  for (long long s : res) {
    if (s < Cn) continue;
    while (nkey[t] >= 0) ++t;
    moves.push_back({s, t});
    nkey[t] = key[s];
    nstamp[t] = stamp[s];
  }
  for (long long s = 0; s < Cn; ++s)
    if (nkey[s] >= 0) slot_of[nkey[s]] = (int32_t)s;

  // 3. new pool and tables; on any failure the context is left as it was
  Shape shn = sh;
  shn.C = Cn;
  const bool tc_new = prefill_tc_supported(shn) && Cn >= 2ll * sh.E;
  uint8_t* nslots = nullptr;
  int32_t* nk = nullptr;
  unsigned long long* ns = nullptr;
  __nv_bfloat16 *nxs = nullptr, *nhs = nullptr;
  const size_t Tk = (size_t)c->cfg.max_tokens * sh.k;
  auto undo = [&]() {
    void* ps[] = {nslots, nk, ns, nxs, nhs};
    for (void* p : ps)
      if (p) cudaFree(p);
    cudaGetLastError();
  };
  bool ok = !fault("resize_alloc");
  if (ok && Cn > 0) ok = cudaMalloc((void**)&nslots, sh.slot_bytes * (size_t)Cn) == cudaSuccess;
  if (ok) ok = cudaMalloc((void**)&nk, sizeof(int32_t) * nC) == cudaSuccess;
  if (ok) ok = cudaMalloc((void**)&ns, sizeof(unsigned long long) * nC) == cudaSuccess;
  if (ok && tc_new && !d.xs) {
    ok = cudaMalloc((void**)&nxs, sizeof(__nv_bfloat16) * (Tk + 256) * sh.d) == cudaSuccess &&
         cudaMalloc((void**)&nhs, sizeof(__nv_bfloat16) * (Tk + 256) * sh.d_ff) == cudaSuccess;
  }
  if (!ok) {
    undo();
    return FT_ENOMEM;
  }
  // 4. survivors device-to-device, runs of consecutive slots in one copy each
  std::sort(moves.begin(), moves.end());
  cudaError_t ce = cudaSuccess;
  for (size_t i = 0; i < moves.size() && ce == cudaSuccess;) {
    size_t j = i + 1;
    while (j < moves.size() && moves[j].first == moves[j - 1].first + 1 && moves[j].second == moves[j - 1].second + 1)
      ++j;
    ce = cudaMemcpyAsync(nslots + (size_t)moves[i].second * sh.slot_bytes, d.slots + (size_t)moves[i].first * sh.slot_bytes,
                         (j - i) * sh.slot_bytes, cudaMemcpyDeviceToDevice, c->s_comp);
    i = j;
  }
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(nk, nkey.data(), sizeof(int32_t) * nC, cudaMemcpyHostToDevice, c->s_comp);
  if (ce == cudaSuccess)
    ce = cudaMemcpyAsync(ns, nstamp.data(), sizeof(unsigned long long) * nC, cudaMemcpyHostToDevice, c->s_comp);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(c->s_comp);
  if (ce != cudaSuccess) {
    cudaStreamSynchronize(c->s_comp);
    undo();
    fprintf(stderr, "ft_moe_resize_cache: %s\n", cudaGetErrorString(ce));
    return FT_ECUDA;
  }
  // 5. commit
  CK(cudaMemcpy(d.slot_of, slot_of.data(), sizeof(int32_t) * slot_of.size(), cudaMemcpyHostToDevice));
  if (d.slots) cudaFree(d.slots);
  cudaFree(d.key_of);
  cudaFree(d.stamp);
  d.slots = nslots;
  d.key_of = nk;
  d.stamp = ns;
  sh.C = Cn;
  c->cfg.cache_slots = Cn;
  prefill_tc_free(d);
  if (nxs) d.xs = nxs, d.hs = nhs;
  if (!tc_new && d.xs) {
    cudaFree(d.xs);
    cudaFree(d.hs);
    d.xs = d.hs = nullptr;
  }
  c->use_tc = tc_new;
  if (tc_new && prefill_tc_init(sh, d, (int)Tk) != cudaSuccess) {
    prefill_tc_free(d);
    c->use_tc = false;  // prefill keeps working on the GEMV path
    cudaGetLastError();
  }
  return FT_OK;
}

ft_status ft_moe_probe_link(ft_ctx* c, uint64_t bytes, double* h2d_gbs, double* zc_gbs) {
  if (!c || bytes == 0 || bytes % 4096) return FT_EINVAL;
  const Shape& sh = c->sh;
  if (bytes > sh.slot_bytes * (size_t)sh.E) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_comp));
  CK(cudaStreamSynchronize(c->s_copy));
  uint8_t* tmp = nullptr;
  CK(cudaMalloc((void**)&tmp, bytes));
  float ms = 0.f;
  cudaError_t e = cudaSuccess;
  for (int rep = 0; rep < 2 && e == cudaSuccess; ++rep) {  // first pass warms up
    e = cudaEventRecord(c->ev_t0, c->s_copy);
    if (e == cudaSuccess) e = cudaMemcpyAsync(tmp, c->pool_host[0], bytes, cudaMemcpyHostToDevice, c->s_copy);
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_t1, c->s_copy);
    if (e == cudaSuccess) e = cudaEventSynchronize(c->ev_t1);
  }
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, c->ev_t0, c->ev_t1);
  if (e == cudaSuccess && h2d_gbs) *h2d_gbs = bytes / (ms * 1e6);
  for (int rep = 0; rep < 2 && e == cudaSuccess; ++rep) {
    e = cudaEventRecord(c->ev_t0, c->s_comp);
    if (e == cudaSuccess) {
      launch_read_probe(c->pool_dev[0], bytes, c->probe_sink, c->s_comp);
      e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaEventRecord(c->ev_t1, c->s_comp);
    if (e == cudaSuccess) e = cudaEventSynchronize(c->ev_t1);
  }
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, c->ev_t0, c->ev_t1);
  if (e == cudaSuccess && zc_gbs) *zc_gbs = bytes / (ms * 1e6);
  cudaFree(tmp);
  CK(e);
  return FT_OK;
}

ft_status ft_moe_profile(ft_ctx* c, int32_t enable) {
  if (!c) return FT_EINVAL;
  c->profiling = enable != 0;
  return FT_OK;
}

ft_status ft_moe_profile_read(ft_ctx* c, ft_kernel_time* out, int32_t cap, int32_t* n_out, int32_t reset) {
  if (!c || !n_out || cap < 0 || (cap > 0 && !out)) return FT_EINVAL;
  CK(cudaStreamSynchronize(c->s_copy));
  CK(cudaStreamSynchronize(c->s_side));
  CK(cudaStreamSynchronize(c->s_comp));
  for (auto& r : c->pend) {
    float ms = 0.f;
    CK(cudaEventElapsedTime(&ms, r.a, r.b));
    ft_ctx::Agg& g = c->agg[r.name];
    g.n += 1;
    g.ms += ms;
    g.bytes += r.bytes;
    g.flops += r.flops;
    c->evpool.push_back(r.a);
    c->evpool.push_back(r.b);
  }
  c->pend.clear();
  int n = 0;
  for (int i = 0; i < P_COUNT; ++i) {
    const ft_ctx::Agg& g = c->agg[i];
    if (g.n == 0) continue;
    if (n < cap) {
      memset(out[n].name, 0, sizeof(out[n].name));
      strncpy(out[n].name, kProfNames[i], sizeof(out[n].name) - 1);
      out[n].launches = g.n;
      out[n].ms = g.ms;
      out[n].bytes = g.bytes;
      out[n].flops = g.flops;
    }
    ++n;
  }
  *n_out = n;
  if (reset) c->agg.assign(P_COUNT, ft_ctx::Agg{});
  return FT_OK;
}

}  // extern "C"
