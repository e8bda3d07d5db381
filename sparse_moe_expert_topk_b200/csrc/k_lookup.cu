// Device-side lookup of one batch of (layer, expert) keys in the shared LRU
// slot cache, with the q* split of the misses.
//
// The pages: one elastic expert cache shared by all MoE layers, one slot per
// (layer, expert) ([paperlens] "設計: 2階建てのエキスパート記憶", paper §3), kept
// as an LRU that follows the router during decode ([techfeed]
// "セマンティック認識キャッシング"); of m missed experts about m B_P / B_H go to
// the GPU cache and the rest run where the weights are ([techfeed]
// "帯域適応型実行（q*ポリシー）"); prefill brings in whole layers ([paperlens]
// "プレフィル: 全層ダブルバッファと「意味の錨」", paper §3.1).
//
// Rules (the readings documented with the C ABI): keys of a batch are taken in
// ascending expert order; hits get fresh stamps first, then the staged misses
// in ascending order; q* = floor((2 m B_P + B_H) / (2 B_H)) clamped to [0, m];
// the first min(q*, C - hits) misses are staged; an insertion takes the free
// slot of lowest index, else the unpinned slot of smallest stamp. Since every
// inserted entry is pinned, the victims of a batch are exactly its q_stage
// smallest (stamp, slot) pairs among unpinned slots (free slots carry stamp 0),
// handed out in increasing order; this kernel finds them with a radix select.
#include "lookup_body.cuh"

namespace ft {

namespace {

using namespace lookup_detail;

__global__ void __launch_bounds__(NT) lookup_kernel(LookupArgs a, int E, long long C, size_t slot_bytes,
                                                    DevState ds) {
  lookup_body(a, E, C, slot_bytes, ds);
}

// Work list of a prefill call: every routed expert, read from its slot.
__global__ void __launch_bounds__(NT) prefill_work_kernel(int layer, int E, DevState ds) {
  __shared__ ScanTmp scan;
  const int tid = threadIdx.x;
  const bool in = tid < E && ds.counts[tid] > 0;
  int n;
  const int r = block_scan_flag(in, scan, n);
  {
    __shared__ int s_ch;
    int ch = in ? (ds.counts[tid] + MMA_CHUNK - 1) / MMA_CHUNK : 0;
    for (int o = 16; o > 0; o >>= 1) ch += __shfl_xor_sync(0xffffffffu, ch, o);
    if (tid == 0) s_ch = 0;
    __syncthreads();
    if ((tid & 31) == 0) atomicAdd(&s_ch, ch);
    __syncthreads();
    const int nch = s_ch < ds.sched_chunks ? s_ch : ds.sched_chunks;
    int32_t* done = ds.sched + N_CLASSES + (size_t)KIND_HIT * ds.sched_chunks;
    for (int i = tid; i < nch; i += NT) done[i] = 0;
    if (tid == 0) ds.sched[KIND_HIT] = 0;
  }
  if (in) {
    WorkItem it;
    it.e = tid;
    it.slot = ds.slot_of[layer * E + tid];
    it.tok_off = ds.offsets[tid];
    it.n_tok = ds.counts[tid];
    if (it.slot < 0) atomicExch(ds.error, (uint32_t)DERR_BAD_INDEX);  // the expert kernels skip it
    ds.work->items[KIND_HIT][r] = it;
  }
  if (tid == 0) {
    ds.work->n_items[KIND_HIT] = n;
    ds.work->n_items[KIND_STAGED] = 0;
    ds.work->n_items[KIND_STREAMED] = 0;
  }
}

}  // namespace

void launch_lookup(const Shape& sh, const LookupArgs& a, DevState& ds, cudaStream_t st) {
  lookup_kernel<<<1, NT, 0, st>>>(a, sh.E, sh.C, sh.slot_bytes, ds);
}

void launch_prefill_work(const Shape& sh, int layer, DevState& ds, cudaStream_t st) {
  prefill_work_kernel<<<1, NT, 0, st>>>(layer, sh.E, ds);
}

}  // namespace ft
