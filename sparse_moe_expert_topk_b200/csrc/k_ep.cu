// Expert parallelism: the kernels on either side of the exchange between
// devices that split the experts of every layer in contiguous blocks.
//
// The pages serve one GPU and note that in a datacenter a fast interconnect
// hides moving experts between devices ([ainew] "UC バークレーと MIT、MoE
// モデルを一般ハードウェアで動かす推論エンジン「FreeToken」公開", opening
// paragraph). Here the experts stay put and the routed rows move: a device
// orders its routed rows by expert (the stable permutation of the router,
// so each owner's rows form one block), sends each block to its owner, the
// owner runs its experts on the rows (ft_moe_expert_rows) and sends the fp32
// outputs back, and the device combines them in rank order, as on one GPU.
//
//   ft_ep_pack     ids -> sanitised ids, stable permutation (the router's
//                  permutation kernels), rows and expert ids in sorted order,
//                  rows per owner
//   ft_ep_combine  y[t] = sum_j w[t,j] Y[inv[t*k+j]] over the returned rows
//   rows_in        (owner side) global expert ids -> local ids, weight 1
#include <atomic>

#include "ft_internal.cuh"

namespace ft {

cudaError_t route_kernels_init();
void launch_combine_rows(const float* ybuf, const float* wts, const int32_t* inv, int T, int k, int d, bool out_f32,
                         void* y, cudaStream_t st);

namespace {

// ids_s[i] = ids[i] if 0 <= ids[i] < E, else E - 1 (counted in *bad).
__global__ void __launch_bounds__(256) ep_sanitize_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                          int32_t* __restrict__ ids_s, int32_t* bad) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= n) return;
  int e = ids[i];
  if (e < 0 || e >= E) {
    e = E - 1;
    if (bad) atomicAdd(bad, 1);
  }
  ids_s[i] = e;
}

// Row p of the send buffer = x[perm[p] / k]; its expert = ids_s[perm[p]].
// grid (n), 128 threads; a row is vecs 16-byte vectors.
__global__ void __launch_bounds__(128) ep_pack_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                                                           const int32_t* __restrict__ ids_s, int k, int vecs,
                                                           uint4* __restrict__ rows, int32_t* __restrict__ eids) {
  const int p = blockIdx.x;
  const int f = perm[p];
  const uint4* src = x + (size_t)(f / k) * vecs;
  uint4* dst = rows + (size_t)p * vecs;
  for (int i = threadIdx.x; i < vecs; i += 128) dst[i] = __ldg(src + i);
  if (threadIdx.x == 0) eids[p] = ids_s[f];
}

// counts[o] = rows whose expert is in owner o's block [o E/G, (o+1) E/G).
__global__ void ep_owner_counts_kernel(const int32_t* __restrict__ offsets, int E, int G, int64_t* __restrict__ counts) {
  const int o = threadIdx.x;
  if (o < G) counts[o] = (int64_t)offsets[(o + 1) * (E / G)] - offsets[o * (E / G)];
}

// Owner side: ids[i] = eids[i] - base (a bad id latches DERR_BAD_INDEX and
// is replaced by local expert 0), wts[i] = 1.
__global__ void __launch_bounds__(256) rows_in_kernel(const int32_t* __restrict__ eids, int n, int base, int E,
                                                      int32_t* __restrict__ ids, float* __restrict__ wts,
                                                      uint32_t* error) {
  const int i = blockIdx.x * 256 + threadIdx.x;
  if (i >= n) return;
  int e = eids[i] - base;
  if (e < 0 || e >= E) {
    atomicExch(error, (uint32_t)DERR_BAD_INDEX);
    e = 0;
  }
  ids[i] = e;
  wts[i] = 1.f;
}

constexpr size_t ALIGN = 256;
size_t up(size_t b) { return (b + ALIGN - 1) / ALIGN * ALIGN; }

// Scratch of ft_ep_pack: sanitised ids [n], counts [E], offsets [E+1],
// perm [n], per-chunk counts of the multi-CTA permutation.
struct PackScratch {
  size_t ids, counts, offsets, perm, chunks, total;
};
PackScratch pack_layout(int n, int E) {
  PackScratch s;
  s.ids = 0;
  s.counts = s.ids + up(sizeof(int32_t) * (size_t)n);
  s.offsets = s.counts + up(sizeof(int32_t) * (size_t)E);
  s.perm = s.offsets + up(sizeof(int32_t) * (size_t)(E + 1));
  s.chunks = s.perm + up(sizeof(int32_t) * (size_t)n);
  s.total = s.chunks + up(sizeof(int32_t) * perm_chunks_ints(n, E));
  return s;
}

constexpr int MAX_DEVICES = 64;
std::atomic<int> g_attr_done[MAX_DEVICES];

}  // namespace

void launch_rows_in(const int32_t* eids, int n, int base, int E, DevState& ds, cudaStream_t st) {
  rows_in_kernel<<<(n + 255) / 256, 256, 0, st>>>(eids, n, base, E, ds.ids, ds.wts, ds.error);
}

}  // namespace ft

extern "C" ft_status ft_ep_pack_scratch_bytes(int32_t T, int32_t top_k, int32_t n_experts, uint64_t* out) {
  using namespace ft;
  if (!out || T < 0 || top_k < 1 || top_k > MAX_K || n_experts < 1 || n_experts > MAX_E) return FT_EINVAL;
  *out = pack_layout(T * top_k, n_experts).total;
  return FT_OK;
}

extern "C" ft_status ft_ep_pack(const int32_t* ids, int32_t T, int32_t top_k, int32_t n_experts, int32_t n_owners,
                                const void* x, int32_t d_model, int32_t wtype, void* rows, int32_t* eids,
                                int64_t* owner_counts, int32_t* inv, int32_t* bad_ids, void* scratch,
                                uint64_t scratch_bytes, void* stream) {
  using namespace ft;
  if (T < 0 || top_k < 1 || top_k > MAX_K || n_experts < 1 || n_experts > MAX_E || n_owners < 1 ||
      n_owners > n_experts || n_experts % n_owners || d_model < 8 || d_model % 8 ||
      (wtype != FT_W_F32 && wtype != FT_W_BF16 && wtype != FT_W_NVFP4) || !owner_counts)
    return FT_EINVAL;
  const cudaStream_t st = (cudaStream_t)stream;
  if (bad_ids && cudaMemsetAsync(bad_ids, 0, sizeof(int32_t), st) != cudaSuccess) return FT_ECUDA;
  if (T == 0) return cudaMemsetAsync(owner_counts, 0, sizeof(int64_t) * n_owners, st) == cudaSuccess ? FT_OK : FT_ECUDA;
  const int n = T * top_k;
  const PackScratch L = pack_layout(n, n_experts);
  if (!ids || !x || !rows || !eids || !inv || !scratch || scratch_bytes < L.total) return FT_EINVAL;
  if (((uintptr_t)x | (uintptr_t)rows) & 15 || (uintptr_t)scratch & (ALIGN - 1)) return FT_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return FT_ECUDA;
  if (!g_attr_done[dev].load(std::memory_order_acquire)) {  // shared-memory limits of the permutation kernels
    if (route_kernels_init() != cudaSuccess) return FT_ECUDA;
    g_attr_done[dev].store(1, std::memory_order_release);
  }
  uint8_t* s = static_cast<uint8_t*>(scratch);
  DevState ds{};
  ds.ids = reinterpret_cast<int32_t*>(s + L.ids);
  ds.counts = reinterpret_cast<int32_t*>(s + L.counts);
  ds.offsets = reinterpret_cast<int32_t*>(s + L.offsets);
  ds.perm = reinterpret_cast<int32_t*>(s + L.perm);
  ds.perm_chunks = reinterpret_cast<int32_t*>(s + L.chunks);
  ds.inv = inv;
  Shape sh{};
  sh.E = n_experts;
  sh.k = top_k;
  ep_sanitize_kernel<<<(n + 255) / 256, 256, 0, st>>>(ids, n, n_experts, ds.ids, bad_ids);
  launch_permute(sh, T, ds, st);
  const int esize = wtype == FT_W_F32 ? 4 : 2;
  ep_pack_rows_kernel<<<n, 128, 0, st>>>(static_cast<const uint4*>(x), ds.perm, ds.ids, top_k,
                                         d_model * esize / 16, static_cast<uint4*>(rows), eids);
  ep_owner_counts_kernel<<<1, 64 * ((n_owners + 63) / 64), 0, st>>>(ds.offsets, n_experts, n_owners, owner_counts);
  return cudaGetLastError() == cudaSuccess ? FT_OK : FT_ECUDA;
}

extern "C" ft_status ft_ep_combine(const float* y_rows, const float* w, const int32_t* inv, int32_t T, int32_t top_k,
                                   int32_t d_model, int32_t wtype, void* y, void* stream) {
  using namespace ft;
  if (T < 0 || top_k < 1 || top_k > MAX_K || d_model < 4 || d_model % 4 ||
      (wtype != FT_W_F32 && wtype != FT_W_BF16 && wtype != FT_W_NVFP4))
    return FT_EINVAL;
  if (T == 0) return FT_OK;
  if (!y_rows || !w || !inv || !y || y == (const void*)y_rows) return FT_EINVAL;
  if (((uintptr_t)y_rows | (uintptr_t)y) & 15) return FT_EINVAL;
  launch_combine_rows(y_rows, w, inv, T, top_k, d_model, wtype == FT_W_F32, y, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? FT_OK : FT_ECUDA;
}
