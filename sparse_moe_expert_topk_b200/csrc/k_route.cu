// Router of one MoE layer: logits, top-k with softmax weights, and the stable
// token -> expert permutation.
//
// Each token passes through k of the layer's E experts ([paperlens]
// "MoEは扉を開けると同時に、別の扉を閉める", paper §1). The pages do not give the
// router function; this follows the reading documented with the C ABI:
// logits s = x W_r^T + b in fp32, the k largest logits (equal logits -> lower
// expert index), softmax over those k.
#include <atomic>

#include <cooperative_groups.h>

#include "f16_scale.cuh"
#include "lookup_body.cuh"

namespace ft {

namespace {

__device__ __forceinline__ void to_f32x8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Logits for 8 experts (one warp each) x up to TT tokens per CTA.
// grid: (ceil(E/8), ceil(T/TT)); block 256.
template <typename AT, int TT>
__global__ void __launch_bounds__(256) router_scores_kernel(const AT* __restrict__ x, const AT* __restrict__ wr,
                                                            const float* __restrict__ bias, int bias_per_token,
                                                            int T, int E, int d, float* __restrict__ scores) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  const int t0 = blockIdx.y * TT;
  if (e >= E) return;
  const int nt = min(TT, T - t0);
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) acc[t] = 0.f;
  constexpr int VN = 16 / sizeof(AT);  // elements per 16-byte vector
  const int nv = d / VN;
  const uint4* wrow = reinterpret_cast<const uint4*>(wr + (size_t)e * d);
  for (int v = lane; v < nv; v += 32) {
    const uint4 wv = __ldg(wrow + v);
#pragma unroll
    for (int t = 0; t < TT; ++t) {
      if (t < nt) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * d) + v);
        if constexpr (sizeof(AT) == 2) {
          float wf[8], xf[8];
          to_f32x8(wv, wf);
          to_f32x8(xv, xf);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[t] = fmaf(wf[i], xf[i], acc[t]);
        } else {
          acc[t] = fmaf(__uint_as_float(wv.x), __uint_as_float(xv.x), acc[t]);
          acc[t] = fmaf(__uint_as_float(wv.y), __uint_as_float(xv.y), acc[t]);
          acc[t] = fmaf(__uint_as_float(wv.z), __uint_as_float(xv.z), acc[t]);
          acc[t] = fmaf(__uint_as_float(wv.w), __uint_as_float(xv.w), acc[t]);
        }
      }
    }
  }
#pragma unroll
  for (int t = 0; t < TT; ++t) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
  }
  if (lane < nt) {
    float a = 0.f;
#pragma unroll
    for (int t = 0; t < TT; ++t)
      if (t == lane) a = acc[t];
    const int tt = t0 + lane;
    float b = 0.f;
    if (bias) b = bias_per_token ? bias[(size_t)tt * E + e] : bias[e];
    scores[(size_t)tt * E + e] = a + b;
  }
}

// Orderable 64-bit key of a logit and its expert: a larger logit gives a
// larger key, equal logits (+0 and -0 are equal) the lower expert index; a NaN
// logit sorts below every number. Key 0 is never a valid key.
__device__ __forceinline__ unsigned long long topk_key(float v, int e) {
  uint32_t u = __float_as_uint(v + 0.0f);  // -0 -> +0
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  if (v != v) u = 0;
  return ((unsigned long long)u << 32) | (0xFFFFFFFFu - (uint32_t)e);
}
__device__ __forceinline__ float topk_key_value(unsigned long long key) {
  const uint32_t t = (uint32_t)(key >> 32);
  return __uint_as_float((t & 0x80000000u) ? (t & 0x7FFFFFFFu) : ~t);
}
__device__ __forceinline__ int topk_key_expert(unsigned long long key) {
  return (int)(0xFFFFFFFFu - (uint32_t)key);
}

// k rounds of a warp-wide maximum over the keys of E experts (expert
// i*32 + lane in lane, slot i); lane j gets the j-th largest key.
template <int PER, bool SHARED>
__device__ __forceinline__ unsigned long long topk_keys(const float* __restrict__ s, int E, int k, int lane,
                                                        unsigned long long& top) {
  unsigned long long key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = i * 32 + lane;
    float v = 0.f;
    if (e < E) {
      if constexpr (SHARED)
        v = s[e];
      else
        v = __ldcg(s + e);  // L2: in the fused kernel other CTAs wrote these
    }
    key[i] = e < E ? topk_key(v, e) : 0ull;
  }
  unsigned long long mine = 0;
  for (int j = 0; j < k; ++j) {
    unsigned long long b = key[0];
#pragma unroll
    for (int i = 1; i < PER; ++i) b = key[i] > b ? key[i] : b;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b, o);
      b = ob > b ? ob : b;
    }
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (key[i] == b) key[i] = 0;  // keys are unique: only the owner's entry matches
    if (lane == j) mine = b;
    if (j == 0) top = b;
  }
  return mine;
}

// One warp per token: the k largest logits (larger first, equal logits ->
// lower index), as k rounds of a warp maximum over (logit, index) keys, then
// softmax over the chosen k. SHARED: the scores are in this CTA's shared
// memory (the cluster routing), else in global memory, read through L2
// (other CTAs of the same launch may have written them). ids_sh, if set,
// receives a copy of the ids (shared memory).
template <bool SHARED = false>
__device__ __forceinline__ void topk_token(const float* __restrict__ scores, int warp, int E, int k,
                                           int32_t* __restrict__ ids, float* __restrict__ wts, int lane,
                                           int32_t* ids_sh = nullptr) {
  const float* s = scores + (size_t)warp * E;  // warp = token index
  unsigned long long top = 0;
  const unsigned long long mine =
      E <= 256 ? topk_keys<8, SHARED>(s, E, k, lane, top) : topk_keys<MAX_E / 32, SHARED>(s, E, k, lane, top);
  const float my_s = topk_key_value(mine), top0 = topk_key_value(top);
  const int my_e = topk_key_expert(mine);
  const float ex = lane < k ? expf(my_s - top0) : 0.f;
  float den = 0.f;
  for (int j = 0; j < k; ++j) den += __shfl_sync(0xffffffffu, ex, j);  // rank order
  if (lane < k) {
    ids[(size_t)warp * k + lane] = my_e;
    wts[(size_t)warp * k + lane] = ex / den;
    if (ids_sh) ids_sh[warp * k + lane] = my_e;
  }
}

__global__ void __launch_bounds__(256) topk_softmax_kernel(const float* __restrict__ scores, int T, int E, int k,
                                                           int32_t* __restrict__ ids, float* __restrict__ wts) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (warp >= T) return;
  topk_token(scores, warp, E, k, ids, wts, threadIdx.x & 31);
}

// Stable counting sort of the n = T*k routing ids by expert, one CTA of 1024
// threads. Sorted order = (expert, flat index t*k+j). Within a 1024-entry
// chunk a thread's rank among equal experts comes from __match_any_sync
// inside its warp plus the counts of the lower warps.
__device__ __forceinline__ void permute_body(const int32_t* __restrict__ ids, int n, int E,
                                             int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                             int32_t* __restrict__ perm, int32_t* __restrict__ inv,
                                             int32_t* smem) {
  int32_t* wcnt = smem;                // [32][E]
  int32_t* run = smem + 32 * E;        // [E] next free position per expert
  int32_t* tot = run + E;              // [E] per-chunk totals
  int32_t* cnt = tot + E;              // [E] counts (kept after the call)
  int32_t* off = cnt + E;              // [E] offsets (kept after the call)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e < E; e += 1024) cnt[e] = 0;
  __syncthreads();
  if (n <= 32) {
    // one warp holds every entry (decode at a few tokens): an entry's place
    // among equal experts is the number of earlier lanes with its expert,
    // the same stable order as the general path below
    if (warp == 0) {
      const bool valid = lane < n;
      const int e = valid ? ids[lane] : E;
      const unsigned same = __match_any_sync(0xffffffffu, e);
      const int rank = __popc(same & ((1u << lane) - 1u));
      if (valid && rank == 0) cnt[e] = __popc(same);
      __syncwarp();
      constexpr int PER = MAX_E / 32;
      int local[PER], sum = 0;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int x = lane * PER + i;
        local[i] = x < E ? cnt[x] : 0;
        sum += local[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int base = incl - sum;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int x = lane * PER + i;
        if (x < E) {
          off[x] = base;
          offsets[x] = base;
          counts[x] = local[i];
        }
        base += local[i];
      }
      if (lane == 31) offsets[E] = incl;
      __syncwarp();
      if (valid) {
        const int pos = off[e] + rank;
        perm[pos] = lane;
        inv[lane] = pos;
      }
    }
    return;
  }
  for (int i = tid; i < n; i += 1024) atomicAdd(&cnt[ids[i]], 1);
  __syncthreads();
  if (warp == 0) {  // exclusive scan of cnt over E <= 512 entries, 16 per lane
    constexpr int PER = MAX_E / 32;
    int local[PER], s = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      local[i] = e < E ? cnt[e] : 0;
      s += local[i];
    }
    int incl = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int base = incl - s;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      if (e < E) {
        run[e] = base;
        off[e] = base;
        offsets[e] = base;
        counts[e] = local[i];
      }
      base += local[i];
    }
    if (lane == 31) offsets[E] = incl;
  }
  __syncthreads();
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int base = 0; base < n; base += 1024) {
    for (int i = tid; i < 32 * E; i += 1024) wcnt[i] = 0;
    __syncthreads();
    const int i = base + tid;
    const bool valid = i < n;
    const int e = valid ? ids[i] : E;  // E = sentinel for padding lanes
    const unsigned same = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(same & lt_mask);
    if (valid && rank == 0) wcnt[warp * E + e] = __popc(same);
    __syncthreads();
    for (int x = tid; x < E; x += 1024) {
      int r = 0;
      for (int w = 0; w < 32; ++w) {
        const int c = wcnt[w * E + x];
        wcnt[w * E + x] = r;
        r += c;
      }
      tot[x] = r;
    }
    __syncthreads();
    if (valid) {
      const int pos = run[e] + wcnt[warp * E + e] + rank;
      perm[pos] = i;
      inv[i] = pos;
    }
    __syncthreads();
    for (int x = tid; x < E; x += 1024) run[x] += tot[x];
    __syncthreads();
  }
}

__global__ void __launch_bounds__(1024) permute_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                       int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ int32_t smem[];
  permute_body(ids, n, E, counts, offsets, perm, inv, smem);
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// BF16 logits of 16 experts (rows e0..e0+15 of W_r) for all T tokens, by one
// CTA of 32 warps: warp w takes K steps [w*S/32, (w+1)*S/32) of 32 values;
// lane (g, q) feeds 16 bytes of rows g and g+8 to the MMA as its A fragment and
// the matching 16 bytes of token rows as the B fragment (the lane-dependent K
// order is the same on both sides). Partial sums are reduced in warp order in
// shared memory (red: 32 warps x 8 values x 32 lanes floats).
__device__ void logits_bf16_block(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ wr,
                                  const float* __restrict__ bias, int bias_per_token, int T, int E, int d, int e0,
                                  float* __restrict__ scores, float* red) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int steps = d / 32;
  const int s0 = (warp * steps) / 32, s1 = ((warp + 1) * steps) / 32;
  const int ra = min(e0 + g, E - 1), rb = min(e0 + g + 8, E - 1);  // clamp: rows past E are not stored
  const uint8_t* pa = reinterpret_cast<const uint8_t*>(wr + (size_t)ra * d) + q * 16;
  const uint8_t* pb = reinterpret_cast<const uint8_t*>(wr + (size_t)rb * d) + q * 16;
  for (int t0 = 0; t0 < T; t0 += 16) {
    const int nt = min(16, T - t0);
    const __nv_bfloat16* xr0 = x + (size_t)(t0 + (g < nt ? g : 0)) * d;
    const __nv_bfloat16* xr1 = x + (size_t)(t0 + (g + 8 < nt ? g + 8 : 0)) * d;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    // RU steps of router rows in flight, then their MMAs in step order (the
    // order, and so every logit, is the one-step loop's)
    constexpr int RU = 4;
    for (int sb = s0; sb < s1; sb += RU) {
      uint4 wa[RU], wb[RU];
#pragma unroll
      for (int u = 0; u < RU; ++u) {
        const int s = sb + u < s1 ? sb + u : s1 - 1;
        wa[u] = __ldg(reinterpret_cast<const uint4*>(pa + (size_t)s * 64));
        wb[u] = __ldg(reinterpret_cast<const uint4*>(pb + (size_t)s * 64));
      }
#pragma unroll
      for (int u = 0; u < RU; ++u) {
        if (sb + u >= s1) break;
        const int s = sb + u;
        const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(xr0 + s * 32 + q * 8));
        mma_bf16_16816(acc[0], wa[u].x, wb[u].x, wa[u].y, wb[u].y, x0.x, x0.y);
        mma_bf16_16816(acc[0], wa[u].z, wb[u].z, wa[u].w, wb[u].w, x0.z, x0.w);
        if (nt > 8) {
          const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(xr1 + s * 32 + q * 8));
          mma_bf16_16816(acc[1], wa[u].x, wb[u].x, wa[u].y, wb[u].y, x1.x, x1.y);
          mma_bf16_16816(acc[1], wa[u].z, wb[u].z, wa[u].w, wb[u].w, x1.z, x1.w);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int c = 0; c < 4; ++c) red[(warp * 8 + t * 4 + c) * 32 + lane] = acc[t][c];
    __syncthreads();
    // thread i < 256 sums accumulator element i over the 32 warps, in warp order
    const int n_out = nt > 8 ? 256 : 128;
    if ((int)threadIdx.x < n_out) {
      const int i = threadIdx.x, t = i >> 7, c = (i >> 5) & 3, l = i & 31;
      float v = 0.f;
#pragma unroll 8
      for (int w = 0; w < 32; ++w) v += red[w * 256 + i];
      // element c of lane l: c = 0,1 expert e0+g, tokens 2q, 2q+1; c = 2,3 expert e0+g+8
      const int tt = t * 8 + 2 * (l & 3) + (c & 1);
      const int tok = t0 + tt;
      const int e = e0 + (l >> 2) + (c >> 1) * 8;
      if (tt < nt && e < E) {
        float b = 0.f;
        if (bias) b = bias_per_token ? bias[(size_t)tok * E + e] : bias[e];
        scores[(size_t)tok * E + e] = v + b;
      }
    }
    __syncthreads();
  }
}

// BF16 logits of up to 32 tokens by the fused decode routing's device
// function, as a kernel of its own: the router of every other small-batch
// call (a prefill of few tokens, the allocation-free entry point) then sums
// each logit in exactly the order the fused decode routing does. grid
// ceil(E/16), 1024 threads, dynamic shared memory for the warp partial sums.
__global__ void __launch_bounds__(1024) router_small_kernel(const __nv_bfloat16* __restrict__ x,
                                                            const __nv_bfloat16* __restrict__ wr,
                                                            const float* __restrict__ bias, int bias_per_token,
                                                            int T, int E, int d, float* __restrict__ scores) {
  extern __shared__ float red_small[];
  logits_bf16_block(x, wr, bias, bias_per_token, T, E, d, blockIdx.x * 16, scores, red_small);
}
constexpr int SMALL_RED_BYTES = sizeof(float) * 32 * 8 * 32;

// BF16 router logits for many tokens (prefill) on mma.sync: CTA = 16 experts
// x 64 tokens, warp w takes tokens t0+16w .. +16 over the full K (steps of 32
// K values, lane-permuted K as in logits_bf16_block; the four warps read the
// same W_r rows, which L1 serves). grid (ceil(E/16), ceil(T/64)), 128 threads.
__global__ void __launch_bounds__(128) router_mma_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const __nv_bfloat16* __restrict__ wr,
                                                         const float* __restrict__ bias, int bias_per_token, int T,
                                                         int E, int d, float* __restrict__ scores) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int e0 = blockIdx.x * 16, t0 = blockIdx.y * 64 + warp * 16;
  if (t0 >= T) return;
  const int nt = min(16, T - t0);
  const int ra = min(e0 + g, E - 1), rb = min(e0 + g + 8, E - 1);
  const uint8_t* pa = reinterpret_cast<const uint8_t*>(wr + (size_t)ra * d) + q * 16;
  const uint8_t* pb = reinterpret_cast<const uint8_t*>(wr + (size_t)rb * d) + q * 16;
  const __nv_bfloat16* xr0 = x + (size_t)(t0 + (g < nt ? g : 0)) * d + q * 8;
  const __nv_bfloat16* xr1 = x + (size_t)(t0 + (g + 8 < nt ? g + 8 : 0)) * d + q * 8;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  const int steps = d / 32;
  constexpr int U = 4;
  for (int s = 0; s < steps; s += U) {
    uint4 wa[U], wb[U], x0[U], x1[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ss = s + u < steps ? s + u : steps - 1;
      wa[u] = __ldg(reinterpret_cast<const uint4*>(pa + (size_t)ss * 64));
      wb[u] = __ldg(reinterpret_cast<const uint4*>(pb + (size_t)ss * 64));
      x0[u] = __ldg(reinterpret_cast<const uint4*>(xr0 + ss * 32));
      x1[u] = __ldg(reinterpret_cast<const uint4*>(xr1 + ss * 32));
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (s + u < steps) {
        mma_bf16_16816(acc[0], wa[u].x, wb[u].x, wa[u].y, wb[u].y, x0[u].x, x0[u].y);
        mma_bf16_16816(acc[0], wa[u].z, wb[u].z, wa[u].w, wb[u].w, x0[u].z, x0[u].w);
        mma_bf16_16816(acc[1], wa[u].x, wb[u].x, wa[u].y, wb[u].y, x1[u].x, x1[u].y);
        mma_bf16_16816(acc[1], wa[u].z, wb[u].z, wa[u].w, wb[u].w, x1[u].z, x1[u].w);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < 2; ++t)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = t * 8 + 2 * q + (c & 1);  // token within the tile
      const int e = e0 + g + (c >> 1) * 8;
      if (j < nt && e < E) {
        const int tok = t0 + j;
        float b = 0.f;
        if (bias) b = bias_per_token ? bias[(size_t)tok * E + e] : bias[e];
        scores[(size_t)tok * E + e] = acc[t][c] + b;
      }
    }
}

// After a fused routing's lookup: the decode prefetch batch of the next layer
// (pf.layer >= 0; it reads that layer's recorded routing counts), then this
// call's counts (s_counts, shared memory) become this layer's record. The
// record is written after the prefetch batch has read its counts, so a
// one-layer model prefetches from its previous call, not from this one.
__device__ __forceinline__ void route_tail(const LookupArgs& la, const LookupArgs& pf, int E, long long C,
                                           size_t slot_bytes, DevState& ds, const int32_t* s_counts) {
  if (pf.layer >= 0) {
    __syncthreads();
    lookup_detail::lookup_body(pf, E, C, slot_bytes, ds);
  }
  if (la.record_counts) {
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) la.record_counts[e] = s_counts[e];
  }
}

// Decode routing in one launch (T <= 32 tokens): CTAs of 32 warps compute the
// logits of 16 (BF16) or 32 (fp32) experts each; the last CTA to finish
// (ticket on ds.route_ctr) runs top-k + softmax, the stable permutation and
// the LRU lookup of the layer. Same device code as the separate kernels, so
// the results are the same. With x16 set (NVFP4 experts), CTA b also writes
// the f16 copy of tokens b, b + grid, ... (to_f16_scaled_row, as the
// standalone conversion kernel does).
template <typename AT>
__global__ void __launch_bounds__(1024) route_decode_kernel(const AT* __restrict__ x, const AT* __restrict__ wr,
                                                            const float* __restrict__ bias, int bias_per_token, int T,
                                                            int E, int d, int k, LookupArgs la, LookupArgs pf,
                                                            long long C, size_t slot_bytes, DevState ds, __half* x16,
                                                            float* xscale) {
  extern __shared__ int32_t smem[];
  __shared__ int s_last;
  __shared__ float s_max[32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if constexpr (sizeof(AT) == 2) {
    // BF16: 16 experts per CTA on the tensor cores (red reuses the dynamic smem)
    logits_bf16_block(x, wr, bias, bias_per_token, T, E, d, blockIdx.x * 16, ds.scores,
                      reinterpret_cast<float*>(smem));
  } else if (blockIdx.x * 32 + warp < E) {
    const int e = blockIdx.x * 32 + warp;
    constexpr int VN = 16 / sizeof(AT);
    const int nv = d / VN;
    const uint4* wrow = reinterpret_cast<const uint4*>(wr + (size_t)e * d);
    for (int t0 = 0; t0 < T; t0 += 8) {
      const int nt = min(8, T - t0);
      float acc[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) acc[t] = 0.f;
      for (int v = lane; v < nv; v += 32) {
        const uint4 wv = __ldg(wrow + v);
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (t < nt) {
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + t) * d) + v);
            if constexpr (sizeof(AT) == 2) {
              float wf[8], xf[8];
              to_f32x8(wv, wf);
              to_f32x8(xv, xf);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[t] = fmaf(wf[i], xf[i], acc[t]);
            } else {
              acc[t] = fmaf(__uint_as_float(wv.x), __uint_as_float(xv.x), acc[t]);
              acc[t] = fmaf(__uint_as_float(wv.y), __uint_as_float(xv.y), acc[t]);
              acc[t] = fmaf(__uint_as_float(wv.z), __uint_as_float(xv.z), acc[t]);
              acc[t] = fmaf(__uint_as_float(wv.w), __uint_as_float(xv.w), acc[t]);
            }
          }
        }
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
      }
      if (lane < nt) {
        float a = 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t)
          if (t == lane) a = acc[t];
        const int tt = t0 + lane;
        float b = 0.f;
        if (bias) b = bias_per_token ? bias[(size_t)tt * E + e] : bias[e];
        ds.scores[(size_t)tt * E + e] = a + b;
      }
    }
  }
  if constexpr (sizeof(AT) == 2) {
    if (x16) {
      for (int t = blockIdx.x; t < T; t += gridDim.x)
        to_f16_scaled_row<1024>(reinterpret_cast<const __nv_bfloat16*>(x) + (size_t)t * d, d, x16 + (size_t)t * d,
                                xscale + t, s_max);
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ds.route_ctr, 1) == (int)gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  if (warp < T) topk_token(ds.scores, warp, E, k, ds.ids, ds.wts, lane);
  __syncthreads();
  permute_body(ds.ids, T * k, E, ds.counts, ds.offsets, ds.perm, ds.inv, smem);
  __syncthreads();
  // counts and offsets are still in this CTA's shared memory (permute_body)
  lookup_detail::lookup_body(la, E, C, slot_bytes, ds, smem + 34 * E, smem + 35 * E);
  route_tail(la, pf, E, C, slot_bytes, ds, smem + 34 * E);
  if (threadIdx.x == 0) *ds.route_ctr = 0;  // ready for the next call
}

// Decode routing (T <= 32, BF16 router, E <= 256) as one thread-block
// cluster of ceil(E/16) CTAs: CTA r computes the logits of experts 16r ..
// 16r+15 (logits_bf16_block, the same sums as the other small-batch router
// paths) and stores them straight into the shared memory of CTA 0; one
// cluster barrier publishes them, and CTA 0 runs top-k + softmax, the stable
// permutation and the LRU lookup with the scores and ids in its own shared
// memory. No global round trip, fence or ticket between the logits and the
// lookup. With x16 set (NVFP4 experts), CTA r also writes the f16 copy of
// tokens r, r + grid, ...
// Dynamic shared memory: [0, sc_off) the logits' partial sums and later the
// permutation's tables, [sc_off, sc_off + 4*T*E) the scores (CTA 0's).
__global__ void __launch_bounds__(1024) route_cluster_kernel(const __nv_bfloat16* __restrict__ x,
                                                             const __nv_bfloat16* __restrict__ wr,
                                                             const float* __restrict__ bias, int bias_per_token, int T,
                                                             int E, int d, int k, LookupArgs la, LookupArgs pf,
                                                             long long C, size_t slot_bytes, DevState ds, __half* x16,
                                                             float* xscale, int sc_off) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) int32_t smem[];
  __shared__ float s_max[32];
  __shared__ int32_t s_ids[32 * MAX_K];
  cg::cluster_group cl = cg::this_cluster();
  const unsigned rank = cl.block_rank();
  float* scores = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(smem) + sc_off);
  float* scores0 = cl.map_shared_rank(scores, 0);
  cl.sync();  // every CTA of the cluster runs before its shared memory is written
  logits_bf16_block(x, wr, bias, bias_per_token, T, E, d, (int)rank * 16, scores0, reinterpret_cast<float*>(smem));
  if (x16) {
    for (int t = (int)rank; t < T; t += (int)cl.num_blocks())
      to_f16_scaled_row<1024>(x + (size_t)t * d, d, x16 + (size_t)t * d, xscale + t, s_max);
  }
  cl.sync();  // the scores are in CTA 0
  if (rank != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp < T) topk_token<true>(scores, warp, E, k, ds.ids, ds.wts, lane, s_ids);
  __syncthreads();
  permute_body(s_ids, T * k, E, ds.counts, ds.offsets, ds.perm, ds.inv, smem);
  __syncthreads();
  // counts and offsets are still in this CTA's shared memory (permute_body)
  lookup_detail::lookup_body(la, E, C, slot_bytes, ds, smem + 34 * E, smem + 35 * E);
  route_tail(la, pf, E, C, slot_bytes, ds, smem + 34 * E);
}

bool g_route_cluster = false;  // cluster launches of 16 x 1024 threads fit on this device

}  // namespace

void launch_router_scores(const Shape& sh, const void* x, const void* w_router, const float* bias, int bias_per_token,
                          int T, float* scores, cudaStream_t st) {
  if (sh.wtype != FT_W_F32 && T <= 32 && sh.d % 32 == 0) {
    router_small_kernel<<<(sh.E + 15) / 16, 1024, SMALL_RED_BYTES, st>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, bias, bias_per_token, T, sh.E, sh.d, scores);
    return;
  }
  if (sh.wtype != FT_W_F32 && T > 32 && sh.d % 32 == 0) {
    dim3 grid((sh.E + 15) / 16, (T + 63) / 64);
    router_mma_kernel<<<grid, 128, 0, st>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, bias,
                                            bias_per_token, T, sh.E, sh.d, scores);
    return;
  }
  constexpr int TT = 8;
  dim3 grid((sh.E + 7) / 8, (T + TT - 1) / TT);
  if (sh.wtype == FT_W_F32)
    router_scores_kernel<float, TT><<<grid, 256, 0, st>>>((const float*)x, (const float*)w_router, bias,
                                                          bias_per_token, T, sh.E, sh.d, scores);
  else
    router_scores_kernel<__nv_bfloat16, TT><<<grid, 256, 0, st>>>((const __nv_bfloat16*)x,
                                                                  (const __nv_bfloat16*)w_router, bias,
                                                                  bias_per_token, T, sh.E, sh.d, scores);
}

// ---------------------------------------------------------------------------
// The same stable counting sort over many CTAs, for large T*k: chunks of 1024
// entries; (1) each chunk counts its experts, (2) one CTA turns the counts into
// the global offsets and, per (expert, chunk), the position of the chunk's
// first entry of that expert (expert-major, chunks in order: stable), (3) each
// chunk ranks its entries among equal experts as permute_body does and
// scatters them.
// ---------------------------------------------------------------------------
constexpr int PCHUNK = 1024;

__global__ void __launch_bounds__(PCHUNK) perm_hist_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                           int32_t* __restrict__ chunk) {
  extern __shared__ int32_t cnt[];  // [E]
  const int tid = threadIdx.x;
  for (int e = tid; e < E; e += PCHUNK) cnt[e] = 0;
  __syncthreads();
  const int i = blockIdx.x * PCHUNK + tid;
  if (i < n) atomicAdd(&cnt[ids[i]], 1);
  __syncthreads();
  for (int e = tid; e < E; e += PCHUNK) chunk[(size_t)blockIdx.x * E + e] = cnt[e];
}

// One CTA of MAX_E threads, thread e = expert e.
__global__ void __launch_bounds__(MAX_E) perm_scan_kernel(int32_t* __restrict__ chunk, int nch, int E,
                                                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int wsum[MAX_E / 32];
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  int tot = 0;
  if (e < E)
    for (int c = 0; c < nch; ++c) tot += chunk[(size_t)c * E + e];
  int incl = tot;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int base = incl - tot;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  if (e < E) {
    counts[e] = tot;
    offsets[e] = base;
    if (e == E - 1) offsets[E] = base + tot;
    int run = base;
    for (int c = 0; c < nch; ++c) {
      const int v = chunk[(size_t)c * E + e];
      chunk[(size_t)c * E + e] = run;
      run += v;
    }
  }
}

__global__ void __launch_bounds__(PCHUNK) perm_scatter_kernel(const int32_t* __restrict__ ids, int n, int E,
                                                              const int32_t* __restrict__ chunk,
                                                              int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  extern __shared__ int32_t wcnt[];  // [32][E]: per warp count, then exclusive prefix over the warps
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int x = tid; x < 32 * E; x += PCHUNK) wcnt[x] = 0;
  __syncthreads();
  const int i = blockIdx.x * PCHUNK + tid;
  const bool valid = i < n;
  const int e = valid ? ids[i] : E;  // E = sentinel for padding lanes
  const unsigned same = __match_any_sync(0xffffffffu, e);
  const int rank = __popc(same & ((1u << lane) - 1u));
  if (valid && rank == 0) wcnt[warp * E + e] = __popc(same);
  __syncthreads();
  for (int x = tid; x < E; x += PCHUNK) {
    int r = 0;
    for (int w = 0; w < 32; ++w) {
      const int c = wcnt[w * E + x];
      wcnt[w * E + x] = r;
      r += c;
    }
  }
  __syncthreads();
  if (valid) {
    const int pos = chunk[(size_t)blockIdx.x * E + e] + wcnt[warp * E + e] + rank;
    perm[pos] = i;
    inv[i] = pos;
  }
}

size_t permute_smem_bytes(int E) { return sizeof(int32_t) * (size_t)(32 * E + 4 * E); }

void launch_topk(const Shape& sh, const float* scores, int T, DevState& ds, cudaStream_t st) {
  const int warps_per_cta = 8;
  topk_softmax_kernel<<<(T + warps_per_cta - 1) / warps_per_cta, 32 * warps_per_cta, 0, st>>>(
      scores, T, sh.E, sh.k, ds.ids, ds.wts);
}

int launch_permute(const Shape& sh, int T, DevState& ds, cudaStream_t st) {
  const int n = T * sh.k;
  if (n <= 2 * PCHUNK) {
    permute_kernel<<<1, 1024, permute_smem_bytes(sh.E), st>>>(ds.ids, n, sh.E, ds.counts, ds.offsets, ds.perm, ds.inv);
    return 1;
  }
  const int nch = (n + PCHUNK - 1) / PCHUNK;
  perm_hist_kernel<<<nch, PCHUNK, sizeof(int32_t) * sh.E, st>>>(ds.ids, n, sh.E, ds.perm_chunks);
  perm_scan_kernel<<<1, MAX_E, 0, st>>>(ds.perm_chunks, nch, sh.E, ds.counts, ds.offsets);
  perm_scatter_kernel<<<nch, PCHUNK, sizeof(int32_t) * 32 * sh.E, st>>>(ds.ids, n, sh.E, ds.perm_chunks, ds.perm,
                                                                         ds.inv);
  return 3;
}

size_t perm_chunks_ints(int max_entries, int E) { return (size_t)((max_entries + PCHUNK - 1) / PCHUNK) * E; }

// ---------------------------------------------------------------------------
// Router + top-k without any allocation (ft_route_topk_static in ft_moe.h).
// The logits scratch is this file-scope device array instead of a buffer the
// library or the caller allocates. Its host-side name is only a stand-in, so
// the device address is looked up once per device with cudaGetSymbolAddress
// and cached.
// ---------------------------------------------------------------------------
namespace {
constexpr int STATIC_MAX_TOKENS = FT_ROUTE_STATIC_MAX_TOKENS;
constexpr int MAX_DEVICES = 64;
static __device__ __align__(256) float g_static_scores[STATIC_MAX_TOKENS * MAX_E];
std::atomic<float*> g_static_ptr[MAX_DEVICES];
}  // namespace

}  // namespace ft

extern "C" ft_status ft_route_topk_static(const void* x_dev, const void* w_router_dev, const float* bias_dev,
                                          int32_t bias_per_token, int32_t T, int32_t n_experts, int32_t d_model,
                                          int32_t top_k, int32_t wtype, int32_t* ids_dev, float* w_dev,
                                          void* stream) {
  using namespace ft;
  if (T < 0 || T > STATIC_MAX_TOKENS || n_experts < 1 || n_experts > MAX_E || top_k < 1 || top_k > MAX_K ||
      top_k > n_experts || d_model < 64 || d_model % 64 || (wtype != FT_W_F32 && wtype != FT_W_BF16 &&
      wtype != FT_W_NVFP4))
    return FT_EINVAL;
  if (T == 0) return FT_OK;
  if (!x_dev || !w_router_dev || !ids_dev || !w_dev) return FT_EINVAL;
  if (((uintptr_t)x_dev | (uintptr_t)w_router_dev) & 15) return FT_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return FT_ECUDA;
  float* scores = g_static_ptr[dev].load(std::memory_order_acquire);
  if (!scores) {  // first call on this device: resolve the array's device address
    if (cudaGetSymbolAddress((void**)&scores, g_static_scores) != cudaSuccess || !scores) return FT_ECUDA;
    g_static_ptr[dev].store(scores, std::memory_order_release);
  }
  Shape sh{};
  sh.E = n_experts;
  sh.k = top_k;
  sh.d = d_model;
  sh.wtype = wtype;
  const cudaStream_t st = (cudaStream_t)stream;
  launch_router_scores(sh, x_dev, w_router_dev, bias_dev, bias_per_token, T, scores, st);
  const int warps_per_cta = 8;
  topk_softmax_kernel<<<(T + warps_per_cta - 1) / warps_per_cta, 32 * warps_per_cta, 0, st>>>(
      scores, T, n_experts, top_k, ids_dev, w_dev);
  return cudaGetLastError() == cudaSuccess ? FT_OK : FT_ECUDA;
}

namespace ft {

size_t route_decode_smem(int E) {
  const size_t red = sizeof(float) * 32 * 8 * 32;  // logits partial sums (BF16)
  const size_t perm = permute_smem_bytes(E);
  return red > perm ? red : perm;
}

static size_t route_cluster_sc_off(int E) {
  const size_t red = sizeof(float) * 32 * 8 * 32, perm = permute_smem_bytes(E);
  return ((red > perm ? red : perm) + 15) & ~size_t(15);
}
constexpr int CLUSTER_MAX_E = 256;  // 16 CTAs of 16 experts
constexpr int CLUSTER_MAX_T = 32;

void launch_route_decode(const Shape& sh, const void* x, const void* w_router, const float* bias, int bias_per_token,
                         int T, const LookupArgs& la, const LookupArgs& pf, DevState& ds, bool to_f16,
                         cudaStream_t st) {
  if (sh.wtype != FT_W_F32 && g_route_cluster && sh.E <= CLUSTER_MAX_E && T <= CLUSTER_MAX_T) {
    const int cs = (sh.E + 15) / 16;
    const int sc_off = (int)route_cluster_sc_off(sh.E);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cs, 1, 1);
    cfg.blockDim = dim3(1024, 1, 1);
    cfg.dynamicSmemBytes = sc_off + sizeof(float) * (size_t)T * sh.E;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, route_cluster_kernel, (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, bias,
                       bias_per_token, T, sh.E, sh.d, sh.k, la, pf, sh.C, sh.slot_bytes, ds,
                       to_f16 ? reinterpret_cast<__half*>(ds.x16) : nullptr, to_f16 ? ds.xscale : nullptr, sc_off);
    return;
  }
  const int grid = sh.wtype == FT_W_F32 ? (sh.E + 31) / 32 : (sh.E + 15) / 16;
  const size_t smem = route_decode_smem(sh.E);
  if (sh.wtype == FT_W_F32)
    route_decode_kernel<float><<<grid, 1024, smem, st>>>((const float*)x, (const float*)w_router, bias,
                                                         bias_per_token, T, sh.E, sh.d, sh.k, la, pf, sh.C,
                                                         sh.slot_bytes, ds, nullptr, nullptr);
  else
    route_decode_kernel<__nv_bfloat16><<<grid, 1024, smem, st>>>(
        (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, bias, bias_per_token, T, sh.E, sh.d, sh.k, la, pf,
        sh.C, sh.slot_bytes, ds, to_f16 ? reinterpret_cast<__half*>(ds.x16) : nullptr, to_f16 ? ds.xscale : nullptr);
}

// Dynamic shared-memory limits of the permutation and fused routing kernels,
// set for the largest supported E (MAX_E): the attribute is per kernel and
// process-wide, so a limit set for a small E would break the launches of a
// context (or ft_ep_pack call) with a larger one.
cudaError_t route_kernels_init() {
  const int E = MAX_E;
  const int smem = (int)permute_smem_bytes(E), smem_f = (int)route_decode_smem(E);
  cudaError_t e = cudaFuncSetAttribute(permute_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(perm_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(sizeof(int32_t) * 32 * E));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(router_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMALL_RED_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(route_decode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_f);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(route_decode_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem_f);
  // the cluster routing: 16 CTAs of 1024 threads (a non-portable cluster
  // size), used only if such a cluster fits on the device
  const int smem_c = (int)(route_cluster_sc_off(CLUSTER_MAX_E) + sizeof(float) * CLUSTER_MAX_T * CLUSTER_MAX_E);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(route_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_c);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(route_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1, 1);
    cfg.blockDim = dim3(1024, 1, 1);
    cfg.dynamicSmemBytes = smem_c;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 16;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t q = cudaOccupancyMaxActiveClusters(&n, route_cluster_kernel, &cfg);
    g_route_cluster = q == cudaSuccess && n >= 1;
    if (q != cudaSuccess) (void)cudaGetLastError();  // not fatal: the other routing kernel stays in use
  }
  return e;
}

}  // namespace ft
