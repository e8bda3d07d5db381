// Grouped GEMV over the routed experts of one layer call (decode path, and the
// on-demand prefill fallback), the fixed-order combine, and a zero-copy read
// probe.
//
// Small-batch decode is memory bound ([paperlens] "壁2: デコードのミスを「どう捌く
// か」が決まっていない", paper §2.2), so each expert's weights are streamed once
// with 128-bit loads and every loaded vector is used for all tokens of the
// chunk. The weight pointer of an expert is its HBM slot (hit / staged) or the
// device address of its blob in the mapped host pool (streamed: the misses
// the q* split leaves where the weights are, [techfeed]
// "帯域適応型実行（q*ポリシー）"). The kernel code, and with it the order of every
// floating-point reduction, is the same whatever the source, so the output of
// an expert does not depend on the cache state ([paperlens]
// "設計: 2階建てのエキスパート記憶", paper §3.3).
//
// Expert math (the reading documented with the C ABI): SwiGLU without biases,
// h = silu(W_gate x) * (W_up x), Y = W_down h, fp32 accumulation. NVFP4
// weights are decoded in registers: e2m1 code x e4m3 scale per 16 values x
// fp32 tensor scale per matrix.
#include "ft_internal.cuh"

namespace ft {

namespace {

constexpr int WARPS = 8;
constexpr int RW_GU = 2;    // gate rows (and as many up rows) per warp
constexpr int RW_DN = 4;    // down rows per warp
constexpr int U = 2;        // 16-byte vectors in flight per row stream and lane

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void bf16x8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// e2m1 magnitude bits placed in an fp32 exponent/mantissa and rescaled by 2^126:
// the 3 magnitude bits (e1 e0 m) at bits 24..22 give 2^(E-127) (1 + m/2) for
// E = e1e0 > 0 and m * 2^-127 for E = 0, i.e. the e2m1 value times 2^-126.
__device__ __forceinline__ float e2m1_f32(uint32_t nib) {
  const uint32_t bits = ((nib & 7u) << 22) | ((nib & 8u) << 28);
  return __uint_as_float(bits) * 8.507059173023462e37f;  // 2^126
}

// e4m3 (FN) byte -> fp32: normal codes shift into place with the exponent
// bias moved from 7 to 127; exponent 0 is subnormal (mantissa/8 * 2^-6).
__device__ __forceinline__ float e4m3_f32(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 24, ex = (b >> 3) & 0xFu, mn = b & 7u;
  if (ex == 0) return __uint_as_float(s) + (s ? -1.f : 1.f) * (float)mn * 0.001953125f;  // mn * 2^-9
  return __uint_as_float(s | ((ex + 120u) << 23) | (mn << 20));
}

// Activation row accessor: 8 consecutive elements starting at element i as fp32.
template <typename XT>
__device__ __forceinline__ void load_x8(const XT* row, int i, float (&f)[8]) {
  if constexpr (sizeof(XT) == 2) {
    bf16x8(__ldg(reinterpret_cast<const uint4*>(row + i)), f);
  } else {
    const float4 a = __ldg(reinterpret_cast<const float4*>(row + i));
    const float4 b = __ldg(reinterpret_cast<const float4*>(row + i) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}

// One 16-byte NVFP4 vector (32 codes, two 16-value scale blocks) of R rows
// against NT activation rows starting at element i0. Per token and row the
// partial sum of a 16-value block is scaled by its e4m3 scale.
template <typename XT, int R, int NT>
__device__ __forceinline__ void nvfp4_vec(const uint4 (&wv)[R], const uint32_t (&sv)[R], const XT* const (&x)[NT],
                                          int i0, float (&acc)[R][NT]) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      float xf0[8], xf1[8];
      load_x8(x[t], i0 + half * 16, xf0);
      load_x8(x[t], i0 + half * 16 + 8, xf1);
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const uint32_t q0 = half ? wv[r].z : wv[r].x;
        const uint32_t q1 = half ? wv[r].w : wv[r].y;
        float p = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) p = fmaf(e2m1_f32((q0 >> (4 * i)) & 15u), xf0[i], p);
#pragma unroll
        for (int i = 0; i < 8; ++i) p = fmaf(e2m1_f32((q1 >> (4 * i)) & 15u), xf1[i], p);
        acc[r][t] = fmaf(e4m3_f32((sv[r] >> (8 * half)) & 0xFFu), p, acc[r][t]);
      }
    }
  }
}

// acc[r][t] += sum_k W_r[k] x_t[k] over the K elements of R weight rows, lane
// strided over 16-byte weight vectors (in increasing order per lane, so the
// result does not depend on U). NVFP4 rows carry their scale rows in sc[r].
template <int WT, typename XT, int R, int NT>
__device__ __forceinline__ void warp_dot(const uint8_t* const (&w)[R], const uint8_t* const (&sc)[R],
                                         const XT* const (&x)[NT], int K, int lane, float (&acc)[R][NT]) {
  constexpr int VALS = WT == FT_W_F32 ? 4 : (WT == FT_W_BF16 ? 8 : 32);  // values per 16-byte vector
  const int nv = K / VALS;
  int v = lane;
  for (; v + 32 * (U - 1) < nv; v += 32 * U) {
    uint4 wv[U][R];
    uint32_t sv[U][R];
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
      for (int r = 0; r < R; ++r) {
        wv[u][r] = ld_stream(w[r] + (size_t)(v + 32 * u) * 16);
        if constexpr (WT == FT_W_NVFP4)
          sv[u][r] = __ldg(reinterpret_cast<const unsigned short*>(sc[r]) + (v + 32 * u));
      }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int vv = v + 32 * u;
      if constexpr (WT == FT_W_F32) {
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          const float4 xa = __ldg(reinterpret_cast<const float4*>(x[t] + vv * 4));
#pragma unroll
          for (int r = 0; r < R; ++r) {
            float a = acc[r][t];
            a = fmaf(__uint_as_float(wv[u][r].x), xa.x, a);
            a = fmaf(__uint_as_float(wv[u][r].y), xa.y, a);
            a = fmaf(__uint_as_float(wv[u][r].z), xa.z, a);
            a = fmaf(__uint_as_float(wv[u][r].w), xa.w, a);
            acc[r][t] = a;
          }
        }
      } else if constexpr (WT == FT_W_BF16) {
        float wf[R][8];
#pragma unroll
        for (int r = 0; r < R; ++r) bf16x8(wv[u][r], wf[r]);
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          float xf[8];
          load_x8(x[t], vv * 8, xf);
#pragma unroll
          for (int r = 0; r < R; ++r) {
            float a = acc[r][t];
#pragma unroll
            for (int i = 0; i < 8; ++i) a = fmaf(wf[r][i], xf[i], a);
            acc[r][t] = a;
          }
        }
      } else {  // NVFP4
        nvfp4_vec<XT, R, NT>(wv[u], sv[u], x, vv * 32, acc);
      }
    }
  }
  // tail: at most U-1 vectors per lane, same per-lane order
  for (; v < nv; v += 32) {
    uint4 wv[R];
    uint32_t sv[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      wv[r] = ld_stream(w[r] + (size_t)v * 16);
      if constexpr (WT == FT_W_NVFP4) sv[r] = __ldg(reinterpret_cast<const unsigned short*>(sc[r]) + v);
    }
    if constexpr (WT == FT_W_F32) {
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        const float4 xa = __ldg(reinterpret_cast<const float4*>(x[t] + v * 4));
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float a = acc[r][t];
          a = fmaf(__uint_as_float(wv[r].x), xa.x, a);
          a = fmaf(__uint_as_float(wv[r].y), xa.y, a);
          a = fmaf(__uint_as_float(wv[r].z), xa.z, a);
          a = fmaf(__uint_as_float(wv[r].w), xa.w, a);
          acc[r][t] = a;
        }
      }
    } else if constexpr (WT == FT_W_BF16) {
      float wf[R][8];
#pragma unroll
      for (int r = 0; r < R; ++r) bf16x8(wv[r], wf[r]);
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        float xf[8];
        load_x8(x[t], v * 8, xf);
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float a = acc[r][t];
#pragma unroll
          for (int i = 0; i < 8; ++i) a = fmaf(wf[r][i], xf[i], a);
          acc[r][t] = a;
        }
      }
    } else {
      nvfp4_vec<XT, R, NT>(wv, sv, x, v * 32, acc);
    }
  }
}

template <int R, int NT>
__device__ __forceinline__ void warp_allreduce(float (&acc)[R][NT]) {
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[r][t] += __shfl_xor_sync(0xffffffffu, acc[r][t], o);
}

struct GemvArgs {
  const WorkLists* work;
  int cls;
  int layer, E, k, d, d_ff;
  long long C;
  size_t slot_bytes;
  const uint8_t* slots;
  const uint8_t* pool;
  const void* x;         // [T, d] activations
  const int32_t* perm;
  const float* tscale;   // [L*E*3]
  float* hbuf;           // [T*k, d_ff]
  float* ybuf;           // [T*k, d]
};

struct MatRef {  // byte offsets of one matrix inside a blob
  size_t codes, scales;
};

__device__ __forceinline__ MatRef mat_ref(int wt, int which, int d, int d_ff) {
  const size_t n = (size_t)d * d_ff;
  MatRef m;
  if (wt == FT_W_NVFP4) {
    m.codes = which * (n / 2);
    m.scales = 3 * (n / 2) + which * (n / 16);
  } else {
    m.codes = which * n * (wt == FT_W_F32 ? 4 : 2);
    m.scales = 0;
  }
  return m;
}

__device__ __forceinline__ size_t row_bytes(int wt, int K) {
  return wt == FT_W_F32 ? (size_t)K * 4 : (wt == FT_W_BF16 ? (size_t)K * 2 : (size_t)K / 2);
}

__device__ __forceinline__ const uint8_t* blob_of(const GemvArgs& a, const WorkItem& it) {
  if (a.cls == KIND_STREAMED) return a.pool + (size_t)it.e * a.slot_bytes;  // a.pool: this layer's chunk
  return a.slots + (size_t)it.slot * a.slot_bytes;
}

// Map unit u of this class to (item, token chunk, row block). Units are
// ordered item-major, then chunk, then row block.
__device__ __forceinline__ bool unit_of(const GemvArgs& a, const int* s_pref, int n_items, int rblocks, int u,
                                        int& item, int& chunk, int& rb) {
  const int qi = u / rblocks;
  rb = u - qi * rblocks;
  if (qi >= s_pref[n_items]) return false;
  int lo = 0, hi = n_items - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_pref[mid] <= qi) lo = mid; else hi = mid - 1;
  }
  item = lo;
  chunk = qi - s_pref[lo];
  return true;
}

template <int WT, typename XT, int NT>
__device__ void gateup_unit(const GemvArgs& a, const WorkItem& it, int chunk, int rb, int warp, int lane) {
  const int f0 = (rb * WARPS + warp) * RW_GU;
  const uint8_t* blob = blob_of(a, it);
  const MatRef mg = mat_ref(WT, 0, a.d, a.d_ff), mu = mat_ref(WT, 1, a.d, a.d_ff);
  const size_t rbytes = row_bytes(WT, a.d);
  const uint8_t* w[2 * RW_GU];
  const uint8_t* sc[2 * RW_GU];
#pragma unroll
  for (int r = 0; r < RW_GU; ++r) {
    w[r] = blob + mg.codes + (size_t)(f0 + r) * rbytes;
    w[RW_GU + r] = blob + mu.codes + (size_t)(f0 + r) * rbytes;
    sc[r] = blob + mg.scales + (size_t)(f0 + r) * (a.d / 16);
    sc[RW_GU + r] = blob + mu.scales + (size_t)(f0 + r) * (a.d / 16);
  }
  const int base = it.tok_off + chunk * TOK_CHUNK;
  const int nt = min(TOK_CHUNK, it.n_tok - chunk * TOK_CHUNK);
  const XT* xr[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int pos = base + (t < nt ? t : 0);
    xr[t] = reinterpret_cast<const XT*>(a.x) + (size_t)(a.perm[pos] / a.k) * a.d;
  }
  float acc[2 * RW_GU][NT];
#pragma unroll
  for (int r = 0; r < 2 * RW_GU; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = 0.f;
  warp_dot<WT, XT, 2 * RW_GU, NT>(w, sc, xr, a.d, lane, acc);
  warp_allreduce(acc);
  float tg = 1.f, tu = 1.f;
  if (WT == FT_W_NVFP4) {
    const float* ts = a.tscale + ((size_t)a.layer * a.E + it.e) * 3;
    tg = ts[0];
    tu = ts[1];
  }
#pragma unroll
  for (int r = 0; r < RW_GU; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      if (lane == r * NT + t && t < nt) {
        const float g = WT == FT_W_NVFP4 ? acc[r][t] * tg : acc[r][t];
        const float u = WT == FT_W_NVFP4 ? acc[RW_GU + r][t] * tu : acc[RW_GU + r][t];
        a.hbuf[(size_t)(base + t) * a.d_ff + f0 + r] = g / (1.f + expf(-g)) * u;
      }
    }
}

template <int WT, int NT>
__device__ void down_unit(const GemvArgs& a, const WorkItem& it, int chunk, int rb, int warp, int lane) {
  const int r0 = (rb * WARPS + warp) * RW_DN;
  const uint8_t* blob = blob_of(a, it);
  const MatRef md = mat_ref(WT, 2, a.d, a.d_ff);
  const size_t rbytes = row_bytes(WT, a.d_ff);
  const uint8_t* w[RW_DN];
  const uint8_t* sc[RW_DN];
#pragma unroll
  for (int r = 0; r < RW_DN; ++r) {
    w[r] = blob + md.codes + (size_t)(r0 + r) * rbytes;
    sc[r] = blob + md.scales + (size_t)(r0 + r) * (a.d_ff / 16);
  }
  const int base = it.tok_off + chunk * TOK_CHUNK;
  const int nt = min(TOK_CHUNK, it.n_tok - chunk * TOK_CHUNK);
  const float* hr[NT];
#pragma unroll
  for (int t = 0; t < NT; ++t) hr[t] = a.hbuf + (size_t)(base + (t < nt ? t : 0)) * a.d_ff;
  float acc[RW_DN][NT];
#pragma unroll
  for (int r = 0; r < RW_DN; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t) acc[r][t] = 0.f;
  warp_dot<WT, float, RW_DN, NT>(w, sc, hr, a.d_ff, lane, acc);
  warp_allreduce(acc);
  float td = 1.f;
  if (WT == FT_W_NVFP4) td = a.tscale[((size_t)a.layer * a.E + it.e) * 3 + 2];
#pragma unroll
  for (int r = 0; r < RW_DN; ++r)
#pragma unroll
    for (int t = 0; t < NT; ++t)
      if (lane == r * NT + t && t < nt)
        a.ybuf[(size_t)(base + t) * a.d + r0 + r] = WT == FT_W_NVFP4 ? acc[r][t] * td : acc[r][t];
}

// Persistent grid-stride kernel over the units of one class. phase 0: gate/up
// + SwiGLU into hbuf; phase 1: down into ybuf.
template <int WT, typename XT, int NTMAX>
__global__ void __launch_bounds__(WARPS * 32) expert_gemv_kernel(GemvArgs a, int phase) {
  __shared__ int s_pref[MAX_E + 1];
  __shared__ WorkItem s_items[MAX_E];
  const int n_items = a.work->n_items[a.cls];
  if (n_items == 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < n_items; i += blockDim.x) s_items[i] = a.work->items[a.cls][i];
  __syncthreads();
  if (tid == 0) {
    int p = 0;
    for (int i = 0; i < n_items; ++i) {
      s_pref[i] = p;
      p += (s_items[i].n_tok + TOK_CHUNK - 1) / TOK_CHUNK;
    }
    s_pref[n_items] = p;
  }
  __syncthreads();
  const int rows_per_cta = WARPS * (phase == 0 ? RW_GU : RW_DN);
  const int rblocks = (phase == 0 ? a.d_ff : a.d) / rows_per_cta;
  const int n_units = s_pref[n_items] * rblocks;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    int item, chunk, rb;
    if (!unit_of(a, s_pref, n_items, rblocks, u, item, chunk, rb)) break;
    const WorkItem it = s_items[item];
    if (a.cls != KIND_STREAMED && (it.slot < 0 || it.slot >= a.C)) continue;  // error already latched
    const int nt = min(TOK_CHUNK, it.n_tok - chunk * TOK_CHUNK);
    // token-count variants up to NTMAX (the caller's T bounds every n_tok)
    if (phase == 0) {
      if (NTMAX == 1 || nt == 1) gateup_unit<WT, XT, 1>(a, it, chunk, rb, warp, lane);
      else if (NTMAX == 2 || nt == 2) gateup_unit<WT, XT, (NTMAX < 2 ? NTMAX : 2)>(a, it, chunk, rb, warp, lane);
      else if (NTMAX == 4 || nt <= 4) gateup_unit<WT, XT, (NTMAX < 4 ? NTMAX : 4)>(a, it, chunk, rb, warp, lane);
      else gateup_unit<WT, XT, NTMAX>(a, it, chunk, rb, warp, lane);
    } else {
      if (NTMAX == 1 || nt == 1) down_unit<WT, 1>(a, it, chunk, rb, warp, lane);
      else if (NTMAX == 2 || nt == 2) down_unit<WT, (NTMAX < 2 ? NTMAX : 2)>(a, it, chunk, rb, warp, lane);
      else if (NTMAX == 4 || nt <= 4) down_unit<WT, (NTMAX < 4 ? NTMAX : 4)>(a, it, chunk, rb, warp, lane);
      else down_unit<WT, NTMAX>(a, it, chunk, rb, warp, lane);
    }
  }
}

// y[t, :] = sum_{j<k} w[t, j] * Y[inv[t*k + j], :], ranks in order, fp32, one
// rounding to the output type. grid: (T, ceil(d / (4*256))). The weights and
// row indices of up to eight ranks are loaded first, then their rows, then
// the sums run in rank order: two dependent memory round trips per eight
// ranks instead of two per rank, with the same arithmetic.
template <typename OT>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ ybuf, const float* __restrict__ wts,
                                                      const int32_t* __restrict__ inv, int k, int d,
                                                      OT* __restrict__ y) {
  const int t = blockIdx.x;
  const int c = (blockIdx.y * 256 + threadIdx.x) * 4;
  if (c >= d) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int B = 8;
  for (int j0 = 0; j0 < k; j0 += B) {
    float w[B];
    int r[B];
    float4 v[B];
#pragma unroll
    for (int j = 0; j < B; ++j) {
      if (j0 + j < k) {
        w[j] = wts[(size_t)t * k + j0 + j];
        r[j] = inv[(size_t)t * k + j0 + j];
      }
    }
#pragma unroll
    for (int j = 0; j < B; ++j)
      if (j0 + j < k) v[j] = *reinterpret_cast<const float4*>(ybuf + (size_t)r[j] * d + c);
#pragma unroll
    for (int j = 0; j < B; ++j) {
      if (j0 + j < k) {
        acc.x = fmaf(w[j], v[j].x, acc.x);
        acc.y = fmaf(w[j], v[j].y, acc.y);
        acc.z = fmaf(w[j], v[j].z, acc.z);
        acc.w = fmaf(w[j], v[j].w, acc.w);
      }
    }
  }
  if constexpr (sizeof(OT) == 4) {
    *reinterpret_cast<float4*>(y + (size_t)t * d + c) = acc;
  } else {
    __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 pk;
    pk.x = *reinterpret_cast<uint32_t*>(&lo);
    pk.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(y + (size_t)t * d + c) = pk;
  }
}

__global__ void read_probe_kernel(const uint4* __restrict__ src, size_t n, unsigned long long* sink) {
  uint32_t x = 0;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = ld_stream(src + i);
    x ^= v.x ^ v.y ^ v.z ^ v.w;
  }
  if (x == 0x9e3779b9u) atomicAdd(sink, 1ull);  // keeps the loads alive
}

int g_gemv_grid = 0;

}  // namespace

cudaError_t expert_kernels_init(int device) {
  int sms = 0;
  cudaError_t err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, expert_gemv_kernel<FT_W_BF16, __nv_bfloat16, 1>,
                                                      WARPS * 32, 0);
  if (err != cudaSuccess) return err;
  g_gemv_grid = sms * (per_sm > 0 ? per_sm : 1);
  return cudaSuccess;
}

template <int WT, typename XT>
void launch_nt(int ntmax, int grid, const GemvArgs& a, int phase, cudaStream_t st) {
  switch (ntmax) {
    case 1: expert_gemv_kernel<WT, XT, 1><<<grid, WARPS * 32, 0, st>>>(a, phase); break;
    case 2: expert_gemv_kernel<WT, XT, 2><<<grid, WARPS * 32, 0, st>>>(a, phase); break;
    case 4: expert_gemv_kernel<WT, XT, 4><<<grid, WARPS * 32, 0, st>>>(a, phase); break;
    default: expert_gemv_kernel<WT, XT, 8><<<grid, WARPS * 32, 0, st>>>(a, phase); break;
  }
}

void launch_gemv_variant(int wtype, int ntmax, int grid, const GemvArgs& a, int phase, cudaStream_t st) {
  switch (wtype) {
    case FT_W_F32: launch_nt<FT_W_F32, float>(ntmax, grid, a, phase, st); break;
    case FT_W_BF16: launch_nt<FT_W_BF16, __nv_bfloat16>(ntmax, grid, a, phase, st); break;
    default: launch_nt<FT_W_NVFP4, __nv_bfloat16>(ntmax, grid, a, phase, st); break;
  }
}

void launch_expert_gemv(const Shape& sh, int cls, int phase, int layer, const void* x, int T, DevState& ds,
                        int max_items, int max_tok, cudaStream_t st) {
  GemvArgs a;
  a.work = ds.work;
  a.cls = cls;
  a.layer = layer;
  a.E = sh.E;
  a.k = sh.k;
  a.d = sh.d;
  a.d_ff = sh.d_ff;
  a.C = sh.C;
  a.slot_bytes = sh.slot_bytes;
  a.slots = ds.slots;
  a.pool = ds.pool_dev;
  a.x = x;
  a.perm = ds.perm;
  a.tscale = ds.tscale;
  a.hbuf = ds.hbuf;
  a.ybuf = ds.ybuf;
  // upper bound of (item x token chunk) pairs, to size the grid without
  // reading the device work list; the kernel strides over the true count
  const long long chunks = (long long)max_items + (long long)max_tok / TOK_CHUNK;
  const int rows = WARPS * (phase == 0 ? RW_GU : RW_DN);
  const long long units = chunks * ((phase == 0 ? sh.d_ff : sh.d) / rows);
  const int grid = (int)(units < g_gemv_grid ? units : g_gemv_grid);
  if (grid <= 0) return;
  const int ntmax = T >= 5 ? 8 : (T >= 3 ? 4 : T);
  launch_gemv_variant(sh.wtype, ntmax, grid, a, phase, st);
}

void launch_combine(const Shape& sh, int T, DevState& ds, void* y, cudaStream_t st) {
  dim3 grid(T, (sh.d / 4 + 255) / 256);
  if (sh.wtype == FT_W_F32)
    combine_kernel<float><<<grid, 256, 0, st>>>(ds.ybuf, ds.wts, ds.inv, sh.k, sh.d, (float*)y);
  else
    combine_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(ds.ybuf, ds.wts, ds.inv, sh.k, sh.d, (__nv_bfloat16*)y);
}

// The same combine over caller buffers: Y rows [*, d] fp32 in sorted order,
// weights [T*k], inv [T*k]; y fp32 or bf16.
void launch_combine_rows(const float* ybuf, const float* wts, const int32_t* inv, int T, int k, int d, bool out_f32,
                         void* y, cudaStream_t st) {
  dim3 grid(T, (d / 4 + 255) / 256);
  if (out_f32)
    combine_kernel<float><<<grid, 256, 0, st>>>(ybuf, wts, inv, k, d, (float*)y);
  else
    combine_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(ybuf, wts, inv, k, d, (__nv_bfloat16*)y);
}

void launch_read_probe(const uint8_t* src, size_t bytes, unsigned long long* sink, cudaStream_t st) {
  read_probe_kernel<<<g_gemv_grid > 0 ? g_gemv_grid : 148, 256, 0, st>>>(reinterpret_cast<const uint4*>(src),
                                                                        bytes / 16, sink);
}

}  // namespace ft
