// Decode grouped GEMV for BF16 and NVFP4 experts on warp-level tensor-core
// MMAs (mma.sync m16n8k16, fp32 accumulate), weights streamed straight from
// HBM slots or from the mapped host pool with 128-bit loads.
//
// Small-batch decode is memory bound ([paperlens] "壁2: デコードのミスを「どう捌く
// か」が決まっていない", paper §2.2): every weight byte is read once, so the
// kernel's job is to keep enough loads in flight and spend few instructions
// per byte. A warp owns 16 weight rows and one chunk of up to 16 tokens; each
// lane loads 16 consecutive bytes of two rows (g and g+8, g = lane / 4) and
// hands them to the MMA unchanged as its A fragment. That assigns the K
// positions of the MMA in a lane-dependent order, which is harmless for a dot
// product as long as the activations use the same order: each lane loads the
// 16 matching bytes of its token's row as the B fragment. No shuffles, no
// shared memory; the accumulation order is fixed by the code, so an expert's
// result does not depend on where its weights were read from ([paperlens]
// "設計: 2階建てのエキスパート記憶", paper §3.3).
//
// Gate/up phase: rows 0..7 of the MMA tile are gate rows f0..f0+7 and rows
// 8..15 the matching up rows, so each lane holds gate and up of the same
// (feature, token) pairs and applies SwiGLU in registers; h is written as a
// 16-bit activation for the down phase: f16 for NVFP4 experts, and for BF16
// experts as two bf16 parts hi + lo (both multiplied by W_down), which keeps h
// to about 2^-16 relative -- a single bf16 rounding of h would spend most of
// the 2e-2 rms error budget that the bf16 output rounding leaves.
// NVFP4: 32 e2m1 codes per lane are converted to f16 pairs (cvt e2m1x2) and
// multiplied by their e4m3 block scale (exact in f16), the per-matrix fp32
// tensor scale is applied to the fp32 result.
#include <cuda_fp16.h>

#include "ft_internal.cuh"

namespace ft {

namespace {

constexpr int WARPS = 8;

__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four bytes of e2m1 pairs -> four f16x2 (byte i -> out[i]; the even element
// of a pair sits in the low nibble and lands in the low half).
__device__ __forceinline__ void e2m1x8_to_f16x8(uint32_t w, uint32_t (&o)[4]) {
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
      : "r"(w));
}

// Two e4m3 scale bytes (low byte = first block) -> f16x2 {s0, s1}.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t s) {
  uint32_t r;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}" : "=r"(r) : "r"(s));
  return r;
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

struct MmaArgs {
  const WorkLists* work;
  int cls, layer, E, k, d, d_ff, nvfp4;
  long long C;
  size_t slot_bytes;
  const uint8_t* slots;
  const uint8_t* pool;
  const void* x;        // [T, d] bf16 activations (BF16) or f16 copy (NVFP4)
  const int32_t* perm;
  const float* tscale;  // [L*E*3]
  uint16_t* h16;        // [T*k, d_ff] bf16 (BF16) or f16 (NVFP4) SwiGLU output
  uint16_t* h16lo;      // [T*k, d_ff] BF16 experts: bf16 residual h - h16 (h = hi + lo to ~2^-16)
  float* ybuf;          // [T*k, d]
};

__device__ __forceinline__ const uint8_t* blob_of(const MmaArgs& a, const WorkItem& it) {
  if (a.cls == KIND_STREAMED) return a.pool + (size_t)it.e * a.slot_bytes;
  return a.slots + (size_t)it.slot * a.slot_bytes;
}

// One BF16 step: 8 K values of rows g and g+8 per lane, two MMAs per token
// tile (and two more for the low part of h in the down phase).
template <int NB, bool LO>
__device__ __forceinline__ void bf16_step(const uint4 wa, const uint4 wb, const uint16_t* const (&xr)[NB],
                                          const uint16_t* const (&xl)[NB], int e0, float (&acc)[NB][4]) {
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr[t] + e0));
    mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
    mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
    if constexpr (LO) {
      const uint4 xo = __ldg(reinterpret_cast<const uint4*>(xl[t] + e0));
      mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xo.x, xo.y);
      mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xo.z, xo.w);
    }
  }
}

// 16 code bytes (32 e2m1 values) and their two e4m3 scales -> 16 f16 pairs.
__device__ __forceinline__ void decode_nvfp4(const uint4 w, uint32_t sc, uint32_t (&h)[16]) {
  e2m1x8_to_f16x8(w.x, *reinterpret_cast<uint32_t(*)[4]>(&h[0]));
  e2m1x8_to_f16x8(w.y, *reinterpret_cast<uint32_t(*)[4]>(&h[4]));
  e2m1x8_to_f16x8(w.z, *reinterpret_cast<uint32_t(*)[4]>(&h[8]));
  e2m1x8_to_f16x8(w.w, *reinterpret_cast<uint32_t(*)[4]>(&h[12]));
  const uint32_t s2 = e4m3x2_to_f16x2(sc);
  const __half2 hs = *reinterpret_cast<const __half2*>(&s2);
  const __half2 lo = __low2half2(hs), hi = __high2half2(hs);
  const uint32_t slo = *reinterpret_cast<const uint32_t*>(&lo), shi = *reinterpret_cast<const uint32_t*>(&hi);
#pragma unroll
  for (int j = 0; j < 8; ++j) h[j] = hmul2(h[j], slo);
#pragma unroll
  for (int j = 8; j < 16; ++j) h[j] = hmul2(h[j], shi);
}

// Where a warp's two weight rows come from: straight from global memory
// (HBM slots: 128-bit non-caching loads) or from the warp's shared-memory
// tile, filled beforehand with cp.async (streamed experts: each warp
// instruction reads a contiguous run of a row, which the host link moves in
// large requests). Both hand the MMAs the same 16-byte vectors in the same
// order, so the arithmetic does not depend on the source.
template <bool STAGED>
struct RowSrc {
  const uint8_t* ga;  // global row g (+ q*16), direct mode
  const uint8_t* gb;  // global row g+8 (+ q*16)
  const uint8_t* ta;  // smem row g of this warp's tile (+ q*16), staged mode
  const uint8_t* tb;
  int s0;             // first step of this warp
  __device__ __forceinline__ uint4 a(int s) const {
    if constexpr (STAGED) return *reinterpret_cast<const uint4*>(ta + (s - s0) * 64);
    else return ld_stream(ga + (size_t)s * 64);
  }
  __device__ __forceinline__ uint4 b(int s) const {
    if constexpr (STAGED) return *reinterpret_cast<const uint4*>(tb + (s - s0) * 64);
    else return ld_stream(gb + (size_t)s * 64);
  }
};

// Scale pair (two e4m3 bytes) of step s for rows g and g+8 (NVFP4).
template <bool STAGED>
struct ScaleSrc {
  const unsigned short* ga;  // global scale row g (+ q)
  const unsigned short* gb;
  const unsigned short* ta;  // smem scale row g (+ q)
  const unsigned short* tb;
  int s0;
  __device__ __forceinline__ uint32_t a(int s) const {
    if constexpr (STAGED) return ta[(s - s0) * 4];
    else return __ldg(ga + s * 4);
  }
  __device__ __forceinline__ uint32_t b(int s) const {
    if constexpr (STAGED) return tb[(s - s0) * 4];
    else return __ldg(gb + s * 4);
  }
};

// acc[t][.] += W[rows g, g+8] . X[tokens] over steps [s0, s1) of 32 K values
// (BF16: lane q covers K = 32 s + 8 q .. +8). U steps of loads in flight;
// steps past s1 reload the last step (its result is not used).
template <int NB, int U, bool LO, class Src>
__device__ __forceinline__ void dot_bf16(const Src& src, int s0, int s1, const uint16_t* const (&xr)[NB],
                                         const uint16_t* const (&xl)[NB], int q, float (&acc)[NB][4]) {
  for (int s = s0; s < s1; s += U) {
    uint4 wa[U], wb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ss = s + u < s1 ? s + u : s1 - 1;
      wa[u] = src.a(ss);
      wb[u] = src.b(ss);
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (s + u < s1) bf16_step<NB, LO>(wa[u], wb[u], xr, xl, (s + u) * 32 + q * 8, acc);
  }
}

// NVFP4: steps of 128 K values (lane q covers K = 128 s + 32 q .. +32: 16
// code bytes and one scale pair per row); eight MMAs per step.
template <int NB, int U, class Src, class Sc>
__device__ __forceinline__ void dot_nvfp4(const Src& src, const Sc& sc, int s0, int s1,
                                          const uint16_t* const (&xr)[NB], int q, float (&acc)[NB][4]) {
  for (int s = s0; s < s1; s += U) {
    uint4 wa[U], wb[U];
    uint32_t ca[U], cb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ss = s + u < s1 ? s + u : s1 - 1;
      wa[u] = src.a(ss);
      wb[u] = src.b(ss);
      ca[u] = sc.a(ss);
      cb[u] = sc.b(ss);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (s + u < s1) {
        uint32_t ha[16], hb[16];
        decode_nvfp4(wa[u], ca[u], ha);
        decode_nvfp4(wb[u], cb[u], hb);
#pragma unroll
        for (int t = 0; t < NB; ++t) {
          const uint4* xp = reinterpret_cast<const uint4*>(xr[t] + (s + u) * 128 + q * 32);
          uint32_t xh[16];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 xv = __ldg(xp + v);
            xh[4 * v] = xv.x;
            xh[4 * v + 1] = xv.y;
            xh[4 * v + 2] = xv.z;
            xh[4 * v + 3] = xv.w;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mma_f16(acc[t], ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1], xh[2 * j], xh[2 * j + 1]);
        }
      }
    }
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Map CTA-unit u of this class to (item, 16-token chunk, 16-row block).
__device__ __forceinline__ bool unit_of(const int* pref, int n_items, int rblocks, int u, int& item, int& chunk,
                                        int& rb) {
  const int qi = u / rblocks;
  rb = u - qi * rblocks;
  if (qi >= pref[n_items]) return false;
  int lo = 0, hi = n_items - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref[mid] <= qi) lo = mid; else hi = mid - 1;
  }
  item = lo;
  chunk = qi - pref[lo];
  return true;
}

constexpr int CHUNK = 16;  // tokens per unit (two n8 tiles)

// Per-warp tile geometry of the staged mode (bytes per row, padded so the
// 8 rows a warp's lanes read at once fall in distinct bank groups).
__host__ __device__ __forceinline__ int tile_row_bytes(int steps_w) { return steps_w * 64 + 16; }
__host__ __device__ __forceinline__ int tile_scale_bytes(int steps_w) { return steps_w * 8 + 16; }
__host__ __device__ __forceinline__ int max_steps_per_warp(int steps) { return (steps + WARPS - 1) / WARPS; }
__host__ __device__ __forceinline__ int warp_tile_bytes(int steps, bool fp4) {
  const int sw = max_steps_per_warp(steps);
  return 16 * tile_row_bytes(sw) + (fp4 ? 16 * tile_scale_bytes(sw) : 0);
}

// One CTA-unit: 16 weight rows x one chunk of <= 16 tokens, the K range split
// over the 8 warps, partial sums reduced in warp order, epilogue by warp 0.
template <int NB, int PHASE, bool FP4, bool STAGED>
__device__ void unit_work(const MmaArgs& a, const WorkItem& it, int chunk, int rb, int warp, int lane,
                          uint8_t* tiles, float* red) {
  const int g = lane >> 2, q = lane & 3;
  const uint8_t* blob = blob_of(a, it);
  const size_t n = (size_t)a.d * a.d_ff;
  const int K = PHASE == 0 ? a.d : a.d_ff;
  const size_t rbytes = FP4 ? (size_t)K / 2 : (size_t)K * 2;
  const size_t sbytes = (size_t)K / 16;
  const int steps = FP4 ? K / 128 : K / 32;
  const int s0 = (warp * steps) / WARPS, s1 = ((warp + 1) * steps) / WARPS;
  // rows 0..7 / 8..15 of the tile: gate / up rows rb*8.. (phase 0), down rows rb*16.. (phase 1)
  auto row_ptr = [&](int r) -> const uint8_t* {
    if (PHASE == 0) return blob + (r < 8 ? 0 : (FP4 ? n / 2 : n * 2)) + (size_t)(rb * 8 + (r & 7)) * rbytes;
    return blob + (FP4 ? n : n * 4) + (size_t)(rb * 16 + r) * rbytes;
  };
  auto scale_ptr = [&](int r) -> const uint8_t* {
    const size_t base = 3 * (n / 2);
    if (PHASE == 0) return blob + base + (r < 8 ? 0 : n / 16) + (size_t)(rb * 8 + (r & 7)) * sbytes;
    return blob + base + 2 * (n / 16) + (size_t)(rb * 16 + r) * sbytes;
  };
  const int sw = max_steps_per_warp(steps);
  uint8_t* tile = tiles + (size_t)warp * warp_tile_bytes(steps, FP4);
  const int trow = tile_row_bytes(sw), tsrow = tile_scale_bytes(sw);
  if (STAGED && s1 > s0) {
    // contiguous per-row runs: flattened (row, byte) index, 16 bytes per lane
    const int nb = (s1 - s0) * 64;
    for (int e = lane * 16; e < 16 * nb; e += 512) {
      const int r = e / nb, off = e - r * nb;
      cp_async16(tile + r * trow + off, row_ptr(r) + (size_t)s0 * 64 + off);
    }
    if (FP4) {
      const int ns = (s1 - s0) * 8;
      uint8_t* st = tile + 16 * trow;
      for (int e = lane * 8; e < 16 * ns; e += 256) {
        const int r = e / ns, off = e - r * ns;
        cp_async8(st + r * tsrow + off, scale_ptr(r) + (size_t)s0 * 8 + off);
      }
    }
    cp_async_wait_all();
    __syncwarp();
  }
  RowSrc<STAGED> src;
  src.ga = row_ptr(g) + q * 16;
  src.gb = row_ptr(g + 8) + q * 16;
  src.ta = tile + g * trow + q * 16;
  src.tb = tile + (g + 8) * trow + q * 16;
  src.s0 = s0;
  const int base = it.tok_off + chunk * CHUNK;
  const int nt = min(CHUNK, it.n_tok - chunk * CHUNK);
  const uint16_t* xr[NB];
  const uint16_t* xl[NB];
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    const int j = t * 8 + g;
    const int pos = base + (j < nt ? j : 0);
    if (PHASE == 0) {
      xr[t] = reinterpret_cast<const uint16_t*>(a.x) + (size_t)(a.perm[pos] / a.k) * a.d;
      xl[t] = xr[t];
    } else {
      xr[t] = a.h16 + (size_t)pos * a.d_ff;
      xl[t] = a.h16lo + (size_t)pos * a.d_ff;
    }
  }
  float acc[NB][4];
#pragma unroll
  for (int t = 0; t < NB; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  if constexpr (FP4) {
    ScaleSrc<STAGED> sc;
    sc.ga = reinterpret_cast<const unsigned short*>(scale_ptr(g)) + q;
    sc.gb = reinterpret_cast<const unsigned short*>(scale_ptr(g + 8)) + q;
    sc.ta = reinterpret_cast<const unsigned short*>(tile + 16 * trow + g * tsrow) + q;
    sc.tb = reinterpret_cast<const unsigned short*>(tile + 16 * trow + (g + 8) * tsrow) + q;
    sc.s0 = s0;
    dot_nvfp4<NB, 4>(src, sc, s0, s1, xr, q, acc);
  } else {
    dot_bf16<NB, (NB == 1 ? 8 : 4), PHASE == 1>(src, s0, s1, xr, xl, q, acc);
  }
  // split-K reduction over the warps, in warp order
#pragma unroll
  for (int t = 0; t < NB; ++t)
#pragma unroll
    for (int c = 0; c < 4; ++c) red[(warp * NB * 4 + t * 4 + c) * 32 + lane] = acc[t][c];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int t = 0; t < NB; ++t)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v = red[(t * 4 + c) * 32 + lane];
        for (int w = 1; w < WARPS; ++w) v += red[(w * NB * 4 + t * 4 + c) * 32 + lane];
        acc[t][c] = v;
      }
    // d0,d1: row g, tokens 2q, 2q+1; d2,d3: row g+8, same tokens (per n8 tile)
    float t0 = 1.f, t1 = 1.f;
    if constexpr (FP4) {
      const float* ts = a.tscale + ((size_t)a.layer * a.E + it.e) * 3;
      t0 = PHASE == 0 ? ts[0] : ts[2];
      t1 = PHASE == 0 ? ts[1] : ts[2];
    }
#pragma unroll
    for (int t = 0; t < NB; ++t) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int j = t * 8 + 2 * q + c;
        if (j >= nt) continue;
        const float v0 = acc[t][c] * t0, v1 = acc[t][2 + c] * t1;
        if (PHASE == 0) {
          const float hv = v0 / (1.f + expf(-v0)) * v1;
          const size_t o = (size_t)(base + j) * a.d_ff + rb * 8 + g;
          if constexpr (FP4) {
            a.h16[o] = __half_as_ushort(__float2half_rn(hv));
          } else {
            const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
            a.h16[o] = __bfloat16_as_ushort(hi);
            a.h16lo[o] = __bfloat16_as_ushort(__float2bfloat16_rn(hv - __bfloat162float(hi)));
          }
        } else {
          float* yr = a.ybuf + (size_t)(base + j) * a.d;
          yr[rb * 16 + g] = v0;
          yr[rb * 16 + g + 8] = v1;
        }
      }
    }
  }
  __syncthreads();  // red and the tiles are reused by the next unit
}

template <int NB, bool FP4, bool STAGED>
__global__ void __launch_bounds__(WARPS * 32) gemv_mma_kernel(MmaArgs a, int phase) {
  extern __shared__ __align__(16) uint8_t tiles[];
  __shared__ int s_pref[MAX_E + 1];
  __shared__ WorkItem s_items[MAX_E];
  __shared__ float red[WARPS * NB * 4 * 32];
  const int n_items = a.work->n_items[a.cls];
  if (n_items == 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < n_items; i += blockDim.x) s_items[i] = a.work->items[a.cls][i];
  __syncthreads();
  if (tid == 0) {
    int p = 0;
    for (int i = 0; i < n_items; ++i) {
      s_pref[i] = p;
      p += (s_items[i].n_tok + CHUNK - 1) / CHUNK;
    }
    s_pref[n_items] = p;
  }
  __syncthreads();
  const int rblocks = phase == 0 ? a.d_ff / 8 : a.d / 16;
  const int n_units = s_pref[n_items] * rblocks;
  for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
    int item, chunk, rb;
    if (!unit_of(s_pref, n_items, rblocks, u, item, chunk, rb)) break;
    const WorkItem it = s_items[item];
    if (a.cls != KIND_STREAMED && (it.slot < 0 || it.slot >= a.C)) continue;  // error already latched
    if (phase == 0) unit_work<NB, 0, FP4, STAGED>(a, it, chunk, rb, warp, lane, tiles, red);
    else unit_work<NB, 1, FP4, STAGED>(a, it, chunk, rb, warp, lane, tiles, red);
  }
}

// bf16 -> f16 copy of the activations (NVFP4 experts take f16 MMA operands).
__global__ void __launch_bounds__(256) to_f16_kernel(const __nv_bfloat16* __restrict__ x, int n, __half* __restrict__ y) {
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) y[i] = __float2half_rn(__bfloat162float(x[i]));
}

int g_grid[2][3] = {{0, 0, 0}, {0, 0, 0}};  // [fp4][NB], direct mode
constexpr int STAGED_SMEM_MAX = 200 * 1024;

}  // namespace

bool gemv_mma_supported(const Shape& sh) {
  if (sh.wtype == FT_W_BF16) return sh.d % 32 == 0 && sh.d_ff % 32 == 0;
  if (sh.wtype == FT_W_NVFP4) return sh.d % 128 == 0 && sh.d_ff % 128 == 0;
  return false;
}

template <int NB, bool FP4>
cudaError_t kernel_setup(int sms) {
  cudaError_t e = cudaFuncSetAttribute(gemv_mma_kernel<NB, FP4, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       STAGED_SMEM_MAX);
  if (e != cudaSuccess) return e;
  int per = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, gemv_mma_kernel<NB, FP4, false>, WARPS * 32, 0);
  g_grid[FP4][NB] = sms * (per > 0 ? per : 1);
  return e;
}

cudaError_t gemv_mma_init(int device) {
  int sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e == cudaSuccess) e = kernel_setup<1, false>(sms);
  if (e == cudaSuccess) e = kernel_setup<2, false>(sms);
  if (e == cudaSuccess) e = kernel_setup<1, true>(sms);
  if (e == cudaSuccess) e = kernel_setup<2, true>(sms);
  return e;
}

template <int NB, bool FP4>
void launch_variant(bool staged, int grid, int dyn, const MmaArgs& a, int phase, cudaStream_t st) {
  if (staged) gemv_mma_kernel<NB, FP4, true><<<grid, WARPS * 32, dyn, st>>>(a, phase);
  else gemv_mma_kernel<NB, FP4, false><<<grid, WARPS * 32, 0, st>>>(a, phase);
}

void launch_to_f16(const void* x, int n, void* y, cudaStream_t st) {
  const int grid = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
  to_f16_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, n, (__half*)y);
}

void launch_gemv_mma(const Shape& sh, int cls, int phase, int layer, const void* x16, int T, DevState& ds,
                     int max_items, int max_tok, cudaStream_t st) {
  MmaArgs a;
  a.work = ds.work;
  a.cls = cls;
  a.layer = layer;
  a.E = sh.E;
  a.k = sh.k;
  a.d = sh.d;
  a.d_ff = sh.d_ff;
  a.nvfp4 = sh.wtype == FT_W_NVFP4;
  a.C = sh.C;
  a.slot_bytes = sh.slot_bytes;
  a.slots = ds.slots;
  a.pool = ds.pool_dev;
  a.x = x16;
  a.perm = ds.perm;
  a.tscale = ds.tscale;
  a.h16 = ds.h16;
  a.h16lo = ds.h16lo;
  a.ybuf = ds.ybuf;
  const int NB = T > 8 ? 2 : 1;
  const long long chunks = (long long)max_items + (long long)max_tok / CHUNK;
  const long long units = chunks * (phase == 0 ? sh.d_ff / 8 : sh.d / 16);
  // Streamed experts come over the host link (~55 GB/s): they are staged
  // through shared memory in contiguous runs, on a few dozen CTAs, leaving
  // the SMs to the HBM work of the hit and staged experts meanwhile.
  const int K = phase == 0 ? sh.d : sh.d_ff;
  const int steps = a.nvfp4 ? K / 128 : K / 32;
  const int smem = WARPS * warp_tile_bytes(steps, a.nvfp4);
  const bool staged = cls == KIND_STREAMED && smem <= STAGED_SMEM_MAX;
  int cap = g_grid[a.nvfp4][NB];
  if (cls == KIND_STREAMED && cap > 64) cap = 64;
  const int grid = (int)(units < cap ? units : cap);
  if (grid <= 0) return;
  if (a.nvfp4) {
    if (NB == 1) launch_variant<1, true>(staged, grid, smem, a, phase, st);
    else launch_variant<2, true>(staged, grid, smem, a, phase, st);
  } else {
    if (NB == 1) launch_variant<1, false>(staged, grid, smem, a, phase, st);
    else launch_variant<2, false>(staged, grid, smem, a, phase, st);
  }
}

}  // namespace ft
