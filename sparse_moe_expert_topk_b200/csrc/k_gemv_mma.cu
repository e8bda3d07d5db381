// Decode grouped GEMV for BF16 and NVFP4 experts on warp-level tensor-core
// MMAs (mma.sync m16n8k16, fp32 accumulate): gate/up + SwiGLU and down in one
// persistent launch per work class, weights read from HBM slots or straight
// from the mapped host pool.
//
// Small-batch decode is memory bound ([paperlens] "壁2: デコードのミスを「どう捌く
// か」が決まっていない", paper §2.2): every weight byte is read once, so the
// kernel keeps many loads in flight and spends few instructions per byte.
//
// Work unit: 16 weight rows x one chunk of <= 16 tokens of one expert, taken
// by atomic ticket; the K range of the unit is split over eight MMA warps
// (split-K), whose partial sums are reduced in warp order through shared
// memory. Two kernels share this arithmetic exactly:
//   * gemv_fused_kernel (staged and streamed experts): a producer warp has the
//     TMA engine copy the unit's weight rows (K slices of <= 2 KB per row,
//     cp.async.bulk) into a 4-stage shared-memory ring that the MMA warps
//     consume. The ring decouples the bytes in flight from registers, a
//     streamed expert's host reads become large contiguous requests, and a
//     staged expert is consumed blob by blob as the copy engine lands it.
//   * gemv_direct_kernel (experts hit in HBM slots): the MMA warps load their
//     fragments straight into registers, several steps in flight and several
//     CTAs per SM, which hides HBM latency better than the ring here.
// Both split K identically (for each ring slice in order, warp w takes the
// same sub-range of its steps), so an expert's result is bit-identical
// whichever kernel computes it.
//
// Inside a warp, lane (g, q) = (lane/4, lane%4) reads 16 consecutive bytes of
// rows g and g+8 per step and hands them to the MMA unchanged as its A
// fragment; that fixes a lane-dependent order of the K positions, which a dot
// product does not care about as long as the activations (B fragment) are
// loaded in the same order. No shuffles, and the summation order is fixed by
// the code, so an expert's result does not depend on where its weights were
// read from ([paperlens] "設計: 2階建てのエキスパート記憶", paper §3.3).
//
// Phase 0 units (gate/up): tile rows 0..7 are gate rows f0..f0+7 and rows
// 8..15 the matching up rows, so one lane holds gate and up of the same
// (feature, token) pairs and applies SwiGLU in registers. h goes to memory as
// f16 (NVFP4 experts) or as bf16 hi + lo parts (BF16 experts: both parts are
// multiplied by W_down, keeping h to ~2^-16; one bf16 rounding of h would eat
// most of the 2e-2 rms budget that the bf16 output rounding leaves).
// Phase 1 units (down) of an (expert, chunk) start once all its phase-0 units
// have published h: units are handed out in ticket order (gate/up tickets
// first) and a down unit waits, bounded, on a per-chunk completion counter.
// A CTA holds tickets in increasing order and finishes them in that order, so
// when it waits on a down unit it holds no unfinished gate/up unit; every unit
// waited for is held by a running CTA that does not wait: no deadlock whatever
// the residency.
//
// NVFP4: 32 e2m1 codes per lane are converted to f16 pairs (cvt e2m1x2) and
// multiplied by their e4m3 block scale (exact in f16: at most 6 significant
// bits, magnitudes 2^-10 .. 2688); the per-matrix fp32 tensor scale is applied
// to the fp32 result. The activation-side f16 MMA operands stay in f16
// range whatever the activations' magnitude: token t enters as
// f16(x_t * 2^-s_t), the power of two bringing max|x_t| into [1, 2) (exact
// scaling; the gate sees g = 2^s_t * sum before SwiGLU); h enters the down
// projection as h' = h * 2^-2 s_t (h scales with x^2), stored as two f16 terms
// h' = 2^24 hi + lo, each multiplied by W_down into its own accumulator and
// joined in fp32, then scaled back by 2^2 s_t. So h' keeps ~22 significant
// bits for any |h'| < 2^40; with max|x'| < 2, |h'| <= 4 |W_gate row|_1
// |W_up row|_1, below 2^40 for any weights whose rows' absolute sums stay
// below 2^19 (at d = 4096 that is a mean |weight| up to 128).
#include <cuda_fp16.h>

#include "f16_scale.cuh"
#include "ft_internal.cuh"
#include "mbarrier.cuh"

namespace ft {

namespace {

constexpr int CHUNK = 16;  // tokens per unit (two n8 tiles)
constexpr long long WAIT_CYCLES = mb::WAIT_CYCLES;
constexpr int NW = 8;                            // MMA (consumer) warps
constexpr int RING_WARPS = NW;
constexpr int THREADS = (NW + 1) * 32;           // + one producer warp
constexpr int NST = 4;                           // ring stages
constexpr int ROWS = 16;                         // weight rows per unit / stage
constexpr int SLICE = 2048;                      // max code bytes per row per stage
constexpr int CODE_RS = SLICE + 16;              // smem row stride: rows start 4 banks apart
constexpr int SC_RS = SLICE / 8 + 16;            // same for the NVFP4 block scales
constexpr int STAGE_BYTES = ROWS * CODE_RS + ROWS * SC_RS;
constexpr int RING_BYTES = NST * STAGE_BYTES;
constexpr float H_SPLIT = 16777216.0f;         // 2^24: h = H_SPLIT * hi + lo (NVFP4)
constexpr float H_SPLIT_INV = 1.0f / 16777216.0f;

// Weight fragment load that skips L1 (every weight byte is read once); kept
// in program order, so a batch of them is issued back to back.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// L2-coherent load (for h, written by other CTAs of the same launch): the
// compiler's own cache-global load, so that it stays ordered after the
// barriers that publish h but can be scheduled ahead of the MMAs around it.
__device__ __forceinline__ uint4 ld_cg(const void* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }

// Register-only MMAs (not volatile: their order per accumulator is fixed by
// the data dependence through d, which is all the summation order needs).
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                        uint32_t b1) {
  asm(
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

struct MmaArgs {
  const WorkLists* work;
  int cls, layer, E, k, d, d_ff;
  long long C;
  size_t slot_bytes;
  const uint8_t* slots;
  const uint8_t* pool;
  const void* x;        // [T, d] bf16 activations (BF16) or scaled f16 copy (NVFP4)
  const float* xscale;  // NVFP4: [T] power of two the f16 copy of token t is to be multiplied by
  const int32_t* perm;
  const float* tscale;  // [L*E*3]
  uint16_t* h16;        // [T*k, d_ff] bf16 (BF16) or f16 (NVFP4) SwiGLU output
  uint16_t* h16lo;      // [T*k, d_ff] BF16: bf16 residual h - h16; NVFP4: f16 rest h - 2^24 h16
  float* ybuf;          // [T*k, d]
  int32_t* ticket;      // this class's unit ticket counter (zeroed by the lookup)
  int32_t* done;        // this class's per-(item, chunk) phase-0 completion counters (zeroed)
  uint32_t* error;
  const uint32_t* landed;  // staged class: landed[item] == epoch once the copy engine wrote the item's slot
  uint32_t epoch;          // (null: the launch was ordered after every copy)
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ const uint8_t* blob_of(const MmaArgs& a, const WorkItem& it) {
  if (a.cls == KIND_STREAMED) return a.pool + (size_t)it.e * a.slot_bytes;
  return a.slots + (size_t)it.slot * a.slot_bytes;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}
__device__ __forceinline__ uint32_t lds16(uint32_t addr) {
  unsigned short r;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(r) : "r"(addr));
  return r;
}
// NVFP4 gate/up epilogue of one (feature, token) pair: v0, v1 are the gate
// and up sums of the scaled f16 activations (x * 2^-s), ts0 / ts1 the tensor
// scales, xs = 2^s. The true gate is g = v0 ts0 xs; the stored value is
// h' = h / xs^2 = (v0 ts0) sigmoid(g) (v1 ts1), the SwiGLU output of the
// scaled token (h scales with x^2), split into two f16 terms
// h' = 2^24 hi + lo. Shared by both GEMV kernels, so that they agree bit for bit.
__device__ __forceinline__ void fp4_gateup_store(float v0, float v1, float ts0, float ts1, float xs, uint16_t* hi_out,
                                                 uint16_t* lo_out) {
  const float gs = v0 * ts0, us = v1 * ts1;
  const float hv = gs / (1.f + expf(-(gs * xs))) * us;
  const __half hi = __float2half_rn(hv * H_SPLIT_INV);
  *hi_out = __half_as_ushort(hi);
  *lo_out = __half_as_ushort(__float2half_rn(fmaf(-__half2float(hi), H_SPLIT, hv)));
}
// NVFP4 down epilogue: the down sum over h' times the tensor scale and xs^2.
__device__ __forceinline__ float fp4_down_value(float v, float ts2, float xs) { return v * (ts2 * (xs * xs)); }

// Barrier among the MMA warps only (the producer warp runs on its own).
__device__ __forceinline__ void mma_warps_sync() { asm volatile("bar.sync 1, %0;" ::"r"(NW * 32) : "memory"); }

// acc[t] += rows g, g+8 of one stage . X over this warp's steps [s0, s1) of
// the stage; step s covers 64 code bytes of each row (32 bf16 / 128 e2m1
// values), lane q its 16-byte quarter; kb = first global step of the stage.
// The activation rows xr / xl (h hi / lo parts for BF16 down units) are read
// in the same lane-permuted K order.
template <int NB, bool FP4, bool P1>
__device__ __forceinline__ void stage_dot(uint32_t code, uint32_t sc, int s0, int s1, int kb,
                                          const uint16_t* const (&xr)[NB], const uint16_t* const (&xl)[NB], int g,
                                          int q, float (&acc)[NB][4], float (&acc2)[NB][4]) {
  const uint32_t ra = code + g * CODE_RS + q * 16, rb = ra + 8 * CODE_RS;
  for (int s = s0; s < s1; ++s) {
    const uint4 wa = lds128(ra + s * 64), wb = lds128(rb + s * 64);
    if constexpr (FP4) {
      const uint32_t ca = lds16(sc + g * SC_RS + s * 8 + q * 2), cb = lds16(sc + (g + 8) * SC_RS + s * 8 + q * 2);
      uint32_t ha[16], hb[16];
      decode_nvfp4(wa, ca, ha);
      decode_nvfp4(wb, cb, hb);
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        const uint16_t* xp = xr[t] + (kb + s) * 128 + q * 32;
        uint32_t xh[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 xv = P1 ? ld_cg(xp + 8 * v) : __ldg(reinterpret_cast<const uint4*>(xp) + v);
          xh[4 * v] = xv.x;
          xh[4 * v + 1] = xv.y;
          xh[4 * v + 2] = xv.z;
          xh[4 * v + 3] = xv.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mma_f16(acc[t], ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1], xh[2 * j], xh[2 * j + 1]);
        if constexpr (P1) {  // the lo term of h into its own accumulator
          const uint16_t* lp = xl[t] + (kb + s) * 128 + q * 32;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const uint4 xv = ld_cg(lp + 8 * v);
            xh[4 * v] = xv.x;
            xh[4 * v + 1] = xv.y;
            xh[4 * v + 2] = xv.z;
            xh[4 * v + 3] = xv.w;
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mma_f16(acc2[t], ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1], xh[2 * j], xh[2 * j + 1]);
        }
      }
    } else {
      const int e0 = (kb + s) * 32 + q * 8;
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        const uint4 xv = P1 ? ld_cg(xr[t] + e0) : __ldg(reinterpret_cast<const uint4*>(xr[t] + e0));
        mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
        mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
        if constexpr (P1) {
          const uint4 xo = ld_cg(xl[t] + e0);
          mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xo.x, xo.y);
          mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xo.z, xo.w);
        }
      }
    }
  }
}

// Map a unit index within a phase to (item, 16-token chunk, row block) and
// the item-chunk index qi.
__device__ __forceinline__ bool unit_of(const int* pref, int n_items, int rblocks, int u, int& item, int& chunk,
                                        int& rb, int& qi) {
  qi = u / rblocks;
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

// Row geometry of a phase: 64-byte steps per row and how they are cut into
// ring slices of <= SLICE bytes (an even number of steps, so an NVFP4
// slice's scales are a multiple of 16 bytes).
struct Geo {
  int steps, nsl, ss;       // steps per row, slices, steps per slice (last may be shorter)
  size_t row_bytes, sc_row; // code / scale bytes per row
};
__device__ __forceinline__ Geo geo_of(const MmaArgs& a, int phase, bool fp4) {
  Geo g;
  const int K = phase == 0 ? a.d : a.d_ff;
  g.row_bytes = fp4 ? (size_t)K / 2 : (size_t)K * 2;
  g.sc_row = fp4 ? (size_t)K / 16 : 0;
  g.steps = (int)(g.row_bytes / 64);
  g.nsl = (int)((g.row_bytes + SLICE - 1) / SLICE);
  g.ss = (g.steps + g.nsl - 1) / g.nsl;
  g.ss += g.ss & 1;
  return g;
}

struct StageMeta {
  int u, slice, flags;
};
constexpr int SM_FIRST = 1, SM_LAST = 2, SM_BAD = 4, SM_END = 8;

// Producer: the last warp fills the ring. Lane 0 takes the tickets (the next
// one always in flight), waits for free slots and posts each stage; then each
// lane issues one bulk copy of the stage (lane i < 16: the codes of smem row i;
// lane 16 + i, NVFP4 only: that row's block scales), so the 16-32 copies of a
// stage go out in parallel instead of one after another.
template <bool FP4>
__device__ void produce(const MmaArgs& a, const WorkItem* items, const int* pref, int n_items, int rb0, int rb1,
                        int U0, int U1, uint8_t* ring, volatile StageMeta* meta, uint32_t full, uint32_t empty,
                        volatile int* abort, int lane) {
  const size_t n = (size_t)a.d * a.d_ff;
  const size_t mat = FP4 ? n / 2 : n * 2;          // code bytes per matrix
  const size_t sc0 = 3 * (n / 2), scm = n / 16;     // NVFP4 scales: start, bytes per matrix
  // per slot (lane 0): the last round posted and whether it carried copies.
  // Only that round can still be in flight at exit (posting a round waits for
  // the consumers to release the one before it); a sentinel or skipped stage
  // posted after a copy round advances the slot's phase, so an older copy
  // round's parity must not be waited on.
  int it = 0;
  int landed_upto = -1;  // items known to be in their slots
  int last_round[NST];
  bool last_copy[NST];
#pragma unroll
  for (int i = 0; i < NST; ++i) last_round[i] = -1, last_copy[i] = false;
  // the next ticket is always in flight while a unit's copies are issued (a
  // global atomic's round trip would otherwise stall every unit); holding it
  // keeps the order argument: every ticket a CTA holds is later than the unit
  // its MMA warps work on
  int nxt = lane == 0 ? atomicAdd(a.ticket, 1) : 0;
  const int row = lane & 15;  // smem row this lane copies
  const bool sc_lane = lane >= 16;
  for (bool done = false; !done;) {
    const int u = __shfl_sync(0xffffffffu, nxt, 0);
    if (u >= U0 + U1) {  // end of work: one sentinel stage
      if (lane == 0) {
        const int slot = it % NST, r = it / NST;
        if (mb::wait(empty + 8 * slot, (r & 1) ^ 1, abort, a.error)) {
          meta[slot].flags = SM_END;
          mb::arrive(full + 8 * slot);
          last_round[slot] = r;
          last_copy[slot] = false;
        }
      }
      break;
    }
    if (lane == 0) nxt = atomicAdd(a.ticket, 1);
    const int phase = u < U0 ? 0 : 1;
    int item, chunk, rb, qi;
    unit_of(pref, n_items, phase == 0 ? rb0 : rb1, phase == 0 ? u : u - U0, item, chunk, rb, qi);
    const WorkItem wi = items[item];
    const bool bad = a.cls != KIND_STREAMED && (wi.slot < 0 || wi.slot >= a.C);  // error already latched
    const uint8_t* blob = bad ? nullptr : blob_of(a, wi);
    if (a.landed && !bad && item > landed_upto) {
      // a staged expert: its slot is readable once the copy stream has
      // written this call's epoch behind the blob's copy (items are in copy order)
      if (lane == 0) {
        const long long t0 = clock64();
        while (ld_acquire(a.landed + item) != a.epoch) {
          if (*abort) break;
          if (clock64() - t0 > WAIT_CYCLES) {
            *abort = 1;
            atomicExch(a.error, (uint32_t)DERR_TIMEOUT);
            break;
          }
        }
      }
      __syncwarp();
      landed_upto = item;
    }
    const Geo g = geo_of(a, phase, FP4);
    // this lane's source row: smem row i -> gate row 8 rb + i (i < 8) or up row
    // 8 rb + i - 8 (phase 0); down row 16 rb + i (phase 1)
    const size_t m = phase == 0 ? (row < 8 ? 0 : 1) : 2;
    const size_t grow = phase == 0 ? (size_t)rb * 8 + (row & 7) : (size_t)rb * 16 + row;
    for (int sl = 0; sl < g.nsl; ++sl, ++it) {
      const int slot = it % NST, r = it / NST;
      int ok = 1;
      if (lane == 0) {
        ok = mb::wait(empty + 8 * slot, (r & 1) ^ 1, abort, a.error) ? 1 : 0;
        if (ok) {
          meta[slot].u = u;
          meta[slot].slice = sl;
          meta[slot].flags = (sl == 0 ? SM_FIRST : 0) | (sl == g.nsl - 1 ? SM_LAST : 0) | (bad ? SM_BAD : 0);
          last_round[slot] = r;
          last_copy[slot] = !bad;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        done = true;
        break;
      }
      const uint32_t bar = full + 8 * slot;
      const int s0 = sl * g.ss, ns = min(g.ss, g.steps - s0);
      const uint32_t cb = (uint32_t)ns * 64, sb = FP4 ? (uint32_t)ns * 8 : 0;
      if (lane == 0) {
        if (bad)
          mb::arrive(bar);
        else
          mb::expect_tx(bar, ROWS * (cb + sb));
      }
      __syncwarp();  // the expected bytes are posted before any copy can complete them
      if (bad) continue;
      const uint32_t code = mb::smem_u32(ring + slot * STAGE_BYTES), scs = code + ROWS * CODE_RS;
      if (!sc_lane)
        mb::bulk_g2s(code + row * CODE_RS, blob + m * mat + grow * g.row_bytes + (size_t)s0 * 64, cb, bar);
      else if (FP4)
        mb::bulk_g2s(scs + row * SC_RS, blob + sc0 + m * scm + grow * g.sc_row + (size_t)s0 * 8, sb, bar);
    }
  }
  // every copy issued must have landed before the CTA's shared memory goes away
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i)
      if (last_copy[i]) mb::wait_quiet(full + 8 * i, last_round[i] & 1, WAIT_CYCLES / 4);
  }
  __syncwarp();
}

template <int NB, bool FP4>
__global__ void __launch_bounds__(THREADS, 1) gemv_fused_kernel(MmaArgs a) {
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ int s_pref[MAX_E + 1];
  __shared__ WorkItem s_items[MAX_E];
  __shared__ float red[NW * NB * 4 * 32];
  __shared__ StageMeta meta[NST];
  __shared__ __align__(8) uint64_t bars[2 * NST];
  __shared__ int s_abort, s_go[2];
  const int n_items = a.work->n_items[a.cls];
  if (n_items == 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < n_items; i += blockDim.x) s_items[i] = a.work->items[a.cls][i];
  const uint32_t full = mb::smem_u32(bars), empty = full + 8 * NST;
  if (tid == 0) {
    s_abort = 0;
    for (int i = 0; i < NST; ++i) {
      mb::init(full + 8 * i, 1);
      mb::init(empty + 8 * i, NW);
    }
    mb::fence_init();
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the chunks per item
    int carry = 0;
    for (int b = 0; b < n_items; b += 32) {
      const int i = b + lane;
      const int c = i < n_items ? (s_items[i].n_tok + CHUNK - 1) / CHUNK : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (i < n_items) s_pref[i] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_pref[n_items] = carry;
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  const int n_qi = s_pref[n_items];
  const int rb0 = a.d_ff / 8, rb1 = a.d / 16;
  const int U0 = n_qi * rb0, U1 = n_qi * rb1;

  if (warp == NW) {
    produce<FP4>(a, s_items, s_pref, n_items, rb0, rb1, U0, U1, ring, meta, full, empty, abort, lane);
  } else {
    const int g = lane >> 2, q = lane & 3;
    float acc[NB][4], acc2[NB][4];
    const uint16_t* xr[NB];
    const uint16_t* xl[NB];
    int phase = 0, item = 0, chunk = 0, rb = 0, qi = 0, base = 0, nt = 0;
    Geo geo{};
    for (int it = 0;; ++it) {
      const int slot = it % NST, r = it / NST;
      // one waiter, then everyone reads its verdict: the exit decision is
      // uniform (the producer may raise the abort flag at any time, so the
      // flag itself is not read here); two verdict slots, because thread 0
      // writes the next one before a slow warp may have read this one
      if (tid == 0) s_go[it & 1] = mb::wait(full + 8 * slot, r & 1, abort, a.error) ? 1 : 0;
      mma_warps_sync();
      if (!s_go[it & 1]) break;
      const int flags = meta[slot].flags;
      if (flags & SM_END) break;
      const int sl = meta[slot].slice;
      if (flags & SM_FIRST) {
        const int u = meta[slot].u;
        phase = u < U0 ? 0 : 1;
        unit_of(s_pref, n_items, phase == 0 ? rb0 : rb1, phase == 0 ? u : u - U0, item, chunk, rb, qi);
        const WorkItem wi = s_items[item];
        geo = geo_of(a, phase, FP4);
        base = wi.tok_off + chunk * CHUNK;
        nt = min(CHUNK, wi.n_tok - chunk * CHUNK);
#pragma unroll
        for (int t = 0; t < NB; ++t) {
          const int j = t * 8 + g;
          const int pos = base + (j < nt ? j : 0);
          if (phase == 0) {
            xr[t] = reinterpret_cast<const uint16_t*>(a.x) + (size_t)(a.perm[pos] / a.k) * a.d;
            xl[t] = xr[t];
          } else {
            xr[t] = a.h16 + (size_t)pos * a.d_ff;
            xl[t] = a.h16lo + (size_t)pos * a.d_ff;
          }
          acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
          acc2[t][0] = acc2[t][1] = acc2[t][2] = acc2[t][3] = 0.f;
        }
        if (phase == 1) {
          // every gate/up unit of this (item, chunk) must have published h
          if (tid == 0) {
            const long long t0 = clock64();
            volatile int32_t* dn = a.done + qi;
            while (*dn < rb0) {
              if (clock64() - t0 > WAIT_CYCLES) {
                atomicExch(a.error, (uint32_t)DERR_TIMEOUT);
                break;
              }
            }
            __threadfence();
          }
          mma_warps_sync();
        }
      }
      if (!(flags & SM_BAD)) {
        const int s0 = sl * geo.ss, ns = min(geo.ss, geo.steps - s0);
        const int w0 = (warp * ns) / NW, w1 = ((warp + 1) * ns) / NW;
        const uint32_t code = mb::smem_u32(ring + slot * STAGE_BYTES), scs = code + ROWS * CODE_RS;
        if (phase == 0)
          stage_dot<NB, FP4, false>(code, scs, w0, w1, s0, xr, xl, g, q, acc, acc2);
        else
          stage_dot<NB, FP4, true>(code, scs, w0, w1, s0, xr, xl, g, q, acc, acc2);
      }
      __syncwarp();
      if (lane == 0) mb::arrive(empty + 8 * slot);  // this warp is done with the stage
      if (!(flags & SM_LAST)) continue;

      // end of the unit: split-K reduction over the warps in warp order, one
      // output pair per thread: thread o < NB*64 takes token tile t, element
      // pair c (rows g and g+8 of lane l's fragment). NVFP4 down units first
      // join the two terms of h in each warp.
      if (FP4 && phase == 1) {
#pragma unroll
        for (int t = 0; t < NB; ++t)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[t][c] = fmaf(acc[t][c], H_SPLIT, acc2[t][c]);
      }
#pragma unroll
      for (int t = 0; t < NB; ++t)
#pragma unroll
        for (int c = 0; c < 4; ++c) red[((warp * NB + t) * 4 + c) * 32 + lane] = acc[t][c];
      mma_warps_sync();
      if (!(flags & SM_BAD) && tid < NB * 64) {
        const int t = tid >> 6, c = (tid >> 5) & 1, l = tid & 31;
        const int lg = l >> 2, lq = l & 3;
        float v0 = 0.f, v1 = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          v0 += red[((w * NB + t) * 4 + c) * 32 + l];
          v1 += red[((w * NB + t) * 4 + c + 2) * 32 + l];
        }
        // row lg (gate / first down row) and lg+8 (up / second down row), token 2 lq + c of tile t
        const int j = t * 8 + 2 * lq + c;
        if (j < nt) {
          float ts0 = 1.f, ts1 = 1.f, ts2 = 1.f, xs = 1.f;
          if constexpr (FP4) {
            const float* ts = a.tscale + ((size_t)a.layer * a.E + s_items[item].e) * 3;
            ts0 = ts[0], ts1 = ts[1], ts2 = ts[2];
            xs = a.xscale[a.perm[base + j] / a.k];
            if (phase == 1) {
              v0 = fp4_down_value(v0, ts2, xs);
              v1 = fp4_down_value(v1, ts2, xs);
            }
          }
          if (phase == 0) {
            const size_t o = (size_t)(base + j) * a.d_ff + rb * 8 + lg;
            if constexpr (FP4) {
              fp4_gateup_store(v0, v1, ts0, ts1, xs, a.h16 + o, a.h16lo + o);
            } else {
              const float hv = v0 / (1.f + expf(-v0)) * v1;
              const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
              a.h16[o] = __bfloat16_as_ushort(hi);
              a.h16lo[o] = __bfloat16_as_ushort(__float2bfloat16_rn(hv - __bfloat162float(hi)));
            }
          } else {
            float* yr = a.ybuf + (size_t)(base + j) * a.d;
            yr[rb * 16 + lg] = v0;
            yr[rb * 16 + lg + 8] = v1;
          }
        }
        if (phase == 0) __threadfence();  // publish h before the unit is counted done
      }
      mma_warps_sync();  // red is free again; h of this unit is published
      if (tid == 0 && phase == 0) atomicAdd(a.done + qi, 1);
    }
  }
  __syncthreads();
}

// One BF16 step: 8 K values of rows g and g+8 per lane, two MMAs per token
// tile (and two more for the low part of h in phase 1).
template <int NB, bool P1>
__device__ __forceinline__ void bf16_step(const uint4 wa, const uint4 wb, const uint16_t* const (&xr)[NB],
                                          const uint16_t* const (&xl)[NB], int e0, float (&acc)[NB][4]) {
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    const uint4 xv = P1 ? ld_cg(xr[t] + e0) : __ldg(reinterpret_cast<const uint4*>(xr[t] + e0));
    mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
    mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
    if constexpr (P1) {
      const uint4 xo = ld_cg(xl[t] + e0);
      mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xo.x, xo.y);
      mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xo.z, xo.w);
    }
  }
}

// acc[t][.] += W[rows g, g+8] . X[tokens] over steps [s0, s1) of 32 K values
// (lane q covers K = 32 s + 8 q .. +8). U steps of loads in flight; steps past
// s1 reload the last step and are not used.
template <int NB, int U, bool P1>
__device__ __forceinline__ void dot_bf16(const uint8_t* ra, const uint8_t* rb, int s0, int s1,
                                         const uint16_t* const (&xr)[NB], const uint16_t* const (&xl)[NB], int q,
                                         float (&acc)[NB][4]) {
  for (int s = s0; s < s1; s += U) {
    uint4 wa[U], wb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ss = s + u < s1 ? s + u : s1 - 1;
      wa[u] = ld_stream(ra + (size_t)ss * 64);
      wb[u] = ld_stream(rb + (size_t)ss * 64);
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (s + u < s1) bf16_step<NB, P1>(wa[u], wb[u], xr, xl, (s + u) * 32 + q * 8, acc);
  }
}

// The same over this warp's K steps of every ring slice (slice j: sub-range
// warp of NW of [j*ss, j*ss + ns_j)), gathered across slice boundaries into
// batches of U loads in flight; the MMAs run in slice order, step by step, so
// the sum is exactly the TMA-ring kernel's.
template <int NB, int U, bool P1, int NWARPS>
__device__ __forceinline__ void dot_bf16_slices(const uint8_t* ra, const uint8_t* rb, const Geo& g, int warp,
                                                const uint16_t* const (&xr)[NB], const uint16_t* const (&xl)[NB],
                                                int q, float (&acc)[NB][4]) {
  int j = 0;
  int lo = (warp * min(g.ss, g.steps)) / NWARPS, hi = ((warp + 1) * min(g.ss, g.steps)) / NWARPS;
  int s = lo;
  for (;;) {
    int st[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      while (s >= hi && j + 1 < g.nsl) {
        ++j;
        const int b0 = j * g.ss, ns = min(g.ss, g.steps - b0);
        lo = b0 + (warp * ns) / NWARPS;
        hi = b0 + ((warp + 1) * ns) / NWARPS;
        s = lo;
      }
      st[u] = s < hi ? s : -1;
      s += s < hi ? 1 : 0;
    }
    if (st[0] < 0) break;
    uint4 wa[U], wb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ss = st[u] >= 0 ? st[u] : st[0];
      wa[u] = ld_stream(ra + (size_t)ss * 64);
      wb[u] = ld_stream(rb + (size_t)ss * 64);
    }
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (st[u] >= 0) bf16_step<NB, P1>(wa[u], wb[u], xr, xl, st[u] * 32 + q * 8, acc);
  }
}

// The same over RT row tiles per step (tile r's rows tstride bytes after
// tile 0's), which share each step's activation fragments: U steps of RT x 2
// weight loads in flight, and per tile the MMAs of bf16_step in its order, so
// every row's sum is the single-tile kernels' exactly.
template <int NB, int RT, int U, bool P1, int NWARPS>
__device__ __forceinline__ void dot_bf16_rt(const uint8_t* ra, const uint8_t* rb, size_t tstride, const Geo& g,
                                            int warp, const uint16_t* const (&xr)[NB], const uint16_t* const (&xl)[NB],
                                            int q, float (&acc)[RT][NB][4]) {
  int j = 0;
  int lo = (warp * min(g.ss, g.steps)) / NWARPS, hi = ((warp + 1) * min(g.ss, g.steps)) / NWARPS;
  int s = lo;
  for (;;) {
    int st[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      while (s >= hi && j + 1 < g.nsl) {
        ++j;
        const int b0 = j * g.ss, ns = min(g.ss, g.steps - b0);
        lo = b0 + (warp * ns) / NWARPS;
        hi = b0 + ((warp + 1) * ns) / NWARPS;
        s = lo;
      }
      st[u] = s < hi ? s : -1;
      s += s < hi ? 1 : 0;
    }
    if (st[0] < 0) break;
    uint4 wa[U][RT], wb[U][RT];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ss = st[u] >= 0 ? st[u] : st[0];
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        wa[u][r] = ld_stream(ra + r * tstride + (size_t)ss * 64);
        wb[u][r] = ld_stream(rb + r * tstride + (size_t)ss * 64);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (st[u] < 0) continue;
      const int e0 = st[u] * 32 + q * 8;
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        const uint4 xv = P1 ? ld_cg(xr[t] + e0) : __ldg(reinterpret_cast<const uint4*>(xr[t] + e0));
        uint4 xo = xv;
        if constexpr (P1) xo = ld_cg(xl[t] + e0);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
          mma_bf16(acc[r][t], wa[u][r].x, wb[u][r].x, wa[u][r].y, wb[u][r].y, xv.x, xv.y);
          mma_bf16(acc[r][t], wa[u][r].z, wb[u][r].z, wa[u][r].w, wb[u][r].w, xv.z, xv.w);
          if constexpr (P1) {
            mma_bf16(acc[r][t], wa[u][r].x, wb[u][r].x, wa[u][r].y, wb[u][r].y, xo.x, xo.y);
            mma_bf16(acc[r][t], wa[u][r].z, wb[u][r].z, wa[u][r].w, wb[u][r].w, xo.z, xo.w);
          }
        }
      }
    }
  }
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Bytes of one warp's code buffers in the NVFP4 direct kernel: two steps of
// RT tiles x (gate or row a, up or row b) x 32 lanes x 16 bytes.
constexpr int fp4_wbuf_bytes(int rt) { return 2 * rt * 2 * 32 * 16; }

// NVFP4: steps of 128 K values (lane q covers K = 128 s + 32 q .. +32: 16
// code bytes and one scale pair per row); RT row tiles per step, the tiles
// tstride code bytes (tsc scale pairs) apart, sharing one activation
// fragment; eight MMAs per step, tile and token tile.
// Each step's code fragments are brought into the warp's own shared-memory
// buffers by cp.async one step ahead of their MMAs (and the block scales into
// registers one step ahead), so a warp's next loads are in flight while it
// decodes and multiplies the current step (with every load of a step waited
// for before its arithmetic, a gate/up unit took about 2.5 us per step). Each
// lane reads back only the 16 bytes it copied. wbuf: shared address of this
// warp's buffers (fp4_wbuf_bytes(RT)).
template <int NB, int RT, bool P1>
__device__ __forceinline__ void dot_nvfp4_async(const uint8_t* ra, const uint8_t* rb, const unsigned short* sa,
                                                const unsigned short* sb, size_t tstride, size_t tsc, int s0, int s1,
                                                const uint16_t* const (&xr)[NB], const uint16_t* const (&xl)[NB],
                                                int q, float (&acc)[RT][NB][4], float (&acc2)[P1 ? RT : 1][NB][4],
                                                uint32_t wbuf, int lane) {
  if (s0 >= s1) return;
  constexpr uint32_t STEP_B = RT * 2 * 32 * 16;
  const uint32_t mine = wbuf + lane * 16;
  auto issue = [&](int s, int b) {
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      cp_async16(mine + b * STEP_B + (2 * r) * 512, ra + r * tstride + (size_t)s * 64);
      cp_async16(mine + b * STEP_B + (2 * r + 1) * 512, rb + r * tstride + (size_t)s * 64);
    }
    cp_async_commit();
  };
  uint32_t ca[RT], cb[RT];
  issue(s0, 0);
#pragma unroll
  for (int r = 0; r < RT; ++r) {
    ca[r] = __ldg(sa + r * tsc + s0 * 4);
    cb[r] = __ldg(sb + r * tsc + s0 * 4);
  }
  for (int s = s0; s < s1; ++s) {
    const int b = (s - s0) & 1;
    uint32_t na[RT], nb[RT];
    if (s + 1 < s1) {
      issue(s + 1, b ^ 1);
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        na[r] = __ldg(sa + r * tsc + (s + 1) * 4);
        nb[r] = __ldg(sb + r * tsc + (s + 1) * 4);
      }
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    uint32_t xh[NB][16];
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const uint16_t* xp = xr[t] + s * 128 + q * 32;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 xv = P1 ? ld_cg(xp + 8 * v) : __ldg(reinterpret_cast<const uint4*>(xp) + v);
        xh[t][4 * v] = xv.x;
        xh[t][4 * v + 1] = xv.y;
        xh[t][4 * v + 2] = xv.z;
        xh[t][4 * v + 3] = xv.w;
      }
    }
    uint32_t xo[P1 ? NB : 1][16];  // the lo term of h (down units)
    if constexpr (P1) {
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        const uint16_t* xp = xl[t] + s * 128 + q * 32;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 xv = ld_cg(xp + 8 * v);
          xo[t][4 * v] = xv.x;
          xo[t][4 * v + 1] = xv.y;
          xo[t][4 * v + 2] = xv.z;
          xo[t][4 * v + 3] = xv.w;
        }
      }
    }
#pragma unroll
    for (int r = 0; r < RT; ++r) {
      uint32_t ha[16], hb[16];
      decode_nvfp4(lds128(mine + b * STEP_B + (2 * r) * 512), ca[r], ha);
      decode_nvfp4(lds128(mine + b * STEP_B + (2 * r + 1) * 512), cb[r], hb);
#pragma unroll
      for (int t = 0; t < NB; ++t) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mma_f16(acc[r][t], ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1], xh[t][2 * j], xh[t][2 * j + 1]);
        if constexpr (P1) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            mma_f16(acc2[r][t], ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1], xo[t][2 * j], xo[t][2 * j + 1]);
        }
      }
    }
    if (s + 1 < s1) {
#pragma unroll
      for (int r = 0; r < RT; ++r) {
        ca[r] = na[r];
        cb[r] = nb[r];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Direct-load variant for experts resident in HBM slots (the hit class): the
// MMA warps load their weight fragments straight into registers, U steps in
// flight, several CTAs per SM, so load latency is hidden by many warps. (The
// TMA ring above serves the staged and streamed classes, whose bytes arrive
// over the host link anyway.)
// ---------------------------------------------------------------------------

// One unit: RT tiles of 16 weight rows x one chunk of <= 16 tokens, the K
// range split over the NW warps, partial sums reduced in warp order, epilogue
// of tile r by warp r. Tile r of unit rb is row block rb*RT + r: gate rows
// 8 (rb*RT + r) + g with the matching up rows (phase 0), down rows
// 16 (rb*RT + r) + g and + 8 (phase 1).
template <int NB, int PHASE, bool FP4, int NW, int RT>
__device__ void direct_unit(const MmaArgs& a, const WorkItem& it, int chunk, int rb, int warp, int lane, float* red,
                            uint32_t wbuf) {
  const int g = lane >> 2, q = lane & 3;
  const uint8_t* blob = blob_of(a, it);
  const size_t n = (size_t)a.d * a.d_ff;
  const int K = PHASE == 0 ? a.d : a.d_ff;
  const size_t rbytes = FP4 ? (size_t)K / 2 : (size_t)K * 2;
  const size_t sbytes = (size_t)K / 16;
  const int steps = FP4 ? K / 128 : K / 32;
  (void)steps;
  const int rows_per_tile = PHASE == 0 ? 8 : 16;  // per weight matrix
  const int blk0 = rb * RT;                       // first row block of the unit
  size_t oa, ob, sa0, sb0;
  if (PHASE == 0) {
    oa = (size_t)(blk0 * 8 + g) * rbytes;
    ob = (FP4 ? n / 2 : n * 2) + (size_t)(blk0 * 8 + g) * rbytes;
    sa0 = 3 * (n / 2) + (size_t)(blk0 * 8 + g) * sbytes;
    sb0 = 3 * (n / 2) + n / 16 + (size_t)(blk0 * 8 + g) * sbytes;
  } else {
    oa = (FP4 ? n : n * 4) + (size_t)(blk0 * 16 + g) * rbytes;
    ob = oa + 8 * rbytes;
    sa0 = 3 * (n / 2) + 2 * (n / 16) + (size_t)(blk0 * 16 + g) * sbytes;
    sb0 = sa0 + 8 * sbytes;
  }
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
  float acc[RT][NB][4];
  float acc2[FP4 && PHASE == 1 ? RT : 1][NB][4];  // NVFP4 down units: the lo term of h
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int t = 0; t < NB; ++t) acc[r][t][0] = acc[r][t][1] = acc[r][t][2] = acc[r][t][3] = 0.f;
#pragma unroll
  for (int r = 0; r < (FP4 && PHASE == 1 ? RT : 1); ++r)
#pragma unroll
    for (int t = 0; t < NB; ++t) acc2[r][t][0] = acc2[r][t][1] = acc2[r][t][2] = acc2[r][t][3] = 0.f;
  // The K steps this warp covers are the TMA-ring kernel's: for each ring
  // slice j in order, sub-range w of NW = 8. With the same MMA order inside a
  // warp and the same warp-order reduction, an expert's output is bit-identical
  // whichever class (and kernel) computes it.
  static_assert(NW == RING_WARPS, "the K partition must match the TMA-ring kernel's");
  const Geo gg = geo_of(a, PHASE, FP4);
  if constexpr (FP4) {
    for (int j = 0; j < gg.nsl; ++j) {
      const int b0 = j * gg.ss, ns = min(gg.ss, gg.steps - b0);
      const int s0 = b0 + (warp * ns) / NW, s1 = b0 + ((warp + 1) * ns) / NW;
      if constexpr (PHASE == 1)
        dot_nvfp4_async<NB, RT, true>(blob + oa + q * 16, blob + ob + q * 16,
                                      reinterpret_cast<const unsigned short*>(blob + sa0) + q,
                                      reinterpret_cast<const unsigned short*>(blob + sb0) + q,
                                      (size_t)rows_per_tile * rbytes, (size_t)rows_per_tile * sbytes / 2, s0, s1, xr,
                                      xl, q, acc, acc2, wbuf, lane);
      else
        dot_nvfp4_async<NB, RT, false>(blob + oa + q * 16, blob + ob + q * 16,
                                       reinterpret_cast<const unsigned short*>(blob + sa0) + q,
                                       reinterpret_cast<const unsigned short*>(blob + sb0) + q,
                                       (size_t)rows_per_tile * rbytes, (size_t)rows_per_tile * sbytes / 2, s0, s1, xr,
                                       xl, q, acc, acc2, wbuf, lane);
    }
    if constexpr (PHASE == 1) {  // join the two terms of h in each warp, as the ring kernel does
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int t = 0; t < NB; ++t)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[r][t][c] = fmaf(acc[r][t][c], H_SPLIT, acc2[r][t][c]);
    }
  } else if constexpr (RT > 1) {
    // several row tiles share each step's activations, a batch of steps in flight
    // steps per load batch: three for the two-tile down units up to 8 tokens
    // (a warp's 6 steps of a d_ff = 1536 row in two batches; measured 4-5%
    // faster than three batches of two), two otherwise
    dot_bf16_rt<NB, RT, (RT == 2 && NB == 1) ? 3 : 2, PHASE == 1, NW>(blob + oa + q * 16, blob + ob + q * 16,
                                           (size_t)rows_per_tile * rbytes, gg, warp, xr, xl, q, acc);
  } else if constexpr (NB == 1) {
    // up to 8 tokens: a warp's steps gathered across slices, 8 loads in flight
    dot_bf16_slices<NB, 8, PHASE == 1, NW>(blob + oa + q * 16, blob + ob + q * 16, gg, warp, xr, xl, q, acc[0]);
  } else {
    // 9..16 tokens: slice by slice, 4 loads in flight, fewer registers and
    // more CTAs per SM (measured faster at this size); the same step order
    for (int j = 0; j < gg.nsl; ++j) {
      const int b0 = j * gg.ss, ns = min(gg.ss, gg.steps - b0);
      const int s0 = b0 + (warp * ns) / NW, s1 = b0 + ((warp + 1) * ns) / NW;
      dot_bf16<NB, 4, PHASE == 1>(blob + oa + q * 16, blob + ob + q * 16, s0, s1, xr, xl, q, acc[0]);
    }
  }
  // split-K reduction over the warps, in warp order; red is [NW][RT][NB][4][32]
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int t = 0; t < NB; ++t)
#pragma unroll
      for (int c = 0; c < 4; ++c) red[(((warp * RT + r) * NB + t) * 4 + c) * 32 + lane] = acc[r][t][c];
  __syncthreads();
  if (warp < RT) {
    const int r = warp;
    float v[NB][4];
#pragma unroll
    for (int t = 0; t < NB; ++t)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float x = red[((r * NB + t) * 4 + c) * 32 + lane];
        for (int w = 1; w < NW; ++w) x += red[(((w * RT + r) * NB + t) * 4 + c) * 32 + lane];
        v[t][c] = x;
      }
    // d0,d1: row g, tokens 2q, 2q+1; d2,d3: row g+8, same tokens (per n8 tile)
    float t0 = 1.f, t1 = 1.f;
    if constexpr (FP4) {
      const float* ts = a.tscale + ((size_t)a.layer * a.E + it.e) * 3;
      t0 = PHASE == 0 ? ts[0] : ts[2];
      t1 = PHASE == 0 ? ts[1] : ts[2];
    }
    const int blk = blk0 + r;
#pragma unroll
    for (int t = 0; t < NB; ++t) {
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int j = t * 8 + 2 * q + c;
        if (j >= nt) continue;
        float v0 = v[t][c], v1 = v[t][2 + c], xs = 1.f;
        if constexpr (FP4) {
          xs = a.xscale[a.perm[base + j] / a.k];
          if (PHASE == 1) {
            v0 = fp4_down_value(v0, t0, xs);
            v1 = fp4_down_value(v1, t1, xs);
          }
        }
        if (PHASE == 0) {
          const size_t o = (size_t)(base + j) * a.d_ff + blk * 8 + g;
          if constexpr (FP4) {
            fp4_gateup_store(v0, v1, t0, t1, xs, a.h16 + o, a.h16lo + o);
          } else {
            const float hv = v0 / (1.f + expf(-v0)) * v1;
            const __nv_bfloat16 hi = __float2bfloat16_rn(hv);
            a.h16[o] = __bfloat16_as_ushort(hi);
            a.h16lo[o] = __bfloat16_as_ushort(__float2bfloat16_rn(hv - __bfloat162float(hi)));
          }
        } else {
          float* yr = a.ybuf + (size_t)(base + j) * a.d;
          yr[blk * 16 + g] = v0;
          yr[blk * 16 + g + 8] = v1;
        }
      }
    }
    if (PHASE == 0) __threadfence();  // publish h before the unit is counted done
  }
  // the caller's barrier ends the unit: red is reused by the next one
}

// Row tiles per unit: NVFP4 rows are a quarter of the BF16 bytes, so a unit
// takes four tiles to keep the loads in flight per warp and the per-unit
// reduction and barriers amortised.
template <bool FP4>
constexpr int tiles_for() { return FP4 ? 4 : 1; }
// Row tiles per down unit. BF16: four sharing each step's h fragments at
// 9-16 tokens; two up to 8, where the 384 four-tile units of a 6-expert call
// left a tail of 12.7 us units on a third of the CTAs (two tiles measured 5%
// faster at 1 and 4 tokens). NVFP4 down units carry two accumulators (the two
// terms of h), so they take two row tiles, which keeps the kernel's registers
// where four gate/up tiles put them (four measured slower: fewer, longer units
// and spills). A unit's row tiles change which rows it covers, not the K order
// of any row, so results do not depend on this choice.
template <bool FP4, int NB>
constexpr int tiles_down_for() { return FP4 ? 2 : (NB == 1 ? 2 : 4); }

template <int NB, bool FP4, int NW>
__global__ void __launch_bounds__(NW * 32) gemv_direct_kernel(MmaArgs a) {
  constexpr int RT = tiles_for<FP4>(), RT1 = tiles_down_for<FP4, NB>();
  constexpr int RTM = RT > RT1 ? RT : RT1;
  __shared__ int s_pref[MAX_E + 1];
  __shared__ WorkItem s_items[MAX_E];
  __shared__ float red[NW * RTM * NB * 4 * 32];
  extern __shared__ __align__(16) uint8_t dsm_direct[];  // NVFP4: per-warp code buffers
  // Tickets taken ahead of the unit being worked on: two for BF16 (measured
  // faster than one), one for NVFP4, whose gate/up units fill about one wave
  // at a few tokens, so a second early ticket would stack two of them on some
  // CTAs while others wait for their h.
  constexpr int AHEAD = FP4 ? 1 : 2;
  __shared__ int s_unit[AHEAD + 1];  // tickets of this unit and the ones after it, in rotation
  const int n_items = a.work->n_items[a.cls];
  if (n_items == 0) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t wbuf = (uint32_t)__cvta_generic_to_shared(dsm_direct) + warp * (FP4 ? fp4_wbuf_bytes(RTM) : 0);
  for (int i = tid; i < n_items; i += blockDim.x) s_items[i] = a.work->items[a.cls][i];
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the chunks per item
    int carry = 0;
    for (int b = 0; b < n_items; b += 32) {
      const int i = b + lane;
      const int c = i < n_items ? (s_items[i].n_tok + CHUNK - 1) / CHUNK : 0;
      int incl = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      if (i < n_items) s_pref[i] = carry + incl - c;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_pref[n_items] = carry;
  }
  __syncthreads();
  const int n_qi = s_pref[n_items];
  const int rb0 = a.d_ff / 8 / RT, rb1 = a.d / 16 / RT1;
  const int U0 = n_qi * rb0, U1 = n_qi * rb1;
  if (tid == 0)
    for (int j = 0; j < AHEAD; ++j) s_unit[j] = atomicAdd(a.ticket, 1);
  __syncthreads();
  for (int i = 0;; ++i) {
    const int u = s_unit[i % (AHEAD + 1)];
    if (u >= U0 + U1) break;
    // The next ticket of the rotation is fetched while this unit runs.
    // Tickets are taken in increasing order and phase-0 tickets all precede
    // phase-1 ones, so a CTA waiting in a phase-1 unit holds no phase-0
    // ticket: every waited-on unit is running or held by a CTA that runs it
    // without waiting.
    int nxt = 0;
    if (tid == 0) nxt = atomicAdd(a.ticket, 1);
    const int phase = u < U0 ? 0 : 1;
    int item, chunk, rb, qi;
    unit_of(s_pref, n_items, phase == 0 ? rb0 : rb1, phase == 0 ? u : u - U0, item, chunk, rb, qi);
    const WorkItem it = s_items[item];
    const bool bad = a.cls != KIND_STREAMED && (it.slot < 0 || it.slot >= a.C);  // error already latched
    if (phase == 1) {
      // wait until every gate/up unit of this (item, chunk) has published h
      if (tid == 0) {
        const long long t0 = clock64();
        volatile int32_t* dn = a.done + qi;
        while (*dn < rb0) {
          if (clock64() - t0 > WAIT_CYCLES) {
            atomicExch(a.error, (uint32_t)DERR_TIMEOUT);
            break;
          }
        }
        __threadfence();
      }
      __syncthreads();
      if (!bad) direct_unit<NB, 1, FP4, NW, RT1>(a, it, chunk, rb, warp, lane, red, wbuf);
    } else {
      if (!bad) direct_unit<NB, 0, FP4, NW, RT>(a, it, chunk, rb, warp, lane, red, wbuf);
    }
    // entry (i + AHEAD) % (AHEAD + 1) held the previous unit's ticket, which
    // every thread read before the last barrier: it is free for the new one
    if (tid == 0) s_unit[(i + AHEAD) % (AHEAD + 1)] = nxt;
    __syncthreads();  // red is free; this unit's h is published; the next ticket is visible
    if (tid == 0 && phase == 0) atomicAdd(a.done + qi, 1);
  }
}

// f16 copy of the bf16 activations for the NVFP4 experts' f16 MMAs, one CTA
// per token (to_f16_scaled_row gives the scaling rule).
__global__ void __launch_bounds__(256) to_f16_scaled_kernel(const __nv_bfloat16* __restrict__ x, int d,
                                                            __half* __restrict__ y, float* __restrict__ xscale) {
  __shared__ float s_max[8];
  const int t = blockIdx.x;
  to_f16_scaled_row<256>(x + (size_t)t * d, d, y + (size_t)t * d, xscale + t, s_max);
}

int g_grid[2][3] = {{0, 0, 0}, {0, 0, 0}};  // [fp4][NB]: resident CTAs (one per SM)

template <int NB, bool FP4>
cudaError_t kernel_setup(int sms) {
  cudaError_t e = cudaFuncSetAttribute(gemv_fused_kernel<NB, FP4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       RING_BYTES);
  if (e != cudaSuccess) return e;
  int per = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, gemv_fused_kernel<NB, FP4>, THREADS, RING_BYTES);
  g_grid[FP4][NB] = sms * (per > 0 ? per : 1);
  return e;
}

template <int NB, bool FP4>
void launch_nb(int grid, const MmaArgs& a, cudaStream_t st) {
  gemv_fused_kernel<NB, FP4><<<grid, THREADS, RING_BYTES, st>>>(a);
}

// Warps per CTA of the direct-load kernel: the ring kernel's eight, so both
// split K the same way (see direct_unit).
template <int NB>
constexpr int warps_for() { return RING_WARPS; }

int g_grid_direct[2][3] = {{0, 0, 0}, {0, 0, 0}};  // [fp4][NB]

// Dynamic shared memory of the direct kernel: the NVFP4 per-warp code buffers.
template <int NB, bool FP4>
constexpr int direct_dyn_smem() {
  constexpr int rtm = tiles_for<FP4>() > tiles_down_for<FP4, NB>() ? tiles_for<FP4>() : tiles_down_for<FP4, NB>();
  return FP4 ? warps_for<NB>() * fp4_wbuf_bytes(rtm) : 0;
}

template <int NB, bool FP4>
cudaError_t direct_setup(int sms) {
  constexpr int NW = warps_for<NB>();
  constexpr int dyn = direct_dyn_smem<NB, FP4>();
  cudaError_t e = cudaFuncSetAttribute(gemv_direct_kernel<NB, FP4, NW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       dyn);
  if (e != cudaSuccess) return e;
  int per = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, gemv_direct_kernel<NB, FP4, NW>, NW * 32, dyn);
  g_grid_direct[FP4][NB] = sms * (per > 0 ? per : 1);
  return e;
}

template <int NB, bool FP4>
void launch_direct(int grid, const MmaArgs& a, cudaStream_t st) {
  constexpr int NW = warps_for<NB>();
  gemv_direct_kernel<NB, FP4, NW><<<grid, NW * 32, direct_dyn_smem<NB, FP4>(), st>>>(a);
}

}  // namespace

bool gemv_mma_supported(const Shape& sh) {
  if (sh.wtype == FT_W_BF16) return sh.d % 32 == 0 && sh.d_ff % 32 == 0;
  // NVFP4: a row's block scales are a multiple of 16 bytes (bulk copies)
  if (sh.wtype == FT_W_NVFP4) return sh.d % 256 == 0 && sh.d_ff % 256 == 0;
  return false;
}

cudaError_t gemv_mma_init(int device) {
  int sms = 0;
  cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (e == cudaSuccess) e = kernel_setup<1, false>(sms);
  if (e == cudaSuccess) e = kernel_setup<2, false>(sms);
  if (e == cudaSuccess) e = kernel_setup<1, true>(sms);
  if (e == cudaSuccess) e = kernel_setup<2, true>(sms);
  if (e == cudaSuccess) e = direct_setup<1, false>(sms);
  if (e == cudaSuccess) e = direct_setup<2, false>(sms);
  if (e == cudaSuccess) e = direct_setup<1, true>(sms);
  if (e == cudaSuccess) e = direct_setup<2, true>(sms);
  return e;
}

void launch_to_f16(const void* x, int T, int d, void* y, float* xscale, cudaStream_t st) {
  to_f16_scaled_kernel<<<T, 256, 0, st>>>((const __nv_bfloat16*)x, d, (__half*)y, xscale);
}

// Both phases of one work class in one launch.
void launch_gemv_mma(const Shape& sh, int cls, int layer, const void* x16, int T, DevState& ds, int max_items,
                     int max_tok, cudaStream_t st) {
  MmaArgs a;
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
  a.x = x16;
  a.xscale = ds.xscale;
  a.perm = ds.perm;
  a.tscale = ds.tscale;
  a.h16 = ds.h16;
  a.h16lo = ds.h16lo;
  a.ybuf = ds.ybuf;
  a.ticket = ds.sched + cls;
  a.done = ds.sched + N_CLASSES + (size_t)cls * ds.sched_chunks;
  a.error = ds.error;
  a.landed = cls == KIND_STAGED && ds.landed_epoch ? ds.landed : nullptr;
  a.epoch = ds.landed_epoch;
  const bool fp4 = sh.wtype == FT_W_NVFP4;
  const int NB = T > 8 ? 2 : 1;
  const long long chunks = (long long)max_items + (long long)max_tok / CHUNK;
  if (cls == KIND_HIT) {
    const int rt1 = NB == 1 ? (fp4 ? tiles_down_for<true, 1>() : tiles_down_for<false, 1>())
                            : (fp4 ? tiles_down_for<true, 2>() : tiles_down_for<false, 2>());
    const long long units = chunks * (sh.d_ff / 8 / (fp4 ? tiles_for<true>() : tiles_for<false>()) + sh.d / 16 / rt1);
    const int cap = g_grid_direct[fp4][NB];
    const int grid = (int)(units < cap ? units : cap);
    if (grid <= 0) return;
    if (fp4) {
      if (NB == 1) launch_direct<1, true>(grid, a, st);
      else launch_direct<2, true>(grid, a, st);
    } else {
      if (NB == 1) launch_direct<1, false>(grid, a, st);
      else launch_direct<2, false>(grid, a, st);
    }
    return;
  }
  const long long units = chunks * (sh.d_ff / 8 + sh.d / 16);
  // Streamed experts come over the host link, which a few CTAs' rings keep
  // busy (BF16: 16 CTAs x 4 stages x 37 KB of bulk reads in flight; NVFP4,
  // whose stages carry fewer bytes, 32 CTAs: measured alone at one token,
  // 16 / 32 CTAs reach 1.00 / 1.00 of the zero-copy read rate for BF16 and
  // 0.89 / 0.98 for NVFP4); the other SMs stay with the HBM work of the hit
  // experts running meanwhile.
  int cap = g_grid[fp4][NB];
  const int stream_ctas = fp4 ? 32 : 16;
  if (cls == KIND_STREAMED && cap > stream_ctas) cap = stream_ctas;
  const int grid = (int)(units < cap ? units : cap);
  if (grid <= 0) return;
  if (fp4) {
    if (NB == 1) launch_nb<1, true>(grid, a, st);
    else launch_nb<2, true>(grid, a, st);
  } else {
    if (NB == 1) launch_nb<1, false>(grid, a, st);
    else launch_nb<2, false>(grid, a, st);
  }
}

}  // namespace ft
