// Decode grouped GEMV for BF16 and NVFP4 experts on warp-level tensor-core
// MMAs (mma.sync m16n8k16, fp32 accumulate): gate/up + SwiGLU and down in one
// persistent launch per work class (experts hit in HBM slots, staged into
// slots by the copy engine, or streamed from the mapped host pool).
//
// Small-batch decode is memory bound ([paperlens] "壁2: デコードのミスを「どう捌く
// か」が決まっていない", paper §2.2): every weight byte is read once, so the
// kernel keeps many bytes in flight and spends few instructions per byte.
//
// Work unit: 16 weight rows x one chunk of <= 16 tokens of one expert. One
// producer warp takes the units by atomic ticket and has the TMA engine copy,
// per K slice, the unit's 16 weight-row pieces AND the matching pieces of the
// chunk's activation rows (x for gate/up, h for down) into one stage of a
// 4-stage shared-memory ring (cp.async.bulk, mbarrier completion, one row per
// lane). Eight MMA warps split each slice's K steps and read every operand
// from shared memory, so no warp waits on a global load; they accumulate over
// the unit's slices and reduce their partial sums in warp order. Host reads
// of a streamed expert are large contiguous requests.
//
// Inside a warp, lane (g, q) = (lane/4, lane%4) reads 16 consecutive bytes of
// rows g and g+8 per step and hands them to the MMA unchanged as its A
// fragment; that fixes a lane-dependent order of the K positions, which a dot
// product does not care about as long as the activations (B fragment) are read
// in the same order. The summation order is fixed by the code and every class
// runs the same kernel, so an expert's result does not depend on where its
// weights were read from ([paperlens] "設計: 2階建てのエキスパート記憶", paper §3.3).
//
// Phase 0 units (gate/up): tile rows 0..7 are gate rows f0..f0+7 and rows
// 8..15 the matching up rows, so one lane holds gate and up of the same
// (feature, token) pairs and applies SwiGLU in registers. h goes to memory as
// f16 (NVFP4 experts) or as bf16 hi + lo parts (BF16 experts: both parts are
// multiplied by W_down, keeping h to ~2^-16; one bf16 rounding of h would eat
// most of the 2e-2 rms budget that the bf16 output rounding leaves).
// Phase 1 units (down) of an (expert, chunk) need all its phase-0 units'
// h: units are handed out in ticket order (gate/up tickets first) and the
// producer, before it copies a down unit's h rows, waits (bounded) on a
// per-chunk completion counter. A CTA holds tickets in increasing order and
// posts each unit's stages before taking the next, so when its producer waits
// every gate/up unit it holds is fully posted and its MMA warps finish it
// alone; every unit waited for is held by a running CTA: no deadlock whatever
// the residency.
//
// NVFP4: 32 e2m1 codes per lane are converted to f16 pairs (cvt e2m1x2) and
// multiplied by their e4m3 block scale (exact in f16); the per-matrix fp32
// tensor scale is applied to the fp32 result.
#include <cuda_fp16.h>

#include "ft_internal.cuh"
#include "mbarrier.cuh"

namespace ft {

namespace {

constexpr int CHUNK = 16;  // tokens per unit (two n8 tiles)
constexpr long long WAIT_CYCLES = mb::WAIT_CYCLES;
constexpr int NW = 8;                   // MMA (consumer) warps
constexpr int THREADS = (NW + 1) * 32;  // + one producer warp
constexpr int NST = 4;                  // ring stages
constexpr int ROWS = 16;                // weight rows per unit

// Stage layout, per K slice of KS values: 16 weight-row pieces, (NVFP4) their
// block scales, up to 16 activation-row pieces and (BF16 down units) the h low
// parts. Rows are padded by 16 bytes so that consecutive rows start 4 banks
// apart and a warp's fragment reads are conflict-free.
template <bool FP4> struct Lay {
  static constexpr int KS = FP4 ? 1024 : 512;                    // K values per slice
  static constexpr int STEP = FP4 ? 128 : 32;                    // K values per MMA step (64 code bytes)
  static constexpr int WROW = (FP4 ? KS / 2 : KS * 2) + 16;      // code bytes per row + pad
  static constexpr int SROW = FP4 ? KS / 16 + 16 : 0;            // scale bytes per row + pad
  static constexpr int XROW = KS * 2 + 16;                       // activation bytes per row + pad (bf16 / f16)
  static constexpr int S_OFF = ROWS * WROW;
  static constexpr int X_OFF = S_OFF + ROWS * SROW;
  static constexpr int L_OFF = X_OFF + CHUNK * XROW;
  static constexpr int BYTES = L_OFF + (FP4 ? 0 : CHUNK * XROW);
};
constexpr int STAGE_BYTES = Lay<false>::BYTES > Lay<true>::BYTES ? Lay<false>::BYTES : Lay<true>::BYTES;
constexpr int RING_BYTES = NST * STAGE_BYTES;
static_assert(STAGE_BYTES % 16 == 0, "stages start 16-byte aligned");

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
  const void* x;        // [T, d] bf16 activations (BF16) or f16 copy (NVFP4)
  const int32_t* perm;
  const float* tscale;  // [L*E*3]
  uint16_t* h16;        // [T*k, d_ff] bf16 (BF16) or f16 (NVFP4) SwiGLU output
  uint16_t* h16lo;      // [T*k, d_ff] BF16 experts: bf16 residual h - h16
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
// Barrier among the MMA warps only (the producer warp runs on its own).
__device__ __forceinline__ void mma_warps_sync() { asm volatile("bar.sync 1, %0;" ::"r"(NW * 32) : "memory"); }

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

// Generic-proxy writes of other CTAs (h), made visible by their release and
// this thread's acquire, before the async proxy (TMA) reads them.
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// K geometry of a phase: steps of 64 code bytes per row, cut into slices of
// KS values (the last may be shorter; NVFP4 slices hold an even number of
// steps, so a slice's scales are a multiple of 16 bytes).
struct Geo {
  int K, steps, nsl, ss;  // K values, steps per row, slices, steps per slice
};
template <bool FP4>
__device__ __forceinline__ Geo geo_of(const MmaArgs& a, int phase) {
  Geo g;
  g.K = phase == 0 ? a.d : a.d_ff;
  g.steps = g.K / Lay<FP4>::STEP;
  g.ss = Lay<FP4>::KS / Lay<FP4>::STEP;
  g.nsl = (g.steps + g.ss - 1) / g.ss;
  return g;
}

// acc[t] += rows g, g+8 of a stage . X over this warp's steps [s0, s1) of the
// stage; the activation rows come from the same stage (row j of token tile t
// is token t*8+g of the chunk, or row 0 for padding lanes, whose results are
// not stored).
template <int NB, bool FP4, bool P1>
__device__ __forceinline__ void stage_dot(uint32_t st, int s0, int s1, int nt, int g, int q, float (&acc)[NB][4]) {
  using L = Lay<FP4>;
  const uint32_t ra = st + g * L::WROW + q * 16, rb = ra + 8 * L::WROW;
  uint32_t xa[NB];
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    const int j = t * 8 + g;
    xa[t] = st + L::X_OFF + (j < nt ? j : 0) * L::XROW;
  }
  for (int s = s0; s < s1; ++s) {
    const uint4 wa = lds128(ra + s * 64), wb = lds128(rb + s * 64);
    if constexpr (FP4) {
      const uint32_t sc = st + L::S_OFF + s * 8 + q * 2;
      const uint32_t ca = lds16(sc + g * L::SROW), cb = lds16(sc + (g + 8) * L::SROW);
      uint32_t ha[16], hb[16];
      decode_nvfp4(wa, ca, ha);
      decode_nvfp4(wb, cb, hb);
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        uint32_t xh[16];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint4 xv = lds128(xa[t] + s * 256 + q * 64 + v * 16);
          xh[4 * v] = xv.x;
          xh[4 * v + 1] = xv.y;
          xh[4 * v + 2] = xv.z;
          xh[4 * v + 3] = xv.w;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mma_f16(acc[t], ha[2 * j], hb[2 * j], ha[2 * j + 1], hb[2 * j + 1], xh[2 * j], xh[2 * j + 1]);
      }
    } else {
#pragma unroll
      for (int t = 0; t < NB; ++t) {
        const uint4 xv = lds128(xa[t] + s * 64 + q * 16);
        mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xv.x, xv.y);
        mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xv.z, xv.w);
        if constexpr (P1) {
          const uint4 xo = lds128(xa[t] + (L::L_OFF - L::X_OFF) + s * 64 + q * 16);
          mma_bf16(acc[t], wa.x, wb.x, wa.y, wb.y, xo.x, xo.y);
          mma_bf16(acc[t], wa.z, wb.z, wa.w, wb.w, xo.z, xo.w);
        }
      }
    }
  }
}

struct StageMeta {
  int u, slice, flags;
};
constexpr int SM_FIRST = 1, SM_LAST = 2, SM_BAD = 4, SM_END = 8;

// Producer: the last warp fills the ring. Lane 0 takes the tickets (the next
// one always in flight), waits for free slots and posts each stage; then the
// lanes issue the stage's bulk copies in parallel: lane i < 16 the code piece
// of weight row i, lane 16 + i (NVFP4) its scales; then lane j < nt the piece
// of activation row j and (BF16 down units) lane 16 + j its h low part.
template <bool FP4>
__device__ void produce(const MmaArgs& a, const WorkItem* items, const int* pref, int n_items, int rb0, int rb1,
                        int U0, int U1, uint8_t* ring, volatile StageMeta* meta, uint32_t full, uint32_t empty,
                        volatile int* abort, int lane) {
  using L = Lay<FP4>;
  const size_t n = (size_t)a.d * a.d_ff;
  const size_t mat = FP4 ? n / 2 : n * 2;           // code bytes per matrix
  const size_t sc0 = 3 * (n / 2), scm = n / 16;      // NVFP4 scales: start, bytes per matrix
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
  int nxt = lane == 0 ? atomicAdd(a.ticket, 1) : 0;
  const int row = lane & 15;
  const bool hi_lane = lane >= 16;
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
    const int base = wi.tok_off + chunk * CHUNK;
    const int nt = min(CHUNK, wi.n_tok - chunk * CHUNK);
    if (!bad && ((a.landed && item > landed_upto) || phase == 1)) {
      if (lane == 0) {
        const long long t0 = clock64();
        if (a.landed && item > landed_upto) {
          // a staged expert: its slot is readable once the copy stream has
          // written this call's epoch behind the blob's copy (items in copy order)
          while (ld_acquire(a.landed + item) != a.epoch) {
            if (*abort) break;
            if (clock64() - t0 > WAIT_CYCLES) {
              *abort = 1;
              atomicExch(a.error, (uint32_t)DERR_TIMEOUT);
              break;
            }
          }
        }
        if (phase == 1) {
          // every gate/up unit of this (item, chunk) must have published h
          while (ld_acquire(reinterpret_cast<const uint32_t*>(a.done + qi)) < (uint32_t)rb0) {
            if (*abort) break;
            if (clock64() - t0 > WAIT_CYCLES) {
              *abort = 1;
              atomicExch(a.error, (uint32_t)DERR_TIMEOUT);
              break;
            }
          }
        }
        fence_proxy_async();
      }
      __syncwarp();
      if (a.landed) landed_upto = max(landed_upto, item);
    }
    // this lane's rows: weight row `row` (phase 0: gate row 8 rb + row for row
    // < 8, else up row 8 rb + row - 8; phase 1: down row 16 rb + row) and
    // activation row `row` of the chunk (x of its token, or its h row)
    const size_t m = phase == 0 ? (row < 8 ? 0 : 1) : 2;
    const size_t grow = phase == 0 ? (size_t)rb * 8 + (row & 7) : (size_t)rb * 16 + row;
    const Geo g = geo_of<FP4>(a, phase);
    const size_t wrow_bytes = FP4 ? (size_t)g.K / 2 : (size_t)g.K * 2, srow_bytes = (size_t)g.K / 16;
    const uint8_t* xsrc = nullptr;
    const uint8_t* lsrc = nullptr;
    if (row < nt) {
      if (phase == 0) {
        const int tok = a.perm[base + row] / a.k;
        xsrc = reinterpret_cast<const uint8_t*>(a.x) + (size_t)tok * a.d * 2;
      } else {
        xsrc = reinterpret_cast<const uint8_t*>(a.h16) + (size_t)(base + row) * a.d_ff * 2;
        if (!FP4) lsrc = reinterpret_cast<const uint8_t*>(a.h16lo) + (size_t)(base + row) * a.d_ff * 2;
      }
    }
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
      const int k0 = s0 * L::STEP, kv = ns * L::STEP;  // first K value and K values of the slice
      const uint32_t cb = FP4 ? (uint32_t)kv / 2 : (uint32_t)kv * 2, sb = FP4 ? (uint32_t)kv / 16 : 0;
      const uint32_t xb = (uint32_t)kv * 2;
      if (lane == 0) {
        if (bad)
          mb::arrive(bar);
        else
          mb::expect_tx(bar, ROWS * (cb + sb) + nt * xb * ((!FP4 && phase == 1) ? 2 : 1));
      }
      __syncwarp();  // the expected bytes are posted before any copy can complete them
      if (bad) continue;
      const uint32_t st = mb::smem_u32(ring + slot * STAGE_BYTES);
      if (!hi_lane)
        mb::bulk_g2s(st + row * L::WROW, blob + m * mat + grow * wrow_bytes + (FP4 ? (size_t)k0 / 2 : (size_t)k0 * 2),
                     cb, bar);
      else if (FP4)
        mb::bulk_g2s(st + L::S_OFF + row * L::SROW, blob + sc0 + m * scm + grow * srow_bytes + (size_t)k0 / 16, sb, bar);
      if (row < nt) {
        if (!hi_lane)
          mb::bulk_g2s(st + L::X_OFF + row * L::XROW, xsrc + (size_t)k0 * 2, xb, bar);
        else if (!FP4 && phase == 1)
          mb::bulk_g2s(st + L::L_OFF + row * L::XROW, lsrc + (size_t)k0 * 2, xb, bar);
      }
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
    float acc[NB][4];
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
        geo = geo_of<FP4>(a, phase);
        base = wi.tok_off + chunk * CHUNK;
        nt = min(CHUNK, wi.n_tok - chunk * CHUNK);
#pragma unroll
        for (int t = 0; t < NB; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
      }
      if (!(flags & SM_BAD)) {
        const int ns = min(geo.ss, geo.steps - sl * geo.ss);
        const int w0 = (warp * ns) / NW, w1 = ((warp + 1) * ns) / NW;
        const uint32_t st = mb::smem_u32(ring + slot * STAGE_BYTES);
        if (phase == 0)
          stage_dot<NB, FP4, false>(st, w0, w1, nt, g, q, acc);
        else
          stage_dot<NB, FP4, true>(st, w0, w1, nt, g, q, acc);
      }
      __syncwarp();
      if (lane == 0) mb::arrive(empty + 8 * slot);  // this warp is done with the stage
      if (!(flags & SM_LAST)) continue;

      // end of the unit: split-K reduction over the warps in warp order, one
      // output pair per thread: thread o < NB*64 takes token tile t, element
      // pair c (rows g and g+8 of lane l's fragment)
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
          if constexpr (FP4) {
            const float* ts = a.tscale + ((size_t)a.layer * a.E + s_items[item].e) * 3;
            v0 *= phase == 0 ? ts[0] : ts[2];
            v1 *= phase == 0 ? ts[1] : ts[2];
          }
          if (phase == 0) {
            const float hv = v0 / (1.f + expf(-v0)) * v1;
            const size_t o = (size_t)(base + j) * a.d_ff + rb * 8 + lg;
            if constexpr (FP4) {
              a.h16[o] = __half_as_ushort(__float2half_rn(hv));
            } else {
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

// bf16 -> f16 copy of the activations (NVFP4 experts take f16 MMA operands).
__global__ void __launch_bounds__(256) to_f16_kernel(const __nv_bfloat16* __restrict__ x, int n, __half* __restrict__ y) {
  for (int i = blockIdx.x * 256 + threadIdx.x; i < n; i += gridDim.x * 256) y[i] = __float2half_rn(__bfloat162float(x[i]));
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

}  // namespace

bool gemv_mma_supported(const Shape& sh) {
  if (sh.wtype == FT_W_BF16) return sh.d % 64 == 0 && sh.d_ff % 64 == 0;
  // NVFP4: a slice's block scales are a multiple of 16 bytes (bulk copies)
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
  return e;
}

void launch_to_f16(const void* x, int n, void* y, cudaStream_t st) {
  const int grid = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
  to_f16_kernel<<<grid, 256, 0, st>>>((const __nv_bfloat16*)x, n, (__half*)y);
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
  const long long units = chunks * (sh.d_ff / 8 + sh.d / 16);
  // Streamed experts come over the host link, which a few CTAs' rings keep
  // busy (16 CTAs x 4 stages of bulk reads in flight); the other SMs stay with
  // the HBM work of the hit experts running meanwhile.
  int cap = g_grid[fp4][NB];
  constexpr int stream_ctas = 16;
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
