// Prefill grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM,
// operands staged by TMA), with SwiGLU fused into the gate/up epilogue.
//
// Prefill pushes thousands of tokens through a layer, so nearly every expert
// is active ([paperlens] "壁1: プレフィルではスパース性が消える", paper §2.1) and
// the whole layer is resident in HBM slots before it computes ([paperlens]
// "プレフィル: 全層ダブルバッファと「意味の錨」", paper §3.1). Per expert the work
// is a GEMM with a ragged number of tokens (about 96 at T=4096, top-6 of 256).
//
// Formulation (swap-AB): the weight rows are the MMA's M = 128 side and the
// expert's tokens the N side (N = tokens rounded up to 16, <= 256), so no
// weight tile is padded:
//   phase 0: D_g[f, p] = W_gate[f, :] . X_s[p, :],  D_u[f, p] = W_up[f, :] . X_s[p, :]
//            H_s[p, f] = bf16(silu(D_g) * D_u)          (two accumulators in TMEM)
//   phase 1: Y[p, r]   = W_down[r, :] . H_s[p, :]        (fp32 into the expert output buffer)
// X_s / H_s hold the activations in expert-sorted order (row p = sorted
// position), so an expert's tokens are consecutive rows.
//
// One persistent CTA per SM: warp 0 issues TMA loads (one elected lane) into a
// 3-stage ring of 128B-swizzled K-major tiles, warp 1 allocates TMEM and
// issues tcgen05.mma (one elected lane), warps 2..5 drain the accumulators
// with tcgen05.ld and run the epilogue. All waits are bounded: a wait that
// runs out latches a device error and the CTA drains and returns.
// No TMA load uses cluster multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <new>

#include "ft_internal.cuh"
#include "mbarrier.cuh"

namespace ft {

struct TcPlan {
  CUtensorMap a_gu;  // BF16: slot pool as rows of d bf16 (gate/up rows)
  CUtensorMap a_dn;  // BF16: slot pool as rows of d_ff bf16 (down rows)
  CUtensorMap b_x;   // X_s [rows, d]
  CUtensorMap b_h;   // H_s [rows, d_ff]
  // NVFP4: the codes of each matrix over the slot pool
  // (3D: bytes of a row, rows of the matrix, slot), phase 0 and phase 1
  CUtensorMap f_code[3];   // gate, up, down: boxes of one k-block (32 code bytes x 128 rows)
  CUtensorMap f_code4[3];  // the same with boxes of four k-blocks (128 bytes x 128 rows, 128B-swizzled)
  bool fp4;
  int sms;
};

namespace {

constexpr int BM = 128;       // weight rows per tile (MMA M)
constexpr int BK = 64;        // K per stage: 64 bf16 = one 128-byte swizzle row
constexpr int MAX_N = 256;    // tokens per MMA (N)
constexpr int BOX_ROWS = 32;  // rows per TMA box of the token operand
constexpr int STAGES = 3;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_BYTES = MAX_N * BK * 2;    // 32 KB
constexpr int STAGE_BYTES = 2 * A_BYTES + B_BYTES;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + 256;
// Warps: 0 TMA, 1 MMA, 2 .. 2 + EPI_WARPS - 1 epilogue. The gate/up epilogue
// (SwiGLU over 128 x 256 accumulators) runs while the MMAs wait for the one
// accumulator buffer, so it takes two warps per TMEM lane quarter, each on
// every other 32-column chunk (one warp per quarter took about as long as a
// unit's main loop).
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (2 + EPI_WARPS) * 32;

using mb::smem_u32;
using mb::WAIT_CYCLES;
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) { mb::init(bar, count); }
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) { mb::expect_tx(bar, bytes); }
__device__ __forceinline__ void mbar_arrive(uint32_t bar) { mb::arrive(bar); }
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) { return mb::try_wait(bar, parity); }
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort, uint32_t* err) {
  return mb::wait(bar, parity, abort, err);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every previously issued tcgen05.mma of this thread completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,"
      "%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, rows of 128 bytes,
// 8-row atoms 1024 bytes apart (SBO), LBO unused (1), descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B (K-major), fp32 D, M x N.
__device__ __forceinline__ uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

struct TcArgs {
  const WorkLists* work;
  const float* tscale;  // NVFP4: [L*E*3] per-matrix tensor scales
  const uint8_t* slots; // NVFP4: the slot pool (block scales are read from it)
  size_t slot_bytes;
  int layer, E;
  int phase;
  int d, d_ff;
  int m_tiles;   // weight-row tiles of 128
  int k_blocks;  // K / 64
  __nv_bfloat16* hs;  // phase 0 output [rows, d_ff]
  float* ybuf;        // phase 1 output [rows, d]
  uint32_t* error;
};

struct Unit {
  int slot, p0, nrows, mt, e;
};

// Units: (item, token tile of <= 256, weight-row tile); item-major so that the
// CTAs working at one time share an expert's activations in L2.
__device__ __forceinline__ bool unit_at(const TcArgs& a, const WorkItem* items, const int* pref, int n_items, int u,
                                        Unit& out) {
  const int q = u / a.m_tiles;
  if (q >= pref[n_items]) return false;
  int lo = 0, hi = n_items - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pref[mid] <= q) lo = mid; else hi = mid - 1;
  }
  const WorkItem it = items[lo];
  const int j = q - pref[lo];
  out.slot = it.slot;
  out.e = it.e;
  out.p0 = it.tok_off + j * MAX_N;
  out.nrows = min(MAX_N, it.n_tok - j * MAX_N);
  out.mt = u - q * a.m_tiles;
  return true;
}

__global__ void __launch_bounds__(THREADS, 1) gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a,
                                                             const __grid_constant__ CUtensorMap tm_b, TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ WorkItem s_items[MAX_E];
  __shared__ int s_pref[MAX_E + 1];
  __shared__ int s_abort;
  __shared__ uint32_t s_tmem;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  // bars: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
  const uint32_t bar_full = smem_u32(bars), bar_empty = bar_full + 8 * STAGES;
  // accumulator buffers: phase 0 uses all 512 TMEM columns (gate | up), one
  // buffer; phase 1 needs 256, so two buffers let the epilogue drain one while
  // the MMAs of the next unit fill the other
  const uint32_t bar_acc_full = bar_full + 16 * STAGES, bar_acc_empty = bar_acc_full + 16;
  const uint32_t bar_drain = bar_acc_empty + 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &s_abort;

  const int n_items = a.work->n_items[KIND_HIT];
  for (int i = threadIdx.x; i < n_items; i += THREADS) s_items[i] = a.work->items[KIND_HIT][i];
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, EPI_WARPS);
    }
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), 512);
    tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int p = 0;
    for (int i = 0; i < n_items; ++i) {
      s_pref[i] = p;
      p += (s_items[i].n_tok + MAX_N - 1) / MAX_N;
    }
    s_pref[n_items] = p;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_units = n_items > 0 ? s_pref[n_items] * a.m_tiles : 0;
  const int two_a = a.phase == 0;

  int last_round[STAGES];  // producer: last ring round issued per stage (-1 none)
#pragma unroll
  for (int s = 0; s < STAGES; ++s) last_round[s] = -1;
  if (warp == 0) {
    // ---------------- TMA producer ----------------
    int it = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const int nb = (un.nrows + BOX_ROWS - 1) / BOX_ROWS;
      const uint32_t bytes = (two_a ? 2 : 1) * A_BYTES + nb * BOX_ROWS * BK * 2;
      int row_a0, row_a1;
      if (two_a) {
        row_a0 = un.slot * 3 * a.d_ff + un.mt * BM;          // gate rows
        row_a1 = un.slot * 3 * a.d_ff + a.d_ff + un.mt * BM;  // up rows
      } else {
        row_a0 = un.slot * 3 * a.d + 2 * a.d + un.mt * BM;    // down rows
        row_a1 = 0;
      }
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
        const int s = it % STAGES, r = it / STAGES;
        if (!mbar_wait(bar_empty + 8 * s, (r & 1) ^ 1, abort, a.error)) break;
        last_round[s] = r;
        if (lane == 0) {
          const uint32_t base = smem_u32(smem + s * STAGE_BYTES);
          mbar_expect_tx(bar_full + 8 * s, bytes);
          tma_load_2d(base, &tm_a, bar_full + 8 * s, kb * BK, row_a0);
          if (two_a) tma_load_2d(base + A_BYTES, &tm_a, bar_full + 8 * s, kb * BK, row_a1);
          for (int b = 0; b < nb; ++b)
            tma_load_2d(base + 2 * A_BYTES + b * BOX_ROWS * 128, &tm_b, bar_full + 8 * s, kb * BK,
                        un.p0 + b * BOX_ROWS);
        }
        __syncwarp();
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    int it = 0, ui = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x, ++ui) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const int n_mma = (un.nrows + 15) & ~15;
      const uint32_t idesc = idesc_bf16(BM, n_mma);
      const int ab = two_a ? 0 : (ui & 1), use = two_a ? ui : (ui >> 1);  // buffer, its use count
      if (!mbar_wait(bar_acc_empty + 8 * ab, (use & 1) ^ 1, abort, a.error)) break;
      const uint32_t dacc = tmem + (uint32_t)(ab * 256);
      tc_fence_after();
      bool ok = true;
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
        const int s = it % STAGES, r = it / STAGES;
        if (!mbar_wait(bar_full + 8 * s, r & 1, abort, a.error)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t base = smem_u32(smem + s * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = sw128_desc(base + 2 * A_BYTES + kk * 32);
            umma_bf16(dacc, sw128_desc(base + kk * 32), bd, idesc, (kb | kk) != 0);
            if (two_a) umma_bf16(tmem + 256, sw128_desc(base + A_BYTES + kk * 32), bd, idesc, (kb | kk) != 0);
          }
          umma_commit(bar_empty + 8 * s);  // stage free once these MMAs have read it
          if (kb == a.k_blocks - 1) umma_commit(bar_acc_full + 8 * ab);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
  } else {
    // ---------------- epilogue (warps 2 .. 2 + EPI_WARPS - 1) ----------------
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int part = (warp - 2) >> 2, parts = EPI_WARPS / 4;  // which of the quarter's column chunks
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int ui = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x, ++ui) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const int ab = two_a ? 0 : (ui & 1), use = two_a ? ui : (ui >> 1);
      if (!mbar_wait(bar_acc_full + 8 * ab, use & 1, abort, a.error)) break;
      tc_fence_after();
      const int row = un.mt * BM + 32 * q + lane;  // weight row = output feature
      for (int c0 = 32 * part; c0 < un.nrows; c0 += 32 * parts) {
        uint32_t g[32];
        tmem_ld32(tmem + (uint32_t)(ab * 256) + lane_base + c0, g);
        if (two_a) {
          uint32_t uu[32];
          tmem_ld32(tmem + lane_base + 256 + c0, uu);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c0 + i < un.nrows) {
              const float gv = __uint_as_float(g[i]), uv = __uint_as_float(uu[i]);
              const float hv = gv / (1.f + expf(-gv)) * uv;
              a.hs[(size_t)(un.p0 + c0 + i) * a.d_ff + row] = __float2bfloat16_rn(hv);
            }
          }
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < un.nrows) a.ybuf[(size_t)(un.p0 + c0 + i) * a.d + row] = __uint_as_float(g[i]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acc_empty + 8 * ab);
    }
  }
  __syncthreads();
  if (warp == 0) {
    // producer tail: every stage's last round must be released by the MMAs
    // (normal exit) or at least have landed (abort) before smem goes away
    for (int s = 0; s < STAGES; ++s) {
      if (last_round[s] < 0) continue;
      const uint32_t bar = *abort ? bar_full + 8 * s : bar_empty + 8 * s;
      const long long t0 = clock64();
      while (!mbar_try_wait(bar, last_round[s] & 1) && clock64() - t0 < WAIT_CYCLES / 4) {
      }
    }
  } else if (warp == 1 && *abort) {
    // let every issued MMA finish before the accumulators are freed
    if (lane == 0) umma_commit(bar_drain);
    __syncwarp();
    const long long t0 = clock64();
    while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < WAIT_CYCLES / 4) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// NVFP4 experts on the same tensor cores. tcgen05 has no MMA kind that takes
// 4-bit weights against 16-bit activations, so the weight tiles are widened
// on chip: the TMA engine brings each tile's e2m1 codes (straight from the
// slot, no bytes added in HBM), eight dequantising warps, which read the
// tile's e4m3 block scales themselves one k-block ahead,
// turn them into the bf16 128B-swizzled tile the bf16 MMA reads (e2m1 x e4m3
// has at most 6 significant bits, exact in bf16), and the per-matrix fp32
// tensor scale multiplies the accumulators in the epilogue. Activations and
// the rest of the pipeline are the bf16 kernel's: tokens on the N side,
// gate and up in two TMEM halves, SwiGLU in the epilogue.
//
// Rings: the A (weights) and B (tokens) tiles in STG stages as above, the
// raw codes in RAW stages of RK k-blocks each, filled by a producer warp of
// their own, so the codes run ahead of the A/B ring. Barriers per A/B stage:
// full (TMA of the token tile), deq (256 dequantising threads wrote the A
// tile), empty (the MMAs that read the stage completed); per raw stage:
// raw_full (TMA of the codes), raw_empty (the dequantising threads read
// them). Two instances: few tokens per expert (weight-bound) STG 2, RAW 2,
// RK 4: each stage fetches 128 contiguous bytes of each of 128 rows (a
// one-k-block stage fetches 32, which kept DRAM at about 2 TB/s whatever the
// ring depth), 128B-swizzled so the dequantising reads are conflict-free;
// many tokens per expert (tensor-bound) STG 3, RAW 2, RK 1.
// Warps: 0 token TMA, 1 MMA, 2..5 epilogue, 6..13 dequantising, 14 code TMA.
// ---------------------------------------------------------------------------
constexpr int F_CODE_BYTES = BM * BK / 2;  // 4 KB: 128 rows x 32 code bytes (64 values)
constexpr int F_RAW_BYTES = 2 * F_CODE_BYTES;
constexpr int F_DEQ_WARPS = 8;
constexpr int F_CODE_WARP = 6 + F_DEQ_WARPS;
constexpr int F_THREADS = (F_CODE_WARP + 1) * 32;
template <int STG, int RAW, int RK>
constexpr int f_smem_bytes() {
  static_assert((3 * STG + 2 * RAW + 5) * 8 <= 256, "barriers");
  return STG * STAGE_BYTES + RAW * RK * F_RAW_BYTES + 1024 + 256;
}
constexpr int F_TOK_PER_EXPERT_DEEP = 128;  // up to this many rows per routed expert: the deep code ring

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Four e2m1 code bytes (8 values, even value in the low nibble) times one
// e4m3 block scale -> four bf16 pairs, exactly.
__device__ __forceinline__ uint4 fp4x8_to_bf16x8(uint32_t codes, uint32_t scale_byte) {
  uint32_t h[4];
  asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %4;\n"
      " cvt.rn.f16x2.e2m1x2 %0, b0;\n cvt.rn.f16x2.e2m1x2 %1, b1;\n"
      " cvt.rn.f16x2.e2m1x2 %2, b2;\n cvt.rn.f16x2.e2m1x2 %3, b3;\n}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(codes));
  uint32_t s2;
  asm("{\n .reg .b16 t;\n cvt.u16.u32 t, %1;\n cvt.rn.f16x2.e4m3x2 %0, t;\n}" : "=r"(s2) : "r"(scale_byte));
  const __half2 sc = __low2half2(*reinterpret_cast<const __half2*>(&s2));
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 v = __hmul2(*reinterpret_cast<const __half2*>(&h[i]), sc);
    const float2 f = __half22float2(v);
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    o[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

struct TcFp4Maps {
  CUtensorMap code_a, code_b;  // phase 0: gate / up codes; phase 1: down codes (b unused)
};

template <int STG, int RAW, int RK>
__global__ void __launch_bounds__(F_THREADS, 1) gemm_tc_fp4_kernel(const __grid_constant__ CUtensorMap tm_b,
                                                                   const __grid_constant__ TcFp4Maps fm, TcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ WorkItem s_items[MAX_E];
  __shared__ int s_pref[MAX_E + 1];
  __shared__ int s_abort;
  __shared__ uint32_t s_tmem;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* raw = smem + STG * STAGE_BYTES;
  constexpr int RAW_STAGE = RK * F_RAW_BYTES;  // RK k-blocks of codes of both matrices
  uint64_t* bars = reinterpret_cast<uint64_t*>(raw + RAW * RAW_STAGE);
  const uint32_t bar_full = smem_u32(bars), bar_empty = bar_full + 8 * STG, bar_deq = bar_empty + 8 * STG;
  const uint32_t bar_rfull = bar_deq + 8 * STG, bar_rempty = bar_rfull + 8 * RAW;
  const uint32_t bar_acc_full = bar_rempty + 8 * RAW, bar_acc_empty = bar_acc_full + 16;
  const uint32_t bar_drain = bar_acc_empty + 16;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &s_abort;
  constexpr int DEQ_THREADS = F_DEQ_WARPS * 32;

  const int n_items = a.work->n_items[KIND_HIT];
  for (int i = threadIdx.x; i < n_items; i += F_THREADS) s_items[i] = a.work->items[KIND_HIT][i];
  if (threadIdx.x == 0) {
    s_abort = 0;
    for (int s = 0; s < STG; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
      mbar_init(bar_deq + 8 * s, DEQ_THREADS);
    }
    for (int r = 0; r < RAW; ++r) {
      mbar_init(bar_rfull + 8 * r, 1);
      mbar_init(bar_rempty + 8 * r, DEQ_THREADS);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_acc_full + 8 * b, 1);
      mbar_init(bar_acc_empty + 8 * b, 4);
    }
    mbar_init(bar_drain, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), 512);
    tmem_relinquish();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int p = 0;
    for (int i = 0; i < n_items; ++i) {
      s_pref[i] = p;
      p += (s_items[i].n_tok + MAX_N - 1) / MAX_N;
    }
    s_pref[n_items] = p;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int n_units = n_items > 0 ? s_pref[n_items] * a.m_tiles : 0;
  const int two_a = a.phase == 0;
  const int n_mat = two_a ? 2 : 1;

  int last_round[STG], last_raw[RAW];  // producer: last round issued per stage (-1 none)
#pragma unroll
  for (int s = 0; s < STG; ++s) last_round[s] = -1;
#pragma unroll
  for (int r = 0; r < RAW; ++r) last_raw[r] = -1;
  if (warp == 0) {
    // ---------------- TMA producer: token tiles ----------------
    int it = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const int nb = (un.nrows + BOX_ROWS - 1) / BOX_ROWS;
      const uint32_t b_bytes = nb * BOX_ROWS * BK * 2;
      bool ok = true;
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
        const int s = it % STG, r = it / STG;
        if (!mbar_wait(bar_empty + 8 * s, (r & 1) ^ 1, abort, a.error)) {
          ok = false;
          break;
        }
        last_round[s] = r;
        if (lane == 0) {
          const uint32_t base = smem_u32(smem + s * STAGE_BYTES);
          mbar_expect_tx(bar_full + 8 * s, b_bytes);
          for (int b = 0; b < nb; ++b)
            tma_load_2d(base + 2 * A_BYTES + b * BOX_ROWS * 128, &tm_b, bar_full + 8 * s, kb * BK,
                        un.p0 + b * BOX_ROWS);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    int it = 0, ui = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x, ++ui) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const int n_mma = (un.nrows + 15) & ~15;
      const uint32_t idesc = idesc_bf16(BM, n_mma);
      const int ab = two_a ? 0 : (ui & 1), use = two_a ? ui : (ui >> 1);
      if (!mbar_wait(bar_acc_empty + 8 * ab, (use & 1) ^ 1, abort, a.error)) break;
      const uint32_t dacc = tmem + (uint32_t)(ab * 256);
      tc_fence_after();
      bool ok = true;
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
        const int s = it % STG, r = it / STG;
        if (!mbar_wait(bar_full + 8 * s, r & 1, abort, a.error) || !mbar_wait(bar_deq + 8 * s, r & 1, abort, a.error)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t base = smem_u32(smem + s * STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd = sw128_desc(base + 2 * A_BYTES + kk * 32);
            umma_bf16(dacc, sw128_desc(base + kk * 32), bd, idesc, (kb | kk) != 0);
            if (two_a) umma_bf16(tmem + 256, sw128_desc(base + A_BYTES + kk * 32), bd, idesc, (kb | kk) != 0);
          }
          umma_commit(bar_empty + 8 * s);
          if (kb == a.k_blocks - 1) umma_commit(bar_acc_full + 8 * ab);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
  } else if (warp == F_CODE_WARP) {
    // ------- TMA producer: weight codes, RK k-blocks per stage, up to RAW stages ahead -------
    int it = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const uint32_t r_bytes = n_mat * RK * F_CODE_BYTES;
      const int row0 = un.mt * BM;
      bool ok = true;
      for (int kb = 0; kb < a.k_blocks; kb += RK, ++it) {  // k_blocks is a multiple of RK
        const int q = it % RAW, rq = it / RAW;
        if (!mbar_wait(bar_rempty + 8 * q, (rq & 1) ^ 1, abort, a.error)) {
          ok = false;
          break;
        }
        last_raw[q] = rq;
        if (lane == 0) {
          const uint32_t rb = smem_u32(raw + q * RAW_STAGE);
          mbar_expect_tx(bar_rfull + 8 * q, r_bytes);
          tma_load_3d(rb, &fm.code_a, bar_rfull + 8 * q, kb * (BK / 2), row0, un.slot);
          if (two_a)
            tma_load_3d(rb + RK * F_CODE_BYTES, &fm.code_b, bar_rfull + 8 * q, kb * (BK / 2), row0, un.slot);
        }
        __syncwarp();
      }
      if (!ok) break;
    }
  } else if (warp < 6) {
    // ---------------- epilogue (warps 2..5) ----------------
    const int q = warp & 3;
    const uint32_t lane_base = (uint32_t)(32 * q) << 16;
    int ui = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x, ++ui) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const int ab = two_a ? 0 : (ui & 1), use = two_a ? ui : (ui >> 1);
      if (!mbar_wait(bar_acc_full + 8 * ab, use & 1, abort, a.error)) break;
      tc_fence_after();
      const float* ts = a.tscale + ((size_t)a.layer * a.E + un.e) * 3;
      const int row = un.mt * BM + 32 * q + lane;
      for (int c0 = 0; c0 < un.nrows; c0 += 32) {
        uint32_t g[32];
        tmem_ld32(tmem + (uint32_t)(ab * 256) + lane_base + c0, g);
        if (two_a) {
          uint32_t uu[32];
          tmem_ld32(tmem + lane_base + 256 + c0, uu);
          tmem_ld_wait();
          const float t0 = ts[0], t1 = ts[1];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if (c0 + i < un.nrows) {
              const float gv = __uint_as_float(g[i]) * t0, uv = __uint_as_float(uu[i]) * t1;
              const float hv = gv / (1.f + expf(-gv)) * uv;
              a.hs[(size_t)(un.p0 + c0 + i) * a.d_ff + row] = __float2bfloat16_rn(hv);
            }
          }
        } else {
          tmem_ld_wait();
          const float t2 = ts[2];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < un.nrows) a.ybuf[(size_t)(un.p0 + c0 + i) * a.d + row] = __uint_as_float(g[i]) * t2;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_acc_empty + 8 * ab);
    }
  } else {
    // ---------------- dequantising warps (6..13) ----------------
    // thread dt owns half-rows dt (and dt + 256 for gate/up): (matrix, row,
    // half) = (i / 256, (i % 256) / 2, i % 2). A k-block's block scales of a
    // row are 4 bytes of the matrix's scale row, the thread's two are the
    // 16-bit half h; one 16-byte load brings a row's scales of 4 k-blocks,
    // issued a group of 4 k-blocks ahead of its use (loading each k-block's
    // scales one k-block ahead held the kernel at the load latency), and the
    // thread's halves of the 4 words are packed into two registers
    const int dt = threadIdx.x - 6 * 32;  // 0..255
    const size_t n = (size_t)a.d * a.d_ff;
    const int K = two_a ? a.d : a.d_ff;   // a multiple of 256: scale rows are 16-byte aligned
    const size_t sc0 = 3 * (n / 2) + (two_a ? 0 : n / 8);  // scales of gate (phase 0) or down (phase 1)
    const uint32_t sel = (dt & 1) ? 0x7632u : 0x5410u;  // bytes 2h, 2h+1 of two words
    int it = 0;
    for (int u = blockIdx.x; u < n_units && !*abort; u += gridDim.x) {
      Unit un;
      if (!unit_at(a, s_items, s_pref, n_items, u, un)) break;
      const uint8_t* blob = a.slots + (size_t)un.slot * a.slot_bytes;
      const uint4* srow[2];
#pragma unroll
      for (int v = 0; v < 2; ++v) {
        const int i = dt + v * DEQ_THREADS;
        const int m = i / (2 * BM), row = un.mt * BM + ((i % (2 * BM)) >> 1);
        srow[v] = reinterpret_cast<const uint4*>(blob + sc0 + m * (n / 16) + (size_t)row * (K / 16));
      }
      uint4 sraw[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
      uint2 scur[2] = {make_uint2(0, 0), make_uint2(0, 0)};
#pragma unroll
      for (int v = 0; v < 2; ++v)
        if (v < n_mat) sraw[v] = __ldg(srow[v]);
      bool ok = true;
      for (int kb = 0; kb < a.k_blocks; ++kb, ++it) {
        const int s = it % STG, r = it / STG, q = (it / RK) % RAW, rq = (it / RK) / RAW, jr = it % RK;
        const int j = kb & 3;
        if (j == 0) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            if (v < n_mat) {
              scur[v] = make_uint2(__byte_perm(sraw[v].x, sraw[v].y, sel), __byte_perm(sraw[v].z, sraw[v].w, sel));
              if (kb + 4 < a.k_blocks) sraw[v] = __ldg(srow[v] + (kb / 4 + 1));
            }
          }
        }
        uint32_t scc[2];
#pragma unroll
        for (int v = 0; v < 2; ++v) scc[v] = ((j < 2 ? scur[v].x : scur[v].y) >> (16 * (j & 1))) & 0xFFFFu;
        if (!mbar_wait(bar_rfull + 8 * q, rq & 1, abort, a.error) ||
            !mbar_wait(bar_empty + 8 * s, (r & 1) ^ 1, abort, a.error)) {
          ok = false;
          break;
        }
        const uint8_t* rb = raw + q * RAW_STAGE;
        uint8_t* ab_tile = smem + s * STAGE_BYTES;
#pragma unroll
        for (int v = 0; v < 2; ++v) {
          if (v >= n_mat) break;
          const int i = dt + v * DEQ_THREADS;
          const int m = i / (2 * BM), row = (i % (2 * BM)) >> 1, h = i & 1;
          // row `row` of the stage holds RK k-blocks of codes (32 bytes each);
          // with RK = 4 the 128-byte rows are 128B-swizzled by the TMA
          const int chunk = RK == 4 ? ((2 * jr + h) ^ (row & 7)) : 2 * jr + h;
          const uint4 codes =
              *reinterpret_cast<const uint4*>(rb + m * RK * F_CODE_BYTES + row * (32 * RK) + chunk * 16);
          const uint32_t s0 = scc[v] & 0xFF, s1 = (scc[v] >> 8) & 0xFF;
          uint8_t* dst = ab_tile + m * A_BYTES + row * 128;
          const int sw = row & 7;
          *reinterpret_cast<uint4*>(dst + (((4 * h + 0) ^ sw) << 4)) = fp4x8_to_bf16x8(codes.x, s0);
          *reinterpret_cast<uint4*>(dst + (((4 * h + 1) ^ sw) << 4)) = fp4x8_to_bf16x8(codes.y, s0);
          *reinterpret_cast<uint4*>(dst + (((4 * h + 2) ^ sw) << 4)) = fp4x8_to_bf16x8(codes.z, s1);
          *reinterpret_cast<uint4*>(dst + (((4 * h + 3) ^ sw) << 4)) = fp4x8_to_bf16x8(codes.w, s1);
        }
        // the MMAs read the tile through the async proxy
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(bar_deq + 8 * s);
        if (jr == RK - 1) mbar_arrive(bar_rempty + 8 * q);
      }
      if (!ok) break;
    }
  }
  __syncthreads();
  if (warp == 0) {
    // producer tail: every stage's last round released (normal exit) or at
    // least landed (abort) before shared memory goes away
    for (int s = 0; s < STG; ++s) {
      if (last_round[s] < 0) continue;
      const uint32_t bar = *abort ? bar_full + 8 * s : bar_empty + 8 * s;
      const long long t0 = clock64();
      while (!mbar_try_wait(bar, last_round[s] & 1) && clock64() - t0 < WAIT_CYCLES / 4) {
      }
    }
  } else if (warp == F_CODE_WARP) {
    // code producer tail: every raw stage's last copy landed
    for (int q = 0; q < RAW; ++q) {
      if (last_raw[q] < 0) continue;
      const long long t0 = clock64();
      while (!mbar_try_wait(bar_rfull + 8 * q, last_raw[q] & 1) && clock64() - t0 < WAIT_CYCLES / 4) {
      }
    }
  } else if (warp == 1 && *abort) {
    if (lane == 0) umma_commit(bar_drain);
    __syncwarp();
    const long long t0 = clock64();
    while (!mbar_try_wait(bar_drain, 0) && clock64() - t0 < WAIT_CYCLES / 4) {
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// X_s[p, :] = x[perm[p] / k, :] (bf16 rows, 16-byte vectors); grid (rows), 256 threads.
__global__ void __launch_bounds__(256) gather_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const int32_t* __restrict__ perm, int k, int d,
                                                          __nv_bfloat16* __restrict__ xs) {
  const int p = blockIdx.x;
  const int t = perm[p] / k;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  uint4* dst = reinterpret_cast<uint4*>(xs + (size_t)p * d);
  for (int i = threadIdx.x; i < d / 8; i += 256) dst[i] = __ldg(src + i);
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool encode_2d(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)BK, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3D byte map over the slot pool: `row_bytes` per row, `rows` rows per slot,
// `slots` slots `slot_bytes` apart, starting `off` bytes into each slot; box
// of box_x bytes x BM rows x 1 slot (box_x = 128 with the 128-byte swizzle).
bool encode_3d_u8(CUtensorMap* m, const uint8_t* slots, size_t off, uint64_t row_bytes, uint64_t rows,
                  uint64_t n_slots, uint64_t slot_bytes, uint32_t box_x, bool swizzle128 = false) {
  cuuint64_t dims[3] = {row_bytes, rows, n_slots};
  cuuint64_t strides[2] = {row_bytes, slot_bytes};
  cuuint32_t box[3] = {box_x, (cuuint32_t)BM, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, (void*)(slots + off), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE,
                              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

bool prefill_tc_supported(const Shape& sh) {
  if (sh.C <= 0 || sh.d % BM || sh.d_ff % BM) return false;
  // NVFP4: the dequantising warps read each row's block scales 16 bytes (four
  // k-blocks) at a time, so the scale rows (K / 16 bytes) are 16-byte multiples
  if (sh.wtype == FT_W_NVFP4) return sh.d % 256 == 0 && sh.d_ff % 256 == 0;
  return sh.wtype == FT_W_BF16;
}

cudaError_t prefill_tc_init(const Shape& sh, DevState& ds, int max_rows) {
  if (!g_encode) {
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", (void**)&g_encode, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !g_encode) return cudaErrorNotSupported;
  }
  TcPlan* p = new (std::nothrow) TcPlan();
  if (!p) return cudaErrorMemoryAllocation;
  ds.tc_plan = p;  // owned by the context (prefill_tc_free)
  const uint64_t C = (uint64_t)sh.C;
  p->fp4 = sh.wtype == FT_W_NVFP4;
  if (!p->fp4) {
    if (!encode_2d(&p->a_gu, ds.slots, C * 3 * sh.d_ff, sh.d, BM)) return cudaErrorInvalidValue;
    if (!encode_2d(&p->a_dn, ds.slots, C * 3 * sh.d, sh.d_ff, BM)) return cudaErrorInvalidValue;
  } else {
    const size_t n = (size_t)sh.d * sh.d_ff;
    const uint8_t* sl = ds.slots;
    const bool ok = encode_3d_u8(&p->f_code[0], sl, 0, sh.d / 2, sh.d_ff, C, sh.slot_bytes, BK / 2) &&
                    encode_3d_u8(&p->f_code[1], sl, n / 2, sh.d / 2, sh.d_ff, C, sh.slot_bytes, BK / 2) &&
                    encode_3d_u8(&p->f_code[2], sl, n, sh.d_ff / 2, sh.d, C, sh.slot_bytes, BK / 2) &&
                    encode_3d_u8(&p->f_code4[0], sl, 0, sh.d / 2, sh.d_ff, C, sh.slot_bytes, 4 * BK / 2, true) &&
                    encode_3d_u8(&p->f_code4[1], sl, n / 2, sh.d / 2, sh.d_ff, C, sh.slot_bytes, 4 * BK / 2, true) &&
                    encode_3d_u8(&p->f_code4[2], sl, n, sh.d_ff / 2, sh.d, C, sh.slot_bytes, 4 * BK / 2, true);
    if (!ok) return cudaErrorInvalidValue;
  }
  if (!encode_2d(&p->b_x, ds.xs, (uint64_t)max_rows + 256, sh.d, BOX_ROWS)) return cudaErrorInvalidValue;
  if (!encode_2d(&p->b_h, ds.hs, (uint64_t)max_rows + 256, sh.d_ff, BOX_ROWS)) return cudaErrorInvalidValue;

  cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tc_fp4_kernel<2, 2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             f_smem_bytes<2, 2, 4>());
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(gemm_tc_fp4_kernel<3, 2, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             f_smem_bytes<3, 2, 1>());
  if (e != cudaSuccess) return e;
  int dev = 0;
  cudaGetDevice(&dev);
  return cudaDeviceGetAttribute(&p->sms, cudaDevAttrMultiProcessorCount, dev);
}

void prefill_tc_free(DevState& ds) {
  delete static_cast<TcPlan*>(ds.tc_plan);
  ds.tc_plan = nullptr;
}

void launch_prefill_gather(const Shape& sh, const void* x, int T, DevState& ds, cudaStream_t st) {
  gather_rows_kernel<<<T * sh.k, 256, 0, st>>>((const __nv_bfloat16*)x, ds.perm, sh.k, sh.d, ds.xs);
}

void launch_gemm_tc(const Shape& sh, int phase, int layer, int T, DevState& ds, cudaStream_t st) {
  const TcPlan& p = *static_cast<const TcPlan*>(ds.tc_plan);
  TcArgs a;
  a.work = ds.work;
  a.tscale = ds.tscale;
  a.slots = ds.slots;
  a.slot_bytes = sh.slot_bytes;
  a.layer = layer;
  a.E = sh.E;
  a.phase = phase;
  a.d = sh.d;
  a.d_ff = sh.d_ff;
  a.m_tiles = (phase == 0 ? sh.d_ff : sh.d) / BM;
  a.k_blocks = (phase == 0 ? sh.d : sh.d_ff) / BK;
  a.hs = ds.hs;
  a.ybuf = ds.ybuf;
  a.error = ds.error;
  if (p.fp4) {
    const CUtensorMap& tb = phase == 0 ? p.b_x : p.b_h;
    TcFp4Maps fm;
    if ((long long)T * sh.k <= (long long)F_TOK_PER_EXPERT_DEEP * sh.E) {
      fm.code_a = p.f_code4[phase == 0 ? 0 : 2];
      fm.code_b = p.f_code4[1];
      gemm_tc_fp4_kernel<2, 2, 4><<<p.sms, F_THREADS, f_smem_bytes<2, 2, 4>(), st>>>(tb, fm, a);
    } else {
      fm.code_a = p.f_code[phase == 0 ? 0 : 2];
      fm.code_b = p.f_code[1];
      gemm_tc_fp4_kernel<3, 2, 1><<<p.sms, F_THREADS, f_smem_bytes<3, 2, 1>(), st>>>(tb, fm, a);
    }
    return;
  }
  gemm_tc_kernel<<<p.sms, THREADS, SMEM_BYTES, st>>>(phase == 0 ? p.a_gu : p.a_dn, phase == 0 ? p.b_x : p.b_h, a);
}

}  // namespace ft
