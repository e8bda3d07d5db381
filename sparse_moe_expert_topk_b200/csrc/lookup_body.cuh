// One lookup batch of the shared LRU slot cache, as a device function for a
// 1024-thread CTA: used by the standalone lookup kernel and by the fused
// decode routing kernel. See k_lookup.cu for the rules it implements.
#pragma once

#include "ft_internal.cuh"

namespace ft {
namespace lookup_detail {

constexpr int NT = 1024;  // threads of the CTA running a lookup
constexpr unsigned long long NOKEY = ~0ull;
constexpr int SLOT_BITS = 20;

struct ScanTmp {
  int warp_tot[32];
  int total;
};

// Exclusive prefix of a 0/1 flag over the 1024 threads; *total = sum.
__device__ __forceinline__ int block_scan_flag(bool f, ScanTmp& s, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned b = __ballot_sync(0xffffffffu, f);
  const int in_warp = __popc(b & ((1u << lane) - 1u));
  __syncthreads();
  if (lane == 0) s.warp_tot[warp] = __popc(b);
  __syncthreads();
  if (warp == 0) {
    const int v = s.warp_tot[lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    s.warp_tot[lane] = incl - v;
    if (lane == 31) s.total = incl;
  }
  __syncthreads();
  total = s.total;
  return s.warp_tot[warp] + in_warp;
}

// Per-class ranks and totals of a class tag (0..2, or -1) over the 1024
// threads in two barriers: rank of the thread among its class (in thread
// order), and per class the count, a token sum and a chunk sum.
struct Scan3Tmp {
  int cnt[3][32], tok[3][32], ch[3][32], base[3][32];
  int tot_cnt[3], tot_tok[3], tot_ch[3];
};
__device__ __forceinline__ int block_scan3(int cls, int tok, int ch, Scan3Tmp& s) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int in_warp = 0;
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    const unsigned b = __ballot_sync(0xffffffffu, cls == c);
    if (cls == c) in_warp = __popc(b & ((1u << lane) - 1u));
    int t = cls == c ? tok : 0, h = cls == c ? ch : 0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      t += __shfl_xor_sync(0xffffffffu, t, o);
      h += __shfl_xor_sync(0xffffffffu, h, o);
    }
    if (lane == 0) {
      s.cnt[c][warp] = __popc(b);
      s.tok[c][warp] = t;
      s.ch[c][warp] = h;
    }
  }
  __syncthreads();
  if (warp < 3) {
    const int c = warp;
    const int v = s.cnt[c][lane];
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    s.base[c][lane] = incl - v;
    int t = s.tok[c][lane], h = s.ch[c][lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      t += __shfl_xor_sync(0xffffffffu, t, o);
      h += __shfl_xor_sync(0xffffffffu, h, o);
    }
    if (lane == 31) s.tot_cnt[c] = incl;
    if (lane == 0) {
      s.tot_tok[c] = t;
      s.tot_ch[c] = h;
    }
  }
  __syncthreads();
  return cls >= 0 ? s.base[cls][warp] + in_warp : 0;
}

__device__ __forceinline__ unsigned long long slot_key(const unsigned long long* stamp, long long s,
                                                       unsigned long long epoch) {
  const unsigned long long st = stamp[s];
  return st < epoch ? ((st << SLOT_BITS) | (unsigned long long)s) : NOKEY;
}

// s_counts / s_offsets: the routing counts and offsets when the calling CTA
// already holds them in shared memory (else null: read from global memory).
__device__ __forceinline__ void lookup_body(const LookupArgs& a, int E, long long C, size_t slot_bytes,
                                            DevState& ds, const int32_t* s_counts = nullptr,
                                            const int32_t* s_offsets = nullptr) {
  const int32_t* counts = s_counts ? s_counts : (a.counts_src ? a.counts_src : ds.counts);
  const bool pf = a.prefetch != 0;
  const int32_t* offsets = s_offsets ? s_offsets : ds.offsets;
  __shared__ int s_e[MAX_E];
  __shared__ int s_slot_of[MAX_E];
  __shared__ int s_slot[MAX_E];
  __shared__ int s_vic[MAX_E];
  __shared__ unsigned long long s_cand[MAX_E];
  __shared__ int s_hist[256];
  __shared__ ScanTmp scan;
  __shared__ Scan3Tmp scan3;
  __shared__ unsigned long long s_prefix, s_mask;
  __shared__ int s_remaining, s_ncand, s_avail;
  __shared__ unsigned long long s_c0, s_epoch, s_bstart;
  __shared__ int s_cbase, s_lbase;

  const int tid = threadIdx.x;
  Mailbox* mb = ds.mbox;
  const int layer = a.layer;
  // the loads every later step depends on go out first, so that their
  // latency overlaps the batch scan: each expert's slot, and the clock
  const int my_slot = tid < E ? ds.slot_of[layer * E + tid] : -1;
  unsigned long long clk0 = 0, bstart0 = 0;
  int cbase0 = 0, lbase0 = 0;
  if (tid == 0) {
    clk0 = ds.clk->clock;
    bstart0 = ds.clk->batch_start;
    if (a.append) {
      cbase0 = mb->n_copy;
      lbase0 = mb->n_lookup;
    }
  }

  // 1. the batch: routed experts (counts > 0) or all E, ascending
  const bool in = tid < E && (a.use_counts ? counts[tid] > 0 : true);
  int n_u;
  const int upos = block_scan_flag(in, scan, n_u);
  if (in) s_e[upos] = tid;
  if (tid < E) s_slot_of[tid] = my_slot;
  __syncthreads();

  // 2. hits
  const bool act = tid < n_u;
  int e = -1, key = -1, sl = -1;
  if (act) {
    e = s_e[tid];
    key = layer * E + e;
    sl = s_slot_of[e];
    if (sl >= C) {  // corrupt table: report and treat as a miss
      atomicExch(ds.error, (uint32_t)DERR_BAD_INDEX);
      sl = -1;
    }
  }
  const bool hit = act && sl >= 0;
  const int hm_rank = block_scan3(act ? (hit ? 0 : 1) : -1, 0, 0, scan3);
  const int h = scan3.tot_cnt[0], m = scan3.tot_cnt[1];
  const int hrank = hit ? hm_rank : 0, mrank = (act && !hit) ? hm_rank : 0;

  // 3. clock and pins
  if (tid == 0) {
    s_c0 = clk0;
    s_bstart = clk0 + 1;
    s_epoch = a.pin_prev ? bstart0 : clk0 + 1;
    s_cbase = cbase0;
    s_lbase = lbase0;
  }
  __syncthreads();
  const unsigned long long c0 = s_c0, epoch = s_epoch;
  if (hit && !pf) ds.stamp[sl] = c0 + 1 + (unsigned long long)hrank;  // a prefetch leaves hits alone

  // 4. q*
  int q, q_stage;
  if (a.limit_q) {
    q = 0;
    if (m > 0) {
      const unsigned long long num = 2ull * (unsigned long long)m * a.bp_mbps + a.bh_mbps;
      const unsigned long long qq = num / (2ull * a.bh_mbps);
      q = (int)(qq > (unsigned long long)m ? m : qq);
    }
    const long long room = C - h;
    q_stage = (long long)q < room ? q : (int)room;
  } else {
    q = -1;
    q_stage = m;
  }
  __syncthreads();  // hit stamps visible before victim selection

  // 5. victims: the q_stage smallest keys among unpinned slots
  if (q_stage > 0) {
    int avail_local = 0;
    for (long long s = tid; s < C; s += NT) avail_local += slot_key(ds.stamp, s, epoch) != NOKEY;
    if (tid == 0) s_avail = 0;
    __syncthreads();
    for (int o = 16; o > 0; o >>= 1) avail_local += __shfl_xor_sync(0xffffffffu, avail_local, o);
    if ((tid & 31) == 0) atomicAdd(&s_avail, avail_local);
    __syncthreads();
    if (s_avail < q_stage) {  // a prefetch stages what fits; a lookup must not run short
      if (tid == 0 && !pf) atomicExch(ds.error, (uint32_t)DERR_NO_VICTIM);
      q_stage = s_avail;
    }
  }
  if (q_stage > 0 && q_stage <= 8) {
    // a few victims: repeated arg-min over the keys above the previous pick
    unsigned long long prev = 0;
    for (int v = 0; v < q_stage; ++v) {
      unsigned long long best = NOKEY;
      for (long long sidx = tid; sidx < C; sidx += NT) {
        const unsigned long long k = slot_key(ds.stamp, sidx, epoch);
        if (k != NOKEY && (v == 0 || k > prev) && k < best) best = k;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long ob = __shfl_xor_sync(0xffffffffu, best, o);
        best = ob < best ? ob : best;
      }
      if ((tid & 31) == 0) s_cand[tid >> 5] = best;
      __syncthreads();
      if (tid < 32) {
        unsigned long long b2 = s_cand[tid];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b2, o);
          b2 = ob < b2 ? ob : b2;
        }
        if (tid == 0) {
          s_prefix = b2;
          s_vic[v] = (int)(b2 & ((1ull << SLOT_BITS) - 1));
        }
      }
      __syncthreads();
      prev = s_prefix;
    }
  } else if (q_stage > 0) {
    if (tid == 0) {
      s_prefix = 0;
      s_mask = 0;
      s_remaining = q_stage;
    }
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += NT) s_hist[i] = 0;
      __syncthreads();
      const unsigned long long pre = s_prefix, msk = s_mask;
      for (long long s = tid; s < C; s += NT) {
        const unsigned long long k = slot_key(ds.stamp, s, epoch);
        if (k != NOKEY && (k & msk) == pre) atomicAdd(&s_hist[(k >> shift) & 255], 1);
      }
      __syncthreads();
      if (tid == 0) {
        int rem = s_remaining, b = 0;
        for (; b < 256; ++b) {
          if (s_hist[b] >= rem) break;
          rem -= s_hist[b];
        }
        s_remaining = rem;
        s_prefix = pre | ((unsigned long long)b << shift);
        s_mask = msk | (255ull << shift);
      }
      __syncthreads();
    }
    const unsigned long long thr = s_prefix;  // the q_stage-th smallest key
    if (tid == 0) s_ncand = 0;
    __syncthreads();
    for (long long s = tid; s < C; s += NT) {
      const unsigned long long k = slot_key(ds.stamp, s, epoch);
      if (k != NOKEY && k <= thr) {
        const int i = atomicAdd(&s_ncand, 1);
        if (i < MAX_E) s_cand[i] = k;
      }
    }
    __syncthreads();
    if (s_ncand != q_stage) {  // cannot happen with unique keys; stay memory safe if it does
      if (tid == 0) atomicExch(ds.error, (uint32_t)DERR_NO_VICTIM);
      q_stage = 0;
    }
    if (tid < q_stage) {
      const unsigned long long mine = s_cand[tid];
      int r = 0;
      for (int j = 0; j < q_stage; ++j) r += s_cand[j] < mine;
      s_vic[r] = (int)(mine & ((1ull << SLOT_BITS) - 1));
    }
    __syncthreads();
  }

  // 6. insert the staged misses
  const bool staged = act && !hit && mrank < q_stage;
  if (staged) {
    const int v = s_vic[mrank];
    const int old = ds.key_of[v];
    if (old >= 0) ds.slot_of[old] = -1;
    ds.key_of[v] = key;
    ds.slot_of[key] = v;
    ds.stamp[v] = c0 + (unsigned long long)(pf ? 0 : h) + 1ull + (unsigned long long)mrank;
    s_slot[tid] = v;
  } else if (act) {
    s_slot[tid] = hit ? sl : -1;
  }
  if (tid == 0) {
    ds.clk->clock = c0 + (unsigned long long)(pf ? 0 : h) + (unsigned long long)q_stage;
    ds.clk->batch_start = s_bstart;
  }
  __syncthreads();
  const int kind = hit ? KIND_HIT : (staged ? KIND_STAGED : KIND_STREAMED);

  // 7. work lists of the routed experts, per class, ascending e, with the
  // tensor-core GEMV scheduling state of each class (ticket and one
  // completion counter per (item, 16-token chunk)) cleared
  if (a.build_work) {
    const int tok = act ? counts[e] : 0;
    const int r = block_scan3(act ? kind : -1, tok, (tok + MMA_CHUNK - 1) / MMA_CHUNK, scan3);
    if (act) {
      WorkItem it;
      it.e = e;
      it.slot = s_slot[tid];
      it.tok_off = offsets[e];
      it.n_tok = tok;
      ds.work->items[kind][r] = it;
    }
    for (int c = 0; c < N_CLASSES; ++c) {
      const int nch = scan3.tot_ch[c] < ds.sched_chunks ? scan3.tot_ch[c] : ds.sched_chunks;
      int32_t* done = ds.sched + N_CLASSES + (size_t)c * ds.sched_chunks;
      for (int i = tid; i < nch; i += NT) done[i] = 0;
    }
    if (tid < N_CLASSES) {
      ds.sched[tid] = 0;
      ds.work->n_items[tid] = scan3.tot_cnt[tid];
      mb->n_tok_cls[tid] = scan3.tot_tok[tid];
    }
  }

  // 8. mailbox for the host (mapped memory) and counters
  const int cbase = s_cbase, lbase = s_lbase;
  if (staged) {
    mb->copy_key[cbase + mrank] = key;
    mb->copy_slot[cbase + mrank] = s_slot[tid];
  }
  if (act && !pf) {
    mb->lookup_e[lbase + tid] = e;
    mb->lookup_kind[lbase + tid] = kind;
  }
  __syncthreads();
  if (tid == 0) {
    mb->n_copy = cbase + q_stage;
    mb->n_lookup = lbase + (pf ? 0 : n_u);
    if (a.is_current) {
      mb->m = m;
      mb->qstar = q;
      mb->qstage = q_stage;
      mb->n_lookup_cur = n_u;
      ds.ctr->last_m = m;
      ds.ctr->last_qstar = q;
      ds.ctr->last_qstage = q_stage;
    } else if (!a.append) {
      mb->m = 0;
      mb->qstar = -1;
      mb->qstage = 0;
      mb->n_lookup_cur = 0;
    }
    if (a.build_work) {
      mb->n_hit_cls = ds.work->n_items[KIND_HIT];
      mb->n_staged_cls = ds.work->n_items[KIND_STAGED];
      mb->n_streamed_cls = ds.work->n_items[KIND_STREAMED];
    }
    mb->pad_error = *ds.error;
    DevCounters* c = ds.ctr;
    if (pf) {
      c->prefetched += q_stage;
      c->bytes_h2d += (unsigned long long)q_stage * slot_bytes;
    } else {
      c->lookups += n_u;
      c->hits += h;
      c->misses += m;
      c->staged += q_stage;
      c->streamed += m - q_stage;
      c->bytes_h2d += (unsigned long long)q_stage * slot_bytes;
      c->bytes_zero_copy += (unsigned long long)(m - q_stage) * slot_bytes;
    }
    // no fence needed: the host reads the mailbox only after an event recorded
    // behind this kernel has completed
  }
}

}  // namespace lookup_detail
}  // namespace ft
