// moe_oracle.cpp -- the routed-MoE layer and its shared LRU expert cache,
// written out plainly in C++: one std::thread per token, each token's layer
// output computed element by element from the slot blobs.
//
// TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and
// bench.py's CPU legs load it (through oracle/cpp.py); it shares no code with
// the CUDA library, and the library never loads it.
//
// What it computes (the pages fix the structure -- [paperlens] "MoEは扉を開
// けると同時に、別の扉を閉める", paper §1: E experts per layer, each token passes
// through k of them -- and not the router or the expert form, so the readings
// documented with the C ABI are taken):
//   s[t,e]  = sum_i x[t,i] W_r[e,i] + b     summed in double in index order,
//                                           rounded once to float
//   ids     = the k largest float logits, larger first, equal -> lower e
//   w_j     = exp(s_j - s_max) / sum over the chosen, in double
//   g_f, u_f = sum_i W[f,i] x_i             in double, rounded to float
//   h_f     = g_f / (1 + exp(-g_f)) * u_f   in float
//   Y_o     = sum_f W_down[o,f] h_f         in double, rounded to float
//   y[t,o]  = sum_j (float) w_j * Y_j[o]    in float, rank order j = 0..k-1
// The weights are decoded from the slot-blob layout of include/ft_moe.h with
// decoders written from the format definitions: bf16 is the top half of an
// IEEE float; e2m1 has a sign bit, two exponent bits with bias 1 and one
// mantissa bit (exponent 0 subnormal: mantissa * 0.5); e4m3 has a sign bit,
// four exponent bits with bias 7 and three mantissa bits (exponent 0
// subnormal: mantissa / 8 * 2^-6; all-ones exponent with all-ones mantissa is
// NaN). An NVFP4 weight is e2m1 x e4m3 block scale x the matrix's fp32 tensor
// scale, the block being 16 consecutive elements along a row.
//
// The cache simulator follows the same readings as the Python oracle's
// ExpertCache (decode lookups in ascending expert order with the q* split
// q* = floor((2 m B_P + B_H) / (2 B_H)) clamped to [0, m], hits stamped
// first, the first min(q*, C - hits) misses inserted, lowest free slot else
// the least recently stamped unpinned slot; prefill with C >= 2E loads a
// whole layer and the next one behind it): [techfeed]
// "帯域適応型実行（q*ポリシー）" and "セマンティック認識キャッシング";
// [paperlens] "プレフィル: 全層ダブルバッファと「意味の錨」", paper §3.1.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <map>
#include <set>
#include <thread>
#include <vector>

namespace {

enum { W_F32 = 0, W_BF16 = 1, W_NVFP4 = 2 };

double e2m1_value(int code) {
  const double sign = (code & 8) ? -1.0 : 1.0;
  const int ex = (code >> 1) & 3, man = code & 1;
  if (ex == 0) return sign * man * 0.5;
  return sign * std::ldexp(1.0 + man / 2.0, ex - 1);
}

double e4m3_value(int code) {
  const double sign = (code & 0x80) ? -1.0 : 1.0;
  const int ex = (code >> 3) & 15, man = code & 7;
  if (ex == 15 && man == 7) return NAN;
  if (ex == 0) return sign * (man / 8.0) * std::ldexp(1.0, -6);
  return sign * std::ldexp(1.0 + man / 8.0, ex - 7);
}

struct Expert {
  const uint8_t* blob;
  int wtype, d, d_ff;
  const float* tscale;  // 3 floats for NVFP4, else unused

  // element (r, c) of matrix m (0 gate [d_ff][d], 1 up [d_ff][d], 2 down [d][d_ff])
  double at(int m, long r, long c) const {
    const long n = (long)d * d_ff;
    const long K = m == 2 ? d_ff : d;
    const long idx = (long)m * n + r * K + c;
    if (wtype == W_F32) {
      float v;
      std::memcpy(&v, blob + 4 * idx, 4);
      return v;
    }
    if (wtype == W_BF16) {
      uint16_t b;
      std::memcpy(&b, blob + 2 * idx, 2);
      const uint32_t u = (uint32_t)b << 16;
      float v;
      std::memcpy(&v, &u, 4);
      return v;
    }
    const uint8_t byte = blob[idx / 2];
    const int code = (c & 1) ? (byte >> 4) : (byte & 15);
    const uint8_t sc = blob[3 * n / 2 + idx / 16];
    return e2m1_value(code) * e4m3_value(sc) * (double)tscale[m];
  }
};

// One token through one expert: Y [d] floats.
void expert_token(const Expert& ex, const double* x, float* Y) {
  const int d = ex.d, dff = ex.d_ff;
  std::vector<float> h(dff);
  for (int f = 0; f < dff; ++f) {
    double g = 0.0, u = 0.0;
    for (int i = 0; i < d; ++i) {
      g += ex.at(0, f, i) * x[i];
      u += ex.at(1, f, i) * x[i];
    }
    const float gf = (float)g, uf = (float)u;
    h[f] = gf / (1.0f + std::exp(-gf)) * uf;
  }
  for (int o = 0; o < d; ++o) {
    double acc = 0.0;
    for (int f = 0; f < dff; ++f) acc += ex.at(2, o, f) * (double)h[f];
    Y[o] = (float)acc;
  }
}

// Router of one token: ids [k] and weights [k] (double).
void route_token(const double* x, const double* wr, const double* b, int E, int d, int k, int32_t* ids, double* w,
                 float* s32) {
  for (int e = 0; e < E; ++e) {
    double s = 0.0;
    for (int i = 0; i < d; ++i) s += x[i] * wr[(long)e * d + i];
    if (b) s += b[e];
    s32[e] = (float)s;
  }
  std::vector<char> taken(E, 0);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (best < 0 || s32[e] > s32[best])) best = e;  // strict: equal keeps the lower index
    taken[best] = 1;
    ids[j] = best;
  }
  const double top = s32[ids[0]];
  double den = 0.0;
  for (int j = 0; j < k; ++j) den += std::exp((double)s32[ids[j]] - top);
  for (int j = 0; j < k; ++j) w[j] = std::exp((double)s32[ids[j]] - top) / den;
}

// --- the shared LRU cache -------------------------------------------------
constexpr int HIT = 0, STAGED = 1, STREAMED = 2;

struct Cache {
  int L, E;
  long C;
  unsigned bp, bh;
  std::vector<long> key_of;
  std::vector<uint64_t> stamp;
  std::map<long, long> slot_of;
  uint64_t clock = 0;
  int prefetched = -1;
  uint64_t n[6] = {0, 0, 0, 0, 0, 0};  // lookups hits misses staged streamed layer_calls

  long victim(const std::set<long>& pinned) const {
    for (long s = 0; s < C; ++s)
      if (key_of[s] < 0) return s;
    long best = -1;
    for (long s = 0; s < C; ++s)
      if (!pinned.count(s) && (best < 0 || stamp[s] < stamp[best])) best = s;
    return best;
  }
  void touch(long s) { stamp[s] = ++clock; }
  bool insert(long key, std::set<long>& pinned) {
    const long s = victim(pinned);
    if (s < 0) return false;
    if (key_of[s] >= 0) slot_of.erase(key_of[s]);
    key_of[s] = key;
    slot_of[key] = s;
    touch(s);
    pinned.insert(s);
    return true;
  }
  // one lookup batch: kinds[i] for experts[i]; returns false on an internal error
  bool batch(int layer, const std::vector<int>& experts, std::set<long>& pinned, bool limit_q, std::vector<int>& kinds,
             int& m, int& q, int& q_stage) {
    std::vector<int> misses;
    kinds.assign(experts.size(), HIT);
    for (size_t i = 0; i < experts.size(); ++i) {
      const long key = (long)layer * E + experts[i];
      auto it = slot_of.find(key);
      if (it != slot_of.end()) {
        touch(it->second);
        pinned.insert(it->second);
      } else {
        misses.push_back((int)i);
      }
    }
    const int h = (int)(experts.size() - misses.size());
    m = (int)misses.size();
    if (limit_q) {
      long long qq = m > 0 ? (2ll * m * bp + bh) / (2ll * bh) : 0;
      q = (int)std::max(0ll, std::min((long long)m, qq));
      q_stage = (int)std::min((long)q, C - h);
    } else {
      q = -1;
      q_stage = m;
    }
    for (int j = 0; j < m; ++j) {
      const int i = misses[j];
      if (j < q_stage) {
        if (!insert((long)layer * E + experts[i], pinned)) return false;
        kinds[i] = STAGED;
      } else {
        kinds[i] = STREAMED;
      }
    }
    n[0] += experts.size();
    n[1] += h;
    n[2] += m;
    n[3] += q_stage;
    n[4] += m - q_stage;
    return true;
  }
};

}  // namespace

extern "C" {

// Router and layer for T tokens, one std::thread per token (at most
// `threads` at a time). x [T][d], wr [E][d], bias NULL / [E] / [T][E] (all
// double, holding the exact values of the caller's bf16 / fp32 data);
// blobs[e] points at expert e's slot blob; tscales [E][3] for NVFP4 (else
// NULL). Out: y [T][d] float, ids [T][k], w [T][k] double. Returns 0, or -1 on
// a bad argument.
int fto_layer_forward(const double* x, int T, int d, int d_ff, int E, int k, const double* wr, const double* bias,
                      int bias_per_token, const uint8_t* const* blobs, int wtype, const float* tscales, int threads,
                      float* y, int32_t* ids, double* w) {
  if (T < 0 || d < 1 || d_ff < 1 || E < 1 || k < 1 || k > E || !x || !wr || !blobs || !y || !ids || !w) return -1;
  if (wtype == W_NVFP4 && (!tscales || d % 16 || d_ff % 16)) return -1;
  if (threads < 1) threads = 1;
  auto one = [&](int t) {
    std::vector<float> s32(E), Y(d), acc(d, 0.0f);
    const double* b = bias ? bias + (bias_per_token ? (long)t * E : 0) : nullptr;
    route_token(x + (long)t * d, wr, b, E, d, k, ids + (long)t * k, w + (long)t * k, s32.data());
    for (int j = 0; j < k; ++j) {
      const int e = ids[(long)t * k + j];
      const Expert ex{blobs[e], wtype, d, d_ff, tscales ? tscales + 3 * (long)e : nullptr};
      expert_token(ex, x + (long)t * d, Y.data());
      const float wj = (float)w[(long)t * k + j];
      for (int o = 0; o < d; ++o) acc[o] += wj * Y[o];
    }
    std::memcpy(y + (long)t * d, acc.data(), sizeof(float) * d);
  };
  for (int t0 = 0; t0 < T; t0 += threads) {
    std::vector<std::thread> pool;
    for (int t = t0; t < std::min(T, t0 + threads); ++t) pool.emplace_back(one, t);
    for (auto& th : pool) th.join();
  }
  return 0;
}

// Router only: ids [T][k] and weights [T][k] of T tokens (arguments as
// fto_layer_forward). Returns 0, or -1 on a bad argument.
int fto_route(const double* x, int T, int d, int E, int k, const double* wr, const double* bias, int bias_per_token,
              int32_t* ids, double* w) {
  if (T < 0 || d < 1 || E < 1 || k < 1 || k > E || !x || !wr || !ids || !w) return -1;
  std::vector<float> s32(E);
  for (int t = 0; t < T; ++t) {
    const double* b = bias ? bias + (bias_per_token ? (long)t * E : 0) : nullptr;
    route_token(x + (long)t * d, wr, b, E, d, k, ids + (long)t * k, w + (long)t * k, s32.data());
  }
  return 0;
}

// Decoded value of one weight element, for pins against the format tables.
double fto_weight(const uint8_t* blob, int wtype, int d, int d_ff, const float* tscale, int m, long r, long c) {
  const Expert ex{blob, wtype, d, d_ff, tscale};
  return ex.at(m, r, c);
}

double fto_e2m1(int code) { return e2m1_value(code & 15); }
double fto_e4m3(int code) { return e4m3_value(code & 255); }

void* fto_cache_new(int L, int E, long C, unsigned bp_mbps, unsigned bh_mbps) {
  if (L < 1 || E < 1 || C < 0 || bh_mbps == 0) return nullptr;
  Cache* c = new Cache{L, E, C, bp_mbps, bh_mbps, std::vector<long>(C, -1), std::vector<uint64_t>(C, 0), {}};
  return c;
}

void fto_cache_free(void* p) { delete static_cast<Cache*>(p); }

// One layer call of the cache (mode 0 decode, 1 prefill) with counts[E]
// tokens per expert. Out: the lookups in order (layer, expert, kind), their
// number, how many belong to this layer, and m, q*, q_stage. Returns 0, or -1
// (no unpinned slot left: an internal error).
int fto_cache_forward(void* p, int layer, int mode, const int32_t* counts, int32_t* look_layer, int32_t* look_e,
                      int32_t* look_kind, int* n_look, int* n_cur, int* m_out, int* q_out, int* qs_out) {
  Cache& c = *static_cast<Cache*>(p);
  const int E = c.E;
  std::vector<int> routed;
  for (int e = 0; e < E; ++e)
    if (counts[e] > 0) routed.push_back(e);
  *n_look = *n_cur = *m_out = *q_out = *qs_out = 0;
  if (routed.empty()) return 0;
  c.n[5] += 1;
  int nl = 0;
  auto emit = [&](int l, const std::vector<int>& ex, const std::vector<int>& kinds) {
    for (size_t i = 0; i < ex.size(); ++i, ++nl) {
      look_layer[nl] = l;
      look_e[nl] = ex[i];
      look_kind[nl] = kinds[i];
    }
  };
  std::vector<int> kinds;
  int m = 0, q = 0, qs = 0;
  if (mode == 0 || c.C < 2l * E) {
    std::set<long> pinned;
    if (!c.batch(layer, routed, pinned, true, kinds, m, q, qs)) return -1;
    c.prefetched = -1;
    emit(layer, routed, kinds);
    *n_look = *n_cur = nl;
    *m_out = m;
    *q_out = q;
    *qs_out = qs;
    return 0;
  }
  std::vector<int> all(E);
  for (int e = 0; e < E; ++e) all[e] = e;
  if (c.prefetched != layer) {
    std::set<long> pinned;
    if (!c.batch(layer, all, pinned, false, kinds, m, q, qs)) return -1;
    emit(layer, all, kinds);
  }
  *n_cur = nl;
  if (layer + 1 < c.L) {
    std::set<long> pinned;
    for (int e = 0; e < E; ++e) pinned.insert(c.slot_of[(long)layer * E + e]);
    int m2, q2, qs2;
    if (!c.batch(layer + 1, all, pinned, false, kinds, m2, q2, qs2)) return -1;
    emit(layer + 1, all, kinds);
    c.prefetched = layer + 1;
  } else {
    c.prefetched = -1;
  }
  *n_look = nl;
  *m_out = m;
  *q_out = -1;
  *qs_out = qs;
  return 0;
}

// Counters: lookups, hits, misses, staged, streamed, layer_calls.
void fto_cache_counters(void* p, uint64_t* out6) {
  const Cache& c = *static_cast<Cache*>(p);
  for (int i = 0; i < 6; ++i) out6[i] = c.n[i];
}

// Contents: key_of [C] (layer * E + e, or -1) and stamp [C].
void fto_cache_contents(void* p, int64_t* key_of, uint64_t* stamp) {
  const Cache& c = *static_cast<Cache*>(p);
  for (long s = 0; s < c.C; ++s) {
    key_of[s] = c.key_of[s];
    stamp[s] = c.stamp[s];
  }
}

}  // extern "C"
