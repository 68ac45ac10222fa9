// Reference oracle for block-sparse mixed-precision causal attention
// (TriAttention, as summarised on the rit.work TriAttention page,
// rit.work/blog/triattention-sparse-mixed-precision-attention).
//
// TEST INFRASTRUCTURE ONLY. This file is a plain, slow, obviously correct CPU
// statement of what the GPU library computes. Only the tests, the smoke check
// and the benchmark's CPU-baseline leg may load it. It shares no code, header,
// table or constant with the CUDA path, and the CUDA path never calls it.
//
// Build: g++ -std=c++17 -O2 -ffp-contract=off -fno-fast-math -fPIC -shared -pthread
// (no FMA contraction: every fp32 step below rounds exactly once, as written).
//
// What it follows, step by step:
//  * Three actions per block of attention links — skip, compute at 4 bits, or
//    compute at 8 bits (TriAttention page, section "Какие связи можно не
//    считать, а какие нельзя удалять", third paragraph).
//  * The action is chosen by the distance of the block to the diagonal: nearest
//    blocks at high precision, the next at low precision, far ones skipped; the
//    first key block and the diagonal block are always kept at high precision
//    (same section, fourth paragraph).
//  * Per head the policy is a pair of boundaries: one between high and low
//    precision, one between kept and skipped blocks (same section, fifth
//    paragraph). Readings: bands are half-open in the block distance
//    d = i - j: int8 iff d < hi, int4 iff hi <= d < keep, skip iff d >= keep;
//    the pair is per query head.
//  * One normalised softmax result over all kept blocks of both precisions
//    (section "Как калибровка распределяет вычисления между головами", last
//    paragraph), and decode reads the same prepared K/V from the compressed
//    cache with the same boundaries.
//  * Codec (a reading; the page names only "4 bits" and "8 bits"): per token
//    and per plane a symmetric scale s = max|x| / 127 (int8) or max|x| / 7
//    (int4), computed in fp32 with IEEE division; code = clamp(rint(x / s)),
//    round half to even, clamped to [-127, 127] or [-7, 7]; an all-zero row
//    has scale 0 and codes 0. The tile's plane applies to Q, K and V alike.
//  * Scores: exact integer dot product of the codes, times both scales, divided
//    by sqrt(D), in float64. Softmax and P.V in float64 (two passes).
//  * GQA head mapping: kv_head = q_head / (Hq / Hkv) (llmis.ru chapter 3.5,
//    section 4 "Grouped-Query Attention").

#include <cmath>
#include <cstdint>
#include <cstring>
#include <cfenv>
#include <algorithm>
#include <thread>
#include <vector>
#include <atomic>
#include <limits>

namespace {

enum Action { NONE = -1, SKIP = 0, INT4 = 4, INT8 = 8 };

enum Flags {
  // Use the bf16 inputs themselves (as float64) instead of codes x scales.
  FLAG_BYPASS_QUANT = 1,
};

float bf16_to_float(uint16_t h) {
  uint32_t u = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// Tile action for query block i and key block j (see the header comment).
int tile_action(int i, int j, int hi, int keep) {
  if (j > i) return NONE;                 // causal: the key block lies in the future
  if (j == 0 || j == i) return INT8;      // protected: sink block and diagonal block
  const int d = i - j;
  if (d < hi) return INT8;
  if (d < keep) return INT4;
  return SKIP;
}

// One row of the codec: fills both planes for a row of D bf16 values.
void quantize_row(const uint16_t* x, int D, int8_t* c8, float* s8, int8_t* c4, float* s4) {
  float a = 0.0f;
  for (int k = 0; k < D; ++k) a = std::max(a, std::fabs(bf16_to_float(x[k])));
  if (a == 0.0f) {
    *s8 = 0.0f;
    *s4 = 0.0f;
    for (int k = 0; k < D; ++k) { c8[k] = 0; c4[k] = 0; }
    return;
  }
  const volatile float sc8 = a / 127.0f;  // one IEEE fp32 division each
  const volatile float sc4 = a / 7.0f;
  *s8 = sc8;
  *s4 = sc4;
  for (int k = 0; k < D; ++k) {
    const float v = bf16_to_float(x[k]);
    const volatile float q8 = v / sc8;
    const volatile float q4 = v / sc4;
    float r8 = std::nearbyint(q8);  // FE_TONEAREST: ties to even
    float r4 = std::nearbyint(q4);
    r8 = std::min(127.0f, std::max(-127.0f, r8));
    r4 = std::min(7.0f, std::max(-7.0f, r4));
    c8[k] = static_cast<int8_t>(r8);
    c4[k] = static_cast<int8_t>(r4);
  }
}

// Both planes of a set of rows, codes kept unpacked (one int8 per value).
struct Planes {
  std::vector<int8_t> c8, c4;
  std::vector<float> s8, s4;
  void build(const uint16_t* x, int64_t rows, int D) {
    c8.resize(rows * D); c4.resize(rows * D); s8.resize(rows); s4.resize(rows);
    for (int64_t r = 0; r < rows; ++r)
      quantize_row(x + r * D, D, &c8[r * D], &s8[r], &c4[r * D], &s4[r]);
  }
};

// Problem description shared by prefill and decode rows.
struct Problem {
  int B, Hq, Hkv, S, D, T;   // S = tokens per (b, kv head) stored in K/V
  const int32_t* hi;
  const int32_t* keep;
  int flags;
  const uint16_t* K;         // [B, Hkv, S, D] bf16
  const uint16_t* V;
  const Planes* kq;          // quantized K, rows indexed like K
  const Planes* vq;
};

// Score and dequantised value access for key row `kr` (flat index into K/V rows)
// under plane `p`, for query row given as both bf16 values and codes.
struct QueryRow {
  const uint16_t* x;   // D bf16 values
  const int8_t* c8; float s8;
  const int8_t* c4; float s4;
};

double score(const Problem& P, const QueryRow& q, int64_t kr, int plane) {
  const int D = P.D;
  if (P.flags & FLAG_BYPASS_QUANT) {
    double acc = 0.0;
    for (int k = 0; k < D; ++k)
      acc += static_cast<double>(bf16_to_float(q.x[k])) *
             static_cast<double>(bf16_to_float(P.K[kr * D + k]));
    return acc / std::sqrt(static_cast<double>(D));
  }
  const int8_t* cq = plane == INT8 ? q.c8 : q.c4;
  const int8_t* ck = plane == INT8 ? &P.kq->c8[kr * D] : &P.kq->c4[kr * D];
  const double sq = plane == INT8 ? q.s8 : q.s4;
  const double sk = plane == INT8 ? P.kq->s8[kr] : P.kq->s4[kr];
  int64_t acc = 0;
  for (int k = 0; k < D; ++k) acc += static_cast<int64_t>(cq[k]) * static_cast<int64_t>(ck[k]);
  return static_cast<double>(acc) * sq * sk / std::sqrt(static_cast<double>(D));
}

double value(const Problem& P, int64_t kr, int plane, int d) {
  const int D = P.D;
  if (P.flags & FLAG_BYPASS_QUANT) return bf16_to_float(P.V[kr * D + d]);
  if (plane == INT8) return static_cast<double>(P.vq->s8[kr]) * P.vq->c8[kr * D + d];
  return static_cast<double>(P.vq->s4[kr]) * P.vq->c4[kr * D + d];
}

// Keys that query position t (in query block i) attends to among positions
// [0, t], with their plane; `group_base` is the first K/V row of (b, kvh).
struct Kept { int64_t row; int plane; };

void kept_keys(const Problem& P, int t, int hi, int keep, int64_t group_base, std::vector<Kept>& out) {
  out.clear();
  const int i = t / P.T;
  for (int u = 0; u <= t; ++u) {
    const int a = tile_action(i, u / P.T, hi, keep);
    if (a == INT8 || a == INT4) out.push_back({group_base + u, a});
  }
}

// Unnormalised partial over a set of kept keys: m = max score, l = sum exp(s - m),
// o = sum exp(s - m) * v. Two passes in float64.
void partial(const Problem& P, const QueryRow& q, const Kept* keys, size_t n,
             double* m_out, double* l_out, double* o_out) {
  const int D = P.D;
  std::vector<double> s(n);
  double m = -std::numeric_limits<double>::infinity();
  for (size_t e = 0; e < n; ++e) { s[e] = score(P, q, keys[e].row, keys[e].plane); m = std::max(m, s[e]); }
  double l = 0.0;
  for (int d = 0; d < D; ++d) o_out[d] = 0.0;
  for (size_t e = 0; e < n; ++e) {
    const double p = std::exp(s[e] - m);
    l += p;
    for (int d = 0; d < D; ++d) o_out[d] += p * value(P, keys[e].row, keys[e].plane, d);
  }
  *m_out = m;
  *l_out = l;
}

// Full attention row: O = o / l, LSE = m + ln l.
void attention_row(const Problem& P, const QueryRow& q, int t, int hq, int b,
                   double* O, double* LSE, std::vector<Kept>& scratch) {
  const int kvh = hq / (P.Hq / P.Hkv);
  const int64_t base = (static_cast<int64_t>(b) * P.Hkv + kvh) * P.S;
  kept_keys(P, t, P.hi[hq], P.keep[hq], base, scratch);
  double m, l;
  partial(P, q, scratch.data(), scratch.size(), &m, &l, O);
  for (int d = 0; d < P.D; ++d) O[d] /= l;
  *LSE = m + std::log(l);
}

template <class F>
void parallel_for(int64_t n, int nthreads, F&& f) {
  if (nthreads <= 1 || n < 2) { for (int64_t r = 0; r < n; ++r) f(r); return; }
  std::atomic<int64_t> next(0);
  std::vector<std::thread> pool;
  for (int w = 0; w < nthreads; ++w)
    pool.emplace_back([&]() {
      std::fesetround(FE_TONEAREST);
      for (int64_t r; (r = next.fetch_add(1)) < n;) f(r);
    });
  for (auto& th : pool) th.join();
}

int check_dims(int B, int Hq, int Hkv, int S, int D, int T) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || D < 2 || T < 1) return 1;
  if (Hq % Hkv != 0 || D % 2 != 0) return 1;
  return 0;
}

}  // namespace

extern "C" {

// ---- codec ---------------------------------------------------------------

// Quantise `rows` rows of D bf16 values (raw bits) into both planes.
// c8/c4 are unpacked (one int8 per value); s8/s4 one fp32 per row.
void oracle_quantize_rows(const uint16_t* x, int64_t rows, int D,
                          int8_t* c8, float* s8, int8_t* c4, float* s4) {
  std::fesetround(FE_TONEAREST);
  for (int64_t r = 0; r < rows; ++r)
    quantize_row(x + r * D, D, c8 + r * D, s8 + r, c4 + r * D, s4 + r);
}

// Pack unpacked int4 codes two per byte: element 2k in the low nibble,
// element 2k+1 in the high nibble, 4-bit two's complement (a layout reading).
void oracle_pack_int4(const int8_t* c4, int64_t n_values, uint8_t* packed) {
  for (int64_t k = 0; k < n_values / 2; ++k) {
    const uint8_t lo = static_cast<uint8_t>(c4[2 * k]) & 0x0F;
    const uint8_t hi = static_cast<uint8_t>(c4[2 * k + 1]) & 0x0F;
    packed[k] = static_cast<uint8_t>(lo | (hi << 4));
  }
}

// ---- policy --------------------------------------------------------------

int oracle_action(int i, int j, int hi, int keep) { return tile_action(i, j, hi, keep); }

// Action of every (query block i, key block j) tile, row-major [nb][nb].
void oracle_action_map(int nb, int hi, int keep, int32_t* out) {
  for (int i = 0; i < nb; ++i)
    for (int j = 0; j < nb; ++j) out[i * nb + j] = tile_action(i, j, hi, keep);
}

// Tile counts by enumeration: out = {int8, int4, skip} over causal tiles.
void oracle_action_counts(int nb, int hi, int keep, int64_t* out) {
  out[0] = out[1] = out[2] = 0;
  for (int i = 0; i < nb; ++i)
    for (int j = 0; j <= i; ++j) {
      const int a = tile_action(i, j, hi, keep);
      if (a == INT8) ++out[0]; else if (a == INT4) ++out[1]; else if (a == SKIP) ++out[2];
    }
}

// ---- prefill -------------------------------------------------------------

// Attention rows of a prefill. Q [B,Hq,S,D], K/V [B,Hkv,S,D] bf16 (raw bits).
// rows: flat row ids (b*Hq + hq)*S + t; O [nrows, D], LSE [nrows] float64.
// hi/keep: per query head. Returns 0, or 1 on invalid dimensions.
int oracle_prefill_rows(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                        int B, int Hq, int Hkv, int S, int D, int T,
                        const int32_t* hi, const int32_t* keep, int flags,
                        const int64_t* rows, int64_t nrows,
                        double* O, double* LSE, int nthreads) {
  if (check_dims(B, Hq, Hkv, S, D, T)) return 1;
  std::fesetround(FE_TONEAREST);
  const int64_t kv_rows = static_cast<int64_t>(B) * Hkv * S;
  Planes kq, vq;
  if (!(flags & FLAG_BYPASS_QUANT)) { kq.build(K, kv_rows, D); vq.build(V, kv_rows, D); }
  Problem P{B, Hq, Hkv, S, D, T, hi, keep, flags, K, V, &kq, &vq};
  parallel_for(nrows, nthreads, [&](int64_t r) {
    const int64_t id = rows[r];
    const int t = static_cast<int>(id % S);
    const int hq = static_cast<int>((id / S) % Hq);
    const int b = static_cast<int>(id / (static_cast<int64_t>(S) * Hq));
    std::vector<int8_t> c8(D), c4(D);
    float s8, s4;
    const uint16_t* x = Q + id * D;
    quantize_row(x, D, c8.data(), &s8, c4.data(), &s4);
    QueryRow q{x, c8.data(), s8, c4.data(), s4};
    std::vector<Kept> scratch;
    attention_row(P, q, t, hq, b, O + r * D, LSE + r, scratch);
  });
  return 0;
}

// Textbook dense causal softmax attention in float64 with GQA, written without
// tiles, codes or policies: O[t] = sum_{u<=t} softmax_u(q_t.k_u / sqrt(D)) v_u.
int oracle_dense_attention(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                           int B, int Hq, int Hkv, int S, int D,
                           double* O, double* LSE, int nthreads) {
  if (check_dims(B, Hq, Hkv, S, D, 1)) return 1;
  const int G = Hq / Hkv;
  parallel_for(static_cast<int64_t>(B) * Hq * S, nthreads, [&](int64_t id) {
    const int t = static_cast<int>(id % S);
    const int hq = static_cast<int>((id / S) % Hq);
    const int b = static_cast<int>(id / (static_cast<int64_t>(S) * Hq));
    const int64_t kv = (static_cast<int64_t>(b) * Hkv + hq / G) * S;
    std::vector<double> s(t + 1);
    double m = -std::numeric_limits<double>::infinity();
    for (int u = 0; u <= t; ++u) {
      double acc = 0.0;
      for (int k = 0; k < D; ++k)
        acc += static_cast<double>(bf16_to_float(Q[id * D + k])) *
               static_cast<double>(bf16_to_float(K[(kv + u) * D + k]));
      s[u] = acc / std::sqrt(static_cast<double>(D));
      m = std::max(m, s[u]);
    }
    double l = 0.0;
    double* o = O + id * D;
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    for (int u = 0; u <= t; ++u) {
      const double p = std::exp(s[u] - m);
      l += p;
      for (int d = 0; d < D; ++d) o[d] += p * bf16_to_float(V[(kv + u) * D + d]);
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    LSE[id] = m + std::log(l);
  });
  return 0;
}

// ---- decode --------------------------------------------------------------

// One new token per sequence attending to its cache. q [B,Hq,D]; K/V
// [B,Hkv,S,D] with S the capacity; kv_len[b] tokens valid (the query sits at
// position kv_len-1, already in the cache, so its block is the diagonal).
// nsplit = 0: one pass. nsplit >= 1: the kept keys are cut into nsplit
// contiguous runs of key blocks, each reduced to (m, l, o) on its own, then
// merged: m* = max m_s, l = sum e^(m_s-m*) l_s, O = sum e^(m_s-m*) o_s / l.
int oracle_decode(const uint16_t* q, const uint16_t* K, const uint16_t* V,
                  int B, int Hq, int Hkv, int S, int D, int T,
                  const int32_t* kv_len, const int32_t* hi, const int32_t* keep,
                  int flags, int nsplit, double* O, double* LSE, int nthreads) {
  if (check_dims(B, Hq, Hkv, S, D, T) || nsplit < 0) return 1;
  for (int b = 0; b < B; ++b) if (kv_len[b] < 1 || kv_len[b] > S) return 1;
  std::fesetround(FE_TONEAREST);
  const int64_t kv_rows = static_cast<int64_t>(B) * Hkv * S;
  Planes kq, vq;
  if (!(flags & FLAG_BYPASS_QUANT)) { kq.build(K, kv_rows, D); vq.build(V, kv_rows, D); }
  Problem P{B, Hq, Hkv, S, D, T, hi, keep, flags, K, V, &kq, &vq};
  parallel_for(static_cast<int64_t>(B) * Hq, nthreads, [&](int64_t id) {
    const int hq = static_cast<int>(id % Hq);
    const int b = static_cast<int>(id / Hq);
    const int t = kv_len[b] - 1;
    std::vector<int8_t> c8(D), c4(D);
    float s8, s4;
    const uint16_t* x = q + id * D;
    quantize_row(x, D, c8.data(), &s8, c4.data(), &s4);
    QueryRow qr{x, c8.data(), s8, c4.data(), s4};
    std::vector<Kept> keys;
    if (nsplit == 0) { attention_row(P, qr, t, hq, b, O + id * D, LSE + id, keys); return; }
    const int kvh = hq / (Hq / Hkv);
    kept_keys(P, t, hi[hq], keep[hq], (static_cast<int64_t>(b) * Hkv + kvh) * S, keys);
    // Split the kept keys at key-block boundaries into nsplit runs.
    std::vector<size_t> cut{0};
    const size_t n = keys.size();
    for (int s = 1; s < nsplit; ++s) {
      size_t c = n * s / nsplit;
      while (c > cut.back() && c < n && (keys[c].row / T) == (keys[c - 1].row / T)) ++c;
      cut.push_back(std::max(c, cut.back()));
    }
    cut.push_back(n);
    std::vector<double> ms, ls, os;
    for (size_t s = 0; s + 1 < cut.size(); ++s) {
      if (cut[s + 1] == cut[s]) continue;
      double m, l;
      std::vector<double> o(D);
      partial(P, qr, keys.data() + cut[s], cut[s + 1] - cut[s], &m, &l, o.data());
      ms.push_back(m); ls.push_back(l); os.insert(os.end(), o.begin(), o.end());
    }
    double mstar = -std::numeric_limits<double>::infinity();
    for (double m : ms) mstar = std::max(mstar, m);
    double l = 0.0;
    double* out = O + id * D;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (size_t s = 0; s < ms.size(); ++s) {
      const double w = std::exp(ms[s] - mstar);
      l += w * ls[s];
      for (int d = 0; d < D; ++d) out[d] += w * os[s * D + d];
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
    LSE[id] = mstar + std::log(l);
  });
  return 0;
}

}  // extern "C"
