// Plain CPU oracle for the Dynamic Memory Sparsification (DMS) inference path.
//
// TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
// the benchmark's CPU-baseline leg load this library.  It shares no code, header,
// table or helper with the CUDA path and never calls it.
//
// Everything here is written to be checked by eye against the pages it follows:
//   [DMS-Qwen3] "基于 DMS 的 KV Cache 压缩实战：为 Qwen3-8B 训练驱逐适配器
//               (Model-Optimizer 实验模块)" (mhpq.cn article on Model-Optimizer
//               experimental/dms)
//   [FastDMS]   the FastDMS announcement post (ai-navigate-news.com), its speed
//               table and its "what changes with DMS" subsystem table.
// Floating point is fp64, with two deliberate exceptions that follow from the
// rule "where floating point decides an integer, both sides decide in the same
// precision": the FP8 page scale and the FP8 codes are computed in fp32, which is
// the precision the quantiser on the GPU uses (the pages fix no precision).
//
// Conventions the pages leave open:
//  * A decision logit alpha_t is computed from token t's own hidden state (or
//    key/query neuron) and decides the fate of key t (no shift).
//  * Key j is visible to query i iff j <= i and (i - j < w or alpha_j <= 0).
//  * Evict iff alpha > 0; alpha == 0 keeps.
//  * Page ids: preallocated pages are numbered row-major over (layer, batch,
//    kv-head, page); further pages come from one ascending counter, and the
//    requests of one call are served in (batch, kv-head) row-major order.
//  * FP8 E4M3 (OCP): one fp32 scale per page for K and one for V.  A prefill
//    writes the survivors of each page with scale = max amax(row) / 448.  A
//    decode append raises the scale to amax(new row) / 448 when that is larger,
//    first re-encoding the page's rows from their decoded values.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ----------------------------------------------------------------------------
// FP8 E4M3 (OCP 8-bit floating point specification, E4M3 variant):
// 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; no infinities; the
// only NaN pattern per sign is S.1111.111; largest finite 448 = 1.75 * 2^8;
// subnormals are m * 2^-9 for m in 1..7.  Encoding rounds to nearest, ties to
// even, and saturates finite overflow to +-448 ("satfinite").
// ----------------------------------------------------------------------------
double e4m3_decode(uint8_t c) {
  const int s = (c >> 7) & 1;
  const int e = (c >> 3) & 0xF;
  const int m = c & 0x7;
  double v;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    v = std::ldexp(static_cast<double>(m), -9);  // subnormal: m/8 * 2^(1-7)
  else
    v = std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

// Round half to even of a non-negative double to an integer-valued double.
double rne(double x) {
  double f = std::floor(x);
  double r = x - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (std::fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

uint8_t e4m3_encode(float xf) {
  const double x = static_cast<double>(xf);
  if (std::isnan(x)) return 0x7F;
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(x);
  if (a >= 448.0) return sign | 0x7E;  // saturate (also +-inf)
  // Smallest normal is 2^-6.  Below it the grid is uniform with step 2^-9.
  if (a < std::ldexp(1.0, -6)) {
    double q = rne(a * 512.0);  // in units of 2^-9, 0..8
    if (q >= 8.0) return sign | (1 << 3);  // rounds up to the smallest normal
    return sign | static_cast<uint8_t>(q);
  }
  int e = static_cast<int>(std::floor(std::log2(a)));
  // Guard against log2 rounding at exact powers of two.
  if (std::ldexp(1.0, e) > a) e -= 1;
  if (std::ldexp(1.0, e + 1) <= a) e += 1;
  double mant = a / std::ldexp(1.0, e);   // in [1, 2)
  double q = rne((mant - 1.0) * 8.0);     // 0..8
  if (q >= 8.0) { q = 0.0; e += 1; }
  if (e > 8 || (e == 8 && q > 6.0)) return sign | 0x7E;  // above 448 after rounding
  return sign | static_cast<uint8_t>(((e + 7) << 3) | static_cast<int>(q));
}

struct Cache {
  int L, B, Hkv, D, w, P, max_pos, maxp, cap, pool_pages, pre_pages, fp8;
  int next_page;
  int status;
  std::vector<int> npos;        // [L,B,Hkv] tokens appended so far
  std::vector<int> count;       // [L,B,Hkv] retained slots
  std::vector<int> npages;      // [L,B,Hkv] pages owned
  std::vector<int> page_table;  // [L,B,Hkv,maxp]
  std::vector<int> slot_pos;    // [L,B,Hkv,cap]
  std::vector<int> ring_slot;   // [L,B,Hkv,w]
  std::vector<uint8_t> ring_evict;
  // Page contents.  kval/vval hold the value as stored (fp32/bf16 input values,
  // or the decoded FP8 value).  Codes and scales are kept for FP8 pages.
  std::vector<double> kval, vval;        // [pool_pages, P, D]
  std::vector<float> kraw, vraw;         // unquantised rows staged during a prefill
  std::vector<uint8_t> kcode, vcode;     // [pool_pages, P, D]
  std::vector<float> kscale, vscale;     // [pool_pages]
  int store_values;
  // Which token's decision logit marks token t (see append): 0 its own, +1
  // token t - 1's (carried per head), -1 token t + 1's (set when it arrives).
  int shift;
  std::vector<uint8_t> carry;  // [L,B,Hkv] shift +1: the last token's own decision

  size_t bh(int l, int b, int h) const { return (static_cast<size_t>(l) * B + b) * Hkv + h; }
};

// Status bits: the same meanings as the library's device status word.
constexpr int ST_POOL_EXHAUSTED = 1;
constexpr int ST_CAPACITY = 2;

// Re-encode every row of page `id` up to `rows` with a larger scale.
void fp8_rescale_page(std::vector<uint8_t>& code, std::vector<double>& val, int P, int D,
                      int id, int rows, float s_old, float s_new) {
  for (int r = 0; r < rows; ++r)
    for (int d = 0; d < D; ++d) {
      size_t o = (static_cast<size_t>(id) * P + r) * D + d;
      float v = static_cast<float>(e4m3_decode(code[o])) * s_old;  // fp32 multiply
      uint8_t c = e4m3_encode(v / s_new);                            // fp32 divide
      code[o] = c;
      val[o] = static_cast<double>(static_cast<float>(e4m3_decode(c)) * s_new);
    }
}

// Write one row into a page slot.  For FP8 pages in decode mode the page scale
// may grow first.  In prefill mode FP8 rows are staged unquantised and encoded
// by fp8_encode_prefill_page once the call has replayed every append.
void store_row(Cache& c, int id, int row, int rows_in_page, const float* krow, const float* vrow,
               bool prefill_mode) {
  const size_t base = (static_cast<size_t>(id) * c.P + row) * c.D;
  if (!c.fp8) {
    for (int d = 0; d < c.D; ++d) {
      c.kval[base + d] = krow[d];
      c.vval[base + d] = vrow[d];
    }
    return;
  }
  if (prefill_mode) {
    for (int d = 0; d < c.D; ++d) {
      c.kraw[base + d] = krow[d];
      c.vraw[base + d] = vrow[d];
    }
    return;
  }
  for (int which = 0; which < 2; ++which) {
    const float* x = which ? vrow : krow;
    std::vector<uint8_t>& code = which ? c.vcode : c.kcode;
    std::vector<double>& val = which ? c.vval : c.kval;
    float& scale = which ? c.vscale[id] : c.kscale[id];
    float amax = 0.0f;
    for (int d = 0; d < c.D; ++d) amax = std::max(amax, std::fabs(x[d]));
    float s_new = amax / 448.0f;
    if (s_new > scale) {
      fp8_rescale_page(code, val, c.P, c.D, id, rows_in_page, scale, s_new);
      scale = s_new;
    }
    for (int d = 0; d < c.D; ++d) {
      uint8_t q = scale > 0.0f ? e4m3_encode(x[d] / scale) : 0;
      code[base + d] = q;
      val[base + d] = static_cast<double>(static_cast<float>(e4m3_decode(q)) * scale);
    }
  }
}

// FP8 encoding of page p of head i once a prefill call has staged its rows.
// Rows holding positions >= pos0 were written by this call ("new"); the others
// were written by an earlier call and hold codes at the page's scale ("old").
// For K and for V separately: the scale becomes the larger of the old scale
// (when the page holds old rows) and max amax(new row) / 448; when it grows the
// old rows are first re-encoded from their decoded values, exactly as a decode
// append re-encodes a page; then the new rows are encoded.  In a first prefill
// every row is new and the scale is max amax(row) / 448 over the page.
void fp8_encode_prefill_page(Cache& c, size_t i, int p, int pos0) {
  const int id = c.page_table[i * c.maxp + p];
  const int rows = std::min(c.P, c.count[i] - p * c.P);
  const int* sp = &c.slot_pos[i * c.cap + static_cast<size_t>(p) * c.P];
  bool any_new = false, any_old = false;
  for (int r = 0; r < rows; ++r) (sp[r] >= pos0 ? any_new : any_old) = true;
  if (!any_new) return;
  for (int which = 0; which < 2; ++which) {
    const std::vector<float>& raw = which ? c.vraw : c.kraw;
    std::vector<uint8_t>& code = which ? c.vcode : c.kcode;
    std::vector<double>& val = which ? c.vval : c.kval;
    float& scale = (which ? c.vscale : c.kscale)[id];
    float amax = 0.0f;
    for (int r = 0; r < rows; ++r)
      if (sp[r] >= pos0)
        for (int d = 0; d < c.D; ++d)
          amax = std::max(amax, std::fabs(raw[(static_cast<size_t>(id) * c.P + r) * c.D + d]));
    const float s_old = any_old ? scale : 0.0f;
    const float s = std::max(s_old, amax / 448.0f);
    if (any_old && s > s_old)
      for (int r = 0; r < rows; ++r) {
        if (sp[r] >= pos0) continue;
        for (int d = 0; d < c.D; ++d) {
          const size_t o = (static_cast<size_t>(id) * c.P + r) * c.D + d;
          const float dec = static_cast<float>(e4m3_decode(code[o])) * s_old;  // fp32 multiply
          code[o] = e4m3_encode(dec / s);                                       // fp32 divide
          val[o] = static_cast<double>(static_cast<float>(e4m3_decode(code[o])) * s);
        }
      }
    scale = s;
    for (int r = 0; r < rows; ++r) {
      if (sp[r] < pos0) continue;
      for (int d = 0; d < c.D; ++d) {
        const size_t o = (static_cast<size_t>(id) * c.P + r) * c.D + d;
        const uint8_t q = s > 0.0f ? e4m3_encode(raw[o] / s) : 0;
        code[o] = q;
        val[o] = static_cast<double>(static_cast<float>(e4m3_decode(q)) * s);
      }
    }
  }
}

// The append rule of the paged DMS cache ([DMS-Qwen3], inference mode, paged KV
// cache): when token t arrives and the token leaving the sliding window
// (t - w) was marked for eviction, t takes that token's slot in place;
// otherwise t takes the next free slot, and the block table grows by one page
// whenever that slot starts a page.  Returns false if the append was dropped
// (pool exhausted or capacity exceeded; the status word records which).
//
// `decision` is token t's own decision (its logit > 0).  Which token it marks
// follows the cache's shift ([DMS-Qwen3], attention: the training path shifts
// the decision logits by one position):
//   0   token t is marked by its own decision;
//   +1  token t is marked by token t - 1's decision (the logits shifted right
//       by one; token 0 takes the padding, "keep");
//   -1  token t's decision marks token t - 1 (set now, in t - 1's ring entry);
//       token t stays unmarked until token t + 1 arrives.
bool append(Cache& c, int l, int b, int h, bool decision, const float* krow, const float* vrow,
            bool prefill_mode) {
  const size_t i = c.bh(l, b, h);
  const int t = c.npos[i];
  int* ring_slot = &c.ring_slot[i * c.w];
  uint8_t* ring_evict = &c.ring_evict[i * c.w];
  bool evict = decision;
  if (c.shift == 1) {
    evict = c.carry[i] != 0;
    c.carry[i] = decision ? 1 : 0;
  } else if (c.shift == -1) {
    evict = false;
    if (t >= 1) ring_evict[(t - 1) % c.w] = decision ? 1 : 0;
  }
  int slot;
  if (t >= c.w && ring_evict[t % c.w]) {
    slot = ring_slot[t % c.w];  // overwrite the evicted token in place
  } else {
    slot = c.count[i];
    if (slot >= c.cap) {
      c.status |= ST_CAPACITY;
      return false;
    }
    if (slot % c.P == 0 && slot / c.P >= c.npages[i]) {
      if (c.next_page >= c.pool_pages) {
        c.status |= ST_POOL_EXHAUSTED;
        return false;
      }
      c.page_table[i * c.maxp + c.npages[i]] = c.next_page++;
      c.npages[i] += 1;
    }
    c.count[i] += 1;
  }
  c.slot_pos[i * c.cap + slot] = t;
  ring_slot[t % c.w] = slot;
  ring_evict[t % c.w] = evict ? 1 : 0;
  c.npos[i] = t + 1;
  if (c.store_values && krow != nullptr) {
    const int p = slot / c.P;
    const int id = c.page_table[i * c.maxp + p];
    const int rows = std::min(c.P, c.count[i] - p * c.P);
    store_row(c, id, slot % c.P, rows, krow, vrow, prefill_mode);
  }
  return true;
}

inline double softmax_attend(const double* q, int D, const std::vector<const double*>& keys,
                             const std::vector<const double*>& vals, double* out) {
  // Dense softmax over the given keys with scale 1/sqrt(D), in fp64.
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
  std::vector<double> s(keys.size());
  double m = -INFINITY;
  for (size_t j = 0; j < keys.size(); ++j) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += q[d] * keys[j][d];
    s[j] = acc * scale;
    m = std::max(m, s[j]);
  }
  double l = 0.0;
  for (size_t j = 0; j < keys.size(); ++j) {
    s[j] = std::exp(s[j] - m);
    l += s[j];
  }
  for (int d = 0; d < D; ++d) out[d] = 0.0;
  for (size_t j = 0; j < keys.size(); ++j)
    for (int d = 0; d < D; ++d) out[d] += s[j] * vals[j][d];
  for (int d = 0; d < D; ++d) out[d] /= l;
  return l;
}

}  // namespace

extern "C" {

int oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

void oracle_e4m3_encode_n(const float* x, uint8_t* out, long n) {
  for (long i = 0; i < n; ++i) out[i] = e4m3_encode(x[i]);
}
void oracle_e4m3_decode_n(const uint8_t* c, double* out, long n) {
  for (long i = 0; i < n; ++i) out[i] = e4m3_decode(c[i]);
}

// Decision logits from the separate adapter ([DMS-Qwen3], "two sources and two
// granularities of the eviction decision", source two): an RMSNorm over the
// pre-attention hidden state, a Linear(hidden -> num_kv_heads), times the alpha
// scale, minus the alpha offset.  The output is laid out (batch, kv-head, token).
//   h      [B,T,hidden]     gamma [hidden]     W [Hkv,hidden]   bias [Hkv] or null
//   offset [B,Hkv] (one offset per head and sequence)
// With layer granularity every head takes head 0's logit.
void oracle_decide_proj(int B, int T, int hidden, int Hkv, const double* h, const double* gamma,
                        const double* W, const double* bias, const double* offset, double scale,
                        double eps, int layer_mode, double* alpha) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      const double* x = h + (static_cast<size_t>(b) * T + t) * hidden;
      double ms = 0.0;
      for (int i = 0; i < hidden; ++i) ms += x[i] * x[i];
      ms /= hidden;
      const double inv = 1.0 / std::sqrt(ms + eps);
      for (int hd = 0; hd < Hkv; ++hd) {
        double z = bias ? bias[hd] : 0.0;
        for (int i = 0; i < hidden; ++i) z += W[static_cast<size_t>(hd) * hidden + i] * (x[i] * inv * gamma[i]);
        alpha[(static_cast<size_t>(b) * Hkv + hd) * T + t] = z * scale - offset[b * Hkv + hd];
      }
      if (layer_mode)
        for (int hd = 1; hd < Hkv; ++hd)
          alpha[(static_cast<size_t>(b) * Hkv + hd) * T + t] = alpha[(static_cast<size_t>(b) * Hkv) * T + t];
    }
}

// Decision logits from an importance score (the KVzap-linear page, workflow:
// a Linear from the layer's hidden state to one score per KV head; tokens
// scoring below the threshold are pruned while the most recent ones are
// kept): score = W_h . x_t + bias_h, alpha = threshold_h - score, so a token
// is marked iff its score is below the threshold.  No normalisation.
//   h [B,T,hidden]  W [Hkv,hidden]  bias [Hkv] or null  threshold [B,Hkv]
// With layer granularity every head takes head 0's logit.
void oracle_decide_score(int B, int T, int hidden, int Hkv, const double* h, const double* W,
                         const double* bias, const double* threshold, int layer_mode, double* alpha) {
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      const double* x = h + (static_cast<size_t>(b) * T + t) * hidden;
      for (int hd = 0; hd < Hkv; ++hd) {
        const int src = layer_mode ? 0 : hd;
        double score = bias ? bias[src] : 0.0;
        for (int i = 0; i < hidden; ++i) score += W[static_cast<size_t>(src) * hidden + i] * x[i];
        alpha[(static_cast<size_t>(b) * Hkv + hd) * T + t] = threshold[b * Hkv + src] - score;
      }
    }
}

// Decision logits from a single neuron ([DMS-Qwen3], source one): the last
// element of a key (group = 1) or of the first query head of each GQA group
// (group = Hq/Hkv), times the scale, minus the offset; that element is then set
// to zero so the rotary embedding does not mix it.  x is [B,T,Hsrc,D] and is
// modified in place.  With layer granularity every head takes head 0's logit,
// and every head's decision neuron is still zeroed.
void oracle_decide_neuron(int B, int T, int Hsrc, int D, int group, int Hkv, double* x,
                          const double* offset, double scale, int layer_mode, double* alpha) {
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t) {
      for (int hd = 0; hd < Hkv; ++hd) {
        double* e = x + ((static_cast<size_t>(b) * T + t) * Hsrc + hd * group) * D + (D - 1);
        alpha[(static_cast<size_t>(b) * Hkv + hd) * T + t] = *e * scale - offset[b * Hkv + hd];
        *e = 0.0;
      }
      if (layer_mode)
        for (int hd = 1; hd < Hkv; ++hd)
          alpha[(static_cast<size_t>(b) * Hkv + hd) * T + t] = alpha[(static_cast<size_t>(b) * Hkv) * T + t];
    }
}

// Rotary embedding, half-split form: for i < D/2 the pair (x_i, x_{i+D/2}) is
// rotated by the angle of (position, i), with cos/sin read from caller tables
// [max_pos, D/2]:  x_i' = x_i c - x_{i+D/2} s,  x_{i+D/2}' = x_{i+D/2} c + x_i s.
// x is [B,T,H,D] (fp64, modified in place); token t sits at position pos0 + t.
// Plain fp64; the caller rounds the result once into the activation dtype when
// it is stored (oracle_round_bf16_n for bf16).
void oracle_rope(int B, int T, int H, int D, double* x, int pos0, const double* cos_t,
                 const double* sin_t) {
  const int half = D / 2;
  for (int b = 0; b < B; ++b)
    for (int t = 0; t < T; ++t)
      for (int hh = 0; hh < H; ++hh) {
        double* e = x + ((static_cast<size_t>(b) * T + t) * H + hh) * D;
        const double* c = cos_t + static_cast<size_t>(pos0 + t) * half;
        const double* s = sin_t + static_cast<size_t>(pos0 + t) * half;
        for (int i = 0; i < half; ++i) {
          const double a = e[i], bb = e[i + half];
          e[i] = a * c[i] - bb * s[i];
          e[i + half] = bb * c[i] + a * s[i];
        }
      }
}

// Round fp64 values to bfloat16 (1 sign bit, 8 exponent bits with bias 127, 7
// stored mantissa bits: 8 significant bits for normal numbers, a fixed quantum
// of 2^-133 below the smallest normal 2^-126), to nearest with ties to even, in
// one step.  Results are returned as the fp32 numbers they denote; values that
// round past the largest finite bf16 (0x7F7F) become infinities.
void oracle_round_bf16_n(const double* x, float* out, long n) {
  const double max_bf16 = std::ldexp(255.0, 120);  // 1.9921875 * 2^127
  for (long idx = 0; idx < n; ++idx) {
    const double v = x[idx];
    if (std::isnan(v) || std::isinf(v) || v == 0.0) {
      out[idx] = static_cast<float>(v);
      continue;
    }
    int e;
    std::frexp(std::fabs(v), &e);  // |v| in [2^(e-1), 2^e)
    const int q = std::max(e - 8, -133);  // exponent of the quantum
    double r = std::ldexp(rne(std::ldexp(std::fabs(v), -q)), q);
    if (r > max_bf16) r = INFINITY;
    out[idx] = static_cast<float>(std::signbit(v) ? -r : r);
  }
}

// DMS-masked prefill attention ([DMS-Qwen3], attention: the sliding window plus
// eviction gate of the training score_mod, taken to its hard inference limit):
// query i of head hq sees key j of KV head hq / (Hq/Hkv) iff
//   j <= i  and  (i - j < w  or  evict[j] == 0),
// and the output row is the fp64 softmax (scale 1/sqrt(D)) over those keys.
//   q [B,T,Hq,D], k/v [B,T,Hkv,D], evict [B,Hkv,T] (0/1), o [B,T,Hq,D]
// rows: optional list of (b, hq, i) triples; if null every row is computed.
void oracle_prefill_attention(int B, int T, int Hq, int Hkv, int D, int w, const double* q,
                              const double* k, const double* v, const uint8_t* evict,
                              const int* rows, long n_rows, double* o) {
  const int g = Hq / Hkv;
  const long total = rows ? n_rows : static_cast<long>(B) * Hq * T;
#pragma omp parallel for schedule(dynamic, 16)
  for (long r = 0; r < total; ++r) {
    int b, hq, i;
    if (rows) {
      b = rows[3 * r];
      hq = rows[3 * r + 1];
      i = rows[3 * r + 2];
    } else {
      b = static_cast<int>(r / (static_cast<long>(Hq) * T));
      hq = static_cast<int>((r / T) % Hq);
      i = static_cast<int>(r % T);
    }
    const int h = hq / g;
    std::vector<const double*> keys, vals;
    for (int j = 0; j <= i; ++j) {
      bool visible = (i - j < w) || evict[(static_cast<size_t>(b) * Hkv + h) * T + j] == 0;
      if (!visible) continue;
      keys.push_back(k + ((static_cast<size_t>(b) * T + j) * Hkv + h) * D);
      vals.push_back(v + ((static_cast<size_t>(b) * T + j) * Hkv + h) * D);
    }
    const double* qq = q + ((static_cast<size_t>(b) * T + i) * Hq + hq) * D;
    double* out = rows ? o + static_cast<size_t>(r) * D : o + ((static_cast<size_t>(b) * T + i) * Hq + hq) * D;
    softmax_attend(qq, D, keys, vals, out);
  }
}

// ---------------------------------------------------------------------------
// Training mode ([DMS-Qwen3], "Gumbel 噪声与可微门控" and "注意力实现": the
// soft-gated attention of the training path, forward only)
// ---------------------------------------------------------------------------
// Gate of each token: gate logit l = (alpha + noise) / tau, probability
// p = sigmoid(l), forward value of the straight-through decision
// (p > 0.5) - p + p, which is exactly 1 or 0 (here: p > 0.5); and the eviction
// penalty of each key from the logits shifted right by one position:
// penalty[k] = logsigmoid(-l[k-1]) = log(1 - p[k-1]) for k >= 1, penalty[0] = 0
// (the padding position is never penalised).  All [B,Hkv,T]; noise may be
// null (zero).
void oracle_train_gate(int B, int Hkv, int T, const double* alpha, const double* noise, double tau,
                       double* prob, double* hard, double* penalty) {
  for (long r = 0; r < static_cast<long>(B) * Hkv; ++r) {
    const double* a = alpha + r * T;
    const double* g = noise ? noise + r * T : nullptr;
    for (int t = 0; t < T; ++t) {
      const double l = (a[t] + (g ? g[t] : 0.0)) / tau;
      const double p = 1.0 / (1.0 + std::exp(-l));
      prob[r * T + t] = p;
      hard[r * T + t] = p > 0.5 ? 1.0 : 0.0;
      // logsigmoid(-l) = -log(1 + exp(l)), in a form that does not overflow
      const double ls = l > 0 ? -(l + std::log1p(std::exp(-l))) : -std::log1p(std::exp(l));
      if (t + 1 < T) penalty[r * T + t + 1] = ls;
    }
    penalty[r * T] = 0.0;
  }
}

// The soft-gated attention of the training path: query i and key j of KV head
// hq / (Hq/Hkv) score s = q.k / sqrt(D); a key inside the window (i - j < w)
// keeps s, a key outside it gets s + penalty[j]; a causal violation (j > i)
// gets the mask value -50000, whose weight exp(-50000 - max) is zero in fp64,
// so those keys are left out; o = softmax(scores) v.  Dense over every key.
//   q [B,T,Hq,D], k/v [B,T,Hkv,D], penalty [B,Hkv,T]; rows as in
//   oracle_prefill_attention.
void oracle_train_attention(int B, int T, int Hq, int Hkv, int D, int w, const double* q, const double* k,
                            const double* v, const double* penalty, const int* rows, long n_rows, double* o) {
  const int g = Hq / Hkv;
  const long total = rows ? n_rows : static_cast<long>(B) * Hq * T;
  const double scale = 1.0 / std::sqrt(static_cast<double>(D));
#pragma omp parallel for schedule(dynamic, 16)
  for (long r = 0; r < total; ++r) {
    int b, hq, i;
    if (rows) {
      b = rows[3 * r];
      hq = rows[3 * r + 1];
      i = rows[3 * r + 2];
    } else {
      b = static_cast<int>(r / (static_cast<long>(Hq) * T));
      hq = static_cast<int>((r / T) % Hq);
      i = static_cast<int>(r % T);
    }
    const int h = hq / g;
    const double* qq = q + ((static_cast<size_t>(b) * T + i) * Hq + hq) * D;
    std::vector<double> s(i + 1);
    double m = -INFINITY;
    for (int j = 0; j <= i; ++j) {
      const double* kk = k + ((static_cast<size_t>(b) * T + j) * Hkv + h) * D;
      double acc = 0.0;
      for (int d = 0; d < D; ++d) acc += qq[d] * kk[d];
      s[j] = acc * scale + (i - j < w ? 0.0 : penalty[(static_cast<size_t>(b) * Hkv + h) * T + j]);
      m = std::max(m, s[j]);
    }
    double l = 0.0;
    for (int j = 0; j <= i; ++j) {
      s[j] = std::exp(s[j] - m);
      l += s[j];
    }
    double* out = rows ? o + static_cast<size_t>(r) * D : o + ((static_cast<size_t>(b) * T + i) * Hq + hq) * D;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int j = 0; j <= i; ++j) {
      const double* vv = v + ((static_cast<size_t>(b) * T + j) * Hkv + h) * D;
      for (int d = 0; d < D; ++d) out[d] += s[j] * vv[d];
    }
    for (int d = 0; d < D; ++d) out[d] /= l;
  }
}

// ---------------------------------------------------------------------------
// Paged cache simulation
// ---------------------------------------------------------------------------
void* oracle_cache_new(int L, int B, int Hkv, int D, int w, int P, int max_pos, int pool_pages,
                       int prealloc_tokens, int fp8, int store_values, int shift) {
  Cache* c = new Cache();
  c->shift = shift;
  c->carry.assign(static_cast<size_t>(L) * B * Hkv, 0);
  c->L = L; c->B = B; c->Hkv = Hkv; c->D = D; c->w = w; c->P = P;
  c->max_pos = max_pos;
  c->maxp = (max_pos + P - 1) / P;
  c->cap = c->maxp * P;
  c->pool_pages = pool_pages;
  c->pre_pages = std::min(c->maxp, (prealloc_tokens + P - 1) / P);
  c->fp8 = fp8;
  c->store_values = store_values;
  c->status = 0;
  const size_t nbh = static_cast<size_t>(L) * B * Hkv;
  c->npos.assign(nbh, 0);
  c->count.assign(nbh, 0);
  c->npages.assign(nbh, 0);
  c->page_table.assign(nbh * c->maxp, -1);
  c->slot_pos.assign(nbh * c->cap, -1);
  c->ring_slot.assign(nbh * w, -1);
  c->ring_evict.assign(nbh * w, 0);
  // Preallocation ([DMS-Qwen3], advanced options, cache preallocation): each
  // (layer, batch, head) starts with enough pages for prealloc_tokens, numbered
  // row-major; if the pool cannot hold them all the status word says so.
  int id = 0;
  for (size_t i = 0; i < nbh; ++i)
    for (int p = 0; p < c->pre_pages; ++p) {
      if (id >= pool_pages) {
        c->status |= ST_POOL_EXHAUSTED;
        break;
      }
      c->page_table[i * c->maxp + p] = id++;
      c->npages[i] += 1;
    }
  c->next_page = id;
  if (store_values) {
    const size_t n = static_cast<size_t>(pool_pages) * P * D;
    c->kval.assign(n, 0.0);
    c->vval.assign(n, 0.0);
    if (fp8) {
      c->kraw.assign(n, 0.0f);
      c->vraw.assign(n, 0.0f);
      c->kcode.assign(n, 0);
      c->vcode.assign(n, 0);
      c->kscale.assign(pool_pages, 0.0f);
      c->vscale.assign(pool_pages, 0.0f);
    }
  }
  return c;
}

void oracle_cache_delete(void* h) { delete static_cast<Cache*>(h); }
// An independent copy of the whole simulated cache (state and pages).
void* oracle_cache_clone(void* h) { return new Cache(*static_cast<const Cache*>(h)); }

int oracle_cache_status(void* h) { return static_cast<Cache*>(h)->status; }

// Prefill of layer l: replay the append rule token by token, for each (b, h) in
// row-major order, continuing from the tokens the layer already holds (a
// later chunk of a chunked prefill).  evict [B,Hkv,T] (0/1); k/v [B,T,Hkv,D] fp32 values or null
// (index-only replay).  FP8 pages the call wrote rows into are encoded at the
// end (fp8_encode_prefill_page).
void oracle_cache_prefill(void* hc, int l, int T, const uint8_t* evict, const float* k,
                          const float* v) {
  Cache& c = *static_cast<Cache*>(hc);
  for (int b = 0; b < c.B; ++b)
    for (int h = 0; h < c.Hkv; ++h) {
      const int pos0 = c.npos[c.bh(l, b, h)];  // tokens held before this call
      for (int t = 0; t < T; ++t) {
        const float* kr = k ? k + ((static_cast<size_t>(b) * T + t) * c.Hkv + h) * c.D : nullptr;
        const float* vr = v ? v + ((static_cast<size_t>(b) * T + t) * c.Hkv + h) * c.D : nullptr;
        append(c, l, b, h, evict[(static_cast<size_t>(b) * c.Hkv + h) * T + t] != 0, kr, vr, true);
      }
      if (c.fp8 && c.store_values && k) {
        const size_t i = c.bh(l, b, h);
        for (int p = 0; p * c.P < c.count[i]; ++p) fp8_encode_prefill_page(c, i, p, pos0);
      }
    }
}

// One decode append for layer l: one token per (b, h), in row-major order.
// evict [B,Hkv]; k/v [B,Hkv,D] or null.
void oracle_cache_append(void* hc, int l, const uint8_t* evict, const float* k, const float* v) {
  Cache& c = *static_cast<Cache*>(hc);
  for (int b = 0; b < c.B; ++b)
    for (int h = 0; h < c.Hkv; ++h) {
      const size_t r = (static_cast<size_t>(b) * c.Hkv + h);
      append(c, l, b, h, evict[r] != 0, k ? k + r * c.D : nullptr, v ? v + r * c.D : nullptr, false);
    }
}

// Copy out the index state of layer l (each array as laid out in the cache).
void oracle_cache_export(void* hc, int l, int* npos, int* count, int* npages, int* page_table,
                         int* slot_pos, int* ring_slot, uint8_t* ring_evict, int* next_page) {
  Cache& c = *static_cast<Cache*>(hc);
  const size_t nb = static_cast<size_t>(c.B) * c.Hkv;
  const size_t o = static_cast<size_t>(l) * nb;
  std::copy(c.npos.begin() + o, c.npos.begin() + o + nb, npos);
  std::copy(c.count.begin() + o, c.count.begin() + o + nb, count);
  std::copy(c.npages.begin() + o, c.npages.begin() + o + nb, npages);
  std::copy(c.page_table.begin() + o * c.maxp, c.page_table.begin() + (o + nb) * c.maxp, page_table);
  std::copy(c.slot_pos.begin() + o * c.cap, c.slot_pos.begin() + (o + nb) * c.cap, slot_pos);
  std::copy(c.ring_slot.begin() + o * c.w, c.ring_slot.begin() + (o + nb) * c.w, ring_slot);
  std::copy(c.ring_evict.begin() + o * c.w, c.ring_evict.begin() + (o + nb) * c.w, ring_evict);
  *next_page = c.next_page;
}

// Copy out page contents: stored values (decoded for FP8), codes and scales.
void oracle_cache_pages(void* hc, double* kval, double* vval, uint8_t* kcode, uint8_t* vcode,
                        float* kscale, float* vscale) {
  Cache& c = *static_cast<Cache*>(hc);
  if (!c.store_values) return;
  std::copy(c.kval.begin(), c.kval.end(), kval);
  std::copy(c.vval.begin(), c.vval.end(), vval);
  if (c.fp8) {
    std::copy(c.kcode.begin(), c.kcode.end(), kcode);
    std::copy(c.vcode.begin(), c.vcode.end(), vcode);
    std::copy(c.kscale.begin(), c.kscale.end(), kscale);
    std::copy(c.vscale.begin(), c.vscale.end(), vscale);
  }
}

// Decode attention of layer l over each head's retained slots [0, count):
// the query heads of one GQA group share their KV head's pages
// ([FastDMS], attention scoring: grouped compact decode attention over
// variable-length per-head live spans).  q [B,Hq,D] -> o [B,Hq,D].
void oracle_cache_decode_attention(void* hc, int l, int Hq, const double* q, double* o) {
  Cache& c = *static_cast<Cache*>(hc);
  const int g = Hq / c.Hkv;
#pragma omp parallel for collapse(2) schedule(static)
  for (int b = 0; b < c.B; ++b)
    for (int hq = 0; hq < Hq; ++hq) {
      const int h = hq / g;
      const size_t i = c.bh(l, b, h);
      std::vector<const double*> keys, vals;
      for (int s = 0; s < c.count[i]; ++s) {
        const int id = c.page_table[i * c.maxp + s / c.P];
        const size_t off = (static_cast<size_t>(id) * c.P + s % c.P) * c.D;
        keys.push_back(&c.kval[off]);
        vals.push_back(&c.vval[off]);
      }
      softmax_attend(q + (static_cast<size_t>(b) * Hq + hq) * c.D, c.D, keys, vals,
                     o + (static_cast<size_t>(b) * Hq + hq) * c.D);
    }
}


// Attention of the T rows of a prefill call into layer l, computed with the
// cache as it is before the call's appends ([DMS-Qwen3], chunked prefill: a
// chunk's queries attend to the cache plus the chunk itself).  Row i of the
// call sits at position pos0 + i (pos0 = tokens the layer already holds) and
// sees, under the DMS mask (key j visible iff j <= i and (i - j < w or j was
// kept)):
//   * every key the cache holds: a slot at position j older than the last w
//     positions is a kept token (a marked one would have been overwritten), a
//     younger one is kept or marked as its ring entry says; values as stored
//     (decoded for FP8 pages);
//   * the call's own keys j <= i, from its inputs.
// q [B,T,Hq,D], k/v [B,T,Hkv,D], evict [B,Hkv,T] (the call's tokens' own
// decisions; which token each marks follows the cache's shift, as in append);
// rows: optional (b, hq, i) triples (i a row of this call), else every row.
// With an empty layer and no shift this is oracle_prefill_attention.
void oracle_cache_prefill_attention(void* hc, int l, int T, int Hq, const double* q, const double* k,
                                    const double* v, const uint8_t* evict, const int* rows, long n_rows,
                                    double* o) {
  Cache& c = *static_cast<Cache*>(hc);
  const int g = Hq / c.Hkv, w = c.w, D = c.D;
  const long total = rows ? n_rows : static_cast<long>(c.B) * Hq * T;
#pragma omp parallel for schedule(dynamic, 16)
  for (long r = 0; r < total; ++r) {
    int b, hq, i;
    if (rows) {
      b = rows[3 * r];
      hq = rows[3 * r + 1];
      i = rows[3 * r + 2];
    } else {
      b = static_cast<int>(r / (static_cast<long>(Hq) * T));
      hq = static_cast<int>((r / T) % Hq);
      i = static_cast<int>(r % T);
    }
    const int h = hq / g;
    const size_t bh = c.bh(l, b, h);
    const int pos0 = c.npos[bh], qi = pos0 + i;
    const uint8_t* ev = evict + (static_cast<size_t>(b) * c.Hkv + h) * T;  // the call's own decisions
    // the mark of the call's token jj under the cache's shift
    auto call_mark = [&](int jj) -> bool {
      if (c.shift == 1) return jj == 0 ? c.carry[bh] != 0 : ev[jj - 1] != 0;
      if (c.shift == -1) return jj + 1 < T ? ev[jj + 1] != 0 : false;
      return ev[jj] != 0;
    };
    std::vector<const double*> keys, vals;
    for (int s = 0; s < c.count[bh]; ++s) {
      const int j = c.slot_pos[bh * c.cap + s];
      // the layer's last token is marked by this call's first decision when
      // a token's decision marks the one before it
      const bool mark = (c.shift == -1 && j == pos0 - 1) ? ev[0] != 0 : c.ring_evict[bh * w + j % w] != 0;
      const bool marked = j >= pos0 - w && mark;
      if (marked && qi - j >= w) continue;
      const int id = c.page_table[bh * c.maxp + s / c.P];
      const size_t off = (static_cast<size_t>(id) * c.P + s % c.P) * D;
      keys.push_back(&c.kval[off]);
      vals.push_back(&c.vval[off]);
    }
    for (int jj = 0; jj <= i; ++jj) {
      const bool visible = (i - jj < w) || !call_mark(jj);
      if (!visible) continue;
      keys.push_back(k + ((static_cast<size_t>(b) * T + jj) * c.Hkv + h) * D);
      vals.push_back(v + ((static_cast<size_t>(b) * T + jj) * c.Hkv + h) * D);
    }
    const double* qq = q + ((static_cast<size_t>(b) * T + i) * Hq + hq) * D;
    double* out = rows ? o + static_cast<size_t>(r) * D : o + ((static_cast<size_t>(b) * T + i) * Hq + hq) * D;
    softmax_attend(qq, D, keys, vals, out);
  }
}

}  // extern "C"
