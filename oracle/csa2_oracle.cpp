// CSA2 CPU oracle -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, deliberately unoptimised C++17 statement of what the CSA2
// sparse-attention step computes.  Only the tests, the smoke check and the
// bench's CPU-baseline / reference leg may load this library; the CUDA library
// never does, and the two share no code (no headers, tables or helpers).
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC.
//
// Sources (page titles of the pages studied; sections named per function):
//  [V41]  "DeepSeek-V4.1-Flash: Pushing the Limits of KV Cache Compression"
//         (fupanwang summary): sections "三个方向一起压小缓存" (CSA2 modes,
//         hierarchical indexer, pool of <=2048 blocks x 8, Top-512, MXFP4 main
//         KV, FP4 indexer q/k, FP8 sliding window) and "后 20 层干脆共用一份 KV"
//         (128-token window, compression ratio 2 / 1, compression weights).
//  [NOTES] "DeepSeek-V4.1" reading notes (dreamax): Full/Reindex/Reuse modes,
//         the SWA branch and the three-set distinction.
//  [OCP]  OCP Microscaling Formats (MX) v1.0: E2M1, E8M0, MXFP4 block of 32.
//
// The pages give no formula for the indexer score, the compression weights or
// the attention scale; the readings used here are the plainest ones, and each
// function states the reading it takes.  Every function below is pinned by
// tests under tests/ (no function is "parity unpinned").
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------------------
// Formats  [OCP] + [V41] "MXFP4 (OCP)", "FP8 window"
// ---------------------------------------------------------------------------

// E2M1 magnitudes: exponent bias 1, one mantissa bit, no inf/NaN.
const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double e2m1_value(int code) {
  double m = kE2M1[code & 7];
  return (code & 8) ? -m : m;
}

// Twice the E2M1 value: an integer in {0, +-1, +-2, +-3, +-4, +-6, +-8, +-12}.
int e2m1_twice(int code) {
  static const int t[8] = {0, 1, 2, 3, 4, 6, 8, 12};
  return (code & 8) ? -t[code & 7] : t[code & 7];
}

double e8m0_value(int byte) { return std::ldexp(1.0, byte - 127); }

// OCP FP8 E4M3 ("FN"): bias 7, subnormals, S.1111.111 is NaN, max 448.
double e4m3_value(int byte) {
  int s = (byte >> 7) & 1, e = (byte >> 3) & 15, m = byte & 7;
  if (e == 15 && m == 7) return std::nan("");
  double v = (e == 0) ? std::ldexp(m / 8.0, -6) : std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

int code_at(const uint8_t* row_codes, int e) {
  uint8_t b = row_codes[e / 2];
  return (e & 1) ? (b >> 4) : (b & 15);
}

float bf16_to_float(uint16_t b) {
  uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Nearest E2M1 magnitude index for a >= 0, ties to the even index (even
// mantissa), saturating at 6.
int e2m1_round_mag(double a) {
  if (a >= 6.0) return 7;
  int i = 0;
  while (!(a < kE2M1[i + 1])) ++i;  // kE2M1[i] <= a < kE2M1[i+1]
  double dlo = a - kE2M1[i], dhi = kE2M1[i + 1] - a;
  if (dlo < dhi) return i;
  if (dhi < dlo) return i + 1;
  return (i % 2 == 0) ? i : i + 1;
}

// One 32-element MXFP4 block [OCP]: X = floor(log2(amax)) - emax(E2M1)=2,
// clamped to [-127, 127]; E8M0 byte = X + 127; elements x * 2^-X rounded to
// E2M1 (nearest, ties to even, saturating); the sign bit is always the sign
// of x.  amax == 0 gives byte 0 and zero magnitudes.
void mxfp4_encode_block(const float* x, uint8_t* codes16, uint8_t* scale) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) amax = std::max(amax, std::fabs(x[i]));
  int X = -127;
  if (amax > 0.0f) {
    int e;
    std::frexp(amax, &e);  // amax = f * 2^e, f in [0.5, 1)  => floor(log2 amax) = e - 1
    X = std::min(127, std::max(-127, (e - 1) - 2));
  }
  *scale = uint8_t(X + 127);
  for (int i = 0; i < 32; i += 2) {
    int c[2];
    for (int j = 0; j < 2; ++j) {
      double v = std::ldexp(double(x[i + j]), -X);
      int mag = e2m1_round_mag(std::fabs(v));
      c[j] = mag | (std::signbit(x[i + j]) ? 8 : 0);
    }
    codes16[i / 2] = uint8_t(c[0] | (c[1] << 4));
  }
}

void mxfp4_encode_row(const float* x, int n, uint8_t* codes, uint8_t* scales) {
  for (int b = 0; b < n / 32; ++b) mxfp4_encode_block(x + 32 * b, codes + 16 * b, scales + b);
}

void mxfp4_decode_row(const uint8_t* codes, const uint8_t* scales, int n, double* out) {
  for (int e = 0; e < n; ++e) out[e] = e2m1_value(code_at(codes, e)) * e8m0_value(scales[e / 32]);
}

// ---------------------------------------------------------------------------
// Own exp for the compression weights (Cody & Waite argument reduction by
// ln 2 with a two-part constant, then the Taylor series of e^r to degree 14 by
// Horner's rule).  Both sides of the parity check must take the same steps, so
// this is written out instead of calling the C library.  ln2 split: hi is ln 2
// rounded to 24 significant bits, lo = ln 2 - hi rounded to double.
// ---------------------------------------------------------------------------
const double kLn2Hi = 0.6931471824645996;         // 11629080 * 2^-24
const double kLn2Lo = -1.904654299957768e-09;     // ln2 - kLn2Hi
const double kInvLn2 = 1.4426950408889634;        // 1 / ln 2

double own_exp(double x) {
  if (x < -745.0) return 0.0;
  if (x > 709.0) return INFINITY;
  double k = std::nearbyint(x * kInvLn2);           // round half to even
  double r = (x - k * kLn2Hi) - k * kLn2Lo;         // |r| <= ~0.3466
  double p = 1.0 / 87178291200.0;                   // 1/14!
  const double inv_fact[14] = {1.0,
                               1.0,
                               1.0 / 2.0,
                               1.0 / 6.0,
                               1.0 / 24.0,
                               1.0 / 120.0,
                               1.0 / 720.0,
                               1.0 / 5040.0,
                               1.0 / 40320.0,
                               1.0 / 362880.0,
                               1.0 / 3628800.0,
                               1.0 / 39916800.0,
                               1.0 / 479001600.0,
                               1.0 / 6227020800.0};
  for (int i = 13; i >= 0; --i) p = std::fma(p, r, inv_fact[i]);
  return std::ldexp(p, int(k));
}

// ---------------------------------------------------------------------------
// Indexer score  [V41] "FP4 indexer q/k"; the pages give no formula; the plainest reading is
//   s_t = sum_h w_h * (q_h . k_t)   (no ReLU), one 128-d key per position
// shared by the 4 indexer heads.  Exactness: per head h and 32-block b the
// doubled-E2M1 integer dot D (|D| <= 4608) times 2^(eq+ek-2) is exact; the
// four block terms are summed in fp64 in order b = 0..3 and rounded once to
// fp32 (d_h).  That sum is the exact block sum whenever the block exponents
// of a head lie within 38 of each other (four 13-bit integers fit fp64's
// 53-bit significand); beyond that the ordered fp64 sum itself is the
// definition (both sides add in this order).  The head
// combination is s = w0*d0, then fmaf(w_h, d_h, s) for h = 1..3, in fp32.
// -0 becomes +0.
// ---------------------------------------------------------------------------
float index_score(const uint8_t* kc, const uint8_t* ks, const uint8_t* qc, const uint8_t* qs,
                  const float* w) {
  float d[4];
  for (int h = 0; h < 4; ++h) {
    double acc = 0.0;
    for (int b = 0; b < 4; ++b) {
      int64_t D = 0;
      for (int i = 0; i < 32; ++i) {
        int e = 32 * b + i;
        D += int64_t(e2m1_twice(code_at(qc + 64 * h, e))) * e2m1_twice(code_at(kc, e));
      }
      int ex = (int(qs[4 * h + b]) - 127) + (int(ks[b]) - 127) - 2;
      double term = double(D) * std::ldexp(1.0, ex);
      acc = acc + term;
    }
    d[h] = float(acc);
  }
  float s = w[0] * d[0];
  for (int h = 1; h < 4; ++h) s = std::fma(w[h], d[h], s);
  if (s == 0.0f) s = 0.0f;
  return s;
}

// Order-preserving map of a score to uint32 (larger score -> larger key).
// The pages rank by score alone; a NaN score (a head sum of +inf and -inf,
// or 0 * inf) has no place in that order.  Reading: every NaN ranks below
// every number, -inf included, and NaNs tie among themselves (so the lower
// position wins): all NaNs map to key 1 (-inf maps to 0x007FFFFF; 0 stays
// free to mean "absent" elsewhere).
uint32_t rank_key(float s) {
  if (std::isnan(s)) return 1u;
  if (s == 0.0f) s = 0.0f;
  uint32_t u;
  std::memcpy(&u, &s, 4);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k by (key descending, id ascending); result ascending by id, padded -1.
void topk_select(const std::vector<uint32_t>& keys, const std::vector<int64_t>& ids, int k,
                 int32_t* out) {
  std::vector<size_t> ord(keys.size());
  for (size_t i = 0; i < ord.size(); ++i) ord[i] = i;
  size_t m = std::min<size_t>(size_t(k), ord.size());
  std::partial_sort(ord.begin(), ord.begin() + m, ord.end(), [&](size_t a, size_t b) {
    if (keys[a] != keys[b]) return keys[a] > keys[b];
    return ids[a] < ids[b];
  });
  std::vector<int64_t> sel;
  for (size_t i = 0; i < m; ++i) sel.push_back(ids[ord[i]]);
  std::sort(sel.begin(), sel.end());
  for (int i = 0; i < k; ++i) out[i] = (size_t(i) < sel.size()) ? int32_t(sel[i]) : -1;
}

template <class F>
void parallel_for(int64_t n, int nthreads, F fn) {
  if (nthreads <= 0) nthreads = int(std::max(1u, std::thread::hardware_concurrency()));
  nthreads = int(std::min<int64_t>(nthreads, std::max<int64_t>(n, 1)));
  if (nthreads <= 1) {
    for (int64_t i = 0; i < n; ++i) fn(i);
    return;
  }
  std::vector<std::thread> th;
  for (int t = 0; t < nthreads; ++t)
    th.emplace_back([&, t] {
      for (int64_t i = t; i < n; i += nthreads) fn(i);
    });
  for (auto& x : th) x.join();
}

const int kHi = 4, kDi = 128, kHq = 16, kD = 512, kBlk = 8;

// Scores of positions [0, L) of one sequence against one indexer query.
std::vector<float> scores_all(const uint8_t* kcodes, const uint8_t* kscales, int64_t row0, int64_t L,
                              const uint8_t* qc, const uint8_t* qs, const float* w) {
  std::vector<float> s(size_t(std::max<int64_t>(L, 0)));
  for (int64_t t = 0; t < L; ++t)
    s[t] = index_score(kcodes + (row0 + t) * 64, kscales + (row0 + t) * 4, qc, qs, w);
  return s;
}

// Full-mode indexer for one query over L visible positions [V41] hierarchical
// indexer: block maxima over 8 positions, the pool = Top-P blocks by (block
// max desc, block id asc), and the layer's own Top-k over ALL L positions.
void index_full_one(const uint8_t* kcodes, const uint8_t* kscales, int64_t row0, int64_t L,
                    const uint8_t* qc, const uint8_t* qs, const float* w, int P, int k,
                    int32_t* pool_out, int32_t* topk_out, float* scores_out) {
  std::vector<float> s = scores_all(kcodes, kscales, row0, L, qc, qs, w);
  if (scores_out)
    for (int64_t t = 0; t < L; ++t) scores_out[t] = s[t];
  int64_t nb = (L + kBlk - 1) / kBlk;
  std::vector<uint32_t> bkey(nb, 0);
  std::vector<int64_t> bid(nb);
  for (int64_t b = 0; b < nb; ++b) {
    bid[b] = b;
    for (int64_t t = b * kBlk; t < std::min(L, (b + 1) * kBlk); ++t)
      bkey[b] = std::max(bkey[b], rank_key(s[t]));
  }
  if (pool_out) topk_select(bkey, bid, P, pool_out);
  std::vector<uint32_t> key(L);
  std::vector<int64_t> id(L);
  for (int64_t t = 0; t < L; ++t) {
    key[t] = rank_key(s[t]);
    id[t] = t;
  }
  topk_select(key, id, k, topk_out);
}

// Attention of one query over a set of keys (= values): fp64 softmax.
// keys: list of (pointer to 512 doubles).
void attend(const uint16_t* q /*[16][512] bf16*/, const std::vector<std::vector<double>>& keys,
            double sm_scale, double* out /*[16][512]*/, double* lse /*[16]*/) {
  for (int h = 0; h < kHq; ++h) {
    double* o = out + h * kD;
    for (int d = 0; d < kD; ++d) o[d] = 0.0;
    if (keys.empty()) {
      if (lse) lse[h] = -INFINITY;
      continue;
    }
    std::vector<double> lg(keys.size());
    double m = -INFINITY;
    for (size_t j = 0; j < keys.size(); ++j) {
      double acc = 0.0;
      for (int d = 0; d < kD; ++d) acc += double(bf16_to_float(q[h * kD + d])) * keys[j][d];
      lg[j] = sm_scale * acc;
      m = std::max(m, lg[j]);
    }
    double l = 0.0;
    for (size_t j = 0; j < keys.size(); ++j) {
      double p = std::exp(lg[j] - m);
      l += p;
      for (int d = 0; d < kD; ++d) o[d] += p * keys[j][d];
    }
    for (int d = 0; d < kD; ++d) o[d] /= l;
    if (lse) lse[h] = m + std::log(l);
  }
}

std::vector<double> main_row(const uint8_t* codes, const uint8_t* scales, int64_t row) {
  std::vector<double> v(kD);
  mxfp4_decode_row(codes + row * (kD / 2), scales + row * (kD / 32), kD, v.data());
  return v;
}

std::vector<double> e4m3_row(const uint8_t* codes, double scale) {
  std::vector<double> v(kD);
  for (int d = 0; d < kD; ++d) v[d] = e4m3_value(codes[d]) * scale;
  return v;
}

}  // namespace

// ===========================================================================
// C ABI of the oracle (called from Python through ctypes).
// Return value: 0 on success, negative on an input the definitions reject.
// ===========================================================================
extern "C" {

double orc_e2m1_value(int code) { return e2m1_value(code); }
double orc_e8m0_value(int byte) { return e8m0_value(byte); }
double orc_e4m3_value(int byte) { return e4m3_value(byte); }
double orc_exp(double x) { return own_exp(x); }
uint32_t orc_rank_key(float s) { return rank_key(s); }

void orc_mxfp4_encode(const float* x, int64_t rows, int n, uint8_t* codes, uint8_t* scales) {
  for (int64_t r = 0; r < rows; ++r)
    mxfp4_encode_row(x + r * n, n, codes + r * (n / 2), scales + r * (n / 32));
}

void orc_mxfp4_decode(const uint8_t* codes, const uint8_t* scales, int64_t rows, int n, double* out) {
  for (int64_t r = 0; r < rows; ++r)
    mxfp4_decode_row(codes + r * (n / 2), scales + r * (n / 32), n, out + r * n);
}

// Scores of `n` cache rows (row ids given) against one indexer query.
void orc_index_scores(const uint8_t* kcodes, const uint8_t* kscales, const int64_t* rows, int64_t n,
                      const uint8_t* qc, const uint8_t* qs, const float* w, float* out) {
  for (int64_t i = 0; i < n; ++i)
    out[i] = index_score(kcodes + rows[i] * 64, kscales + rows[i] * 4, qc, qs, w);
}

// Top-k of explicit keys/ids (test helper for the selection rule).
void orc_topk(const uint32_t* keys, const int64_t* ids, int64_t n, int k, int32_t* out) {
  std::vector<uint32_t> kk(keys, keys + n);
  std::vector<int64_t> ii(ids, ids + n);
  topk_select(kk, ii, k, out);
}

// Full-mode decode indexer for a batch.  q codes [B][4][64], q scales
// [B][4][4], w [B][4]; sequence b occupies cache rows seq_row_off[b] ..
// + seq_len[b].  pool_out [B][P] (may be null), topk_out [B][k],
// scores_out [B][max_len] or null.
int orc_index_full(const uint8_t* kcodes, const uint8_t* kscales, const uint8_t* qc, const uint8_t* qs,
                   const float* w, const int64_t* seq_row_off, const int32_t* seq_len, int B, int P, int k,
                   int32_t* pool_out, int32_t* topk_out, float* scores_out, int64_t max_len, int nthreads) {
  parallel_for(B, nthreads, [&](int64_t b) {
    index_full_one(kcodes, kscales, seq_row_off[b], seq_len[b], qc + b * kHi * 64, qs + b * kHi * 4,
                   w + b * kHi, P, k, pool_out ? pool_out + b * P : nullptr, topk_out + b * k,
                   scores_out ? scores_out + b * max_len : nullptr);
  });
  return 0;
}

// Reindex-mode indexer [V41]/[NOTES]: score only the positions of the pool
// blocks (8 positions each, those < seq_len) with this layer's q and w against
// the nearest Full layer's indexer K, then Top-k by (score desc, position asc).
int orc_index_reindex(const uint8_t* kcodes, const uint8_t* kscales, const uint8_t* qc, const uint8_t* qs,
                      const float* w, const int64_t* seq_row_off, const int32_t* seq_len,
                      const int32_t* pool, int B, int P, int k, int32_t* topk_out, int nthreads) {
  parallel_for(B, nthreads, [&](int64_t b) {
    std::vector<uint32_t> key;
    std::vector<int64_t> id;
    for (int i = 0; i < P; ++i) {
      int32_t blk = pool[b * P + i];
      if (blk < 0) continue;
      for (int j = 0; j < kBlk; ++j) {
        int64_t t = int64_t(blk) * kBlk + j;
        if (t >= seq_len[b]) continue;
        int64_t row = seq_row_off[b] + t;
        float s = index_score(kcodes + row * 64, kscales + row * 4, qc + b * kHi * 64, qs + b * kHi * 4,
                              w + b * kHi);
        key.push_back(rank_key(s));
        id.push_back(t);
      }
    }
    topk_select(key, id, k, topk_out + b * k);
  });
  return 0;
}

// Sparse attention decode [V41]: one softmax over the selected MXFP4 main-KV
// rows (topk, -1 skipped) followed by the first win_len rows of the FP8 E4M3
// window (times its per-(sequence, layer) fp32 scale).  Keys = values (shared
// latent).  out [B][16][512] fp64, lse [B][16] fp64 (may be null).
int orc_attn_decode(const uint16_t* q, const uint8_t* mcodes, const uint8_t* mscales,
                    const int64_t* seq_row_off, const int32_t* seq_len, const int32_t* topk, int k,
                    const uint8_t* win, const float* win_scale, const int32_t* win_len, double sm_scale,
                    double* out, double* lse, int B, int nthreads) {
  int bad = 0;
  parallel_for(B, nthreads, [&](int64_t b) {
    std::vector<std::vector<double>> keys;
    for (int j = 0; j < k; ++j) {
      int32_t t = topk[b * k + j];
      if (t < 0) continue;
      if (t >= seq_len[b]) {
        bad = 1;
        continue;
      }
      keys.push_back(main_row(mcodes, mscales, seq_row_off[b] + t));
    }
    for (int r = 0; r < win_len[b]; ++r)
      keys.push_back(e4m3_row(win + (b * 128 + r) * int64_t(kD), double(win_scale[b])));
    attend(q + b * kHq * kD, keys, sm_scale, out + b * kHq * kD, lse ? lse + b * kHq : nullptr);
  });
  return bad ? -1 : 0;
}

// Compression + quantisation of new cache entries [V41]: m tokens become one
// entry, entries have disjoint sources and no absolute position encoding; the
// weights are a softmax over the pair's per-token logits (the plainest
// reading of a weighting formula the page prints garbled).
// ratio 1: c = x.  ratio 2: entry j merges raw rows 2j, 2j+1:
//   m = max(z0, z1); a = exp(z0-m); b = exp(z1-m); w0 = a/(a+b); w1 = b/(a+b)
//   c_i = fp32( fma(w0, x0_i, w1*x1_i) )   (fp64, own exp)
// Indexer row: W_idx given -> r_j = fp32( sum_i c_i * W[i][j] ) by an fp64
// fma chain in order i = 0..511; else the 128-d idx_raw rows are merged with
// the same weights.  Both rows are then MXFP4-encoded.  c_out [n][512] and
// r_out [n][128] (may be null) receive the fp32 rows before quantisation.
int orc_compress(const uint16_t* raw, const float* logits, const float* w_idx, const uint16_t* idx_raw,
                 int64_t n_entries, int ratio, uint8_t* mcodes, uint8_t* mscales, uint8_t* icodes,
                 uint8_t* iscales, float* c_out, float* r_out, int nthreads) {
  if (ratio != 1 && ratio != 2) return -1;
  parallel_for(n_entries, nthreads, [&](int64_t j) {
    double w0 = 1.0, w1 = 0.0;
    if (ratio == 2) {
      double z0 = logits[2 * j], z1 = logits[2 * j + 1];
      double m = std::max(z0, z1);
      double a = own_exp(z0 - m), b = own_exp(z1 - m);
      double s = a + b;
      w0 = a / s;
      w1 = b / s;
    }
    auto merge = [&](const uint16_t* src, int64_t stride, int n, float* c) {
      for (int i = 0; i < n; ++i) {
        if (ratio == 1) {
          c[i] = bf16_to_float(src[j * stride + i]);
        } else {
          double x0 = bf16_to_float(src[(2 * j) * stride + i]);
          double x1 = bf16_to_float(src[(2 * j + 1) * stride + i]);
          c[i] = float(std::fma(w0, x0, w1 * x1));
        }
      }
    };
    float c[kD], r[kDi];
    merge(raw, kD, kD, c);
    mxfp4_encode_row(c, kD, mcodes + j * (kD / 2), mscales + j * (kD / 32));
    if (w_idx) {
      for (int o = 0; o < kDi; ++o) {
        double acc = 0.0;
        for (int i = 0; i < kD; ++i) acc = std::fma(double(c[i]), double(w_idx[i * kDi + o]), acc);
        r[o] = float(acc);
      }
    } else {
      merge(idx_raw, kDi, kDi, r);
    }
    mxfp4_encode_row(r, kDi, icodes + j * (kDi / 2), iscales + j * (kDi / 32));
    if (c_out) std::memcpy(c_out + j * kD, c, sizeof(c));
    if (r_out) std::memcpy(r_out + j * kDi, r, sizeof(r));
  });
  return 0;
}

// Causal prefill indexer for one sequence: query i at raw position q_pos[i]
// sees entries j with (j+1)*ratio - 1 <= q_pos[i] (entry j holds raw tokens
// ratio*j .. ratio*j+ratio-1), capped at n_entries.  Same Full-mode selection
// as decode over those visible entries.
int orc_index_prefill(const uint8_t* kcodes, const uint8_t* kscales, int64_t row0, int64_t n_entries,
                      const uint8_t* qc, const uint8_t* qs, const float* w, const int32_t* q_pos,
                      const int32_t* q_ids, int64_t nq, int ratio, int P, int k, int32_t* pool_out,
                      int32_t* topk_out, int nthreads) {
  parallel_for(nq, nthreads, [&](int64_t ii) {
    int64_t i = q_ids ? q_ids[ii] : ii;
    int64_t vis = std::min<int64_t>(n_entries, (int64_t(q_pos[i]) + 1) / ratio);
    index_full_one(kcodes, kscales, row0, vis, qc + i * kHi * 64, qs + i * kHi * 4, w + i * kHi, P, k,
                   pool_out ? pool_out + ii * P : nullptr, topk_out + ii * k, nullptr);
  });
  return 0;
}

// Causal prefill attention: query i attends its selected entries plus the
// raw FP8 window rows max(0, p-127) .. p (one fp32 scale for the tensor).
int orc_attn_prefill(const uint16_t* q, const int32_t* q_pos, const int32_t* q_ids, int64_t nq,
                     const uint8_t* mcodes, const uint8_t* mscales, int64_t row0, int64_t n_entries,
                     int ratio, const int32_t* topk, int k, const uint8_t* raw_win, float win_scale,
                     double sm_scale, double* out, double* lse, int nthreads) {
  int bad = 0;
  parallel_for(nq, nthreads, [&](int64_t ii) {
    int64_t i = q_ids ? q_ids[ii] : ii;
    int64_t p = q_pos[i];
    int64_t vis = std::min<int64_t>(n_entries, (p + 1) / ratio);
    std::vector<std::vector<double>> keys;
    for (int j = 0; j < k; ++j) {
      int32_t t = topk[ii * k + j];
      if (t < 0) continue;
      if (t >= vis) {
        bad = 1;
        continue;
      }
      keys.push_back(main_row(mcodes, mscales, row0 + t));
    }
    for (int64_t r = std::max<int64_t>(0, p - 127); r <= p; ++r)
      keys.push_back(e4m3_row(raw_win + r * kD, double(win_scale)));
    attend(q + i * kHq * kD, keys, sm_scale, out + ii * kHq * kD, lse ? lse + ii * kHq : nullptr);
  });
  return bad ? -1 : 0;
}

}  // extern "C"
