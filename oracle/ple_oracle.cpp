// CPU oracle for the hashed n-gram (PLE / Engram) embedding lookup.
//
// TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link,
// load or call this file; only the tests, the package's smoke check and the
// benchmark's CPU-baseline leg do.  It shares no code, header, constant or
// helper with the CUDA library: the hash, the remainder, the gather and the
// gradient fold are written out here once more, in the plainest scalar form.
//
// What it follows (NeMo AutoModel API page "nemo_automodel.components.models.
// qwen3_8_flash_next.engram", class Qwen3_8_FlashNextNGramEmbedding):
//  * heads are grouped by n-gram order: the first heads_per_ngram heads hash
//    bigrams, the next group trigrams, up to ngram_size (class docstring);
//  * previous-token context resets AFTER an EOS token and never crosses a
//    packed-segment boundary (class docstring; _shift_right_after_eos;
//    _hash_input_ids "n-gram history stays inside a segment");
//  * signed int64 overflow (wrapping), positive remainders modulo the
//    per-head prime, plus the global head offset (class docstring;
//    parameters layer_multipliers [ngram_size], ngram_heads_vocab_sizes,
//    ngram_heads_offsets);
//  * the page does not print the combine.  The reading adopted: the order-m
//    hash is h_m = sum_{k<m} ctx_k * mult[k] (wrapping), ctx_0 the current
//    token, ctx_k the token k back or the sentinel 0 when that position lies
//    before the context start, and row = offset_j + ((h % p_j) + p_j) % p_j;
//  * _lookup_ngram_ids returns the heads' rows concatenated per token:
//    output [T, H, D] with heads ascending;
//  * the table is a plain embedding parameter, so the backward pass adds the
//    gradients of all hits of a row into that row.  The page fixes no
//    summation order; the order adopted (and checked bit for bit) is: the
//    hits of row r in ascending flat index i = t*H + j, cut into chunks of 32
//    consecutive hits; each chunk summed left to right starting from its
//    first element; the chunk sums summed left to right starting from the
//    first; the result added once into table_grad[r].  Parity unpinned by
//    the page for that order itself: it is the library's contract, held here
//    by closed-form cases only this order produces (the pins in
//    tests/test_oracle_pins.py), while the sums' values are pinned against
//    fp64 index_add and exact integer gradients.
//
// Build: g++ -O2 -ffp-contract=off -std=c++17 -shared -fPIC (no fast-math,
// so every float add below is one IEEE round-to-nearest add).
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <thread>
#include <utility>
#include <vector>

namespace {

constexpr int64_t kChunk = 32;  // hits per chunk in the gradient fold

float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

float grad_at(const void* grad, int grad_is_bf16, int64_t i, int32_t D, int32_t d) {
  const int64_t k = i * D + d;
  if (grad_is_bf16) return bf16_to_float(static_cast<const uint16_t*>(grad)[k]);
  return static_cast<const float*>(grad)[k];
}

// Wrapping int64 product and sum, done in uint64 (two's complement).
int64_t wrap_mul(int64_t a, int64_t b) {
  return static_cast<int64_t>(static_cast<uint64_t>(a) * static_cast<uint64_t>(b));
}
int64_t wrap_add(int64_t a, int64_t b) {
  return static_cast<int64_t>(static_cast<uint64_t>(a) + static_cast<uint64_t>(b));
}

// Rows of every token of sequences [s0, s1).
void rows_of_sequences(const int64_t* tokens, const int32_t* cu, int32_t s0, int32_t s1,
                       int32_t n, int32_t G, int64_t eos, const int64_t* mult,
                       const int64_t* prime, const int64_t* offset, int64_t* rows) {
  const int32_t H = (n - 1) * G;
  std::vector<int64_t> ctx(n);
  for (int32_t s = s0; s < s1; ++s) {
    int64_t start = cu[s];  // first position whose token may serve as context
    for (int64_t t = cu[s]; t < cu[s + 1]; ++t) {
      ctx[0] = tokens[t];
      for (int32_t k = 1; k < n; ++k) ctx[k] = (t - k >= start) ? tokens[t - k] : 0;
      for (int32_t m = 2; m <= n; ++m) {
        int64_t h = 0;
        for (int32_t k = 0; k < m; ++k) h = wrap_add(h, wrap_mul(ctx[k], mult[k]));
        for (int32_t g = 0; g < G; ++g) {
          const int32_t j = (m - 2) * G + g;
          int64_t r = h % prime[j];
          if (r < 0) r += prime[j];
          rows[t * H + j] = offset[j] + r;
        }
      }
      if (tokens[t] == eos) start = t + 1;  // the reset takes effect after the EOS
    }
  }
}

int check_cu(const int32_t* cu, int32_t S, int64_t T) {
  if (S < 0 || cu[0] != 0 || cu[S] != T) return -1;
  for (int32_t s = 0; s < S; ++s)
    if (cu[s + 1] < cu[s]) return -1;
  return 0;
}

// Stable order of hits by row: (row, i) pairs sorted lexicographically.
std::vector<std::pair<int64_t, int64_t>> sorted_hits(const int64_t* rows, int64_t N) {
  std::vector<std::pair<int64_t, int64_t>> p(N);
  for (int64_t i = 0; i < N; ++i) p[i] = {rows[i], i};
  std::sort(p.begin(), p.end());
  return p;
}

// Sum of one row's hits [a, b) of the sorted list, in the fixed chunked order.
void fold_row(const std::vector<std::pair<int64_t, int64_t>>& p, int64_t a, int64_t b,
              const void* grad, int grad_is_bf16, int32_t D, float* out) {
  std::vector<float> chunk(D);
  for (int64_t c0 = a; c0 < b; c0 += kChunk) {
    const int64_t c1 = std::min(b, c0 + kChunk);
    for (int32_t d = 0; d < D; ++d) chunk[d] = grad_at(grad, grad_is_bf16, p[c0].second, D, d);
    for (int64_t e = c0 + 1; e < c1; ++e)
      for (int32_t d = 0; d < D; ++d) chunk[d] = chunk[d] + grad_at(grad, grad_is_bf16, p[e].second, D, d);
    if (c0 == a)
      for (int32_t d = 0; d < D; ++d) out[d] = chunk[d];
    else
      for (int32_t d = 0; d < D; ++d) out[d] = out[d] + chunk[d];
  }
}

}  // namespace

extern "C" {

// Row ids [T, H] for packed tokens.  Returns 0, or -1 for malformed
// cu_seqlens (cu[0] != 0, cu[S] != T, or decreasing).
int oracle_ple_rows(const int64_t* tokens, int64_t T, const int32_t* cu_seqlens, int32_t num_seqs,
                    int32_t ngram_size, int32_t heads_per_ngram, int64_t eos_id,
                    const int64_t* mults, const int64_t* primes, const int64_t* offsets,
                    int64_t* rows) {
  if (check_cu(cu_seqlens, num_seqs, T) != 0) return -1;
  rows_of_sequences(tokens, cu_seqlens, 0, num_seqs, ngram_size, heads_per_ngram, eos_id, mults,
                    primes, offsets, rows);
  return 0;
}

// Same result with the sequences dealt round-robin to nthreads std::threads.
int oracle_ple_rows_mt(const int64_t* tokens, int64_t T, const int32_t* cu_seqlens, int32_t num_seqs,
                       int32_t ngram_size, int32_t heads_per_ngram, int64_t eos_id,
                       const int64_t* mults, const int64_t* primes, const int64_t* offsets,
                       int64_t* rows, int32_t nthreads) {
  if (check_cu(cu_seqlens, num_seqs, T) != 0) return -1;
  if (nthreads < 1) nthreads = 1;
  std::vector<std::thread> pool;
  for (int32_t w = 0; w < nthreads; ++w)
    pool.emplace_back([=] {
      for (int32_t s = w; s < num_seqs; s += nthreads)
        rows_of_sequences(tokens, cu_seqlens, s, s + 1, ngram_size, heads_per_ngram, eos_id, mults,
                          primes, offsets, rows);
    });
  for (auto& th : pool) th.join();
  return 0;
}

// out[i, :] = table[rows[i], :] as raw bytes.  Returns 0, or -1 if a row is
// outside [0, num_rows).
int oracle_ple_gather(const int64_t* rows, int64_t N, const void* table, int64_t num_rows,
                      int64_t row_bytes, void* out) {
  for (int64_t i = 0; i < N; ++i)
    if (rows[i] < 0 || rows[i] >= num_rows) return -1;
  const char* src = static_cast<const char*>(table);
  char* dst = static_cast<char*>(out);
  for (int64_t i = 0; i < N; ++i) std::memcpy(dst + i * row_bytes, src + rows[i] * row_bytes, row_bytes);
  return 0;
}

int oracle_ple_gather_mt(const int64_t* rows, int64_t N, const void* table, int64_t num_rows,
                         int64_t row_bytes, void* out, int32_t nthreads) {
  for (int64_t i = 0; i < N; ++i)
    if (rows[i] < 0 || rows[i] >= num_rows) return -1;
  if (nthreads < 1) nthreads = 1;
  std::vector<std::thread> pool;
  for (int32_t w = 0; w < nthreads; ++w)
    pool.emplace_back([=] {
      const int64_t a = N * w / nthreads, b = N * (w + 1) / nthreads;
      const char* src = static_cast<const char*>(table);
      char* dst = static_cast<char*>(out);
      for (int64_t i = a; i < b; ++i) std::memcpy(dst + i * row_bytes, src + rows[i] * row_bytes, row_bytes);
    });
  for (auto& th : pool) th.join();
  return 0;
}

// bf16 bit pattern of an fp8 e4m3 code (OCP 8-bit floating point spec,
// "E4M3": 1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no
// infinities, S.1111.111 is NaN).  Every e4m3 value is exactly a bf16 value.
uint16_t e4m3_to_bf16_bits(uint8_t code) {
  const uint16_t sign = static_cast<uint16_t>(code & 0x80) << 8;
  const int e = (code >> 3) & 0xF, m = code & 0x7;
  if (e == 0xF && m == 0x7) return sign | 0x7FC0;       // NaN
  if (e == 0 && m == 0) return sign;                     // +-0
  if (e == 0) {                                          // subnormal: m * 2^-9
    int p = 2;
    while (!((m >> p) & 1)) --p;                         // leading one of m
    const int exp = p - 9 + 127;
    const int frac = (m - (1 << p)) << (7 - p);
    return sign | static_cast<uint16_t>(exp << 7) | static_cast<uint16_t>(frac);
  }
  return sign | static_cast<uint16_t>((e - 7 + 127) << 7) | static_cast<uint16_t>(m << 4);
}

// out[i, :] = bf16(table[rows[i], :]) for an fp8 e4m3 table [num_rows, D].
int oracle_ple_gather_e4m3(const int64_t* rows, int64_t N, const uint8_t* table, int64_t num_rows, int64_t D,
                           uint16_t* out) {
  for (int64_t i = 0; i < N; ++i)
    if (rows[i] < 0 || rows[i] >= num_rows) return -1;
  for (int64_t i = 0; i < N; ++i)
    for (int64_t d = 0; d < D; ++d) out[i * D + d] = e4m3_to_bf16_bits(table[rows[i] * D + d]);
  return 0;
}

// Number of distinct rows among rows[0..N).
int64_t oracle_ple_count_unique(const int64_t* rows, int64_t N) {
  std::vector<int64_t> r(rows, rows + N);
  std::sort(r.begin(), r.end());
  return static_cast<int64_t>(std::unique(r.begin(), r.end()) - r.begin());
}

// Per-row gradient sums in the fixed order.  Writes the touched rows in
// ascending order to uniq_rows[0..U) and their sums to sums[U, D]; returns U
// (the caller sizes both from oracle_ple_count_unique).
int64_t oracle_ple_grad_sums(const int64_t* rows, int64_t N, const void* grad, int grad_is_bf16,
                             int32_t D, int64_t* uniq_rows, float* sums) {
  const auto p = sorted_hits(rows, N);
  int64_t u = 0;
  for (int64_t a = 0; a < N;) {
    int64_t b = a + 1;
    while (b < N && p[b].first == p[a].first) ++b;
    uniq_rows[u] = p[a].first;
    fold_row(p, a, b, grad, grad_is_bf16, D, sums + u * D);
    ++u;
    a = b;
  }
  return u;
}

// Same, with the rows dealt to nthreads std::threads after one sort.
int64_t oracle_ple_grad_sums_mt(const int64_t* rows, int64_t N, const void* grad, int grad_is_bf16,
                                int32_t D, int64_t* uniq_rows, float* sums, int32_t nthreads) {
  const auto p = sorted_hits(rows, N);
  std::vector<int64_t> starts;
  for (int64_t a = 0; a < N; ++a)
    if (a == 0 || p[a].first != p[a - 1].first) starts.push_back(a);
  const int64_t U = static_cast<int64_t>(starts.size());
  starts.push_back(N);
  if (nthreads < 1) nthreads = 1;
  std::vector<std::thread> pool;
  for (int32_t w = 0; w < nthreads; ++w)
    pool.emplace_back([&, w] {
      for (int64_t u = U * w / nthreads; u < U * (w + 1) / nthreads; ++u) {
        uniq_rows[u] = p[starts[u]].first;
        fold_row(p, starts[u], starts[u + 1], grad, grad_is_bf16, D, sums + u * D);
      }
    });
  for (auto& th : pool) th.join();
  return U;
}

// table_grad[r, :] = table_grad[r, :] + S_r for every touched row r (dense
// [num_rows, D] fp32).  Returns 0, or -1 if a row is outside [0, num_rows).
int oracle_ple_grad_apply(const int64_t* rows, int64_t N, const void* grad, int grad_is_bf16,
                          int32_t D, int64_t num_rows, float* table_grad) {
  for (int64_t i = 0; i < N; ++i)
    if (rows[i] < 0 || rows[i] >= num_rows) return -1;
  const auto p = sorted_hits(rows, N);
  std::vector<float> s(D);
  for (int64_t a = 0; a < N;) {
    int64_t b = a + 1;
    while (b < N && p[b].first == p[a].first) ++b;
    fold_row(p, a, b, grad, grad_is_bf16, D, s.data());
    float* dst = table_grad + p[a].first * D;
    for (int32_t d = 0; d < D; ++d) dst[d] = dst[d] + s[d];
    a = b;
  }
  return 0;
}

// ---------------------------------------------------------------------------
// Segment-aware causal dilated depthwise convolution (NeMo AutoModel engram
// API page, Qwen3_8_FlashNextPLELayer._causal_short_conv and
// _segmented_conv): every packed segment is convolved as if it started a
// fresh row, with (K-1)*dilation zeros of history ahead of it, one filter of
// K taps per channel (depthwise), tap k reading the position
// dilation*(K-1-k) tokens back.  Plain fp64 loops in the order of that
// definition.
// ---------------------------------------------------------------------------
int oracle_conv_forward(const double* x, int64_t T, int64_t C, const int32_t* cu_seqlens, int32_t num_seqs,
                        const double* w, int32_t K, int32_t dilation, const double* bias, double* y) {
  if (T < 0 || C < 1 || K < 1 || dilation < 1 || num_seqs < 1) return -1;
  if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -2;
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int64_t start = cu_seqlens[s];
    for (int64_t t = start; t < cu_seqlens[s + 1]; ++t) {
      for (int64_t c = 0; c < C; ++c) {
        double acc = bias != nullptr ? bias[c] : 0.0;
        for (int32_t k = 0; k < K; ++k) {
          const int64_t src = t - static_cast<int64_t>(dilation) * (K - 1 - k);
          if (src >= start) acc += w[c * K + k] * x[src * C + c];  // before the segment: zero history
        }
        y[t * C + c] = acc;
      }
    }
  }
  return 0;
}

// Gradients of the convolution above for an output gradient dy: every tap
// (t, k) that read x[src, c] sends w[c, k] * dy[t, c] to dx[src, c] and
// dy[t, c] * x[src, c] to dw[c, k]; db[c] sums dy[., c].  dx, dw and db are
// overwritten; any of them may be null.
int oracle_conv_backward(const double* dy, const double* x, int64_t T, int64_t C, const int32_t* cu_seqlens,
                         int32_t num_seqs, const double* w, int32_t K, int32_t dilation, double* dx, double* dw,
                         double* db) {
  if (T < 0 || C < 1 || K < 1 || dilation < 1 || num_seqs < 1) return -1;
  if (cu_seqlens[0] != 0 || cu_seqlens[num_seqs] != T) return -2;
  if (dx != nullptr) std::fill(dx, dx + T * C, 0.0);
  if (dw != nullptr) std::fill(dw, dw + C * K, 0.0);
  if (db != nullptr) std::fill(db, db + C, 0.0);
  for (int32_t s = 0; s < num_seqs; ++s) {
    const int64_t start = cu_seqlens[s];
    for (int64_t t = start; t < cu_seqlens[s + 1]; ++t) {
      for (int64_t c = 0; c < C; ++c) {
        const double g = dy[t * C + c];
        if (db != nullptr) db[c] += g;
        for (int32_t k = 0; k < K; ++k) {
          const int64_t src = t - static_cast<int64_t>(dilation) * (K - 1 - k);
          if (src < start) continue;
          if (dx != nullptr) dx[src * C + c] += w[c * K + k] * g;
          if (dw != nullptr) dw[c * K + k] += g * x[src * C + c];
        }
      }
    }
  }
  return 0;
}

}  // extern "C"
