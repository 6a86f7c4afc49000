// The PLE layer's short convolution: a causal, dilated, depthwise 1-D
// convolution over packed tokens in which every packed segment starts with
// zero history (Qwen3_8_FlashNextPLELayer._causal_short_conv and
// _segmented_conv, NeMo AutoModel engram API page):
//   y[t, c] = bias[c] + sum_k w[c, k] * x[t - dilation*(K-1-k), c],
// a tap before the first position of t's segment reading zero.
//
// HBM-bound: x is read once from DRAM and y written once.  A thread owns one
// 16-byte vector of channels (8 bf16 or 4 fp32) and walks a chunk of tokens
// one residue class modulo the dilation at a time (the taps of a token lie
// in its class), keeping the class's previous rows in registers, so every
// load and store of a warp covers 512 consecutive bytes of a token row and
// each row is loaded once (plus K-1 rows of history per class and chunk).
// The backward pass computes dx (the same taps looking ahead, inside the
// segment) and per-chunk partial sums of dw and db in one sweep when both
// are asked for (dy and x read once; a thread owns 4 channels there so that
// both tensors' rows fit its registers), or either alone in a kernel of its
// own; a last kernel adds the chunk partials in chunk order (deterministic)
// and adds the result once into the caller's dw and db.
#include <cuda_bf16.h>

#include <type_traits>

#include "common.cuh"

namespace ple {
namespace {

constexpr int kConvThreads = 128;     // channel vectors per block
constexpr int kConvChunk = 128;       // tokens per block, forward
constexpr int kConvBwdChunk = 256;    // least tokens per block, backward (doubled for wide rows)
constexpr int64_t kMaxPartials = 1024;  // at most this many backward chunks (their partial sums)
constexpr int kMaxTaps = 8;

// Blocks per SM the register budget is cut for (measured: more rows in
// flight beats fewer, until the row registers start to spill); larger K
// holds more rows and gets fewer blocks.
constexpr int fwd_min_blocks(int K) { return K <= 4 ? 5 : K <= 5 ? 4 : K <= 7 ? 3 : 2; }
constexpr int dx_min_blocks(int K) { return K <= 4 ? 4 : K <= 7 ? 3 : 2; }
constexpr int dw_min_blocks(int K) { return K <= 4 ? 4 : K <= 5 ? 3 : 2; }
constexpr int bwd_min_blocks(int K, bool bf16) {
  return bf16 ? (K <= 4 ? 4 : K <= 6 ? 3 : 2) : (K <= 2 ? 4 : K <= 4 ? 3 : 2);
}

template <bool BF16>
struct Vec {
  static constexpr int n = BF16 ? 8 : 4;  // channels per 16-byte vector
};

template <bool BF16>
__device__ __forceinline__ void unpack(const uint4& u, float* v) {
  if constexpr (BF16) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  } else {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  }
}

template <bool BF16>
__device__ __forceinline__ uint4 pack(const float* v) {
  if constexpr (BF16) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);  // .x = low half
      w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    return make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3]));
  }
}

__device__ __forceinline__ uint4 ld_vec(const unsigned char* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Four channels: 8 bytes of bf16 or 16 bytes of fp32 (the fused backward's
// unit, half the registers per row of a 16-byte bf16 vector).
template <bool BF16>
struct Quad {
  using type = typename std::conditional<BF16, uint2, uint4>::type;
  static constexpr int bytes = BF16 ? 8 : 16;
};

template <bool BF16>
__device__ __forceinline__ typename Quad<BF16>::type ld_quad(const unsigned char* p) {
  return __ldg(reinterpret_cast<const typename Quad<BF16>::type*>(p));
}

template <bool BF16>
__device__ __forceinline__ typename Quad<BF16>::type zero_quad() {
  typename Quad<BF16>::type z;
  if constexpr (BF16) z = make_uint2(0, 0); else z = make_uint4(0, 0, 0, 0);
  return z;
}

template <bool BF16>
__device__ __forceinline__ void unpack4(const typename Quad<BF16>::type& u, float* v) {
  if constexpr (BF16) {
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xffff0000u);
  } else {
    v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y); v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
  }
}

template <bool BF16>
__device__ __forceinline__ void st_quad(unsigned char* p, const float* v) {
  if constexpr (BF16) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    const uint2 u = make_uint2(*reinterpret_cast<const uint32_t*>(&a), *reinterpret_cast<const uint32_t*>(&b));
    asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(u.x), "r"(u.y) : "memory");
  } else {
    st_cs(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]), __float_as_uint(v[3])));
  }
}

// The packed segment of the positions a thread walks (in increasing order).
// Bounds are clamped to [0, T]; with a malformed cu_seqlens (flagged by
// check_cu) a position the array does not cover is treated as a segment of
// its own, so every access stays inside the tensors.
struct Segment {
  const int32_t* cu;
  int32_t num_seqs, s;
  int64_t T, lo, hi;
  __device__ void load() {
    lo = min(max(static_cast<int64_t>(__ldg(cu + s)), int64_t{0}), T);
    hi = min(max(static_cast<int64_t>(__ldg(cu + s + 1)), int64_t{0}), T);
  }
  __device__ void start(int64_t t) {  // the last s with cu[s] <= t (binary search)
    int32_t a = 0, b = num_seqs - 1;
    while (a < b) {
      const int32_t mid = (a + b + 1) >> 1;
      if (static_cast<int64_t>(__ldg(cu + mid)) <= t) a = mid; else b = mid - 1;
    }
    s = a;
    load();
  }
  __device__ void advance(int64_t t) {  // to the segment holding t (empty segments skipped)
    while (t >= hi && s + 1 < num_seqs) {
      ++s;
      load();
    }
  }
  __device__ int64_t first(int64_t t) const { return t >= lo && t < hi ? lo : t; }    // history starts here
  __device__ int64_t end(int64_t t) const { return t >= lo && t < hi ? hi : t + 1; }  // lookahead ends here
};

// The taps of chain position t that stay inside t's segment: `back` chain
// steps before t (capped at K-1) and `ahead` steps after it (capped).  Kept
// incrementally along a chain; a division only when the chain enters a
// segment.  Equivalent to t - j d >= first(t) and t + j d < end(t).
template <int K>
struct ChainTaps {
  int64_t lo = 1, hi = 0, rem = 0;  // segment [lo, hi) of the last step; chain steps left in it
  int back = 0, ahead = 0;
  __device__ __forceinline__ void step(Segment& sg, int64_t t, int64_t d) {
    if (t >= lo && t < hi) {  // one chain step further inside the same segment
      back = min(back + 1, K - 1);
      --rem;
      ahead = rem < K - 1 ? static_cast<int>(rem) : K - 1;
    } else {
      sg.advance(t);
      lo = sg.first(t);
      hi = sg.end(t);
      back = static_cast<int>(min((t - lo) / d, static_cast<int64_t>(K - 1)));
      rem = (hi - 1 - t) / d;
      ahead = static_cast<int>(min(rem, static_cast<int64_t>(K - 1)));
    }
  }
  // n steps inside the segment, each with all K - 1 taps behind and ahead
  __device__ __forceinline__ void skip(int n) {
    back = K - 1;
    rem -= n;
    ahead = rem < K - 1 ? static_cast<int>(rem) : K - 1;
  }
};

// Block (0, 0) checks cu_seqlens once per launch: cu[0] == 0, cu[S] == T,
// non-decreasing.  Bad input only raises a flag.
__device__ void check_cu(const int32_t* __restrict__ cu, int32_t num_seqs, int64_t T, unsigned int* status) {
  if (blockIdx.x != 0 || blockIdx.y != 0) return;
  bool bad = false;
  if (threadIdx.x == 0) bad = (cu[0] != 0) || (static_cast<int64_t>(cu[num_seqs]) != T);
  for (int32_t i = threadIdx.x; i < num_seqs; i += blockDim.x) bad |= cu[i + 1] < cu[i];
  if (bad) raise_flag(status, PLE_ERR_BAD_SEQLENS);
}

// Forward.  Block (token chunk bx, vector block by); thread = one channel
// vector.  The taps of token t lie at t, t - d, ..., t - (K-1) d: all in
// t's residue class modulo the dilation d.  So a thread walks the chunk one
// residue class (chain) at a time, K chain steps per iteration, holding the
// chain's previous K rows in registers (static indices): one new row load
// per output, K of them in flight; the K-1 rows before the chunk come from
// one load each at the start of every chain.
template <bool BF16, int K>
__global__ void __launch_bounds__(kConvThreads, fwd_min_blocks(K))
conv_forward_kernel(const unsigned char* __restrict__ x, int64_t T, int64_t nvec, const int32_t* __restrict__ cu,
                    int32_t num_seqs, const float* __restrict__ w, int dilation,
                    const float* __restrict__ bias, unsigned char* __restrict__ y, unsigned int* status) {
  constexpr int V = Vec<BF16>::n;
  check_cu(cu, num_seqs, T, status);
  const int64_t cv = static_cast<int64_t>(blockIdx.y) * kConvThreads + threadIdx.x;  // channel vector
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kConvChunk;
  if (cv >= nvec || t0 >= T) return;
  const int64_t C = nvec * V, row = C * (BF16 ? 2 : 4);
  float wr[V][K], b[V];
#pragma unroll
  for (int v = 0; v < V; ++v) {
    b[v] = bias != nullptr ? __ldg(bias + cv * V + v) : 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) wr[v][k] = __ldg(w + (cv * V + v) * K + k);
  }
  const int64_t t1 = min(T, t0 + kConvChunk), d = dilation;
  const unsigned char* xc = x + cv * 16;
  unsigned char* yc = y + cv * 16;
  Segment sg{cu, num_seqs, 0, T, 0, 0};
  constexpr int U = 2 * K;  // chain steps per iteration: U row loads in flight
  for (int64_t r = 0; r < d && t0 + r < t1; ++r) {
    sg.start(t0 + r);
    uint4 prev[K], cur[U];  // chain rows: prev = the K steps before cur
#pragma unroll
    for (int j = 1; j < K; ++j) {  // steps -1 .. -(K-1) before the chain's first token
      const int64_t t = t0 + r - static_cast<int64_t>(K - j) * d;
      prev[j] = t >= 0 ? ld_vec(xc + t * row) : make_uint4(0, 0, 0, 0);
    }
    for (int64_t tb = t0 + r; tb < t1; tb += U * d) {
#pragma unroll
      for (int m = 0; m < U; ++m) {
        const int64_t t = tb + m * d;
        cur[m] = t < t1 ? ld_vec(xc + t * row) : make_uint4(0, 0, 0, 0);
      }
      // interior iteration: every token of it, with all K taps, inside the
      // chunk and one segment; then no per-token segment test (same sums)
      sg.advance(tb);
      const bool interior = tb + (U - 1) * d < t1 && tb - (K - 1) * d >= sg.lo && tb + (U - 1) * d < sg.hi;
      if (interior) {
#pragma unroll
        for (int m = 0; m < U; ++m) {
          float acc[V];
#pragma unroll
          for (int v = 0; v < V; ++v) acc[v] = b[v];
#pragma unroll
          for (int k = 0; k < K; ++k) {
            const int j = K - 1 - k;
            float xv[V];
            unpack<BF16>(m - j >= 0 ? cur[m - j] : prev[K + m - j], xv);
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = fmaf(wr[v][k], xv[v], acc[v]);
          }
          st_cs(yc + (tb + m * d) * row, pack<BF16>(acc));
        }
      } else {
#pragma unroll
        for (int m = 0; m < U; ++m) {
          const int64_t t = tb + m * d;
          if (t < t1) {
            sg.advance(t);
            const int64_t seg_lo = sg.first(t);
            float acc[V];
#pragma unroll
            for (int v = 0; v < V; ++v) acc[v] = b[v];
#pragma unroll
            for (int k = 0; k < K; ++k) {
              const int j = K - 1 - k;  // chain steps back
              if (t - j * d >= seg_lo) {  // before the segment: zero history
                float xv[V];
                unpack<BF16>(m - j >= 0 ? cur[m - j] : prev[K + m - j], xv);
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] = fmaf(wr[v][k], xv[v], acc[v]);
              }
            }
            st_cs(yc + t * row, pack<BF16>(acc));
          }
        }
      }
#pragma unroll
      for (int m = 0; m < K; ++m) prev[m] = cur[U - K + m];
    }
  }
}

// dx of the backward: dx[t] = sum_k w[k] * dy[t + d (K-1-k)] over the taps
// that stay inside t's segment, the forward's structure mirrored: residue
// chains of the chunk, 2K chain steps per iteration.  Each iteration loads
// the dy rows of the next one while it computes from the rows the iteration
// before loaded (and the first K-1 of its own loads), so a thread always has
// a full iteration of rows in flight.
template <bool BF16, int K>
__global__ void __launch_bounds__(kConvThreads, dx_min_blocks(K))
conv_dx_kernel(const unsigned char* __restrict__ dy, int64_t T, int64_t nvec, const int32_t* __restrict__ cu,
               int32_t num_seqs, const float* __restrict__ w, int dilation, unsigned char* __restrict__ dx,
               unsigned int* status) {
  constexpr int V = Vec<BF16>::n;
  constexpr int U = 2 * K;  // chain steps per iteration
  check_cu(cu, num_seqs, T, status);
  const int64_t cv = static_cast<int64_t>(blockIdx.y) * kConvThreads + threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kConvChunk;
  if (cv >= nvec || t0 >= T) return;
  const int64_t C = nvec * V, row = C * (BF16 ? 2 : 4);
  float wr[V][K];
#pragma unroll
  for (int v = 0; v < V; ++v)
#pragma unroll
    for (int k = 0; k < K; ++k) wr[v][k] = __ldg(w + (cv * V + v) * K + k);
  const int64_t t1 = min(T, t0 + kConvChunk), d = dilation;
  const unsigned char* gc = dy + cv * 16;
  unsigned char* dxc = dx + cv * 16;
  Segment sg{cu, num_seqs, 0, T, 0, 0};
  for (int64_t r = 0; r < d && t0 + r < t1; ++r) {
    sg.start(t0 + r);
    uint4 cur[U], nxt[U];  // dy of this iteration's steps and of the next U steps
#pragma unroll
    for (int m = 0; m < U; ++m) {
      const int64_t t = t0 + r + m * d;
      cur[m] = t < T ? ld_vec(gc + t * row) : make_uint4(0, 0, 0, 0);
    }
    for (int64_t tb = t0 + r; tb < t1; tb += U * d) {
#pragma unroll
      for (int m = 0; m < U; ++m) {  // K-1 of them are read now, all of them next iteration
        const int64_t t = tb + (U + m) * d;
        nxt[m] = t < T && tb + m * d < t1 ? ld_vec(gc + t * row) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int m = 0; m < U; ++m) {
        const int64_t t = tb + m * d;
        if (t < t1) {
          sg.advance(t);
          const int64_t seg_hi = sg.end(t);
          float acc[V];
#pragma unroll
          for (int v = 0; v < V; ++v) acc[v] = 0.f;
#pragma unroll
          for (int k = 0; k < K; ++k) {
            const int j = K - 1 - k;  // chain steps ahead
            if (t + j * d < seg_hi) {  // x[t] fed output t + j d through tap k
              float gv[V];
              unpack<BF16>(m + j < U ? cur[m + j] : nxt[m + j - U], gv);
#pragma unroll
              for (int v = 0; v < V; ++v) acc[v] = fmaf(wr[v][k], gv[v], acc[v]);
            }
          }
          st_cs(dxc + t * row, pack<BF16>(acc));
        }
      }
#pragma unroll
      for (int m = 0; m < U; ++m) cur[m] = nxt[m];
    }
  }
}

// dweight / dbias of the backward: this chunk's partial sums, written to
// part[chunk][K + 1][c] (tap k in row k, the bias in row K).  Residue chains again:
// output t read x at chain steps 0..K-1 back; per 2K chain steps a thread
// loads the 2K rows of dy and of x, the K-1 x rows before them come from the
// previous iteration.  The order of a chunk's sum: class by class modulo the
// dilation, each class in ascending tokens (a fixed function of the sizes).
template <bool BF16, int K>
__global__ void __launch_bounds__(kConvThreads, dw_min_blocks(K))
conv_dw_kernel(const unsigned char* __restrict__ dy, const unsigned char* __restrict__ x, int64_t T, int64_t nvec,
               const int32_t* __restrict__ cu, int32_t num_seqs, int dilation, int64_t chunk,
               float* __restrict__ part, unsigned int* status) {
  constexpr int V = Vec<BF16>::n;
  constexpr int U = 2 * K;
  check_cu(cu, num_seqs, T, status);
  const int64_t cv = static_cast<int64_t>(blockIdx.y) * kConvThreads + threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * chunk;
  if (cv >= nvec) return;
  const int64_t C = nvec * V, row = C * (BF16 ? 2 : 4);
  float gw[V][K], gb[V];
#pragma unroll
  for (int v = 0; v < V; ++v) {
    gb[v] = 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) gw[v][k] = 0.f;
  }
  const int64_t t1 = min(T, t0 + chunk), d = dilation;
  const unsigned char* xc = x + cv * 16;
  const unsigned char* gc = dy + cv * 16;
  Segment sg{cu, num_seqs, 0, T, 0, 0};
  for (int64_t r = 0; r < d && t0 + r < t1; ++r) {
    sg.start(t0 + r);
    uint4 xp[K], xn[U], gn[U];  // x: the K steps before / this iteration's steps; dy: this iteration's steps
#pragma unroll
    for (int j = 1; j < K; ++j) {
      const int64_t t = t0 + r - static_cast<int64_t>(K - j) * d;
      xp[j] = t >= 0 ? ld_vec(xc + t * row) : make_uint4(0, 0, 0, 0);
    }
    for (int64_t tb = t0 + r; tb < t1; tb += U * d) {
#pragma unroll
      for (int m = 0; m < U; ++m) {
        const int64_t t = tb + m * d;
        xn[m] = t < t1 ? ld_vec(xc + t * row) : make_uint4(0, 0, 0, 0);
        gn[m] = t < t1 ? ld_vec(gc + t * row) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int m = 0; m < U; ++m) {
        const int64_t t = tb + m * d;
        if (t < t1) {
          sg.advance(t);
          const int64_t seg_lo = sg.first(t);
          float g[V];
          unpack<BF16>(gn[m], g);
#pragma unroll
          for (int v = 0; v < V; ++v) gb[v] += g[v];
#pragma unroll
          for (int k = 0; k < K; ++k) {
            const int j = K - 1 - k;  // chain steps back
            if (t - j * d >= seg_lo) {  // output t read x[t - j d] through tap k
              float xv[V];
              unpack<BF16>(m - j >= 0 ? xn[m - j] : xp[K + m - j], xv);
#pragma unroll
              for (int v = 0; v < V; ++v) gw[v][k] = fmaf(g[v], xv[v], gw[v][k]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < K; ++m) xp[m] = xn[U - K + m];
    }
  }
  float* pc = part + static_cast<int64_t>(blockIdx.x) * C * (K + 1) + cv * V;
#pragma unroll
  for (int k = 0; k <= K; ++k) {  // V consecutive floats per row: coalesced across the warp
#pragma unroll
    for (int v = 0; v < V; v += 4)
      *reinterpret_cast<float4*>(pc + k * C + v) =
          k < K ? make_float4(gw[v][k], gw[v + 1][k], gw[v + 2][k], gw[v + 3][k])
                : make_float4(gb[v], gb[v + 1], gb[v + 2], gb[v + 3]);
  }
}

// The whole backward in one sweep (dx and this chunk's dweight / dbias
// partials), dy and x each read once.  A thread holds four channels (half a
// 16-byte bf16 vector, so that the rows of both tensors, both rings and the
// weight-gradient accumulators fit the register budget of four blocks per
// SM).  Along a residue chain, K steps per iteration: x at steps -(K-1) ..
// K-1 and dy at steps 0 .. 2K-2 of the iteration, and the next iteration's
// rows already in flight.  dx and the partial sums
// come out bit-identical to conv_dx_kernel and conv_dw_kernel (same
// per-output tap order, same per-chunk token order).
template <bool BF16, int K>
__global__ void __launch_bounds__(kConvThreads, bwd_min_blocks(K, BF16))
conv_backward_kernel(const unsigned char* __restrict__ dy, const unsigned char* __restrict__ x, int64_t T,
                     int64_t nquad, const int32_t* __restrict__ cu, int32_t num_seqs, const float* __restrict__ w,
                     int dilation, int64_t chunk, unsigned char* __restrict__ dx, float* __restrict__ part,
                     unsigned int* status) {
  using Q = typename Quad<BF16>::type;
  constexpr int U = K, L = K - 1, LS = L > 0 ? L : 1;
  check_cu(cu, num_seqs, T, status);
  const int64_t cq = static_cast<int64_t>(blockIdx.y) * kConvThreads + threadIdx.x;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * chunk;
  if (cq >= nquad) return;
  const int64_t C = nquad * 4, row = C * (BF16 ? 2 : 4);
  float wr[4][K], gw[4][K], gb[4];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    gb[v] = 0.f;
#pragma unroll
    for (int k = 0; k < K; ++k) {
      wr[v][k] = __ldg(w + (cq * 4 + v) * K + k);
      gw[v][k] = 0.f;
    }
  }
  const int64_t t1 = min(T, t0 + chunk), d = dilation;
  const unsigned char* xc = x + cq * Quad<BF16>::bytes;
  const unsigned char* gc = dy + cq * Quad<BF16>::bytes;
  unsigned char* dxc = dx + cq * Quad<BF16>::bytes;
  Segment sg{cu, num_seqs, 0, T, 0, 0};
  for (int64_t r = 0; r < d && t0 + r < t1; ++r) {
    sg.start(t0 + r);
    ChainTaps<K> ct;
    // x at steps -L .. -1 (xp) and 0 .. U-1 (xn); dy at steps 0 .. L-1 (ga) and L .. L+U-1 (gn)
    Q xp[LS], ga[LS], xn[U], gn[U];
#pragma unroll
    for (int i = 0; i < L; ++i) {
      const int64_t tx = t0 + r - static_cast<int64_t>(L - i) * d, tg = t0 + r + i * d;
      xp[i] = tx >= 0 ? ld_quad<BF16>(xc + tx * row) : zero_quad<BF16>();
      ga[i] = tg < T ? ld_quad<BF16>(gc + tg * row) : zero_quad<BF16>();
    }
#pragma unroll
    for (int m = 0; m < U; ++m) {
      const int64_t t = t0 + r + m * d, tg = t0 + r + (L + m) * d;
      xn[m] = t < t1 ? ld_quad<BF16>(xc + t * row) : zero_quad<BF16>();
      gn[m] = tg < T && t < t1 ? ld_quad<BF16>(gc + tg * row) : zero_quad<BF16>();
    }
    for (int64_t tb = t0 + r; tb < t1; tb += U * d) {
      Q xq[U], gq[U];  // the next iteration's rows, in flight during this one's arithmetic
#pragma unroll
      for (int m = 0; m < U; ++m) {
        const int64_t t = tb + (U + m) * d, tg = tb + (U + L + m) * d;
        xq[m] = t < t1 ? ld_quad<BF16>(xc + t * row) : zero_quad<BF16>();
        gq[m] = tg < T && t < t1 ? ld_quad<BF16>(gc + tg * row) : zero_quad<BF16>();
      }
      // interior iteration: its K tokens inside the chunk, and every one with
      // all K taps behind and ahead inside the segment of the previous chain
      // step; then no per-token segment bookkeeping or tap tests (same sums)
      const bool interior = tb + (U - 1) * d < t1 && tb - static_cast<int64_t>(L) * d >= ct.lo &&
                            tb - d >= ct.lo && tb + static_cast<int64_t>(U - 1 + L) * d < ct.hi;
      if (interior) {
#pragma unroll
        for (int m = 0; m < U; ++m) {
          float g[4];
          unpack4<BF16>(m < L ? ga[m] : gn[m - L], g);
#pragma unroll
          for (int v = 0; v < 4; ++v) gb[v] += g[v];
#pragma unroll
          for (int k = 0; k < K; ++k) {
            const int j = K - 1 - k;
            float xv[4];
            unpack4<BF16>(m - j >= 0 ? xn[m - j] : xp[L + m - j], xv);
#pragma unroll
            for (int v = 0; v < 4; ++v) gw[v][k] = fmaf(g[v], xv[v], gw[v][k]);
          }
          if (dx != nullptr) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < K; ++k) {
              const int j = K - 1 - k;
              float gv[4];
              unpack4<BF16>(m + j < L ? ga[m + j] : gn[m + j - L], gv);
#pragma unroll
              for (int v = 0; v < 4; ++v) acc[v] = fmaf(wr[v][k], gv[v], acc[v]);
            }
            st_quad<BF16>(dxc + (tb + m * d) * row, acc);
          }
        }
        ct.skip(U);
      } else {
#pragma unroll
        for (int m = 0; m < U; ++m) {
          const int64_t t = tb + m * d;
          if (t < t1) {
            ct.step(sg, t, d);
            float g[4];
            unpack4<BF16>(m < L ? ga[m] : gn[m - L], g);
#pragma unroll
            for (int v = 0; v < 4; ++v) gb[v] += g[v];
#pragma unroll
            for (int k = 0; k < K; ++k) {
              const int j = K - 1 - k;
              if (j <= ct.back) {  // output t read x[t - j d] through tap k
                float xv[4];
                unpack4<BF16>(m - j >= 0 ? xn[m - j] : xp[L + m - j], xv);
#pragma unroll
                for (int v = 0; v < 4; ++v) gw[v][k] = fmaf(g[v], xv[v], gw[v][k]);
              }
            }
            if (dx != nullptr) {
              float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int k = 0; k < K; ++k) {
                const int j = K - 1 - k;
                if (j <= ct.ahead) {  // x[t] fed output t + j d through tap k
                  float gv[4];
                  unpack4<BF16>(m + j < L ? ga[m + j] : gn[m + j - L], gv);
#pragma unroll
                  for (int v = 0; v < 4; ++v) acc[v] = fmaf(wr[v][k], gv[v], acc[v]);
                }
              }
              st_quad<BF16>(dxc + t * row, acc);
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < L; ++i) {
        xp[i] = xn[U - L + i];
        ga[i] = gn[U - L + i];
      }
#pragma unroll
      for (int m = 0; m < U; ++m) {
        xn[m] = xq[m];
        gn[m] = gq[m];
      }
    }
  }
  float* pc = part + static_cast<int64_t>(blockIdx.x) * C * (K + 1) + cq * 4;
#pragma unroll
  for (int k = 0; k <= K; ++k)
    *reinterpret_cast<float4*>(pc + k * C) =
        k < K ? make_float4(gw[0][k], gw[1][k], gw[2][k], gw[3][k]) : make_float4(gb[0], gb[1], gb[2], gb[3]);
}

// dw[c, k] += sum over chunks (in chunk order) of the partials; db likewise.
__global__ void conv_reduce_kernel(const float* __restrict__ part, int64_t nchunks, int64_t C, int K,
                                   float* __restrict__ dw, float* __restrict__ db) {
  const int64_t n = C * (K + 1);
  const int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= n) return;
  wait_for_prior_grid();
  float sum = part[e];
  int64_t q = 1;
  for (; q < nchunks; q += 32) {  // up to 32 loads in flight, added in order
    float v[32];
#pragma unroll
    for (int u = 0; u < 32; ++u) v[u] = q + u < nchunks ? __ldcs(part + (q + u) * n + e) : 0.f;
#pragma unroll
    for (int u = 0; u < 32; ++u)
      if (q + u < nchunks) sum += v[u];
  }
  const int k = static_cast<int>(e / C);  // part[q] is [K + 1][C]
  const int64_t c = e - k * C;
  if (k < K) {
    if (dw != nullptr) dw[c * K + k] += sum;
  } else if (db != nullptr) {
    db[c] += sum;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ple_status_t check_conv_args(const void* x, ple_dtype_t dtype, int64_t T, int64_t C, const int32_t* cu,
                             int32_t S, const float* w, int32_t K, int32_t dilation) {
  if (T < 0 || C < 1 || K < 1 || dilation < 1) return PLE_ERR_INVALID_ARG;
  if (dtype != PLE_F32 && dtype != PLE_BF16) return PLE_ERR_INVALID_ARG;
  if (K > kMaxTaps) return PLE_ERR_UNSUPPORTED;
  if (T == 0) return PLE_OK;
  if (x == nullptr || cu == nullptr || w == nullptr || S < 1) return PLE_ERR_INVALID_ARG;
  if (T > (int64_t{1} << 40) || C > (int64_t{1} << 24)) return PLE_ERR_UNSUPPORTED;
  if ((C * (dtype == PLE_F32 ? 4 : 2)) % 16 != 0 || !aligned16(x)) return PLE_ERR_ALIGNMENT;
  if ((reinterpret_cast<uintptr_t>(cu) & 3u) != 0 || (reinterpret_cast<uintptr_t>(w) & 3u) != 0)
    return PLE_ERR_ALIGNMENT;
  return PLE_OK;
}

// Tokens per backward block: 2 * kConvBwdChunk when the blocks of that
// chunk still fill kConvBwdWave slots (a longer chunk loads fewer history
// and lookahead rows per token), else kConvBwdChunk; and few enough blocks
// along the tokens that at most kMaxPartials partial sums are kept.  A
// function of the sizes only (not of the device), so that the summation
// order and the workspace size are too.  Measured on the B200 at 32768
// tokens: 8192 channels 345.1 -> 330.7 us with 512-token chunks, 2048
// channels 109.6 -> 126.0 us (too few blocks), hence the rule.
constexpr int64_t kConvBwdWave = 4 * 148;  // four blocks on each of the B200's SMs
int64_t conv_chunk_bwd(int64_t T, int64_t C) {
  const int64_t need = (T + kMaxPartials - 1) / kMaxPartials;
  const int64_t quad_blocks = (C / 4 + kConvThreads - 1) / kConvThreads;
  const int64_t longer = 2 * kConvBwdChunk;
  const int64_t chunk = (T + longer - 1) / longer * quad_blocks >= kConvBwdWave ? longer : kConvBwdChunk;
  return need > chunk ? need : chunk;
}
int64_t conv_chunks_bwd(int64_t T, int64_t C) {
  const int64_t c = conv_chunk_bwd(T, C);
  return (T + c - 1) / c;
}

}  // namespace
}  // namespace ple

using namespace ple;

extern "C" {

ple_status_t ple_conv_forward(const void* x, ple_dtype_t dtype, int64_t T, int64_t C, const int32_t* cu_seqlens,
                              int32_t num_seqs, const float* weight, int32_t K, int32_t dilation, const float* bias,
                              void* y, void* stream) {
  ple_status_t st = check_conv_args(x, dtype, T, C, cu_seqlens, num_seqs, weight, K, dilation);
  if (st != PLE_OK || T == 0) return st;
  if (y == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned16(y) || (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 3u) != 0)) return PLE_ERR_ALIGNMENT;
  cudaError_t e;
  unsigned int* status = status_word(nullptr, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  const bool bf = dtype == PLE_BF16;
  const int64_t nvec = C / (bf ? 8 : 4);
  // grid.x: token chunks (T <= 2^40 keeps them < 2^31); grid.y: channel blocks (C <= 2^24 keeps them <= 32768)
  const dim3 grid(static_cast<unsigned>((T + kConvChunk - 1) / kConvChunk),
                  static_cast<unsigned>((nvec + kConvThreads - 1) / kConvThreads));
  const auto s = static_cast<cudaStream_t>(stream);
  const auto* xb = static_cast<const unsigned char*>(x);
  auto* yb = static_cast<unsigned char*>(y);
#define PLE_CONV_FWD(KK)                                                                                    \
  case KK:                                                                                                  \
    if (bf)                                                                                                 \
      conv_forward_kernel<true, KK><<<grid, kConvThreads, 0, s>>>(xb, T, nvec, cu_seqlens, num_seqs, weight, \
                                                                   dilation, bias, yb, status);             \
    else                                                                                                    \
      conv_forward_kernel<false, KK><<<grid, kConvThreads, 0, s>>>(xb, T, nvec, cu_seqlens, num_seqs, weight, \
                                                                    dilation, bias, yb, status);            \
    break;
  switch (K) {
    PLE_CONV_FWD(1) PLE_CONV_FWD(2) PLE_CONV_FWD(3) PLE_CONV_FWD(4)
    PLE_CONV_FWD(5) PLE_CONV_FWD(6) PLE_CONV_FWD(7) PLE_CONV_FWD(8)
    default: return PLE_ERR_UNSUPPORTED;
  }
#undef PLE_CONV_FWD
  return check_launch();
}

size_t ple_conv_backward_workspace_bytes(int64_t T, int64_t C, int32_t K) {
  if (T <= 0 || C < 1 || K < 1 || K > kMaxTaps) return 0;
  return static_cast<size_t>(conv_chunks_bwd(T, C)) * static_cast<size_t>(C) * static_cast<size_t>(K + 1) *
         sizeof(float);
}

ple_status_t ple_conv_backward(const void* dy, const void* x, ple_dtype_t dtype, int64_t T, int64_t C,
                               const int32_t* cu_seqlens, int32_t num_seqs, const float* weight, int32_t K,
                               int32_t dilation, void* dx, float* dweight, float* dbias, void* workspace,
                               size_t workspace_bytes, void* stream) {
  ple_status_t st = check_conv_args(x, dtype, T, C, cu_seqlens, num_seqs, weight, K, dilation);
  if (st != PLE_OK || T == 0) return st;
  if (dy == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned16(dy) || (dx != nullptr && !aligned16(dx))) return PLE_ERR_ALIGNMENT;
  const bool want_params = dweight != nullptr || dbias != nullptr;
  if (want_params) {
    if (workspace == nullptr || workspace_bytes < ple_conv_backward_workspace_bytes(T, C, K))
      return PLE_ERR_WORKSPACE;
    if (!aligned16(workspace)) return PLE_ERR_ALIGNMENT;
  } else if (dx == nullptr) {
    return PLE_OK;  // nothing asked for
  }
  cudaError_t e;
  unsigned int* status = status_word(nullptr, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  const bool bf = dtype == PLE_BF16;
  const int64_t nvec = C / (bf ? 8 : 4);
  const int64_t chunk = conv_chunk_bwd(T, C), nchunks = conv_chunks_bwd(T, C);
  const unsigned vblocks = static_cast<unsigned>((nvec + kConvThreads - 1) / kConvThreads);
  const auto s = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(workspace);
  const auto* g = static_cast<const unsigned char*>(dy);
  const auto* xb = static_cast<const unsigned char*>(x);
  auto* dxb = static_cast<unsigned char*>(dx);
  const dim3 dx_grid(static_cast<unsigned>((T + kConvChunk - 1) / kConvChunk), vblocks);
  const dim3 dw_grid(static_cast<unsigned>(nchunks), vblocks);
  const int64_t nquad = C / 4;
  const dim3 fused_grid(static_cast<unsigned>(nchunks),
                        static_cast<unsigned>((nquad + kConvThreads - 1) / kConvThreads));
#define PLE_CONV_BWD(KK)                                                                                          \
  case KK:                                                                                                        \
    if (dx != nullptr && want_params) {                                                                           \
      if (bf)                                                                                                     \
        conv_backward_kernel<true, KK><<<fused_grid, kConvThreads, 0, s>>>(g, xb, T, nquad, cu_seqlens, num_seqs, \
                                                                           weight, dilation, chunk, dxb, part,    \
                                                                           status);                               \
      else                                                                                                        \
        conv_backward_kernel<false, KK><<<fused_grid, kConvThreads, 0, s>>>(g, xb, T, nquad, cu_seqlens,          \
                                                                            num_seqs, weight, dilation, chunk,    \
                                                                            dxb, part, status);                   \
    } else if (dx != nullptr) {                                                                                   \
      if (bf)                                                                                                     \
        conv_dx_kernel<true, KK><<<dx_grid, kConvThreads, 0, s>>>(g, T, nvec, cu_seqlens, num_seqs, weight,       \
                                                                  dilation, dxb, status);                         \
      else                                                                                                        \
        conv_dx_kernel<false, KK><<<dx_grid, kConvThreads, 0, s>>>(g, T, nvec, cu_seqlens, num_seqs, weight,      \
                                                                   dilation, dxb, status);                        \
    } else {                                                                                                      \
      if (bf)                                                                                                     \
        conv_dw_kernel<true, KK><<<dw_grid, kConvThreads, 0, s>>>(g, xb, T, nvec, cu_seqlens, num_seqs, dilation, \
                                                                  chunk, part, status);                           \
      else                                                                                                        \
        conv_dw_kernel<false, KK><<<dw_grid, kConvThreads, 0, s>>>(g, xb, T, nvec, cu_seqlens, num_seqs,          \
                                                                   dilation, chunk, part, status);                \
    }                                                                                                             \
    break;
  switch (K) {
    PLE_CONV_BWD(1) PLE_CONV_BWD(2) PLE_CONV_BWD(3) PLE_CONV_BWD(4)
    PLE_CONV_BWD(5) PLE_CONV_BWD(6) PLE_CONV_BWD(7) PLE_CONV_BWD(8)
    default: return PLE_ERR_UNSUPPORTED;
  }
#undef PLE_CONV_BWD
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  if (want_params) {
    const int64_t n = C * (K + 1);
    e = launch_after(conv_reduce_kernel, dim3(static_cast<unsigned>((n + 63) / 64)), dim3(64), 0, s,
                     static_cast<const float*>(part), nchunks, C, static_cast<int>(K), dweight, dbias);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return check_launch();
}

}  // extern "C"
