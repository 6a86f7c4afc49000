// Backward path: the table gradient of the row gather.  The embedding table
// of Qwen3_8_FlashNextOwnerShardedEmbedding (NeMo AutoModel engram API
// page) is an ordinary parameter, so the rows' gradients are the sums of
// grad_out over the hits of each row.  The page fixes no summation order;
// this file implements a fixed one, so the result is bit-identical run to
// run:
//   hits of row r in ascending flat index i = t*H + j, cut into chunks of 32
//   consecutive hits; each chunk summed left to right from its first element
//   (fp32); the chunk sums summed left to right from the first; the row sum
//   added once into table_grad[r].
//
// Pipeline (all in the caller's workspace, no allocation, no inter-block
// waiting):
//   1. keys_kernel: 32-bit keys from the int64 rows (bad rows -> key R),
//      per-tile histogram of the first digit;
//   2. LSD radix sort, 8-bit digits, stable (reduce-then-scan per pass:
//      histogram, one-block exclusive scan, rank-and-scatter), values = i;
//   3. fold_kernel: one warp per 32 sorted positions ("window"); finds the
//      chunk starts in its window (a chunk start is a position whose offset
//      from its run's first position is a multiple of 32), folds each chunk
//      it starts, and either adds a whole single-chunk run into table_grad
//      or stores the chunk sum in a slot of the workspace;
//   4. fold_heavy_kernel: one warp per run longer than 32 folds its chunk
//      sums in order and adds the result into table_grad.
// The final add is a vector fp32 reduction (red.global.add) issued by the one
// warp that owns the row, so it is the single add table_grad + S_r.
#include "common.cuh"

namespace ple {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortThreads * kSortItems;  // keys per sort tile
constexpr int kRadix = 256;
constexpr int kWarpsPerSortBlock = kSortThreads / 32;
constexpr int kChunk = 32;
constexpr uint32_t kNoKey = 0xffffffffu;  // past the end; never a real key
constexpr int kScanThreads = 1024;
constexpr int kFoldThreads = 256;
constexpr int kFoldBatch = 8;             // grad rows loaded ahead in the fold

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---------------------------------------------------------------------------
// radix sort
// ---------------------------------------------------------------------------

// Warp-aggregated shared-memory histogram update for one key per lane.
__device__ __forceinline__ void hist_add(uint32_t* h, bool valid, uint32_t digit) {
  const unsigned peers = __match_any_sync(kFull, valid ? digit : 0x100u);
  if (valid && (peers & lanemask_lt()) == 0) atomicAdd(&h[digit], __popc(peers));
}

__global__ void __launch_bounds__(kSortThreads)
keys_kernel(const int64_t* __restrict__ rows, int64_t N, int64_t num_rows, uint32_t* __restrict__ keys,
            uint32_t* __restrict__ hist, int num_tiles, int* __restrict__ mc_count, unsigned int* status) {
  __shared__ uint32_t h[kRadix];
  h[threadIdx.x] = 0;
  if (blockIdx.x == 0 && threadIdx.x == 0) *mc_count = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSortTile;
  bool bad = false;
#pragma unroll 4
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * kSortThreads + threadIdx.x;
    const bool valid = i < N;
    uint32_t key = 0;
    if (valid) {
      const int64_t v = rows[i];
      const bool ok = v >= 0 && v < num_rows;
      bad |= !ok;
      key = ok ? static_cast<uint32_t>(v) : static_cast<uint32_t>(num_rows);
      keys[i] = key;
    }
    hist_add(h, valid, key & (kRadix - 1));
  }
  if (bad) raise_flag(status, PLE_ERR_BAD_ROW);
  __syncthreads();
  hist[threadIdx.x * num_tiles + blockIdx.x] = h[threadIdx.x];
}

__global__ void __launch_bounds__(kSortThreads)
hist_kernel(const uint32_t* __restrict__ keys, int64_t N, int shift, uint32_t* __restrict__ hist,
            int num_tiles) {
  __shared__ uint32_t h[kRadix];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSortTile;
#pragma unroll 4
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * kSortThreads + threadIdx.x;
    const bool valid = i < N;
    const uint32_t key = valid ? keys[i] : 0;
    hist_add(h, valid, (key >> shift) & (kRadix - 1));
  }
  __syncthreads();
  hist[threadIdx.x * num_tiles + blockIdx.x] = h[threadIdx.x];
}

// Exclusive scan, in place, of M counters laid out digit-major
// ([digit][tile]), by one block: each thread owns a contiguous run.
__global__ void __launch_bounds__(kScanThreads) scan_kernel(uint32_t* __restrict__ a, int M) {
  __shared__ uint32_t warp_tot[kScanThreads / 32];
  const int per = (M + kScanThreads - 1) / kScanThreads;
  const int beg = min(M, threadIdx.x * per), end = min(M, beg + per);
  uint32_t s = 0;
  for (int i = beg; i < end; ++i) s += a[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = s;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_tot[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t y = __shfl_up_sync(kFull, w, d);
      if (lane >= d) w += y;
    }
    warp_tot[lane] = w;  // inclusive
  }
  __syncthreads();
  uint32_t run = incl - s + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int i = beg; i < end; ++i) {
    const uint32_t v = a[i];
    a[i] = run;
    run += v;
  }
}

// Stable rank-and-scatter of one 4096-key tile.  Keys are held striped
// (item r of thread x is tile position r*256 + x), so the order
// (r, warp, lane) is the tile order.  Per (item round, warp, digit) counts
// go to shared memory; one pass per digit turns them into exclusive
// offsets; the destination is the tile's scanned global digit offset plus
// that offset plus the rank among equal digits inside the warp.
constexpr size_t kScatterSmem =
    sizeof(uint16_t) * kSortItems * kWarpsPerSortBlock * kRadix + sizeof(uint32_t) * kRadix;

template <bool kIdentityVals>
__global__ void __launch_bounds__(kSortThreads)
scatter_kernel(const uint32_t* __restrict__ kin, const uint32_t* __restrict__ vin, uint32_t* __restrict__ kout,
               uint32_t* __restrict__ vout, const uint32_t* __restrict__ offs, int64_t N, int shift,
               int num_tiles) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t* cnt = reinterpret_cast<uint16_t*>(smem);  // [items][warps][radix]
  uint32_t* tile_base = reinterpret_cast<uint32_t*>(cnt + kSortItems * kWarpsPerSortBlock * kRadix);
  const int warp = threadIdx.x >> 5;
  {
    uint32_t* c32 = reinterpret_cast<uint32_t*>(cnt);
    constexpr int words = kSortItems * kWarpsPerSortBlock * kRadix / 2;
#pragma unroll 4
    for (int k = threadIdx.x; k < words; k += kSortThreads) c32[k] = 0;
  }
  tile_base[threadIdx.x] = offs[threadIdx.x * num_tiles + blockIdx.x];
  const int64_t base = static_cast<int64_t>(blockIdx.x) * kSortTile;
  uint32_t key[kSortItems], val[kSortItems];
  uint8_t rank[kSortItems];
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * kSortThreads + threadIdx.x;
    key[r] = i < N ? kin[i] : kNoKey;
    val[r] = i < N ? (kIdentityVals ? static_cast<uint32_t>(i) : vin[i]) : 0;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * kSortThreads + threadIdx.x;
    const bool valid = i < N;
    const uint32_t digit = (key[r] >> shift) & (kRadix - 1);
    const unsigned peers = __match_any_sync(kFull, valid ? digit : 0x100u);
    const unsigned lower = __popc(peers & lanemask_lt());
    rank[r] = static_cast<uint8_t>(lower);
    if (valid && lower == 0) cnt[(r * kWarpsPerSortBlock + warp) * kRadix + digit] = __popc(peers);
  }
  __syncthreads();
  {
    const int d = threadIdx.x;
    uint32_t run = 0;
    for (int rw = 0; rw < kSortItems * kWarpsPerSortBlock; ++rw) {
      const uint32_t c = cnt[rw * kRadix + d];
      cnt[rw * kRadix + d] = static_cast<uint16_t>(run);
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = base + r * kSortThreads + threadIdx.x;
    if (i < N) {
      const uint32_t digit = (key[r] >> shift) & (kRadix - 1);
      const uint32_t dst =
          tile_base[digit] + cnt[(r * kWarpsPerSortBlock + warp) * kRadix + digit] + rank[r];
      if (dst < N) {  // always true when the counts are consistent
        kout[dst] = key[r];
        vout[dst] = val[r];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// gradient columns: lane l owns columns [l*CPL, (l+1)*CPL) when D = 32*CPL
// (CPL > 0); for other D <= 256 (CPL = 0) lane l owns columns l, l+32, ...
// ---------------------------------------------------------------------------
constexpr int kMaxColsPerLane = 8;

template <int CPL>
struct Cols {
  static constexpr int n = CPL > 0 ? CPL : kMaxColsPerLane;
  float v[n];
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <int CPL, bool BF16>
__device__ __forceinline__ void load_cols(const void* __restrict__ base, int64_t row, int D, Cols<CPL>& x) {
  const int lane = threadIdx.x & 31;
  if constexpr (CPL == 0) {
#pragma unroll
    for (int k = 0; k < kMaxColsPerLane; ++k) {
      const int d = lane + 32 * k;
      float f = 0.f;
      if (d < D) {
        const int64_t e = row * D + d;
        f = BF16 ? __uint_as_float(static_cast<uint32_t>(__ldg(static_cast<const uint16_t*>(base) + e)) << 16)
                 : __ldg(static_cast<const float*>(base) + e);
      }
      x.v[k] = f;
    }
  } else if constexpr (BF16) {
    const uint16_t* p = static_cast<const uint16_t*>(base) + row * D + lane * CPL;
    if constexpr (CPL == 1) {
      x.v[0] = __uint_as_float(static_cast<uint32_t>(__ldg(p)) << 16);
    } else if constexpr (CPL == 2) {
      const uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p));
      x.v[0] = bf16_lo(w);
      x.v[1] = bf16_hi(w);
    } else if constexpr (CPL == 4) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
      x.v[0] = bf16_lo(w.x); x.v[1] = bf16_hi(w.x); x.v[2] = bf16_lo(w.y); x.v[3] = bf16_hi(w.y);
    } else {
      static_assert(CPL == 8, "CPL");
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
      x.v[0] = bf16_lo(w.x); x.v[1] = bf16_hi(w.x); x.v[2] = bf16_lo(w.y); x.v[3] = bf16_hi(w.y);
      x.v[4] = bf16_lo(w.z); x.v[5] = bf16_hi(w.z); x.v[6] = bf16_lo(w.w); x.v[7] = bf16_hi(w.w);
    }
  } else {
    const float* p = static_cast<const float*>(base) + row * D + lane * CPL;
    if constexpr (CPL == 1) {
      x.v[0] = __ldg(p);
    } else if constexpr (CPL == 2) {
      const float2 w = __ldg(reinterpret_cast<const float2*>(p));
      x.v[0] = w.x; x.v[1] = w.y;
    } else {
#pragma unroll
      for (int k = 0; k < CPL; k += 4) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(p + k));
        x.v[k] = w.x; x.v[k + 1] = w.y; x.v[k + 2] = w.z; x.v[k + 3] = w.w;
      }
    }
  }
}

// fp32 chunk-sum slots in the workspace (plain loads / stores).
template <int CPL>
__device__ __forceinline__ void store_slot(float* __restrict__ base, int64_t slot, int D, const Cols<CPL>& x) {
  const int lane = threadIdx.x & 31;
  if constexpr (CPL == 0) {
#pragma unroll
    for (int k = 0; k < kMaxColsPerLane; ++k)
      if (lane + 32 * k < D) base[slot * D + lane + 32 * k] = x.v[k];
  } else {
    float* p = base + slot * D + lane * CPL;
#pragma unroll
    for (int k = 0; k < CPL; ++k) p[k] = x.v[k];
  }
}

// One fp32 reduction per column into table_grad (the single final add).
template <int CPL>
__device__ __forceinline__ void red_add_row(float* __restrict__ tg, int64_t row, int D, const Cols<CPL>& x) {
  const int lane = threadIdx.x & 31;
  if constexpr (CPL == 0) {
#pragma unroll
    for (int k = 0; k < kMaxColsPerLane; ++k)
      if (lane + 32 * k < D) atomicAdd(tg + row * D + lane + 32 * k, x.v[k]);
  } else {
    float* p = tg + row * D + lane * CPL;
    if constexpr (CPL == 1) {
      asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(x.v[0]) : "memory");
    } else if constexpr (CPL == 2) {
      asm volatile("red.global.add.v2.f32 [%0], {%1,%2};" ::"l"(p), "f"(x.v[0]), "f"(x.v[1]) : "memory");
    } else {
#pragma unroll
      for (int k = 0; k < CPL; k += 4)
        asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p + k), "f"(x.v[k]), "f"(x.v[k + 1]),
                     "f"(x.v[k + 2]), "f"(x.v[k + 3])
                     : "memory");
    }
  }
}

// First position of the run of sorted keys that holds position p (known
// not to be a run start): the warp probes p - 32*2^l, l = 0..31, then
// narrows the bracket 32 ways per step.  Keys before the run are smaller,
// so "key != run key" is a prefix property of positions.
__device__ int64_t find_run_start(const uint32_t* __restrict__ K, int64_t p, uint32_t key) {
  const int lane = threadIdx.x & 31;
  const int64_t probe = p - (static_cast<int64_t>(32) << lane);
  const bool before = probe < 0 || K[probe] != key;
  const unsigned bm = __ballot_sync(kFull, before);
  // lo: a position known to be before the run (or -1); hi: known inside.
  const int l = __ffs(bm) - 1;  // bm != 0: lane 31 probes below 0 for any p < 2^36
  int64_t lo = max(static_cast<int64_t>(-1), p - (static_cast<int64_t>(32) << l));
  int64_t hi = l == 0 ? p : p - (static_cast<int64_t>(32) << (l - 1));
  while (hi - lo > 1) {
    // probes q_j = lo + step*(j+1); those below hi are "in range"
    const int64_t step = (hi - lo + 31) / 32;
    const int64_t q = lo + step * (lane + 1);
    const bool in_range = q < hi;
    const int nb = __popc(__ballot_sync(kFull, in_range && K[q] != key));  // before-run probes: a prefix
    const int nr = __popc(__ballot_sync(kFull, in_range));
    const int64_t lo_next = lo + step * nb;
    if (nb < nr) hi = lo + step * (nb + 1);  // first in-range probe inside the run
    lo = lo_next;
  }
  return hi;
}

// Level 1: one warp per window of 32 sorted positions.
template <int CPL, bool BF16>
__global__ void __launch_bounds__(kFoldThreads)
fold_kernel(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I, int64_t N, uint32_t bad_key,
            const void* __restrict__ grad, int D, float* __restrict__ table_grad, float* __restrict__ csum,
            int* __restrict__ mc_len, int* __restrict__ mc_list, int* __restrict__ mc_count) {
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x) >> 5;
  const int64_t p0 = w * 32;
  if (p0 >= N) return;
  const int64_t pa = p0 + lane, pb = p0 + 32 + lane;
  const uint32_t kA = pa < N ? K[pa] : kNoKey;
  const uint32_t kB = pb < N ? K[pb] : kNoKey;
  const uint32_t iA = pa < N ? I[pa] : 0;
  const uint32_t iB = pb < N ? I[pb] : 0;
  const uint32_t k_before = p0 > 0 ? K[p0 - 1] : kNoKey;
  uint32_t prevA = __shfl_up_sync(kFull, kA, 1);
  uint32_t prevB = __shfl_up_sync(kFull, kB, 1);
  const uint32_t kA31 = __shfl_sync(kFull, kA, 31);
  if (lane == 0) {
    prevA = k_before;
    prevB = kA31;
  }
  const bool headA = pa < N && kA != prevA;
  const bool headB = pb < N && kB != prevB;
  const uint64_t hm = static_cast<uint64_t>(__ballot_sync(kFull, headA)) |
                      (static_cast<uint64_t>(__ballot_sync(kFull, headB)) << 32);
  const uint32_t key0 = __shfl_sync(kFull, kA, 0);
  const int64_t s0 = (hm & 1ull) ? p0 : find_run_start(K, p0, key0);

  auto run_start = [&](int idx) -> int64_t {  // first position of the run holding p0 + idx
    const uint64_t le = hm & (idx >= 63 ? ~0ull : ((2ull << idx) - 1));
    return le ? p0 + (63 - __clzll(le)) : s0;
  };
  const bool csA = pa < N && ((pa - run_start(lane)) & (kChunk - 1)) == 0;
  const bool csB = pb < N && ((pb - run_start(32 + lane)) & (kChunk - 1)) == 0;
  const uint64_t cm = static_cast<uint64_t>(__ballot_sync(kFull, csA)) |
                      (static_cast<uint64_t>(__ballot_sync(kFull, csB)) << 32);
  // A window may hold no chunk start only at the tail, when its positions
  // finish a chunk that started in the previous window (folded there).
  if ((cm & 0xffffffffull) == 0) return;
  const int a = __ffsll(static_cast<long long>(cm & 0xffffffffull)) - 1;
  const uint32_t hiw = static_cast<uint32_t>(cm >> 32);
  const int b = hiw ? 32 + __ffs(hiw) - 1 : static_cast<int>(N - p0);

  Cols<CPL> acc;
#pragma unroll
  for (int k = 0; k < Cols<CPL>::n; ++k) acc.v[k] = 0.f;
  int c = a;  // current chunk start (relative)
  for (int e0 = a; e0 < b; e0 += kFoldBatch) {
    Cols<CPL> g[kFoldBatch];
#pragma unroll
    for (int u = 0; u < kFoldBatch; ++u) {
      const int e = e0 + u;
      if (e < b) {
        const uint32_t idx = e < 32 ? __shfl_sync(kFull, iA, e) : __shfl_sync(kFull, iB, e - 32);
        load_cols<CPL, BF16>(grad, idx, D, g[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kFoldBatch; ++u) {
      const int e = e0 + u;
      if (e < b) {
        if ((cm >> e) & 1ull) {
          c = e;
#pragma unroll
          for (int k = 0; k < Cols<CPL>::n; ++k) acc.v[k] = g[u].v[k];
        } else {
#pragma unroll
          for (int k = 0; k < Cols<CPL>::n; ++k) acc.v[k] = acc.v[k] + g[u].v[k];
        }
        const int nxt = e + 1;
        const bool chunk_end = nxt == b || ((cm >> nxt) & 1ull);
        if (chunk_end) {
          const uint32_t key = c < 32 ? __shfl_sync(kFull, kA, c) : __shfl_sync(kFull, kB, c - 32);
          if (key != bad_key) {
            const bool is_head = (hm >> c) & 1ull;
            const bool run_ends = (p0 + nxt >= N) || ((hm >> nxt) & 1ull);
            if (is_head && run_ends) {
              red_add_row<CPL>(table_grad, key, D, acc);
            } else {
              const int64_t pos = p0 + c;
              store_slot<CPL>(csum, 2 * (pos >> 5) + (is_head ? 1 : 0), D, acc);
              if (lane == 0) {
                if (is_head) mc_list[atomicAdd(mc_count, 1)] = static_cast<int>(pos);
                if (run_ends) {
                  const int64_t s = run_start(c);
                  mc_len[s >> 5] = static_cast<int>(p0 + nxt - s);
                }
              }
            }
          }
        }
      }
    }
  }
}

// Level 2: one warp per run longer than 32 hits.
template <int CPL>
__global__ void __launch_bounds__(kFoldThreads)
fold_heavy_kernel(const uint32_t* __restrict__ K, int64_t N, uint32_t bad_key, const float* __restrict__ csum,
                  const int* __restrict__ mc_len, const int* __restrict__ mc_list, const int* __restrict__ mc_count,
                  int D, float* __restrict__ table_grad) {
  const int lane = threadIdx.x & 31;
  const int count = *mc_count;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kFoldThreads / 32);
  for (int64_t q = (static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x) >> 5; q < count; q += nwarps) {
    const int64_t c0 = mc_list[q];
    const int64_t len = min(static_cast<int64_t>(mc_len[c0 >> 5]), N - c0);  // clamp: never past the end
    const int nc = static_cast<int>((len + kChunk - 1) / kChunk);
    const uint32_t key = K[c0];
    if (key >= bad_key) continue;
    Cols<CPL> acc, x;
    auto load_slot = [&](int64_t slot, Cols<CPL>& y) {
      if constexpr (CPL == 0) {
#pragma unroll
        for (int k = 0; k < kMaxColsPerLane; ++k)
          y.v[k] = (lane + 32 * k < D) ? csum[slot * D + lane + 32 * k] : 0.f;
      } else {
        const float* p = csum + slot * D + lane * CPL;
#pragma unroll
        for (int k = 0; k < CPL; ++k) y.v[k] = p[k];
      }
    };
    load_slot(2 * (c0 >> 5) + 1, acc);
    for (int m = 1; m < nc; ++m) {
      load_slot(2 * ((c0 + static_cast<int64_t>(m) * kChunk) >> 5), x);
#pragma unroll
      for (int k = 0; k < Cols<CPL>::n; ++k) acc.v[k] = acc.v[k] + x.v[k];
    }
    red_add_row<CPL>(table_grad, key, D, acc);
  }
}

// Non-deterministic reference: one warp per hit, fp32 reductions.
template <int CPL, bool BF16>
__global__ void __launch_bounds__(kFoldThreads)
atomic_kernel(const int64_t* __restrict__ rows, int64_t N, int64_t num_rows, const void* __restrict__ grad, int D,
              float* __restrict__ table_grad, unsigned int* status) {
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kFoldThreads / 32);
  bool bad = false;
  for (int64_t i = (static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x) >> 5; i < N; i += nwarps) {
    const int64_t r = rows[i];
    if (r < 0 || r >= num_rows) {
      bad = true;
      continue;
    }
    Cols<CPL> x;
    load_cols<CPL, BF16>(grad, i, D, x);
    red_add_row<CPL>(table_grad, r, D, x);
  }
  if (bad && (threadIdx.x & 31) == 0) raise_flag(status, PLE_ERR_BAD_ROW);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Layout {
  size_t keys[2], vals[2], hist, csum, mc_len, mc_list, mc_count, total;
  int num_tiles;
  int64_t nwin;
};

size_t align_up(size_t x) { return (x + 255) & ~size_t{255}; }

Layout layout_for(int64_t N, int D) {
  Layout L{};
  L.num_tiles = static_cast<int>((N + kSortTile - 1) / kSortTile);
  L.nwin = (N + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  for (int b = 0; b < 2; ++b) L.keys[b] = take(sizeof(uint32_t) * N);
  for (int b = 0; b < 2; ++b) L.vals[b] = take(sizeof(uint32_t) * N);
  L.hist = take(sizeof(uint32_t) * kRadix * static_cast<size_t>(L.num_tiles));
  L.csum = take(sizeof(float) * 2 * static_cast<size_t>(L.nwin) * D);
  L.mc_len = take(sizeof(int) * L.nwin);
  L.mc_list = take(sizeof(int) * L.nwin);
  L.mc_count = take(sizeof(int));
  L.total = off;
  return L;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int cols_per_lane(int D) {
  if (D == 32 || D == 64 || D == 128 || D == 256) return D / 32;
  return 0;
}

ple_status_t check_grad_args(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* grad,
                             ple_dtype_t gdt, const float* tg) {
  if (plan == nullptr || N < 0) return PLE_ERR_INVALID_ARG;
  if (gdt != PLE_F32 && gdt != PLE_BF16) return PLE_ERR_INVALID_ARG;
  if (N == 0) return PLE_OK;
  if (rows == nullptr || grad == nullptr || tg == nullptr) return PLE_ERR_INVALID_ARG;
  if (plan->head_dim > 32 * kMaxColsPerLane) return PLE_ERR_UNSUPPORTED;
  if (!aligned(rows, 8) || !aligned(grad, 16) || !aligned(tg, 16)) return PLE_ERR_ALIGNMENT;
  if ((static_cast<int64_t>(plan->head_dim) * (gdt == PLE_F32 ? 4 : 2)) % 16 != 0) return PLE_ERR_ALIGNMENT;
  return PLE_OK;
}

bool g_scatter_smem_set[64];

}  // namespace
}  // namespace ple

using namespace ple;

extern "C" {

size_t ple_grad_scatter_workspace_bytes(const ple_plan_t* plan, int64_t N) {
  if (plan == nullptr || N <= 0) return 0;
  return layout_for(N, plan->head_dim).total;
}

ple_status_t ple_grad_scatter(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* grad,
                              ple_dtype_t gdt, float* table_grad, void* workspace, size_t ws_bytes,
                              void* stream) {
  ple_status_t st = check_grad_args(plan, rows, N, grad, gdt, table_grad);
  if (st != PLE_OK || N == 0) return st;
  if (plan->num_rows >= static_cast<int64_t>(kNoKey) || N >= (int64_t{1} << 31)) return PLE_ERR_UNSUPPORTED;
  const int D = plan->head_dim;
  const Layout L = layout_for(N, D);
  if (workspace == nullptr || ws_bytes < L.total) return PLE_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return PLE_ERR_ALIGNMENT;
  cudaError_t e;
  unsigned int* status = status_word(&e);
  if (status == nullptr) return cuda_fail(e);
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !g_scatter_smem_set[dev]) {
    e = cudaFuncSetAttribute(scatter_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kScatterSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(scatter_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(kScatterSmem));
    if (e != cudaSuccess) return cuda_fail(e);
    g_scatter_smem_set[dev] = true;
  }
  auto* ws = static_cast<unsigned char*>(workspace);
  uint32_t* keys[2] = {reinterpret_cast<uint32_t*>(ws + L.keys[0]), reinterpret_cast<uint32_t*>(ws + L.keys[1])};
  uint32_t* vals[2] = {reinterpret_cast<uint32_t*>(ws + L.vals[0]), reinterpret_cast<uint32_t*>(ws + L.vals[1])};
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  float* csum = reinterpret_cast<float*>(ws + L.csum);
  int* mc_len = reinterpret_cast<int*>(ws + L.mc_len);
  int* mc_list = reinterpret_cast<int*>(ws + L.mc_list);
  int* mc_count = reinterpret_cast<int*>(ws + L.mc_count);
  const auto s = static_cast<cudaStream_t>(stream);

  // key bits: keys lie in [0, num_rows] (num_rows marks a bad row)
  int bits = 0;
  while (bits < 32 && (static_cast<uint64_t>(plan->num_rows) >> bits) != 0) ++bits;
  const int passes = (bits + 7) / 8;
  const int M = kRadix * L.num_tiles;

  keys_kernel<<<L.num_tiles, kSortThreads, 0, s>>>(rows, N, plan->num_rows, keys[0], hist, L.num_tiles, mc_count,
                                                   status);
  int cur = 0;
  for (int p = 0; p < passes; ++p) {
    if (p > 0) hist_kernel<<<L.num_tiles, kSortThreads, 0, s>>>(keys[cur], N, 8 * p, hist, L.num_tiles);
    scan_kernel<<<1, kScanThreads, 0, s>>>(hist, M);
    if (p == 0)
      scatter_kernel<true><<<L.num_tiles, kSortThreads, kScatterSmem, s>>>(keys[cur], nullptr, keys[1 - cur],
                                                                          vals[1 - cur], hist, N, 0, L.num_tiles);
    else
      scatter_kernel<false><<<L.num_tiles, kSortThreads, kScatterSmem, s>>>(
          keys[cur], vals[cur], keys[1 - cur], vals[1 - cur], hist, N, 8 * p, L.num_tiles);
    cur = 1 - cur;
  }
  const uint32_t* Ks = keys[cur];
  const uint32_t* Is = vals[cur];
  const uint32_t bad_key = static_cast<uint32_t>(plan->num_rows);
  const unsigned fold_blocks = static_cast<unsigned>((L.nwin * 32 + kFoldThreads - 1) / kFoldThreads);
  const unsigned heavy_blocks = static_cast<unsigned>(sm_count() * 4);
  const int cpl = cols_per_lane(D);
  const bool bf = gdt == PLE_BF16;
#define PLE_FOLD(CPL)                                                                                      \
  do {                                                                                                     \
    if (bf)                                                                                                \
      fold_kernel<CPL, true><<<fold_blocks, kFoldThreads, 0, s>>>(Ks, Is, N, bad_key, grad, D, table_grad, \
                                                                  csum, mc_len, mc_list, mc_count);        \
    else                                                                                                   \
      fold_kernel<CPL, false><<<fold_blocks, kFoldThreads, 0, s>>>(Ks, Is, N, bad_key, grad, D, table_grad, \
                                                                   csum, mc_len, mc_list, mc_count);       \
    fold_heavy_kernel<CPL><<<heavy_blocks, kFoldThreads, 0, s>>>(Ks, N, bad_key, csum, mc_len, mc_list,     \
                                                                 mc_count, D, table_grad);                 \
  } while (0)
  switch (cpl) {
    case 1: PLE_FOLD(1); break;
    case 2: PLE_FOLD(2); break;
    case 4: PLE_FOLD(4); break;
    case 8: PLE_FOLD(8); break;
    default: PLE_FOLD(0); break;
  }
#undef PLE_FOLD
  return check_launch();
}

ple_status_t ple_grad_scatter_atomic(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* grad,
                                     ple_dtype_t gdt, float* table_grad, void* stream) {
  ple_status_t st = check_grad_args(plan, rows, N, grad, gdt, table_grad);
  if (st != PLE_OK || N == 0) return st;
  cudaError_t e;
  unsigned int* status = status_word(&e);
  if (status == nullptr) return cuda_fail(e);
  const int D = plan->head_dim;
  const auto s = static_cast<cudaStream_t>(stream);
  const unsigned blocks = static_cast<unsigned>(
      std::min<int64_t>((N * 32 + kFoldThreads - 1) / kFoldThreads, static_cast<int64_t>(sm_count()) * 16));
  const bool bf = gdt == PLE_BF16;
#define PLE_ATOMIC(CPL)                                                                                   \
  do {                                                                                                    \
    if (bf)                                                                                               \
      atomic_kernel<CPL, true><<<blocks, kFoldThreads, 0, s>>>(rows, N, plan->num_rows, grad, D, table_grad, \
                                                               status);                                   \
    else                                                                                                  \
      atomic_kernel<CPL, false><<<blocks, kFoldThreads, 0, s>>>(rows, N, plan->num_rows, grad, D,          \
                                                                table_grad, status);                      \
  } while (0)
  switch (cols_per_lane(D)) {
    case 1: PLE_ATOMIC(1); break;
    case 2: PLE_ATOMIC(2); break;
    case 4: PLE_ATOMIC(4); break;
    case 8: PLE_ATOMIC(8); break;
    default: PLE_ATOMIC(0); break;
  }
#undef PLE_ATOMIC
  return check_launch();
}

}  // extern "C"
