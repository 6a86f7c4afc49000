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
#include <atomic>

#include "common.cuh"

namespace ple {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kSortThreads = 256;
constexpr int kSortItems = 4;
constexpr int kSortTile = kSortThreads * kSortItems;  // keys per sort tile
constexpr int kRadix = 256;
constexpr int kWarpsPerSortBlock = kSortThreads / 32;
constexpr int kChunk = 32;
constexpr uint32_t kNoKey = 0xffffffffu;  // past the end; never a real key
constexpr int kFoldThreads = 256;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---------------------------------------------------------------------------
// radix sort
//
// Tiles of 4096 keys; inside a tile warp w owns positions [512w, 512w+512),
// read in 16 rounds of 32, so (warp, round, lane) is the tile order.
// Histograms are stored tile-major, hist[tile][digit].  Tiles form groups of
// 32: the last block of a group to finish its histogram (atomic ticket, no
// waiting) turns the group's histograms into in-group exclusive prefixes and
// writes the group's digit totals.  A scatter block then derives its global
// digit offsets from the (few) group totals itself, so no device-wide scan
// kernel is needed.
// ---------------------------------------------------------------------------
constexpr int kTilesPerGroup = 32;

// Warp-aggregated shared-memory histogram update for one key per lane.
__device__ __forceinline__ void hist_add(uint32_t* h, bool valid, uint32_t digit) {
  const unsigned peers = __match_any_sync(kFull, valid ? digit : 0x100u);
  if (valid && (peers & lanemask_lt()) == 0) atomicAdd(&h[digit], __popc(peers));
}

__device__ __forceinline__ int64_t tile_pos(int64_t tile, int warp, int r, int lane) {
  return tile * kSortTile + warp * (kSortTile / kWarpsPerSortBlock) + r * 32 + lane;
}

// Block-wide exclusive sum over the 256 threads (one value per thread).
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t x, uint32_t* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp; ++w) before += warp_tot[w];
  return before + incl - x;
}

// Publish this block's histogram.  The last block of a group of 32 tiles to
// arrive (atomic ticket, nobody waits) turns the group's histograms into
// in-group exclusive prefixes and writes the group's digit totals; the last
// group to finish then turns the group totals into gbase[group][digit] =
// (keys of smaller digits) + (keys of this digit in earlier groups).  A
// scatter block's global offset for digit d is gbase[its group][d] +
// hist[its tile][d].
__device__ void publish_histogram(const uint32_t* h, uint32_t* __restrict__ hist, uint32_t* __restrict__ gtot,
                                  unsigned int* __restrict__ tickets, int num_tiles) {
  __shared__ bool is_last;
  __shared__ uint32_t warp_tot[kWarpsPerSortBlock];
  const int tile = blockIdx.x, d = threadIdx.x;
  const int ngroups = (num_tiles + kTilesPerGroup - 1) / kTilesPerGroup;
  unsigned int* group_done = tickets + ngroups;  // one more counter after the per-group tickets
  hist[static_cast<int64_t>(tile) * kRadix + d] = h[d];
  __threadfence();
  __syncthreads();
  const int g = tile / kTilesPerGroup;
  const int first = g * kTilesPerGroup;
  const int n = min(kTilesPerGroup, num_tiles - first);
  if (threadIdx.x == 0) is_last = atomicAdd(&tickets[g], 1u) == static_cast<unsigned>(n - 1);
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  {
    uint32_t v[kTilesPerGroup];
    uint32_t* col = hist + static_cast<int64_t>(first) * kRadix + d;
#pragma unroll
    for (int k = 0; k < kTilesPerGroup; ++k) v[k] = k < n ? __ldcg(col + k * kRadix) : 0;  // all loads first
    uint32_t run = 0;
#pragma unroll
    for (int k = 0; k < kTilesPerGroup; ++k) {
      if (k < n) col[k * kRadix] = run;
      run += v[k];
    }
    gtot[static_cast<int64_t>(g) * kRadix + d] = run;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    tickets[g] = 0;  // ready for the next pass / call
    is_last = atomicAdd(group_done, 1u) == static_cast<unsigned>(ngroups - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  // exclusive prefix over groups per digit, then the digit base over digits
  uint32_t total = 0;
#pragma unroll 8
  for (int k = 0; k < ngroups; ++k) total += __ldcg(gtot + static_cast<int64_t>(k) * kRadix + d);
  const uint32_t digit_base = block_exclusive_sum(total, warp_tot);
  uint32_t run = digit_base;
  for (int k0 = 0; k0 < ngroups; k0 += 8) {
    uint32_t v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = k0 + k < ngroups ? __ldcg(gtot + static_cast<int64_t>(k0 + k) * kRadix + d) : 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if (k0 + k < ngroups) gtot[static_cast<int64_t>(k0 + k) * kRadix + d] = run;
      run += v[k];
    }
  }
  if (threadIdx.x == 0) *group_done = 0;
}

__global__ void __launch_bounds__(kSortThreads)
keys_kernel(const int64_t* __restrict__ rows, int64_t N, int64_t num_rows, uint32_t* __restrict__ keys,
            uint32_t* __restrict__ hist, uint32_t* __restrict__ gtot, unsigned int* __restrict__ tickets,
            int num_tiles, unsigned int* status) {
  __shared__ uint32_t h[kRadix];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  bool bad = false;
#pragma unroll 4
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = tile_pos(blockIdx.x, warp, r, lane);
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
  publish_histogram(h, hist, gtot, tickets, num_tiles);
}

__global__ void __launch_bounds__(kSortThreads)
hist_kernel(const uint32_t* __restrict__ keys, int64_t N, int shift, uint32_t* __restrict__ hist,
            uint32_t* __restrict__ gtot, unsigned int* __restrict__ tickets, int num_tiles) {
  __shared__ uint32_t h[kRadix];
  h[threadIdx.x] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t key[kSortItems];
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = tile_pos(blockIdx.x, warp, r, lane);
    key[r] = i < N ? keys[i] : 0;
  }
#pragma unroll
  for (int r = 0; r < kSortItems; ++r)
    hist_add(h, tile_pos(blockIdx.x, warp, r, lane) < N, (key[r] >> shift) & (kRadix - 1));
  __syncthreads();
  publish_histogram(h, hist, gtot, tickets, num_tiles);
}

// Stable rank-and-scatter of one tile.  Rank of a key = its tile's global
// digit offset + the keys of that digit in earlier warps of the tile + the
// keys of that digit earlier in its own warp (running per-warp counts,
// updated round by round after every lane has read them).
template <bool kIdentityVals>
__global__ void __launch_bounds__(kSortThreads)
scatter_kernel(const uint32_t* __restrict__ kin, const uint32_t* __restrict__ vin, uint32_t* __restrict__ kout,
               uint32_t* __restrict__ vout, const uint32_t* __restrict__ hist, const uint32_t* __restrict__ gtot,
               int64_t N, int shift, int num_tiles) {
  __shared__ uint32_t wh[kWarpsPerSortBlock][kRadix];
  __shared__ uint32_t tile_base[kRadix];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, d = threadIdx.x;
  const int tile = blockIdx.x;
  const int g = tile / kTilesPerGroup;

  uint32_t key[kSortItems], val[kSortItems];
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const int64_t i = tile_pos(tile, warp, r, lane);
    key[r] = i < N ? kin[i] : kNoKey;
    val[r] = i < N ? (kIdentityVals ? static_cast<uint32_t>(i) : vin[i]) : 0;
  }
  tile_base[d] = gtot[static_cast<int64_t>(g) * kRadix + d] + hist[static_cast<int64_t>(tile) * kRadix + d];
#pragma unroll
  for (int w = 0; w < kWarpsPerSortBlock; ++w) wh[w][d] = 0;
  __syncthreads();
  uint16_t rank[kSortItems];
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    const bool valid = tile_pos(tile, warp, r, lane) < N;
    const uint32_t digit = (key[r] >> shift) & (kRadix - 1);
    const unsigned peers = __match_any_sync(kFull, valid ? digit : 0x100u);
    const unsigned lower = __popc(peers & lanemask_lt());
    rank[r] = valid ? static_cast<uint16_t>(wh[warp][digit] + lower) : 0;
    __syncwarp();
    if (valid && lower == 0) wh[warp][digit] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  {
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kWarpsPerSortBlock; ++w) {
      const uint32_t c = wh[w][d];
      wh[w][d] = run;
      run += c;
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kSortItems; ++r) {
    if (tile_pos(tile, warp, r, lane) < N) {
      const uint32_t digit = (key[r] >> shift) & (kRadix - 1);
      const uint32_t dst = tile_base[digit] + wh[warp][digit] + rank[r];
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

// Level 1 works on windows of 32 sorted positions, one warp per window.
// One round trip brings the window's keys and hit indices, the next 32 keys
// (a chunk that starts in this window may end in the next) and the previous
// 32 keys (to find where the run holding the window's first position starts;
// only runs longer than 32 need the search).  The warp folds the chunks that
// START in its window: positions [a, b) relative to p0, b being the first
// chunk start of the next window (or the end).
struct Window {
  uint64_t hm;   // run starts among positions p0 .. p0+63
  uint64_t cm;   // chunk starts among positions p0 .. p0+63
  int64_t p0, s0;
  int a, b;
  uint32_t kA, kB, iA, iB;
  __device__ int64_t run_start(int idx) const {  // first position of the run holding p0 + idx
    const uint64_t le = hm & (idx >= 63 ? ~0ull : ((2ull << idx) - 1));
    return le ? p0 + (63 - __clzll(le)) : s0;
  }
  __device__ uint32_t key_at(int e) const {  // warp-uniform e in [0, 64)
    const uint32_t ka = __shfl_sync(kFull, kA, e & 31), kb = __shfl_sync(kFull, kB, e & 31);
    return e < 32 ? ka : kb;
  }
};

__device__ __forceinline__ bool window_setup(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I,
                                             int64_t N, int64_t w, Window& W) {
  const int lane = threadIdx.x & 31;
  const int64_t p0 = w * 32;
  const int64_t pa = p0 + lane, pb = p0 + 32 + lane, pc = p0 - 32 + lane;
  W.p0 = p0;
  W.kA = pa < N ? K[pa] : kNoKey;
  W.kB = pb < N ? K[pb] : kNoKey;
  const uint32_t kC = p0 > 0 ? K[pc] : kNoKey;  // p0 is a multiple of 32, so pc >= 0 here
  W.iA = pa < N ? I[pa] : 0;
  W.iB = pb < N ? I[pb] : 0;
  uint32_t prevA = __shfl_up_sync(kFull, W.kA, 1);
  uint32_t prevB = __shfl_up_sync(kFull, W.kB, 1);
  const uint32_t kA31 = __shfl_sync(kFull, W.kA, 31);
  const uint32_t kC31 = __shfl_sync(kFull, kC, 31);
  if (lane == 0) {
    prevA = kC31;
    prevB = kA31;
  }
  const bool headA = pa < N && W.kA != prevA;
  const bool headB = pb < N && W.kB != prevB;
  W.hm = static_cast<uint64_t>(__ballot_sync(kFull, headA)) |
         (static_cast<uint64_t>(__ballot_sync(kFull, headB)) << 32);
  const uint32_t key0 = __shfl_sync(kFull, W.kA, 0);
  W.s0 = p0;
  if (!(W.hm & 1ull)) {
    // p0 > 0 here; the run started among the previous 32 positions unless
    // all of them hold key0
    const unsigned differ = __ballot_sync(kFull, kC != key0);
    W.s0 = differ ? p0 - 32 + (32 - __clz(differ)) : find_run_start(K, p0 - 32, key0);
  }
  const bool csA = pa < N && ((pa - W.run_start(lane)) & (kChunk - 1)) == 0;
  const bool csB = pb < N && ((pb - W.run_start(32 + lane)) & (kChunk - 1)) == 0;
  W.cm = static_cast<uint64_t>(__ballot_sync(kFull, csA)) | (static_cast<uint64_t>(__ballot_sync(kFull, csB)) << 32);
  // A window may hold no chunk start only at the tail, when its positions
  // finish a chunk that started in the previous window (folded there).
  if ((W.cm & 0xffffffffull) == 0) return false;
  W.a = __ffsll(static_cast<long long>(W.cm & 0xffffffffull)) - 1;
  const uint32_t hiw = static_cast<uint32_t>(W.cm >> 32);
  W.b = hiw ? 32 + __ffs(hiw) - 1 : static_cast<int>(N - p0);
  return true;
}

// Bookkeeping of a finished chunk [c, nxt) (relative positions) whose sum the
// calling lanes hold: returns true if the chunk is a whole run (the caller
// adds it into table_grad), false if its sum goes to a chunk-sum slot
// (returned in *slot); lane `leader` records heavy-run metadata.
__device__ __forceinline__ bool chunk_is_whole_run(const Window& W, int c, int nxt, int64_t N, bool leader,
                                                   int64_t* slot, int* __restrict__ mc_len,
                                                   int* __restrict__ mc_list, int* __restrict__ mc_count) {
  const bool is_head = (W.hm >> c) & 1ull;
  const bool run_ends = (W.p0 + nxt >= N) || ((W.hm >> nxt) & 1ull);
  if (is_head && run_ends) return true;
  const int64_t pos = W.p0 + c;
  *slot = 2 * (pos >> 5) + (is_head ? 1 : 0);
  if (leader) {
    if (is_head) mc_list[atomicAdd(mc_count, 1)] = static_cast<int>(pos);
    if (run_ends) {
      const int64_t s = W.run_start(c);
      mc_len[s >> 5] = static_cast<int>(W.p0 + nxt - s);
    }
  }
  return false;
}

__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

template <bool BF16>
__device__ __forceinline__ void unpack16(const uint4& y, float* v) {
  if constexpr (BF16) {
    v[0] = bf16_lo(y.x); v[1] = bf16_hi(y.x); v[2] = bf16_lo(y.y); v[3] = bf16_hi(y.y);
    v[4] = bf16_lo(y.z); v[5] = bf16_hi(y.z); v[6] = bf16_lo(y.w); v[7] = bf16_hi(y.w);
  } else {
    v[0] = __uint_as_float(y.x); v[1] = __uint_as_float(y.y);
    v[2] = __uint_as_float(y.z); v[3] = __uint_as_float(y.w);
  }
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

constexpr int kWideWarps = 4;  // warps per block of the wide fold
constexpr int kWideLoads = 8;  // 16-byte async copies per lane per batch

// Wide fold: a grad row spans L lanes that each copy 16 bytes, so one
// instruction fetches 32/L rows.  A batch of rows is staged in shared memory
// by asynchronous copies (no registers held while they are in flight).  A run
// of a single hit is added into table_grad by the lane group that fetched it.
// Hits of longer runs are folded in order: every L-lane group keeps the same
// running chunk sum (lane `sub` of a group owns CPLN = 16/elem columns) and
// adds row after row from the staging buffer; the groups write finished
// chunks in turn.
template <int L, bool BF16>
__global__ void __launch_bounds__(kWideWarps * 32, 8)
fold_wide_kernel(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I, int64_t N, uint32_t bad_key,
                 const void* __restrict__ grad, int D, float* __restrict__ table_grad, float* __restrict__ csum,
                 int* __restrict__ mc_len, int* __restrict__ mc_list, int* __restrict__ mc_count) {
  constexpr int RPI = 32 / L;                                            // rows per copy instruction
  constexpr int CPLN = BF16 ? 8 : 4;                                     // fp32 columns per lane
  constexpr int BATCH = kWideLoads * RPI < 64 ? kWideLoads * RPI : 64;   // hits per batch
  constexpr int LOADS = BATCH / RPI;                                     // copies per lane per batch
  __shared__ uint4 stage[kWideWarps][kWideLoads][32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / L, sub = lane % L;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kWideWarps + warp;
  if (w * 32 >= N) return;
  Window W;
  if (!window_setup(K, I, N, w, W)) return;
  const size_t row_bytes = static_cast<size_t>(D) * (BF16 ? 2 : 4);
  const unsigned char* gbase = static_cast<const unsigned char*>(grad) + sub * 16;
  // positions holding a run of exactly one hit
  const uint64_t next_is_head = (W.hm >> 1) | (W.p0 + 63 >= N ? (1ull << (N - 1 - W.p0)) : 0ull);
  const uint64_t single = W.hm & next_is_head;

  float acc[CPLN];
#pragma unroll
  for (int k = 0; k < CPLN; ++k) acc[k] = 0.f;
  int c = W.a, turn = 0;
  for (int e0 = W.a; e0 < W.b; e0 += BATCH) {
#pragma unroll
    for (int s = 0; s < LOADS; ++s) {
      const int e = e0 + s * RPI + grp;
      const int src = e & 31;
      const uint32_t ia = __shfl_sync(kFull, W.iA, src), ib = __shfl_sync(kFull, W.iB, src);
      if (e < W.b) cp_async16(&stage[warp][s][lane], gbase + static_cast<size_t>(e < 32 ? ia : ib) * row_bytes);
    }
    cp_async_wait_all();
    __syncwarp();
#pragma unroll
    for (int s = 0; s < LOADS; ++s) {
      const int e = e0 + s * RPI + grp;
      const int src = e & 31;
      const uint32_t ka = __shfl_sync(kFull, W.kA, src), kb = __shfl_sync(kFull, W.kB, src);
      const uint32_t key = e < 32 ? ka : kb;
      if (e < W.b && ((single >> e) & 1ull) && key != bad_key) {
        float v[CPLN];
        unpack16<BF16>(stage[warp][s][lane], v);
        float* dst = table_grad + static_cast<int64_t>(key) * D + sub * CPLN;
#pragma unroll
        for (int k = 0; k < CPLN; k += 4) red_add4(dst + k, v[k], v[k + 1], v[k + 2], v[k + 3]);
      }
    }
    const int nb = min(BATCH, W.b - e0);
    uint64_t multi = (~single >> e0) & (nb >= 64 ? ~0ull : ((1ull << nb) - 1));
    while (multi) {
      const int t = __ffsll(static_cast<long long>(multi)) - 1;
      multi &= multi - 1;
      const int e = e0 + t;
      float v[CPLN];
      unpack16<BF16>(stage[warp][t / RPI][sub + L * (t % RPI)], v);
      if ((W.cm >> e) & 1ull) {
        c = e;
#pragma unroll
        for (int k = 0; k < CPLN; ++k) acc[k] = v[k];
      } else {
#pragma unroll
        for (int k = 0; k < CPLN; ++k) acc[k] = acc[k] + v[k];
      }
      const int nxt = e + 1;
      if (nxt == W.b || ((W.cm >> nxt) & 1ull)) {  // chunk [c, nxt) complete
        const uint32_t key = W.key_at(c);
        if (key != bad_key) {
          const int writer = turn % RPI;
          int64_t slot = 0;
          const bool whole = chunk_is_whole_run(W, c, nxt, N, lane == 0, &slot, mc_len, mc_list, mc_count);
          if (grp == writer) {
            float* dst = (whole ? table_grad + static_cast<int64_t>(key) * D : csum + slot * D) + sub * CPLN;
            if (whole) {
#pragma unroll
              for (int k = 0; k < CPLN; k += 4) red_add4(dst + k, acc[k], acc[k + 1], acc[k + 2], acc[k + 3]);
            } else {
#pragma unroll
              for (int k = 0; k < CPLN; k += 4)
                *reinterpret_cast<float4*>(dst + k) = make_float4(acc[k], acc[k + 1], acc[k + 2], acc[k + 3]);
            }
          }
          ++turn;
        }
      }
    }
    __syncwarp();  // the next batch reuses the staging buffer
  }
}

// Generic fold for row sizes the wide fold does not cover: lanes own
// columns l, l+32, ... of every row; one warp-wide load per hit.
template <bool BF16>
__global__ void __launch_bounds__(kFoldThreads, 3)
fold_generic_kernel(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I, int64_t N, uint32_t bad_key,
                    const void* __restrict__ grad, int D, float* __restrict__ table_grad, float* __restrict__ csum,
                    int* __restrict__ mc_len, int* __restrict__ mc_list, int* __restrict__ mc_count) {
  constexpr int kBatch = 4;
  const int lane = threadIdx.x & 31;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * kFoldThreads + threadIdx.x) >> 5;
  if (w * 32 >= N) return;
  Window W;
  if (!window_setup(K, I, N, w, W)) return;
  Cols<0> acc;
#pragma unroll
  for (int k = 0; k < Cols<0>::n; ++k) acc.v[k] = 0.f;
  int c = W.a;
  for (int e0 = W.a; e0 < W.b; e0 += kBatch) {
    Cols<0> g[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = e0 + u;
      if (e < W.b) {
        const uint32_t ia = __shfl_sync(kFull, W.iA, e & 31), ib = __shfl_sync(kFull, W.iB, e & 31);
        load_cols<0, BF16>(grad, e < 32 ? ia : ib, D, g[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = e0 + u;
      if (e < W.b) {
        if ((W.cm >> e) & 1ull) {
          c = e;
#pragma unroll
          for (int k = 0; k < Cols<0>::n; ++k) acc.v[k] = g[u].v[k];
        } else {
#pragma unroll
          for (int k = 0; k < Cols<0>::n; ++k) acc.v[k] = acc.v[k] + g[u].v[k];
        }
        const int nxt = e + 1;
        if (nxt == W.b || ((W.cm >> nxt) & 1ull)) {
          const uint32_t key = W.key_at(c);
          if (key != bad_key) {
            int64_t slot = 0;
            if (chunk_is_whole_run(W, c, nxt, N, lane == 0, &slot, mc_len, mc_list, mc_count))
              red_add_row<0>(table_grad, key, D, acc);
            else
              store_slot<0>(csum, slot, D, acc);
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
    Cols<CPL> acc;
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
    constexpr int kAhead = 8;  // chunk sums loaded ahead of the in-order adds
    for (int m0 = 1; m0 < nc; m0 += kAhead) {
      Cols<CPL> y[kAhead];
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
        if (m0 + u < nc) load_slot(2 * ((c0 + static_cast<int64_t>(m0 + u) * kChunk) >> 5), y[u]);
#pragma unroll
      for (int u = 0; u < kAhead; ++u)
        if (m0 + u < nc) {
#pragma unroll
          for (int k = 0; k < Cols<CPL>::n; ++k) acc.v[k] = acc.v[k] + y[u].v[k];
        }
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
  size_t keys[2], vals[2], hist, gtot, csum, mc_len, mc_list, zeroed, total;
  size_t zeroed_bytes;  // tickets of every pass + the heavy-run counter, cleared per call
  int num_tiles, num_groups, max_passes;
  int64_t nwin;
};

size_t align_up(size_t x) { return (x + 255) & ~size_t{255}; }

Layout layout_for(int64_t N, int D) {
  Layout L{};
  L.num_tiles = static_cast<int>((N + kSortTile - 1) / kSortTile);
  L.num_groups = (L.num_tiles + kTilesPerGroup - 1) / kTilesPerGroup;
  L.max_passes = 4;
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
  L.gtot = take(sizeof(uint32_t) * kRadix * static_cast<size_t>(L.num_groups));
  L.csum = take(sizeof(float) * 2 * static_cast<size_t>(L.nwin) * D);
  L.mc_len = take(sizeof(int) * L.nwin);
  L.mc_list = take(sizeof(int) * L.nwin);
  L.zeroed_bytes = sizeof(unsigned int) * (static_cast<size_t>(L.max_passes) * (L.num_groups + 1) + 1);
  L.zeroed = take(L.zeroed_bytes);
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
  auto* ws = static_cast<unsigned char*>(workspace);
  uint32_t* keys[2] = {reinterpret_cast<uint32_t*>(ws + L.keys[0]), reinterpret_cast<uint32_t*>(ws + L.keys[1])};
  uint32_t* vals[2] = {reinterpret_cast<uint32_t*>(ws + L.vals[0]), reinterpret_cast<uint32_t*>(ws + L.vals[1])};
  uint32_t* hist = reinterpret_cast<uint32_t*>(ws + L.hist);
  uint32_t* gtot = reinterpret_cast<uint32_t*>(ws + L.gtot);
  float* csum = reinterpret_cast<float*>(ws + L.csum);
  int* mc_len = reinterpret_cast<int*>(ws + L.mc_len);
  int* mc_list = reinterpret_cast<int*>(ws + L.mc_list);
  unsigned int* tickets = reinterpret_cast<unsigned int*>(ws + L.zeroed);
  int* mc_count = reinterpret_cast<int*>(tickets + static_cast<size_t>(L.max_passes) * (L.num_groups + 1));
  const auto s = static_cast<cudaStream_t>(stream);

  // key bits: keys lie in [0, num_rows] (num_rows marks a bad row)
  int bits = 0;
  while (bits < 32 && (static_cast<uint64_t>(plan->num_rows) >> bits) != 0) ++bits;
  const int passes = (bits + 7) / 8;

  e = cudaMemsetAsync(tickets, 0, L.zeroed_bytes, s);
  if (e != cudaSuccess) return cuda_fail(e);
  keys_kernel<<<L.num_tiles, kSortThreads, 0, s>>>(rows, N, plan->num_rows, keys[0], hist, gtot, tickets,
                                                   L.num_tiles, status);
  int cur = 0;
  for (int p = 0; p < passes; ++p) {
    if (p > 0)
      hist_kernel<<<L.num_tiles, kSortThreads, 0, s>>>(keys[cur], N, 8 * p, hist, gtot,
                                                       tickets + static_cast<size_t>(p) * (L.num_groups + 1),
                                                       L.num_tiles);
    if (p == 0)
      scatter_kernel<true><<<L.num_tiles, kSortThreads, 0, s>>>(keys[cur], nullptr, keys[1 - cur], vals[1 - cur],
                                                                hist, gtot, N, 0, L.num_tiles);
    else
      scatter_kernel<false><<<L.num_tiles, kSortThreads, 0, s>>>(keys[cur], vals[cur], keys[1 - cur],
                                                                 vals[1 - cur], hist, gtot, N, 8 * p, L.num_tiles);
    cur = 1 - cur;
  }
  const uint32_t* Ks = keys[cur];
  const uint32_t* Is = vals[cur];
  const uint32_t bad_key = static_cast<uint32_t>(plan->num_rows);
  const unsigned fold_blocks = static_cast<unsigned>((L.nwin * 32 + kFoldThreads - 1) / kFoldThreads);
  const unsigned heavy_blocks = static_cast<unsigned>(sm_count() * 4);
  const bool bf = gdt == PLE_BF16;
  const int lanes_per_row = static_cast<int>(static_cast<int64_t>(D) * (bf ? 2 : 4) / 16);
  const unsigned wide_blocks = static_cast<unsigned>((L.nwin + kWideWarps - 1) / kWideWarps);
#define PLE_FOLD_WIDE(LW)                                                                                   \
  case LW:                                                                                                  \
    if (bf)                                                                                                 \
      fold_wide_kernel<LW, true><<<wide_blocks, kWideWarps * 32, 0, s>>>(Ks, Is, N, bad_key, grad, D,       \
                                                                         table_grad, csum, mc_len, mc_list, \
                                                                         mc_count);                         \
    else                                                                                                    \
      fold_wide_kernel<LW, false><<<wide_blocks, kWideWarps * 32, 0, s>>>(Ks, Is, N, bad_key, grad, D,      \
                                                                          table_grad, csum, mc_len, mc_list, \
                                                                          mc_count);                        \
    break;
  switch (lanes_per_row) {
    PLE_FOLD_WIDE(1)
    PLE_FOLD_WIDE(2)
    PLE_FOLD_WIDE(4)
    PLE_FOLD_WIDE(8)
    PLE_FOLD_WIDE(16)
    PLE_FOLD_WIDE(32)
    default:
      if (bf)
        fold_generic_kernel<true><<<fold_blocks, kFoldThreads, 0, s>>>(Ks, Is, N, bad_key, grad, D, table_grad,
                                                                       csum, mc_len, mc_list, mc_count);
      else
        fold_generic_kernel<false><<<fold_blocks, kFoldThreads, 0, s>>>(Ks, Is, N, bad_key, grad, D, table_grad,
                                                                        csum, mc_len, mc_list, mc_count);
  }
#undef PLE_FOLD_WIDE
  switch (cols_per_lane(D)) {
    case 1: fold_heavy_kernel<1><<<heavy_blocks, kFoldThreads, 0, s>>>(Ks, N, bad_key, csum, mc_len, mc_list, mc_count, D, table_grad); break;
    case 2: fold_heavy_kernel<2><<<heavy_blocks, kFoldThreads, 0, s>>>(Ks, N, bad_key, csum, mc_len, mc_list, mc_count, D, table_grad); break;
    case 4: fold_heavy_kernel<4><<<heavy_blocks, kFoldThreads, 0, s>>>(Ks, N, bad_key, csum, mc_len, mc_list, mc_count, D, table_grad); break;
    case 8: fold_heavy_kernel<8><<<heavy_blocks, kFoldThreads, 0, s>>>(Ks, N, bad_key, csum, mc_len, mc_list, mc_count, D, table_grad); break;
    default: fold_heavy_kernel<0><<<heavy_blocks, kFoldThreads, 0, s>>>(Ks, N, bad_key, csum, mc_len, mc_list, mc_count, D, table_grad); break;
  }
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

// ---------------------------------------------------------------------------
// Gradient scatter without any allocation by anyone.
//
// Some callers cannot hand the library a workspace: a serving process whose
// device memory is reserved up front and may not grow while requests run, a
// host plugin that is not allowed to call the CUDA allocator, or a hot loop
// where cudaMalloc could synchronise the device and stall every stream.  For
// them the library keeps one fixed scratch area
// of kNoAllocScratchBytes in device memory (allocated with the module, held by
// every GPU that loads the library until the process exits) and runs the same
// deterministic sort-and-fold kernels in it.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t{32} << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch, one per device.  In host code the
// array's name only stands in for the symbol; its device address has to be
// looked up with that device current.
std::atomic<void*> g_noalloc_addr[64];

}  // namespace

extern "C" {

ple_status_t ple_grad_scatter_noalloc(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* grad,
                                      ple_dtype_t gdt, float* table_grad, void* stream) {
  if (plan == nullptr || N < 0) return PLE_ERR_INVALID_ARG;
  if (N == 0) return check_grad_args(plan, rows, N, grad, gdt, table_grad);
  if (ple_grad_scatter_workspace_bytes(plan, N) > kNoAllocScratchBytes) return PLE_ERR_WORKSPACE;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return PLE_ERR_UNSUPPORTED;
  void* scratch = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (scratch == nullptr) {  // first call on this device: look the address up
    e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    g_noalloc_addr[dev].store(scratch, std::memory_order_release);
  }
  return ple_grad_scatter(plan, rows, N, grad, gdt, table_grad, scratch, kNoAllocScratchBytes, stream);
}

size_t ple_grad_scatter_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

}  // extern "C"
