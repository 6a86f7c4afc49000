// Stable LSD radix sort of 32-bit keys with 32-bit values (the hit index),
// shared by the table gradient and the host-memory tier: key_hist_kernel
// turns int64 rows into keys and counts the digits of every pass, then one
// sort_pass_kernel per 8-bit digit (see the comment above SortArgs).
// Everything lives in an anonymous namespace: each translation unit that
// includes this header gets its own copy of the kernels.
#ifndef PLE_SORT_CUH_
#define PLE_SORT_CUH_

#include "common.cuh"

namespace ple {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kRadix = 256;

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ---------------------------------------------------------------------------
// radix sort: LSD, 8-bit digits, stable, one kernel per pass
//
// key_hist_kernel turns the int64 rows into 32-bit keys and counts the
// digits of every pass at once, so the global start of each digit is known
// before the first pass.  Each pass is one sort_pass_kernel launch in which
// a block takes one tile of consecutive positions (2048, 4096 or 8192 keys,
// by the key count), in the order of a ticket counter (a block only ever waits
// for tiles with lower tickets, whose blocks are already running).  The
// block counts its keys per digit and publishes the counts at once.  The
// keys of a digit in all earlier tiles are summed over three levels, so
// that no tile waits on a long chain:
//   tiles of its group of 32 tiles before it (their counts);
//   groups of its supergroup of 32 groups before its group (group totals,
//   published by the last tile of each group as soon as it has its level);
//   supergroups before its supergroup (totals published by the last tile of
//   each supergroup).
// Between the first level and the other two the block ranks its keys by
// digit (per-warp lane masks per digit, per-warp running counts: stable) and stages the tile
// in shared memory in digit order, while the other groups publish.
// A published word is READY | count; the count is the payload, so plain
// relaxed loads and stores suffice.  Keys then go to digit start + earlier
// count + rank, written from the staged tile so that the writes are
// coalesced.
//
// Every wait is bounded in time (the device's global nanosecond timer,
// limit chosen by the host per call).  A warp whose wait runs out raises
// PLE_ERR_TIMEOUT and sets the call's abort word in the workspace; every
// other waiting warp sees that word at its next poll and gives up too, later
// passes return at their first instruction, and the kernels that consume
// the sort (the gradient's fold, the prefetch's finalize) check the word
// and write nothing.  A stuck sort thus ends within about one wait limit,
// leaves its outputs (table_grad, the cache) untouched, and every access on
// the way stays inside the workspace.
// ---------------------------------------------------------------------------
constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
// Keys per thread: 32 (8192-key tiles, 2 blocks per SM) from kHugeTileKeys
// keys on, 16 (4096-key tiles, 2 blocks per SM) from kBigTileKeys, else 8
// (2048-key tiles, 3 blocks per SM): fewer tiles shorten the look-back and
// the waves of tiles, but below about 3 * 2^17 keys there are too few of
// them to fill the SMs (measured on the B200: 2048-key tiles win at 262144
// keys, 4096-key tiles at 524288; at 2097152 keys 8192-key tiles take a
// pass from two waves to one, 286.7 -> 276.5 us for the whole gradient).
constexpr int64_t kBigTileKeys = 3 << 17;
constexpr int64_t kHugeTileKeys = 37 << 15;  // 1212416 = 296 tiles of 4096: one wave of 2 blocks per SM
inline int sort_items(int64_t N) { return N >= kHugeTileKeys ? 32 : N >= kBigTileKeys ? 16 : 8; }
// Dynamic shared memory of a sort pass: the staged tile (keys, values) and,
// for 32 keys per thread, the ranks (registers would not hold them).
inline size_t sort_pass_smem(int items) {
  const size_t tile = static_cast<size_t>(kSortThreads) * items;
  return tile * 8 + (items > 16 ? tile * 2 : 0);
}
constexpr int kMaxPasses = 4;
constexpr int kGroupBits = 5;                         // 32 tiles per group, 32 groups per supergroup
constexpr uint32_t kReady = 0x80000000u;              // look-back word: READY | count (count < 2^31)

// Block-wide exclusive sum (every thread passes one value); *total gets the sum.
__device__ __forceinline__ uint32_t block_exclusive_sum(uint32_t x, uint32_t* warp_tot, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t y = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += y;
  }
  __syncthreads();  // warp_tot may still be read by a previous call
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  uint32_t before = 0, all = 0;
  for (int w = 0; w < nwarps; ++w) {
    const uint32_t t = warp_tot[w];
    if (w < warp) before += t;
    all += t;
  }
  *total = all;
  return before + incl - x;
}

__device__ __forceinline__ uint4 ld_relaxed_v4(const uint32_t* p) {
  uint4 v;
  asm volatile("ld.relaxed.gpu.global.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// What a bounded wait needs: where to raise the error, the call's abort
// word (cleared at the start of every sort), and the limit in nanoseconds.
struct WaitCtl {
  unsigned int* status;
  uint32_t* abort;
  uint64_t wait_ns;
};

__device__ __forceinline__ void st_relaxed(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ bool all_ready(const uint4& x) {
  return (x.x & x.y & x.z & x.w & kReady) != 0;
}

// Per-digit sums of the published count rows [first, last) of one level
// (row q: 256 words at rows + q * 256), by the whole block: warp w takes
// rows first + w, first + w + 8, ... (up to 4 rows in flight per warp, each
// lane reading 8 digits as two 16-byte loads); rows not yet fully published
// are loaded again, round after round; the warps' partial sums meet in
// `part`.  Returns the sum for digit threadIdx.x (threads < 256).
__device__ uint32_t level_sum(const uint32_t* rows, int64_t first, int64_t last, uint32_t (*part)[kRadix],
                              const WaitCtl& wc) {
  if (first >= last) return 0;  // block-uniform
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint32_t acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int64_t q0 = first; q0 < last; q0 += 4 * kSortWarps) {
    uint4 x[4][2];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t q = q0 + warp + k * kSortWarps;
      if (q < last) {
        x[k][0] = ld_relaxed_v4(rows + q * kRadix + lane * 8);
        x[k][1] = ld_relaxed_v4(rows + q * kRadix + lane * 8 + 4);
      } else {
        x[k][0] = x[k][1] = make_uint4(kReady, kReady, kReady, kReady);
      }
    }
    uint64_t t0 = 0;
    for (int round = 0;; ++round) {
      bool ready = true;
#pragma unroll
      for (int k = 0; k < 4; ++k) ready &= all_ready(x[k][0]) && all_ready(x[k][1]);
      if (__all_sync(kFull, ready)) break;
      // give up when the limit has passed since the first poll, or (looked
      // at every 16th round, off the common short waits) when another warp
      // of the call has given up; a warp-uniform decision
      const uint64_t now = global_ns();
      if (round == 0) t0 = now;
      bool give_up = round > 0 && now - t0 >= wc.wait_ns;
      if ((round & 15) == 15 && lane == 0) give_up |= ld_relaxed(wc.abort) != 0;
      if (__any_sync(kFull, give_up)) {
        if (lane == 0) {
          raise_flag(wc.status, PLE_ERR_TIMEOUT);
          st_relaxed(wc.abort, 1u);
        }
        break;
      }
      __nanosleep(64);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int64_t q = q0 + warp + k * kSortWarps;
        if (q < last && !(all_ready(x[k][0]) && all_ready(x[k][1]))) {
          x[k][0] = ld_relaxed_v4(rows + q * kRadix + lane * 8);
          x[k][1] = ld_relaxed_v4(rows + q * kRadix + lane * 8 + 4);
        }
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[0] += x[k][0].x & ~kReady; acc[1] += x[k][0].y & ~kReady;
      acc[2] += x[k][0].z & ~kReady; acc[3] += x[k][0].w & ~kReady;
      acc[4] += x[k][1].x & ~kReady; acc[5] += x[k][1].y & ~kReady;
      acc[6] += x[k][1].z & ~kReady; acc[7] += x[k][1].w & ~kReady;
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) part[warp][lane * 8 + j] = acc[j];
  __syncthreads();
  uint32_t sum = 0;
  if (threadIdx.x < kRadix)
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) sum += part[w][threadIdx.x];
  __syncthreads();  // part is reused by the next level
  return sum;
}

struct SortArgs {
  int64_t N;
  int64_t tiles, groups, supers;
  int passes;
  uint32_t* keys[2];
  uint32_t* vals[2];
  uint32_t* hist;          // [kMaxPasses][256] digit totals of every pass (zeroed before the sort)
  unsigned int* tickets;   // [kMaxPasses] tile tickets (zeroed before the sort)
  uint32_t* look;          // [passes][tiles + groups + supers][256] published counts
  WaitCtl wc;              // bounded waits; wc.abort is zeroed before the sort with hist and tickets
};

// Clears the digit totals, the tile tickets and the call's abort word
// before key_hist_kernel adds to them.
__global__ void clear_kernel(uint32_t* words, int n) {
  wait_for_prior_grid();  // (launched early, behind the caller's previous kernel)
  for (int i = threadIdx.x; i < n; i += blockDim.x) words[i] = 0;
  allow_next_grid();
}

// Keys from the int64 rows (a row outside [0, num_rows) becomes the key
// num_rows, sorted last and skipped by the fold) and the digit counts of
// every pass.  Also clears the look-back words of every pass and the fold's
// run counters.
__global__ void __launch_bounds__(kSortThreads)
key_hist_kernel(const int64_t* __restrict__ rows, int64_t num_rows, const SortArgs a, unsigned int* run_done,
                int64_t nwin) {
  __shared__ uint32_t h[kMaxPasses][kRadix];
  const int tid = threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kSortThreads;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * kSortThreads + tid;
  for (int k = tid; k < kMaxPasses * kRadix; k += kSortThreads) (&h[0][0])[k] = 0;
  wait_for_prior_grid();  // the totals it adds to are cleared by the previous kernel
  const int64_t look_words = static_cast<int64_t>(a.passes) * (a.tiles + a.groups + a.supers) * kRadix;
  for (int64_t i = g; i < look_words; i += stride) a.look[i] = 0;
  if (run_done != nullptr)
    for (int64_t i = g; i < nwin; i += stride) run_done[i] = 0;
  __syncthreads();
  bool bad = false;
  constexpr int kIlp = 4;  // row loads in flight per thread
  for (int64_t i0 = g; i0 < a.N; i0 += kIlp * stride) {
    int64_t v[kIlp];
#pragma unroll
    for (int u = 0; u < kIlp; ++u) v[u] = i0 + u * stride < a.N ? __ldcs(rows + i0 + u * stride) : 0;
#pragma unroll
    for (int u = 0; u < kIlp; ++u) {
      const int64_t i = i0 + u * stride;
      if (i < a.N) {
        const bool ok = v[u] >= 0 && v[u] < num_rows;
        bad |= !ok;
        const uint32_t key = ok ? static_cast<uint32_t>(v[u]) : static_cast<uint32_t>(num_rows);
        a.keys[0][i] = key;
        for (int p = 0; p < a.passes; ++p) atomicAdd(&h[p][(key >> (8 * p)) & (kRadix - 1)], 1u);
      }
    }
  }
  if (bad) raise_flag(a.wc.status, PLE_ERR_BAD_ROW);
  __syncthreads();
  for (int k = tid; k < a.passes * kRadix; k += kSortThreads) {
    const uint32_t c = (&h[0][0])[k];
    if (c) atomicAdd(a.hist + k, c);
  }
  allow_next_grid();
}

template <int ITEMS>
__global__ void __launch_bounds__(kSortThreads, ITEMS > 8 ? 2 : 3) sort_pass_kernel(const SortArgs a, const int pass) {
  constexpr int kSortTile = kSortThreads * ITEMS;   // positions per tile
  constexpr int kWarpSpan = kSortTile / kSortWarps;  // positions per warp within a tile
  __shared__ uint32_t wh[kSortWarps][kRadix];
  extern __shared__ __align__(16) uint32_t sort_dyn[];
  uint32_t* stage_k = sort_dyn;               // [kSortTile]
  uint32_t* stage_v = sort_dyn + kSortTile;   // [kSortTile]
  uint16_t* rank_s = reinterpret_cast<uint16_t*>(sort_dyn + 2 * kSortTile);  // [kSortTile], ITEMS > 16 only
  __shared__ uint32_t base_s[kRadix];
  __shared__ uint32_t start_s[kRadix];
  __shared__ uint32_t warp_tot[kSortWarps];
  __shared__ int64_t tile_s;
  __shared__ uint32_t abort_s;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  wait_for_prior_grid();
  if (tid == 0) {
    abort_s = ld_relaxed(a.wc.abort);  // an earlier wait of this sort gave up: nothing more to do
    tile_s = atomicAdd(a.tickets + pass, 1u);
  }
  if (tid < kRadix) start_s[tid] = 0;  // the tile's digit counts first
  {  // global start of every digit of this pass (while the ticket is on its way)
    const uint32_t c = tid < kRadix ? __ldcg(a.hist + pass * kRadix + tid) : 0;
    uint32_t all;
    const uint32_t start = block_exclusive_sum(c, warp_tot, &all);  // (its barriers publish tile_s, start_s)
    if (tid < kRadix) base_s[tid] = start;
  }
  allow_next_grid();
  if (abort_s != 0) return;  // block-uniform (read after the barriers above)
  const int64_t t = tile_s;
  const int64_t N = a.N, i0 = t * kSortTile + warp * kWarpSpan;
  const int shift = 8 * pass;
  const bool odd = pass & 1;  // (selects, not indexes: the parameter arrays stay in the constant bank)
  const uint32_t* kin = odd ? a.keys[1] : a.keys[0];
  const uint32_t* vin = odd ? a.vals[1] : a.vals[0];
  uint32_t* kout = odd ? a.keys[0] : a.keys[1];
  uint32_t* vout = odd ? a.vals[0] : a.vals[1];
  uint32_t* tile_rows = a.look + static_cast<int64_t>(pass) * (a.tiles + a.groups + a.supers) * kRadix;

  uint32_t key[ITEMS], val[ITEMS];
#pragma unroll
  for (int r = 0; r < ITEMS; ++r) {
    const int64_t i = i0 + r * 32 + lane;
    key[r] = i < N ? kin[i] : 0;
    val[r] = i < N ? (pass == 0 ? static_cast<uint32_t>(i) : vin[i]) : 0;
  }
  // digit counts of the tile (shared-memory atomics), published at once so
  // that later tiles' look-backs do not wait for this tile's ranking
#pragma unroll
  for (int r = 0; r < ITEMS; ++r)
    if (i0 + r * 32 + lane < N) atomicAdd(&start_s[(key[r] >> shift) & (kRadix - 1)], 1u);
  __syncthreads();
  const uint32_t count = tid < kRadix ? start_s[tid] : 0;  // keys of digit tid in this tile
  if (tid < kRadix) st_relaxed(tile_rows + t * kRadix + tid, kReady | count);
  // keys of digit tid in the earlier tiles of its group (wh is the scratch),
  // so that the group's total is published early
  uint32_t* group_rows = tile_rows + a.tiles * kRadix;
  uint32_t* super_rows = group_rows + a.groups * kRadix;
  const int64_t g = t >> kGroupBits, sg = g >> kGroupBits;
  uint32_t before = level_sum(tile_rows, g << kGroupBits, t, wh, a.wc);
  if ((t & 31) == 31 && tid < kRadix) st_relaxed(group_rows + g * kRadix + tid, kReady | (before + count));
  // then everything local to the tile (its ranks, the tile staged in digit
  // order) while the other groups' totals are published
  uint32_t tile_n;
  const uint32_t local_start = block_exclusive_sum(count, warp_tot, &tile_n);
  if (tid < kRadix) start_s[tid] = local_start;
  uint32_t* match = stage_k + warp * kRadix;  // free until the tile is staged: one lane mask per digit and warp
  for (int k = tid; k < kSortWarps * kRadix; k += kSortThreads) {
    (&wh[0][0])[k] = 0;
    stage_k[k] = 0;
  }
  __syncthreads();
  // rank among the same digit within the warp's positions, in order: the
  // lanes holding one digit find each other by OR-ing their bit into the
  // digit's mask (three shared-memory operations instead of eight ballots:
  // the ranking was ALU-bound)
  constexpr bool kRankInSmem = ITEMS > 16;
  uint16_t rank[kRankInSmem ? 1 : ITEMS];
#pragma unroll
  for (int r = 0; r < ITEMS; ++r) {
    const bool valid = i0 + r * 32 + lane < N;
    const uint32_t digit = (key[r] >> shift) & (kRadix - 1);
    if (valid) atomicOr(match + digit, 1u << lane);
    __syncwarp();
    const unsigned peers = valid ? match[digit] : 0u;
    const unsigned lower = __popc(peers & lanemask_lt());
    const uint16_t rk = valid ? static_cast<uint16_t>(wh[warp][digit] + lower) : 0;  // < kWarpSpan
    if constexpr (kRankInSmem)
      rank_s[warp * kWarpSpan + r * 32 + lane] = rk;
    else
      rank[r] = rk;
    __syncwarp();
    if (valid && lower == 0) {
      wh[warp][digit] += __popc(peers);
      match[digit] = 0;
    }
    __syncwarp();
  }
  __syncthreads();
  if (tid < kRadix) {  // per-warp offsets within each digit
    uint32_t run = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = wh[w][tid];
      wh[w][tid] = run;
      run += c;
    }
  }
  __syncthreads();
  // stage the tile in digit order (consecutive positions within a digit)
#pragma unroll
  for (int r = 0; r < ITEMS; ++r) {
    if (i0 + r * 32 + lane < N) {
      const uint32_t digit = (key[r] >> shift) & (kRadix - 1);
      uint32_t rk;
      if constexpr (kRankInSmem)
        rk = rank_s[warp * kWarpSpan + r * 32 + lane];
      else
        rk = rank[r];
      const uint32_t pos = start_s[digit] + wh[warp][digit] + rk;
      stage_k[pos] = key[r];
      stage_v[pos] = val[r];
    }
  }
  __syncthreads();
  // keys of digit tid in the earlier groups and supergroups (wh is the scratch again)
  before += level_sum(group_rows, sg << kGroupBits, g, wh, a.wc);
  if ((t & 1023) == 1023 && tid < kRadix) st_relaxed(super_rows + sg * kRadix + tid, kReady | (before + count));
  before += level_sum(super_rows, 0, sg, wh, a.wc);
  if (tid < kRadix) base_s[tid] += before;
  __syncthreads();
  // coalesced writes: consecutive threads, consecutive destinations within a digit
  for (uint32_t j = tid; j < tile_n; j += kSortThreads) {
    const uint32_t k2 = stage_k[j];
    const uint32_t digit = (k2 >> shift) & (kRadix - 1);
    const uint32_t dst = base_s[digit] + (j - start_s[digit]);
    if (dst < N) {  // always true when the counts are consistent
      kout[dst] = k2;
      vout[dst] = stage_v[j];
    }
  }
}

// ---------------------------------------------------------------------------
// host side: the sort's buffers inside a caller's workspace, and its launches
// ---------------------------------------------------------------------------
inline size_t align256(size_t x) { return (x + 255) & ~size_t{255}; }

struct SortLayout {
  size_t keys[2], vals[2], look, zeroed, zeroed_bytes;
  int64_t tiles, groups, supers;
  int items;  // keys per thread of the sort passes
};

// Places the sort's buffers for N keys at byte offset *off (advanced past them).
inline SortLayout sort_layout(int64_t N, size_t* off) {
  SortLayout L{};
  L.items = sort_items(N);
  const int64_t tile = static_cast<int64_t>(kSortThreads) * L.items;
  L.tiles = (N + tile - 1) / tile;
  L.groups = (L.tiles + 31) >> kGroupBits;
  L.supers = (L.groups + 31) >> kGroupBits;
  auto take = [&](size_t bytes) {
    const size_t at = *off;
    *off = align256(*off + bytes);
    return at;
  };
  for (int b = 0; b < 2; ++b) L.keys[b] = take(sizeof(uint32_t) * N);
  for (int b = 0; b < 2; ++b) L.vals[b] = take(sizeof(uint32_t) * N);
  // the look-back rows are sized for the smaller tiles whatever the tiling,
  // so the workspace never shrinks as N grows (a workspace sized for some N
  // serves every smaller N)
  const int64_t small_tiles = (N + kSortThreads * 8 - 1) / (kSortThreads * 8);
  const int64_t small_groups = (small_tiles + 31) >> kGroupBits, small_supers = (small_groups + 31) >> kGroupBits;
  L.look = take(sizeof(uint32_t) * kRadix * kMaxPasses * static_cast<size_t>(small_tiles + small_groups + small_supers));
  L.zeroed_bytes = sizeof(uint32_t) * (kMaxPasses * kRadix + kMaxPasses + 1);  // totals, tickets, abort word
  L.zeroed = take(L.zeroed_bytes);
  return L;
}

// 8-bit digit passes for keys in [0, num_rows] (num_rows marks a bad row).
inline int sort_passes(int64_t num_rows) {
  int bits = 0;
  while (bits < 32 && (static_cast<uint64_t>(num_rows) >> bits) != 0) ++bits;
  return (bits + 7) / 8 > 1 ? (bits + 7) / 8 : 1;
}

// The call's abort word (non-zero once a wait of the sort gave up).
inline uint32_t* sort_abort_word(const SortLayout& L, unsigned char* ws) {
  return reinterpret_cast<uint32_t*>(ws + L.zeroed) + kMaxPasses * kRadix + kMaxPasses;
}

// Where the sort leaves its result (keys, values) for keys below num_rows.
inline void sorted_result(const SortLayout& L, int64_t num_rows, unsigned char* ws, const uint32_t** keys,
                          const uint32_t** vals) {
  const int b = sort_passes(num_rows) & 1;
  *keys = reinterpret_cast<const uint32_t*>(ws + L.keys[b]);
  *vals = reinterpret_cast<const uint32_t*>(ws + L.vals[b]);
}

// Sorts the N rows (keys in [0, num_rows]; a row outside [0, num_rows)
// becomes the key num_rows) with their hit indices: clear, key_hist, one pass
// per 8-bit digit, all launched with programmatic dependent launch.  On
// success *sorted_keys / *sorted_vals point at the result; run_done (nullable)
// [nwin] is cleared on the way.
inline ple_status_t launch_sort(const int64_t* rows, int64_t N, int64_t num_rows, unsigned char* ws,
                                const SortLayout& L, unsigned int* run_done, int64_t nwin, unsigned int* status,
                                cudaStream_t s, const uint32_t** sorted_keys, const uint32_t** sorted_vals) {
  SortArgs sa{};
  sa.N = N;
  sa.tiles = L.tiles;
  sa.groups = L.groups;
  sa.supers = L.supers;
  for (int b = 0; b < 2; ++b) {
    sa.keys[b] = reinterpret_cast<uint32_t*>(ws + L.keys[b]);
    sa.vals[b] = reinterpret_cast<uint32_t*>(ws + L.vals[b]);
  }
  sa.look = reinterpret_cast<uint32_t*>(ws + L.look);
  sa.hist = reinterpret_cast<uint32_t*>(ws + L.zeroed);
  sa.tickets = sa.hist + kMaxPasses * kRadix;
  sa.wc.status = status;
  sa.wc.abort = sort_abort_word(L, ws);
  sa.wc.wait_ns = wait_limit_ns();
  sa.passes = sort_passes(num_rows);
  cudaError_t e = launch_after(clear_kernel, dim3(1), dim3(kSortThreads), 0, s, sa.hist,
                               static_cast<int>(L.zeroed_bytes / sizeof(uint32_t)));
  if (e != cudaSuccess) return cuda_fail(e);
  // few blocks: each adds its digit counts to the same 256 * passes totals
  int64_t hist_blocks = (N + kSortThreads - 1) / kSortThreads;
  if (hist_blocks > int64_t{2} * sm_count()) hist_blocks = int64_t{2} * sm_count();
  e = launch_after(key_hist_kernel, dim3(static_cast<unsigned>(hist_blocks)), dim3(kSortThreads), 0, s, rows,
                   num_rows, sa, run_done, nwin);
  if (e != cudaSuccess) return cuda_fail(e);
  const size_t smem = sort_pass_smem(L.items);
  if (L.items == 32) {  // more than 48 KB of dynamic shared memory: allowed once per device and context
    static std::atomic<unsigned long long> allowed[64];  // context id + 1, per device
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned long long ctx = 0;
    current_context_id(&ctx);
    if (dev >= 64 || allowed[dev].load(std::memory_order_acquire) != ctx + 1) {
      e = cudaFuncSetAttribute(sort_pass_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(sort_pass_smem(32)));
      if (e != cudaSuccess) return cuda_fail(e);
      if (dev < 64) allowed[dev].store(ctx + 1, std::memory_order_release);
    }
  }
  for (int p = 0; p < sa.passes; ++p) {
    const dim3 grid(static_cast<unsigned>(L.tiles));
    e = L.items == 32   ? launch_after(sort_pass_kernel<32>, grid, dim3(kSortThreads), smem, s, sa, p)
        : L.items == 16 ? launch_after(sort_pass_kernel<16>, grid, dim3(kSortThreads), smem, s, sa, p)
                        : launch_after(sort_pass_kernel<8>, grid, dim3(kSortThreads), smem, s, sa, p);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *sorted_keys = sa.keys[sa.passes & 1];
  *sorted_vals = sa.vals[sa.passes & 1];
  return PLE_OK;
}

}  // namespace
}  // namespace ple

#endif  // PLE_SORT_CUH_
