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
// Pipeline (all in the caller's workspace, no allocation):
//   0. clear_kernel: zeroes the digit totals, the tile tickets and the
//      call's abort word;
//   1. key_hist_kernel: 32-bit keys from the int64 rows (bad rows -> key R)
//      and the digit counts of every radix pass;
//   2. sort_pass_kernel, once per 8-bit digit: LSD radix sort, stable,
//      values = hit index (tiles find their offsets by look-back);
//   3. fold kernel: one warp per window of 32 sorted positions; it folds the
//      chunks that start in its window (a chunk start is a position whose
//      offset from its run's first position is a multiple of 32), adds a
//      whole single-chunk run into table_grad, or stores the chunk sum of a
//      longer run in a slot; the writer that completes a long run (per-run
//      counter) folds that run's chunk sums in order and adds the result;
//   4. finish_long_runs_kernel: the same second level for the runs of more
//      than kLongChunks chunks, which the fold lists instead (hot rows).
//      If a wait of the sort gave up (the call's abort word is set), the
//      fold writes nothing.
// The final add is made once per row by the lanes that own it: a vector fp32
// reduction (red.global.add) when that gives the IEEE sum, else a plain
// IEEE add (subnormals: see the comment above any_tiny), so it is the single
// add table_grad + S_r.
#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "sort.cuh"

namespace ple {
namespace {

constexpr int kChunk = 32;
constexpr uint32_t kNoKey = 0xffffffffu;  // past the end; never a real key
constexpr int kFoldThreads = 256;  // threads per block of the atomic variant

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

// The single final add table_grad[r] + S_r must be the IEEE fp32 add,
// subnormals included, but the fp32 reductions of global memory
// (red.global.add.f32 in every vector width, atomicAdd) flush subnormal
// operands and results to zero on the B200 (checked against IEEE adds on the
// device).  For |x| >= 2^-100 the two agree: a subnormal table_grad value is
// then below half an ulp of x and cannot change the rounded sum, and x + t
// cannot be subnormal unless it is exactly 0 (t and x are then multiples of
// 2^-124).  So the reduction is used when every value of a lane's group is
// at least 2^-100 in magnitude (one integer test per group), and any other
// group (zeros, tiny and subnormal sums, which real gradients almost never
// produce) is added element by element with an IEEE add:
//   - by the deterministic folds, as a plain load, add and store: each row's
//     final add is made once per call, by the lane group that owns the row
//     (a compare-and-swap loop anywhere in the fold kernel made it about 20 %
//     slower, even out of line and never executed);
//   - by the atomic variant, whose hits of one row race, as a
//     compare-and-swap loop around the add.
constexpr uint32_t kExactBelow = 0x0D800000u;  // bits of 2^-100

// True if some |v[q]| < 2^-100 (zeros and subnormals included; NaN is not).
template <int n>
__device__ __forceinline__ bool any_tiny(const float* v) {
  uint32_t m = 0xffffffffu;
#pragma unroll
  for (int q = 0; q < n; ++q) m = min(m, __float_as_uint(v[q]) & 0x7fffffffu);
  return m < kExactBelow;
}

// p += x with an IEEE add; kShared: other threads may add to *p meanwhile.
template <bool kShared>
__device__ __forceinline__ void add_exact(float* p, float x) {
  if constexpr (kShared) {
    unsigned* q = reinterpret_cast<unsigned*>(p);
    unsigned old = __ldcg(q);
    for (;;) {
      const unsigned want = __float_as_uint(__fadd_rn(__uint_as_float(old), x));
      const unsigned seen = atomicCAS(q, old, want);
      if (seen == old) break;
      old = seen;
    }
  } else {
    __stcg(p, __fadd_rn(__ldcg(p), x));
  }
}

__device__ __forceinline__ void red_v4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

template <bool kShared>
__device__ __forceinline__ void red_add1(float* p, float a) {
  if (any_tiny<1>(&a))
    add_exact<kShared>(p, a);
  else
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}

template <bool kShared>
__device__ __forceinline__ void red_add2(float* p, float a, float b) {
  const float v[2] = {a, b};
  if (any_tiny<2>(v)) {
    add_exact<kShared>(p, a);
    add_exact<kShared>(p + 1, b);
  } else {
    asm volatile("red.global.add.v2.f32 [%0], {%1,%2};" ::"l"(p), "f"(a), "f"(b) : "memory");
  }
}

template <bool kShared>
__device__ __forceinline__ void red_add4(float* p, float a, float b, float c, float d) {
  const float v[4] = {a, b, c, d};
  if (any_tiny<4>(v)) {
    add_exact<kShared>(p, a);
    add_exact<kShared>(p + 1, b);
    add_exact<kShared>(p + 2, c);
    add_exact<kShared>(p + 3, d);
  } else {
    red_v4(p, a, b, c, d);
  }
}

// One fp32 reduction per column into table_grad (the single final add of a
// fold, kShared = false; or one hit's add in the atomic variant, kShared).
template <int CPL, bool kShared>
__device__ __forceinline__ void red_add_row(float* __restrict__ tg, int64_t row, int D, const Cols<CPL>& x) {
  const int lane = threadIdx.x & 31;
  if constexpr (CPL == 0) {
#pragma unroll
    for (int k = 0; k < kMaxColsPerLane; ++k)
      if (lane + 32 * k < D) red_add1<kShared>(tg + row * D + lane + 32 * k, x.v[k]);
  } else {
    float* p = tg + row * D + lane * CPL;
    if constexpr (CPL == 1) {
      red_add1<kShared>(p, x.v[0]);
    } else if constexpr (CPL == 2) {
      red_add2<kShared>(p, x.v[0], x.v[1]);
    } else {
#pragma unroll
      for (int k = 0; k < CPL; k += 4) red_add4<kShared>(p + k, x.v[k], x.v[k + 1], x.v[k + 2], x.v[k + 3]);
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

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const unsigned dst = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(gmem_src) : "memory");
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

// Runs longer than 32 hits: each chunk sum goes to a slot; the run is
// identified by its first position s (no two such runs start in one 32-position
// window).  Every chunk writer adds 1 to done[s/32], except the writer of the
// run's last chunk, which knows the run's length and adds kDoneTarget - nc + 1
// instead; so the counter reaches kDoneTarget exactly once, when every chunk
// sum is stored, and the writer that brings it there folds the chunk sums in
// order (second level) and makes the run's single final add.  Nobody waits.
constexpr unsigned kDoneTarget = 1u << 30;

// A run of more than kLongChunks chunks is not finished by the warp that
// completes it (one warp would fold its chunk sums at one short batch per
// memory round trip) but listed for finish_long_runs_kernel.
// (Runs up to this length finish inside the fold at no visible cost: its other warps keep the memory
// busy meanwhile; a 64-chunk threshold cost backward_stress, whose longest runs have 266 chunks, 10 us.)
constexpr int kLongChunks = 512;

struct LongRun {
  int64_t s;     // first sorted position of the run
  int32_t nc;    // its chunks
  uint32_t key;  // its row
};

struct RunBook {
  int* len;               // [windows] run length, written by the last chunk's writer
  unsigned* done;         // [windows] completion counters, cleared before the fold
  const uint32_t* abort;  // the sort's abort word: non-zero, the fold writes nothing
  LongRun* long_runs;     // [long_cap] runs left to finish_long_runs_kernel
  unsigned* long_count;   // their count (cleared with the completion counters)
  unsigned long_cap;
};

// Lists a completed run for finish_long_runs_kernel (by one lane).
__device__ __forceinline__ void list_long_run(const RunBook& rb, int64_t s, int nc, uint32_t key) {
  const unsigned at = atomicAdd(rb.long_count, 1u);
  if (at < rb.long_cap) rb.long_runs[at] = LongRun{s, nc, key};  // (always: long_cap bounds the runs)
}

__device__ __forceinline__ int64_t chunk_slot(int64_t s, int m) {
  return m == 0 ? 2 * (s >> 5) + 1 : 2 * ((s + static_cast<int64_t>(m) * kChunk) >> 5);
}

// Where the sum of chunk [c, nxt) goes: a whole run -> returns true; else the
// chunk-sum slot in *slot.
__device__ __forceinline__ bool chunk_is_whole_run(const Window& W, int c, int nxt, int64_t N, int64_t* slot) {
  const bool is_head = (W.hm >> c) & 1ull;
  const bool run_ends = (W.p0 + nxt >= N) || ((W.hm >> nxt) & 1ull);
  if (is_head && run_ends) return true;
  const int64_t pos = W.p0 + c;
  *slot = 2 * (pos >> 5) + (is_head ? 1 : 0);
  return false;
}

// Called by the lanes `gmask` (leader lane `leader`) after they stored the sum
// of chunk [c, nxt) of a run longer than 32 in its slot.  Returns, to all of
// them, the run's chunk count if this chunk completed the run, else 0.
__device__ __forceinline__ int chunk_stored(const Window& W, int c, int nxt, int64_t N, unsigned gmask, int leader,
                                            const RunBook& rb, int64_t* run_start) {
  const int lane = threadIdx.x & 31;
  const bool run_ends = (W.p0 + nxt >= N) || ((W.hm >> nxt) & 1ull);
  const int64_t s = W.run_start(c);
  *run_start = s;
  __threadfence();  // this lane's part of the chunk sum, before the count
  __syncwarp(gmask);
  int nc = 0;
  if (lane == leader) {
    unsigned inc = 1;
    if (run_ends) {
      const int len = static_cast<int>(W.p0 + nxt - s);
      rb.len[s >> 5] = len;
      __threadfence();
      inc = kDoneTarget - static_cast<unsigned>((len + kChunk - 1) / kChunk) + 1;
    }
    const unsigned old = atomicAdd(rb.done + (s >> 5), inc);
    if (old + inc == kDoneTarget) nc = (__ldcg(rb.len + (s >> 5)) + kChunk - 1) / kChunk;
  }
  nc = __shfl_sync(gmask, nc, leader);
  if (nc) __threadfence();  // the other writers' chunk sums, before reading them
  return nc;
}


// Second level of a long run, by a whole warp after its window is folded:
// the run's chunk sums go through the warp's staging buffer (`stage_vecs`
// 16-byte vectors) by asynchronous copies, a buffer-full per round trip, and
// lane l adds column vectors l, l+32 of them in order; one final reduction.
__device__ void finish_run_staged(const float* csum, int64_t s, int nc, int D, uint32_t key, float* table_grad,
                                  uint4* stage, int stage_vecs) {
  const int lane = threadIdx.x & 31;
  const int vps = D / 4;                 // 16-byte vectors per chunk sum (D <= 256: <= 64)
  const int cap = stage_vecs / vps;      // chunk sums per round (>= 16 for the wide fold's buffers)
  float acc[2][4];
  for (int m0 = 0; m0 < nc; m0 += cap) {
    const int np = min(cap, nc - m0);
    for (int v = lane; v < np * vps; v += 32) {
      const int m = m0 + v / vps, col = v % vps;
      cp_async16(stage + v, csum + chunk_slot(s, m) * D + col * 4);
    }
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    for (int mm = 0; mm < np; ++mm) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int col = lane + 32 * j;
        if (col < vps) {
          const uint4 x = stage[mm * vps + col];
          const float f[4] = {__uint_as_float(x.x), __uint_as_float(x.y), __uint_as_float(x.z), __uint_as_float(x.w)};
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[j][q] = (m0 + mm == 0) ? f[q] : acc[j][q] + f[q];
        }
      }
    }
    __syncwarp();  // the next round overwrites the buffer
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int col = lane + 32 * j;
    if (col < vps)
      red_add4<false>(table_grad + static_cast<int64_t>(key) * D + col * 4, acc[j][0], acc[j][1], acc[j][2],
                      acc[j][3]);
  }
}

// Wide fold.  A grad row spans L lanes that each copy 16 bytes, so one copy
// instruction fetches 32/L rows.  The chunks that start in the window are
// taken in rounds of whole chunks covering at most kWideRows positions (a
// chunk has at most 32 hits, so it never straddles two rounds); the rows of
// a round are staged in shared memory with asynchronous copies in one round
// trip.  The L-lane groups of the warp then fold the round's chunks
// independently from shared memory, each in the fixed order, lane `sub` of a
// group owning CPLN = 16/elem columns; group g takes the chunks that start at
// a position = g modulo the number of groups (32/L), so it only visits its
// own chunks.  A finished chunk that is a whole run is added into
// table_grad by its group; otherwise it goes to its chunk-sum slot.
constexpr int kWideRows = 32;  // staged rows per warp and round

// Columns of the staged grad row that lane `sub` of an L-lane group folds:
// 4-column blocks at 4*sub + 4*L*h, h = 0 .. CPLN/4 - 1 (fp32 grad: one block,
// the lane's own 16 bytes; bf16 grad: two blocks, one from each half of the
// row).  So every 16-byte fp32 reduction instruction of the group covers 4*L
// consecutive columns of the table_grad row: whole sectors.
template <int L, bool BF16>
__device__ __forceinline__ int lane_col(int sub, int q) {  // fp32 column of acc[q], q a multiple of 4
  return 4 * sub + L * q;
}

template <int L, bool BF16>
__device__ __forceinline__ void load_lane_cols(const uint4* row, int sub, float* v) {
  if constexpr (BF16) {
    const uint2* r = reinterpret_cast<const uint2*>(row);  // 4 bf16 per 8 bytes
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint2 y = r[sub + L * h];
      v[4 * h] = bf16_lo(y.x); v[4 * h + 1] = bf16_hi(y.x); v[4 * h + 2] = bf16_lo(y.y); v[4 * h + 3] = bf16_hi(y.y);
    }
  } else {
    const uint4 y = row[sub];
    v[0] = __uint_as_float(y.x); v[1] = __uint_as_float(y.y); v[2] = __uint_as_float(y.z); v[3] = __uint_as_float(y.w);
  }
}

// One warp per block: a block retires as soon as its window is folded, so a
// warp that finishes a long run (its chunk sums folded in order) holds no
// other warp's share of the SM.  Measured on the B200 against 2-8 warps per
// block: backward_stress 279.6 -> 267.5 us, 64-byte rows 213.7 -> 210.6 us,
// the others within 1 %.
template <int L>
__host__ __device__ constexpr int wide_warps() {
  return 1;
}
// per warp after the rows: 64 keys, 64 hit ids, 32 chunk descriptors, 2 pending long runs, a count
constexpr int kWideTail = 64 * 4 + 64 * 4 + 32 * 4 + 48;
constexpr uint32_t kChunkWhole = 1u << 8;  // chunk descriptor: the chunk is a whole run
constexpr uint32_t kChunkSkip = 1u << 9;   // chunk descriptor: rows outside the table (dropped)

template <int L>
__host__ __device__ constexpr size_t wide_smem() {
  return static_cast<size_t>(wide_warps<L>()) * (kWideRows * L * 16 + kWideTail);
}

struct PendingRun {
  int64_t s;
  int nc;
  uint32_t key;
};

// Bits 0, n, 2n, ... of a 64-bit word.
template <int n>
__host__ __device__ constexpr uint64_t every_nth_bit() {
  uint64_t m = 0;
  for (int b = 0; b < 64; b += n) m |= 1ull << b;
  return m;
}

// Resident one-warp blocks per SM: 32 (the SM's block limit; <= 64
// registers) for rows of up to 128 bytes, 24 (<= 85 registers) for larger
// rows, whose staging (up to 17 KB a block) bounds the count first.
template <int L>
__host__ __device__ constexpr int wide_min_blocks() {
  return L <= 8 ? 32 : 24;
}

template <int L, bool BF16>
__global__ void __launch_bounds__(wide_warps<L>() * 32, wide_min_blocks<L>())
fold_wide_kernel(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I, int64_t N, uint32_t bad_key,
                 const void* __restrict__ grad, int D, float* __restrict__ table_grad, float* __restrict__ csum,
                 const RunBook rb) {
  constexpr int RPI = 32 / L;         // rows per copy instruction = lane groups per warp
  constexpr int CPLN = BF16 ? 8 : 4;  // fp32 columns per lane
  extern __shared__ __align__(16) unsigned char wide_smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / L, sub = lane % L;
  uint4* rows_s = reinterpret_cast<uint4*>(wide_smem_raw + warp * (kWideRows * L * 16 + kWideTail));
  uint32_t* keys_s = reinterpret_cast<uint32_t*>(rows_s + kWideRows * L);  // 64 keys
  uint32_t* ids_s = keys_s + 64;                                           // 64 hit ids
  uint32_t* desc_s = ids_s + 64;                                           // 32 chunk descriptors
  PendingRun* pend = reinterpret_cast<PendingRun*>(desc_s + 32);           // long runs this warp completed
  int* npend = reinterpret_cast<int*>(pend + 2);
  const int64_t w = static_cast<int64_t>(blockIdx.x) * wide_warps<L>() + warp;
  wait_for_prior_grid();
  allow_next_grid();
  if (w * 32 >= N) return;
  const uint32_t aborted = ld_relaxed(rb.abort);  // (in flight with the window's loads)
  Window W;
  const bool any = window_setup(K, I, N, w, W);
  if (!any || aborted != 0) return;  // nothing to fold, or the sort gave up: no write at all
  const size_t row_bytes = static_cast<size_t>(D) * (BF16 ? 2 : 4);
  const unsigned char* gbase = static_cast<const unsigned char*>(grad) + sub * 16;
  keys_s[lane] = W.kA;
  keys_s[32 + lane] = W.kB;
  ids_s[lane] = W.iA;
  ids_s[32 + lane] = W.iB;
  if (lane == 0) *npend = 0;
  __syncwarp();

  const uint64_t in_range = (W.b >= 64 ? ~0ull : ((1ull << W.b) - 1)) & ~((1ull << W.a) - 1);
  uint64_t rem = W.cm & in_range;  // chunk starts still to fold
  while (rem) {
    // the round: whole chunks from the first remaining start, at most kWideRows positions
    const int r0 = __ffsll(static_cast<long long>(rem)) - 1;
    int r1 = W.b;
    if (W.b - r0 > kWideRows) {
      const uint64_t later = rem & ~(1ull << r0) & ((2ull << (r0 + kWideRows)) - 1);
      r1 = 63 - __clzll(later);  // a later chunk start within reach exists: chunks are <= 32 long
    }
    for (int e = r0 + grp; e < r1; e += RPI) {
      const uint32_t id = ids_s[e];  // < N for a sorted workspace; kept inside grad_out whatever it holds
      cp_async16(rows_s + (e - r0) * L + sub, gbase + static_cast<size_t>(id < N ? id : 0) * row_bytes);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    const uint64_t starts = rem & ((r1 >= 64 ? ~0ull : ((1ull << r1) - 1)));
    rem &= ~starts;
    // chunk starts of the round relative to r0 (a round spans at most 32 positions); lane j
    // describes the chunk starting at r0 + j (while the rows are on their way): where it ends,
    // whether it is a whole run, whether its rows are outside the table
    const uint32_t st32 = static_cast<uint32_t>(starts >> r0);
    if ((st32 >> lane) & 1u) {
      const uint32_t above = st32 & ~((2u << lane) - 1u);  // (lane 31: 2u << 31 wraps to 0, nothing above)
      const int nrel = above ? __ffs(above) - 1 : r1 - r0;
      const int c = r0 + lane, nxt = r0 + nrel;
      const bool is_head = (W.hm >> c) & 1ull;
      const bool run_ends = (W.p0 + nxt >= N) || ((W.hm >> nxt) & 1ull);  // nxt < 64 unless the data ends there
      desc_s[lane] = static_cast<uint32_t>(nrel) | (is_head && run_ends ? kChunkWhole : 0u) |
                     (keys_s[c] >= bad_key ? kChunkSkip : 0u);
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    // this group's chunks: those starting at a position = grp mod RPI (relative position
    // j = c - r0, so j = grp - r0 mod RPI)
    uint32_t mine = st32 & static_cast<uint32_t>(every_nth_bit<RPI>() >> ((r0 - grp) & (RPI - 1)));
    while (mine) {
      const int j = __ffs(mine) - 1;
      mine &= mine - 1;
      const uint32_t dsc = desc_s[j];
      if (dsc & kChunkSkip) continue;
      const int nrel = static_cast<int>(dsc & 0xFFu);
      float acc[CPLN];
      load_lane_cols<L, BF16>(rows_s + j * L, sub, acc);
      for (int e = j + 1; e < nrel; ++e) {
        float v[CPLN];
        load_lane_cols<L, BF16>(rows_s + e * L, sub, v);
#pragma unroll
        for (int q = 0; q < CPLN; ++q) acc[q] = acc[q] + v[q];
      }
      const int c = r0 + j;
      const uint32_t key = keys_s[c];
      if (dsc & kChunkWhole) {
        float* dst = table_grad + static_cast<int64_t>(key) * D;
        if (!any_tiny<CPLN>(acc)) {
#pragma unroll
          for (int q = 0; q < CPLN; q += 4)
            red_v4(dst + lane_col<L, BF16>(sub, q), acc[q], acc[q + 1], acc[q + 2], acc[q + 3]);
        } else {
#pragma unroll
          for (int q = 0; q < CPLN; ++q) add_exact<false>(dst + lane_col<L, BF16>(sub, q & ~3) + (q & 3), acc[q]);
        }
      } else {
        const int nxt = r0 + nrel;
        const bool is_head = (W.hm >> c) & 1ull;
        const int64_t slot = 2 * ((W.p0 + c) >> 5) + (is_head ? 1 : 0);
        float* dst = csum + slot * D;
#pragma unroll
        for (int q = 0; q < CPLN; q += 4)
          *reinterpret_cast<float4*>(dst + lane_col<L, BF16>(sub, q)) =
              make_float4(acc[q], acc[q + 1], acc[q + 2], acc[q + 3]);
        const unsigned gmask = L == 32 ? kFull : (((1u << L) - 1u) << (grp * L));
        int64_t s = 0;
        const int nc = chunk_stored(W, c, nxt, N, gmask, grp * L, rb, &s);
        if (nc && sub == 0) {  // this chunk completed a long run
          if (nc > kLongChunks) {
            list_long_run(rb, s, nc, key);
          } else {  // fold it once the window is done
            const int at = atomicAdd(npend, 1);  // at most 2: a window holds chunks of at most 2 long runs
            if (at < 2) pend[at] = PendingRun{s, nc, key};
          }
        }
      }
    }
    __syncwarp();  // the next round reuses the staging buffer and the descriptors
  }
  const int n = min(*npend, 2);
  for (int q = 0; q < n; ++q)
    finish_run_staged(csum, pend[q].s, pend[q].nc, D, pend[q].key, table_grad, rows_s, kWideRows * L);
}

// Resident one-warp blocks per SM of the generic fold (<= 85 registers).
// One warp per block, as in the wide fold: a block retires as soon as its
// window is folded.  Measured on the B200 against 8-warp blocks: the
// gradient at D = 96 998.5 -> 795.6 us, D = 40 779.3 -> 650.3 us, D = 200
// 1328.3 -> 1201.2 us (same bits).
constexpr int kGenericBlocks = 24;

// Generic fold for row sizes the wide fold does not cover: lanes own
// columns l, l+32, ... of every row; one warp-wide load per hit.
template <bool BF16>
__global__ void __launch_bounds__(32, kGenericBlocks)
fold_generic_kernel(const uint32_t* __restrict__ K, const uint32_t* __restrict__ I, int64_t N, uint32_t bad_key,
                    const void* __restrict__ grad, int D, float* __restrict__ table_grad, float* __restrict__ csum,
                    const RunBook rb) {
  constexpr int kBatch = 4;
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x);  // one warp per block, one window per warp
  wait_for_prior_grid();
  allow_next_grid();
  if (w * 32 >= N) return;
  const uint32_t aborted = ld_relaxed(rb.abort);
  Window W;
  const bool any = window_setup(K, I, N, w, W);
  if (!any || aborted != 0) return;
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
        const uint32_t id = e < 32 ? ia : ib;
        load_cols<0, BF16>(grad, id < N ? id : 0, D, g[u]);
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
          if (key < bad_key) {
            int64_t slot = 0;
            if (chunk_is_whole_run(W, c, nxt, N, &slot)) {
              red_add_row<0, false>(table_grad, key, D, acc);
            } else {
              store_slot<0>(csum, slot, D, acc);
              int64_t s = 0;
              const int nc = chunk_stored(W, c, nxt, N, kFull, 0, rb, &s);
              if (nc > kLongChunks) {
                if (lane == 0) list_long_run(rb, s, nc, key);
              } else if (nc) {  // second level by the whole warp, lanes owning columns l, l+32, ...
                Cols<0> sum;
#pragma unroll
                for (int q = 0; q < Cols<0>::n; ++q) {
                  const int d = lane + 32 * q;
                  sum.v[q] = d < D ? __ldcg(csum + chunk_slot(s, 0) * D + d) : 0.f;
                }
                for (int m = 1; m < nc; ++m) {
#pragma unroll
                  for (int q = 0; q < Cols<0>::n; ++q) {
                    const int d = lane + 32 * q;
                    if (d < D) sum.v[q] = sum.v[q] + __ldcg(csum + chunk_slot(s, m) * D + d);
                  }
                }
                red_add_row<0, false>(table_grad, key, D, sum);
              }
            }
          }
        }
      }
    }
  }
}

// Second level of the listed long runs.  One block per (run, 32-column
// slice): lane l of warp 0 owns column 32 g + l and adds the run's chunk sums
// in order, left to right from the first (the order finish_run_staged uses),
// then makes the run's single final add into table_grad.  All eight warps
// stream the slice's chunk sums into a ring of kFinStages stages of
// kFinStage slices in shared memory with asynchronous copies, kFinStages - 1
// stages ahead (one warp alone keeps too few copies in flight), and the
// slices of one run go to different SMs.
constexpr int kFinThreads = 256;
constexpr int kFinStage = 128;  // chunk sums per stage
constexpr int kFinStages = 3;   // stages in the ring: 3 * 128 slices of 128 bytes = 48 KB
constexpr size_t kFinSmem = static_cast<size_t>(kFinStages) * kFinStage * 32 * sizeof(float);

__global__ void __launch_bounds__(kFinThreads)
finish_long_runs_kernel(const LongRun* __restrict__ runs, const unsigned* __restrict__ count, unsigned cap,
                        const float* __restrict__ csum, int D, float* __restrict__ table_grad,
                        const uint32_t* abort) {
  extern __shared__ __align__(16) float fin_ring[];  // [kFinStages][kFinStage][32]
  wait_for_prior_grid();
  if (ld_relaxed(abort) != 0) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int groups = (D + 31) / 32;
  const int64_t items = static_cast<int64_t>(min(ld_relaxed(count), cap)) * groups;  // (count <= cap)
  for (int64_t item = blockIdx.x; item < items; item += gridDim.x) {
    const LongRun run = runs[item / groups];
    const int c0 = 32 * static_cast<int>(item % groups);
    const int cols = min(32, D - c0);  // a multiple of 4: grad rows are 16-byte multiples
    const int vps = cols / 4;          // 16-byte vectors per slice
    const int64_t nst = (run.nc + kFinStage - 1) / kFinStage;
    auto load_stage = [&](int64_t k) {  // chunk sums k*S .. k*S+S-1 into stage k mod kFinStages
      float* st = fin_ring + (k % kFinStages) * kFinStage * 32;
      for (int idx = tid; idx < kFinStage * vps; idx += kFinThreads) {
        const int i = idx / vps, v = idx - i * vps;
        const int64_t m = k * kFinStage + i;
        if (m < run.nc)
          cp_async16(st + i * 32 + 4 * v, csum + chunk_slot(run.s, static_cast<int>(m)) * D + c0 + 4 * v);
      }
    };
    for (int64_t k = 0; k < kFinStages - 1; ++k) {
      if (k < nst) load_stage(k);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    float acc = 0.f;
    for (int64_t k = 0; k < nst; ++k) {
      if (k + kFinStages - 1 < nst) load_stage(k + kFinStages - 1);  // into the stage read at k - 1
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group %0;" ::"n"(kFinStages - 1) : "memory");  // this thread's part of stage k
      __syncthreads();                                                            // everyone's part
      if (warp == 0 && lane < cols) {
        const float* st = fin_ring + (k % kFinStages) * kFinStage * 32;
        const int cnt = static_cast<int>(min(static_cast<int64_t>(kFinStage), run.nc - k * kFinStage));
        for (int i = 0; i < cnt; ++i) acc = (k == 0 && i == 0) ? st[i * 32 + lane] : acc + st[i * 32 + lane];
      }
      __syncthreads();  // the stage just read is refilled two iterations on
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    if (warp == 0 && lane < cols) red_add1<false>(table_grad + static_cast<int64_t>(run.key) * D + c0 + lane, acc);
    __syncthreads();  // the next item's first stages overwrite the ring
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
    red_add_row<CPL, true>(table_grad, r, D, x);
  }
  if (bad && (threadIdx.x & 31) == 0) raise_flag(status, PLE_ERR_BAD_ROW);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct Layout {
  SortLayout sort;
  size_t csum, run_len, run_done, long_runs, total_bytes;
  int64_t nwin, long_cap;
};

Layout layout_for(int64_t N, int D) {
  Layout L{};
  L.nwin = (N + 31) / 32;
  size_t off = 0;
  L.sort = sort_layout(N, &off);
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L.csum = take(sizeof(float) * 2 * static_cast<size_t>(L.nwin) * D);
  L.run_len = take(sizeof(int) * L.nwin);
  L.run_done = take(sizeof(unsigned int) * (L.nwin + 1));  // + the long-run count
  L.long_cap = L.nwin / (kLongChunks + 1) + 1;  // a long run spans more than kLongChunks windows
  L.long_runs = take(sizeof(LongRun) * static_cast<size_t>(L.long_cap));
  L.total_bytes = off;
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
  return layout_for(N, plan->head_dim).total_bytes;
}

}  // extern "C"

namespace {

// The deterministic gradient with an explicit row bound: rows in
// [0, num_rows) are summed into table_grad [num_rows, head_dim], others are
// dropped (and flagged).  The phases: kPrepare sorts the rows into the
// workspace (it does not read grad_out); kApply folds grad_out in the
// sorted order (it does not read the rows); kBoth does both in order.
enum Phase { kPrepare = 1, kApply = 2, kBoth = 3 };

ple_status_t grad_scatter_bounded(const ple_plan_t* plan, const int64_t* rows, int64_t N, int64_t num_rows,
                                  const void* grad, ple_dtype_t gdt, float* table_grad, void* workspace,
                                  size_t ws_bytes, void* stream, int phases = kBoth) {
  if (plan == nullptr || N < 0) return PLE_ERR_INVALID_ARG;
  if ((phases & kApply) && gdt != PLE_F32 && gdt != PLE_BF16) return PLE_ERR_INVALID_ARG;
  if (N == 0) return PLE_OK;
  if ((phases & kPrepare) && rows == nullptr) return PLE_ERR_INVALID_ARG;
  if ((phases & kApply) && (grad == nullptr || table_grad == nullptr)) return PLE_ERR_INVALID_ARG;
  if (plan->head_dim > 32 * kMaxColsPerLane) return PLE_ERR_UNSUPPORTED;
  if ((phases & kPrepare) && !aligned(rows, 8)) return PLE_ERR_ALIGNMENT;
  if ((phases & kApply) && (!aligned(grad, 16) || !aligned(table_grad, 16) ||
                            (static_cast<int64_t>(plan->head_dim) * (gdt == PLE_F32 ? 4 : 2)) % 16 != 0))
    return PLE_ERR_ALIGNMENT;
  if (num_rows < 1) return PLE_ERR_INVALID_ARG;
  if (num_rows >= static_cast<int64_t>(kNoKey) || N >= (int64_t{1} << 31)) return PLE_ERR_UNSUPPORTED;
  const int D = plan->head_dim;
  const Layout L = layout_for(N, D);
  if (workspace == nullptr || ws_bytes < L.total_bytes) return PLE_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return PLE_ERR_ALIGNMENT;
  cudaError_t e;
  unsigned int* status = status_word(plan, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  auto* ws = static_cast<unsigned char*>(workspace);
  const auto s = static_cast<cudaStream_t>(stream);
  float* csum = reinterpret_cast<float*>(ws + L.csum);
  RunBook rb;
  rb.len = reinterpret_cast<int*>(ws + L.run_len);
  rb.done = reinterpret_cast<unsigned int*>(ws + L.run_done);
  rb.abort = sort_abort_word(L.sort, ws);
  rb.long_count = rb.done + L.nwin;
  rb.long_runs = reinterpret_cast<LongRun*>(ws + L.long_runs);
  rb.long_cap = static_cast<unsigned>(L.long_cap);
  const uint32_t* Ks = nullptr;
  const uint32_t* Is = nullptr;
  if (phases & kPrepare) {
    ple_status_t st = launch_sort(rows, N, num_rows, ws, L.sort, rb.done, L.nwin + 1, status, s, &Ks, &Is);
    if (st != PLE_OK) return st;
    if (!(phases & kApply)) return check_launch();
  } else {
    sorted_result(L.sort, num_rows, ws, &Ks, &Is);
  }
  const uint32_t bad_key = static_cast<uint32_t>(num_rows);
  const dim3 fold_grid(static_cast<unsigned>(L.nwin));  // the generic fold: one warp per block
  const bool bf = gdt == PLE_BF16;
  const int lanes_per_row = static_cast<int>(static_cast<int64_t>(D) * (bf ? 2 : 4) / 16);
  auto fold = [&](auto kernel, dim3 grid, int threads, size_t smem) {
    return launch_after(kernel, grid, dim3(threads), smem, s, Ks, Is, N, bad_key, grad, D, table_grad, csum, rb);
  };
#define PLE_WIDE(LW, BF)                                                                                  \
  case 2 * LW + BF:                                                                                       \
    e = fold(fold_wide_kernel<LW, BF>,                                                                    \
             dim3(static_cast<unsigned>((L.nwin + wide_warps<LW>() - 1) / wide_warps<LW>())),            \
             wide_warps<LW>() * 32, wide_smem<LW>());                                                     \
    break;
  switch (lanes_per_row * 2 + (bf ? 1 : 0)) {
    PLE_WIDE(1, 0) PLE_WIDE(1, 1) PLE_WIDE(2, 0) PLE_WIDE(2, 1) PLE_WIDE(4, 0) PLE_WIDE(4, 1)
    PLE_WIDE(8, 0) PLE_WIDE(8, 1) PLE_WIDE(16, 0) PLE_WIDE(16, 1) PLE_WIDE(32, 0) PLE_WIDE(32, 1)
    default:
      e = bf ? fold(fold_generic_kernel<true>, fold_grid, 32, 0)
             : fold(fold_generic_kernel<false>, fold_grid, 32, 0);
  }
#undef PLE_WIDE
  if (e != cudaSuccess) return cuda_fail(e);
  // the long runs the fold listed (none in most calls: the blocks read the count and return)
  const int64_t items = L.long_cap * ((D + 31) / 32);
  const unsigned fin_blocks = static_cast<unsigned>(std::min<int64_t>(items, sm_count()));
  e = launch_after(finish_long_runs_kernel, dim3(fin_blocks), dim3(kFinThreads), kFinSmem, s,
                   static_cast<const LongRun*>(rb.long_runs), static_cast<const unsigned*>(rb.long_count),
                   rb.long_cap, static_cast<const float*>(csum), D, table_grad, rb.abort);
  if (e != cudaSuccess) return cuda_fail(e);
  return check_launch();
}

}  // namespace

extern "C" {

ple_status_t ple_grad_scatter(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* grad,
                              ple_dtype_t gdt, float* table_grad, void* workspace, size_t ws_bytes,
                              void* stream) {
  if (plan == nullptr) return PLE_ERR_INVALID_ARG;
  return grad_scatter_bounded(plan, rows, N, plan->num_rows, grad, gdt, table_grad, workspace, ws_bytes, stream);
}

ple_status_t ple_grad_prepare(const ple_plan_t* plan, const int64_t* rows, int64_t N, void* workspace,
                              size_t ws_bytes, void* stream) {
  if (plan == nullptr) return PLE_ERR_INVALID_ARG;
  return grad_scatter_bounded(plan, rows, N, plan->num_rows, nullptr, PLE_F32, nullptr, workspace, ws_bytes, stream,
                              kPrepare);
}

ple_status_t ple_grad_apply(const ple_plan_t* plan, int64_t N, const void* grad, ple_dtype_t gdt, float* table_grad,
                            void* workspace, size_t ws_bytes, void* stream) {
  if (plan == nullptr) return PLE_ERR_INVALID_ARG;
  return grad_scatter_bounded(plan, nullptr, N, plan->num_rows, grad, gdt, table_grad, workspace, ws_bytes, stream,
                              kApply);
}

ple_status_t ple_grad_scatter_cache(const ple_plan_t* plan, const int64_t* slots, int64_t N, const void* grad,
                                    ple_dtype_t gdt, float* cache_grad, int64_t cache_rows, void* workspace,
                                    size_t ws_bytes, void* stream) {
  if (plan == nullptr) return PLE_ERR_INVALID_ARG;
  return grad_scatter_bounded(plan, slots, N, cache_rows, grad, gdt, cache_grad, workspace, ws_bytes, stream);
}

ple_status_t ple_grad_scatter_atomic(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* grad,
                                     ple_dtype_t gdt, float* table_grad, void* stream) {
  ple_status_t st = check_grad_args(plan, rows, N, grad, gdt, table_grad);
  if (st != PLE_OK || N == 0) return st;
  cudaError_t e;
  unsigned int* status = status_word(plan, static_cast<cudaStream_t>(stream), &e);
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

// Device address of g_noalloc_scratch, one per device, with the id of the
// context it was looked up in.  In host code the array's name only stands in
// for the symbol; its device address has to be looked up with that device
// current, and again when the runtime has loaded the module into a new
// context (after cudaDeviceReset).
std::atomic<void*> g_noalloc_addr[64];
std::atomic<unsigned long long> g_noalloc_ctx[64];

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
  unsigned long long ctx = 0;
  const bool have_ctx = current_context_id(&ctx);
  void* scratch = g_noalloc_addr[dev].load(std::memory_order_acquire);
  if (scratch == nullptr || (have_ctx && g_noalloc_ctx[dev].load(std::memory_order_acquire) != ctx)) {
    // first call on this device (or in a new context): look the address up
    e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned long long now = 0;
    if (current_context_id(&now)) g_noalloc_ctx[dev].store(now, std::memory_order_relaxed);
    g_noalloc_addr[dev].store(scratch, std::memory_order_release);
  }
  return ple_grad_scatter(plan, rows, N, grad, gdt, table_grad, scratch, kNoAllocScratchBytes, stream);
}

size_t ple_grad_scatter_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

}  // extern "C"
