// Forward path: row hashing (_hash_input_ids), the fused hash + row gather
// (forward of Qwen3_8_FlashNextNGramEmbedding) and the plain row gather
// (_lookup_ngram_ids), NeMo AutoModel engram API page.
//
// The gather is HBM-bound: every hit reads one table row and writes one
// output row.  A block stages the byte offsets of its hits in shared memory,
// then streams the rows as flat 16-byte vectors: vector q of the block's
// output is column (q mod V) of hit (q div V), V = row_bytes / 16, so the
// stores of a warp are contiguous and each row is read by V consecutive
// lanes.  UNROLL independent loads are in flight per thread before the
// matching stores are issued.  An fp8 E4M3 table is widened to bf16 on the
// way (8 bytes of codes in, 16 bytes of bf16 out per unit).
#include <atomic>

#include "common.cuh"

namespace ple {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kBlock = 256;     // threads per block of the gather kernels
constexpr int kUnroll = 8;      // 16-byte loads in flight per thread
constexpr int kHashWarps = 4;   // warps per block of the stand-alone hash

// Block 0 checks cu_seqlens once per launch: cu[0] == 0, cu[S] == T and
// non-decreasing.  Bad input only raises a flag; all indexing stays in range.
__device__ void check_seqlens(const int32_t* __restrict__ cu, int32_t num_seqs, int64_t T,
                              unsigned int* status) {
  if (blockIdx.x != 0) return;
  bool bad = false;
  if (threadIdx.x == 0) bad = (cu[0] != 0) || (static_cast<int64_t>(cu[num_seqs]) != T);
  for (int32_t s = threadIdx.x; s < num_seqs; s += blockDim.x) bad |= cu[s + 1] < cu[s];
  if (bad) raise_flag(status, PLE_ERR_BAD_SEQLENS);
}

// Order hashes h_2..h_n of token t, the token of this lane.  Called by a
// whole warp; lanes hold consecutive tokens (valid lanes form a prefix).
// The previous tokens come from lower lanes by shuffle; the first k lanes
// load the k-token halo before the warp's first token from global memory.
// Context slot k is kept while position t-k is inside t's packed sequence
// and no EOS sits in positions t-k .. t-1; otherwise it and every slot
// beyond it hold the sentinel 0.
__device__ __forceinline__ void order_hashes(const HashParams& hp, const int64_t* __restrict__ tokens,
                                             const int32_t* __restrict__ cu, int32_t num_seqs, int64_t t,
                                             bool valid, int64_t (&hs)[kMaxOrder - 1]) {
  const int lane = threadIdx.x & 31;
  const int64_t tok = valid ? tokens[t] : 0;
  // the halo (tokens before the warp's first) is loaded together with the
  // lane's own token, ahead of the segment search: one round trip, not two
  int64_t halo[kMaxOrder];
#pragma unroll
  for (int k = 1; k < kMaxOrder; ++k)
    halo[k] = (k < hp.ngram_size && lane < k && valid && t - k >= 0) ? tokens[t - k] : 0;
  const int64_t seq_start = valid ? static_cast<int64_t>(cu[find_sequence(cu, num_seqs, t)]) : 0;
  uint64_t h = static_cast<uint64_t>(tok) * static_cast<uint64_t>(hp.mults[0]);
  bool keep = valid;
#pragma unroll
  for (int k = 1; k < kMaxOrder; ++k) {
    if (k < hp.ngram_size) {
      int64_t prev = __shfl_up_sync(kFull, tok, k);
      if (lane < k) prev = halo[k];
      keep = keep && (t - k >= seq_start) && (prev != hp.eos_id);
      const int64_t ctx = keep ? prev : 0;
      h += static_cast<uint64_t>(ctx) * static_cast<uint64_t>(hp.mults[k]);
      hs[k - 1] = static_cast<int64_t>(h);
    }
  }
}

// Same order hashes for a lane whose token is not the next position after
// the previous lane's (slices cross row boundaries): every preceding token is
// loaded from global memory.
__device__ __forceinline__ void order_hashes_direct(const HashParams& hp, const int64_t* __restrict__ tokens,
                                                    const int32_t* __restrict__ cu, int32_t num_seqs, int64_t t,
                                                    bool valid, int64_t (&hs)[kMaxOrder - 1]) {
  const int64_t tok = valid ? tokens[t] : 0;
  const int64_t seq_start = valid ? static_cast<int64_t>(cu[find_sequence(cu, num_seqs, t)]) : 0;
  uint64_t h = static_cast<uint64_t>(tok) * static_cast<uint64_t>(hp.mults[0]);
  bool keep = valid;
#pragma unroll
  for (int k = 1; k < kMaxOrder; ++k) {
    if (k < hp.ngram_size) {
      keep = keep && (t - k >= seq_start) && (t - k >= 0);
      const int64_t prev = keep ? tokens[t - k] : 0;
      keep = keep && (prev != hp.eos_id);
      const int64_t ctx = keep ? prev : 0;
      h += static_cast<uint64_t>(ctx) * static_cast<uint64_t>(hp.mults[k]);
      hs[k - 1] = static_cast<int64_t>(h);
    }
  }
}

// rows of the tokens of this lane for every head, head j of order 2 + j/G.
template <typename Emit>
__device__ __forceinline__ void rows_of_token(const HashParams& hp, const HeadConst* consts,
                                              const int64_t (&hs)[kMaxOrder - 1], Emit emit) {
  const int G = hp.heads_per_ngram;
#pragma unroll
  for (int m = 0; m < kMaxOrder - 1; ++m) {
    if (m < hp.ngram_size - 1) {
      for (int g = 0; g < G; ++g) {
        const int j = m * G + g;
        const HeadConst c = consts[j];
        emit(j, c.offset + static_cast<int64_t>(floor_mod(hs[m], c)));
      }
    }
  }
}

__device__ __forceinline__ void load_consts(const HashParams& hp, HeadConst* consts) {
  for (int j = threadIdx.x; j < hp.num_heads; j += blockDim.x) consts[j] = hp.head[j];
}

// ---------------------------------------------------------------------------
// Stand-alone hash: one warp per 32 tokens, staged through shared memory so
// that the int64 [T, H] rows are written with coalesced stores.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kHashWarps * 32)
hash_kernel(const HashParams hp, const int64_t* __restrict__ tokens, int64_t T,
            const int32_t* __restrict__ cu, int32_t num_seqs, int64_t* __restrict__ rows,
            unsigned int* status) {
  extern __shared__ __align__(16) unsigned char smem[];
  HeadConst* consts = reinterpret_cast<HeadConst*>(smem);
  const int H = hp.num_heads;
  int64_t* stage = reinterpret_cast<int64_t*>(consts + H) + (threadIdx.x >> 5) * 32 * H;
  load_consts(hp, consts);
  check_seqlens(cu, num_seqs, T, status);
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int64_t t_first = (static_cast<int64_t>(blockIdx.x) * kHashWarps + (threadIdx.x >> 5)) * 32;
  if (t_first >= T) return;
  const int64_t t = t_first + lane;
  const bool valid = t < T;
  int64_t hs[kMaxOrder - 1];
  order_hashes(hp, tokens, cu, num_seqs, t, valid, hs);
  rows_of_token(hp, consts, hs, [&](int j, int64_t row) { stage[lane * H + j] = row; });
  __syncwarp();
  const int n = static_cast<int>(min(static_cast<int64_t>(32), T - t_first)) * H;
  int64_t* dst = rows + t_first * H;
  for (int q = lane; q < n; q += 32) dst[q] = stage[q];
}

// ---------------------------------------------------------------------------
// Row streaming shared by the fused lookup and the gather: `lanes` threads
// (a warp or a block) copy nhits rows, vector q of the output being column
// q mod V of hit q div V (V = row bytes / 16).
// ---------------------------------------------------------------------------
template <int VL, int kLanes>
__device__ __forceinline__ void copy_hits(const unsigned char* __restrict__ table,
                                          const int64_t* __restrict__ rowoff, int nhits, int v_rt,
                                          unsigned char* __restrict__ out, int tid) {
  const int V = VL >= 0 ? (1 << VL) : v_rt;
  const int total = nhits * V;
  for (int base = tid; base < total; base += kLanes * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int q = base + u * kLanes;
      if (q < total) {
        const int hit = VL >= 0 ? (q >> VL) : q / V;
        const int col = q - hit * V;
        const int64_t off = rowoff[hit];
        v[u] = off >= 0 ? ld_nc(table + off + col * 16) : make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int q = base + u * kLanes;
      if (q < total) st_cs(out + static_cast<int64_t>(q) * 16, v[u]);
    }
  }
}

// E4M3 -> bf16 widening, two codes per 32-bit word, on the integer and
// bf16x2 pipes.  For a code c = S.EEEE.MMM the pattern S.0000EEEE.MMM0000
// read as bf16 is (-1)^S 2^(E-127) (1 + M/8) for E > 0 and the subnormal
// (-1)^S (M/8) 2^-126 for E = 0; one exact bf16 multiply by 2^120 turns both
// into the E4M3 value (bias 7: 2^(E-7) (1 + M/8), and M 2^-9).  The two NaN
// codes S.1111.111 would come out as +-480; they are patched to S | 0x7FC0.
constexpr uint32_t kBf16x2Two120 = 0x7B807B80u;  // {2^120, 2^120}

__device__ __forceinline__ uint32_t e4m3_pair_to_bf16x2(uint32_t codes4, int pair) {
  // a = {c_lo, c_hi} in the low byte of each half; b = the same in the high byte
  const uint32_t a = __byte_perm(codes4, 0, pair ? 0x4342 : 0x4140);
  const uint32_t b = __byte_perm(codes4, 0, pair ? 0x3424 : 0x1404);
  const uint32_t x = ((a << 4) & 0x07F007F0u) | (b & 0x80008000u);
  uint32_t y;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(y) : "r"(x), "r"(kBf16x2Two120));
  return y;
}

// The NaN patch of one pair (rare path).
__device__ __noinline__ uint32_t e4m3_pair_nan_patch(uint32_t codes4, int pair, uint32_t y) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t c = (codes4 >> (16 * pair + 8 * h)) & 0xFFu;
    if ((c & 0x7Fu) == 0x7Fu) y = (y & (0xFFFF0000u >> (16 * h))) | ((((c & 0x80u) << 8) | 0x7FC0u) << (16 * h));
  }
  return y;
}

// Eight codes to eight bf16 values (one 16-byte store).
__device__ __forceinline__ uint4 widen8(const uint2 c) {
  uint4 o = make_uint4(e4m3_pair_to_bf16x2(c.x, 0), e4m3_pair_to_bf16x2(c.x, 1), e4m3_pair_to_bf16x2(c.y, 0),
                       e4m3_pair_to_bf16x2(c.y, 1));
  // a byte b with (b & 0x7F) == 0x7F becomes 0x80 after +1 on its low 7 bits
  const uint32_t nan = (((c.x & 0x7F7F7F7Fu) + 0x01010101u) | ((c.y & 0x7F7F7F7Fu) + 0x01010101u)) & 0x80808080u;
  if (nan != 0) {
    o.x = e4m3_pair_nan_patch(c.x, 0, o.x);
    o.y = e4m3_pair_nan_patch(c.x, 1, o.y);
    o.z = e4m3_pair_nan_patch(c.y, 0, o.z);
    o.w = e4m3_pair_nan_patch(c.y, 1, o.w);
  }
  return o;
}

// Widening variant of copy_hits for an E4M3 table: the unit is 8 bytes of
// codes (V8 = row bytes / 8 per row) and becomes one 16-byte bf16 store at
// byte 16 q of the output, so the stores of a warp stay contiguous.  Twice
// as many units as vectors: twice the unroll keeps the bytes in flight.
constexpr int kWidenUnroll = 2 * kUnroll;

template <int VL, int kLanes>
__device__ __forceinline__ void widen_hits(const unsigned char* __restrict__ table,
                                           const int64_t* __restrict__ rowoff, int nhits, int v_rt,
                                           unsigned char* __restrict__ out, int tid) {
  constexpr int VL8 = VL >= 0 ? VL + 1 : -1;
  const int V = VL8 >= 0 ? (1 << VL8) : 2 * v_rt;
  const int total = nhits * V;
  for (int base = tid; base < total; base += kLanes * kWidenUnroll) {
    uint2 v[kWidenUnroll];
#pragma unroll
    for (int u = 0; u < kWidenUnroll; ++u) {
      const int q = base + u * kLanes;
      if (q < total) {
        const int hit = VL8 >= 0 ? (q >> VL8) : q / V;
        const int col = q - hit * V;
        const int64_t off = rowoff[hit];
        v[u] = off >= 0 ? ld_nc8(table + off + col * 8) : make_uint2(0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < kWidenUnroll; ++u) {
      const int q = base + u * kLanes;
      if (q < total) st_cs(out + static_cast<int64_t>(q) * 16, widen8(v[u]));
    }
  }
}

template <int VL, int kLanes, bool kWiden>
__device__ __forceinline__ void stream_hits(const unsigned char* __restrict__ table,
                                            const int64_t* __restrict__ rowoff, int nhits, int v_rt,
                                            unsigned char* __restrict__ out, int tid) {
  if constexpr (kWiden)
    widen_hits<VL, kLanes>(table, rowoff, nhits, v_rt, out, tid);
  else
    copy_hits<VL, kLanes>(table, rowoff, nhits, v_rt, out, tid);
}

// Fused lookup.  Every warp owns TW consecutive tokens and works alone (no
// block barrier after the constants are staged): its first TW lanes hash the
// tokens, the warp turns the order hashes into TW*H row offsets in its own
// slice of shared memory, then streams those rows.  Warps drift apart, so one
// warp's hashing overlaps other warps' copies.
// Output tokens of a lookup: all T packed tokens, or (global slice) for each
// of the T / row_len rows the positions [start, start + width) of the row.
struct OutMap {
  int64_t count;    // output tokens
  int64_t row_len;  // slice mode only
  int64_t start;
  int64_t width;
};

template <int TW, int VL, bool kSlice, bool kWiden>
__global__ void __launch_bounds__(kBlock, 4)
lookup_kernel(const HashParams hp, const int64_t* __restrict__ tokens, int64_t T,
              const int32_t* __restrict__ cu, int32_t num_seqs, const unsigned char* __restrict__ table,
              int64_t num_rows, int32_t row_bytes, unsigned char* __restrict__ out,
              int64_t* __restrict__ rows_out, const OutMap om, unsigned int* status) {
  static_assert(TW <= 32, "the first TW lanes hash the warp's tokens");
  extern __shared__ __align__(16) unsigned char smem[];
  const int H = hp.num_heads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  HeadConst* consts = reinterpret_cast<HeadConst*>(smem);
  int64_t* hsh = reinterpret_cast<int64_t*>(consts + H) + warp * TW * (kMaxOrder - 1);  // [TW][7]
  int64_t* rowoff = reinterpret_cast<int64_t*>(consts + H) + (kBlock / 32) * TW * (kMaxOrder - 1) +
                    warp * TW * H;                                                        // [TW*H]
  load_consts(hp, consts);
  check_seqlens(cu, num_seqs, T, status);
  __syncthreads();
  allow_next_grid();  // a dependent launch waits for this grid's completion before it reads anything

  const int64_t Tout = kSlice ? om.count : T;
  const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * (kBlock / 32) + warp) * TW;  // first output token
  if (t0 >= Tout) return;
  {
    const int64_t o = t0 + lane;
    const bool valid = lane < TW && o < Tout;
    int64_t hs[kMaxOrder - 1];
    if constexpr (kSlice) {
      const int64_t t = valid ? (o / om.width) * om.row_len + om.start + o % om.width : 0;
      order_hashes_direct(hp, tokens, cu, num_seqs, t, valid, hs);
    } else {
      order_hashes(hp, tokens, cu, num_seqs, o, valid, hs);
    }
    if (lane < TW) {
#pragma unroll
      for (int m = 0; m < kMaxOrder - 1; ++m) hsh[lane * (kMaxOrder - 1) + m] = hs[m];
    }
  }
  __syncwarp();
  const int ntok = static_cast<int>(min(static_cast<int64_t>(TW), Tout - t0));
  const int nhits = ntok * H;
  const int G = hp.heads_per_ngram;
  for (int q = lane; q < nhits; q += 32) {
    const int tl = q / H;
    const int j = q - tl * H;
    const HeadConst c = consts[j];
    const int64_t row = c.offset + static_cast<int64_t>(floor_mod(hsh[tl * (kMaxOrder - 1) + j / G], c));
    // always true for a validated plan; kept so that no table read can leave the table
    rowoff[q] = row < num_rows ? row * row_bytes : -1;
    if (rows_out != nullptr) rows_out[t0 * H + q] = row;
  }
  __syncwarp();
  const int64_t out_row_bytes = static_cast<int64_t>(row_bytes) * (kWiden ? 2 : 1);
  stream_hits<VL, 32, kWiden>(table, rowoff, nhits, row_bytes >> 4, out + t0 * H * out_row_bytes, lane);
}

constexpr int kGatherHits = 512;  // hits per block of the plain gather

template <int VL, bool kWiden>
__global__ void __launch_bounds__(kBlock, 4)
gather_kernel(const int64_t* __restrict__ rows, int64_t N, int64_t num_rows,
              const unsigned char* __restrict__ table, int32_t row_bytes, unsigned char* __restrict__ out,
              unsigned int* status) {
  __shared__ int64_t rowoff[kGatherHits];
  const int64_t h0 = static_cast<int64_t>(blockIdx.x) * kGatherHits;
  const int nh = static_cast<int>(min(static_cast<int64_t>(kGatherHits), N - h0));
  bool bad = false;
  for (int q = threadIdx.x; q < nh; q += kBlock) {
    const int64_t r = rows[h0 + q];
    const bool ok = r >= 0 && r < num_rows;
    bad |= !ok;
    rowoff[q] = ok ? r * row_bytes : -1;
  }
  if (bad) raise_flag(status, PLE_ERR_BAD_ROW);
  __syncthreads();
  const int64_t out_row_bytes = static_cast<int64_t>(row_bytes) * (kWiden ? 2 : 1);
  stream_hits<VL, kBlock, kWiden>(table, rowoff, nh, row_bytes >> 4, out + h0 * out_row_bytes, threadIdx.x);
}

int log2_exact(int v) {
  for (int k = 0; k < 31; ++k)
    if ((1 << k) == v) return k;
  return -1;
}

template <int TW, bool kSlice, bool kWiden>
ple_status_t launch_lookup(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu,
                           int32_t S, const void* table, void* out, int64_t* rows_out, const OutMap& om,
                           unsigned int* status, cudaStream_t stream) {
  const int H = plan->hp.num_heads;
  constexpr int kWarps = kBlock / 32;
  const size_t smem = H * sizeof(HeadConst) + kWarps * TW * (kMaxOrder - 1) * sizeof(int64_t) +
                      static_cast<size_t>(kWarps) * TW * H * sizeof(int64_t);
  if (smem > 48 * 1024) return PLE_ERR_UNSUPPORTED;  // not reached: TW*H <= 512 keeps it under 48 KB
  const int64_t warps = ((kSlice ? om.count : T) + TW - 1) / TW;
  const dim3 grid(static_cast<unsigned>((warps + kWarps - 1) / kWarps));
  const auto* tb = static_cast<const unsigned char*>(table);
  auto* ob = static_cast<unsigned char*>(out);
  const int rb = plan->row_bytes;
  const int64_t R = plan->num_rows;
#define PLE_LOOKUP_CASE(VL)                                                                            \
  case VL:                                                                                             \
    lookup_kernel<TW, VL, kSlice, kWiden><<<grid, kBlock, smem, stream>>>(plan->hp, tokens, T, cu, S, tb, R, \
                                                                          rb, ob, rows_out, om, status);     \
    break;
  switch (log2_exact(rb >> 4)) {
    PLE_LOOKUP_CASE(0)
    PLE_LOOKUP_CASE(1)
    PLE_LOOKUP_CASE(2)
    PLE_LOOKUP_CASE(3)
    PLE_LOOKUP_CASE(4)
    PLE_LOOKUP_CASE(5)
    PLE_LOOKUP_CASE(6)
    default:
      lookup_kernel<TW, -1, kSlice, kWiden><<<grid, kBlock, smem, stream>>>(plan->hp, tokens, T, cu, S, tb, R, rb,
                                                                            ob, rows_out, om, status);
  }
#undef PLE_LOOKUP_CASE
  return check_launch();
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

ple_status_t check_hash_args(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu,
                             int32_t S) {
  if (plan == nullptr || T < 0) return PLE_ERR_INVALID_ARG;
  if (T == 0) return PLE_OK;
  if (tokens == nullptr || cu == nullptr || S < 1) return PLE_ERR_INVALID_ARG;
  if (T > (int64_t{1} << 40)) return PLE_ERR_UNSUPPORTED;
  if (!aligned(tokens, 8) || !aligned(cu, 4)) return PLE_ERR_ALIGNMENT;
  return PLE_OK;
}

}  // namespace
}  // namespace ple

using namespace ple;

extern "C" {

ple_status_t ple_hash(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu,
                      int32_t S, int64_t* rows, void* stream) {
  ple_status_t st = check_hash_args(plan, tokens, T, cu, S);
  if (st != PLE_OK || T == 0) return st;
  if (rows == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(rows, 8)) return PLE_ERR_ALIGNMENT;
  cudaError_t e;
  unsigned int* status = status_word(plan, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  const int H = plan->hp.num_heads;
  const size_t smem = H * sizeof(HeadConst) + static_cast<size_t>(kHashWarps) * 32 * H * sizeof(int64_t);
  if (smem > 48 * 1024) {  // once per device and context, for the largest size a plan can ask for
    static std::atomic<unsigned long long> allowed[64];  // context id + 1, per device
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned long long ctx = 0;
    current_context_id(&ctx);
    if (dev >= 64 || allowed[dev].load(std::memory_order_acquire) != ctx + 1) {
      const size_t most = kMaxHeads * sizeof(HeadConst) + static_cast<size_t>(kHashWarps) * 32 * kMaxHeads * sizeof(int64_t);
      e = cudaFuncSetAttribute(hash_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(most));
      if (e != cudaSuccess) return cuda_fail(e);
      if (dev < 64) allowed[dev].store(ctx + 1, std::memory_order_release);
    }
  }
  const int64_t warps = (T + 31) / 32;
  const dim3 grid(static_cast<unsigned>((warps + kHashWarps - 1) / kHashWarps));
  hash_kernel<<<grid, kHashWarps * 32, smem, static_cast<cudaStream_t>(stream)>>>(plan->hp, tokens, T, cu, S,
                                                                                   rows, status);
  return check_launch();
}

}  // extern "C"

namespace {

template <bool kSlice>
ple_status_t dispatch_lookup(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu, int32_t S,
                             const void* table, void* out, int64_t* rows_out, const OutMap& om, void* stream) {
  cudaError_t e;
  unsigned int* status = status_word(plan, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  const auto s = static_cast<cudaStream_t>(stream);
  const int64_t Tout = kSlice ? om.count : T;
  // tokens per warp: at most about 1K 16-byte vectors of copy work per warp,
  // and enough warps to fill every SM several times over
  const int64_t vec_per_token = static_cast<int64_t>(plan->hp.num_heads) * (plan->row_bytes >> 4);
  int tw = 32;
  while (tw > 1 && (tw * vec_per_token > 1024 || (Tout + tw - 1) / tw < 32LL * sm_count())) tw >>= 1;
  while (tw > 1 && tw * plan->hp.num_heads > 512) tw >>= 1;  // row offsets of 8 warps stay <= 32 KB
  const bool widen = plan->table_dtype == PLE_F8E4M3;
#define PLE_TW_CASE(TWV)                                                                                      \
  case TWV:                                                                                                   \
    return widen ? launch_lookup<TWV, kSlice, true>(plan, tokens, T, cu, S, table, out, rows_out, om, status, s) \
                 : launch_lookup<TWV, kSlice, false>(plan, tokens, T, cu, S, table, out, rows_out, om, status, s);
  switch (tw) {
    PLE_TW_CASE(32)
    PLE_TW_CASE(16)
    PLE_TW_CASE(8)
    PLE_TW_CASE(4)
    PLE_TW_CASE(2)
    PLE_TW_CASE(1)
    default:
      return PLE_ERR_UNSUPPORTED;  // not reached: tw is a power of two in 1..32
  }
#undef PLE_TW_CASE
}

ple_status_t gather_bounded(const ple_plan_t* plan, const int64_t* rows, int64_t N, int64_t R, const void* table,
                            void* out, void* stream) {
  if (plan == nullptr || N < 0) return PLE_ERR_INVALID_ARG;
  if (N == 0) return PLE_OK;
  if (rows == nullptr || table == nullptr || out == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(rows, 8) || !aligned(table, 16) || !aligned(out, 16)) return PLE_ERR_ALIGNMENT;
  cudaError_t e;
  unsigned int* status = status_word(plan, static_cast<cudaStream_t>(stream), &e);
  if (status == nullptr) return cuda_fail(e);
  const dim3 grid(static_cast<unsigned>((N + kGatherHits - 1) / kGatherHits));
  const auto s = static_cast<cudaStream_t>(stream);
  const auto* tb = static_cast<const unsigned char*>(table);
  auto* ob = static_cast<unsigned char*>(out);
  const int rb = plan->row_bytes;
  const bool widen = plan->table_dtype == PLE_F8E4M3;
#define PLE_GATHER_CASE(VL)                                                                   \
  case VL:                                                                                    \
    if (widen)                                                                                \
      gather_kernel<VL, true><<<grid, kBlock, 0, s>>>(rows, N, R, tb, rb, ob, status);        \
    else                                                                                      \
      gather_kernel<VL, false><<<grid, kBlock, 0, s>>>(rows, N, R, tb, rb, ob, status);       \
    break;
  switch (log2_exact(rb >> 4)) {
    PLE_GATHER_CASE(0)
    PLE_GATHER_CASE(1)
    PLE_GATHER_CASE(2)
    PLE_GATHER_CASE(3)
    PLE_GATHER_CASE(4)
    PLE_GATHER_CASE(5)
    PLE_GATHER_CASE(6)
    default:
      if (widen)
        gather_kernel<-1, true><<<grid, kBlock, 0, s>>>(rows, N, R, tb, rb, ob, status);
      else
        gather_kernel<-1, false><<<grid, kBlock, 0, s>>>(rows, N, R, tb, rb, ob, status);
  }
#undef PLE_GATHER_CASE
  return check_launch();
}

ple_status_t check_lookup_ptrs(const void* table, void* out, int64_t* rows_out) {
  if (table == nullptr || out == nullptr) return PLE_ERR_INVALID_ARG;
  if (!aligned(table, 16) || !aligned(out, 16) || (rows_out != nullptr && !aligned(rows_out, 8)))
    return PLE_ERR_ALIGNMENT;
  return PLE_OK;
}

}  // namespace

extern "C" {

ple_status_t ple_lookup(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu,
                        int32_t S, const void* table, void* out, int64_t* rows_out, void* stream) {
  ple_status_t st = check_hash_args(plan, tokens, T, cu, S);
  if (st != PLE_OK || T == 0) return st;
  st = check_lookup_ptrs(table, out, rows_out);
  if (st != PLE_OK) return st;
  return dispatch_lookup<false>(plan, tokens, T, cu, S, table, out, rows_out, OutMap{T, T, 0, T}, stream);
}

ple_status_t ple_lookup_slice(const ple_plan_t* plan, const int64_t* tokens, int64_t T, const int32_t* cu,
                              int32_t S, int64_t row_len, int64_t start, int64_t end, const void* table, void* out,
                              int64_t* rows_out, void* stream) {
  ple_status_t st = check_hash_args(plan, tokens, T, cu, S);
  if (st != PLE_OK) return st;
  if (row_len < 1 || T % row_len != 0 || start < 0 || start > end || end > row_len) return PLE_ERR_INVALID_ARG;
  const int64_t count = (T / row_len) * (end - start);
  if (count == 0) return PLE_OK;
  st = check_lookup_ptrs(table, out, rows_out);
  if (st != PLE_OK) return st;
  return dispatch_lookup<true>(plan, tokens, T, cu, S, table, out, rows_out, OutMap{count, row_len, start,
                                                                                    end - start}, stream);
}

ple_status_t ple_gather(const ple_plan_t* plan, const int64_t* rows, int64_t N, const void* table, void* out,
                        void* stream) {
  if (plan == nullptr) return PLE_ERR_INVALID_ARG;
  return gather_bounded(plan, rows, N, plan->num_rows, table, out, stream);
}

ple_status_t ple_gather_cache(const ple_plan_t* plan, const int64_t* slots, int64_t N, const void* cache,
                              int64_t cache_rows, void* out, void* stream) {
  if (plan == nullptr || cache_rows < 0) return PLE_ERR_INVALID_ARG;
  return gather_bounded(plan, slots, N, cache_rows, cache, out, stream);
}

}  // extern "C"
