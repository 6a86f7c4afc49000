"""Seeded synthetic inputs for the hashed n-gram (PLE / Engram) lookup.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It holds none of the lookup's own arithmetic (no context
shift, no hash combine, no remainder, no gather, no gradient fold): it only
draws token streams, packed-sequence boundaries, hash constants and table /
gradient values, all from fixed seeds.

Table and gradient values come from one counter-based generator so that any
single element can be regenerated on the host without a host copy of a
multi-gigabyte table.  Its definition (the CUDA twin in ``synth/fill.cu``
implements the same definition independently):

* ``u(seed, i)`` is the ``(i+1)``-th output of SplitMix64 (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014; the
  finaliser constants are Stafford's "Mix13" as used by Vigna's reference
  ``splitmix64.c``) started from state ``seed * 0xD1B54A32D192ED03``.
* ``s = sum of the four 16-bit fields of u`` is an exact integer in
  ``[0, 262140]`` (Irwin-Hall of four uniforms; mean 131070, standard
  deviation ``sqrt((65536**2 - 1) / 3)``).
* value ``= float32(s - 131070) * k`` with ``k = float32(sigma / sd)``; the
  integer is exactly representable, so the one fp32 multiply rounds the same
  way on every IEEE machine.
* bf16 values are the fp32 value rounded to nearest-even on its top 16 bits.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
SEED_MUL = 0xD1B54A32D192ED03
MIX_C1 = 0xBF58476D1CE4E5B9
MIX_C2 = 0x94D049BB133111EB
IH4_MEAN = 131070
IH4_SD = math.sqrt((65536.0 ** 2 - 1.0) / 3.0)

DTYPE_F32 = 0
DTYPE_BF16 = 1
DTYPE_E4M3 = 2  # fp8 e4m3 codes: uniform random finite codes (8 per counter output)


def value_scale(sigma: float) -> np.float32:
    """fp32 factor that maps the centred Irwin-Hall sum to standard deviation sigma."""
    return np.float32(sigma / IH4_SD)


def _mix64(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX_C1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX_C2)
    return z ^ (z >> np.uint64(31))


def counter_u64(seed: int, idx: np.ndarray) -> np.ndarray:
    """u(seed, i) for an array of non-negative indices (uint64 result)."""
    idx = np.asarray(idx, dtype=np.uint64)
    state0 = np.uint64((seed * SEED_MUL) & MASK64)
    with np.errstate(over="ignore"):
        z = state0 + (idx + np.uint64(1)) * np.uint64(GOLDEN)
        return _mix64(z)


def counter_f32(seed: int, idx: np.ndarray, sigma: float) -> np.ndarray:
    """fp32 values of the generator at flat indices ``idx``."""
    u = counter_u64(seed, idx)
    m = np.uint64(0xFFFF)
    s = (u & m) + ((u >> np.uint64(16)) & m) + ((u >> np.uint64(32)) & m) + (u >> np.uint64(48))
    centred = (s.astype(np.int64) - IH4_MEAN).astype(np.float32)
    return centred * value_scale(sigma)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest-even), returned as uint16 bit patterns."""
    b = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def counter_e4m3(seed: int, idx: np.ndarray) -> np.ndarray:
    """fp8 e4m3 codes: byte (i mod 8) of u(seed, i div 8); the two NaN codes
    (x.1111.111) become the largest finite code of their sign."""
    idx = np.asarray(idx, dtype=np.uint64)
    u = counter_u64(seed, idx // np.uint64(8))
    code = ((u >> (np.uint64(8) * (idx % np.uint64(8)))) & np.uint64(0xFF)).astype(np.uint8)
    nan = (code & 0x7F) == 0x7F
    code[nan] ^= 0x01
    return code


def counter_values(seed: int, idx: np.ndarray, sigma: float, dtype: int) -> np.ndarray:
    """Values as stored: fp32 array, bf16 bit patterns as uint16, or fp8 codes as uint8."""
    if dtype == DTYPE_E4M3:
        return counter_e4m3(seed, idx)
    v = counter_f32(seed, idx, sigma)
    if dtype == DTYPE_F32:
        return v
    if dtype == DTYPE_BF16:
        return f32_to_bf16_bits(v)
    raise ValueError(f"unknown dtype code {dtype}")


def table_rows(seed: int, rows: np.ndarray, dim: int, sigma: float, dtype: int) -> np.ndarray:
    """Regenerate whole rows ``[len(rows), dim]`` of a generated table."""
    rows = np.asarray(rows, dtype=np.int64).reshape(-1)
    idx = (rows[:, None].astype(np.uint64) * np.uint64(dim)) + np.arange(dim, dtype=np.uint64)[None, :]
    return counter_values(seed, idx, sigma, dtype)


def dense_values(seed: int, count: int, sigma: float, dtype: int) -> np.ndarray:
    return counter_values(seed, np.arange(count, dtype=np.uint64), sigma, dtype)


# ---------------------------------------------------------------------------
# token streams and packing
# ---------------------------------------------------------------------------

def packed_lengths(total: int, num_seqs: int, lo: int, hi: int, rng: np.random.Generator) -> np.ndarray:
    """Sequence lengths drawn uniformly in [lo, hi], rescaled to sum to ``total``.

    Each rescaled length is clipped back into [lo, hi] where the total allows;
    the remainder lands on the last sequence.
    """
    raw = rng.integers(lo, hi + 1, size=num_seqs).astype(np.float64)
    lens = np.floor(raw * (total / raw.sum())).astype(np.int64)
    lens = np.clip(lens, 1, None)
    lens[-1] += total - lens.sum()
    if lens[-1] < 1:  # extremely skewed draws: fall back to an even split
        lens[:] = total // num_seqs
        lens[-1] += total - lens.sum()
    return lens


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=cu[1:])
    if cu[-1] >= 2 ** 31:
        raise ValueError("packed length does not fit int32 cu_seqlens")
    return cu.astype(np.int32)


def uniform_ids(n: int, lo: int, hi: int, rng: np.random.Generator) -> np.ndarray:
    return rng.integers(lo, hi, size=n, dtype=np.int64)


def zipf_ids(n: int, s: float, vocab: int, rng: np.random.Generator) -> np.ndarray:
    """Zipf(s)-distributed ids over ranks 1..vocab-1, mapped by a seeded
    permutation onto the ids [1, vocab) (id 0 is kept for EOS)."""
    ranks = np.arange(1, vocab, dtype=np.float64)
    w = ranks ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    r = np.searchsorted(cdf, rng.random(n), side="right")
    r = np.minimum(r, vocab - 2)
    perm = rng.permutation(vocab - 1).astype(np.int64) + 1
    return perm[r]


def inject_eos(tokens: np.ndarray, rate: float, eos: int, rng: np.random.Generator) -> np.ndarray:
    out = tokens.copy()
    out[rng.random(len(out)) < rate] = eos
    return out


def repeat_spans(tokens: np.ndarray, span: int, p: float, rng: np.random.Generator) -> np.ndarray:
    """For every aligned ``span``-token block after the first, with probability
    p, overwrite it with a copy of a uniformly chosen earlier block."""
    out = tokens.copy()
    nblk = len(out) // span
    for b in range(1, nblk):
        if rng.random() < p:
            src = int(rng.integers(0, b))
            out[b * span:(b + 1) * span] = out[src * span:(src + 1) * span]
    return out


# ---------------------------------------------------------------------------
# hash constants
# ---------------------------------------------------------------------------

_MR_BASES = (2, 3, 5, 7, 11, 13, 17, 19, 23, 29, 31, 37)


def is_prime(n: int) -> bool:
    """Deterministic Miller-Rabin for n < 3.3e24 with the first twelve prime bases."""
    if n < 2:
        return False
    for p in _MR_BASES:
        if n % p == 0:
            return n == p
    d, r = n - 1, 0
    while d % 2 == 0:
        d //= 2
        r += 1
    for a in _MR_BASES:
        x = pow(a, d, n)
        if x in (1, n - 1):
            continue
        for _ in range(r - 1):
            x = x * x % n
            if x == n - 1:
                break
        else:
            return False
    return True


def consecutive_primes(start: int, count: int) -> list[int]:
    """The ``count`` smallest primes >= start."""
    out, x = [], start
    while len(out) < count:
        if is_prime(x):
            out.append(x)
        x += 1
    return out


def exclusive_prefix(values) -> list[int]:
    out, acc = [], 0
    for v in values:
        out.append(acc)
        acc += int(v)
    return out


def signed_mults(count: int, rng: np.random.Generator) -> np.ndarray:
    return rng.integers(-(2 ** 63), 2 ** 63 - 1, size=count, dtype=np.int64, endpoint=True)


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

@dataclass
class Workload:
    name: str
    tokens: np.ndarray            # int64 [T]
    cu_seqlens: np.ndarray        # int32 [S+1]
    ngram_size: int
    heads_per_ngram: int
    eos_id: int
    mults: np.ndarray             # int64 [ngram_size]
    primes: np.ndarray            # int64 [H]
    offsets: np.ndarray           # int64 [H]
    num_rows: int
    head_dim: int
    table_dtype: int              # DTYPE_F32 / DTYPE_BF16
    table_seed: int
    table_sigma: float
    grad_dtype: int
    grad_seed: int
    grad_sigma: float
    notes: dict = field(default_factory=dict)

    @property
    def num_heads(self) -> int:
        return (self.ngram_size - 1) * self.heads_per_ngram

    @property
    def num_tokens(self) -> int:
        return int(self.tokens.shape[0])

    @property
    def num_hits(self) -> int:
        return self.num_tokens * self.num_heads

    @property
    def table_elem_bytes(self) -> int:
        return {DTYPE_F32: 4, DTYPE_BF16: 2, DTYPE_E4M3: 1}[self.table_dtype]

    @property
    def grad_elem_bytes(self) -> int:
        return 4 if self.grad_dtype == DTYPE_F32 else 2

    @property
    def table_bytes(self) -> int:
        return self.num_rows * self.head_dim * self.table_elem_bytes

    def table_rows(self, rows) -> np.ndarray:
        return table_rows(self.table_seed, rows, self.head_dim, self.table_sigma, self.table_dtype)

    def grad_rows(self, hits) -> np.ndarray:
        """grad_out rows for flat hit indices i = t*H + j."""
        return table_rows(self.grad_seed, hits, self.head_dim, self.grad_sigma, self.grad_dtype)


def _hash_constants(n: int, G: int, prime_start: int, rng: np.random.Generator):
    H = (n - 1) * G
    primes = consecutive_primes(prime_start, H)
    offsets = exclusive_prefix(primes)
    mults = signed_mults(n, rng)
    return (np.asarray(mults, np.int64), np.asarray(primes, np.int64),
            np.asarray(offsets, np.int64), int(sum(primes)))


def _packed_stream(total, lo, hi, seed):
    rng = np.random.default_rng(seed)
    nseq = max(1, int(round(total / ((lo + hi) / 2))))
    return rng, packed_lengths(total, nseq, lo, hi, rng)


VOCAB = 151936


def tiny(seed: int = 0) -> Workload:
    """Two packed sequences (100 + 156), ids uniform in [1,1000), EOS 0 at 1 %,
    n=3, 2 heads per order, primes 4093/4099/8191/8209, D=32 fp32."""
    rng = np.random.default_rng(seed)
    lens = [100, 156]
    tok = inject_eos(uniform_ids(sum(lens), 1, 1000, rng), 0.01, 0, rng)
    primes = [4093, 4099, 8191, 8209]
    mults = signed_mults(3, rng)
    return Workload("tiny", tok, cu_seqlens_from_lengths(lens), 3, 2, 0, mults,
                    np.asarray(primes, np.int64), np.asarray(exclusive_prefix(primes), np.int64),
                    sum(primes), 32, DTYPE_F32, seed + 101, 0.02, DTYPE_F32, seed + 202, 1.0)


def single_layer_bf16(seed: int = 0, total: int = 32768) -> Workload:
    """8 packed sequences (lengths uniform 1k-8k, rescaled to 32768 tokens),
    Zipf(1.1) ids over the 151936-id vocabulary, EOS 0.5 %, n=3, 8 heads per
    order, 16 consecutive primes >= 1,000,000, D=64 bf16 (about 2 GB)."""
    rng = np.random.default_rng(seed)
    lens = packed_lengths(total, 8, 1024, 8192, rng)
    tok = inject_eos(zipf_ids(total, 1.1, VOCAB, rng), 0.005, 0, rng)
    mults, primes, offsets, R = _hash_constants(3, 8, 1_000_000, rng)
    return Workload("single_layer_bf16", tok, cu_seqlens_from_lengths(lens), 3, 8, 0, mults, primes,
                    offsets, R, 64, DTYPE_BF16, seed + 101, 0.02, DTYPE_BF16, seed + 202, 1.0)


def large_table_fp8(seed: int = 0, total: int = 65536) -> Workload:
    """The large-table workload with the table stored as fp8 e4m3 (the pages'
    checkpoint format): 25.8 GB, rows widened to bf16 by the lookup."""
    w = large_table(seed, total)
    w.name = "large_table_fp8"
    w.table_dtype = DTYPE_E4M3
    return w


def large_table(seed: int = 0, total: int = 65536) -> Workload:
    """65536 packed tokens (lengths 1k-8k), Zipf(1.1), n=4, 8 heads per order
    (24 heads), 24 consecutive primes >= 8,400,000 (~2.0e8 rows), D=128 bf16
    (about 51.6 GB)."""
    rng, lens = _packed_stream(total, 1024, 8192, seed)
    tok = inject_eos(zipf_ids(total, 1.1, VOCAB, rng), 0.005, 0, rng)
    mults, primes, offsets, R = _hash_constants(4, 8, 8_400_000, rng)
    return Workload("large_table", tok, cu_seqlens_from_lengths(lens), 4, 8, 0, mults, primes,
                    offsets, R, 128, DTYPE_BF16, seed + 101, 0.02, DTYPE_BF16, seed + 202, 1.0)


def backward_stress(seed: int = 0, total: int = 131072) -> Workload:
    """131072 packed tokens, Zipf(1.3) ids with 64-token repeated spans,
    EOS 0.5 %, n=3, 16 heads, primes as the single-layer workload, D=128,
    bf16 grad_out N(0,1) summed into an fp32 table gradient."""
    rng, lens = _packed_stream(total, 1024, 8192, seed)
    tok = zipf_ids(total, 1.3, VOCAB, rng)
    tok = repeat_spans(tok, 64, 0.5, rng)
    tok = inject_eos(tok, 0.005, 0, rng)
    mults, primes, offsets, R = _hash_constants(3, 8, 1_000_000, rng)
    return Workload("backward_stress", tok, cu_seqlens_from_lengths(lens), 3, 8, 0, mults, primes,
                    offsets, R, 128, DTYPE_BF16, seed + 101, 0.02, DTYPE_BF16, seed + 202, 1.0)


def backward_stress_small(seed: int = 0, total: int = 131072) -> Workload:
    """The backward-stress tokens and hits with 16 primes >= 125,000 (2.0 M
    rows): a 0.5 GB table and a 1 GB fp32 gradient, for profiler captures of
    the backward kernels that replay each launch many times."""
    w = backward_stress(seed, total)
    rng = np.random.default_rng(seed + 7)
    mults, primes, offsets, R = _hash_constants(3, 8, 125_000, rng)
    w.name = "backward_stress_small"
    w.primes, w.offsets, w.num_rows = primes, offsets, R
    return w


def sweep_point(tokens: int = 131072, head_dim: int = 128, ngram_size: int = 3, heads_per_ngram: int = 8,
                table_gb: float = 16.0, ids: str = "zipf", seed: int = 0,
                table_dtype: int = DTYPE_BF16) -> Workload:
    """One point of the sweep: per-head primes are consecutive primes >=
    table_bytes / (elem * D * H), so the table holds about ``table_gb`` GB
    (table_dtype=DTYPE_E4M3 for an fp8 table)."""
    rng, lens = _packed_stream(tokens, 1024, 8192, seed)
    if ids == "zipf":
        tok = zipf_ids(tokens, 1.1, VOCAB, rng)
    elif ids == "uniform":
        tok = uniform_ids(tokens, 1, VOCAB, rng)
    else:
        raise ValueError(ids)
    tok = inject_eos(tok, 0.005, 0, rng)
    H = (ngram_size - 1) * heads_per_ngram
    elem = {DTYPE_F32: 4, DTYPE_BF16: 2, DTYPE_E4M3: 1}[table_dtype]
    per_head = max(3, int(table_gb * 1e9 / (elem * head_dim * H)))
    mults, primes, offsets, R = _hash_constants(ngram_size, heads_per_ngram, per_head, rng)
    name = f"sweep_T{tokens}_D{head_dim}_n{ngram_size}_{ids}_{table_gb:g}GB" + ("_fp8" if table_dtype == DTYPE_E4M3 else "")
    return Workload(name, tok, cu_seqlens_from_lengths(lens), ngram_size, heads_per_ngram, 0, mults,
                    primes, offsets, R, head_dim, table_dtype, seed + 101, 0.02, DTYPE_BF16, seed + 202, 1.0)


WORKLOADS = {
    "tiny": tiny,
    "single_layer_bf16": single_layer_bf16,
    "large_table": large_table,
    "backward_stress": backward_stress,
    "large_table_fp8": large_table_fp8,
    "backward_stress_small": backward_stress_small,
}
