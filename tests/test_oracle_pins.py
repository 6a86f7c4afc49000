"""Pins for the CPU oracle: each check holds it to something other than itself.

* hand-worked rows (tests/golden/hand_worked.txt, derived on paper);
* special multipliers that reduce the hash to a plain token shift;
* brute force over every token string of length <= 5 over {EOS, 1, 2, 3}
  and every packing, against a restatement that walks the segment
  explicitly and wraps Python big integers modulo 2^64;
* invariants: rows inside their head's range, head ranges disjoint, the
  n-gram after an EOS hashes as at a sequence start, packing position does
  not matter;
* the gather against torch.nn.functional.embedding (same definition, library);
* the gradient against torch.index_add_ in fp64 (integer-valued gradients are
  exact in any order), the per-row-sum invariant, and closed-form values that
  only the adopted chunked order (chunks of 32, left folds from the first
  element, one final add) produces.
"""
import itertools
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import oracle
import synth
from conftest import ROOT, read_golden_blocks

pytestmark = pytest.mark.filterwarnings("ignore::DeprecationWarning")

M64 = 1 << 64


# ---------------------------------------------------------------------------
# hash / rows
# ---------------------------------------------------------------------------

def test_hand_worked_cases():
    cases, _ = read_golden_blocks("hand_worked.txt")
    assert len(cases) == 6
    for c in cases:
        got = oracle.rows(c["tokens"], c["cu_seqlens"], c["ngram_size"][0], c["heads_per_ngram"][0],
                          c["eos"][0], c["mults"], c["primes"], c["offsets"])
        assert got.reshape(-1).tolist() == c["rows"], c["name"]


def _ref_rows_bigint(tokens, cu, n, G, eos, mults, primes, offsets):
    """Independent restatement: for each token, walk back inside its own
    segment collecting at most n-1 earlier tokens, stopping at an EOS; hash
    with unbounded integers, wrap to signed 64 bits, floor remainder."""
    H = (n - 1) * G
    T = len(tokens)
    out = np.zeros((T, H), dtype=np.int64)
    for s in range(len(cu) - 1):
        seg = tokens[cu[s]:cu[s + 1]]
        for loc in range(len(seg)):
            history = []
            back = loc - 1
            while back >= 0 and len(history) < n - 1 and seg[back] != eos:
                history.append(int(seg[back]))
                back -= 1
            ctx = [int(seg[loc])] + history + [0] * (n - 1 - len(history))
            for m in range(2, n + 1):
                h = sum(ctx[k] * int(mults[k]) for k in range(m)) % M64
                if h >= 1 << 63:
                    h -= M64
                for g in range(G):
                    j = (m - 2) * G + g
                    out[cu[s] + loc, j] = int(offsets[j]) + h % int(primes[j])
    return out


def _compositions(L):
    """All ways to split L tokens into >= 1 consecutive segments, plus one
    packing with empty segments at both ends and in the middle."""
    outs = []
    for cuts in itertools.product([0, 1], repeat=max(L - 1, 0)):
        cu = [0] + [i + 1 for i, c in enumerate(cuts) if c] + [L]
        outs.append(cu)
    half = L // 2
    outs.append([0, 0, half, half, L, L])
    return outs


@pytest.mark.parametrize("n", [2, 3, 4])
@pytest.mark.parametrize("mult_kind", ["small", "extreme", "random"])
def test_brute_force_all_short_strings(n, mult_kind):
    rng = np.random.default_rng(1000 + n)
    if mult_kind == "small":
        mults = [1, 7, 49, 343][:n]
    elif mult_kind == "extreme":
        mults = [2 ** 63 - 1, -(2 ** 63), -1, 2 ** 62 + 3][:n]
    else:
        mults = synth.signed_mults(n, rng).tolist()
    G = 2
    primes = [5, 7, 11, 13, 17, 19][: (n - 1) * G]
    offsets = synth.exclusive_prefix(primes)
    eos = 0
    # pack every case as its own run of sequences in one large packed batch
    all_tok, all_cu = [], [0]
    for L in range(1, 6):
        for s in itertools.product(range(4), repeat=L):
            for cu in _compositions(L):
                base = len(all_tok)
                all_tok.extend(s)
                all_cu.extend(base + c for c in cu[1:])
    tok = np.asarray(all_tok, np.int64)
    cu = np.asarray(all_cu, np.int32)
    got = oracle.rows(tok, cu, n, G, eos, mults, primes, offsets)
    ref = _ref_rows_bigint(all_tok, all_cu, n, G, eos, mults, primes, offsets)
    np.testing.assert_array_equal(got, ref)


def _shift_within_segments(tok, cu, k, eos):
    """Token k positions back, or 0 where that position is before the segment
    start or an EOS lies in between (numpy shift and masks)."""
    T = len(tok)
    seg_start = np.repeat(cu[:-1], np.diff(cu))
    out = np.zeros(T, np.int64)
    ok = np.arange(T) - k >= seg_start
    for d in range(1, k + 1):
        prev = np.concatenate([np.full(d, -1, np.int64), tok[:-d]]) if d < T else np.full(T, -1, np.int64)
        ok &= prev != eos
    src = np.arange(T) - k
    out[ok] = tok[src[ok]]
    return out


@pytest.mark.parametrize("which", [0, 1, 2, 3])
def test_shift_only_multipliers(which):
    """A multiplier vector with a single 1 at slot k makes every order-m head
    (m > k) a plain remainder of the token k back (or of 0)."""
    w = synth.tiny(seed=3)
    n = 4
    G = 2
    mults = [0] * n
    mults[which] = 1
    primes = synth.consecutive_primes(1009, (n - 1) * G)
    offsets = synth.exclusive_prefix(primes)
    got = oracle.rows(w.tokens, w.cu_seqlens, n, G, w.eos_id, mults, primes, offsets)
    shifted = _shift_within_segments(w.tokens, w.cu_seqlens.astype(np.int64), which, w.eos_id)
    for j in range(len(primes)):
        m = 2 + j // G
        expect = offsets[j] + (np.mod(shifted, primes[j]) if which < m else 0)
        np.testing.assert_array_equal(got[:, j], expect)


def test_rows_in_head_ranges_and_ranges_disjoint():
    for w in (synth.tiny(0), synth.tiny(5)):
        r = oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults,
                        w.primes, w.offsets)
        lo, hi = w.offsets, w.offsets + w.primes
        assert np.all(r >= lo[None, :]) and np.all(r < hi[None, :])
        order = np.argsort(lo)
        assert np.all(hi[order][:-1] <= lo[order][1:])


def test_eos_reset_equals_sequence_start():
    rng = np.random.default_rng(7)
    mults = synth.signed_mults(4, rng)
    primes = synth.consecutive_primes(100_003, 6)
    offsets = synth.exclusive_prefix(primes)
    body = rng.integers(1, 1000, 9)
    with_eos = np.concatenate([[11, 12, 13, 0], body])  # EOS at position 3
    a = oracle.rows(with_eos, [0, len(with_eos)], 4, 2, 0, mults, primes, offsets)
    b = oracle.rows(body, [0, len(body)], 4, 2, 0, mults, primes, offsets)
    np.testing.assert_array_equal(a[4:], b)
    # the EOS's own n-gram still sees its predecessors
    c = oracle.rows(with_eos[:4], [0, 4], 4, 2, 0, mults, primes, offsets)
    np.testing.assert_array_equal(a[:4], c)


def test_packing_position_invariance():
    rng = np.random.default_rng(11)
    mults = synth.signed_mults(3, rng)
    primes = synth.consecutive_primes(7919, 4)
    offsets = synth.exclusive_prefix(primes)
    seqs = [rng.integers(0, 30, L) for L in (17, 1, 40, 0, 23)]
    packed = np.concatenate(seqs)
    cu = synth.cu_seqlens_from_lengths([len(s) for s in seqs])
    full = oracle.rows(packed, cu, 3, 2, 0, mults, primes, offsets)
    for s, (a, b) in zip(seqs, zip(cu[:-1], cu[1:])):
        alone = oracle.rows(s, [0, len(s)], 3, 2, 0, mults, primes, offsets)
        np.testing.assert_array_equal(full[a:b], alone)


def test_malformed_cu_seqlens_rejected():
    with pytest.raises(ValueError):
        oracle.rows([1, 2, 3], [0, 2], 2, 1, 0, [1, 1], [7], [0])
    with pytest.raises(ValueError):
        oracle.rows([1, 2, 3], [0, 2, 1, 3], 2, 1, 0, [1, 1], [7], [0])


def test_production_constants():
    _, g = read_golden_blocks("production_constants.txt")
    primes = g["primes_prefix"]
    # the printed offsets are the exclusive prefix sums of the printed primes
    assert synth.exclusive_prefix(primes) == g["offsets_prefix"]
    assert str(g["offsets_prefix"][-1] + primes[-1]).startswith(str(g["offset_9_leading_digits"][0]))
    # the printed primes are the consecutive primes from 2e7 on
    assert synth.consecutive_primes(20_000_000, 8) == primes
    # all 16 heads (ngram 3, 8 per order): their sum, padded to a multiple of 128,
    # is the printed padded row count
    all16 = synth.consecutive_primes(20_000_000, 16)
    total = sum(all16)
    assert (total + 127) // 128 * 128 == g["padded_rows"][0]
    # rows of a random stream under the production constants stay in range
    rng = np.random.default_rng(0)
    tok = rng.integers(0, 248_320, 3000)
    tok[rng.random(3000) < 0.01] = g["eos_token_id"][0]
    offs = synth.exclusive_prefix(all16)
    r = oracle.rows(tok, [0, 1000, 3000], 3, 8, g["eos_token_id"][0], g["multipliers"], all16, offs)
    assert r.min() >= 0 and r.max() < total
    np.testing.assert_array_equal(r, _ref_rows_bigint(tok.tolist(), [0, 1000, 3000], 3, 8,
                                                      g["eos_token_id"][0], g["multipliers"], all16, offs))


def test_multithreaded_rows_match():
    w = synth.single_layer_bf16(0, total=8192)
    a = oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                    w.offsets)
    b = oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                    w.offsets, threads=4)
    np.testing.assert_array_equal(a, b)


# ---------------------------------------------------------------------------
# gather
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_gather_matches_torch_embedding(dtype):
    rng = np.random.default_rng(5)
    table = rng.integers(0, 2 ** 15, size=(997, 24)).astype(dtype) if dtype == np.uint16 else \
        rng.standard_normal((997, 24)).astype(np.float32)
    rows = rng.integers(0, 997, size=(50, 6))
    got = oracle.gather(rows, table)
    t = torch.from_numpy(table.astype(np.int64) if dtype == np.uint16 else table)
    ref = torch.nn.functional.embedding(torch.from_numpy(rows), t).numpy().astype(dtype)
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(oracle.gather(rows, table, threads=3), got)


def test_gather_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.gather(np.array([0, 5]), np.zeros((5, 4), np.float32))
    with pytest.raises(ValueError):
        oracle.gather(np.array([-1]), np.zeros((5, 4), np.float32))


# ---------------------------------------------------------------------------
# gradient
# ---------------------------------------------------------------------------

def _index_add_fp64(rows, grad_f32, R):
    D = grad_f32.shape[-1]
    out = torch.zeros(R, D, dtype=torch.float64)
    out.index_add_(0, torch.from_numpy(rows.reshape(-1)), torch.from_numpy(grad_f32.reshape(-1, D)).double())
    return out.numpy()


def test_grad_integer_values_exact():
    rng = np.random.default_rng(9)
    R, D, N = 300, 16, 5000
    rows = rng.integers(0, R, N)
    rows[:700] = 17  # a heavy row spanning many chunks
    grad = rng.integers(-50, 51, size=(N, D)).astype(np.float32)
    tg = oracle.grad_apply(rows, grad, np.zeros((R, D), np.float32))
    np.testing.assert_array_equal(tg.astype(np.float64), _index_add_fp64(rows, grad, R))
    # bf16 storage of the same small integers is exact too
    gb = synth.f32_to_bf16_bits(grad)
    tb = oracle.grad_apply(rows, gb, np.zeros((R, D), np.float32))
    np.testing.assert_array_equal(tb, tg)


def test_grad_random_close_to_fp64_and_row_sum_invariant():
    w = synth.tiny(0)
    r = oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                    w.offsets)
    grad = synth.dense_values(w.grad_seed, r.size * w.head_dim, 1.0, synth.DTYPE_F32).reshape(-1, w.head_dim)
    tg = oracle.grad_apply(r, grad, np.zeros((w.num_rows, w.head_dim), np.float32))
    ref = _index_add_fp64(r, grad, w.num_rows)
    np.testing.assert_allclose(tg, ref, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(tg.astype(np.float64).sum(0), grad.astype(np.float64).sum(0), rtol=1e-5, atol=1e-4)
    uniq, sums = oracle.grad_sums(r, grad)
    np.testing.assert_array_equal(uniq, np.unique(r))
    np.testing.assert_array_equal(sums, tg[uniq])
    u2, s2 = oracle.grad_sums(r, grad, threads=3)
    np.testing.assert_array_equal(u2, uniq)
    np.testing.assert_array_equal(s2, sums)


def _single_row_grad(values, D=2):
    N = len(values)
    rows = np.full(N, 3, np.int64)
    grad = np.repeat(np.asarray(values, np.float32)[:, None], D, axis=1)
    return rows, grad


def test_grad_chunk_of_32_closed_form():
    """2^24 followed by 39 ones on one row.  fp32 spacing at 2^24 is 2, so a
    single left fold loses every 1 (2^24); chunks of 32 give 2^24 (31 ones
    lost) + 8 = 16777224; chunks of 16 would give 16777240, a pairwise tree
    16777256."""
    rows, grad = _single_row_grad([2.0 ** 24] + [1.0] * 39)
    tg = oracle.grad_apply(rows, grad, np.zeros((5, 2), np.float32))
    assert tg[3, 0] == np.float32(16777224.0)


def test_grad_ascending_index_order_closed_form():
    """Same multiset in the reverse index order: chunk 0 = 32 ones = 32,
    chunk 1 = 7 ones then 2^24 = 16777223 -> 16777224 (tie to even), sum
    16777256: the order of hits inside a row is ascending flat index."""
    rows, grad = _single_row_grad([1.0] * 39 + [2.0 ** 24])
    tg = oracle.grad_apply(rows, grad, np.zeros((5, 2), np.float32))
    assert tg[3, 0] == np.float32(16777256.0)


def test_grad_single_final_add_and_negative_zero():
    # the row sum is formed first and added once: 2^24 + (1 + 1) = 16777218,
    # while adding the hits into the row one by one would leave 2^24
    rows, grad = _single_row_grad([1.0, 1.0])
    tg = np.full((5, 2), 2.0 ** 24, np.float32)
    oracle.grad_apply(rows, grad, tg)
    assert tg[3, 0] == np.float32(16777218.0) and tg[0, 0] == np.float32(2.0 ** 24)
    # folds start from the first element, not from +0: -0 + -0 stays -0
    rows, grad = _single_row_grad([-0.0])
    tg = np.full((5, 2), -0.0, np.float32)
    oracle.grad_apply(rows, grad, tg)
    assert np.signbit(tg[3, 0])


def test_grad_subnormal_sums_exact():
    """Gradients and prefill that are integer multiples of 2^-149 (fp32
    subnormals): every partial sum is exact in fp32 (|sum| < 2^-125), so
    whatever the order the result is the integer sum times 2^-149.  A
    flush-to-zero add anywhere in the fold would lose them."""
    rng = np.random.default_rng(8)
    N, D, R = 700, 4, 9
    rows = rng.integers(0, R, N)
    rows[:100] = 2  # one row with a long run (several chunks)
    k = rng.integers(-1000, 1000, (N, D))
    m = rng.integers(-1000, 1000, (R, D))
    g = (k * 2.0 ** -149).astype(np.float32)
    assert np.all(np.abs(g) < np.float32(2.0 ** -126))
    tg = (m * 2.0 ** -149).astype(np.float32)
    oracle.grad_apply(rows, g, tg)
    want = m.copy()
    np.add.at(want, rows, k)
    np.testing.assert_array_equal(tg, (want * 2.0 ** -149).astype(np.float32))
    # bf16 subnormals: bits S.00000000.MMMMMMM = +-M * 2^-133, sums exact below 2^-109
    kb = rng.integers(-127, 128, (N, D))
    bits = (np.where(kb < 0, 0x8000, 0) | np.abs(kb)).astype(np.uint16)
    tg = np.zeros((R, D), np.float32)
    oracle.grad_apply(rows, bits, tg)
    want = np.zeros((R, D), np.int64)
    np.add.at(want, rows, kb)
    np.testing.assert_array_equal(tg, (want * 2.0 ** -133).astype(np.float32))


def test_grad_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.grad_apply(np.array([0, 9]), np.zeros((2, 4), np.float32), np.zeros((5, 4), np.float32))


# ---------------------------------------------------------------------------
# global-slice lookup
# ---------------------------------------------------------------------------

def test_slice_keeps_context_before_the_boundary():
    """A shard [start, end) of a row hashes with the tokens before `start`
    (the API page: hashing the full tensor preserves the preceding raw tokens
    and EOS resets at a CP boundary): its first tokens differ from hashing the
    shard's tokens alone, and equal the full rows restricted to the shard."""
    rng = np.random.default_rng(21)
    n, G = 3, 2
    mults = synth.signed_mults(n, rng)
    primes = synth.consecutive_primes(5003, (n - 1) * G)
    offsets = synth.exclusive_prefix(primes)
    row_len, B = 40, 3
    tok = rng.integers(1, 50, row_len * B)
    tok[row_len + 17] = 0  # an EOS just before the shard of row 1
    cu = np.arange(0, row_len * B + 1, row_len)
    table = rng.standard_normal((sum(primes), 8)).astype(np.float32)
    vals, sel = oracle.lookup_slice(tok, cu, n, G, 0, mults, primes, offsets, table, row_len, 18, 30)
    full = oracle.rows(tok, cu, n, G, 0, mults, primes, offsets).reshape(B, row_len, -1)
    np.testing.assert_array_equal(sel, full[:, 18:30])
    np.testing.assert_array_equal(vals, table[full[:, 18:30]])
    alone = oracle.rows(tok[18:30], [0, 12], n, G, 0, mults, primes, offsets)
    assert not np.array_equal(sel[0, :2], alone[:2])   # row 0: context from positions 16, 17
    np.testing.assert_array_equal(sel[0, 2:], alone[2:])
    # row 1: the EOS at position 17 resets the context, so its shard hashes as if alone
    alone1 = oracle.rows(tok[row_len + 18:row_len + 30], [0, 12], n, G, 0, mults, primes, offsets)
    np.testing.assert_array_equal(sel[1], alone1)


def test_slice_bounds_rejected():
    with pytest.raises(ValueError):
        oracle.slice_positions(10, 4, 0, 2)
    with pytest.raises(ValueError):
        oracle.slice_positions(8, 4, 3, 2)
    assert oracle.slice_positions(8, 4, 1, 3).tolist() == [1, 2, 5, 6]
    assert oracle.slice_positions(8, 4, 2, 2).size == 0


# ---------------------------------------------------------------------------
# fp8 e4m3 table widening
# ---------------------------------------------------------------------------

def test_e4m3_widening_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8).reshape(16, 16)
    got = oracle.gather_e4m3(np.arange(16), codes)  # [16, 16] bf16 bits
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float32)
    ref_bits = ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    finite = ~torch.isnan(ref).numpy()
    np.testing.assert_array_equal(got[finite], ref_bits[finite])
    # the two NaN codes stay NaN, with their sign
    nan_got = synth.bf16_bits_to_f32(got[~finite])
    assert np.all(np.isnan(nan_got)) and (~finite).sum() == 2
    # exactness: bf16 -> fp32 equals torch's fp8 -> fp32 on every finite code
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(got[finite]), ref.numpy()[finite])


def test_e4m3_spot_values():
    table = np.array([[0x38, 0x7E, 0x01, 0x80, 0xB8, 0x08, 0x07, 0x00] * 2], np.uint8)
    v = synth.bf16_bits_to_f32(oracle.gather_e4m3(np.array([0]), table))[0, :8]
    assert v.tolist() == [1.0, 448.0, 2.0 ** -9, -0.0, -1.0, 2.0 ** -6, 7 * 2.0 ** -9, 0.0]
    assert np.signbit(v[3])


# ---------------------------------------------------------------------------
# segment-aware causal dilated depthwise convolution (PLE layer's short conv):
# the API page builds it per packed segment as "history zeros ahead of the
# segment, then its own F.conv1d" (_segmented_conv); torch's conv1d on each
# zero-padded segment is therefore an independent statement of the same
# definition
# ---------------------------------------------------------------------------

def _conv_cases():
    rng = np.random.default_rng(17)
    # segments: empty, shorter than the receptive field, one token, long
    lens = [0, 5, 1, 40, 9, 10, 0, 27]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    for C, K, d in [(3, 4, 3), (5, 1, 1), (2, 4, 1), (4, 3, 5), (1, 8, 2)]:
        yield rng, cu, C, K, d


def _torch_segment_conv(x, cu, w, d, b):
    import torch
    out = []
    K = w.shape[1]
    for s in range(len(cu) - 1):
        if cu[s + 1] == cu[s]:
            continue  # an empty segment has no output rows
        seg = torch.from_numpy(x[cu[s]:cu[s + 1]]).T[None]  # [1, C, L]
        seg = torch.nn.functional.pad(seg, ((K - 1) * d, 0))
        y = torch.nn.functional.conv1d(seg, torch.from_numpy(w)[:, None, :], None if b is None else torch.from_numpy(b),
                                       dilation=d, groups=w.shape[0])
        out.append(y[0].T.numpy())
    return np.concatenate(out) if out else np.zeros((0, x.shape[1]))


def test_conv_matches_per_segment_conv1d():
    for rng, cu, C, K, d in _conv_cases():
        T = int(cu[-1])
        x = rng.standard_normal((T, C))
        w = rng.standard_normal((C, K))
        b = rng.standard_normal(C)
        for bias in (None, b):
            y = oracle.conv_forward(x, cu, w, d, bias)
            np.testing.assert_allclose(y, _torch_segment_conv(x, cu, w, d, bias), rtol=1e-12, atol=1e-12)


def test_conv_closed_forms():
    rng = np.random.default_rng(3)
    cu = np.array([0, 7, 7, 20, 21], np.int32)
    T, C, K, d = 21, 3, 4, 3
    x = rng.standard_normal((T, C))
    # only the last tap: the identity
    w = np.zeros((C, K)); w[:, K - 1] = 1.0
    np.testing.assert_array_equal(oracle.conv_forward(x, cu, w, d), x)
    # only tap K-1-m: a shift by m*d inside each segment, zeros at its start
    for m in range(1, K):
        w = np.zeros((C, K)); w[:, K - 1 - m] = 1.0
        want = np.zeros_like(x)
        for s in range(len(cu) - 1):
            lo, hi = cu[s], cu[s + 1]
            if hi - lo > m * d:
                want[lo + m * d:hi] = x[lo:hi - m * d]
        np.testing.assert_array_equal(oracle.conv_forward(x, cu, w, d), want)
    # bias alone
    b = rng.standard_normal(C)
    np.testing.assert_array_equal(oracle.conv_forward(x, cu, np.zeros((C, K)), d, b), np.broadcast_to(b, (T, C)))


def test_conv_causal_and_segment_local():
    rng = np.random.default_rng(4)
    cu = np.array([0, 12, 30], np.int32)
    x = rng.standard_normal((30, 2))
    w = rng.standard_normal((2, 4))
    y = oracle.conv_forward(x, cu, w, 3)
    x2 = x.copy()
    x2[20:] += 100.0  # later positions of segment 1
    y2 = oracle.conv_forward(x2, cu, w, 3)
    np.testing.assert_array_equal(y2[:20], y[:20])
    x3 = x.copy()
    x3[:12] -= 50.0   # all of segment 0
    y3 = oracle.conv_forward(x3, cu, w, 3)
    np.testing.assert_array_equal(y3[12:], y[12:])


def test_conv_backward_matches_autograd_and_adjoint():
    import torch
    for rng, cu, C, K, d in _conv_cases():
        T = int(cu[-1])
        x = rng.standard_normal((T, C))
        w = rng.standard_normal((C, K))
        dy = rng.standard_normal((T, C))
        dx, dw, db = oracle.conv_backward(dy, x, cu, w, d)
        xt = torch.from_numpy(x).requires_grad_(True)
        wt = torch.from_numpy(w).requires_grad_(True)
        bt = torch.zeros(C, dtype=torch.float64, requires_grad=True)
        outs = []
        for s in range(len(cu) - 1):
            if cu[s + 1] == cu[s]:
                continue
            seg = torch.nn.functional.pad(xt[cu[s]:cu[s + 1]].T[None], ((K - 1) * d, 0))
            outs.append(torch.nn.functional.conv1d(seg, wt[:, None, :], bt, dilation=d, groups=C)[0].T)
        (torch.cat(outs) * torch.from_numpy(dy)).sum().backward()
        np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(dw, wt.grad.numpy(), rtol=1e-12, atol=1e-11)
        np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-12, atol=1e-12)
        # adjoint identity on integers (exact in fp64): <conv(x), dy> = <x, dx>
        xi = rng.integers(-8, 9, (T, C)).astype(np.float64)
        wi = rng.integers(-4, 5, (C, K)).astype(np.float64)
        gi = rng.integers(-8, 9, (T, C)).astype(np.float64)
        dxi, dwi, _ = oracle.conv_backward(gi, xi, cu, wi, d)
        assert float((oracle.conv_forward(xi, cu, wi, d) * gi).sum()) == float((xi * dxi).sum())
        assert float((oracle.conv_forward(xi, cu, wi, d) * gi).sum()) == float((wi * dwi).sum())


# ---------------------------------------------------------------------------
# the oracle under AddressSanitizer / UndefinedBehaviorSanitizer
# ---------------------------------------------------------------------------

_SANITIZED_RUN = r"""
import hashlib, sys
import numpy as np
sys.path.insert(0, sys.argv[1])
import oracle, synth
h = hashlib.sha256()
rng = np.random.default_rng(3)
for n, G in ((2, 1), (3, 2), (4, 3)):
    lens = [0, 1, 7, 300, 0, 55]
    tok = rng.integers(0, 20, sum(lens))
    cu = synth.cu_seqlens_from_lengths(lens)
    mults = synth.signed_mults(n, rng)
    primes = synth.consecutive_primes(97, (n - 1) * G)
    offs = synth.exclusive_prefix(primes)
    rows = oracle.rows(tok, cu, n, G, 0, mults, primes, offs)
    rows_mt = oracle.rows(tok, cu, n, G, 0, mults, primes, offs, threads=3)
    table = rng.standard_normal((int(sum(primes)), 8)).astype(np.float32)
    out = oracle.gather(rows, table)
    codes = rng.integers(0, 256, (int(sum(primes)), 16)).astype(np.uint8)
    wide = oracle.gather_e4m3(rows, codes)
    g = rng.standard_normal((rows.size, 8)).astype(np.float32)
    uniq, sums = oracle.grad_sums(rows, g)
    _, sums_mt = oracle.grad_sums(rows, g, threads=3)
    tg = oracle.grad_apply(rows, g, np.zeros_like(table))
    x = rng.standard_normal((len(tok), 5))
    dy = rng.standard_normal((len(tok), 5))
    w = rng.standard_normal((5, 4))
    y = oracle.conv_forward(x, cu, w, n, rng.standard_normal(5))
    dx, dw, db = oracle.conv_backward(dy, x, cu, w, n)
    for a in (rows, rows_mt, out, wide, uniq, sums, sums_mt, tg, y, dx, dw, db):
        h.update(np.ascontiguousarray(a).tobytes())
print(h.hexdigest())
"""


def _libs_exist():
    import shutil

    if shutil.which("gcc") is None:
        return None
    out = []
    for lib in ("libasan.so", "libubsan.so"):
        p = subprocess.run(["gcc", f"-print-file-name={lib}"], capture_output=True, text=True).stdout.strip()
        if not os.path.isabs(p) or not os.path.exists(p):
            return None
        out.append(p)
    return out


def test_oracle_clean_under_asan_and_ubsan():
    """The oracle built with -fsanitize=address,undefined runs rows, gathers
    (bf16 / fp32 / E4M3), gradient sums (one and several threads) and the
    conv on ragged inputs (empty and one-token segments) without a report,
    and gives the same bytes as the normal build."""
    libs = _libs_exist()
    if libs is None:
        pytest.skip("gcc sanitizer runtimes not found")
    oracle.build(sanitize=True)
    env = dict(os.environ, PLE_ORACLE_SANITIZED="1", LD_PRELOAD=":".join(libs),
               ASAN_OPTIONS="detect_leaks=0:verify_asan_link_order=0:halt_on_error=1",
               UBSAN_OPTIONS="halt_on_error=1:print_stacktrace=1")
    r = subprocess.run([sys.executable, "-c", _SANITIZED_RUN, ROOT], env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-4000:]
    assert "runtime error" not in r.stderr and "AddressSanitizer" not in r.stderr, r.stderr[-4000:]
    plain = subprocess.run([sys.executable, "-c", _SANITIZED_RUN, ROOT], capture_output=True, text=True, timeout=600)
    assert plain.returncode == 0, plain.stderr[-2000:]
    assert r.stdout.strip() == plain.stdout.strip()
