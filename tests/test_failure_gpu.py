"""Failure detection on the GPU without a GPU fault.

The only waits between the blocks of a kernel are the radix sort's
look-back waits.  Each is bounded in time; the tests shorten the limit to 0
through include/ple_debug.h, so that every wait that does not succeed at
its first poll gives up, and check what the library promises then:

  * the call returns promptly and ple_status reports PLE_ERR_TIMEOUT;
  * the gradient is not applied at all (table_grad keeps its prefill,
    every row of it, bit for bit) and a prefetch reports zero distinct rows;
  * a call that happened to need no second poll is exact, as usual;
  * with the default limit restored, the same process computes exact
    results again (nothing stuck in the device or the workspace).

No kernel is made to fault, trap or hang: a wait that runs out is the normal
bounded-wait path, taken here with a limit of zero.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import custom_workload, dev_i32, dev_i64, small_table, torch_to_values

pytestmark = pytest.mark.gpu

R = 1_000_003  # 20-bit keys: three sort passes
D = 16


@pytest.fixture
def zero_wait_limit():
    prev = ple.set_wait_limit_ns(0)
    try:
        yield
    finally:
        ple.set_wait_limit_ns(prev)


def _inputs(N, seed, dev):
    rng = np.random.default_rng(seed)
    rows = rng.integers(0, R, N).astype(np.int64)
    g = synth.dense_values(seed, N * D, 1.0, synth.DTYPE_BF16).reshape(N, D)
    grad = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).to(dev)
    return rows, g, dev_i64(rows, dev), grad


def _plan():
    return ple.Plan(2, 1, 0, [1, 1], [R], [0], R, D, torch.bfloat16)


def test_sort_wait_timeout_leaves_table_grad_untouched(cuda_device, zero_wait_limit):
    dev = cuda_device
    plan = _plan()
    prefill = synth.dense_values(77, R * D, 0.5, synth.DTYPE_F32).reshape(R, D)
    timed_out = 0
    for attempt, N in enumerate([1 << 22, 1 << 23, 1 << 23]):
        rows_np, g_host, rows, grad = _inputs(N, 40 + attempt, dev)
        tg = torch.from_numpy(prefill).to(dev)
        ws = ple.alloc_workspace(plan, N, dev)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        ple.ple_grad_scatter(plan, rows, grad, tg, workspace=ws)
        st = ple.ple_status(dev)
        elapsed = time.perf_counter() - t0
        assert elapsed < 10.0, f"a call with a zero wait limit took {elapsed:.1f} s"
        got = tg.cpu().numpy()
        if st == ple.PLE_ERR_TIMEOUT:
            timed_out += 1
            # nothing applied: every row keeps its prefill, bit for bit
            np.testing.assert_array_equal(got.view(np.uint32), prefill.view(np.uint32))
        else:
            assert st == ple.PLE_OK
            ref = oracle.grad_apply(rows_np, g_host, prefill.copy())
            np.testing.assert_array_equal(got.view(np.uint32), ref.view(np.uint32))
        if timed_out:
            break
    assert timed_out, "no wait ran out even with a zero limit"


def test_prepare_apply_timeout_applies_nothing(cuda_device, zero_wait_limit):
    """The abort word travels in the workspace from the prepare to the apply."""
    dev = cuda_device
    plan = _plan()
    N = 1 << 23
    for seed in (50, 51, 52):
        _, _, rows, grad = _inputs(N, seed, dev)
        ws = ple.alloc_workspace(plan, N, dev)
        ple.ple_grad_prepare(plan, rows, ws)
        tg = torch.zeros(R, D, device=dev)
        ple.ple_grad_apply(plan, N, grad, tg, ws)
        st = ple.ple_status(dev)
        if st == ple.PLE_ERR_TIMEOUT:
            assert not tg.any()
            return
        assert st == ple.PLE_OK
    pytest.fail("no wait ran out even with a zero limit")


def test_prefetch_timeout_reports_no_rows(cuda_device, zero_wait_limit):
    dev = cuda_device
    rng = np.random.default_rng(9)
    T = 1 << 18
    tok = rng.integers(1, 1 << 30, T)
    w = custom_workload("pf_timeout", tok, [0, T], 3, 8, 0, synth.signed_mults(3, rng),
                        synth.consecutive_primes(100_003, 16), 8, synth.DTYPE_BF16, synth.DTYPE_BF16)
    plan = ple.Plan.from_workload(w)
    host_table = torch.zeros(w.num_rows, w.head_dim, dtype=torch.bfloat16).pin_memory()
    tokens, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    for _ in range(3):
        buf = ple.Prefetched(plan, T, dev)
        buf.num_unique.fill_(-7)
        ple.ple_prefetch(plan, tokens, cu, host_table, buf)
        st = ple.ple_status(dev)
        if st == ple.PLE_ERR_TIMEOUT:
            assert int(buf.num_unique.item()) == 0
            return
        assert st == ple.PLE_OK
    pytest.fail("no wait ran out even with a zero limit")


def test_default_limit_restored_gives_exact_results(cuda_device):
    """Runs after the zero-limit tests in the same process: the default
    limit is back and the same sizes are exact again."""
    dev = cuda_device
    assert ple.set_wait_limit_ns(ple.default_wait_limit_ns()) == ple.default_wait_limit_ns()
    plan = _plan()
    N = 1 << 22
    rows_np, g_host, rows, grad = _inputs(N, 60, dev)
    tg = torch.zeros(R, D, device=dev)
    ple.ple_grad_scatter(plan, rows, grad, tg)
    assert ple.ple_status(dev) == ple.PLE_OK
    ref = oracle.grad_apply(rows_np, g_host, np.zeros((R, D), np.float32))
    np.testing.assert_array_equal(tg.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    # and a small forward through the same library state
    w = synth.tiny(0)
    plan_t = ple.Plan.from_workload(w)
    host_table, table = small_table(w, dev)
    out = ple.ple_lookup(plan_t, dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev), table)
    assert ple.ple_status(dev) == ple.PLE_OK
    ref_rows = oracle.rows(w.tokens, w.cu_seqlens, w.ngram_size, w.heads_per_ngram, w.eos_id, w.mults, w.primes,
                           w.offsets)
    np.testing.assert_array_equal(torch_to_values(out), oracle.gather(ref_rows, host_table))


def test_status_is_per_plan_and_taken_once(cuda_device):
    """Two plans raise PLE_ERR_BAD_ROW on two streams: each plan's status
    reports its own flag exactly once, and one plan's read leaves the other
    plan's flag in place."""
    dev = cuda_device
    w = synth.tiny(0)
    p1, p2 = ple.Plan.from_workload(w), ple.Plan.from_workload(w)
    _, table = small_table(w, dev)
    bad = dev_i64(np.array([3, w.num_rows, 5], np.int64), dev)
    good = dev_i64(np.array([3, 4, 5], np.int64), dev)
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    with torch.cuda.stream(s1):
        ple.ple_gather(p1, bad, table)
    with torch.cuda.stream(s2):
        ple.ple_gather(p2, bad, table)
        ple.ple_gather(p2, good, table)
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        assert ple.ple_status(dev, plan=p1) == ple.PLE_ERR_BAD_ROW
        assert ple.ple_status(dev, plan=p1) == ple.PLE_OK  # taken once
    with torch.cuda.stream(s2):
        assert ple.ple_status(dev, plan=p2) == ple.PLE_ERR_BAD_ROW  # untouched by p1's read
        assert ple.ple_status(dev, plan=p2) == ple.PLE_OK
    # a plan-less read takes every word: a third plan's flag is seen there
    p3 = ple.Plan.from_workload(w)
    ple.ple_gather(p3, bad, table)
    assert ple.ple_status(dev) == ple.PLE_ERR_BAD_ROW
    assert ple.ple_status(dev, plan=p3) == ple.PLE_OK


def test_status_word_of_a_destroyed_plan_is_not_inherited(cuda_device):
    """A new plan that takes over a destroyed plan's status word does not
    see that plan's unread flags."""
    dev = cuda_device
    w = synth.tiny(0)
    _, table = small_table(w, dev)
    bad = dev_i64(np.array([w.num_rows + 1], np.int64), dev)
    for _ in range(3):
        p = ple.Plan.from_workload(w)
        ple.ple_gather(p, bad, table)
        torch.cuda.synchronize()
        del p  # its flag stays unread
        q = ple.Plan.from_workload(w)
        ple.ple_gather(q, dev_i64(np.array([1, 2], np.int64), dev), table)
        assert ple.ple_status(dev, plan=q) == ple.PLE_OK
        del q
    ple.ple_status(dev)  # clear the device
