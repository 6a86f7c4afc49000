"""ple_grad_scatter_noalloc: the gradient for callers that cannot allocate.

Serving processes with device memory reserved up front, plugin hosts that
may not call the CUDA allocator, or hot loops where cudaMalloc would
synchronise the device cannot pass the workspace ple_grad_scatter needs.
The no-allocation entry point runs the same kernels in a fixed scratch area
that the library keeps in device memory.  These tests call it through the C
ABI and hold it to the workspace entry point's result and to the CPU
oracle, bit for bit (the gradient is deterministic), on calls in a row with
different inputs, so that anything a call leaves behind in the shared
scratch area would show.  The last call uses the largest hit count whose
workspace fits the scratch area (the sort's 4096-key tiles).
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from hashed_gram_embedding_ple_b200 import binding
from gpu_util import custom_workload


def _plan(D=128):
    return ple.Plan(2, 1, 0, [1, 1], [70_001], [0], 70_001, D, torch.float32)


def test_noalloc_rejects_sizes_beyond_scratch():
    """Checked on the host before any launch (no GPU needed)."""
    lib = ple.lib()
    plan = _plan()
    cap = lib.ple_grad_scatter_noalloc_scratch_bytes()
    assert cap == 32 << 20
    n = 1
    while ple.workspace_bytes(plan, n) <= cap:
        n *= 2
    rc = lib.ple_grad_scatter_noalloc(plan.handle, ctypes.c_void_p(0x1000), n, ctypes.c_void_p(0x2000),
                                      binding.PLE_BF16, ctypes.c_void_p(0x3000), None)
    assert rc == binding.PLE_ERR_WORKSPACE


def _inputs(N, D, seed, dev):
    rng = np.random.default_rng(seed)
    rows = synth.zipf_ids(N, 1.3, 70_001, rng)
    w = custom_workload("noalloc", np.zeros(1, np.int64), [0, 1], 2, 1, 0, [1, 1], [70_001], D, synth.DTYPE_F32,
                        synth.DTYPE_BF16, seed=seed)
    g = synth.dense_values(w.grad_seed, N * D, 1.0, synth.DTYPE_BF16).reshape(N, D)
    grad = torch.from_numpy(g.view(np.int16)).view(torch.bfloat16).to(dev)
    return rows, g, torch.from_numpy(rows).to(dev), grad


def _largest_fitting(plan, cap):
    lo, hi = 1, 1
    while ple.workspace_bytes(plan, hi) <= cap:
        lo, hi = hi, 2 * hi
    while hi - lo > 1:  # workspace_bytes is non-decreasing in N
        mid = (lo + hi) // 2
        if ple.workspace_bytes(plan, mid) <= cap:
            lo = mid
        else:
            hi = mid
    return lo


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_and_oracle(cuda_device):
    dev = cuda_device
    lib = ple.lib()
    D = 128
    plan = _plan(D)
    cap = lib.ple_grad_scatter_noalloc_scratch_bytes()
    n_max = _largest_fitting(plan, cap)
    assert n_max >= 3 << 17, "the largest fitting size must reach the 4096-key sort tiles"
    stream = torch.cuda.current_stream(dev).cuda_stream
    for call, (N, seed) in enumerate([(3 * 4096 + 777, 11), (40_000, 12), (n_max, 13)]):
        assert ple.workspace_bytes(plan, N) <= cap
        rows_np, g_host, rows, grad = _inputs(N, D, seed, dev)
        ref = torch.zeros(70_001, D, device=dev)
        ple.ple_grad_scatter(plan, rows, grad, ref)
        got = torch.zeros(70_001, D, device=dev)
        rc = lib.ple_grad_scatter_noalloc(plan.handle, rows.data_ptr(), N, grad.data_ptr(), binding.PLE_BF16,
                                          got.data_ptr(), stream)
        assert rc == binding.PLE_OK, f"call {call}: status {rc}"
        assert ple.ple_status(dev) == ple.PLE_OK
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32)), f"call {call} differs"
        want = oracle.grad_apply(rows_np, g_host, np.zeros((70_001, D), np.float32))
        np.testing.assert_array_equal(got.cpu().numpy().view(np.uint32), want.view(np.uint32),
                                      err_msg=f"call {call} differs from the oracle")
