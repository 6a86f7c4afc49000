"""The hot path captured into a CUDA graph and replayed.

A serving or training loop can capture the lookup and the deterministic
gradient once and replay them: every call is asynchronous on the given
stream, takes its scratch from the caller's workspace and launches a fixed
set of kernels.  The first call of a plan on a device looks up the library's
device addresses and clears the plan's status word, so it is made before the
capture.  The replays must give the same bits as eager calls.
"""
import numpy as np
import pytest
import torch

import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import dev_i32, dev_i64, device_grad, device_table

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tokens", [20_000, 200_000])  # 2048- and 8192-key sort tiles
def test_lookup_and_gradient_replay_from_a_graph(cuda_device, tokens):
    dev = cuda_device
    w = synth.sweep_point(tokens=tokens, head_dim=64, ngram_size=3, heads_per_ngram=8, table_gb=0.5, seed=3)
    plan = ple.Plan.from_workload(w)
    table = device_table(w, dev)
    tok, cu = dev_i64(w.tokens, dev), dev_i32(w.cu_seqlens, dev)
    T, H, D = w.num_tokens, w.num_heads, w.head_dim
    grad = device_grad(w, dev)
    ws = ple.alloc_workspace(plan, T * H, dev)
    out = torch.empty(T, H, D, dtype=torch.bfloat16, device=dev)
    rows = torch.empty(T, H, dtype=torch.int64, device=dev)
    tg = torch.zeros(w.num_rows, D, device=dev)

    def step():
        ple.ple_lookup(plan, tok, cu, table, out=out, rows_out=rows)
        ple.ple_grad_scatter(plan, rows.view(-1), grad, tg, workspace=ws)

    step()  # eager, also the plan's first call on the device
    assert ple.ple_status(dev, plan=plan) == ple.PLE_OK
    ref_out, ref_rows, ref_tg = out.clone(), rows.clone(), tg.clone()

    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        step()  # warm the side stream too (outside the capture)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    for _ in range(3):
        out.zero_()
        rows.zero_()
        tg.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert ple.ple_status(dev, plan=plan) == ple.PLE_OK
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(rows, ref_rows)
        assert torch.equal(tg.view(torch.int32), ref_tg.view(torch.int32))
    del graph


def test_conv_replay_from_a_graph(cuda_device):
    dev = cuda_device
    rng = np.random.default_rng(8)
    lens = [700, 0, 3000, 1, 2000]
    T, C, K, d = sum(lens), 512, 4, 3
    x = torch.from_numpy(rng.standard_normal((T, C)).astype(np.float32)).to(dev).to(torch.bfloat16)
    dy = torch.from_numpy(rng.standard_normal((T, C)).astype(np.float32)).to(dev).to(torch.bfloat16)
    wt = torch.from_numpy(rng.standard_normal((C, K)).astype(np.float32)).to(dev)
    cu = dev_i32(synth.cu_seqlens_from_lengths(lens), dev)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    dw, db = torch.zeros(C, K, device=dev), torch.zeros(C, device=dev)
    ws = torch.empty(ple.conv_workspace_bytes(T, C, K), dtype=torch.uint8, device=dev)

    def step():
        ple.conv_forward(x, cu, wt, d, out=y)
        ple.conv_backward(dy, x, cu, wt, d, dx=dx, dweight=dw, dbias=db, workspace=ws)

    step()
    assert ple.ple_status(dev) == ple.PLE_OK
    ref = [t.clone() for t in (y, dx, dw, db)]
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.current_stream(dev).wait_stream(side)
    for _ in range(2):
        for t in (y, dx, dw, db):
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        got = (y, dx, dw, db)
        for a, b in zip(got, ref):
            assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                               b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))
    assert ple.ple_status(dev) == ple.PLE_OK
    del graph
