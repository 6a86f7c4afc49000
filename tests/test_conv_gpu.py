"""The PLE layer's short convolution (segment-aware, causal, dilated,
depthwise) through the C ABI against the oracle.

Tolerances follow from the arithmetic: an output is an fp32 sum of at most
K + 1 terms (at most K + 1 roundings of at most 2^-24 of the magnitude sum
mag = |b| + sum |w x|), then rounded to the output type (bf16: half an ulp,
at most 2^-8 of the value); dw and db are fp32 sums over chunks of 256 or
512 tokens added in chunk order (at most 1024 chunks): at most (512 + 1024)
roundings of 2^-24 of their magnitude sums, inside 2^-14 of them.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import hashed_gram_embedding_ple_b200 as ple
from gpu_util import dev_i32, torch_to_values, values_to_torch

pytestmark = pytest.mark.gpu


def _as_f64(v, dtype_code):
    return synth.bf16_bits_to_f32(v).astype(np.float64) if dtype_code == synth.DTYPE_BF16 else v.astype(np.float64)


def _inputs(T, C, K, dt, seed):
    rng = np.random.default_rng(seed)
    x = synth.dense_values(seed + 1, T * C, 1.0, dt).reshape(T, C)
    g = synth.dense_values(seed + 2, T * C, 1.0, dt).reshape(T, C)
    w = rng.standard_normal((C, K)).astype(np.float32)
    b = rng.standard_normal(C).astype(np.float32)
    return x, g, w, b


def _check_close(got, ref, mag, rel, abs_scale):
    err = np.abs(got - ref)
    bound = rel * np.abs(ref) + abs_scale * mag + 1e-30
    assert np.all(err <= bound), f"max excess {np.max(err - bound)} at {np.unravel_index(np.argmax(err - bound), err.shape)}"


def run_case(dev, lens, C, K, d, dt, seed=0, with_bias=True):
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    x, g, w, b = _inputs(T, C, K, dt, seed)
    bias = b if with_bias else None
    xf, gf = _as_f64(x, dt), _as_f64(g, dt)
    xt, gt = values_to_torch(x, dt).to(dev), values_to_torch(g, dt).to(dev)
    wt = torch.from_numpy(w).to(dev)
    bt = torch.from_numpy(b).to(dev) if with_bias else None
    cut = dev_i32(cu, dev)
    y = ple.conv_forward(xt, cut, wt, d, bt)
    dw0 = np.linspace(-1, 1, C * K, dtype=np.float32).reshape(C, K)  # accumulate into a non-zero start
    db0 = np.linspace(1, 2, C, dtype=np.float32)
    dwt, dbt = torch.from_numpy(dw0.copy()).to(dev), torch.from_numpy(db0.copy()).to(dev)
    dx, _, _ = ple.conv_backward(gt, xt, cut, wt, d, dweight=dwt, dbias=dbt)
    assert ple.ple_status() == ple.PLE_OK
    rel_out = 2.0 ** -8 if dt == synth.DTYPE_BF16 else 0.0
    # forward
    ref = oracle.conv_forward(xf, cu, w, d, bias)
    mag = oracle.conv_forward(np.abs(xf), cu, np.abs(w), d, None if bias is None else np.abs(bias))
    _check_close(_as_f64(torch_to_values(y), dt), ref, mag, rel_out, 2.0 ** -20)
    # backward
    rdx, rdw, rdb = oracle.conv_backward(gf, xf, cu, w, d)
    mdx, mdw, mdb = oracle.conv_backward(np.abs(gf), np.abs(xf), cu, np.abs(w), d)
    _check_close(_as_f64(torch_to_values(dx), dt), rdx, mdx, rel_out, 2.0 ** -20)
    _check_close(dwt.cpu().numpy().astype(np.float64), dw0 + rdw, mdw + np.abs(dw0), 2.0 ** -23, 2.0 ** -14)
    _check_close(dbt.cpu().numpy().astype(np.float64), db0 + rdb, mdb + np.abs(db0), 2.0 ** -23, 2.0 ** -14)
    # the parameter gradients are bit-identical run to run; dx and y are elementwise
    dwt2, dbt2 = torch.from_numpy(dw0.copy()).to(dev), torch.from_numpy(db0.copy()).to(dev)
    dx2, _, _ = ple.conv_backward(gt, xt, cut, wt, d, dweight=dwt2, dbias=dbt2)
    assert torch.equal(dwt2.view(torch.int32), dwt.view(torch.int32))
    assert torch.equal(dbt2.view(torch.int32), dbt.view(torch.int32))
    assert torch.equal(dx2.view(torch.int16 if dt == synth.DTYPE_BF16 else torch.int32),
                       dx.view(torch.int16 if dt == synth.DTYPE_BF16 else torch.int32))
    # dx with the parameter gradients runs as one sweep, each alone as its own
    # kernel: the same sums in the same order, bit for bit
    dx3, _, _ = ple.conv_backward(gt, xt, cut, wt, d)
    dwt3, dbt3 = torch.from_numpy(dw0.copy()).to(dev), torch.from_numpy(db0.copy()).to(dev)
    ple.conv_backward(gt, xt, cut, wt, d, want_dx=False, dweight=dwt3, dbias=dbt3)
    assert torch.equal(dx3.view(torch.int16 if dt == synth.DTYPE_BF16 else torch.int32),
                       dx.view(torch.int16 if dt == synth.DTYPE_BF16 else torch.int32))
    assert torch.equal(dwt3.view(torch.int32), dwt.view(torch.int32))
    assert torch.equal(dbt3.view(torch.int32), dbt.view(torch.int32))


@pytest.mark.parametrize("C,K,d,dt", [
    (8, 4, 3, synth.DTYPE_BF16),     # one 16-byte channel vector
    (24, 4, 3, synth.DTYPE_BF16),    # 3 vectors
    (1032, 4, 3, synth.DTYPE_BF16),  # 129 vectors: two channel blocks, a ragged one
    (12, 1, 1, synth.DTYPE_F32),     # K = 1: a per-channel scale
    (20, 8, 2, synth.DTYPE_F32),
    (16, 3, 7, synth.DTYPE_BF16),
    (64, 2, 1, synth.DTYPE_F32),
    # long reach (K-1)*dilation: the history rows come from far back
    (16, 4, 6, synth.DTYPE_BF16),
    (8, 8, 3, synth.DTYPE_F32),
])
def test_conv_ragged_segments(cuda_device, C, K, d, dt):
    # empty segments, one-token segments, segments shorter than the receptive field
    lens = [0, 1, 5, 40, 0, 9, 10, 3, 200, 1]
    run_case(cuda_device, lens, C, K, d, dt, seed=C + K)


def test_conv_many_chunks(cuda_device):
    # crosses many forward (64-token) and backward (256-token) chunks, and segments inside them
    rng = np.random.default_rng(5)
    lens = list(rng.integers(1, 700, 14)) + [0, 2]
    run_case(cuda_device, lens, 64, 4, 3, synth.DTYPE_BF16, seed=9)
    run_case(cuda_device, lens, 32, 4, 3, synth.DTYPE_F32, seed=10, with_bias=False)


def test_conv_single_segment_and_dx_only(cuda_device):
    dev = cuda_device
    T, C, K, d = 777, 16, 4, 3
    x, g, w, b = _inputs(T, C, K, synth.DTYPE_BF16, 3)
    cu = np.array([0, T], np.int32)
    xt, gt = values_to_torch(x, synth.DTYPE_BF16).to(dev), values_to_torch(g, synth.DTYPE_BF16).to(dev)
    dx, dw, db = ple.conv_backward(gt, xt, dev_i32(cu, dev), torch.from_numpy(w).to(dev), d)
    assert dw is None and db is None
    rdx, _, _ = oracle.conv_backward(_as_f64(g, 1), _as_f64(x, 1), cu, w, d)
    mdx, _, _ = oracle.conv_backward(np.abs(_as_f64(g, 1)), np.abs(_as_f64(x, 1)), cu, np.abs(w), d)
    _check_close(_as_f64(torch_to_values(dx), 1), rdx, mdx, 2.0 ** -8, 2.0 ** -20)


def test_conv_empty_and_host_errors(cuda_device):
    dev = cuda_device
    x = torch.empty(0, 8, dtype=torch.bfloat16, device=dev)
    cu = torch.zeros(2, dtype=torch.int32, device=dev)
    w = torch.zeros(8, 4, device=dev)
    assert ple.conv_forward(x, cu, w, 3).shape == (0, 8)
    with pytest.raises(ple.PleError):
        ple.conv_forward(torch.zeros(4, 8, dtype=torch.bfloat16, device=dev), torch.tensor([0, 4], dtype=torch.int32,
                         device=dev), torch.zeros(8, 9, device=dev), 3)  # K > 8
    with pytest.raises(ple.PleError):
        ple.conv_forward(torch.zeros(4, 4, dtype=torch.bfloat16, device=dev), torch.tensor([0, 4], dtype=torch.int32,
                         device=dev), torch.zeros(4, 4, device=dev), 3)  # 8-byte rows


def test_conv_malformed_seqlens_flagged(cuda_device):
    dev = cuda_device
    T, C = 50, 8
    x = torch.ones(T, C, dtype=torch.bfloat16, device=dev)
    w = torch.ones(C, 4, device=dev)
    for cu in ([0, 30, 20, 50], [0, 30, 60], [5, 50]):  # decreasing, past the end, not starting at 0
        ple.conv_forward(x, torch.tensor(cu, dtype=torch.int32, device=dev), w, 3)
        assert ple.ple_status() == ple.PLE_ERR_BAD_SEQLENS


def test_conv_full_size_sampled(cuda_device):
    """The bench's conv workload (32768 packed tokens of the single-layer
    packing, 8192 bf16 channels, K = 4, dilation 3): every token of 256
    sampled ones and dw / db of 64 sampled channels against the oracle."""
    from synth import gpu as sgpu

    dev = cuda_device
    w_ = synth.single_layer_bf16(0)
    cu = w_.cu_seqlens
    T, C, K, d = int(cu[-1]), 8192, 4, 3
    xt = torch.empty(T, C, dtype=torch.bfloat16, device=dev)
    gt = torch.empty(T, C, dtype=torch.bfloat16, device=dev)
    sgpu.fill_(xt, 11, 1.0)
    sgpu.fill_(gt, 12, 1.0)
    rng = np.random.default_rng(0)
    w = rng.standard_normal((C, K)).astype(np.float32)
    b = rng.standard_normal(C).astype(np.float32)
    cut = dev_i32(cu, dev)
    y = ple.conv_forward(xt, cut, torch.from_numpy(w).to(dev), d, torch.from_numpy(b).to(dev))
    dwt = torch.zeros(C, K, device=dev)
    dbt = torch.zeros(C, device=dev)
    dx, _, _ = ple.conv_backward(gt, xt, cut, torch.from_numpy(w).to(dev), d, dweight=dwt, dbias=dbt)
    assert ple.ple_status() == ple.PLE_OK
    span = (K - 1) * d
    seg_of = np.searchsorted(cu, np.arange(T), side="right") - 1
    for t in rng.integers(0, T, 256):
        # y[t] reads positions max(segment start, t - span) .. t: the oracle on
        # exactly that window (taken as one segment) gives y[t] at its end
        lo = max(int(cu[seg_of[t]]), int(t) - span)
        idx = np.arange(lo, t + 1, dtype=np.uint64)
        xs = _as_f64(synth.counter_values(11, idx[:, None] * np.uint64(C) + np.arange(C, dtype=np.uint64), 1.0,
                                          synth.DTYPE_BF16), 1)
        win = np.array([0, t + 1 - lo], np.int32)
        ref = oracle.conv_forward(xs, win, w, d, b)[-1]
        mag = oracle.conv_forward(np.abs(xs), win, np.abs(w), d, np.abs(b))[-1]
        _check_close(_as_f64(torch_to_values(y[t:t + 1]), 1)[0], ref, mag, 2.0 ** -8, 2.0 ** -20)
    cols = rng.choice(C, 64, replace=False)
    allrows = np.arange(T, dtype=np.uint64)[:, None] * np.uint64(C)
    xs = _as_f64(synth.counter_values(11, allrows + cols.astype(np.uint64), 1.0, synth.DTYPE_BF16), 1)
    gs = _as_f64(synth.counter_values(12, allrows + cols.astype(np.uint64), 1.0, synth.DTYPE_BF16), 1)
    rdx, rdw, rdb = oracle.conv_backward(gs, xs, cu, w[cols], d)
    mdx, mdw, mdb = oracle.conv_backward(np.abs(gs), np.abs(xs), cu, np.abs(w[cols]), d)
    _check_close(dwt.cpu().numpy()[cols].astype(np.float64), rdw, mdw, 2.0 ** -23, 2.0 ** -14)
    _check_close(dbt.cpu().numpy()[cols].astype(np.float64), rdb, mdb, 2.0 ** -23, 2.0 ** -14)
    _check_close(_as_f64(torch_to_values(dx[:, torch.from_numpy(cols).to(dev)]), 1), rdx, mdx, 2.0 ** -8, 2.0 ** -20)
