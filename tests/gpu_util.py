"""Helpers for the GPU tests: move seeded inputs to the device and back."""
import numpy as np
import torch

import synth


def dev_i64(a, device):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int64)).to(device)


def dev_i32(a, device):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


TORCH_DTYPE = {synth.DTYPE_F32: torch.float32, synth.DTYPE_BF16: torch.bfloat16,
               synth.DTYPE_E4M3: torch.float8_e4m3fn}


def values_to_torch(v: np.ndarray, dtype_code: int) -> torch.Tensor:
    """Host generator output (fp32, bf16 bits as uint16 or fp8 codes as
    uint8) as a CPU tensor."""
    if dtype_code == synth.DTYPE_F32:
        return torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32))
    if dtype_code == synth.DTYPE_E4M3:
        return torch.from_numpy(np.ascontiguousarray(v, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return torch.from_numpy(np.ascontiguousarray(v, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def torch_to_values(t: torch.Tensor) -> np.ndarray:
    """Device tensor back to the host representation (fp32, bf16 bits or fp8 codes)."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8).numpy()
    return t.numpy()


def small_table(w, device):
    """Whole table generated on the host (small workloads only)."""
    v = synth.dense_values(w.table_seed, w.num_rows * w.head_dim, w.table_sigma, w.table_dtype)
    host = v.reshape(w.num_rows, w.head_dim)
    return host, values_to_torch(host, w.table_dtype).to(device)


def device_table(w, device):
    """Table generated on the device by the twin generator (large workloads)."""
    from synth import gpu as sgpu

    t = torch.empty(w.num_rows, w.head_dim, dtype=TORCH_DTYPE[w.table_dtype], device=device)
    sgpu.fill_(t, w.table_seed, w.table_sigma)
    return t


def device_grad(w, device, num_hits=None):
    from synth import gpu as sgpu

    n = w.num_hits if num_hits is None else num_hits
    dt = torch.float32 if w.grad_dtype == synth.DTYPE_F32 else torch.bfloat16
    g = torch.empty(n, w.head_dim, dtype=dt, device=device)
    sgpu.fill_(g, w.grad_seed, w.grad_sigma)
    return g


def host_grad(w, num_hits=None):
    n = w.num_hits if num_hits is None else num_hits
    return synth.dense_values(w.grad_seed, n * w.head_dim, w.grad_sigma, w.grad_dtype).reshape(n, w.head_dim)


def custom_workload(name, tokens, cu, n, G, eos, mults, primes, D, table_dtype=synth.DTYPE_F32,
                    grad_dtype=synth.DTYPE_F32, seed=0):
    primes = np.asarray(primes, np.int64)
    offsets = np.asarray(synth.exclusive_prefix(primes), np.int64)
    return synth.Workload(name, np.asarray(tokens, np.int64), np.asarray(cu, np.int32), n, G, eos,
                          np.asarray(mults, np.int64), primes, offsets, int(primes.sum()), D, table_dtype,
                          seed + 101, 0.02, grad_dtype, seed + 202, 1.0)
