"""Helpers shared by the GPU parity tests: moving bf16 bit patterns between
numpy and CUDA tensors, and the parity tolerance.

Parity bar (per output tensor):
    max |gpu - oracle| <= 1e-2 * max |oracle| + 1e-3
with bf16 storage and fp32 accumulation on the GPU and the float64 oracle on
the CPU.
"""
import numpy as np

from oracle import flashsvd_oracle as oracle

REL_TOL = 1e-2
ABS_TOL = 1e-3


def dev_bf16(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy())
    return t.view(torch.bfloat16).cuda()


def host_bits(t) -> np.ndarray:
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f64(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return oracle.from_bf16(host_bits(t))
    return t.detach().double().cpu().numpy()


def parity_err(gpu: np.ndarray, ref: np.ndarray):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    err = float(np.max(np.abs(gpu - ref))) if ref.size else 0.0
    bound = REL_TOL * (float(np.max(np.abs(ref))) if ref.size else 0.0) + ABS_TOL
    return err, bound


def assert_parity(gpu, ref, what=""):
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    err, bound = parity_err(gpu, ref)
    assert err <= bound, f"{what}: max|gpu-oracle| = {err:.3e} > {bound:.3e}"
    return err, bound
