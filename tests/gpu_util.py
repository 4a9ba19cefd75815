"""Shared helpers of the GPU parity tests: move seeded numpy inputs to the device, run the
CUDA path through the C ABI, and compare with the oracle."""
import numpy as np
import torch

from moe_grouped_gemm_sm_b200 import synth


def dev(arr, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def bf16_dev(bits):
    return dev(np.ascontiguousarray(bits, np.uint16).view(np.int16), torch.bfloat16)


def host(t):
    return t.cpu().numpy()


def bf16_host_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_close(d, ref, what=""):
    """The accuracy bound |D - ref| <= 2^-7·|ref| + 1e-2·rms(ref), element by element."""
    import oracle
    ok, ratio = oracle.tolerance_ok(d, ref)
    if not ok:
        err = np.abs(d - ref)
        i = np.unravel_index(np.argmax(err / (2 ** -7 * np.abs(ref) + 1e-2 * np.sqrt(np.mean(ref ** 2)))), ref.shape)
        raise AssertionError(f"{what}: worst error/bound = {ratio:.3f} at {i}: got {d[i]}, ref {ref[i]}")
    return ratio


def sentinel_fill(shape):
    return torch.full(shape, synth.sentinel_bf16(), dtype=torch.int16, device="cuda").view(torch.bfloat16) \
        if synth.sentinel_bf16() < 0x8000 else \
        torch.full(shape, synth.sentinel_bf16() - 0x10000, dtype=torch.int16, device="cuda").view(torch.bfloat16)
