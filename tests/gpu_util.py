"""Helpers for the GPU parity tests: moving seeded numpy inputs to the device and
comparing against the oracle with the stated tolerances."""
import numpy as np
import torch

# Attention tolerance (bf16 inputs, fp32 accumulation), applied to the kernels' fp32
# result; the bf16 output must be exactly that result rounded to nearest even.
MAX_ABS = 1e-2
REL_L2 = 2e-3


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_f16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.float16).cuda()


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).astype(np.int32)).cuda()


def dev_u32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32).view(np.int32)).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close_attn(got: np.ndarray, want: np.ndarray, what: str = ""):
    err = np.abs(got - want)
    rel = np.linalg.norm((got - want).ravel()) / max(np.linalg.norm(want.ravel()), 1e-30)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)


def both_outputs(run):
    """run(out_dtype) -> tensor.  Returns the fp32 result after checking that the bf16
    output is exactly its round-to-nearest-even."""
    o32 = run(torch.float32)
    o16 = run(torch.bfloat16)
    torch.cuda.synchronize()
    assert o16.dtype == torch.bfloat16 and o32.dtype == torch.float32
    assert torch.equal(o16, o32.to(torch.bfloat16)), "bf16 output is not the rounded fp32 result"
    return o32
