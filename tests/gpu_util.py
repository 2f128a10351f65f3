"""Helpers shared by the GPU parity tests: host numpy <-> device tensors, the
comparison against the oracle, and the device status check."""
import numpy as np
import torch

from paged_kv_cache_380_b200 import ops


def dev(a: np.ndarray, tag: str) -> torch.Tensor:
    """Host array (bf16/f16 as uint16 bits) -> CUDA tensor of the real dtype."""
    a = np.ascontiguousarray(a)
    if tag == "bf16":
        return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
    if tag == "f16":
        return torch.from_numpy(a.view(np.float16)).cuda()
    if tag in ("f32", "i8", "i32", "i64"):
        return torch.from_numpy(a).cuda()
    raise ValueError(tag)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor -> host numpy with bf16/f16 as uint16 bits (exact bytes)."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def assert_close(got: np.ndarray, want: np.ndarray, atol: float, what: str):
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want)
    i = np.unravel_index(np.argmax(err), err.shape)
    assert err.max() <= atol, f"{what}: max abs err {err.max():.3e} at {i} (got {got[i]}, want {want[i]}) > {atol}"


def assert_status_ok():
    code, detail = ops.device_status()
    assert code == 0, f"device status {code} ({ops.error_string(code)}), detail {detail}"
