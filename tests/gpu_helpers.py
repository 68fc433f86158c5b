"""Helpers shared by the GPU parity tests (numpy <-> torch marshalling, bounds)."""
import numpy as np
import torch

TOL = 1e-3   # |y - y_ref| <= TOL * sum_k |s_g x_k| per element


def dev():
    return torch.device("cuda:0")


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).to(dev()).view(torch.bfloat16)


def fp16_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.int16)).to(dev()).view(torch.float16)


def words_dev(words: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(words, dtype=np.uint32).view(np.int32)).to(dev())


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def words_host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def bits16_host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def assert_within(y, y_ref, bound, tol=TOL, what=""):
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - y_ref)
    lim = tol * bound
    bad = err > lim
    if bad.any():
        idx = np.argwhere(bad)[:5]
        details = [(tuple(i), float(y[tuple(i)]), float(y_ref[tuple(i)]), float(lim[tuple(i)])) for i in idx]
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} elements outside "
                             f"{tol}*sum|s x|; first (index, got, ref, limit): {details}")
    return float((err / np.maximum(bound, 1e-300)).max())
