"""Helpers shared by the tests: tensor <-> numpy bit views, buffer allocation."""
import numpy as np
import torch


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy array of its bit patterns (CPU copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def from_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def act_buffers(M, K, dev, colwise=True):
    q_row = torch.empty((M, K), dtype=torch.uint8, device=dev)
    s_row = torch.empty((K // 128, M), dtype=torch.float32, device=dev)
    if not colwise:
        return q_row, s_row, None, None
    q_col = torch.empty((K, M), dtype=torch.uint8, device=dev)
    s_col = torch.empty((M // 128, K), dtype=torch.float32, device=dev)
    return q_row, s_row, q_col, s_col


def weight_buffers(N, K, dev, transposed=True):
    q = torch.empty((N, K), dtype=torch.uint8, device=dev)
    s = torch.empty((N // 128, K // 128), dtype=torch.float32, device=dev)
    qT = torch.empty((K, N), dtype=torch.uint8, device=dev) if transposed else None
    return q, s, qT


def assert_bytes_equal(got: np.ndarray, want: np.ndarray, what: str):
    if got.shape != want.shape:
        raise AssertionError(f"{what}: shape {got.shape} != {want.shape}")
    bad = np.argwhere(got.view(np.uint8).reshape(got.shape[0], -1) != want.view(np.uint8).reshape(want.shape[0], -1))
    if bad.size:
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} differing bytes, first at {i}")
