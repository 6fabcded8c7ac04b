"""Helpers shared by the GPU parity tests: run the CUDA path (through the C
ABI) and the CPU oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import serq_oracle as O

TOL_REL = 1e-2     # |y - y_ref| <= 1e-2 * max(|y_ref|, 1e-3)
TOL_FLOOR = 1e-3


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_act(a: np.ndarray, act_dtype: str) -> torch.Tensor:
    t = dev(a.astype(np.float32))
    return t.to(torch.bfloat16) if act_dtype == "bf16" else t


def expected_packed(ol: O.PreparedLayer):
    """Packed bytes the oracle's codes give in the library's storage format."""
    wq = O.pack_int4_rows(np.ascontiguousarray(ol.q_w.T))
    N = ol.q_w.shape[1]
    rpad = (ol.r + 31) // 32 * 32
    qr = np.zeros((N, rpad), np.int8)
    if ol.r:
        qr[:, :ol.r] = ol.q_r.T
    rq = O.pack_int4_rows(qr) if rpad else np.zeros((N, 0), np.uint8)
    return wq, rq


def act_bytes(codes: np.ndarray, bits: int) -> np.ndarray:
    if bits == 4:
        return O.pack_int4_rows(codes)
    return codes.astype(np.int8).view(np.uint8)


def assert_y_close(y_gpu: torch.Tensor, y_ref: np.ndarray):
    y = y_gpu.float().cpu().numpy().astype(np.float64)
    err = np.abs(y - y_ref)
    bound = TOL_REL * np.maximum(np.abs(y_ref), TOL_FLOOR)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{bad.sum()} of {bad.size} outputs outside tolerance; first at {tuple(i)}: "
                             f"gpu {y[tuple(i)]!r} ref {y_ref[tuple(i)]!r}")


def bits(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
