"""Seeded synthetic inputs for the SERQ quantized linear.

This module only draws random numbers and rounds them to storage formats.  It
holds none of the method's arithmetic (no smoothing, ranking, quantization or
GEMM), so both the CPU oracle's tests and the CUDA path can take their inputs
from it without sharing any of the method.

Workloads (all seeded with numpy PCG64):

* ``tiny``   -- one 256x256 layer, 16 tokens, 4 outlier channels x50, 64
  calibration tokens, r = 16, fp32 activations.
* ``llama2_7b`` -- Llama-2-7B decoder-layer projections: q/k/v/o 4096x4096,
  gate/up 4096x11008, down 11008x4096; weights ~ N(0, 0.02^2); activations
  ~ N(0, 1) with round(0.5% of K) channels scaled by a factor drawn
  log-uniformly in [20, 100] (fixed per layer input); 512 calibration tokens;
  bf16 activations.
* ``llama3_8b`` -- Llama-3-8B projections (GQA k/v 4096x1024, MLP 14336).

The outlier structure stands in for the channel-wise activation outliers the
SERQ notes (papernotes.org, ICLR 2026, "research background") describe for
LLaMA-2/3; the pages' own LLaMA checkpoints and WikiText/Pile calibration data
are not available, so these synthetic draws replace them.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Tuple

import numpy as np

WEIGHT_STD = 0.02


# --------------------------------------------------------------------------
# storage-format helpers (bf16 <-> fp32 bit patterns, round-to-nearest-even)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 array whose values are exactly representable in bf16."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# --------------------------------------------------------------------------
# draws
# --------------------------------------------------------------------------
def draw_weight(rng: np.random.Generator, K: int, N: int) -> np.ndarray:
    """W is d_in x d_out (K x N), Y = X W, entries ~ N(0, 0.02^2), fp32."""
    w = rng.standard_normal((K, N), dtype=np.float32)
    w *= np.float32(WEIGHT_STD)
    return w


def draw_outlier_channels(rng: np.random.Generator, K: int, n_out: int,
                          fixed_factor: float | None = None) -> Tuple[np.ndarray, np.ndarray]:
    """Pick ``n_out`` distinct channels and a magnitude factor for each."""
    ch = np.sort(rng.choice(K, size=n_out, replace=False)).astype(np.int64)
    if fixed_factor is not None:
        fac = np.full(n_out, fixed_factor, dtype=np.float32)
    else:
        fac = np.exp(rng.uniform(np.log(20.0), np.log(100.0), size=n_out)).astype(np.float32)
    return ch, fac


def draw_activations(rng: np.random.Generator, M: int, K: int,
                     channels: np.ndarray, factors: np.ndarray) -> np.ndarray:
    """Tokens x channels, ~ N(0,1) with the given outlier channels scaled."""
    x = rng.standard_normal((M, K), dtype=np.float32)
    if len(channels):
        x[:, channels] *= factors[None, :]
    return x


@dataclasses.dataclass
class LayerInput:
    """One activation stream feeding one or more projections."""
    name: str
    K: int
    X: np.ndarray          # M x K fp32 (bf16-representable when bf16 is set)
    X_calib: np.ndarray    # n_calib x K fp32 (same rounding)
    channels: np.ndarray
    factors: np.ndarray


@dataclasses.dataclass
class Projection:
    name: str
    input: str             # which LayerInput feeds it
    W: np.ndarray          # K x N fp32


@dataclasses.dataclass
class Workload:
    name: str
    M: int
    rank: int
    mode: str              # "w4a4" or "w4a8"
    act_dtype: str         # "f32" or "bf16"
    inputs: Dict[str, LayerInput]
    projections: List[Projection]
    groups: Dict[str, List[str]]   # shared-input groups: input name -> projections

    def shapes(self):
        return [(p.name, p.W.shape[0], p.W.shape[1]) for p in self.projections]


def _n_outliers(K: int) -> int:
    return int(round(0.005 * K))


def _make_input(rng, name, M, K, n_calib, bf16, n_out=None, fixed_factor=None):
    n_out = _n_outliers(K) if n_out is None else n_out
    ch, fac = draw_outlier_channels(rng, K, n_out, fixed_factor)
    X = draw_activations(rng, M, K, ch, fac)
    Xc = draw_activations(rng, n_calib, K, ch, fac)
    if bf16:
        X = round_to_bf16(X)
        Xc = round_to_bf16(Xc)
    return LayerInput(name, K, X, Xc, ch, fac)


# projection tables (name, input stream, K, N)
LLAMA2_7B = [
    ("q_proj", "attn_in", 4096, 4096),
    ("k_proj", "attn_in", 4096, 4096),
    ("v_proj", "attn_in", 4096, 4096),
    ("o_proj", "o_in", 4096, 4096),
    ("gate_proj", "mlp_in", 4096, 11008),
    ("up_proj", "mlp_in", 4096, 11008),
    ("down_proj", "down_in", 11008, 4096),
]

LLAMA3_8B = [
    ("q_proj", "attn_in", 4096, 4096),
    ("k_proj", "attn_in", 4096, 1024),
    ("v_proj", "attn_in", 4096, 1024),
    ("o_proj", "o_in", 4096, 4096),
    ("gate_proj", "mlp_in", 4096, 14336),
    ("up_proj", "mlp_in", 4096, 14336),
    ("down_proj", "down_in", 14336, 4096),
]


def _table_workload(name, table, M, rank, mode, seed, n_calib=512, only=None,
                    m_scale=None):
    rng = np.random.default_rng(seed)
    inputs: Dict[str, LayerInput] = {}
    projs: List[Projection] = []
    groups: Dict[str, List[str]] = {}
    for pname, iname, K, N in table:
        if iname not in inputs:
            inputs[iname] = _make_input(rng, iname, M, K, n_calib, bf16=True)
        # every weight is drawn (keeps the stream identical whether or not a
        # subset is requested)
        W = draw_weight(rng, K, N)
        if only is not None and pname not in only:
            continue
        projs.append(Projection(pname, iname, W))
        groups.setdefault(iname, []).append(pname)
    inputs = {k: v for k, v in inputs.items() if k in groups}
    return Workload(name, M, rank, mode, "bf16", inputs, projs, groups)


def tiny(seed: int = 0) -> Workload:
    """16 tokens x 256 -> 256, 4 outlier channels x50, r = 16, W4A4, fp32."""
    rng = np.random.default_rng(seed)
    inp = _make_input(rng, "x", 16, 256, 64, bf16=False, n_out=4, fixed_factor=50.0)
    W = draw_weight(rng, 256, 256)
    return Workload("tiny", 16, 16, "w4a4", "f32", {"x": inp},
                    [Projection("linear", "x", W)], {"x": ["linear"]})


def llama2_7b(M: int = 2048, seed: int = 1, only=None) -> Workload:
    """Llama-2-7B-shaped projections, W4A4, r = 128 (M = 2048 prefill)."""
    return _table_workload("llama2_7b", LLAMA2_7B, M, 128, "w4a4", seed, only=only)


def llama3_8b(M: int = 4096, seed: int = 2, only=None) -> Workload:
    """Llama-3-8B-shaped projections, W4A8, r = 128 (M = 4096)."""
    return _table_workload("llama3_8b", LLAMA3_8B, M, 128, "w4a8", seed, only=only)


def custom_layer(M: int, K: int, N: int, rank: int, mode: str = "w4a4",
                 act_dtype: str = "bf16", seed: int = 7, n_calib: int = 64,
                 n_outliers: int | None = None) -> Workload:
    """One layer of arbitrary shape with the same distributions (for sweeps)."""
    rng = np.random.default_rng(seed)
    inp = _make_input(rng, "x", M, K, n_calib, bf16=(act_dtype == "bf16"),
                      n_out=n_outliers)
    W = draw_weight(rng, K, N)
    return Workload(f"layer_{M}x{K}x{N}_r{rank}", M, rank, mode, act_dtype,
                    {"x": inp}, [Projection("linear", "x", W)], {"x": ["linear"]})


@dataclasses.dataclass
class MLPBlock:
    """Llama MLP: gate/up (K x F) -> silu(g)*u -> down (F x K)."""
    M: int
    rank: int
    X: np.ndarray           # M x K bf16-representable fp32
    X_calib: np.ndarray     # n_calib x K
    Wg: np.ndarray          # K x F
    Wu: np.ndarray          # K x F
    Wd: np.ndarray          # F x K
    H_calib: np.ndarray     # n_calib x F: fp32 unquantized silu(Xc Wg) * (Xc Wu)


def _silu_f64(x):
    return x / (1.0 + np.exp(-x))


def mlp_block(M: int = 4096, K: int = 4096, F: int = 11008, rank: int = 128,
              seed: int = 3, n_calib: int = 512) -> MLPBlock:
    """Synthetic MLP block.  The calibration activations of down_proj are the
    block's own full-precision intermediate on the calibration tokens (a plain
    forward of the unquantized model, not part of the method)."""
    rng = np.random.default_rng(seed)
    inp = _make_input(rng, "mlp_in", M, K, n_calib, bf16=True)
    Wg = draw_weight(rng, K, F)
    Wu = draw_weight(rng, K, F)
    Wd = draw_weight(rng, F, K)
    xc = inp.X_calib.astype(np.float64)
    h = _silu_f64(xc @ Wg.astype(np.float64)) * (xc @ Wu.astype(np.float64))
    return MLPBlock(M, rank, inp.X, inp.X_calib, Wg, Wu, Wd, h.astype(np.float32))


def factor_pair(K: int, N: int, r: int, seed: int = 11, err_std: float = 3e-3):
    """Two seeded low-rank factors shaped like the scaled-SVD factors of a
    4-bit weight's quantization error (L1: K x r, entries ~ N(0, 1/K);
    L2: r x N, entries ~ N(0, err_std^2 K / r)), as inputs of the two-factor
    comparator's preparation."""
    rng = np.random.default_rng(seed)
    L1 = (rng.standard_normal((K, r)) / np.sqrt(K)).astype(np.float32)
    L2 = (err_std * np.sqrt(K / r) * rng.standard_normal((r, N))).astype(np.float32)
    return L1, L2
