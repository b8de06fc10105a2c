"""Seeded synthetic inputs for the multi-LoRA shrink / expand path.

This module draws numbers and lays them out; it holds none of the method's
arithmetic.  The CUDA path, the oracle, the tests and the benchmark all take
their inputs from here, so both sides of every comparison see the same bits.

Recipe (numpy Generator(PCG64(seed))): values are drawn in float64 in the fixed
order idx -> x -> A_i -> B_i -> y, cast to float32 and rounded to fp16 / bf16
(round-to-nearest-even, by torch on the CPU).  fp16/bf16 arrays are handed out
as numpy uint16 bit patterns; indices are int32.

  x, y       ~ N(0, 1)
  A_i, B_i   ~ N(0, 0.02)   (0.02 read as the standard deviation)

The five workloads are shaped like the layers the pages serve (Llama-class
q_proj / qkv / gate_up / down projections, decode and prefill batches); no
model weights or datasets are involved.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

F16, BF16 = 0, 1
DTYPE_NAME = {F16: "f16", BF16: "bf16"}
TORCH_DTYPE = {F16: torch.float16, BF16: torch.bfloat16}


@dataclass
class Problem:
    """One LoRA-wrapped projection applied to one batch.

    A: list of [S, r, D] stacks (one per slice, or a single shared one),
    B: list of [S, D_out_i, r] stacks, y: [T, sum(D_out)] with slice i's
    columns starting at col_off[i].  Exactly one of idx (per-token, BGMV)
    or seg_starts / seg_adapter (segments, SGMV) describes the adapters.
    """
    name: str
    dtype: int
    T: int
    D: int
    r: int
    S: int
    d_out: List[int]
    scale: float
    x: np.ndarray
    A: List[np.ndarray]
    B: List[np.ndarray]
    y: np.ndarray
    idx: Optional[np.ndarray] = None
    seg_starts: Optional[np.ndarray] = None
    seg_adapter: Optional[np.ndarray] = None
    shared_A: bool = False
    col_off: List[int] = field(default_factory=list)

    @property
    def n_slices(self) -> int:
        return len(self.B)

    @property
    def segmented(self) -> bool:
        return self.seg_starts is not None


def _round_bits(vals: np.ndarray, dtype: int) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(vals, dtype=np.float32))
    return t.to(TORCH_DTYPE[dtype]).view(torch.int16).numpy().view(np.uint16)


def draw_idx(rng, T, S, kind, frac_neg=0.0, zipf_s=1.1):
    """Per-token adapter indices (-1 = base model only)."""
    if kind == "uniform":            # every token has an adapter, uniform over slots
        idx = rng.integers(0, S, size=T)
    elif kind == "uniform_neg":      # uniform over {-1, 0, .., S-1}
        idx = rng.integers(-1, S, size=T)
    elif kind == "frac_neg":         # exactly round(frac*T) tokens -1, rest uniform
        idx = rng.integers(0, S, size=T)
        n_neg = int(round(frac_neg * T))
        idx[rng.choice(T, size=n_neg, replace=False)] = -1
    elif kind == "zipf":             # slot k has weight (k+1)^-s; then frac_neg of -1
        w = (np.arange(S, dtype=np.float64) + 1.0) ** (-zipf_s)
        idx = rng.choice(S, size=T, p=w / w.sum())
        n_neg = int(round(frac_neg * T))
        idx[rng.choice(T, size=n_neg, replace=False)] = -1
    elif kind == "none":             # no token has an adapter
        idx = np.full(T, -1)
    elif kind == "single":           # every token on slot 0
        idx = np.zeros(T)
    else:
        raise ValueError(kind)
    return np.ascontiguousarray(idx, dtype=np.int32)


def draw_values(rng, shape, kind, std):
    if kind == "normal":
        return rng.normal(0.0, std, size=shape)
    if kind == "int":                # {-1, 0, 1}: products and sums stay integers
        return rng.integers(-1, 2, size=shape).astype(np.float64)
    raise ValueError(kind)


def make_problem(name, dtype, T, D, r, S, d_out, scale=1.0, seed=0,
                 idx_kind="uniform", frac_neg=0.0, segments=None,
                 shared_A=False, values="normal", y_kind=None) -> Problem:
    """Draw one problem.  segments = (seg_starts, seg_adapter) switches to the
    segment form; values="int" gives x, A, B in {-1,0,1} and y in [-8, 8]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if segments is None:
        idx = draw_idx(rng, T, S, idx_kind, frac_neg)
        ss = sa = None
    else:
        idx = None
        ss = np.ascontiguousarray(segments[0], dtype=np.int32)
        sa = np.ascontiguousarray(segments[1], dtype=np.int32)
    n_a = 1 if shared_A else len(d_out)
    x = _round_bits(draw_values(rng, (T, D), values, 1.0), dtype)
    A = [_round_bits(draw_values(rng, (S, r, D), values, 0.02), dtype) for _ in range(n_a)]
    B = [_round_bits(draw_values(rng, (S, o, r), values, 0.02), dtype) for o in d_out]
    ncol = int(sum(d_out))
    yk = y_kind or ("int8" if values == "int" else "normal")
    if yk == "int8":
        yv = rng.integers(-8, 9, size=(T, ncol)).astype(np.float64)
    else:
        yv = rng.normal(0.0, 1.0, size=(T, ncol))
    y = _round_bits(yv, dtype)
    col_off = list(np.concatenate([[0], np.cumsum(d_out)[:-1]]).astype(int))
    return Problem(name=name, dtype=dtype, T=T, D=D, r=r, S=S, d_out=list(d_out),
                   scale=scale, x=x, A=A, B=B, y=y, idx=idx, seg_starts=ss,
                   seg_adapter=sa, shared_A=shared_A, col_off=col_off)


def prefill_segments(rng_seed, n_seq, seq_len, S):
    """n_seq contiguous sequences of seq_len tokens, each on its own slot
    drawn as a random permutation of the slots."""
    rng = np.random.Generator(np.random.PCG64(rng_seed))
    starts = np.arange(n_seq + 1, dtype=np.int32) * seq_len
    adapters = rng.permutation(S)[:n_seq].astype(np.int32)
    return starts, adapters


# The five workloads.  Each entry returns the list of projections that make
# one step of that workload.  `dtype` draws the same workload in another
# element type (same seeds and shapes).
def config(n: int, dtype: Optional[int] = None) -> List[Problem]:
    def dt(default):
        return default if dtype is None else dtype
    if n == 1:   # tiny BGMV
        return [make_problem("tiny_bgmv", dt(F16), T=32, D=1024, r=8, S=4, d_out=[1024],
                             scale=1.0, seed=1, idx_kind="uniform_neg")]
    if n == 2:   # decode at a Llama-3-8B q_proj shape
        return [make_problem("decode_q_proj", dt(F16), T=256, D=4096, r=16, S=32,
                             d_out=[4096], scale=2.0, seed=2, idx_kind="uniform")]
    if n == 3:   # fused-slice decode: qkv, gate_up, down
        return [
            make_problem("decode_qkv", dt(BF16), T=512, D=4096, r=64, S=8,
                         d_out=[4096, 1024, 1024], seed=3, idx_kind="frac_neg",
                         frac_neg=0.25),
            make_problem("decode_gate_up", dt(BF16), T=512, D=4096, r=64, S=8,
                         d_out=[14336, 14336], seed=3, idx_kind="frac_neg",
                         frac_neg=0.25),
            make_problem("decode_down", dt(BF16), T=512, D=14336, r=64, S=8,
                         d_out=[4096], seed=3, idx_kind="frac_neg", frac_neg=0.25),
        ]
    if n == 4:   # prefill, 8 sequences x 1024 tokens, one slot each
        seg = prefill_segments(4, 8, 1024, 8)
        return [make_problem("prefill_sgmv", dt(BF16), T=8192, D=4096, r=64, S=8,
                             d_out=[4096], seed=4, segments=seg)]
    if n == 5:   # large mixed batch, Zipf(1.1) popularity, 10% base-only, unsorted
        return [make_problem("large_mixed", dt(BF16), T=4096, D=8192, r=32, S=128,
                             d_out=[8192], seed=5, idx_kind="zipf", frac_neg=0.10)]
    raise ValueError(n)


CONFIG_NAMES = {1: "tiny_bgmv", 2: "decode_q_proj", 3: "fused_decode",
                4: "prefill_sgmv", 5: "large_mixed"}
