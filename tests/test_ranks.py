"""GPU parity with per-slot ranks ("Add multi-LoRA support", Features list:
LoRAs of different ranks in one batch).  The stacks keep the call's rank r;
a slot of rank k < r has zero rows of A and zero columns of B past k.  With
the ranks recorded in the workspace (lora_set_slot_ranks) every path must
give the oracle's result on the zero-padded stacks, write buf columns past
a slot's rank as exact zeros, and never read the padding: it is filled with
NaN here (past k in A; in B past the tensor-core tile width, k rounded up to
16, 32 or 64), and the results must not change."""
import dataclasses

import numpy as np
import pytest
import torch

from gather_matmul_b200 import ops
from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from gpu_util import Dev, assert_buf_close, assert_y_close, oracle_expand, oracle_shrink


def _ranked(p, ranks, poison):
    """p with each slot's padding zeroed (the oracle's stacks) and a copy whose
    padding is NaN (the GPU's stacks when poison is set)."""
    nan = np.uint16(0x7FC0 if p.dtype == W.BF16 else 0x7E00)
    A0 = [a.copy() for a in p.A]
    B0 = [b.copy() for b in p.B]
    A1 = [a.copy() for a in p.A]
    B1 = [b.copy() for b in p.B]
    for g, k in enumerate(ranks):
        k16 = 16 if k <= 16 else (32 if k <= 32 else 64)     # tensor-core B tile width
        for a0, a1 in zip(A0, A1):
            a0[g, k:] = 0
            a1[g, k:] = nan if poison else 0
        for b0, b1 in zip(B0, B1):
            b0[g, :, k:] = 0
            b1[g, :, k:k16] = 0
            b1[g, :, k16:] = nan if poison else 0
    return dataclasses.replace(p, A=A0, B=B0), dataclasses.replace(p, A=A1, B=B1)


PATHS = [
    # name, T, S, r, segments
    ("cuda-core-items", 60, 8, 64, None),
    ("tensor-core-grouped", 400, 8, 64, None),
    ("tensor-core-grouped-r32", 300, 6, 32, None),
    ("segments", None, 8, 64, (np.array([0, 100, 101, 230, 300, 460]), np.array([0, 3, -1, 5, 2]))),
]
RANKS = {8: [8, 16, 32, 64, 8, 16, 40, 64], 6: [8, 16, 32, 24, 8, 32]}


@pytest.mark.parametrize("poison", [False, True], ids=["zero-padding", "nan-padding"])
@pytest.mark.parametrize("name,T,S,r,seg", PATHS, ids=[c[0] for c in PATHS])
def test_mixed_ranks(name, T, S, r, seg, poison):
    ranks = RANKS[S]
    T = T if seg is None else int(seg[0][-1])
    p = W.make_problem("ranks", W.BF16, T=T, D=2056, r=r, S=S, d_out=[1024, 264], scale=0.75,
                       seed=T + S + r, idx_kind="uniform_neg", segments=seg)
    ref, gpu = _ranked(p, ranks, poison)
    d = Dev(gpu)
    ops.set_slot_ranks(torch.tensor(ranks, dtype=torch.int32, device="cuda"), S, d.meta)
    buf_ref, cabs = oracle_shrink(ref)
    buf = d.shrink()
    y = d.expand()
    torch.cuda.synchronize()
    assert_buf_close(buf, buf_ref, cabs)
    # columns past each token's slot rank (rounded up to 8) are exact zeros
    idx = ref.idx if not ref.segmented else np.repeat(seg[1], np.diff(seg[0]))
    g = buf.detach().cpu().numpy()
    for t in range(T):
        if 0 <= idx[t] < S:
            k8 = -(-ranks[idx[t]] // 8) * 8
            assert np.all(g[:, t, k8:] == 0)
    assert_y_close(ref, y, oracle_expand(ref, buf_ref))


def test_clearing_ranks_restores_full_rank():
    p = W.make_problem("clear", W.BF16, T=300, D=1024, r=32, S=4, d_out=[512], seed=5,
                       idx_kind="uniform")
    d = Dev(p)
    ops.set_slot_ranks(torch.tensor([8, 8, 8, 8], dtype=torch.int32, device="cuda"), p.S, d.meta)
    ops.set_slot_ranks(None, p.S, d.meta)
    buf_ref, cabs = oracle_shrink(p)
    assert_buf_close(d.shrink(), buf_ref, cabs)
