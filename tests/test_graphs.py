"""Graph specialisation on has_lora (gather_matmul_b200.graphs.LoraGraphSet),
after "[LoRA] LoRA cuda graph specialization", Implementation list: a step is
captured twice, with and without its LoRA calls, and a batch without any
active adapter replays the graph without them.

Checked on a small decoder-projection stand-in (a base matmul followed by the
LoRA update of its output): the graph without LoRA records none of this
library's kernels (by the library's launch counter and by the kernel nodes of
the captured graph), the graph with LoRA does, each replay reproduces the
eager step bit for bit, and the dispatch picks the graph from the batch's
host indices."""
import numpy as np
import pytest
import torch

from gather_matmul_b200 import ops
from gather_matmul_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _stand_in(idx_kind, seed=70):
    p = W.make_problem("graph", W.BF16, T=64, D=1024, r=16, S=4, d_out=[512, 256], scale=0.5,
                       seed=seed, idx_kind=idx_kind)
    td = torch.bfloat16
    mk = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(td).cuda()
    g = torch.Generator(device="cuda").manual_seed(seed)
    d = dict(
        x=mk(p.x), A=[mk(a) for a in p.A], B=[mk(b) for b in p.B],
        W=torch.randn(sum(p.d_out), p.D, generator=g, device="cuda").to(td) * 0.02,
        y=torch.empty(p.T, sum(p.d_out), dtype=td, device="cuda"),
        idx=torch.from_numpy(p.idx).cuda(),
        buf=torch.empty(len(p.A), p.T, p.r, dtype=torch.float32, device="cuda"),
        meta=ops.workspace(p.T, p.S))
    return p, d


def _step(p, d):
    def step(has_lora):
        torch.matmul(d["x"], d["W"].t(), out=d["y"])          # the base projection
        if has_lora:
            ops.bgmv(d["x"], d["A"], d["B"], d["idx"], d["y"], d["buf"], d["meta"], p.scale,
                     y_col_off=p.col_off)
    return step


def _graph_kernel_names(g):
    """Names of the kernel nodes of a captured (kept) graph."""
    from cuda.bindings import driver as cu
    graph = cu.CUgraph(g.raw_cuda_graph())
    err, _, n = cu.cuGraphGetNodes(graph, 0)
    assert err == cu.CUresult.CUDA_SUCCESS
    err, nodes, n = cu.cuGraphGetNodes(graph, n)
    assert err == cu.CUresult.CUDA_SUCCESS
    names = []
    for node in nodes[:n]:
        err, t = cu.cuGraphNodeGetType(node)
        if t != cu.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
            continue
        err, params = cu.cuGraphKernelNodeGetParams(node)
        assert err == cu.CUresult.CUDA_SUCCESS
        err, name = cu.cuFuncGetName(params.func)
        assert err == cu.CUresult.CUDA_SUCCESS
        names.append(name.decode() if isinstance(name, bytes) else str(name))
    return names


def test_graph_without_lora_records_no_library_kernel():
    from gather_matmul_b200.graphs import LoraGraphSet
    p, d = _stand_in("uniform_neg")
    gs = LoraGraphSet(_step(p, d)).capture()
    assert gs.lora_launches[False] == 0
    assert gs.lora_launches[True] >= 1


def test_graph_nodes_hold_library_kernels_only_with_lora():
    from gather_matmul_b200.graphs import LoraGraphSet
    p, d = _stand_in("uniform_neg")
    gs = LoraGraphSet(_step(p, d)).capture(keep_graph=True)
    without = _graph_kernel_names(gs.graphs[False])
    with_lora = _graph_kernel_names(gs.graphs[True])
    lib = lambda names: [n for n in names if "lora" in n]
    assert len(without) >= 1 and lib(without) == []          # the base matmul only
    assert len(lib(with_lora)) == gs.lora_launches[True]


def test_replays_match_eager_and_dispatch_follows_the_indices():
    from gather_matmul_b200.graphs import LoraGraphSet
    p, d = _stand_in("uniform_neg")
    step = _step(p, d)
    step(True)
    torch.cuda.synchronize()
    y_lora = d["y"].clone()
    step(False)
    torch.cuda.synchronize()
    y_base = d["y"].clone()
    assert not torch.equal(y_lora, y_base)
    gs = LoraGraphSet(step).capture()
    d["y"].fill_(7)
    assert gs.replay_for(p.idx, p.S) is True
    torch.cuda.synchronize()
    assert torch.equal(d["y"], y_lora)
    # an idle batch (every index -1, or outside [0, S)): the graph without LoRA
    idle = np.full(p.T, -1, dtype=np.int32)
    idle[3] = p.S
    d["idx"].copy_(torch.from_numpy(idle))
    d["y"].fill_(7)
    assert gs.replay_for(idle, p.S) is False
    torch.cuda.synchronize()
    assert torch.equal(d["y"], y_base)
