"""CUDA-graph capture of the hot path.

A serving loop records a whole attention step once and replays it; every device call of the
C ABI is asynchronous on its stream (no allocation, no synchronisation), so the ring step,
the Ulysses pass through permutes and the fused Ulysses kernel (with and without its tail
split) can be captured into a CUDA graph.  Each is captured after one eager warm-up, replayed on new inputs copied into the
captured buffers, and compared bit for bit with the same calls run eagerly on those inputs.
The captured launches keep their programmatic (dependent-launch) edges.
"""

import math

import pytest
import torch

import context_long_sequence_non_b200 as cp
from context_long_sequence_non_b200 import build as build_mod
from context_long_sequence_non_b200 import workloads as W
from context_long_sequence_non_b200.paths import UlyssesPlan, ring_attention

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build_mod.build()
    cp.lib()
    yield
    assert cp.device_error() == 0


def _capture(fn):
    """Warm `fn` up on a side stream, then record it into a graph; returns (graph, outputs)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = fn()
    return graph, outs


def _refill(tensors, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    for t in tensors:
        t.copy_(W.randn(tuple(t.shape), g, sigma, "bf16"))


@pytest.mark.parametrize("n_split", [0, 1])
def test_ring_step_graph_replay(n_split):
    # 8 chunks of 600 keys against a 1100-row Q slice of 36 heads: 180 work items, so with
    # n_split = 0 each chunk's last, partial wave (32 items) runs as two key ranges
    # (attention + combine launches per chunk)
    Bn, Sq, H, D, S_c, n_c = 1, 1100, 36, 128, 600, 8
    q = torch.empty(Bn, Sq, H, D, dtype=torch.bfloat16, device=DEV)
    ks = [torch.empty(Bn, S_c, H, D, dtype=torch.bfloat16, device=DEV) for _ in range(n_c)]
    vs = [torch.empty_like(k) for k in ks]
    _refill([q, *ks, *vs], 1)
    step = lambda: ring_attention(q, ks, vs, n_split=n_split)
    graph, (o_g, l_g) = _capture(step)
    for trial in range(2):
        _refill([q, *ks, *vs], 100 + trial)
        graph.replay()
        o_e, l_e = step()
        torch.cuda.synchronize()
        assert torch.equal(o_g, o_e) and torch.equal(l_g, l_e), trial
        assert torch.isfinite(o_g.float()).all()


@pytest.mark.parametrize("mode", ["plain", "batched", "qk_norm"])
def test_ulysses_plan_graph_replay(mode):
    P, S_l, H, D = 4, 400, 8, 128
    shards = [torch.empty(P, S_l, H, D, dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    _refill(shards, 2)
    norm = None
    if mode == "qk_norm":
        norm = (W.norm_weights(D, 1).to(DEV), W.norm_weights(D, 2).to(DEV))
    plan = UlyssesPlan(P, S_l, H, D, device=DEV, batched=mode == "batched", qk_norm=norm)
    graph, _ = _capture(lambda: plan.run(*shards))  # the graph writes plan.out / plan.lse
    for trial in range(2):
        _refill(shards, 200 + trial)
        graph.replay()
        torch.cuda.synchronize()
        o_r, l_r = plan.out.clone(), plan.lse.clone()
        o_e, l_e = plan.run(*shards)
        torch.cuda.synchronize()
        assert torch.equal(o_r, o_e) and torch.equal(l_r, l_e), trial


@pytest.mark.parametrize("split", [False, True])
def test_fused_ulysses_graph_replay(split):
    # split: 4 groups x 16 heads x 7 tile pairs = 448 items, the last wave's 4 in key ranges
    P, S_l, H, D = (4, 400, 64, 128) if split else (8, 272, 16, 64)
    shards = [torch.empty(P, S_l, H, D, dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    _refill(shards, 3)
    out = torch.empty(P, S_l, H, D, dtype=torch.bfloat16, device=DEV)
    lse = torch.empty(P, H // P, P * S_l, device=DEV)
    if split:
        ws = torch.empty(cp.ulysses_workspace_bytes(P, S_l, H, D), dtype=torch.uint8, device=DEV)
        assert ws.numel() > 0
        run = lambda: cp.ulysses_fwd_split(*shards, P, out=out, lse=lse, scale=1 / math.sqrt(D),
                                           workspace=ws)
    else:
        run = lambda: cp.ulysses_fwd(*shards, P, out=out, lse=lse, scale=1 / math.sqrt(D))
    graph, _ = _capture(run)
    for trial in range(2):
        _refill(shards, 300 + trial)
        graph.replay()
        torch.cuda.synchronize()
        o_r, l_r = out.clone(), lse.clone()
        run()
        torch.cuda.synchronize()
        assert torch.equal(o_r, out) and torch.equal(l_r, lse), trial
