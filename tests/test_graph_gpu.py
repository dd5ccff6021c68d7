"""The library's call sequences are capturable in a CUDA graph (no allocation,
no host synchronisation inside a call): a captured step replays with the
eager step's output bits, on the streaming and on the grouped-GEMM paths."""
import pytest
import torch

import moe_inputs
import mixture_experts_routed_sigmoid_b200 as moe

pytestmark = pytest.mark.gpu


def _replay_equals_eager(step, out):
    step()
    torch.cuda.synchronize()
    want = out.clone()
    out.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int32), want.view(torch.int32))
    del graph


@pytest.mark.parametrize("m", [8, 300])  # 64 routed rows stream; 2400 use the grouped GEMMs
def test_ffn_step_replays_bit_identical(m):
    cfg = moe_inputs.FfnConfig("g", m, 512, 256, 32, 8, w_std=0.05)
    inp = moe_inputs.ffn_inputs(cfg, seed=m, device="cuda")
    ids = torch.empty((m, cfg.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((m, cfg.top_k), dtype=torch.float32, device="cuda")
    y = torch.empty((m, cfg.hidden), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_ffn_workspace(m, cfg.hidden, cfg.inter, cfg.top_k, cfg.n_experts),
                     dtype=torch.uint8, device="cuda")

    def step():
        moe.moe_route_topk(inp["logits"], inp["bias"], cfg.top_k, ids=ids, weights=w)
        moe.moe_ffn_forward(inp["x"], ids, w, inp["W_gate"], inp["W_up"], inp["W_down"], y=y,
                            ws=ws)

    _replay_equals_eager(step, y)


def test_matmul_id_replays_bit_identical():
    cfg = moe_inputs.DECODE
    inp = moe_inputs.matmul_id_inputs(cfg, seed=2, device="cuda")
    y = torch.empty((cfg.m, cfg.top_k, cfg.n), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.moe_matmul_id_workspace(cfg.m, cfg.n, cfg.k, cfg.top_k, cfg.n_experts),
                     dtype=torch.uint8, device="cuda")
    _replay_equals_eager(lambda: moe.moe_matmul_id(inp["x"], inp["ids"], inp["W"], y=y, ws=ws), y)
