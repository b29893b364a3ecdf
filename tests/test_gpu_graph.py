"""The layer's calls are asynchronous, allocate nothing and never
synchronize, so a whole training step can be captured in a CUDA graph: the
replayed graph must give bit-for-bit the results of the same calls run
eagerly on an identical copy of the state."""
from __future__ import annotations

import pytest
import torch

import workloads
import int8_quantized_act_b200 as ql
from parity_util import dev, new_status, status_word

pytestmark = pytest.mark.gpu


class State:
    def __init__(self, d, B):
        self.M, self.K = d["x_bf16"].shape
        self.N = d["w"].shape[0]
        M, K, N = self.M, self.K, self.N
        self.B = B
        self.x, self.dy = dev(d["x_bf16"]), dev(d["dy_bf16"])
        self.bias = dev(d["bias"])
        self.st = new_status()
        self.wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
        self.sw = torch.empty(N, device="cuda")
        ql.qlinear_quantize_rows(dev(d["w"]), self.wq, self.sw, self.st, hadamard_block=B,
                                 flags=ql.QL_REJECT_ZERO_ROWS)
        self.m = torch.zeros((N, K), device="cuda")
        self.v = torch.zeros((N, K), device="cuda")
        self.y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        self.xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
        self.sx = torch.empty(M, device="cuda")
        self.dx = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
        self.dw = torch.empty((N, K), device="cuda")
        self.db = torch.empty(N, device="cuda")
        self.ws = torch.empty(ql.qlinear_bwd_workspace_bytes(M, N, K, B), dtype=torch.uint8,
                              device="cuda")

    def step(self, t):
        ql.qlinear_fwd(self.x, self.wq, self.sw, self.bias, self.B, self.y, self.xq, self.sx,
                       self.st)
        ql.qlinear_bwd(self.dy, self.wq, self.sw, self.xq, self.sx, self.B, self.dx, self.dw,
                       self.db, self.ws, self.st)
        ql.qweight_update_sr(self.wq, self.sw, self.dw, ql.Optim(), self.m, self.v, 77, t,
                             self.st)

    def outputs(self):
        return [self.y, self.xq, self.sx, self.dx, self.dw, self.db, self.wq, self.sw, self.m,
                self.v]


@pytest.mark.parametrize("M", [17, 600])
def test_train_step_replays_bit_exactly_from_a_cuda_graph(M):
    d = workloads.rotated_layer(M=M, seed=4)
    eager, graphed = State(d, 128), State(d, 128)
    # warm-up outside the capture (one-time kernel attribute setup)
    eager.step(1)
    graphed.step(1)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.step(2)
    g.replay()
    eager.step(2)
    assert status_word(eager.st) == 0 and status_word(graphed.st) == 0
    for a, b in zip(eager.outputs(), graphed.outputs()):
        assert torch.equal(a, b)
