"""GPU parity: one decoder layer's seven projections captured in a CUDA graph.

The model pages decode under CUDA graphs ("Llama 3.1 8B Instruct W8A8" and
"Qwen3 8B FP8", "Against bf16").  Here a layer's projections at M = 1 are
captured once, in the order a decode step runs them -- q|k|v on one input
(one grouped launch), o, gate|up on one input (one grouped launch), down --
with static input and output buffers.  The graph is replayed on two different
sets of inputs copied into those buffers, and every output of every
projection is compared with the oracle (bit for bit for int8, within the
output tolerance for E4M3).  The same is done for the small-M path (M = 8
and M = 32, seven qlinear_forward calls, workspaces included) so that the
graph-replayed split-K sums are checked too.
"""
import numpy as np
import pytest
import torch

import fp8_linear_layers_b200 as ql
import oracle
from fp8_linear_layers_b200 import synthetic
from tests._util import assert_y_close, bits, f32_dev, oracle_forward_par, u8_dev

pytestmark = pytest.mark.gpu

INPUT_OF = {"q_proj": "qkv", "k_proj": "qkv", "v_proj": "qkv", "o_proj": "o", "gate_proj": "gate_up",
            "up_proj": "gate_up", "down_proj": "down"}


def _layer(scheme, shapes, M):
    ws = {}
    for name, N, K in shapes:
        w = synthetic.make_w(N, K, seed=0, tag=f"layer.{name}")
        ws[name] = oracle.quantize_weight(scheme, w)
    ks = {INPUT_OF[n]: K for n, _, K in shapes}
    return ws, ks


# the E4M3 row scheme at M = 1 and 8 (M = 32 runs the kernels W8A8 runs there)
@pytest.mark.parametrize("scheme,model,M", [(ql.W8A8_INT8_ROW, "llama", 1), (ql.W8A8_INT8_ROW, "llama", 8),
                                            (ql.W8A8_INT8_ROW, "llama", 32), (ql.FP8_E4M3_ROW, "llama", 1),
                                            (ql.FP8_E4M3_ROW, "llama", 8), (ql.FP8_E4M3_BLOCK128, "qwen", 1),
                                            (ql.FP8_E4M3_BLOCK128, "qwen", 8), (ql.FP8_E4M3_BLOCK128, "qwen", 32)])
def test_layer_in_one_cuda_graph(cuda, scheme, model, M):
    shapes = synthetic.LLAMA31_8B if model == "llama" else synthetic.QWEN3_8B
    ws, ks = _layer(scheme, shapes, M)
    d_w = {n: (u8_dev(wq), f32_dev(sw)) for n, (wq, sw) in ws.items()}
    d_x = {g: torch.empty((M, K), dtype=torch.bfloat16, device="cuda") for g, K in ks.items()}
    d_y = {n: torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for n, N, _ in shapes}
    d_ws = {n: ql.new_workspace(ql.forward_workspace_bytes(scheme, M, N, K)) for n, N, K in shapes}
    stream = torch.cuda.Stream()

    def layer():
        if M == 1:
            for names in (("q_proj", "k_proj", "v_proj"), ("o_proj",), ("gate_proj", "up_proj"),
                          ("down_proj",)):
                x = d_x[INPUT_OF[names[0]]]
                if len(names) > 1:
                    ql.gemv_grouped(scheme, [(x, *d_w[n], d_y[n]) for n in names], stream=stream)
                else:
                    ql.gemv(scheme, x, *d_w[names[0]], y=d_y[names[0]], stream=stream)
        else:
            for n, _, _ in shapes:
                ql.forward(scheme, d_x[INPUT_OF[n]], *d_w[n], workspace=d_ws[n], y=d_y[n], stream=stream)

    def set_inputs(seed):
        xs = {}
        for g, K in ks.items():
            oc = 0 if model == "qwen" else synthetic.outlier_count(K)
            xs[g] = synthetic.make_x(M, K, seed=seed, tag=f"layer.x.{g}", outliers=oc)
            d_x[g].copy_(torch.from_numpy(xs[g].view(np.int16)).view(torch.bfloat16))
        return xs

    set_inputs(100)
    with torch.cuda.stream(stream):
        layer()  # warm the launch path before capture
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        layer()
    for seed in (1, 2):
        xs = set_inputs(seed)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        assert ql.device_status()[0] == 0
        for n, N, K in shapes:
            ref = oracle_forward_par(scheme, xs[INPUT_OF[n]], *ws[n])
            got = bits(d_y[n])
            assert_y_close(got, ref, f"graph replay seed {seed}: {n} M={M} scheme {scheme}")
            if scheme == ql.W8A8_INT8_ROW:
                assert np.array_equal(got, ref), f"{n}: int8 outputs must match the oracle exactly"
    del graph
