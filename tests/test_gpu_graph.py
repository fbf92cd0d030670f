"""The layer calls inside CUDA graphs: a prepared MLP pair, a prepared
attention block and a one-shot SwiGLU pair are captured once and replayed;
each replay must equal the eager call bit for bit, and must follow new
contents of the captured input buffer."""
import numpy as np
import pytest
import torch

import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import from_dev, to_dev

pytestmark = pytest.mark.gpu


def _capture(fn):
    """Warms fn up on a side stream, then captures it; returns the graph."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_prepared_mlp_and_attention_replay_in_graphs():
    M, D, F, H, T = 384, 256, 1024, 2, 2
    d = {k: to_dev(v) for k, v in syn.mlp_inputs(M, D, F, seed=21).items()}
    a = {k: to_dev(v) for k, v in syn.attn_inputs(M, D, seed=22).items()}
    X2 = to_dev(syn.normal_bf16((M, D), 1.0, seed=23, tid=0))
    mlp = tp.MlpPair(d["W_up"], d["b_up"], d["W_down"], d["b_down"], T)
    att = tp.AttnBlock(a["W_qkv"], a["W_o"], H, T)
    X = d["X"].clone()
    Ym = torch.empty((M, D), dtype=torch.int16, device="cuda")
    Ya = torch.empty((M, D), dtype=torch.int16, device="cuda")
    mlp.workspace(M, X.device)  # workspaces exist before capture
    att.workspace(M, X.device)
    g = _capture(lambda: (mlp(X, Ym), att(X, Ya)))
    for xin in (d["X"], X2):
        X.copy_(xin)
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(Ym), from_dev(mlp(xin)))
        assert np.array_equal(from_dev(Ya), from_dev(att(xin)))
    del g
    mlp.close()
    att.close()
    assert tp.tp_check_device_error() == 0


def test_one_shot_swiglu_replays_in_a_graph():
    M, D, F, T = 300, 256, 512, 2
    s = {k: to_dev(v) for k, v in syn.swiglu_inputs(M, D, F, seed=24).items()}
    Y = torch.empty((M, D), dtype=torch.int16, device="cuda")
    nb = tp.tp_swiglu_workspace_bytes(M, D, F, T)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")

    def call():
        tp._check(tp.tp_swiglu_mlp_pair(s["X"], M, D, F, s["W_in"], s["b_in"], s["W_out"], s["b_out"], T, Y, ws, nb),
                  "tp_swiglu_mlp_pair")
    g = _capture(call)
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    eager = tp.swiglu_mlp_pair(s["X"], s["W_in"], s["b_in"], s["W_out"], s["b_out"], T)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(Y), from_dev(eager))


def test_prepared_joint_attention_replays_in_a_graph():
    # The joint layer forks its text-stream projections onto a side stream and
    # joins them back; inside a capture that becomes two branches of the graph.
    Mi, Mt, D, H, T = 300, 77, 256, 2, 2
    d = {k: to_dev(v) for k, v in syn.joint_attn_inputs(Mi, Mt, D, seed=25).items()}
    layer = tp.JointAttnBlock(d["W_qkv_img"], d["W_qkv_txt"], d["W_o_img"], d["W_o_txt"], H, T)
    Xi, Xt = d["X_img"].clone(), d["X_txt"].clone()
    Yi = torch.empty((Mi, D), dtype=torch.int16, device="cuda")
    Yt = torch.empty((Mt, D), dtype=torch.int16, device="cuda")
    nb = tp.tp_joint_attn_run_workspace_bytes(Mi, Mt, D, H, T)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")

    def run():
        stream = torch.cuda.current_stream().cuda_stream
        assert tp.tp_joint_attn_run(layer.handle, Xi, Mi, Xt, Mt, Yi, Yt, ws, nb, stream) == 0

    g = _capture(run)
    for seed in (26, 27):
        Xi.copy_(to_dev(syn.normal_bf16((Mi, D), 1.0, seed=seed, tid=0)))
        Xt.copy_(to_dev(syn.normal_bf16((Mt, D), 1.0, seed=seed, tid=1)))
        g.replay()
        torch.cuda.synchronize()
        ei, et = layer(Xi, Xt)
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(Yi), from_dev(ei)) and np.array_equal(from_dev(Yt), from_dev(et))
    del g
    layer.close()
    assert tp.tp_check_device_error() == 0
