"""Dual-stream joint attention on the GPU against the fp64 oracle: the image
and text streams' projections sharded alike, one SDPA over both streams'
tokens, each stream's rows through its own out-projection.  Small ragged
streams, the degenerate cases (one stream empty; both streams sharing
weights, which must equal the attention block on the concatenation bit for
bit), the prepared handle, and the Flux-scale 4096 + 512 tokens on sampled
rows."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


def _run(dd, Mi, Mt, heads, T):
    Yi, Yt = tp.joint_attn_block(dd["X_img"][:Mi], dd["X_txt"][:Mt], dd["W_qkv_img"], dd["W_qkv_txt"],
                                 dd["W_o_img"], dd["W_o_txt"], heads, T)
    torch.cuda.synchronize()
    return from_dev(Yi), from_dev(Yt)


def _inputs(Mi, Mt, D, heads, seed):
    d = syn.joint_attn_inputs(Mi, Mt, D, seed)
    return d, {k: to_dev(v) for k, v in d.items()}


@pytest.mark.parametrize("Mi,Mt,D,heads,T", [
    (200, 77, 256, 2, 2),     # ragged both streams
    (128, 128, 512, 4, 4),
    (300, 5, 384, 3, 1),      # a handful of text tokens
    (513, 1, 256, 2, 2),      # one text token beside a ragged image stream
])
def test_joint_small(Mi, Mt, D, heads, T):
    d, dd = _inputs(Mi, Mt, D, heads, seed=Mi + Mt)
    f = {k: f64(v) for k, v in d.items()}
    gi, gt = _run(dd, Mi, Mt, heads, T)
    ri, rt = o.joint_attn_sharded_summed(f["X_img"], f["X_txt"], f["W_qkv_img"], f["W_qkv_txt"], f["W_o_img"],
                                         f["W_o_txt"], heads, T)
    both = np.concatenate([gi, gt])
    assert_parity(both, np.concatenate([ri, rt]), f"joint Mi={Mi} Mt={Mt} T={T}")
    assert_parity(gt, rt, "joint text stream")


def test_one_empty_stream_is_the_attention_block():
    Mi, Mt, D, heads, T = 200, 77, 256, 2, 2
    d, dd = _inputs(Mi, Mt, D, heads, seed=7)
    for which in ("img", "txt"):
        X, Wq, Wo = dd[f"X_{which}"], dd[f"W_qkv_{which}"], dd[f"W_o_{which}"]
        ref = from_dev(tp.attn_block(X, Wq, Wo, heads, T))
        if which == "img":
            gi, gt = _run(dd, Mi, 0, heads, T)
            assert gt.shape == (0, D) and np.array_equal(gi, ref)
        else:
            gi, gt = _run(dd, 0, Mt, heads, T)
            assert gi.shape == (0, D) and np.array_equal(gt, ref)


def test_shared_weights_equal_attention_over_the_concatenation():
    Mi, Mt, D, heads, T = 300, 130, 256, 2, 2
    d, dd = _inputs(Mi, Mt, D, heads, seed=8)
    Yi, Yt = tp.joint_attn_block(dd["X_img"], dd["X_txt"], dd["W_qkv_img"], dd["W_qkv_img"], dd["W_o_img"],
                                 dd["W_o_img"], heads, T)
    Y = tp.attn_block(torch.cat([dd["X_img"], dd["X_txt"]]), dd["W_qkv_img"], dd["W_o_img"], heads, T)
    torch.cuda.synchronize()
    # same kernels, same per-element arithmetic: identical bits
    assert np.array_equal(np.concatenate([from_dev(Yi), from_dev(Yt)]), from_dev(Y))


@pytest.fixture(scope="module")
def flux_joint():
    c = syn.CONFIGS["flux_joint_attn"]
    d = syn.joint_attn_inputs(c["M_img"], c["M_txt"], c["D"], c["seed"])
    return c, d


def test_flux_joint_sampled_rows_and_prepared(flux_joint):
    c, d = flux_joint
    Mi, Mt, D, H, T = c["M_img"], c["M_txt"], c["D"], c["H"], c["T"]
    dd = {k: to_dev(v) for k, v in d.items()}
    gi, gt = _run(dd, Mi, Mt, H, T)
    rng = np.random.default_rng(0)
    ri = np.sort(np.concatenate([[0, 127, 128, Mi - 1], rng.choice(Mi, 28, replace=False)]))
    rt = np.sort(np.concatenate([[0, Mt - 1], rng.choice(Mt, 14, replace=False)]))
    f = {k: f64(v) for k, v in d.items()}
    oi, ot = o.joint_attn_rows(f["X_img"], f["X_txt"], f["W_qkv_img"], f["W_qkv_txt"], f["W_o_img"], f["W_o_txt"],
                               H, ri, rt, tp_degree=T)
    assert_parity(np.concatenate([gi[ri], gt[rt]]), np.concatenate([oi, ot]), "flux joint attention, sampled rows")
    layer = tp.JointAttnBlock(dd["W_qkv_img"], dd["W_qkv_txt"], dd["W_o_img"], dd["W_o_txt"], H, T)
    Yi, Yt = layer(dd["X_img"], dd["X_txt"])
    torch.cuda.synchronize()
    assert np.array_equal(from_dev(Yi), gi) and np.array_equal(from_dev(Yt), gt)
    layer.close()
    assert tp.tp_check_device_error() == 0


def test_bench_step_sequence_matches_one_shot():
    # bench.py times the joint block as one call of the prepared layer (which
    # runs the two streams' projections side by side: five launches) and, for
    # the per-kernel breakdown, as its six step-level calls (one batched slice
    # launch, two row-range QKV GEMMs, one SDPA, two row-range
    # out-projections); both must give exactly the one-shot result.
    import bench
    wl = bench.JointAttnWorkload(dict(kind="joint", M_img=300, M_txt=77, D=256, H=2, T=2, seed=9))
    d = wl.host_inputs(0)
    g = {k: to_dev(v) for k, v in d.items()}
    kernels = wl.kernels(tp, g, "cuda")
    assert [k.name for k in kernels if k.composite] == ["joint_layer"]
    n0 = tp.tp_kernel_launches()
    for k in kernels:
        k.fn()
    assert tp.tp_kernel_launches() - n0 == 5 + 6
    torch.cuda.synchronize()
    gi, gt = _run(g, 300, 77, 2, 2)
    assert np.array_equal(from_dev(wl.bufs["Y_img"]), gi) and np.array_equal(from_dev(wl.bufs["Y_txt"]), gt)
    assert np.array_equal(from_dev(wl.bufs["Yj_img"]), gi) and np.array_equal(from_dev(wl.bufs["Yj_txt"]), gt)


def test_joint_layers_from_two_host_threads():
    # Two threads, each on its own stream, call the joint layer (which forks
    # onto the device's side stream) at the same time; each result must equal
    # the single-threaded one.
    import threading
    Mi, Mt, D, heads, T = 300, 77, 256, 2, 2
    runs = []
    for seed in (31, 32):
        d, dd = _inputs(Mi, Mt, D, heads, seed=seed)
        runs.append((dd, _run(dd, Mi, Mt, heads, T)))
    errors, results = [], [None, None]

    def worker(i):
        try:
            dd = runs[i][0]
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                for _ in range(3):
                    Yi, Yt = tp.joint_attn_block(dd["X_img"], dd["X_txt"], dd["W_qkv_img"], dd["W_qkv_txt"],
                                                 dd["W_o_img"], dd["W_o_txt"], heads, T, stream=st)
            st.synchronize()
            results[i] = (from_dev(Yi), from_dev(Yt))
        except Exception as e:  # noqa: BLE001 - reported below
            errors.append(e)

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=120)
    assert not errors, errors
    for i in range(2):
        assert np.array_equal(results[i][0], runs[i][1][0]) and np.array_equal(results[i][1], runs[i][1][1])
    assert tp.tp_check_device_error() == 0

