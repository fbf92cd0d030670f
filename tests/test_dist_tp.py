"""Tensor parallelism across processes, host side: two gloo ranks on CPU.

Each rank holds only its own shards (colwise W_up,r / b_up,r, rowwise
W_down,r; for attention its heads of W_qkv and its rowwise W_o,r), computes
its partial sum with the oracle (the per-rank compute is supplied by the
test; the GPU computes it with tp_*_rank_partial), and
``tensor_transformer_layers_b200.dist.allreduce_layer`` runs the one
AllReduce(sum) at the block boundary and the finish step, which adds the
rowwise bias once.  Every rank must end with the unsharded layer's output
("Tensor parallelism" page: the colwise -> rowwise pair needs a single
AllReduce; the validation method compares the sharded output with the
single-device one)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

WORLD = 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _inputs(seed):
    rng = np.random.default_rng(seed)
    M, D, F, heads = 6, 256, 64, 2
    return dict(
        X=rng.standard_normal((M, D)),
        W_up=rng.standard_normal((F, D)) / 16, b_up=rng.standard_normal(F) * 0.1,
        W_down=rng.standard_normal((D, F)) / 8, b_down=rng.standard_normal(D) * 0.1,
        W_qkv=rng.standard_normal((3 * D, D)) / 16, W_o=rng.standard_normal((D, D)) / 16, heads=heads)


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    import datetime

    import torch.distributed as dist

    import oracle as o
    from tensor_transformer_layers_b200.dist import allreduce_layer
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        d = _inputs(5)
        T = WORLD
        seen = []

        def mlp_partial():  # this rank's shards only; no rowwise bias
            H = o.mlp_colwise_shard(d["X"], d["W_up"], d["b_up"], T, rank)
            p = torch.from_numpy(o.mlp_rowwise_partial(H, d["W_down"], T, rank))
            seen.append(p.clone())
            return p

        Y = allreduce_layer(mlp_partial, lambda s: s + torch.from_numpy(d["b_down"])[None, :])

        def attn_partial():
            O_r = o.attn_shard_output(d["X"], d["W_qkv"], d["heads"], T, rank)
            return torch.from_numpy(o.linear(O_r, o.slice_rowwise(d["W_o"], T, rank)))

        A = allreduce_layer(attn_partial, lambda s: s)
        np.save(os.path.join(out_dir, f"mlp{rank}.npy"), Y.numpy())
        np.save(os.path.join(out_dir, f"part{rank}.npy"), seen[0].numpy())
        np.save(os.path.join(out_dir, f"attn{rank}.npy"), A.numpy())
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("tp_ranks")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(out))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return out


def test_every_rank_gets_the_unsharded_mlp(ranks):
    import oracle as o
    d = _inputs(5)
    want = o.mlp_unsharded(d["X"], d["W_up"], d["b_up"], d["W_down"], d["b_down"])
    for r in range(WORLD):
        got = np.load(ranks / f"mlp{r}.npy")
        assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def test_ranks_hold_different_shards_and_the_bias_is_added_once(ranks):
    import oracle as o
    d = _inputs(5)
    parts = [np.load(ranks / f"part{r}.npy") for r in range(WORLD)]
    assert not np.allclose(parts[0], parts[1])  # partial sums of different shards, not replicas
    Y = np.load(ranks / "mlp0.npy")
    assert np.allclose(Y, parts[0] + parts[1] + d["b_down"][None, :], rtol=0, atol=1e-12)
    # a bias added by every rank before the sum would be off by (T - 1) * b_down
    full_no_bias = o.mlp_unsharded(d["X"], d["W_up"], d["b_up"], d["W_down"], None)
    assert np.allclose(Y - full_no_bias, np.tile(d["b_down"], (Y.shape[0], 1)), atol=1e-12)


def test_every_rank_gets_the_unsharded_attention(ranks):
    import oracle as o
    d = _inputs(5)
    want = o.attn_unsharded(d["X"], d["W_qkv"], d["W_o"], d["heads"])
    for r in range(WORLD):
        got = np.load(ranks / f"attn{r}.npy")
        assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def test_single_process_needs_no_collective():
    from tensor_transformer_layers_b200.dist import allreduce_layer
    t = torch.arange(4.0)
    assert torch.equal(allreduce_layer(lambda: t.clone(), lambda s: s * 2), t * 2)


# ---------------------------------------------------------------------------
# Context parallelism across processes: Ulysses all-to-all regrouping and the
# Ring rotation of key/value blocks, two gloo ranks, oracle compute.
# ---------------------------------------------------------------------------

def _cp_inputs():
    rng = np.random.default_rng(11)
    M, H, d = 8, 4, 16
    return rng.standard_normal((M, 3 * H * d)), H, d


def _attend(qkv, n_heads, d):
    import oracle as o
    c = n_heads * d
    return np.concatenate([o.sdpa(qkv[:, h * d:(h + 1) * d], qkv[:, c + h * d:c + (h + 1) * d],
                                  qkv[:, 2 * c + h * d:2 * c + (h + 1) * d]) for h in range(n_heads)], axis=1)


def _cp_rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(WORLD))
    import datetime

    import torch.distributed as dist

    import oracle as o
    from tensor_transformer_layers_b200.dist import ring_attention, ulysses_attention
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=60))
    try:
        QKV, H, d = _cp_inputs()
        U, M = WORLD, QKV.shape[0]
        Ms = M // U
        local = torch.from_numpy(QKV[rank * Ms:(rank + 1) * Ms].copy())

        def pack(x):  # by destination head group: packed rowwise, blocks [1, 1, 1]
            return torch.from_numpy(np.stack([o.slice_packed_rowwise(x.numpy(), [1, 1, 1], U, u) for u in range(U)]))

        def attend(recv):  # [U, Ms, ...] = all tokens, this rank's heads
            return torch.from_numpy(_attend(recv.reshape(M, -1).numpy(), H // U, d).reshape(U, Ms, -1))

        def unpack(back):  # [U, Ms, (H/U) d] -> [Ms, H d]
            return torch.cat([back[u] for u in range(U)], dim=1)

        Yu = ulysses_attention(local, pack, attend, unpack)

        def attend_block(q_rows, kv_rows):  # per head: normalised O and natural log-sum-exp
            q, kv = q_rows.numpy(), kv_rows.numpy()
            c = H * d
            res = [o.sdpa(q[:, h * d:(h + 1) * d], kv[:, c + h * d:c + (h + 1) * d],
                          kv[:, 2 * c + h * d:2 * c + (h + 1) * d], return_lse=True) for h in range(H)]
            return [r[0] for r in res], [r[1] for r in res]

        def merge(parts):
            outs = []
            for h in range(H):
                Oh, _ = o.attn_merge(np.stack([p[0][h] for p in parts]), np.stack([p[1][h] for p in parts]))
                outs.append(Oh)
            return np.concatenate(outs, axis=1)

        Yr = ring_attention(local, local, attend_block, merge)
        np.save(os.path.join(out_dir, f"ulysses{rank}.npy"), Yu.numpy())
        np.save(os.path.join(out_dir, f"ring{rank}.npy"), Yr)
    finally:
        dist.destroy_process_group()


@pytest.fixture(scope="module")
def cp_ranks(tmp_path_factory):
    out = tmp_path_factory.mktemp("cp_ranks")
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_cp_rank_main, args=(r, port, str(out))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return out


def test_ulysses_ranks_get_their_tokens_of_the_full_attention(cp_ranks):
    QKV, H, d = _cp_inputs()
    full = _attend(QKV, H, d)
    Ms = QKV.shape[0] // WORLD
    for r in range(WORLD):
        assert np.array_equal(np.load(cp_ranks / f"ulysses{r}.npy"), full[r * Ms:(r + 1) * Ms])


def test_ring_ranks_get_their_tokens_of_the_full_attention(cp_ranks):
    QKV, H, d = _cp_inputs()
    full = _attend(QKV, H, d)
    Ms = QKV.shape[0] // WORLD
    for r in range(WORLD):
        got = np.load(cp_ranks / f"ring{r}.npy")
        assert np.max(np.abs(got - full[r * Ms:(r + 1) * Ms])) <= 1e-12
