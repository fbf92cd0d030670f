"""a1 on the GPU: shard slices must be bit-exact copies of the oracle's slices."""
import numpy as np
import pytest
import torch

import oracle as o
import tensor_transformer_layers_b200 as tp
from tests._util import from_dev, to_dev

pytestmark = pytest.mark.gpu


def _bits(shape, seed):
    return np.random.default_rng(seed).integers(0, 1 << 16, size=shape, dtype=np.uint16)


@pytest.mark.parametrize("rows,cols,T", [
    (8, 8, 1), (16, 64, 2), (24, 48, 3), (40, 8, 5),
    (12288, 3072, 4),    # Flux-scale FFN-in weight
    (24576, 6144, 8),    # wide block FFN-in weight
])
def test_colwise_bit_exact(rows, cols, T):
    W = _bits((rows, cols), rows + cols)
    Wd = to_dev(W)
    out = torch.empty((rows // T, cols), dtype=torch.int16, device="cuda")
    for r in range(T):
        out.fill_(0x5A5A)
        assert tp.tp_shard_weight(Wd, rows, cols, tp.TP_COLWISE, T, r, out) == 0
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out), o.slice_colwise(W, T, r))


@pytest.mark.parametrize("rows,cols,T", [
    (8, 8, 1), (16, 64, 2), (24, 48, 3), (5, 80, 5), (3, 64, 8),
    (3072, 12288, 4),    # Flux-scale FFN-out weight
    (3072, 3072, 4),     # Flux attention out-projection
    (6144, 24576, 8),    # wide block FFN-out weight
    (6144, 6144, 8),     # wide block out-projection
])
def test_rowwise_bit_exact(rows, cols, T):
    W = _bits((rows, cols), rows * 7 + cols)
    Wd = to_dev(W)
    out = torch.empty((rows, cols // T), dtype=torch.int16, device="cuda")
    for r in range(T):
        out.fill_(0x5A5A)
        assert tp.tp_shard_weight(Wd, rows, cols, tp.TP_ROWWISE, T, r, out) == 0
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out), o.slice_rowwise(W, T, r))


@pytest.mark.parametrize("heads,T", [(2, 2), (4, 1), (24, 4), (48, 8)])
def test_qkv_heads_bit_exact(heads, T):
    D = heads * 128
    W = _bits((3 * D, D), heads + T)
    Wd = to_dev(W)
    out = torch.empty((3 * D // T, D), dtype=torch.int16, device="cuda")
    for r in range(T):
        out.fill_(0x5A5A)
        assert tp.tp_shard_qkv_heads(Wd, D, heads, T, r, out) == 0
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out), o.slice_qkv_heads(W, heads, T, r))


@pytest.mark.parametrize("heads,T", [(2, 2), (4, 1), (24, 4), (48, 8)])
def test_qkv_heads_all_bit_exact(heads, T):
    D = heads * 128
    W = _bits((3 * D, D), heads * 3 + T)
    out = torch.full((T, 3 * D // T, D), 0x5A5A, dtype=torch.int16, device="cuda")
    assert tp.tp_shard_qkv_heads_all(to_dev(W), D, heads, T, out) == 0
    torch.cuda.synchronize()
    h = from_dev(out)
    for r in range(T):
        assert np.array_equal(h[r], o.slice_qkv_heads(W, heads, T, r))


@pytest.mark.parametrize("n,T", [(16, 2), (12288, 4), (24576, 8)])
def test_bias_bit_exact(n, T):
    b = _bits((n,), n)
    bd = to_dev(b)
    out = torch.empty((n // T,), dtype=torch.int16, device="cuda")
    for r in range(T):
        assert tp.tp_shard_bias(bd, n, T, r, out) == 0
        torch.cuda.synchronize()
        assert np.array_equal(from_dev(out), o.slice_colwise(b, T, r))


def test_slice_leaves_neighbours_untouched():
    # A shard written into the middle of a larger buffer must not spill over.
    W = _bits((64, 96), 1)
    Wd = to_dev(W)
    buf = torch.full((3, 64 * 48), 0x1234, dtype=torch.int16, device="cuda")
    assert tp.tp_shard_weight(Wd, 64, 96, tp.TP_ROWWISE, 2, 1, buf[1]) == 0
    torch.cuda.synchronize()
    h = from_dev(buf)
    assert np.all(h[0] == 0x1234) and np.all(h[2] == 0x1234)
    assert np.array_equal(h[1].reshape(64, 48), o.slice_rowwise(W, 2, 1))
