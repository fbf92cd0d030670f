"""a8 on the GPU: Y = bf16(sum_r parts[r] + bias) against the oracle's sum."""
import numpy as np
import pytest
import torch

import oracle as o
import synthetic as syn
import tensor_transformer_layers_b200 as tp
from tests._util import assert_parity, f64, from_dev, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,T,bias", [
    (1, 8, 1, False), (3, 8, 2, True), (37, 136, 3, True), (64, 128, 8, True), (5, 64, 11, True),
    (4608, 3072, 4, True),   # Flux-scale partials
    (4608, 3072, 8, True),
])
def test_reduce_partials(M, N, T, bias):
    parts = syn.bf16_bits_to_f32(syn.normal_bf16((T, M, N), 1.0, seed=M + N, tid=200)).copy()
    # fp32 partials with full mantissas: add a small perturbation that bf16 could not hold
    parts += np.float32(1e-3) * syn.bf16_bits_to_f32(syn.normal_bf16((T, M, N), 1.0, seed=M + N, tid=201))
    b = syn.normal_bf16((N,), 0.02, seed=N, tid=202) if bias else None
    Y = torch.empty((M, N), dtype=torch.int16, device="cuda")
    Pd = torch.from_numpy(parts).cuda()
    bd = to_dev(b) if bias else None
    assert tp.tp_reduce_partials(Pd, M, N, T, bd, Y) == 0
    torch.cuda.synchronize()
    ref = o.reduce_partials([parts[r].astype(np.float64) for r in range(T)], f64(b) if bias else None)
    g = from_dev(Y)
    assert_parity(g, ref, "reduce")
    # the only roundings are the fp32 adds and one final bf16 rounding
    err = np.abs(f64(g) - ref)
    assert np.all(err <= np.abs(ref) * 2.0 ** -8 + 1e-5 * T)
