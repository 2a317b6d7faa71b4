"""The standalone split-KV decode attention op against the oracle.

Covers the long-context case (32768 keys, the 32K-prefill workload's
attention per KV head) that is too slow to reach through a whole-model oracle
run, ragged splits (more splits than keys, splits that do not divide the key
count), and reuse of one workspace across calls.
"""
import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import binding

pytestmark = pytest.mark.gpu

ATOL, RTOL = 3e-5, 1e-4


def _case(G, d, n, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    q = torch.randn(G, d, generator=g) * 0.3
    K = torch.randn(n, d, generator=g).to(torch.bfloat16)
    V = torch.randn(n, d, generator=g).to(torch.bfloat16)
    return q, K, V


def _oracle(q, K, V):
    Kf, Vf = K.float().numpy(), V.float().numpy()
    return np.stack([oracle.attend(q[h].numpy(), Kf, Vf) for h in range(q.shape[0])])


def _gpu(q, K, V, splits, ws=None):
    G, d = q.shape
    if ws is None:
        ws = torch.zeros(binding.attention_workspace_bytes(G, d, splits), dtype=torch.uint8,
                         device="cuda")
    out = torch.empty(G, d, device="cuda")
    binding.attention_decode(q.cuda(), K.cuda(), V.cuda(), K.shape[0], splits, ws, out)
    torch.cuda.synchronize()
    return out.cpu().numpy(), ws


@pytest.mark.parametrize("G,d,n,splits", [
    (4, 128, 1, 1), (4, 128, 1, 8), (4, 128, 300, 3), (4, 128, 4096, 16),
    (7, 64, 551, 5), (2, 64, 17, 40), (8, 64, 1000, 7), (1, 128, 64, 1),
    (4, 128, 32768, 18), (4, 128, 32768, 64),
])
def test_attention_op_matches_oracle(cuda_ok, G, d, n, splits):
    q, K, V = _case(G, d, n, seed=n * 31 + splits)
    got, _ = _gpu(q, K, V, splits)
    want = _oracle(q, K, V)
    np.testing.assert_allclose(got, want, atol=ATOL, rtol=RTOL)


def test_attention_op_reuses_its_workspace(cuda_ok):
    q, K, V = _case(4, 128, 777, seed=3)
    a, ws = _gpu(q, K, V, 9)
    b, _ = _gpu(q, K, V, 9, ws)
    q2, K2, V2 = _case(4, 128, 777, seed=4)
    c, _ = _gpu(q2, K2, V2, 9, ws)
    assert np.array_equal(a, b)
    np.testing.assert_allclose(c, _oracle(q2, K2, V2), atol=ATOL, rtol=RTOL)


def test_attention_op_rejects_bad_arguments(cuda_ok):
    q, K, V = _case(3, 128, 10, seed=1)   # 3 query heads per KV head: unsupported
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    out = torch.empty(3, 128, device="cuda")
    with pytest.raises(binding.MkError) as e:
        binding.attention_decode(q.cuda(), K.cuda(), V.cuda(), 10, 1, ws, out)
    assert e.value.code == -9
