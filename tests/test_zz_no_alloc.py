"""The allocation-free attention entry point.

mk_attention_decode_noalloc exists for callers that cannot allocate device
memory themselves (a plugin whose host owns all device memory, a real-time
loop that must stay out of allocators, code limited to the buffers it is
handed).  It must give the same result as mk_attention_decode with a
caller-provided workspace, call after call, although its scratch is one
static array shared by every call, and both must match the oracle's
attention.  This file is collected last so that a run stopping at its first
failure has run every other test already; it also passes on its own in a
fresh process (the first call sets the array up).
"""
import numpy as np
import pytest
import torch

import oracle
from persistent_megakernel_03_b200 import binding

pytestmark = pytest.mark.gpu

ATOL, RTOL = 3e-5, 1e-4   # the attention op's tolerance against the oracle


def _inputs(G, d, n, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    q = (torch.randn(G, d, generator=g) * 0.3).cuda()
    K = torch.randn(n, d, generator=g).to(torch.bfloat16).cuda()
    V = torch.randn(n, d, generator=g).to(torch.bfloat16).cuda()
    return q, K, V


def _with_workspace(q, K, V, splits, stream=None):
    G, d = q.shape
    ws = torch.zeros(binding.attention_workspace_bytes(G, d, splits), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty(G, d, device="cuda")
    binding.attention_decode(q, K, V, K.shape[0], splits, ws, out, stream=stream)
    return out


def _noalloc(q, K, V, splits, stream=None):
    out = torch.empty(q.shape, device="cuda")
    binding.attention_decode_noalloc(q, K, V, K.shape[0], splits, out, stream=stream)
    return out


def _oracle(q, K, V):
    qh, Kh, Vh = q.cpu().numpy(), K.float().cpu().numpy(), V.float().cpu().numpy()
    return np.stack([oracle.attend(qh[h], Kh, Vh) for h in range(qh.shape[0])])


# (G, head_dim, keys, splits): the last case fills the static array exactly
# (8 query heads x head_dim 128 x 64 splits = 270,592 bytes with the ticket).
CASES = [(4, 128, 2000, 64), (7, 64, 333, 5), (8, 128, 64 * 64 + 17, 64)]


def test_noalloc_matches_workspace_entry_point_and_oracle_twice_in_a_row(cuda_ok):
    # calls in a row on the shared scratch: a later call must not see an
    # earlier call's leftovers (different sizes, so stale partials would show)
    for call, (G, d, n, splits) in enumerate(CASES):
        q, K, V = _inputs(G, d, n, seed=10 + call)
        got = _noalloc(q, K, V, splits)
        want = _with_workspace(q, K, V, splits)
        torch.cuda.synchronize()
        np.testing.assert_allclose(got.cpu().numpy(), want.cpu().numpy(), atol=ATOL, rtol=RTOL)
        np.testing.assert_allclose(got.cpu().numpy(), _oracle(q, K, V), atol=ATOL, rtol=RTOL)


def test_noalloc_on_a_side_stream_at_full_capacity(cuda_ok):
    side = torch.cuda.Stream()
    G, d, n, splits = CASES[-1]
    q, K, V = _inputs(G, d, n, seed=30)
    torch.cuda.synchronize()
    with torch.cuda.stream(side):
        got1 = _noalloc(q, K, V, splits, stream=side)
        got2 = _noalloc(q, K, V, splits, stream=side)
    side.synchronize()
    want = _with_workspace(q, K, V, splits)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got1.cpu().numpy(), got2.cpu().numpy())
    np.testing.assert_allclose(got1.cpu().numpy(), want.cpu().numpy(), atol=ATOL, rtol=RTOL)


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_ok):
    q, K, V = _inputs(8, 128, 100, seed=1)
    with pytest.raises(binding.MkError) as e:
        _noalloc(q, K, V, 65)
    assert e.value.code == -1
    assert "static array" in str(e.value)
