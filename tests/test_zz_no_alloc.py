"""moga_permute_noalloc: the permute for callers that cannot allocate device memory.

Some callers have no allocator when they run the layer (plugins of another
runtime that owns the device memory, services with a fixed, pre-planned memory
budget where cudaMalloc is not allowed while serving, plain C callers).  The
no-allocation entry point keeps its scratch in a library-owned device array.
This test calls it through the C ABI and checks that it gives exactly the
outputs of the workspace-taking moga_permute, on two calls in a row with
different inputs (the second call finds the first call's data in the shared
array), then that an oversized N is refused before any launch.

The file sorts last so that a run stopping at the first failure has already
run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def _outputs(torch, dev, N, M):
    return (torch.empty(N, dtype=torch.int32, device=dev), torch.empty(M + 1, dtype=torch.int32, device=dev),
            torch.empty(M, dtype=torch.int32, device=dev), torch.empty(1, dtype=torch.int32, device=dev))


# the last two cases reach the array's bound: 2048 tiles of 2048 tokens at
# 32 groups fill both the histogram and the offset halves of the scratch
@pytest.mark.parametrize("N,M", [(282360, 20), (32760, 5), (4194304, 32), (4194304 - 77, 32)])
def test_noalloc_matches_workspace_permute_twice(cuda_device, N, M):
    import torch
    import sparse_attention_long_moga_b200 as moga
    L = moga._lib.lib()
    P = moga._ptr
    rs = np.random.default_rng(N + M)
    for call in range(2):
        # skewed group sizes, and one empty group on the second call
        probs = rs.dirichlet(np.ones(M) * (0.5 + call))
        g_host = rs.choice(M, size=N, p=probs).astype(np.int32)
        if call == 1:
            g_host[g_host == M - 1] = 0
        g = torch.from_numpy(g_host).to(cuda_device)
        ref = moga.moga_permute(g, M)
        perm, cu, counts, mx = _outputs(torch, cuda_device, N, M)
        st = L.moga_permute_noalloc(P(g), N, M, P(perm), P(cu), P(counts), P(mx), moga._stream())
        assert st == 0, L.moga_last_error()
        moga.device_status()
        for got, want in zip((perm, cu, counts, mx), ref):
            assert torch.equal(got, want)


def test_noalloc_rejects_oversized_n(cuda_device):
    import sparse_attention_long_moga_b200 as moga
    L = moga._lib.lib()
    fake = ctypes.c_void_p(4096)
    st = L.moga_permute_noalloc(fake, 4194305, 5, fake, fake, fake, fake, None)
    assert st == 3 and b"scratch limit" in L.moga_last_error()
