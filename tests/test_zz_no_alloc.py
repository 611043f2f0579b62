"""csa_topk_noalloc: the top-k entry point for callers that cannot allocate device
memory themselves (a host that fixes its device-memory budget at start-up, a plug-in
inside an application that owns the device allocator, C code without an allocator).
Its scratch is a library-owned static device array, so it must give exactly the
indices of csa_topk with a caller workspace, and those of the oracle's full sort --
on two calls in a row, since the array keeps whatever the previous call left.

This file is collected last on purpose: a failure here leaves every other test already
run.  It also passes on its own in a fresh process (the first call sets the array's
device address up)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_compressed_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


# every shape takes the chunked path, which uses the static array as its scratch
@pytest.mark.parametrize("B,T,N,k", [(1, 1, 262144, 1024), (8, 1, 16384, 512), (2, 3, 40000, 700),
                                     (1, 1, 1 << 20, 2048)])
def test_noalloc_matches_workspace_topk_twice(csa, B, T, N, k):
    nv = np.full((B, T), N, np.int32)
    if B * T > 1:
        nv.reshape(-1)[1] = N // 2                         # a ragged row
    assert 0 < csa.csa_topk_workspace_size(B, T, N, k) <= csa.NOALLOC_SCRATCH_BYTES
    g_nv = torch.from_numpy(nv).cuda()
    for call in range(2):                                  # two calls in a row on the shared array
        s = synth.draw_scores(40 + call, f"noalloc/{B}/{T}/{N}", B, T, N, ties=4)
        g_s = s.cuda()
        want = csa.csa_topk(g_s, g_nv, k)                  # existing entry point, caller workspace
        got = csa.csa_topk_noalloc(g_s, g_nv, k)
        torch.cuda.synchronize()
        assert torch.equal(got, want), f"call {call}"
        assert np.array_equal(got.cpu().numpy(), oracle.topk(s.numpy(), nv, k)), f"call {call} vs oracle"


def test_noalloc_rejects_more_scratch_than_the_array(csa):
    B, T, N, k = 4, 1, 1 << 20, 1024                       # needs ~4 x 8.7 MiB of scratch
    assert csa.csa_topk_workspace_size(B, T, N, k) > csa.NOALLOC_SCRATCH_BYTES
    s = torch.zeros((B, T, N), device="cuda")
    nv = torch.full((B, T), N, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.csa_topk_noalloc(s, nv, k)
    assert e.value.status == csa.CSA_ERR_UNSUPPORTED
    assert csa.csa_poll_status() == csa.CSA_OK
