"""csa_n_valid (the causality rule computed by the library) against the oracle, and the
failure-detection path of the bounded waits: a wait that nothing completes runs out,
the kernel returns, csa_poll_status reports CSA_ERR_TIMEOUT once and then CSA_OK, and
the context stays usable.  No GPU fault, trap or hang is involved: the wait is bounded
by the GPU's global timer (a few milliseconds here)."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def csa():
    from long_context_compressed_b200 import csa
    return csa


@pytest.mark.parametrize("ratio,N", [(4, 1024), (4, 262144), (128, 8192), (1, 5)])
def test_n_valid_matches_oracle(csa, ratio, N):
    pos = np.concatenate([np.arange(-3, 2 * ratio + 3), [ratio * N - 2, ratio * N - 1, ratio * N, ratio * N + 7],
                          np.arange(4088, 4096), (np.arange(4096) * 31 + 126976)]).astype(np.int64)
    got = csa.csa_n_valid(torch.from_numpy(pos).cuda(), ratio, 0, N).cpu().numpy()
    assert np.array_equal(got, oracle.n_visible(pos, ratio, N))


def test_n_valid_tiny_golden(csa, golden):
    """The tiny workload's queries (positions 4088..4095, m = 4, N = 1024)."""
    g = golden("tiny_n_valid.json")
    pos = torch.arange(4088, 4096, dtype=torch.int64).cuda()
    assert csa.csa_n_valid(pos, 4, 0, 1024).cpu().tolist() == g["n_valid"]


@pytest.mark.parametrize("G", [1, 2, 3, 4])
def test_n_valid_of_shards_sums_to_the_whole(csa, G):
    """A shard holding entries [lo, hi) sees clamp(n - lo, 0, hi - lo) of them; over the
    shards these add up to the whole sequence's count."""
    from long_context_compressed_b200 import shard
    N = 12000
    pos = torch.tensor([0, 3, 4 * 3000 - 1, 4 * 6000 + 2, 4 * N - 1, 4 * N + 100], dtype=torch.int64).cuda()
    whole = oracle.n_visible(pos.cpu().numpy(), 4, N)
    parts = []
    for g in range(G):
        lo, hi = shard.shard_range(N, G, g)
        loc = csa.csa_n_valid(pos, 4, lo, hi).cpu().numpy()
        assert np.array_equal(loc, np.clip(whole - lo, 0, hi - lo))
        parts.append(loc)
    assert np.array_equal(np.sum(parts, 0), whole)


def test_bounded_wait_runs_out_and_reports_timeout(csa):
    assert csa.csa_poll_status() == csa.CSA_OK                  # nothing pending
    csa.csa_test_bounded_wait(False, 2_000_000)                 # nothing completes the barrier: 2 ms
    assert csa.csa_poll_status() == csa.CSA_ERR_TIMEOUT         # the kernel returned and recorded it
    assert csa.csa_poll_status() == csa.CSA_OK                  # read once, then cleared
    csa.csa_test_bounded_wait(True, 2_000_000)                  # completed barrier: no timeout
    assert csa.csa_poll_status() == csa.CSA_OK
    # the context is still usable
    pos = torch.arange(8, dtype=torch.int64).cuda()
    assert csa.csa_n_valid(pos, 4, 0, 100).cpu().tolist() == [0, 0, 0, 1, 1, 1, 1, 2]


def test_bounded_wait_rejects_bad_limits(csa):
    for bad in (0, 999, 10 ** 9 + 1):
        with pytest.raises(csa.CsaError) as e:
            csa.csa_test_bounded_wait(False, bad)
        assert e.value.status == csa.CSA_ERR_INVALID
    assert csa.csa_poll_status() == csa.CSA_OK
