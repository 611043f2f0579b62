"""Top-k parity: bit-exact indices against the oracle's full sort on the same fp32
score buffers (drawn by the seeded generator, with planted exact ties and +-0.0)."""
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


def _run(csa, scores, nv, k):
    g = csa.csa_topk(scores.cuda(), torch.from_numpy(nv).cuda(), k).cpu().numpy()
    ref = oracle.topk(scores.numpy(), nv, k)
    assert np.array_equal(g, ref), f"mismatch in {np.argwhere((g != ref).any(-1))[:5].tolist()}"
    return g


@pytest.mark.parametrize("B,T,N,k", [
    (1, 8, 1024, 64),          # tiny: row-resident path
    (8, 1, 16384, 512),        # flash decode: chunk path (few rows)
    (1, 1, 262144, 1024),      # pro 1M decode: chunk path (long row)
    (1, 96, 5000, 512),        # many rows, ragged N: row path
    (2, 3, 40000, 700),        # N above the resident limit: chunk path, odd k
    (1, 1, 1 << 20, 2048),     # maximum N and k
])
def test_topk_shapes(csa, B, T, N, k):
    s = synth.draw_scores(0, f"topk/{B}/{T}/{N}", B, T, N, ties=8)
    nv = np.full((B, T), N, np.int32)
    _run(csa, s, nv, k)


@pytest.mark.parametrize("N", [3000, 20000, 100000])
def test_topk_ragged_n_valid(csa, N):
    """Rows with n_valid below N (the tail must be ignored even if it holds large values),
    n_valid < k (all valid then -1), n_valid == k, and n_valid == 0."""
    B, T, k = 1, 6, 512
    s = synth.draw_scores(1, f"topk/ragged/{N}", B, T, N, ties=4)
    nv = np.array([[N, N - 1, N // 2 + 3, k, k - 7, 0]], np.int32)
    s[0, 2, nv[0, 2]:] = 1e30                            # huge values past n_valid must not be chosen
    _run(csa, s, nv, k)


@pytest.mark.parametrize("N", [2048, 50000])
def test_topk_all_equal_and_signed_zero(csa, N):
    """Degenerate rows: every score equal (the k lowest indices win), all +-0.0 mixed,
    and a row where exactly k-1 values exceed a tied block."""
    B, T, k = 1, 3, 256
    s = torch.zeros(B, T, N)
    s[0, 0] = 3.25
    s[0, 1] = torch.where(torch.arange(N) % 3 == 0, torch.tensor(-0.0), torch.tensor(0.0))
    s[0, 2] = 1.0
    pos = synth.uniform(2, "topk/eqpos", (k - 1,)) * N
    s[0, 2, pos.long()] = 2.0
    nv = np.full((B, T), N, np.int32)
    g = _run(csa, s, nv, k)
    assert g[0, 0].tolist() == list(range(k))
    assert g[0, 1].tolist() == list(range(k))


def test_topk_workloads_chunk_and_row_paths_agree(csa):
    """The same rows through both paths (as one batch of many rows and as few rows)."""
    N, k = 16384, 512
    s = synth.draw_scores(3, "topk/paths", 1, 80, N, ties=4)
    nv = np.full((1, 80), N, np.int32)
    many = csa.csa_topk(s.cuda(), torch.from_numpy(nv).cuda(), k).cpu()        # row path (80 rows)
    few = torch.cat([csa.csa_topk(s[:, i:i + 8].contiguous().cuda(), torch.from_numpy(nv[:, i:i + 8]).cuda(), k).cpu()
                     for i in range(0, 80, 8)], 1)                            # chunk path (8 rows)
    assert torch.equal(many, few)


def test_topk_workspace_stays_zero(csa):
    """The long-row path leaves its workspace zero-filled, so calls can repeat."""
    N, k = 262144, 1024
    ws = csa.topk_workspace(1, 1, N, k)
    for seed in range(3):
        s = synth.draw_scores(seed, "topk/ws", 1, 1, N)
        nv = np.full((1, 1), N, np.int32)
        g = csa.csa_topk(s.cuda(), torch.from_numpy(nv).cuda(), k, workspace=ws).cpu().numpy()
        assert np.array_equal(g, oracle.topk(s.numpy(), nv, k))
        torch.cuda.synchronize()
        assert int(ws.count_nonzero()) == 0
