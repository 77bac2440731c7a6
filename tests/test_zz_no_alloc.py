"""The allocation-free top-k entry point (dsa_topk_from_scores_noalloc).

Some callers cannot allocate device memory while they run a decode step, for
example code being captured into a CUDA graph or a serving loop that forbids
allocation after start-up.  This entry point uses a static scratch array inside
the library instead of a caller workspace.  The test calls it through the C ABI
twice in a row (the second call finds the first call's leftovers in the shared
scratch) and requires the same selected indices as the workspace entry point;
index output is compared exactly.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_attention_decode_relu_b200 import dsa

pytestmark = pytest.mark.gpu


def _scores(rng, T, L, kind, ld=None):
    if kind == "ties":
        s = rng.integers(0, 50, size=(T, L)).astype(np.float32)
    elif kind == "equal":
        s = np.full((T, L), 0.5, np.float32)
    else:
        s = rng.standard_normal((T, L)).astype(np.float32)
    ld = ld or (L + 3) // 4 * 4
    out = torch.zeros((T, ld), dtype=torch.float32, device="cuda")
    out[:, :L] = torch.from_numpy(s).cuda()
    return out, s.astype(np.float64)


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_noalloc_topk_matches_workspace_entry_two_calls_in_a_row():
    rng = np.random.default_rng(2024)
    # Every call works in the one scratch array: the second finds the first
    # one's leftovers there, the third checks a shorter context on the same
    # scratch after two larger calls, and the last gives the scores a row
    # stride far beyond the scratch's own row length.
    cases = [(8, 262144, 2048, "ties", [262143 - i for i in range(8)], None),
             (3, 200000, 777, "normal", [199999, 1000, 150000], None),
             (3, 40000, 777, "normal", [39999, 1000, 20000], None),
             (8, 40000, 2048, "equal", [39999 - 977 * i for i in range(8)], 40000 + 64 + 64)]
    for T, L, k, kind, pos, ld in cases:
        scores, s_np = _scores(rng, T, L, kind, ld)
        ref = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
        ws = dsa.workspace(T, L, k)
        dsa.dsa_topk_from_scores(scores, L, pos, k, ref, ws)
        got = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
        dsa.dsa_topk_from_scores_noalloc(scores, L, pos, k, got)
        dsa.dsa_device_status()
        assert torch.equal(got, ref), (T, L, k, kind)
        assert np.array_equal(got.cpu().numpy(), oracle.topk(s_np, np.array(pos, np.int32), k)), (T, L, k, kind)


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")
def test_noalloc_rejects_sizes_beyond_its_scratch():
    scores = torch.zeros((1, 262148), dtype=torch.float32, device="cuda")
    sel = torch.empty((1, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_topk_from_scores_noalloc(scores, 262145, [10], 16, sel)
    assert e.value.status == dsa.ERR_INVALID_ARG
    assert "no-allocation scratch limit" in str(e.value)
