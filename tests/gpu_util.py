"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs."""
import numpy as np
import torch

from sparse_attention_decode_relu_b200 import dsa

ATOL = 2e-2       # max |gpu - oracle| over all outputs (bf16 output)
REL_L2 = 1e-2     # ||gpu - oracle||_2 / ||oracle||_2
SCORE_BAND = 2.0 ** -15   # fp32 indexer error bound factor on the oracle's magnitude sum


def round_up(x, m):
    return (x + m - 1) // m * m


def gpu_scores(w, d):
    ld = round_up(w.L, 4)
    scores = torch.empty((w.T, ld), dtype=torch.float32, device="cuda")
    dsa.dsa_index_scores(d["q_idx"], d["w_idx"], d["k_idx"], w.pos, scores, k_scale=d["k_scale"])
    torch.cuda.synchronize()
    return scores[:, : w.L].double().cpu().numpy()


def gpu_decode(w, d, topk=None, ws=None):
    out, sel = dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], topk or w.topk,
                          k_scale=d["k_scale"], ws=ws)
    dsa.dsa_device_status()
    return out.double().cpu().numpy(), sel.cpu().numpy()


def check_attention(got, ref, what=""):
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert np.all(np.isfinite(got)), what
    assert err.max() <= ATOL, f"{what}: max abs err {err.max():.3e}"
    assert rel <= REL_L2, f"{what}: rel L2 err {rel:.3e}"
    return err.max(), rel


def check_scores(gs, os_, mag, pos):
    """GPU fp32 scores against the oracle's fp64 scores: -inf where invisible,
    within 2^-15 of the magnitude sum elsewhere (exact when inputs are integers)."""
    T, L = gs.shape
    vis = np.arange(L)[None, :] <= pos[:, None]
    assert np.all(np.isneginf(gs[~vis]))
    d = np.abs(gs[vis] - os_[vis])
    tol = SCORE_BAND * mag[vis]
    bad = d > tol
    assert not bad.any(), f"{bad.sum()} scores outside the fp32 band, worst {d[bad].max():.3e}"
    return d.max()


def check_selection_band(sel_gpu, sel_ora, s_ora, mag, pos, topk):
    """Float inputs: the GPU set may differ from the oracle's only at positions
    whose oracle score is within the fp32 band of the oracle's topk-th score."""
    for t in range(sel_gpu.shape[0]):
        a = sel_gpu[t][sel_gpu[t] >= 0]
        b = sel_ora[t][sel_ora[t] >= 0]
        assert np.all(np.diff(a) > 0), "not ascending"
        assert len(a) == len(b)
        if np.array_equal(a, b):
            continue
        n = int(pos[t]) + 1
        assert n > topk, "everything visible must be selected"
        order = np.lexsort((np.arange(n), -s_ora[t, :n]))
        s_tau = order[topk - 1]
        tau = s_ora[t, s_tau]
        for s in np.setxor1d(a, b):
            slack = SCORE_BAND * (mag[t, s] + mag[t, s_tau])
            assert abs(s_ora[t, s] - tau) <= slack, f"t={t} s={s}: {s_ora[t, s]} vs tau {tau}"
