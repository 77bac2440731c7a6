"""GPU parity of the rows beyond the core step: sliding-window decode, the step
with an attention sink, and the short-context bypass (NaiveAI research page,
"Hybrid SWA-DSA Architecture" and "A faster microbenchmark is not a faster
model").  Every call goes through the C ABI; the CPU oracle is the reference."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_attention
from sparse_attention_decode_relu_b200 import dsa, synth

pytestmark = pytest.mark.gpu


def _sink(seed):
    return np.random.default_rng(seed).standard_normal(64).astype(np.float32)


@pytest.mark.parametrize("L,T,window,with_sink", [(4096, 1, 128, False), (4096, 8, 128, True), (300, 8, 128, True),
                                                  (100, 3, 128, False), (5000, 2, 1, False), (5000, 2, 2048, True)])
def test_swa_decode_matches_oracle(L, T, window, with_sink):
    w = synth.make_workload("swa", L=L, T=T, key_dtype="bf16", recipe="normal", seed=L + T)
    pos = np.array([L - 1 - 37 * t for t in range(T)], np.int32)
    pos[-1] = min(pos[-1], 90)   # one query near the start: a short window
    q = torch.from_numpy(w.q.view(np.int16)).view(torch.bfloat16).cuda()
    kv = torch.from_numpy(w.kv.view(np.int16)).view(torch.bfloat16).cuda()
    out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device="cuda")
    sink = _sink(window) if with_sink else None
    ws = dsa.workspace(T, L, window)
    dsa.dsa_swa_decode(q, kv, pos, window, out, ws, sink=None if sink is None else torch.from_numpy(sink).cuda())
    dsa.dsa_device_status()
    ref = oracle.swa_decode(w.q, w.kv, pos, window, sink=sink)
    check_attention(out.double().cpu().numpy(), ref, f"swa L={L} T={T} W={window}")


def test_swa_rejects_bad_window():
    q = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((16, 2, 4, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    ws = dsa.workspace(1, 16, 128)
    for bad in (0, 2049):
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_swa_decode(q, kv, [15], bad, out, ws)
        assert e.value.status == dsa.ERR_INVALID_ARG


@pytest.mark.parametrize("name", ["tiny_decode", "sweep_L16384_T8"])
def test_decode_with_sink_matches_oracle(name):
    w = synth.config(name)
    d = dsa.to_device(w)
    sink = _sink(7)
    ws = dsa.workspace(w.T, w.L, w.topk)
    out = torch.empty((w.T, 64, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((w.T, w.topk), dtype=torch.int32, device="cuda")
    dsa.dsa_decode_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk, out, sel, ws,
                      k_scale=d["k_scale"], sink=torch.from_numpy(sink).cuda())
    dsa.dsa_device_status()
    sel_np = sel.cpu().numpy()
    # the sink does not change the selection; the attention uses it
    _, sel_ref = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, w.topk)
    if w.recipe == "int":
        assert np.array_equal(sel_np, sel_ref)
    check_attention(out.double().cpu().numpy(), oracle.sparse_attn(w.q, w.kv, sel_np, sink=sink), name + " sink")


@pytest.mark.parametrize("name", ["sweep_L200_T1", "sweep_L200_T8", "int_L2048_T8"])
def test_short_context_bypass_is_exact(name):
    """With every query seeing at most topk positions the bypass selects all of
    them by position; the result equals the scored path bit for bit."""
    if name == "int_L2048_T8":
        w = synth.make_workload(name, L=2048, T=8, key_dtype="bf16", recipe="int", seed=21)
    else:
        w = synth.config(name)
    assert int(w.pos.max()) + 1 <= w.topk
    d = dsa.to_device(w)
    ws = dsa.workspace(w.T, w.L, w.topk)
    res = []
    for bypass in (True, False):
        dsa.dsa_set_short_context_bypass(bypass)
        try:
            out, sel = dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk,
                                  k_scale=d["k_scale"], ws=ws)
            dsa.dsa_device_status()
        finally:
            dsa.dsa_set_short_context_bypass(True)
        res.append((out.view(torch.int16).clone(), sel.clone()))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    n = w.pos + 1
    for t in range(w.T):
        s = res[0][1][t].cpu().numpy()
        assert s[: n[t]].tolist() == list(range(n[t])) and np.all(s[n[t]:] == -1)


def test_device_positions_replay_one_graph_across_steps():
    """One CUDA graph of the step with positions in device memory serves several
    decode positions: each replay equals the host-position entry point bit for
    bit and the oracle's selection exactly (integer inputs)."""
    w = synth.config("sweep_L16384_T8_int")
    d = dsa.to_device(w)
    T, L, k = w.T, w.L, w.topk
    ws = dsa.workspace(T, L, k)
    pos_dev = torch.tensor(w.pos, dtype=torch.int32, device="cuda")
    out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((T, k), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()

    def step():
        dsa.dsa_decode_devpos_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], pos_dev, k, out, sel, ws,
                                 k_scale=d["k_scale"])

    with torch.cuda.stream(s):
        step()
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step()
    for positions in (w.pos, w.pos - 3000, np.array([16383, 100, 5000, 2047, 2048, 9000, 16000, 0], np.int32)):
        pos_dev.copy_(torch.from_numpy(positions.astype(np.int32)))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        dsa.dsa_device_status()
        ref_o, ref_s = dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], positions, k,
                                  k_scale=d["k_scale"], ws=dsa.workspace(T, L, k))
        dsa.dsa_device_status()
        assert torch.equal(sel, ref_s) and torch.equal(out.view(torch.int16), ref_o.view(torch.int16))
        o_ora, s_ora = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, positions, k)
        assert np.array_equal(sel.cpu().numpy(), s_ora)
        check_attention(out.double().cpu().numpy(), o_ora, f"device positions {positions.tolist()}")
    del g


def test_device_position_out_of_range_is_clamped_and_flagged():
    w = synth.config("tiny_decode")
    d = dsa.to_device(w)
    ws = dsa.workspace(w.T, w.L, w.topk)
    out = torch.empty((1, 64, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((1, w.topk), dtype=torch.int32, device="cuda")
    pos_dev = torch.tensor([w.L + 5], dtype=torch.int32, device="cuda")
    dsa.dsa_decode_devpos_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], pos_dev, w.topk, out, sel, ws,
                             k_scale=d["k_scale"])
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_device_status()
    assert e.value.status == dsa.ERR_DEVICE and "0x10" in str(e.value)
    # clamped to the last position: the same result as pos = L - 1
    ref_o, ref_s = dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], [w.L - 1], w.topk,
                              k_scale=d["k_scale"], ws=ws)
    dsa.dsa_device_status()
    assert torch.equal(sel, ref_s)
