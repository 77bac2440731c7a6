"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle on
the same seeded inputs.  Selected index sets must match exactly on integer
inputs (and on the GPU's own scores); outputs must agree within max-abs 2e-2
and relative-L2 1e-2."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (check_attention, check_scores, check_selection_band, gpu_decode, gpu_scores, round_up)
from sparse_attention_decode_relu_b200 import dsa, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    dsa.lib()
    yield
    dsa.dsa_device_status()


def _custom(name, L, T, key_dtype, recipe, seed, pos=None, topk=2048):
    return synth.make_workload(name, L=L, T=T, key_dtype=key_dtype, recipe=recipe, seed=seed, topk=topk, pos=pos)


# Small and medium cases: several indexer tiles, ragged tails, both key formats,
# T in {1, 3, 5, 6, 7, 8}, queries at scattered positions.
SMALL = [
    ("tiny_decode", None),
    ("ragged_bf16_T3", dict(L=3001, T=3, key_dtype="bf16", recipe="normal", seed=41, pos=np.array([3000, 1500, 2047]))),
    ("ragged_fp8_T3", dict(L=2999, T=3, key_dtype="fp8", recipe="normal", seed=42, pos=np.array([2998, 2500, 10]))),
    ("ragged_fp8_T8_int", dict(L=5000, T=8, key_dtype="fp8", recipe="int", seed=43)),
    # T = 5, 6, 7 (uneven query halves) at contexts where the fused first radix pass
    # counts groups of 2, 4 and 8 keys
    ("ragged_fp8_T6", dict(L=20000, T=6, key_dtype="fp8", recipe="normal", seed=44,
                           pos=np.array([19999, 17000, 16383, 12000, 19000, 5000]))),
    ("ragged_fp8_T5", dict(L=40000, T=5, key_dtype="fp8", recipe="normal", seed=45,
                           pos=np.array([39999, 33000, 20000, 39000, 2100]))),
    ("ragged_bf16_T7_int", dict(L=70001, T=7, key_dtype="bf16", recipe="int", seed=46,
                                pos=np.array([70000, 69000, 65535, 40000, 70000, 1000, 66000]))),
    ("sweep_L2200_T8", None),
    ("sweep_L2200_T1", None),
    ("sweep_L2200_T1_int", None),
    ("sweep_L200_T8", None),
    ("sweep_L200_T1", None),
    ("sweep_L16384_T1", None),
    ("sweep_L16384_T8", None),
    ("verify_block", None),
    ("verify_block_int", None),
    ("long_decode", None),
    ("long_decode_int", None),
]


def _workload(name, kw):
    return synth.config(name) if kw is None else _custom(name, **kw)


@pytest.mark.parametrize("name,kw", SMALL, ids=[s[0] for s in SMALL])
def test_indexer_scores(name, kw):
    w = _workload(name, kw)
    d = dsa.to_device(w)
    gs = gpu_scores(w, d)
    os_ = oracle.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    mag = oracle.index_magnitude(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    check_scores(gs, os_, mag, w.pos)
    if w.recipe == "int":
        assert np.array_equal(gs, os_)   # every score is an exact fp32 integer or half-integer


def test_indexer_decodes_every_e4m3_code():
    """Every finite E4M3 code (subnormals and both zeros included) widened by the
    indexer, at every dim position: key row s holds one code at dim s % 64 (twice,
    at two dim offsets); the queries are +1 and -1 on every dim of head 0, so the
    scores are ReLU(+-value) of each code, exact in fp32."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    L = 2 * len(codes)
    k = np.zeros((L, 64), np.uint8)
    for s in range(L):
        k[s, (s + 7 * (s >= len(codes))) % 64] = codes[s % len(codes)]
    w = synth.make_workload("codes", L=L, T=2, key_dtype="fp8", recipe="int", seed=5)
    w.k_idx = k
    w.k_scale = np.ones(L, np.float32)
    qf = np.zeros((2, 16, 64), np.float32)
    qf[0, 0, :] = 1.0
    qf[1, 0, :] = -1.0
    w.q_idx = synth.f32_to_bf16_bits(qf)
    w.w_idx = np.zeros((2, 16), np.float32)
    w.w_idx[:, 0] = 1.0
    w.pos = np.array([L - 1, L - 1], np.int32)
    d = dsa.to_device(w, with_kv=False)
    gs = gpu_scores(w, d)
    os_ = oracle.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    assert np.array_equal(gs, os_)
    assert (gs > 0).sum() == 2 * 2 * 126   # 126 positive and 126 negative non-zero codes, twice


@pytest.mark.parametrize("name,kw", SMALL, ids=[s[0] for s in SMALL])
def test_decode_step(name, kw):
    w = _workload(name, kw)
    d = dsa.to_device(w)
    out, sel = gpu_decode(w, d)
    # 1. the selection equals the exact top-k of the GPU's own fp32 scores
    gs = gpu_scores(w, d)
    assert np.array_equal(sel, oracle.topk(gs, w.pos, w.topk))
    # 2. against the oracle's fp64 selection: exact on integer inputs, band otherwise
    ref_out, ref_sel, s_ora = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, w.topk,
                                            want_scores=True)
    if w.recipe == "int":
        assert np.array_equal(sel, ref_sel)
    else:
        mag = oracle.index_magnitude(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
        check_selection_band(sel, ref_sel, s_ora, mag, w.pos, w.topk)
    # 3. attention: on the GPU's own selection (isolates the attention kernel) and end to end
    check_attention(out, oracle.sparse_attn(w.q, w.kv, sel), name + " (gpu selection)")
    check_attention(out, ref_out, name + " (end to end)")


@pytest.mark.parametrize("L,T", [(1, 1), (2, 1), (2047, 8), (2048, 8), (2049, 8), (2052, 8), (2056, 8), (2055, 1)])
def test_edge_contexts(L, T):
    """Context lengths straddling topk inside an 8-token block, and L = 1."""
    w = _custom("edge", L=L, T=T, key_dtype="fp8", recipe="int", seed=L)
    d = dsa.to_device(w)
    out, sel = gpu_decode(w, d)
    ref_out, ref_sel = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, w.topk)
    assert np.array_equal(sel, ref_sel)
    check_attention(out, ref_out, f"L={L} T={T}")


@pytest.mark.parametrize("topk", [1, 2, 7, 100, 1000, 2047])
def test_small_topk(topk):
    w = _custom("k", L=6000, T=2, key_dtype="bf16", recipe="int", seed=topk, topk=topk)
    d = dsa.to_device(w)
    out, sel = gpu_decode(w, d, topk=topk)
    ref_out, ref_sel = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, topk)
    assert np.array_equal(sel, ref_sel)
    check_attention(out, ref_out, f"topk={topk}")


def _topk_gpu(scores_np, pos, topk, ld=None):
    T, L = scores_np.shape
    ld = ld or round_up(L, 4)
    s = torch.full((T, ld), float("nan"), dtype=torch.float32, device="cuda")
    s[:, :L] = torch.from_numpy(scores_np.astype(np.float32)).cuda()
    sel = torch.empty((T, topk), dtype=torch.int32, device="cuda")
    ws = dsa.workspace(T, L, topk)
    dsa.dsa_topk_from_scores(s, L, pos, topk, sel, ws)
    dsa.dsa_device_status()
    return sel.cpu().numpy()


@pytest.mark.parametrize("case", ["all_equal", "signed_zero", "ties_at_threshold", "few_distinct", "huge_tie",
                                  "negative", "spread", "inf"])
def test_topk_stage_exact(case):
    rng = np.random.default_rng(sum(map(ord, case)))
    T, L, k = 3, 50000, 2048
    if case == "all_equal":
        s = np.full((T, L), 3.5)
    elif case == "signed_zero":
        s = np.where(rng.random((T, L)) < 0.5, -0.0, 0.0)
        s[:, ::97] = 1.0
    elif case == "ties_at_threshold":
        s = rng.integers(0, 40, size=(T, L)).astype(np.float64)
    elif case == "few_distinct":
        s = rng.choice([-1.0, 2.0, 2.0 + 2 ** -20, 7.0], size=(T, L))
    elif case == "huge_tie":   # more than 8192 candidates in the threshold bin: global-memory path
        s = np.zeros((T, L))
        s[:, rng.choice(L, 100, replace=False)] = 5.0
    elif case == "negative":
        s = -rng.random((T, L)) * 1e30
    elif case == "inf":
        s = rng.standard_normal((T, L))
        s[:, ::1000] = np.inf
        s[:, 5::1000] = -np.inf
    else:
        s = rng.standard_normal((T, L)) * np.exp(rng.uniform(-30, 30, size=(T, L)))
    s = s.astype(np.float32).astype(np.float64)
    pos = np.array([L - 1, L // 2, 3000], np.int32)
    assert np.array_equal(_topk_gpu(s, pos, k), oracle.topk(s, pos, k))


def test_topk_stage_wide_score_stride():
    """A score row stride far above the workspace's own row length: the
    candidate lists keep the workspace's stride (every score tied, so every
    visible position is a candidate)."""
    T, L, k = 8, 40000, 2048
    s = np.full((T, L), 1.25)
    pos = np.array([L - 1 - 977 * t for t in range(T)], np.int32)
    ld = round_up(L, 64) + 64
    got = _topk_gpu(s, pos, k, ld=ld)
    assert np.array_equal(got, oracle.topk(s, pos, k))
    assert np.array_equal(got, _topk_gpu(s, pos, k))


def test_topk_stage_many_chunks():
    rng = np.random.default_rng(7)
    T, L = 2, 1 << 20
    s = rng.integers(0, 5000, size=(T, L)).astype(np.float32).astype(np.float64)
    pos = np.array([L - 1, L - 12345], np.int32)
    for k in (2048, 1, 333):
        assert np.array_equal(_topk_gpu(s, pos, k), oracle.topk(s, pos, k))


def test_attention_stage_with_sink_and_padding():
    rng = np.random.default_rng(8)
    w = _custom("sink", L=9000, T=4, key_dtype="bf16", recipe="normal", seed=9, pos=np.array([8999, 4000, 100, 7000]))
    d = dsa.to_device(w)
    sel = np.full((4, 2048), -1, np.int32)
    for t in range(4):
        m = min(int(w.pos[t]) + 1, [2048, 1500, 101, 33][t])
        sel[t, :m] = np.sort(rng.choice(int(w.pos[t]) + 1, m, replace=False))
    sink = rng.standard_normal(64).astype(np.float32) * 3
    out = torch.empty((4, 64, 128), dtype=torch.bfloat16, device="cuda")
    ws = dsa.workspace(4, w.L, 2048)
    sel_t = torch.from_numpy(sel).cuda()
    for sk in (None, sink):
        dsa.dsa_sparse_attn(d["q"], d["kv"], sel_t, w.pos, out, ws,
                            sink=None if sk is None else torch.from_numpy(sk).cuda())
        dsa.dsa_device_status()
        check_attention(out.double().cpu().numpy(), oracle.sparse_attn(w.q, w.kv, sel, sink=sk), "sink")


def test_bad_selected_index_is_flagged_not_read():
    w = _custom("bad", L=3000, T=1, key_dtype="bf16", recipe="normal", seed=10)
    d = dsa.to_device(w)
    sel = np.arange(2048, dtype=np.int32)[None, :].copy()
    sel[0, 5] = 10 ** 9          # outside the cache
    sel[0, 6] = int(w.pos[0]) + 0   # fine
    out = torch.empty((1, 64, 128), dtype=torch.bfloat16, device="cuda")
    ws = dsa.workspace(1, w.L, 2048)
    dsa.dsa_sparse_attn(d["q"], d["kv"], torch.from_numpy(sel).cuda(), w.pos, out, ws)
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_device_status()
    assert e.value.status == dsa.ERR_DEVICE
    ok = sel.copy()
    ok[0, 5] = -1
    check_attention(out.double().cpu().numpy(), oracle.sparse_attn(w.q, w.kv, ok), "skipped bad row")
    dsa.dsa_device_status()   # the error word was cleared


def test_determinism_bitwise():
    w = synth.config("verify_block")
    d = dsa.to_device(w)
    ws = dsa.workspace(w.T, w.L, w.topk)
    outs, sels, scs = [], [], []
    for _ in range(20):
        o, s = dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk,
                          k_scale=d["k_scale"], ws=ws)
        outs.append(o.view(torch.int16).clone())
        sels.append(s.clone())
        scs.append(torch.from_numpy(gpu_scores(w, d)))
    for i in range(1, 20):
        assert torch.equal(outs[0], outs[i]) and torch.equal(sels[0], sels[i]) and torch.equal(scs[0], scs[i])


def test_graph_capture_replays_the_step():
    w = synth.config("long_decode")
    d = dsa.to_device(w)
    ws = dsa.workspace(w.T, w.L, w.topk)
    out = torch.empty((w.T, 64, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((w.T, w.topk), dtype=torch.int32, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        dsa.dsa_decode_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk, out, sel, ws,
                          k_scale=d["k_scale"])
    torch.cuda.synchronize()
    ref_o, ref_s = out.clone(), sel.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        dsa.dsa_decode_ws(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk, out, sel, ws,
                          k_scale=d["k_scale"])
    out.zero_()
    sel.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_o.view(torch.int16)) and torch.equal(sel, ref_s)
    del g


@pytest.mark.slow
@pytest.mark.parametrize("name", ["sweep_L262144_T8", "sweep_L262144_T1", "sweep_L262144_T1_int"])
def test_sweep_256k(name):
    w = synth.config(name)
    d = dsa.to_device(w)
    out, sel = gpu_decode(w, d)
    ref_out, ref_sel, s_ora = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, w.topk,
                                            want_scores=True)
    if w.recipe == "int":
        assert np.array_equal(sel, ref_sel)
    else:
        mag = oracle.index_magnitude(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
        check_selection_band(sel, ref_sel, s_ora, mag, w.pos, w.topk)
    check_attention(out, oracle.sparse_attn(w.q, w.kv, sel), name)
    check_attention(out, ref_out, name + " end to end")


@pytest.mark.slow
def test_verify_1m_planted():
    """The 1M-context planted workload at full size: the selection is exactly the
    planted set for every query, and the output matches the oracle."""
    w = synth.config("verify_1m")
    d = dsa.to_device(w)
    out, sel = gpu_decode(w, d)
    for t in range(w.T):
        assert np.array_equal(sel[t], w.planted)
    check_attention(out, oracle.sparse_attn(w.q, w.kv, sel), "verify_1m")
    gs = gpu_scores(w, d)
    os_ = oracle.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    mag = oracle.index_magnitude(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    check_scores(gs, os_, mag, w.pos)


@pytest.mark.slow
def test_verify_1m_integer_twin_selection():
    w = synth.config("verify_1m_int")
    d = dsa.to_device(w, with_kv=False)
    gs = gpu_scores(w, d)
    os_ = oracle.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    assert np.array_equal(gs, os_)
    sel = torch.empty((w.T, w.topk), dtype=torch.int32, device="cuda")
    ld = round_up(w.L, 4)
    s = torch.empty((w.T, ld), dtype=torch.float32, device="cuda")
    dsa.dsa_index_scores(d["q_idx"], d["w_idx"], d["k_idx"], w.pos, s, k_scale=d["k_scale"])
    dsa.dsa_topk_from_scores(s, w.L, w.pos, w.topk, sel, dsa.workspace(w.T, w.L, w.topk))
    dsa.dsa_device_status()
    assert np.array_equal(sel.cpu().numpy(), oracle.topk(os_, w.pos, w.topk))


def _ctrl_words_zero(ws):
    words = ws[:1024].view(torch.int32)
    return all(int(words[i]) == 0 for i in dsa.WS_WORDS_ZERO_AFTER_CALL)


def test_workspace_control_words_left_zero_and_checked():
    """Each launch leaves the workspace's grid-barrier and per-query words at zero
    (and advances its launch counter), so a workspace needs zeroing only once; a
    launch that finds the barrier words non-zero reports it (device error word)
    and skips the work that depends on the barrier."""
    w = synth.config("tiny_decode")
    d = dsa.to_device(w)
    ws = dsa.workspace(w.T, w.L, w.topk)
    ref_o, ref_s = gpu_decode(w, d, ws=ws)
    assert _ctrl_words_zero(ws)
    assert int(ws[:1024].view(torch.int32)[64]) == 1   # one launch so far
    o1, s1 = gpu_decode(w, d, ws=ws)                    # the other histogram buffer, same result
    assert np.array_equal(s1, ref_s) and np.array_equal(o1, ref_o) and _ctrl_words_zero(ws)
    ws[:4].view(torch.int32).fill_(1 << 16)       # an arrival count no launch can start from
    out, sel = dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk,
                          k_scale=d["k_scale"], ws=ws)
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_device_status()
    assert e.value.status == dsa.ERR_DEVICE and "0x8" in str(e.value)
    ws[: dsa.WS_CTRL_BYTES].zero_()
    o2, s2 = gpu_decode(w, d, ws=ws)
    assert np.array_equal(s2, ref_s) and np.array_equal(o2, ref_o)


def test_barrier_wait_timeout_is_reported_and_recovers():
    """Failure detection of the single cooperative kernel: with the test hook,
    every wait between blocks of one launch waits for a block that never comes.  Each
    bounded wait runs out (about 1 ms here), the launch reports the wait-timeout
    bit alone, leaves the workspace control words at zero, and the next call on
    the same workspace matches the oracle again."""
    w = synth.config("tiny_decode")   # 4096 positions, one query: every phase and barrier runs
    d = dsa.to_device(w)
    ws = dsa.workspace(w.T, w.L, w.topk)
    ref_o, ref_s = gpu_decode(w, d, ws=ws)
    dsa.dsa_debug_fail_next_barriers(2_000_000)
    dsa.decode(d["q"], d["q_idx"], d["w_idx"], d["k_idx"], d["kv"], d["pos"], w.topk, k_scale=d["k_scale"], ws=ws)
    with pytest.raises(dsa.DsaError) as e:
        dsa.dsa_device_status()
    assert e.value.status == dsa.ERR_DEVICE and "word 0x1 " in str(e.value)
    assert _ctrl_words_zero(ws)
    o2, s2 = gpu_decode(w, d, ws=ws)   # the hook covered one launch only
    assert np.array_equal(s2, ref_s) and np.array_equal(o2, ref_o)
    ora_o, ora_s = oracle.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, w.topk)
    assert np.array_equal(s2, ora_s)
    check_attention(o2, ora_o, "after a timed-out launch")
