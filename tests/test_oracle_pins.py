"""Pins for the CPU oracle: each check ties the oracle to something other than
itself (a library routine, a closed form, brute force, or a hand-worked or
spec-printed fixture under tests/golden/).  Runs on CPU."""
import math
import os

import numpy as np
import pytest
import torch

from sparse_attention_decode_relu_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- codecs
def test_e4m3_spec_table(orc):
    """Printed E4M3 values of the OCP OFP8 spec (Table 1)."""
    for line in open(os.path.join(GOLD, "e4m3_spec.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        got = orc.e4m3(int(code, 16))
        if val == "nan":
            assert math.isnan(got), code
        else:
            assert got == float(val), code
            assert math.copysign(1.0, got) == math.copysign(1.0, float(val)), code


def test_e4m3_all_codes_match_torch(orc):
    """All 256 codes against torch's float8_e4m3fn widening (a library routine)."""
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([orc.e4m3(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_matches_torch(orc):
    rng = np.random.default_rng(5)
    bits = np.concatenate([rng.integers(0, 1 << 16, 4000), [0, 0x8000, 0x3F80, 0xBF80, 0x7F7F, 0x0001]]).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]  # finite values only
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([orc.bf16(b) for b in bits])
    assert np.array_equal(got, ref)


# ---------------------------------------------------------------- indexer
def _hand():
    d = {}
    ks = []
    for line in open(os.path.join(GOLD, "indexer_hand.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, *vals = line.split()
        if key == "k":
            ks.append([float(v) for v in vals])
        else:
            d[key] = vals
    q_idx = np.zeros((1, 16, 64), np.float32)
    q_idx[0, 0, :3] = [float(v) for v in d["q0"]]
    q_idx[0, 5, :3] = [float(v) for v in d["q5"]]
    w = np.zeros((1, 16), np.float32)
    w[0, 0] = float(d["w0"][0])
    w[0, 5] = float(d["w5"][0])
    k = np.zeros((len(ks), 64), np.float32)
    k[:, :3] = np.array(ks)
    return d, synth.f32_to_bf16_bits(q_idx), w, k


def test_indexer_hand_worked(orc):
    d, q_idx, w, k = _hand()
    pos = np.array([int(d["pos"][0])], np.int32)
    for keys, scale in ((synth.f32_to_bf16_bits(k), None), (synth.f32_to_e4m3_codes(k), np.ones(len(k), np.float32))):
        s = orc.index_scores(q_idx, w, keys, scale, pos)
        assert s[0].tolist() == [float(v) for v in d["scores"]]
        s4 = orc.index_scores(q_idx, w, keys, scale, np.array([4], np.int32))
        assert s4[0].tolist() == [float(v) for v in d["scores_pos4"]]
    s = orc.index_scores(q_idx, w, synth.f32_to_bf16_bits(k), None, pos)
    for kk in (1, 2, 3, 4, 5, 6, 7):
        assert orc.topk(s, pos, kk)[0].tolist() == [int(v) for v in d["topk%d" % kk]], kk


def _rand_idx(rng, T, L, fp8):
    q_idx = synth.f32_to_bf16_bits(rng.standard_normal((T, 16, 64), dtype=np.float32))
    w = rng.random((T, 16), dtype=np.float32)
    kf = rng.standard_normal((L, 64), dtype=np.float32)
    if fp8:
        return q_idx, w, synth.f32_to_e4m3_codes(kf), (0.5 + 1.5 * rng.random(L)).astype(np.float32)
    return q_idx, w, synth.f32_to_bf16_bits(kf), None


def _dequant(keys, scale):
    if keys.dtype == np.uint8:
        k = torch.from_numpy(keys).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    else:
        k = synth.bf16_bits_to_f32(keys).astype(np.float64)
    return k if scale is None else k * scale.astype(np.float64)[:, None]


@pytest.mark.parametrize("fp8", [False, True])
def test_indexer_one_hot_head_is_relu_matmul(orc, fp8):
    """w = e_j reduces the indexer to ReLU(K q_j) for one head: a plain matmul."""
    rng = np.random.default_rng(11)
    T, L = 2, 300
    q_idx, _, keys, scale = _rand_idx(rng, T, L, fp8)
    K = _dequant(keys, scale)
    pos = np.array([L - 1, 137], np.int32)
    for j in (0, 7, 15):
        w = np.zeros((T, 16), np.float32)
        w[:, j] = 1.0
        s = orc.index_scores(q_idx, w, keys, scale, pos)
        for t in range(T):
            qj = synth.bf16_bits_to_f32(q_idx[t, j]).astype(np.float64)
            ref = np.maximum(K @ qj, 0.0)
            n = pos[t] + 1
            np.testing.assert_allclose(s[t, :n], ref[:n], rtol=1e-12, atol=1e-12)
            assert np.all(np.isneginf(s[t, n:]))


@pytest.mark.parametrize("fp8", [False, True])
def test_indexer_relu_free_regime_is_one_matmul(orc, fp8):
    """If every head's dot product is positive the ReLU is inactive and the score
    is linear: I[t,s] = k[s] . (sum_j w[t,j] q_idx[t,j])  (one matmul)."""
    rng = np.random.default_rng(12)
    T, L = 3, 257
    q_idx = synth.f32_to_bf16_bits(rng.random((T, 16, 64), dtype=np.float32) + 0.1)
    w = (rng.random((T, 16), dtype=np.float32) * 2 - 0.5).astype(np.float32)  # includes negative weights
    kf = rng.random((L, 64), dtype=np.float32) + 0.05
    if fp8:
        keys, scale = synth.f32_to_e4m3_codes(kf), (0.5 + 1.5 * rng.random(L)).astype(np.float32)
    else:
        keys, scale = synth.f32_to_bf16_bits(kf), None
    K = _dequant(keys, scale)
    Q = synth.bf16_bits_to_f32(q_idx).astype(np.float64)
    pos = np.full(T, L - 1, np.int32)
    s = orc.index_scores(q_idx, w, keys, scale, pos)
    combined = np.einsum("tj,tjd->td", w.astype(np.float64), Q)
    ref = combined @ K.T
    np.testing.assert_allclose(s, ref, rtol=1e-11, atol=1e-9)


def test_indexer_properties(orc):
    rng = np.random.default_rng(13)
    T, L = 2, 200
    q_idx, w, keys, scale = _rand_idx(rng, T, L, True)
    pos = np.full(T, L - 1, np.int32)
    base = orc.index_scores(q_idx, w, keys, scale, pos)
    # zero weights -> zero scores
    assert np.all(orc.index_scores(q_idx, np.zeros_like(w), keys, scale, pos) == 0.0)
    # non-negative weights -> non-negative scores; negating every query flips the
    # sign of every dot product, so the score becomes sum_j w_j ReLU(-dot)
    assert np.all(base >= 0.0)
    neg = orc.index_scores(q_idx ^ np.uint16(0x8000), w, keys, scale, pos)
    K = _dequant(keys, scale)
    Q = synth.bf16_bits_to_f32(q_idx).astype(np.float64)
    dots = np.einsum("tjd,sd->tjs", Q, K)
    np.testing.assert_allclose(base, np.einsum("tj,tjs->ts", w.astype(np.float64), np.maximum(dots, 0)), rtol=1e-12)
    np.testing.assert_allclose(neg, np.einsum("tj,tjs->ts", w.astype(np.float64), np.maximum(-dots, 0)), rtol=1e-12)
    # the per-token scale is a positive factor on the score
    s2 = orc.index_scores(q_idx, w, keys, 2 * scale, pos)
    np.testing.assert_allclose(s2, 2 * base, rtol=1e-14)
    # permuting the heads (with their weights) changes nothing
    perm = rng.permutation(16)
    np.testing.assert_allclose(orc.index_scores(q_idx[:, perm], w[:, perm], keys, scale, pos), base, rtol=1e-12)


def test_indexer_integer_inputs_give_exact_integers(orc):
    w = synth.config("tiny_decode")
    s = orc.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    assert np.all(s == np.round(s))
    assert s.max() < 2 ** 24


# ---------------------------------------------------------------- error-band magnitude
def test_index_magnitude_hand_worked(orc):
    """The magnitude sum M = scale * sum_j |w_j| * sum_d |q_jd k_d| of the
    hand-worked example, worked out by hand in the fixture (bf16 and E4M3 keys,
    with and without per-token scales, an invisible position)."""
    d, q_idx, w, k = _hand()
    pos = np.array([int(d["pos"][0])], np.int32)
    scale = np.array([float(v) for v in d["scale"]], np.float32)
    for keys, ones in ((synth.f32_to_bf16_bits(k), None), (synth.f32_to_e4m3_codes(k), np.ones(len(k), np.float32))):
        assert orc.index_magnitude(q_idx, w, keys, ones, pos)[0].tolist() == [float(v) for v in d["magnitude"]]
        m4 = orc.index_magnitude(q_idx, w, keys, ones, np.array([4], np.int32))
        assert m4[0].tolist() == [float(v) for v in d["magnitude_pos4"]]
    e4 = synth.f32_to_e4m3_codes(k)
    got = orc.index_magnitude(q_idx, w, e4, scale, pos)[0].tolist()
    assert got == [float(v) for v in d["magnitude_scaled"]]


@pytest.mark.parametrize("fp8", [False, True])
def test_index_magnitude_matches_numpy(orc, fp8):
    """Against a numpy restatement on dequantised inputs: |w| @ (|Q| |K8|^T),
    times the per-token scale; negative weights count by their absolute value,
    scales are not uniform, invisible positions give 0."""
    rng = np.random.default_rng(31 + fp8)
    T, L = 3, 333
    q_idx, w, keys, scale = _rand_idx(rng, T, L, fp8)
    w = (w * 2 - 1).astype(np.float32)   # mixed signs
    pos = np.array([L - 1, 200, 0], np.int32)
    got = orc.index_magnitude(q_idx, w, keys, scale, pos)
    Q = np.abs(synth.bf16_bits_to_f32(q_idx).astype(np.float64))
    K8 = np.abs(_dequant(keys, None))
    ref = np.einsum("tj,tjs->ts", np.abs(w.astype(np.float64)), np.einsum("tjd,sd->tjs", Q, K8))
    if scale is not None:
        ref = ref * scale.astype(np.float64)[None, :]
    ref[np.arange(L)[None, :] > pos[:, None]] = 0.0
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=0)


def test_index_magnitude_bounds_the_score(orc):
    """|I| <= M always (triangle inequality, ReLU is 1-Lipschitz through 0), with
    equality when every query, key and weight is non-negative (then nothing is
    cancelled or clipped)."""
    rng = np.random.default_rng(33)
    T, L = 2, 250
    q_idx, w, keys, scale = _rand_idx(rng, T, L, True)
    w = (w * 2 - 1).astype(np.float32)
    pos = np.full(T, L - 1, np.int32)
    s = orc.index_scores(q_idx, w, keys, scale, pos)
    m = orc.index_magnitude(q_idx, w, keys, scale, pos)
    assert np.all(np.abs(s) <= m * (1 + 1e-12))
    qp = synth.f32_to_bf16_bits(rng.random((T, 16, 64), dtype=np.float32))
    wp = rng.random((T, 16), dtype=np.float32)
    kp = synth.f32_to_e4m3_codes(rng.random((L, 64), dtype=np.float32) * 3)
    np.testing.assert_allclose(orc.index_scores(qp, wp, kp, scale, pos), orc.index_magnitude(qp, wp, kp, scale, pos),
                               rtol=1e-13, atol=0)


# ---------------------------------------------------------------- top-k
def _brute_topk(scores, pos, k):
    T = scores.shape[0]
    out = np.full((T, k), -1, np.int32)
    for t in range(T):
        n = int(pos[t]) + 1
        idx = np.arange(n)
        if n <= k:
            out[t, :n] = idx
            continue
        order = np.lexsort((idx, -scores[t, :n]))  # primary: score desc, then position asc
        out[t] = np.sort(order[:k])
    return out


@pytest.mark.parametrize("k", [1, 4, 8, 33])
def test_topk_matches_full_sort(orc, k):
    rng = np.random.default_rng(20 + k)
    for trial in range(20):
        T, L = 4, int(rng.integers(1, 64))
        scores = rng.integers(-3, 4, size=(T, L)).astype(np.float64)  # heavy ties
        if trial % 2:
            scores = rng.standard_normal((T, L))
        pos = rng.integers(0, L, size=T).astype(np.int32)
        assert np.array_equal(orc.topk(scores, pos, k), _brute_topk(scores, pos, k))


def test_topk_special_cases(orc):
    L = 50
    pos = np.array([L - 1, 10, 0], np.int32)
    eq = np.full((3, L), 7.0)
    sel = orc.topk(eq, pos, 8)
    assert sel[0].tolist() == list(range(8))                  # all equal -> lowest positions
    assert sel[1].tolist() == list(range(8))
    assert sel[2].tolist() == [0] + [-1] * 7                  # pos = 0 -> one candidate
    sel = orc.topk(eq, pos, 11)
    assert sel[1].tolist() == list(range(11))                 # n == k -> everything
    z = np.zeros((1, 4))
    z[0, 1] = -0.0
    assert orc.topk(z, np.array([3], np.int32), 2)[0].tolist() == [0, 1]   # -0 equals +0
    bad = np.zeros((1, 4))
    bad[0, 2] = np.nan
    with pytest.raises(ValueError):
        orc.topk(bad, np.array([3], np.int32), 2)


# ---------------------------------------------------------------- attention
def _torch_masked_attention(q_bits, kv_bits, sel, sink=None):
    """Dense attention over all L rows with a boolean mask (torch SDPA, fp64)."""
    T = q_bits.shape[0]
    L = kv_bits.shape[0]
    q = torch.from_numpy(synth.bf16_bits_to_f32(q_bits).astype(np.float64))           # [T,64,128]
    kv = torch.from_numpy(synth.bf16_bits_to_f32(kv_bits).astype(np.float64))         # [L,2,4,128]
    K = kv[:, 0].permute(1, 0, 2)                                                      # [4,L,128]
    V = kv[:, 1].permute(1, 0, 2)
    out = torch.empty(T, 64, 128, dtype=torch.float64)
    for t in range(T):
        mask = torch.zeros(L, dtype=torch.bool)
        s = sel[t][sel[t] >= 0]
        mask[torch.from_numpy(s.astype(np.int64))] = True
        qt = q[t].reshape(4, 16, 128)
        if sink is None:
            o = torch.nn.functional.scaled_dot_product_attention(qt, K, V, attn_mask=mask[None, None, :])
        else:  # a sink is an extra key whose logit is sink[h] and whose value is zero
            z = torch.einsum("ghd,gld->ghl", qt, K) / math.sqrt(128)
            z = z.masked_fill(~mask[None, None, :], -math.inf)
            zs = torch.from_numpy(sink.astype(np.float64)).reshape(4, 16, 1)
            p = torch.softmax(torch.cat([z, zs], dim=-1), dim=-1)[..., :L]
            o = torch.einsum("ghl,gld->ghd", p, V)
        out[t] = o.reshape(64, 128)
    return out.numpy()


@pytest.mark.parametrize("k", [1, 7, 64])
def test_attention_matches_torch_sdpa(orc, k):
    rng = np.random.default_rng(30 + k)
    T, L = 3, 150
    q = synth.f32_to_bf16_bits(rng.standard_normal((T, 64, 128), dtype=np.float32))
    kv = synth.f32_to_bf16_bits(rng.standard_normal((L, 2, 4, 128), dtype=np.float32))
    sel = np.full((T, k), -1, np.int32)
    for t in range(T):
        m = int(rng.integers(1, k + 1))
        sel[t, :m] = np.sort(rng.choice(L, m, replace=False))
    got = orc.sparse_attn(q, kv, sel)
    np.testing.assert_allclose(got, _torch_masked_attention(q, kv, sel), rtol=1e-11, atol=1e-12)


def test_attention_sink_matches_torch(orc):
    rng = np.random.default_rng(39)
    T, L, k = 2, 90, 16
    q = synth.f32_to_bf16_bits(rng.standard_normal((T, 64, 128), dtype=np.float32))
    kv = synth.f32_to_bf16_bits(rng.standard_normal((L, 2, 4, 128), dtype=np.float32))
    sel = np.sort(np.stack([rng.choice(L, k, replace=False) for _ in range(T)]), axis=1).astype(np.int32)
    sink = rng.standard_normal(64).astype(np.float32)
    np.testing.assert_allclose(orc.sparse_attn(q, kv, sel, sink=sink),
                               _torch_masked_attention(q, kv, sel, sink=sink), rtol=1e-11, atol=1e-12)


def test_attention_closed_forms(orc):
    rng = np.random.default_rng(40)
    L = 40
    q = synth.f32_to_bf16_bits(rng.standard_normal((1, 64, 128), dtype=np.float32))
    kv = synth.f32_to_bf16_bits(rng.standard_normal((L, 2, 4, 128), dtype=np.float32))
    V = synth.bf16_bits_to_f32(kv[:, 1]).astype(np.float64)        # [L,4,128]
    # one selected row -> its V row, for every head of its group
    sel = np.array([[17, -1, -1]], np.int32)
    out = orc.sparse_attn(q, kv, sel)
    for h in range(64):
        assert np.array_equal(out[0, h], V[17, h // 16])
    # zero query -> uniform weights -> mean of the selected V rows
    rows = np.array([[1, 5, 9, 30]], np.int32)
    out = orc.sparse_attn(np.zeros_like(q), kv, rows)
    for h in range(64):
        np.testing.assert_allclose(out[0, h], V[rows[0], h // 16].mean(axis=0), rtol=1e-13, atol=1e-15)
    # constant V across the selected rows -> that V
    kv2 = kv.copy()
    kv2[:, 1] = kv2[3, 1]
    out = orc.sparse_attn(q, kv2, rows)
    for h in range(64):
        np.testing.assert_allclose(out[0, h], V[3, h // 16], rtol=1e-13)


def test_dense_causal_when_everything_fits(orc):
    """L <= topk: every visible position is selected and the step is dense causal
    attention (torch SDPA with a causal mask at the query positions)."""
    w = synth.make_workload("t", L=200, T=8, key_dtype="fp8", recipe="normal", seed=17)
    out, sel = orc.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, 2048)
    for t in range(8):
        n = w.pos[t] + 1
        assert sel[t, :n].tolist() == list(range(n)) and np.all(sel[t, n:] == -1)
    q = torch.from_numpy(synth.bf16_bits_to_f32(w.q).astype(np.float64))
    kv = torch.from_numpy(synth.bf16_bits_to_f32(w.kv).astype(np.float64))
    K, V = kv[:, 0].permute(1, 0, 2), kv[:, 1].permute(1, 0, 2)
    for t in range(8):
        mask = torch.arange(200) <= int(w.pos[t])
        ref = torch.nn.functional.scaled_dot_product_attention(q[t].reshape(4, 16, 128), K, V,
                                                               attn_mask=mask[None, None, :])
        np.testing.assert_allclose(out[t], ref.reshape(64, 128).numpy(), rtol=1e-11, atol=1e-12)


def test_decode_is_composition(orc):
    w = synth.make_workload("t", L=3000, T=2, key_dtype="bf16", recipe="normal", seed=3, topk=256)
    out, sel, sc = orc.decode(w.q, w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.kv, w.pos, 256, want_scores=True)
    sc2 = orc.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    assert np.array_equal(sc, sc2)
    sel2 = orc.topk(sc2, w.pos, 256)
    assert np.array_equal(sel, sel2)
    assert np.array_equal(sel, _brute_topk(sc2, w.pos, 256))
    assert np.array_equal(out, orc.sparse_attn(w.q, w.kv, sel2))


@pytest.mark.slow
def test_planted_margin_full_size(orc):
    """The 1M-context planted workload: every planted token outscores every
    background token by at least 2x, so the oracle selects exactly the planted set."""
    w = synth.config("verify_1m")
    s = orc.index_scores(w.q_idx, w.w_idx, w.k_idx, w.k_scale, w.pos)
    planted = np.zeros(w.L, bool)
    planted[w.planted] = True
    assert len(w.planted) == 2048
    assert w.planted.max() < w.pos.min()
    for t in range(w.T):
        background = ~planted & (np.arange(w.L) <= w.pos[t])
        assert s[t, planted].min() >= 2.0 * s[t, background].max()
    sel = orc.topk(s, w.pos, 2048)
    for t in range(w.T):
        assert np.array_equal(sel[t], w.planted)


@pytest.mark.parametrize("window,with_sink", [(128, False), (128, True), (1, False), (300, True)])
def test_window_attention_matches_band_mask(orc, window, with_sink):
    """Sliding-window attention equals dense attention under a band mask
    pos - window < s <= pos (torch, built here from the mask, not from the
    oracle's selection), with the sink as an extra zero-valued key."""
    rng = np.random.default_rng(50 + window)
    T, L = 3, 260
    q = synth.f32_to_bf16_bits(rng.standard_normal((T, 64, 128), dtype=np.float32))
    kv = synth.f32_to_bf16_bits(rng.standard_normal((L, 2, 4, 128), dtype=np.float32))
    pos = np.array([259, 100, 5], np.int32)
    sink = rng.standard_normal(64).astype(np.float32) if with_sink else None
    got = orc.swa_decode(q, kv, pos, window, sink=sink)
    qd = torch.from_numpy(synth.bf16_bits_to_f32(q).astype(np.float64))
    kd = torch.from_numpy(synth.bf16_bits_to_f32(kv).astype(np.float64))
    K, V = kd[:, 0].permute(1, 0, 2), kd[:, 1].permute(1, 0, 2)
    s = torch.arange(L)
    for t in range(T):
        mask = (s <= int(pos[t])) & (s > int(pos[t]) - window)
        z = torch.einsum("ghd,gld->ghl", qd[t].reshape(4, 16, 128), K) / math.sqrt(128)
        z = z.masked_fill(~mask[None, None, :], -math.inf)
        if sink is not None:
            z = torch.cat([z, torch.from_numpy(sink.astype(np.float64)).reshape(4, 16, 1)], dim=-1)
        p = torch.softmax(z, dim=-1)[..., :L]
        ref = torch.einsum("ghl,gld->ghd", p, V).reshape(64, 128).numpy()
        np.testing.assert_allclose(got[t], ref, rtol=1e-11, atol=1e-12)
    sel = orc.window_select(pos, window)
    n = min(6, window)   # query 2 sees positions 0..5
    assert sel[2, :n].tolist() == list(range(6 - n, 6)) and np.all(sel[2, n:] == -1)
