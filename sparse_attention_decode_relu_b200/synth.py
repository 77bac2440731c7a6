"""Seeded synthetic inputs for the DSA decode/verify step.

This module is shared by the CUDA path's tests and benchmark and by the CPU
oracle's tests.  It only *draws and encodes inputs*: it holds none of the
step's arithmetic (no indexer scores, no selection, no attention).  Both sides
receive the same bits.

Shapes follow the step described on the NaiveAI research page (naive.ai/en/research,
"Technical Details > Hybrid SWA-DSA Architecture": DSA selects the top 2,048 tokens,
GQA with four KV groups, a lightweight indexer with 16 query heads):

    q        [T][64][128]     bf16 bits (uint16)   backbone queries, 64 heads
    q_idx    [T][16][64]      bf16 bits (uint16)   indexer queries, 16 heads x 64
    w_idx    [T][16]          float32              indexer head weights
    k_idx    [L][64]          bf16 bits (uint16) or FP8-E4M3 codes (uint8)
    k_scale  [L]              float32 per-token scale (FP8 keys only)
    kv       [L][2][4][128]   bf16 bits: K plane (4 groups x 128), then V plane
    pos      [T]              int32, query t sees cached positions s <= pos[t]

Recipes ("indexer recipe"; K/V and q are always N(0,1) rounded to bf16):
    normal  : q_idx, k_idx ~ N(0,1); w ~ U(0,1); FP8 scale ~ U(0.5, 2)
    int     : q_idx, k_idx uniform integers in [-3, 3]; w uniform integers in
              {0..3}; FP8 scale uniform in {0.5, 1, 2}.  Every indexer score is
              then an exactly representable fp32 value, which makes the selected
              index set exactly reproducible.
    planted : 32 non-overlapping runs of 64 consecutive tokens whose keys are a
              shared direction u ~ N(0,1)^64 (FP8) with a large per-token scale;
              indexer queries are u + N(0, 0.5^2) per head and query.  The
              planted 2,048 tokens then outscore every background token.

Encodings: bf16 is float32 rounded to nearest-even on the upper 16 bits; FP8
E4M3 uses torch's float8_e4m3fn conversion after clipping to +-448 (torch does
not saturate).  Sub-streams of numpy's PCG64 are keyed by (seed, tensor id) so a
tensor's bits do not depend on which other tensors were drawn.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

H, G, D = 64, 4, 128          # backbone query heads, KV groups, head dim
HI, DI = 16, 64               # indexer heads, indexer dim
TOPK = 2048
ROW_ELEMS = 2 * G * D         # bf16 elements per cached token row (K then V)

_STREAM = {"q": 1, "q_idx": 2, "w": 3, "k_idx": 4, "scale": 5, "kv": 6, "plant": 7}


def _rng(seed: int, what: str) -> np.random.Generator:
    return np.random.default_rng([int(seed), _STREAM[what]])


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> float32 (exact widening)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    """Encode float32 as FP8-E4M3 codes (uint8), saturating at +-448."""
    import torch

    t = torch.from_numpy(np.clip(np.asarray(x, np.float32), -448.0, 448.0))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


@dataclasses.dataclass
class Workload:
    name: str
    L: int
    T: int
    key_dtype: str               # "bf16" | "fp8"
    recipe: str                  # "normal" | "int" | "planted"
    seed: int
    topk: int = TOPK
    q: np.ndarray = None
    q_idx: np.ndarray = None
    w_idx: np.ndarray = None
    k_idx: np.ndarray = None
    k_scale: Optional[np.ndarray] = None
    pos: np.ndarray = None
    planted: Optional[np.ndarray] = None   # planted positions (sorted), planted recipe only
    _kv: Optional[np.ndarray] = None

    @property
    def kv(self) -> np.ndarray:
        """[L][2][4][128] bf16 bits, drawn on first use (2 GiB at L = 2^20)."""
        if self._kv is None:
            self._kv = make_kv(self.L, self.seed)
        return self._kv

    def key_bytes_per_token(self) -> int:
        return DI * 2 if self.key_dtype == "bf16" else DI + 4


def make_kv(L: int, seed: int, chunk: int = 1 << 16) -> np.ndarray:
    rng = _rng(seed, "kv")
    out = np.empty((L, 2, G, D), dtype=np.uint16)
    flat = out.reshape(L, ROW_ELEMS)
    for s0 in range(0, L, chunk):
        s1 = min(L, s0 + chunk)
        flat[s0:s1] = f32_to_bf16_bits(rng.standard_normal((s1 - s0, ROW_ELEMS), dtype=np.float32))
    return out


def _planted_starts(L: int, rng: np.random.Generator, runs: int = 32, run_len: int = 64, T: int = 8):
    """32 non-overlapping run starts in [0, L - T - run_len], one per stratum."""
    hi = L - T - run_len
    width = (hi + 1) // runs
    if width < run_len:
        raise ValueError("context too short for planted runs")
    starts = np.array([i * width + int(rng.integers(0, width - run_len + 1)) for i in range(runs)], dtype=np.int64)
    return starts


def make_workload(name: str, L: int, T: int, key_dtype: str, recipe: str, seed: int,
                  topk: int = TOPK, pos: Optional[np.ndarray] = None,
                  plant_amplitude: float = 8.0) -> Workload:
    if key_dtype not in ("bf16", "fp8"):
        raise ValueError(key_dtype)
    if recipe not in ("normal", "int", "planted"):
        raise ValueError(recipe)
    if recipe == "planted" and key_dtype != "fp8":
        raise ValueError("the planted recipe carries its amplitude in the FP8 per-token scale")
    if pos is None:
        pos = np.arange(L - T, L, dtype=np.int32)
    pos = np.asarray(pos, dtype=np.int32)
    assert pos.shape == (T,)

    q = f32_to_bf16_bits(_rng(seed, "q").standard_normal((T, H, D), dtype=np.float32))
    r_qi, r_w, r_k, r_s = (_rng(seed, x) for x in ("q_idx", "w", "k_idx", "scale"))
    planted = None
    if recipe == "int":
        q_idx_f = r_qi.integers(-3, 4, size=(T, HI, DI)).astype(np.float32)
        w = r_w.integers(0, 4, size=(T, HI)).astype(np.float32)
        k_f = r_k.integers(-3, 4, size=(L, DI)).astype(np.float32)
        scale = np.array([0.5, 1.0, 2.0], np.float32)[r_s.integers(0, 3, size=L)]
    else:
        q_idx_f = r_qi.standard_normal((T, HI, DI), dtype=np.float32)
        w = r_w.random((T, HI), dtype=np.float32)
        k_f = r_k.standard_normal((L, DI), dtype=np.float32)
        scale = (0.5 + 1.5 * r_s.random(L, dtype=np.float32)).astype(np.float32)
        if recipe == "planted":
            rp = _rng(seed, "plant")
            u = rp.standard_normal(DI, dtype=np.float32)
            u = bf16_bits_to_f32(f32_to_bf16_bits(u))
            starts = _planted_starts(L, rp, T=T)
            planted = (starts[:, None] + np.arange(64)[None, :]).reshape(-1)
            k_f[planted] = u[None, :]
            scale[planted] = np.float32(plant_amplitude)
            q_idx_f = u[None, None, :] + 0.5 * q_idx_f
    q_idx = f32_to_bf16_bits(q_idx_f)
    if key_dtype == "bf16":
        k_idx = f32_to_bf16_bits(k_f)
        k_scale = None
    else:
        k_idx = f32_to_e4m3_codes(k_f)
        k_scale = scale.astype(np.float32)
    return Workload(name=name, L=L, T=T, key_dtype=key_dtype, recipe=recipe, seed=seed, topk=topk,
                    q=q, q_idx=q_idx, w_idx=w.astype(np.float32), k_idx=k_idx, k_scale=k_scale,
                    pos=pos, planted=None if planted is None else np.sort(planted))


# Named workloads: the four fixed configurations and the context sweep, each with
# an integer twin (same shapes, integer recipe) used for exact-selection checks.
_BASE = {
    "tiny_decode": dict(L=4096, T=1, key_dtype="bf16", recipe="int", seed=0),
    "verify_block": dict(L=32768, T=8, key_dtype="bf16", recipe="normal", seed=1),
    "long_decode": dict(L=131072, T=1, key_dtype="fp8", recipe="normal", seed=2),
    "verify_1m": dict(L=1 << 20, T=8, key_dtype="fp8", recipe="planted", seed=3),
}
_seed = 10
for _L in (200, 2200, 16384, 262144):
    for _T in (1, 8):
        _BASE[f"sweep_L{_L}_T{_T}"] = dict(L=_L, T=_T, key_dtype="fp8", recipe="normal", seed=_seed)
        _seed += 1

CONFIGS = dict(_BASE)
for _n, _c in _BASE.items():
    if _c["recipe"] != "int":
        CONFIGS[_n + "_int"] = dict(_c, recipe="int")


def config(name: str, **overrides) -> Workload:
    c = dict(CONFIGS[name])
    c.update(overrides)
    return make_workload(name, **c)
