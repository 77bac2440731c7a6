"""Host-side checks of the C ABI: the library builds, loads and exports every
entry point include/dsa_decode.h declares, and argument validation rejects bad
input before any CUDA call (so these run without a GPU)."""
import ctypes
import os
import re

import pytest

from sparse_attention_decode_relu_b200 import build, dsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa_decode.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", text)))


def test_header_declares_the_step_and_stages():
    names = declared_symbols()
    for n in ("dsa_decode", "dsa_decode_ws", "dsa_workspace_bytes", "dsa_index_scores", "dsa_topk_from_scores",
              "dsa_sparse_attn", "dsa_device_status", "dsa_status_str", "dsa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(build.build())
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_only_declared_symbols_are_exported():
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", build.build()], capture_output=True, text=True, check=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if " T " in l)
    assert exported == declared_symbols()


def test_workspace_bytes():
    L = dsa.lib()
    assert L.dsa_workspace_bytes(0, 100, 16) == 0
    assert L.dsa_workspace_bytes(9, 100, 16) == 0
    assert L.dsa_workspace_bytes(1, 100, 0) == 0
    assert L.dsa_workspace_bytes(1, 100, 2049) == 0
    a = L.dsa_workspace_bytes(1, 4096, 2048)
    b = L.dsa_workspace_bytes(8, 1 << 20, 2048)
    assert 0 < a < b and a % 256 == 0 and b % 256 == 0
    # scores + candidates dominate: at least 12 bytes per (query, position)
    assert b >= 12 * 8 * (1 << 20)


def _t(ptr, dtype, shape, stride=None, scale=None):
    d = dsa.dsa_tensor_t()
    d.data = ptr
    d.dtype = dtype
    d.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for s in reversed(shape):
            stride.insert(0, acc)
            acc *= s
    for i, (s, st) in enumerate(zip(shape, stride)):
        d.shape[i] = s
        d.stride[i] = st
    d.scale = scale
    return d


def _args(T=2, L=5000, topk=2048, k_dtype=dsa.BF16, pos=None, q_shape=None, kv_stride=None, k_stride=None,
          base=0x10000):
    q = _t(base, dsa.BF16, q_shape or (T, 64, 128))
    qi = _t(base, dsa.BF16, (T, 16, 64))
    w = _t(base, dsa.F32, (T, 16))
    k = _t(base, k_dtype, (L, 64), k_stride)
    kv = _t(base, dsa.BF16, (L, 2, 4, 128), kv_stride)
    out = _t(base, dsa.BF16, (T, 64, 128))
    sel = _t(base, dsa.I32, (T, topk))
    p = pos if pos is not None else [L - T + i for i in range(T)]
    return q, qi, w, k, kv, (ctypes.c_int32 * len(p))(*p), topk, out, sel


def _call(*a):
    L = dsa.lib()
    q, qi, w, k, kv, pos, topk, out, sel = a
    r = ctypes.byref
    st = L.dsa_decode_ws(r(q), r(qi), r(w), r(k), r(kv), pos, topk, r(out), r(sel), None, 0x100000, 1 << 40)
    return st, L.dsa_last_error().decode()


@pytest.mark.parametrize("kw,expect,msg", [
    (dict(T=9), dsa.ERR_UNSUPPORTED, "T = 9"),
    (dict(topk=0), dsa.ERR_INVALID_ARG, "topk"),
    (dict(topk=4096), dsa.ERR_INVALID_ARG, "topk"),
    (dict(pos=[4999, 5000]), dsa.ERR_INVALID_ARG, "pos[1]"),
    (dict(pos=[-1, 3]), dsa.ERR_INVALID_ARG, "pos[0]"),
    (dict(k_dtype=dsa.F32), dsa.ERR_INVALID_ARG, "k_idx_cache"),
    (dict(q_shape=(2, 32, 128)), dsa.ERR_UNSUPPORTED, "q"),
    (dict(kv_stride=(1000, 512, 128, 1)), dsa.ERR_INVALID_ARG, "kv_cache"),
    (dict(k_stride=(70, 1)), dsa.ERR_INVALID_ARG, "row stride"),
    (dict(base=0x10008), dsa.ERR_INVALID_ARG, "aligned"),
])
def test_validation_rejects_before_launch(kw, expect, msg):
    st, err = _call(*_args(**kw))
    assert st == expect, err
    assert msg in err


def test_validation_null_and_mismatch():
    a = list(_args())
    a[4] = _t(0x10000, dsa.BF16, (4000, 2, 4, 128))   # kv L differs from key-cache L
    st, err = _call(*a)
    assert st == dsa.ERR_INVALID_ARG and "kv_cache" in err
    a = list(_args())
    a[0] = _t(0, dsa.BF16, (2, 64, 128))
    st, err = _call(*a)
    assert st == dsa.ERR_INVALID_ARG and "null" in err
    L = dsa.lib()
    assert L.dsa_status_str(4) == b"device-side anomaly"


def test_new_entry_points_validate_before_launch():
    """Sliding-window decode, the step with a sink and the step with device
    positions reject bad arguments on the host, before any launch."""
    L = dsa.lib()
    r = ctypes.byref
    q, qi, w, k, kv, pos, topk, out, sel = _args()
    # sliding-window decode: window outside [1, 2048]
    for bad in (0, 2049):
        st = L.dsa_swa_decode(r(q), r(kv), pos, bad, None, r(out), None, 0x100000, 1 << 40)
        assert st == dsa.ERR_INVALID_ARG and "window" in L.dsa_last_error().decode()
    # sliding-window decode: a sink that is not 16-byte aligned
    st = L.dsa_swa_decode(r(q), r(kv), pos, 128, 0x10004, r(out), None, 0x100000, 1 << 40)
    assert st == dsa.ERR_INVALID_ARG and "sink" in L.dsa_last_error().decode()
    # the step with a sink: the sink is required
    st = L.dsa_decode_sink_ws(r(q), r(qi), r(w), r(k), r(kv), pos, topk, None, r(out), r(sel), None, 0x100000,
                              1 << 40)
    assert st == dsa.ERR_INVALID_ARG and "sink" in L.dsa_last_error().decode()
    # the step with device positions: null or misaligned position array
    st = L.dsa_decode_devpos_ws(r(q), r(qi), r(w), r(k), r(kv), None, topk, None, r(out), r(sel), None, 0x100000,
                                1 << 40)
    assert st == dsa.ERR_INVALID_ARG and "pos_device" in L.dsa_last_error().decode()
    st = L.dsa_decode_devpos_ws(r(q), r(qi), r(w), r(k), r(kv), 0x10002, topk, None, r(out), r(sel), None,
                                0x100000, 1 << 40)
    assert st == dsa.ERR_INVALID_ARG and "pos_device" in L.dsa_last_error().decode()
    # ... and the other arguments are still checked (topk out of range)
    st = L.dsa_decode_devpos_ws(r(q), r(qi), r(w), r(k), r(kv), 0x10000, 4096, None, r(out), r(sel), None, 0x100000,
                                1 << 40)
    assert st == dsa.ERR_INVALID_ARG and "topk" in L.dsa_last_error().decode()


def test_barrier_fault_hook_validates_its_limit():
    L = dsa.lib()
    for bad in (0, 999, 2_000_000_001, -5):
        assert L.dsa_debug_fail_next_barriers(bad) == dsa.ERR_INVALID_ARG
    assert b"limit_cycles" in L.dsa_last_error()
