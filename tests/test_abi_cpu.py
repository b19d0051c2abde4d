"""Host-side checks of the C ABI library that need no GPU: it loads, it exports
every function include/neox_shard.h declares, its host arithmetic and its
argument validation (which runs before any CUDA call)."""
import ctypes
import os
import re

import pytest

from mixed_precision_zero_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fn in sorted(os.listdir(inc)):
        if not fn.endswith(".h"):
            continue
        text = open(os.path.join(inc, fn)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*[A-Za-z_][\w\s\*]*?\b(neox_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_library_exports_every_declared_function():
    names = declared_functions()
    assert "neox_shard_step" in names and "neox_shard_create" in names and len(names) >= 10
    L = ctypes.CDLL(_abi.LIB_PATH)
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_state_accounting_matches_page():
    """16 bytes per parameter: 175B parameters -> 2.8 TB, FP16 weights 350 GB."""
    facts = dict(ln.split() for ln in open(os.path.join(GOLDEN, "state_accounting.txt"))
                 if ln.strip() and not ln.startswith("#"))
    n = int(facts["params"])
    assert _abi.neox_model_state_bytes(n, _abi.NEOX_FP16, _abi.NEOX_FP16) == int(facts["state_bytes"])
    assert _abi.neox_model_state_bytes(n, _abi.NEOX_BF16, _abi.NEOX_BF16) == int(facts["state_bytes"])
    assert 2 * n == int(facts["fp16_weight_bytes"])


def test_status_strings():
    for s in range(5):
        assert _abi.neox_status_string(s)
    assert _abi.neox_status_string(99) == "unknown status"


def _desc(n=16, **kw):
    d = _abi.neox_shard_desc()
    d.numel = n
    d.wdtype = kw.get("wdtype", _abi.NEOX_FP16)
    d.gdtype = kw.get("gdtype", _abi.NEOX_FP16)
    d.master = kw.get("master", 4096)
    d.exp_avg = kw.get("exp_avg", 8192)
    d.exp_avg_sq = kw.get("exp_avg_sq", 12288)
    d.default_weight_decay = kw.get("wd", 0.1)
    d.max_grads = kw.get("max_grads", 1)
    d.flags = kw.get("flags", 0)
    return d


def _hp(**kw):
    base = dict(beta1=0.9, beta2=0.95, eps=1e-8, clip_norm=1.0, predivide=1.0, init_scale=65536.0,
                scale_factor=2.0, min_scale=1.0, scale_window=1000)
    base.update(kw)
    return _abi.neox_hparams(**base)


@pytest.mark.parametrize("desc_kw,hp_kw,why", [
    ({}, {"beta1": 1.0}, "beta1"),
    ({}, {"beta2": -0.1}, "beta2"),
    ({}, {"eps": float("nan")}, "eps"),
    ({}, {"predivide": 0.0}, "predivide"),
    ({}, {"init_scale": 0.0}, "init_scale"),
    ({}, {"scale_factor": 0.5}, "scale_factor"),
    ({}, {"min_scale": -1.0}, "min_scale"),
    ({}, {"scale_window": 0}, "scale_window"),
    ({}, {"hysteresis": -1}, "hysteresis"),
    ({}, {"optimizer": 2}, "optimizer"),
    ({"wdtype": 7}, {}, "dtype"),
    ({"master": 0}, {}, "non-NULL"),
    ({"exp_avg": 8194}, {}, "aligned"),
    ({"max_grads": 65}, {}, "max_grads"),
    ({"flags": 2}, {}, "flags"),
    ({"wd": float("inf")}, {}, "weight decay"),
])
def test_create_rejects_invalid_arguments_before_cuda(desc_kw, hp_kw, why):
    h = ctypes.c_void_p()
    st = _abi.lib().neox_shard_create(ctypes.byref(_desc(**desc_kw)), ctypes.byref(_hp(**hp_kw)), 0,
                                      ctypes.byref(h))
    assert st == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert h.value is None
    assert why in _abi.neox_last_error(None)


def test_create_rejects_bad_segment_tables():
    L = _abi.lib()
    for segs in ([(0, 8, 0.1), (9, 8, 0.1)], [(0, 8, 0.1), (8, 0, 0.1), (8, 8, 0.1)], [(0, 15, 0.1)],
                 [(1, 16, 0.1)]):
        arr = (_abi.neox_segment * len(segs))(*[_abi.neox_segment(*s) for s in segs])
        d = _desc(16)
        d.segs = ctypes.cast(arr, ctypes.POINTER(_abi.neox_segment))
        d.nsegs = len(segs)
        h = ctypes.c_void_p()
        assert L.neox_shard_create(ctypes.byref(d), ctypes.byref(_hp()), 0, ctypes.byref(h)) == \
            _abi.NEOX_ERR_INVALID_ARGUMENT
    for bad in (None,):
        assert L.neox_shard_create(None, ctypes.byref(_hp()), 0, ctypes.byref(ctypes.c_void_p())) == \
            _abi.NEOX_ERR_INVALID_ARGUMENT


def test_null_handle_calls():
    L = _abi.lib()
    assert L.neox_shard_step(None, None, 1, None, 1e-3, None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_shard_set_state(None, 1.0, 0, 0) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_shard_get_state(None, None, None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_shard_set_hparams(None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_shard_scratch_bytes(None) == 0
    assert L.neox_shard_get_hysteresis(None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_shard_set_hysteresis(None, 1) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_ipc_export(None, None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_ipc_open(None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert L.neox_ipc_close(None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    assert "non-NULL" in _abi.lib().neox_ipc_last_error().decode()
    L.neox_shard_destroy(None)


def test_multi_create_rejects_invalid_arguments_before_cuda():
    L = _abi.lib()
    h = ctypes.c_void_p()
    hp = _hp()
    grads = (ctypes.c_void_p * 1)(4096)
    good_t = _abi.neox_tensor(16, 0.1, 4096, 8192, 12288, 16384, ctypes.cast(grads, ctypes.POINTER(ctypes.c_void_p)))
    cases = [
        (_abi.neox_tensor_set(-1, 1, 0, 0, None), "ntensors"),
        (_abi.neox_tensor_set(1, 0, 0, 0, ctypes.pointer(good_t)), "num_grads"),
        (_abi.neox_tensor_set(1, 65, 0, 0, ctypes.pointer(good_t)), "num_grads"),
        (_abi.neox_tensor_set(1, 1, 5, 0, ctypes.pointer(good_t)), "dtype"),
        (_abi.neox_tensor_set(1, 1, 0, 0, ctypes.pointer(
            _abi.neox_tensor(16, 0.1, 4096, 8194, 12288, 16384, ctypes.cast(grads, ctypes.POINTER(ctypes.c_void_p))))),
         "aligned"),
        (_abi.neox_tensor_set(1, 1, 0, 0, ctypes.pointer(_abi.neox_tensor(16, 0.1, 4096, 8192, 12288, 16384, None))),
         "non-NULL"),
        (_abi.neox_tensor_set(1, 1, 0, 0, ctypes.pointer(
            _abi.neox_tensor(16, float("nan"), 4096, 8192, 12288, 16384,
                             ctypes.cast(grads, ctypes.POINTER(ctypes.c_void_p))))), "weight decay"),
    ]
    for tset, why in cases:
        assert L.neox_multi_create(ctypes.byref(tset), ctypes.byref(hp), 0, ctypes.byref(h)) == \
            _abi.NEOX_ERR_INVALID_ARGUMENT
        assert why in L.neox_multi_last_error(None).decode()
    assert L.neox_multi_step(None, 1e-3, None, None) == _abi.NEOX_ERR_INVALID_ARGUMENT
    L.neox_multi_destroy(None)


def test_noalloc_rejects_invalid_arguments_before_cuda():
    """The allocation-free step validates everything before its first CUDA
    call, so a caller learns of a bad argument without a device: a segment
    table beyond the static scratch's 1024 entries, a hysteresis count its
    caller-held scaler state cannot carry, K outside [1, 64], a bad scale.
    The caller's state is left as it was."""
    nseg = 1025
    segs = (_abi.neox_segment * nseg)(*[_abi.neox_segment(4 * i, 4, 0.1) for i in range(nseg)])
    fake = 0x100000  # never dereferenced: validation fails first

    def desc(n=4 * nseg, with_segs=True):
        return _abi.neox_shard_desc(n, _abi.NEOX_FP16, _abi.NEOX_FP16,
                                    ctypes.cast(segs, ctypes.POINTER(_abi.neox_segment)) if with_segs else None,
                                    nseg if with_segs else 0, 0.1, fake, fake, fake, 1)

    hp = _abi.neox_hparams(0.9, 0.95, 1e-8, 1.0, 1.0, 1024.0, 2.0, 1.0, 1000, 1, 0)
    hp_hyst = _abi.neox_hparams(0.9, 0.95, 1e-8, 1.0, 1.0, 1024.0, 2.0, 1.0, 1000, 2, 0)
    cases = [(desc(), hp, 1, 1024.0, "1024"),
             (desc(with_segs=False), hp_hyst, 1, 1024.0, "hysteresis"),
             (desc(with_segs=False), hp, 0, 1024.0, "num_grads"),
             (desc(with_segs=False), hp, 65, 1024.0, "num_grads"),
             (desc(with_segs=False), hp, 1, 0.0, "scale")]
    for d, h, k, scale, why in cases:
        state = _abi.neox_scaler_state(scale, 3, 7)
        with pytest.raises(_abi.NeoxError) as ei:
            _abi.neox_shard_step_noalloc(d, h, state, [fake] * k, fake, 1e-3, 0)
        assert ei.value.status == _abi.NEOX_ERR_INVALID_ARGUMENT and why in str(ei.value), (why, str(ei.value))
        assert (state.scale, state.good, state.t) == (scale, 3, 7)
