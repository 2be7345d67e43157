"""The C-ABI library on a machine without a GPU: it loads, it exports every
entry point include/saga.h declares, and argument validation rejects bad
calls before anything touches CUDA."""
import ctypes
import os
import re

import pytest

from long_context_decoding_saga_b200 import build as build_mod
from long_context_decoding_saga_b200 import saga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return saga.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "saga.h")).read()
    return sorted(set(re.findall(r"SAGA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declares_the_binding_names():
    assert set(declared_symbols()) == set(saga.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.saga_abi_version() == 102


def _shape(**kw):
    base = dict(batch=1, h_q=8, h_k=1, h_v=8, d=64, l_cap=1024)
    base.update(kw)
    return saga.SagaShape.of(**base)


FAKE = ctypes.c_void_p(0x100000)  # never dereferenced: validation fails first


def _decode(lib, shape, seq_len=10, n_top=4, R=2, step=0, out_dtype=0, ptrs=True, sel_idx=None, sel_count=None):
    p = FAKE if ptrs else None
    return lib.saga_decode_attn(ctypes.byref(shape), p, p, p, seq_len, None, n_top, R, step, p, p, out_dtype,
                                sel_count, sel_idx, p, 1 << 30, None)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), saga.SAGA_ERR_UNSUPPORTED),
    (dict(h_q=6, h_k=4), saga.SAGA_ERR_ARG),
    (dict(h_q=8, h_v=3), saga.SAGA_ERR_ARG),
    (dict(h_q=12, h_k=3, h_v=2), saga.SAGA_ERR_UNSUPPORTED),
    (dict(h_q=128, h_k=1), saga.SAGA_ERR_UNSUPPORTED),
    (dict(batch=0), saga.SAGA_ERR_ARG),
    (dict(l_cap=0), saga.SAGA_ERR_ARG),
])
def test_bad_shapes_rejected(lib, kw, code):
    s = _shape(**kw)
    assert _decode(lib, s) == code
    assert lib.saga_last_error()
    assert lib.saga_workspace_bytes(ctypes.byref(s)) == 0


@pytest.mark.parametrize("kw", [dict(seq_len=0), dict(seq_len=1025), dict(n_top=0), dict(R=0), dict(step=-1),
                                dict(out_dtype=7), dict(ptrs=False), dict(sel_idx=FAKE)])
def test_bad_arguments_rejected(lib, kw):
    assert _decode(lib, _shape(), **kw) == saga.SAGA_ERR_ARG
    assert lib.saga_last_error()


def test_append_and_select_validation(lib):
    s = _shape()
    assert lib.saga_kv_append(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, 1024, None, None) == saga.SAGA_ERR_ARG
    assert lib.saga_kv_append(ctypes.byref(s), None, FAKE, FAKE, FAKE, 0, None, None) == saga.SAGA_ERR_ARG
    assert lib.atopn_select_threshold(FAKE, 4, 10, 6, 3, FAKE, FAKE, 256, None) == saga.SAGA_ERR_ARG
    assert lib.atopn_select_threshold(FAKE, 4, 10, 12, 0, FAKE, FAKE, 256, None) == saga.SAGA_ERR_ARG
    assert lib.atopn_select_threshold(FAKE, 4, 10, 12, 3, FAKE, None, 0, None) == saga.SAGA_ERR_WORKSPACE
    assert lib.atopn_refresh_threshold(ctypes.byref(s), FAKE, FAKE, 5, None, 0, FAKE, FAKE, 1, None) == saga.SAGA_ERR_ARG


def test_binding_refuses_cpu_tensors(lib):
    import torch
    s = _shape()
    with pytest.raises(ValueError):
        saga.saga_kv_append(s, torch.zeros(1, 1, 1024, 64, dtype=torch.bfloat16),
                            torch.zeros(1, 8, 1024, 64, dtype=torch.bfloat16),
                            torch.zeros(1, 1, 64, dtype=torch.bfloat16), torch.zeros(1, 8, 64, dtype=torch.bfloat16), 0)


def _step(lib, shape, k_new=FAKE, v_new=FAKE, seq_len=10):
    p = FAKE
    return lib.saga_decode_step(ctypes.byref(shape), p, k_new, v_new, p, p, seq_len, None, 4, 2, 0, p, p, 0, None,
                                None, p, 1 << 30, None)


def test_decode_step_validation(lib):
    s = _shape()
    assert _step(lib, s, k_new=None) == saga.SAGA_ERR_ARG
    assert _step(lib, s, v_new=None) == saga.SAGA_ERR_ARG
    assert _step(lib, s, k_new=ctypes.c_void_p(0x100008)) == saga.SAGA_ERR_ARG  # not 16-byte aligned
    assert _step(lib, s, seq_len=0) == saga.SAGA_ERR_ARG
    assert _step(lib, _shape(d=96)) == saga.SAGA_ERR_UNSUPPORTED
    assert lib.saga_last_error()


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), saga.SAGA_ERR_UNSUPPORTED),
    (dict(h_k=3, h_q=6), saga.SAGA_ERR_UNSUPPORTED),
    (dict(h_k=18, h_q=36), saga.SAGA_ERR_UNSUPPORTED),
    (dict(h_q=10, h_k=4), saga.SAGA_ERR_ARG),
    (dict(tokens=0), saga.SAGA_ERR_ARG),
    (dict(hidden=0), saga.SAGA_ERR_ARG),
    (dict(h_k=0), saga.SAGA_ERR_ARG),
])
def test_merge_rejects_bad_shapes(lib, kw, code):
    base = dict(tokens=128, hidden=256, d=64, h_q=8, h_k=4)
    base.update(kw)
    s = saga.SagaMergeShape(base["tokens"], base["hidden"], base["d"], base["h_q"], base["h_k"])
    assert lib.saga_merge_workspace_bytes(ctypes.byref(s)) == 0
    rc = lib.saga_key_head_merge(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None)
    assert rc == code
    assert lib.saga_merge_last_error()


def test_merge_rejects_null_and_misaligned(lib):
    s = saga.SagaMergeShape(128, 256, 64, 8, 4)
    odd = ctypes.c_void_p(0x100008)
    assert lib.saga_key_head_merge(ctypes.byref(s), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                   None) == saga.SAGA_ERR_ARG
    assert lib.saga_key_head_merge(ctypes.byref(s), odd, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                                   None) == saga.SAGA_ERR_ARG
    assert lib.saga_key_head_merge(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1 << 30,
                                   None) == saga.SAGA_ERR_WORKSPACE


WS = ctypes.c_void_p(0x100000)  # 256-byte aligned, never dereferenced


def _qkv(lib, shape, hidden=256, x=FAKE, pos=0, ws=WS):
    return lib.saga_qkv_project(ctypes.byref(shape), hidden, x, FAKE, FAKE, FAKE, FAKE, pos, None, ws, 1 << 30, None)


def test_qkv_projection_validation(lib):
    s = _shape()
    assert _qkv(lib, _shape(batch=17)) == saga.SAGA_ERR_UNSUPPORTED
    assert _qkv(lib, s, hidden=0) == saga.SAGA_ERR_ARG
    assert _qkv(lib, s, hidden=100) == saga.SAGA_ERR_ARG  # not a multiple of 8
    assert _qkv(lib, s, x=None) == saga.SAGA_ERR_ARG
    assert _qkv(lib, s, x=ctypes.c_void_p(0x100008)) == saga.SAGA_ERR_ARG  # not 16-byte aligned
    assert _qkv(lib, s, pos=1024) == saga.SAGA_ERR_ARG
    assert _qkv(lib, s, pos=-1) == saga.SAGA_ERR_ARG
    assert _qkv(lib, _shape(d=96)) == saga.SAGA_ERR_UNSUPPORTED
    assert _qkv(lib, _shape(h_q=4096, h_k=64, h_v=64, d=128), hidden=1 << 16) == saga.SAGA_ERR_UNSUPPORTED
    assert _qkv(lib, s, ws=None) == saga.SAGA_ERR_WORKSPACE
    assert _qkv(lib, s, ws=ctypes.c_void_p(0x100010)) == saga.SAGA_ERR_WORKSPACE  # not 256-byte aligned
    assert lib.saga_qkv_workspace_bytes(ctypes.byref(_shape(batch=17)), 256) == 0
    assert lib.saga_qkv_workspace_bytes(ctypes.byref(s), 12) == 0
    assert lib.saga_qkv_workspace_bytes(ctypes.byref(s), 16384) == 256
    assert _qkv(lib, s, hidden=16392) == saga.SAGA_ERR_UNSUPPORTED
    assert lib.saga_last_error()
