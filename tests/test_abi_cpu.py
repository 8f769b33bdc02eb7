"""The C-ABI library loads and exports what include/dory.h declares; host-side
validation returns the documented codes (no GPU needed, no kernel runs)."""
import ctypes
import os
import re

import pytest

from looped_ngpt_b200 import _lib
from synthetic import TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "dory.h")) as f:
        txt = f.read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dory_[a-z_0-9]+)\s*\(", txt)))


def test_exports_every_declared_symbol():
    lib = _lib.load()
    names = _declared()
    assert len(names) >= 13
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES)


def test_strerror_names_codes():
    lib = _lib.load()
    assert lib.dory_strerror(0) == b"ok"
    assert b"cache" in lib.dory_strerror(-3)
    assert lib.dory_strerror(-99) == b"unknown error"


def _cfg(shape, **over):
    lt = (ctypes.c_uint8 * shape.n_blocks)(*shape.layer_types)
    vals = dict(d=shape.d, n_q_heads=shape.n_q_heads,
                n_kv_heads=shape.n_kv_heads, head_dim=shape.head_dim,
                ffn=shape.ffn, vocab=shape.vocab, n_in_blocks=shape.n_in,
                n_rec_blocks=shape.n_rec, n_out_blocks=shape.n_out,
                layer_types=lt, swa_window=shape.swa_window,
                rope_theta_swa=shape.rope_theta_swa,
                rope_theta_full=shape.rope_theta_full, wfmt=0)
    vals.update(over)
    return _lib.DoryConfig(**vals), lt


@pytest.mark.parametrize("over,code", [
    (dict(n_q_heads=3, n_kv_heads=2), -1),   # Hq % Hkv != 0
    (dict(head_dim=96), -2),
    (dict(wfmt=7), -2),                      # unknown weight format
    (dict(d=300), -2),
    (dict(n_rec_blocks=0), -1),
    (dict(swa_window=0), -1),
])
def test_init_rejects_bad_config(over, code):
    lib = _lib.load()
    cfg, _keep = _cfg(TINY, **over)
    h = ctypes.c_void_p()
    assert lib.dory_init_weights(ctypes.byref(cfg), None, 0,
                                 ctypes.byref(h)) == code
    assert not h.value


def test_init_rejects_missing_or_misaligned_tensor():
    lib = _lib.load()
    cfg, _keep = _cfg(TINY)
    h = ctypes.c_void_p()
    arr = (_lib.DoryTensor * 1)(_lib.DoryTensor(b"embed", 0x1000, 8))
    assert lib.dory_init_weights(ctypes.byref(cfg), arr, 1, ctypes.byref(h)) == -1
    arr = (_lib.DoryTensor * 1)(_lib.DoryTensor(b"embed", 0x1001, 8))
    assert lib.dory_init_weights(ctypes.byref(cfg), arr, 1, ctypes.byref(h)) == -1
    assert lib.dory_init_weights(None, None, 0, ctypes.byref(h)) == -1


def test_null_handles_rejected():
    lib = _lib.load()
    n = ctypes.c_int64()
    assert lib.dory_kv_cache_bytes(None, 1, 8, 1, 1, 1, ctypes.byref(n)) == -1
    assert lib.dory_workspace_bytes(None, 1, 1, ctypes.byref(n)) == -1
    assert lib.dory_prefill(None, None, None, 1, 1, 1, 1, 0, None, None, None,
                            0, None) == -1
    assert lib.dory_decode_step(None, None, None, 1, 1, 1, None, None, None,
                                0, None) == -1
    assert lib.dory_sync_status(None, None) == -1


def test_debug_gemm_arguments_validated_before_any_launch():
    """Bad shapes and pointers are rejected by the host checks alone (no
    device work), for the plain and the K-split debug GEMM."""
    lib = _lib.load()
    n = ctypes.c_int(0)
    p = ctypes.c_void_p(0x1000)
    # null operands, K not a multiple of 64, lda < K, no split slabs
    assert lib.dory_debug_gemm_bf16(None, 64, p, p, 1, 1, 64, None) == -1
    assert lib.dory_debug_gemm_bf16(p, 96, p, p, 1, 1, 96, None) == -1
    assert lib.dory_debug_gemm_bf16(p, 32, p, p, 1, 1, 64, None) == -1
    assert lib.dory_debug_gemm_bf16_split(p, 64, p, p, 1, 1, 64, 0,
                                          ctypes.byref(n), None) == -1
    assert lib.dory_debug_gemm_bf16_split(p, 64, p, p, 1, 1, 64, 4, None,
                                          None) == -1
    assert lib.dory_debug_gemm_bf16_split(p, 64, p, p, 0, 1, 64, 4,
                                          ctypes.byref(n), None) == -1
    assert n.value == 0


def test_debug_gemm_unbuildable_descriptor_is_an_error():
    """An operand the TMA descriptor cannot describe (a base address that is
    not 16-byte aligned) makes the launcher enqueue nothing; the entry point
    must report DORY_ERR_CUDA, never DORY_OK.  The A descriptor is built
    first and fails, so no kernel is launched on any machine."""
    lib = _lib.load()
    n = ctypes.c_int(0)
    bad = ctypes.c_void_p(0x1002)
    p = ctypes.c_void_p(0x1000)
    assert lib.dory_debug_gemm_bf16(bad, 64, p, p, 1, 128, 64, None) == -4
    assert lib.dory_debug_gemm_bf16_split(bad, 64, p, p, 1, 128, 64, 4,
                                          ctypes.byref(n), None) == -4
    assert n.value == 0
