"""The C ABI library loads on a CPU-only host, exports every entry point
declared in include/tq.h, and validates arguments on the host before any
device work (no compute calls here)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ["tq_create", "tq_destroy", "tq_encode_kv", "tq_attention_scores", "tq_decode_attention",
              "tq_dequantize", "tq_packed_bytes", "tq_get_status"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    import kv_cache_vector_10_b200 as tq
    out = subprocess.check_output(["nm", "-D", "--defined-only", tq.LIB_PATH]).decode()
    exported = set(l.split()[-1] for l in out.splitlines() if " T " in l)
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        assert hasattr(tq.lib, n)
    assert set(tq.EXPORTED) == set(_declared())


def test_create_validates_arguments_on_host():
    import kv_cache_vector_10_b200 as tq
    lib = tq.lib
    out = ctypes.c_void_p()
    cases = [((0, 3, 128, 42), "TQ_ERR_ZERO_DIM"), ((96, 3, 128, 42), "TQ_ERR_DIM"),
             ((130, 3, 128, 42), "TQ_ERR_DIM"), ((128, 1, 128, 42), "TQ_ERR_BITS"),
             ((128, 6, 128, 42), "TQ_ERR_BITS"), ((128, 3, 0, 42), "TQ_ERR_ZERO_PROJ"),
             ((128, 3, 48, 42), "TQ_ERR_PROJ"), ((128, 3, 512, 42), "TQ_ERR_PROJ"),
             ((512, 3, 128, 42), "TQ_ERR_DIM"), ((256, 3, 224, 42), "TQ_ERR_PROJ"),
             ((256, 3, 256, 42), "TQ_ERR_PROJ")]
    for args, want in cases:
        code = lib.tq_create(*args, ctypes.byref(out))
        assert lib.tq_status_string(code).decode() == want, (args, code)
        assert out.value is None
    assert lib.tq_create(128, 3, 128, 42, None) != 0
    # head_dim 256 runs the Walsh-Hadamard rotation only (the Haar operands
    # do not fit in a CTA's shared memory)
    code = lib.tq_create_ex(256, 3, 128, 42, tq.TQ_ROT_HAAR, ctypes.byref(out))
    assert lib.tq_status_string(code).decode() == "TQ_ERR_DIM" and out.value is None


def test_null_and_empty_arguments():
    import kv_cache_vector_10_b200 as tq
    lib = tq.lib
    assert lib.tq_row_bytes(None, tq.TQ_KEYS) == 0
    assert lib.tq_packed_bytes(None, 1, 1, 16, tq.TQ_BOTH) == 0
    assert tq.STATUS_NAMES[lib.tq_encode_kv(None, None, None, 0, 1, 1, 1, 0, 0, 128, None, 0, None)] == "TQ_ERR_NULL"
    assert tq.STATUS_NAMES[lib.tq_ensure_heads(None, 4)] == "TQ_ERR_NULL"
    assert tq.STATUS_NAMES[lib.tq_get_status(None, None, None, None)] == "TQ_ERR_NULL"
    assert tq.STATUS_NAMES[lib.tq_decode_attention(None, 1, None, 0, 1, 1, 1, None, 0, None, 0, None)] == "TQ_ERR_NULL"
    assert lib.tq_decode_workspace_bytes(None, 1, 1, 1, 1) == 0
    lib.tq_destroy(None)
    for code, name in tq.STATUS_NAMES.items():
        assert lib.tq_status_string(code).decode() == name


def test_no_cpu_fallback_without_a_gpu():
    """On a host without an sm_100 device, creation fails loudly."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    import kv_cache_vector_10_b200 as tq
    with pytest.raises(tq.TQError):
        tq.tq_create(128, 3, 128, 42)
