"""The C ABI library loads, exports every symbol include/msa.h declares, and rejects bad
arguments on the host before touching the GPU (these tests run without a GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

from top_document_sparse_b200 import msa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(msa_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_four_calls_of_the_path():
    names = header_functions()
    for n in ("msa_encode_memory", "msa_route", "msa_sparse_attend", "msa_step"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = msa.lib()
    for name in header_functions():
        assert hasattr(lib, name), name


def test_binding_signatures_cover_the_header():
    assert set(header_functions()) == set(msa.SIGNATURES)


def test_exported_symbols_are_only_the_abi():
    out = os.popen(f"nm -D --defined-only {msa._build.LIB}").read()
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert exported == set(header_functions())


def test_status_strings_and_version():
    lib = msa.lib()
    assert lib.msa_status_string(0) == b"ok"
    assert lib.msa_status_string(1) == b"invalid argument"
    assert lib.msa_version() >= 10000


def _cfg(**kw):
    off = np.asarray(kw.pop("offsets", [0, 100, 228]), dtype=np.int64)
    base = dict(n_docs=off.size - 1, chunk_len=64, n_kv_heads=2, head_dim=64, n_router_heads=8,
                router_dim=128, dtype=msa.MSA_F32, rope_theta=1e6, max_local_position=1024)
    base.update(kw)
    c = msa.MemoryConfig(**{k: v for k, v in base.items()})
    c.doc_token_offsets = off.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    return c, off


@pytest.mark.parametrize("kw,status", [
    (dict(offsets=[0, 10, 10]), 1),        # empty document
    (dict(offsets=[5, 10]), 1),            # offsets[0] != 0
    (dict(chunk_len=1), 2),
    (dict(chunk_len=65), 2),
    (dict(head_dim=96), 2),
    (dict(router_dim=96), 2),
    (dict(n_router_heads=1, router_dim=32), 2),  # width 32 is not a multiple of 64
    (dict(dtype=7), 1),
    (dict(rope_theta=0.5), 1),
    (dict(max_local_position=0), 1),
])
def test_memory_create_rejects_bad_configs_without_a_gpu(kw, status):
    cfg, _keep = _cfg(**kw)
    h = ctypes.c_void_p()
    st = msa.lib().msa_memory_create(ctypes.byref(cfg), ctypes.byref(h))
    assert st == status
    assert not h.value
    assert msa.lib().msa_last_error()


def test_calls_reject_null_handles():
    lib = msa.lib()
    assert lib.msa_memory_destroy(None) == 1
    assert lib.msa_route(None, None, None, 1, 1, 1, None, None, None, None, None, 0, None) == 1
    assert lib.msa_sparse_attend(None, None, None, 1, 1, 1, 8, None, None, None, None, None, None,
                                 8, 0, None, None, 0, None) == 1
    assert lib.msa_encode_memory(None, 0, 1, None, None, None, None, None, None, None) == 1
    assert lib.msa_step(None, None, None, None, None, None, None, None, None, None) == 1
    assert lib.msa_route_workspace_size(None, 1, 1, 1) == 0
    assert lib.msa_device_error(None, None) == 1


def test_adaptive_interleave_validates_before_touching_the_gpu():
    """msa_interleave_adaptive rejects a null n_rounds and a NaN stop score (INVALID_ARG, with a
    message) before any CUDA call, so these checks run on a machine without a GPU."""
    import ctypes
    lib = msa.lib()
    n = ctypes.c_int32(0)
    assert lib.msa_interleave_adaptive(None, None, None, 1, 1, 1, 1, 0.5, None, None, None, None,
                                       None, None, 0, None) == 1
    assert b"n_rounds" in lib.msa_last_error()
    assert lib.msa_interleave_adaptive(None, None, None, 1, 1, 1, 1, float("nan"), None, None,
                                       None, None, ctypes.addressof(n), None, 0, None) == 1
    assert b"NaN" in lib.msa_last_error()
    assert lib.msa_interleave_adaptive(None, None, None, 1, 1, 1, 1, float("-inf"), None, None,
                                       None, None, ctypes.addressof(n), None, 0, None) == 1
    assert b"null" in lib.msa_last_error()
    assert lib.msa_interleave(None, None, None, 1, 1, 1, 1, None, None, None, None, None, 0,
                              None) == 1
