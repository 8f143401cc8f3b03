"""The C ABI library loads without a GPU, exports every symbol of include/dsa.h, and validates
arguments on the host (these calls return before touching CUDA)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dsa():
    from sparse_attention_long_indexer_b200.build import build
    build()
    import sparse_attention_long_indexer_b200 as m
    return m


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(dsa):
    lib = ctypes.CDLL(dsa.LIBRARY_PATH)
    names = _declared()
    assert set(names) == set(dsa.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings_and_version(dsa):
    for code in range(7):
        assert dsa.dsa_status_string(code) and dsa.dsa_status_string(code) != "unknown status"
    assert dsa.dsa_status_string(99) == "unknown status"
    assert dsa.dsa_version() >= 100


def test_workspace_bytes(dsa):
    prod = dsa.make_dims(1, 4096, 4096)
    n = dsa.dsa_workspace_bytes(prod, 2048)
    assert n >= 4096 * 2048 * 4 and n % 256 == 0
    # decode rows up to 131072 keys keep every key's score (4 B); longer rows keep a top-k list
    # of (key, position) pairs per 8192-key chunk
    dec = dsa.make_dims(64, 1, 131072)
    assert dsa.dsa_workspace_bytes(dec, 2048) >= 64 * 131072 * 4
    long_rows = dsa.make_dims(4, 1, 140000)
    assert dsa.dsa_workspace_bytes(long_rows, 2048) >= 4 * ((140000 + 8191) // 8192) * 2048 * 8
    tiny = dsa.make_dims(1, 512, 512, 4, 32, 8, 64, 16)
    assert dsa.dsa_workspace_bytes(tiny, 64) > dsa.dsa_workspace_bytes(dsa.make_dims(1, 512, 512), 64)  # padding
    for bad in [dsa.make_dims(1, 10, 5), dsa.make_dims(-1, 1, 1), dsa.make_dims(1, 1, 1, n_idx_heads=65),
                dsa.make_dims(1, 1, 1, idx_dim=24), dsa.make_dims(1, 1, 1, d_latent=520)]:
        assert dsa.dsa_workspace_bytes(bad, 16) == 0
    assert dsa.dsa_workspace_bytes(prod, 0) == 0
    assert dsa.dsa_workspace_bytes(prod, 4096) == 0


def test_host_validation_returns_before_any_launch(dsa):
    lib = dsa._lib
    dims = dsa.make_dims(1, 8, 8)
    n = dsa.dsa_workspace_bytes(dims, 4)
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: every call below fails validation
    P = ctypes.c_void_p
    # unsupported dims
    big = dsa.make_dims(1, 8, 8, n_heads=129)
    assert lib.dsa_indexer_topk(ctypes.byref(big), fake, fake, fake, fake, fake, 4, fake, fake, n, None) == \
        dsa.DSA_ERR_UNSUPPORTED
    # workspace too small / missing / misaligned
    assert lib.dsa_indexer_topk(ctypes.byref(dims), fake, fake, fake, fake, fake, 4, fake, fake, n - 256, None) == \
        dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_sparse_mla_attn(ctypes.byref(dims), fake, fake, fake, 4, fake, fake, None, n, None) == \
        dsa.DSA_ERR_WORKSPACE
    assert lib.dsa_forward(ctypes.byref(dims), fake, fake, fake, fake, fake, 4, fake, fake, None, fake, fake,
                           P((1 << 20) + 8), n, None) == dsa.DSA_ERR_WORKSPACE
    # null tensors / misaligned tensors
    assert lib.dsa_indexer_topk(ctypes.byref(dims), None, fake, fake, fake, fake, 4, fake, fake, n, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_sparse_mla_attn(ctypes.byref(dims), P((1 << 20) + 2), fake, fake, 4, fake, fake, fake, n,
                                   None) == dsa.DSA_ERR_INVALID_ARG
    # bad top-k, null dims
    assert lib.dsa_indexer_topk(ctypes.byref(dims), fake, fake, fake, fake, fake, 0, fake, fake, n, None) == \
        dsa.DSA_ERR_INVALID_ARG
    assert lib.dsa_indexer_topk(None, fake, fake, fake, fake, fake, 4, fake, fake, n, None) == dsa.DSA_ERR_INVALID_ARG
    # an empty problem succeeds without work
    empty = dsa.make_dims(0, 8, 8)
    ne = dsa.dsa_workspace_bytes(empty, 4)
    assert lib.dsa_forward(ctypes.byref(empty), None, None, None, None, None, 4, None, None, None, None, None,
                           fake, ne, None) == dsa.DSA_OK
