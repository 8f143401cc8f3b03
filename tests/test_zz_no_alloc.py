"""Decode selection without a workspace: dsa_indexer_topk_decode_noalloc.

Some callers cannot allocate device memory for a call -- serving runtimes that plan every
buffer ahead, plugin interfaces that hand a kernel only its inputs and outputs, loops that
cannot afford cudaMalloc's implicit synchronisation. This entry point keeps its scratch (the
per-chunk top-k lists of the decode selection) in a device array inside the library. The test
calls it through the C ABI twice in a row and checks each call's selections against the
workspace entry point, dsa_indexer_topk, and a few sequences of each against the oracle. The
first call uses top-k 2048 over five 8192-key chunks per sequence, the second top-k 64 over two
chunks, so the second call's slots sit where the first left longer lists and larger counts:
leftovers in the shared array would show. It also checks that oversized problems are refused.
"""
import ctypes

import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu


def _lib():
    import sparse_attention_long_indexer_b200 as dsa
    lib = dsa._lib
    P = ctypes.c_void_p
    lib.dsa_indexer_topk_decode_noalloc.argtypes = [ctypes.POINTER(dsa.dsa_dims), P, P, P, P, P, ctypes.c_int32, P, P,
                                                    P]
    lib.dsa_indexer_topk_decode_noalloc.restype = ctypes.c_int
    return dsa, lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_noalloc_decode_matches_workspace_entry_point():
    from tests.dsa_cases import RowOracle, check_selection
    dsa, lib = _lib()
    stream = torch.cuda.current_stream()
    calls = [(31, synthetic.config("decode", batch=6, max_len=40000, len_range=(3000, 40000))),
             (32, synthetic.config("decode", batch=6, max_len=9000, len_range=(1000, 9000), topk=64))]
    for seed, cfg in calls:                              # two calls in a row, different inputs and sizes
        dims = dsa.dims_for(cfg)
        ws = dsa.Workspace.create(dims, cfg.topk)
        g = synthetic.gen_all(cfg, seed, "cuda")
        scales = torch.cat([g["q_scale"].reshape(-1), g["k_scale"].reshape(-1)]).contiguous()
        ref = dsa.indexer_topk(dims, g["q_idx"], g["w"], g["k_idx"], g["q_scale"], g["k_scale"], g["lengths"],
                               cfg.topk, ws)
        out = torch.full_like(ref, -7)
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        rc = lib.dsa_indexer_topk_decode_noalloc(ctypes.byref(dims), _p(g["q_idx"]), _p(g["w"]), _p(g["k_idx"]),
                                                 _p(scales), _p(g["lengths"]), cfg.topk, _p(out), _p(status),
                                                 ctypes.c_void_p(stream.cuda_stream))
        assert rc == dsa.DSA_OK, dsa.dsa_status_string(rc)
        torch.cuda.synchronize()
        ws.check()
        assert status.tolist() == [0, 0]
        lengths = g["lengths"].tolist()
        got_all = out.cpu().numpy()
        for b in range(cfg.batch):
            n = min(cfg.topk, lengths[b])
            got, exp = got_all[b, 0].tolist(), ref[b, 0].tolist()
            assert sorted(got[:n]) == sorted(exp[:n])          # same selected set
            assert all(x == -1 for x in got[n:])               # padding after the selection
        ro = RowOracle(cfg, seed)
        for b in (0, cfg.batch - 1):                           # and the oracle agrees, up to near-ties
            _, scores = ro.indexer(b, 0)
            check_selection(got_all[b, 0], scores, cfg.topk, ro.pos(b, 0))


def test_noalloc_decode_refuses_sizes_beyond_its_array():
    dsa, lib = _lib()
    dummy = torch.zeros(64, dtype=torch.uint8, device="cuda")
    too_many = dsa.make_dims(129, 1, 65536)                # 129 sequences x 8 chunks > 1024 slots
    assert lib.dsa_indexer_topk_decode_noalloc(ctypes.byref(too_many), _p(dummy), _p(dummy), _p(dummy), _p(dummy),
                                               _p(dummy), 2048, _p(dummy), None, None) == dsa.DSA_ERR_UNSUPPORTED
    prefill = dsa.make_dims(1, 8, 8)                        # n_q != 1
    assert lib.dsa_indexer_topk_decode_noalloc(ctypes.byref(prefill), _p(dummy), _p(dummy), _p(dummy), _p(dummy),
                                               _p(dummy), 4, _p(dummy), None, None) == dsa.DSA_ERR_UNSUPPORTED
