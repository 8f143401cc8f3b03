"""Python binding of the DSA forward-path C ABI (``include/dsa.h``, ``libdsa.so``).

Argument marshalling only: every step of the path (lightning indexer, top-k selection,
sparse MLA attention) runs in the library's CUDA kernels. PyTorch supplies device memory
and streams. There is no CPU fallback: importing this package raises if ``libdsa.so`` is
missing, and every call raises ``DSAError`` on a non-OK status.

Functions with the C names take torch tensors (device memory, contiguous, the dtypes
stated in ``include/dsa.h``); ``forward`` / ``indexer_topk`` / ``sparse_mla_attn``
allocate outputs for convenience.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"{_LIB_PATH} is missing: build it with `python -m sparse_attention_long_indexer_b200.build` "
        "(the DSA path has no CPU fallback)")
_lib = ctypes.CDLL(_LIB_PATH)

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_CUDA = 0, 1, 2, 3
DSA_ERR_DEVICE_TIMEOUT, DSA_ERR_INDEX_RANGE, DSA_ERR_WORKSPACE = 4, 5, 6

LIBRARY_PATH = _LIB_PATH
EXPORTED = ("dsa_workspace_bytes", "dsa_workspace_init", "dsa_indexer_topk", "dsa_sparse_mla_attn",
            "dsa_forward", "dsa_get_device_status", "dsa_status_string", "dsa_version",
            "dsa_indexer_topk_decode_noalloc", "dsa_masked_mqa_attn", "dsa_indexer_topk_scores",
            "dsa_indexer_kl_loss", "dsa_set_wait_budget_ns")


class dsa_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q", ctypes.c_int32), ("max_len", ctypes.c_int32),
                ("n_idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("d_latent", ctypes.c_int32), ("d_rope", ctypes.c_int32), ("softmax_scale", ctypes.c_float)]


_P = ctypes.c_void_p
_DIMS = ctypes.POINTER(dsa_dims)
_lib.dsa_workspace_bytes.argtypes = [_DIMS, ctypes.c_int32]
_lib.dsa_workspace_bytes.restype = ctypes.c_size_t
_lib.dsa_workspace_init.argtypes = [_P, ctypes.c_size_t, _P]
_lib.dsa_workspace_init.restype = ctypes.c_int
_lib.dsa_indexer_topk.argtypes = [_DIMS, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_indexer_topk.restype = ctypes.c_int
_lib.dsa_indexer_topk_scores.argtypes = [_DIMS, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_indexer_topk_scores.restype = ctypes.c_int
_lib.dsa_indexer_kl_loss.argtypes = [_DIMS, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_indexer_kl_loss.restype = ctypes.c_int
_lib.dsa_sparse_mla_attn.argtypes = [_DIMS, _P, _P, _P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_sparse_mla_attn.restype = ctypes.c_int
_lib.dsa_masked_mqa_attn.argtypes = [_DIMS, _P, _P, _P, ctypes.c_int32, _P, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_masked_mqa_attn.restype = ctypes.c_int
_lib.dsa_forward.argtypes = [_DIMS, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
_lib.dsa_forward.restype = ctypes.c_int
_lib.dsa_get_device_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint32)]
_lib.dsa_get_device_status.restype = ctypes.c_int
_lib.dsa_status_string.argtypes = [ctypes.c_int]
_lib.dsa_status_string.restype = ctypes.c_char_p
_lib.dsa_set_wait_budget_ns.argtypes = [ctypes.c_uint64]
_lib.dsa_set_wait_budget_ns.restype = ctypes.c_int
_lib.dsa_version.argtypes = []
_lib.dsa_version.restype = ctypes.c_int32


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {dsa_status_string(status)} (status {status})")


def dsa_status_string(status: int) -> str:
    return _lib.dsa_status_string(int(status)).decode()


def dsa_set_wait_budget_ns(ns: int):
    """Test setting: budget of the indexer's pipeline waits in ns (0 = the default 2 s)."""
    _check(_lib.dsa_set_wait_budget_ns(int(ns)), "dsa_set_wait_budget_ns")


def dsa_version() -> int:
    return int(_lib.dsa_version())


def make_dims(batch, n_q, max_len, n_idx_heads=64, idx_dim=128, n_heads=128, d_latent=512, d_rope=64,
              softmax_scale=None) -> dsa_dims:
    if softmax_scale is None:
        softmax_scale = 1.0 / float(d_latent + d_rope) ** 0.5
    return dsa_dims(batch, n_q, max_len, n_idx_heads, idx_dim, n_heads, d_latent, d_rope, softmax_scale)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("DSA tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status: int, where: str):
    if status != DSA_OK:
        raise DSAError(status, where)


def _expect(t: torch.Tensor, dtype, name: str):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be device memory")


# ----------------------------------------------------------------------------- C-named calls
def dsa_workspace_bytes(dims: dsa_dims, topk: int) -> int:
    return int(_lib.dsa_workspace_bytes(ctypes.byref(dims), int(topk)))


def dsa_workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.dsa_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "dsa_workspace_init")


def dsa_indexer_topk(dims, q_idx, w, k_idx, scales, lengths, topk, out_idx, ws, stream=None):
    _check(_lib.dsa_indexer_topk(ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(scales), _ptr(lengths),
                                 int(topk), _ptr(out_idx), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_indexer_topk")


def dsa_indexer_topk_scores(dims, q_idx, w, k_idx, scales, lengths, topk, out_idx, out_scores, ws, stream=None):
    _check(_lib.dsa_indexer_topk_scores(ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(scales),
                                        _ptr(lengths), int(topk), _ptr(out_idx), _ptr(out_scores), _ptr(ws),
                                        ws.numel(), _stream(stream)), "dsa_indexer_topk_scores")


def dsa_indexer_kl_loss(dims, q, latent_kv, idx, idx_scores, lse, topk, loss, ws, stream=None):
    _check(_lib.dsa_indexer_kl_loss(ctypes.byref(dims), _ptr(q), _ptr(latent_kv), _ptr(idx), _ptr(idx_scores),
                                    _ptr(lse), int(topk), _ptr(loss), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_indexer_kl_loss")


def dsa_sparse_mla_attn(dims, q, latent_kv, idx, topk, out, lse, ws, stream=None):
    _check(_lib.dsa_sparse_mla_attn(ctypes.byref(dims), _ptr(q), _ptr(latent_kv), _ptr(idx), int(topk), _ptr(out),
                                    _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "dsa_sparse_mla_attn")


def dsa_masked_mqa_attn(dims, q, latent_kv, idx, topk, out, lse, ws, stream=None):
    _check(_lib.dsa_masked_mqa_attn(ctypes.byref(dims), _ptr(q), _ptr(latent_kv), _ptr(idx), int(topk), _ptr(out),
                                    _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "dsa_masked_mqa_attn")


def dsa_forward(dims, q_idx, w, k_idx, scales, lengths, topk, q, latent_kv, out_idx, out, lse, ws, stream=None):
    _check(_lib.dsa_forward(ctypes.byref(dims), _ptr(q_idx), _ptr(w), _ptr(k_idx), _ptr(scales), _ptr(lengths),
                            int(topk), _ptr(q), _ptr(latent_kv), _ptr(out_idx), _ptr(out), _ptr(lse), _ptr(ws),
                            ws.numel(), _stream(stream)), "dsa_forward")


def dsa_get_device_status(ws: torch.Tensor, stream=None):
    detail = ctypes.c_uint32(0)
    st = int(_lib.dsa_get_device_status(_ptr(ws), _stream(stream), ctypes.byref(detail)))
    return st, int(detail.value)


# ----------------------------------------------------------------------------- conveniences
@dataclass
class Workspace:
    """A device workspace sized for (dims, topk), status word zeroed."""
    dims: dsa_dims
    topk: int
    buf: torch.Tensor

    @staticmethod
    def create(dims: dsa_dims, topk: int, device=None, stream=None) -> "Workspace":
        n = dsa_workspace_bytes(dims, topk)
        if n == 0:
            raise DSAError(DSA_ERR_INVALID_ARG, "dsa_workspace_bytes")
        buf = torch.empty(n + 256, dtype=torch.uint8, device=device or "cuda")
        off = (-buf.data_ptr()) % 256
        buf = buf[off:off + n]
        dsa_workspace_init(buf, stream)
        return Workspace(dims, topk, buf)

    def check(self, stream=None):
        """Raises DSAError if a kernel recorded a device-side error since the last check."""
        st, detail = dsa_get_device_status(self.buf, stream)
        if st != DSA_OK:
            raise DSAError(st, f"device status (detail 0x{detail:08x})")


def _scales(q_scale: torch.Tensor, k_scale: torch.Tensor) -> torch.Tensor:
    return torch.cat([q_scale.reshape(-1), k_scale.reshape(-1)]).to(torch.float32).contiguous()


def indexer_topk(dims, q_idx, w, k_idx, q_scale, k_scale, lengths, topk, ws: Workspace, stream=None):
    """Returns int32 [B, n_q, topk] selected positions (-1 padded, unspecified order)."""
    _expect(q_idx, torch.uint8, "q_idx")
    _expect(k_idx, torch.uint8, "k_idx")
    _expect(w, torch.bfloat16, "w")
    out_idx = torch.empty((dims.batch, dims.n_q, topk), dtype=torch.int32, device=q_idx.device)
    dsa_indexer_topk(dims, q_idx, w, k_idx, _scales(q_scale, k_scale), lengths.to(torch.int32).contiguous(), topk,
                     out_idx, ws.buf, stream)
    return out_idx


def sparse_mla_attn(dims, q, latent_kv, idx, topk, ws: Workspace, stream=None):
    """Returns (out bf16 [B, n_q, H, d_latent], lse fp32 [B, n_q, H])."""
    _expect(q, torch.bfloat16, "q")
    _expect(latent_kv, torch.bfloat16, "latent_kv")
    out = torch.empty((dims.batch, dims.n_q, dims.n_heads, dims.d_latent), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((dims.batch, dims.n_q, dims.n_heads), dtype=torch.float32, device=q.device)
    dsa_sparse_mla_attn(dims, q, latent_kv, idx.to(torch.int32).contiguous(), topk, out, lse, ws.buf, stream)
    return out, lse


def indexer_topk_scores(dims, q_idx, w, k_idx, q_scale, k_scale, lengths, topk, ws: Workspace, stream=None):
    """Returns (idx int32 [B, n_q, topk], scores fp32 [B, n_q, topk]); -1 / -inf padded."""
    _expect(q_idx, torch.uint8, "q_idx")
    _expect(k_idx, torch.uint8, "k_idx")
    _expect(w, torch.bfloat16, "w")
    out_idx = torch.empty((dims.batch, dims.n_q, topk), dtype=torch.int32, device=q_idx.device)
    out_scores = torch.empty((dims.batch, dims.n_q, topk), dtype=torch.float32, device=q_idx.device)
    dsa_indexer_topk_scores(dims, q_idx, w, k_idx, _scales(q_scale, k_scale), lengths.to(torch.int32).contiguous(),
                            topk, out_idx, out_scores, ws.buf, stream)
    return out_idx, out_scores


def indexer_kl_loss(dims, q, latent_kv, idx, idx_scores, lse, topk, ws: Workspace, stream=None):
    """Returns the per-query indexer-alignment KL terms, fp32 [B, n_q]."""
    loss = torch.empty((dims.batch, dims.n_q), dtype=torch.float32, device=q.device)
    dsa_indexer_kl_loss(dims, q, latent_kv, idx.to(torch.int32).contiguous(), idx_scores.contiguous(),
                        lse.contiguous(), topk, loss, ws.buf, stream)
    return loss


def masked_mqa_attn(dims, q, latent_kv, idx, topk, ws: Workspace, stream=None):
    """The masked dense mode of the attention. Returns (out, lse) like ``sparse_mla_attn``."""
    _expect(q, torch.bfloat16, "q")
    _expect(latent_kv, torch.bfloat16, "latent_kv")
    out = torch.empty((dims.batch, dims.n_q, dims.n_heads, dims.d_latent), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((dims.batch, dims.n_q, dims.n_heads), dtype=torch.float32, device=q.device)
    dsa_masked_mqa_attn(dims, q, latent_kv, idx.to(torch.int32).contiguous(), topk, out, lse, ws.buf, stream)
    return out, lse


def forward(dims, q_idx, w, k_idx, q_scale, k_scale, lengths, topk, q, latent_kv, ws: Workspace, stream=None,
            return_idx: bool = True):
    """The whole DSA forward path. Returns (idx or None, out, lse)."""
    dev = q.device
    out = torch.empty((dims.batch, dims.n_q, dims.n_heads, dims.d_latent), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((dims.batch, dims.n_q, dims.n_heads), dtype=torch.float32, device=dev)
    out_idx = torch.empty((dims.batch, dims.n_q, topk), dtype=torch.int32, device=dev) if return_idx else None
    dsa_forward(dims, q_idx, w, k_idx, _scales(q_scale, k_scale), lengths.to(torch.int32).contiguous(), topk, q,
                latent_kv, out_idx, out, lse, ws.buf, stream)
    return out_idx, out, lse


def dims_for(cfg) -> dsa_dims:
    """dsa_dims of a workload description with the fields of ``synthetic.DSAConfig``."""
    return make_dims(cfg.batch, cfg.n_q, cfg.max_len, cfg.n_idx_heads, cfg.idx_dim, cfg.n_heads, cfg.d_latent,
                     cfg.d_rope, cfg.softmax_scale)
