"""Seeded synthetic inputs for the DeepSeek Sparse Attention (DSA) forward path.

This module draws numbers and stores them in the formats the path consumes:
FP8 E4M3 codes with one fp32 scale per token for the lightning indexer, bf16
for the indexer head weights, the attention queries and the latent KV cache.
It contains no step of the method itself (no score, no selection, no
attention), so both the CUDA path (driven by the tests and the bench) and the
CPU oracle take their inputs from here without sharing any of the method's
arithmetic.

Determinism across devices.  Every element is a pure function of
(seed, tensor id, flat element index):

* a 32-bit integer mixer (xor-shift / odd-multiply rounds whose constants are
  below 2**30, so every product fits in a signed int64 and torch computes it
  exactly on CPU and CUDA alike) turns the counter into two 32-bit words;
* the four 16-bit halves are summed (Irwin-Hall of order 4, a bounded
  approximation of a normal law with mean 0 and unit variance after scaling);
  the sum is an exact integer below 2**18, converted exactly to fp32 and
  multiplied once by an fp32 constant (one IEEE-rounded product);
* FP8 quantisation uses a per-token power-of-two scale (exact scaling, below
  the E4M3 maximum) and one round-to-nearest-even cast; bf16 is a
  round-to-nearest-even cast.

So a row generated on the CPU for the oracle has the same bits as the same row
generated on the GPU for the kernels; a GPU test pins this.

Workloads follow the DeepSeek-V3.2-Exp DSA description (lightning indexer with
FP8 inputs and few heads, top-k = 2048, MLA in MQA mode with one 512+64-d
latent row per token, 128K context): see ``CONFIGS``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional, Sequence

import torch

__all__ = [
    "DSAConfig", "CONFIGS", "config", "mix32_int", "normal_rows", "lengths",
    "quantize_e4m3_rows", "quantize_e4m3_rows_amax", "gen_q_idx", "gen_k_idx", "gen_w", "gen_q", "gen_kv",
    "gen_all", "TENSOR_IDS",
]

_M32 = 0xFFFFFFFF
_C1 = 0x2C1B3C6D  # odd, < 2**30
_C2 = 0x297A2D39  # odd, < 2**30
_IH_MEAN = 4 * 65535 // 2          # mean of the sum of four 16-bit uniforms (131070)
_IH_STD = math.sqrt(4 * (65536.0 ** 2 - 1.0) / 12.0)
E4M3_MAX = 448.0

# one stream per input tensor
TENSOR_IDS = {"q_idx": 1, "k_idx": 2, "w": 3, "q": 4, "kv": 5, "lengths": 6, "sample": 7}

_CHUNK = 1 << 25  # elements per generation chunk (bounds temporaries to ~1 GB)


# ----------------------------------------------------------------------------- configs
@dataclass(frozen=True)
class DSAConfig:
    """Shapes and source distributions of one DSA workload.

    Query ``i`` of sequence ``b`` sits at position ``len_b - n_q + i``; prefill
    has ``n_q == max_len == L`` (so position ``i``), decode has ``n_q == 1``.
    """
    name: str
    batch: int
    n_q: int
    max_len: int
    n_idx_heads: int      # H_I, lightning-indexer heads
    idx_dim: int          # d_I, indexer head dim
    n_heads: int          # H, attention query heads sharing one latent row (MQA mode)
    d_latent: int         # d_c, compressed latent (also the value)
    d_rope: int           # d_r, decoupled RoPE part of the key
    topk: int             # k, selected tokens per query
    q_idx_std: float = 1.0
    k_idx_std: float = 1.0
    w_std: float = 0.125
    qkv_std: float = 1.0
    len_range: Optional[tuple] = None   # decode: lengths ~ U[lo, hi] (inclusive)
    # per-token FP8 scale: "pow2" = the power of two above amax/256 (exact scaling), or
    # "amax" = amax/448 rounded to fp32 (a general positive scale; generate on the CPU)
    fp8_scale: str = "pow2"
    description: str = field(default="", compare=False)

    @property
    def d_qk(self) -> int:
        return self.d_latent + self.d_rope

    @property
    def d_v(self) -> int:
        return self.d_latent

    @property
    def softmax_scale(self) -> float:
        """1/sqrt(d_qk), rounded to fp32 (the value both sides are given)."""
        return float(torch.tensor(1.0 / math.sqrt(self.d_qk), dtype=torch.float32))

    @property
    def is_decode(self) -> bool:
        return self.len_range is not None


_PROD = dict(n_idx_heads=64, idx_dim=128, n_heads=128, d_latent=512, d_rope=64, topk=2048,
             q_idx_std=1.0, k_idx_std=1.0, w_std=0.125, qkv_std=1.0)

CONFIGS = {
    "tiny": DSAConfig(
        name="tiny", batch=1, n_q=512, max_len=512, n_idx_heads=4, idx_dim=32, n_heads=8,
        d_latent=64, d_rope=16, topk=64, q_idx_std=1.0 / math.sqrt(32), k_idx_std=1.0 / math.sqrt(32),
        w_std=0.5, qkv_std=1.0,
        description="tiny causal prefill L=512, H_I=4 d_I=32, H=8, latent 64+16, k=64"),
    "prefill_4k": DSAConfig(name="prefill_4k", batch=1, n_q=4096, max_len=4096, **_PROD,
                            description="causal prefill L=4096, k=2048"),
    "prefill_32k": DSAConfig(name="prefill_32k", batch=1, n_q=32768, max_len=32768, **_PROD,
                             description="causal prefill L=32768, k=2048"),
    "prefill_128k": DSAConfig(name="prefill_128k", batch=1, n_q=131072, max_len=131072, **_PROD,
                              description="causal prefill L=131072 (128K), k=2048"),
    "decode": DSAConfig(name="decode", batch=64, n_q=1, max_len=131072, len_range=(4096, 131072),
                        **_PROD, description="decode: 64 sequences, len ~ U[4096,131072], 1 query each"),
}


def config(name: str, **overrides) -> DSAConfig:
    """A named config, optionally with fields replaced (e.g. a shorter L for a test)."""
    return replace(CONFIGS[name], **overrides) if overrides else CONFIGS[name]


# ----------------------------------------------------------------------------- integer mixer
def mix32_int(x: int) -> int:
    """Reference (pure Python) form of the 32-bit mixer used for every element."""
    x &= _M32
    x ^= x >> 16
    x = (x * _C1) & _M32
    x ^= x >> 15
    x = (x * _C2) & _M32
    x ^= x >> 16
    return x


def _mix32(x: torch.Tensor) -> torch.Tensor:
    # x: int64 with values in [0, 2**32); every product stays below 2**62
    x = x ^ (x >> 16)
    x = (x * _C1) & _M32
    x = x ^ (x >> 15)
    x = (x * _C2) & _M32
    x = x ^ (x >> 16)
    return x


def _stream_key(seed: int, tensor: str) -> int:
    return mix32_int(((seed & _M32) * 0x9E3779B1 + TENSOR_IDS[tensor] * 0x7F4A7C15) & _M32)


def _words(flat: torch.Tensor, key: int):
    lo = flat & _M32
    hi = flat >> 32
    h1 = _mix32(lo ^ key)
    h1 = _mix32((h1 + hi * 0x3C6EF35F + 0x1B873593) & _M32)
    h2 = _mix32(h1 ^ 0x68E31DA4)
    return h1, h2


def _irwin_hall(flat: torch.Tensor, key: int, std: float) -> torch.Tensor:
    h1, h2 = _words(flat, key)
    s = (h1 & 0xFFFF) + (h1 >> 16) + (h2 & 0xFFFF) + (h2 >> 16) - _IH_MEAN
    c = torch.tensor(std / _IH_STD, dtype=torch.float32, device=flat.device)
    return s.to(torch.float32) * c


def normal_rows(seed: int, tensor: str, rows, row_len: int, std: float, device="cpu") -> torch.Tensor:
    """fp32 [len(rows), row_len]; element (r, c) is drawn from counter r*row_len + c.

    ``rows`` is a sequence / int64 tensor of row ids, or a ``range``.
    """
    key = _stream_key(seed, tensor)
    if isinstance(rows, range):
        assert rows.step == 1
        r0, n = rows.start, len(rows)
        out = torch.empty((n, row_len), dtype=torch.float32, device=device)
        per = max(1, _CHUNK // row_len)
        cols = torch.arange(row_len, dtype=torch.int64, device=device)
        for a in range(0, n, per):
            b = min(n, a + per)
            rid = torch.arange(r0 + a, r0 + b, dtype=torch.int64, device=device)
            flat = rid[:, None] * row_len + cols[None, :]
            out[a:b] = _irwin_hall(flat, key, std)
        return out
    rid = torch.as_tensor(rows, dtype=torch.int64, device=device).reshape(-1)
    cols = torch.arange(row_len, dtype=torch.int64, device=device)
    return _irwin_hall(rid[:, None] * row_len + cols[None, :], key, std)


def _pow2(k: torch.Tensor) -> torch.Tensor:
    """2**k in fp32 built from its IEEE bits (exact; k clamped to the normal range)."""
    return ((k.to(torch.int32) + 127).clamp(1, 254) << 23).view(torch.float32)


def quantize_e4m3_rows(x: torch.Tensor):
    """Per-row FP8 E4M3 codes (uint8) and fp32 scales.

    The scale is the power of two 2**(e-8) where amax = m * 2**e, 0.5 <= m < 1 (1 if
    amax == 0), so |x / scale| < 256 <= 448 and x / scale is exact; the only rounding is
    the round-to-nearest-even cast to E4M3. (A division by amax/448 would round twice, and
    torch rounds a division by a Python scalar differently on CPU and CUDA.)
    """
    amax = x.abs().amax(dim=1)
    _, e = torch.frexp(amax)
    nz = amax > 0
    scale = torch.where(nz, _pow2(e - 8), torch.ones_like(amax))
    inv = torch.where(nz, _pow2(8 - e), torch.zeros_like(amax))
    y = x * inv[:, None]
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale


def quantize_e4m3_rows_amax(x: torch.Tensor):
    """Per-row FP8 E4M3 codes (uint8) and fp32 scales scale = amax / 448.

    The scale is amax/448 computed in float64 and rounded to fp32 (1 if amax == 0), so it is
    in general not a power of two. Codes are x / scale computed in float64, clamped to
    [-448, 448], rounded to fp32 and then to E4M3 (round to nearest even). Deterministic on
    the CPU; tests generate these inputs there and upload them.
    """
    amax = x.abs().amax(dim=1).double()
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax)).float()
    y = (x.double() / scale.double()[:, None]).clamp(-E4M3_MAX, E4M3_MAX).float()
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale


def _quantizer(cfg: "DSAConfig"):
    if cfg.fp8_scale == "pow2":
        return quantize_e4m3_rows
    if cfg.fp8_scale == "amax":
        return quantize_e4m3_rows_amax
    raise ValueError(f"unknown fp8_scale {cfg.fp8_scale!r}")


# ----------------------------------------------------------------------------- lengths
def lengths(cfg: DSAConfig, seed: int) -> torch.Tensor:
    """int32 [B]: L for prefill, U[lo, hi] (seeded) for decode."""
    if cfg.len_range is None:
        return torch.full((cfg.batch,), cfg.max_len, dtype=torch.int32)
    lo, hi = cfg.len_range
    key = _stream_key(seed, "lengths")
    vals = [lo + mix32_int(mix32_int(b ^ key) + 0x165667B1) % (hi - lo + 1) for b in range(cfg.batch)]
    return torch.tensor(vals, dtype=torch.int32)


# ----------------------------------------------------------------------------- tensors
def _token_rows(cfg: DSAConfig, b_i):
    """flat query-token ids b*n_q+i for a list of (b, i)."""
    return [b * cfg.n_q + i for (b, i) in b_i]


def gen_q_idx(cfg: DSAConfig, seed: int, device="cpu", tokens=None):
    """Indexer queries: (uint8 E4M3 [T, H_I, d_I], fp32 scale [T]).

    ``tokens``: None = all B*n_q query tokens (flat order b*n_q+i), else a list of flat ids.
    """
    rl = cfg.n_idx_heads * cfg.idx_dim
    if tokens is None:
        n = cfg.batch * cfg.n_q
        codes = torch.empty((n, rl), dtype=torch.uint8, device=device)
        scale = torch.empty((n,), dtype=torch.float32, device=device)
        per = max(1, _CHUNK // rl)
        for a in range(0, n, per):
            b = min(n, a + per)
            c, s = _quantizer(cfg)(normal_rows(seed, "q_idx", range(a, b), rl, cfg.q_idx_std, device))
            codes[a:b], scale[a:b] = c, s
    else:
        codes, scale = _quantizer(cfg)(normal_rows(seed, "q_idx", tokens, rl, cfg.q_idx_std, device))
    return codes.view(-1, cfg.n_idx_heads, cfg.idx_dim), scale


def gen_k_idx(cfg: DSAConfig, seed: int, device="cpu", b: Optional[int] = None, s_range=None):
    """Indexer keys: (uint8 E4M3, fp32 scale).

    All: ([B, max_len, d_I], [B, max_len]); one sequence ``b`` and ``s_range``: ([n, d_I], [n]).
    """
    rl = cfg.idx_dim
    if b is None:
        n = cfg.batch * cfg.max_len
        codes = torch.empty((n, rl), dtype=torch.uint8, device=device)
        scale = torch.empty((n,), dtype=torch.float32, device=device)
        per = max(1, _CHUNK // rl)
        for a in range(0, n, per):
            e = min(n, a + per)
            c, s = _quantizer(cfg)(normal_rows(seed, "k_idx", range(a, e), rl, cfg.k_idx_std, device))
            codes[a:e], scale[a:e] = c, s
        return codes.view(cfg.batch, cfg.max_len, rl), scale.view(cfg.batch, cfg.max_len)
    s_range = range(cfg.max_len) if s_range is None else s_range
    rows = range(b * cfg.max_len + s_range.start, b * cfg.max_len + s_range.stop)
    return _quantizer(cfg)(normal_rows(seed, "k_idx", rows, rl, cfg.k_idx_std, device))


def _bf16_rows(seed, tensor, rows, row_len, std, device):
    if isinstance(rows, range):
        n = len(rows)
        out = torch.empty((n, row_len), dtype=torch.bfloat16, device=device)
        per = max(1, _CHUNK // row_len)
        for a in range(0, n, per):
            e = min(n, a + per)
            out[a:e] = normal_rows(seed, tensor, range(rows.start + a, rows.start + e), row_len, std,
                                   device).to(torch.bfloat16)
        return out
    return normal_rows(seed, tensor, rows, row_len, std, device).to(torch.bfloat16)


def gen_w(cfg: DSAConfig, seed: int, device="cpu", tokens=None):
    """Indexer head weights, bf16 [T, H_I] (T = all B*n_q tokens or the listed flat ids)."""
    rows = range(cfg.batch * cfg.n_q) if tokens is None else tokens
    return _bf16_rows(seed, "w", rows, cfg.n_idx_heads, cfg.w_std, device)


def gen_q(cfg: DSAConfig, seed: int, device="cpu", tokens=None):
    """Attention queries in MQA form, bf16 [T, H, d_qk]."""
    rows = range(cfg.batch * cfg.n_q) if tokens is None else tokens
    rl = cfg.n_heads * cfg.d_qk
    return _bf16_rows(seed, "q", rows, rl, cfg.qkv_std, device).view(-1, cfg.n_heads, cfg.d_qk)


def gen_kv(cfg: DSAConfig, seed: int, device="cpu", b: Optional[int] = None, positions=None):
    """Latent KV rows (512 latent | 64 rope), bf16.

    All: [B, max_len, d_qk]; sequence ``b`` with ``positions`` (range or list): [n, d_qk].
    """
    if b is None:
        out = _bf16_rows(seed, "kv", range(cfg.batch * cfg.max_len), cfg.d_qk, cfg.qkv_std, device)
        return out.view(cfg.batch, cfg.max_len, cfg.d_qk)
    if isinstance(positions, range):
        rows = range(b * cfg.max_len + positions.start, b * cfg.max_len + positions.stop)
    else:
        rows = [b * cfg.max_len + int(p) for p in positions]
    return _bf16_rows(seed, "kv", rows, cfg.d_qk, cfg.qkv_std, device)


def gen_all(cfg: DSAConfig, seed: int, device="cpu") -> dict:
    """Every input tensor of the workload, in the layouts the C ABI takes."""
    q_idx, q_scale = gen_q_idx(cfg, seed, device)
    k_idx, k_scale = gen_k_idx(cfg, seed, device)
    return dict(
        q_idx=q_idx.view(cfg.batch, cfg.n_q, cfg.n_idx_heads, cfg.idx_dim),
        q_scale=q_scale.view(cfg.batch, cfg.n_q),
        w=gen_w(cfg, seed, device).view(cfg.batch, cfg.n_q, cfg.n_idx_heads),
        k_idx=k_idx, k_scale=k_scale,
        q=gen_q(cfg, seed, device).view(cfg.batch, cfg.n_q, cfg.n_heads, cfg.d_qk),
        kv=gen_kv(cfg, seed, device),
        lengths=lengths(cfg, seed).to(device),
    )


def sample_rows(n_total: int, n: int, seed: int, extra: Sequence[int] = ()) -> list:
    """Seeded distinct sample of ``n`` ids in [0, n_total) plus ``extra`` ids, sorted."""
    key = _stream_key(seed, "sample")
    chosen, i = set(int(e) for e in extra if 0 <= e < n_total), 0
    target = min(n_total, n + len(chosen))
    while len(chosen) < target:
        chosen.add(mix32_int(i ^ key) % n_total)
        i += 1
    return sorted(chosen)
