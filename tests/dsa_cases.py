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
# oracle score lies within 1e-3 (relative) of the k-th score I_k; attention max-abs 1e-2 and
# relative L2 5e-3, both per query row. Reading for a k-th score near zero (w may be negative,
# so I_k can sit at 0 where a relative band is empty): where |I_k| < 0.05 x RMS of the row's
# scores, the band is 1e-3 x 0.05 x RMS instead; the rows where that floor decided anything
# are counted and reported. lse has no stated bound; its error budget (fp32 logits, bf16-rounded
# weights) is far below 2e-3 absolute, which the tests use.
NEAR_TIE_REL = 1e-3
NEAR_ZERO_FRAC = 0.05
OUT_MAX_ABS = 1e-2
OUT_REL_L2 = 5e-3
LSE_MAX_ABS = 2e-3

# Near-tie statistics of every checked configuration, printed at the end of the session
# (tests/conftest.py): name -> [rows checked, rows with a near-tie swap, swapped pairs,
# rows where the near-zero floor was needed].
NEAR_TIE_REPORT = {}


def report_near_ties(name, rows, stats):
    """Adds the SelectionCheck results of ``rows`` query rows to the session report."""
    r = NEAR_TIE_REPORT.setdefault(name, [0, 0, 0, 0])
    r[0] += rows
    for st in stats:
        r[1] += 1 if st.ties else 0
        r[2] += st.ties
        r[3] += 1 if st.floor_used else 0


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


class SelectionCheck(tuple):
    """(ties, floor_used): pairs swapped inside the near-tie band, and whether the near-zero
    floor of the band was needed to accept them."""
    __slots__ = ()

    def __new__(cls, ties=0, floor_used=False):
        return super().__new__(cls, (ties, floor_used))

    ties = property(lambda self: self[0])
    floor_used = property(lambda self: self[1])


def check_selection(gpu_row, scores: np.ndarray, k: int, pos: int) -> SelectionCheck:
    """Asserts the GPU index row is a valid top-k of ``scores`` up to near-ties.

    Layout: the min(k, pos+1) selected positions first (any order), then -1 padding."""
    g = [int(x) for x in gpu_row]
    n = max(pos + 1, 0)
    m = min(k, n)
    assert len(g) == k, f"row width {len(g)} != {k}"
    assert all(x >= 0 for x in g[:m]), "padding before the end of the selection"
    assert all(x == -1 for x in g[m:]), "entries after the selection are not -1 padding"
    valid = g[:m]
    assert len(set(valid)) == len(valid), "duplicate indices"
    assert all(0 <= x <= pos for x in valid), "index beyond the causal limit"
    if n == 0:
        return SelectionCheck()
    exact = set(oracle.select_topk(scores, k).tolist())
    diff = exact.symmetric_difference(valid)
    if not diff:
        return SelectionCheck()
    kth = float(np.sort(scores)[::-1][m - 1])
    rms = math.sqrt(float(np.mean(scores ** 2)))
    band = NEAR_TIE_REL * abs(kth)
    floor = NEAR_TIE_REL * NEAR_ZERO_FRAC * rms if abs(kth) < NEAR_ZERO_FRAC * rms else 0.0
    dist = [abs(scores[s] - kth) for s in diff]
    bad = [d for d in dist if d > max(band, floor)]
    assert not bad, (f"{len(bad)} selections differ beyond the near-tie band (k-th={kth}, band={band}, "
                     f"floor={floor}, worst={max(bad)})")
    return SelectionCheck(len(diff) // 2, any(d > band for d in dist))


def compare_attention(out_gpu: np.ndarray, lse_gpu: np.ndarray, out_ref: np.ndarray, lse_ref: np.ndarray):
    """max-abs of out, relative L2 of out per query row (the leading axis of [rows, H, d_v]) and
    over all rows, max-abs of lse (finite entries), asserted against the bounds."""
    out_gpu, out_ref = np.asarray(out_gpu, np.float64), np.asarray(out_ref, np.float64)
    if out_gpu.ndim == 2:
        out_gpu, out_ref = out_gpu[None], out_ref[None]
        lse_gpu, lse_ref = np.asarray(lse_gpu)[None], np.asarray(lse_ref)[None]
    d = out_gpu - out_ref
    max_abs = float(np.abs(d).max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(out_ref), 1e-30)) if d.size else 0.0
    row_rel = 0.0
    for r in range(d.shape[0]):
        nr = float(np.linalg.norm(out_ref[r]))
        nd = float(np.linalg.norm(d[r]))
        row_rel = max(row_rel, nd / nr if nr > 0 else (0.0 if nd == 0 else math.inf))
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), "lse finiteness differs"
    assert not np.isnan(out_gpu).any(), "NaN in out"
    lse_err = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert max_abs <= OUT_MAX_ABS, f"out max-abs {max_abs}"
    assert rel <= OUT_REL_L2, f"out rel-L2 {rel}"
    assert row_rel <= OUT_REL_L2, f"out rel-L2 of one query row {row_rel}"
    assert lse_err <= LSE_MAX_ABS, f"lse max-abs {lse_err}"
    return max_abs, max(rel, row_rel), lse_err
