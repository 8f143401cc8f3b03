"""Plant plausible mistakes in the oracle (CPU only) and check that the pins catch each one.

A pin set that passes on a wrong oracle would not be evidence; every mutant below
must make at least one test of ``test_oracle_pins`` fail.
"""
import numpy as np
import pytest

import oracle
import oracle.dsa_oracle as od
import tests.test_oracle_pins as pins


def _relu_after_sum(q, w, k):
    return np.maximum(w @ (q @ k.T), 0.0)


def _no_relu(q, w, k):
    return w @ (q @ k.T)


def _unweighted(q, w, k):
    return np.maximum(q @ k.T, 0.0).sum(0)


def _abs_weights(q, w, k):
    return np.abs(w) @ np.maximum(q @ k.T, 0.0)


def _ties_to_higher(scores, k):
    n = scores.shape[0]
    return np.lexsort((-np.arange(n), -scores))[: min(k, n)]


def _bottom_k(scores, k):
    n = scores.shape[0]
    return np.lexsort((np.arange(n), scores))[: min(k, n)]


def _value_is_rope_end(q, kv, d_v, tau):
    out, lse = od.__dict__["_orig_attn"](q, kv, d_v, tau)
    if kv.shape[0] == 0:
        return out, lse
    z = tau * (q @ kv.T)
    p = np.exp(z - z.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    return p @ kv[:, -d_v:], lse


def _lse_without_tau(q, kv, d_v, tau):
    out, lse = od.__dict__["_orig_attn"](q, kv, d_v, tau)
    if kv.shape[0] == 0:
        return out, lse
    z = q @ kv.T
    return out, z.max(1) + np.log(np.exp(z - z.max(1, keepdims=True)).sum(1))


def _softmax_over_heads(q, kv, d_v, tau):
    if kv.shape[0] == 0:
        return np.zeros((q.shape[0], d_v)), np.full(q.shape[0], -np.inf)
    z = tau * (q @ kv.T)
    p = np.exp(z - z.max(0, keepdims=True))
    l = p.sum(0, keepdims=True)
    return (p / l) @ kv[:, :d_v], z.max(1) + np.log(np.exp(z - z.max(1, keepdims=True)).sum(1))


def _no_scale_e4m3(codes, scale=None):
    return od._E4M3[np.asarray(codes, dtype=np.uint8)]


def _e4m3_bias_8(codes, scale=None):
    return od.__dict__["_orig_e4m3"](codes, scale) * 0.5


def _driver(q_of, k_of):
    """indexer_topk_row with the decoding of q and k replaced (planted scale mistakes)."""
    def row(q_codes, q_scale, w_bits, k_codes, k_scale, pos, topk):
        if pos < 0:
            return np.zeros(0, dtype=np.int64), np.zeros(0)
        q = q_of(q_codes, q_scale)
        k = k_of(k_codes, np.asarray(k_scale, dtype=np.float64), q_scale, pos)
        scores = od.index_scores(q, od.decode_bf16(w_bits), k)
        return od.select_topk(scores, topk).astype(np.int64), scores
    return row


def _q_scaled(q_codes, q_scale):
    return od.decode_e4m3(q_codes, np.full(q_codes.shape[0], q_scale))


MUTANTS_DRIVER = {
    # keys decoded without their scales
    "driver_k_scale_dropped": _driver(_q_scaled, lambda kc, ks, qs, pos: od.decode_e4m3(kc[: pos + 1])),
    # every key takes the scale of the next token
    "driver_k_scale_shifted": _driver(
        _q_scaled, lambda kc, ks, qs, pos: od.decode_e4m3(kc[: pos + 1], np.roll(ks, -1)[: pos + 1])),
    # the query's scale applied to the keys (query unscaled, key scales unused)
    "driver_q_scale_on_keys": _driver(
        lambda qc, qs: od.decode_e4m3(qc),
        lambda kc, ks, qs, pos: od.decode_e4m3(kc[: pos + 1], np.full(pos + 1, qs))),
}

def _target_logits_summed(q, kv, tau):
    z = (tau * (q @ kv.T)).sum(0)                 # heads summed before the softmax
    e = np.exp(z - z.max())
    return e / e.sum()


def _target_unnormalised_heads(q, kv, tau):
    z = tau * (q @ kv.T)
    a = np.exp(z - z.max()).sum(0)                # no per-head softmax normalisation
    return a / a.sum()


def _kl_reversed(p, scores):
    q = np.exp(scores - scores.max())
    q /= q.sum()
    nz = q > 0
    return float(np.sum(q[nz] * (np.log(q[nz]) - np.log(np.maximum(p[nz], 1e-300)))))


def _kl_log2(p, scores):
    return od.__dict__["_orig_kl"](p, scores) / np.log(2.0)


def _kl_row_keeps_padding(q_bits, kv_bits, idx, sc, tau):
    idx = np.asarray(idx, dtype=np.int64)
    sel = np.where(idx >= 0, idx, 0)
    p = od.attention_head_sum_target(od.decode_bf16(q_bits), od.decode_bf16(kv_bits[sel]), tau)
    return od.indexer_kl(p, np.asarray(sc, dtype=np.float64))


def _masked_ignores_mask(q, kv, mask, d_v, tau):
    return od.sparse_mla_attention(q, kv, d_v, tau)


def _masked_zero_logits(q, kv, mask, d_v, tau):
    z = np.where(np.asarray(mask)[None, :], tau * (q @ kv.T), 0.0)     # masked logits 0, not -inf
    e = np.exp(z - z.max(1, keepdims=True))
    return (e @ kv[:, :d_v]) / e.sum(1, keepdims=True), z.max(1) + np.log(e.sum(1))


MUTANTS = {
    **{n: ("indexer_topk_row", f) for n, f in MUTANTS_DRIVER.items()},
    "masked_mode_ignores_mask": ("masked_dense_mqa_attention", _masked_ignores_mask),
    "masked_logits_zero_not_minus_inf": ("masked_dense_mqa_attention", _masked_zero_logits),
    "target_logits_summed_over_heads": ("attention_head_sum_target", _target_logits_summed),
    "target_heads_not_normalised": ("attention_head_sum_target", _target_unnormalised_heads),
    "kl_reversed": ("indexer_kl", _kl_reversed),
    "kl_in_bits": ("indexer_kl", _kl_log2),
    "kl_row_keeps_padding": ("indexer_kl_row", _kl_row_keeps_padding),
    "relu_after_sum": ("index_scores", _relu_after_sum),
    "no_relu": ("index_scores", _no_relu),
    "unweighted_heads": ("index_scores", _unweighted),
    "abs_weights": ("index_scores", _abs_weights),
    "ties_to_higher": ("select_topk", _ties_to_higher),
    "bottom_k": ("select_topk", _bottom_k),
    "value_from_rope_end": ("sparse_mla_attention", _value_is_rope_end),
    "lse_without_tau": ("sparse_mla_attention", _lse_without_tau),
    "softmax_over_heads": ("sparse_mla_attention", _softmax_over_heads),
    "scale_dropped": ("decode_e4m3", _no_scale_e4m3),
    "e4m3_wrong_bias": ("decode_e4m3", _e4m3_bias_8),
}

PIN_TESTS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _run_pins():
    failed = []
    for fn in PIN_TESTS:
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        try:
            if params:
                names = [s.strip() for s in params[0].args[0].split(",")]
                for vals in params[0].args[1]:
                    fn(**dict(zip(names, vals if len(names) > 1 else (vals,))))
            else:
                fn()
        except Exception:
            failed.append(fn.__name__)
    return failed


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_planted_mistake(mutant, monkeypatch):
    name, fake = MUTANTS[mutant]
    monkeypatch.setitem(od.__dict__, "_orig_attn", od.sparse_mla_attention)
    monkeypatch.setitem(od.__dict__, "_orig_e4m3", od.decode_e4m3)
    monkeypatch.setitem(od.__dict__, "_orig_kl", od.indexer_kl)
    monkeypatch.setattr(od, name, fake)
    monkeypatch.setattr(oracle, name, fake)
    assert _run_pins(), f"no pin caught mutant {mutant}"


def test_unmutated_oracle_passes_every_pin():
    assert _run_pins() == []
