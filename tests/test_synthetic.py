"""The seeded input generator: exact integer mixing, determinism, row access, moments."""
import math

import numpy as np
import pytest
import torch

import oracle
import synthetic
from synthetic import _mix32, _stream_key, _words, mix32_int


def test_mixer_torch_matches_python_ints():
    xs = [0, 1, 2, 0x7FFFFFFF, 0x80000000, 0xFFFFFFFF, 123456789, 0xDEADBEEF]
    xs += list(np.random.default_rng(0).integers(0, 1 << 32, size=200, dtype=np.int64))
    t = _mix32(torch.tensor(xs, dtype=torch.int64))
    assert t.tolist() == [mix32_int(int(x)) for x in xs]


def test_words_handle_counters_beyond_32_bits():
    key = _stream_key(5, "q")
    flat = torch.tensor([3, (1 << 32) + 3, (1 << 34) + 3], dtype=torch.int64)
    h1, _ = _words(flat, key)
    assert len(set(h1.tolist())) == 3
    lo, hi = 3, 1
    ref = mix32_int((mix32_int(lo ^ key) + hi * 0x3C6EF35F + 0x1B873593) & 0xFFFFFFFF)
    assert h1[1].item() == ref


def test_rows_are_a_pure_function_of_the_counter():
    a = synthetic.normal_rows(7, "q", range(10, 20), 33, 1.0)
    b = synthetic.normal_rows(7, "q", [15, 10, 19], 33, 1.0)
    assert torch.equal(a[[5, 0, 9]], b)
    assert not torch.equal(a, synthetic.normal_rows(8, "q", range(10, 20), 33, 1.0))
    assert not torch.equal(a, synthetic.normal_rows(7, "kv", range(10, 20), 33, 1.0))


def test_moments_are_standard_normal_like():
    x = synthetic.normal_rows(1, "q", range(0, 512), 1024, 2.0).double()
    assert abs(x.mean().item()) < 0.01
    assert abs(x.std().item() - 2.0) < 0.01
    assert x.abs().max().item() <= 2.0 * math.sqrt(12.0) + 1e-5      # Irwin-Hall(4) bound


def test_e4m3_quantisation_uses_exact_power_of_two_scales():
    x = synthetic.normal_rows(3, "q_idx", range(0, 64), 256, 1.0)
    x[5] = 0.0
    codes, scale = synthetic.quantize_e4m3_rows(x)
    s = scale.double().numpy()
    m, _ = np.frexp(s)
    assert (m == 0.5).all()                                    # powers of two
    dec = oracle.decode_e4m3(codes.numpy(), scale.numpy())
    xd = x.double().numpy()
    amax = np.abs(xd).max(1)
    nz = amax > 0
    assert (amax[nz] / s[nz] < 256).all() and (amax[nz] / s[nz] >= 128).all()
    assert (dec[~nz] == 0).all() and (s[~nz] == 1).all()
    # round to nearest: within half an E4M3 step of the exact scaled value
    err = np.abs(dec - xd)
    assert (err <= np.maximum(np.abs(xd) * 2.0 ** -4, s[:, None] * 2.0 ** -10) + 1e-30).all()
    # and exactly the RNE cast of x / scale
    ref = torch.from_numpy(xd / s[:, None]).float().to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(ref, codes)


def test_e4m3_quantisation_with_amax_scales():
    x = synthetic.normal_rows(4, "k_idx", range(0, 64), 128, 1.0)
    x[7] = 0.0
    codes, scale = synthetic.quantize_e4m3_rows_amax(x)
    s = scale.double().numpy()
    xd = x.double().numpy()
    amax = np.abs(xd).max(1)
    nz = amax > 0
    assert (s > 0).all() and (s[~nz] == 1).all()
    np.testing.assert_allclose(s[nz], amax[nz] / 448.0, rtol=2.0 ** -24)   # amax/448 rounded to fp32
    m, _ = np.frexp(s[nz])
    assert (m != 0.5).sum() > 50                                            # general, not powers of two
    dec = oracle.decode_e4m3(codes.numpy(), scale.numpy())
    assert np.isfinite(dec).all() and (np.abs(dec) <= 448.0 * s[:, None] * (1 + 2.0 ** -20)).all()
    # within half an E4M3 step (plus the fp32 rounding of x / scale) of the exact value
    err = np.abs(dec - xd)
    assert (err <= np.maximum(np.abs(xd) * 2.0 ** -4, s[:, None] * 2.0 ** -10) * (1 + 1e-6) + 1e-30).all()
    # the row maximum maps to the top code
    top = np.abs(oracle.decode_e4m3(codes.numpy()))[nz].max(1)
    assert (top == 448.0).all()
    cfg = synthetic.config("tiny", n_q=16, max_len=16, fp8_scale="amax")
    qc, qs = synthetic.gen_q_idx(cfg, 2)
    ref_c, ref_s = synthetic.quantize_e4m3_rows_amax(
        synthetic.normal_rows(2, "q_idx", range(0, 16), cfg.n_idx_heads * cfg.idx_dim, cfg.q_idx_std))
    assert torch.equal(qc.reshape(16, -1), ref_c) and torch.equal(qs, ref_s)


def test_row_subsets_match_full_generation():
    cfg = synthetic.config("tiny", n_q=48, max_len=48)
    g = synthetic.gen_all(cfg, 9)
    qc, qs = synthetic.gen_q_idx(cfg, 9, tokens=[5, 17])
    assert torch.equal(qc, g["q_idx"][0, [5, 17]]) and torch.equal(qs, g["q_scale"][0, [5, 17]])
    kc, ks = synthetic.gen_k_idx(cfg, 9, b=0, s_range=range(3, 30))
    assert torch.equal(kc, g["k_idx"][0, 3:30]) and torch.equal(ks, g["k_scale"][0, 3:30])
    assert torch.equal(synthetic.gen_kv(cfg, 9, b=0, positions=[4, 2]), g["kv"][0, [4, 2]])
    assert torch.equal(synthetic.gen_q(cfg, 9, tokens=[7]), g["q"][0, [7]])
    assert torch.equal(synthetic.gen_w(cfg, 9, tokens=[7]), g["w"][0, [7]])


def test_decode_lengths_are_seeded_and_in_range():
    cfg = synthetic.config("decode")
    a, b = synthetic.lengths(cfg, 0), synthetic.lengths(cfg, 0)
    assert torch.equal(a, b) and a.shape == (64,)
    assert int(a.min()) >= 4096 and int(a.max()) <= 131072
    assert len(set(a.tolist())) > 60
    assert synthetic.lengths(synthetic.config("prefill_4k"), 0).tolist() == [4096]


def test_sample_rows_is_seeded_and_distinct():
    s = synthetic.sample_rows(1000, 20, 3, extra=[0, 999])
    assert s == synthetic.sample_rows(1000, 20, 3, extra=[0, 999])
    assert len(s) == 22 and 0 in s and 999 in s and len(set(s)) == 22


@pytest.mark.gpu
def test_cpu_and_cuda_generate_identical_bits():
    for name in ["tiny", "prefill_4k"]:
        cfg = synthetic.config(name, n_q=256, max_len=256) if name != "tiny" else synthetic.config(name)
        a = synthetic.gen_all(cfg, 21, "cpu")
        b = synthetic.gen_all(cfg, 21, "cuda")
        for k in a:
            ta, tb = a[k], b[k].cpu()
            if ta.dtype == torch.bfloat16:
                ta, tb = ta.view(torch.int16), tb.view(torch.int16)
            assert torch.equal(ta, tb), (name, k)
