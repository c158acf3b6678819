"""The seeded input generators: statistics, bf16 rounding and the workload recipes."""
import numpy as np
import torch

import msa_synth as syn


def test_irwin_hall_moments_and_determinism():
    x = syn.fill(11, syn.STREAM_K, 2, 0, 0, 512, 1024)
    assert abs(float(x.mean())) < 0.01
    assert abs(float(x.var()) - 1.0) < 0.01
    assert float(np.abs(x).max()) <= 2 * np.sqrt(3.0) + 1e-6     # Irwin-Hall(4) support
    y = syn.fill(11, syn.STREAM_K, 2, 0, 100, 10, 1024)
    assert np.array_equal(x[100:110], y)                          # counter-based: any row range


def test_bf16_rounding_matches_torch():
    x = syn.fill(1, syn.STREAM_V, 0, 0, 0, 64, 1024) * np.float32(3.7)
    mine = syn.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    assert np.array_equal(syn.bf16_bits_to_f32(mine), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_document_length_laws():
    u = syn.doc_lengths_uniform(0, 64, 200, 1000)
    assert u.min() >= 200 and u.max() <= 1000 and 25_000 < u.sum() < 50_000
    ln = syn.doc_lengths_lognormal(1, 10_000)
    assert 850 < np.median(ln) < 950 and ln.min() >= 64 and ln.max() <= 8192
    ex = syn.doc_lengths_exact_total(3, 1000, 1_000_000)
    assert ex.sum() == 1_000_000 and np.all(ex % 64 == 0)


def test_topics_and_targets():
    t = syn.topics(0, 10)
    np.testing.assert_allclose(np.linalg.norm(t.astype(np.float64), axis=1), 4.0, rtol=1e-6)
    tg = syn.pick_targets(2, 100, 16)
    assert len(set(tg.tolist())) == 16 and tg.max() < 100
