"""The seeded synthetic inputs (moe_inputs.py): determinism, independent streams, the stated
distributions, and the Zipf(1.1) routing recipe (Gumbel-max over log-popularity draws the top
choice with probability p_e)."""
import numpy as np
import torch

import moe_inputs as mi


def test_streams_are_deterministic_and_independent():
    wl = mi.WORKLOADS["tiny"]
    assert np.array_equal(mi.activations(wl, 1, 2), mi.activations(wl, 1, 2))
    assert not np.array_equal(mi.activations(wl, 1, 2), mi.activations(wl, 1, 3))
    assert not np.array_equal(mi.activations(wl, 1, 2), mi.activations(wl, 2, 2))
    assert not np.array_equal(mi.router_logits(wl, 0, 0), mi.router_logits(wl, 0, 1))
    a13, a2 = mi.expert_weights(wl, 0, 3)
    b13, b2 = mi.expert_weights(wl, 0, 3)
    c13, _ = mi.expert_weights(wl, 0, 4)
    assert np.array_equal(a13, b13) and np.array_equal(a2, b2) and not np.array_equal(a13, c13)


def test_bf16_conversion_is_round_to_nearest_even():
    # halfway cases between two bf16 values round to the even mantissa
    lo = np.float32(1.0)
    ulp = np.float32(2.0 ** -7)
    vals = np.array([lo + ulp / 2, lo + ulp + ulp / 2, -(lo + ulp / 2), 3.0e38, 1e-40], np.float32)
    bits = mi.to_bf16_bits(vals)
    assert bits[0] == 0x3F80            # 1 + ulp/2 -> 1 (even)
    assert bits[1] == 0x3F82            # 1 + 3 ulp/2 -> 1 + 2 ulp (even)
    assert bits[2] == 0xBF80
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)
    back = mi.bf16_bits_to_f32(bits)
    assert back[0] == 1.0 and back[1] == np.float32(1.0 + 2 * 2.0 ** -7)


def test_weight_and_activation_distributions():
    wl = mi.Workload("d", H=512, I=256, E=2, k=1, T=64, w_std=0.02)
    w13, w2 = mi.expert_weights(wl, 0, 0)
    for w in (w13, w2):
        f = mi.bf16_bits_to_f32(w).astype(np.float64)
        assert abs(f.mean()) < 0.02 * 0.02
        assert abs(f.std() / 0.02 - 1.0) < 0.02
    x = mi.bf16_bits_to_f32(mi.activations(wl)).astype(np.float64)
    assert abs(x.mean()) < 0.02 and abs(x.std() - 1.0) < 0.02


def test_zipf_routing_draws_the_top_choice_with_its_popularity():
    wl = mi.Workload("z", H=256, I=128, E=64, k=8, T=20000, routing="zipf")
    logp = mi.zipf_log_popularity(wl, 0)
    p = np.exp(logp)
    assert abs(p.sum() - 1.0) < 1e-12
    # rank r (1-based) of the popularity order has p proportional to r^-1.1
    ps = np.sort(p)[::-1]
    r = np.arange(1, 65, dtype=np.float64)
    assert np.allclose(ps / ps[0], r ** -1.1, rtol=1e-12)
    # Gumbel-max: the arg-max of log p + Gumbel noise is expert e with probability p_e
    lg = mi.bf16_bits_to_f32(mi.router_logits(wl, 0, 0)).reshape(wl.T, wl.E)
    top1 = np.argmax(lg, axis=1)
    freq = np.bincount(top1, minlength=wl.E) / wl.T
    for e in np.argsort(-p)[:4]:
        sigma = np.sqrt(p[e] * (1 - p[e]) / wl.T)
        assert abs(freq[e] - p[e]) < 5 * sigma + 2e-3, (e, freq[e], p[e])
    # top-k counts follow the popularity order (the skew the prefill workload relies on)
    topk = np.argsort(-lg, axis=1, kind="stable")[:, : wl.k]
    counts = np.bincount(topk.ravel(), minlength=wl.E)
    rank_p = np.argsort(np.argsort(-p))
    rank_c = np.argsort(np.argsort(-counts))
    rho = np.corrcoef(rank_p, rank_c)[0, 1]
    assert rho > 0.95
