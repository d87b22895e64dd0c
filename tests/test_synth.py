"""The shared input generator: seeded, exact bf16 rounding, stated shapes."""

import numpy as np
import torch

from synth import (WORKLOADS, bf16_bits_from_f64, bf16_bits_to_f32, make_decode, make_prefill,
                   random_distinct_keys)


def test_bf16_rne_matches_torch_on_fp32_inputs():
    # for fp32-representable inputs there is no double rounding, so torch's
    # fp32 -> bf16 round-to-nearest-even is an independent reference
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-20, 20, 100000),
                        [0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38, -3.0e38]])
    x = x.astype(np.float32)
    ours = bf16_bits_from_f64(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (ours == ref).all()


def test_bf16_rne_ties_to_even_from_fp64():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert bf16_bits_to_f32(bf16_bits_from_f64(np.array([1 + 2.0 ** -8])))[0] == 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 and 1+2^-6: even is 1 + 2^-6
    assert bf16_bits_to_f32(bf16_bits_from_f64(np.array([1 + 3 * 2.0 ** -8])))[0] == 1 + 2.0 ** -6
    # just above the halfway point rounds up (fp64 sees it; fp32 would not)
    v = 1 + 2.0 ** -8 + 2.0 ** -40
    assert bf16_bits_to_f32(bf16_bits_from_f64(np.array([v])))[0] == 1 + 2.0 ** -7


def test_prefill_is_seeded_and_shaped():
    a = make_prefill("causal_1k_h64", T_q=8, T_k=40, q_offset=32)
    b = make_prefill("causal_1k_h64", T_q=8, T_k=40, q_offset=32)
    assert a["q"].shape == (8, 64, 128) and a["k"].shape == (40, 128) and a["w"].shape == (8, 64)
    assert a["q"].dtype == np.uint16 and a["w"].dtype == np.float32
    assert all((a[n] == b[n]).all() for n in ("q", "k", "w"))
    c = make_prefill("chunk_1m_h64", T_q=4, T_k=30, q_offset=26)
    assert (c["w"] < 0).any() and (c["w"] > 0).any()


def test_visible_pair_counts_of_workloads():
    assert WORKLOADS["causal_1k_h64"].visible_pairs == 1024 * 1025 // 2
    assert WORKLOADS["chunk_128k_h32"].visible_pairs == 1_040_191_488
    assert WORKLOADS["chunk_1m_h64"].visible_pairs == 4_286_580_736
    assert WORKLOADS["decode_64x128k_h64"].visible_pairs == 64 * 131072


def test_decode_shapes_and_lengths():
    x = make_decode("decode_64x128k_h64", B=3, t_cap=50, seq_len=[50, 7, 0])
    assert x["k"].shape == (3, 50, 128) and x["q"].shape == (3, 64, 128)
    assert x["seq_len"].tolist() == [50, 7, 0]


def test_random_distinct_keys():
    s = random_distinct_keys(1, 0, 100, 60, exclude=np.arange(10))
    assert len(set(s.tolist())) == 60 and s.min() >= 10 and s.max() < 100


def test_recipes_match_their_stated_distributions():
    # w ~ N(0, 1/8) (variance 1/8); the 1M-chunk recipe draws |N(0, 1/8)| with a
    # negative sign at probability 0.4
    x = make_prefill("causal_16k_h64", T_q=2048, T_k=2048, q_offset=0, seed=5)
    assert abs(float(x["w"].astype(np.float64).var()) - 1.0 / 8.0) < 0.01
    assert abs(float(x["w"].mean())) < 0.01
    y = make_prefill("chunk_1m_h64", T_q=2048, T_k=4096, q_offset=2048, seed=6)
    neg = float((y["w"] < 0).mean())
    assert abs(neg - 0.4) < 0.02
    assert abs(float((y["w"].astype(np.float64) ** 2).mean()) - 1.0 / 8.0) < 0.01


def test_lowrank_keys_live_near_a_rank_16_subspace():
    # k = U z + 0.3 e with U (128 x 16): the energy outside the top 16
    # directions is the isotropic noise, about 0.09 * 112 / (128 + 0.09 * 128)
    from synth import bf16_bits_to_f32
    x = make_prefill("causal_16k_h64", T_q=1, T_k=4096, q_offset=4095, seed=8)
    k = bf16_bits_to_f32(x["k"]).astype(np.float64)
    s = np.linalg.svd(k, compute_uv=False) ** 2
    outside = float(s[16:].sum() / s.sum())
    assert 0.04 < outside < 0.11
    # the gauss recipe has no such structure
    g = make_prefill("causal_1k_h64", T_q=1, T_k=1024, q_offset=1023, seed=9)
    sg = np.linalg.svd(bf16_bits_to_f32(g["k"]).astype(np.float64), compute_uv=False) ** 2
    assert float(sg[16:].sum() / sg.sum()) > 0.7
