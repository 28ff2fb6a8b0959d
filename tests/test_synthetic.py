"""The seeded input generators: determinism, bf16 rounding and the planted structure."""
import numpy as np

import synthetic as sy


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.00390625, 1.005859375, 1.0078125 + 2 ** -9, -2.5, 3.0e38], np.float32)
    bits = sy.bf16_round(x)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1.0); 1 + 1.5*2^-8 rounds up
    assert bits.tolist() == [0x3F80, 0x3F80, 0x3F81, 0x3F81, 0xC020, 0x7F62]
    np.testing.assert_array_equal(sy.bf16_bits_to_f32(bits)[:2], [1.0, 1.0])


def test_same_seed_same_bits_and_heads_independent():
    w = sy.workload("llama8b_gqa_32k", M=1024, Hq=4, Hkv=2, n_heavy=8)
    a = sy.layer_inputs(w, seed=7)
    b = sy.layer_inputs(w, seed=7)
    c = sy.layer_inputs(w, seed=8)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    assert not np.array_equal(a[0], c[0])
    q3, k3, v3 = sy.head_inputs(w, 3, seed=7)
    np.testing.assert_array_equal(q3, a[0][0, 3])
    np.testing.assert_array_equal(k3, a[1][0, 1])
    np.testing.assert_array_equal(v3, a[2][0, 1])


def test_heavy_tokens_and_shared_direction():
    w = sy.workload("tiny_1h_2k")
    q, k, _ = (sy.bf16_bits_to_f32(x).astype(np.float64) for x in sy.head_inputs(w, 0))
    # heavy keys carry +3u along the same direction the queries carry +1u
    u = q.mean(axis=0)
    u /= np.linalg.norm(u)
    proj = k @ u
    heavy = sy._heavy_positions(w, sy.DEFAULT_SEED, 0, 0)
    assert heavy[0] == 0 and len(set(heavy.tolist())) == w.n_heavy == 16
    rest = np.setdiff1d(np.arange(w.M), heavy)
    assert proj[heavy].mean() > 2.5 and abs(proj[rest].mean()) < 0.2


def test_slash_term_period():
    w = sy.workload("llama8b_gqa_32k", M=4096, Hq=1, Hkv=1, n_heavy=1)
    q, k, _ = (sy.bf16_bits_to_f32(x).astype(np.float64) for x in sy.head_inputs(w, 0))
    # q_i . k_j is ~0.25*C larger when i = j (mod 64)
    same = np.mean([q[i] @ k[i + 64 * 3] for i in range(0, 1000)])
    diff = np.mean([q[i] @ k[i + 64 * 3 + 5] for i in range(0, 1000)])
    assert same - diff > 0.15 * w.C


def test_video_grid_structure():
    w = sy.workload("video_dit_118k", M=3 * 4096, Hq=1, Hkv=1)
    q, k, _ = (sy.bf16_bits_to_f32(x).astype(np.float64) for x in sy.head_inputs(w, 0))
    same_frame = np.mean([q[i] @ k[i + 1] for i in range(0, 2000, 7)])
    same_pos = np.mean([q[i] @ k[i + 4096] for i in range(0, 2000, 7)])
    neither = np.mean([q[i] @ k[i + 4096 + 1] for i in range(0, 2000, 7)])
    assert same_frame - neither > 0.3 * w.C and same_pos - neither > 0.3 * w.C


def test_tau_vector():
    w = sy.workload("llama8b_gqa_256k")
    t = sy.tau_vector(w)
    assert t.shape == (32,) and t.dtype == np.float32
    assert (t >= 0.80).all() and (t <= 0.95).all() and len(set(t.tolist())) == 32
    np.testing.assert_array_equal(t, sy.tau_vector(w))
    assert (sy.tau_vector(sy.workload("llama8b_gqa_128k")) == np.float32(0.9)).all()


def test_video_length_is_whole_blocks():
    w = sy.workload("video_dit_118k")
    assert w.M == 29 * 4096 and w.M % w.block == 0 and w.nb == 928
