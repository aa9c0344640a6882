"""The seeded input generator: determinism, independence of streams, recipe."""
import numpy as np

from recurrent_state_memory_b200 import inputs as I


def test_streams_are_deterministic_and_order_free():
    a = I.normal(7, "q", (3, 5))
    _ = I.normal(7, "k", (1000,))
    b = I.normal(7, "q", (3, 5))
    assert np.array_equal(a, b)
    assert not np.array_equal(a, I.normal(8, "q", (3, 5)))
    assert not np.array_equal(a, I.normal(7, "k", (3, 5)))


def test_blocked_generation_matches_single_block():
    n = (1 << 21) + 17                      # spans two blocks of the threaded path
    x = I.normal(3, "v", (n,))
    y = I._normal_block(3, "v", 0, n)
    assert np.array_equal(x, y)


def test_normal_moments():
    x = I.normal(1, "m", (1 << 20,))
    assert abs(x.mean()) < 5e-3 and abs(x.std() - 1.0) < 5e-3


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.14159265], dtype=np.float32)
    r = I.bf16_bits_to_f32(I.to_bf16_bits(x))
    assert r[0] == 1.0 and r[1] == 1.0                       # tie rounds to even
    assert r[2] == np.float32(1.0 + 4 * 2 ** -8)             # tie rounds up to even
    assert r[3] == -2.5
    assert abs(r[4] - 3.140625) < 1e-7


def test_fwd_recipe():
    p = I.make_fwd(B=2, T=70, H=3, dk=32, dv=16, dtype="bf16", seed=5, rotation=True, s0_std=0.02)
    q = p.widened("q")
    assert q.shape == (2, 70, 3, 32) and p.q.dtype == np.uint16
    assert np.allclose(np.linalg.norm(q, axis=-1), 1.0, atol=2e-2)
    assert p.g.shape == (2, 70, 3, 16) and p.theta.shape == (2, 70, 3, 16)
    assert np.all(np.abs(p.theta) <= np.pi) and np.all((p.beta > 0) & (p.beta < 1))
    assert abs(p.S0.std() - 0.02) < 2e-3
    s = p.head_slice(1, 2)
    assert np.array_equal(s.q[0, :, 0], p.q[1, :, 2]) and np.array_equal(s.S0[0, 0], p.S0[1, 2])
    slow = I.make_fwd(B=1, T=64, H=1, dk=32, dv=32, dtype="f32", seed=2, gate="slow")
    assert abs(slow.g.mean() + 2.0) < 0.1          # a = -x, x ~ N(2, 1)
