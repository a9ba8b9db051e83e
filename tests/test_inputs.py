"""The seeded input generator that the oracle and the CUDA path share (hinm_inputs.py).

It holds none of the method's arithmetic, but every parity test reads its bytes, so its
recipe is pinned here: bf16 rounding against an independent implementation (torch's own
fp32 -> bf16 conversion, round to nearest even), exact widening, determinism, the draw
order, and the workloads' shapes and parameters.
"""
import numpy as np
import pytest

import hinm_inputs as hi

torch = pytest.importorskip("torch")


def _torch_bf16_bits(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_bf16_rounding_matches_torch_on_random_values():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100_000).astype(np.float32),
                        (rng.standard_normal(10_000) * 1e-30).astype(np.float32),
                        (rng.standard_normal(10_000) * 1e30).astype(np.float32)])
    np.testing.assert_array_equal(hi.f32_to_bf16_bits(a), _torch_bf16_bits(a))


def test_bf16_rounding_halfway_cases_go_to_even():
    # bit patterns exactly halfway between two bf16 values: the lower 16 bits are 0x8000
    u = np.array([0x3F808000,   # 1.00390625: between 0x3F80 (even) and 0x3F81 -> 0x3F80
                  0x3F818000,   # between 0x3F81 (odd) and 0x3F82 (even)     -> 0x3F82
                  0xBF808000,   # negative, even below                        -> 0xBF80
                  0x3F808001,   # just above halfway                          -> 0x3F81
                  0x3F807FFF,   # just below halfway                          -> 0x3F80
                  0x00008000,   # smallest subnormal region, halfway to even  -> 0x0000
                  0x7F7FFFFF],  # largest finite fp32: rounds up to +inf      -> 0x7F80
                 dtype=np.uint32)
    want = np.array([0x3F80, 0x3F82, 0xBF80, 0x3F81, 0x3F80, 0x0000, 0x7F80], dtype=np.uint16)
    got = hi.f32_to_bf16_bits(u.view(np.float32))
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(got, _torch_bf16_bits(u.view(np.float32)))


def test_bf16_widening_is_exact_and_round_trips():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    f = hi.bf16_bits_to_f32(bits)
    finite = np.isfinite(f)
    np.testing.assert_array_equal(hi.f32_to_bf16_bits(f[finite]), bits[finite])
    np.testing.assert_array_equal(f.view(np.uint32) & 0xFFFF, np.zeros(f.size, np.uint32))


def test_draws_are_deterministic_and_in_the_stated_order():
    a = hi.custom(64, 48, 16, 64, seed=5, t_s=0.5, v_s=None, random_perm=True)
    b = hi.custom(64, 48, 16, 64, seed=5, t_s=0.5, v_s=None, random_perm=True)
    np.testing.assert_array_equal(a.W_bits, b.W_bits)
    np.testing.assert_array_equal(a.X_bits, b.X_bits)
    np.testing.assert_array_equal(a.perm, b.perm)
    # the recipe: W (fp32 normal x 0.02), then X (normal), then the permutation
    rng = np.random.Generator(np.random.PCG64(5))
    W = rng.standard_normal((64, 48), dtype=np.float32) * np.float32(0.02)
    X = rng.standard_normal((48, 16), dtype=np.float32)
    perm = rng.permutation(48)
    np.testing.assert_array_equal(a.W_bits, hi.f32_to_bf16_bits(W))
    np.testing.assert_array_equal(a.X_bits, hi.f32_to_bf16_bits(X))
    np.testing.assert_array_equal(a.perm, perm)
    c = hi.custom(64, 48, 16, 64, seed=6, t_s=0.5, v_s=None, random_perm=True)
    assert not np.array_equal(a.W_bits, c.W_bits)


def test_outliers_and_identity_order():
    w = hi.custom(256, 256, 8, 128, seed=3, t_s=0.5, v_s=0.0, outlier_frac=0.01)
    np.testing.assert_array_equal(w.perm, np.arange(256))
    big = np.abs(hi.bf16_bits_to_f32(w.W_bits)) > 0.02 * 10 * 0.5
    frac = big.mean()
    assert 0.003 < frac < 0.02  # about 1 % of the weights were scaled by 10


def test_workload_shapes_and_parameters():
    assert (hi.tiny_hinm().M, hi.tiny_hinm().K, hi.tiny_hinm().N, hi.tiny_hinm().T) == (256, 256, 16, 64)
    cases = {
        "pure24": (hi.pure24, (4096, 4096, 2048, 128, 0.5, 0.0)),
        "up": (hi.hinm_up_proj, (11008, 4096, 4096, 128, 0.75, 0.6)),
        "decode": (hi.decode_down_proj, (4096, 11008, 16, 128, 0.625, 0.4)),
    }
    for name, (make, want) in cases.items():
        # small replicas through the same constructors: only the shapes differ
        w = make(M=256, K=256, N=16) if name != "decode" else make(M=256, K=512, N=16)
        assert (w.T, w.t_s, w.v_s) == want[3:], name
    up = hi.hinm_up_proj(M=256, K=256, N=16)
    assert not np.array_equal(up.perm, np.arange(256))  # the up-projection's order is random
    s = hi.llama_sweep_layer(3, "down", 512, 0.625)
    assert (s.M, s.K, s.N, s.T, s.t_s, s.v_s) == (4096, 11008, 512, 128, 0.625, None)
    assert s.meta["seed"] == 1000 * 3 + 6
