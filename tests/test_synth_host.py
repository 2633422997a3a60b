"""The C twin of the seeded generator (synth/hostgen.c) against the NumPy
definition: bit for bit on scattered coordinates, in fp32 and bf16, and the
threaded amax against NumPy's max over the same whole tensor."""
import numpy as np
import pytest

import synth
from synth import fast


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_twin_draws_equal_numpy_bit_for_bit(dtype):
    rng = np.random.default_rng(1)
    for _ in range(6):
        seed = int(rng.integers(0, 2 ** 63))
        stream, layer, b, h = (int(rng.integers(0, 4)), int(rng.integers(0, 4096)),
                               int(rng.integers(0, 256)), int(rng.integers(0, 256)))
        pos = rng.integers(0, 2 ** 24, size=3000)
        D = int(rng.choice([64, 128, 200]))
        a = fast.normal(seed, stream, layer, b, pos, h, D, dtype)
        ref = synth.normal(seed, stream, layer, b, pos[:, None], h, np.arange(D)[None, :], dtype)
        assert np.array_equal(a.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_twin_amax_equals_numpy_max(dtype):
    for batch, pos0, n_pos, H, D in [(3, 17, 700, 5, 64), (1, 0, 1, 2, 128), (2, 5000, 33, 8, 128)]:
        K = synth.kv_tokens(9, 1, 4, batch, pos0, n_pos, H, D, dtype)
        want = np.abs(K).max(axis=(0, 1, 3))
        got = fast.amax(9, 1, 4, batch, pos0, n_pos, H, D, dtype)
        assert np.array_equal(got, want)
