"""The input generator's bfloat16 rounding (weights of the bf16 parity cases) against PyTorch's
float32 -> bfloat16 conversion (round to nearest, ties to even), on random values and on ties."""
import numpy as np
import torch

import synth


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 0.02,
                        rng.standard_normal(1000).astype(np.float32) * 1e4,
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 0.0, -0.0], np.float32)])
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    got = synth.round_bf16(a)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    # ties go to the even significand: 1 + 2^-8 -> 1, 1 + 3 * 2^-8 -> 1 + 2^-6
    assert got[-5] == 1.0 and got[-4] == 1.0 + 2 ** -6
