"""The output tolerance reading, shown on the CPU with the oracle alone.

The layer's outputs are stored in the activation format (bf16: 8 significant
bits). Rounding the EXACT result to bf16 moves an element by up to half an
ulp, 2^-8 of its magnitude, so any element beyond ~5 x rms can exceed a plain
2e-2 x rms bound with no arithmetic error at all. The parity tests therefore
measure the error beyond half an ulp of the output format (parity_helpers).
"""
import numpy as np
import torch

import oracle
from parity_helpers import OUT_RTOL_RMS, half_ulp, out_err, rel_rms_err


def test_exact_result_rounded_to_bf16_breaks_plain_bound_but_not_reading():
    # every slot on a zero expert: the exact output is x itself
    T, d = 64, 32
    g = torch.Generator().manual_seed(0)
    x = torch.randn(T, d, generator=g)
    x[5, 7] = 9.03125 - 2 ** -12  # one 9-sigma element just under a bf16 tie
    wr = torch.zeros(3, d)
    b = torch.tensor([-1e3, 0.0, 0.0])  # expert 0 routed, experts 1-2 zero
    wg = torch.zeros(1, 4, d)
    out, idx, _ = oracle.layer(x, wr, b, wg, wg, torch.zeros(1, d, 4), 1, 2, 1.0)
    assert np.all(idx >= 1)
    np.testing.assert_allclose(out, x.double().numpy(), rtol=0, atol=1e-15)
    stored = torch.from_numpy(out).to(torch.bfloat16).double().numpy()
    assert rel_rms_err(stored, out) > OUT_RTOL_RMS          # plain bound fails
    assert out_err(stored, out, torch.bfloat16) <= 1e-12     # reading: exact


def test_half_ulp_of_bf16():
    assert half_ulp(np.array([1.0]), torch.bfloat16)[0] == 2 ** -8
    assert half_ulp(np.array([9.0]), torch.bfloat16)[0] == 2 ** -5
    assert half_ulp(np.array([0.75]), torch.bfloat16)[0] == 2 ** -9
    v = np.random.default_rng(0).standard_normal(10000) * 3
    r = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(r - v) <= half_ulp(v, torch.bfloat16) * (1 + 1e-12))
