"""The output-error measure that smoke() applies, checked on the CPU against
the parity tests' own helper and on cases with a known answer."""
import numpy as np
import torch

from __graft_entry__ import output_error
from parity_helpers import out_err


def test_matches_the_parity_helper():
    rng = np.random.default_rng(3)
    ref = rng.standard_normal((64, 256)) * 3.0
    got = torch.tensor(ref + rng.standard_normal(ref.shape) * 1e-2).to(torch.bfloat16)
    got = got.double().numpy()
    assert output_error(got, ref) == out_err(got, ref, torch.bfloat16)


def test_exact_result_rounded_to_bf16_has_no_error():
    rng = np.random.default_rng(4)
    ref = rng.standard_normal((32, 128)) * 10.0
    got = torch.tensor(ref).to(torch.bfloat16).double().numpy()
    assert output_error(got, ref) == 0.0


def test_error_beyond_half_an_ulp_is_counted():
    ref = np.ones((4, 4))  # rms 1; half an ulp of 1.0 in bf16 is 2^-8
    got = ref.copy()
    got[1, 2] += 0.05
    assert abs(output_error(got, ref) - (0.05 - 2.0 ** -8)) < 1e-12
