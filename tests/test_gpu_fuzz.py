"""Layer shapes chosen to reach every path of the library, run through the
same staged-and-fused parity check as the named workloads: logits, selection
and flags, dispatch, expert rows and combine against the oracle; the fused
layer against the oracle and, bit for bit, against the staged calls.

Paths covered (by the rules the host applies): the one-launch small router
(T <= 256), the CUDA-core split-K router (256 < T < 512) and the tensor-core
router (bf16, T >= 512); the one-block and multi-kernel dispatch; the
CUDA-core FFN (f32, or d or F not a multiple of 128); single-CTA tensor-core
GEMMs with 64-, 128- and 256-token tiles, with and without a split
contraction; and the CTA-pair GEMMs with their dynamic schedule. Also the
narrowest widths the limits allow, a single routed expert (a dense FFN), and
one token past each batch-size threshold.
"""
import pytest

from moe_synth import MoEShape
from test_gpu_parity import run_staged_and_fused

pytestmark = pytest.mark.gpu

SHAPES = [
    # tiny batches: split contraction in both GEMMs, small router
    MoEShape("fz_t1", T=1, d=256, n_routed=12, n_zero=3, top_k=4, ffn=256),
    MoEShape("fz_t3_nozero", T=3, d=384, n_routed=5, n_zero=0, top_k=2, ffn=128),
    # 64-token tiles
    MoEShape("fz_t17_zipf", T=17, d=256, n_routed=33, n_zero=7, top_k=6, ffn=384,
             routing="zipf"),
    MoEShape("fz_t64", T=64, d=512, n_routed=24, n_zero=8, top_k=8, ffn=256),
    # 128-token tiles, small router
    MoEShape("fz_t130", T=130, d=256, n_routed=9, n_zero=2, top_k=3, ffn=512),
    # CUDA-core split-K router
    MoEShape("fz_t300", T=300, d=384, n_routed=20, n_zero=4, top_k=5, ffn=256),
    # tensor-core router, single-CTA GEMMs
    MoEShape("fz_t700_zipf", T=700, d=256, n_routed=16, n_zero=4, top_k=4, ffn=384,
             routing="zipf"),
    # CTA pairs (T > 1024, d and F multiples of 256)
    MoEShape("fz_t1030_pairs", T=1030, d=512, n_routed=12, n_zero=3, top_k=3, ffn=512),
    MoEShape("fz_t1300_pairs_zipf", T=1300, d=256, n_routed=7, n_zero=1, top_k=2, ffn=768,
             routing="zipf"),
    # T > 1024 but d not a multiple of 256: single-CTA 256-token tiles
    MoEShape("fz_t1100_single", T=1100, d=384, n_routed=8, n_zero=2, top_k=2, ffn=384),
    # CUDA-core FFN in bf16 (d, F not multiples of 128) and in f32
    MoEShape("fz_t90_simt", T=90, d=200, n_routed=6, n_zero=2, top_k=2, ffn=136),
    MoEShape("fz_t50_f32", T=50, d=128, n_routed=5, n_zero=1, top_k=3, ffn=128,
             act_dtype="f32"),
    # the narrowest layers the limits allow (router boxes wider than the rows)
    MoEShape("fz_d8", T=33, d=8, n_routed=3, n_zero=1, top_k=2, ffn=8),
    MoEShape("fz_d16_f32", T=20, d=16, n_routed=4, n_zero=2, top_k=3, ffn=24,
             act_dtype="f32"),
    # one routed expert: a dense SwiGLU FFN on tensor cores, with and without
    # zero experts beside it
    MoEShape("fz_dense", T=100, d=256, n_routed=1, n_zero=0, top_k=1, ffn=256),
    MoEShape("fz_n1_zero", T=70, d=128, n_routed=1, n_zero=3, top_k=2, ffn=128),
    # one token past each batch-size threshold: small router (256), tensor-core
    # router (512), CTA pairs (1024), one-block dispatch (4096)
    MoEShape("fz_t257", T=257, d=128, n_routed=6, n_zero=2, top_k=2, ffn=128),
    MoEShape("fz_t512", T=512, d=128, n_routed=6, n_zero=2, top_k=2, ffn=128),
    MoEShape("fz_t1025_pairs", T=1025, d=256, n_routed=4, n_zero=1, top_k=1, ffn=256),
    MoEShape("fz_t4097", T=4097, d=128, n_routed=8, n_zero=2, top_k=2, ffn=128),
    # tensor-core router with 103 experts: three 40-expert plane tiles, the
    # last one and its last quarter only partly used
    MoEShape("fz_t600_e103", T=600, d=256, n_routed=91, n_zero=12, top_k=5, ffn=128),
]


@pytest.mark.parametrize("i", range(len(SHAPES)), ids=[s.name for s in SHAPES])
def test_path_shapes(i):
    run_staged_and_fused(SHAPES[i], 100 + i)
