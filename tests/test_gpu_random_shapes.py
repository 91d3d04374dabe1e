"""Seeded random shapes through the one-call path, on the bf16 metadata and on
the fp8 copy, every unit against the oracle: kv-heads 1-8 (3 included), group
sizes 1-16, D 64/128/256, ragged lengths with empty and one-page sequences,
prefix and window from 0 up, budgets from one page up, and up to 40 units (so
both the single launch and the separate kernels run, and the page-major and
ring fp8 scorers)."""
import random

import pytest

from long_context_decoding_b200 import workloads as wl
from test_gpu_fp8 import Fp8Run, check_fp8
from test_gpu_parity import Run, check_one_call, small

pytestmark = pytest.mark.gpu


def _shape(i):
    r = random.Random(1000 + i)
    Hkv = r.choice([1, 2, 3, 4, 8])
    G = r.choice([1, 2, 4, 8, 16])
    D = r.choice([64, 128, 256])
    B = r.randint(1, max(1, 40 // Hkv))
    lens = tuple(r.choice([0, 1, 15, 16, 17]) if r.random() < 0.15 else r.randint(18, 6000)
                 for _ in range(B))
    return dict(B=B, Hq=Hkv * G, Hkv=Hkv, D=D, lens=lens, prefix=r.choice([0, 1, 16, 40, 128]),
                window=r.choice([0, 15, 16, 100, 512]), budget=r.choice([16, 64, 160, 480, 1024]),
                seed=7 + i)


@pytest.mark.parametrize("i", range(12))
def test_random_shape_one_call(i, cuda):
    check_one_call(Run(wl.make_case(small(**_shape(i)), cuda)))


@pytest.mark.parametrize("i", range(12, 20))
def test_random_shape_fp8(i, cuda):
    check_fp8(Fp8Run(wl.make_case(small(**_shape(i)), cuda)))
