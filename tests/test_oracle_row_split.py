"""The full-size parity tests run the oracle on whole heads with their input
rows split over worker processes; that split must give exactly the oracle's
one-call S (the per-range maxima merge by an exact max)."""
import math

import numpy as np
import torch

from kvz_testutil import f64, oracle_head_rows_parallel
from oracle import kvz_oracle as orc


def test_row_split_equals_one_call():
    g = torch.Generator().manual_seed(5)
    G, n_c, n_in, d = 3, 300, 1000, 32
    Q = torch.randn((G, n_in, d), generator=g).to(torch.bfloat16)
    Kc = (torch.randn((n_c, d), generator=g) * 2).to(torch.bfloat16)
    Ki = torch.randn((n_in, d), generator=g).to(torch.bfloat16)
    scale = float(np.float32(1.0 / math.sqrt(d)))
    whole = orc.score(f64(Q), f64(Kc), f64(Ki), scale)
    split = oracle_head_rows_parallel(Q, Kc, Ki, scale, rows_per_job=96, row_block=17)
    np.testing.assert_array_equal(split, whole)
