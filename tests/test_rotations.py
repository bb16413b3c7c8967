"""Host rotation generator of the library (lsh_attn_make_rotations) against the
repository's seeded generator: the same Philox4x32-10 + Box-Muller definition,
so a seed below 2^32 must give the synthetic inputs' rotations bit for bit."""
import numpy as np
import pytest
import torch

import lsh_attention_02_b200 as lsh
from lsh_attention_02_b200 import synth


@pytest.mark.parametrize("seed,nb,nh,dtype", [(1000, 16, 1, "f32"), (1002, 1024, 4, "bf16"), (7, 2, 3, "bf16"),
                                              (123456789, 192, 8, "f32"), (1004, 8192, 2, "bf16")])
def test_rotations_match_synthetic_generator(seed, nb, nh, dtype):
    desc = lsh.make_desc(1, 1, 64, 64, nb, nh, 64, True, lsh.LSH_BF16 if dtype == "bf16" else lsh.LSH_F32)
    got = lsh.make_rotations(desc, seed).float().numpy()
    w = synth.Workload("t", 1, 1, 64, 64, nb, nh, 64, True, dtype, False, seed)
    want = synth.make_inputs(w)["R"]
    assert got.shape == want.shape
    np.testing.assert_array_equal(got, want)


def test_rotations_statistics_and_seed_dependence():
    desc = lsh.make_desc(1, 1, 64, 64, 4096, 4, 64, False, lsh.LSH_F32)
    a = lsh.make_rotations(desc, 1).numpy().ravel().astype(np.float64)
    b = lsh.make_rotations(desc, 2).numpy().ravel()
    c = lsh.make_rotations(desc, 1 + (1 << 32)).numpy().ravel()     # the high seed word changes the key
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01     # 524288 N(0, 1) draws
    assert not np.array_equal(a, b) and not np.array_equal(a, c)
    np.testing.assert_array_equal(a, lsh.make_rotations(desc, 1).numpy().ravel())


def test_rotations_argument_errors():
    L = lsh.load_library()
    good = lsh.make_desc(1, 1, 64, 64, 16, 1, 64, False, lsh.LSH_F32)
    buf = torch.empty(64 * 8)
    assert L.lsh_attn_make_rotations(1, None, lsh._ptr(buf)) == -1
    assert L.lsh_attn_make_rotations(1, lsh.ctypes.byref(good), None) == -1
    bad = lsh.make_desc(1, 1, 64, 64, 15, 1, 64, False, lsh.LSH_F32)
    assert L.lsh_attn_make_rotations(1, lsh.ctypes.byref(bad), lsh._ptr(buf)) == -2
