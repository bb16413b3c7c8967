"""Allocation-free sort entry point (lsh_attn_sort_static) against the
workspace sort (lsh_attn_sort): the permutation must be identical, bit for
bit, on consecutive calls that share the fixed scratch.  Kept in a file of its
own that is collected last, so it runs both alone and after the other tests.
"""
import numpy as np
import pytest
import torch

import lsh_attention_02_b200 as lsh
from lsh_attention_02_b200 import synth

pytestmark = pytest.mark.gpu


def _buckets(S, L, nb, seed):
    b = np.random.default_rng(seed).integers(0, nb, size=(S, L))
    return torch.from_numpy(b.astype(np.uint16).view(np.int16).reshape(1, S, 1, L)).cuda()


def _both(desc, bk):
    ref = torch.full(bk.shape, -1, dtype=torch.int32, device="cuda")
    got = torch.full(bk.shape, -1, dtype=torch.int32, device="cuda")
    lsh.lsh_attn_sort(desc, bk, ref)
    lsh.lsh_attn_sort_static(desc, bk, got)
    torch.cuda.synchronize()
    return ref, got


def test_static_sort_matches_workspace_sort_hashed_64k():
    """Buckets of the 64K-token, 4-round, 1024-bucket workload from the hash
    entry point; two static calls in a row, each equal to lsh_attn_sort."""
    w = synth.WORKLOADS["long_64k"]
    inp = synth.make_inputs(w, with_dy=False)
    x = torch.from_numpy(inp["x"]).cuda().to(torch.bfloat16)
    R = torch.from_numpy(inp["R"]).cuda().to(torch.bfloat16)
    desc = lsh.desc_for(x, w.n_buckets, w.n_hashes, w.chunk, w.causal)
    bk = torch.empty((w.B, w.H, w.n_hashes, w.L), dtype=torch.int16, device="cuda")
    lsh.lsh_attn_hash(desc, x, R, bk)
    for _ in range(2):
        ref, got = _both(desc, bk)
        assert torch.equal(ref, got)
        assert int(got.min()) == 0 and int(got.max()) == w.L - 1


@pytest.mark.parametrize("L,nb", [(4160, 200), (65536, 1024)])
def test_static_sort_two_calls_new_inputs(L, nb):
    """Second call on different buckets: nothing left in the scratch by the
    first call may leak into the second (one- and two-pass radix plans)."""
    S = 8
    desc = lsh.make_desc(1, S, L, 64, nb, 1, 64, False, lsh.LSH_BF16)
    for seed in (11, 12):
        ref, got = _both(desc, _buckets(S, L, nb, seed))
        assert torch.equal(ref, got)


def test_static_sort_rejects_oversize():
    """A problem whose scratch exceeds the fixed limit is refused before any
    launch, with the limit in the message; perm is left untouched."""
    S, L, nb = 32, 131072, 1024                       # 6 B per position -> 24 MiB > 16 MiB
    desc = lsh.make_desc(1, S, L, 64, nb, 1, 64, False, lsh.LSH_BF16)
    bk = _buckets(S, L, nb, 3)
    perm = torch.full(bk.shape, -1, dtype=torch.int32, device="cuda")
    with pytest.raises(lsh.LshAttnError) as ei:
        lsh.lsh_attn_sort_static(desc, bk, perm)
    assert ei.value.status == -7
    assert str(16 << 20) in str(ei.value)
    torch.cuda.synchronize()
    assert int(perm.max()) == -1
