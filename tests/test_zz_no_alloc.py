"""The scratch-free ternarise entry point (tw_ternarize_pack_noalloc).

It serves callers that cannot allocate device memory where they need a
matrix packed (a plugin whose host framework owns the device-memory budget,
a loop that must not call cudaMalloc).  Its results must equal those of
tw_ternarize_pack, which takes a caller workspace: the same packed bytes,
the same fp64 mean|W| and fp32 scale, bit for bit (the tolerance every
ternarisation test here uses).  Two calls in a row — a larger matrix, then a
smaller one — show that the shared scratch array's leftover contents from
one call do not leak into the next.  This file is collected last.
"""
import numpy as np
import pytest

from tests import gpu_util as G
from ternary_weight_decoder_b200 import synth

pytestmark = pytest.mark.gpu


def _both(api, dev, N, K, seed):
    W = G.to_dev(synth.weights(seed, 3, N, K), dev)
    p0, m0, s0 = api.ternarize_pack(W)
    p1, m1, s1 = api.ternarize_pack_noalloc(W)
    api.check()
    return (p0.cpu().numpy(), m0.cpu().numpy(), s0.cpu().numpy(),
            p1.cpu().numpy(), m1.cpu().numpy(), s1.cpu().numpy())


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    dev = G.torch_dev()
    api = G.api()
    for (N, K, seed) in [(1536, 8960, 1), (300, 1536, 2)]:
        p0, m0, s0, p1, m1, s1 = _both(api, dev, N, K, seed)
        assert p1.size == p0.size == api.packed_bytes(N, K)
        assert (p1 == p0).all(), f"packed codes differ for {N}x{K}"
        assert m1[0] == m0[0] and s1[0] == s0[0], (N, K, m0, m1, s0, s1)


def test_noalloc_rejects_rows_beyond_its_scratch():
    dev = G.torch_dev()
    api = G.api()
    import torch
    W = torch.zeros((api.NOALLOC_MAX_N + 1, 128), dtype=torch.float32, device=dev)
    with pytest.raises(api.TernaryError) as e:
        api.ternarize_pack_noalloc(W)
    assert e.value.status == 2 and "TW_NOALLOC_MAX_N" in str(e.value)
    # a successful call after the failure leaves no stale message behind
    api.ternarize_pack_noalloc(W[:16].contiguous())
    assert api.tw_last_error() == b""
    api.check()
