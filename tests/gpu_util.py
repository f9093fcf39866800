"""Shared helpers of the GPU parity tests: build/load the library, run the
CUDA path through the C ABI, and compare with the oracle."""
import numpy as np
import pytest

from oracle import oracle as orc
from tests import layout_spec

Y_RTOL = 1e-6   # fp32 outputs vs the fp64 oracle (four fp32 roundings < 2.4e-7)


def api():
    from ternary_weight_decoder_b200 import build
    build.build()
    from ternary_weight_decoder_b200 import api as a
    return a


def torch_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def to_dev(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def ternarize_gpu(W, dev):
    a = api()
    packed, mean_abs, wscale = a.ternarize_pack(to_dev(W, dev))
    a.check()
    return packed, mean_abs, wscale


def assert_y_close(y_gpu, y_orc, ctx=""):
    y_gpu = np.asarray(y_gpu, np.float64)
    assert np.isfinite(y_gpu).all(), f"non-finite output {ctx}"
    err = np.abs(y_gpu - y_orc)
    bad = err > Y_RTOL * np.abs(y_orc)
    assert not bad.any(), (f"{ctx}: {int(bad.sum())} outputs off; worst rel "
                           f"{float((err / np.maximum(np.abs(y_orc), 1e-300)).max()):.3e}")


def check_packed_against_oracle(W, packed, mean_abs, wscale, N, K):
    """Codes (through the layout spec), mean and wscale against the oracle."""
    codes, mean = orc.ternarize(W)
    got_mean = float(mean_abs.cpu().numpy()[0])
    assert got_mean == mean, (got_mean, mean)
    assert float(wscale.cpu().numpy()[0]) == np.float32(mean)
    want = layout_spec.pack(codes)
    got = packed.cpu().numpy()[:want.size]
    assert (got == want).all(), "packed bytes differ from the layout of the oracle codes"
    return codes, mean
