"""The seeded input generator: pinned to numpy's Philox and to torch's encoders."""
import numpy as np
import pytest
import torch

import synth
from synth import workloads


@pytest.mark.parametrize("key,ctr", [((0, 0), (0, 0, 0, 0)), ((7, 9), (5, 1, 2, 3)),
                                     ((2**64 - 1, 12345), (2**64 - 2, 2**63, 17, 2**40))])
def test_philox_matches_numpy(key, ctr):
    # numpy's Philox4x64-10 increments the counter before producing a block.
    whole = sum(int(w) << (64 * i) for i, w in enumerate(ctr))
    whole = (whole - 1) % 2**256
    prev = [(whole >> (64 * i)) & (2**64 - 1) for i in range(4)]
    bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=np.array(prev, dtype=np.uint64))
    want = bg.random_raw(4)
    got = synth.philox4x64_10(np.array(ctr, dtype=np.uint64), np.array(key, dtype=np.uint64))
    assert [int(v) for v in got] == [int(v) for v in want]


def test_normal_moments_and_thread_independence():
    a = synth.normal(1 << 18, "f32", 0.0, 1.0, seed=0, stream=1, threads=1)
    b = synth.normal(1 << 18, "f32", 0.0, 1.0, seed=0, stream=1, threads=7)
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1.0) < 0.01
    c = synth.normal(1 << 18, "f32", 1.0, 0.2, seed=0, stream=3)
    assert abs(c.mean() - 1.0) < 0.002 and abs(c.std() - 0.2) < 0.002
    d = synth.normal(1 << 18, "f32", 0.0, 1.0, seed=0, stream=2)
    assert abs(np.corrcoef(a, d)[0, 1]) < 0.01  # streams are independent


def test_storage_encoders_match_torch():
    f = synth.normal(1 << 16, "f32", 0.0, 3.0, seed=1, stream=1)
    bf = synth.normal(1 << 16, "bf16", 0.0, 3.0, seed=1, stream=1)
    want = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf, want)
    h = synth.normal(1 << 16, "f16", 0.0, 3.0, seed=1, stream=1)
    assert np.array_equal(h.view(np.uint16), f.astype(np.float16).view(np.uint16))
    e = workloads.encode(f.astype(np.float64), "bf16")
    assert np.array_equal(e, want)


def test_nonzero_redraws_zeros():
    # std so small that about a third of the bf16 values round to zero
    plain = synth.normal(1 << 14, "bf16", 0.0, 1e-40, seed=0, stream=1)
    assert (plain & 0x7FFF == 0).sum() > 1000
    nz = synth.normal(1 << 14, "bf16", 0.0, 1e-40, seed=0, stream=1, nonzero=True)
    assert (nz & 0x7FFF == 0).sum() == 0
    keep = plain & 0x7FFF != 0
    assert np.array_equal(plain[keep], nz[keep])  # only the zeros were redrawn


def test_workload_shapes():
    w = workloads.WORKLOADS["c1_f32_1024x64"]
    d = workloads.make_inputs(w)
    assert d["x"].shape == (1024 * 64,) and d["x"].dtype == np.float32
    assert d["gamma"].shape == (64,) and d["alpha"][0] == np.float32(0.5)
    w3 = workloads.WORKLOADS["c3_f32_100003x17_inf"]
    assert np.isinf(workloads.make_params(w3)["alpha"][0])
    assert w.fwd_bytes() == 524804 and w.bwd_bytes() == 787208
