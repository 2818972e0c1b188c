"""The seeded generator: published splitmix64 outputs, determinism, slice independence."""
import numpy as np

import synth


def test_splitmix64_published_seed0_outputs():
    lib = synth._load()
    # the first outputs of splitmix64 seeded with 0, as published with the generator
    assert lib.synth_u64(0, 0) == 0xE220A8397B1DCDAF
    assert lib.synth_u64(0, 1) == 0x6E789E6AA1B965F4
    assert lib.synth_u64(0, 2) == 0x06C45D188009454F


def test_normals_have_the_requested_moments():
    z = synth.normal_f16(synth.stream_key(0, 99), 200, 500, 0.0, 2.0).astype(np.float64)
    assert abs(z.mean()) < 0.02 and abs(z.std() - 2.0) < 0.02


def test_workloads_are_deterministic_and_planted():
    w = synth.scaled(synth.WORKLOADS["decode_q_proj"], K=512, N=64)
    X1, W1, b1, c1 = synth.make_inputs(w)
    X2, W2, b2, c2 = synth.make_inputs(w)
    assert b1 is None and b2 is None
    assert np.array_equal(X1.view(np.uint16), X2.view(np.uint16))
    assert np.array_equal(W1.view(np.uint16), W2.view(np.uint16))
    assert np.array_equal(c1, c2) and len(set(c1.tolist())) == 6
    regular = np.setdiff1d(np.arange(512), c1)
    assert np.abs(X1[:, regular]).max() < 6.0 < np.abs(X1[:, c1]).max(axis=0).min()
    X3, _, _, _ = synth.make_inputs(w, seed=1)
    assert not np.array_equal(X1, X3)


def test_tiny_workload_matches_its_definition():
    X, W, b, cols = synth.make_inputs(synth.WORKLOADS["tiny"])
    assert X.shape == (16, 256) and W.shape == (256, 256) and b.shape == (256,)
    assert list(cols) == [7, 200] and not b.any()
    assert abs(W.astype(np.float64).std() - 0.02) < 0.002
