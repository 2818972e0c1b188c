"""int8_linear_forward_noalloc (static scratch, no workspace) against int8_linear_forward.

Collected last on purpose: it must give the same answers whether it runs alone in a fresh
process (the first call sets the scratch up) or after every other test has used the GPU.
Two calls go back to back on one stream, the second with fewer outlier columns and other
shapes than the first, so that it runs over what the first left in the shared scratch.
"""
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import synth

from gpu_helpers import assert_y_close, to_dev, to_np

pytestmark = pytest.mark.gpu


def _layer(w: synth.Workload, seed: int):
    X, W, b, _ = synth.make_inputs(w, seed=seed)
    Xd, Wd = to_dev(X), to_dev(W)
    bd = None if b is None else to_dev(b)
    Wq, ws = i8.int8_quant_weight(Wd)
    return Xd, Wq, ws, bd


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    base = synth.WORKLOADS["decode_q_proj"]
    cases = [
        (synth.scaled(base, n_outlier_cols=40, bias_std=0.01), 1),   # M=8, K=N=4096
        (synth.scaled(base, M=13, K=2048, N=640, n_outlier_cols=3), 2),
    ]
    layers = [(w, _layer(w, seed)) for w, seed in cases]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for w, (X, Wq, ws, b) in layers:
        Y = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
        outs.append(i8.int8_linear_forward_noalloc(X, Wq, ws, b, w.threshold, Y, dev_status=status))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (w, (X, Wq, ws, b)), Y in zip(layers, outs):
        Y_ref = i8.int8_linear_forward(X, Wq, ws, b, w.threshold)
        torch.cuda.synchronize()
        assert_y_close(to_np(Y), to_np(Y_ref), f"noalloc {w.M}x{w.K}x{w.N}")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = synth.scaled(synth.WORKLOADS["decode_q_proj"], M=17, K=256, N=128)
    X, Wq, ws, b = _layer(w, 3)
    Y = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
    with pytest.raises(i8.Int8mmError) as e:
        i8.int8_linear_forward_noalloc(X, Wq, ws, b, w.threshold, Y)
    assert e.value.status == -10
