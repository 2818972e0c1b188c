"""int8_linear_forward_noalloc (static scratch, no workspace) against int8_linear_forward.

Some callers cannot allocate device memory at the point where they run the layer: a stream
that is being captured into a CUDA graph, an allocator that must not grow in the middle of a
step, or a plain C host that has no way to hand a workspace through.  The no-alloc entry point
serves them from a static device array.  It runs the same kernels as int8_linear_forward, so
its Y must be the same bits.

Collected last on purpose: it must give the same answers whether it runs alone in a fresh
process (the first call looks the scratch up) or after every other test has used the GPU.
"""
import pytest
import torch

import int8_mixed_precision_absmax_b200 as i8
import synth

from gpu_helpers import to_dev

pytestmark = pytest.mark.gpu


def _layer(w: synth.Workload, seed: int):
    X, W, b, _ = synth.make_inputs(w, seed=seed)
    Xd, Wd = to_dev(X), to_dev(W)
    bd = None if b is None else to_dev(b)
    Wq, ws = i8.int8_quant_weight(Wd)
    return Xd, Wq, ws, bd


def _run_in_a_row(cases):
    """The no-alloc calls back to back on one stream, then the workspace forward of each."""
    layers = [(w, _layer(w, seed)) for w, seed in cases]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    outs = []
    for w, (X, Wq, ws, b) in layers:
        Y = torch.full((w.M, w.N), float("nan"), dtype=torch.float16, device="cuda")
        outs.append(i8.int8_linear_forward_noalloc(X, Wq, ws, b, w.threshold, Y, dev_status=status))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for (w, (X, Wq, ws, b)), Y in zip(layers, outs):
        Y_ref = i8.int8_linear_forward(X, Wq, ws, b, w.threshold)
        torch.cuda.synchronize()
        assert torch.equal(Y.view(torch.int16), Y_ref.view(torch.int16)), \
            f"noalloc {w.M}x{w.K}x{w.N}: Y differs from int8_linear_forward"


def test_noalloc_two_scratch_calls_in_a_row():
    """Both calls take the few-token pair, whose outlier list, codes and row scales live in the
    static scratch; the second has fewer outlier columns and smaller M and K, so it runs over
    what the first left behind."""
    base = synth.WORKLOADS["decode_q_proj"]
    _run_in_a_row([
        (synth.scaled(base, M=13, K=2048, N=640, n_outlier_cols=40, bias_std=0.01), 1),
        (synth.scaled(base, M=9, K=1024, N=384, n_outlier_cols=3), 2),
    ])


def test_noalloc_other_routes():
    """A decode-shaped call (one kernel, no scratch) and a long-row call (the cluster kernel,
    no scratch) between two scratch calls."""
    base = synth.WORKLOADS["decode_q_proj"]
    _run_in_a_row([
        (synth.scaled(base, M=16, K=4096, N=512, n_outlier_cols=7), 3),
        (synth.scaled(base, M=8, K=4096, N=1024, n_outlier_cols=6), 4),
        (synth.scaled(base, M=12, K=12288, N=256, n_outlier_cols=5), 5),
        (synth.scaled(base, M=10, K=512, N=256, n_outlier_cols=0), 6),
    ])


def test_noalloc_rejects_shapes_beyond_its_scratch():
    w = synth.scaled(synth.WORKLOADS["decode_q_proj"], M=17, K=256, N=128)
    X, Wq, ws, b = _layer(w, 3)
    Y = torch.empty((w.M, w.N), dtype=torch.float16, device="cuda")
    with pytest.raises(i8.Int8mmError) as e:
        i8.int8_linear_forward_noalloc(X, Wq, ws, b, w.threshold, Y)
    assert e.value.status == -10
