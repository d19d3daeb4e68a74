"""Host logic of bench.py's end-to-end step: the six x and six y of a step live in one device
buffer each, as views, so that a step moves its inputs and results with one copy each way."""
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def _layer():
    g = torch.Generator().manual_seed(0)
    return [(object(), torch.randn(M, bench.K_HEAD, generator=g).to(torch.bfloat16),
             torch.empty(M, N, dtype=torch.float32)) for (N, M) in bench.GEMV_SHAPES]


def test_views_cover_every_operand_once():
    layer = _layer()
    x_dev, y_dev, x_host, y_host, ops = bench.stage_step_io(layer, "cpu", lambda t: t.clone())
    assert len(ops) == len(layer)
    assert x_dev.numel() == sum(x.numel() for (_, x, _) in layer)
    assert y_dev.numel() == sum(y.numel() for (_, _, y) in layer)
    for (w, x, y), (w2, xv, yv) in zip(layer, ops):
        assert w2 is w and torch.equal(xv, x) and yv.shape == y.shape
        assert xv.is_contiguous() and yv.is_contiguous()
        assert (xv.data_ptr() - x_dev.data_ptr()) % 16 == 0
        assert (yv.data_ptr() - y_dev.data_ptr()) % 16 == 0
    # bytes moved per step match the per-tensor sums the JSON line reports
    assert x_host.numel() * x_host.element_size() == 266240
    assert y_host.numel() * y_host.element_size() == 1331200


def test_one_copy_each_way_moves_all_operands():
    layer = _layer()
    x_dev, y_dev, x_host, y_host, ops = bench.stage_step_io(layer, "cpu", lambda t: t.clone())
    x_dev.zero_()
    x_dev.copy_(x_host)                      # the step's single input copy
    for (_, x, _), (_, xv, _) in zip(layer, ops):
        assert torch.equal(xv, x)
    for k, (_, _, yv) in enumerate(ops):     # what the six GEMVs would write
        yv.fill_(k + 1)
    y_host.copy_(y_dev)                      # the step's single output copy
    o = 0
    for k, (_, _, yv) in enumerate(ops):
        assert torch.all(y_host[o:o + yv.numel()] == k + 1)
        o += yv.numel()
