"""The nn.Module / custom-op layer without a GPU: the op's shape-only
implementation, and the static-FP8 calibration observers (plain torch)."""

import torch

from weight_only_quantized_prologue_b200 import module as M


def test_op_fake_kernel_gives_the_output_shape():
    x = torch.empty((7, 64), dtype=torch.bfloat16, device="meta")
    y = torch.ops.dqgemm.linear(x, 1, 96)
    assert y.shape == (7, 96) and y.dtype == torch.bfloat16 and y.device.type == "meta"


def test_calibration_records_the_input_range_of_every_linear():
    torch.manual_seed(0)
    model = torch.nn.Sequential(torch.nn.Linear(16, 32), torch.nn.ReLU(), torch.nn.Linear(32, 8))
    batches = [torch.randn(4, 16) * (i + 1) for i in range(3)]
    scales = M.calibrate_static_fp8(model, batches)
    assert set(scales) == {"0", "2"}
    a0 = max(b.abs().max().item() for b in batches)
    with torch.no_grad():
        a2 = max(model[1](model[0](b)).abs().max().item() for b in batches)
    # observers keep min and max; the scale is max(|min|, |max|) / 448 in fp32
    assert scales["0"] == float(torch.tensor(a0, dtype=torch.float32) / 448.0)
    assert scales["2"] == float(torch.tensor(a2, dtype=torch.float32) / 448.0)
    # hooks are removed afterwards
    assert not model[0]._forward_pre_hooks and not model[2]._forward_pre_hooks


def test_op_traces_through_torch_export():
    # the pages' flow starts from torch.export; a model calling the op exports
    # with the op as one node, shaped by the fake implementation alone (no
    # library call, so no GPU)
    class Wrap(torch.nn.Module):
        def forward(self, x):
            return torch.relu(torch.ops.dqgemm.linear(x, 12345, 64))

    ep = torch.export.export(Wrap(), (torch.empty(4, 128, dtype=torch.bfloat16),))
    targets = [n.target for n in ep.graph.nodes if n.op == "call_function"]
    assert torch.ops.dqgemm.linear.default in targets
    out = [n for n in ep.graph.nodes if n.op == "output"][0].args[0][0]
    assert tuple(out.meta["val"].shape) == (4, 64) and out.meta["val"].dtype == torch.bfloat16
