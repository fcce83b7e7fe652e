"""Device-side failure path: a bounded wait that runs out.

Every device-side wait of the library is bounded and reports
EDIT_ERR_TIMEOUT through the workspace status word instead of hanging the
GPU. The wait drill (edit_attn_set_wait_drill) makes the fused GroupNorm's
grid barrier wait for one block more than it launched, with a 1 ms limit: a
flag that nothing sets. The test checks the reported status and wait site,
and that the context stays usable: the next calls, on the same workspace and
on a fresh one, are clean and match the oracle. No fault, trap or hang is
involved."""
import numpy as np
import pytest
import torch

import oracle.edit_oracle as O
from linear_compressed_attention_b200 import binding as bd
from linear_compressed_attention_b200.inputs import make_inputs

pytestmark = pytest.mark.gpu

EDIT_ERR_TIMEOUT = -7
SITE_GN_BARRIER = 30


def max_rel(g, o):
    return float(np.max(np.abs(np.asarray(g, np.float64) - o)) / np.max(np.abs(o)))


def test_gn_grid_barrier_wait_runs_out_and_context_survives():
    # bf16, 8 channels per group: the fused GroupNorm kernel (the one with the grid barrier) runs
    cfg = dict(B=1, H=16, W=16, C=128, c_red=64, gn_groups=8, heads=2, dtype="bf16", seed=46, nonzero_affine=True)
    d = make_inputs(**cfg)
    ref = O.edit_forward(d["x"], 16, 16, d, 2)
    layer = bd.EditAttention(d, 1, 16, 16, 128, 2, "bf16")
    x = torch.from_numpy(d["x"]).to("cuda", torch.bfloat16)
    assert bd.edit_attn_set_wait_drill(1, 1_000_000) == 0
    try:
        layer.forward(x)
    finally:
        assert bd.edit_attn_set_wait_drill(0, 0) == 0
    torch.cuda.synchronize()
    assert layer.status() == EDIT_ERR_TIMEOUT
    words = layer.intermediate("status", (8,), torch.int32).cpu().tolist()
    site, _, seen, expected, launched = words[1:6]
    assert site == SITE_GN_BARRIER, words
    assert expected == launched + 1 and 0 < seen < expected, words
    # the same workspace, drill disarmed: the call resets the status block and is clean
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.status() == 0
    assert max_rel(y.float().cpu().numpy(), ref) <= 2e-2
    # a fresh workspace as well
    fresh = bd.EditAttention(d, 1, 16, 16, 128, 2, "bf16")
    y2 = fresh.forward(x)
    torch.cuda.synchronize()
    assert fresh.status() == 0
    assert torch.equal(y, y2)
