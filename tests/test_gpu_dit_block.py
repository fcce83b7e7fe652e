"""The DiT block around the attention (EDiT self-attention with its output
Linear, gated residuals with LayerNorm modulation, cross-attention over the
caption tokens, tanh-GELU MLP) through the C ABI against the fp64 oracle's
dit_block_forward on the same seeded inputs: max |gpu - oracle| /
max |oracle| within 1e-4 (fp32) and 2e-2 (bf16, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import oracle.edit_oracle as O
from linear_compressed_attention_b200 import binding as bd
from linear_compressed_attention_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}

CASES = [
    ("bf16_d64", dict(dtype="bf16", B=2, H=6, W=7, C=128, c_red=64, gn_groups=8, heads=2, seed=81,
                      nonzero_affine=True), dict(n_cap=9, hidden=512)),
    ("bf16_d72", dict(dtype="bf16", B=1, H=12, W=10, C=1152, c_red=288, gn_groups=32, heads=16, seed=82,
                      nonzero_affine=True), dict(n_cap=150, hidden=4608)),
    ("bf16_d32_odd", dict(dtype="bf16", B=1, H=9, W=5, C=128, c_red=64, gn_groups=4, heads=4, seed=83,
                          nonzero_affine=True), dict(n_cap=1, hidden=256)),
    ("f32", dict(dtype="f32", B=2, H=5, W=7, C=64, c_red=16, gn_groups=4, heads=2, seed=84, nonzero_affine=True),
     dict(n_cap=6, hidden=128)),
    ("px1024", dict(WORKLOADS["px1024"]), dict(n_cap=300, hidden=4608)),
]


@pytest.mark.parametrize("name,cfg,blk", CASES, ids=[c[0] for c in CASES])
def test_dit_block_matches_oracle(name, cfg, blk):
    d = make_inputs(**cfg, dit_block=blk)
    B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    block = bd.DitBlock(d, B, H, W, blk["n_cap"], C, heads, cfg["dtype"])
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", block.tdtype)  # noqa: E731
    x, y, t6 = dev(d["x"]), dev(d["y"]), dev(d["t6"])
    outs = [block.forward(x, y, t6).clone() for _ in range(2)]
    torch.cuda.synchronize()
    assert block.status() == 0
    assert torch.equal(outs[0], outs[1])
    ref = O.dit_block_forward(d["x"], d["y"], d["t6"], H, W, d, heads)
    g = outs[0].float().cpu().numpy()
    err = float(np.max(np.abs(g - ref)) / np.max(np.abs(ref)))
    print(name, err)
    assert err <= TOL[cfg["dtype"]], err
