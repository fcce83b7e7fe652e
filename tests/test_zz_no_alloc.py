"""The linear attention entry point that allocates nothing.

Callers that may not allocate device memory (a plugin handed only its input
and output buffers, code running under a memory pool that forbids ad-hoc
allocation) use edit_linear_attention_noalloc, whose scratch is an array
compiled into the library. Through the C ABI, on two calls in a row, its
output must match the linear attention step of edit_attn_forward on the same
q, k, v, within the fp32 tolerance of the other parity tests.
"""
import pytest
import torch

from linear_compressed_attention_b200 import binding as bd
from linear_compressed_attention_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32": dict(WORKLOADS["tiny_fp32"]),
    "two_images_odd_grid": dict(B=2, H=7, W=5, C=96, c_red=24, gn_groups=4, heads=3, dtype="f32", seed=41,
                                nonzero_affine=True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_matches_layer_forward(name):
    cfg = CASES[name]
    d = make_inputs(**cfg)
    B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    N, M = H * W, ((H + 1) // 2) * ((W + 1) // 2)
    layer = bd.EditAttention(d, B, H, W, C, heads, "f32")
    ref = layer.forward(torch.from_numpy(d["x"]).cuda())
    torch.cuda.synchronize()
    assert layer.status() == 0
    q = layer.intermediate("Q", (B, N, C)).clone()
    k = layer.intermediate("K", (B, M, C)).clone()
    v = layer.intermediate("V", (B, M, C)).clone()
    scale = ref.abs().max().item()
    for _ in range(2):
        out = torch.full_like(ref, float("nan"))
        rc = bd.edit_linear_attention_noalloc(q, k, v, B, N, M, C, heads, bd.EDIT_F32, d["attn_eps"], out)
        assert rc == 0, bd.status_string(rc)
        torch.cuda.synchronize()
        err = (out - ref).abs().max().item() / scale
        assert err <= 1e-4, err
