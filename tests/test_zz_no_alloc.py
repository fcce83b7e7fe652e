"""The linear attention entry point that allocates nothing.

Callers that may not allocate device memory (a plugin handed only its input
and output buffers, code running under a memory pool that forbids ad-hoc
allocation) use edit_linear_attention_noalloc, whose scratch is an array
compiled into the library. Through the C ABI, on two calls in a row, its
output must match the linear attention step of edit_attn_forward on the same
q, k, v, within the fp32 tolerance of the other parity tests; and, on seeded
q, k, v of its own, the fp64 oracle's linear attention (eq. (y_i) of the EDiT
notes page) within the bars of the other parity tests: 1e-4 for fp32 and
2e-2 for bf16 (fp32 accumulation), max |gpu - oracle| / max |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle.edit_oracle as O
from linear_compressed_attention_b200 import binding as bd
from linear_compressed_attention_b200.inputs import WORKLOADS, make_attention_inputs, make_inputs

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


ORACLE_CASES = [
    # (dtype, B, N, M, C, heads): d = 72 (the workloads' head width), d = 128 (the apply kernel's shared
    # memory above 48 KB), a ragged token count, two images
    ("bf16", 1, 4096, 1024, 1152, 16),
    ("bf16", 2, 333, 77, 256, 2),
    ("f32", 1, 1000, 250, 256, 2),
    ("f32", 2, 130, 37, 96, 3),
]


@pytest.mark.parametrize("case", ORACLE_CASES, ids=lambda c: "-".join(map(str, c)))
def test_noalloc_matches_oracle(case):
    dtype, B, N, M, C, heads = case
    q, k, v = make_attention_inputs(B, N, M, C, seed=51, dtype=dtype)
    eps = 1e-6
    ref, _, _ = O.linear_attention(q, k, v, heads, eps)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    code = bd.EDIT_BF16 if dtype == "bf16" else bd.EDIT_F32
    dq, dk, dv = (torch.from_numpy(a).to("cuda", tdt) for a in (q, k, v))
    tol = 2e-2 if dtype == "bf16" else 1e-4
    first = None
    for _ in range(2):
        out = torch.full_like(dq, float("nan"))
        rc = bd.edit_linear_attention_noalloc(dq, dk, dv, B, N, M, C, heads, code, eps, out)
        assert rc == 0, bd.status_string(rc)
        torch.cuda.synchronize()
        y = out.float().cpu().numpy()
        err = float(np.max(np.abs(y - ref)) / np.max(np.abs(ref)))
        assert err <= tol, (case, err)
        if first is None:
            first = out.clone()
        else:
            assert torch.equal(first, out)     # the second call leaves nothing of the first behind
