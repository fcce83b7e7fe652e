"""Parity of the ablation variants (query / key / value processing of the
ablation table on the EDiT notes page) and of the optional output Linear,
CUDA path through the C ABI against the fp64 CPU oracle on the same seeded
inputs. Metric and bars as the layer tests: max |gpu - oracle| / max |oracle|,
1e-4 (fp32 storage) and 2e-2 (bf16 storage, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import oracle.edit_oracle as O
from linear_compressed_attention_b200 import binding as bd
from linear_compressed_attention_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
VARIANTS = [(q, k, v) for q in ("cf", "none") for (k, v) in (("sc", "sc"), ("cf", "none"), ("none", "none"))]
TABLE_ROWS = [("cf", "sc", "sc"), ("cf", "cf", "none"), ("none", "sc", "sc"), ("cf", "none", "none")]


def max_rel(g, o):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    return float(np.max(np.abs(g - o)) / max(np.max(np.abs(o)), 1e-30))


def check_variant(cfg, d, qkv, proj):
    layer = bd.EditAttention(d, cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"], cfg["dtype"],
                             variant=qkv, out_proj=proj)
    x = torch.from_numpy(d["x"]).to("cuda", layer.tdtype)
    y = layer.forward(x)
    torch.cuda.synchronize()
    assert layer.status() == 0
    ref, it = O.edit_variant_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"], *qkv, out_proj=proj,
                                     return_intermediates=True)
    errs = {"out": max_rel(y.float().cpu().numpy(), ref)}
    B, heads, dh = cfg["B"], cfg["heads"], cfg["C"] // cfg["heads"]
    Sz = layer.intermediate("Sz", (B, heads, dh, dh + 1), torch.float32).cpu().numpy()
    errs["S"] = max_rel(Sz[..., :dh], it["S"])
    errs["z"] = max_rel(Sz[..., dh], it["z"])
    tol = TOL[cfg["dtype"]]
    assert all(v <= tol for v in errs.values()), (qkv, proj, errs, tol)
    return errs


SMALL = [
    dict(dtype="bf16", B=2, H=9, W=7, C=128, c_red=64, gn_groups=8, heads=2),      # d = 64, odd grid, N % 8 != 0
    dict(dtype="bf16", B=1, H=12, W=10, C=1152, c_red=288, gn_groups=32, heads=16),  # d = 72, the workload widths
    dict(dtype="f32", B=2, H=5, W=7, C=48, c_red=12, gn_groups=3, heads=3),
]


@pytest.mark.parametrize("proj", [False, True], ids=["y", "proj"])
@pytest.mark.parametrize("qkv", VARIANTS, ids=lambda v: "-".join(v))
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: f"{s['dtype']}-{s['C']}")
def test_variant_small(shape, qkv, proj):
    cfg = dict(shape, seed=41, nonzero_affine=True, variant_weights=True)
    check_variant(cfg, make_inputs(**cfg), qkv, proj)


@pytest.mark.parametrize("qkv", TABLE_ROWS, ids=lambda v: "-".join(v))
def test_table_rows_px1024(qkv):
    """The ablation table's four rows on the 4096-token workload (uncompressed
    rows: 4096 keys per head)."""
    cfg = dict(WORKLOADS["px1024"], variant_weights=True)
    print(qkv, check_variant(cfg, make_inputs(**cfg), qkv, qkv == ("cf", "sc", "sc")))


@pytest.mark.parametrize("qkv", TABLE_ROWS, ids=lambda v: "-".join(v))
def test_table_rows_px2048(qkv):
    """The ablation table's four rows on the 16,384-token workload, the size
    from which the plan takes the kernels the benchmark times at 65,536
    tokens: the tap-reuse conv (W = 128), the 384-column ring GEMM (also for
    the key ConvFusion's 2C-strided output and the output Linear) and the
    uncompressed rows' operand transpose over 16,384 tokens."""
    cfg = dict(WORKLOADS["px2048"], variant_weights=True)
    print(qkv, check_variant(cfg, make_inputs(**cfg), qkv, qkv == ("cf", "sc", "sc")))


@pytest.mark.slow
@pytest.mark.parametrize("qkv,proj", [(("cf", "none", "none"), False), (("cf", "cf", "none"), False),
                                      (("cf", "sc", "sc"), True), (("none", "sc", "sc"), False)],
                         ids=["cf-none-none", "cf-cf-none", "cf-sc-sc-proj", "none-sc-sc"])
def test_table_rows_px4096_full_size(qkv, proj):
    """The ablation rows at the size and in the launch configuration the
    benchmark times them (65,536 tokens, 5% outlier tokens), every output
    element and S, z against the oracle; the uncompressed rows sum over all
    65,536 keys per head."""
    cfg = dict(WORKLOADS["px4096"], variant_weights=True)
    print(qkv, proj, check_variant(cfg, make_inputs(**cfg), qkv, proj))


def test_default_variant_is_the_layer():
    cfg = dict(dtype="bf16", B=1, H=16, W=16, C=256, c_red=64, gn_groups=4, heads=4, seed=43, variant_weights=True)
    d = make_inputs(**cfg)
    a = bd.EditAttention(d, 1, 16, 16, 256, 4, "bf16")
    b = bd.EditAttention(d, 1, 16, 16, 256, 4, "bf16", variant=("cf", "sc", "sc"))
    x = torch.from_numpy(d["x"]).to("cuda", torch.bfloat16)
    ya, yb = a.forward(x), b.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(ya, yb)


def test_variant_uncompressed_operands():
    """Without the compressor the channel-major operands hold ReLU(K') and V'
    for all N tokens, zero past N."""
    cfg = dict(dtype="bf16", B=2, H=5, W=3, C=128, c_red=64, gn_groups=8, heads=2, seed=44, variant_weights=True)
    d = make_inputs(**cfg)
    layer = bd.EditAttention(d, 2, 5, 3, 128, 2, "bf16", variant=("none", "none", "none"))
    x = torch.from_numpy(d["x"]).to("cuda", torch.bfloat16)
    layer.forward(x)
    torch.cuda.synchronize()
    lay = layer.layout
    Mp, NP, dh = lay["Mp"], lay["NP"], 64
    assert Mp == 16
    KT = layer.intermediate("KT", (2, 128, Mp)).float().cpu()
    VTx = layer.intermediate("VTx", (2, 2, NP, Mp)).float().cpu()
    Kp = layer.intermediate("KVp", (2, 15, 256)).float().cpu()
    assert torch.equal(KT[..., :15], torch.relu(Kp[..., :128]).transpose(1, 2))
    assert torch.equal(VTx[:, :, :dh, :15].reshape(2, 128, 15), Kp[..., 128:].transpose(1, 2))
    assert torch.all(KT[..., 15:] == 0) and torch.all(VTx[:, :, :dh, 15:] == 0)
