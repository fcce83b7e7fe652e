"""Row-band sequence parallelism on the GPU: the library's band entry points
(edit_attn_band_partials / edit_attn_band_finish) for every band of one
image, run one band after another on one device (each band with its own
workspace, the records gathered in band order as the ranks' all-gather would
give them). The bands' outputs, put together, must match the fp64 oracle's
unsharded layer within the bf16 bar (2e-2, max |gpu - oracle| / max
|oracle|), and the unsharded CUDA layer closely (the split changes only the
order of the two global sums)."""
import numpy as np
import pytest
import torch

import oracle.edit_oracle as O
from linear_compressed_attention_b200 import binding as bd
from linear_compressed_attention_b200 import seqpar
from linear_compressed_attention_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

CASES = [
    ("odd_grid", dict(B=1, H=9, W=7, C=128, c_red=64, gn_groups=8, heads=2, dtype="bf16", seed=63,
                      nonzero_affine=True), 2),
    ("widths_72", dict(B=1, H=32, W=32, C=1152, c_red=288, gn_groups=32, heads=16, dtype="bf16", seed=64,
                       nonzero_affine=True), 3),
    ("px1024", dict(WORKLOADS["px1024"]), 4),
    ("px2048", dict(WORKLOADS["px2048"]), 8),
]


def run_bands(d, H, W, C, heads, world):
    x = torch.from_numpy(d["x"][0]).to("cuda", torch.bfloat16).reshape(H, W, C)
    bands = [seqpar.band_bounds(H, world, r) for r in range(world)]
    layers = [seqpar.BandLayer(d, H, W, C, heads) for _ in bands]
    exts = []
    for r0, n in bands:
        top, bot = seqpar.halo(H, r0, n)
        exts.append(x[r0 - top:r0 + n + bot].contiguous())
    records = torch.empty((world, layers[0].record_bytes), dtype=torch.uint8, device="cuda")
    for r, ((r0, n), layer, ext) in enumerate(zip(bands, layers, exts)):
        layer.partials(ext, r0, n, record=records[r])
    outs = [layer.finish(ext, records, r0, n) for (r0, n), layer, ext in zip(bands, layers, exts)]
    torch.cuda.synchronize()
    assert all(layer.status() == 0 for layer in layers)
    return torch.cat(outs).float().cpu().numpy()


@pytest.mark.parametrize("name,cfg,world", CASES, ids=[c[0] for c in CASES])
def test_bands_match_the_layer(name, cfg, world):
    d = make_inputs(**cfg)
    H, W, C, heads = cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    y = run_bands(d, H, W, C, heads, world)
    ref = O.edit_forward(d["x"], H, W, d, heads)[0].reshape(H, W, C)
    err = float(np.max(np.abs(y - ref)) / np.max(np.abs(ref)))
    layer = bd.EditAttention(d, 1, H, W, C, heads, "bf16")
    full = layer.forward(torch.from_numpy(d["x"]).to("cuda", torch.bfloat16))
    torch.cuda.synchronize()
    full = full.float().cpu().numpy()[0].reshape(H, W, C)
    diff = float(np.max(np.abs(y - full)) / np.max(np.abs(full)))
    print(name, world, "vs oracle", err, "vs unsharded", diff)
    assert err <= 2e-2 and diff <= 2e-2


def test_band_arguments_are_checked():
    cfg = dict(B=1, H=8, W=8, C=128, c_red=64, gn_groups=8, heads=2, dtype="bf16", seed=65)
    d = make_inputs(**cfg)
    layer = seqpar.BandLayer(d, 8, 8, 128, 2)
    for row0, rows in ((1, 4), (0, 3), (6, 4), (-2, 4), (0, 0)):
        with pytest.raises(ValueError):
            layer._bind(row0, rows)
