"""Row-band sequence parallelism on the host (CPU): the band split, the
halo exchange and the record all-gather of linear_compressed_attention_b200
.seqpar, run on 2 and 3 gloo ranks with the fp64 oracle's band arithmetic as
the backend (tests/oracle_band.py). Every rank's band of the output,
gathered, must equal the unsharded oracle layer (eq. (y_i) with ConvFusion
and the Spatial Compressor) to fp64 rounding: the split changes only the
order of the two global sums."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.edit_oracle as O
from linear_compressed_attention_b200 import seqpar
from linear_compressed_attention_b200.inputs import make_inputs
from tests.oracle_band import OracleBand

CASES = {
    "even": dict(B=1, H=12, W=10, C=64, c_red=16, gn_groups=4, heads=2, dtype="f32", seed=61, nonzero_affine=True),
    "odd": dict(B=1, H=11, W=7, C=48, c_red=12, gn_groups=3, heads=3, dtype="f32", seed=62, nonzero_affine=True),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("H,world", [(12, 1), (12, 2), (12, 6), (11, 2), (11, 3), (11, 6), (512, 8), (1, 1)])
def test_band_bounds_cover_the_image_on_even_rows(H, world):
    bands = [seqpar.band_bounds(H, world, r) for r in range(world)]
    assert bands[0][0] == 0 and sum(rows for _, rows in bands) == H
    for (r0, n), (r1, _) in zip(bands, bands[1:]):
        assert r0 + n == r1 and r1 % 2 == 0 and n >= 1
    assert max(n for _, n in bands) - min(n for _, n in bands) <= 2
    with pytest.raises(ValueError):
        seqpar.band_bounds(H, (H + 1) // 2 + 1, 0)


@pytest.mark.parametrize("name,world", [("even", 2), ("even", 3), ("odd", 4)])
def test_bands_in_one_process_equal_the_layer(name, world):
    """The decomposition alone: every band's partials, then every band's
    finish with all records, in one process."""
    cfg = CASES[name]
    d = make_inputs(**cfg)
    H, W, C = cfg["H"], cfg["W"], cfg["C"]
    x = torch.from_numpy(d["x"][0].astype(np.float64)).reshape(H, W, C)
    bands = [seqpar.band_bounds(H, world, r) for r in range(world)]
    be = OracleBand(d, H, W, cfg["heads"])
    exts = []
    for r0, n in bands:
        top, bot = seqpar.halo(H, r0, n)
        exts.append(x[r0 - top:r0 + n + bot])
    recs = torch.stack([be.partials(e, r0, n) for e, (r0, n) in zip(exts, bands)])
    y = torch.cat([be.finish(e, recs, r0, n) for e, (r0, n) in zip(exts, bands)]).numpy()
    ref = O.edit_forward(d["x"], H, W, d, cfg["heads"])[0].reshape(H, W, C)
    assert np.max(np.abs(y - ref)) <= 1e-10 * np.max(np.abs(ref))


def _rank_main(rank, world, port, name, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        cfg = CASES[name]
        d = make_inputs(**cfg)
        H, W, C = cfg["H"], cfg["W"], cfg["C"]
        r0, n = seqpar.band_bounds(H, world, rank)
        x_band = torch.from_numpy(d["x"][0].astype(np.float64)).reshape(H, W, C)[r0:r0 + n].clone()
        y = seqpar.sharded_forward(x_band, H, OracleBand(d, H, W, cfg["heads"]), rank, world)
        torch.save({"row0": r0, "y": y}, os.path.join(out, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world", [("even", 2), ("odd", 3)])
def test_sharded_forward_on_gloo_ranks(tmp_path, name, world):
    mp.spawn(_rank_main, args=(world, _free_port(), name, str(tmp_path)), nprocs=world, join=True)
    parts = sorted((torch.load(os.path.join(tmp_path, f"r{r}.pt")) for r in range(world)), key=lambda p: p["row0"])
    y = torch.cat([p["y"] for p in parts]).numpy()
    cfg = CASES[name]
    ref = O.edit_forward(make_inputs(**cfg)["x"], cfg["H"], cfg["W"], make_inputs(**cfg), cfg["heads"])[0]
    ref = ref.reshape(cfg["H"], cfg["W"], cfg["C"])
    assert y.shape == ref.shape
    assert np.max(np.abs(y - ref)) <= 1e-10 * np.max(np.abs(ref))
