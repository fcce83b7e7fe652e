"""Row-band sequence parallelism: one EDiT layer over several ranks.

One image's rows are split into bands, one per rank (include/edit_attn.h,
edit_attn_band_*). The layer's only global steps are the GroupNorm statistics
of the 3x3 conv output and the per-head [S | z] sums of eq. (y_i) on the EDiT
notes page; everything else reads at most a pixel's 3x3 neighbourhood. A step:

1. ``exchange_halo``: each rank sends its first row to the rank above and its
   last row to the rank below, and receives their neighbouring rows (point to
   point, into local buffers), giving its band with one halo row on each side
   (none at the image borders);
2. ``backend.partials``: the band's record of partial sums (the library's
   edit_attn_band_partials on a GPU);
3. ``gather_records``: an all-gather of the records, in band order;
4. ``backend.finish``: every rank sums all records in band order (the same
   totals on every rank, no floating-point all-reduce) and computes its rows
   of the output (edit_attn_band_finish).

This module is host orchestration over torch.distributed; the arithmetic runs
in the backend. ``BandLayer`` is the CUDA backend (argument marshalling for the
C ABI only).
"""
from __future__ import annotations

import ctypes

from . import binding as bd


def band_bounds(H: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [row0, row0 + rows) of band `rank` of `world`: the ceil(H/2) row
    pairs split as evenly as possible (the first bands take one pair more),
    so every band boundary is an even row."""
    pairs = (H + 1) // 2
    if world < 1 or world > pairs or not 0 <= rank < world:
        raise ValueError(f"cannot split {H} rows into {world} bands of whole row pairs")
    base, extra = divmod(pairs, world)
    p0 = rank * base + min(rank, extra)
    p1 = p0 + base + (1 if rank < extra else 0)
    row0, row1 = 2 * p0, min(H, 2 * p1)
    return row0, row1 - row0


def halo(H: int, row0: int, rows: int) -> tuple[int, int]:
    """(top, bottom) halo rows of a band: one on each side that has a neighbour."""
    return (1 if row0 > 0 else 0), (1 if row0 + rows < H else 0)


def exchange_halo(x_band, H: int, row0: int, rows: int, rank: int, world: int, group=None):
    """The band [rows, W, C] with its halo rows from the neighbouring ranks:
    returns x_ext [rows + top + bottom, W, C]. Point-to-point sends and
    receives into local buffers, posted together (no ordering deadlock)."""
    import torch
    import torch.distributed as dist

    top, bot = halo(H, row0, rows)
    ops, recv_top, recv_bot = [], None, None
    if top:
        recv_top = torch.empty_like(x_band[0])
        ops.append(dist.P2POp(dist.irecv, recv_top, rank - 1, group))
        ops.append(dist.P2POp(dist.isend, x_band[0].contiguous(), rank - 1, group))
    if bot:
        recv_bot = torch.empty_like(x_band[-1])
        ops.append(dist.P2POp(dist.irecv, recv_bot, rank + 1, group))
        ops.append(dist.P2POp(dist.isend, x_band[-1].contiguous(), rank + 1, group))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    parts = ([recv_top[None]] if top else []) + [x_band] + ([recv_bot[None]] if bot else [])
    return torch.cat(parts, 0).contiguous()


def gather_records(record, world: int, group=None):
    """All ranks' records [world, nbytes], in band (rank) order."""
    import torch
    import torch.distributed as dist

    out = [torch.empty_like(record) for _ in range(world)]
    dist.all_gather(out, record, group=group)
    return torch.stack(out, 0).contiguous()


def sharded_forward(x_band, H: int, backend, rank: int, world: int, group=None):
    """One layer step of this rank's band: its rows of the output."""
    row0, rows = band_bounds(H, world, rank)
    if x_band.shape[0] != rows:
        raise ValueError(f"rank {rank} holds {x_band.shape[0]} rows, its band has {rows}")
    x_ext = exchange_halo(x_band, H, row0, rows, rank, world, group)
    record = backend.partials(x_ext, row0, rows)
    records = gather_records(record, world, group)
    return backend.finish(x_ext, records, row0, rows)


class EditBand(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("row0", ctypes.c_int), ("rows", ctypes.c_int)]


def _lib():
    L = bd.lib()
    if not getattr(L, "_band_types", False):
        i, p = ctypes.c_int, ctypes.c_void_p
        Wp, Bp = ctypes.POINTER(bd.EditAttnWeights), ctypes.POINTER(EditBand)
        L.edit_attn_band_workspace_bytes.argtypes = [i, i, i, Bp, Wp]
        L.edit_attn_band_workspace_bytes.restype = ctypes.c_size_t
        L.edit_attn_band_record_bytes.argtypes = [i, i, Wp]
        L.edit_attn_band_record_bytes.restype = ctypes.c_size_t
        L.edit_attn_band_partials.argtypes = [p, i, i, i, Bp, Wp, p, p]
        L.edit_attn_band_partials.restype = i
        L.edit_attn_band_finish.argtypes = [p, i, i, i, Bp, Wp, p, i, p, p]
        L.edit_attn_band_finish.restype = i
        L._band_types = True
    return L


def band_workspace_bytes(W, C, heads, band: EditBand, weights: bd.EditAttnWeights) -> int:
    return int(_lib().edit_attn_band_workspace_bytes(W, C, heads, ctypes.byref(band), ctypes.byref(weights)))


def band_record_bytes(C, heads, weights: bd.EditAttnWeights) -> int:
    return int(_lib().edit_attn_band_record_bytes(C, heads, ctypes.byref(weights)))


def band_partials(x_ext, W, C, heads, band: EditBand, weights, record, stream=None) -> int:
    return int(_lib().edit_attn_band_partials(bd._ptr(x_ext), W, C, heads, ctypes.byref(band), ctypes.byref(weights),
                                              bd._ptr(record), bd._stream(stream)))


def band_finish(x_ext, W, C, heads, band: EditBand, weights, records, nrecords, out, stream=None) -> int:
    return int(_lib().edit_attn_band_finish(bd._ptr(x_ext), W, C, heads, ctypes.byref(band), ctypes.byref(weights),
                                            bd._ptr(records), int(nrecords), bd._ptr(out), bd._stream(stream)))


class BandLayer:
    """The CUDA backend of ``sharded_forward``: one image of H x W tokens,
    bf16 weights on the device (from the synthetic-input dict), a workspace
    sized for the largest band this rank is given."""

    def __init__(self, arrays: dict, H: int, W: int, C: int, heads: int, device="cuda"):
        import torch

        self.torch = torch
        self.H, self.W, self.C, self.heads = H, W, C, heads
        self.device = device
        self.w = {n: torch.from_numpy(arrays[n]).to(device=device, dtype=torch.bfloat16) for n in bd.WEIGHT_NAMES}
        self.consts = dict(c_red=arrays["c_red"], gn_groups=arrays["gn_groups"], gn_eps=arrays["gn_eps"],
                           leaky_slope=arrays["leaky_slope"], attn_eps=arrays["attn_eps"])
        self.struct = bd.make_weights_struct(self.w, bd.EDIT_BF16, **self.consts)
        self.record_bytes = band_record_bytes(C, heads, self.struct)
        self.workspace = None

    def _bind(self, row0, rows):
        band = EditBand(self.H, row0, rows)
        need = band_workspace_bytes(self.W, self.C, self.heads, band, self.struct)
        if need == 0:
            raise ValueError(f"band rows [{row0}, {row0 + rows}) of {self.H} rejected")
        if self.workspace is None or self.workspace.numel() < need:
            self.workspace = self.torch.empty(need, dtype=self.torch.uint8, device=self.device)
            self.struct.workspace = self.workspace.data_ptr()
            self.struct.workspace_bytes = self.workspace.numel()
        return band

    def partials(self, x_ext, row0, rows, record=None):
        band = self._bind(row0, rows)
        if record is None:
            record = self.torch.empty(self.record_bytes, dtype=self.torch.uint8, device=self.device)
        rc = band_partials(x_ext, self.W, self.C, self.heads, band, self.struct, record)
        if rc != 0:
            raise bd.EditError(rc)
        return record

    def finish(self, x_ext, records, row0, rows, out=None):
        band = self._bind(row0, rows)
        if out is None:
            out = self.torch.empty((rows, self.W, self.C), dtype=self.torch.bfloat16, device=self.device)
        rc = band_finish(x_ext, self.W, self.C, self.heads, band, self.struct, records, records.shape[0], out)
        if rc != 0:
            raise bd.EditError(rc)
        return out

    def status(self) -> int:
        return bd.edit_attn_read_status(self.workspace)
