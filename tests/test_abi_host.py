"""The C-ABI library loads on a machine without a GPU, exports every entry
point the header declares, and rejects bad arguments on the host with the
documented codes before touching the device (no compute calls here)."""
import ctypes
import os
import re

import pytest

from linear_compressed_attention_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "edit_attn.h")).read()
    return re.findall(r"^EDIT_API\s+[\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M)


def test_header_declares_the_boundary():
    names = header_functions()
    assert set(names) == set(bd.EXPORTS)
    for must in ("edit_attn_forward", "mmedit_hybrid_forward"):
        assert must in names


def test_library_exports_every_declared_symbol():
    L = bd.lib()
    for n in header_functions():
        assert hasattr(L, n), n
        assert ctypes.cast(getattr(L, n), ctypes.c_void_p).value


def fake_struct(dtype=bd.EDIT_BF16, c_red=288, groups=32, ws_bytes=1 << 40, base=0x10000):
    s = bd.EditAttnWeights()
    s.dtype, s.c_red, s.gn_groups = dtype, c_red, groups
    s.gn_eps, s.leaky_slope, s.attn_eps = 1e-5, 0.01, 1e-6
    for k, n in enumerate(bd.WEIGHT_NAMES):
        setattr(s, n, base + 0x1000 * (k + 1))   # never dereferenced: validation fails first
    s.workspace = 0x100000
    s.workspace_bytes = ws_bytes
    return s


def fwd(s, B=1, H=64, W=64, C=1152, heads=16, x=0x200000, out=0x400000):
    return bd.lib().edit_attn_forward(ctypes.c_void_p(x), B, H, W, C, heads, ctypes.byref(s),
                                      ctypes.c_void_p(out), None)


def test_workspace_query_is_host_only_and_monotone():
    s = fake_struct()
    a = bd.edit_attn_workspace_bytes(1, 64, 64, 1152, 16, s)
    b = bd.edit_attn_workspace_bytes(1, 128, 128, 1152, 16, s)
    assert 0 < a < b
    assert a % 256 == 0
    assert bd.edit_attn_workspace_bytes(1, 64, 64, 1152, 7, s) == 0        # C % heads
    f = fake_struct(dtype=bd.EDIT_F32, c_red=16, groups=4)
    assert bd.edit_attn_workspace_bytes(1, 16, 16, 64, 2, f) > 0


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), -2), (dict(H=0), -2), (dict(W=-1), -2), (dict(heads=0), -2), (dict(heads=5), -2),
    (dict(x=0), -1), (dict(out=0), -1), (dict(x=0x200008), -3), (dict(out=0x400004), -3),
])
def test_forward_rejects_bad_arguments(kw, code):
    assert fwd(fake_struct(), **kw) == code


def test_forward_rejects_bad_weights_and_workspace():
    s = fake_struct()
    s.q_w = None
    assert fwd(s) == -1
    s = fake_struct()
    s.k_b = 0x10008
    assert fwd(s) == -3
    s = fake_struct()
    s.dtype = 7
    assert fwd(s) == -4
    s = fake_struct(ws_bytes=1024)
    assert fwd(s) == -5
    s = fake_struct()
    s.workspace = 0x100010          # 16- but not 256-byte aligned
    assert fwd(s) == -3
    s = fake_struct(c_red=100, groups=4)   # no tensor-core conv tile for this width
    assert fwd(s) == -8
    s = fake_struct(c_red=288, groups=5)   # groups must divide c_red
    assert fwd(s) == -2
    assert fwd(fake_struct(), C=1000, heads=8) == -8     # C % 128 for bf16


def test_mm_rejects_bad_arguments():
    m = bd.MMEditWeights()
    m.img = fake_struct()
    for k, n in enumerate(bd.TEXT_NAMES):
        setattr(m, n, 0x800000 + 0x1000 * k)
    m.workspace, m.workspace_bytes = 0x100000, 1 << 40
    L = bd.lib()
    call = lambda **kw: L.mmedit_hybrid_forward(  # noqa: E731
        ctypes.c_void_p(kw.get("xi", 0x200000)), ctypes.c_void_p(kw.get("xt", 0x300000)), 1, 64, 64,
        kw.get("nt", 333), 1536, kw.get("heads", 24), ctypes.byref(m), ctypes.c_void_p(0x400000),
        ctypes.c_void_p(kw.get("ot", 0x500000)), None)
    assert call(nt=-1) == -2
    assert call(xt=0) == -1
    assert call(ot=0x500002) == -3
    assert call(heads=12) == -8        # d = 128: no SDPA kernel for it
    m.eta_mode = 7
    assert call() == -8                # unknown mixing-weight mode
    m.eta_mode = bd.EDIT_ETA_EXACT
    assert bd.mmedit_workspace_bytes(1, 64, 64, 333, 1536, 24, m) > bd.mmedit_workspace_bytes(1, 64, 64, 0, 1536, 24, m)


def test_side_stream_is_optional_and_needs_its_events():
    """A side stream is lent by the caller with its four events; NULL (the
    default) is accepted and runs every kernel on the call's stream."""
    s = fake_struct(ws_bytes=1024)
    assert s.side_stream is None
    assert fwd(s) == -5                     # NULL side stream passes validation up to the workspace
    s = fake_struct()
    s.side_stream = 0x7000
    assert fwd(s) == -1                     # events missing
    for i in range(bd.SIDE_EVENTS):
        s.side_events[i] = 0x7100 + i
    s.side_events[2] = None
    assert fwd(s) == -1
    m = bd.MMEditWeights()
    m.img = fake_struct()
    for k, n in enumerate(bd.TEXT_NAMES):
        setattr(m, n, 0x800000 + 0x1000 * k)
    m.workspace, m.workspace_bytes = 0x100000, 1 << 40
    m.side_stream = 0x7000
    rc = bd.lib().mmedit_hybrid_forward(ctypes.c_void_p(0x200000), ctypes.c_void_p(0x300000), 1, 64, 64, 333, 1536,
                                        24, ctypes.byref(m), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x500000), None)
    assert rc == -1


def test_wait_drill_arguments():
    assert bd.edit_attn_set_wait_drill(-1, 0) == -2
    assert bd.edit_attn_set_wait_drill(1, 10) == -2            # limit below 1 us
    assert bd.edit_attn_set_wait_drill(1, 3_000_000_000) == -2  # above the library's own 2 s
    assert bd.edit_attn_set_wait_drill(1, 1_000_000) == 0
    assert bd.edit_attn_set_wait_drill(0, 0) == 0


def test_status_strings():
    assert bd.status_string(0) == "ok"
    assert bd.status_string(-7) == "device wait timed out"
    assert bd.status_string(-99) == "unknown status"


def test_workspace_layout_offsets():
    s = fake_struct()
    lay = bd.edit_attn_workspace_layout(1, 64, 64, 1152, 16, s)
    offs = [lay[k] for k in ("U", "G", "Q", "KVp", "KT", "VTx", "gn_stats", "Sz")]
    assert lay["K"] == -1 and lay["V"] == -1          # bf16 EDiT keeps K, V channel-major only
    assert lay["Mp"] == 32 * 32 and lay["Wop"] == 32 and lay["NP"] == 80
    assert lay["status"] == 0
    assert all(o % 256 == 0 for o in offs)
    assert len(set(offs)) == len(offs)
    assert max(offs) < bd.edit_attn_workspace_bytes(1, 64, 64, 1152, 16, s)


def test_noalloc_rejects_requests_beyond_its_scratch():
    L = bd.lib()
    p = lambda a: ctypes.c_void_p(a)  # noqa: E731  (never dereferenced: rejected before any launch)
    # 64 images x 16 heads x 72 x 73 x 4 B per block > the fixed scratch
    rc = L.edit_linear_attention_noalloc(p(0x1000), p(0x2000), p(0x3000), 64, 4096, 1024, 1152, 16, bd.EDIT_BF16,
                                         ctypes.c_float(1e-6), p(0x4000), None)
    assert rc == -9 and bd.status_string(rc) == "request exceeds the library's fixed scratch"
    assert L.edit_linear_attention_noalloc(None, p(0x2000), p(0x3000), 1, 8, 4, 64, 2, 0, ctypes.c_float(1e-6),
                                           p(0x4000), None) == -1
    # grid limits: more than 65535 images or heads is a shape error, not a failed launch
    assert L.edit_linear_attention_noalloc(p(0x1000), p(0x2000), p(0x3000), 70000, 8, 4, 8, 2, 0,
                                           ctypes.c_float(1e-6), p(0x4000), None) == -8
    assert L.edit_linear_attention_noalloc(p(0x1000), p(0x2000), p(0x3000), 1, 8, 4, 70000, 70000, 0,
                                           ctypes.c_float(1e-6), p(0x4000), None) == -8
    assert L.edit_linear_attention_noalloc(p(0x1000), p(0x2000), p(0x3000), 1, 8, 4, 258, 1, 0,
                                           ctypes.c_float(1e-6), p(0x4000), None) == -8   # d > 128


def fake_variant(q="cf", k="sc", v="sc", proj=False, base=0x900000):
    var = bd.make_variant_struct(q, k, v)
    for j, n in enumerate(bd.VARIANT_NAMES):
        if n.startswith("o_") and not proj:
            continue
        setattr(var, n, base + 0x1000 * (j + 1))
    return var


def vfwd(s, var, B=1, H=64, W=64, C=1152, heads=16):
    return bd.lib().edit_attn_variant_forward(ctypes.c_void_p(0x200000), B, H, W, C, heads, ctypes.byref(s),
                                              ctypes.byref(var), ctypes.c_void_p(0x400000), None)


def test_variant_workspace_and_processing_checks():
    s = fake_struct()
    base = bd.edit_attn_workspace_bytes(1, 64, 64, 1152, 16, s)
    assert bd.edit_attn_variant_workspace_bytes(1, 64, 64, 1152, 16, s, fake_variant()) == base
    # uncompressed keys/values (M = N) and the output Linear's buffer need more
    assert bd.edit_attn_variant_workspace_bytes(1, 64, 64, 1152, 16, s, fake_variant("cf", "none", "none")) > base
    assert bd.edit_attn_variant_workspace_bytes(1, 64, 64, 1152, 16, s, fake_variant(proj=True)) > base
    for bad in (("cf", "sc", "none"), ("sc", "sc", "sc"), ("cf", "none", "sc"), ("cf", "cf", "cf")):
        assert bd.edit_attn_variant_workspace_bytes(1, 64, 64, 1152, 16, s, fake_variant(*bad)) == 0
        assert vfwd(s, fake_variant(*bad)) == -8
    lay = bd.edit_attn_variant_workspace_layout(1, 64, 64, 1152, 16, s, fake_variant("none", "none", "none"))
    assert lay["Mp"] == 4096 and lay["Wop"] == 4096
    lay = bd.edit_attn_variant_workspace_layout(1, 5, 3, 1152, 16, s, fake_variant("none", "none", "none"))
    assert lay["Mp"] == 16


def test_variant_rejects_missing_weights_it_reads_only():
    # no ConvFusion anywhere: its weights, c_red and gn_groups are not read
    s = fake_struct(c_red=0, groups=0)
    for n in ("cf3_w", "cf3_b", "gn_gamma", "gn_beta", "cf1_w", "cf1_b", "kdw_w", "kdw_b", "vdw_w", "vdw_b"):
        setattr(s, n, None)
    var = fake_variant("none", "none", "none")
    assert bd.edit_attn_variant_workspace_bytes(1, 64, 64, 1152, 16, s, var) > 0
    s.workspace_bytes = 1024
    assert vfwd(s, var) == -5                       # validation passes up to the workspace size
    assert vfwd(s, fake_variant("cf", "none", "none")) == -2   # ConvFusion needs c_red / gn_groups
    s = fake_struct()
    var = fake_variant("cf", "cf", "none")
    var.kcf1_b = None
    assert vfwd(s, var) == -1
    var = fake_variant(proj=True)
    var.o_b = None
    assert vfwd(s, var) == -1
    var = fake_variant(proj=True)
    var.o_w = 0x900008
    assert vfwd(s, var) == -3
    s.kdw_w = None
    assert vfwd(s, fake_variant()) == -1            # the compressor reads the depthwise weights
    assert bd.lib().edit_attn_variant_forward(ctypes.c_void_p(0x200000), 1, 8, 8, 128, 2, ctypes.byref(s), None,
                                              ctypes.c_void_p(0x400000), None) == -1


def _device_present():
    import torch
    return torch.cuda.is_available()


@pytest.mark.skipif(_device_present(), reason="needs a host without a GPU: the call must reach a failing CUDA call")
def test_cuda_failure_is_a_status_not_a_crash():
    """Arguments that pass every host check reach the first CUDA runtime call
    (the status reset), which fails here for want of a device: the call
    returns EDIT_ERR_CUDA instead of crashing, for the layer, a variant and
    MM-EDiT alike. (Skipped where a GPU exists: the fake pointers would then
    reach a real device.)"""
    s = fake_struct(ws_bytes=1 << 40)
    assert fwd(s) == -6
    assert vfwd(s, fake_variant("none", "none", "none", proj=True)) == -6
    m = bd.MMEditWeights()
    m.img = s
    for k, n in enumerate(bd.TEXT_NAMES):
        setattr(m, n, 0x800000 + 0x1000 * k)
    m.workspace, m.workspace_bytes = 0x100000, 1 << 40
    rc = bd.lib().mmedit_hybrid_forward(ctypes.c_void_p(0x200000), ctypes.c_void_p(0x300000), 1, 64, 64, 333, 1152,
                                        16, ctypes.byref(m), ctypes.c_void_p(0x400000), ctypes.c_void_p(0x500000), None)
    assert rc == -6
    assert bd.status_string(rc) == "CUDA error"


def _regions(lay, B, H, W, C, heads, c_red, bf16, compress):
    """(name, offset, bytes) of the intermediates the layout reports, sized as
    the header documents them."""
    es = 2 if bf16 else 4
    N = H * W
    M = ((H + 1) // 2) * ((W + 1) // 2) if compress else N
    d = C // heads
    size = {
        "U": B * N * c_red * es, "G": B * N * c_red * es, "Q": B * N * C * es, "KVp": B * N * 2 * C * es,
        "K": B * M * C * es, "V": B * M * C * es, "gn_stats": None, "Sz": B * heads * d * (d + 1) * 4,
        "KT": B * C * lay["Mp"] * 2, "VTx": B * heads * lay["NP"] * lay["Mp"] * 2,
    }
    out = []
    for name, nbytes in size.items():
        off = lay[name]
        if off < 0 or not nbytes:
            continue
        out.append((name, off, nbytes))
    return out


@pytest.mark.parametrize("dtype", [bd.EDIT_BF16, bd.EDIT_F32])
def test_workspace_regions_disjoint_and_inside(dtype):
    import itertools
    shapes = [(1, 64, 64, 1152, 16, 288, 32), (2, 9, 7, 128, 2, 64, 8), (1, 1, 1, 128, 4, 64, 4),
              (3, 12, 20, 384, 6, 256, 8), (1, 5, 130, 128, 1, 128, 8)]
    if dtype == bd.EDIT_F32:
        shapes = [(2, 5, 7, 48, 3, 12, 3), (1, 1, 1, 32, 2, 8, 2), (1, 11, 4, 72, 1, 24, 6)]
    procs = [("cf", "sc", "sc"), ("cf", "cf", "none"), ("none", "sc", "sc"), ("cf", "none", "none"),
             ("none", "none", "none")]
    for (B, H, W, C, heads, cr, g), qkv, proj in itertools.product(shapes, procs, (False, True)):
        s = fake_struct(dtype=dtype, c_red=cr, groups=g)
        var = fake_variant(*qkv, proj=proj)
        total = bd.edit_attn_variant_workspace_bytes(B, H, W, C, heads, s, var)
        assert total > 0, (B, H, W, C, heads, qkv)
        lay = bd.edit_attn_variant_workspace_layout(B, H, W, C, heads, s, var)
        cr_used = cr if "cf" in qkv[:2] else 0   # U and G exist only when a ConvFusion runs
        regs = _regions(lay, B, H, W, C, heads, cr_used, dtype == bd.EDIT_BF16, qkv[1] == "sc")
        for name, off, nbytes in regs:
            assert off % 256 == 0 and off + nbytes <= total, (name, off, nbytes, total)
        for (n1, o1, b1), (n2, o2, b2) in itertools.combinations(regs, 2):
            assert o1 + b1 <= o2 or o2 + b2 <= o1, (qkv, n1, o1, b1, n2, o2, b2)


def test_band_entry_points_validate_on_the_host():
    from linear_compressed_attention_b200 import seqpar
    s = fake_struct(ws_bytes=1024)
    L = seqpar._lib()
    ok = seqpar.EditBand(64, 32, 32)
    assert seqpar.band_workspace_bytes(64, 1152, 16, ok, s) > 0
    assert seqpar.band_record_bytes(1152, 16, s) % 256 == 0
    assert seqpar.band_record_bytes(1152, 16, s) >= 32 * 2 * 8 + 16 * 72 * 73 * 4
    for bad in ((64, 1, 31), (64, 0, 33), (64, 40, 30), (0, 0, 1), (64, 0, 0)):
        assert seqpar.band_workspace_bytes(64, 1152, 16, seqpar.EditBand(*bad), s) == 0, bad
    assert seqpar.band_workspace_bytes(64, 1152, 16, seqpar.EditBand(63, 32, 31), s) > 0   # last band may be odd
    f = fake_struct(dtype=bd.EDIT_F32, c_red=16, groups=4)
    assert seqpar.band_workspace_bytes(16, 64, 2, seqpar.EditBand(16, 0, 8), f) == 0          # bf16 only
    p = ctypes.c_void_p
    rc = L.edit_attn_band_partials(p(0x200000), 64, 1152, 16, ctypes.byref(ok), ctypes.byref(s), p(0x300000), None)
    assert rc == -5                                    # workspace too small, nothing launched
    s = fake_struct()
    rc = L.edit_attn_band_partials(p(0x200000), 64, 1152, 16, ctypes.byref(ok), ctypes.byref(s), p(0x300010), None)
    assert rc == -3                                    # record not 256-byte aligned
    rc = L.edit_attn_band_finish(p(0x200000), 64, 1152, 16, ctypes.byref(ok), ctypes.byref(s), p(0x300000), 0,
                                 p(0x400000), None)
    assert rc == -2                                    # no records
