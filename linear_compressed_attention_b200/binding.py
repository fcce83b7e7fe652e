"""ctypes binding of libedit_attn.so (include/edit_attn.h).

Argument marshalling only: torch tensors are passed as device pointers, the
stream as the current torch stream handle. Every step of the layer runs in the
library's CUDA kernels; there is no fallback. Loading raises if the library
has not been built.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libedit_attn.so")

EDIT_F32, EDIT_BF16 = 0, 1
WEIGHT_NAMES = ("cf3_w", "cf3_b", "gn_gamma", "gn_beta", "cf1_w", "cf1_b", "q_w", "q_b", "k_w", "k_b",
                "v_w", "v_b", "kdw_w", "kdw_b", "vdw_w", "vdw_b")
TEXT_NAMES = ("tq_w", "tq_b", "tk_w", "tk_b", "tv_w", "tv_b")
EXPORTS = ("edit_attn_workspace_bytes", "edit_attn_forward", "mmedit_workspace_bytes", "mmedit_hybrid_forward",
           "edit_attn_read_status", "edit_status_string", "edit_attn_workspace_layout",
           "edit_attn_set_stage_events", "edit_attn_kernel_launches", "edit_linear_attention_noalloc",
           "edit_attn_variant_workspace_bytes", "edit_attn_variant_forward", "edit_attn_variant_workspace_layout",
           "edit_attn_set_wait_drill", "edit_attn_band_workspace_bytes", "edit_attn_band_record_bytes",
           "edit_attn_band_partials", "edit_attn_band_finish", "edit_dit_block_workspace_bytes",
           "edit_dit_block_forward")
STAGE_EVENTS_EDIT, STAGE_EVENTS_MM = 9, 12
PROC = {"none": 0, "cf": 1, "sc": 2}
VARIANT_NAMES = ("kcf3_w", "kcf3_b", "kgn_gamma", "kgn_beta", "kcf1_w", "kcf1_b", "o_w", "o_b")


SIDE_EVENTS = 4
_SIDE_FIELDS = [("side_stream", ctypes.c_void_p), ("side_events", ctypes.c_void_p * SIDE_EVENTS)]


class EditAttnWeights(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int), ("c_red", ctypes.c_int), ("gn_groups", ctypes.c_int),
                ("gn_eps", ctypes.c_float), ("leaky_slope", ctypes.c_float), ("attn_eps", ctypes.c_float)] + \
               [(n, ctypes.c_void_p) for n in WEIGHT_NAMES] + \
               [("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)] + _SIDE_FIELDS


EDIT_ETA_RATIO, EDIT_ETA_EXACT = 0, 1


class MMEditWeights(ctypes.Structure):
    _fields_ = [("img", EditAttnWeights)] + [(n, ctypes.c_void_p) for n in TEXT_NAMES] + \
               [("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t)] + _SIDE_FIELDS + \
               [("eta_mode", ctypes.c_int)]


DIT_NAMES = ("o_w", "o_b", "sst", "cq_w", "cq_b", "ck_w", "ck_b", "cv_w", "cv_b", "co_w", "co_b",
             "fc1_w", "fc1_b", "fc2_w", "fc2_b")


class DitBlockWeights(ctypes.Structure):
    _fields_ = [("attn", EditAttnWeights)] + [(n, ctypes.c_void_p) for n in DIT_NAMES] + \
               [("hidden", ctypes.c_int), ("ln_eps", ctypes.c_float), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)] + _SIDE_FIELDS


class EditAttnVariant(ctypes.Structure):
    _fields_ = [("q_proc", ctypes.c_int), ("k_proc", ctypes.c_int), ("v_proc", ctypes.c_int)] + \
               [(n, ctypes.c_void_p) for n in VARIANT_NAMES]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("status", "U", "G", "Q", "KVp", "K", "V", "gn_stats", "Sz", "KT",
                                              "VTx", "Mp", "Wop", "NP")]


_lib = None


def lib():
    """Load the shared library (raises RuntimeError if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build() "
                           "(python -m linear_compressed_attention_b200.build)")
    L = ctypes.CDLL(LIB_PATH)
    i, p, sz = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
    W, MW = ctypes.POINTER(EditAttnWeights), ctypes.POINTER(MMEditWeights)
    L.edit_attn_workspace_bytes.argtypes = [i, i, i, i, i, W]
    L.edit_attn_workspace_bytes.restype = sz
    L.edit_attn_forward.argtypes = [p, i, i, i, i, i, W, p, p]
    L.edit_attn_forward.restype = i
    L.mmedit_workspace_bytes.argtypes = [i, i, i, i, i, i, MW]
    L.mmedit_workspace_bytes.restype = sz
    L.mmedit_hybrid_forward.argtypes = [p, p, i, i, i, i, i, i, MW, p, p, p]
    L.mmedit_hybrid_forward.restype = i
    L.edit_attn_read_status.argtypes = [p, p, ctypes.POINTER(ctypes.c_int)]
    L.edit_attn_read_status.restype = i
    L.edit_status_string.argtypes = [i]
    L.edit_status_string.restype = ctypes.c_char_p
    L.edit_attn_workspace_layout.argtypes = [i, i, i, i, i, W, ctypes.POINTER(WsLayout)]
    L.edit_attn_workspace_layout.restype = i
    L.edit_attn_set_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i]
    L.edit_attn_set_stage_events.restype = i
    L.edit_attn_kernel_launches.argtypes = []
    L.edit_attn_kernel_launches.restype = ctypes.c_uint64
    L.edit_attn_set_wait_drill.argtypes = [i, ctypes.c_uint64]
    L.edit_attn_set_wait_drill.restype = i
    L.edit_linear_attention_noalloc.argtypes = [p, p, p, i, i, i, i, i, i, ctypes.c_float, p, p]
    L.edit_linear_attention_noalloc.restype = i
    DW = ctypes.POINTER(DitBlockWeights)
    L.edit_dit_block_workspace_bytes.argtypes = [i, i, i, i, i, i, DW]
    L.edit_dit_block_workspace_bytes.restype = sz
    L.edit_dit_block_forward.argtypes = [p, p, p, i, i, i, i, i, i, DW, p, p]
    L.edit_dit_block_forward.restype = i
    V = ctypes.POINTER(EditAttnVariant)
    L.edit_attn_variant_workspace_bytes.argtypes = [i, i, i, i, i, W, V]
    L.edit_attn_variant_workspace_bytes.restype = sz
    L.edit_attn_variant_forward.argtypes = [p, i, i, i, i, i, W, V, p, p]
    L.edit_attn_variant_forward.restype = i
    L.edit_attn_variant_workspace_layout.argtypes = [i, i, i, i, i, W, V, ctypes.POINTER(WsLayout)]
    L.edit_attn_variant_workspace_layout.restype = i
    _lib = L
    return L


class EditError(RuntimeError):
    def __init__(self, code):
        self.code = code
        super().__init__(f"edit_attn error {code}: {status_string(code)}")


def status_string(code: int) -> str:
    return lib().edit_status_string(int(code)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_weights_struct(w: dict, dtype_code: int, c_red: int, gn_groups: int, gn_eps: float, leaky_slope: float,
                        attn_eps: float, workspace=None) -> EditAttnWeights:
    """Fill the C struct from a dict of device tensors named as in the header."""
    s = EditAttnWeights()
    s.dtype = dtype_code
    s.c_red, s.gn_groups = int(c_red), int(gn_groups)
    s.gn_eps, s.leaky_slope, s.attn_eps = float(gn_eps), float(leaky_slope), float(attn_eps)
    for n in WEIGHT_NAMES:
        t = w.get(n)
        setattr(s, n, None if t is None else t.data_ptr())
    if workspace is not None:
        s.workspace = workspace.data_ptr()
        s.workspace_bytes = workspace.numel() * workspace.element_size()
    return s


def make_mm_struct(img: EditAttnWeights, w: dict, workspace=None) -> MMEditWeights:
    s = MMEditWeights()
    s.img = img
    for n in TEXT_NAMES:
        t = w.get(n)
        setattr(s, n, None if t is None else t.data_ptr())
    if workspace is not None:
        s.workspace = workspace.data_ptr()
        s.workspace_bytes = workspace.numel() * workspace.element_size()
    return s


# ----------------------------------------------------------- C-ABI mirrors
def edit_attn_workspace_bytes(B, H, W, C, heads, weights: EditAttnWeights) -> int:
    return int(lib().edit_attn_workspace_bytes(B, H, W, C, heads, ctypes.byref(weights)))


def edit_attn_forward(x, B, H, W, C, heads, weights: EditAttnWeights, out, stream=None) -> int:
    """x, out: device tensors [B, H*W, C]; returns the status code (0 = OK)."""
    return int(lib().edit_attn_forward(_ptr(x), B, H, W, C, heads, ctypes.byref(weights), _ptr(out),
                                       _stream(stream)))


def mmedit_workspace_bytes(B, H, W, N_T, C, heads, weights: MMEditWeights) -> int:
    return int(lib().mmedit_workspace_bytes(B, H, W, N_T, C, heads, ctypes.byref(weights)))


def mmedit_hybrid_forward(x_img, x_txt, B, H, W, N_T, C, heads, weights: MMEditWeights, out_img, out_txt,
                          stream=None) -> int:
    return int(lib().mmedit_hybrid_forward(_ptr(x_img), _ptr(x_txt), B, H, W, N_T, C, heads,
                                           ctypes.byref(weights), _ptr(out_img), _ptr(out_txt), _stream(stream)))


def edit_attn_read_status(workspace, stream=None) -> int:
    st = ctypes.c_int(0)
    rc = lib().edit_attn_read_status(_ptr(workspace), _stream(stream), ctypes.byref(st))
    if rc != 0:
        raise EditError(rc)
    return int(st.value)


def edit_attn_workspace_layout(B, H, W, C, heads, weights: EditAttnWeights) -> dict:
    lay = WsLayout()
    rc = lib().edit_attn_workspace_layout(B, H, W, C, heads, ctypes.byref(weights), ctypes.byref(lay))
    if rc != 0:
        raise EditError(rc)
    return {n: int(getattr(lay, n)) for n, _ in WsLayout._fields_}


_stage_keepalive = None


def edit_attn_set_stage_events(handles) -> int:
    """handles: list of raw cudaEvent_t values (ints), or None to clear."""
    global _stage_keepalive
    if handles is None:
        _stage_keepalive = None
        return int(lib().edit_attn_set_stage_events(None, 0))
    arr = (ctypes.c_void_p * len(handles))(*handles)
    _stage_keepalive = arr
    return int(lib().edit_attn_set_stage_events(arr, len(handles)))


def edit_attn_kernel_launches() -> int:
    return int(lib().edit_attn_kernel_launches())


def edit_attn_set_wait_drill(gn_extra_arrivals: int, limit_ns: int) -> int:
    return int(lib().edit_attn_set_wait_drill(int(gn_extra_arrivals), int(limit_ns)))


def set_side(struct, side) -> None:
    """Lend a side stream to a weights struct: `side` is (stream, [4 events])
    of torch.cuda objects, or None for none."""
    if side is None:
        struct.side_stream = None
        for i in range(SIDE_EVENTS):
            struct.side_events[i] = None
        return
    stream, events = side
    struct.side_stream = stream.cuda_stream
    for i, e in enumerate(events):
        struct.side_events[i] = e.cuda_event


def make_side(device=None):
    """A side stream and its events for the library's concurrent branches,
    owned by the caller (kept alive by the returned tuple)."""
    import torch
    stream = torch.cuda.Stream(device=device)
    events = [torch.cuda.Event(enable_timing=False) for _ in range(SIDE_EVENTS)]
    with torch.cuda.stream(stream):
        for e in events:
            e.record(stream)  # torch creates the event handle at its first record
    return stream, events


def make_variant_struct(q_proc="cf", k_proc="sc", v_proc="sc", w: dict | None = None) -> EditAttnVariant:
    """Processing names 'cf' / 'sc' / 'none'; `w` holds the key ConvFusion
    weights and/or the output Linear (o_w, o_b) as device tensors, or None."""
    v = EditAttnVariant()
    v.q_proc, v.k_proc, v.v_proc = PROC[q_proc], PROC[k_proc], PROC[v_proc]
    for n in VARIANT_NAMES:
        t = (w or {}).get(n)
        setattr(v, n, None if t is None else t.data_ptr())
    return v


def edit_attn_variant_workspace_bytes(B, H, W, C, heads, weights: EditAttnWeights, variant: EditAttnVariant) -> int:
    return int(lib().edit_attn_variant_workspace_bytes(B, H, W, C, heads, ctypes.byref(weights),
                                                       ctypes.byref(variant)))


def edit_attn_variant_forward(x, B, H, W, C, heads, weights: EditAttnWeights, variant: EditAttnVariant, out,
                              stream=None) -> int:
    return int(lib().edit_attn_variant_forward(_ptr(x), B, H, W, C, heads, ctypes.byref(weights),
                                               ctypes.byref(variant), _ptr(out), _stream(stream)))


def edit_attn_variant_workspace_layout(B, H, W, C, heads, weights: EditAttnWeights, variant) -> dict:
    lay = WsLayout()
    vp = None if variant is None else ctypes.byref(variant)
    rc = lib().edit_attn_variant_workspace_layout(B, H, W, C, heads, ctypes.byref(weights), vp, ctypes.byref(lay))
    if rc != 0:
        raise EditError(rc)
    return {n: int(getattr(lay, n)) for n, _ in WsLayout._fields_}


def edit_linear_attention_noalloc(q, k, v, B, N, M, C, heads, dtype_code, attn_eps, out, stream=None) -> int:
    """Linear attention step with the library's static scratch (no workspace);
    q, out [B, N, C], k, v [B, M, C] device tensors. Returns the status code."""
    return int(lib().edit_linear_attention_noalloc(_ptr(q), _ptr(k), _ptr(v), B, N, M, C, heads, dtype_code,
                                                   float(attn_eps), _ptr(out), _stream(stream)))


# ----------------------------------------------------------- convenience
class EditAttention:
    """One EDiT (or MM-EDiT) layer with weights and workspace on a CUDA device.

    ``arrays`` is the dict the synthetic-input generator returns (numpy
    float32, bf16-exact for bf16); tensors are copied to the device once.
    """

    def __init__(self, arrays: dict, B: int, H: int, W: int, C: int, heads: int, dtype: str = "bf16",
                 n_txt: int = 0, mm: bool | None = None, device="cuda", variant: tuple | None = None,
                 out_proj: bool = False, side: bool = True, eta: str = "ratio"):
        """``variant`` = (q_proc, k_proc, v_proc) names ('cf', 'sc', 'none') and/or
        ``out_proj`` select edit_attn_variant_forward; weights a variant does
        not read are not copied to the device (NULL in the structs). With
        ``side`` the layer lends the library a side stream and its events
        (created here, owned by this object) for the concurrent branches.
        ``eta`` ('ratio' | 'exact') picks MM-EDiT's mixing weights."""
        import torch
        self.torch = torch
        self.B, self.H, self.W, self.C, self.heads, self.n_txt = B, H, W, C, heads, int(n_txt or 0)
        self.mm = bool(self.n_txt) if mm is None else bool(mm)
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        self.code = EDIT_BF16 if dtype == "bf16" else EDIT_F32
        self.is_variant = variant is not None or out_proj
        q, k, v = variant or ("cf", "sc", "sc")
        names = WEIGHT_NAMES + (TEXT_NAMES if self.mm else ())
        if self.is_variant:
            skip = set()
            if q != "cf":
                skip |= {"cf3_w", "cf3_b", "gn_gamma", "gn_beta", "cf1_w", "cf1_b"}
            if k != "sc":
                skip |= {"kdw_w", "kdw_b", "vdw_w", "vdw_b"}
            names = tuple(n for n in names if n not in skip)
            names += (("kcf3_w", "kcf3_b", "kgn_gamma", "kgn_beta", "kcf1_w", "kcf1_b") if k == "cf" else ())
            names += (("o_w", "o_b") if out_proj else ())
        self.w = {n: torch.from_numpy(np.ascontiguousarray(arrays[n])).to(device=device, dtype=self.tdtype)
                  for n in names}
        self.consts = dict(c_red=arrays["c_red"], gn_groups=arrays["gn_groups"], gn_eps=arrays["gn_eps"],
                           leaky_slope=arrays["leaky_slope"], attn_eps=arrays["attn_eps"])
        s = make_weights_struct(self.w, self.code, **self.consts)
        self.variant = make_variant_struct(q, k, v, self.w) if self.is_variant else None
        if self.mm:
            m = make_mm_struct(s, self.w)
            nbytes = mmedit_workspace_bytes(B, H, W, self.n_txt, C, heads, m)
        elif self.is_variant:
            nbytes = edit_attn_variant_workspace_bytes(B, H, W, C, heads, s, self.variant)
        else:
            nbytes = edit_attn_workspace_bytes(B, H, W, C, heads, s)
        if nbytes == 0:
            raise ValueError("shape/dtype rejected by the workspace query")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.struct = make_weights_struct(self.w, self.code, workspace=self.workspace, **self.consts)
        self.mm_struct = make_mm_struct(self.struct, self.w, self.workspace) if self.mm else None
        if self.mm_struct is not None:
            self.mm_struct.eta_mode = {"ratio": EDIT_ETA_RATIO, "exact": EDIT_ETA_EXACT}[eta]
        self.side = make_side(device) if side and self.code == EDIT_BF16 else None
        self.set_side(self.side)
        self.layout = edit_attn_variant_workspace_layout(B, H, W, C, heads, self.struct, self.variant)

    def set_side(self, side) -> None:
        """Lend (stream, events) to the library, or None to run every kernel
        on the call's stream."""
        set_side(self.struct, side)
        if self.mm_struct is not None:
            set_side(self.mm_struct, side)

    def forward(self, x, out=None, stream=None):
        if out is None:
            out = self.torch.empty_like(x)
        if self.is_variant:
            rc = edit_attn_variant_forward(x, self.B, self.H, self.W, self.C, self.heads, self.struct, self.variant,
                                           out, stream)
        else:
            rc = edit_attn_forward(x, self.B, self.H, self.W, self.C, self.heads, self.struct, out, stream)
        if rc != 0:
            raise EditError(rc)
        return out

    def forward_mm(self, x_img, x_txt, out_img=None, out_txt=None, stream=None):
        if out_img is None:
            out_img = self.torch.empty_like(x_img)
        if out_txt is None and x_txt is not None:
            out_txt = self.torch.empty_like(x_txt)
        rc = mmedit_hybrid_forward(x_img, x_txt, self.B, self.H, self.W, self.n_txt, self.C, self.heads,
                                   self.mm_struct, out_img, out_txt, stream)
        if rc != 0:
            raise EditError(rc)
        return out_img, out_txt

    def status(self, stream=None) -> int:
        return edit_attn_read_status(self.workspace, stream)

    def intermediate(self, name: str, shape, dtype=None):
        """View of an intermediate kept in the workspace (valid after the call completes)."""
        torch = self.torch
        off = self.layout[name]
        dt = dtype or self.tdtype
        n = int(np.prod(shape))
        es = torch.empty((), dtype=dt).element_size()
        return self.workspace[off:off + n * es].view(dt).view(*shape)


# ----------------------------------------------------------- DiT block
def edit_dit_block_workspace_bytes(B, H, W, N_T, C, heads, weights: DitBlockWeights) -> int:
    return int(lib().edit_dit_block_workspace_bytes(B, H, W, N_T, C, heads, ctypes.byref(weights)))


def edit_dit_block_forward(x, y, t6, B, H, W, N_T, C, heads, weights: DitBlockWeights, out, stream=None) -> int:
    return int(lib().edit_dit_block_forward(_ptr(x), _ptr(y), _ptr(t6), B, H, W, N_T, C, heads,
                                            ctypes.byref(weights), _ptr(out), _stream(stream)))


class DitBlock:
    """One DiT block (EDiT self-attention, cross-attention over the caption
    tokens, MLP) with weights and workspace on a CUDA device; ``arrays`` is
    the synthetic-input dict drawn with ``dit_block=...``."""

    def __init__(self, arrays: dict, B: int, H: int, W: int, N_T: int, C: int, heads: int, dtype: str = "bf16",
                 device="cuda", side: bool = True):
        import torch
        self.torch = torch
        self.B, self.H, self.W, self.N_T, self.C, self.heads = B, H, W, N_T, C, heads
        self.tdtype = torch.bfloat16 if dtype == "bf16" else torch.float32
        code = EDIT_BF16 if dtype == "bf16" else EDIT_F32
        names = WEIGHT_NAMES + DIT_NAMES
        self.w = {n: torch.from_numpy(np.ascontiguousarray(arrays[n])).to(device=device, dtype=self.tdtype)
                  for n in names}
        consts = dict(c_red=arrays["c_red"], gn_groups=arrays["gn_groups"], gn_eps=arrays["gn_eps"],
                      leaky_slope=arrays["leaky_slope"], attn_eps=arrays["attn_eps"])
        s = DitBlockWeights()
        s.attn = make_weights_struct(self.w, code, **consts)
        for n in DIT_NAMES:
            setattr(s, n, self.w[n].data_ptr())
        s.hidden = int(arrays["fc1_w"].shape[0])
        s.ln_eps = float(arrays["ln_eps"])
        nbytes = edit_dit_block_workspace_bytes(B, H, W, N_T, C, heads, s)
        if nbytes == 0:
            raise ValueError("shape/dtype rejected by the DiT block workspace query")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        s.workspace = self.workspace.data_ptr()
        s.workspace_bytes = nbytes
        self.struct = s
        self.side = make_side(device) if side and code == EDIT_BF16 else None
        set_side(self.struct, self.side)

    def forward(self, x, y, t6, out=None, stream=None):
        if out is None:
            out = self.torch.empty_like(x)
        rc = edit_dit_block_forward(x, y, t6, self.B, self.H, self.W, self.N_T, self.C, self.heads, self.struct, out,
                                    stream)
        if rc != 0:
            raise EditError(rc)
        return out

    def status(self, stream=None) -> int:
        return edit_attn_read_status(self.workspace, stream)
