"""Seeded synthetic inputs and the workload table.

This module holds no arithmetic of the method: it only draws random numbers,
rounds them to the storage precision and names the workloads. The CUDA path
and the CPU oracle both consume what it returns.

Recipe (per workload): ``numpy.random.default_rng(seed)`` (PCG64), float32
normal draws in this order: X [B, N, C]; the outlier token indices (when the
workload has outliers: exactly round(0.05 N) distinct tokens per batch item,
all channels scaled by 8); then the weights cf3_w, cf1_w, q_w, k_w, v_w,
kdw_w, vdw_w, each N(0, 1/fan_in) with fan_in = 9C, Cr, C, C, C, 9, 9; for
MM-EDiT workloads then x_txt [B, N_T, C] and the prompt weights tq_w, tk_w,
tv_w (fan_in C). Biases are 0, GroupNorm gamma = 1 and beta = 0, unless
``nonzero_affine`` asks for random ones (drawn after the weights, so the
stream above is unchanged). ``variant_weights`` adds, drawn after all of
that, the key's own ConvFusion weights kcf3_w, kcf1_w (fan_in 9C, Cr) and the
output projection o_w (fan_in C), then (with ``nonzero_affine``) their
biases and GroupNorm affine. ``dit_block`` (dict with n_cap, hidden) adds,
after all of that, the DiT block's inputs and weights (see make_inputs). bf16
workloads round every array once to bf16 (round-to-nearest-even) and hand out
float32 arrays holding exactly those values.
"""
from __future__ import annotations

import numpy as np

# Workloads shaped like the pages' 512..8192 px text-to-image resolutions.
WORKLOADS = {
    "tiny_fp32": dict(dtype="f32", B=1, H=16, W=16, C=64, c_red=16, gn_groups=4,
                      heads=2, seed=0, outliers=False, n_txt=None),
    "px512_b2": dict(dtype="bf16", B=2, H=32, W=32, C=1152, c_red=288, gn_groups=32,
                     heads=16, seed=1, outliers=False, n_txt=None),
    "px1024": dict(dtype="bf16", B=1, H=64, W=64, C=1152, c_red=288, gn_groups=32,
                   heads=16, seed=2, outliers=False, n_txt=None),
    "px2048": dict(dtype="bf16", B=1, H=128, W=128, C=1152, c_red=288, gn_groups=32,
                   heads=16, seed=2, outliers=False, n_txt=None),
    "px4096": dict(dtype="bf16", B=1, H=256, W=256, C=1152, c_red=288, gn_groups=32,
                   heads=16, seed=3, outliers=True, n_txt=None),
    "px8192": dict(dtype="bf16", B=1, H=512, W=512, C=1152, c_red=288, gn_groups=32,
                   heads=16, seed=3, outliers=True, n_txt=None),
    "mm1024": dict(dtype="bf16", B=1, H=64, W=64, C=1536, c_red=384, gn_groups=32,
                   heads=24, seed=4, outliers=False, n_txt=333),
}

DECLARED = dict(gn_eps=1e-5, leaky_slope=0.01, attn_eps=1e-6)


def round_bf16(a):
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(a.shape)


def _normal(rng, shape, var):
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(np.sqrt(var))


def make_inputs(B, H, W, C, c_red, gn_groups, heads, seed, dtype="bf16",
                outliers=False, n_txt=None, nonzero_affine=False, variant_weights=False, dit_block=None,
                **_ignored):
    """Draw one workload. Returns a dict with x (and x_txt) plus every weight
    under the C header's names and the declared constants; arrays are float32
    (bf16-exact for bf16 workloads). Shapes: x [B, H*W, C]; cf3_w [Cr, 3, 3, C];
    cf1_w [C, Cr]; q_w/k_w/v_w [C, C]; kdw_w/vdw_w [C, 3, 3]; biases [out]."""
    rng = np.random.default_rng(seed)
    N = H * W
    x = rng.standard_normal((B, N, C), dtype=np.float32)
    if outliers:
        k = int(round(0.05 * N))
        for b in range(B):
            idx = rng.choice(N, k, replace=False)
            x[b, idx, :] *= np.float32(8.0)
    d = {"x": x}
    d["cf3_w"] = _normal(rng, (c_red, 3, 3, C), 1.0 / (9 * C))
    d["cf1_w"] = _normal(rng, (C, c_red), 1.0 / c_red)
    d["q_w"] = _normal(rng, (C, C), 1.0 / C)
    d["k_w"] = _normal(rng, (C, C), 1.0 / C)
    d["v_w"] = _normal(rng, (C, C), 1.0 / C)
    d["kdw_w"] = _normal(rng, (C, 3, 3), 1.0 / 9)
    d["vdw_w"] = _normal(rng, (C, 3, 3), 1.0 / 9)
    if n_txt is not None:
        d["x_txt"] = rng.standard_normal((B, n_txt, C), dtype=np.float32)
        d["tq_w"] = _normal(rng, (C, C), 1.0 / C)
        d["tk_w"] = _normal(rng, (C, C), 1.0 / C)
        d["tv_w"] = _normal(rng, (C, C), 1.0 / C)
    zeros = lambda n: np.zeros((n,), dtype=np.float32)  # noqa: E731
    d["cf3_b"] = zeros(c_red)
    d["gn_gamma"] = np.ones((c_red,), dtype=np.float32)
    d["gn_beta"] = zeros(c_red)
    for name in ("cf1_b", "q_b", "k_b", "v_b", "kdw_b", "vdw_b"):
        d[name] = zeros(C)
    if n_txt is not None:
        for name in ("tq_b", "tk_b", "tv_b"):
            d[name] = zeros(C)
    if nonzero_affine:
        d["cf3_b"] = _normal(rng, (c_red,), 0.01)
        d["gn_gamma"] = (1.0 + _normal(rng, (c_red,), 0.01)).astype(np.float32)
        d["gn_beta"] = _normal(rng, (c_red,), 0.01)
        for name in ("cf1_b", "q_b", "k_b", "v_b", "kdw_b", "vdw_b"):
            d[name] = _normal(rng, (C,), 0.01)
        if n_txt is not None:
            for name in ("tq_b", "tk_b", "tv_b"):
                d[name] = _normal(rng, (C,), 0.01)
    if variant_weights:
        d["kcf3_w"] = _normal(rng, (c_red, 3, 3, C), 1.0 / (9 * C))
        d["kcf1_w"] = _normal(rng, (C, c_red), 1.0 / c_red)
        d["o_w"] = _normal(rng, (C, C), 1.0 / C)
        d["kcf3_b"] = zeros(c_red)
        d["kgn_gamma"] = np.ones((c_red,), dtype=np.float32)
        d["kgn_beta"] = zeros(c_red)
        d["kcf1_b"] = zeros(C)
        d["o_b"] = zeros(C)
        if nonzero_affine:
            d["kcf3_b"] = _normal(rng, (c_red,), 0.01)
            d["kgn_gamma"] = (1.0 + _normal(rng, (c_red,), 0.01)).astype(np.float32)
            d["kgn_beta"] = _normal(rng, (c_red,), 0.01)
            d["kcf1_b"] = _normal(rng, (C,), 0.01)
            d["o_b"] = _normal(rng, (C,), 0.01)
    if dit_block:
        # the DiT block around the attention: caption tokens y [B, n_cap, C], the
        # sample's timestep modulation t6 [B, 6, C] (N(0, 0.1^2)), the block's
        # modulation table sst [6, C] (N(0, 1/C)), the attention's output Linear,
        # the cross-attention Linears and the MLP (hidden units), fan-in variances
        n_cap, hidden = dit_block["n_cap"], dit_block["hidden"]
        d["y"] = rng.standard_normal((B, n_cap, C), dtype=np.float32)
        d["t6"] = _normal(rng, (B, 6, C), 0.01)
        d["sst"] = _normal(rng, (6, C), 1.0 / C)
        if "o_w" not in d:
            d["o_w"] = _normal(rng, (C, C), 1.0 / C)
            d["o_b"] = zeros(C)
        for n in ("cq_w", "ck_w", "cv_w", "co_w"):
            d[n] = _normal(rng, (C, C), 1.0 / C)
        d["fc1_w"] = _normal(rng, (hidden, C), 1.0 / C)
        d["fc2_w"] = _normal(rng, (C, hidden), 1.0 / hidden)
        for n in ("cq_b", "ck_b", "cv_b", "co_b", "fc2_b"):
            d[n] = zeros(C)
        d["fc1_b"] = zeros(hidden)
        if nonzero_affine:
            for n in ("cq_b", "ck_b", "cv_b", "co_b", "fc2_b", "o_b"):
                d[n] = _normal(rng, (C,), 0.01)
            d["fc1_b"] = _normal(rng, (hidden,), 0.01)
    if dtype == "bf16":
        d = {k: round_bf16(v) for k, v in d.items()}
    d.update(dict(c_red=c_red, gn_groups=gn_groups, **DECLARED))
    if dit_block:
        d["ln_eps"] = 1e-6
    return d


def make_workload(name, **overrides):
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    return cfg, make_inputs(**cfg)


def make_attention_inputs(B, N, M, C, seed, dtype="bf16"):
    """Operands of the linear-attention step alone: q [B, N, C] and k [B, M, C]
    non-negative (|N(0, 1)| draws, like the ReLU feature maps the layer feeds
    it), v [B, M, C] ~ N(0, 1); drawn in that order from
    ``numpy.random.default_rng(seed)`` and rounded once to bf16 for bf16."""
    rng = np.random.default_rng(seed)
    q = np.abs(rng.standard_normal((B, N, C), dtype=np.float32))
    k = np.abs(rng.standard_normal((B, M, C), dtype=np.float32))
    v = rng.standard_normal((B, M, C), dtype=np.float32)
    if dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    return q, k, v
