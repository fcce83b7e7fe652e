"""Plain fp64 CPU oracle for the EDiT linear compressed attention forward pass
and the MM-EDiT hybrid.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this module: only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` use it. It shares no code with the
CUDA library (no kernels, headers, helpers, tables or pre/post-processing).

Source: the paper-notes page "EDiT: Efficient Diffusion Transformers with
Linear Compressed Attention" (ICCV 2025, arXiv 2503.16726), section
"Method in detail" (方法详解):

* ConvFusion query, eq. (Q^EDiT):
  Q = ReLU(Linear(X + Conv(LeakyReLU(GN(Conv(X)))))), with the sequence
  reshaped to its 2D grid, the first conv a 3x3 channel compressor and the
  second a 1x1 channel restorer.
* Spatial Compressor, eq. (K^EDiT, V^EDiT, phi_SC):
  K = ReLU(phi_SC(X)), V = phi_SC(X), phi_SC(X) = Conv(Linear(X)) with a 3x3
  depthwise conv of stride 2 (4x fewer key/value tokens).
* Linear attention, eq. (y_i): y_i = Q_i (sum_j K_j^T V_j) / (Q_i sum_j K_j).
* MM-EDiT, eq. (A^Hybrid) and the token-ratio approximation
  eta = N_I / (N_I + N_T), or the exact normaliser it stands in for.

Everything is float64, computed from the given (possibly bf16-rounded) inputs
with no intermediate rounding. Library primitives used as steps: numpy matmul
(``@``), sums, exp, max. Readings of points the page leaves open are marked
``[R#]``; the list is kept with the design notes of this repository.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(closed forms, brute force, PyTorch-CPU fp64 library special cases and
invariants); the choice of readings R1 and R12 themselves cannot be pinned by
the page ("parity unpinned" for those readings only, not for the arithmetic).
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


def _f64(a):
    return np.asarray(a, dtype=F64)


# --------------------------------------------------------------------------
# Primitives (each one is the textbook definition written out)
# --------------------------------------------------------------------------

def grid_view(x, H, W):
    """[B, N, C] token sequence -> [B, H, W, C] grid, token n = h*W + w.

    ConvFusion "key design": the 1D sequence is reshaped to the 2D image
    shape before the 2D convolutions. Row-major order is reading [R10].
    """
    x = _f64(x)
    B, N, C = x.shape
    assert N == H * W, (N, H, W)
    return x.reshape(B, H, W, C)


def conv3x3_same(X, w, b):
    """3x3 cross-correlation, stride 1, zero padding 1, with bias [R2].

    X: [B, H, W, Cin]; w: [Cout, 3, 3, Cin] (tap (kh, kw) reads input pixel
    (h + kh - 1, w + kw - 1)); b: [Cout]. Returns [B, H, W, Cout].
    ConvFusion eq. (Q^EDiT), inner Conv: "the first (3x3) conv compresses the
    channel dimension".
    """
    X, w, b = _f64(X), _f64(w), _f64(b)
    B, H, W, _ = X.shape
    Xp = np.zeros((B, H + 2, W + 2, X.shape[3]), dtype=F64)
    Xp[:, 1:H + 1, 1:W + 1, :] = X
    out = np.broadcast_to(b, (B, H, W, w.shape[0])).copy()
    for kh in range(3):
        for kw in range(3):
            out += Xp[:, kh:kh + H, kw:kw + W, :] @ w[:, kh, kw, :].T
    return out


def group_norm_stats(U, groups):
    """Per (batch, group) mean and biased variance over all pixels and the
    channels of the group (reading [R3]). U: [B, H, W, Cr].
    Returns (mean [B, G], var [B, G])."""
    U = _f64(U)
    B, H, W, Cr = U.shape
    assert Cr % groups == 0
    cpg = Cr // groups
    Ug = U.reshape(B, H * W, groups, cpg)
    mean = Ug.mean(axis=(1, 3))
    var = ((Ug - mean[:, None, :, None]) ** 2).mean(axis=(1, 3))
    return mean, var


def group_norm(U, groups, gamma, beta, eps):
    """GroupNorm with affine gamma/beta: gamma*(U - mean)/sqrt(var + eps) + beta.
    ConvFusion eq. (Q^EDiT), GN step ("Group Normalization for stability")."""
    U = _f64(U)
    B, H, W, Cr = U.shape
    cpg = Cr // groups
    mean, var = group_norm_stats(U, groups)
    mu_c = np.repeat(mean, cpg, axis=1)[:, None, None, :]
    var_c = np.repeat(var, cpg, axis=1)[:, None, None, :]
    return _f64(gamma) * (U - mu_c) / np.sqrt(var_c + eps) + _f64(beta)


def leaky_relu(x, slope):
    x = _f64(x)
    return np.where(x >= 0.0, x, slope * x)


def relu(x):
    x = _f64(x)
    return np.maximum(x, 0.0)


def linear(x, w, b):
    """torch-style Linear: y = x w^T + b, w: [out, in]."""
    return _f64(x) @ _f64(w).T + _f64(b)


def dwconv3x3_s2(Y, w, b):
    """Depthwise 3x3 conv, stride 2, zero padding 1, with bias [R11].

    Y: [B, H, W, C]; w: [C, 3, 3]; b: [C]. Output pixel (i, j) of channel c is
    b[c] + sum_{a, e in 0..2} w[c, a, e] * Y[2i + a - 1, 2j + e - 1, c], for
    i < ceil(H/2), j < ceil(W/2). Spatial Compressor eq. (phi_SC): "3x3
    depthwise conv, stride 2, reduces the number of keys/values by 4x".
    """
    Y, w, b = _f64(Y), _f64(w), _f64(b)
    B, H, W, C = Y.shape
    Ho, Wo = (H + 1) // 2, (W + 1) // 2
    Yp = np.zeros((B, H + 2, W + 2, C), dtype=F64)
    Yp[:, 1:H + 1, 1:W + 1, :] = Y
    out = np.broadcast_to(b, (B, Ho, Wo, C)).copy()
    for a in range(3):
        for e in range(3):
            # padded row index of tap a for output row i is 2i + a
            out += Yp[:, a:a + 2 * Ho - 1:2, e:e + 2 * Wo - 1:2, :] * w[:, a, e]
    return out


def compressed_count(H, W):
    """Number of key/value tokens after the stride-2, padding-1 compressor."""
    return ((H + 1) // 2) * ((W + 1) // 2)


def linear_attention(Q, K, V, heads, eps):
    """Per-head linear attention, eq. (y_i) with the declared eps [R7]:

        S_h = sum_j K_jh^T V_jh   (d x d),  z_h = sum_j K_jh   (d)
        y_ih = (Q_ih S_h) / (Q_ih . z_h + eps)

    Q: [B, N, C]; K, V: [B, M, C]; heads are contiguous channel blocks of
    d = C / heads [R9]; the sums run over the M compressed tokens [R6].
    Returns (y [B, N, C], S [B, heads, d, d], z [B, heads, d]).
    """
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, N, C = Q.shape
    d = C // heads
    y = np.empty_like(Q)
    S = np.empty((B, heads, d, d), dtype=F64)
    z = np.empty((B, heads, d), dtype=F64)
    for bi in range(B):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            Kh, Vh, Qh = K[bi, :, sl], V[bi, :, sl], Q[bi, :, sl]
            S[bi, h] = Kh.T @ Vh
            z[bi, h] = Kh.sum(axis=0)
            num = Qh @ S[bi, h]
            den = Qh @ z[bi, h] + eps
            y[bi, :, sl] = num / den[:, None]
    return y, S, z


def sdpa(q, k, v, heads):
    """Scaled dot-product attention per head, softmax(q k^T / sqrt(d)) v,
    normalised over its own key set [R12]. q: [B, Nq, C]; k, v: [B, Nk, C].
    An empty key set (Nk == 0) returns zeros: it only ever appears with a
    mixing weight of exactly 0 (eta = 1 when there are no prompt tokens)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Nq, C = q.shape
    Nk = k.shape[1]
    d = C // heads
    out = np.zeros((B, Nq, C), dtype=F64)
    if Nk == 0:
        return out
    scale = 1.0 / math.sqrt(d)
    for bi in range(B):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            s = (q[bi, :, sl] @ k[bi, :, sl].T) * scale
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[bi, :, sl] = p @ v[bi, :, sl]
    return out


def softmax_log_normaliser(q, k, heads):
    """log sum_j exp(q . k_j / sqrt(d)) per query row and head, the
    normaliser of sdpa() [R12]. q: [B, Nq, C]; k: [B, Nk, C]. Returns
    [B, Nq, heads]; -inf for an empty key set."""
    q, k = _f64(q), _f64(k)
    B, Nq, C = q.shape
    Nk = k.shape[1]
    d = C // heads
    out = np.full((B, Nq, heads), -np.inf)
    if Nk == 0:
        return out
    scale = 1.0 / math.sqrt(d)
    for bi in range(B):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            s = (q[bi, :, sl] @ k[bi, :, sl].T) * scale
            m = s.max(axis=1)
            out[bi, :, h] = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    return out


def mix_ratio(N_I, N_T):
    """eta = N_I / (N_I + N_T): eq. (A^Hybrid) normaliser approximated by
    the token-count ratio (eta_I and eta_P both take it [R13])."""
    return N_I / float(N_I + N_T)


# --------------------------------------------------------------------------
# EDiT layer
# --------------------------------------------------------------------------

def convfusion_residual(X, cf3_w, cf3_b, groups, gamma, beta, gn_eps, slope, cf1_w, cf1_b):
    """R = X + Conv1x1(LeakyReLU(GN(Conv3x3(X)))), the argument of the Linear
    in ConvFusion, eq. (Q^EDiT). X: [B, H, W, C] grid. Returns
    (R [B, H, W, C], U, gn_mean, gn_var, Lk) with U = Conv3x3(X) and
    Lk = LeakyReLU(GN(U))."""
    U = conv3x3_same(X, cf3_w, cf3_b)
    gn_mean, gn_var = group_norm_stats(U, groups)
    G = group_norm(U, groups, gamma, beta, gn_eps)
    Lk = leaky_relu(G, slope)
    # the 1x1 conv restoring the channels is a per-pixel Linear Cr -> C
    R = _f64(X) + linear(Lk, cf1_w, cf1_b)
    return R, U, gn_mean, gn_var, Lk


def edit_branches(x, H, W, w, heads):
    """The three branches of one EDiT layer, step by step.

    x: [B, N=H*W, C]. w: dict with the weights and declared constants
    (see tests/ and the C header for the names). Returns a dict of every
    intermediate, all float64:
      U  = Conv3x3(X)                                  [B, H, W, Cr]
      gn_mean, gn_var                                  [B, G]
      Lk = LeakyReLU(GN(U))                            [B, H, W, Cr]
      R  = X + Conv1x1(Lk)                             [B, N, C]
      Q  = ReLU(Linear_Q(R))                           [B, N, C]
      Kp, Vp = Linear_K(X), Linear_V(X)                [B, N, C]
      K  = ReLU(DW(Kp)), V = DW(Vp)                    [B, M, C]
    """
    B, N, C = np.shape(x)
    X = grid_view(x, H, W)
    # ConvFusion, eq. (Q^EDiT)
    R, U, gn_mean, gn_var, Lk = convfusion_residual(
        X, w["cf3_w"], w["cf3_b"], w["gn_groups"], w["gn_gamma"], w["gn_beta"], w["gn_eps"],
        w["leaky_slope"], w["cf1_w"], w["cf1_b"])
    Q = relu(linear(R, w["q_w"], w["q_b"]))
    # Spatial Compressor, eq. (phi_SC): Linear first, then the depthwise conv;
    # separate K and V weights [R1]
    Kp = linear(X, w["k_w"], w["k_b"])
    Vp = linear(X, w["v_w"], w["v_b"])
    K = relu(dwconv3x3_s2(Kp, w["kdw_w"], w["kdw_b"]))
    V = dwconv3x3_s2(Vp, w["vdw_w"], w["vdw_b"])
    Ho, Wo = K.shape[1], K.shape[2]
    return {
        "U": U, "gn_mean": gn_mean, "gn_var": gn_var, "Lk": Lk,
        "R": R.reshape(B, N, C), "Q": Q.reshape(B, N, C),
        "Kp": Kp.reshape(B, N, C), "Vp": Vp.reshape(B, N, C),
        "K": K.reshape(B, Ho * Wo, C), "V": V.reshape(B, Ho * Wo, C),
    }


def edit_forward(x, H, W, w, heads, return_intermediates=False):
    """EDiT linear compressed attention layer: out = y, eq. (y_i), with no
    1/sqrt(d) and no output projection [R8]. x: [B, H*W, C] -> [B, H*W, C]."""
    br = edit_branches(x, H, W, w, heads)
    y, S, z = linear_attention(br["Q"], br["K"], br["V"], heads, w["attn_eps"])
    if return_intermediates:
        br.update({"S": S, "z": z, "y": y})
        return y, br
    return y


# --------------------------------------------------------------------------
# MM-EDiT hybrid
# --------------------------------------------------------------------------

def mmedit_forward(x_img, x_txt, H, W, w, heads, return_intermediates=False, eta="ratio"):
    """MM-EDiT hybrid attention, eq. (A^Hybrid).

    Image rows: eta * A_lin(Q_I, K_I, V_I) + (1 - eta) * A(Q_I, K_P, V_P).
    Text rows:  eta * A(Q_P, K_I, V_I)     + (1 - eta) * A(Q_P, K_P, V_P).
    Q_I, K_I, V_I are the EDiT query and the compressed keys/values; the
    prompt side uses plain Linear projections, A is softmax attention with
    scale 1/sqrt(d) normalised per block [R12].

    eta="ratio": the page's approximation eta = N_I / (N_I + N_T) for both
    rows [R13]. eta="exact": the normaliser the page says the ratio stands in
    for [R22]: each query normalises once over all keys, image keys weighted by
    the linear kernel (Q_i . K_j, plus the layer's eps) and prompt keys by
    exp(q . k / sqrt(d)). Per query row and head that is
      image rows: eta_i = (Q_i z + eps) / (Q_i z + eps + sum_P exp(q.k/sqrt(d)))
      text rows:  eta_i = Z_I / (Z_I + Z_P), Z = sum_j exp(q.k_j/sqrt(d)) over
                  the image (I) or prompt (P) keys, i.e. one softmax over both.
    Returns (out_img [B, N_I, C], out_txt [B, N_T, C]).
    """
    x_txt = _f64(x_txt)
    B, N_T, C = x_txt.shape
    N_I = H * W
    br = edit_branches(x_img, H, W, w, heads)
    y_lin, S, z = linear_attention(br["Q"], br["K"], br["V"], heads, w["attn_eps"])
    Qp = linear(x_txt, w["tq_w"], w["tq_b"])
    Kp = linear(x_txt, w["tk_w"], w["tk_b"])
    Vp = linear(x_txt, w["tv_w"], w["tv_b"])
    a_ip = sdpa(br["Q"], Kp, Vp, heads)
    a_pi = sdpa(Qp, br["K"], br["V"], heads)
    a_pp = sdpa(Qp, Kp, Vp, heads)
    if eta == "ratio":
        eta = mix_ratio(N_I, N_T)
        out_img = eta * y_lin + (1.0 - eta) * a_ip
        out_txt = eta * a_pi + (1.0 - eta) * a_pp
    elif eta == "exact":
        d = C // heads
        Q = br["Q"]
        den = np.empty((B, N_I, heads))           # Q_i z + eps, the linear part's normaliser
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            den[:, :, h] = np.einsum("bnc,bc->bn", Q[:, :, sl], z[:, h]) + w["attn_eps"]
        # eta = A / (A + B) written as 1 / (1 + exp(log B - log A)), which stays finite
        eta_i = 1.0 / (1.0 + np.exp(softmax_log_normaliser(Q, Kp, heads) - np.log(den)))
        eta_p = 1.0 / (1.0 + np.exp(softmax_log_normaliser(Qp, Kp, heads) -
                                    softmax_log_normaliser(Qp, br["K"], heads)))
        per_col = lambda e: np.repeat(e, d, axis=2)  # noqa: E731  (heads -> their d columns)
        out_img = per_col(eta_i) * y_lin + (1.0 - per_col(eta_i)) * a_ip
        out_txt = per_col(eta_p) * a_pi + (1.0 - per_col(eta_p)) * a_pp
        eta = (eta_i, eta_p)
    else:
        raise ValueError(f"eta must be 'ratio' or 'exact', not {eta!r}")
    if return_intermediates:
        br.update({"S": S, "z": z, "y": y_lin, "Qp": Qp, "Kp_txt": Kp,
                   "Vp_txt": Vp, "A_ip": a_ip, "A_pi": a_pi, "A_pp": a_pp,
                   "eta": eta})
        return out_img, out_txt, br
    return out_img, out_txt


# --------------------------------------------------------------------------
# Ablation variants of the query/key/value processing, optional output
# projection
# --------------------------------------------------------------------------

PROC_NONE, PROC_CF, PROC_SC = "none", "cf", "sc"
# (q, k, v) processing combinations with equal key and value counts: the
# ablation table "Query/Key/Value processing" (消融实验) lists (CF, SC, SC),
# (CF, CF, -), (-, SC, SC) and (CF, -, -); the query choice is independent of
# the key/value choice, so both queries go with every key/value pair.
KV_PAIRS = ((PROC_SC, PROC_SC), (PROC_CF, PROC_NONE), (PROC_NONE, PROC_NONE))


def edit_variant_forward(x, H, W, w, heads, q_proc=PROC_CF, k_proc=PROC_SC, v_proc=PROC_SC, out_proj=False,
                         return_intermediates=False):
    """One EDiT layer with the query, key and value processing chosen as in the
    ablation table of the EDiT notes page (section 消融实验, "Query/Key/Value
    processing"), followed by an optional output projection.

    Readings [R20] (the table names only the processing, not the formula):
      query  cf:   Q = ReLU(Linear_Q(X + Conv1x1(LeakyReLU(GN(Conv3x3(X))))))
             none: Q = ReLU(Linear_Q(X))      (the ReLU feature map stays)
      key    sc:   K = ReLU(DW_K(Linear_K(X)))                       M tokens
             cf:   K = ReLU(Linear_K(X + Conv1x1_K(LeakyReLU(GN_K(Conv3x3_K(X))))))
                   with the key's own ConvFusion weights (kcf3_w, kcf3_b,
                   kgn_gamma, kgn_beta, kcf1_w, kcf1_b)             N tokens
             none: K = ReLU(Linear_K(X))                             N tokens
      value  sc:   V = DW_V(Linear_V(X));  none: V = Linear_V(X)
    then y = eq. (y_i) over the M (or N) key/value tokens and, with
    out_proj, out = y o_w^T + o_b (the attention block's output Linear;
    the page's layer has none [R8], so it is an option here [R21]).
    (cf, sc, sc) without out_proj is edit_forward.
    """
    if q_proc not in (PROC_CF, PROC_NONE) or (k_proc, v_proc) not in KV_PAIRS:
        raise ValueError(f"unsupported processing ({q_proc}, {k_proc}, {v_proc})")
    B, N, C = np.shape(x)
    X = grid_view(x, H, W)
    it = {}
    if q_proc == PROC_CF:
        R = convfusion_residual(X, w["cf3_w"], w["cf3_b"], w["gn_groups"], w["gn_gamma"], w["gn_beta"],
                                w["gn_eps"], w["leaky_slope"], w["cf1_w"], w["cf1_b"])[0]
        Q = relu(linear(R, w["q_w"], w["q_b"]))
    else:
        Q = relu(linear(X, w["q_w"], w["q_b"]))
    Kp = linear(X, w["k_w"], w["k_b"])
    Vp = linear(X, w["v_w"], w["v_b"])
    if k_proc == PROC_SC:
        K = relu(dwconv3x3_s2(Kp, w["kdw_w"], w["kdw_b"]))
        V = dwconv3x3_s2(Vp, w["vdw_w"], w["vdw_b"])
    else:
        if k_proc == PROC_CF:
            RK = convfusion_residual(X, w["kcf3_w"], w["kcf3_b"], w["gn_groups"], w["kgn_gamma"], w["kgn_beta"],
                                     w["gn_eps"], w["leaky_slope"], w["kcf1_w"], w["kcf1_b"])[0]
            K = relu(linear(RK, w["k_w"], w["k_b"]))
        else:
            K = relu(Kp)
        V = Vp
    Q = Q.reshape(B, N, C)
    K = K.reshape(B, -1, C)
    V = V.reshape(B, -1, C)
    y, S, z = linear_attention(Q, K, V, heads, w["attn_eps"])
    out = linear(y, w["o_w"], w["o_b"]) if out_proj else y
    if return_intermediates:
        it.update({"Q": Q, "K": K, "V": V, "S": S, "z": z, "y": y})
        return out, it
    return out


# --------------------------------------------------------------------------
# The DiT block around the attention [R23]
# --------------------------------------------------------------------------

def layer_norm(x, eps):
    """LayerNorm over the last axis without affine weights: (x - mean) /
    sqrt(biased var + eps)."""
    x = _f64(x)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps)


def gelu_tanh(x):
    """GELU with the tanh approximation: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = _f64(x)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def dit_block_forward(x, y, t6, H, W, w, heads):
    """One text-to-image DiT block of the PixArt-Sigma kind with EDiT as its
    self-attention [R23] (the notes page: EDiT replaces the attention of
    PixArt-Sigma's blocks; the block itself is that model's, not the page's).

    x: [B, N, C] image tokens; y: [B, N_T, C] caption tokens; t6: [B, 6, C]
    the sample's timestep modulation. With m = sst + t6 split into
    (shift_a, scale_a, gate_a, shift_f, scale_f, gate_f):
      x1 = x + gate_a * (EDiT(LN(x) (1 + scale_a) + shift_a) o_w^T + o_b)
      x2 = x1 + (A(x1 cq_w^T + cq_b, y ck_w^T + ck_b, y cv_w^T + cv_b) co_w^T + co_b)
      out = x2 + gate_f * (GELU(LN(x2) (1 + scale_f) + shift_f) fc1_w^T + fc1_b) fc2_w^T + fc2_b)
    with LN the LayerNorm without affine (eps w["ln_eps"]), A softmax attention
    per head (scale 1/sqrt(d)) and GELU the tanh form."""
    x, y, t6 = _f64(x), _f64(y), _f64(t6)
    m = _f64(w["sst"])[None] + t6                      # [B, 6, C]
    sh_a, sc_a, g_a, sh_f, sc_f, g_f = (m[:, k][:, None, :] for k in range(6))
    h1 = layer_norm(x, w["ln_eps"]) * (1.0 + sc_a) + sh_a
    a = linear(edit_forward(h1, H, W, w, heads), w["o_w"], w["o_b"])
    x1 = x + g_a * a
    q = linear(x1, w["cq_w"], w["cq_b"])
    k = linear(y, w["ck_w"], w["ck_b"])
    v = linear(y, w["cv_w"], w["cv_b"])
    x2 = x1 + linear(sdpa(q, k, v, heads), w["co_w"], w["co_b"])
    h2 = layer_norm(x2, w["ln_eps"]) * (1.0 + sc_f) + sh_f
    f = gelu_tanh(linear(h2, w["fc1_w"], w["fc1_b"]))
    return x2 + g_f * linear(f, w["fc2_w"], w["fc2_b"])
