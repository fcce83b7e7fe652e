"""Pins for the fp64 oracle, against things other than the oracle itself:
hand-worked values from the EDiT notes page's definitions, closed forms,
brute force on tiny inputs, invariants, and special cases that reduce to
PyTorch CPU float64 library routines (conv2d, group_norm, avg_pool2d,
scaled_dot_product_attention). The last section plants plausible mistakes in
copies of the oracle and checks that a pin catches each one.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle.edit_oracle as O
from linear_compressed_attention_b200.inputs import make_inputs, make_workload

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))

torch.set_default_dtype(torch.float64)


def rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def small_cfg(**kw):
    c = dict(B=2, H=6, W=5, C=16, c_red=8, gn_groups=2, heads=2, seed=11,
             dtype="f32", nonzero_affine=True)
    c.update(kw)
    return c


# ---------------------------------------------------------------- hand-worked

def test_linear_attention_hand_worked():
    g = GOLDEN["linear_attention"]
    Q = np.array(g["Q"], float)[None]
    K = np.array(g["K"], float)[None]
    V = np.array(g["V"], float)[None]
    y, S, z = O.linear_attention(Q, K, V, heads=1, eps=0.0)
    assert np.allclose(S[0, 0], g["S"], rtol=0, atol=1e-14)
    assert np.allclose(z[0, 0], g["z"], rtol=0, atol=1e-14)
    assert np.allclose(y[0], g["y"], rtol=1e-15, atol=1e-15)


def test_dwconv_hand_worked():
    g = GOLDEN["dwconv_s2"]
    Y = np.array(g["Y"], float)[None, :, :, None]
    out = O.dwconv3x3_s2(Y, np.ones((1, 3, 3)), np.zeros(1))
    assert np.array_equal(out[0, :, :, 0], np.array(g["out"], float))


def test_mix_ratio_exact():
    g = GOLDEN["mix_ratio"]
    eta = O.mix_ratio(g["N_I"], g["N_T"])
    assert Fraction(eta).limit_denominator(100000) == Fraction(g["numerator"], g["denominator"])
    assert eta == g["numerator"] / g["denominator"]
    assert O.mix_ratio(4096, 0) == 1.0


@pytest.mark.parametrize("H,W,M", GOLDEN["compressed_count"]["cases"])
def test_compressed_count(H, W, M):
    assert O.compressed_count(H, W) == M == math.ceil(H / 2) * math.ceil(W / 2)
    if H * W <= 400:
        Y = np.random.default_rng(0).standard_normal((1, H, W, 3))
        out = O.dwconv3x3_s2(Y, np.ones((3, 3, 3)), np.zeros(3))
        assert out.shape[1] * out.shape[2] == M


# ------------------------------------------------- brute force / closed forms

def _brute_linear_attention(Q, K, V, eps):
    """Explicit O(N*M) form: y_i = sum_j (Q_i.K_j) V_j / (sum_j Q_i.K_j + eps),
    with pure Python loops (associativity of the matrix product)."""
    N, d = Q.shape
    M = K.shape[0]
    y = np.zeros((N, V.shape[1]))
    for i in range(N):
        num = [0.0] * V.shape[1]
        den = 0.0
        for j in range(M):
            a = sum(Q[i, t] * K[j, t] for t in range(d))
            den += a
            for c in range(V.shape[1]):
                num[c] += a * V[j, c]
        for c in range(V.shape[1]):
            y[i, c] = num[c] / (den + eps)
    return y


def test_linear_attention_vs_brute_force():
    rng = np.random.default_rng(3)
    heads, d = 2, 3
    Q = np.maximum(rng.standard_normal((1, 5, heads * d)), 0) + 0.01
    K = np.maximum(rng.standard_normal((1, 7, heads * d)), 0) + 0.01
    V = rng.standard_normal((1, 7, heads * d))
    y, S, z = O.linear_attention(Q, K, V, heads, eps=1e-6)
    for h in range(heads):
        sl = slice(h * d, (h + 1) * d)
        ref = _brute_linear_attention(Q[0, :, sl], K[0, :, sl], V[0, :, sl], 1e-6)
        assert rel(y[0, :, sl], ref) < 1e-12
        # S and z against the sums written element by element
        for a in range(d):
            assert abs(z[0, h, a] - sum(K[0, j, h * d + a] for j in range(7))) < 1e-12
            for b in range(d):
                s = sum(K[0, j, h * d + a] * V[0, j, h * d + b] for j in range(7))
                assert abs(S[0, h, a, b] - s) < 1e-12


def test_sdpa_vs_textbook_softmax_and_torch():
    rng = np.random.default_rng(4)
    heads, d = 3, 4
    q = rng.standard_normal((2, 5, heads * d))
    k = rng.standard_normal((2, 6, heads * d))
    v = rng.standard_normal((2, 6, heads * d))
    out = O.sdpa(q, k, v, heads)
    # textbook softmax without max subtraction, pure Python loops
    for bi in range(2):
        for h in range(heads):
            for i in range(5):
                w = []
                for j in range(6):
                    s = sum(q[bi, i, h * d + t] * k[bi, j, h * d + t] for t in range(d))
                    w.append(math.exp(s / math.sqrt(d)))
                tot = sum(w)
                for c in range(d):
                    ref = sum(w[j] * v[bi, j, h * d + c] for j in range(6)) / tot
                    assert abs(out[bi, i, h * d + c] - ref) < 1e-12
    tq = torch.tensor(q).reshape(2, 5, heads, d).transpose(1, 2)
    tk = torch.tensor(k).reshape(2, 6, heads, d).transpose(1, 2)
    tv = torch.tensor(v).reshape(2, 6, heads, d).transpose(1, 2)
    ref = F.scaled_dot_product_attention(tq, tk, tv).transpose(1, 2).reshape(2, 5, heads * d)
    assert rel(out, ref.numpy()) < 1e-12


# --------------------------------------------- library special cases (torch)

def test_conv3x3_vs_torch_conv2d():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((2, 7, 5, 6))
    w = rng.standard_normal((4, 3, 3, 6))
    b = rng.standard_normal(4)
    out = O.conv3x3_same(X, w, b)
    ref = F.conv2d(torch.tensor(X).permute(0, 3, 1, 2), torch.tensor(w).permute(0, 3, 1, 2),
                   torch.tensor(b), stride=1, padding=1).permute(0, 2, 3, 1)
    assert rel(out, ref.numpy()) < 1e-13


def test_group_norm_vs_torch():
    rng = np.random.default_rng(6)
    U = rng.standard_normal((2, 4, 3, 8)) * 3 + 1
    gam, bet = rng.standard_normal(8), rng.standard_normal(8)
    out = O.group_norm(U, 2, gam, bet, 1e-5)
    ref = F.group_norm(torch.tensor(U).permute(0, 3, 1, 2), 2, torch.tensor(gam),
                       torch.tensor(bet), eps=1e-5).permute(0, 2, 3, 1)
    assert rel(out, ref.numpy()) < 1e-12


def test_linear_leaky_relu_vs_torch():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((3, 5))
    w, b = rng.standard_normal((4, 5)), rng.standard_normal(4)
    assert rel(O.linear(x, w, b), F.linear(torch.tensor(x), torch.tensor(w), torch.tensor(b)).numpy()) < 1e-14
    assert rel(O.leaky_relu(x, 0.01), F.leaky_relu(torch.tensor(x), 0.01).numpy()) < 1e-15
    assert rel(O.relu(x), F.relu(torch.tensor(x)).numpy()) < 1e-15


@pytest.mark.parametrize("H,W", [(6, 6), (5, 7), (1, 1), (2, 3), (9, 4)])
def test_dwconv_vs_torch_depthwise(H, W):
    rng = np.random.default_rng(H * 100 + W)
    C = 5
    Y = rng.standard_normal((2, H, W, C))
    w, b = rng.standard_normal((C, 3, 3)), rng.standard_normal(C)
    out = O.dwconv3x3_s2(Y, w, b)
    ref = F.conv2d(torch.tensor(Y).permute(0, 3, 1, 2), torch.tensor(w)[:, None], torch.tensor(b),
                   stride=2, padding=1, groups=C).permute(0, 2, 3, 1)
    assert out.shape == tuple(ref.shape)
    assert rel(out, ref.numpy()) < 1e-13


def test_dwconv_centre_tap_is_subsampling_and_uniform_is_avgpool():
    rng = np.random.default_rng(8)
    Y = rng.standard_normal((1, 7, 6, 3))
    w = np.zeros((3, 3, 3))
    w[:, 1, 1] = 1.0
    out = O.dwconv3x3_s2(Y, w, np.zeros(3))
    assert np.array_equal(out, Y[:, ::2, ::2, :])
    out = O.dwconv3x3_s2(Y, np.full((3, 3, 3), 1.0 / 9), np.zeros(3))
    ref = F.avg_pool2d(torch.tensor(Y).permute(0, 3, 1, 2), 3, 2, 1,
                       count_include_pad=True).permute(0, 2, 3, 1)
    assert rel(out, ref.numpy()) < 1e-14


def _torch_edit_layer(d, cfg):
    """A second composition of the layer from PyTorch CPU float64 library
    routines, with the explicit quadratic form for the attention step."""
    B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    t = {k: torch.tensor(np.asarray(v, np.float64)) for k, v in d.items() if isinstance(v, np.ndarray)}
    X = t["x"].reshape(B, H, W, C).permute(0, 3, 1, 2)
    U = F.conv2d(X, t["cf3_w"].permute(0, 3, 1, 2), t["cf3_b"], padding=1)
    G = F.group_norm(U, d["gn_groups"], t["gn_gamma"], t["gn_beta"], eps=d["gn_eps"])
    L = F.leaky_relu(G, d["leaky_slope"])
    R = X + F.conv2d(L, t["cf1_w"][:, :, None, None], t["cf1_b"])
    Rt = R.permute(0, 2, 3, 1).reshape(B, H * W, C)
    Q = F.relu(F.linear(Rt, t["q_w"], t["q_b"]))
    Kp = F.linear(t["x"], t["k_w"], t["k_b"]).reshape(B, H, W, C).permute(0, 3, 1, 2)
    Vp = F.linear(t["x"], t["v_w"], t["v_b"]).reshape(B, H, W, C).permute(0, 3, 1, 2)
    K = F.relu(F.conv2d(Kp, t["kdw_w"][:, None], t["kdw_b"], stride=2, padding=1, groups=C))
    V = F.conv2d(Vp, t["vdw_w"][:, None], t["vdw_b"], stride=2, padding=1, groups=C)
    K = K.permute(0, 2, 3, 1).reshape(B, -1, C)
    V = V.permute(0, 2, 3, 1).reshape(B, -1, C)
    dh = C // heads
    q = Q.reshape(B, -1, heads, dh).transpose(1, 2)
    k = K.reshape(B, -1, heads, dh).transpose(1, 2)
    v = V.reshape(B, -1, heads, dh).transpose(1, 2)
    A = q @ k.transpose(-1, -2)                     # [B, h, N, M] = Q_i . K_j
    y = (A @ v) / (A.sum(-1, keepdim=True) + d["attn_eps"])
    return y.transpose(1, 2).reshape(B, -1, C).numpy(), Q.numpy(), K.numpy(), V.numpy()


@pytest.mark.parametrize("cfgkw", [dict(), dict(H=5, W=7), dict(H=1, W=1, B=1), dict(H=4, W=3, heads=4)])
def test_edit_layer_vs_torch_composition(cfgkw):
    cfg = small_cfg(**cfgkw)
    d = make_inputs(**cfg)
    y, inter = O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"], return_intermediates=True)
    y_t, Q_t, K_t, V_t = _torch_edit_layer(d, cfg)
    assert rel(inter["Q"], Q_t) < 1e-12
    assert rel(inter["K"], K_t) < 1e-12
    assert rel(inter["V"], V_t) < 1e-12
    assert rel(y, y_t) < 1e-11


def test_tiny_workload_vs_torch_composition():
    cfg, d = make_workload("tiny_fp32")
    y = O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"])
    y_t = _torch_edit_layer(d, cfg)[0]
    assert rel(y, y_t) < 1e-11


def test_zero_conv3x3_collapses_to_library_ops():
    """With a zero 3x3 conv, U = 0, GN(0) = beta, and
    Q = ReLU(Linear(X + Conv1x1(LeakyReLU(beta))))."""
    cfg = small_cfg()
    d = make_inputs(**cfg)
    d["cf3_w"] = np.zeros_like(d["cf3_w"])
    d["cf3_b"] = np.zeros_like(d["cf3_b"])
    _, inter = O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"], return_intermediates=True)
    beta = torch.tensor(d["gn_beta"].astype(np.float64))
    res = F.linear(F.leaky_relu(beta, 0.01), torch.tensor(d["cf1_w"].astype(np.float64)),
                   torch.tensor(d["cf1_b"].astype(np.float64)))
    Q = F.relu(F.linear(torch.tensor(d["x"].astype(np.float64)) + res,
                        torch.tensor(d["q_w"].astype(np.float64)), torch.tensor(d["q_b"].astype(np.float64))))
    assert rel(inter["Q"], Q.numpy()) < 1e-13


# ----------------------------------------------------------------- invariants

def _layer(cfg, d):
    return O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"], return_intermediates=True)


def test_denominator_positive_and_convex_combination():
    cfg = small_cfg(nonzero_affine=False)
    d = make_inputs(**cfg)
    y, it = _layer(cfg, d)
    dh = cfg["C"] // cfg["heads"]
    for bi in range(cfg["B"]):
        for h in range(cfg["heads"]):
            sl = slice(h * dh, (h + 1) * dh)
            den = it["Q"][bi, :, sl] @ it["z"][bi, h] + d["attn_eps"]
            assert den.min() >= d["attn_eps"]
            big = den > 1e3 * d["attn_eps"]
            Vh = it["V"][bi, :, sl]
            lo, hi = Vh.min(axis=0), Vh.max(axis=0)
            yh = y[bi, big][:, sl]
            assert np.all(yh >= lo - 1e-9) and np.all(yh <= hi + 1e-9)


def test_scale_laws():
    rng = np.random.default_rng(9)
    Q = np.maximum(rng.standard_normal((1, 9, 8)), 0) + 0.1
    K = np.maximum(rng.standard_normal((1, 6, 8)), 0) + 0.1
    V = rng.standard_normal((1, 6, 8))
    y0 = O.linear_attention(Q, K, V, 2, 0.0)[0]
    assert rel(O.linear_attention(3.0 * Q, K, V, 2, 0.0)[0], y0) < 1e-14
    assert rel(O.linear_attention(Q, 0.25 * K, V, 2, 0.0)[0], y0) < 1e-14
    assert rel(O.linear_attention(Q, K, -2.5 * V, 2, 0.0)[0], -2.5 * y0) < 1e-14


def test_batch_independence():
    cfg = small_cfg(B=2)
    d = make_inputs(**cfg)
    y = O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"])
    for bi in range(2):
        yb = O.edit_forward(d["x"][bi:bi + 1], cfg["H"], cfg["W"], d, cfg["heads"])
        assert np.array_equal(yb[0], y[bi])


def test_shared_kv_weights_gives_literal_reading():
    """Reading R1: with the same Linear and depthwise weights for K and V,
    K = ReLU(phi_SC(X)) and V = phi_SC(X), i.e. K == ReLU(V)."""
    cfg = small_cfg()
    d = make_inputs(**cfg)
    d["v_w"], d["v_b"], d["vdw_w"], d["vdw_b"] = d["k_w"], d["k_b"], d["kdw_w"], d["kdw_b"]
    _, it = _layer(cfg, d)
    assert np.array_equal(it["K"], np.maximum(it["V"], 0.0))


# ----------------------------------------------------------------- MM-EDiT

def _torch_mm(d, cfg):
    B, C, heads = cfg["B"], cfg["C"], cfg["heads"]
    y, Q, K, V = _torch_edit_layer(d, cfg)
    t = {k: torch.tensor(np.asarray(v, np.float64)) for k, v in d.items() if isinstance(v, np.ndarray)}
    Qp = F.linear(t["x_txt"], t["tq_w"], t["tq_b"])
    Kp = F.linear(t["x_txt"], t["tk_w"], t["tk_b"])
    Vp = F.linear(t["x_txt"], t["tv_w"], t["tv_b"])
    dh = C // heads

    def att(q, k, v):
        sh = lambda a: a.reshape(B, -1, heads, dh).transpose(1, 2)  # noqa: E731
        return F.scaled_dot_product_attention(sh(torch.as_tensor(q)), sh(torch.as_tensor(k)),
                                              sh(torch.as_tensor(v))).transpose(1, 2).reshape(B, -1, C)

    NI, NT = cfg["H"] * cfg["W"], d["x_txt"].shape[1]
    eta = Fraction(NI, NI + NT)
    e = float(eta)
    out_i = e * torch.tensor(y) + (1 - e) * att(Q, Kp, Vp)
    out_p = e * att(Qp, K, V) + (1 - e) * att(Qp, Kp, Vp)
    return out_i.numpy(), out_p.numpy()


def test_mmedit_vs_torch_composition():
    cfg = small_cfg(n_txt=5)
    d = make_inputs(**cfg)
    oi, op = O.mmedit_forward(d["x"], d["x_txt"], cfg["H"], cfg["W"], d, cfg["heads"])
    ri, rp = _torch_mm(d, cfg)
    assert rel(oi, ri) < 1e-11 and rel(op, rp) < 1e-11


def test_mmedit_without_text_is_edit():
    cfg = small_cfg(n_txt=0)
    d = make_inputs(**cfg)
    oi, op = O.mmedit_forward(d["x"], d["x_txt"], cfg["H"], cfg["W"], d, cfg["heads"])
    y = O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"])
    assert op.shape == (cfg["B"], 0, cfg["C"])
    assert np.array_equal(oi, y)


def test_mmedit_exact_eta_prompt_rows_are_one_softmax_over_all_keys():
    """Exact eta, prompt rows: one softmax over the image and prompt keys
    together (PyTorch CPU fp64 scaled_dot_product_attention on the
    concatenated key and value sets)."""
    cfg = small_cfg(n_txt=5)
    d = make_inputs(**cfg)
    B, C, heads = cfg["B"], cfg["C"], cfg["heads"]
    _, op, it = O.mmedit_forward(d["x"], d["x_txt"], cfg["H"], cfg["W"], d, heads, return_intermediates=True,
                                 eta="exact")
    dh = C // heads
    sh = lambda a: torch.as_tensor(a).reshape(B, -1, heads, dh).transpose(1, 2)  # noqa: E731
    k = np.concatenate([it["K"], it["Kp_txt"]], axis=1)
    v = np.concatenate([it["V"], it["Vp_txt"]], axis=1)
    ref = F.scaled_dot_product_attention(sh(it["Qp"]), sh(k), sh(v)).transpose(1, 2).reshape(B, -1, C).numpy()
    assert rel(op, ref) < 1e-12


def test_mmedit_exact_eta_image_rows_brute_force():
    """Exact eta, image rows, pure-Python loops on a tiny case: every key
    weighted once, image keys by Q_i . K_j, prompt keys by
    exp(q . k / sqrt(d)), one normalisation with the layer's eps:
    out_i = (sum_j w_j v_j) / (sum_j w_j + eps)."""
    cfg = dict(B=1, H=3, W=3, C=8, c_red=4, gn_groups=2, heads=2, dtype="f32", seed=71, n_txt=3,
               nonzero_affine=True)
    d = make_inputs(**cfg)
    oi, _, it = O.mmedit_forward(d["x"], d["x_txt"], 3, 3, d, 2, return_intermediates=True, eta="exact")
    Q, K, V, Kp, Vp = (np.asarray(it[n])[0] for n in ("Q", "K", "V", "Kp_txt", "Vp_txt"))
    dh, eps = 4, d["attn_eps"]
    for i in range(Q.shape[0]):
        for h in range(2):
            cols = range(h * dh, (h + 1) * dh)
            dot = lambda a, b: sum(a[c] * b[c] for c in cols)  # noqa: E731
            ws = [dot(Q[i], K[j]) for j in range(K.shape[0])] + \
                 [math.exp(dot(Q[i], Kp[j]) / math.sqrt(dh)) for j in range(Kp.shape[0])]
            vs = [V[j] for j in range(V.shape[0])] + [Vp[j] for j in range(Vp.shape[0])]
            tot = sum(ws) + eps
            for c in cols:
                want = sum(wj * vj[c] for wj, vj in zip(ws, vs)) / tot
                assert abs(oi[0, i, c] - want) <= 1e-12 * max(1.0, abs(want))


def test_mmedit_exact_eta_without_prompt_tokens_is_edit():
    cfg = small_cfg(n_txt=0)
    d = make_inputs(**cfg)
    oi, op = O.mmedit_forward(d["x"], d["x_txt"], cfg["H"], cfg["W"], d, cfg["heads"], eta="exact")
    assert np.array_equal(oi, O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"]))
    assert op.shape == (cfg["B"], 0, cfg["C"])


# ------------------------------------------ planted mistakes must be caught

def _mutant_layer(monkeypatch, name, fn):
    monkeypatch.setattr(O, name, fn)


MUTANTS = {
    "S_transposed": ("linear_attention", lambda orig: (lambda Q, K, V, heads, eps: _la_transposed(Q, K, V, heads, eps))),
    "conv_taps_flipped": ("conv3x3_same", lambda orig: (lambda X, w, b: orig(X, w[:, ::-1, ::-1, :], b))),
    "dwconv_off_by_one": ("dwconv3x3_s2", lambda orig: (lambda Y, w, b: _dw_shifted(orig, Y, w, b))),
    "gn_unbiased_var": ("group_norm", lambda orig: (lambda U, g, ga, be, eps: _gn_unbiased(U, g, ga, be, eps))),
    "leaky_sign": ("leaky_relu", lambda orig: (lambda x, s: np.where(np.asarray(x) >= 0, x, -s * np.asarray(x)))),
    "dropped_bias": ("linear", lambda orig: (lambda x, w, b: np.asarray(x, float) @ np.asarray(w, float).T)),
    "eta_swapped": ("mix_ratio", lambda orig: (lambda NI, NT: NT / float(NI + NT))),
}


def _la_transposed(Q, K, V, heads, eps):
    Q, K, V = (np.asarray(a, float) for a in (Q, K, V))
    B, N, C = Q.shape
    d = C // heads
    y = np.empty_like(Q)
    for bi in range(B):
        for h in range(heads):
            sl = slice(h * d, (h + 1) * d)
            S = (K[bi, :, sl].T @ V[bi, :, sl]).T
            z = K[bi, :, sl].sum(0)
            y[bi, :, sl] = (Q[bi, :, sl] @ S) / (Q[bi, :, sl] @ z + eps)[:, None]
    return y, None, None


def _dw_shifted(orig, Y, w, b):
    out = orig(Y, w, b)
    Y = np.asarray(Y, float)
    Ypad = np.concatenate([Y[:, 1:], np.zeros_like(Y[:, :1])], axis=1)
    return orig(Ypad, w, b) if out.shape[1] > 1 else out * 1.5


def _gn_unbiased(U, groups, gamma, beta, eps):
    U = np.asarray(U, float)
    B, H, W, Cr = U.shape
    cpg = Cr // groups
    Ug = U.reshape(B, -1, groups, cpg)
    mean = Ug.mean(axis=(1, 3))
    var = ((Ug - mean[:, None, :, None]) ** 2).sum(axis=(1, 3)) / (Ug.shape[1] * cpg - 1)
    mu = np.repeat(mean, cpg, 1)[:, None, None, :]
    vv = np.repeat(var, cpg, 1)[:, None, None, :]
    return gamma * (U - mu) / np.sqrt(vv + eps) + beta


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(monkeypatch, mutant):
    name, make = MUTANTS[mutant]
    orig = getattr(O, name)
    cfg = small_cfg(n_txt=4, H=6, W=6)
    d = make_inputs(**cfg)
    ri, rp = _torch_mm(d, cfg)
    oi, op = O.mmedit_forward(d["x"], d["x_txt"], cfg["H"], cfg["W"], d, cfg["heads"])
    assert rel(oi, ri) < 1e-11 and rel(op, rp) < 1e-11
    monkeypatch.setattr(O, name, make(orig))
    oi, op = O.mmedit_forward(d["x"], d["x_txt"], cfg["H"], cfg["W"], d, cfg["heads"])
    assert max(rel(oi, ri), rel(op, rp)) > 1e-3, mutant


# ------------------------------------------- ablation variants, output Linear

VARIANTS = [(q, k, v) for q in (O.PROC_CF, O.PROC_NONE) for (k, v) in O.KV_PAIRS]


def _torch_variant_layer(d, cfg, qp, kp, vp, proj):
    """The variant layers composed from PyTorch CPU float64 library routines
    (conv2d, group_norm, leaky_relu, linear, relu, depthwise conv2d), with the
    explicit quadratic form for the attention step."""
    B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    t = {k: torch.tensor(np.asarray(v, np.float64)) for k, v in d.items() if isinstance(v, np.ndarray)}
    X = t["x"].reshape(B, H, W, C).permute(0, 3, 1, 2)

    def convfusion_feature(pre, lin_w, lin_b):
        U = F.conv2d(X, t[pre + "cf3_w"].permute(0, 3, 1, 2), t[pre + "cf3_b"], padding=1)
        G = F.group_norm(U, d["gn_groups"], t[pre + "gn_gamma"], t[pre + "gn_beta"], eps=d["gn_eps"])
        R = X + F.conv2d(F.leaky_relu(G, d["leaky_slope"]), t[pre + "cf1_w"][:, :, None, None], t[pre + "cf1_b"])
        return F.relu(F.linear(R.permute(0, 2, 3, 1).reshape(B, H * W, C), lin_w, lin_b))

    Q = convfusion_feature("", t["q_w"], t["q_b"]) if qp == "cf" else F.relu(F.linear(t["x"], t["q_w"], t["q_b"]))
    if kp == "sc":
        Kp = F.linear(t["x"], t["k_w"], t["k_b"]).reshape(B, H, W, C).permute(0, 3, 1, 2)
        Vp = F.linear(t["x"], t["v_w"], t["v_b"]).reshape(B, H, W, C).permute(0, 3, 1, 2)
        K = F.relu(F.conv2d(Kp, t["kdw_w"][:, None], t["kdw_b"], stride=2, padding=1, groups=C))
        V = F.conv2d(Vp, t["vdw_w"][:, None], t["vdw_b"], stride=2, padding=1, groups=C)
        K = K.permute(0, 2, 3, 1).reshape(B, -1, C)
        V = V.permute(0, 2, 3, 1).reshape(B, -1, C)
    else:
        K = convfusion_feature("k", t["k_w"], t["k_b"]) if kp == "cf" else F.relu(F.linear(t["x"], t["k_w"], t["k_b"]))
        V = F.linear(t["x"], t["v_w"], t["v_b"])
    dh = C // heads
    q = Q.reshape(B, -1, heads, dh).transpose(1, 2)
    k = K.reshape(B, -1, heads, dh).transpose(1, 2)
    v = V.reshape(B, -1, heads, dh).transpose(1, 2)
    A = q @ k.transpose(-1, -2)
    y = ((A @ v) / (A.sum(-1, keepdim=True) + d["attn_eps"])).transpose(1, 2).reshape(B, -1, C)
    out = F.linear(y, t["o_w"], t["o_b"]) if proj else y
    return out.numpy(), K.numpy()


@pytest.mark.parametrize("proj", [False, True])
@pytest.mark.parametrize("qkv", VARIANTS, ids=lambda v: "-".join(v))
def test_variant_vs_torch_composition(qkv, proj):
    cfg = small_cfg(H=5, W=6, variant_weights=True)
    d = make_inputs(**cfg)
    out, it = O.edit_variant_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"], *qkv, out_proj=proj,
                                     return_intermediates=True)
    ref, K_t = _torch_variant_layer(d, cfg, *qkv, proj)
    n_kv = O.compressed_count(5, 6) if qkv[1] == "sc" else 30
    assert it["K"].shape == (cfg["B"], n_kv, cfg["C"]) and it["V"].shape == it["K"].shape
    assert rel(it["K"], K_t) < 1e-12
    assert rel(out, ref) < 1e-11


def test_variant_default_is_edit_layer():
    cfg = small_cfg(variant_weights=True)
    d = make_inputs(**cfg)
    y = O.edit_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"])
    assert np.array_equal(O.edit_variant_forward(d["x"], cfg["H"], cfg["W"], d, cfg["heads"]), y)


def test_variant_uncompressed_vs_brute_force():
    """(-, -, -) keys/values: K = ReLU(x Wk^T + bk), V = x Wv^T + bv over all N
    tokens, attention in the explicit O(N^2) loop form."""
    cfg = small_cfg(B=1, H=3, W=2, C=4, c_red=2, gn_groups=1, heads=2, variant_weights=True)
    d = make_inputs(**cfg)
    out = O.edit_variant_forward(d["x"], 3, 2, d, 2, "none", "none", "none")
    x = np.asarray(d["x"][0], float)
    kw, kb, vw, vb, qw, qb = (np.asarray(d[n], float) for n in ("k_w", "k_b", "v_w", "v_b", "q_w", "q_b"))
    lin = lambda w, b: np.array([[b[o] + sum(x[n, i] * w[o, i] for i in range(4)) for o in range(4)]
                                 for n in range(6)])  # noqa: E731
    Q, K, V = np.maximum(lin(qw, qb), 0), np.maximum(lin(kw, kb), 0), lin(vw, vb)
    for h in range(2):
        sl = slice(2 * h, 2 * h + 2)
        ref = _brute_linear_attention(Q[:, sl], K[:, sl], V[:, sl], d["attn_eps"])
        assert rel(out[0, :, sl], ref) < 1e-12


def test_variant_special_cases():
    cfg = small_cfg(variant_weights=True)
    d = make_inputs(**cfg)
    H, W, h = cfg["H"], cfg["W"], cfg["heads"]
    # identity output Linear with zero bias leaves y unchanged
    e = dict(d, o_w=np.eye(cfg["C"]), o_b=np.zeros(cfg["C"]))
    assert np.array_equal(O.edit_variant_forward(d["x"], H, W, e, h, out_proj=True),
                          O.edit_variant_forward(d["x"], H, W, e, h))
    # a zero 1x1 conv makes the ConvFusion query the plain ReLU(Linear) query
    e = dict(d, cf1_w=np.zeros_like(d["cf1_w"]), cf1_b=np.zeros_like(d["cf1_b"]))
    a = O.edit_variant_forward(d["x"], H, W, e, h, "cf", "none", "none")
    b = O.edit_variant_forward(d["x"], H, W, e, h, "none", "none", "none")
    assert rel(a, b) < 1e-13
    # key ConvFusion with the query's weights and Linear gives K == Q
    e = dict(d, kcf3_w=d["cf3_w"], kcf3_b=d["cf3_b"], kgn_gamma=d["gn_gamma"], kgn_beta=d["gn_beta"],
             kcf1_w=d["cf1_w"], kcf1_b=d["cf1_b"], k_w=d["q_w"], k_b=d["q_b"])
    _, it = O.edit_variant_forward(d["x"], H, W, e, h, "cf", "cf", "none", return_intermediates=True)
    assert np.array_equal(it["K"], it["Q"])
    with pytest.raises(ValueError):
        O.edit_variant_forward(d["x"], H, W, d, h, "cf", "sc", "none")


VARIANT_MUTANTS = {
    "convfusion_without_1x1": ("convfusion_residual", ("cf", "cf", "none"),
                               lambda orig: (lambda X, *a: (np.asarray(X, float),) + orig(X, *a)[1:])),
    "relu_dropped": ("relu", ("none", "none", "none"), lambda orig: (lambda x: np.asarray(x, float))),
    "linear_transposed": ("linear", ("none", "none", "none"),
                          lambda orig: (lambda x, w, b: np.asarray(x, float) @ np.asarray(w, float) + b)),
}


@pytest.mark.parametrize("mutant", sorted(VARIANT_MUTANTS))
def test_variant_planted_mistake_is_caught(monkeypatch, mutant):
    name, qkv, make = VARIANT_MUTANTS[mutant]
    cfg = small_cfg(H=4, W=5, variant_weights=True)
    d = make_inputs(**cfg)
    ref = _torch_variant_layer(d, cfg, *qkv, True)[0]
    assert rel(O.edit_variant_forward(d["x"], 4, 5, d, cfg["heads"], *qkv, out_proj=True), ref) < 1e-11
    monkeypatch.setattr(O, name, make(getattr(O, name)))
    assert rel(O.edit_variant_forward(d["x"], 4, 5, d, cfg["heads"], *qkv, out_proj=True), ref) > 1e-3, mutant


# ------------------------------------------------ the DiT block around EDiT

DIT = dict(n_cap=7, hidden=64)


def _torch_dit_block(d, cfg):
    """The block from PyTorch CPU float64 library routines: layer_norm,
    linear, scaled_dot_product_attention, gelu(approximate='tanh'), and the
    EDiT layer's own torch composition for the self-attention."""
    B, H, W, C, heads = cfg["B"], cfg["H"], cfg["W"], cfg["C"], cfg["heads"]
    t = {k: torch.tensor(np.asarray(v, np.float64)) for k, v in d.items() if isinstance(v, np.ndarray)}
    m = t["sst"][None] + t["t6"]
    sh_a, sc_a, g_a, sh_f, sc_f, g_f = (m[:, k][:, None, :] for k in range(6))
    x = t["x"]
    h1 = F.layer_norm(x, (C,), eps=d["ln_eps"]) * (1 + sc_a) + sh_a
    y_att, _, _, _ = _torch_edit_layer(dict(d, x=h1.numpy()), cfg)
    x1 = x + g_a * F.linear(torch.tensor(y_att), t["o_w"], t["o_b"])
    dh = C // heads
    sh = lambda a: a.reshape(B, -1, heads, dh).transpose(1, 2)  # noqa: E731
    q = F.linear(x1, t["cq_w"], t["cq_b"])
    k = F.linear(t["y"], t["ck_w"], t["ck_b"])
    v = F.linear(t["y"], t["cv_w"], t["cv_b"])
    a = F.scaled_dot_product_attention(sh(q), sh(k), sh(v)).transpose(1, 2).reshape(B, -1, C)
    x2 = x1 + F.linear(a, t["co_w"], t["co_b"])
    h2 = F.layer_norm(x2, (C,), eps=d["ln_eps"]) * (1 + sc_f) + sh_f
    f = F.gelu(F.linear(h2, t["fc1_w"], t["fc1_b"]), approximate="tanh")
    return (x2 + g_f * F.linear(f, t["fc2_w"], t["fc2_b"])).numpy()


@pytest.mark.parametrize("cfgkw", [dict(), dict(H=5, W=7, B=1), dict(H=4, W=4, heads=4)])
def test_dit_block_vs_torch_composition(cfgkw):
    cfg = small_cfg(**cfgkw)
    d = make_inputs(**cfg, dit_block=DIT)
    out = O.dit_block_forward(d["x"], d["y"], d["t6"], cfg["H"], cfg["W"], d, cfg["heads"])
    assert rel(out, _torch_dit_block(d, cfg)) < 1e-11


def test_layer_norm_and_gelu_vs_torch():
    x = np.random.default_rng(5).standard_normal((3, 7, 24))
    assert rel(O.layer_norm(x, 1e-6), F.layer_norm(torch.tensor(x), (24,), eps=1e-6).numpy()) < 1e-13
    assert rel(O.gelu_tanh(x), F.gelu(torch.tensor(x), approximate="tanh").numpy()) < 1e-13


def test_dit_block_special_cases():
    """Zero gates and a zero cross-attention output Linear leave x unchanged;
    with zero gates only, the block is x plus the cross-attention alone."""
    cfg = small_cfg()
    d = make_inputs(**cfg, dit_block=DIT)
    H, W, heads = cfg["H"], cfg["W"], cfg["heads"]
    z = dict(d)
    z["t6"] = d["t6"].copy()
    z["t6"][:, 2] = -d["sst"][2]
    z["t6"][:, 5] = -d["sst"][5]
    z["co_w"] = np.zeros_like(d["co_w"])
    z["co_b"] = np.zeros_like(d["co_b"])
    assert np.array_equal(O.dit_block_forward(d["x"], d["y"], z["t6"], H, W, z, heads), np.asarray(d["x"], float))
    z2 = dict(z, co_w=d["co_w"], co_b=d["co_b"])
    q = O.linear(d["x"], d["cq_w"], d["cq_b"])
    k, v = O.linear(d["y"], d["ck_w"], d["ck_b"]), O.linear(d["y"], d["cv_w"], d["cv_b"])
    want = np.asarray(d["x"], float) + O.linear(O.sdpa(q, k, v, heads), d["co_w"], d["co_b"])
    assert rel(O.dit_block_forward(d["x"], d["y"], z2["t6"], H, W, z2, heads), want) < 1e-13
