"""Test infrastructure: the EDiT layer for one row band of an image, in fp64
from the oracle's primitives, as the CPU backend of the sequence-parallel
orchestration (linear_compressed_attention_b200.seqpar).

A band holds rows [row0, row0 + rows) of an H x W image plus one halo row on
each side that has a neighbour. Its record is the band's share of the layer's
two global sums (ConvFusion eq. (Q^EDiT): the GroupNorm statistics of
Conv3x3(X); eq. (y_i): S = sum_j K_j^T V_j and z = sum_j K_j); the finish
step sums every band's record in band order and computes the band's rows of
eq. (y_i). The arithmetic is the oracle's; only the split is new here."""
import numpy as np
import torch

import oracle.edit_oracle as O
from linear_compressed_attention_b200.seqpar import halo


def dwconv_band(Kp, w, b, top, Ho):
    """Stride-2 depthwise conv for the band's compressed rows: output row i
    reads rows 2i - 1 + top .. 2i + 1 + top of Kp (the band's K' rows with
    `top` halo rows above), zero outside Kp and outside the image's columns."""
    R, W, C = Kp.shape
    Wo = (W + 1) // 2
    P = np.zeros((R + 2, W + 2, C))
    P[1:-1, 1:-1] = Kp
    out = np.broadcast_to(np.asarray(b, np.float64), (Ho, Wo, C)).copy()
    for a in range(3):
        for e in range(3):
            out += P[top + a:top + a + 2 * Ho - 1:2, e:e + 2 * Wo - 1:2, :] * np.asarray(w, np.float64)[:, a, e]
    return out


class OracleBand:
    """partials() / finish() of one band, fp64; records are float64 arrays
    carried in uint8 tensors (opaque to the orchestration)."""

    def __init__(self, w, H, W, heads):
        self.w, self.H, self.W, self.heads = w, H, W, heads
        self.keep = {}

    def partials(self, x_ext, row0, rows):
        w, W = self.w, self.W
        X = x_ext.double().numpy()
        top, _ = halo(self.H, row0, rows)
        G = w["gn_groups"]
        U = O.conv3x3_same(X[None], w["cf3_w"], w["cf3_b"])[0][top:top + rows]
        Ug = U.reshape(rows * W, G, -1)
        gn = np.stack([Ug.sum(axis=(0, 2)), (Ug * Ug).sum(axis=(0, 2))], axis=1)       # [G][2]
        Ho = (rows + 1) // 2
        Kp = O.linear(X[:rows + top], w["k_w"], w["k_b"])
        Vp = O.linear(X[:rows + top], w["v_w"], w["v_b"])
        K = O.relu(dwconv_band(Kp, w["kdw_w"], w["kdw_b"], top, Ho)).reshape(-1, Kp.shape[2])
        V = dwconv_band(Vp, w["vdw_w"], w["vdw_b"], top, Ho).reshape(-1, Kp.shape[2])
        d = K.shape[1] // self.heads
        Sz = np.empty((self.heads, d, d + 1))
        for h in range(self.heads):
            sl = slice(h * d, (h + 1) * d)
            Sz[h, :, :d] = K[:, sl].T @ V[:, sl]
            Sz[h, :, d] = K[:, sl].sum(axis=0)
        self.keep[row0] = U
        rec = np.concatenate([gn.ravel(), Sz.ravel()])
        return torch.from_numpy(rec).view(torch.uint8)

    def finish(self, x_ext, records, row0, rows):
        w, W, H = self.w, self.W, self.H
        X = x_ext.double().numpy()
        top, _ = halo(H, row0, rows)
        G = w["gn_groups"]
        recs = records.contiguous().view(torch.float64).numpy()
        tot = np.zeros_like(recs[0])
        for r in range(recs.shape[0]):          # band order
            tot = tot + recs[r]
        gn = tot[:2 * G].reshape(G, 2)
        C = X.shape[2]
        d = C // self.heads
        Sz = tot[2 * G:].reshape(self.heads, d, d + 1)
        U = self.keep[row0]
        cpg = U.shape[2] // G
        count = H * W * cpg
        mean = gn[:, 0] / count
        var = gn[:, 1] / count - mean * mean
        mu, sd = np.repeat(mean, cpg), np.sqrt(np.repeat(var, cpg) + w["gn_eps"])
        Gn = w["gn_gamma"] * (U - mu) / sd + w["gn_beta"]
        R = X[top:top + rows] + O.linear(O.leaky_relu(Gn, w["leaky_slope"]), w["cf1_w"], w["cf1_b"])
        Q = O.relu(O.linear(R, w["q_w"], w["q_b"])).reshape(rows * W, C)
        y = np.empty_like(Q)
        for h in range(self.heads):
            sl = slice(h * d, (h + 1) * d)
            y[:, sl] = (Q[:, sl] @ Sz[h, :, :d]) / (Q[:, sl] @ Sz[h, :, d] + w["attn_eps"])[:, None]
        return torch.from_numpy(y.reshape(rows, W, C))
