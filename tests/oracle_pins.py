"""Independent pins for the fp64 oracle.

Each pin checks the oracle against something other than itself: a closed
form (identity, box sum, shifted gather, affine field, constant input), a
brute-force sum over the whole grid of the bilinear kernel
g(a,b) = max(0, 1-|a-b|) ("用PyTorch实战DCNv1", section 2), PyTorch's own
bilinear sampler (grid_sample, zero padding), finite differences and the
adjoint identity for the gradients. The pins are functions of the oracle
library handle so that the mutation test can rerun them against deliberately
broken builds of the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

F32 = np.float32


# ---------------------------------------------------------------- helpers
def base_grid(Ho, Wo, kh, kw, stride, pad, dil):
    """by[ho, i], bx[wo, j]: regular grid points of the kernel window."""
    by = np.arange(Ho)[:, None] * stride[0] - pad[0] + np.arange(kh)[None, :] * dil[0]
    bx = np.arange(Wo)[:, None] * stride[1] - pad[1] + np.arange(kw)[None, :] * dil[1]
    return by, bx


def positions32(off, Ho, Wo, kh, kw, stride, pad, dil, s):
    """fp32 sampling positions py, px [B,Ho,Wo,G,K]; s must make s*d exact."""
    by, bx = base_grid(Ho, Wo, kh, kw, stride, pad, dil)
    K = kh * kw
    byk = np.repeat(by, kw, axis=1)  # [Ho, K], k = i*kw + j
    bxk = np.tile(bx, (1, kh))       # [Wo, K]
    d = off.astype(F32)
    py = F32(s) * d[..., 1] + byk[None, :, None, None, :].astype(F32)
    px = F32(s) * d[..., 0] + bxk[None, None, :, None, :].astype(F32)
    return py.astype(np.float64), px.astype(np.float64)


def brute_force_forward(x, off, mask, G, kh, kw, stride, pad, dil, s, softmax):
    """out = sum_k m_k sum_{every grid q} g(qx,px) g(qy,py) x(q), by full sums."""
    B, H, W, GC = x.shape
    C = GC // G
    Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
    py, px = positions32(off, Ho, Wo, kh, kw, stride, pad, dil, s)
    m = mask.astype(np.float64)
    if softmax:
        e = np.exp(m - m.max(-1, keepdims=True))
        m = e / e.sum(-1, keepdims=True)
    qy = np.arange(H, dtype=np.float64)
    qx = np.arange(W, dtype=np.float64)
    gy = np.maximum(0.0, 1.0 - np.abs(qy - py[..., None]))  # [B,Ho,Wo,G,K,H]
    gx = np.maximum(0.0, 1.0 - np.abs(qx - px[..., None]))  # [B,Ho,Wo,G,K,W]
    xg = x.reshape(B, H, W, G, C).astype(np.float64)
    # sum over k, qy, qx: m * gy * gx * x[b, qy, qx, g, c]
    out = np.einsum("bhwgk,bhwgky,bhwgkx,byxgc->bhwgc", m, gy, gx, xg, optimize=True)
    return out.reshape(B, Ho, Wo, GC)


def grid_sample_forward(x, off, mask, G, kh, kw, stride, pad, dil, s, softmax):
    """The same sum with torch's bilinear grid_sample (zeros padding,
    align_corners=False: pixel centre i sits at normalised (2i+1)/n - 1)."""
    B, H, W, GC = x.shape
    C = GC // G
    Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
    py, px = positions32(off, Ho, Wo, kh, kw, stride, pad, dil, s)
    m = torch.from_numpy(mask.astype(np.float64))
    if softmax:
        m = torch.softmax(m, dim=-1)
    xt = torch.from_numpy(x.astype(np.float64)).reshape(B, H, W, G, C)
    out = torch.zeros(B, Ho, Wo, G, C, dtype=torch.float64)
    for g in range(G):
        xin = xt[:, :, :, g, :].permute(0, 3, 1, 2)  # [B,C,H,W]
        for k in range(kh * kw):
            gx = (2.0 * px[:, :, :, g, k] + 1.0) / W - 1.0
            gy = (2.0 * py[:, :, :, g, k] + 1.0) / H - 1.0
            grid = torch.from_numpy(np.stack([gx, gy], -1))
            v = torch.nn.functional.grid_sample(xin, grid, mode="bilinear", padding_mode="zeros",
                                                align_corners=False)  # [B,C,Ho,Wo]
            out[:, :, :, g, :] += m[:, :, :, g, k, None] * v.permute(0, 2, 3, 1)
    return out.reshape(B, Ho, Wo, GC).numpy()


def rand_case(seed, B, H, W, G, C, kh, kw, stride, pad, dil, off_std, quant=None):
    rng = np.random.default_rng(seed)
    Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
    x = rng.standard_normal((B, H, W, G * C))
    off = rng.standard_normal((B, Ho, Wo, G, kh * kw, 2)) * off_std
    if quant is not None:
        # odd multiples of quant/2: fp32-exact positions that never sit on a grid line
        off = np.round(off / quant) * quant + quant / 2
    off = off.astype(F32).astype(np.float64)
    mask = rng.standard_normal((B, Ho, Wo, G, kh * kw))
    return x, off, mask


GEOMS = [
    # (H, W, kh, kw, stride, pad, dil)
    (7, 9, 3, 3, (1, 1), (1, 1), (1, 1)),
    (8, 6, 3, 3, (2, 2), (1, 1), (1, 1)),
    (9, 8, 3, 3, (1, 1), (2, 2), (2, 2)),
    (6, 11, 3, 5, (1, 2), (1, 2), (1, 1)),
    (5, 5, 1, 1, (1, 1), (0, 0), (1, 1)),
]


# ---------------------------------------------------------------- core pins
def pin_identity(lib):
    """Zero offsets and a one-hot centre mask reproduce x exactly."""
    rng = np.random.default_rng(11)
    for pad, dil in (((1, 1), (1, 1)), ((2, 2), (2, 2))):
        x = rng.standard_normal((2, 6, 7, 3 * 4))
        Ho, Wo = oracle.out_hw(6, 7, 3, 3, 1, 1, *pad, *dil)
        off = np.zeros((2, Ho, Wo, 3, 9, 2))
        mask = np.zeros((2, Ho, Wo, 3, 9))
        mask[..., 4] = 1.0
        out = oracle.dcn_forward(x, off, mask, G=3, pad=pad, dil=dil, lib=lib)
        assert np.array_equal(out, x), "identity"


def pin_box_sum(lib):
    """Zero offsets, unit masks: zero-padded window sum (integral image)."""
    rng = np.random.default_rng(12)
    for (H, W, kh, kw, stride, pad, dil) in GEOMS:
        G, C = 2, 3
        x = rng.standard_normal((1, H, W, G * C))
        Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
        off = np.zeros((1, Ho, Wo, G, kh * kw, 2))
        mask = np.ones((1, Ho, Wo, G, kh * kw))
        out = oracle.dcn_forward(x, off, mask, G=G, kh=kh, kw=kw, stride=stride, pad=pad, dil=dil, lib=lib)
        xp = np.zeros((H + 2 * pad[0] + dil[0] * kh, W + 2 * pad[1] + dil[1] * kw, G * C))
        xp[pad[0]:pad[0] + H, pad[1]:pad[1] + W] = x[0]
        ref = np.zeros((Ho, Wo, G * C))
        for i in range(kh):
            for j in range(kw):
                ys = i * dil[0]
                xs = j * dil[1]
                ref += xp[ys:ys + (Ho - 1) * stride[0] + 1:stride[0], xs:xs + (Wo - 1) * stride[1] + 1:stride[1]]
        if (kh, kw, stride, dil) == (3, 3, (1, 1), (1, 1)):
            # second, independent route: summed-area table of the padded map
            S = np.zeros((xp.shape[0] + 1, xp.shape[1] + 1, G * C))
            S[1:, 1:] = xp.cumsum(0).cumsum(1)
            box = S[3:3 + Ho, 3:3 + Wo] - S[:Ho, 3:3 + Wo] - S[3:3 + Ho, :Wo] + S[:Ho, :Wo]
            assert np.allclose(box, ref, atol=1e-12)
        assert np.allclose(out[0], ref, rtol=0, atol=1e-12), "box sum"


def pin_shifted_gather(lib):
    """Integer offsets (dx != dy) give exact shifted gathers, zero outside."""
    rng = np.random.default_rng(13)
    for (H, W, kh, kw, stride, pad, dil) in GEOMS:
        G, C, B = 2, 3, 2
        K = kh * kw
        x = rng.standard_normal((B, H, W, G * C))
        Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
        off = rng.integers(-3, 4, size=(B, Ho, Wo, G, K, 2)).astype(np.float64)
        off[..., 0] += 1.0  # keep dx and dy statistically different
        mask = rng.standard_normal((B, Ho, Wo, G, K))
        out = oracle.dcn_forward(x, off, mask, G=G, kh=kh, kw=kw, stride=stride, pad=pad, dil=dil, lib=lib)
        by, bx = base_grid(Ho, Wo, kh, kw, stride, pad, dil)
        ref = np.zeros((B, Ho, Wo, G, C))
        xg = x.reshape(B, H, W, G, C)
        bb, hh, ww, gg, ii, jj = np.meshgrid(np.arange(B), np.arange(Ho), np.arange(Wo), np.arange(G),
                                             np.arange(kh), np.arange(kw), indexing="ij")
        kk = ii * kw + jj
        yy = by[hh, ii] + off[bb, hh, ww, gg, kk, 1].astype(int)
        xx = bx[ww, jj] + off[bb, hh, ww, gg, kk, 0].astype(int)
        ok = (yy >= 0) & (yy < H) & (xx >= 0) & (xx < W)
        vals = np.where(ok[..., None], xg[bb, np.clip(yy, 0, H - 1), np.clip(xx, 0, W - 1), gg], 0.0)
        ref = (mask[bb, hh, ww, gg, kk][..., None] * vals).sum(axis=(4, 5))
        assert np.allclose(out.reshape(B, Ho, Wo, G, C), ref, rtol=0, atol=1e-12), "shifted gather"


def pin_affine_field(lib):
    """Bilinear interpolation is exact on x = a + b*y + c*x inside the map."""
    rng = np.random.default_rng(14)
    H, W, G, C = 12, 10, 2, 3
    a, bcoef, ccoef = rng.standard_normal((3, G * C))
    yy, xx = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    x = (a + bcoef * yy[..., None] + ccoef * xx[..., None])[None]
    Ho, Wo = H, W
    off = rng.uniform(-0.9, 0.9, size=(1, Ho, Wo, G, 9, 2))
    off = np.round(off * 1024) / 1024  # fp32-exact positions
    mask = rng.standard_normal((1, Ho, Wo, G, 9))
    out = oracle.dcn_forward(x, off, mask, G=G, lib=lib)
    py, px = positions32(off, Ho, Wo, 3, 3, (1, 1), (1, 1), (1, 1), 1.0)
    inside = ((py >= 0) & (py <= H - 1) & (px >= 0) & (px <= W - 1)).all(axis=(3, 4))
    field = a.reshape(G, C)[None, None, None, :, None, :] + \
        bcoef.reshape(G, C)[None, None, None, :, None, :] * py[..., None] + \
        ccoef.reshape(G, C)[None, None, None, :, None, :] * px[..., None]
    ref = (mask[..., None] * field).sum(axis=4).reshape(1, Ho, Wo, G * C)
    assert inside.sum() > 20
    assert np.allclose(out[inside], ref[inside], rtol=0, atol=1e-11), "affine field"


def pin_softmax_constant(lib):
    """Softmax modulation of a constant map returns the constant inside it."""
    rng = np.random.default_rng(15)
    H, W, G, C = 10, 9, 3, 2
    kappa = 1.75
    x = np.full((1, H, W, G * C), kappa)
    off = rng.uniform(-0.45, 0.45, size=(1, H, W, G, 9, 2))
    mask = rng.standard_normal((1, H, W, G, 9)) * 3.0
    out = oracle.dcn_forward(x, off, mask, G=G, softmax=True, lib=lib)
    py, px = positions32(off, H, W, 3, 3, (1, 1), (1, 1), (1, 1), 1.0)
    inside = ((py >= 0) & (py <= H - 1) & (px >= 0) & (px <= W - 1)).all(axis=(3, 4))
    assert inside.sum() > 10
    assert np.allclose(out[inside], kappa, rtol=0, atol=1e-13), "softmax constant"
    # border pixels, whose taps leave the map, lose part of the unit weight
    assert (out[~inside] <= kappa + 1e-13).all() and out[~inside].mean() < 0.95 * kappa


def pin_softmax_vs_raw(lib):
    """Softmax mode equals raw mode fed with scipy's softmax over K."""
    from scipy.special import softmax

    x, off, mask = rand_case(16, 2, 7, 8, 3, 4, 3, 3, (1, 1), (1, 1), (1, 1), 2.0)
    a = oracle.dcn_forward(x, off, mask, G=3, softmax=True, lib=lib)
    b = oracle.dcn_forward(x, off, softmax(mask, axis=-1), G=3, softmax=False, lib=lib)
    assert np.allclose(a, b, rtol=0, atol=1e-13), "softmax vs raw"


def pin_brute_force(lib):
    """The four-corner sum equals the sum over every grid point (random
    fractional offsets, out-of-range taps included), and matches grid_sample."""
    for n, (H, W, kh, kw, stride, pad, dil) in enumerate(GEOMS):
        for s, softmax in ((1.0, False), (0.5, True)):
            x, off, mask = rand_case(20 + n, 2, H, W, 2, 3, kh, kw, stride, pad, dil, 2.5)
            out = oracle.dcn_forward(x, off, mask, G=2, kh=kh, kw=kw, stride=stride, pad=pad, dil=dil,
                                     offset_scale=s, softmax=softmax, lib=lib)
            ref = brute_force_forward(x, off, mask, 2, kh, kw, stride, pad, dil, s, softmax)
            assert np.allclose(out, ref, rtol=0, atol=1e-12), "brute force"
            gs = grid_sample_forward(x, off, mask, 2, kh, kw, stride, pad, dil, s, softmax)
            assert np.allclose(out, gs, rtol=0, atol=1e-10), "grid_sample"


# ---------------------------------------------------------------- backward pins
def _loss(lib, x, off, mask, go, G, geom, s, softmax):
    H, W, kh, kw, stride, pad, dil = geom
    out = oracle.dcn_forward(x, off, mask, G=G, kh=kh, kw=kw, stride=stride, pad=pad, dil=dil,
                             offset_scale=s, softmax=softmax, lib=lib)
    return float((go * out).sum())


def pin_backward_fd(lib):
    """Finite differences of <grad_out, out> for the offset and the mask, and
    the adjoint identity <grad_out, F(x')> = <grad_x, x'> (out is linear in x)."""
    for softmax in (False, True):
        geom = (6, 7, 3, 3, (1, 1), (1, 1), (1, 1))
        H, W, kh, kw, stride, pad, dil = geom
        G, C = 2, 4
        # offsets on a 2^-12 lattice keep base + d + h exact in fp32
        x, off, mask = rand_case(31, 1, H, W, G, C, kh, kw, stride, pad, dil, 1.5, quant=2.0 ** -12)
        rng = np.random.default_rng(32)
        Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
        go = rng.standard_normal((1, Ho, Wo, G * C))
        s = 0.5
        gr = oracle.dcn_backward(x, off, mask, go, G=G, offset_scale=s, softmax=softmax, lib=lib)
        py, px = positions32(off, Ho, Wo, kh, kw, stride, pad, dil, s)
        h = 2.0 ** -10
        checked = 0
        for idx in map(tuple, rng.integers([0, 0, 0, 0, 0], [1, Ho, Wo, G, 9], size=(40, 5))):
            for comp, pos in ((0, px[idx]), (1, py[idx])):
                frac = pos - np.floor(pos)
                if frac < 4 * h * s or frac > 1 - 4 * h * s:
                    continue  # the derivative jumps on grid lines
                op, om = off.copy(), off.copy()
                op[idx + (comp,)] += h
                om[idx + (comp,)] -= h
                fd = (_loss(lib, x, op, mask, go, G, geom, s, softmax)
                      - _loss(lib, x, om, mask, go, G, geom, s, softmax)) / (2 * h)
                assert abs(fd - gr["grad_offset"][idx + (comp,)]) < 1e-9 * (1 + abs(fd)), "fd offset"
                checked += 1
            hm = 1e-6
            mp, mm = mask.copy(), mask.copy()
            mp[idx] += hm
            mm[idx] -= hm
            fd = (_loss(lib, x, off, mp, go, G, geom, s, softmax)
                  - _loss(lib, x, off, mm, go, G, geom, s, softmax)) / (2 * hm)
            assert abs(fd - gr["grad_mask"][idx]) < 1e-7 * (1 + abs(fd)), "fd mask"
        assert checked > 40
        # adjoint identity for grad_x, and each unit vector for a handful of entries
        xp = rng.standard_normal(x.shape)
        lhs = _loss(lib, xp, off, mask, go, G, geom, s, softmax)
        rhs = float((gr["grad_x"] * xp).sum())
        assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs)), "adjoint grad_x"
        for flat in rng.integers(0, x.size, size=8):
            e = np.zeros(x.size)
            e[flat] = 1.0
            v = _loss(lib, e.reshape(x.shape), off, mask, go, G, geom, s, softmax)
            assert abs(v - gr["grad_x"].reshape(-1)[flat]) < 1e-12, "unit grad_x"


def pin_backward_autograd(lib):
    """The offset and mask gradients agree with torch.autograd through the
    grid_sample formulation (a third, library route)."""
    geom = (5, 6, 3, 3, (1, 1), (1, 1), (1, 1))
    H, W, kh, kw, stride, pad, dil = geom
    G, C = 2, 3
    x, off, mask = rand_case(41, 1, H, W, G, C, kh, kw, stride, pad, dil, 1.2, quant=2.0 ** -12)
    rng = np.random.default_rng(42)
    go = rng.standard_normal((1, H, W, G * C))
    gr = oracle.dcn_backward(x, off, mask, go, G=G, lib=lib)
    by, bx = base_grid(H, W, kh, kw, stride, pad, dil)
    byk = torch.from_numpy(np.repeat(by, kw, axis=1).astype(np.float64))
    bxk = torch.from_numpy(np.tile(bx, (1, kh)).astype(np.float64))
    offt = torch.from_numpy(off).requires_grad_(True)
    mt = torch.from_numpy(mask).requires_grad_(True)
    xt = torch.from_numpy(x).requires_grad_(True)
    out = torch.zeros(1, H, W, G, C, dtype=torch.float64)
    for g in range(G):
        xin = xt.reshape(1, H, W, G, C)[:, :, :, g, :].permute(0, 3, 1, 2)
        for k in range(9):
            px = bxk[None, None, :, k] + offt[:, :, :, g, k, 0]
            py = byk[None, :, None, k] + offt[:, :, :, g, k, 1]
            grid = torch.stack([(2 * px + 1) / W - 1, (2 * py + 1) / H - 1], -1)
            v = torch.nn.functional.grid_sample(xin, grid, mode="bilinear", padding_mode="zeros",
                                                align_corners=False)
            out[:, :, :, g, :] = out[:, :, :, g, :] + mt[:, :, :, g, k, None] * v.permute(0, 2, 3, 1)
    (out.reshape(1, H, W, G * C) * torch.from_numpy(go)).sum().backward()
    assert np.allclose(gr["grad_offset"], offt.grad.numpy(), rtol=0, atol=1e-9), "autograd offset"
    assert np.allclose(gr["grad_mask"], mt.grad.numpy(), rtol=0, atol=1e-10), "autograd mask"
    assert np.allclose(gr["grad_x"], xt.grad.numpy(), rtol=0, atol=1e-10), "autograd x"


# ---------------------------------------------------------------- aggregation pins
def agg_case(seed, B=1, cams=2, scales=((5, 7), (3, 4)), A=3, P=2, G=2, C=3, lo=-0.1, hi=1.1, quant=None):
    rng = np.random.default_rng(seed)
    hw = sum(h * w for h, w in scales)
    rows = cams * hw
    feat = rng.standard_normal((B, rows, G * C))
    shape = np.array([[list(s) for s in scales]] * cams, dtype=np.int32)
    start = np.array([[c * hw + sum(h * w for h, w in scales[:s]) for s in range(len(scales))]
                      for c in range(cams)], dtype=np.int32)
    loc = rng.uniform(lo, hi, size=(B, A, P, cams, 2))
    if quant is not None:
        loc = np.round(loc / quant) * quant
    loc = loc.astype(F32)
    w = rng.standard_normal((B, A, P, cams, len(scales), G))
    return feat, shape, start, loc, w


def agg_pos32(u, n):
    """fp32 position u*n - 0.5 with one rounding (the product and the shift
    are exact in fp64 for a 24-bit u and a small integer n)."""
    return (u.astype(np.float64) * n - 0.5).astype(F32).astype(np.float64)


def agg_brute_force(feat, shape, start, loc, w):
    """Explicit per-camera, per-scale maps and a sum over every grid point."""
    B, rows, GC = feat.shape
    _, A, P, cams, S, G = w.shape
    C = GC // G
    out = np.zeros((B, A, G, C))
    for b in range(B):
        for cam in range(cams):
            for s in range(S):
                Hs, Ws = int(shape[cam, s, 0]), int(shape[cam, s, 1])
                r0 = int(start[cam, s])
                fmap = feat[b, r0:r0 + Hs * Ws].reshape(Hs, Ws, G, C)
                px = agg_pos32(loc[b, :, :, cam, 0], Ws)  # [A,P]
                py = agg_pos32(loc[b, :, :, cam, 1], Hs)
                gy = np.maximum(0, 1 - np.abs(np.arange(Hs) - py[..., None]))
                gx = np.maximum(0, 1 - np.abs(np.arange(Ws) - px[..., None]))
                out[b] += np.einsum("apg,apy,apx,yxgc->agc", w[b, :, :, cam, s, :], gy, gx, fmap)
    return out.reshape(B, A, GC)


def pin_agg_brute_force(lib):
    for seed in range(3):
        feat, shape, start, loc, w = agg_case(50 + seed)
        out = oracle.agg_forward(feat, shape, start, loc, w, lib=lib)
        ref = agg_brute_force(feat, shape, start, loc, w)
        assert np.allclose(out, ref, rtol=0, atol=1e-12), "agg brute force"


def pin_agg_grid_sample(lib):
    feat, shape, start, loc, w = agg_case(60, cams=3, scales=((6, 9), (4, 5), (2, 3)), A=4, P=3)
    out = oracle.agg_forward(feat, shape, start, loc, w, lib=lib)
    B, rows, GC = feat.shape
    _, A, P, cams, S, G = w.shape
    C = GC // G
    ref = torch.zeros(B, A, G, C, dtype=torch.float64)
    for cam in range(cams):
        for s in range(S):
            Hs, Ws = int(shape[cam, s, 0]), int(shape[cam, s, 1])
            r0 = int(start[cam, s])
            fm = torch.from_numpy(feat[:, r0:r0 + Hs * Ws]).reshape(B, Hs, Ws, G, C)
            px = torch.from_numpy(agg_pos32(loc[:, :, :, cam, 0], Ws))
            py = torch.from_numpy(agg_pos32(loc[:, :, :, cam, 1], Hs))
            grid = torch.stack([(2 * px + 1) / Ws - 1, (2 * py + 1) / Hs - 1], -1)  # [B,A,P,2]
            for g in range(G):
                v = torch.nn.functional.grid_sample(fm[..., g, :].permute(0, 3, 1, 2), grid,
                                                    mode="bilinear", padding_mode="zeros",
                                                    align_corners=False)  # [B,C,A,P]
                ref[:, :, g, :] += (torch.from_numpy(w[:, :, :, cam, s, g])[:, None] * v).sum(-1).permute(0, 2, 1)
    assert np.allclose(out, ref.reshape(B, A, GC).numpy(), rtol=0, atol=1e-10), "agg grid_sample"


def pin_agg_backward(lib):
    """Finite differences (locations on a 2^-14 lattice keep loc*size exact),
    linearity in the weights, and the adjoint identity for grad_feat."""
    feat, shape, start, loc, w = agg_case(70, quant=2.0 ** -14)
    rng = np.random.default_rng(71)
    B, rows, GC = feat.shape
    _, A, P, cams, S, G = w.shape
    go = rng.standard_normal((B, A, GC))
    gr = oracle.agg_backward(feat, shape, start, loc, w, go, lib=lib)

    def loss(f, l, ww):
        return float((go * oracle.agg_forward(f, shape, start, l, ww, lib=lib)).sum())

    h = 2.0 ** -12
    checked = 0
    for idx in map(tuple, rng.integers([0, 0, 0, 0, 0], [B, A, P, cams, 2], size=(30, 5))):
        lp, lm = loc.copy(), loc.copy()
        lp[idx] += F32(h)
        lm[idx] -= F32(h)
        # skip when any scale's position crosses a grid line
        cam, comp = idx[3], idx[4]
        crosses = False
        for s in range(S):
            n = shape[cam, s, 1 - comp]
            a_ = float(lm[idx]) * n - 0.5
            b_ = float(lp[idx]) * n - 0.5
            if np.floor(a_) != np.floor(b_) or a_ == np.floor(a_):
                crosses = True
        if crosses:
            continue
        fd = (loss(feat, lp, w) - loss(feat, lm, w)) / (2 * h)
        assert abs(fd - gr["grad_loc"][idx]) < 1e-9 * (1 + abs(fd)), "agg fd loc"
        checked += 1
    assert checked > 10
    for idx in map(tuple, rng.integers([0] * 6, [B, A, P, cams, S, G], size=(12, 6))):
        wp = w.copy()
        wp[idx] += 1.0
        assert abs(loss(feat, loc, wp) - loss(feat, loc, w) - gr["grad_weights"][idx]) < 1e-10, "agg w"
    fp = rng.standard_normal(feat.shape)
    lhs = loss(fp, loc, w)
    rhs = float((gr["grad_feat"] * fp).sum())
    assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs)), "agg adjoint"


def pin_agg_grad_feat_budget(lib):
    """The aggregation's grad_feat budget by brute force over every (anchor,
    point, camera, scale, group, corner), positions formed in fp32; and, for
    non-negative weights and grad_out, the absolute sum is grad_feat itself."""
    for B in (1, 2):
        feat, shape, start, loc, w = agg_case(420 + B, B=B, quant=2.0 ** -12)
        rng = np.random.default_rng(430 + B)
        _, rows, GC = feat.shape
        _, A, P, cams, S, G = w.shape
        C = GC // G
        go = rng.standard_normal((B, A, GC))
        bud = oracle.agg_grad_feat_budget(feat, shape, start, loc, w, go, lib=lib)
        absum = np.zeros((B, rows, GC))
        n = np.zeros((B, rows, G))
        for b in range(B):
            for a in range(A):
                for p in range(P):
                    for cam in range(cams):
                        for s in range(S):
                            Hs, Ws = shape[cam, s]
                            px = agg_pos32(loc[b, a, p, cam, 0:1], Ws)[0]
                            py = agg_pos32(loc[b, a, p, cam, 1:2], Hs)[0]
                            y0, x0 = int(np.floor(py)), int(np.floor(px))
                            for qy in (y0, y0 + 1):
                                for qx in (x0, x0 + 1):
                                    if not (0 <= qy < Hs and 0 <= qx < Ws):
                                        continue
                                    wgt = max(0.0, 1 - abs(qx - px)) * max(0.0, 1 - abs(qy - py))
                                    if wgt == 0.0:
                                        continue
                                    row = start[cam, s] + qy * Ws + qx
                                    for g in range(G):
                                        sl = slice(g * C, (g + 1) * C)
                                        absum[b, row, sl] += np.abs(w[b, a, p, cam, s, g] * wgt * go[b, a, sl])
                                        n[b, row, g] += 1
        assert np.allclose(bud["abs_sum"], absum, rtol=1e-12, atol=1e-14), "agg abs_sum"
        assert np.array_equal(bud["terms"], n), "agg terms"
    feat, shape, start, loc, w = agg_case(440, quant=2.0 ** -12)
    go = np.abs(np.random.default_rng(441).standard_normal((1, w.shape[1], feat.shape[2])))
    w = np.abs(w)
    gr = oracle.agg_backward(feat, shape, start, loc, w, go, lib=lib)
    bud = oracle.agg_grad_feat_budget(feat, shape, start, loc, w, go, lib=lib)
    assert np.allclose(bud["abs_sum"], gr["grad_feat"], rtol=1e-12, atol=1e-14), "agg abs_sum vs grad_feat"


CORE_PINS = [pin_identity, pin_box_sum, pin_shifted_gather, pin_affine_field, pin_softmax_constant,
             pin_softmax_vs_raw, pin_brute_force]
def pin_backward_right_derivative_at_minus_one(lib):
    """At a sampling position exactly on p = -1 the value is zero, and the
    offset gradient is the derivative from the right (the floor() support
    convention): it equals the forward difference (L(p + h) - L(p)) / h, which
    is exact because the interpolation is linear inside the cell [-1, 0)."""
    rng = np.random.default_rng(301)
    B, H, W, G, C = 1, 4, 5, 1, 3
    x = rng.standard_normal((B, H, W, G * C))
    go = rng.standard_normal((B, H, W, G * C))
    mask = np.zeros((B, H, W, G, 9))
    off = np.zeros((B, H, W, G, 9, 2))
    # output (0, 2), point (0, 1): base (-1, 2) with pad 1; output (2, 0), point (1, 0): base (2, -1)
    mask[0, 0, 2, 0, 1] = 0.7
    mask[0, 2, 0, 0, 3] = -1.3
    geom = (H, W, 3, 3, (1, 1), (1, 1), (1, 1))
    g = oracle.dcn_backward(x, off, mask, go, G=G, lib=lib)
    h = 2.0 ** -10
    L0 = _loss(lib, x, off, mask, go, G, geom, 1.0, False)
    for (ho, wo, k, axis) in ((0, 2, 1, 1), (2, 0, 3, 0)):
        o2 = off.copy()
        o2[0, ho, wo, 0, k, axis] = h
        fd = (_loss(lib, x, o2, mask, go, G, geom, 1.0, False) - L0) / h
        an = g["grad_offset"][0, ho, wo, 0, k, axis]
        assert abs(an) > 1e-3, "right derivative at p = -1 is not zero for this input"
        assert abs(an - fd) <= 1e-9 * (1 + abs(fd)), f"right derivative at p = -1: {an} vs {fd}"


def pin_grad_x_budget(lib):
    """The error budget of grad_x: per element, the number of contributions and
    the sum of their absolute values, by brute force over every (item, point,
    corner) with positions formed in fp32; and, for non-negative modulation and
    grad_out (no cancellation), the absolute sum is the oracle's grad_x itself."""
    B, G, C = 2, 2, 3
    for softmax in (False, True):
        for geom in GEOMS[:4]:
            H, W, kh, kw, stride, pad, dil = geom
            x, off, mask = rand_case(411, B, H, W, G, C, kh, kw, stride, pad, dil, 1.5, quant=2.0 ** -10)
            Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
            rng = np.random.default_rng(412)
            go = rng.standard_normal((B, Ho, Wo, G * C))
            s = 0.75
            bud = oracle.dcn_grad_x_budget(off, mask, go, x_shape=x.shape, G=G, kh=kh, kw=kw, stride=stride,
                                           pad=pad, dil=dil, offset_scale=s, softmax=softmax, lib=lib)
            py, px = positions32(off, Ho, Wo, kh, kw, stride, pad, dil, s)
            K = kh * kw
            if softmax:
                e = np.exp(mask - mask.max(axis=-1, keepdims=True))
                m = e / e.sum(axis=-1, keepdims=True)
            else:
                m = mask
            A = np.zeros((B, H, W, G * C))
            n = np.zeros((B, H, W, G))
            for b in range(B):
                for ho in range(Ho):
                    for wo in range(Wo):
                        for g in range(G):
                            for k in range(K):
                                yy, xx = py[b, ho, wo, g, k], px[b, ho, wo, g, k]
                                y0, x0 = int(np.floor(yy)), int(np.floor(xx))
                                for qy in (y0, y0 + 1):
                                    for qx in (x0, x0 + 1):
                                        if not (0 <= qy < H and 0 <= qx < W):
                                            continue
                                        wgt = max(0.0, 1 - abs(qx - xx)) * max(0.0, 1 - abs(qy - yy))
                                        if wgt == 0.0:
                                            continue
                                        gsl = slice(g * C, (g + 1) * C)
                                        A[b, qy, qx, gsl] += np.abs(m[b, ho, wo, g, k] * wgt * go[b, ho, wo, gsl])
                                        n[b, qy, qx, g] += 1
            assert np.allclose(bud["abs_sum"], A, rtol=1e-12, atol=1e-14), "grad_x abs_sum"
            assert np.array_equal(bud["terms"], n), "grad_x terms"
    # no cancellation: the absolute sum equals grad_x
    H, W, kh, kw, stride, pad, dil = GEOMS[0]
    x, off, mask = rand_case(413, 1, H, W, G, C, kh, kw, stride, pad, dil, 1.5, quant=2.0 ** -10)
    Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
    go = np.abs(np.random.default_rng(414).standard_normal((1, Ho, Wo, G * C)))
    mask = np.abs(mask)
    gr = oracle.dcn_backward(x, off, mask, go, G=G, lib=lib)
    bud = oracle.dcn_grad_x_budget(off, mask, go, x_shape=x.shape, G=G, lib=lib)
    assert np.allclose(bud["abs_sum"], gr["grad_x"], rtol=1e-12, atol=1e-14), "abs_sum vs grad_x"


BACKWARD_PINS = [pin_backward_fd, pin_backward_autograd, pin_backward_right_derivative_at_minus_one,
                 pin_grad_x_budget]
AGG_PINS = [pin_agg_brute_force, pin_agg_grid_sample, pin_agg_backward, pin_agg_grad_feat_budget]
ALL_PINS = CORE_PINS + BACKWARD_PINS + AGG_PINS


# ---------------------------------------------------------------- deformable RoI pooling pins
def roi_case(seed, B=2, H=13, W=17, C=3, N=6, P=(3, 4), scale=0.5, margin=2.0, off_std=0.5, quant=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, W, C))
    rois = []
    for n in range(N):
        b = n % B
        w_img, h_img = W / scale, H / scale
        x1 = rng.uniform(margin / scale, w_img / 2)
        y1 = rng.uniform(margin / scale, h_img / 2)
        x2 = rng.uniform(x1 + 1.0, w_img - margin / scale)
        y2 = rng.uniform(y1 + 1.0, h_img - margin / scale)
        rois.append([b, x1, y1, x2, y2])
    rois = np.array(rois, dtype=np.float32)
    off = (rng.standard_normal((N, P[0], P[1], 2)) * off_std).astype(np.float32)
    if quant is not None:
        off = (np.round(off / quant) * quant).astype(np.float32)
    return x, rois, off


def roi_positions32(rois, off, P, S, scale, gamma):
    """fp32 sample positions py, px [N, PH, PW, S, S] in the oracle's operation order."""
    f = np.float32
    r = rois.astype(f)
    x1, y1, x2, y2 = r[:, 1] * f(scale), r[:, 2] * f(scale), r[:, 3] * f(scale), r[:, 4] * f(scale)
    rw = np.maximum(x2 - x1, f(1)).astype(f)
    rh = np.maximum(y2 - y1, f(1)).astype(f)
    bw, bh = (rw / f(P[1])).astype(f), (rh / f(P[0])).astype(f)
    sw, sh = (bw / f(S)).astype(f), (bh / f(S)).astype(f)
    i = np.arange(P[0], dtype=f)[None, :, None, None, None]
    j = np.arange(P[1], dtype=f)[None, None, :, None, None]
    sy = (np.arange(S, dtype=f) + f(0.5))[None, None, None, :, None]
    sx = (np.arange(S, dtype=f) + f(0.5))[None, None, None, None, :]
    dx = ((f(gamma) * off[..., 0]).astype(f) * rw[:, None, None]).astype(f)[..., None, None]
    dy = ((f(gamma) * off[..., 1]).astype(f) * rh[:, None, None]).astype(f)[..., None, None]
    by0 = (y1[:, None, None, None, None] + (i * bh[:, None, None, None, None]).astype(f)).astype(f)
    bx0 = (x1[:, None, None, None, None] + (j * bw[:, None, None, None, None]).astype(f)).astype(f)
    py = ((by0 + (sy * sh[:, None, None, None, None]).astype(f)).astype(f) + dy).astype(f)
    px = ((bx0 + (sx * sw[:, None, None, None, None]).astype(f)).astype(f) + dx).astype(f)
    return py.astype(np.float64), px.astype(np.float64)


def pin_roi_brute_force(lib):
    """Average over S x S samples of the sum over every grid point of G(q,p) x(q)."""
    for seed, (P, S, scale, gamma) in enumerate((((3, 4), 2, 0.5, 0.1), ((2, 2), 3, 1.0, 0.3),
                                                 ((5, 3), 1, 0.25, 1.0))):
        x, rois, off = roi_case(80 + seed, P=P, scale=scale, margin=-1.0, off_std=2.0)
        out = oracle.roi_pool_forward(x, rois, off, pooled=P, sampling=S, spatial_scale=scale, gamma=gamma,
                                      lib=lib)
        py, px = roi_positions32(rois, off, P, S, scale, gamma)
        B, H, W, C = x.shape
        gy = np.maximum(0, 1 - np.abs(np.arange(H) - py[..., None]))
        gx = np.maximum(0, 1 - np.abs(np.arange(W) - px[..., None]))
        xb = x[rois[:, 0].astype(int)]  # [N, H, W, C]
        ref = np.einsum("nijabh,nijabw,nhwc->nijc", gy, gx, xb) / (S * S)
        assert np.allclose(out, ref, rtol=0, atol=1e-12), "roi brute force"


def pin_roi_bad_batch_index(lib):
    """Regions naming no image (batch index -1, B, 7.5 or NaN) pool to zeros;
    the other regions still equal the brute-force sum over every grid point."""
    P, S, scale, gamma = (3, 2), 2, 0.5, 0.3
    x, rois, off = roi_case(85, B=2, P=P, scale=scale, margin=-1.0, off_std=1.0)
    bad = {1: -1.0, 2: 2.0, 3: 7.5, 4: float("nan")}
    for n, v in bad.items():
        rois[n, 0] = v
    out = oracle.roi_pool_forward(x, rois, off, pooled=P, sampling=S, spatial_scale=scale, gamma=gamma, lib=lib)
    assert np.all(out[list(bad)] == 0.0), "roi bad batch index"
    good = [n for n in range(rois.shape[0]) if n not in bad]
    py, px = roi_positions32(rois[good], off[good], P, S, scale, gamma)
    B, H, W, C = x.shape
    gy = np.maximum(0, 1 - np.abs(np.arange(H) - py[..., None]))
    gx = np.maximum(0, 1 - np.abs(np.arange(W) - px[..., None]))
    xb = x[rois[good, 0].astype(int)]
    ref = np.einsum("nijabh,nijabw,nhwc->nijc", gy, gx, xb) / (S * S)
    assert np.allclose(out[good], ref, rtol=0, atol=1e-12), "roi bad batch index, other regions"


def pin_roi_affine(lib):
    """On x = a + b*y + c*x the pooled value is the field at the mean sample position."""
    rng = np.random.default_rng(90)
    B, H, W, C = 2, 20, 24, 3
    a, bcoef, ccoef = rng.standard_normal((3, C))
    yy, xx = np.meshgrid(np.arange(H), np.arange(W), indexing="ij")
    x = np.broadcast_to(a + bcoef * yy[..., None] + ccoef * xx[..., None], (B, H, W, C)).copy()
    _, rois, off = roi_case(91, B=B, H=H, W=W, C=C, N=8, P=(3, 2), scale=0.5, margin=5.0, off_std=0.3)
    out = oracle.roi_pool_forward(x, rois, off, pooled=(3, 2), sampling=2, spatial_scale=0.5, gamma=0.2,
                                  lib=lib)
    py, px = roi_positions32(rois, off, (3, 2), 2, 0.5, 0.2)
    assert (py >= 0).all() and (py <= H - 1).all() and (px >= 0).all() and (px <= W - 1).all()
    my, mx = py.mean(axis=(-1, -2)), px.mean(axis=(-1, -2))
    ref = a + bcoef * my[..., None] + ccoef * mx[..., None]
    assert np.allclose(out, ref, rtol=0, atol=1e-11), "roi affine"


def pin_roi_constant(lib):
    x = np.full((1, 9, 9, 2), -2.5)
    _, rois, off = roi_case(92, B=1, H=9, W=9, C=2, N=5, P=(2, 2), scale=1.0, margin=2.5, off_std=0.1)
    out = oracle.roi_pool_forward(x, rois, off, pooled=(2, 2), sampling=2, spatial_scale=1.0, gamma=0.1, lib=lib)
    assert np.allclose(out, -2.5, rtol=0, atol=1e-13), "roi constant"


def pin_roi_torchvision(lib):
    """Zero offsets reduce to RoIAlign (torchvision, aligned=False) for regions inside the map."""
    import torchvision

    x, rois, off = roi_case(93, B=2, H=21, W=19, C=4, N=10, P=(4, 3), scale=0.5, margin=3.0)
    off[:] = 0
    out = oracle.roi_pool_forward(x, rois, off, pooled=(4, 3), sampling=2, spatial_scale=0.5, gamma=0.1, lib=lib)
    ref = torchvision.ops.roi_align(torch.from_numpy(x).permute(0, 3, 1, 2).contiguous(),
                                    torch.from_numpy(rois.astype(np.float64)), output_size=(4, 3),
                                    spatial_scale=0.5, sampling_ratio=2, aligned=False)
    assert np.allclose(out, ref.permute(0, 2, 3, 1).numpy(), rtol=0, atol=1e-5), "roi torchvision"


ROI_PINS = [pin_roi_brute_force, pin_roi_bad_batch_index, pin_roi_affine, pin_roi_constant, pin_roi_torchvision]
ALL_PINS = ALL_PINS + ROI_PINS


# ---------------------------------------------------------------- pointwise projection pins
def pin_proj_conv2d(lib):
    """The projection equals PyTorch's 1x1 convolution with bias (fp64), Cout != Cin."""
    rng = np.random.default_rng(101)
    v = rng.standard_normal((2, 5, 7, 12))
    w = rng.standard_normal((20, 12))
    b = rng.standard_normal(20)
    out = oracle.pointwise_projection(v, w, b, lib=lib)
    ref = torch.nn.functional.conv2d(torch.from_numpy(v).permute(0, 3, 1, 2), torch.from_numpy(w)[:, :, None, None],
                                     torch.from_numpy(b))
    assert np.allclose(out, ref.permute(0, 2, 3, 1).numpy(), rtol=0, atol=1e-12), "projection vs conv2d"
    out0 = oracle.pointwise_projection(v, w, None, lib=lib)
    ref0 = torch.nn.functional.conv2d(torch.from_numpy(v).permute(0, 3, 1, 2), torch.from_numpy(w)[:, :, None, None])
    assert np.allclose(out0, ref0.permute(0, 2, 3, 1).numpy(), rtol=0, atol=1e-12), "projection without bias"


def pin_proj_closed_forms(lib):
    """A permutation matrix permutes channels exactly; a zero matrix leaves the bias."""
    rng = np.random.default_rng(102)
    v = rng.standard_normal((3, 4, 16))
    perm = rng.permutation(16)
    w = np.eye(16)[perm]  # out[o] = v[perm[o]]
    assert np.array_equal(oracle.pointwise_projection(v, w, lib=lib), v[..., perm]), "projection permutation"
    b = rng.standard_normal(9)
    out = oracle.pointwise_projection(v, np.zeros((9, 16)), b, lib=lib)
    assert np.array_equal(out, np.broadcast_to(b, out.shape)), "projection bias only"


def pin_proj_composed_identity(lib):
    """Zero offsets with a one-hot centre mask make the core the identity (3x3, pad 1), so the
    composed operator is a 1x1 convolution of x itself."""
    rng = np.random.default_rng(103)
    B, H, W, G, C = 2, 6, 5, 2, 8
    x = rng.standard_normal((B, H, W, G * C))
    off = np.zeros((B, H, W, G, 9, 2))
    mask = np.zeros((B, H, W, G, 9))
    mask[..., 4] = 1.0
    w = rng.standard_normal((24, G * C))
    b = rng.standard_normal(24)
    out = oracle.dcn_forward_proj(x, off, mask, w, b, G=G, lib=lib)
    ref = torch.nn.functional.conv2d(torch.from_numpy(x).permute(0, 3, 1, 2), torch.from_numpy(w)[:, :, None, None],
                                     torch.from_numpy(b))
    assert np.allclose(out, ref.permute(0, 2, 3, 1).numpy(), rtol=0, atol=1e-12), "composed identity"


PROJ_PINS = [pin_proj_conv2d, pin_proj_closed_forms, pin_proj_composed_identity]
ALL_PINS = ALL_PINS + PROJ_PINS


# ---------------------------------------------------------------- modulated deformable convolution pins
def _dconv_case(seed, B=2, H=7, W=9, G=2, C=3, cout=5, kh=3, kw=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, W, G * C)), rng.standard_normal((cout, kh * kw, G * C)),
            rng.standard_normal(cout))


def _tv_offset_mask(off, mask):
    """ours: offset [B,Ho,Wo,G,K,(dx,dy)], mask [B,Ho,Wo,G,K] -> torchvision's
    offset [B, 2*G*K, Ho, Wo] with (dy, dx) per (g, k), mask [B, G*K, Ho, Wo]."""
    B, Ho, Wo, G, K, _ = off.shape
    tv_off = np.stack([off[..., 1], off[..., 0]], axis=-1).reshape(B, Ho, Wo, G * K * 2).transpose(0, 3, 1, 2)
    tv_mask = mask.reshape(B, Ho, Wo, G * K).transpose(0, 3, 1, 2)
    return torch.from_numpy(np.ascontiguousarray(tv_off)), torch.from_numpy(np.ascontiguousarray(tv_mask))


def pin_dconv_torchvision(lib):
    """Equals torchvision's deform_conv2d (DCNv2 with mask) on several geometries;
    offsets on a 1/256 lattice so the fp32 positions are exact."""
    from torchvision.ops import deform_conv2d

    for n, (kh, kw, stride, pad, dil) in enumerate([(3, 3, (1, 1), (1, 1), (1, 1)), (3, 2, (2, 1), (1, 0), (1, 2)),
                                                    (1, 3, (1, 2), (0, 2), (2, 1))]):
        x, w, b = _dconv_case(400 + n, kh=kh, kw=kw)
        B, H, W, GC = x.shape
        G = 2
        Ho, Wo = oracle.out_hw(H, W, kh, kw, *stride, *pad, *dil)
        rng = np.random.default_rng(410 + n)
        off = np.round(rng.standard_normal((B, Ho, Wo, G, kh * kw, 2)) * 1.5 * 256) / 256
        mask = rng.uniform(0.0, 1.0, (B, Ho, Wo, G, kh * kw))
        out = oracle.deform_conv_forward(x, off, mask, w, b, G=G, kh=kh, kw=kw, stride=stride, pad=pad, dil=dil,
                                         lib=lib)
        tv_off, tv_mask = _tv_offset_mask(off, mask)
        tv_w = torch.from_numpy(w.reshape(w.shape[0], kh, kw, GC).transpose(0, 3, 1, 2).copy())
        ref = deform_conv2d(torch.from_numpy(x).permute(0, 3, 1, 2).contiguous(), tv_off, tv_w, torch.from_numpy(b),
                            stride=stride, padding=pad, dilation=dil, mask=tv_mask)
        assert np.allclose(out, ref.permute(0, 2, 3, 1).numpy(), rtol=0, atol=1e-10), f"deform conv vs torchvision {n}"


def pin_dconv_regular_conv(lib):
    """Zero offsets and unit modulation reduce it to an ordinary convolution."""
    x, w, b = _dconv_case(420, B=2, H=8, W=6, G=3, C=2, cout=4)
    B, H, W, GC = x.shape
    for stride, pad, dil in [((1, 1), (1, 1), (1, 1)), ((2, 1), (2, 0), (2, 1))]:
        Ho, Wo = oracle.out_hw(H, W, 3, 3, *stride, *pad, *dil)
        off = np.zeros((B, Ho, Wo, 3, 9, 2))
        mask = np.ones((B, Ho, Wo, 3, 9))
        out = oracle.deform_conv_forward(x, off, mask, w, b, G=3, stride=stride, pad=pad, dil=dil, lib=lib)
        ref = torch.nn.functional.conv2d(torch.from_numpy(x).permute(0, 3, 1, 2),
                                         torch.from_numpy(w.reshape(4, 3, 3, GC).transpose(0, 3, 1, 2).copy()),
                                         torch.from_numpy(b), stride=stride, padding=pad, dilation=dil)
        assert np.allclose(out, ref.permute(0, 2, 3, 1).numpy(), rtol=0, atol=1e-11), "deform conv vs conv2d"


def pin_dconv_softmax_vs_raw(lib):
    """Softmax mode equals raw mode fed with scipy's softmax of the logits over the
    K points of each (pixel, group)."""
    from scipy.special import softmax

    x, w, b = _dconv_case(430, B=1, H=6, W=7, G=2, C=3, cout=3)
    Ho, Wo = oracle.out_hw(6, 7, 3, 3, 1, 1, 1, 1, 1, 1)
    rng = np.random.default_rng(431)
    off = rng.standard_normal((1, Ho, Wo, 2, 9, 2)) * 1.5
    logits = rng.standard_normal((1, Ho, Wo, 2, 9)) * 2.0
    a = oracle.deform_conv_forward(x, off, logits, w, b, G=2, softmax=True, lib=lib)
    r = oracle.deform_conv_forward(x, off, softmax(logits, axis=-1), w, b, G=2, softmax=False, lib=lib)
    assert np.allclose(a, r, rtol=0, atol=1e-12), "deform conv softmax vs raw"


DCONV_PINS = [pin_dconv_torchvision, pin_dconv_regular_conv, pin_dconv_softmax_vs_raw]
ALL_PINS = ALL_PINS + DCONV_PINS
