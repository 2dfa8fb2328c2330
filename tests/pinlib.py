"""Independent formulations and invariant checks that pin the CPU oracle.

Nothing here calls the oracle's C code: these are second and third ways to compute
the same quantities (explicit im2col + matmul, a dense per-channel band matrix, and
torch's float64 CPU convolutions with autograd), written from the definitions:

* parakeet.cpp PR #102, "What changes": the depthwise conv is the sum over k of
  x[t+k, c] * w[k, c] over the input padded to T + K - 1 frames; the old graph computed
  the same conv as im2col + mul_mat.
* NeMo PR #16114, "What does this PR do ?": conv0 (3x3, stride 2, 1 -> C) -> ReLU ->
  masking -> conv_dw1 (depthwise 3x3, stride 2), with pre/post masking and causal padding.

``pin_battery(o)`` runs a quick selection of every pin against an ``oracle.Oracle`` and
returns the list of failures; the mutation test uses it to show that planted mistakes in
the oracle are caught.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch
import torch.nn.functional as Fnn

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def clamp_lengths(lengths, B, T):
    if lengths is None:
        return [T] * B
    return [min(max(int(v), 0), T) for v in lengths]


# ----------------------------------------------------------------------------------
# conv1d: second formulation, explicit im2col + matmul (the old parakeet path)
# ----------------------------------------------------------------------------------
def im2col_fwd(x, w, bias, lengths, pad_left):
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    B, T, C = x.shape
    K = w.shape[0]
    pad_right = K - 1 - pad_left
    Ls = clamp_lengths(lengths, B, T)
    y = np.zeros((B, T, C))
    for b in range(B):
        xm = x[b].copy()
        xm[Ls[b]:] = 0.0
        xp = np.concatenate([np.zeros((pad_left, C)), xm, np.zeros((pad_right, C))], axis=0)
        for c in range(C):
            cols = np.stack([xp[t:t + K, c] for t in range(T)], axis=0) if T else np.zeros((0, K))
            y[b, :, c] = cols @ w[:, c] + (0.0 if bias is None else float(bias[c]))
        y[b, Ls[b]:] = 0.0
    return y


def im2col_dw(x, dy, K, lengths, pad_left):
    x = np.asarray(x, np.float64)
    dy = np.asarray(dy, np.float64)
    B, T, C = x.shape
    pad_right = K - 1 - pad_left
    Ls = clamp_lengths(lengths, B, T)
    dw = np.zeros((K, C))
    db = np.zeros(C)
    for b in range(B):
        xm = x[b].copy()
        xm[Ls[b]:] = 0.0
        dz = dy[b].copy()
        dz[Ls[b]:] = 0.0
        xp = np.concatenate([np.zeros((pad_left, C)), xm, np.zeros((pad_right, C))], axis=0)
        for c in range(C):
            cols = np.stack([xp[t:t + K, c] for t in range(T)], axis=0) if T else np.zeros((0, K))
            dw[:, c] += cols.T @ dz[:, c]
        db += dz.sum(axis=0)
    return dw, db


def band_matrix(wc, T, pad_left):
    """Dense T x T matrix A with (A @ x)[t] = sum_k x[t + k - pad_left] * wc[k] (zero outside)."""
    K = wc.shape[0]
    A = np.zeros((T, T))
    for t in range(T):
        for s in range(T):
            k = s - t + pad_left
            if 0 <= k < K:
                A[t, s] = wc[k]
    return A


def band_dx(dy, w, lengths, pad_left):
    """dx = M A^T M dy per channel: the data gradient as the transpose of the forward matrix."""
    dy = np.asarray(dy, np.float64)
    w = np.asarray(w, np.float64)
    B, T, C = dy.shape
    Ls = clamp_lengths(lengths, B, T)
    dx = np.zeros_like(dy)
    for b in range(B):
        m = (np.arange(T) < Ls[b]).astype(np.float64)
        for c in range(C):
            A = band_matrix(w[:, c], T, pad_left)
            dx[b, :, c] = m * (A.T @ (m * dy[b, :, c]))
    return dx


# ----------------------------------------------------------------------------------
# third formulation: torch float64 CPU convolutions + autograd (a library routine)
# ----------------------------------------------------------------------------------
def torch_conv1d_all(x, w, bias, dy, lengths, pad_left):
    x = torch.tensor(np.asarray(x, np.float64), requires_grad=True)
    w_t = torch.tensor(np.asarray(w, np.float64), requires_grad=True)
    B, T, C = x.shape
    K = w_t.shape[0]
    b_t = torch.tensor(np.asarray(bias, np.float64) if bias is not None else np.zeros(C),
                       requires_grad=True)
    Ls = clamp_lengths(lengths, B, T)
    mask = (torch.arange(T)[None, :] < torch.tensor(Ls)[:, None]).double()[:, :, None]
    inp = Fnn.pad((x * mask).permute(0, 2, 1), (pad_left, K - 1 - pad_left))
    y = Fnn.conv1d(inp, w_t.t().unsqueeze(1), b_t, groups=C).permute(0, 2, 1) * mask
    dy_t = torch.tensor(np.asarray(dy, np.float64))
    (y * dy_t).sum().backward()
    return (y.detach().numpy(), x.grad.numpy(), w_t.grad.numpy(), b_t.grad.numpy())


def torch_subsample(mel, w0, b0, w1, b1, lengths, causal):
    mel = torch.tensor(np.asarray(mel, np.float64))
    B, T, F = mel.shape
    C = np.asarray(w0).shape[-1]
    pt, pb = (2, 0) if causal else (1, 1)
    Ls = clamp_lengths(lengths, B, T)
    m0 = (torch.arange(T)[None, :] < torch.tensor(Ls)[:, None]).double()
    inp = Fnn.pad((mel * m0[:, :, None])[:, None], (1, 1, pt, pb))
    W0 = torch.tensor(np.asarray(w0, np.float64)).permute(2, 0, 1)[:, None]
    W1 = torch.tensor(np.asarray(w1, np.float64)).permute(2, 0, 1)[:, None]
    h = torch.relu(Fnn.conv2d(inp, W0, torch.tensor(np.asarray(b0, np.float64)), stride=2))
    T2 = h.shape[2]
    L2 = [(v + 1) // 2 for v in Ls]
    m2 = (torch.arange(T2)[None, :] < torch.tensor(L2)[:, None]).double()[:, None, :, None]
    h = h * m2
    o = Fnn.conv2d(Fnn.pad(h, (1, 1, pt, pb)), W1, torch.tensor(np.asarray(b1, np.float64)),
                   stride=2, groups=C)
    T4 = o.shape[2]
    L4 = [(v + 1) // 2 for v in L2]
    m4 = (torch.arange(T4)[None, :] < torch.tensor(L4)[:, None]).double()[:, None, :, None]
    o = o * m4
    return o.permute(0, 2, 3, 1).numpy(), np.array(L4, dtype=np.int32)


def torch_subsample_grads(mel, w0, b0, w1, b1, dout, lengths, causal):
    """Gradients of sum(out * dout) with respect to (w0, b0, w1, b1) by float64 autograd through
    the torch formulation above (conv2d, relu, masks); returns numpy arrays in [3,3,C] / [C]."""
    mel = torch.tensor(np.asarray(mel, np.float64))
    B, T, F = mel.shape
    C = np.asarray(w0).shape[-1]
    pt, pb = (2, 0) if causal else (1, 1)
    Ls = clamp_lengths(lengths, B, T)
    W0 = torch.tensor(np.asarray(w0, np.float64)).permute(2, 0, 1)[:, None].clone().requires_grad_(True)
    W1 = torch.tensor(np.asarray(w1, np.float64)).permute(2, 0, 1)[:, None].clone().requires_grad_(True)
    B0 = torch.tensor(np.asarray(b0, np.float64)).requires_grad_(True)
    B1 = torch.tensor(np.asarray(b1, np.float64)).requires_grad_(True)
    m0 = (torch.arange(T)[None, :] < torch.tensor(Ls)[:, None]).double()
    inp = Fnn.pad((mel * m0[:, :, None])[:, None], (1, 1, pt, pb))
    h = torch.relu(Fnn.conv2d(inp, W0, B0, stride=2))
    L2 = [(v + 1) // 2 for v in Ls]
    h = h * (torch.arange(h.shape[2])[None, :] < torch.tensor(L2)[:, None]).double()[:, None, :, None]
    o = Fnn.conv2d(Fnn.pad(h, (1, 1, pt, pb)), W1, B1, stride=2, groups=C)
    L4 = [(v + 1) // 2 for v in L2]
    o = o * (torch.arange(o.shape[2])[None, :] < torch.tensor(L4)[:, None]).double()[:, None, :, None]
    loss = (o * torch.tensor(np.asarray(dout, np.float64)).permute(0, 3, 1, 2)).sum()
    loss.backward()
    g = lambda W: W.grad[:, 0].permute(1, 2, 0).numpy()
    return g(W0), B0.grad.numpy(), g(W1), B1.grad.numpy()


def torch_subsample_kinks(mel, w0, b0, w1, dout, lengths, causal, delta, delta_rel):
    """Brute-force recount of the kink budget of the subsampler backward, written from its
    definition with torch float64 tensors: z = b0 + patches @ w0 over melpad's 3x3 stride-2
    patches (torch's unfold), S = |b0| + |patches| @ |w0|, dh = the gradient of
    sum(mask4 * conv_dw1(pad(h)) * dout) with respect to h by autograd; a valid h pixel
    (row < ceil(len/2)) counts when |z| <= delta + delta_rel * S, and the budget sums |dh| (db0)
    and |dh| |patch tap| (dw0, per tap) over those pixels.  Returns (kdw0 [3,3,C], kdb0 [C])."""
    mel = torch.tensor(np.asarray(mel, np.float64))
    B, T, F = mel.shape
    W0 = torch.tensor(np.asarray(w0, np.float64)).reshape(9, -1)
    C = W0.shape[1]
    pt, pb = (2, 0) if causal else (1, 1)
    Ls = clamp_lengths(lengths, B, T)
    m0 = (torch.arange(T)[None, :] < torch.tensor(Ls)[:, None]).double()
    inp = Fnn.pad((mel * m0[:, :, None])[:, None], (1, 1, pt, pb))
    TP, FP = inp.shape[2], inp.shape[3]
    T2, F2 = (TP - 3) // 2 + 1, (FP - 3) // 2 + 1
    patches = Fnn.unfold(inp, kernel_size=3, stride=2)            # [B, 9, T2*F2], tap = 3p + q
    bb = torch.tensor(np.asarray(b0, np.float64))
    z = torch.einsum("bkn,kc->bnc", patches, W0) + bb          # [B, T2*F2, C]
    S = torch.einsum("bkn,kc->bnc", patches.abs(), W0.abs()) + bb.abs()
    L2 = [(v + 1) // 2 for v in Ls]
    rows = torch.arange(T2)[:, None].expand(T2, F2).reshape(-1)
    valid = rows[None, :] < torch.tensor(L2)[:, None]          # [B, T2*F2]
    hv = torch.zeros(B, C, T2, F2, dtype=torch.float64, requires_grad=True)
    W1 = torch.tensor(np.asarray(w1, np.float64)).permute(2, 0, 1)[:, None]
    o = Fnn.conv2d(Fnn.pad(hv, (1, 1, pt, pb)), W1, None, stride=2, groups=C)
    L4 = [(v + 1) // 2 for v in L2]
    o = o * (torch.arange(o.shape[2])[None, :] < torch.tensor(L4)[:, None]).double()[:, None, :, None]
    (o * torch.tensor(np.asarray(dout, np.float64)).permute(0, 3, 1, 2)).sum().backward()
    dh = hv.grad.permute(0, 2, 3, 1).reshape(B, T2 * F2, C).abs()
    sel = (valid[:, :, None] & (z.abs() <= delta + delta_rel * S)).double()
    kdb0 = (sel * dh).sum(dim=(0, 1))
    kdw0 = torch.einsum("bkn,bnc->kc", patches.abs(), sel * dh)
    return kdw0.reshape(3, 3, C).numpy(), kdb0.numpy()


def subsample_kink_checks(o, rng, B, T, F, C, causal):
    """The oracle's kink budget against the brute-force recount above, at thresholds that take
    no pixel, about half of them, and all of them; returns failure strings."""
    fails = []
    mel = rng.standard_normal((B, T, F)); w0 = rng.standard_normal((3, 3, C)) / 3
    b0 = rng.standard_normal(C) * 0.3; w1 = rng.standard_normal((3, 3, C)) / 3
    L = rng.integers(0, T + 1, size=B).astype(np.int32)
    L[0] = T
    T4, F4 = (((T + 1) // 2 + 1) // 2, ((F + 1) // 2 + 1) // 2)
    dout = rng.standard_normal((B, T4, F4, C))
    for delta, delta_rel in ((0.0, 0.0), (0.3, 0.0), (0.05, 0.2), (1e300, 0.0)):
        got = o.dw_subsample_bwd_kinks(mel, w0, b0, w1, dout, L, causal, delta, delta_rel)
        ref = torch_subsample_kinks(mel, w0, b0, w1, dout, L, causal, delta, delta_rel)
        for name, gv, rv in zip(("kdw0", "kdb0"), got, ref):
            if gv.shape != rv.shape or rel_err(gv, rv) > 1e-12:
                fails.append(f"kink budget {name} {B, T, F, C, causal, delta, delta_rel}")
        if delta == 0.0 and delta_rel == 0.0 and (np.any(got[0] != 0.0) or np.any(got[1] != 0.0)):
            fails.append(f"kink budget not exactly 0 without kinks {B, T, F, C, causal}")
    return fails


def subsample_bwd_checks(o, rng, B, T, F, C, causal):
    """The oracle's subsampler backward against float64 autograd, and dw1 / db1 against exact
    finite differences of <dout, out> (out is linear in w1 and b1).  Returns failure strings."""
    fails = []
    mel = rng.standard_normal((B, T, F)); w0 = rng.standard_normal((3, 3, C)) / 3
    b0 = rng.standard_normal(C) * 0.3; w1 = rng.standard_normal((3, 3, C)) / 3; b1 = rng.standard_normal(C)
    L = rng.integers(0, T + 1, size=B).astype(np.int32)
    L[0] = T
    out, _ = o.dw_subsample_fwd(mel, w0, b0, w1, b1, L, causal)
    dout = rng.standard_normal(out.shape)
    got = o.dw_subsample_bwd(mel, w0, b0, w1, dout, L, causal)
    ref = torch_subsample_grads(mel, w0, b0, w1, b1, dout, L, causal)
    for name, gv, rv in zip(("dw0", "db0", "dw1", "db1"), got, ref):
        if gv.shape != rv.shape or rel_err(gv, rv) > 1e-11:
            fails.append(f"autograd subsample bwd {name} {B, T, F, C, causal}")
    base = float((out * dout).sum())
    for (p, q, c) in ((0, 0, 0), (2, 1, C - 1), (1, 2, C // 2)):
        w1e = w1.copy(); w1e[p, q, c] += 1.0
        oe, _ = o.dw_subsample_fwd(mel, w0, b0, w1e, b1, L, causal)
        if abs(float((oe * dout).sum()) - base - got[2][p, q, c]) > 1e-9 * max(1.0, abs(base)):
            fails.append(f"finite difference dw1 {p, q, c}")
    b1e = b1.copy(); b1e[0] += 1.0
    oe, _ = o.dw_subsample_fwd(mel, w0, b0, w1, b1e, L, causal)
    if abs(float((oe * dout).sum()) - base - got[3][0]) > 1e-9 * max(1.0, abs(base)):
        fails.append("finite difference db1")
    return fails


def torch_dwconv2d_all(x, w, bias, dy, lengths, stride, pads):
    """Depthwise conv2d with input and output length masks through torch float64 (conv2d with
    groups=C) and autograd: returns (y, dx, dW [KT,KF,C], dbias) for loss = sum(y * dy)."""
    (st, sf), (pt, pb, pf) = stride, pads
    x = torch.tensor(np.asarray(x, np.float64), requires_grad=True)
    B, T, F, C = x.shape
    KT, KF = np.asarray(w).shape[:2]
    W = torch.tensor(np.asarray(w, np.float64)).permute(2, 0, 1)[:, None].clone().requires_grad_(True)
    bb = torch.tensor(np.asarray(bias, np.float64) if bias is not None else np.zeros(C)).requires_grad_(True)
    Ls = clamp_lengths(lengths, B, T)
    m = (torch.arange(T)[None, :] < torch.tensor(Ls)[:, None]).double()[:, :, None, None]
    xin = Fnn.pad((x * m).permute(0, 3, 1, 2), (pf, pf, pt, pb))
    y = Fnn.conv2d(xin, W, bb, stride=(st, sf), groups=C)
    To = y.shape[2]
    Lo = [min(To, max(0, (L + pt + pb - KT) // st + 1) if L + pt + pb - KT >= 0 else 0) for L in Ls]
    y = y * (torch.arange(To)[None, :] < torch.tensor(Lo)[:, None]).double()[:, None, :, None]
    y = y.permute(0, 2, 3, 1)
    (y * torch.tensor(np.asarray(dy, np.float64))).sum().backward()
    return y.detach().numpy(), x.grad.numpy(), W.grad[:, 0].permute(1, 2, 0).numpy(), bb.grad.numpy()


def conv2d_checks(o, rng, B, T, F, C, KT, KF, stride, pads):
    """The oracle's depthwise conv2d forward and gradients against torch autograd; returns
    failure strings."""
    import oracle as _oracle_mod  # only for the shape rule
    fails = []
    To, Fo = _oracle_mod.conv2d_out_shape(T, F, KT, KF, stride, pads)
    x = rng.standard_normal((B, T, F, C)); w = rng.standard_normal((KT, KF, C)); b = rng.standard_normal(C)
    dy = rng.standard_normal((B, To, Fo, C))
    L = rng.integers(0, T + 1, size=B).astype(np.int32)
    L[0] = T
    y, ol = o.dwconv2d_fwd(x, w, b, L, stride, pads)
    dx = o.dwconv2d_bwd_dx(dy, w, L, T, F, stride, pads)
    gw, gb = o.dwconv2d_bwd_dw(x, dy, KT, KF, L, stride, pads)
    tag = (B, T, F, C, KT, KF, stride, pads)
    if To == 0 or Fo == 0:  # the window does not fit the padded input: no output, zero gradients
        if y.size or np.any(dx != 0.0) or np.any(gw != 0.0) or np.any(gb != 0.0) or np.any(ol != 0):
            fails.append(f"conv2d empty output {tag}")
        return fails
    ry, rdx, rgw, rgb = torch_dwconv2d_all(x, w, b, dy, L, stride, pads)
    if y.shape != ry.shape or rel_err(y, ry) > 1e-12:
        fails.append(f"torch conv2d fwd {tag}")
    if rel_err(dx, rdx) > 1e-12:
        fails.append(f"torch conv2d dx {tag}")
    if rel_err(gw, rgw) > 1e-12 or rel_err(gb, rgb) > 1e-12:
        fails.append(f"torch conv2d dw {tag}")
    return fails


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def rel_err(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    if a.size == 0:
        return 0.0
    scale = max(np.max(np.abs(b)), 1e-300)
    return float(np.max(np.abs(a - b)) / scale)


# ----------------------------------------------------------------------------------
# a quick battery of every kind of pin, for the mutation test
# ----------------------------------------------------------------------------------
def np_stream_fwd(x, w, bias, cache, L):
    """One chunk of the streaming causal conv written out directly in numpy: the chunk's valid
    frames appended to the K-1 cached ones, the K-tap sum, the output mask, the new cache."""
    B, T, C = x.shape
    K = w.shape[0]
    y = np.zeros((B, T, C))
    cout = np.zeros((B, K - 1, C))
    for b in range(B):
        n = T if L is None else int(min(max(L[b], 0), T))
        xcat = np.concatenate([cache[b], x[b, :n]], axis=0)  # [K-1+n, C]
        for t in range(n):
            y[b, t] = (0.0 if bias is None else bias) + (xcat[t:t + K] * w).sum(axis=0)
        cout[b] = xcat[n:n + K - 1]
    return y, cout


def stream_chunked_vs_whole(o, rng, B, C, K, T, n_chunks, bias=True):
    """Feed random chunks (valid lengths 0..T, some below K-1) through ``o.dwconv1d_stream_fwd``
    from a zero cache; compare every valid output with the causal conv (im2col formulation) of
    each stream's concatenated valid frames, masked outputs with exact zeros, and the final
    cache with the stream's last K-1 frames.  Returns a list of failure strings."""
    fails = []
    w = rng.standard_normal((K, C)); b = rng.standard_normal(C) if bias else None
    cache = np.zeros((B, K - 1, C))
    seen = [np.zeros((0, C)) for _ in range(B)]
    outs = [[] for _ in range(B)]
    for _ in range(n_chunks):
        x = rng.standard_normal((B, T, C))
        L = rng.integers(0, T + 1, size=B).astype(np.int32)
        y, cache = o.dwconv1d_stream_fwd(x, w, b, cache, L)
        for i in range(B):
            if np.any(y[i, L[i]:] != 0.0):
                fails.append(f"stream masked frames not zero {B, C, K, T}")
            seen[i] = np.concatenate([seen[i], x[i, :L[i]]])
            outs[i].append(y[i, :L[i]])
    for i in range(B):
        n = seen[i].shape[0]
        if n == 0:
            continue
        whole = im2col_fwd(seen[i][None], w, b, None, K - 1)[0]
        got = np.concatenate(outs[i])
        if rel_err(got, whole) > 1e-12:
            fails.append(f"stream chunked != whole {B, C, K, T}")
        last = np.concatenate([np.zeros((K - 1, C)), seen[i]])[-(K - 1):] if K > 1 else np.zeros((0, C))
        if not np.array_equal(cache[i], last):
            fails.append(f"stream cache != last frames {B, C, K, T}")
    return fails


def pin_battery(o):
    """Run a fast selection of pins against oracle ``o``; returns a list of failure strings."""
    fails = []
    rng = np.random.default_rng(123)

    # golden, hand-worked values
    g = load_golden("dwconv1d_worked_example.json")
    x = np.array(g["x"], float); w = np.array(g["w"], float); bias = np.array(g["bias"], float)
    dy = np.array(g["dy"], float); L = np.array(g["lengths"], np.int32)
    s = g["symmetric"]
    if not np.array_equal(o.dwconv1d_fwd(x, w, bias, L, s["pad_left"]), np.array(s["y"], float)):
        fails.append("golden fwd symmetric")
    if not np.array_equal(o.dwconv1d_bwd_dx(dy, w, L, s["pad_left"]), np.array(s["dx"], float)):
        fails.append("golden dx")
    dw, db = o.dwconv1d_bwd_dw(x, dy, 3, L, s["pad_left"])
    if not (np.array_equal(dw, np.array(s["dw"], float)) and np.array_equal(db, np.array(s["dbias"], float))):
        fails.append("golden dw/dbias")
    cz = g["causal_no_bias"]
    if not np.array_equal(o.dwconv1d_fwd(x, w, None, L, cz["pad_left"]), np.array(cz["y"], float)):
        fails.append("golden fwd causal")
    gs = load_golden("subsample_worked_example.json")
    for mode, causal in (("symmetric", False), ("causal", True)):
        e = gs[mode]
        out, ol = o.dw_subsample_fwd(np.array(gs["mel"], float), np.array(e["w0"], float),
                                     np.array(e["b0"], float), np.array(gs["w1"], float),
                                     np.array(gs["b1"], float), np.array(gs["lengths"], np.int32),
                                     causal)
        if not (np.array_equal(out, np.array(e["out"], float)) and list(ol) == e["out_lengths"]):
            fails.append(f"golden subsample {mode}")

    # second formulations (im2col, band matrix) and torch autograd on small random cases
    for (B, T, C, K, pl) in ((3, 11, 5, 4, 1), (2, 7, 3, 9, 8), (1, 2, 2, 5, 2), (2, 16, 9, 3, 1)):
        x = rng.standard_normal((B, T, C)); w = rng.standard_normal((K, C))
        bias = rng.standard_normal(C); dy = rng.standard_normal((B, T, C))
        L = rng.integers(0, T + 1, size=B).astype(np.int32)
        y = o.dwconv1d_fwd(x, w, bias, L, pl)
        if rel_err(y, im2col_fwd(x, w, bias, L, pl)) > 1e-12:
            fails.append(f"im2col fwd {B, T, C, K, pl}")
        if rel_err(o.dwconv1d_bwd_dx(dy, w, L, pl), band_dx(dy, w, L, pl)) > 1e-12:
            fails.append(f"band dx {B, T, C, K, pl}")
        dw, db = o.dwconv1d_bwd_dw(x, dy, K, L, pl)
        rdw, rdb = im2col_dw(x, dy, K, L, pl)
        if rel_err(dw, rdw) > 1e-12 or rel_err(db, rdb) > 1e-12:
            fails.append(f"im2col dw {B, T, C, K, pl}")
        ty, tdx, tdw, tdb = torch_conv1d_all(x, w, bias, dy, L, pl)
        if rel_err(y, ty) > 1e-12:
            fails.append(f"torch fwd {B, T, C, K, pl}")

    for causal in (False, True):
        B, T, F, C = 2, 13, 10, 3
        mel = rng.standard_normal((B, T, F)); w0 = rng.standard_normal((3, 3, C))
        w1 = rng.standard_normal((3, 3, C)); b0 = rng.standard_normal(C); b1 = rng.standard_normal(C)
        L = np.array([13, 6], np.int32)
        out, ol = o.dw_subsample_fwd(mel, w0, b0, w1, b1, L, causal)
        ref, rl = torch_subsample(mel, w0, b0, w1, b1, L, causal)
        if out.shape != ref.shape or rel_err(out, ref) > 1e-12 or not np.array_equal(ol, rl):
            fails.append(f"torch subsample causal={causal}")

    # streaming chunks: the whole-stream causal conv, and the direct numpy statement
    for (B, C, K, T, n) in ((3, 4, 4, 5, 6), (2, 3, 9, 3, 8), (2, 2, 1, 4, 3)):
        fails += stream_chunked_vs_whole(o, rng, B, C, K, T, n)
    x = rng.standard_normal((3, 6, 5)); w = rng.standard_normal((3, 5)); bias = rng.standard_normal(5)
    cache = rng.standard_normal((3, 2, 5)); L = np.array([6, 0, 1], np.int32)
    y, c = o.dwconv1d_stream_fwd(x, w, bias, cache, L)
    ry, rc = np_stream_fwd(x, w, bias, cache, L)
    if rel_err(y, ry) > 1e-12 or not np.array_equal(c, rc):
        fails.append("numpy stream")

    # subsampler backward: autograd and exact finite differences; its kink budget: brute force
    for causal in (False, True):
        fails += subsample_bwd_checks(o, rng, 2, 13, 10, 3, causal)
        fails += subsample_kink_checks(o, rng, 3, 14, 9, 4, causal)

    # general depthwise conv2d: torch autograd, symmetric and causal, strides 1 and 2
    for (KT, KF, stride, pads) in ((3, 3, (2, 2), (1, 1, 1)), (3, 2, (1, 2), (2, 0, 1)), (2, 3, (2, 1), (0, 1, 0))):
        fails += conv2d_checks(o, rng, 2, 11, 9, 3, KT, KF, stride, pads)
    return fails
