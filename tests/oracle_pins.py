"""Pins of the CPU oracle: checks against facts fixed by the pages and by
mathematics, never against the oracle's own formula.

Each ``pin_*`` function takes an oracle library handle (``oracle.load()`` or
a deliberately mutated build) and raises AssertionError when the oracle
disagrees with the fact.  ``test_oracle_pins.py`` runs them on the real
oracle; ``test_oracle_mutants.py`` checks that every planted mistake in the
oracle makes at least one of them fail.

Sources (pages as titled):
* "Mamba ... 并行扫描" (mhpq.cn) §2.3 -- the unrolled closed form
  x_k = A^k x_0 + sum_i A^{k-i} B u_i, and the combine operator
  (A1, B1) (+) (A2, B2) = (A2 A1, A2 B1 + B2) evaluated as a prefix scan;
* "Mamba状态空间模型的硬件感知推理优化" (ybb.press) §2.1 -- the augmented
  matrix M_t = [[A, B x_t], [0, 1]] whose prefix product gives the state;
  §2.2 -- Blelloch up-sweep / down-sweep; §4 -- the scalar-decay (Mamba-2)
  closed form with cumulative products, evaluated in log space (§6.2);
  §4 -- chunked parallel/serial hybrid scan;
* "Mamba与选择性SSM" (mlqm.cn) §5.4 -- decode keeps only the state.
"""
from __future__ import annotations

import numpy as np
from scipy.special import expit

import oracle

REL = 1e-10  # double-precision agreement, relative to the largest reference value


def _close(got, ref, rel=REL, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} != {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    scale = max(float(np.max(np.abs(ref))), 1e-300)
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert err <= rel * scale, f"{what}: max|err| {err:.3e} > {rel:.1e} * {scale:.3e}"


def _softplus(s):
    return np.logaddexp(0.0, s)  # library form of log(1 + e^s)


def _silu(z):
    return z * expit(z)  # library logistic sigmoid


def _rand_scan(rng, batch=2, dim=3, N=4, L=24, gate=True, h0=True):
    return dict(
        u=rng.standard_normal((batch, dim, L)),
        delta=rng.standard_normal((batch, dim, L)),
        A=-np.exp(rng.uniform(0.0, np.log(10.0), (dim, N))),
        B=rng.standard_normal((batch, N, L)),
        C=rng.standard_normal((batch, N, L)),
        D=rng.standard_normal(dim),
        z=rng.standard_normal((batch, dim, L)) if gate else None,
        delta_bias=rng.uniform(-3.0, 0.5, dim),
        h0=rng.standard_normal((batch, dim, N)) if h0 else None,
    )


def _discretise(inp):
    """dt', dA (b,d,n,t), dBu (b,d,n,t) from the definitions."""
    dt = _softplus(inp["delta"] + inp["delta_bias"][None, :, None])
    dA = np.exp(dt[:, :, None, :] * inp["A"][None, :, :, None])
    dBu = dt[:, :, None, :] * inp["B"][:, None, :, :] * inp["u"][:, :, None, :]
    return dt, dA, dBu


def _readout(inp, h_all):
    """y from states h_all (b,d,n,t): C.h + D u, then the silu(z) gate."""
    y = np.einsum("bnt,bdnt->bdt", inp["C"], h_all) + inp["D"][None, :, None] * inp["u"]
    if inp["z"] is not None:
        y = y * _silu(inp["z"])
    return y


def _run(lib, inp, **kw):
    args = dict(inp)
    args.update(kw)
    return oracle.scan_fwd(args["u"], args["delta"], args["A"], args["B"], args["C"], args["D"],
                           args["z"], args["delta_bias"], args.get("delta_softplus", True),
                           args["h0"], nthreads=2, lib=lib)


# ---------------------------------------------------------------- Mamba-1 pins
def pin_closed_form(lib):
    """P1: h_k = (prod_{j<=k} dA_j) h_0 + sum_{i<=k} (prod_{i<j<=k} dA_j) dBu_i (O(L^2))."""
    rng = np.random.default_rng(11)
    inp = _rand_scan(rng, L=20)
    _, dA, dBu = _discretise(inp)
    b, d, n, L = dA.shape
    h_all = np.zeros((b, d, n, L))
    for k in range(L):
        acc = np.prod(dA[..., : k + 1], axis=-1) * inp["h0"]
        for i in range(k + 1):
            acc = acc + np.prod(dA[..., i + 1: k + 1], axis=-1) * dBu[..., i]
        h_all[..., k] = acc
    y, h_last = _run(lib, inp)
    _close(y, _readout(inp, h_all), what="closed form y")
    _close(h_last, h_all[..., -1], what="closed form h_L")


def pin_augmented_matrix(lib):
    """P2: [h_t; 1] = M_t ... M_1 [h_0; 1] with M_t = [[dA_t, dBu_t], [0, 1]]."""
    rng = np.random.default_rng(12)
    inp = _rand_scan(rng, batch=1, dim=4, N=3, L=17)
    _, dA, dBu = _discretise(inp)
    b, d, n, L = dA.shape
    M = np.zeros((b, d, n, L, 2, 2))
    M[..., 0, 0] = dA
    M[..., 0, 1] = dBu
    M[..., 1, 1] = 1.0
    prefix = np.broadcast_to(np.eye(2), (b, d, n, 2, 2)).copy()
    v0 = np.stack([inp["h0"], np.ones_like(inp["h0"])], axis=-1)
    h_all = np.zeros((b, d, n, L))
    for t in range(L):
        prefix = np.matmul(M[..., t, :, :], prefix)
        h_all[..., t] = np.einsum("...ij,...j->...i", prefix, v0)[..., 0]
    y, h_last = _run(lib, inp)
    _close(y, _readout(inp, h_all), what="augmented matrix y")
    _close(h_last, h_all[..., -1], what="augmented matrix h_L")


def _combine(p, q):
    """(a1, b1) (+) (a2, b2) = (a2 a1, a2 b1 + b2): p first, then q."""
    return (q[0] * p[0], q[0] * p[1] + q[1])


def pin_blelloch_order(lib):
    """P3: the combine operator folded in Blelloch up/down-sweep order gives the
    same inclusive states as the sequential recurrence."""
    rng = np.random.default_rng(13)
    inp = _rand_scan(rng, batch=1, dim=2, N=3, L=32, h0=True)
    _, dA, dBu = _discretise(inp)
    L = dA.shape[-1]
    a = [dA[..., t] for t in range(L)]
    bb = [dBu[..., t] for t in range(L)]
    # up-sweep
    tree = [(a[t], bb[t]) for t in range(L)]
    step = 1
    while step < L:
        for i in range(2 * step - 1, L, 2 * step):
            tree[i] = _combine(tree[i - step], tree[i])
        step *= 2
    # down-sweep (exclusive prefixes); identity is (1, 0)
    tree[L - 1] = (np.ones_like(a[0]), np.zeros_like(bb[0]))
    step = L // 2
    while step >= 1:
        for i in range(2 * step - 1, L, 2 * step):
            left = tree[i - step]
            tree[i - step] = tree[i]
            tree[i] = _combine(tree[i], left)
        step //= 2
    h_all = np.zeros(dA.shape)
    for t in range(L):
        excl = tree[t]
        inc = _combine(excl, (a[t], bb[t]))
        h_all[..., t] = inc[0] * inp["h0"] + inc[1]
    y, h_last = _run(lib, inp)
    _close(y, _readout(inp, h_all), what="Blelloch y")
    _close(h_last, h_all[..., -1], what="Blelloch h_L")


def pin_lti_convolution(lib):
    """P4: with delta, B, C constant in time the scan is a causal convolution of u
    with K_k = sum_n C_n dA_n^k dt' B_n, plus D u, then the gate."""
    rng = np.random.default_rng(14)
    batch, dim, N, L = 2, 3, 5, 40
    inp = _rand_scan(rng, batch, dim, N, L, gate=True, h0=False)
    inp["delta"] = np.repeat(rng.standard_normal((batch, dim, 1)), L, axis=2)
    inp["B"] = np.repeat(rng.standard_normal((batch, N, 1)), L, axis=2)
    inp["C"] = np.repeat(rng.standard_normal((batch, N, 1)), L, axis=2)
    y, _ = _run(lib, inp)
    ref = np.zeros((batch, dim, L))
    for b in range(batch):
        for d in range(dim):
            dt = _softplus(inp["delta"][b, d, 0] + inp["delta_bias"][d])
            dA = np.exp(dt * inp["A"][d])
            k = np.arange(L)
            K = np.sum(inp["C"][b, :, 0][:, None] * dA[:, None] ** k[None, :] * dt
                       * inp["B"][b, :, 0][:, None], axis=0)
            conv = np.convolve(inp["u"][b, d], K)[:L]
            ref[b, d] = (conv + inp["D"][d] * inp["u"][b, d]) * _silu(inp["z"][b, d])
    _close(y, ref, what="LTI convolution")


def pin_split_resume(lib):
    """P5: scan [0, m) -> h_m, resume [m, L) from h_m == one scan over [0, L)."""
    rng = np.random.default_rng(15)
    inp = _rand_scan(rng, L=30)
    y, h_last = _run(lib, inp)
    m = 13
    first = {k: (v[..., :m] if k in ("u", "delta", "z", "B", "C") and v is not None else v)
             for k, v in inp.items()}
    y1, hm = _run(lib, first)
    second = {k: (v[..., m:] if k in ("u", "delta", "z", "B", "C") and v is not None else v)
              for k, v in inp.items()}
    second["h0"] = hm
    y2, hl2 = _run(lib, second)
    _close(np.concatenate([y1, y2], axis=-1), y, rel=0.0, what="split y")
    _close(hl2, h_last, rel=0.0, what="split h_L")


def pin_prefix_sum_case(lib):
    """P6a: A = 0, softplus off, delta = 1, no bias, B = C = 1, D = 0, no gate
    -> dA = 1, h_t[n] = cumsum(u), y = N * cumsum(u)."""
    rng = np.random.default_rng(16)
    batch, dim, N, L = 2, 3, 7, 50
    u = rng.standard_normal((batch, dim, L))
    y, h_last = oracle.scan_fwd(u, np.ones_like(u), np.zeros((dim, N)), np.ones((batch, N, L)),
                                np.ones((batch, N, L)), np.zeros(dim), None, None, False, None,
                                nthreads=1, lib=lib)
    _close(y, N * np.cumsum(u, axis=-1), what="prefix-sum y")
    _close(h_last, np.repeat(np.sum(u, axis=-1)[..., None], N, axis=-1), what="prefix-sum h_L")


def pin_memoryless_case(lib):
    """P6b: a very fast decay (dA underflows) leaves h_t = dt' B_t u_t, so
    y_t = dt'_t u_t (C_t . B_t) + D u_t: no memory of earlier steps."""
    rng = np.random.default_rng(17)
    inp = _rand_scan(rng, batch=2, dim=3, N=4, L=25, gate=False, h0=True)
    inp["A"] = np.full_like(inp["A"], -1e6)
    inp["delta_bias"] = np.full_like(inp["delta_bias"], 1.0)  # dt' >= softplus(1 - |delta|) > 0.01
    inp["delta"] = np.clip(inp["delta"], -3.0, 3.0)
    y, h_last = _run(lib, inp)
    dt = _softplus(inp["delta"] + 1.0)
    cb = np.einsum("bnt,bnt->bt", inp["C"], inp["B"])
    ref = dt * inp["u"] * cb[:, None, :] + inp["D"][None, :, None] * inp["u"]
    _close(y, ref, what="memoryless y")
    _close(h_last, dt[:, :, None, -1] * inp["B"][:, None, :, -1] * inp["u"][:, :, None, -1],
           what="memoryless h_L")


def pin_gate_and_skip(lib):
    """The gate multiplies the whole of C.h + D u by z * sigmoid(z); the skip
    adds exactly D u before it."""
    rng = np.random.default_rng(18)
    inp = _rand_scan(rng)
    y_gated, h1 = _run(lib, inp)
    y_plain, h2 = _run(lib, inp, z=None)
    _close(y_gated, y_plain * _silu(inp["z"]), what="gate")
    _close(h1, h2, rel=0.0, what="gate leaves the state alone")
    y_nod, _ = _run(lib, inp, z=None, D=None)
    _close(y_plain - y_nod, inp["D"][None, :, None] * inp["u"], what="skip")


def pin_softplus_and_bias(lib):
    """dt' = softplus(delta + bias): equal to the scan with softplus off fed the
    library softplus of delta + bias, and the bias acts only through the sum."""
    rng = np.random.default_rng(19)
    inp = _rand_scan(rng)
    y, h = _run(lib, inp)
    pre = _softplus(inp["delta"] + inp["delta_bias"][None, :, None])
    y2, h2 = _run(lib, inp, delta=pre, delta_bias=None, delta_softplus=False)
    _close(y2, y, rel=1e-12, what="softplus")
    _close(h2, h, rel=1e-12, what="softplus h")
    y3, _ = _run(lib, inp, delta=inp["delta"] + inp["delta_bias"][None, :, None],
                 delta_bias=None)
    _close(y3, y, rel=1e-13, what="bias placement")
    # softplus off: dt' is delta + bias itself
    y4, _ = _run(lib, inp, delta_softplus=False)
    y5, _ = _run(lib, inp, delta=inp["delta"] + inp["delta_bias"][None, :, None],
                 delta_bias=None, delta_softplus=False)
    _close(y4, y5, rel=1e-13, what="softplus off")


def pin_decode_steps(lib):
    """P7: L decode steps from h0 reproduce the sequence scan exactly."""
    rng = np.random.default_rng(20)
    inp = _rand_scan(rng, batch=2, dim=3, N=5, L=12)
    y, h_last = _run(lib, inp)
    st = inp["h0"].copy()
    ys = []
    for t in range(inp["u"].shape[-1]):
        yt, st = oracle.scan_step(st, inp["u"][..., t], inp["delta"][..., t], inp["A"],
                                  inp["B"][..., t], inp["C"][..., t], inp["D"], inp["z"][..., t],
                                  inp["delta_bias"], True, lib=lib)
        ys.append(yt)
    _close(np.stack(ys, axis=-1), y, rel=0.0, what="decode y")
    _close(st, h_last, rel=0.0, what="decode state")


# ---------------------------------------------------------------- Mamba-2 pins
def _rand_ssd(rng, batch=2, L=20, H=3, P=4, N=5, gate=False, h0=True):
    return dict(
        x=rng.standard_normal((batch, L, H, P)),
        delta=rng.standard_normal((batch, L, H)),
        A=-np.exp(rng.uniform(0.0, np.log(16.0), H)),
        B=rng.standard_normal((batch, L, N)),
        C=rng.standard_normal((batch, L, N)),
        D=rng.standard_normal(H),
        z=rng.standard_normal((batch, L, H, P)) if gate else None,
        delta_bias=rng.uniform(-3.0, 0.5, H),
        h0=rng.standard_normal((batch, H, P, N)) if h0 else None,
    )


def _run_ssd(lib, inp, **kw):
    a = dict(inp)
    a.update(kw)
    return oracle.ssd_fwd(a["x"], a["delta"], a["A"], a["B"], a["C"], a["D"], a["z"],
                          a["delta_bias"], a.get("delta_softplus", True), a["h0"], nthreads=2,
                          lib=lib)


def pin_ssd_is_mamba1(lib):
    """P8: one head of the scalar-decay scan is the Mamba-1 scan over P channels
    whose decay rates are all A_h and whose B, C are shared."""
    rng = np.random.default_rng(21)
    inp = _rand_ssd(rng, batch=2, L=15, H=1, P=4, N=3, gate=True)
    y, h_last = _run_ssd(lib, inp)
    P, N = 4, 3
    u = np.transpose(inp["x"][:, :, 0, :], (0, 2, 1))  # (b, P, L)
    dl = np.repeat(inp["delta"][:, None, :, 0], P, axis=1)
    z = np.transpose(inp["z"][:, :, 0, :], (0, 2, 1))
    y1, h1 = oracle.scan_fwd(u, dl, np.full((P, N), inp["A"][0]),
                             np.transpose(inp["B"], (0, 2, 1)), np.transpose(inp["C"], (0, 2, 1)),
                             np.full(P, inp["D"][0]), z, np.full(P, inp["delta_bias"][0]), True,
                             inp["h0"][:, 0], nthreads=1, lib=lib)
    _close(np.transpose(y[:, :, 0, :], (0, 2, 1)), y1, rel=1e-13, what="SSD vs Mamba-1 y")
    _close(h_last[:, 0], h1, rel=1e-13, what="SSD vs Mamba-1 h_L")


def ssd_quadratic(inp):
    """Closed form of the scalar-decay scan with cumulative log-decays:
    y_t = sum_{k<=t} (C_t . B_k) exp(cum_t - cum_k) dt'_k x_k
          + exp(cum_t) S_0 C_t + D x_t   (then the optional gate)."""
    x, Bm, Cm = inp["x"], inp["B"], inp["C"]
    batch, L, H, P = x.shape
    dt = _softplus(inp["delta"] + inp["delta_bias"][None, None, :])  # (b, L, H)
    cum = np.cumsum(dt * inp["A"][None, None, :], axis=1)  # log of the cumulative product
    G = np.einsum("btn,bkn->btk", Cm, Bm)
    y = np.zeros_like(x)
    h_last = np.zeros((batch, H, P, Bm.shape[2]))
    mask = np.tril(np.ones((L, L), dtype=bool))
    for b in range(batch):
        for h in range(H):
            seg = cum[b, :, h][:, None] - cum[b, :, h][None, :]
            W = np.where(mask, G[b] * np.exp(np.where(mask, seg, 0.0)), 0.0)
            y[b, :, h, :] = W @ (dt[b, :, h][:, None] * x[b, :, h, :])
            wend = np.exp(cum[b, -1, h] - cum[b, :, h]) * dt[b, :, h]
            h_last[b, h] = (wend[:, None] * x[b, :, h, :]).T @ Bm[b]
            if inp["h0"] is not None:
                y[b, :, h, :] += np.exp(cum[b, :, h])[:, None] * (Cm[b] @ inp["h0"][b, h].T)
                h_last[b, h] += np.exp(cum[b, -1, h]) * inp["h0"][b, h]
            y[b, :, h, :] += inp["D"][h] * x[b, :, h, :]
    if inp["z"] is not None:
        y = y * _silu(inp["z"])
    return y, h_last


def ssd_chunked(inp, chunk):
    """The chunked (parallel within a chunk, serial between chunks) form:
    per chunk a masked quadratic part, a chunk state, and the carried state
    read out through C with the decay from the chunk start."""
    x, Bm, Cm = inp["x"], inp["B"], inp["C"]
    batch, L, H, P = x.shape
    N = Bm.shape[2]
    dt = _softplus(inp["delta"] + inp["delta_bias"][None, None, :])
    y = np.zeros_like(x)
    h_last = np.zeros((batch, H, P, N))
    for b in range(batch):
        for h in range(H):
            S = inp["h0"][b, h].copy() if inp["h0"] is not None else np.zeros((P, N))
            for c0 in range(0, L, chunk):
                sl = slice(c0, min(L, c0 + chunk))
                la = dt[b, sl, h] * inp["A"][h]
                cum = np.cumsum(la)
                Q = cum.shape[0]
                mask = np.tril(np.ones((Q, Q), dtype=bool))
                seg = np.where(mask, cum[:, None] - cum[None, :], 0.0)
                G = Cm[b, sl] @ Bm[b, sl].T
                xs = dt[b, sl, h][:, None] * x[b, sl, h, :]
                yc = np.where(mask, G * np.exp(seg), 0.0) @ xs
                yc += np.exp(cum)[:, None] * (Cm[b, sl] @ S.T)
                S = np.exp(cum[-1]) * S + (np.exp(cum[-1] - cum)[:, None] * xs).T @ Bm[b, sl]
                y[b, sl, h, :] = yc + inp["D"][h] * x[b, sl, h, :]
            h_last[b, h] = S
    if inp["z"] is not None:
        y = y * _silu(inp["z"])
    return y, h_last


def pin_ssd_quadratic(lib):
    """P9: the sequential scalar-decay scan equals its log-space closed form."""
    rng = np.random.default_rng(22)
    inp = _rand_ssd(rng, batch=2, L=24, H=3, P=4, N=5, gate=True)
    y, h_last = _run_ssd(lib, inp)
    yq, hq = ssd_quadratic(inp)
    _close(y, yq, what="SSD quadratic y")
    _close(h_last, hq, what="SSD quadratic h_L")


def pin_ssd_chunked(lib):
    """P10 (oracle side): the chunked hybrid form, for several chunk lengths
    including ragged last chunks, equals the sequential scan."""
    rng = np.random.default_rng(23)
    inp = _rand_ssd(rng, batch=1, L=37, H=2, P=3, N=4, gate=False)
    y, h_last = _run_ssd(lib, inp)
    for q in (4, 8, 16, 37, 64):
        yc, hc = ssd_chunked(inp, q)
        _close(y, yc, what=f"SSD chunk {q} y")
        _close(h_last, hc, what=f"SSD chunk {q} h_L")


# ---- the convolution stage in front of the scan -------------------------------
# Page "从硬件感知到算法革命" (tencentcloud) §3: a local convolution over time
# (kernel size 4) feeds the selective SSM; SiLU is the block's activation.


def _rand_conv(rng, batch=2, dim=3, L=30, K=4, prev=True):
    x = rng.standard_normal((batch, dim, L))
    w = rng.standard_normal((dim, K)) * 0.7
    b = rng.standard_normal(dim) * 0.3
    xp = rng.standard_normal((batch, dim, K - 1)) if prev and K > 1 else None
    return x, w, b, xp


def _conv_numpy(x, w, b, xp):
    """The causal depthwise convolution by np.convolve: the channel's inputs
    with the preceding window prepended, convolved with the taps reversed
    (np.convolve flips its kernel), the causal outputs kept; then SiLU."""
    batch, dim, L = x.shape
    K = w.shape[1]
    out = np.empty_like(x)
    for bb in range(batch):
        for d in range(dim):
            prev = xp[bb, d] if xp is not None else np.zeros(K - 1)
            xe = np.concatenate([prev, x[bb, d]])
            pre = np.convolve(xe, w[d, ::-1])[K - 1:K - 1 + L] + (b[d] if b is not None else 0.0)
            out[bb, d] = _silu(pre)
    return out


def pin_conv_numpy(lib):
    """C1: the convolution stage equals np.convolve's causal outputs plus the
    bias, through SiLU, for widths 1..4, with and without the preceding
    window and the bias."""
    rng = np.random.default_rng(31)
    for K in (1, 2, 3, 4):
        for prev in (True, False):
            x, w, b, xp = _rand_conv(rng, K=K, prev=prev)
            for bias in (b, None):
                got = oracle.conv_silu(x, w, bias, xp, lib=lib)
                _close(got, _conv_numpy(x, w, bias, xp), what=f"conv K={K} prev={prev}")


def pin_conv_one_tap(lib):
    """C2: one tap of weight 1 and no bias leave u = silu(x) = x expit(x)."""
    rng = np.random.default_rng(32)
    x = rng.standard_normal((2, 3, 17)) * 3
    got = oracle.conv_silu(x, np.ones((3, 1)), None, None, lib=lib)
    _close(got, x * expit(x), what="one-tap conv")


def pin_conv_split_resume(lib):
    """C3: convolving [0, m) and then [m, L) with the last width-1 inputs
    before m as the preceding window gives the one-pass result."""
    rng = np.random.default_rng(33)
    x, w, b, xp = _rand_conv(rng, L=40, K=4)
    whole = oracle.conv_silu(x, w, b, xp, lib=lib)
    m = 13
    first = oracle.conv_silu(x[..., :m], w, b, xp, lib=lib)
    second = oracle.conv_silu(x[..., m:], w, b, x[..., m - 3:m], lib=lib)
    _close(np.concatenate([first, second], axis=-1), whole, what="conv split/resume")


def pin_conv_feeds_scan(lib):
    """C4: the convolution stage runs before the scan and its output is the u
    of both the input term and the skip term: scan_fwd_conv equals the scan
    fed with the np.convolve reference of the stage."""
    rng = np.random.default_rng(34)
    inp = _rand_scan(rng, L=26)
    x, w, b, xp = _rand_conv(rng, batch=2, dim=3, L=26, K=4)
    y, h = oracle.scan_fwd_conv(x, w, b, xp, inp["delta"], inp["A"], inp["B"], inp["C"],
                                inp["D"], inp["z"], inp["delta_bias"], True, inp["h0"], lib=lib)
    u = _conv_numpy(x, w, b, xp)
    yr, hr = oracle.scan_fwd(u, inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"], inp["z"],
                             inp["delta_bias"], True, inp["h0"], lib=lib)
    _close(y, yr, what="conv feeding the scan: y")
    _close(h, hr, what="conv feeding the scan: h_L")


# ---- gradients (reverse mode) -----------------------------------------------------


def pin_backward_finite_differences(lib):
    """G1: every gradient of the backward oracle equals the central finite
    difference of sum(y * dy) computed with the (separately pinned) forward
    oracle, on sampled entries of every input, with and without softplus."""
    rng = np.random.default_rng(41)
    for softplus in (True, False):
        inp = _rand_scan(rng, batch=2, dim=3, N=4, L=9)
        if not softplus:  # keep dt' = delta + bias positive and moderate
            inp["delta"] = np.abs(inp["delta"]) * 0.3
            inp["delta_bias"] = np.full(3, 0.05)
        dy = rng.standard_normal(inp["u"].shape)
        names = ["u", "delta", "A", "B", "C", "D", "z", "delta_bias", "h0"]

        def loss(vals):
            y, _ = oracle.scan_fwd(vals["u"], vals["delta"], vals["A"], vals["B"], vals["C"],
                                   vals["D"], vals["z"], vals["delta_bias"], softplus, vals["h0"],
                                   lib=lib)
            return float(np.sum(y * dy))

        g = oracle.scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy, inp["D"],
                            inp["z"], inp["delta_bias"], softplus, inp["h0"], lib=lib)
        key = {"u": "du", "delta": "ddelta", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
               "z": "dz", "delta_bias": "ddelta_bias", "h0": "dh0"}
        for name in names:
            grad = g[key[name]]
            flat = inp[name].reshape(-1)
            for idx in rng.choice(flat.size, size=min(6, flat.size), replace=False):
                eps = 1e-5 * max(1.0, abs(flat[idx]))
                plus = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
                minus = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
                plus[name].reshape(-1)[idx] += eps
                minus[name].reshape(-1)[idx] -= eps
                fd = (loss(plus) - loss(minus)) / (2 * eps)
                scale = max(1.0, float(np.max(np.abs(grad))))
                assert abs(grad.reshape(-1)[idx] - fd) <= 1e-6 * scale, \
                    (name, int(idx), float(grad.reshape(-1)[idx]), fd, softplus)


MAMBA1_PINS = [pin_closed_form, pin_augmented_matrix, pin_blelloch_order, pin_lti_convolution,
               pin_split_resume, pin_prefix_sum_case, pin_memoryless_case, pin_gate_and_skip,
               pin_softplus_and_bias, pin_decode_steps]
SSD_PINS = [pin_ssd_is_mamba1, pin_ssd_quadratic, pin_ssd_chunked]
CONV_PINS = [pin_conv_numpy, pin_conv_one_tap, pin_conv_split_resume, pin_conv_feeds_scan]
BWD_PINS = [pin_backward_finite_differences]
ALL_PINS = MAMBA1_PINS + SSD_PINS + CONV_PINS + BWD_PINS
