"""Seeded synthetic inputs for the selective scan and the scalar-decay scan.

This module only draws random numbers and rounds them to the storage type.
It holds none of the scan's arithmetic, so both the CPU oracle and the CUDA
path can take their inputs from here.

Distributions (the workload descriptions this library is measured on):

* u, z, B, C ~ N(0, 1); delta ~ N(0, 1);
* A[d, n] = -exp(U(ln 1, ln 10)) -- a log-uniform decay rate in [1, 10]
  (the S4D/Mamba initialisation range named on the page "Mamba ... 硬件感知
  ... 并行扫描", section 3.1);
* bias_d such that softplus(bias_d) is log-uniform in [s_lo, s_hi]
  ([1e-3, 1e-1] by default, [1e-4, 1e-2] for the long-sequence workload);
  bias_d = log(expm1(s_d)) is the inverse of softplus;
* D_d ~ N(0, 1);
* Mamba-2 heads: A_h = -exp(U(ln 1, ln 16)).

Tensor rows come in blocks of 64, each block from its own stream
``default_rng([seed, tensor_id, block])``, so any subset of rows can be
regenerated on its own: the oracle can be run on sampled channels of a
workload too large for it, and the blocks are generated in parallel threads.  bf16 tensors are rounded to nearest-even
from the float32 draw; both sides receive exactly those values.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# Tensor ids of the per-row streams.
T_A, T_D, T_BIAS, T_U, T_DELTA, T_Z, T_B, T_C, T_X, T_H0 = range(10)

# The workloads: the first is small enough for the oracle to finish in well
# under a second; the others are the shapes of one Mamba layer of the
# 130M and 2.8B models, a genomics-length sequence and a Mamba-2 layer.
CONFIGS = {
    "tiny_fp32": dict(kind="scan", batch=1, dim=64, dstate=16, seqlen=256, dtype="f32",
                      gate=True, s_range=(1e-3, 1e-1), seed=0),
    "mamba130m_layer": dict(kind="scan", batch=8, dim=1536, dstate=16, seqlen=2048, dtype="bf16",
                            gate=True, s_range=(1e-3, 1e-1), seed=1),
    "mamba2p8b_layer": dict(kind="scan", batch=4, dim=5120, dstate=16, seqlen=4096, dtype="bf16",
                            gate=True, s_range=(1e-3, 1e-1), seed=2),
    "long_seq": dict(kind="scan", batch=1, dim=1024, dstate=16, seqlen=1 << 20, dtype="bf16",
                     gate=True, s_range=(1e-4, 1e-2), seed=3),
    "mamba2_ssd": dict(kind="ssd", batch=2, seqlen=4096, nheads=80, headdim=64, dstate=128,
                       chunk=256, dtype="bf16", gate=False, s_range=(1e-3, 1e-1), seed=4),
}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return the bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """float32 values representable in ``dtype`` ("f32" or "bf16")."""
    x = np.asarray(x, dtype=np.float32)
    return bf16_bits_to_f32(to_bf16_bits(x)).reshape(x.shape) if dtype == "bf16" else x


def _stream(seed: int, tensor: int, row: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tensor), int(row)])


ROWS_PER_STREAM = 64


def normal_rows(seed: int, tensor: int, rows, length: int, dtype: str = "f32",
                threads: int | None = None, bits: bool = False) -> np.ndarray:
    """N(0,1) rows ``rows`` (iterable of ints) of one tensor, each ``length`` long,
    rounded to ``dtype``; returned as float32 of shape (len(rows), length), or,
    with ``bits`` and dtype "bf16", as the uint16 bfloat16 bit patterns.

    Row r is row r % 64 of the (64, length) block drawn from the stream
    ``default_rng([seed, tensor, r // 64])``, so a row's values do not depend
    on which other rows are requested."""
    rows = [int(r) for r in rows]
    as_bits = bits and dtype == "bf16"
    out = np.empty((len(rows), length), dtype=np.uint16 if as_bits else np.float32)
    blocks: dict[int, list[tuple[int, int]]] = {}
    for i, r in enumerate(rows):
        blocks.setdefault(r // ROWS_PER_STREAM, []).append((i, r % ROWS_PER_STREAM))

    def fill(item):
        blk, members = item
        need = max(m for _, m in members) + 1
        v = _stream(seed, tensor, blk).standard_normal((ROWS_PER_STREAM, length),
                                                        dtype=np.float32)[:need]
        v = to_bf16_bits(v).reshape(v.shape) if as_bits else round_to(v, dtype)
        for i, m in members:
            out[i] = v[m]

    items = list(blocks.items())
    n = threads or min(32, os.cpu_count() or 1)
    if len(items) == 1 or n == 1 or len(rows) * length < (1 << 20):
        for it in items:
            fill(it)
    else:
        with ThreadPoolExecutor(n) as ex:
            list(ex.map(fill, items))
    return out


def log_uniform(rng: np.random.Generator, lo: float, hi: float, size) -> np.ndarray:
    return np.exp(rng.uniform(np.log(lo), np.log(hi), size))


def scan_params(seed: int, dim: int, dstate: int, s_range=(1e-3, 1e-1)):
    """A (dim, dstate), D (dim), delta_bias (dim) as float32."""
    A = -log_uniform(_stream(seed, T_A), 1.0, 10.0, (dim, dstate)).astype(np.float32)
    D = _stream(seed, T_D).standard_normal(dim).astype(np.float32)
    s = log_uniform(_stream(seed, T_BIAS), s_range[0], s_range[1], dim)
    bias = np.log(np.expm1(s)).astype(np.float32)  # inverse of softplus
    return A, D, bias


def make_scan_inputs(batch: int, dim: int, dstate: int, seqlen: int, dtype: str = "f32",
                     gate: bool = True, seed: int = 0, s_range=(1e-3, 1e-1),
                     channels=None, h0: bool = False, bits: bool = False) -> dict:
    """Inputs of one selective scan, as float32 arrays holding values exactly
    representable in ``dtype``.

    Layouts: u, delta, z (batch, dim, seqlen); B, C (batch, dstate, seqlen);
    A (dim, dstate); D, delta_bias (dim); h0 (batch, dim, dstate).

    ``channels`` (a list of (b, d) pairs) restricts u/delta/z/h0 to those
    rows, returned with shape (1, len(channels), seqlen), together with the
    matching A/D/bias rows; B and C are then those of the batch of the
    channels, which must all share one b.  With ``bits`` and dtype "bf16" the
    sequence tensors come back as uint16 bfloat16 bit patterns.
    """
    A, D, bias = scan_params(seed, dim, dstate, s_range)
    if channels is None:
        rows = range(batch * dim)
        bsel = list(range(batch))
        dsel = np.arange(dim)
        shape = (batch, dim, seqlen)
    else:
        channels = [(int(b), int(d)) for b, d in channels]
        bs = {b for b, _ in channels}
        if len(bs) != 1:
            raise ValueError("sampled channels must share one batch index")
        rows = [b * dim + d for b, d in channels]
        bsel = [channels[0][0]]
        dsel = np.array([d for _, d in channels])
        shape = (1, len(channels), seqlen)
    out = {
        "A": np.ascontiguousarray(A[dsel]), "D": np.ascontiguousarray(D[dsel]),
        "delta_bias": np.ascontiguousarray(bias[dsel]),
        "u": normal_rows(seed, T_U, rows, seqlen, dtype, bits=bits).reshape(shape),
        "delta": normal_rows(seed, T_DELTA, rows, seqlen, dtype, bits=bits).reshape(shape),
        "z": (normal_rows(seed, T_Z, rows, seqlen, dtype, bits=bits).reshape(shape)
              if gate else None),
    }
    bc_rows = [b * dstate + n for b in bsel for n in range(dstate)]
    out["B"] = normal_rows(seed, T_B, bc_rows, seqlen, dtype, bits=bits).reshape(
        len(bsel), dstate, seqlen)
    out["C"] = normal_rows(seed, T_C, bc_rows, seqlen, dtype, bits=bits).reshape(
        len(bsel), dstate, seqlen)
    out["h0"] = (normal_rows(seed, T_H0, rows, dstate, "f32").reshape(shape[0], shape[1], dstate)
                 if h0 else None)
    return out


def make_grouped_bc(batch: int, ngroups: int, dstate: int, seqlen: int, dtype: str = "bf16",
                    seed: int = 5) -> dict:
    """Grouped B and C, (batch, ngroups, dstate, seqlen) ~ N(0, 1), rounded to
    ``dtype`` (float32 arrays)."""
    rng = np.random.default_rng([seed, 11, ngroups])
    shape = (batch, ngroups, dstate, seqlen)
    return {"B": round_to(rng.standard_normal(shape).astype(np.float32), dtype),
            "C": round_to(rng.standard_normal(shape).astype(np.float32), dtype)}


def make_conv_params(dim: int, width: int = 4, seed: int = 9, batch: int | None = None,
                     prev: bool = False) -> dict:
    """Parameters of the convolution stage in front of the scan (float32):
    weight (dim, width) ~ N(0, 1/width), bias (dim) ~ N(0, 0.1^2) and, with
    ``prev``, a preceding window x_prev (batch, dim, width - 1) ~ N(0, 1)."""
    rng = np.random.default_rng([seed, 7, width])
    out = {"weight": (rng.standard_normal((dim, width)) / np.sqrt(width)).astype(np.float32),
           "bias": (0.1 * rng.standard_normal(dim)).astype(np.float32), "x_prev": None}
    if prev:
        out["x_prev"] = rng.standard_normal((batch, dim, width - 1)).astype(np.float32)
    return out


def make_ssd_inputs(batch: int, seqlen: int, nheads: int, headdim: int, dstate: int,
                    dtype: str = "bf16", gate: bool = False, seed: int = 4,
                    s_range=(1e-3, 1e-1), h0: bool = False) -> dict:
    """Inputs of one Mamba-2 scalar-decay scan (float32 arrays).

    Layouts: x, z (batch, seqlen, nheads, headdim); delta (batch, seqlen, nheads);
    B, C (batch, seqlen, dstate); A, D, delta_bias (nheads);
    h0 (batch, nheads, headdim, dstate).
    """
    A = -log_uniform(_stream(seed, T_A), 1.0, 16.0, nheads).astype(np.float32)
    D = _stream(seed, T_D).standard_normal(nheads).astype(np.float32)
    s = log_uniform(_stream(seed, T_BIAS), s_range[0], s_range[1], nheads)
    bias = np.log(np.expm1(s)).astype(np.float32)
    x = normal_rows(seed, T_X, range(batch), seqlen * nheads * headdim, dtype)
    dl = normal_rows(seed, T_DELTA, range(batch), seqlen * nheads, dtype)
    Bm = normal_rows(seed, T_B, range(batch), seqlen * dstate, dtype)
    Cm = normal_rows(seed, T_C, range(batch), seqlen * dstate, dtype)
    z = normal_rows(seed, T_Z, range(batch), seqlen * nheads * headdim, dtype) if gate else None
    out = {
        "A": A, "D": D, "delta_bias": bias,
        "x": x.reshape(batch, seqlen, nheads, headdim),
        "delta": dl.reshape(batch, seqlen, nheads),
        "B": Bm.reshape(batch, seqlen, dstate), "C": Cm.reshape(batch, seqlen, dstate),
        "z": z.reshape(batch, seqlen, nheads, headdim) if gate else None,
        "h0": (normal_rows(seed, T_H0, range(batch * nheads), headdim * dstate, "f32")
               .reshape(batch, nheads, headdim, dstate) if h0 else None),
    }
    return out
