"""Seeded synthetic inputs for the LongSpark drafting round (host side).

This module only draws numbers: it holds none of the method's arithmetic. Both the CPU
oracle (through the tests) and the CUDA library (through the tests and the bench) are fed
from it. Large tensors are drawn on the GPU by ``synth/synth.cu``, which implements the
same definition; the two are compared bit for bit by a GPU test.

Generator: SplitMix64 (G. L. Steele, D. Lea, C. H. Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), used counter-based: ``draw(key, n)`` is output number n
(0-based) of the SplitMix64 stream whose state starts at ``key``, i.e. the finaliser
applied to ``key + (n + 1) * gamma`` (mod 2^64). A tensor's stream key is
``draw(seed, tensor_id)``; its element at logical coordinates (r, b, l, p, h, d) uses the
counter ``r<<52 | b<<44 | l<<38 | p<<16 | h<<9 | d`` (hidden vectors put their index x in
the low 16 bits, i.e. h = x >> 9, d = x & 511).

Values called "~N(0,1)" are an Irwin-Hall stand-in: the sum of the four 16-bit fields of
one draw, centred (minus 131070, exact in fp32) and multiplied by the fp32 constant
``INV_STD`` = 1/sqrt((65536^2 - 1)/3) (unit variance), optionally times an fp32 per-head
scale, each product rounded to nearest even in fp32; bf16 tensors then round that fp32
value to nearest even. Tails are bounded at +-3.46 sigma.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
INV_STD = np.float32(1.0 / np.sqrt((65536.0 ** 2 - 1.0) / 3.0))
CENTRE = 131070

# tensor ids (part of each stream key)
PREFIX_K, PREFIX_V, VERIFY_K, VERIFY_V, VERIFY_HIDDEN, QUERY, LAST_HIDDEN = 1, 2, 3, 4, 5, 6, 7
HEAD_SCALE, DRAFT, TARGET, ACCEPT, PREFIX_LEN, MISMATCH = 8, 9, 10, 11, 12, 13

SH_R, SH_B, SH_L, SH_P, SH_H = 52, 44, 38, 16, 9


def _finalise(z):
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def draw(key, n):
    """Output number ``n`` of the SplitMix64 stream starting at ``key`` (vectorised)."""
    key = np.uint64(key)
    n = np.asarray(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _finalise(key + (n + np.uint64(1)) * GAMMA)


def stream_key(seed: int, tensor_id: int) -> int:
    return int(draw(np.uint64(seed), tensor_id))


def pack(r=0, b=0, l=0, p=0, h=0, d=0):
    """Counter of the element at logical coordinates (arrays broadcast)."""
    u = lambda x, s: np.asarray(x, dtype=np.uint64) << np.uint64(s)  # noqa: E731
    return u(r, SH_R) | u(b, SH_B) | u(l, SH_L) | u(p, SH_P) | u(h, SH_H) | np.asarray(d, dtype=np.uint64)


def normal_f32(bits, scale=None):
    """fp32 value of the Irwin-Hall stand-in for N(0,1) from 64-bit draws."""
    m = np.uint64(0xFFFF)
    s = (bits & m) + ((bits >> np.uint64(16)) & m) + ((bits >> np.uint64(32)) & m) + (bits >> np.uint64(48))
    z = (s.astype(np.int64) - CENTRE).astype(np.float32) * INV_STD
    if scale is not None:
        z = z * np.asarray(scale, dtype=np.float32)
    return z.astype(np.float32)


def f32_to_bf16_bits(x):
    """Round fp32 to bf16, nearest even, returned as uint16 bit patterns (finite input)."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return u.astype(np.uint16)


def fill_normal(seed, tensor_id, shape, r0=0, b0=0, l0=0, p0=0, x0=0, head_dim=0,
                scale=None, dtype="bf16"):
    """Block of a tensor with logical dims (r, b, l, p, x), ``shape`` = (nr, nb, nl, np, nx).

    The block starts at coordinates (r0, b0, l0, p0, x0). With ``head_dim`` > 0 the
    innermost index x is split into (h, d) = (x // head_dim, x % head_dim) (K/V/q rows);
    with 0 it is a hidden index. ``scale`` is an fp32 [L][Hkv] per-head multiplier
    (K/V only). Returns uint16 bf16 bits or float32, shaped ``shape``.
    """
    nr, nb, nl, npos, nx = shape
    r = (np.arange(nr, dtype=np.uint64) + np.uint64(r0)).reshape(nr, 1, 1, 1, 1)
    b = (np.arange(nb, dtype=np.uint64) + np.uint64(b0)).reshape(1, nb, 1, 1, 1)
    l = (np.arange(nl, dtype=np.uint64) + np.uint64(l0)).reshape(1, 1, nl, 1, 1)
    p = (np.arange(npos, dtype=np.uint64) + np.uint64(p0)).reshape(1, 1, 1, npos, 1)
    x = np.arange(nx, dtype=np.int64) + int(x0)
    if head_dim > 0:
        h, d = x // head_dim, x % head_dim
    else:
        h, d = x >> 9, x & 511
    ctr = pack(r, b, l, p, h.reshape(1, 1, 1, 1, nx), d.reshape(1, 1, 1, 1, nx))
    bits = draw(stream_key(seed, tensor_id), ctr)
    sc = None
    if scale is not None:
        scale = np.asarray(scale, dtype=np.float32)
        ll = np.arange(nl) + l0
        sc = scale[ll][:, h].reshape(1, 1, nl, 1, nx)
    z = normal_f32(bits, sc)
    return f32_to_bf16_bits(z) if dtype == "bf16" else z


def head_scales(seed, n_layers, n_kv_heads, lo=0.5, hi=2.0):
    """fp32 [L][Hkv] per-head scales ~U(lo, hi): 24-bit uniform, fp32 multiply-add."""
    ctr = pack(l=np.arange(n_layers).reshape(-1, 1), h=np.arange(n_kv_heads).reshape(1, -1))
    u = (draw(stream_key(seed, HEAD_SCALE), ctr) >> np.uint64(40)).astype(np.float32) * np.float32(2.0 ** -24)
    return (np.float32(lo) + u * np.float32(hi - lo)).astype(np.float32)


def uniform53(seed, tensor_id, ctr):
    return (draw(stream_key(seed, tensor_id), ctr) >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def truncated_geometric_p(mean, block):
    """p with E[a] = mean for P(a = k) proportional to p (1 - p)^k on k = 0..block."""
    def m(p):
        k = np.arange(block + 1)
        w = p * (1 - p) ** k
        return float((k * w).sum() / w.sum())
    lo, hi = 1e-9, 1 - 1e-9
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if m(mid) > mean:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


def accept_lengths(seed, n_rounds, batch, block, mean=None):
    """int32 [rounds][batch] accepted-draft counts a in 0..block.

    ``mean=None`` draws a uniformly from {0..block}; otherwise truncated-geometric with
    that mean, sampled by inverse CDF from a 53-bit uniform.
    """
    ctr = pack(r=np.arange(n_rounds).reshape(-1, 1), b=np.arange(batch).reshape(1, -1))
    u = uniform53(seed, ACCEPT, ctr)
    if mean is None:
        return np.minimum((u * (block + 1)).astype(np.int64), block).astype(np.int32)
    p = truncated_geometric_p(mean, block)
    w = p * (1 - p) ** np.arange(block + 1)
    cdf = np.cumsum(w / w.sum())
    cdf[-1] = 1.0
    return np.searchsorted(cdf, u, side="right").clip(0, block).astype(np.int32)


def token_ids(seed, n_rounds, batch, block, accept, vocab):
    """Draft ids int32 [rounds][batch][B] and target ids int32 [rounds][batch][B+1].

    The target repeats the draft for i < a, differs from it at i = a (when a < B) and
    is random elsewhere, so the greedy scan of that pair accepts exactly a drafts.
    """
    r = np.arange(n_rounds).reshape(-1, 1, 1)
    b = np.arange(batch).reshape(1, -1, 1)
    i = np.arange(block + 1).reshape(1, 1, -1)
    draft = (draw(stream_key(seed, DRAFT), pack(r=r, b=b, p=i[..., :block])) % np.uint64(vocab)).astype(np.int64)
    target = (draw(stream_key(seed, TARGET), pack(r=r, b=b, p=i)) % np.uint64(vocab)).astype(np.int64)
    off = (draw(stream_key(seed, MISMATCH), pack(r=r, b=b)) % np.uint64(vocab - 1)).astype(np.int64)
    a = np.asarray(accept).reshape(n_rounds, batch, 1)
    d_pad = np.concatenate([draft, np.zeros((n_rounds, batch, 1), np.int64)], axis=2)
    target = np.where(i < a, d_pad, target)
    mism = (d_pad + 1 + off) % vocab
    target = np.where((i == a) & (a < block), mism, target)
    return draft.astype(np.int32), target.astype(np.int32)


def prefix_lengths(seed, batch, lo, hi):
    """int64 [batch] prefix lengths uniform on {lo..hi}."""
    u = uniform53(seed, PREFIX_LEN, pack(b=np.arange(batch)))
    return (lo + np.minimum((u * (hi - lo + 1)).astype(np.int64), hi - lo)).astype(np.int64)


# ----------------------------------------------------------------------------------
# device twin (synth/synth.cu) — the same draws, written straight into GPU memory
# ----------------------------------------------------------------------------------
_LIB = None


def device_lib():
    """ctypes handle of synth/libls_synth.so (built by the package build step)."""
    global _LIB
    if _LIB is None:
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libls_synth.so")
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        lib.lss_fill_normal.restype = ctypes.c_int
        lib.lss_fill_normal.argtypes = [
            ctypes.c_void_p, ctypes.c_int, ctypes.c_uint64,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int32, ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p]
        _LIB = lib
    return _LIB


def device_fill_normal(out_ptr, seed, tensor_id, shape, r0=0, b0=0, l0=0, p0=0, head_dim=0,
                       scale_ptr=None, scale_heads=0, dtype="bf16", stream=0, x0=0, scale_layers=None):
    """Same values as :func:`fill_normal` written to device memory.

    ``out_ptr`` is a device pointer to a contiguous (nr, nb, nl, np, nx) array;
    ``scale_ptr`` a device fp32 [L][scale_heads] array or None.
    """
    nr, nb, nl, npos, nx = shape
    if scale_ptr:
        # the kernel reads scale[l][h] for l < l0 + nl and h < (x0 + nx) / head_dim: the
        # [L][scale_heads] array the caller passes must cover them
        if head_dim <= 0 or (x0 + nx + head_dim - 1) // head_dim > scale_heads:
            raise ValueError("per-head scales need head_dim > 0 and columns within scale_heads heads")
        if scale_layers is not None and l0 + nl > scale_layers:
            raise ValueError(f"layers {l0}..{l0 + nl - 1} past the {scale_layers}-layer scale array")
    rc = device_lib().lss_fill_normal(
        ctypes.c_void_p(out_ptr), 1 if dtype == "bf16" else 0,
        ctypes.c_uint64(stream_key(seed, tensor_id)),
        nr, nb, nl, npos, nx, r0, b0, l0, p0, x0, head_dim,
        ctypes.c_void_p(scale_ptr or 0), scale_heads, float(INV_STD), ctypes.c_void_p(stream))
    if rc != 0:
        raise RuntimeError(f"lss_fill_normal failed with {rc}")
