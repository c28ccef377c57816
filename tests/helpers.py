"""Shared helpers of the parity tests: oracle-built caches and comparisons."""
from __future__ import annotations

import numpy as np

import synth
from oracle import codec, rotation as ro

# Tolerance of scores and attention outputs (fp32 accumulation against the
# float64 oracle): |gpu - ref| <= ATOL + RTOL |ref| elementwise.
ATOL, RTOL = 1e-3, 2e-3


def assert_close(gpu, ref, atol=ATOL, rtol=RTOL, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    bad = np.abs(gpu - ref) > atol + rtol * np.abs(ref)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]!r} ref={ref[tuple(i)]!r}")


def oracle_rotation(d, bits, seed, rope=0.0, kind="hadamard"):
    rnd = synth.rotation_randomness(d, seed, dense=(kind == "dense"))
    return ro.build_rotation(d, bits, rnd, kind, rope_base=rope), rnd


def oracle_records(rot, x, pos=None):
    """Encode rows of x with the oracle; returns (codes, signs, norms, enc)."""
    e = codec.encode(rot, np.asarray(x, dtype=np.float64).reshape(-1, rot.d), pos)
    codes = codec.pack_planes(e["codes"], rot.bits)
    signs = codec.pack_bits(e["signs"])
    norms = np.stack([e["norm"], e["rnorm"]], axis=1).astype(np.float32)
    return codes, signs, norms, e


def compare_records(rot, gpu, enc, x_norm_scale=None):
    """Parity of GPU records (codes, signs, norms as numpy) with an oracle encode.

    Codes: identical except on coordinates the oracle flags (within 1e-5 of a
    threshold).  Signs: compared on vectors whose codes all match, except
    flagged bits.  Norms: ||x|| to 1e-6 relative; ||r|| to 1e-6 relative plus
    2e-6 ||x|| absolute (fp32 rotation error ~1e-7 per unit coordinate, summed
    over d coordinates of the residual), on vectors whose codes all match.
    Returns a dict of counts for reporting."""
    gc, gs, gn = gpu
    n = enc["codes"].shape[0]
    g_codes = codec.unpack_planes(gc.reshape(n, -1), rot.bits, rot.d)
    g_signs = codec.unpack_bits(gs.reshape(n, -1), rot.m)
    g_norms = np.asarray(gn, dtype=np.float64).reshape(n, 2)
    diff = g_codes != enc["codes"]
    unflagged = diff & ~enc["code_flags"]
    assert not unflagged.any(), f"{unflagged.sum()} unflagged code mismatches (first {np.argwhere(unflagged)[0]})"
    same = ~diff.any(axis=1)
    sdiff = (g_signs != enc["signs"]) & ~enc["sign_flags"] & same[:, None]
    assert not sdiff.any(), f"{sdiff.sum()} unflagged sign mismatches (first {np.argwhere(sdiff)[0]})"
    nx = enc["norm"]
    np.testing.assert_allclose(g_norms[:, 0], nx, rtol=1e-6, atol=1e-30)
    nr = enc["rnorm"][same]
    assert np.all(np.abs(g_norms[same, 1] - nr) <= 1e-6 * nr + 2e-6 * nx[same])
    return {"code_mismatch_flagged": int(diff.sum()), "flagged": int(enc["code_flags"].sum()),
            "vectors_all_codes_equal": int(same.sum())}


def _oracle_slice(rot_o, x, pos=None):
    """The oracle's own records of one (sequence, KV head) slice x [T, d] of
    the synthetic input, as [1, 1, T, ...] arrays."""
    codes, signs, norms, enc = oracle_records(rot_o, x, pos)
    T = x.shape[0]
    return tuple(a.reshape(1, 1, T, -1) for a in (codes, signs, norms)), enc


def check_and_substitute(rot_o, cache, b, j, x, pos=None):
    """GPU encode parity of the first T = len(x) records of slice (b, j) of a
    device cache [B, H, cap, ...] (codes equal except boundary-flagged
    coordinates), then those records are overwritten with the oracle's own
    encoding of x, so that an attention launch over the cache and the oracle
    read the same bytes without the oracle reading anything the GPU wrote.
    Returns the oracle records as [1, 1, T, ...] arrays."""
    rec, enc = _oracle_slice(rot_o, x, pos)
    T = x.shape[0]
    compare_records(rot_o, tuple(a[b, j, :T].cpu().numpy().reshape(T, -1) for a in cache), enc)
    import torch
    for a, r in zip(cache, rec):
        a[b, j, :T] = torch.from_numpy(np.ascontiguousarray(r[0, 0])).to(a.device)
    return rec
