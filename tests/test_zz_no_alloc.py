"""The allocation-free decode entry point against the regular one.

Some callers cannot allocate device memory (a runtime that fixes its memory
budget at start-up and forbids cudaMalloc afterwards, or a host that gives the
library no allocator).  tq_decode_attention_noalloc serves them from a fixed
scratch array inside the library.  This test calls it through the C ABI,
twice in a row with different shapes (the second call must not be disturbed
by what the first left in the shared scratch), and compares each result with
tq_decode_attention on a caller-provided workspace.  It sits in a file that
pytest collects last and passes both alone and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import synth
from helpers import ATOL, RTOL, assert_close

pytestmark = pytest.mark.gpu
D = 128


def _bind():
    from vector_quantization_b200 import tq
    fn = tq._lib.tq_decode_attention_noalloc
    c_i, c_i64, c_p, c_f = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p, ctypes.c_float
    fn.restype = c_i
    fn.argtypes = [c_p, c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_i, c_i, c_i, c_i64, c_p, c_f, c_p, c_p]
    return tq, fn


def _case(tq, G, T, B, Hkv, seed, dev):
    rk = tq.Rotation(D, 2, synth.rotation_randomness(D, seed), rope_base=10000.0, rope_max_pos=T + 8)
    rv = tq.Rotation(D, 2, synth.rotation_randomness(D, seed + 1))
    k = torch.from_numpy(synth.heavy_tailed((B, Hkv, T, D), seed + 2)).to(dev)
    v = torch.from_numpy(synth.heavy_tailed((B, Hkv, T, D), seed + 3)).to(dev)
    kc = tq.quantize_kv(rk, k, apply_rope=True, pos_period=T)
    vc = tq.quantize_kv(rv, v)
    q = torch.from_numpy(synth.heavy_tailed((B, Hkv * G, D), seed + 4)).to(dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    return rk, rv, kc, vc, q, qpos


def _noalloc(fn, rk, rv, kc, vc, q, qpos, T, out):
    B, Hq, _ = q.shape
    Hkv, cap = kc[0].shape[1], kc[0].shape[2]
    st = fn(rk.handle, rv.handle, q.data_ptr(), 0, qpos.data_ptr(), kc[0].data_ptr(), kc[1].data_ptr(),
            kc[2].data_ptr(), vc[0].data_ptr(), vc[1].data_ptr(), vc[2].data_ptr(), cap, B, Hq, Hkv, T, None,
            1.0 / np.sqrt(D), out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    return st


def test_noalloc_matches_regular_entry_point_twice(cuda_device):
    tq, fn = _bind()
    dev = cuda_device
    cases = [dict(G=4, T=3000, B=2, Hkv=2, seed=71), dict(G=1, T=334, B=1, Hkv=3, seed=81)]
    for c in cases:
        rk, rv, kc, vc, q, qpos = _case(tq, c["G"], c["T"], c["B"], c["Hkv"], c["seed"], dev)
        ref = tq.decode_attention(rk, rv, q, qpos, kc, vc, c["T"])
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(fn, rk, rv, kc, vc, q, qpos, c["T"], out) == tq.TQ_OK
        torch.cuda.synchronize()
        assert torch.isfinite(out).all()
        assert_close(out.cpu().numpy(), ref.cpu().numpy(), ATOL, RTOL, what=f"noalloc {c}")


def test_noalloc_rejects_requests_beyond_its_scratch(cuda_device):
    tq, fn = _bind()
    dev = cuda_device
    rk, rv, kc, vc, q, qpos = _case(tq, 4, 64, 1, 1, 91, dev)
    # 4096 sequences of 2^20 tokens need far more than the fixed scratch.
    # The cache and output pointers are NULL: the size check must answer
    # first, and were it ever to move behind the pointer checks the call would
    # still return an error (TQ_EINVAL) instead of launching over buffers far
    # smaller than the sizes claimed.
    B, Hkv, T = 512, 8, 1 << 20
    assert tq.decode_workspace_size(rk, rv, B, 4 * Hkv, Hkv, T) > (16 << 20)
    st = fn(rk.handle, rv.handle, q.data_ptr(), 0, qpos.data_ptr(), None, None, None, None, None, None,
            T, B, 4 * Hkv, Hkv, T, None, 0.088, None, torch.cuda.current_stream().cuda_stream)
    assert st == tq.TQ_EWORKSPACE
