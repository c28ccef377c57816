"""GPU parity of the sign-residual record mode ([TurboESM] §2.D: the residual
kept as one sign bit per rotated coordinate plus the mean magnitude e, and
x~ = Pi^T (||x|| c[idx] + e (2z - 1))) against the oracle's own encode
(codec.encode_sign_residual) and its dequantized attention.

A handle built with residual = TQ_RES_SIGN holds S = I and the estimator
constant 1, so every kernel of the codec runs unchanged on it; the encoders
store e = ||r||_1 / d in place of ||r||.  Records are compared as for the QJL
mode (codes identical except flagged coordinates; sign bits on vectors whose
codes all match, except where |r_i| < 1e-5 ||r||; e within 1e-6 e + 3e-7 ||x||:
each |r_i| moves by at most ||x|| times the rotation's error of about 1.5e-7
per unit coordinate).  Attention is compared with the oracle's textbook
softmax attention over the dequantized keys and values, within
1e-3 + 2e-3 |ref|."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_close
from oracle import attention as at
from oracle import codec
from oracle import rotation as ro
from oracle import search as osearch

pytestmark = pytest.mark.gpu


def _rots(d, bits, seed, rope=0.0, kind="hadamard"):
    from vector_quantization_b200 import tq
    rnd = synth.rotation_randomness(d, seed, dense=(kind == "dense"))
    g = tq.Rotation(d, bits, rnd, kind, rope_base=rope, rope_max_pos=(1 << 20) + 8, residual="sign")
    o = ro.build_rotation(d, bits, rnd, kind, rope_base=rope)
    return g, o


def _check_records(o, gpu, x, pos=None):
    gc, gs, gn = (np.asarray(a) for a in gpu)
    n = x.shape[0]
    e = codec.encode_sign_residual(o, x, pos)
    base = codec.encode(o, x, pos)
    g_codes = codec.unpack_planes(gc.reshape(n, -1), o.bits, o.d)
    g_signs = codec.unpack_bits(gs.reshape(n, -1), o.d)
    diff = g_codes != e["codes"]
    assert not (diff & ~base["code_flags"]).any()
    same = ~diff.any(axis=1)
    rn = np.sqrt(np.sum(e["r"] ** 2, axis=1))
    flag = np.abs(e["r"]) < 1e-5 * rn[:, None]
    assert not ((g_signs != e["signs"]) & ~flag & same[:, None]).any()
    gn = gn.reshape(n, 2).astype(np.float64)
    np.testing.assert_allclose(gn[:, 0], e["norm"], rtol=1e-6, atol=1e-30)
    assert np.all(np.abs(gn[same, 1] - e["ebar"][same]) <= 1e-6 * e["ebar"][same] + 3e-7 * e["norm"][same])
    return e


@pytest.mark.parametrize("d,n", [(128, 200), (128, 3000), (128, 17000), (64, 3000), (64, 17000)])
def test_sign_mode_encode_parity(cuda_device, d, n):
    """All encode kernels (block per vector, warp per vector, and the 128-row
    tile kernels) in sign mode, keys with RoPE."""
    from vector_quantization_b200 import tq
    g, o = _rots(d, 2, 401 + d, rope=10000.0)
    x = synth.heavy_tailed((n, d), 402)
    pos = (np.arange(n) % 4096).astype(np.int64)
    gpu = tq.quantize_kv(g, torch.from_numpy(x).to(cuda_device).to(torch.bfloat16), apply_rope=True,
                         pos_period=4096)
    torch.cuda.synchronize()
    xb = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    _check_records(o, tuple(a.cpu().numpy() for a in gpu), xb, pos)


@pytest.mark.parametrize("d,bits,dtype", [(128, 2, torch.bfloat16), (128, 3, torch.float32), (64, 1, torch.bfloat16),
                                           (64, 2, torch.float32)])
def test_sign_mode_encode_parity_no_rope(cuda_device, d, bits, dtype):
    """The 128-row tile kernels in sign mode without RoPE (the value
    launches: a bf16 input enters the rotation product as one operand, fp32
    as a hi + lo pair), 17000 rows: 132 full tiles and a ragged one."""
    from vector_quantization_b200 import tq
    g, o = _rots(d, bits, 407 + d + bits)
    x = synth.heavy_tailed((17000, d), 408 + bits)
    xt = torch.from_numpy(x).to(cuda_device).to(dtype)
    gpu = tq.quantize_kv(g, xt)
    torch.cuda.synchronize()
    _check_records(o, tuple(a.cpu().numpy() for a in gpu), xt.float().cpu().numpy().astype(np.float64))


def _oracle_cache(o, x, pos=None, cap=None):
    """The oracle's sign-mode records of x [B, H, T, d] packed as a cache
    [B, H, cap, ...] (so both sides read the same bytes), and the encodings."""
    B, H, T, d = x.shape
    cap = cap or T
    codes = np.zeros((B, H, cap, o.bits * d // 8), np.uint8)
    signs = np.zeros((B, H, cap, d // 8), np.uint8)
    norms = np.zeros((B, H, cap, 2), np.float32)
    encs = {}
    for b in range(B):
        for h in range(H):
            e = codec.encode_sign_residual(o, x[b, h], pos)
            codes[b, h, :T] = codec.pack_planes(e["codes"], o.bits)
            signs[b, h, :T] = codec.pack_bits(e["signs"])
            norms[b, h, :T] = np.stack([e["norm"], e["ebar"]], 1)
            encs[b, h] = e
    return (codes, signs, norms), encs


def _dequant(o, e):
    return codec.dequantize_sign_residual(o, e["codes"], e["signs"], e["norm"].astype(np.float32),
                                          e["ebar"].astype(np.float32))


@pytest.mark.parametrize("bits,G", [(2, 4), (1, 8), (3, 2)])
def test_sign_mode_decode_parity(cuda_device, bits, G):
    """Decode over an oracle-packed sign-mode cache (T odd, stride even)."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    d, B, Hkv, T = 128, 2, 2, 777
    gk, ok = _rots(d, bits, 411 + bits, rope=10000.0)
    gv, ov = _rots(d, bits, 412 + bits)
    xk = synth.heavy_tailed((B, Hkv, T, d), 413)
    xv = synth.heavy_tailed((B, Hkv, T, d), 414)
    kc, ek = _oracle_cache(ok, xk, np.arange(T), cap=T + 1)
    vc, ev = _oracle_cache(ov, xv, None, cap=T + 1)
    q = synth.heavy_tailed((B, Hkv * G, d), 415)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention(gk, gv, torch.from_numpy(q).to(dev), qpos,
                              tuple(torch.from_numpy(a).to(dev) for a in kc),
                              tuple(torch.from_numpy(a).to(dev) for a in vc), T)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for b in range(B):
        for h in range(Hkv * G):
            j = h // G
            qr = ro.apply_rope(q[b, h:h + 1], np.array([T - 1]), ok.rope_base)
            ref = at.exact_attention(qr, _dequant(ok, ek[b, j]), _dequant(ov, ev[b, j]), 1 / np.sqrt(d))
            assert_close(out[b, h:h + 1], ref, what=f"b={b} h={h}")


def test_sign_mode_window_decode_parity(cuda_device):
    """The packed part in sign-residual records plus a full-precision window
    (fp32 keys before RoPE, token i at position T + i): against textbook
    attention over the oracle's dequantized rows followed by the window's."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    d, B, Hkv, G, T, R, W = 128, 2, 2, 4, 500, 37, 64
    gk, ok = _rots(d, 2, 431, rope=10000.0)
    gv, ov = _rots(d, 2, 432)
    xk = synth.heavy_tailed((B, Hkv, T, d), 433)
    xv = synth.heavy_tailed((B, Hkv, T, d), 434)
    kc, ek = _oracle_cache(ok, xk, np.arange(T))
    vc, ev = _oracle_cache(ov, xv)
    kw = synth.heavy_tailed((B, Hkv, W, d), 435).astype(np.float32)
    vw = synth.heavy_tailed((B, Hkv, W, d), 436).astype(np.float32)
    q = synth.heavy_tailed((B, Hkv * G, d), 437)
    qpos = T + R - 1
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    out = tq.decode_attention_window(gk, gv, to(q), torch.full((B,), qpos, dtype=torch.int64, device=dev),
                                     tuple(map(to, kc)), tuple(map(to, vc)), T, to(kw), to(vw), R)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for b in range(B):
        for h in range(Hkv * G):
            j = h // G
            qr = ro.apply_rope(q[b, h:h + 1], np.array([qpos]), ok.rope_base)
            keys = np.concatenate([_dequant(ok, ek[b, j]),
                                   ro.apply_rope(kw[b, j, :R].astype(np.float64), T + np.arange(R), ok.rope_base)])
            vals = np.concatenate([_dequant(ov, ev[b, j]), vw[b, j, :R].astype(np.float64)])
            ref = at.exact_attention(qr, keys, vals, 1 / np.sqrt(d))
            assert_close(out[b, h:h + 1], ref, what=f"window b={b} h={h}")


def test_sign_mode_fused_append_equals_separate(cuda_device):
    """The fused decode-step append with sign-residual handles writes the
    same records as the scatter encode of the new rows, and the decode that
    follows gives the same output, bit for bit."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    d, B, Hkv, G, T = 128, 2, 2, 4, 400
    cap = T + 4
    gk, _ = _rots(d, 2, 441, rope=10000.0)
    gv, _ = _rots(d, 2, 442)
    kc = tq.quantize_kv(gk, synth.heavy_tailed_torch((B, Hkv, cap, d), [443, 1], dev), apply_rope=True,
                        pos_period=cap)
    vc = tq.quantize_kv(gv, synth.heavy_tailed_torch((B, Hkv, cap, d), [443, 2], dev))
    kc = tuple(a.view(B, Hkv, cap, -1) for a in kc)
    vc = tuple(a.view(B, Hkv, cap, -1) for a in vc)
    q = synth.heavy_tailed_torch((B, Hkv * G, d), [443, 3], dev)
    k_new = synth.heavy_tailed_torch((B, Hkv, d), [443, 4], dev)
    v_new = synth.heavy_tailed_torch((B, Hkv, d), [443, 5], dev)
    q_pos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    ka, va = tuple(a.clone() for a in kc), tuple(a.clone() for a in vc)
    seqs = torch.arange(B * Hkv, dtype=torch.int64, device=dev)
    flat = lambda c: tuple(a.view(B * Hkv * cap, -1) for a in c)
    tq.quantize_kv_pair_scatter(gk, k_new.view(B * Hkv, d), gv, v_new.view(B * Hkv, d), seqs * cap + T - 1,
                                flat(ka), flat(va), pos=torch.full((B * Hkv,), T - 1, dtype=torch.int64, device=dev),
                                apply_rope=True)
    out_a = tq.decode_attention(gk, gv, q, q_pos, ka, va, T)
    kb, vb = tuple(a.clone() for a in kc), tuple(a.clone() for a in vc)
    out_b = tq.decode_attention_append(gk, gv, q, q_pos, k_new, v_new, kb, vb, T)
    torch.cuda.synchronize()
    for x, y in zip(ka + va, kb + vb):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    assert torch.equal(out_a, out_b)


@pytest.mark.parametrize("d,bits", [(64, 2), (64, 1), (128, 3)])
def test_sign_mode_encoder_parity(cuda_device, d, bits):
    """Encoder attention (the tensor-core kernel for d = 64 and 1-2 bit codes,
    the mma.sync kernel otherwise) over oracle-packed sign-mode caches."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    B, H, S = 1, 2, 300
    gk, ok = _rots(d, bits, 421 + d, rope=10000.0)
    gv, ov = _rots(d, bits, 422 + d)
    xk = synth.lognormal_channels((B, H, S, d), 423)
    xv = synth.lognormal_channels((B, H, S, d), 424)
    xq = synth.lognormal_channels((B, H, S, d), 425)
    kc, ek = _oracle_cache(ok, xk, np.arange(S))
    vc, ev = _oracle_cache(ov, xv)
    out = tq.encoder_attention(gk, gv, torch.from_numpy(xq).to(dev), tuple(torch.from_numpy(a).to(dev) for a in kc),
                               tuple(torch.from_numpy(a).to(dev) for a in vc), S)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for h in range(H):
        qr = ro.apply_rope(xq[0, h], np.arange(S), ok.rope_base)
        ref = at.exact_attention(qr, _dequant(ok, ek[0, h]), _dequant(ov, ev[0, h]), 1 / np.sqrt(d))
        assert_close(out[0, h], ref, what=f"head {h}")


def test_sign_mode_search_parity(cuda_device):
    from vector_quantization_b200 import tq
    dev = cuda_device
    d, N, nq, k = 256, 3000, 12, 10
    g, o = _rots(d, 2, 431, kind="dense")
    U = synth.haar_basis(d, 432)
    db = synth.anisotropic(N, d, 433, basis=U)
    qs = synth.anisotropic(nq, d, 434, basis=U)
    # the dense encode in sign mode, against the oracle's records
    packed = tq.quantize_dense(g, torch.from_numpy(db).to(dev))
    torch.cuda.synchronize()
    e = _check_records(o, tuple(a.cpu().numpy() for a in packed), db)
    # search over the oracle's own records, uploaded
    orec = (codec.pack_planes(e["codes"], o.bits), codec.pack_bits(e["signs"]),
            np.stack([e["norm"], e["ebar"]], 1).astype(np.float32))
    sc, ids = tq.search_topk(g, torch.from_numpy(qs).to(dev), tuple(torch.from_numpy(a).to(dev) for a in orec), k)
    torch.cuda.synchronize()
    xt = _dequant(o, e)
    ref = qs.astype(np.float64) @ xt.T
    sc, ids = sc.cpu().numpy(), ids.cpu().numpy()
    tol = lambda r: 1e-3 + 2e-3 * np.abs(r)
    for q in range(nq):
        ref_at = ref[q, ids[q]]
        assert np.all(np.abs(sc[q] - ref_at) <= tol(ref_at))
        _, oid = osearch.topk_desc(ref[q:q + 1], k)
        kth = ref[q, oid[0, -1]]
        assert set(np.nonzero(ref[q] > kth + 2 * tol(kth))[0].tolist()) <= set(ids[q].tolist())
