"""GPU parity of the NSN record mode ([NSNQuant] §1, §4) against the oracle:
tq_nsn_shift + the codec (s1, o and the records of the shifted rows), and
tq_decode_attention_nsn over NSN records (oracle-packed, and end to end)."""
import math

import numpy as np
import pytest
import torch

import synth
from helpers import assert_close, compare_records, oracle_rotation
from oracle import attention as at
from oracle import codec

pytestmark = pytest.mark.gpu


def _gpu_rot(d, bits, seed, rope):
    from vector_quantization_b200 import tq
    return tq.Rotation(d, bits, synth.rotation_randomness(d, seed), "hadamard", rope_base=rope,
                       rope_max_pos=(1 << 16) if rope else 0)


def _offset_rows(shape, seed, offset=4.0):
    """Heavy-tailed rows plus 8 channels offset by +-offset in every token of
    a block (the case NSN's shift removes)."""
    x = synth.heavy_tailed(shape, seed).astype(np.float64)
    g = np.random.default_rng(seed)
    *lead, L, d = shape
    for idx in np.ndindex(*lead):
        ch = g.choice(d, 8, replace=False)
        x[idx][:, ch] += offset * np.where(g.random(8) < 0.5, -1.0, 1.0)
    return x.astype(np.float32)


@pytest.mark.parametrize("d,bits,rope,dtype", [(128, 2, 10000.0, torch.float32), (128, 3, 0.0, torch.bfloat16),
                                               (64, 2, 10000.0, torch.bfloat16), (64, 1, 0.0, torch.float32)])
@pytest.mark.parametrize("L", [300, 20000])
def test_nsn_encode_parity(cuda_device, d, bits, rope, dtype, L):
    """s1, o and the records of the shifted rows against nsn_encode; L = 20000
    takes the tensor-core encode for the shifted rows."""
    from vector_quantization_b200 import tq
    nb = 2
    x = _offset_rows((nb, L, d), 30 + d + bits)
    xt = torch.from_numpy(x).to(cuda_device).to(dtype)
    xin = xt.float().cpu().numpy().astype(np.float64)   # the rows as the GPU sees them
    g = _gpu_rot(d, bits, 40 + bits, rope)
    o_rot, _ = oracle_rotation(d, bits, 40 + bits, rope=rope)
    rec, s1, o = tq.quantize_kv_nsn(g, xt, apply_rope=bool(rope), pos_offset=5)
    torch.cuda.synchronize()
    for b in range(nb):
        e = codec.nsn_encode(o_rot, xin[b], np.arange(L) + 5 if rope else None)
        np.testing.assert_allclose(s1[b].cpu().numpy(), e["s1"], rtol=2e-6, atol=0)
        np.testing.assert_allclose(o[b].cpu().numpy(), e["o"], rtol=0, atol=2e-6 * math.sqrt(d))
        compare_records(o_rot, tuple(a[b].cpu().numpy() for a in rec), e)


def _nsn_caches(rot, x, pos, cap):
    """Oracle NSN records of blocks x [B, H, T, d] in caches of capacity cap
    (records past T poisoned), s1 [B, H, cap] (NaN past T), o [B, H, d]."""
    B, H, T, d = x.shape
    codes = np.full((B, H, cap, rot.bits * d // 8), 0xFF, np.uint8)
    signs = np.full((B, H, cap, rot.m // 8), 0xFF, np.uint8)
    norms = np.full((B, H, cap, 2), np.nan, np.float32)
    s1 = np.full((B, H, cap), np.nan, np.float32)
    o = np.zeros((B, H, d), np.float32)
    for b in range(B):
        for h in range(H):
            e = codec.nsn_encode(rot, x[b, h], pos)
            codes[b, h, :T] = codec.pack_planes(e["codes"], rot.bits)
            signs[b, h, :T] = codec.pack_bits(e["signs"])
            norms[b, h, :T] = np.stack([e["norm"], e["rnorm"]], axis=1)
            s1[b, h, :T] = e["s1"]
            o[b, h] = e["o"]
    return (codes, signs, norms), s1, o


@pytest.mark.parametrize("G,bits,T", [(4, 2, 300), (1, 3, 17), (8, 1, 1000), (2, 2, 1)])
def test_nsn_decode_parity(cuda_device, G, bits, T):
    from vector_quantization_b200 import tq
    d, B, Hkv = 128, 2, 2
    Hq, cap = G * Hkv, T + 8 - (T % 4)
    rk, rv = _gpu_rot(d, bits, 60 + bits, 10000.0), _gpu_rot(d, bits, 70 + bits, 0.0)
    ork, _ = oracle_rotation(d, bits, 60 + bits, rope=10000.0)
    orv, _ = oracle_rotation(d, bits, 70 + bits)
    k = _offset_rows((B, Hkv, T, d), 80 + G).astype(np.float64)
    v = _offset_rows((B, Hkv, T, d), 90 + G).astype(np.float64)
    kc, ks1, ko = _nsn_caches(ork, k, np.arange(T), cap)
    vc, vs1, vo = _nsn_caches(orv, v, None, cap)
    dev = cuda_device
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    q = synth.heavy_tailed((B, Hq, d), 7 + G)
    q_pos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention_nsn(rk, rv, to(q), q_pos, tuple(map(to, kc)), tuple(map(to, vc)), to(ks1), to(ko),
                                  to(vs1), to(vo), T)
    torch.cuda.synchronize()
    ref = at.decode_attention_nsn(ork, orv, q, [T - 1] * B, tuple(a[:, :, :T] for a in kc),
                                  tuple(a[:, :, :T] for a in vc), ks1[:, :, :T], ko, vs1[:, :, :T], vo,
                                  1 / math.sqrt(d))
    assert_close(out.cpu().numpy(), ref, what=f"NSN decode G {G} bits {bits} T {T}")


def test_nsn_decode_ragged_lengths(cuda_device):
    from vector_quantization_b200 import tq
    d, B, Hkv, G, T, bits = 128, 3, 2, 4, 500, 2
    Hq, cap = G * Hkv, 504
    rk, rv = _gpu_rot(d, bits, 61, 10000.0), _gpu_rot(d, bits, 71, 0.0)
    ork, _ = oracle_rotation(d, bits, 61, rope=10000.0)
    orv, _ = oracle_rotation(d, bits, 71)
    k = _offset_rows((B, Hkv, T, d), 81).astype(np.float64)
    v = _offset_rows((B, Hkv, T, d), 91).astype(np.float64)
    kc, ks1, ko = _nsn_caches(ork, k, np.arange(T), cap)
    vc, vs1, vo = _nsn_caches(orv, v, None, cap)
    dev = cuda_device
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    lens = [500, 1, 0]
    q = synth.heavy_tailed((B, Hq, d), 5)
    q_pos = torch.tensor([max(n - 1, 0) for n in lens], dtype=torch.int64, device=dev)
    out = tq.decode_attention_nsn(rk, rv, to(q), q_pos, tuple(map(to, kc)), tuple(map(to, vc)), to(ks1), to(ko),
                                  to(vs1), to(vo), T, seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    assert np.all(out[2] == 0)
    for b in range(2):
        # the shift o of a block covers all T tokens; attention reads the first lens[b]
        n = lens[b]
        ref = at.decode_attention_nsn(ork, orv, q[b:b + 1], [n - 1], tuple(a[b:b + 1, :, :n] for a in kc),
                                      tuple(a[b:b + 1, :, :n] for a in vc), ks1[b:b + 1, :, :n], ko[b:b + 1],
                                      vs1[b:b + 1, :, :n], vo[b:b + 1], 1 / math.sqrt(d))
        assert_close(out[b:b + 1], ref, what=f"NSN ragged seq {b}")


def test_nsn_end_to_end(cuda_device):
    """GPU NSN encode of keys (RoPE) and values, then GPU NSN decode, against
    the oracle's encode and decode of the same rows."""
    from vector_quantization_b200 import tq
    d, B, Hkv, G, T, bits = 128, 2, 2, 4, 1500, 2
    Hq, cap = G * Hkv, 1500
    dev = cuda_device
    rk, rv = _gpu_rot(d, bits, 62, 10000.0), _gpu_rot(d, bits, 72, 0.0)
    ork, _ = oracle_rotation(d, bits, 62, rope=10000.0)
    orv, _ = oracle_rotation(d, bits, 72)
    k = _offset_rows((B, Hkv, T, d), 83)
    v = _offset_rows((B, Hkv, T, d), 93)
    kr, ks1, ko = tq.quantize_kv_nsn(rk, torch.from_numpy(k).to(dev), apply_rope=True)
    vr, vs1, vo = tq.quantize_kv_nsn(rv, torch.from_numpy(v).to(dev))
    q = synth.heavy_tailed((B, Hq, d), 9)
    q_pos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention_nsn(rk, rv, torch.from_numpy(q).to(dev), q_pos, kr, vr, ks1, ko, vs1, vo, T)
    torch.cuda.synchronize()
    okc, oks1, oko = _nsn_caches(ork, k.astype(np.float64), np.arange(T), cap)
    ovc, ovs1, ovo = _nsn_caches(orv, v.astype(np.float64), None, cap)
    ref = at.decode_attention_nsn(ork, orv, q, [T - 1] * B, okc, ovc, oks1, oko, ovs1, ovo, 1 / math.sqrt(d))
    assert_close(out.cpu().numpy(), ref, what="NSN end to end")


def test_nsn_shift_small_blocks_and_zero_rows(cuda_device):
    """Blocks of one, two and 257 rows (one chunk, o written directly; two
    chunks) with an all-zero row (s1 = 0, nothing added to o; its record is
    the zero vector's) against nsn_encode."""
    from vector_quantization_b200 import tq
    d = 128
    g = _gpu_rot(d, 2, 44, 10000.0)
    o_rot, _ = oracle_rotation(d, 2, 44, rope=10000.0)
    for L in (1, 2, 257):
        x = _offset_rows((3, L, d), 50 + L)
        x[1, 0] = 0.0
        xt = torch.from_numpy(x).to(cuda_device)
        rec, s1, o = tq.quantize_kv_nsn(g, xt, apply_rope=True)
        torch.cuda.synchronize()
        for b in range(3):
            e = codec.nsn_encode(o_rot, x[b].astype(np.float64), np.arange(L))
            np.testing.assert_allclose(s1[b].cpu().numpy(), e["s1"], rtol=2e-6, atol=0)
            np.testing.assert_allclose(o[b].cpu().numpy(), e["o"], rtol=0, atol=2e-6 * math.sqrt(d))
            # a one-row block shifts its row to x' = 0 up to rounding, whose
            # direction is noise: its records are not compared
            if L > 1:
                compare_records(o_rot, tuple(a[b].cpu().numpy() for a in rec), e)


def test_nsn_decode_empty_cache(cuda_device):
    from vector_quantization_b200 import tq
    d, B, Hkv, G = 128, 1, 2, 4
    rk, rv = _gpu_rot(d, 2, 63, 10000.0), _gpu_rot(d, 2, 73, 0.0)
    dev = cuda_device
    cap = 8
    kc = tq.empty_records(rk, (B, Hkv, cap), dev)
    vc = tq.empty_records(rv, (B, Hkv, cap), dev)
    z1 = torch.zeros((B, Hkv, cap), dtype=torch.float32, device=dev)
    zo = torch.zeros((B, Hkv, d), dtype=torch.float32, device=dev)
    q = torch.ones((B, G * Hkv, d), dtype=torch.float32, device=dev)
    out = tq.decode_attention_nsn(rk, rv, q, torch.zeros((B,), dtype=torch.int64, device=dev), kc, vc, z1, zo, z1,
                                  zo, 0)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def _append_case(G, bits, dtype, T, seed, dev):
    """Oracle NSN caches of the first T - 1 tokens of each block (o from
    those tokens; token T - 1 and its s1 poisoned) and the raw rows of token
    T - 1, in the dtype the GPU reads."""
    from vector_quantization_b200 import tq
    d, B, Hkv = 128, 2, 2
    Hq, cap = G * Hkv, T + 4 - T % 4
    rk, rv = _gpu_rot(d, bits, seed, 10000.0), _gpu_rot(d, bits, seed + 10, 0.0)
    ork, _ = oracle_rotation(d, bits, seed, rope=10000.0)
    orv, _ = oracle_rotation(d, bits, seed + 10)
    kt = torch.from_numpy(_offset_rows((B, Hkv, T, d), seed + 20)).to(dtype)
    vt = torch.from_numpy(_offset_rows((B, Hkv, T, d), seed + 30)).to(dtype)
    k64, v64 = (a.float().numpy().astype(np.float64) for a in (kt, vt))
    kc, ks1, ko = _nsn_caches(ork, k64[:, :, :T - 1], np.arange(T - 1), cap)
    vc, vs1, vo = _nsn_caches(orv, v64[:, :, :T - 1], None, cap)
    qt = torch.from_numpy(synth.heavy_tailed((B, Hq, d), seed + 40)).to(dtype)
    return dict(rk=rk, rv=rv, ork=ork, orv=orv, k64=k64, v64=v64, kc=kc, ks1=ks1, ko=ko, vc=vc, vs1=vs1, vo=vo,
                k_new=kt[:, :, T - 1].contiguous().to(dev), v_new=vt[:, :, T - 1].contiguous().to(dev),
                q=qt.to(dev), q64=qt.float().numpy().astype(np.float64), B=B, Hkv=Hkv, cap=cap)


@pytest.mark.parametrize("G,bits,dtype", [(4, 2, torch.float32), (8, 3, torch.bfloat16), (1, 1, torch.float32)])
def test_nsn_append_against_oracle(cuda_device, G, bits, dtype):
    """The fused NSN append writes token T - 1 from the raw rows (key after
    RoPE, both shifted by their block's o): records and s1 against the
    oracle's nsn_append with the same o; the output against the oracle's NSN
    attention over all T records, the last ones the oracle's own."""
    from vector_quantization_b200 import tq
    T, dev, d = 600, cuda_device, 128
    c = _append_case(G, bits, dtype, T, 100 + 3 * G + bits, dev)
    B, Hkv = c["B"], c["Hkv"]
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    kcd, vcd = tuple(map(to, c["kc"])), tuple(map(to, c["vc"]))
    ks1d, vs1d = to(c["ks1"]), to(c["vs1"])
    q_pos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention_nsn_append(c["rk"], c["rv"], c["q"], q_pos, c["k_new"], c["v_new"], kcd, vcd, ks1d,
                                         to(c["ko"]), vs1d, to(c["vo"]), T)
    torch.cuda.synchronize()
    kc, vc = tuple(np.array(a) for a in c["kc"]), tuple(np.array(a) for a in c["vc"])
    ks1, vs1 = c["ks1"].copy(), c["vs1"].copy()
    for side, (ot, x64, o, cache, s1, gcache, gs1, pos) in enumerate(
            ((c["ork"], c["k64"], c["ko"], kc, ks1, kcd, ks1d, [T - 1]),
             (c["orv"], c["v64"], c["vo"], vc, vs1, vcd, vs1d, None))):
        for b in range(B):
            for j in range(Hkv):
                e = codec.nsn_append(ot, x64[b, j, T - 1:T], pos, o[b, j])
                compare_records(ot, tuple(a[b, j, T - 1:T].cpu().numpy() for a in gcache), e)
                np.testing.assert_allclose(gs1[b, j, T - 1].item(), e["s1"][0], rtol=2e-6, atol=0)
                cache[0][b, j, T - 1] = codec.pack_planes(e["codes"], ot.bits)[0]
                cache[1][b, j, T - 1] = codec.pack_bits(e["signs"])[0]
                cache[2][b, j, T - 1] = (e["norm"][0], e["rnorm"][0])
                s1[b, j, T - 1] = e["s1"][0]
    ref = at.decode_attention_nsn(c["ork"], c["orv"], c["q64"], [T - 1] * B, tuple(a[:, :, :T] for a in kc),
                                  tuple(a[:, :, :T] for a in vc), ks1[:, :, :T], c["ko"], vs1[:, :, :T], c["vo"],
                                  1 / math.sqrt(d))
    assert_close(out.cpu().numpy(), ref, what=f"NSN append G {G} bits {bits}")


def test_nsn_append_equals_append_then_decode(cuda_device):
    """Ragged lengths (T, 1, 0): the fused call's output equals
    decode_attention_nsn over the caches it wrote, bit for bit; the empty
    sequence's records stay as they were and its output is zero."""
    from vector_quantization_b200 import tq
    T, dev = 333, cuda_device
    c = _append_case(4, 2, torch.bfloat16, T, 150, dev)
    B = c["B"]
    to = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    # a third sequence of length 0 next to lengths T and 1
    pad = lambda a: np.concatenate([a, a[:1]], axis=0)
    kcd, vcd = tuple(to(pad(a)) for a in c["kc"]), tuple(to(pad(a)) for a in c["vc"])
    ks1d, vs1d, kod, vod = (to(pad(a)) for a in (c["ks1"], c["vs1"], c["ko"], c["vo"]))
    before = tuple(a[2].clone() for a in kcd + vcd)
    k_new = torch.cat([c["k_new"], c["k_new"][:1]])
    v_new = torch.cat([c["v_new"], c["v_new"][:1]])
    q = torch.cat([c["q"], c["q"][:1]])
    lens = torch.tensor([T, 1, 0], dtype=torch.int32, device=dev)
    q_pos = torch.tensor([T - 1, 0, 0], dtype=torch.int64, device=dev)
    out_a = tq.decode_attention_nsn_append(c["rk"], c["rv"], q, q_pos, k_new, v_new, kcd, vcd, ks1d, kod, vs1d, vod,
                                           T, seq_lens=lens)
    out_b = tq.decode_attention_nsn(c["rk"], c["rv"], q, q_pos, kcd, vcd, ks1d, kod, vs1d, vod, T, seq_lens=lens)
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b)
    assert torch.all(out_a[2] == 0)
    for x, y in zip(before, tuple(a[2] for a in kcd + vcd)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))   # bytes: the poisoned norms are NaN
    assert torch.isfinite(ks1d[1, :, 0]).all() and torch.isfinite(vs1d[1, :, 0]).all()
