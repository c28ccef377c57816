"""GPU parity of the fused decode-step append (tq_decode_attention_append):
the new token's records equal those of a separate pair encode bit for bit,
the output equals that of the separate encode + decode exactly, and against
the oracle (records, and attention over oracle-packed history plus the new
token) the usual tolerances hold."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_close, compare_records, oracle_records, oracle_rotation
from oracle import attention as at

pytestmark = pytest.mark.gpu
D = 128


def _rots(bits, seed, T):
    from vector_quantization_b200 import tq
    rk = tq.Rotation(D, bits, synth.rotation_randomness(D, [seed, 1]), rope_base=10000.0, rope_max_pos=T + 8)
    rv = tq.Rotation(D, bits, synth.rotation_randomness(D, [seed, 2]))
    return rk, rv


@pytest.mark.parametrize("bits,G,dtype", [(2, 4, torch.bfloat16), (3, 8, torch.float32), (1, 1, torch.bfloat16),
                                          (2, 2, torch.float32)])
@pytest.mark.parametrize("ragged", [False, True])
def test_append_equals_separate_encode_and_decode(cuda_device, bits, G, dtype, ragged):
    from vector_quantization_b200 import tq
    dev = cuda_device
    B, Hkv, T, seed = 3, 2, 1000, 40 + bits * 10 + G
    Hq, cap = G * Hkv, T + 4
    rk, rv = _rots(bits, seed, T)
    hist_k = synth.heavy_tailed_torch((B, Hkv, cap, D), [seed, 3], dev).to(dtype)
    hist_v = synth.heavy_tailed_torch((B, Hkv, cap, D), [seed, 4], dev).to(dtype)
    kc = tq.quantize_kv(rk, hist_k, apply_rope=True, pos_period=cap)
    vc = tq.quantize_kv(rv, hist_v)
    kc = tuple(a.view(B, Hkv, cap, -1) for a in kc)
    vc = tuple(a.view(B, Hkv, cap, -1) for a in vc)
    lens = [T, 1, 0] if ragged else [T] * B
    seq_lens = torch.tensor(lens, dtype=torch.int32, device=dev) if ragged else None
    q_pos = torch.tensor([max(n - 1, 0) for n in lens], dtype=torch.int64, device=dev)
    q = synth.heavy_tailed_torch((B, Hq, D), [seed, 5], dev).to(dtype)
    k_new = synth.heavy_tailed_torch((B, Hkv, D), [seed, 6], dev).to(dtype)
    v_new = synth.heavy_tailed_torch((B, Hkv, D), [seed, 7], dev).to(dtype)
    # separate: scatter encode of the new rows, then decode
    ka, va = tuple(a.clone() for a in kc), tuple(a.clone() for a in vc)
    rows = [(b * Hkv + j, b) for b in range(B) for j in range(Hkv) if lens[b] >= 1]
    sel = torch.tensor([r for r, _ in rows], dtype=torch.int64, device=dev)
    out_rows = torch.tensor([r * cap + lens[b] - 1 for r, b in rows], dtype=torch.int64, device=dev)
    pos = torch.tensor([lens[b] - 1 for _, b in rows], dtype=torch.int64, device=dev)
    flat = lambda c: tuple(a.view(B * Hkv * cap, -1) for a in c)
    tq.quantize_kv_pair_scatter(rk, k_new.view(B * Hkv, D)[sel], rv, v_new.view(B * Hkv, D)[sel], out_rows,
                                flat(ka), flat(va), pos=pos, apply_rope=True)
    out_a = tq.decode_attention(rk, rv, q, q_pos, ka, va, T, seq_lens=seq_lens)
    # fused
    kb, vb = tuple(a.clone() for a in kc), tuple(a.clone() for a in vc)
    out_b = tq.decode_attention_append(rk, rv, q, q_pos, k_new, v_new, kb, vb, T, seq_lens=seq_lens)
    torch.cuda.synchronize()
    for x, y in zip(ka + va, kb + vb):
        assert torch.equal(x, y)
    assert torch.equal(out_a, out_b)
    if ragged:
        assert torch.all(out_b[2] == 0)


@pytest.mark.parametrize("bits,G", [(2, 4), (3, 2)])
def test_append_against_oracle(cuda_device, bits, G):
    """History records packed by the oracle (token T - 1 poisoned); the
    fused call writes token T - 1 from the raw new rows, whose records are
    checked against the oracle's encoding, and the output against the
    oracle's attention over all T tokens."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    B, Hkv, T, seed = 2, 2, 777, 90 + bits
    Hq, cap = G * Hkv, T + 1 + (T + 1) % 2
    rk, rv = _rots(bits, seed, T)
    rk_o, _ = oracle_rotation(D, bits, [seed, 1], rope=10000.0)
    rv_o, _ = oracle_rotation(D, bits, [seed, 2])
    k = synth.heavy_tailed((B, Hkv, T, D), [seed, 3])
    v = synth.heavy_tailed((B, Hkv, T, D), [seed, 4])
    pos = np.tile(np.arange(T), B * Hkv)
    ko = oracle_records(rk_o, k.reshape(-1, D), pos)
    vo = oracle_records(rv_o, v.reshape(-1, D))

    def cache(rec, poison):
        arrs = []
        for a, fill in zip(rec[:3], (0xFF, 0xFF, np.nan)):
            full = np.full((B, Hkv, cap) + a.shape[1:], fill, dtype=a.dtype)
            full[:, :, :T] = a.reshape(B, Hkv, T, -1)
            if poison:
                full[:, :, T - 1] = fill
            arrs.append(torch.from_numpy(full).to(dev))
        return tuple(arrs)
    kc, vc = cache(ko, True), cache(vo, True)
    q = torch.from_numpy(synth.heavy_tailed((B, Hq, D), [seed, 5])).to(dev)
    q_pos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    k_new = torch.from_numpy(np.ascontiguousarray(k[:, :, T - 1])).to(dev)
    v_new = torch.from_numpy(np.ascontiguousarray(v[:, :, T - 1])).to(dev)
    out = tq.decode_attention_append(rk, rv, q, q_pos, k_new, v_new, kc, vc, T)
    torch.cuda.synchronize()
    enc_last = lambda e: {key: (val.reshape(B, Hkv, T, *val.shape[1:])[:, :, T - 1].reshape(B * Hkv, *val.shape[1:])
                                if isinstance(val, np.ndarray) and val.shape[:1] == (B * Hkv * T,) else val)
                          for key, val in e.items()}
    got_k = tuple(a[:, :, T - 1].reshape(B * Hkv, -1).cpu().numpy() for a in kc)
    got_v = tuple(a[:, :, T - 1].reshape(B * Hkv, -1).cpu().numpy() for a in vc)
    compare_records(rk_o, got_k, enc_last(ko[3]))
    compare_records(rv_o, got_v, enc_last(vo[3]))
    ref = at.decode_attention(rk_o, rv_o, q.cpu().numpy(), [T - 1] * B,
                              tuple(np.asarray(a).reshape(B, Hkv, T, -1) for a in ko[:3]),
                              tuple(np.asarray(a).reshape(B, Hkv, T, -1) for a in vo[:3]), 1 / np.sqrt(D))
    assert_close(out.cpu().numpy(), ref, what=f"append bits {bits} G {G}")
