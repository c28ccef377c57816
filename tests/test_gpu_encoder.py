"""GPU parity of tq_encoder_attention against the oracle (oracle-packed caches)."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_close, compare_records, oracle_records, oracle_rotation
from oracle import attention as at

pytestmark = pytest.mark.gpu


def _gpu_rot(d, bits, seed, rope, max_pos=1 << 16):
    from vector_quantization_b200 import tq
    return tq.Rotation(d, bits, synth.rotation_randomness(d, seed), rope_base=rope, rope_max_pos=max_pos)


def _packed(orot, x, cap, pos=None):
    B, H, T, d = x.shape
    c, s, n, _ = oracle_records(orot, x.reshape(-1, d), None if pos is None else np.tile(pos, B * H))
    def place(a, fill):
        out = np.full((B, H, cap) + a.shape[1:], fill, dtype=a.dtype)
        out[:, :, :T] = a.reshape(B, H, T, -1)
        return out
    return place(c, 0xFF), place(s, 0xFF), place(n, np.float32(np.nan))


def run(d, bits, B, Hq, Hkv, S, T, seed, q_dtype=torch.float32, law="heavy", q_off=0):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    cap = T + 4 + ((T + 4) & 1)
    rk_o, _ = oracle_rotation(d, bits, 300 + seed, rope=10000.0)
    rv_o, _ = oracle_rotation(d, bits, 400 + seed)
    rk, rv = _gpu_rot(d, bits, 300 + seed, 10000.0), _gpu_rot(d, bits, 400 + seed, 0.0)
    gen = synth.heavy_tailed if law == "heavy" else synth.lognormal_channels
    k = gen((B, Hkv, T, d), 10 + seed)
    v = gen((B, Hkv, T, d), 20 + seed)
    q = torch.from_numpy(gen((B, Hq, S, d), 30 + seed)).to(dev).to(q_dtype)
    kc = _packed(rk_o, k, cap, np.arange(T))
    vc = _packed(rv_o, v, cap)
    to = lambda c: tuple(torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in c)
    out = tq.encoder_attention(rk, rv, q, to(kc), to(vc), T, q_pos_offset=q_off)
    torch.cuda.synchronize()
    ref = at.encoder_attention(rk_o, rv_o, q.float().cpu().numpy(), tuple(a[:, :, :T] for a in kc),
                               tuple(a[:, :, :T] for a in vc), 1 / np.sqrt(d), q_pos_offset=q_off)
    return out.cpu().numpy(), ref


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3])
def test_encoder_parity_bits(cuda_device, d, bits):
    gpu, ref = run(d, bits, 1, 2, 2, 70, 150, seed=d + bits)
    assert_close(gpu, ref, what=f"d={d} bits={bits}")


@pytest.mark.parametrize("S,T", [(1, 1), (8, 16), (64, 128), (65, 129), (130, 300), (200, 1000)])
def test_encoder_parity_shapes(cuda_device, S, T):
    gpu, ref = run(64, 2, 2, 2, 2, S, T, seed=S + T, law="lognormal")
    assert_close(gpu, ref, what=f"S={S} T={T}")


def test_encoder_gqa_bf16_offset(cuda_device):
    gpu, ref = run(128, 2, 1, 4, 2, 33, 257, seed=5, q_dtype=torch.bfloat16, q_off=1000)
    assert_close(gpu, ref)


@pytest.mark.parametrize("bits", [1, 2])
def test_encoder_gqa_d64_several_query_tiles(cuda_device, bits):
    # d = 64: four query heads on two KV heads, 300 queries (three 128-query
    # tiles, the last ragged) against 161 keys (an odd number of 32-key tiles)
    gpu, ref = run(64, bits, 1, 4, 2, 300, 161, seed=11 + bits, q_dtype=torch.bfloat16, q_off=7)
    assert_close(gpu, ref, what=f"bits={bits}")


def test_encoder_empty_cache(cuda_device):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    rk, rv = _gpu_rot(64, 2, 1, 10000.0), _gpu_rot(64, 2, 2, 0.0)
    z = tq.empty_records(rk, (1, 1, 2), dev)
    out = tq.encoder_attention(rk, rv, torch.randn(1, 1, 5, 64, device=dev), z, z, 0)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_esm2_layer_full_size_sampled(cuda_device):
    """One ESM-2-650M-shaped layer at full size (batch 8, 20 heads, 1024
    tokens, head_dim 64, bf16 log-normal channels + 2% outliers x15, RoPE,
    2+1 bits) in the launch configuration the bench times.  GPU encode of
    the whole layer; sampled heads' records are checked against the oracle's
    encoding of the same inputs (codes equal except boundary-flagged
    coordinates: with x15 outlier channels a flipped code there moves a logit
    by more than the output tolerance) and replaced by the oracle's records;
    one full-size attention launch; the sampled heads' outputs against the
    oracle's attention over its own records."""
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    cfg = synth.CONFIGS["esm2_650m_encoder"]
    B, H, T, d = cfg["batch"], cfg["heads"], cfg["tokens"], cfg["head_dim"]
    seed = cfg["seed"]
    rk_o, _ = oracle_rotation(d, 2, seed, rope=10000.0)
    rv_o, _ = oracle_rotation(d, 2, seed + 1)
    rk, rv = _gpu_rot(d, 2, seed, 10000.0), _gpu_rot(d, 2, seed + 1, 0.0)
    k = torch.from_numpy(synth.lognormal_channels((B, H, T, d), [seed, 0, 1])).to(dev).to(torch.bfloat16)
    v = torch.from_numpy(synth.lognormal_channels((B, H, T, d), [seed, 0, 2])).to(dev).to(torch.bfloat16)
    q = torch.from_numpy(synth.lognormal_channels((B, H, T, d), [seed, 0, 3])).to(dev).to(torch.bfloat16)
    kc = tq.quantize_kv(rk, k, apply_rope=True, pos_period=T)
    vc = tq.quantize_kv(rv, v)
    torch.cuda.synchronize()
    rng = np.random.default_rng(0)
    heads = [(0, 0), (B - 1, H - 1)] + [tuple(int(y) for y in x) for x in rng.integers(0, [B, H], size=(2, 2))]
    refs = {}
    for b, h in heads:
        kk = k[b, h].float().cpu().numpy()
        vv = v[b, h].float().cpu().numpy()
        qq = q[b, h].float().cpu().numpy()[None, None]
        recs = []
        for rot_o, x, pos, cache in ((rk_o, kk, np.arange(T), kc), (rv_o, vv, None, vc)):
            codes, signs, norms, enc = oracle_records(rot_o, x, pos)
            compare_records(rot_o, tuple(a[b, h].cpu().numpy().reshape(T, -1) for a in cache), enc)
            for a, r in zip(cache, (codes, signs, norms)):
                a[b, h] = torch.from_numpy(np.ascontiguousarray(r)).to(dev)
            recs.append(tuple(a.reshape(1, 1, T, -1) for a in (codes, signs, norms)))
        refs[b, h] = at.encoder_attention(rk_o, rv_o, qq, recs[0], recs[1], 1 / np.sqrt(d))[0, 0]
    out = tq.encoder_attention(rk, rv, q, kc, vc, T)
    torch.cuda.synchronize()
    for b, h in heads:
        assert_close(out[b, h].cpu().numpy(), refs[b, h], what=f"head ({b},{h}) full launch")