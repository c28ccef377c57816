"""GPU parity of tq_decode_attention against the oracle.

The caches are packed by the oracle, so both sides score the same bytes; the
tolerance is the benchmark spec's bound |gpu - ref| <= 1e-3 + 2e-3 |ref|."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_close, check_and_substitute, oracle_records, oracle_rotation
from oracle import attention as at

pytestmark = pytest.mark.gpu
D = 128


def _gpu_rot(bits, seed, rope):
    from vector_quantization_b200 import tq
    rnd = synth.rotation_randomness(D, seed)
    return tq.Rotation(D, bits, rnd, "hadamard", rope_base=rope, rope_max_pos=(1 << 20) + 8)


def _packed_cache(orot, x, cap, pos=None, poison=True):
    """Oracle-packed cache [B, H, cap, ...]; records past T poisoned (0xFF
    bytes, NaN norms) so that any read past T shows up as NaN."""
    B, H, T, d = x.shape
    codes, signs, norms, _ = oracle_records(orot, x.reshape(-1, d), None if pos is None else np.tile(pos, B * H))
    def place(a, fill):
        out = np.full((B, H, cap) + a.shape[1:], fill, dtype=a.dtype)
        out[:, :, :T] = a.reshape(B, H, T, -1)
        return out
    nan = np.float32(np.nan) if poison else np.float32(0)
    return (place(codes, 0xFF if poison else 0), place(signs, 0xFF if poison else 0), place(norms, nan))


def _to_dev(cache, dev):
    return tuple(torch.from_numpy(np.ascontiguousarray(a)).to(dev) for a in cache)


def run_decode(bits, G, T, B=2, Hkv=2, q_dtype=torch.float32, seed=0, cap_pad=6, rope=10000.0):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    Hq = G * Hkv
    cap = T + cap_pad + ((T + cap_pad) & 1)   # cache_stride must be even
    rk_o, _ = oracle_rotation(D, bits, 500 + seed, rope=rope)
    rv_o, _ = oracle_rotation(D, bits, 600 + seed)
    rk, rv = _gpu_rot(bits, 500 + seed, rope), _gpu_rot(bits, 600 + seed, 0.0)
    k = synth.heavy_tailed((B, Hkv, T, D), 700 + seed)
    v = synth.heavy_tailed((B, Hkv, T, D), 800 + seed)
    kc = _packed_cache(rk_o, k, cap, np.arange(T))
    vc = _packed_cache(rv_o, v, cap)
    q = torch.from_numpy(synth.heavy_tailed((B, Hq, D), 900 + seed)).to(dev).to(q_dtype)
    q_pos = torch.full((B,), max(T - 1, 0), dtype=torch.int64, device=dev)
    out = tq.decode_attention(rk, rv, q, q_pos, _to_dev(kc, dev), _to_dev(vc, dev), T)
    torch.cuda.synchronize()
    ref = at.decode_attention(rk_o, rv_o, q.float().cpu().numpy(), [max(T - 1, 0)] * B,
                              tuple(a[:, :, :T] for a in kc), tuple(a[:, :, :T] for a in vc), 1 / np.sqrt(D))
    return out.cpu().numpy(), ref


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("bits", [1, 2, 3])
def test_decode_parity_heads_bits(cuda_device, G, bits):
    gpu, ref = run_decode(bits, G, 300, seed=G * 10 + bits)
    assert_close(gpu, ref, what=f"G={G} bits={bits}")


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65, 1000, 5000])
def test_decode_parity_lengths(cuda_device, T):
    gpu, ref = run_decode(2, 4, T, seed=T)
    assert_close(gpu, ref, what=f"T={T}")


def test_decode_one_sequence_many_splits(cuda_device):
    """One sequence with one KV head and 8 query heads over 80000 tokens:
    313 splits, whose merge weights (10 KB) take the merge kernel past the
    default 48 KB of shared memory."""
    out, ref = run_decode(2, 8, 80000, B=1, Hkv=1, seed=7)
    assert_close(out, ref, what="G 8, 313 splits")


def test_decode_bf16_query(cuda_device):
    gpu, ref = run_decode(2, 4, 777, q_dtype=torch.bfloat16, seed=3)
    assert_close(gpu, ref)


def test_decode_no_rope(cuda_device):
    gpu, ref = run_decode(3, 2, 200, seed=4, rope=0.0)
    assert_close(gpu, ref)


def test_decode_sequence_limit(cuda_device):
    """B * Hkv sequences fill the split kernel's grid rows, which CUDA caps at
    65535: at the cap the workspace query answers, one past it the query
    gives 0 and the call returns TQ_EUNSUPPORTED on the host, before any
    pointer is looked at or anything is launched."""
    from vector_quantization_b200 import tq
    rk, rv = _gpu_rot(2, 1, 10000.0), _gpu_rot(2, 2, 0.0)
    assert tq.decode_workspace_size(rk, rv, 65535, 4, 1, 16) > 0
    assert tq.decode_workspace_size(rk, rv, 65536, 4, 1, 16) == 0
    assert tq.decode_workspace_size(rk, rv, 32768, 8, 2, 16) == 0
    st = tq._lib.tq_decode_attention(rk.handle, rv.handle, None, 0, None, None, None, None, None, None, None, 16,
                                     65536, 4, 1, 16, None, 0.125, None, None, 0, None)
    assert st == tq.TQ_EUNSUPPORTED


def test_decode_empty_cache(cuda_device):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    rk, rv = _gpu_rot(2, 1, 10000.0), _gpu_rot(2, 2, 0.0)
    q = torch.randn(1, 4, D, device=dev)
    z = tq.empty_records(rk, (1, 1, 2), dev)
    out = tq.decode_attention(rk, rv, q, torch.zeros(1, dtype=torch.int64, device=dev), z, z, 0)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_tiny_workload_end_to_end(cuda_device):
    """1 head, d 128, 1024 fp32 tokens (N(0,1) + 4 outlier channels x20),
    RoPE base 10000 on K, 2-bit codes + 1-bit QJL (m 128), one fp32 query:
    GPU encode + GPU decode against oracle encode + oracle decode."""
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    T = 1024
    cfg = synth.CONFIGS["tiny_d128_t1024"]
    seed = cfg["seed"]
    rk_o, _ = oracle_rotation(D, 2, seed, rope=10000.0)
    rv_o, _ = oracle_rotation(D, 2, seed + 50)
    rk, rv = _gpu_rot(2, seed, 10000.0), _gpu_rot(2, seed + 50, 0.0)
    k = synth.heavy_tailed((1, 1, T, D), seed + 1)
    v = synth.heavy_tailed((1, 1, T, D), seed + 2)
    q = synth.heavy_tailed((1, 1, D), seed + 3)
    kt, vt = torch.from_numpy(k).to(dev), torch.from_numpy(v).to(dev)
    kcache = tq.quantize_kv(rk, kt, apply_rope=True, pos_period=T)
    vcache = tq.quantize_kv(rv, vt)
    out = tq.decode_attention(rk, rv, torch.from_numpy(q).to(dev), torch.tensor([T - 1], device=dev), kcache,
                              vcache, T)
    torch.cuda.synchronize()
    kco = _packed_cache(rk_o, k, T, np.arange(T), poison=False)
    vco = _packed_cache(rv_o, v, T, poison=False)
    ref = at.decode_attention(rk_o, rv_o, q, [T - 1], kco, vco, 1 / np.sqrt(D))
    # code parity first (identical except flagged coordinates)
    from helpers import compare_records
    _, _, _, ek = oracle_records(rk_o, k.reshape(-1, D), np.arange(T))
    compare_records(rk_o, tuple(t.cpu().numpy() for t in kcache), ek)
    assert_close(out.cpu().numpy(), ref, what="tiny end-to-end")


@pytest.mark.parametrize("bits", [2, 3])
def test_decode_full_size_sampled(cuda_device, bits):
    """The Llama-3.1-8B-shaped decode layer at full size (batch 16, 32 query
    heads over 8 KV heads, 32768 cached tokens, heavy-tailed bf16 K/V, RoPE)
    in the launch configuration the bench times.  The caches are GPU-encoded;
    sampled (sequence, KV head) slices are checked against the oracle's
    encoding of the same inputs and replaced by the oracle's records; one
    full-size decode launch; the sampled outputs against the oracle's
    attention over its own records."""
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    cfg = synth.CONFIGS["llama31_8b_gqa_decode"]
    B, Hq, Hkv, T, seed = cfg["batch"], cfg["q_heads"], cfg["kv_heads"], cfg["tokens"], cfg["seed"]
    G = Hq // Hkv
    rk = tq.Rotation(D, bits, synth.rotation_randomness(D, [seed, 11]), rope_base=10000.0, rope_max_pos=T)
    rv = tq.Rotation(D, bits, synth.rotation_randomness(D, [seed, 12]))
    rk_o, _ = oracle_rotation(D, bits, [seed, 11], rope=10000.0)
    rv_o, _ = oracle_rotation(D, bits, [seed, 12])
    samples = [(0, 0), (B - 1, Hkv - 1), (7, 3)]
    xk = synth.heavy_tailed_torch((B, Hkv, T, D), [seed, 13], dev)
    kc = tq.quantize_kv(rk, xk, apply_rope=True, pos_period=T)
    xk_s = {bj: xk[bj].float().cpu().numpy() for bj in samples}
    del xk
    xv = synth.heavy_tailed_torch((B, Hkv, T, D), [seed, 14], dev)
    vc = tq.quantize_kv(rv, xv)
    xv_s = {bj: xv[bj].float().cpu().numpy() for bj in samples}
    del xv
    torch.cuda.synchronize()
    ko = {bj: check_and_substitute(rk_o, kc, *bj, xk_s[bj], np.arange(T)) for bj in samples}
    vo = {bj: check_and_substitute(rv_o, vc, *bj, xv_s[bj]) for bj in samples}
    q = synth.heavy_tailed_torch((B, Hq, D), [seed, 15], dev)
    q_pos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention(rk, rv, q, q_pos, kc, vc, T)
    torch.cuda.synchronize()
    for b, j in samples:
        qq = q[b:b + 1, j * G:(j + 1) * G].float().cpu().numpy()
        ref = at.decode_attention(rk_o, rv_o, qq, [T - 1], ko[b, j], vo[b, j], 1 / np.sqrt(D))
        assert_close(out[b:b + 1, j * G:(j + 1) * G].cpu().numpy(), ref, what=f"bits {bits} seq {b} kv-head {j}")


def test_decode_70b_slice_full_size_sampled(cuda_device):
    """The Llama-3.1-70B-shaped long-context slice at full size (one
    sequence, 64 query heads over 8 KV heads: G = 8, 2^20 cached tokens,
    2+1 bits) in the launch configuration the bench times; one KV head's
    slice is checked against and replaced by the oracle's records, and its
    8 query heads' outputs are checked against the oracle's attention."""
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    c = synth.CONFIGS["llama31_70b_long_slice"]
    Hq, Hkv, T, seed = c["q_heads"], c["kv_heads"], c["tokens"], c["seed"]
    G = Hq // Hkv
    rk = tq.Rotation(D, 2, synth.rotation_randomness(D, [seed, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(D, 2, synth.rotation_randomness(D, [seed, 2]))
    rk_o, _ = oracle_rotation(D, 2, [seed, 1], rope=c["rope_base"])
    rv_o, _ = oracle_rotation(D, 2, [seed, 2])
    j = Hkv - 1
    xk = synth.heavy_tailed_torch((1, Hkv, T, D), [seed, 3], dev)
    kc = tq.quantize_kv(rk, xk, apply_rope=True, pos_period=T)
    xk_j = xk[0, j].float().cpu().numpy()
    del xk
    xv = synth.heavy_tailed_torch((1, Hkv, T, D), [seed, 4], dev)
    vc = tq.quantize_kv(rv, xv)
    xv_j = xv[0, j].float().cpu().numpy()
    del xv
    torch.cuda.synchronize()
    kk = check_and_substitute(rk_o, kc, 0, j, xk_j, np.arange(T))
    vv = check_and_substitute(rv_o, vc, 0, j, xv_j)
    q = synth.heavy_tailed_torch((1, Hq, D), [seed, 5], dev)
    q_pos = torch.full((1,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention(rk, rv, q, q_pos, kc, vc, T)
    torch.cuda.synchronize()
    qq = q[:, j * G:(j + 1) * G].float().cpu().numpy()
    ref = at.decode_attention(rk_o, rv_o, qq, [T - 1], kk, vv, 1 / np.sqrt(D))
    assert_close(out[:, j * G:(j + 1) * G].cpu().numpy(), ref, what=f"70B slice kv-head {j}")

@pytest.mark.parametrize("bits,G", [(2, 4), (3, 8), (1, 1)])
def test_decode_ragged_batch(cuda_device, bits, G):
    """Per-sequence lengths (seq_lens, device int32): sequence b attends to its
    own first seq_lens[b] records, with lengths 0, 1, 17, 300 and the maximum T
    in one call.  Records past a sequence's length are poisoned (NaN norms,
    0xFF bytes) so a read past it would show; an empty sequence gives zeros."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    lens = [0, 1, 17, 300, 1000]
    B, Hkv, T = len(lens), 2, max(lens)
    Hq, cap = G * Hkv, T + 4
    seed = 40 + bits + G
    rk_o, _ = oracle_rotation(D, bits, 500 + seed, rope=10000.0)
    rv_o, _ = oracle_rotation(D, bits, 600 + seed)
    rk, rv = _gpu_rot(bits, 500 + seed, 10000.0), _gpu_rot(bits, 600 + seed, 0.0)
    k = synth.heavy_tailed((B, Hkv, T, D), 700 + seed)
    v = synth.heavy_tailed((B, Hkv, T, D), 800 + seed)
    kc = list(_packed_cache(rk_o, k, cap, np.arange(T)))
    vc = list(_packed_cache(rv_o, v, cap))
    for b, n in enumerate(lens):
        for cache in (kc, vc):
            cache[0][b, :, n:] = 0xFF
            cache[1][b, :, n:] = 0xFF
            cache[2][b, :, n:] = np.nan
    q = torch.from_numpy(synth.heavy_tailed((B, Hq, D), 900 + seed)).to(dev)
    qpos = [max(n - 1, 0) for n in lens]
    out = tq.decode_attention(rk, rv, q, torch.tensor(qpos, dtype=torch.int64, device=dev), _to_dev(kc, dev),
                              _to_dev(vc, dev), T, seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for b, n in enumerate(lens):
        ref = at.decode_attention(rk_o, rv_o, q[b:b + 1].cpu().numpy(), [qpos[b]],
                                  tuple(a[b:b + 1, :, :n] for a in kc), tuple(a[b:b + 1, :, :n] for a in vc),
                                  1 / np.sqrt(D))
        assert_close(out[b:b + 1], ref, what=f"sequence {b} of length {n}")
    assert np.all(out[0] == 0.0)


def test_decode_length_outside_range_gives_nan(cuda_device):
    """A seq_lens entry above T (or negative) cannot be checked on the host
    (device memory); that sequence's outputs are NaN, the others unaffected."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    B, Hkv, G, T = 3, 1, 4, 64
    rk_o, _ = oracle_rotation(D, 2, 71, rope=10000.0)
    rv_o, _ = oracle_rotation(D, 2, 72)
    rk, rv = _gpu_rot(2, 71, 10000.0), _gpu_rot(2, 72, 0.0)
    kc = _packed_cache(rk_o, synth.heavy_tailed((B, Hkv, T, D), 73), T, np.arange(T))
    vc = _packed_cache(rv_o, synth.heavy_tailed((B, Hkv, T, D), 74), T)
    q = torch.from_numpy(synth.heavy_tailed((B, G * Hkv, D), 75)).to(dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention(rk, rv, q, qpos, _to_dev(kc, dev), _to_dev(vc, dev), T,
                              seq_lens=torch.tensor([T, T + 1, -3], dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    assert np.all(np.isfinite(out[0])) and np.all(np.isnan(out[1])) and np.all(np.isnan(out[2]))
