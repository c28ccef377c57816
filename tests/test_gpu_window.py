"""GPU parity of tq_decode_attention_window (packed cache plus a full-precision
window of recent tokens, [NSNQuant] §4 "Résidus") against the oracle.

The packed caches of the small cases are written by the oracle, so both sides
score the same bytes; the full-size case encodes on the GPU, checks the
sampled slices against the oracle's encoding and replaces them by it.  Window
keys and values are the same float32 (or bf16-rounded) values on both sides.
Tolerance: |gpu - ref| <= 1e-3 + 2e-3 |ref|."""
import numpy as np
import pytest
import torch

import synth
from helpers import assert_close, check_and_substitute, compare_records, oracle_records, oracle_rotation
from oracle import attention as at

pytestmark = pytest.mark.gpu
D = 128


def _gpu_rot(bits, seed, rope):
    from vector_quantization_b200 import tq
    return tq.Rotation(D, bits, synth.rotation_randomness(D, seed), "hadamard", rope_base=rope,
                       rope_max_pos=(1 << 20) + 8)


def _packed_cache(orot, x, cap, pos=None):
    """Oracle-packed cache [B, H, cap, ...]; records past T poisoned (0xFF bytes, NaN norms)."""
    B, H, T, d = x.shape
    out = [np.full((B, H, cap, orot.bits * d // 8), 0xFF, np.uint8), np.full((B, H, cap, orot.m // 8), 0xFF, np.uint8),
           np.full((B, H, cap, 2), np.nan, np.float32)]
    if T:
        codes, signs, norms, _ = oracle_records(orot, x.reshape(-1, d), None if pos is None else np.tile(pos, B * H))
        for a, src in zip(out, (codes, signs, norms)):
            a[:, :, :T] = src.reshape(B, H, T, -1)
    return tuple(out)


def _window(shape, seed, dtype, cap):
    """Window values [B, H, R, D] as the device dtype rounds them, in an array of capacity cap (NaN past R)."""
    B, H, R, _ = shape
    x = torch.from_numpy(synth.heavy_tailed(shape, seed)).to(dtype)
    full = torch.full((B, H, cap, D), float("nan"), dtype=dtype)
    full[:, :, :R] = x
    return full, x.double().numpy()


def run_window(bits, G, T, R, B=2, Hkv=2, q_dtype=torch.float32, w_dtype=torch.float32, seed=0, rope=10000.0,
               cap_pad=3):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    Hq = G * Hkv
    cap = T + 6 + (T & 1)
    rk_o, _ = oracle_rotation(D, bits, 1500 + seed, rope=rope)
    rv_o, _ = oracle_rotation(D, bits, 1600 + seed)
    rk, rv = _gpu_rot(bits, 1500 + seed, rope), _gpu_rot(bits, 1600 + seed, 0.0)
    kc = _packed_cache(rk_o, synth.heavy_tailed((B, Hkv, T, D), 1700 + seed), cap, np.arange(T))
    vc = _packed_cache(rv_o, synth.heavy_tailed((B, Hkv, T, D), 1800 + seed), cap)
    kw, kw_ref = _window((B, Hkv, R, D), 1900 + seed, w_dtype, R + cap_pad)
    vw, vw_ref = _window((B, Hkv, R, D), 2000 + seed, w_dtype, R + cap_pad)
    q = torch.from_numpy(synth.heavy_tailed((B, Hq, D), 2100 + seed)).to(q_dtype).to(dev)
    qpos = [T + R + b for b in range(B)]
    out = tq.decode_attention_window(rk, rv, q, torch.tensor(qpos, dtype=torch.int64, device=dev),
                                     tuple(torch.from_numpy(a).to(dev) for a in kc),
                                     tuple(torch.from_numpy(a).to(dev) for a in vc), T, kw.to(dev), vw.to(dev), R)
    torch.cuda.synchronize()
    ref = at.decode_attention_window(rk_o, rv_o, q.double().cpu().numpy(), qpos, tuple(a[:, :, :T] for a in kc),
                                     tuple(a[:, :, :T] for a in vc), kw_ref, vw_ref, 1 / np.sqrt(D))
    return out.cpu().numpy(), ref


@pytest.mark.parametrize("R", [1, 37, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_window_parity_heads(cuda_device, G, R):
    gpu, ref = run_window(2, G, 300, R, seed=G * 10 + R)
    assert_close(gpu, ref, what=f"G={G} R={R}")


@pytest.mark.parametrize("bits", [1, 3])
def test_window_parity_bits(cuda_device, bits):
    gpu, ref = run_window(bits, 4, 513, 64, seed=bits)
    assert_close(gpu, ref, what=f"bits={bits}")


@pytest.mark.parametrize("R", [1, 200, 1024])
def test_window_without_packed_part(cuda_device, R):
    gpu, ref = run_window(2, 4, 0, R, seed=R)
    assert_close(gpu, ref, what=f"T=0 R={R}")


def test_window_bf16(cuda_device):
    gpu, ref = run_window(2, 4, 1000, 96, q_dtype=torch.bfloat16, w_dtype=torch.bfloat16, seed=5)
    assert_close(gpu, ref)


def test_window_no_rope(cuda_device):
    gpu, ref = run_window(2, 2, 77, 21, seed=6, rope=0.0)
    assert_close(gpu, ref)


def test_window_long_packed_part(cuda_device):
    # several splits of the packed part plus a window at its largest size
    gpu, ref = run_window(2, 4, 20000, 1024, B=1, Hkv=1, seed=7)
    assert_close(gpu, ref)


def test_empty_window_is_plain_decode(cuda_device):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    T, B, Hkv, G = 333, 2, 2, 4
    rk_o, _ = oracle_rotation(D, 2, 31, rope=10000.0)
    rv_o, _ = oracle_rotation(D, 2, 32)
    rk, rv = _gpu_rot(2, 31, 10000.0), _gpu_rot(2, 32, 0.0)
    kc = tuple(torch.from_numpy(a).to(dev) for a in
               _packed_cache(rk_o, synth.heavy_tailed((B, Hkv, T, D), 33), T + 1, np.arange(T)))
    vc = tuple(torch.from_numpy(a).to(dev) for a in _packed_cache(rv_o, synth.heavy_tailed((B, Hkv, T, D), 34), T + 1))
    q = torch.from_numpy(synth.heavy_tailed((B, G * Hkv, D), 35)).to(dev)
    qpos = torch.full((B,), T, dtype=torch.int64, device=dev)
    w = torch.zeros((B, Hkv, 4, D), device=dev)
    a = tq.decode_attention(rk, rv, q, qpos, kc, vc, T)
    b = tq.decode_attention_window(rk, rv, q, qpos, kc, vc, T, w, w, 0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_window_rejects_bad_arguments(cuda_device):
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    rk, rv = _gpu_rot(2, 41, 10000.0), _gpu_rot(2, 42, 0.0)
    z = tq.empty_records(rk, (1, 1, 2), dev)
    q = torch.zeros((1, 4, D), device=dev)
    qpos = torch.zeros(1, dtype=torch.int64, device=dev)
    w = torch.zeros((1, 1, 2000, D), device=dev)
    with pytest.raises(tq.TQError, match="unsupported"):
        tq.decode_attention_window(rk, rv, q, qpos, z, z, 0, w, w, 1025)
    with pytest.raises(tq.TQError):
        tq.decode_attention_window(rk, rv, q, qpos, z, z, 0, w[:, :, :5], w[:, :, :5], 6)   # stride < R
    assert tq.decode_window_workspace_size(rk, rv, 1, 4, 1, 10, 1025) == 0
    assert tq.decode_window_workspace_size(rk, rv, 1, 4, 1, 10, 8) > tq.decode_workspace_size(rk, rv, 1, 4, 1, 10)


def test_streaming_append_and_flush(cuda_device):
    """Decode steps over a growing cache: each step appends its token to the
    window; a full window is quantized (positions T .. T+W-1) into the packed
    part and emptied.  GPU flushes with tq_quantize_kv_pair; the oracle encodes
    the same rows itself.  Checked at every step against the oracle."""
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    B, Hkv, G, W, T0, steps = 2, 2, 4, 16, 50, 40
    Hq = G * Hkv
    cap = T0 + steps + 2
    rk_o, _ = oracle_rotation(D, 2, 51, rope=10000.0)
    rv_o, _ = oracle_rotation(D, 2, 52)
    rk, rv = _gpu_rot(2, 51, 10000.0), _gpu_rot(2, 52, 0.0)
    k_all = synth.heavy_tailed((B, Hkv, T0 + steps, D), 53)
    v_all = synth.heavy_tailed((B, Hkv, T0 + steps, D), 54)
    qs = synth.heavy_tailed((steps, B, Hq, D), 55)
    kc_np = _packed_cache(rk_o, k_all[:, :, :T0], cap, np.arange(T0))
    vc_np = _packed_cache(rv_o, v_all[:, :, :T0], cap)
    kc = tuple(torch.from_numpy(a).to(dev) for a in kc_np)
    vc = tuple(torch.from_numpy(a).to(dev) for a in vc_np)
    kw = torch.zeros((B, Hkv, W, D), device=dev)
    vw = torch.zeros((B, Hkv, W, D), device=dev)
    T, R = T0, 0
    for step in range(steps):
        t = T0 + step                     # position of the token this step appends
        kw[:, :, R] = torch.from_numpy(k_all[:, :, t]).to(dev)
        vw[:, :, R] = torch.from_numpy(v_all[:, :, t]).to(dev)
        R += 1
        q = torch.from_numpy(qs[step]).to(dev)
        qpos = torch.full((B,), t, dtype=torch.int64, device=dev)
        out = tq.decode_attention_window(rk, rv, q, qpos, kc, vc, T, kw, vw, R)
        torch.cuda.synchronize()
        ref = at.decode_attention_window(rk_o, rv_o, qs[step], [t] * B, tuple(a[:, :, :T] for a in kc_np),
                                         tuple(a[:, :, :T] for a in vc_np), k_all[:, :, T:T + R],
                                         v_all[:, :, T:T + R], 1 / np.sqrt(D))
        assert_close(out.cpu().numpy(), ref, what=f"step {step} T={T} R={R}")
        if R == W:                        # flush: quantize the window into records T .. T+W-1
            for b in range(B):
                for j in range(Hkv):
                    tq.quantize_kv_pair(rk, kw[b, j], rv, vw[b, j], pos_offset=T, apply_rope=True,
                                        out_k=tuple(a[b, j, T:T + W] for a in kc),
                                        out_v=tuple(a[b, j, T:T + W] for a in vc))
            torch.cuda.synchronize()
            rows = slice(T, T + W)
            for a_np, src in zip(kc_np, oracle_records(rk_o, k_all[:, :, rows].reshape(-1, D),
                                                       np.tile(np.arange(T, T + W), B * Hkv))[:3]):
                a_np[:, :, rows] = src.reshape(B, Hkv, W, -1)
            for a_np, src in zip(vc_np, oracle_records(rv_o, v_all[:, :, rows].reshape(-1, D), None)[:3]):
                a_np[:, :, rows] = src.reshape(B, Hkv, W, -1)
            gpu_k = tuple(a[:, :, rows].reshape(B * Hkv * W, -1).cpu().numpy() for a in kc)
            _, _, _, enc = oracle_records(rk_o, k_all[:, :, rows].reshape(-1, D), np.tile(np.arange(T, T + W), B * Hkv))
            compare_records(rk_o, gpu_k, enc)
            T, R = T + W, 0


def test_window_full_size_sampled(cuda_device):
    """The bench's window workload at full size, in its launch configuration:
    the Llama-3.1-8B-shaped layer (batch 16, 32 query heads over 8 KV heads,
    2+1 bits) whose 32768 tokens are 32640 packed ones plus a bf16 window of
    the last 128.  GPU-encoded caches; sampled slices checked against the
    oracle's encoding and replaced by the oracle's records; one launch; the
    sampled outputs against the oracle."""
    from vector_quantization_b200 import tq
    dev = torch.device("cuda:0")
    c = synth.CONFIGS["llama31_8b_gqa_decode"]
    B, Hq, Hkv, T, seed = c["batch"], c["q_heads"], c["kv_heads"], c["tokens"], c["seed"]
    G, R = Hq // Hkv, 128
    Tp = T - R
    rk = tq.Rotation(D, 2, synth.rotation_randomness(D, [seed, 8, 1]), rope_base=c["rope_base"], rope_max_pos=T)
    rv = tq.Rotation(D, 2, synth.rotation_randomness(D, [seed, 8, 2]))
    rk_o, _ = oracle_rotation(D, 2, [seed, 8, 1], rope=c["rope_base"])
    rv_o, _ = oracle_rotation(D, 2, [seed, 8, 2])
    samples = [(0, 0), (B - 1, Hkv - 1), (5, 6)]
    xk = synth.heavy_tailed_torch((B, Hkv, T, D), [seed, 8, 3], dev)
    kc = tq.quantize_kv(rk, xk, apply_rope=True, pos_period=T)
    kw = xk[:, :, Tp:].to(torch.bfloat16).contiguous()
    xk_s = {bj: xk[bj][:Tp].float().cpu().numpy() for bj in samples}
    del xk
    xv = synth.heavy_tailed_torch((B, Hkv, T, D), [seed, 8, 4], dev)
    vc = tq.quantize_kv(rv, xv)
    vw = xv[:, :, Tp:].to(torch.bfloat16).contiguous()
    xv_s = {bj: xv[bj][:Tp].float().cpu().numpy() for bj in samples}
    del xv
    torch.cuda.synchronize()
    ko = {bj: check_and_substitute(rk_o, kc, *bj, xk_s[bj], np.arange(Tp)) for bj in samples}
    vo = {bj: check_and_substitute(rv_o, vc, *bj, xv_s[bj]) for bj in samples}
    q = synth.heavy_tailed_torch((B, Hq, D), [seed, 8, 5], dev)
    qpos = torch.full((B,), T - 1, dtype=torch.int64, device=dev)
    out = tq.decode_attention_window(rk, rv, q, qpos, kc, vc, Tp, kw, vw, R)
    torch.cuda.synchronize()
    for b, j in samples:
        qq = q[b:b + 1, j * G:(j + 1) * G].float().cpu().numpy()
        ref = at.decode_attention_window(rk_o, rv_o, qq, [T - 1], ko[b, j], vo[b, j],
                                         kw[b:b + 1, j:j + 1].double().cpu().numpy(),
                                         vw[b:b + 1, j:j + 1].double().cpu().numpy(), 1 / np.sqrt(D))
        assert_close(out[b:b + 1, j * G:(j + 1) * G].cpu().numpy(), ref, what=f"seq {b} kv-head {j}")


def test_window_ragged_batch(cuda_device):
    """Per-sequence packed lengths with a window of R tokens after each: the
    window of sequence b sits at positions seq_lens[b] .. seq_lens[b] + R - 1,
    lengths 0, 5 and 300 in one call."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    lens, R, G, Hkv, bits = [0, 5, 300], 40, 4, 2, 2
    B, T = len(lens), max(lens)
    cap = T + 6
    rk_o, _ = oracle_rotation(D, bits, 1531, rope=10000.0)
    rv_o, _ = oracle_rotation(D, bits, 1631)
    rk, rv = _gpu_rot(bits, 1531, 10000.0), _gpu_rot(bits, 1631, 0.0)
    kc = list(_packed_cache(rk_o, synth.heavy_tailed((B, Hkv, T, D), 1731), cap, np.arange(T)))
    vc = list(_packed_cache(rv_o, synth.heavy_tailed((B, Hkv, T, D), 1831), cap))
    for b, n in enumerate(lens):
        for cache in (kc, vc):
            cache[0][b, :, n:] = 0xFF
            cache[1][b, :, n:] = 0xFF
            cache[2][b, :, n:] = np.nan
    kw, kw_ref = _window((B, Hkv, R, D), 1931, torch.float32, R + 2)
    vw, vw_ref = _window((B, Hkv, R, D), 2031, torch.float32, R + 2)
    q = torch.from_numpy(synth.heavy_tailed((B, G * Hkv, D), 2131)).to(dev)
    qpos = [n + R - 1 for n in lens]
    out = tq.decode_attention_window(rk, rv, q, torch.tensor(qpos, dtype=torch.int64, device=dev),
                                     tuple(torch.from_numpy(a).to(dev) for a in kc),
                                     tuple(torch.from_numpy(a).to(dev) for a in vc), T, kw.to(dev), vw.to(dev), R,
                                     seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    for b, n in enumerate(lens):
        ref = at.decode_attention_window(rk_o, rv_o, q[b:b + 1].double().cpu().numpy(), [qpos[b]],
                                         tuple(a[b:b + 1, :, :n] for a in kc), tuple(a[b:b + 1, :, :n] for a in vc),
                                         kw_ref[b:b + 1], vw_ref[b:b + 1], 1 / np.sqrt(D))
        assert_close(out[b:b + 1], ref, what=f"sequence {b}: {n} packed + {R} window tokens")


def test_window_flush_in_one_call_matches_per_sequence_flushes(cuda_device):
    """A ragged batch's windows flushed by one tq_quantize_kv_pair_scatter call
    (row (b, j, i) -> record (b Hkv + j) cap + T_b + i, key position T_b + i)
    give the same records, bit for bit, as one tq_quantize_kv_pair call per
    (sequence, KV head)."""
    from vector_quantization_b200 import tq
    dev = cuda_device
    lens, Hkv, R, bits = [100, 37, 0], 2, 16, 2
    B, cap = len(lens), 140
    rk, rv = _gpu_rot(bits, 1541, 10000.0), _gpu_rot(bits, 1641, 0.0)
    kw = torch.from_numpy(synth.heavy_tailed((B, Hkv, R, D), 1741)).to(torch.bfloat16).to(dev)
    vw = torch.from_numpy(synth.heavy_tailed((B, Hkv, R, D), 1841)).to(torch.bfloat16).to(dev)

    def fresh():
        return (tuple(torch.zeros((B, Hkv, cap, w), dtype=torch.uint8, device=dev) for w in (rk.code_bytes, rk.sign_bytes))
                + (torch.zeros((B, Hkv, cap, 2), dtype=torch.float32, device=dev),))
    ka, va, kb, vb = fresh(), fresh(), fresh(), fresh()
    for b, n in enumerate(lens):
        for j in range(Hkv):
            tq.quantize_kv_pair(rk, kw[b, j], rv, vw[b, j], apply_rope=True, pos_period=R, pos_offset=n,
                                out_k=tuple(a[b, j, n:n + R] for a in ka), out_v=tuple(a[b, j, n:n + R] for a in va))
    rows = np.array([(b * Hkv + j) * cap + lens[b] + i for b in range(B) for j in range(Hkv) for i in range(R)],
                    dtype=np.int64)
    pos = np.array([lens[b] + i for b in range(B) for j in range(Hkv) for i in range(R)], dtype=np.int64)
    tq.quantize_kv_pair_scatter(rk, kw, rv, vw, torch.from_numpy(rows).to(dev), kb, vb,
                                pos=torch.from_numpy(pos).to(dev), apply_rope=True)
    torch.cuda.synchronize()
    for x, y in zip(ka + va, kb + vb):
        assert torch.equal(x, y)
