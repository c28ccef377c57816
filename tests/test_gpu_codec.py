"""GPU parity of the handle tables and of tq_quantize_kv against the oracle."""
import numpy as np
import pytest
import torch

import synth
from helpers import compare_records, oracle_records, oracle_rotation
from oracle import rotation as ro

pytestmark = pytest.mark.gpu


def _gpu_rot(d, bits, seed, rope=0.0, kind="hadamard", max_pos=(1 << 20) + 8):
    from vector_quantization_b200 import tq
    rnd = synth.rotation_randomness(d, seed, dense=(kind == "dense"))
    return tq.Rotation(d, bits, rnd, kind, rope_base=rope, rope_max_pos=max_pos)


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 1), (128, 2), (128, 3)])
def test_export_matches_oracle(cuda_device, d, bits):
    g = _gpu_rot(d, bits, 21)
    o, _ = oracle_rotation(d, bits, 21)
    ex = g.export()
    np.testing.assert_allclose(ex["pi"], o.pi, rtol=0, atol=1e-7)
    np.testing.assert_array_equal(ex["s"], o.s.astype(np.float32))
    np.testing.assert_allclose(ex["levels"], o.levels, rtol=1e-10)
    np.testing.assert_allclose(ex["thresholds"], o.thresholds, rtol=1e-10, atol=1e-15)


def _run_encode(d, bits, n, dtype, rope, seed, period=None, offset=0, pos_array=False, out_stride=1, scale=1.0,
                max_pos=(1 << 20) + 8):
    from vector_quantization_b200 import tq
    g = _gpu_rot(d, bits, seed, rope=10000.0 if rope else 0.0, max_pos=max_pos)
    o, _ = oracle_rotation(d, bits, seed, rope=10000.0 if rope else 0.0)
    x = synth.heavy_tailed((n, d), seed + 1) * np.float32(scale)
    xt = torch.from_numpy(x).to(cuda_device_of()).to(dtype)
    x_used = xt.float().cpu().numpy()
    period = period or n
    pos = (np.arange(n) % period + offset).astype(np.int64)
    kw = dict(apply_rope=rope)
    if rope:
        if pos_array:
            kw["pos"] = torch.from_numpy(pos).to(xt.device)
        else:
            kw.update(pos_period=period, pos_offset=offset)
    if out_stride > 1:
        out = tq.empty_records(g, (n * out_stride,), xt.device)
        for t in out:
            t.fill_(0)
        tq.quantize_kv(g, xt, out=out, out_stride=out_stride, **kw)
        gpu = tuple(t[::out_stride].cpu().numpy() for t in out)
    else:
        gpu = tuple(t.cpu().numpy() for t in tq.quantize_kv(g, xt, **kw))
    torch.cuda.synchronize()
    _, _, _, enc = oracle_records(o, x_used, pos if rope else None)
    return compare_records(o, gpu, enc)


def cuda_device_of():
    return torch.device("cuda:0")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_parity(cuda_device, d, bits, dtype):
    _run_encode(d, bits, 1031, dtype, rope=True, seed=100 + bits)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_parity_large_batch(cuda_device, d, bits, dtype):
    """Batches of 16384 or more vectors take the tensor-core rotation kernel
    (128-row tiles, d = 64 and 128): several tiles per CTA group and a ragged
    last tile."""
    _run_encode(d, bits, 16384 + 1031, dtype, rope=True, seed=200 + bits)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_parity_small_batch(cuda_device, d, bits, dtype):
    """Batches of at most 256 vectors (a decode step's appended keys and
    values) take the block-per-vector kernel."""
    _run_encode(d, bits, 256, dtype, rope=True, seed=220 + bits, period=100, offset=(1 << 20) - 150)


def test_encode_small_batch_positions_array_strided(cuda_device):
    _run_encode(128, 3, 128, torch.bfloat16, rope=True, seed=230, offset=77, pos_array=True, out_stride=5)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [1, 2, 3])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_parity_large_batch_no_rope(cuda_device, d, bits, dtype):
    """Large batches without RoPE: bf16 rows go to the tensor core as they
    are staged, fp32 rows through the fp16 hi/lo split."""
    _run_encode(d, bits, 2 * 16384 + 389, dtype, rope=False, seed=250 + bits)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_encode_large_batch_far_positions(cuda_device, d, dtype):
    """Tensor-core kernel at the top of its RoPE range: positions up to
    2^22 - 1, where pos * theta_0 needs the widest reduction by 2 pi."""
    n = 16384 + 259
    _run_encode(d, 2, n, dtype, rope=True, seed=240, offset=(1 << 22) - n, max_pos=1 << 22)


@pytest.mark.parametrize("d", [64, 128])
def test_encode_large_batch_positions_past_reduction_range(cuda_device, d):
    """A handle whose positions may pass 2^22 takes the table-driven kernel."""
    n = 16384 + 3
    _run_encode(d, 3, n, torch.bfloat16, rope=True, seed=241, offset=(1 << 22) + 100,
                max_pos=(1 << 22) + 100 + n)


@pytest.mark.parametrize("d", [64, 128])
def test_encode_large_batch_positions_array_strided(cuda_device, d):
    _run_encode(d, 2, 16384 + 77, torch.bfloat16, rope=True, seed=210, period=5000, offset=3,
                pos_array=True, out_stride=2)


@pytest.mark.parametrize("n", [1, 7, 33, 4099])
def test_encode_ragged_counts_no_rope(cuda_device, n):
    _run_encode(128, 2, n, torch.float32, rope=False, seed=7)


def test_encode_positions_period_offset_and_array(cuda_device):
    _run_encode(128, 2, 600, torch.bfloat16, rope=True, seed=8, period=256, offset=(1 << 20) - 300)
    _run_encode(128, 3, 600, torch.float32, rope=True, seed=9, period=600, offset=12345, pos_array=True)


def test_encode_strided_output(cuda_device):
    _run_encode(128, 2, 300, torch.float32, rope=True, seed=10, out_stride=3)


@pytest.mark.parametrize("scale", [1e-10, 1e10])
def test_encode_scale_range(cuda_device, scale):
    _run_encode(128, 2, 200, torch.float32, rope=True, seed=11, scale=scale)


def test_encode_zero_vectors(cuda_device):
    from vector_quantization_b200 import tq
    g = _gpu_rot(128, 2, 12, rope=10000.0)
    x = torch.zeros((5, 128), device=cuda_device)
    codes, signs, norms = tq.quantize_kv(g, x, apply_rope=True, pos_period=5)
    torch.cuda.synchronize()
    assert torch.all(norms == 0)
    # every code = 2 (upper-middle): plane 0 all zero, plane 1 all ones
    assert torch.all(codes[:, :16] == 0) and torch.all(codes[:, 16:] == 0xFF)
    assert torch.all(signs == 0xFF)


def test_encode_rejects_bad_arguments(cuda_device):
    from vector_quantization_b200 import tq
    g = _gpu_rot(128, 2, 13, rope=10000.0)
    x = torch.zeros((4, 128), device=cuda_device)
    with pytest.raises(tq.TQError):  # position beyond the RoPE table
        tq.quantize_kv(g, x, apply_rope=True, pos_period=4, pos_offset=(1 << 21))
    g2 = _gpu_rot(128, 2, 13)
    with pytest.raises(tq.TQError):  # RoPE asked of a handle without RoPE
        tq.quantize_kv(g2, x, apply_rope=True, pos_period=4)


def test_bounded_wait_gives_up_and_context_stays_usable(cuda_device):
    """A wait on an mbarrier phase that nothing completes returns after its
    poll limit with a status the host reads; the context keeps working."""
    from vector_quantization_b200 import tq
    assert tq.wait_selftest(arrive=False) == 0
    assert tq.wait_selftest(arrive=True) == 1
    assert tq.tensor_core_selftest() == 0


def test_tensor_core_selftest(cuda_device):
    from vector_quantization_b200 import tq
    assert tq.tensor_core_selftest() == 0


def test_encode_70b_slice_full_size_sampled(cuda_device):
    """The bench's encode workload at full size: 8 KV heads x 2^20 tokens,
    d = 128, bf16, 2+1 bits, keys with RoPE (position = token index) and
    values without, each as one launch like the bench.  Sampled rows (tile
    edges, the last rows, and a seeded random set) against the oracle over the
    same bf16 inputs."""
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["llama31_70b_long_slice"]
    Hkv, d, T, seed = c["kv_heads"], c["head_dim"], c["tokens"], c["seed"]
    dev = cuda_device_of()
    n = Hkv * T
    rng = np.random.default_rng([seed, 77])
    rows = np.unique(np.concatenate([
        np.array([0, 1, 127, 128, 129, 255, 256, T - 1, T, T + 1, n - 129, n - 128, n - 2, n - 1]),
        rng.integers(0, n, size=1500)]))
    for apply_rope, tag in ((True, 3), (False, 4)):
        rnd = synth.rotation_randomness(d, [seed, 1 if apply_rope else 2])
        g = tq.Rotation(d, 2, rnd, rope_base=c["rope_base"] if apply_rope else 0.0, rope_max_pos=T)
        o = ro.build_rotation(d, 2, rnd, rope_base=c["rope_base"] if apply_rope else 0.0)
        x = synth.heavy_tailed_torch((1, Hkv, T, d), [seed, tag], dev)
        out = tq.empty_records(g, (1, Hkv, T), dev)
        kw = dict(apply_rope=True, pos_period=T) if apply_rope else {}
        tq.quantize_kv(g, x, out=out, **kw)
        torch.cuda.synchronize()
        idx = torch.from_numpy(rows).to(dev)
        xs = x.reshape(n, d).index_select(0, idx).float().cpu().numpy()
        gpu = tuple(t.reshape(n, -1).index_select(0, idx).cpu().numpy() for t in out)
        _, _, _, enc = oracle_records(o, xs, (rows % T).astype(np.int64) if apply_rope else None)
        compare_records(o, gpu, enc)
        del x, out


def test_encode_esm2_cache_full_size_sampled(cuda_device):
    """The bench's ESM-2-650M-shaped cache encode at full size: 33 layers x
    [8, 20, 1024, 64] bf16 keys (RoPE at the token's position) and values,
    2+1 bits, each as one launch like the bench (5.4M vectors, the d = 64
    tensor-core encode at two CTAs per SM), with the config's log-normal
    channel law.  Sampled rows (tile edges, the last rows, a seeded random
    set) against the oracle over the same bf16 inputs."""
    from vector_quantization_b200 import tq
    c = synth.CONFIGS["esm2_650m_encoder"]
    L, B, H, T, d, seed = c["layers"], c["batch"], c["heads"], c["tokens"], c["head_dim"], c["seed"]
    dev = cuda_device_of()
    n = L * B * H * T
    rng = np.random.default_rng([seed, 78])
    rows = np.unique(np.concatenate([
        np.array([0, 1, 127, 128, 129, 255, 256, T - 1, T, T + 1, n - 129, n - 128, n - 2, n - 1]),
        rng.integers(0, n, size=1500)]))
    for apply_rope, tag in ((True, 1), (False, 2)):
        rnd = synth.rotation_randomness(d, [seed, 9, tag])
        g = tq.Rotation(d, 2, rnd, rope_base=c["rope_base"] if apply_rope else 0.0, rope_max_pos=T)
        o = ro.build_rotation(d, 2, rnd, rope_base=c["rope_base"] if apply_rope else 0.0)
        x = synth.lognormal_channels_torch((L * B * H, T, d), [seed, 9, tag + 2], dev).reshape(n, d)
        out = tq.empty_records(g, (n,), dev)
        kw = dict(apply_rope=True, pos_period=T) if apply_rope else {}
        tq.quantize_kv(g, x, out=out, **kw)
        torch.cuda.synchronize()
        idx = torch.from_numpy(rows).to(dev)
        xs = x.index_select(0, idx).float().cpu().numpy()
        gpu = tuple(t.reshape(n, -1).index_select(0, idx).cpu().numpy() for t in out)
        _, _, _, enc = oracle_records(o, xs, (rows % T).astype(np.int64) if apply_rope else None)
        compare_records(o, gpu, enc)
        del x, out


@pytest.mark.parametrize("n", [1, 128, 256, 300])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_kv_pair_equals_two_calls(cuda_device, n, dtype):
    """The decode-step append call (keys with RoPE, values without, one launch
    up to 256 rows) writes the same records as two tq_quantize_kv calls."""
    from vector_quantization_b200 import tq
    dev = cuda_device_of()
    rk = _gpu_rot(128, 2, 260, rope=10000.0)
    rv = _gpu_rot(128, 2, 261)
    k = torch.from_numpy(synth.heavy_tailed((n, 128), 262)).to(dev).to(dtype)
    v = torch.from_numpy(synth.heavy_tailed((n, 128), 263)).to(dev).to(dtype)
    stride = 3
    kw = dict(apply_rope=True, pos_period=n, pos_offset=(1 << 20) - n)
    pk, pv = tq.empty_records(rk, (n * stride,), dev), tq.empty_records(rv, (n * stride,), dev)
    sk, sv = tq.empty_records(rk, (n * stride,), dev), tq.empty_records(rv, (n * stride,), dev)
    for t in (*pk, *pv, *sk, *sv):
        t.zero_()
    tq.quantize_kv_pair(rk, k, rv, v, out_k=pk, out_v=pv, out_stride=stride, **kw)
    tq.quantize_kv(rk, k, out=sk, out_stride=stride, **kw)
    tq.quantize_kv(rv, v, out=sv, out_stride=stride)
    torch.cuda.synchronize()
    for a, b in zip((*pk, *pv), (*sk, *sv)):
        assert torch.equal(a, b)


@pytest.mark.parametrize("d,bits,kind,seed", [(128, 2, "hadamard", 7), (64, 3, "hadamard", 2**33 + 5),
                                              (128, 1, "dense", 99)])
def test_seeded_build_matches_oracle_from_its_own_generator(cuda_device, d, bits, kind, seed):
    """tq_build_rotation_seeded draws D, S (and the Gaussian of a dense Pi)
    with the library's Philox4x32-10; the oracle draws them with its own
    implementation of that generator and builds its handle from them.  The
    exported tables agree, and encoding with the seeded handle gives the
    oracle's records."""
    from vector_quantization_b200 import tq
    from oracle import philox
    g = tq.Rotation(d, bits, seed, kind)
    o = ro.build_rotation(d, bits, philox.rotation_draws(d, seed, dense=(kind == "dense")), kind)
    ex = g.export()
    np.testing.assert_allclose(ex["pi"], o.pi, rtol=0, atol=2e-7)
    np.testing.assert_array_equal(ex["s"], o.s.astype(np.float32))
    np.testing.assert_allclose(ex["levels"], o.levels, rtol=1e-10)
    if kind == "hadamard":
        x = synth.heavy_tailed((300, d), seed % 1000 + 3)
        gpu = tq.quantize_kv(g, torch.from_numpy(x).to(cuda_device))
        codes, signs, norms, enc = oracle_records(o, x)
        compare_records(o, tuple(a.cpu().numpy() for a in gpu), enc)


@pytest.mark.parametrize("n", [100, 300])
def test_scatter_encode_places_rows_at_their_records(cuda_device, n):
    """tq_quantize_kv_scatter: row i lands in record out_rows[i] (keys with
    RoPE at their own positions), with the oracle's codes; rows whose target
    lies outside the arrays are skipped and every other record is untouched."""
    from vector_quantization_b200 import tq
    d, bits, nrec = 128, 2, 1000
    g = _gpu_rot(d, bits, 61, rope=10000.0)
    o, _ = oracle_rotation(d, bits, 61, rope=10000.0)
    rng = np.random.default_rng(62)
    x = synth.heavy_tailed((n, d), 63)
    pos = rng.integers(0, 5000, size=n).astype(np.int64)
    rows = rng.permutation(nrec)[:n].astype(np.int64)
    rows[3], rows[7] = -1, nrec + 5                      # skipped
    dev = cuda_device
    out = tuple(torch.full((nrec, w), 0xAB, dtype=torch.uint8, device=dev) for w in (g.code_bytes, g.sign_bytes))
    out = out + (torch.full((nrec, 2), -7.0, dtype=torch.float32, device=dev),)
    tq.quantize_kv_scatter(g, torch.from_numpy(x).to(dev), torch.from_numpy(rows).to(dev), out,
                           pos=torch.from_numpy(pos).to(dev), apply_rope=True)
    torch.cuda.synchronize()
    got = tuple(a.cpu().numpy() for a in out)
    keep = (rows >= 0) & (rows < nrec)
    _, _, _, enc = oracle_records(o, x[keep], pos[keep])
    compare_records(o, tuple(a[rows[keep]] for a in got), enc)
    untouched = np.setdiff1d(np.arange(nrec), rows[keep])
    assert np.all(got[0][untouched] == 0xAB) and np.all(got[1][untouched] == 0xAB)
    assert np.all(got[2][untouched] == -7.0)
