"""Thin ctypes binding of ``libtq.so`` (argument marshalling only).

Every function here checks shapes and dtypes of torch tensors, passes raw
device pointers and sizes to the C ABI declared in ``include/tq.h`` and raises
:class:`TQError` on a non-zero status.  All arithmetic runs in the library's
CUDA kernels; there is no fallback of any kind: if ``libtq.so`` is missing or
fails to load, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EWORKSPACE, TQ_ECUDA, TQ_ENOMEM = 0, -1, -2, -3, -4, -5
TQ_ROT_HADAMARD, TQ_ROT_DENSE = 0, 1
TQ_F32, TQ_BF16 = 0, 1
TQ_RES_QJL, TQ_RES_SIGN = 0, 1


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.tq_status_string(status).decode()} ({status})")


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m vector_quantization_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    c_i, c_i64, c_sz, c_p, c_d, c_f = (ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p,
                                       ctypes.c_double, ctypes.c_float)
    sig = {
        "tq_status_string": (ctypes.c_char_p, [c_i]),
        "tq_version": (c_i, []),
        "tq_lloyd_max": (c_i, [c_i, c_i, c_p, c_p]),
        "tq_build_rotation": (c_i, [c_i, c_i, c_i, c_p, c_p, c_p, c_i, c_d, c_i64, ctypes.POINTER(c_p)]),
        "tq_build_rotation_seeded": (c_i, [c_i, c_i, c_i, c_i, ctypes.c_uint64, c_i, c_d, c_i64, ctypes.POINTER(c_p)]),
        "tq_build_rotation_ex": (c_i, [c_i, c_i, c_i, c_i, c_p, c_p, c_p, c_i, c_d, c_i64, ctypes.POINTER(c_p)]),
        "tq_rotation_draws": (c_i, [c_i, c_i, ctypes.c_uint64, c_i, c_p, c_p, c_p]),
        "tq_free_rotation": (c_i, [c_p]),
        "tq_rotation_export": (c_i, [c_p, c_p, c_p, c_p, c_p]),
        "tq_rotation_dims": (c_i, [c_p, c_p, c_p, c_p, c_p, c_p]),
        "tq_quantize_kv": (c_i, [c_p, c_p, c_i, c_i64, c_i64, c_p, c_i64, c_i64, c_i, c_p, c_p, c_p, c_i64, c_p]),
        "tq_quantize_kv_pair": (c_i, [c_p, c_p, c_p, c_p, c_i, c_i64, c_i64, c_p, c_i64, c_i64, c_i,
                                      c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_p]),
        "tq_decode_attention": (c_i, [c_p, c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_i, c_i, c_i,
                                      c_i64, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "tq_decode_attention_append": (c_i, [c_p, c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64,
                                             c_i, c_i, c_i, c_i64, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "tq_nsn_shift": (c_i, [c_p, c_p, c_i, c_i64, c_i64, c_i64, c_i64, c_i, c_p, c_p, c_p, c_p]),
        "tq_decode_attention_nsn": (c_i, [c_p, c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_p,
                                          c_i64, c_i, c_i, c_i, c_i64, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "tq_decode_attention_nsn_append": (c_i, [c_p, c_p, c_p, c_i] + [c_p] * 13 +
                                           [c_i64, c_i, c_i, c_i, c_i64, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "tq_decode_workspace_size": (c_sz, [c_p, c_p, c_i, c_i, c_i, c_i64]),
        "tq_decode_partials": (c_i, [c_p, c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_i, c_i, c_i,
                                     c_i64, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "tq_decode_merge_partials": (c_i, [c_p, c_p, c_i, c_i, c_i, c_i, c_p, c_p]),
        "tq_search_merge_topk": (c_i, [c_p, c_p, c_i, c_i, c_i, c_p, c_p, c_p, c_p]),
        "tq_decode_attention_window": (c_i, [c_p, c_p, c_p, c_i, c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_p, c_p,
                                             c_i, c_i64, c_i, c_i, c_i, c_i, c_i64, c_p, c_f, c_p, c_p, c_sz, c_p]),
        "tq_decode_window_workspace_size": (c_sz, [c_p, c_p, c_i, c_i, c_i, c_i64, c_i]),
        "tq_profile_next_decode": (c_i, [c_p, c_p]),
        "tq_encoder_attention": (c_i, [c_p, c_p, c_p, c_i, c_i64, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_i, c_i,
                                       c_i, c_i, c_i64, c_f, c_p, c_p, c_sz, c_p]),
        "tq_encoder_workspace_size": (c_sz, [c_p, c_i, c_i, c_i]),
        "tq_quantize_dense": (c_i, [c_p, c_p, c_i64, c_i64, c_p, c_p, c_p, c_p, c_sz, c_p]),
        "tq_quantize_kv_scatter": (c_i, [c_p, c_p, c_i, c_i64, c_i64, c_p, c_i64, c_i64, c_i, c_p, c_p, c_p, c_p,
                                         c_i64, c_p]),
        "tq_quantize_kv_pair_scatter": (c_i, [c_p, c_p, c_p, c_p, c_i, c_i64, c_i64, c_p, c_i64, c_i64, c_i,
                                              c_p, c_p, c_p, c_p, c_p, c_p, c_p, c_i64, c_p]),
        "tq_quantize_dense_workspace_size": (c_sz, [c_p, c_i64]),
        "tq_search_topk": (c_i, [c_p, c_p, c_i, c_p, c_p, c_p, c_i64, c_i, c_p, c_p, c_p, c_sz, c_p]),
        "tq_search_workspace_size": (c_sz, [c_p, c_i, c_i64, c_i]),
        "tq_tensor_core_selftest": (c_i, [c_p]),
        "tq_wait_selftest": (c_i, [c_i, c_p]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def _check(status: int, where: str):
    if status != TQ_OK:
        raise TQError(status, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream_ptr(stream) -> int | None:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def version() -> int:
    return _lib.tq_version()


def wait_selftest(arrive: bool) -> int:
    """1 if a bounded mbarrier wait saw its phase complete, 0 if it gave up."""
    done = ctypes.c_int(-1)
    _check(_lib.tq_wait_selftest(1 if arrive else 0, ctypes.byref(done)), "tq_wait_selftest")
    return done.value


def tensor_core_selftest() -> int:
    """Run the device self-test of the tcgen05 path; returns the number of
    wrong elements of a 128^3 exact product (0 when working)."""
    bad = ctypes.c_int64()
    _check(_lib.tq_tensor_core_selftest(ctypes.byref(bad)), "tq_tensor_core_selftest")
    return bad.value


def lloyd_max(d: int, bits: int):
    """Host-only Lloyd-Max codebook of the library: (levels, thresholds) float64."""
    lv = np.zeros(1 << bits)
    th = np.zeros((1 << bits) - 1)
    _check(_lib.tq_lloyd_max(d, bits, lv.ctypes.data, th.ctypes.data), "tq_lloyd_max")
    return lv, th


def rotation_draws(d: int, seed: int, kind: str = "hadamard", m: int | None = None) -> dict:
    """Host-only: the draws a handle built from ``seed`` uses (the library's
    Philox4x32-10 streams): signs int8 [d], gauss_s float32 [m, d] and, for
    ``kind='dense'``, gauss_pi float64 [d, d]."""
    m = d if m is None else m
    kind_code = {"hadamard": TQ_ROT_HADAMARD, "dense": TQ_ROT_DENSE}[kind]
    signs = np.zeros(d, np.int8)
    gs = np.zeros((m, d), np.float32)
    gp = np.zeros((d, d), np.float64) if kind == "dense" else None
    _check(_lib.tq_rotation_draws(d, kind_code, int(seed) & (2**64 - 1), m, signs.ctypes.data,
                                  None if gp is None else gp.ctypes.data, gs.ctypes.data), "tq_rotation_draws")
    return {"signs": signs, "gauss_s": gs, "gauss_pi": gp}


class Rotation:
    """A codec handle (rotation, QJL matrix, codebook, RoPE tables) on the
    current CUDA device.  ``randomness`` is either a dict of draws (``signs``,
    ``gauss_s`` and, for ``kind='dense'``, ``gauss_pi``) or an integer seed,
    from which the library draws them itself (tq_build_rotation_seeded)."""

    def __init__(self, d: int, bits: int, randomness, kind: str = "hadamard",
                 rope_base: float = 0.0, rope_max_pos: int = 1 << 21, residual: str = "qjl"):
        kind_code = {"hadamard": TQ_ROT_HADAMARD, "dense": TQ_ROT_DENSE}[kind]
        res_code = {"qjl": TQ_RES_QJL, "sign": TQ_RES_SIGN}[residual]
        h = ctypes.c_void_p()
        if isinstance(randomness, (int, np.integer)):
            _check(_lib.tq_build_rotation_seeded(d, bits, kind_code, res_code, int(randomness) & (2**64 - 1), d,
                                                 float(rope_base), int(rope_max_pos), ctypes.byref(h)),
                   "tq_build_rotation_seeded")
        else:
            signs = np.ascontiguousarray(randomness["signs"], dtype=np.int8)
            gs = np.ascontiguousarray(randomness["gauss_s"], dtype=np.float32)
            gp = randomness.get("gauss_pi")
            gp = None if gp is None else np.ascontiguousarray(gp, dtype=np.float64)
            _check(_lib.tq_build_rotation_ex(d, bits, kind_code, res_code, signs.ctypes.data,
                                             None if gp is None else gp.ctypes.data, gs.ctypes.data, gs.shape[0],
                                             float(rope_base), int(rope_max_pos), ctypes.byref(h)),
                   "tq_build_rotation_ex")
        self._h = h
        dd, mm, bb = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
        cb, sb = ctypes.c_int64(), ctypes.c_int64()
        _check(_lib.tq_rotation_dims(h, ctypes.byref(dd), ctypes.byref(mm), ctypes.byref(bb), ctypes.byref(cb),
                                     ctypes.byref(sb)), "tq_rotation_dims")
        self.d, self.m, self.bits = dd.value, mm.value, bb.value
        self.code_bytes, self.sign_bytes = cb.value, sb.value
        self.kind = kind
        self.residual = residual
        self.rope_base = rope_base

    @property
    def handle(self):
        return self._h

    def export(self) -> dict:
        d, m, n = self.d, self.m, 1 << self.bits
        pi = np.zeros((d, d), np.float32)
        s = np.zeros((m, d), np.float32)
        lv = np.zeros(n)
        th = np.zeros(n - 1)
        _check(_lib.tq_rotation_export(self._h, pi.ctypes.data, s.ctypes.data, lv.ctypes.data, th.ctypes.data),
               "tq_rotation_export")
        return {"pi": pi, "s": s, "levels": lv, "thresholds": th}

    def close(self):
        if getattr(self, "_h", None):
            _lib.tq_free_rotation(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def empty_records(rot: Rotation, shape, device):
    """Allocate (codes, signs, norms) arrays for ``shape`` records."""
    import torch
    shape = tuple(shape)
    codes = torch.empty(shape + (rot.code_bytes,), dtype=torch.uint8, device=device)
    signs = torch.empty(shape + (rot.sign_bytes,), dtype=torch.uint8, device=device)
    norms = torch.empty(shape + (2,), dtype=torch.float32, device=device)
    return codes, signs, norms


def quantize_kv(rot: Rotation, x, *, pos=None, pos_period: int | None = None, pos_offset: int = 0,
                apply_rope: bool = False, out=None, out_stride: int = 1, stream=None):
    """Encode the rows of ``x`` ([n, d] or [..., d], float32/bfloat16, CUDA).

    Returns (codes, signs, norms).  With ``out`` the records are written into
    the given arrays (row i at record i * out_stride of each)."""
    d = x.shape[-1]
    x2 = x.reshape(-1, d)
    if x2.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    n = x2.shape[0]
    ld = x2.stride(0) if n > 1 else d
    if out is None:
        out = empty_records(rot, x.shape[:-1], x.device)
    codes, signs, norms = out
    if pos is not None and pos.dtype.is_floating_point:
        raise TypeError("pos must be int64")
    period = pos_period if pos_period is not None else max(n, 1)
    _check(_lib.tq_quantize_kv(rot.handle, _ptr(x2), _dtype_code(x2), n, ld, _ptr(pos), period, pos_offset,
                               1 if apply_rope else 0, _ptr(codes), _ptr(signs), _ptr(norms), out_stride,
                               _stream_ptr(stream)), "tq_quantize_kv")
    return codes, signs, norms


def quantize_kv_pair(rot_k: Rotation, xk, rot_v: Rotation, xv, *, pos=None, pos_period: int | None = None,
                     pos_offset: int = 0, apply_rope: bool = False, out_k=None, out_v=None, out_stride: int = 1,
                     stream=None):
    """Encode the keys ``xk`` (RoPE as in :func:`quantize_kv`) and values
    ``xv`` (no RoPE) a decode step appends, in one call; both [n, d] or
    [..., d] of one dtype and row stride.  Returns ((k records), (v records))."""
    d = xk.shape[-1]
    k2, v2 = xk.reshape(-1, d), xv.reshape(-1, d)
    if k2.stride(-1) != 1 or v2.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    if k2.shape != v2.shape or k2.dtype != v2.dtype or k2.stride(0) != v2.stride(0):
        raise ValueError("keys and values must share shape, dtype and row stride")
    n = k2.shape[0]
    ld = k2.stride(0) if n > 1 else d
    if out_k is None:
        out_k = empty_records(rot_k, xk.shape[:-1], xk.device)
    if out_v is None:
        out_v = empty_records(rot_v, xv.shape[:-1], xv.device)
    if pos is not None and pos.dtype.is_floating_point:
        raise TypeError("pos must be int64")
    period = pos_period if pos_period is not None else max(n, 1)
    _check(_lib.tq_quantize_kv_pair(rot_k.handle, _ptr(k2), rot_v.handle, _ptr(v2), _dtype_code(k2), n, ld, _ptr(pos),
                                    period, pos_offset, 1 if apply_rope else 0, _ptr(out_k[0]), _ptr(out_k[1]),
                                    _ptr(out_k[2]), _ptr(out_v[0]), _ptr(out_v[1]), _ptr(out_v[2]), out_stride,
                                    _stream_ptr(stream)), "tq_quantize_kv_pair")
    return out_k, out_v


def _rows_of(x, d):
    x2 = x.reshape(-1, d)
    if x2.stride(-1) != 1:
        raise ValueError("x rows must be contiguous")
    return x2, (x2.stride(0) if x2.shape[0] > 1 else d)


def _record_count(cache):
    codes, signs, norms = cache
    for t in cache:
        if not t.is_contiguous():
            raise ValueError("record arrays must be contiguous")
    n = codes.numel() // codes.shape[-1]
    if signs.numel() // signs.shape[-1] != n or norms.numel() // 2 != n:
        raise ValueError("codes, signs and norms must hold the same number of records")
    return n


def quantize_kv_scatter(rot: Rotation, x, out_rows, out, *, pos=None, pos_period: int | None = None,
                        pos_offset: int = 0, apply_rope: bool = False, stream=None):
    """Encode the rows of ``x`` ([n, d] or [..., d]) into records
    ``out_rows[i]`` (int64 device tensor [n]) of the arrays ``out`` (codes,
    signs, norms of any shape [..., record]); rows whose target lies outside
    the arrays are skipped.  Returns ``out``."""
    d = x.shape[-1]
    x2, ld = _rows_of(x, d)
    n = x2.shape[0]
    rows = out_rows.contiguous()
    if rows.dtype != __import__("torch").int64 or rows.numel() != n:
        raise ValueError("out_rows must be int64 with one entry per row")
    period = pos_period if pos_period is not None else max(n, 1)
    _check(_lib.tq_quantize_kv_scatter(rot.handle, _ptr(x2), _dtype_code(x2), n, ld, _ptr(pos), period, pos_offset,
                                       1 if apply_rope else 0, _ptr(out[0]), _ptr(out[1]), _ptr(out[2]), _ptr(rows),
                                       _record_count(out), _stream_ptr(stream)), "tq_quantize_kv_scatter")
    return out


def quantize_kv_nsn(rot: Rotation, x, *, apply_rope: bool = False, pos_offset: int = 0, out=None, stream=None):
    """NSN record mode ([NSNQuant] §1): x [..., L, d] (float32/bfloat16) as
    blocks of L tokens (row t of a block at position pos_offset + t).  Each
    block is shifted by tq_nsn_shift and the shifted rows x' are encoded by
    the codec without RoPE.  Returns ((codes, signs, norms), s1, o) with the
    records and s1 shaped [..., L] and o [..., d].  With ``out`` (record arrays
    [..., cap, ...], cap >= L) the records land in the first L slots of each
    block."""
    import torch
    *lead, L, d = x.shape
    nb = int(np.prod(lead)) if lead else 1
    x3 = x.reshape(nb * L, d)
    if x3.stride(-1) != 1 or (nb * L > 1 and x3.stride(0) != d):
        x3 = x3.contiguous()
    xs = torch.empty((nb * L, d), dtype=torch.float32, device=x.device)
    s1 = torch.empty((nb * L,), dtype=torch.float32, device=x.device)
    o = torch.empty((nb, d), dtype=torch.float32, device=x.device)
    _check(_lib.tq_nsn_shift(rot.handle, _ptr(x3), _dtype_code(x3), nb, L, d, pos_offset, 1 if apply_rope else 0,
                             _ptr(xs), _ptr(s1), _ptr(o), _stream_ptr(stream)), "tq_nsn_shift")
    if out is None:
        rec = quantize_kv(rot, xs, stream=stream)
        rec = tuple(a.view(*lead, L, -1) for a in rec)
    else:
        cap = out[0].shape[-2]
        if cap == L:
            quantize_kv(rot, xs, out=tuple(a.view(nb * L, -1) for a in out), stream=stream)
        else:
            rows = (torch.arange(nb, device=x.device, dtype=torch.int64).repeat_interleave(L) * cap +
                    torch.arange(L, device=x.device, dtype=torch.int64).repeat(nb))
            quantize_kv_scatter(rot, xs, rows, tuple(a.view(nb * cap, -1) for a in out), stream=stream)
        rec = out
    return rec, s1.view(*lead, L), o.view(*lead, d)


def quantize_kv_pair_scatter(rot_k: Rotation, xk, rot_v: Rotation, xv, out_rows, out_k, out_v, *, pos=None,
                             pos_period: int | None = None, pos_offset: int = 0, apply_rope: bool = False,
                             stream=None):
    """Keys (RoPE as in quantize_kv) and values into records ``out_rows[i]``
    of ``out_k`` and ``out_v`` (one launch for up to 256 rows)."""
    d = xk.shape[-1]
    k2, ld = _rows_of(xk, d)
    v2, ldv = _rows_of(xv, d)
    if k2.shape != v2.shape or k2.dtype != v2.dtype or ld != ldv:
        raise ValueError("keys and values must share shape, dtype and row stride")
    n = k2.shape[0]
    rows = out_rows.contiguous()
    if rows.dtype != __import__("torch").int64 or rows.numel() != n:
        raise ValueError("out_rows must be int64 with one entry per row")
    nrec = _record_count(out_k)
    if _record_count(out_v) != nrec:
        raise ValueError("key and value arrays must hold the same number of records")
    period = pos_period if pos_period is not None else max(n, 1)
    _check(_lib.tq_quantize_kv_pair_scatter(rot_k.handle, _ptr(k2), rot_v.handle, _ptr(v2), _dtype_code(k2), n, ld,
                                            _ptr(pos), period, pos_offset, 1 if apply_rope else 0, _ptr(out_k[0]),
                                            _ptr(out_k[1]), _ptr(out_k[2]), _ptr(out_v[0]), _ptr(out_v[1]),
                                            _ptr(out_v[2]), _ptr(rows), nrec, _stream_ptr(stream)),
           "tq_quantize_kv_pair_scatter")
    return out_k, out_v


def profile_next_decode(ev_begin, ev_end):
    """Have the next decode_attention call (this thread) record the two
    torch.cuda.Event objects around its split-KV kernel."""
    for ev in (ev_begin, ev_end):
        if ev is not None and not ev.cuda_event:
            ev.record()  # torch creates the underlying cudaEvent lazily, on first record
    _check(_lib.tq_profile_next_decode(ev_begin.cuda_event if ev_begin is not None else None,
                                       ev_end.cuda_event if ev_end is not None else None), "tq_profile_next_decode")


def decode_workspace_size(rot_k: Rotation, rot_v: Rotation, B: int, Hq: int, Hkv: int, T: int) -> int:
    return _lib.tq_decode_workspace_size(rot_k.handle, rot_v.handle, B, Hq, Hkv, T)


def alloc_workspace(nbytes: int, device):
    import torch
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def _seq_lens(seq_lens, B, device):
    """Per-sequence lengths as a contiguous int32 device tensor [B], or None."""
    if seq_lens is None:
        return None
    import torch
    t = torch.as_tensor(seq_lens, dtype=torch.int32, device=device).contiguous()
    if t.shape != (B,):
        raise ValueError(f"seq_lens must have shape ({B},)")
    return t


def decode_attention(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, T: int, *, seq_lens=None,
                     scale: float | None = None, out=None, workspace=None, stream=None):
    """One decode step: q [B, Hq, d] against caches (codes, signs, norms) of
    shape [B, Hkv, cap, ...]; attends to the first T records of each
    sequence, or to the first seq_lens[b] (each <= T) of sequence b.
    Returns out [B, Hq, d] float32."""
    import torch
    B, Hq, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    for t in (kc, ks, kn, vc, vs, vn):
        if not t.is_contiguous():
            raise ValueError("cache arrays must be contiguous")
    q = q.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(rot_k, rot_v, B, Hq, Hkv, T)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    lens = _seq_lens(seq_lens, B, q.device)
    _check(_lib.tq_decode_attention(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), _ptr(q_pos), _ptr(kc),
                                    _ptr(ks), _ptr(kn), _ptr(vc), _ptr(vs), _ptr(vn), cap, B, Hq, Hkv, T, _ptr(lens),
                                    float(scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                    _stream_ptr(stream)), "tq_decode_attention")
    return out


def decode_attention_append(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_new, v_new, k_cache, v_cache, T: int, *,
                            seq_lens=None, scale: float | None = None, out=None, workspace=None, stream=None):
    """One decode step that first appends the new token: k_new, v_new
    [B, Hkv, d] (or [B*Hkv, d]) in q's dtype are encoded into record T - 1
    (seq_lens[b] - 1 for sequence b) of each sequence, the key with RoPE at
    q_pos[b]; then q [B, Hq, d] attends to the first T (seq_lens[b]) records.
    One launch does the append and the query preparation.  Returns out
    [B, Hq, d] float32."""
    import torch
    B, Hq, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    for t in (kc, ks, kn, vc, vs, vn):
        if not t.is_contiguous():
            raise ValueError("cache arrays must be contiguous")
    if k_new.dtype != q.dtype or v_new.dtype != q.dtype:
        raise ValueError("k_new and v_new must have the query's dtype")
    if k_new.numel() != B * Hkv * d or v_new.numel() != B * Hkv * d:
        raise ValueError("k_new and v_new must hold B * Hkv rows of d")
    q, k_new, v_new = q.contiguous(), k_new.contiguous(), v_new.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(rot_k, rot_v, B, Hq, Hkv, T)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    lens = _seq_lens(seq_lens, B, q.device)
    _check(_lib.tq_decode_attention_append(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), _ptr(q_pos),
                                           _ptr(k_new), _ptr(v_new), _ptr(kc), _ptr(ks), _ptr(kn), _ptr(vc), _ptr(vs),
                                           _ptr(vn), cap, B, Hq, Hkv, T, _ptr(lens), float(scale), _ptr(out),
                                           _ptr(workspace), workspace.numel(), _stream_ptr(stream)),
           "tq_decode_attention_append")
    return out


def decode_attention_nsn(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, k_s1, k_o, v_s1, v_o,
                         T: int, *, seq_lens=None, scale: float | None = None, out=None, workspace=None, stream=None):
    """decode_attention over NSN records (quantize_kv_nsn): k_s1, v_s1
    [B, Hkv, cap] float32 beside the caches, k_o, v_o [B, Hkv, d] float32.
    Returns out [B, Hq, d] float32."""
    import torch
    B, Hq, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    side = (k_s1, k_o, v_s1, v_o)
    for t in (kc, ks, kn, vc, vs, vn) + side:
        if not t.is_contiguous():
            raise ValueError("cache and NSN arrays must be contiguous")
    if k_s1.shape[-1] != cap or v_s1.shape[-1] != cap or k_o.numel() != B * Hkv * d or v_o.numel() != B * Hkv * d:
        raise ValueError("s1 arrays must be [B, Hkv, cap] and shifts [B, Hkv, d]")
    q = q.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(rot_k, rot_v, B, Hq, Hkv, T)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    lens = _seq_lens(seq_lens, B, q.device)
    _check(_lib.tq_decode_attention_nsn(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), _ptr(q_pos), _ptr(kc),
                                        _ptr(ks), _ptr(kn), _ptr(vc), _ptr(vs), _ptr(vn), _ptr(k_s1), _ptr(k_o),
                                        _ptr(v_s1), _ptr(v_o), cap, B, Hq, Hkv, T, _ptr(lens), float(scale), _ptr(out),
                                        _ptr(workspace), workspace.numel(), _stream_ptr(stream)),
           "tq_decode_attention_nsn")
    return out


def decode_attention_nsn_append(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_new, v_new, k_cache, v_cache, k_s1, k_o,
                                v_s1, v_o, T: int, *, seq_lens=None, scale: float | None = None, out=None,
                                workspace=None, stream=None):
    """decode_attention_append over NSN records: each new row (the key after
    RoPE at q_pos[b]) is shifted by its sequence's o (k_o, v_o [B, Hkv, d],
    not changed) and its s1 written into k_s1 / v_s1 [B, Hkv, cap] next to
    its record; then decode_attention_nsn over the first T (seq_lens[b])
    records.  Returns out [B, Hq, d] float32."""
    import torch
    B, Hq, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    for t in (kc, ks, kn, vc, vs, vn, k_s1, k_o, v_s1, v_o):
        if not t.is_contiguous():
            raise ValueError("cache and NSN arrays must be contiguous")
    if k_s1.shape[-1] != cap or v_s1.shape[-1] != cap or k_o.numel() != B * Hkv * d or v_o.numel() != B * Hkv * d:
        raise ValueError("s1 arrays must be [B, Hkv, cap] and shifts [B, Hkv, d]")
    if k_new.dtype != q.dtype or v_new.dtype != q.dtype:
        raise ValueError("k_new and v_new must have the query's dtype")
    if k_new.numel() != B * Hkv * d or v_new.numel() != B * Hkv * d:
        raise ValueError("k_new and v_new must hold B * Hkv rows of d")
    q, k_new, v_new = q.contiguous(), k_new.contiguous(), v_new.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(rot_k, rot_v, B, Hq, Hkv, T)
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    lens = _seq_lens(seq_lens, B, q.device)
    _check(_lib.tq_decode_attention_nsn_append(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), _ptr(q_pos),
                                               _ptr(k_new), _ptr(v_new), _ptr(kc), _ptr(ks), _ptr(kn), _ptr(vc),
                                               _ptr(vs), _ptr(vn), _ptr(k_s1), _ptr(k_o), _ptr(v_s1), _ptr(v_o), cap,
                                               B, Hq, Hkv, T, _ptr(lens), float(scale), _ptr(out), _ptr(workspace),
                                               workspace.numel(), _stream_ptr(stream)),
           "tq_decode_attention_nsn_append")
    return out


def decode_partials(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, T: int, *, seq_lens=None,
                    scale: float | None = None, out=None, workspace=None, stream=None):
    """Partial softmax records of one decode step over this call's tokens:
    returns [B, Hq, 2 + 2 d] float32 (max, sum, O_code[d], O_z[d] per query
    head), to be combined with other token ranges by decode_merge_partials."""
    import torch
    B, Hq, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    for t in (kc, ks, kn, vc, vs, vn):
        if not t.is_contiguous():
            raise ValueError("cache arrays must be contiguous")
    q = q.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, 2 + 2 * d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(decode_workspace_size(rot_k, rot_v, B, Hq, Hkv, T), q.device)
    lens = _seq_lens(seq_lens, B, q.device)
    _check(_lib.tq_decode_partials(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), _ptr(q_pos), _ptr(kc),
                                   _ptr(ks), _ptr(kn), _ptr(vc), _ptr(vs), _ptr(vn), cap, B, Hq, Hkv, T, _ptr(lens),
                                   float(scale), _ptr(out), _ptr(workspace), workspace.numel(), _stream_ptr(stream)),
           "tq_decode_partials")
    return out


def decode_merge_partials(rot_v: Rotation, partials, Hkv: int, *, out=None, stream=None):
    """Attention output [B, Hq, d] from partial records [P, B, Hq, 2 + 2 d]."""
    import torch
    P, B, Hq, rec = partials.shape
    d = (rec - 2) // 2
    partials = partials.contiguous()
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=partials.device)
    _check(_lib.tq_decode_merge_partials(rot_v.handle, _ptr(partials), P, B, Hq, Hkv, _ptr(out), _stream_ptr(stream)),
           "tq_decode_merge_partials")
    return out


def search_merge_topk(cand_scores, cand_ids, k: int, *, id_offsets=None, stream=None):
    """Best k of L candidate lists per query: cand_scores [L, nq, k] float32,
    cand_ids [L, nq, k] int64, id_offsets [L] int64 or None.  Returns
    (scores [nq, k], ids [nq, k])."""
    import torch
    L, nq, kk = cand_scores.shape
    if kk != k or cand_ids.shape != cand_scores.shape:
        raise ValueError("candidate lists must be [L, nq, k]")
    cs, ci = cand_scores.contiguous(), cand_ids.contiguous()
    offs = None if id_offsets is None else torch.as_tensor(id_offsets, dtype=torch.int64,
                                                          device=cs.device).contiguous()
    scores = torch.empty((nq, k), dtype=torch.float32, device=cs.device)
    ids = torch.empty((nq, k), dtype=torch.int64, device=cs.device)
    _check(_lib.tq_search_merge_topk(_ptr(cs), _ptr(ci), L, nq, k, _ptr(offs), _ptr(scores), _ptr(ids),
                                     _stream_ptr(stream)), "tq_search_merge_topk")
    return scores, ids


def decode_window_workspace_size(rot_k: Rotation, rot_v: Rotation, B: int, Hq: int, Hkv: int, T: int,
                                 R: int) -> int:
    return _lib.tq_decode_window_workspace_size(rot_k.handle, rot_v.handle, B, Hq, Hkv, T, R)


def decode_attention_window(rot_k: Rotation, rot_v: Rotation, q, q_pos, k_cache, v_cache, T: int, k_window,
                            v_window, R: int, *, seq_lens=None, scale: float | None = None, out=None, workspace=None,
                            stream=None):
    """One decode step over the first T records of the packed caches (or
    seq_lens[b] of sequence b) plus the first R tokens of the full-precision
    windows k_window, v_window ([B, Hkv, cap_w, d], float32 or bfloat16, keys
    before RoPE); window token i sits at position T + i (seq_lens[b] + i).
    Returns out [B, Hq, d] float32."""
    import torch
    B, Hq, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    for t in (kc, ks, kn, vc, vs, vn, k_window, v_window):
        if not t.is_contiguous():
            raise ValueError("cache and window arrays must be contiguous")
    if k_window.shape != v_window.shape or k_window.dtype != v_window.dtype:
        raise ValueError("k_window and v_window must share shape and dtype")
    q = q.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(decode_window_workspace_size(rot_k, rot_v, B, Hq, Hkv, T, R), q.device)
    lens = _seq_lens(seq_lens, B, q.device)
    _check(_lib.tq_decode_attention_window(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), _ptr(q_pos), _ptr(kc),
                                           _ptr(ks), _ptr(kn), _ptr(vc), _ptr(vs), _ptr(vn), cap, _ptr(k_window),
                                           _ptr(v_window), _dtype_code(k_window), k_window.shape[2], R, B, Hq, Hkv,
                                           T, _ptr(lens), float(scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                           _stream_ptr(stream)), "tq_decode_attention_window")
    return out


def encoder_attention(rot_k: Rotation, rot_v: Rotation, q, k_cache, v_cache, T: int, *, q_pos_offset: int = 0,
                      scale: float | None = None, out=None, workspace=None, stream=None):
    """Bidirectional attention: q [B, Hq, S, d] against caches [B, Hkv, cap, ...]
    (first T records of each sequence).  Returns out [B, Hq, S, d] float32."""
    import torch
    B, Hq, S, d = q.shape
    kc, ks, kn = k_cache
    vc, vs, vn = v_cache
    Hkv, cap = kc.shape[1], kc.shape[2]
    q = q.contiguous()
    if scale is None:
        scale = 1.0 / float(np.sqrt(d))
    if out is None:
        out = torch.empty((B, Hq, S, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(_lib.tq_encoder_workspace_size(rot_k.handle, B, Hq, S), q.device)
    _check(_lib.tq_encoder_attention(rot_k.handle, rot_v.handle, _ptr(q), _dtype_code(q), q_pos_offset, _ptr(kc),
                                     _ptr(ks), _ptr(kn), _ptr(vc), _ptr(vs), _ptr(vn), cap, B, Hq, Hkv, S, T,
                                     float(scale), _ptr(out), _ptr(workspace), workspace.numel(),
                                     _stream_ptr(stream)), "tq_encoder_attention")
    return out


def quantize_dense(rot: Rotation, x, *, out=None, workspace=None, stream=None):
    """Encode rows of x ([n, d] float32, CUDA) with a dense-rotation handle.
    Returns (codes, signs, norms)."""
    import torch
    if x.dtype != torch.float32:
        raise TypeError("quantize_dense takes float32 input")
    x2 = x.reshape(-1, x.shape[-1])
    n = x2.shape[0]
    ld = x2.stride(0) if n > 1 else x2.shape[1]
    if out is None:
        out = empty_records(rot, (n,), x.device)
    codes, signs, norms = out
    if workspace is None:
        workspace = alloc_workspace(_lib.tq_quantize_dense_workspace_size(rot.handle, n), x.device)
    _check(_lib.tq_quantize_dense(rot.handle, _ptr(x2), n, ld, _ptr(codes), _ptr(signs), _ptr(norms),
                                  _ptr(workspace), workspace.numel(), _stream_ptr(stream)), "tq_quantize_dense")
    return codes, signs, norms


def search_workspace_size(rot: Rotation, nq: int, N: int, k: int) -> int:
    return _lib.tq_search_workspace_size(rot.handle, nq, N, k)


def search_topk(rot: Rotation, queries, db, k: int = 10, *, workspace=None, stream=None):
    """Top-k inner products of queries ([nq, d] float32) against the packed
    database db = (codes, signs, norms).  Returns (scores [nq, k], ids [nq, k])."""
    import torch
    q = queries.contiguous()
    nq = q.shape[0]
    codes, signs, norms = db
    N = codes.shape[0]
    scores = torch.empty((nq, k), dtype=torch.float32, device=q.device)
    ids = torch.empty((nq, k), dtype=torch.int64, device=q.device)
    if workspace is None:
        workspace = alloc_workspace(search_workspace_size(rot, nq, N, k), q.device)
    _check(_lib.tq_search_topk(rot.handle, _ptr(q), nq, _ptr(codes), _ptr(signs), _ptr(norms), N, k, _ptr(scores),
                               _ptr(ids), _ptr(workspace), workspace.numel(), _stream_ptr(stream)), "tq_search_topk")
    return scores, ids
