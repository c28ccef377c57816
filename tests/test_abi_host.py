"""CPU checks of the C ABI: the library loads, exports every declared entry
point, and its host-only codebook agrees with the oracle."""
import ctypes
import os
import re

import numpy as np
import pytest

from conftest import ROOT
from oracle import codebook as cb

HEADER = os.path.join(ROOT, "include", "tq.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    from vector_quantization_b200 import tq
    lib = ctypes.CDLL(tq.LIB_PATH)
    names = _declared()
    assert len(names) >= 10
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_and_version():
    from vector_quantization_b200 import tq
    assert tq.version() >= 100
    for code in (0, -1, -2, -3, -4, -5):
        assert tq._lib.tq_status_string(code)


@pytest.mark.parametrize("d,bits", [(3, 2), (64, 1), (64, 2), (128, 2), (128, 3), (1536, 1), (1536, 3)])
def test_library_codebook_matches_oracle(d, bits):
    from vector_quantization_b200 import tq
    lv, th = tq.lloyd_max(d, bits)
    olv, oth = cb.lloyd_max(d, bits)
    # Two independent fixed-point iterations (incomplete beta by continued
    # fraction vs scipy) stop a few 1e-12 apart: Lloyd-Max converges linearly.
    # Thresholds that close move a code only inside the 1e-5 flag band.
    np.testing.assert_allclose(lv, olv, rtol=1e-10, atol=1e-15)
    np.testing.assert_allclose(th, oth, rtol=1e-10, atol=1e-15)


def test_bad_arguments_are_rejected_on_host():
    from vector_quantization_b200 import tq
    lv = np.zeros(4)
    assert tq._lib.tq_lloyd_max(2, 2, lv.ctypes.data, lv.ctypes.data) == tq.TQ_EINVAL
    assert tq._lib.tq_lloyd_max(64, 9, lv.ctypes.data, lv.ctypes.data) == tq.TQ_EINVAL
    h = ctypes.c_void_p()
    g = np.zeros((64, 64), np.float32)
    s = np.ones(64, np.int8)
    # m != d, bits out of range, bad kind, bad signs: all rejected before any device call
    assert tq._lib.tq_build_rotation(64, 2, 0, s.ctypes.data, None, g.ctypes.data, 32, 0.0, 0, ctypes.byref(h)) == tq.TQ_EINVAL
    assert tq._lib.tq_build_rotation(64, 4, 0, s.ctypes.data, None, g.ctypes.data, 64, 0.0, 0, ctypes.byref(h)) == tq.TQ_EINVAL
    assert tq._lib.tq_build_rotation(64, 2, 7, s.ctypes.data, None, g.ctypes.data, 64, 0.0, 0, ctypes.byref(h)) == tq.TQ_EINVAL
    bad = s.copy()
    bad[3] = 0
    assert tq._lib.tq_build_rotation(64, 2, 0, bad.ctypes.data, None, g.ctypes.data, 64, 0.0, 0, ctypes.byref(h)) == tq.TQ_EINVAL
    assert tq._lib.tq_build_rotation(96, 2, 0, np.ones(96, np.int8).ctypes.data, None, np.zeros((96, 96), np.float32).ctypes.data,
                                     96, 0.0, 0, ctypes.byref(h)) == tq.TQ_EUNSUPPORTED
    assert tq._lib.tq_decode_workspace_size(None, None, 1, 1, 1, 10) == 0
    assert tq._lib.tq_decode_window_workspace_size(None, None, 1, 1, 1, 10, 4) == 0
    assert tq._lib.tq_quantize_kv(None, None, 0, 1, 64, None, 1, 0, 0, None, None, None, 1, None) == tq.TQ_EINVAL
    # window decode: null handles rejected on the host, before any device call
    assert tq._lib.tq_decode_attention_window(None, None, None, 0, None, None, None, None, None, None, None, 0,
                                              None, None, 0, 0, 0, 1, 4, 1, 0, None, 0.125, None, None, 0,
                                              None) == tq.TQ_EINVAL
    assert tq._lib.tq_decode_attention(None, None, None, 0, None, None, None, None, None, None, None, 0,
                                       1, 4, 1, 0, None, 0.125, None, None, 0, None) == tq.TQ_EINVAL
    # NSN: null handle or buffers rejected on the host
    assert tq._lib.tq_nsn_shift(None, None, 0, 1, 4, 128, 0, 0, None, None, None, None) == tq.TQ_EINVAL
    assert tq._lib.tq_decode_attention_nsn(None, None, None, 0, None, None, None, None, None, None, None, None, None,
                                           None, None, 0, 1, 4, 1, 1, None, 0.125, None, None, 0, None) == tq.TQ_EINVAL
    # fused append: missing new rows or handles rejected on the host
    assert tq._lib.tq_decode_attention_append(None, None, None, 0, None, None, None, None, None, None, None, None,
                                              None, 0, 1, 4, 1, 1, None, 0.125, None, None, 0, None) == tq.TQ_EINVAL
    # fused NSN append: missing new rows, side arrays or handles rejected on the host
    assert tq._lib.tq_decode_attention_nsn_append(None, None, None, 0, None, None, None, None, None, None, None, None,
                                                  None, None, None, None, None, 4, 1, 4, 1, 1, None, 0.125, None,
                                                  None, 0, None) == tq.TQ_EINVAL


def test_window_binding_checks_shapes_before_any_call():
    """The binding rejects window arrays of different shape or dtype, and
    non-contiguous ones, before it reaches the library (no GPU needed)."""
    import torch
    from vector_quantization_b200 import tq
    rec = (torch.zeros((1, 1, 4, 32), dtype=torch.uint8), torch.zeros((1, 1, 4, 16), dtype=torch.uint8),
           torch.zeros((1, 1, 4, 2)))
    q = torch.zeros((1, 4, 128))
    qpos = torch.zeros(1, dtype=torch.int64)
    kw = torch.zeros((1, 1, 8, 128))
    with pytest.raises(ValueError, match="share shape and dtype"):
        tq.decode_attention_window(None, None, q, qpos, rec, rec, 4, kw, torch.zeros((1, 1, 9, 128)), 2)
    with pytest.raises(ValueError, match="share shape and dtype"):
        tq.decode_attention_window(None, None, q, qpos, rec, rec, 4, kw, kw.to(torch.bfloat16), 2)
    with pytest.raises(ValueError, match="contiguous"):
        tq.decode_attention_window(None, None, q, qpos, rec, rec, 4, kw.transpose(2, 3), kw.transpose(2, 3), 2)


@pytest.mark.parametrize("d,kind,seed", [(128, "hadamard", 0), (64, "hadamard", 2**40 + 7), (96, "dense", 1234567)])
def test_library_seeded_draws_match_oracle_generator(d, kind, seed):
    """The library's Philox4x32-10 draws (host code, no GPU) against the
    oracle's own implementation of the same published generator: signs and
    the float32 QJL Gaussians bit for bit, the float64 dense Gaussians to a
    few ulps (the two sides call different libm builds for log/cos/sin)."""
    from vector_quantization_b200 import tq
    from oracle import philox
    lib = tq.rotation_draws(d, seed, kind)
    ora = philox.rotation_draws(d, seed, dense=(kind == "dense"))
    np.testing.assert_array_equal(lib["signs"], ora["signs"])
    # float64 draws that differ in the last ulp may round to different
    # float32 values only when they sit on a float32 rounding midpoint
    np.testing.assert_allclose(lib["gauss_s"], ora["gauss_s"], rtol=2**-23, atol=0)
    assert np.mean(lib["gauss_s"] == ora["gauss_s"]) > 0.999
    if kind == "dense":
        np.testing.assert_allclose(lib["gauss_pi"], ora["gauss_pi"], rtol=1e-14, atol=1e-300)
    else:
        assert lib["gauss_pi"] is None


def test_library_seeded_draws_reject_bad_sizes():
    from vector_quantization_b200 import tq
    assert tq._lib.tq_rotation_draws(0, 0, 1, 128, None, None, None) == tq.TQ_EINVAL
    assert tq._lib.tq_rotation_draws(128, 7, 1, 128, None, None, None) == tq.TQ_EINVAL
    assert tq._lib.tq_rotation_draws(128, 0, 1, 128, None, None, None) == tq.TQ_OK


def test_binding_without_the_library_raises_on_import(tmp_path):
    """A copy of the package without libtq.so: importing the binding raises
    ImportError naming the missing library (no fallback path exists)."""
    import os
    import shutil
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    pkg = tmp_path / "vector_quantization_b200"
    pkg.mkdir()
    for name in ("__init__.py", "tq.py", "sharded.py", "build.py"):
        shutil.copy(os.path.join(root, "vector_quantization_b200", name), pkg / name)
    code = ("import sys; sys.path.insert(0, sys.argv[1])\n"
            "try:\n"
            "    import vector_quantization_b200.tq\n"
            "except ImportError as e:\n"
            "    print('raised', 'libtq.so' in str(e))\n"
            "else:\n"
            "    print('imported')\n")
    run = subprocess.run([sys.executable, "-c", code, str(tmp_path)], capture_output=True, text=True, timeout=300)
    assert run.stdout.strip() == "raised True", run.stdout + run.stderr
