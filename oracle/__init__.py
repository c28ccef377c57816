"""CPU oracle for the rotation + Lloyd-Max + QJL vector codec.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call, link
or execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code, table or constant
generator with the CUDA library; the two meet only on the seeded inputs from
``synth``.

Everything is plain NumPy/SciPy in float64, with explicit codebooks, unpacked
bit arrays and a two-pass softmax, written for a reader to check against the
pages by eye.  Citations name the page and its section:

* [TurboESM]  "TurboESM: Ultra-Efficient 3-Bit KV Cache Quantization for
  Protein Language Models with Orthogonal Rotation and QJL Correction"
  (gist.science, paper 2603.26110), "Résumé technique" sections 1-5.
* [TurboQuant] the TurboQuant digest (news.hada.io topic 27867): sections
  "Principe de fonctionnement de TurboQuant" (Étape 1, Étape 2),
  "QJL : une technique 1 bit à surcharge nulle", "Expériences et résultats".
* [NSNQuant]  "NSNQuant: A Double Normalization Approach for Calibration-Free
  Low-Bit Vector Quantization of KV Cache" (gist.science, paper 2505.18231),
  "Résumé Technique", Méthodologie §2 (Transformée de Hadamard).

Parity status per function is stated in each module header.
"""
from .codebook import (coord_pdf, coord_mass, coord_first_moment, lloyd_max,
                       codebook_mse, walsh_coefficients)
from .rotation import (sylvester_hadamard, hadamard_rotation, dense_rotation,
                       round_to_bf16, apply_rope, Rotation, build_rotation)
from .codec import (encode, pack_planes, unpack_planes, pack_bits, unpack_bits,
                    dequantize, score_from_codes, QJL_CONST)
from .attention import decode_attention, encoder_attention, exact_attention
from .search import search_scores, topk_desc, exact_mips_topk, recall_at_k
from .memory import record_bytes, cache_bytes

__all__ = [n for n in dir() if not n.startswith("_")]
