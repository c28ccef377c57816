"""Inner-product top-k search from packed codes (float64 oracle).

TEST INFRASTRUCTURE ONLY (see the package header).

[TurboQuant] "Expériences et résultats" / "Performances en recherche
vectorielle": the codec serves brute-force maximum-inner-product search with
no large codebooks; quality is a recall figure against the exact search.

  score(q, x_n) = ||x_n|| <Pi q, c[idx_n]> + ||r_n|| sqrt(pi/2)/m <S Pi q, 2 z_n - 1>

(the same estimator as attention, without RoPE and without 1/sqrt(d)).
Top-k is taken in descending score order with ties broken toward the lower
id.  recall@k = |approx top-k  ∩  exact top-k| / k averaged over queries,
the exact top-k coming from float64 brute-force MIPS on the raw vectors.
Absolute recall values: parity unpinned (the pages print figures only for
GloVe d = 200, which is not available here); the tests pin the top-k routine
against a stable sort and check that recall rises with bits.
"""
from __future__ import annotations

import numpy as np

from .codec import score_from_codes, unpack_bits, unpack_planes
from .rotation import Rotation


def search_scores(rot: Rotation, queries, codes, signs, norms) -> np.ndarray:
    """Estimated inner products [nq, N] from packed (codes, signs, norms)."""
    c = unpack_planes(codes, rot.bits, rot.d)
    z = unpack_bits(signs, rot.m)
    nrm = np.asarray(norms, dtype=np.float64)
    return score_from_codes(rot, np.atleast_2d(queries), c, z, nrm[:, 0], nrm[:, 1])


def topk_desc(scores, k: int):
    """Per row, the k largest scores (descending) and their ids; ties go to
    the lower id.  Returns (values [nq, k], ids [nq, k] int64)."""
    s = np.atleast_2d(np.asarray(scores, dtype=np.float64))
    ids = np.argsort(-s, axis=1, kind="stable")[:, :k]
    return np.take_along_axis(s, ids, axis=1), ids.astype(np.int64)


def exact_mips_topk(queries, db, k: int):
    """Exact float64 brute-force maximum-inner-product top-k."""
    s = np.atleast_2d(np.asarray(queries, dtype=np.float64)) @ np.asarray(db, dtype=np.float64).T
    return topk_desc(s, k)


def recall_at_k(approx_ids, exact_ids) -> float:
    """Mean over queries of |approx ∩ exact| / k."""
    a = np.asarray(approx_ids)
    e = np.asarray(exact_ids)
    k = e.shape[1]
    return float(np.mean([len(set(a[i].tolist()) & set(e[i].tolist())) / k for i in range(len(a))]))
