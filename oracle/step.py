"""The whole indexer step in the oracle, from raw input buffers.

TEST INFRASTRUCTURE ONLY (see ``oracle.lsa_oracle``).  Inputs are raw numpy arrays as
stored on the device: bf16 as uint16 bit patterns, e4m3 as uint8 codes, fp32 as
float32.  Every decode and every arithmetic step is the oracle's own.
"""
from __future__ import annotations

import numpy as np

from . import lsa_oracle as O


def decode(raw, dtype: str) -> np.ndarray:
    """Raw storage -> float64.  dtype in {"f32", "bf16", "e4m3"}."""
    if dtype == "f32":
        return np.asarray(raw, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return O.decode_bf16(np.asarray(raw).view(np.uint16))
    if dtype == "e4m3":
        return O.decode_e4m3(np.asarray(raw).view(np.uint8))
    raise ValueError(dtype)


def decode_keys(K_raw, kscale, kdtype: str) -> np.ndarray:
    """K_IComp rows [n][dI] as float64, with the per-entry e4m3 scale applied."""
    K = decode(K_raw, kdtype)
    if kdtype == "e4m3":
        K = K * np.asarray(kscale, dtype=np.float32).astype(np.float64)[:, None]
    return K


def project(h_raw, Wd_raw, Wu_raw, Ww_raw, H, dI, wdtype):
    """(q [H][dI], w [H]) for one (sequence, layer) from raw storage."""
    return O.project_query(decode(h_raw, wdtype), decode(Wd_raw, wdtype),
                           decode(Wu_raw, wdtype), decode(Ww_raw, wdtype), H, dI,
                           bf16_boundaries=(wdtype == "bf16"))


def score_layer(q, w, b, K_raw, kscale, kdtype):
    """(z [n], I [n], mark [n]) of one (sequence, layer) for the given query."""
    z = O.head_fused_logits(q, w, float(np.float32(b)), decode_keys(K_raw, kscale, kdtype))
    return z, O.sigmoid(z), O.threshold_mark(z)


def select(marks_by_layer, z_by_layer, k):
    """Union, per-layer new sets, fetch lists and the top-k of one sequence."""
    U, news = O.or_union(marks_by_layer)
    idx_U = O.compact(U)
    key = O.fetched_key(z_by_layer, marks_by_layer)
    return {
        "union": U,
        "new": news,
        "idx_new": [O.compact(m) for m in news],
        "idx_union": idx_U,
        "topk": O.topk_in_fetched(idx_U, key, k),
        "key": key,
    }
