"""Python binding of liblsa, the B200 (sm_100a) library for the Lookahead Sparse
Attention indexer step: scoring, OR-union, compaction, cold->hot gather, top-k in the
fetched set and cross-layer vote labels.

The functions keep the C names and only marshal arguments: tensors become raw
pointers, dtypes become lsa_dtype codes, and the current torch CUDA stream is passed
unless one is given.  Every computation runs in liblsa's kernels; a nonzero status
raises LsaError.  Shapes and layouts are documented in include/lsa.h.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_UNSUPPORTED, LSA_ERR_CAPACITY = 0, 1, 2, 3
LSA_ERR_NOMEM, LSA_ERR_CUDA, LSA_ERR_TIMEOUT, LSA_ERR_RANGE = 4, 5, 6, 7
LSA_F32, LSA_BF16, LSA_E4M3 = 0, 1, 2


class LsaError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({detail})")


def lib():
    return _abi.load()


def status_string(code: int) -> str:
    return lib().lsa_status_string(code).decode()


def dtype_code(t) -> int:
    dt = t.dtype if isinstance(t, torch.Tensor) else t
    if dt == torch.float32:
        return LSA_F32
    if dt == torch.bfloat16:
        return LSA_BF16
    if dt in (torch.uint8, torch.float8_e4m3fn):
        return LSA_E4M3
    raise TypeError(f"no lsa_dtype for {dt}")


def _p(t):
    """Raw pointer of a tensor (None -> NULL); plain ints pass through.  The library reads
    and writes every array densely in the layout the header gives, so a strided view is
    refused here rather than read as if it were dense."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError(f"tensor of shape {tuple(t.shape)} with strides {t.stride()} is not contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, where: str):
    if rc != LSA_OK:
        raise LsaError(rc, where, lib().lsa_last_error().decode())


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device workspace (torch allocations are 512-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def kernel_launches() -> int:
    """Kernels liblsa has launched in this process so far."""
    return int(lib().lsa_kernel_launches())


# ----------------------------------------------------------------------------- scoring

def lsa_index_project_workspace_bytes(B, L, D, r, H, dI, wdt) -> int:
    return int(lib().lsa_index_project_workspace_bytes(B, L, D, r, H, dI, wdt))


def lsa_index_project(B, L, D, r, H, dI, wdt, h, W_down, W_up, W_w, layer, q_out, w_out,
                      workspace, stream=None):
    _check(lib().lsa_index_project(B, L, D, r, H, dI, wdt, _p(h), _p(W_down), _p(W_up), _p(W_w),
                                   layer, _p(q_out), _p(w_out), _p(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(stream)),
           "lsa_index_project")


def lsa_index_score_workspace_bytes(B, L, N, D, r, H, dI, wdt, kdt) -> int:
    return int(lib().lsa_index_score_workspace_bytes(B, L, N, D, r, H, dI, wdt, kdt))


def lsa_index_score(B, L, N, D, r, H, dI, wdt, h, W_down, W_up, W_w, bias, kdt, K, kscale,
                    layer, q_in, w_in, q_out, w_out, mask, logit, score, workspace, status=None,
                    stream=None):
    rc = lib().lsa_index_score(B, L, N, D, r, H, dI, wdt, _p(h), _p(W_down), _p(W_up), _p(W_w),
                               _p(bias), kdt, _p(K), _p(kscale), layer, _p(q_in), _p(w_in),
                               _p(q_out), _p(w_out), _p(mask), _p(logit), _p(score), _p(status),
                               _p(workspace), 0 if workspace is None else workspace.numel(),
                               _stream(stream))
    _check(rc, "lsa_index_score")


# ----------------------------------------------------------------------------- selection

def lsa_select_union(B, Nw, mask_l, U, new_l, stream=None):
    _check(lib().lsa_select_union(B, Nw, _p(mask_l), _p(U), _p(new_l), _stream(stream)),
           "lsa_select_union")


def lsa_compact(B, N, bits, cap, idx, count, status=None, stream=None):
    _check(lib().lsa_compact(B, N, _p(bits), cap, _p(idx), _p(count), _p(status), _stream(stream)),
           "lsa_compact")


def lsa_select_fetch_workspace_bytes(B, N) -> int:
    return int(lib().lsa_select_fetch_workspace_bytes(B, N))


def lsa_select_fetch(B, L, N, mask, U, new_l, cap, idx_new, cnt_new, idx_U, cnt_U, workspace, logit=None,
                     key_U=None, status=None, stream=None):
    _check(lib().lsa_select_fetch(B, L, N, _p(mask), _p(U), _p(new_l), cap, _p(idx_new), _p(cnt_new), _p(idx_U),
                                  _p(cnt_U), _p(logit), _p(key_U), _p(status), _p(workspace),
                                  0 if workspace is None else workspace.numel(), _stream(stream)), "lsa_select_fetch")


def lsa_topk_keyed(B, k, idx, cap, count, key, topk, topk_count, stream=None):
    _check(lib().lsa_topk_keyed(B, k, _p(idx), cap, _p(count), _p(key), _p(topk), _p(topk_count), _stream(stream)),
           "lsa_topk_keyed")


def lsa_topk_workspace_bytes(B, cap) -> int:
    return int(lib().lsa_topk_workspace_bytes(B, cap))


def lsa_topk(B, L, N, k, idx, cap, count, logit, topk, topk_count, workspace, stream=None):
    _check(lib().lsa_topk(B, L, N, k, _p(idx), cap, _p(count), _p(logit), _p(topk), _p(topk_count),
                          _p(workspace), 0 if workspace is None else workspace.numel(),
                          _stream(stream)), "lsa_topk")


def lsa_fine_score_workspace_bytes(B, H, dI, kdt) -> int:
    return int(lib().lsa_fine_score_workspace_bytes(B, H, dI, kdt))


def lsa_fine_score(B, N, H, dI, qdt, q, w, kdt, K, kscale, idx, cap, count, score, workspace, status=None,
                   stream=None):
    _check(lib().lsa_fine_score(B, N, H, dI, qdt, _p(q), _p(w), kdt, _p(K), _p(kscale), _p(idx), cap, _p(count),
                                _p(score), _p(status), _p(workspace), 0 if workspace is None else workspace.numel(),
                                _stream(stream)), "lsa_fine_score")


def lsa_topk_noalloc(B, L, N, k, idx, cap, count, logit, topk, topk_count, stream=None):
    """lsa_topk with its scratch in the library's built-in device array (no workspace)."""
    _check(lib().lsa_topk_noalloc(B, L, N, k, _p(idx), cap, _p(count), _p(logit), _p(topk), _p(topk_count),
                                  _stream(stream)), "lsa_topk_noalloc")


def lsa_gather_cold(B, N, row_bytes, cold_host, idx, count, cap, hot, status=None, stream=None):
    _check(lib().lsa_gather_cold(B, N, row_bytes, _p(cold_host), _p(idx), _p(count), cap, _p(hot),
                                 _p(status), _stream(stream)), "lsa_gather_cold")


# ----------------------------------------------------------------------------- hot pool

def lsa_hot_pool_state_bytes(B, N, slots) -> int:
    return int(lib().lsa_hot_pool_state_bytes(B, N, slots))


def lsa_hot_pool_workspace_bytes(B, N, slots) -> int:
    return int(lib().lsa_hot_pool_workspace_bytes(B, N, slots))


def lsa_hot_pool_layout(B, N, slots):
    """Byte offsets of (slot_of, entry_of, stamp, resident) inside the state."""
    off = (ctypes.c_size_t * 4)()
    _check(lib().lsa_hot_pool_layout(B, N, slots, off), "lsa_hot_pool_layout")
    return tuple(int(x) for x in off)


def lsa_hot_pool_reset(B, N, slots, state, stream=None):
    _check(lib().lsa_hot_pool_reset(B, N, slots, _p(state), _stream(stream)), "lsa_hot_pool_reset")


def lsa_hot_pool_update(B, N, slots, row_bytes, trigger, U, cold_host, hot, state, moved, status,
                        workspace, stream=None):
    _check(lib().lsa_hot_pool_update(B, N, slots, row_bytes, trigger, _p(U), _p(cold_host), _p(hot), _p(state),
                                     _p(moved), _p(status), _p(workspace),
                                     0 if workspace is None else workspace.numel(), _stream(stream)),
           "lsa_hot_pool_update")


# ----------------------------------------------------------------------------- training step

def lsa_index_train_step_workspace_bytes(P, N, D, r, H, dI) -> int:
    return int(lib().lsa_index_train_step_workspace_bytes(P, N, D, r, H, dI))


def lsa_index_train_step(P, N, D, r, H, dI, wdt, h, W_down, W_up, W_w, bias, kdt, K, kscale, labels, gamma,
                         c_in, q_in, w_in, loss, dW_down, dW_up, dW_w, dbias, workspace, status=None, stream=None):
    _check(lib().lsa_index_train_step(P, N, D, r, H, dI, wdt, _p(h), _p(W_down), _p(W_up), _p(W_w), float(bias), kdt,
                                      _p(K), _p(kscale), _p(labels), float(gamma), _p(c_in), _p(q_in), _p(w_in),
                                      _p(loss), _p(dW_down), _p(dW_up), _p(dW_w), _p(dbias), _p(status),
                                      _p(workspace), 0 if workspace is None else workspace.numel(),
                                      _stream(stream)), "lsa_index_train_step")


# ----------------------------------------------------------------------------- self-check

def lsa_check_bounded_wait(limit_us, status, stream=None):
    _check(lib().lsa_check_bounded_wait(limit_us, _p(status), _stream(stream)), "lsa_check_bounded_wait")


# ----------------------------------------------------------------------------- labels

def lsa_vote_labels_workspace_bytes(L, P, N) -> int:
    return int(lib().lsa_vote_labels_workspace_bytes(L, P, N))


def lsa_vote_labels(L, P, N, logits, top_p, theta, golden, counts, scores, gamma, loss,
                    workspace, stream=None):
    _check(lib().lsa_vote_labels(L, P, N, _p(logits), float(top_p), theta, _p(golden), _p(counts),
                                 _p(scores), float(gamma), _p(loss), _p(workspace),
                                 0 if workspace is None else workspace.numel(), _stream(stream)),
           "lsa_vote_labels")
