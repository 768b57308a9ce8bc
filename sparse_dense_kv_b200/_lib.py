"""ctypes binding of libs3r.so: argument marshalling only.

Every function has the name of the C entry point it calls and takes torch tensors where
the C function takes device pointers. Tensors must already live on the GPU with the dtype
and layout the header states; the binding checks dtype/device/contiguity, passes
`data_ptr()` and the current CUDA stream, and raises S3RError on any non-OK status. No
step of the hot path runs in Python.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs3r.so")

S3R_OK = 0
STATUS_NAMES = {
    0: "S3R_OK", 1: "S3R_ERR_INVALID_ARG", 2: "S3R_ERR_UNSUPPORTED", 3: "S3R_ERR_CUDA",
    4: "S3R_ERR_WORKSPACE", 5: "S3R_ERR_DEVICE_BOUNDS", 6: "S3R_ERR_NONFINITE",
    7: "S3R_ERR_TIMEOUT",
}
PAGE_SIZE = 16
MAX_K = 8


class S3RError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


class KVCacheDesc(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int64), ("k_pool", ctypes.c_void_p),
                ("v_pool", ctypes.c_void_p)]


class BatchDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_requests", ctypes.c_int32),
                ("req_ids", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("max_pages_per_req", ctypes.c_int32)]


class SchedConfig(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int32), ("policy", ctypes.c_int32), ("evict", ctypes.c_int32),
                ("cap0", ctypes.c_int32), ("cap_min", ctypes.c_int32), ("cap_max", ctypes.c_int32),
                ("u_low", ctypes.c_double), ("u_high", ctypes.c_double), ("b_high", ctypes.c_double),
                ("c0", ctypes.c_double), ("c_tok", ctypes.c_double), ("c_kv", ctypes.c_double),
                ("c_xfer", ctypes.c_double), ("c_rec", ctypes.c_double), ("c_pre", ctypes.c_double),
                ("max_iters", ctypes.c_int64)]


class SchedResult(ctypes.Structure):
    _fields_ = [("tokens", ctypes.c_int64), ("transferred", ctypes.c_int64),
                ("recomputed", ctypes.c_int64), ("prefilled", ctypes.c_int64),
                ("evictions", ctypes.c_int64), ("iterations", ctypes.c_int64),
                ("max_active", ctypes.c_int32), ("done", ctypes.c_int32), ("stalled", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("time", ctypes.c_double)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libs3r.so is not built ({LIB_PATH}); run python sparse_dense_kv_b200/build.py")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t
    C, B = ctypes.POINTER(KVCacheDesc), ctypes.POINTER(BatchDesc)
    sig = {
        "s3r_workspace_size": (SZ, [C, I32, I32, I32, I32, I32]),
        "s3r_workspace_init": (ctypes.c_int, [P, SZ, P]),
        "s3r_verify_attn": (ctypes.c_int, [C, B, I32, P, P, P, P, P, P, P, SZ, P]),
        "s3r_select_kv": (ctypes.c_int, [C, B, P, P, I32, I32, I32, P, I32, P, P, SZ, P]),
        "s3r_select_from_scores": (ctypes.c_int, [C, B, P, I32, I32, I32, P, I32, P, P, SZ, P]),
        "s3r_position_scores": (ctypes.c_int, [C, B, P, P, I32, P, I32, P, SZ, P]),
        "s3r_select_kv_pages": (ctypes.c_int, [C, B, P, P, I32, I32, I32, P, I32, P, P, SZ, P]),
        "s3r_select_pages_from_scores": (ctypes.c_int, [C, B, P, I32, I32, I32, P, I32, P, P, SZ, P]),
        "s3r_sparse_draft_attn": (ctypes.c_int, [C, B, P, P, I32, P, P, I32, P, I32, P, P, P, P, SZ, P]),
        "s3r_draft_sample": (ctypes.c_int, [B, P, I32, P, I32, U64, P, P, P, P, SZ, P]),
        "s3r_draft_sample_noalloc": (ctypes.c_int, [B, P, I32, P, I32, U64, P, P, P]),
        "s3r_spec_sample": (ctypes.c_int, [B, I32, P, P, P, I32, U64, P, P, P, P, P, SZ, P]),
        "s3r_draft_argmax": (ctypes.c_int, [B, P, I32, P, I32, P, P, SZ, P]),
        "s3r_sched_simulate": (ctypes.c_int, [ctypes.POINTER(SchedConfig), I32, P, P, P, ctypes.c_int64,
                                              P, ctypes.c_int64, ctypes.POINTER(SchedResult), P,
                                              ctypes.c_int64]),
        "s3r_choose_horizon": (ctypes.c_int, [P, P, I32, ctypes.c_double, ctypes.c_double,
                                              ctypes.c_double, ctypes.c_double, P]),
        "s3r_horizon_step": (ctypes.c_int, [P, P, P, P, I32, ctypes.c_double, ctypes.c_double,
                                            ctypes.c_double, ctypes.c_double, ctypes.c_double, P, P]),
        "s3r_choose_horizon_costs": (ctypes.c_int, [P, P, I32, P, ctypes.c_double, ctypes.c_double, P]),
        "s3r_horizon_step_costs": (ctypes.c_int, [P, P, P, P, I32, ctypes.c_double, P, ctypes.c_double,
                                                  ctypes.c_double, P, P]),
        "s3r_greedy_verify": (ctypes.c_int, [B, I32, P, P, I32, P, P, P, SZ, P]),
        "s3r_commit": (ctypes.c_int, [B, I32, P, P, P, P]),
        "s3r_philox": (ctypes.c_int, [U64, I32, P, P, I64, P, P, P]),
        "s3r_get_error": (ctypes.c_int, [P, P, P]),
        "s3r_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "s3r_launch_count": (U64, []),
        "s3r_last_error_message": (ctypes.c_char_p, []),
        "s3r_set_verify_kernel": (ctypes.c_int, [I32]),
        "s3r_set_wait_limit": (ctypes.c_int, [I32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
lib = _lib


def _check(status: int, what: str):
    if status != S3R_OK:
        if status == 3:
            what = f"{what} ({_lib.s3r_last_error_message().decode()})"
        raise S3RError(status, what)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, dtype=None, what="tensor", allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{what} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a torch.Tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    if t.device.type != "cuda":
        raise ValueError(f"{what} must be a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def make_cache(k_pool: torch.Tensor, v_pool: torch.Tensor, num_q_heads: int) -> KVCacheDesc:
    """Descriptor of bf16 pools [num_pages][num_kv_heads][16][head_dim]."""
    P, H, S, D = k_pool.shape
    if v_pool.shape != k_pool.shape or S != PAGE_SIZE:
        raise ValueError("pools must be [num_pages][num_kv_heads][16][head_dim] and equal")
    desc = KVCacheDesc(num_q_heads, H, D, S, P, _ptr(k_pool, torch.bfloat16, "k_pool").value,
                       _ptr(v_pool, torch.bfloat16, "v_pool").value)
    desc._refs = (k_pool, v_pool)          # the descriptor keeps its tensors alive
    return desc


def make_batch(seq_lens: torch.Tensor, page_table: torch.Tensor | None = None,
               req_ids: torch.Tensor | None = None, batch: int | None = None) -> BatchDesc:
    """Batch descriptor; covers req_ids (or all requests) of int32 seq_lens / page_table."""
    nr = seq_lens.numel()
    if batch is None:
        batch = req_ids.numel() if req_ids is not None else nr
    pt = _ptr(page_table, torch.int32, "page_table", allow_none=True)
    mp = page_table.shape[1] if page_table is not None else 0
    rid = _ptr(req_ids, torch.int32, "req_ids", allow_none=True)
    desc = BatchDesc(batch, nr, rid.value if rid is not None else None,
                     _ptr(seq_lens, torch.int32, "seq_lens").value,
                     pt.value if pt is not None else None, mp)
    desc._refs = (seq_lens, page_table, req_ids)
    return desc


def s3r_workspace_size(cache: KVCacheDesc, num_requests: int, max_pages_per_req: int,
                       max_k: int, vocab: int, sel_stride: int) -> int:
    n = _lib.s3r_workspace_size(ctypes.byref(cache), num_requests, max_pages_per_req, max_k,
                                vocab, sel_stride)
    if n == 0:
        raise S3RError(1, "s3r_workspace_size")
    return int(n)


def s3r_workspace_init(ws: torch.Tensor, stream=None):
    _check(_lib.s3r_workspace_init(_ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)),
           "s3r_workspace_init")


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zeroed workspace (uint8 CUDA tensor, 256-byte aligned by the caching allocator)."""
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    if ws.data_ptr() % 256:
        raise RuntimeError("workspace allocation is not 256-byte aligned")
    s3r_workspace_init(ws)
    return ws


def s3r_verify_attn(cache, batch, k, q, k_new, v_new, out, lse, score_logits, ws, stream=None):
    bf, f32 = torch.bfloat16, torch.float32
    _check(_lib.s3r_verify_attn(
        ctypes.byref(cache), ctypes.byref(batch), k, _ptr(q, bf, "q"), _ptr(k_new, bf, "k_new"),
        _ptr(v_new, bf, "v_new"), _ptr(out, bf, "out"), _ptr(lse, f32, "lse"),
        _ptr(score_logits, f32, "score_logits", allow_none=True), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream)), "s3r_verify_attn")


def _select_kv(fn, cache, batch, score_logits, lse, k_prev, budget_bp, window, sel_idx,
               sel_count, ws, stream):
    f32, i32 = torch.float32, torch.int32
    _check(getattr(_lib, fn)(
        ctypes.byref(cache), ctypes.byref(batch), _ptr(score_logits, f32, "score_logits"),
        _ptr(lse, f32, "lse"), k_prev, budget_bp, window, _ptr(sel_idx, i32, "sel_idx"),
        sel_idx.shape[-1], _ptr(sel_count, i32, "sel_count"), _ptr(ws, torch.uint8, "ws"),
        ws.numel(), _stream(stream)), fn)


def _select_from_scores(fn, cache, batch, scores, budget_bp, window, sel_idx, sel_count, ws,
                        stream):
    f32, i32 = torch.float32, torch.int32
    _check(getattr(_lib, fn)(
        ctypes.byref(cache), ctypes.byref(batch), _ptr(scores, f32, "scores"), scores.shape[-1],
        budget_bp, window, _ptr(sel_idx, i32, "sel_idx"), sel_idx.shape[-1],
        _ptr(sel_count, i32, "sel_count"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)), fn)


def s3r_position_scores(cache, batch, score_logits, lse, k_prev, scores, ws, stream=None):
    """scores: fp32 [NR][H_kv][stride] receiving sigma_j for every committed j < L."""
    f32 = torch.float32
    _check(_lib.s3r_position_scores(
        ctypes.byref(cache), ctypes.byref(batch), _ptr(score_logits, f32, "score_logits"),
        _ptr(lse, f32, "lse"), k_prev, _ptr(scores, f32, "scores"), scores.shape[-1],
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "s3r_position_scores")


def s3r_select_kv(cache, batch, score_logits, lse, k_prev, budget_bp, window, sel_idx,
                  sel_count, ws, stream=None):
    _select_kv("s3r_select_kv", cache, batch, score_logits, lse, k_prev, budget_bp, window,
               sel_idx, sel_count, ws, stream)


def s3r_select_kv_pages(cache, batch, score_logits, lse, k_prev, budget_bp, window, sel_idx,
                        sel_count, ws, stream=None):
    _select_kv("s3r_select_kv_pages", cache, batch, score_logits, lse, k_prev, budget_bp,
               window, sel_idx, sel_count, ws, stream)


def s3r_select_from_scores(cache, batch, scores, budget_bp, window, sel_idx, sel_count, ws,
                           stream=None):
    _select_from_scores("s3r_select_from_scores", cache, batch, scores, budget_bp, window,
                        sel_idx, sel_count, ws, stream)


def s3r_select_pages_from_scores(cache, batch, scores, budget_bp, window, sel_idx, sel_count,
                                 ws, stream=None):
    _select_from_scores("s3r_select_pages_from_scores", cache, batch, scores, budget_bp,
                        window, sel_idx, sel_count, ws, stream)


def _rows(t, inner, what):
    """Pointer and request stride (elements) of a [num_requests][...] view whose per-request
    part of `inner` elements is contiguous (e.g. block[:, i] of a [R][k+1][H][d] tensor)."""
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda" or t.dtype != torch.bfloat16:
        raise TypeError(f"{what} must be a bf16 CUDA tensor")
    if t[0].numel() != inner or not t[0].is_contiguous():
        raise ValueError(f"{what}: each request's rows must be contiguous ({inner} elements)")
    return ctypes.c_void_p(t.data_ptr()), int(t.stride(0)) if t.shape[0] > 1 else inner


def s3r_sparse_draft_attn(cache, batch, draft_step, q, k_new, v_new, sel_idx, sel_count, out,
                          lse, ws, stream=None):
    """q [NR][H_q][d] and k_new / v_new [NR][H_kv][d], each possibly a strided view."""
    bf, i32 = torch.bfloat16, torch.int32
    qp, qs = _rows(q, cache.num_q_heads * cache.head_dim, "q")
    kp, ks = _rows(k_new, cache.num_kv_heads * cache.head_dim, "k_new")
    vp, vs = _rows(v_new, cache.num_kv_heads * cache.head_dim, "v_new")
    if ks != vs:
        raise ValueError("k_new and v_new must share a request stride")
    _check(_lib.s3r_sparse_draft_attn(
        ctypes.byref(cache), ctypes.byref(batch), _ptr(draft_step, i32, "draft_step"),
        qp, qs, kp, vp, ks,
        _ptr(sel_idx, i32, "sel_idx"), sel_idx.shape[-1], _ptr(sel_count, i32, "sel_count"),
        _ptr(out, bf, "out"), _ptr(lse, torch.float32, "lse", allow_none=True),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "s3r_sparse_draft_attn")


def _norms(t, what):
    """s3r_row_norm [NR][k] as a float64 tensor [NR][k][2] (float max, float unused, double sum)."""
    if t is not None and (t.dtype != torch.float64 or t.shape[-1] != 2):
        raise TypeError(f"{what} must be a float64 [NR][k][2] tensor (s3r_row_norm records)")
    return _ptr(t, torch.float64, what, allow_none=True)


def row_norms(t) -> tuple:
    """(max, sum) arrays of a q_norm tensor written by s3r_draft_sample."""
    raw = t.detach().cpu().contiguous()
    mx = raw.view(torch.float32)[..., 0]
    return mx.numpy(), raw[..., 1].numpy()


def s3r_draft_sample(batch, draft_step, k, q_logits, vocab, seed, draft_tokens, ws, stream=None,
                     margins=None, q_norm=None):
    """margins: optional fp32 [NR][k] tensor receiving each draw's boundary margin; q_norm:
    optional float64 [NR][k][2] tensor receiving the rows' normalisers (s3r_row_norm)."""
    _check(_lib.s3r_draft_sample(
        ctypes.byref(batch), _ptr(draft_step, torch.int32, "draft_step"), k,
        _ptr(q_logits, torch.float32, "q_logits"), vocab, seed,
        _ptr(draft_tokens, torch.int32, "draft_tokens"),
        _ptr(margins, torch.float32, "margins", allow_none=True), _norms(q_norm, "q_norm"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "s3r_draft_sample")


def s3r_draft_sample_noalloc(batch, draft_step, k, q_logits, vocab, seed, draft_tokens, err_word,
                             stream=None):
    """s3r_draft_sample with the library's static scratch instead of a workspace; err_word
    is a device int32 tensor of one element that receives the device-side status bits."""
    st = _lib.s3r_draft_sample_noalloc(
        ctypes.byref(batch), _ptr(draft_step, torch.int32, "draft_step"), k,
        _ptr(q_logits, torch.float32, "q_logits"), vocab, seed,
        _ptr(draft_tokens, torch.int32, "draft_tokens"), _ptr(err_word, torch.int32, "err_word"),
        _stream(stream))
    if st == 2 and _lib.s3r_last_error_message():
        raise S3RError(st, "s3r_draft_sample_noalloc: " + _lib.s3r_last_error_message().decode())
    _check(st, "s3r_draft_sample_noalloc")


def s3r_spec_sample(batch, k, p_logits, q_logits, draft_tokens, vocab, seed, out_tokens, n_out,
                    ws, stream=None, margins=None, q_norm=None):
    """margins: optional fp32 [NR][k+1] tensor receiving the decisions' boundary margins;
    q_norm: the draft rows' normalisers s3r_draft_sample wrote (optional)."""
    f32, i32 = torch.float32, torch.int32
    _check(_lib.s3r_spec_sample(
        ctypes.byref(batch), k, _ptr(p_logits, f32, "p_logits"),
        _ptr(q_logits, f32, "q_logits", allow_none=(k == 0)),
        _ptr(draft_tokens, i32, "draft_tokens", allow_none=(k == 0)), vocab, seed,
        _ptr(out_tokens, i32, "out_tokens"), _ptr(n_out, i32, "n_out"),
        _ptr(margins, f32, "margins", allow_none=True), _norms(q_norm, "q_norm"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "s3r_spec_sample")


def s3r_draft_argmax(batch, draft_step, k, q_logits, vocab, draft_tokens, ws, stream=None):
    _check(_lib.s3r_draft_argmax(
        ctypes.byref(batch), _ptr(draft_step, torch.int32, "draft_step"), k,
        _ptr(q_logits, torch.float32, "q_logits"), vocab,
        _ptr(draft_tokens, torch.int32, "draft_tokens"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream(stream)), "s3r_draft_argmax")


def s3r_greedy_verify(batch, k, p_logits, draft_tokens, vocab, out_tokens, n_out, ws, stream=None):
    i32 = torch.int32
    _check(_lib.s3r_greedy_verify(
        ctypes.byref(batch), k, _ptr(p_logits, torch.float32, "p_logits"),
        _ptr(draft_tokens, i32, "draft_tokens", allow_none=(k == 0)), vocab,
        _ptr(out_tokens, i32, "out_tokens"), _ptr(n_out, i32, "n_out"),
        _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream(stream)), "s3r_greedy_verify")


def s3r_commit(batch, k, n_out, seq_lens, stats=None, stream=None):
    _check(_lib.s3r_commit(
        ctypes.byref(batch), k, _ptr(n_out, torch.int32, "n_out"),
        _ptr(seq_lens, torch.int32, "seq_lens"), _ptr(stats, torch.int64, "stats", allow_none=True),
        _stream(stream)), "s3r_commit")


def s3r_choose_horizon(accepted, decided, c_draft, c_verify, prior_alpha=0.5, prior_weight=4.0):
    """Host call: draft length in [1, len(accepted)] from per-position counts (sequences of
    float; the first len(accepted) positions)."""
    k_max = len(accepted)
    if len(decided) != k_max:
        raise ValueError("accepted and decided differ in length")
    arr = ctypes.c_double * max(k_max, 1)
    a, d, out = arr(*accepted), arr(*decided), ctypes.c_int32(0)
    _check(_lib.s3r_choose_horizon(ctypes.cast(a, ctypes.c_void_p), ctypes.cast(d, ctypes.c_void_p),
                                   k_max, float(c_draft), float(c_verify), float(prior_alpha),
                                   float(prior_weight), ctypes.cast(ctypes.pointer(out), ctypes.c_void_p)),
           "s3r_choose_horizon")
    return int(out.value)


def s3r_choose_horizon_costs(accepted, decided, round_cost, prior_alpha=0.5, prior_weight=4.0):
    """Host call: draft length in [1, len(accepted)] from per-position counts and the cost of a
    round at each length 1..len(accepted) (round_cost)."""
    k_max = len(accepted)
    if len(decided) != k_max or len(round_cost) != k_max:
        raise ValueError("accepted, decided and round_cost differ in length")
    arr = ctypes.c_double * max(k_max, 1)
    a, d, c, out = arr(*accepted), arr(*decided), arr(*round_cost), ctypes.c_int32(0)
    _check(_lib.s3r_choose_horizon_costs(ctypes.cast(a, ctypes.c_void_p), ctypes.cast(d, ctypes.c_void_p), k_max,
                                         ctypes.cast(c, ctypes.c_void_p), float(prior_alpha), float(prior_weight),
                                         ctypes.cast(ctypes.pointer(out), ctypes.c_void_p)),
           "s3r_choose_horizon_costs")
    return int(out.value)


def s3r_horizon_step(stats_now, stats_last, accepted, decided, k_max, decay, c_draft, c_verify,
                     prior_alpha=-1.0, prior_weight=4.0):
    """Host call: decay / add the counts and choose k. stats_now, stats_last: numpy int64
    [2 + 2*MAX_K] (stats_last is updated); accepted, decided: numpy float64 [MAX_K] (updated).
    prior_alpha < 0 pools the prior. Returns (k, prior used)."""
    import numpy as np
    now = np.ascontiguousarray(stats_now, dtype=np.int64)
    for a, dt in ((stats_last, np.int64), (accepted, np.float64), (decided, np.float64)):
        if not (isinstance(a, np.ndarray) and a.dtype == dt and a.flags.c_contiguous):
            raise TypeError("stats_last / accepted / decided must be contiguous numpy arrays")
    if now.size != 2 + 2 * MAX_K or stats_last.size != now.size or accepted.size != MAX_K or decided.size != MAX_K:
        raise ValueError("counter arrays of the s3r_commit layout")
    k, prior = ctypes.c_int32(0), ctypes.c_double(0.0)
    vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    _check(_lib.s3r_horizon_step(vp(now), vp(stats_last), vp(accepted), vp(decided), k_max, float(decay),
                                 float(c_draft), float(c_verify), float(prior_alpha), float(prior_weight),
                                 ctypes.cast(ctypes.pointer(prior), ctypes.c_void_p),
                                 ctypes.cast(ctypes.pointer(k), ctypes.c_void_p)), "s3r_horizon_step")
    return int(k.value), float(prior.value)


def s3r_horizon_step_costs(stats_now, stats_last, accepted, decided, k_max, decay, round_cost,
                           prior_alpha=-1.0, prior_weight=4.0):
    """s3r_horizon_step choosing with the cost of a round at each length 1..k_max
    (round_cost, a sequence of k_max floats). Returns (k, prior used)."""
    import numpy as np
    now = np.ascontiguousarray(stats_now, dtype=np.int64)
    for a, dt in ((stats_last, np.int64), (accepted, np.float64), (decided, np.float64)):
        if not (isinstance(a, np.ndarray) and a.dtype == dt and a.flags.c_contiguous):
            raise TypeError("stats_last / accepted / decided must be contiguous numpy arrays")
    if now.size != 2 + 2 * MAX_K or stats_last.size != now.size or accepted.size != MAX_K or decided.size != MAX_K:
        raise ValueError("counter arrays of the s3r_commit layout")
    if len(round_cost) != k_max:
        raise ValueError("one round cost per draft length 1..k_max")
    cost = (ctypes.c_double * max(k_max, 1))(*[float(c) for c in round_cost])
    k, prior = ctypes.c_int32(0), ctypes.c_double(0.0)
    vp = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    _check(_lib.s3r_horizon_step_costs(vp(now), vp(stats_last), vp(accepted), vp(decided), k_max, float(decay),
                                       ctypes.cast(cost, ctypes.c_void_p), float(prior_alpha), float(prior_weight),
                                       ctypes.cast(ctypes.pointer(prior), ctypes.c_void_p),
                                       ctypes.cast(ctypes.pointer(k), ctypes.c_void_p)), "s3r_horizon_step_costs")
    return int(k.value), float(prior.value)


def s3r_sched_simulate(prompt_len, resp_len, tau, *, capacity, policy="aimd", evict="offload",
                       cap0=16, cap_min=1, cap_max=4096, u_low=0.85, u_high=0.97, b_high=1.0,
                       costs=(10.0, 0.0, 0.00074, 0.094, 0.5, 0.5), pressure=None,
                       max_iters=1 << 20, trace=True):
    """Host call: the KV-aware admission model over numpy inputs; returns (totals dict,
    trace int32 [iterations][8] or None)."""
    import numpy as np
    prompt = np.ascontiguousarray(prompt_len, dtype=np.int32)
    resp = np.ascontiguousarray(resp_len, dtype=np.int32)
    tau = np.ascontiguousarray(tau, dtype=np.uint8)
    if tau.ndim != 2 or tau.shape[0] != prompt.size or resp.size != prompt.size:
        raise ValueError("tau must be [num_requests][rounds]")
    pr = None if pressure is None else np.ascontiguousarray(pressure, dtype=np.int32)
    cfg = SchedConfig(capacity, {"aimd": 0, "fixed": 1}[policy], {"offload": 0, "recompute": 1}[evict],
                      cap0, cap_min, cap_max, u_low, u_high, b_high, *costs, max_iters)
    res = SchedResult()
    cap_rows = int(max_iters) if trace else 0
    cap_rows = min(cap_rows, 1 << 22)
    tr = np.zeros((cap_rows, 8), dtype=np.int32) if cap_rows else None
    vp = lambda a: None if a is None else a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    _check(_lib.s3r_sched_simulate(ctypes.byref(cfg), prompt.size, vp(prompt), vp(resp), vp(tau),
                                   tau.shape[1], vp(pr), 0 if pr is None else pr.size,
                                   ctypes.byref(res), vp(tr), cap_rows), "s3r_sched_simulate")
    tot = {f: getattr(res, f) for f, _ in SchedResult._fields_ if f != "reserved"}
    return tot, (tr[: min(res.iterations, cap_rows)] if tr is not None else None)


def s3r_philox(seed, stream_id, request, position, words=None, u=None, stream=None):
    _check(_lib.s3r_philox(
        seed, stream_id, _ptr(request, torch.int32, "request"),
        _ptr(position, torch.int32, "position"), request.numel(),
        _ptr(words, torch.int32, "words", allow_none=True),
        _ptr(u, torch.float32, "u", allow_none=True), _stream(stream)), "s3r_philox")


def s3r_get_error(ws, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(_lib.s3r_get_error(_ptr(ws, torch.uint8, "ws"), ctypes.byref(v), _stream(stream)),
           "s3r_get_error")
    return int(v.value)


def s3r_status_string(status: int) -> str:
    return _lib.s3r_status_string(status).decode()


def s3r_set_verify_kernel(which: int):
    """0: automatic (tcgen05 kernel where supported), 1: mma.sync kernel."""
    _check(_lib.s3r_set_verify_kernel(which), "s3r_set_verify_kernel")


def s3r_set_wait_limit(polls: int):
    """Bound on the tcgen05 verify's waits of one role for another (0: the default)."""
    _check(_lib.s3r_set_wait_limit(polls), "s3r_set_wait_limit")


def s3r_launch_count() -> int:
    return int(_lib.s3r_launch_count())
