"""Python binding of libbsa: one function per C-ABI call, same names.

Each function only marshals torch tensors (device memory, the current CUDA
stream) into the C call and raises on a non-zero status; every step of the
computation runs in libbsa's kernels.  Outputs are allocated with torch when
not passed in.  All calls are asynchronous on the current stream.
"""

import ctypes

import torch

from . import _lib
from ._lib import Shape, check

__all__ = [
    "n_blocks",
    "version",
    "score_blocks",
    "score_blocks_gather",
    "block_drift",
    "select_topp_mask",
    "max_intervals",
    "interval_runs",
    "interval_width_for_merge",
    "kept_to_intervals",
    "intervals_to_kept",
    "tail_workspace_bytes",
    "tail_stats",
    "coarse_tail",
    "tail_refinement",
    "tail_reconstruct",
    "complement_lists",
    "quantize_fp8",
    "sparse_attn_fwd_fp8",
    "reorder_workspace_bytes",
    "reorder_tokens",
    "permute_tokens",
    "sparse_attn_fwd",
    "sparse_attn_refresh",
    "refresh_refinement",
    "apply_correction",
]


def n_blocks(L, blk):
    return (L + blk - 1) // blk


def version():
    return _lib.load().bsa_version()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, dtype, shape, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    return t


def _shape(q, blk):
    B, H, L, D = q.shape
    return Shape(B, H, L, D, blk)


def score_blocks(q, k, blk, q_pool=None, k_pool=None, probs=None, candidates=None):
    """Block means of Q and K and the per-query-block softmax of their logits.

    q, k: bf16 [B,H,L,D].  Returns (q_pool, k_pool, probs): float32
    [B,H,NB,D], [B,H,NB,D], [B,H,NB,NB].  With `candidates` (uint8
    [B,H,NB,NB]) each row's softmax runs over its candidate blocks only.
    """
    B, H, L, D = q.shape
    nb = n_blocks(L, blk)
    _need(q, torch.bfloat16, (B, H, L, D), "q")
    _need(k, torch.bfloat16, (B, H, L, D), "k")
    dev = q.device
    q_pool = q_pool if q_pool is not None else torch.empty((B, H, nb, D), dtype=torch.float32, device=dev)
    k_pool = k_pool if k_pool is not None else torch.empty((B, H, nb, D), dtype=torch.float32, device=dev)
    probs = probs if probs is not None else torch.empty((B, H, nb, nb), dtype=torch.float32, device=dev)
    _need(q_pool, torch.float32, (B, H, nb, D), "q_pool")
    _need(k_pool, torch.float32, (B, H, nb, D), "k_pool")
    _need(probs, torch.float32, (B, H, nb, nb), "probs")
    if candidates is None:
        check("bsa_score_blocks", _lib.load().bsa_score_blocks(
            _shape(q, blk), _ptr(q), _ptr(k), _ptr(q_pool), _ptr(k_pool), _ptr(probs), _stream()))
    else:
        _need(candidates, torch.uint8, (B, H, nb, nb), "candidates")
        check("bsa_score_blocks_restricted", _lib.load().bsa_score_blocks_restricted(
            _shape(q, blk), _ptr(q), _ptr(k), _ptr(candidates), _ptr(q_pool), _ptr(k_pool), _ptr(probs),
            _stream()))
    return q_pool, k_pool, probs


def score_blocks_gather(q, k, perm, blk, q_out=None, k_out=None, q_pool=None, k_pool=None, probs=None,
                        copies=True):
    """permute_tokens(q), permute_tokens(k) and score_blocks of the results in
    one pass.  Returns (q_out, k_out, q_pool, k_pool, probs); with
    copies=False the reordered q and k are not written (q_out = k_out = None),
    for sparse_attn_fwd(..., in_rows=perm)."""
    B, H, L, D = q.shape
    nb = n_blocks(L, blk)
    _need(q, torch.bfloat16, (B, H, L, D), "q")
    _need(k, torch.bfloat16, (B, H, L, D), "k")
    _need(perm, torch.int32, (L,), "perm")
    dev = q.device
    if copies:
        q_out = q_out if q_out is not None else torch.empty_like(q)
        k_out = k_out if k_out is not None else torch.empty_like(k)
    else:
        q_out = k_out = None
    q_pool = q_pool if q_pool is not None else torch.empty((B, H, nb, D), dtype=torch.float32, device=dev)
    k_pool = k_pool if k_pool is not None else torch.empty((B, H, nb, D), dtype=torch.float32, device=dev)
    probs = probs if probs is not None else torch.empty((B, H, nb, nb), dtype=torch.float32, device=dev)
    if copies:
        for name, t in (("q_out", q_out), ("k_out", k_out)):
            _need(t, torch.bfloat16, (B, H, L, D), name)
    _need(q_pool, torch.float32, (B, H, nb, D), "q_pool")
    _need(k_pool, torch.float32, (B, H, nb, D), "k_pool")
    _need(probs, torch.float32, (B, H, nb, nb), "probs")
    check("bsa_score_blocks_gather", _lib.load().bsa_score_blocks_gather(
        _shape(q, blk), _ptr(q), _ptr(k), _ptr(perm), _ptr(q_out), _ptr(k_out), _ptr(q_pool), _ptr(k_pool),
        _ptr(probs), _stream()))
    return q_out, k_out, q_pool, k_pool, probs


def block_drift(q_pool_ref, k_pool_ref, q_pool, k_pool, L, blk, drift=None):
    """Per-head query-key drift of the block means since a reference step:
    max of the relative Frobenius changes of the Q and K means.  Inputs
    float32 [B,H,NB,D]; returns float32 [B*H] on the device."""
    B, H, nb, D = q_pool.shape
    for name, t in (("q_pool_ref", q_pool_ref), ("k_pool_ref", k_pool_ref), ("q_pool", q_pool), ("k_pool", k_pool)):
        _need(t, torch.float32, (B, H, nb, D), name)
    drift = drift if drift is not None else torch.empty((B * H,), dtype=torch.float32, device=q_pool.device)
    _need(drift, torch.float32, (B * H,), "drift")
    check("bsa_block_drift", _lib.load().bsa_block_drift(
        Shape(B, H, L, D, blk), _ptr(q_pool_ref), _ptr(k_pool_ref), _ptr(q_pool), _ptr(k_pool), _ptr(drift),
        _stream()))
    return drift


def select_topp_mask(probs, p, L, blk, D=128, mask=None, kept_idx=None, kept_cnt=None, candidates=None):
    """Cumulative top-p selection per query block.

    probs: float32 [B,H,NB,NB]; p: per-head thresholds (sequence of H floats
    in (0,1]) or one float for every head.  Returns (mask uint8, kept_idx
    int32, kept_cnt int32).  With `candidates` (uint8 [B,H,NB,NB]) the search
    runs over each row's candidate blocks only.
    """
    B, H, nb, _ = probs.shape
    _need(probs, torch.float32, (B, H, nb, nb), "probs")
    if isinstance(p, (int, float)):
        p = [float(p)] * H
    p = [float(x) for x in p]
    if len(p) != H:
        raise ValueError("p must have one value per head")
    dev = probs.device
    mask = mask if mask is not None else torch.empty((B, H, nb, nb), dtype=torch.uint8, device=dev)
    kept_idx = kept_idx if kept_idx is not None else torch.empty((B, H, nb, nb), dtype=torch.int32, device=dev)
    kept_cnt = kept_cnt if kept_cnt is not None else torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    _need(mask, torch.uint8, (B, H, nb, nb), "mask")
    _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
    _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    parr = (ctypes.c_float * H)(*p)
    if candidates is None:
        check("bsa_select_topp_mask", _lib.load().bsa_select_topp_mask(
            Shape(B, H, L, D, blk), _ptr(probs), parr, _ptr(mask), _ptr(kept_idx), _ptr(kept_cnt), _stream()))
    else:
        _need(candidates, torch.uint8, (B, H, nb, nb), "candidates")
        check("bsa_select_topp_mask_restricted", _lib.load().bsa_select_topp_mask_restricted(
            Shape(B, H, L, D, blk), _ptr(probs), parr, _ptr(candidates), _ptr(mask), _ptr(kept_idx),
            _ptr(kept_cnt), _stream()))
    return mask, kept_idx, kept_cnt


def max_intervals(NB):
    """Most runs (intervals) a row of NB key blocks can have."""
    return (NB + 1) // 2


def interval_runs(kept_idx, kept_cnt, L, blk, D=128, n_runs=None, hist=None, status=None):
    """Runs of consecutive kept blocks per row, and their histogram.

    kept_idx int32 [B,H,NB,NB], kept_cnt int32 [B,H,NB].  Returns (n_runs
    int32 [B,H,NB], hist int32 [max_intervals(NB) + 1]).  A passed-in hist is
    accumulated into (not cleared); a new one starts at zero.
    """
    B, H, nb = kept_cnt.shape
    _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
    _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    dev = kept_cnt.device
    n_runs = n_runs if n_runs is not None else torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    hist = hist if hist is not None else torch.zeros(max_intervals(nb) + 1, dtype=torch.int32, device=dev)
    _need(n_runs, torch.int32, (B, H, nb), "n_runs")
    _need(hist, torch.int32, (max_intervals(nb) + 1,), "hist")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_interval_runs", _lib.load().bsa_interval_runs(
        Shape(B, H, L, D, blk), _ptr(kept_idx), _ptr(kept_cnt), _ptr(n_runs), _ptr(hist), _ptr(status), _stream()))
    return n_runs, hist


def interval_width_for_merge(hist, q):
    """Interval width for a merge percentage q in (0, 1] (host computation in
    libbsa): the smallest W >= 1 that at least ceil(q * rows) rows fit.
    hist: the interval_runs histogram (any device; copied to the host)."""
    h = hist.detach().to("cpu", torch.int32).contiguous() if isinstance(hist, torch.Tensor) else \
        torch.tensor(list(hist), dtype=torch.int32)
    arr = (ctypes.c_int32 * h.numel())(*h.tolist())
    w = ctypes.c_int(0)
    check("bsa_interval_width_for_merge", _lib.load().bsa_interval_width_for_merge(
        arr, h.numel(), float(q), ctypes.byref(w)))
    return w.value


def kept_to_intervals(kept_idx, kept_cnt, W, L, blk, D=128, intervals=None, n_int=None, n_runs=None, status=None):
    """Encode kept lists as interval pairs of width W (rows with more runs are
    merged by filling their smallest gaps).  Returns (intervals int32
    [B,H,NB,W,2], n_int int32 [B,H,NB], n_runs int32 [B,H,NB])."""
    B, H, nb = kept_cnt.shape
    _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
    _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    dev = kept_cnt.device
    intervals = intervals if intervals is not None else torch.empty((B, H, nb, W, 2), dtype=torch.int32, device=dev)
    n_int = n_int if n_int is not None else torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    n_runs = n_runs if n_runs is not None else torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    _need(intervals, torch.int32, (B, H, nb, W, 2), "intervals")
    _need(n_int, torch.int32, (B, H, nb), "n_int")
    _need(n_runs, torch.int32, (B, H, nb), "n_runs")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_kept_to_intervals", _lib.load().bsa_kept_to_intervals(
        Shape(B, H, L, D, blk), _ptr(kept_idx), _ptr(kept_cnt), int(W), _ptr(intervals), _ptr(n_int),
        _ptr(n_runs), _ptr(status), _stream()))
    return intervals, n_int, n_runs


def intervals_to_kept(intervals, n_int, L, blk, D=128, mask=None, kept_idx=None, kept_cnt=None, want_mask=True,
                      status=None):
    """Decode interval pairs (int32 [B,H,NB,W,2], n_int int32 [B,H,NB]) into
    (mask uint8 or None, kept_idx int32 [B,H,NB,NB], kept_cnt int32 [B,H,NB]),
    the lists sparse_attn_fwd takes."""
    B, H, nb, W, _ = intervals.shape
    _need(intervals, torch.int32, (B, H, nb, W, 2), "intervals")
    _need(n_int, torch.int32, (B, H, nb), "n_int")
    dev = n_int.device
    if want_mask:
        mask = mask if mask is not None else torch.empty((B, H, nb, nb), dtype=torch.uint8, device=dev)
        _need(mask, torch.uint8, (B, H, nb, nb), "mask")
    else:
        mask = None
    kept_idx = kept_idx if kept_idx is not None else torch.empty((B, H, nb, nb), dtype=torch.int32, device=dev)
    kept_cnt = kept_cnt if kept_cnt is not None else torch.empty((B, H, nb), dtype=torch.int32, device=dev)
    _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
    _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_intervals_to_kept", _lib.load().bsa_intervals_to_kept(
        Shape(B, H, L, D, blk), _ptr(intervals), _ptr(n_int), int(W), _ptr(mask), _ptr(kept_idx), _ptr(kept_cnt),
        _ptr(status), _stream()))
    return mask, kept_idx, kept_cnt


def tail_workspace_bytes(B, H, L, D, blk):
    """Device bytes of the workspace tail_stats and coarse_tail share."""
    return _lib.load().bsa_tail_workspace_bytes(Shape(B, H, L, D, blk))


def tail_stats(k, v, blk, ws=None, status=None):
    """Block moments and pooled covariance of K and V (D = 128).  Returns
    (kbar, s2, vbar float32 [B,H,NB,D], C float32 [B,H,D,D], ws); ws holds the
    operand tables coarse_tail reads."""
    B, H, L, D = k.shape
    nb = n_blocks(L, blk)
    _need(k, torch.bfloat16, (B, H, L, D), "k")
    _need(v, torch.bfloat16, (B, H, L, D), "v")
    dev = k.device
    nbytes = tail_workspace_bytes(B, H, L, D, blk)
    if nbytes == 0:
        raise ValueError("unsupported shape for the coarse tail (D must be 128)")
    ws = ws if ws is not None else torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _need(ws, torch.uint8, (ws.numel(),), "ws")
    kbar, s2, vbar = (torch.empty((B, H, nb, D), dtype=torch.float32, device=dev) for _ in range(3))
    C = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_tail_stats", _lib.load().bsa_tail_stats(
        Shape(B, H, L, D, blk), _ptr(k), _ptr(v), _ptr(kbar), _ptr(s2), _ptr(vbar), _ptr(C), _ptr(ws), ws.numel(),
        _ptr(status), _stream()))
    return kbar, s2, vbar, C, ws


def coarse_tail(q, mask, blk, ws, status=None):
    """(lbar float32 [B,H,L], obar bf16 [B,H,L,D]) over the blocks each query
    block omits (mask uint8 [B,H,NB,NB], 1 = kept); ws from tail_stats."""
    B, H, L, D = q.shape
    nb = n_blocks(L, blk)
    _need(q, torch.bfloat16, (B, H, L, D), "q")
    _need(mask, torch.uint8, (B, H, nb, nb), "mask")
    _need(ws, torch.uint8, (ws.numel(),), "ws")
    lbar = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    obar = torch.empty_like(q)
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_coarse_tail", _lib.load().bsa_coarse_tail(
        Shape(B, H, L, D, blk), _ptr(q), _ptr(mask), _ptr(ws), ws.numel(), _ptr(lbar), _ptr(obar), _ptr(status),
        _stream()))
    return lbar, obar


def tail_refinement(l_T, o_T, lbar, obar):
    """(d_l float32 [B,H,L], d_o bf16 [B,H,L,D]) cached at a dense refresh."""
    B, H, L, D = o_T.shape
    _need(l_T, torch.float32, (B, H, L), "l_T")
    _need(o_T, torch.bfloat16, (B, H, L, D), "o_T")
    _need(lbar, torch.float32, (B, H, L), "lbar")
    _need(obar, torch.bfloat16, (B, H, L, D), "obar")
    d_l, d_o = torch.empty_like(lbar), torch.empty_like(obar)
    check("bsa_tail_refinement", _lib.load().bsa_tail_refinement(
        Shape(B, H, L, D, 0), _ptr(l_T), _ptr(o_T), _ptr(lbar), _ptr(obar), _ptr(d_l), _ptr(d_o), _stream()))
    return d_l, d_o


def tail_reconstruct(l_S, o_S, lbar, obar, d_l, d_o):
    """(o bf16 [B,H,L,D], lse float32 [B,H,L]): the sparse part merged with the
    reconstructed tail."""
    B, H, L, D = o_S.shape
    for name, t in (("l_S", l_S), ("lbar", lbar), ("d_l", d_l)):
        _need(t, torch.float32, (B, H, L), name)
    for name, t in (("o_S", o_S), ("obar", obar), ("d_o", d_o)):
        _need(t, torch.bfloat16, (B, H, L, D), name)
    o, lse = torch.empty_like(o_S), torch.empty_like(l_S)
    check("bsa_tail_reconstruct", _lib.load().bsa_tail_reconstruct(
        Shape(B, H, L, D, 0), _ptr(l_S), _ptr(o_S), _ptr(lbar), _ptr(obar), _ptr(d_l), _ptr(d_o), _ptr(o),
        _ptr(lse), _stream()))
    return o, lse


def complement_lists(mask, L, blk, D=128):
    """The blocks each row does not keep: (idx int32 [B,H,NB,NB], cnt int32 [B,H,NB])."""
    B, H, nb, _ = mask.shape
    _need(mask, torch.uint8, (B, H, nb, nb), "mask")
    idx = torch.empty((B, H, nb, nb), dtype=torch.int32, device=mask.device)
    cnt = torch.empty((B, H, nb), dtype=torch.int32, device=mask.device)
    check("bsa_complement_lists", _lib.load().bsa_complement_lists(
        Shape(B, H, L, D, blk), _ptr(mask), _ptr(idx), _ptr(cnt), _stream()))
    return idx, cnt


def quantize_fp8(x, blk, codes=None, scales=None):
    """E4M3 codes (uint8 [B,H,L,D]) and per-block scales (float32 [B,H,NB]) of
    a bf16 [B,H,L,D] tensor: scale = amax / 448 per (b, h, block)."""
    B, H, L, D = x.shape
    nb = n_blocks(L, blk)
    _need(x, torch.bfloat16, (B, H, L, D), "x")
    codes = codes if codes is not None else torch.empty((B, H, L, D), dtype=torch.uint8, device=x.device)
    scales = scales if scales is not None else torch.empty((B, H, nb), dtype=torch.float32, device=x.device)
    _need(codes, torch.uint8, (B, H, L, D), "codes")
    _need(scales, torch.float32, (B, H, nb), "scales")
    check("bsa_quantize_fp8", _lib.load().bsa_quantize_fp8(
        Shape(B, H, L, D, blk), _ptr(x), _ptr(codes), _ptr(scales), _stream()))
    return codes, scales


def sparse_attn_fwd_fp8(q8, q_scale, k8, k_scale, v, blk, kept_idx=None, kept_cnt=None, R=None, alpha=None,
                        o=None, lse=None, status=None):
    """Block-sparse attention with S = Q.K^T from E4M3 codes (blk 128, D 128);
    otherwise as sparse_attn_fwd.  Returns (o bf16, lse float32)."""
    B, H, L, D = v.shape
    nb = n_blocks(L, blk)
    _need(v, torch.bfloat16, (B, H, L, D), "v")
    for name, t in (("q8", q8), ("k8", k8)):
        _need(t, torch.uint8, (B, H, L, D), name)
    for name, t in (("q_scale", q_scale), ("k_scale", k_scale)):
        _need(t, torch.float32, (B, H, nb), name)
    if kept_idx is not None:
        _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
        _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    if R is not None:
        _need(R, torch.bfloat16, (B, H, L, D), "R")
        _need(alpha, torch.float32, (H,), "alpha")
    o = o if o is not None else torch.empty_like(v)
    lse = lse if lse is not None else torch.empty((B, H, L), dtype=torch.float32, device=v.device)
    _need(o, torch.bfloat16, (B, H, L, D), "o")
    _need(lse, torch.float32, (B, H, L), "lse")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_sparse_attn_fwd_fp8", _lib.load().bsa_sparse_attn_fwd_fp8(
        Shape(B, H, L, D, blk), _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(k_scale), _ptr(v), _ptr(kept_idx),
        _ptr(kept_cnt), _ptr(R), _ptr(alpha), _ptr(o), _ptr(lse), _ptr(status), _stream()))
    return o, lse


def reorder_workspace_bytes(T, Hh, W):
    return int(_lib.load().bsa_reorder_workspace_bytes(T, Hh, W))


def reorder_tokens(T, Hh, W, device="cuda", perm=None, inv=None, workspace=None):
    """Hilbert-curve order of a (T, Hh, W) latent grid: (perm, inv) int32 [L]."""
    L = T * Hh * W
    perm = perm if perm is not None else torch.empty(L, dtype=torch.int32, device=device)
    inv = inv if inv is not None else torch.empty(L, dtype=torch.int32, device=device)
    _need(perm, torch.int32, (L,), "perm")
    _need(inv, torch.int32, (L,), "inv")
    nbytes = reorder_workspace_bytes(T, Hh, W)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=perm.device)
    _need(workspace, torch.uint8, (workspace.numel(),), "workspace")
    check("bsa_reorder_tokens", _lib.load().bsa_reorder_tokens(
        T, Hh, W, _ptr(perm), _ptr(inv), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream()))
    return perm, inv


def permute_tokens(x, perm, inverse=False, out=None):
    """Gather rows into curve order (inverse=False) or scatter them back."""
    B, H, L, D = x.shape
    _need(x, torch.bfloat16, (B, H, L, D), "x")
    _need(perm, torch.int32, (L,), "perm")
    out = out if out is not None else torch.empty_like(x)
    _need(out, torch.bfloat16, (B, H, L, D), "out")
    check("bsa_permute_tokens", _lib.load().bsa_permute_tokens(
        Shape(B, H, L, D, 0), _ptr(x), _ptr(perm), _ptr(out), 1 if inverse else 0, _stream()))
    return out


def sparse_attn_fwd(q, k, v, blk, kept_idx=None, kept_cnt=None, R=None, alpha=None,
                    o=None, lse=None, status=None, out_rows=None, in_rows=None):
    """Block-sparse attention over the kept blocks (dense when kept_* are None).

    Returns (o bf16 [B,H,L,D], lse float32 [B,H,L]).  With R / alpha the
    epilogue adds alpha_h * R.  `status` (int32 [1] on the device, zeroed by
    the caller) receives BSA_DEV_* bits.  With `out_rows` (int32 [L], a
    permutation; blk 128) output row r goes to row out_rows[r] of o and lse.
    With `in_rows` (int32 [L], a permutation; blk = D = 128) the attention
    runs over the tokens in that order with q, k, v, R, o and lse all in the
    caller's order: token t is row in_rows[t] (bsa_sparse_attn_fwd_gather).
    """
    B, H, L, D = q.shape
    nb = n_blocks(L, blk)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, (B, H, L, D), name)
    if kept_idx is not None:
        _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
        _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    if R is not None:
        _need(R, torch.bfloat16, (B, H, L, D), "R")
        _need(alpha, torch.float32, (H,), "alpha")
    o = o if o is not None else torch.empty_like(q)
    lse = lse if lse is not None else torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, (B, H, L, D), "o")
    _need(lse, torch.float32, (B, H, L), "lse")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    if in_rows is not None:
        if out_rows is not None:
            raise ValueError("in_rows writes the output through the same rows: pass no out_rows")
        _need(in_rows, torch.int32, (L,), "in_rows")
        check("bsa_sparse_attn_fwd_gather", _lib.load().bsa_sparse_attn_fwd_gather(
            Shape(B, H, L, D, blk), _ptr(q), _ptr(k), _ptr(v), _ptr(in_rows), _ptr(kept_idx), _ptr(kept_cnt),
            _ptr(R), _ptr(alpha), _ptr(o), _ptr(lse), _ptr(status), _stream()))
    elif out_rows is None:
        check("bsa_sparse_attn_fwd", _lib.load().bsa_sparse_attn_fwd(
            Shape(B, H, L, D, blk), _ptr(q), _ptr(k), _ptr(v), _ptr(kept_idx), _ptr(kept_cnt),
            _ptr(R), _ptr(alpha), _ptr(o), _ptr(lse), _ptr(status), _stream()))
    else:
        _need(out_rows, torch.int32, (L,), "out_rows")
        check("bsa_sparse_attn_fwd_scatter", _lib.load().bsa_sparse_attn_fwd_scatter(
            Shape(B, H, L, D, blk), _ptr(q), _ptr(k), _ptr(v), _ptr(kept_idx), _ptr(kept_cnt),
            _ptr(R), _ptr(alpha), _ptr(out_rows), _ptr(o), _ptr(lse), _ptr(status), _stream()))
    return o, lse


def sparse_attn_fwd_intervals(q, k, v, blk, intervals, n_int, R=None, alpha=None, o=None, lse=None, status=None):
    """Block-sparse attention with the kept blocks given as interval pairs
    (int32 [B,H,NB,W,2] and int32 [B,H,NB], as kept_to_intervals returns
    them), walked by the kernel itself; blk 128.  Same result as
    sparse_attn_fwd on intervals_to_kept of the same pairs."""
    B, H, L, D = q.shape
    nb = n_blocks(L, blk)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, (B, H, L, D), name)
    if intervals.dim() != 5:
        raise ValueError("intervals must be int32 [B,H,NB,W,2]")
    W = intervals.shape[3]
    _need(intervals, torch.int32, (B, H, nb, W, 2), "intervals")
    _need(n_int, torch.int32, (B, H, nb), "n_int")
    if R is not None:
        _need(R, torch.bfloat16, (B, H, L, D), "R")
        _need(alpha, torch.float32, (H,), "alpha")
    o = o if o is not None else torch.empty_like(q)
    lse = lse if lse is not None else torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    _need(o, torch.bfloat16, (B, H, L, D), "o")
    _need(lse, torch.float32, (B, H, L), "lse")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_sparse_attn_fwd_intervals", _lib.load().bsa_sparse_attn_fwd_intervals(
        Shape(B, H, L, D, blk), _ptr(q), _ptr(k), _ptr(v), _ptr(intervals), _ptr(n_int), W,
        _ptr(R), _ptr(alpha), _ptr(o), _ptr(lse), _ptr(status), _stream()))
    return o, lse


def sparse_attn_refresh(q, k, v, blk, kept_idx, kept_cnt, want_r=True, want_mass=True, out=None, status=None):
    """Dense refresh in one pass over every key block.

    Returns (o_dense, lse_dense, o_sparse, lse_sparse, R, kept_mass): the dense
    and the kept-block attention (bf16 O, float32 LSE), R = bf16(bf16(o_dense)
    - bf16(o_sparse)) (None unless want_r) and the kept share of the attention
    weight per row (None unless want_mass).  blk must be 128.  `out` may hold
    preallocated tensors under the same names.
    """
    B, H, L, D = q.shape
    nb = n_blocks(L, blk)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, torch.bfloat16, (B, H, L, D), name)
    _need(kept_idx, torch.int32, (B, H, nb, nb), "kept_idx")
    _need(kept_cnt, torch.int32, (B, H, nb), "kept_cnt")
    out = dict(out or {})
    dev = q.device
    o_d = out.get("o_dense", None)
    o_d = o_d if o_d is not None else torch.empty_like(q)
    o_s = out.get("o_sparse", None)
    o_s = o_s if o_s is not None else torch.empty_like(q)
    l_d = out.get("lse_dense", None)
    l_d = l_d if l_d is not None else torch.empty((B, H, L), dtype=torch.float32, device=dev)
    l_s = out.get("lse_sparse", None)
    l_s = l_s if l_s is not None else torch.empty((B, H, L), dtype=torch.float32, device=dev)
    R = out.get("R", None) if want_r else None
    R = R if (R is not None or not want_r) else torch.empty_like(q)
    mass = out.get("kept_mass", None) if want_mass else None
    mass = mass if (mass is not None or not want_mass) else torch.empty((B, H, L), dtype=torch.float32, device=dev)
    for name, t in (("o_dense", o_d), ("o_sparse", o_s)):
        _need(t, torch.bfloat16, (B, H, L, D), name)
    for name, t in (("lse_dense", l_d), ("lse_sparse", l_s)):
        _need(t, torch.float32, (B, H, L), name)
    if R is not None:
        _need(R, torch.bfloat16, (B, H, L, D), "R")
    if mass is not None:
        _need(mass, torch.float32, (B, H, L), "kept_mass")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    check("bsa_sparse_attn_refresh", _lib.load().bsa_sparse_attn_refresh(
        Shape(B, H, L, D, blk), _ptr(q), _ptr(k), _ptr(v), _ptr(kept_idx), _ptr(kept_cnt),
        _ptr(o_d), _ptr(l_d), _ptr(o_s), _ptr(l_s), _ptr(R), _ptr(mass), _ptr(status), _stream()))
    return o_d, l_d, o_s, l_s, R, mass


def refresh_refinement(o_dense, o_sparse, out=None):
    """R = bf16(o_dense - o_sparse)."""
    B, H, L, D = o_dense.shape
    _need(o_dense, torch.bfloat16, (B, H, L, D), "o_dense")
    _need(o_sparse, torch.bfloat16, (B, H, L, D), "o_sparse")
    out = out if out is not None else torch.empty_like(o_dense)
    _need(out, torch.bfloat16, (B, H, L, D), "out")
    check("bsa_refresh_refinement", _lib.load().bsa_refresh_refinement(
        Shape(B, H, L, D, 0), _ptr(o_dense), _ptr(o_sparse), _ptr(out), _stream()))
    return out


def apply_correction(o_sparse, R, alpha, out=None):
    """o = bf16(o_sparse + alpha_h * R)."""
    B, H, L, D = o_sparse.shape
    _need(o_sparse, torch.bfloat16, (B, H, L, D), "o_sparse")
    _need(R, torch.bfloat16, (B, H, L, D), "R")
    _need(alpha, torch.float32, (H,), "alpha")
    out = out if out is not None else torch.empty_like(o_sparse)
    _need(out, torch.bfloat16, (B, H, L, D), "out")
    check("bsa_apply_correction", _lib.load().bsa_apply_correction(
        Shape(B, H, L, D, 0), _ptr(o_sparse), _ptr(R), _ptr(alpha), _ptr(out), _stream()))
    return out
