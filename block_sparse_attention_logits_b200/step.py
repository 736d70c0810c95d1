"""One pass of the hot path over one batch, as the benchmark times it.

The pass (DFSAttn abstract: Hilbert reorder, block scoring; head-wise top-p
and GSRS abstracts: cumulative top-p selection per query block; CalibAtt
Fig. 5(b): attention over the kept blocks only; RECAP section 1: the cached
refinement scaled per head):

  with a latent grid (Hilbert order), gather=True:
    score_blocks_gather  block means of Q, K in curve order, read through perm
                         (no reordered copies)
    select_topp_mask     kept lists from the GPU's own block scores
    sparse_attn_fwd      (in_rows = perm) attention whose Q, K and V tiles are
                         gathered rows of the grid-order tensors, with the fused
                         O + alpha*R epilogue writing O and LSE in grid order
  with a latent grid, gather=False:
    score_blocks_gather  Q, K gathered into curve order inside the pooling pass
    permute_tokens       V gathered into curve order (on a side stream, beside
                         the block softmax and the selection, when given one)
    select_topp_mask     kept lists from the GPU's own block scores
    sparse_attn_fwd      attention with the fused O + alpha*R epilogue, writing
                         O and LSE straight back to grid order (row map = perm)
  without one:
    score_blocks -> select_topp_mask -> sparse_attn_fwd (+ alpha*R)

Every call is one of this library's C calls (api.py); nothing here computes.
`run_step` works on a dict of caller-owned buffers, so a head chunk of a
larger job can run the same pass on slices of the full buffers.
"""

import torch

from . import api


def alloc_buffers(B, H, L, D, blk, device, copies=True):
    """Device buffers of one pass: curve-order copies (unless copies=False),
    scores, lists, outputs."""
    nb = api.n_blocks(L, blk)
    dev = torch.device(device)
    bf = dict(dtype=torch.bfloat16, device=dev)
    cp = (lambda: torch.empty((B, H, L, D), **bf)) if copies else (lambda: None)
    return dict(
        qh=cp(), kh=cp(), vh=cp(),
        qp=torch.empty((B, H, nb, D), dtype=torch.float32, device=dev),
        kp=torch.empty((B, H, nb, D), dtype=torch.float32, device=dev),
        probs=torch.empty((B, H, nb, nb), dtype=torch.float32, device=dev),
        mask=torch.empty((B, H, nb, nb), dtype=torch.uint8, device=dev),
        idx=torch.empty((B, H, nb, nb), dtype=torch.int32, device=dev),
        cnt=torch.empty((B, H, nb), dtype=torch.int32, device=dev),
        oh=torch.empty((B, H, L, D), **bf),
        o=torch.empty((B, H, L, D), **bf),
        lse=torch.empty((B, H, L), dtype=torch.float32, device=dev),
    )


def run_step(b, q, k, v, blk, p, perm=None, R=None, alpha=None, status=None, events=None, gather=False,
             side=None):
    """One pass on buffers `b` (from alloc_buffers, or slices of them).

    q, k, v: bf16 [B,H,L,D] in grid order.  perm: the Hilbert order (int32
    [L], from api.reorder_tokens) or None for no reorder.  p: top-p, one float
    or one per head.  R (bf16 [B,H,L,D]) and alpha (float32 [H]) enable the
    fused correction; R is in curve order when perm is given without gather,
    in grid order otherwise.  gather (with perm): the attention gathers its
    tiles from the grid-order tensors, no reordered copies are made.
    events: optional three CUDA events recorded before scoring, after
    selection and after attention.  side: optional second CUDA stream for
    the V gather of the reordered-copies form: it starts when pooling is
    done (both are HBM-bound) and runs beside block softmax and selection
    (latency-bound); the attention waits for it.
    Returns (o, lse) in grid order.
    """
    B, H, L, D = q.shape
    if events:
        events[0].record()
    if perm is not None and gather:
        api.score_blocks_gather(q, k, perm, blk, None, None, b["qp"], b["kp"], b["probs"], copies=False)
        api.select_topp_mask(b["probs"], p, L, blk, D, b["mask"], b["idx"], b["cnt"])
        if events:
            events[1].record()
        api.sparse_attn_fwd(q, k, v, blk, b["idx"], b["cnt"], R, alpha, b["o"], b["lse"], status=status,
                            in_rows=perm)
        if events:
            events[2].record()
        return b["o"], b["lse"]
    v_done = None
    if perm is not None:
        api.score_blocks_gather(q, k, perm, blk, b["qh"], b["kh"], b["qp"], b["kp"], b["probs"])
        if side is not None:
            pooled = torch.cuda.Event()
            pooled.record()
            side.wait_event(pooled)
            with torch.cuda.stream(side):
                api.permute_tokens(v, perm, out=b["vh"])
                v_done = torch.cuda.Event()
                v_done.record()
        else:
            api.permute_tokens(v, perm, out=b["vh"])
        qs, ks, vs = b["qh"], b["kh"], b["vh"]
    else:
        qs, ks, vs = q, k, v
        api.score_blocks(qs, ks, blk, b["qp"], b["kp"], b["probs"])
    api.select_topp_mask(b["probs"], p, L, blk, D, b["mask"], b["idx"], b["cnt"])
    if v_done is not None:
        torch.cuda.current_stream().wait_event(v_done)
    if events:
        events[1].record()
    o = b["o"] if perm is not None else b["oh"]
    api.sparse_attn_fwd(qs, ks, vs, blk, b["idx"], b["cnt"], R, alpha, o, b["lse"], status=status, out_rows=perm)
    if events:
        events[2].record()
    return o, b["lse"]
