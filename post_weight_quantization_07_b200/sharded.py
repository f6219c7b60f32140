"""One layer quantised by several GPUs: tokens and rows sharded.

H = 2 Xhat^T Xhat and the QEP cross term D = (X - Xhat)^T Xhat are sums over
calibration tokens, so rank r computes them over its own token shard
(oc_qep_terms) and one all-reduce of the two n x n matrices (NCCL over NVLink
under torch.distributed) gives every rank the layer's global terms.  QEP and
GPTQ treat the rows of W independently given H and D, so rank r then finishes
its own shard of rows (oc_quantize_from_terms); the inverse-Hessian
factorisation is repeated on every rank (it depends only on H).

The compute and reduction steps are parameters so that the same orchestration
can be exercised without GPUs; by default they are the library's calls and
torch.distributed.all_reduce.
"""
from __future__ import annotations


def shard_range(total: int, rank: int, world: int, align: int = 1):
    """[start, stop) of shard `rank` of `total` items split into `world`
    contiguous shards whose sizes differ by at most `align` (starts are
    multiples of `align`)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    units = (total + align - 1) // align
    base, extra = divmod(units, world)
    start = (rank * base + min(rank, extra)) * align
    stop = ((rank + 1) * base + min(rank + 1, extra)) * align
    return min(start, total), min(stop, total)


def quantize_layer_sharded(W_rows, X_tok, Xhat_tok, alpha, damp, wbits, groupsize, act_order, *,
                           group=None, terms=None, finish=None, all_reduce=None):
    """QEP + GPTQ of the rows W_rows of a layer whose calibration tokens are
    sharded over the ranks of `group` (X_tok, Xhat_tok: this rank's tokens).

    Every rank must call this with its own shards, in the same order (one
    collective per term).  Returns (H, D, finish(...)'s results for W_rows).
    """
    if terms is None or finish is None:
        from . import oc_qep_terms, oc_quantize_from_terms
        terms = terms or oc_qep_terms
        finish = finish or oc_quantize_from_terms
    if all_reduce is None:
        import torch.distributed as dist

        def all_reduce(t):
            dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    H, D = terms(X_tok, Xhat_tok)
    all_reduce(H)
    all_reduce(D)
    return H, D, finish(W_rows, H, D, alpha, damp, wbits, groupsize, act_order)
