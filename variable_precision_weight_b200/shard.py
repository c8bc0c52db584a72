"""The read split over ranks: host-side plumbing around the C-ABI calls.

Every rank reads a contiguous range of each layer's 64-row blocks (``fl_shard_blocks``,
balanced by the bytes the blocks' depths read) with the ordinary GEMV calls on pointer
offsets into the plane store, writes its rows into one local buffer, and the ranks exchange
those buffers with one all-gather. The gate's vocabulary is split with the head's blocks:
each rank reduces its logits to a partial (``fl_logit_gate_partial``), the partials are
all-gathered, and every rank merges the same records in rank order
(``fl_logit_gate_merge``), so all ranks take the same escalation decision.

Only argument marshalling and torch.distributed calls live here; every step of the read runs
in libfl.
"""
from __future__ import annotations

from . import fl

STORE_BYTES_PER_BLOCK_GROUP = 8448  # bytes of one 64-row block per 128-column group in the plane store


def plan(levels_host, ins, nranks: int):
    """Per layer, the first-block list of every rank (nranks + 1 entries).

    levels_host: list of host uint8 arrays (one per layer); ins: the layers' input widths."""
    return [fl.fl_shard_blocks(lv, inn, nranks) for lv, inn in zip(levels_host, ins)]


def rank_rows(plans, rank: int):
    """Rows this rank owns in each layer: [(layer, first row, row count)], and their total."""
    rows, total = [], 0
    for li, first in enumerate(plans):
        b0, b1 = first[rank], first[rank + 1]
        rows.append((li, 64 * b0, 64 * (b1 - b0)))
        total += 64 * (b1 - b0)
    return rows, total


def local_items(layers, plans, rank: int, y_local, batch: int = 1, to_levels=None):
    """fl_gemv_problem tuples for this rank's block ranges.

    layers: [(store, out, in, levels, x)] with device tensors; to_levels: the layers' device
    to-levels for a residual pass. y_local: this rank's flat output buffer; the rows of each
    layer it owns are one [batch][rows] block, blocks back to back in layer order. A layer whose
    range is empty is left out. Returns (items, [(layer, element offset in y_local, rows)])."""
    items, placed, off = [], [], 0
    rows, total = rank_rows(plans, rank)
    for (li, r0, n), (store, out, inn, lv, x) in zip(rows, layers):
        if n == 0:
            continue
        b0 = r0 // 64
        sub_store = store[b0 * STORE_BYTES_PER_BLOCK_GROUP * (inn // 128):]
        lt = None if to_levels is None else to_levels[li][b0:]
        items.append((sub_store, n, inn, lv[b0:], lt, x, y_local[off:off + batch * n]))
        placed.append((li, off, n))
        off += batch * n
    assert off == batch * total
    return items, placed


def gather_rows(y_local, counts, group=None, out=None):
    """All ranks' output rows, in rank order: each rank's buffer [rows_r] (or [batch][rows_r])
    is padded to the largest count, one all-gather, padding dropped. Returns a list of the ranks'
    buffers.

    A buffer already as wide as the largest count (rows at the front) is sent as it is, with no
    copy; ``out`` (len(counts) x that many elements) is then filled in place, so the call can sit
    in a captured CUDA graph with no allocation."""
    import torch
    import torch.distributed as dist
    width = max(counts)
    lead = y_local.shape[:-1]
    if y_local.shape[-1] == width and y_local.is_contiguous():
        pad = y_local
    else:
        pad = torch.zeros((*lead, width), dtype=y_local.dtype, device=y_local.device)
        pad[..., :y_local.shape[-1]] = y_local
    if out is None:
        out = torch.empty(len(counts) * pad.numel(), dtype=y_local.dtype, device=y_local.device)
    dist.all_gather_into_tensor(out, pad.view(-1), group=group)
    out = out.view(len(counts), *lead, width)
    return [out[r][..., :c] for r, c in enumerate(counts)]


def gather_partials(partial_local, nranks: int, group=None, out=None):
    """The ranks' gate partials ([batch] records of 32 bytes, as a uint8 tensor of batch * 32
    bytes) gathered into one [nranks][batch] buffer, rank order, for fl_logit_gate_merge
    (``out``, nranks * batch * 32 bytes, is filled in place when given)."""
    import torch
    import torch.distributed as dist
    if out is None:
        out = torch.empty(nranks * partial_local.numel(), dtype=partial_local.dtype, device=partial_local.device)
    dist.all_gather_into_tensor(out, partial_local.contiguous().view(-1), group=group)
    return out.view(nranks, partial_local.numel())
