"""Context-parallel decode of long sequences across GPUs: the plumbing around
kv4_decode_partials and kv4_merge_partials.

TTKV promo (arXiv 2604.19769), opening section: contexts of about a million
tokens need several GPUs. KV4-RL review, sec. 3: the softmax partials
(max, sum, output) of disjoint position sets merge exactly. So each rank
holds a contiguous range of every sequence's INT4 pages (and one rank the
INT8 side cache), attends it with kv4_decode_partials, the ranks all-gather
their partials -- (D + 4) * 4 bytes per (sequence, query head), whatever the
context length -- and every rank merges them with kv4_merge_partials.

The exchange is a torch.distributed all_gather into a stacked buffer (NCCL for
device tensors, gloo for host tensors): no other collective is needed, and no
rank reads another rank's memory.
"""
import numpy as np
import torch

from . import kv4_decode_partials, kv4_merge_partials

PAGE_TOKENS = 16


def int4_pages(lens, sink=16, recent=128):
    """Logical page range [first, end) of the INT4 region of each sequence."""
    lens = np.asarray(lens, np.int64)
    first = np.full(lens.shape, sink // PAGE_TOKENS, np.int64)
    hi = lens - recent
    end = np.where(hi > sink, (hi + PAGE_TOKENS - 1) // PAGE_TOKENS, first)
    return first, end


def shard_pages(lens, n_shards, sink=16, recent=128):
    """Split every sequence's INT4 pages into n_shards contiguous ranges of
    near-equal length. Returns (page_begin, page_end), int32 [n_shards][B]:
    shard r attends pages [page_begin[r][b], page_end[r][b]) of sequence b."""
    first, end = int4_pages(lens, sink, recent)
    n = end - first
    r = np.arange(n_shards + 1, dtype=np.int64)[:, None]
    bounds = first[None, :] + (r * n[None, :]) // n_shards
    return bounds[:-1].astype(np.int32), bounds[1:].astype(np.int32)


def gather_partials(partials, group=None):
    """All-gather of each rank's partials [B][Hq][D+4] into [world][B][Hq][D+4]
    (rank order), on the tensors' device."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(partials.shape), dtype=partials.dtype, device=partials.device)
    if partials.is_cuda:
        dist.all_gather_into_tensor(out, partials.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), partials.contiguous(), group=group)
    return out


def decode_context_parallel(cache, q, seq_lens, page_table, softmax_scale, page_begin, page_end, with_int8, out,
                            group=None, num_workers=0, stream=None):
    """One decode step of this rank's shard of every sequence, then the
    exchange of partials and the exact merge into `out` [B][Hq][D] on every
    rank. page_begin/page_end: this rank's device int32 [B] page ranges;
    with_int8: whether this rank attends the INT8 sink/recent positions (one
    rank per sequence does)."""
    B, Hq, D = q.shape
    partials = torch.empty((B, Hq, D + 4), dtype=torch.float32, device=q.device)
    kv4_decode_partials(cache.handle, q, seq_lens, page_table, softmax_scale, cache.workspace(B, Hq, num_workers),
                        partials, page_begin, page_end, with_int8, num_workers=num_workers, stream=stream)
    gathered = gather_partials(partials, group)
    kv4_merge_partials(gathered, out, stream=stream)
    return out
