"""Multi-device forms of the search and the decode step: one process per GPU
(torch.distributed; NCCL on GPUs), each holding one shard.

* Search over a database split across ranks ("TurboQuant explainer"
  (m.163.com), "向量搜索": inner-product search over very large sets of
  quantized vectors): every rank runs tq_search_topk on its shard, the per-rank
  top-k lists (ids, estimates) are all-gathered, and tq_search_merge takes the
  global top-k (shard offsets added, ties to the lower global id).  The top-k
  of the union of per-shard top-k lists is the global top-k.
* Decode attention over a sequence split across ranks: rank r holds tokens
  [t_r, t_{r+1}) of every sequence as a KV cache of its own; it runs
  tq_decode_attn_partial, the partials (m, l, o_rot) are all-gathered, and
  tq_decode_attn_merge applies the log-sum-exp merge and the inverse rotation.

The only exchange is one all-gather of small tensors (n_q x k pairs; batch x
heads x (d_pad + 2) floats).  The per-rank compute and the merge are passed in
as functions; the defaults call the library.  The orchestration is plain
tensor plumbing and runs over gloo on CPU tensors as well.
"""
import torch
import torch.distributed as dist

from . import tq_decode_attn_merge, tq_decode_attn_partial, tq_search_merge, tq_search_topk


def shard_bounds(n, world, rank):
    """[lo, hi) of shard `rank` when n items are split as evenly as possible over `world` ranks
    (the first n % world ranks take one more)."""
    base, rem = divmod(int(n), int(world))
    lo = rank * base + min(rank, rem)
    return lo, lo + base + (1 if rank < rem else 0)


def local_seq_lens(seq_lens, lo, hi):
    """Per-sequence token counts inside the shard [lo, hi) of every sequence."""
    return (seq_lens.to(torch.int64) - lo).clamp(min=0, max=hi - lo).to(seq_lens.dtype)


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


def all_gather_stacked(t, group=None):
    """[world, *t.shape]: t from every rank, in rank order."""
    world, _ = _world(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def sharded_search_topk(local_topk, merge, n_db, group=None):
    """Global top-k of a database split over the ranks with shard_bounds(n_db, world, rank).

    local_topk() -> (ids int32 [n_q, k] shard-local, scores fp32 [n_q, k]) on this rank's shard;
    merge(ids [world, n_q, k], scores [world, n_q, k], offsets list[world]) -> (ids, scores)."""
    world, _ = _world(group)
    ids, scores = local_topk()
    offsets = [shard_bounds(n_db, world, r)[0] for r in range(world)]
    return merge(all_gather_stacked(ids, group), all_gather_stacked(scores, group), offsets)


def sequence_split_decode(local_partial, merge, group=None):
    """Decode attention over sequences split across ranks by token ranges.

    local_partial() -> partial [batch, n_q_heads, P] of this rank's tokens;
    merge(partials [world, batch, n_q_heads, P]) -> out [batch, n_q_heads, d]."""
    return merge(all_gather_stacked(local_partial(), group))


# ---- the library's per-rank compute and merges ------------------------------
def library_search(p, q, codes, norms, rnorms, n_local, k, workspace):
    """(local_topk, merge) for sharded_search_topk that run the library's kernels."""
    def local_topk():
        ids = torch.empty((q.shape[0], k), dtype=torch.int32, device=q.device)
        scores = torch.empty((q.shape[0], k), dtype=torch.float32, device=q.device)
        tq_search_topk(p, q, codes, norms, rnorms, n_local, k, ids, scores, workspace)
        return ids, scores

    def merge(ids, scores, offsets):
        out_i = torch.empty(ids.shape[1:], dtype=torch.int32, device=ids.device)
        out_s = torch.empty(ids.shape[1:], dtype=torch.float32, device=ids.device)
        tq_search_merge(ids, scores, offsets, k, out_i, out_s)
        return out_i, out_s

    return local_topk, merge


def library_decode(kp, vp, q, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens_local, max_tokens_local,
                   workspace, scale=0.0):
    """(local_partial, merge) for sequence_split_decode that run the library's kernels."""
    def local_partial():
        part = torch.empty((q.shape[0], q.shape[1], kp.d_pad + 2), dtype=torch.float32, device=q.device)
        tq_decode_attn_partial(kp, vp, q, n_kv_heads, kcodes, knorms, krnorms, vcodes, vnorms, seq_lens_local,
                               max_tokens_local, part, workspace, scale=scale)
        return part

    def merge(parts):
        out = torch.empty((q.shape[0], q.shape[1], kp.d), dtype=torch.float32, device=q.device)
        tq_decode_attn_merge(vp, parts, out)
        return out

    return local_partial, merge
