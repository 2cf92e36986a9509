"""Key-sharded attention forward over several GPUs (one process per GPU).

For a context too long for one GPU's share of the work, each rank holds one
contiguous range of the keys and values and all query rows. Each computes
its range's partial result with ``attn_fwd_partial`` (normalised O_r in fp32
and LSE_r; when the range's own grid would leave SMs idle, its keys are split
over more CTAs and merged on the device first), the ranks all-gather the
partials (NCCL over NVLink), and every rank merges them with
``merge_partials``:

    LSE = ln sum_r exp(LSE_r),   O = sum_r exp(LSE_r - LSE) O_r,

the online-softmax update of "FlashAttention (TR)", section "Çevrimiçi
Softmax Hesaplama", applied to whole key ranges — exact in real arithmetic.
The causal mask stays the full sequence's (bottom-right aligned): a rank
passes the number of keys held by the ranks after it as ``kv_tail``.

The exchange is two all-gathers (O and LSE) of B*Hq*Nq*(d+1) fp32 values
per rank in all.
"""
from __future__ import annotations


def shard_bounds(n_keys: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous key range [lo, hi) of `rank`: near-equal shares in rank
    order, the first n_keys % world ranks holding one key more."""
    if world <= 0 or not 0 <= rank < world or n_keys < 0:
        raise ValueError("need world > 0, 0 <= rank < world, n_keys >= 0")
    base, extra = divmod(n_keys, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def attention_kv_sharded(q, k_shard, v_shard, n_keys: int, causal: bool = False,
                         scale: float | None = None, group=None, partial_fn=None, merge_fn=None):
    """Attention of q over the full key sequence whose range
    ``shard_bounds(n_keys, world, rank)`` this rank holds in k_shard, v_shard.

    q: [B, Hq, Nq, d] (every rank the same rows); k_shard, v_shard:
    [B, Hkv, hi - lo, d]. Returns (o [B, Hq, Nq, d] bf16, lse [B, Hq, Nq]) on
    every rank. ``partial_fn`` / ``merge_fn`` default to the library's
    attn_fwd_partial / merge_partials.
    """
    import torch
    import torch.distributed as dist

    from . import attn_fwd_partial, merge_partials
    partial_fn = partial_fn or attn_fwd_partial
    merge_fn = merge_fn or merge_partials
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if n_keys < world:
        raise ValueError("every rank must hold at least one key")
    lo, hi = shard_bounds(n_keys, world, rank)
    if k_shard.shape[2] != hi - lo or v_shard.shape != k_shard.shape:
        raise ValueError(f"rank {rank} must hold keys [{lo}, {hi}) of {n_keys}")
    o_r, lse_r = partial_fn(q, k_shard, v_shard, causal=causal, scale=scale, kv_tail=n_keys - hi)
    o_all = torch.empty((world, *o_r.shape), dtype=o_r.dtype, device=o_r.device)
    lse_all = torch.empty((world, *lse_r.shape), dtype=lse_r.dtype, device=lse_r.device)
    dist.all_gather(list(o_all.unbind(0)), o_r.contiguous(), group=group)
    dist.all_gather(list(lse_all.unbind(0)), lse_r.contiguous(), group=group)
    return merge_fn(o_all, lse_all)
