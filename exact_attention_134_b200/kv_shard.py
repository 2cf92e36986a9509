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

The exchange is one all-gather: each rank's O and LSE are written into one
packed buffer (O, then LSE, padded to a multiple of 4 floats), so
B*Hq*Nq*(d+1) fp32 values per rank cross the interconnect in a single
collective, and the merge reads the gathered parts in place.
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

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if n_keys < world:
        raise ValueError("every rank must hold at least one key")
    lo, hi = shard_bounds(n_keys, world, rank)
    if k_shard.shape[2] != hi - lo or v_shard.shape != k_shard.shape:
        raise ValueError(f"rank {rank} must hold keys [{lo}, {hi}) of {n_keys}")
    B, Hq, Nq, d = q.shape
    rows = B * Hq * Nq
    stride = (rows * d + rows + 3) // 4 * 4  # the library's packed layout (partial_packed_floats)
    if partial_fn is None:  # the library's fp32 partial, written straight into the packed buffer
        from . import attn_fwd_partial
        buf = torch.empty(stride, dtype=torch.float32, device=q.device)
        attn_fwd_partial(q, k_shard, v_shard, causal=causal, scale=scale, kv_tail=n_keys - hi,
                         out=buf[:rows * d].view(B, Hq, Nq, d), lse=buf[rows * d:rows * d + rows].view(B, Hq, Nq))
    else:  # another partial (same packing, in its own dtype)
        o_p, lse_p = partial_fn(q, k_shard, v_shard, causal=causal, scale=scale, kv_tail=n_keys - hi)
        buf = torch.zeros(stride, dtype=o_p.dtype, device=o_p.device)
        buf[:rows * d].copy_(o_p.reshape(-1))
        buf[rows * d:rows * d + rows].copy_(lse_p.reshape(-1))
    parts = torch.empty((world, stride), dtype=buf.dtype, device=buf.device)
    dist.all_gather(list(parts.unbind(0)), buf, group=group)  # the one exchange
    if merge_fn is None:
        from . import merge_partials_packed
        return merge_partials_packed(parts, B, Hq, Nq, d)
    return merge_fn(parts[:, :rows * d].reshape(world, B, Hq, Nq, d),
                    parts[:, rows * d:rows * d + rows].reshape(world, B, Hq, Nq))
