"""Multi-GPU VC-Attention: Ulysses sequence parallelism and the CFG split.

Pages "NVIDIA Shows How TensorRT LLM VisualGen Speeds Up FLUX 3 Image Klein on
Blackwell" (the 8-GPU configurations) and "Accelerating FLUX 3 Image Generation
on NVIDIA Blackwell GPUs", section "Multi-GPU Scaling Performance": one
denoising step runs on several B200s with a classifier-free-guidance split
(`cfg_size`: the conditional and unconditional branches on different GPUs) and
Ulysses sequence parallelism (`ulysses_size`). Each GPU holds a slice of the
sequence for every head; an all-to-all turns that into the whole sequence for
a slice of the heads; attention runs per head; a second all-to-all returns the
output to the sequence slices.

Everything VC-Attention computes is per (b,h) (grouping, permutation, scales,
repair list, the fused kernel), so after the first exchange `vc_attn_fwd` runs
unchanged on the local heads. The CFG branches are independent batches: no
collective on the attention path. The exchange is
``torch.distributed.all_to_all_single`` (NCCL over NVLink / NVSwitch on the
GPUs, gloo on the CPU in the tests); the bf16 rows travel as int32 pairs, bit
for bit.
"""
from __future__ import annotations

from . import vcattn


def _dist():
    import torch.distributed as dist
    return dist


def make_groups(cfg_size: int, ulysses_size: int):
    """Split the default process group into `cfg_size` Ulysses groups of
    `ulysses_size` consecutive ranks: rank = cfg_rank * ulysses_size + sp_rank.

    Every rank must call this (group creation is collective). Returns
    (cfg_rank, sp_rank, sp_group)."""
    dist = _dist()
    world, rank = dist.get_world_size(), dist.get_rank()
    if cfg_size < 1 or ulysses_size < 1 or cfg_size * ulysses_size != world:
        raise ValueError(f"cfg_size x ulysses_size = {cfg_size} x {ulysses_size} != world size {world}")
    groups = [dist.new_group(list(range(c * ulysses_size, (c + 1) * ulysses_size))) for c in range(cfg_size)]
    cfg_rank, sp_rank = divmod(rank, ulysses_size)
    return cfg_rank, sp_rank, groups[cfg_rank]


def _a2a(send, group):
    """all_to_all_single over the leading dimension (one block per rank of the
    group), moving the bytes as int32 (both NCCL and gloo carry int32)."""
    import torch
    dist = _dist()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv.view(torch.int32), send.view(torch.int32), group=group)
    return recv


def seq_to_heads(x, group):
    """[B, H, n, d] (this rank's sequence slice, every head) ->
    [B, H/P, P*n, d] (the whole sequence, this rank's heads), P = group size.
    Sequence slice r comes from group rank r, so the slices concatenate in
    rank order; this rank gets heads [r*H/P, (r+1)*H/P) for its group rank r."""
    dist = _dist()
    P = dist.get_world_size(group)
    B, H, n, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    hp = H // P
    send = x.reshape(B, P, hp, n, d).permute(1, 0, 2, 3, 4).contiguous()  # block r: heads of rank r
    recv = _a2a(send, group)                                               # block r: sequence slice r
    return recv.permute(1, 2, 0, 3, 4).reshape(B, hp, P * n, d)


def heads_to_seq(y, group):
    """Inverse of seq_to_heads: [B, H/P, N, d] -> [B, H, N/P, d]."""
    dist = _dist()
    P = dist.get_world_size(group)
    B, hp, N, d = y.shape
    if N % P:
        raise ValueError(f"sequence of {N} does not split over {P} ranks")
    n = N // P
    send = y.reshape(B, hp, P, n, d).permute(2, 0, 1, 3, 4).contiguous()  # block r: sequence slice r
    recv = _a2a(send, group)                                              # block r: heads of rank r
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * hp, n, d)


def ulysses_attention(q, k, v, group, p=None, perm=None, ws=None, stream=None):
    """O = VC-Attention of the full sequence, from and to this rank's slice.

    q, k, v: bf16 [B, H, n, 128] CUDA tensors, this rank's sequence slice (the
    slices of the group's ranks, in group-rank order, make the sequence). perm
    (optional, int32 [B, H/P, N] on the device): the permutation of this rank's
    heads from an earlier step. Returns bf16 [B, H, n, 128]."""
    qh, kh, vh = (seq_to_heads(t, group) for t in (q, k, v))
    oh = vcattn.fwd(qh, kh, vh, perm=perm, p=p, ws=ws, stream=stream)
    return heads_to_seq(oh, group)
