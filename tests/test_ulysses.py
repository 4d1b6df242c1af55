"""Ulysses sequence parallelism and the CFG split (bit_attention_diffusion_b200.ulysses).

CPU: gloo ranks (spawned processes). Each rank holds its sequence slice of a
synthetic head set; the exchange gathers the whole sequence of its heads, the
oracle (standing in for the GPU kernel, which is per head too) computes
VC-Attention for them, and the second exchange returns the output slices. The
result must equal, bit for bit, the oracle run on the full tensors in one
process: the exchange moves bytes only, and every step of the method is per
(b,h). GPU: the same call through the CUDA kernel in a one-rank NCCL group.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, N, seed):
    from bit_attention_diffusion_b200 import synth
    return synth.make_inputs(synth.custom(B, H, N, seed=seed))


def _bf16_tensor(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def _bits(t):
    import torch
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _rank_main(rank, world, port, cfg_size, B, H, N, seed, out):
    import datetime
    import sys

    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import oracle
    from bit_attention_diffusion_b200 import ulysses

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        cfg_rank, sp_rank, group = ulysses.make_groups(cfg_size, world // cfg_size)
        P = world // cfg_size
        x = _inputs(B * cfg_size, H, N, seed)          # batch element c = CFG branch c
        n = N // P
        sl = slice(sp_rank * n, (sp_rank + 1) * n)
        mine = {c: _bf16_tensor(x[c][cfg_rank:cfg_rank + 1, :, sl]) for c in "qkv"}
        qh, kh, vh = (ulysses.seq_to_heads(mine[c], group) for c in "qkv")
        # the exchange: this rank's heads, the whole sequence, in order
        hp = H // P
        heads = range(sp_rank * hp, (sp_rank + 1) * hp)
        assert np.array_equal(_bits(qh)[0], x["q"][cfg_rank, sp_rank * hp:(sp_rank + 1) * hp])
        outs = []
        for j, h in enumerate(heads):
            r = oracle.vc_attention_head(_bits(qh)[0, j], _bits(kh)[0, j], _bits(vh)[0, j])
            outs.append(oracle.to_bf16_bits(r["out"]))
        oh = _bf16_tensor(np.stack(outs)[None])
        o = ulysses.heads_to_seq(oh, group)
        out[rank] = (cfg_rank, sp_rank, _bits(o))
        # round trip of the exchange alone
        back = ulysses.heads_to_seq(ulysses.seq_to_heads(mine["v"], group), group)
        assert np.array_equal(_bits(back), _bits(mine["v"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,cfg_size,H", [(2, 1, 4), (4, 2, 4), (4, 1, 8)])
def test_ulysses_exchange_equals_single_process_oracle(orc, world, cfg_size, H):
    B, N, seed = 1, 512, 4242
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, _free_port(), cfg_size, B, H, N, seed, out), nprocs=world,
                           start_method="spawn")
        res = dict(out)
    x = _inputs(B * cfg_size, H, N, seed)
    P = world // cfg_size
    n = N // P
    for c in range(cfg_size):
        full = np.stack([orc.to_bf16_bits(orc.vc_attention_head(x["q"][c, h], x["k"][c, h], x["v"][c, h])["out"])
                         for h in range(H)])
        for rank, (cfg_rank, sp_rank, o) in res.items():
            if cfg_rank != c:
                continue
            assert np.array_equal(o[0], full[:, sp_rank * n:(sp_rank + 1) * n]), (rank, c)


def _grid_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    from bit_attention_diffusion_b200 import ulysses
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        try:
            ulysses.make_groups(3, 2)
            bad = False
        except ValueError:
            bad = True
        cfg_rank, sp_rank, group = ulysses.make_groups(2, 2)
        out[rank] = (bad, cfg_rank, sp_rank, dist.get_world_size(group), dist.get_rank(group))
    finally:
        dist.destroy_process_group()


def test_cfg_by_ulysses_grid_of_four_ranks():
    """The pages' Base-model layout on 8 GPUs is cfg_size 2 x ulysses_size 4;
    here 2 x 2: ranks 0,1 take CFG branch 0 and 2,3 branch 1, each pair one
    Ulysses group; a grid that does not cover the world is rejected."""
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_grid_main, args=(4, _free_port(), out), nprocs=4, start_method="spawn")
        res = dict(out)
    assert res == {0: (True, 0, 0, 2, 0), 1: (True, 0, 1, 2, 1), 2: (True, 1, 0, 2, 0), 3: (True, 1, 1, 2, 1)}


@pytest.mark.gpu
def test_ulysses_attention_one_rank_matches_the_oracle():
    """One NCCL rank on the GPU (every run here has one GPU, so both exchanges
    are all_to_all_single over a group of one): the output of the kernel behind
    the exchange, row by row against the oracle run on each head (relative L2
    <= 1e-3 per head, bf16 against bf16)."""
    import datetime

    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from bit_attention_diffusion_b200 import build_lib, synth, ulysses
    build_lib.build()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        B, H, N = 2, 3, 700
        x = synth.make_inputs(synth.custom(B, H, N, seed=77))
        q, k, v = (_bf16_tensor(x[c]).cuda() for c in "qkv")
        _, _, group = ulysses.make_groups(1, 1)
        o = ulysses.ulysses_attention(q, k, v, group)
        torch.cuda.synchronize()
        got_bits = o.view(torch.int16).cpu().numpy().view(np.uint16)
        val = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        for b in range(B):
            for h in range(H):
                r = oracle.vc_attention_head(x["q"][b, h], x["k"][b, h], x["v"][b, h])
                ref = val(oracle.to_bf16_bits(r["out"]))
                got = val(got_bits[b, h])
                assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-3, (b, h)
    finally:
        dist.destroy_process_group()
