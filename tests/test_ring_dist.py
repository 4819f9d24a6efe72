"""The ring schedule of quantized_attention_05_b200.ring on CPU ranks (gloo,
world size 2 and 3): each rank's result over the whole sequence equals the
LSE merge (oracle) of the per-chunk quantised attention (oracle) over the
chunks it should see -- all of them, or those not after it for causal.
The per-chunk attention and the merge are the oracle's here; the schedule,
the exchanges and the causal skipping are the product code's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W

WORK = W.TINY.scaled(B=1, Hq=2, Hkv=1, N=768, D=64, seed=51)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_attn(q, k, v, causal, sm_scale):
    import oracle as O
    z = O.quantize_qkv_i8f8(q, k, v)
    r = O.attention_i8f8(z, causal=causal, sm_scale=sm_scale)
    return torch.from_numpy(r["out_f64"]), torch.from_numpy(r["lse"])


class _OracleMerge:
    def __init__(self, like):
        self.out, self.lse = None, None

    def add(self, out, lse):
        from oracle.merge import merge_step
        if self.out is None:
            self.out, self.lse = out.numpy(), lse.numpy()
        else:
            self.out, self.lse = merge_step(self.out, self.lse, out.numpy(), lse.numpy())

    def result(self, out):
        return torch.from_numpy(self.out), torch.from_numpy(self.lse)


def _worker(rank, world, port, causal, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantized_attention_05_b200.ring import ring_attention
        q, k, v = W.make_qkv(WORK)
        c = WORK.N // world
        sl = slice(rank * c, (rank + 1) * c)
        out, lse = ring_attention(q[:, :, sl], k[:, :, sl].contiguous(), v[:, :, sl].contiguous(),
                                  causal=causal, attn=_oracle_attn, merger=_OracleMerge)
        q_out.put((rank, out.numpy(), lse.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, False), (2, True), (3, True)])
def test_ring_schedule_matches_merged_chunks(world, causal):
    ctx = mp.get_context("spawn")
    qo = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, qo)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, o, l = qo.get(timeout=300)
        res[r] = (o, l)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    # single process: merge of the chunks each rank should see
    from oracle.merge import merge_partials
    q, k, v = W.make_qkv(WORK)
    c = WORK.N // world
    for r in range(world):
        sl = slice(r * c, (r + 1) * c)
        parts = []
        for j in range(world):
            if causal and j > r:
                continue
            kj = slice(j * c, (j + 1) * c)
            o, l = _oracle_attn(q[:, :, sl], k[:, :, kj], v[:, :, kj], causal and j == r, None)
            parts.append((o.numpy(), l.numpy()))
        ref_o, ref_l = merge_partials(parts)
        np.testing.assert_allclose(res[r][0], ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(res[r][1], ref_l, rtol=0, atol=1e-12)
