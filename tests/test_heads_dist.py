"""Head parallelism (quantized_attention_05_b200.heads) on CPU ranks (gloo,
world size 2, 3 and 5, with an uneven split and a rank without heads), with
full tensors on every rank and with each rank holding only its own slice.

Every KV-head group is a problem of its own, so:
* the gathered result equals, bit for bit, the per-slice results of the same
  attention function put side by side (this pins the split, the padding,
  the collective and the reassembly);
* and it equals the oracle's single call over all heads up to the oracle's
  own fp64 summation order, which depends on the array shapes and can move
  an fp32 rounding by one unit (2^-24 relative).
The per-slice attention is the oracle's here; the split, the padding and the
collective are the product code's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W
from quantized_attention_05_b200.heads import kv_head_range

WORK = W.TINY.scaled(B=2, Hq=8, Hkv=4, N=200, D=64, seed=91)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _oracle_attn(q, k, v, causal, sm_scale):
    import oracle as O
    r = O.attention_i8f8(O.quantize_qkv_i8f8(q.contiguous(), k.contiguous(), v.contiguous()),
                         causal=causal, sm_scale=sm_scale)
    return torch.from_numpy(r["out_f64"]), torch.from_numpy(r["lse"])


def _worker(rank, world, port, causal, q_out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from quantized_attention_05_b200.heads import head_parallel_attention, shard_heads
        q, k, v = (t.double() for t in W.make_qkv(WORK))     # bf16 values, fp64 outputs
        out, lse = head_parallel_attention(q, k, v, causal=causal, attn=_oracle_attn)
        part, plse, (h0, h1) = head_parallel_attention(q, k, v, causal=causal, gather=False,
                                                       attn=_oracle_attn)
        # sliced inputs: this rank holds only its own heads (copies, so no
        # view of the full tensors reaches the call)
        qs, ks, vs = (t.clone() for t in shard_heads(q, k, v, rank, world))
        sout, slse = head_parallel_attention(qs, ks, vs, causal=causal, attn=_oracle_attn,
                                             heads=(WORK.Hq, WORK.Hkv))
        q_out.put((rank, out.numpy(), lse.numpy(), part.numpy(), plse.numpy(), h0, h1,
                   sout.numpy(), slse.numpy(), tuple(qs.shape), tuple(ks.shape)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_kv_head_ranges_cover_every_head_once():
    for Hkv in (1, 4, 7, 8):
        for world in (1, 2, 3, 5, 8):
            ranges = [kv_head_range(Hkv, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == Hkv
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [g1 - g0 for g0, g1 in ranges]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)


@pytest.mark.parametrize("world,causal", [(2, False), (3, True), (5, False)])
def test_gathered_heads_equal_one_call_over_all_heads(world, causal):
    ctx = mp.get_context("spawn")
    qo = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, causal, qo)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = qo.get(timeout=300)
        res[item[0]] = item[1:]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    import oracle as O
    q, k, v = (t.double() for t in W.make_qkv(WORK))
    G = WORK.Hq // WORK.Hkv
    side_o = np.zeros((WORK.B, WORK.Hq, WORK.N, WORK.D))
    side_l = np.zeros((WORK.B, WORK.Hq, WORK.N))
    for r in range(world):
        g0, g1 = kv_head_range(WORK.Hkv, r, world)
        if g1 > g0:
            o, l = _oracle_attn(q[:, g0 * G:g1 * G], k[:, g0:g1], v[:, g0:g1], causal, None)
            side_o[:, g0 * G:g1 * G], side_l[:, g0 * G:g1 * G] = o.numpy(), l.numpy()
    full = O.attention_i8f8(O.quantize_qkv_i8f8(q, k, v), causal=causal)
    for r in range(world):
        out, lse, part, plse, h0, h1, sout, slse, qshape, kshape = res[r]
        np.testing.assert_array_equal(sout, side_o)
        np.testing.assert_array_equal(slse, side_l)
        g0, g1 = kv_head_range(WORK.Hkv, r, world)
        assert qshape[1] == (g1 - g0) * G and kshape[1] == g1 - g0
        np.testing.assert_array_equal(out, side_o)
        np.testing.assert_array_equal(lse, side_l)
        np.testing.assert_allclose(out, full["out_f64"], rtol=2.0 ** -22, atol=1e-12)
        np.testing.assert_allclose(lse, full["lse"], rtol=2.0 ** -22, atol=1e-12)
        g0, g1 = kv_head_range(WORK.Hkv, r, world)
        assert (h0, h1) == (g0 * G, g1 * G)
        np.testing.assert_array_equal(part, side_o[:, h0:h1])
        np.testing.assert_array_equal(plse, side_l[:, h0:h1])


def test_sliced_call_rejects_a_wrong_slice():
    """With heads=(Hq, Hkv) every rank must pass exactly its own slice."""
    import quantized_attention_05_b200.heads as Hm
    orig = (Hm.dist.get_world_size, Hm.dist.get_rank)
    Hm.dist.get_world_size, Hm.dist.get_rank = (lambda g=None: 2), (lambda g=None: 1)
    try:
        q, k, v = W.make_qkv(WORK)
        with pytest.raises(ValueError, match="expected the slices"):
            Hm.head_parallel_attention(q, k, v, heads=(WORK.Hq, WORK.Hkv), attn=lambda *a: None)
    finally:
        Hm.dist.get_world_size, Hm.dist.get_rank = orig
