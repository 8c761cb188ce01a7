"""The head-group partition of one attention call across ranks (bit_flashattention_b200/
partition.py), on CPU: the ranks' ranges cover every (batch, kv head) group exactly once,
and world-size-2 gloo ranks that each quantise and attend only their groups (with the
oracle) produce slices of O, m and l that assemble, bit for bit, into the single-process
result of the whole call.  No collective is on the data path; the test gathers the
slices only to compare them."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_flashattention_b200 import partition


@pytest.mark.parametrize("B,Hkv", [(1, 8), (4, 8), (1, 1), (3, 5), (2, 3)])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_ranges_cover_every_group_once(B, Hkv, world):
    seen = []
    sizes = []
    for r in range(world):
        u0, u1 = partition.group_range(B, Hkv, world, r)
        sizes.append(u1 - u0)
        for b, g0, g1 in partition.group_slices(u0, u1, Hkv):
            assert 0 <= b < B and 0 <= g0 < g1 <= Hkv
            seen += [b * Hkv + g for g in range(g0, g1)]
    assert sorted(seen) == list(range(B * Hkv))
    assert len(seen) == len(set(seen))
    assert max(sizes) - min(sizes) <= 1


def test_slices_stay_inside_one_batch_and_keep_order():
    # 3 batches x 5 kv heads over 4 ranks: rank 1 takes groups 4..7 = (b0, g4) and (b1, g0..g2)
    u0, u1 = partition.group_range(3, 5, 4, 1)
    assert (u0, u1) == (4, 8)
    assert partition.group_slices(u0, u1, 5) == [(0, 4, 5), (1, 0, 3)]
    with pytest.raises(ValueError):
        partition.group_range(1, 8, 2, 2)


def test_call_blocks_merge_whole_batches():
    sl = partition.group_slices(*partition.group_range(4, 8, 2, 1), 8)
    assert partition.call_blocks(sl, 8) == [(2, 4, 0, 8)]
    sl = partition.group_slices(*partition.group_range(3, 5, 4, 1), 5)
    assert partition.call_blocks(sl, 5) == [(0, 1, 4, 5), (1, 2, 0, 3)]
    sl = partition.group_slices(0, 15, 5)
    assert partition.call_blocks(sl, 5) == [(0, 3, 0, 5)]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _case():
    from bit_flashattention_b200 import configs, gen
    import oracle
    w = configs.scaled(configs.get("qwen3-8b-4k"), B=2, Hq=6, Hkv=3, N=256, bc=128)
    q, k, v = gen.inputs(w)
    qc, kc, _ = gen.inputs(w, calib=True)
    s, sinv = oracle.calibrate(qc, kc, w.alpha)
    return w, q, k, v, s, sinv


def _attend_groups(w, q, k, v, s, sinv, slices):
    """Oracle forward of the given (b, g0, g1) head slices: {(b, h): (o_bf16 [N, d], m, l)}."""
    import oracle
    G = w.Hq // w.Hkv
    out = {}
    for b, g0, g1 in slices:
        qs = np.ascontiguousarray(q[b:b + 1, g0 * G:g1 * G])
        ks = np.ascontiguousarray(k[b:b + 1, g0:g1])
        vs = np.ascontiguousarray(v[b:b + 1, g0:g1])
        qz = oracle.quantize_all(qs, ks, vs, np.ascontiguousarray(s[g0:g1]), np.ascontiguousarray(sinv[g0:g1]))
        r = oracle.attn_fwd(qz, w.causal, w.bc)
        n = w.N
        for hh in range((g1 - g0) * G):
            sl = slice(hh * n, (hh + 1) * n)
            out[(b, g0 * G + hh)] = (r["o_bf16"][sl], r["m"][sl], r["l"][sl])
    return out


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), OMP_NUM_THREADS="2")
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, qq, kk, vv, s, sinv = _case()
        u0, u1 = partition.group_range(w.B, w.Hkv, world, rank)
        mine = _attend_groups(w, qq, kk, vv, s, sinv, partition.group_slices(u0, u1, w.Hkv))
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)          # test only: assemble the slices
        if rank == 0:
            whole = {}
            for part in gathered:
                assert not (set(part) & set(whole))
                whole.update(part)
            q.put(whole)
    finally:
        dist.destroy_process_group()


def test_two_ranks_assemble_the_single_process_result():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    whole = q.get(timeout=300)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    w, qq, kk, vv, s, sinv = _case()
    import oracle
    qz = oracle.quantize_all(qq, kk, vv, s, sinv)
    ref = oracle.attn_fwd(qz, w.causal, w.bc)
    assert len(whole) == w.B * w.Hq
    for (b, h), (o, m, l) in whole.items():
        sl = slice((b * w.Hq + h) * w.N, (b * w.Hq + h + 1) * w.N)
        assert np.array_equal(o, ref["o_bf16"][sl]), (b, h)
        assert np.array_equal(m, ref["m"][sl]) and np.array_equal(l, ref["l"][sl]), (b, h)
