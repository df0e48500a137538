"""The cross-GPU shard level of the tree on CPU, with gloo ranks (world sizes
2 and 4).

Each rank computes the root of its own subtree (the CPU oracle stands in for
the rank's GPU kernels), the ranks exchange their results with
tp.gather_shards (the all-gather the multi-GPU path uses), and every rank
applies the tree's shard level.  The result must be bitwise the oracle's
one-device (T = 1) result: row-parallel GEMM over K shards, the non-invariant
baseline's left-to-right shard sum, and the vocabulary-parallel logprob with
the shard layout of vocab_shard.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    import synth
    from invariant_tree_ordered_b200 import tp, vocab_shard

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T, t = world, rank
        # ---- row-parallel GEMM: K = 8 leaves of 32, rank t holds K shard t
        M, N, K, leaf = 5, 24, 256, 32
        a = synth.normal_bf16(600, (M, K))
        b = synth.normal_bf16(601, (K, N), std=0.1)
        ks = K // T
        a_t = np.ascontiguousarray(a[:, t * ks:(t + 1) * ks])
        b_t = np.ascontiguousarray(b[t * ks:(t + 1) * ks])
        q_t = oracle.gemm_tree(a_t, b_t, b_nk=False, T=1, leaf=leaf)
        parts = tp.gather_shards(torch.from_numpy(q_t), None).numpy()
        c = np.empty((M, N), dtype=np.float32)
        for i in range(M):
            for n in range(N):
                c[i, n] = oracle.tree_sum(parts[:, i, n])
        gemm_ok = np.array_equal(_bits(c), _bits(oracle.gemm_tree(a, b, b_nk=False, T=1, leaf=leaf)))
        # ---- the baseline: one chain per shard, summed left to right
        n_t = oracle.gemm_noninv(a_t, b_t, b_nk=False, T=1)
        nparts = tp.gather_shards(torch.from_numpy(n_t), None).numpy()
        acc = nparts[0].copy()
        for j in range(1, T):
            acc = (acc + nparts[j]).astype(np.float32)
        noninv_ok = np.array_equal(_bits(acc), _bits(oracle.gemm_noninv(a, b, b_nk=False, T=T)))
        # ---- vocabulary-parallel logprob
        V, H, lf = 1500, 64, 32
        hid = synth.normal_bf16(610, (6, H))
        w = synth.normal_bf16(611, (V, H), std=0.5)
        tg = synth.uniform_int32(612, 6, 0, V)
        v0, vs, lvs = vocab_shard(V, T, t)
        w_t = np.ascontiguousarray(w[v0:v0 + vs])
        _, m, s = oracle.logprob(hid, w_t, np.zeros(6, dtype=np.int32), T=1, leaf=lf, vpad=lvs * 64, stats=True)
        z = oracle.gemm_tree(hid, w_t, b_nk=True, T=1, leaf=lf)
        part = np.zeros((6, 4), dtype=np.float32)
        part[:, 0], part[:, 1] = m, s
        for i in range(6):
            if v0 <= tg[i] < v0 + vs:
                part[i, 2], part[i, 3] = z[i, tg[i] - v0], 1.0
        gathered = tp.gather_shards(torch.from_numpy(part), None).numpy()
        out = np.empty(6, dtype=np.float32)
        for i in range(6):
            mm, ss = oracle.tree_ms(gathered[:, i, 0], gathered[:, i, 1])
            owner = [j for j in range(T) if gathered[j, i, 3] == 1.0]
            assert len(owner) == 1
            zt = np.float32(gathered[owner[0], i, 2])
            out[i] = np.float32(np.float32(zt - np.float32(mm)) - np.float32(oracle.log(float(ss))))
        lp_ok = np.array_equal(_bits(out), _bits(oracle.logprob(hid, w, tg, T=1, leaf=lf)))
        q.put((rank, bool(gemm_ok), bool(noninv_ok), bool(lp_ok)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_shard_exchange_reproduces_one_device_bits(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert [r[0] for r in res] == list(range(world))
    for rank, gemm_ok, noninv_ok, lp_ok in res:
        assert gemm_ok, f"rank {rank}: row-parallel GEMM differs from T = 1"
        assert noninv_ok, f"rank {rank}: baseline differs from its T-shard definition"
        assert lp_ok, f"rank {rank}: vocabulary-parallel logprob differs from T = 1"


def test_vocab_shard_layout():
    sys.path.insert(0, ROOT)
    from invariant_tree_ordered_b200 import vocab_shard
    V = 151936
    for T in (1, 2, 4, 8):
        shards = [vocab_shard(V, T, t) for t in range(T)]
        assert sum(vs for _, vs, _ in shards) == V
        assert all(lvs * T * 64 == 152064 for _, _, lvs in shards)  # ceil(V / 512) * 512 padded columns
        assert [v0 for v0, _, _ in shards] == [t * 152064 // T for t in range(T)]
    assert vocab_shard(100, 8, 3) == (192, 0, 1)  # a shard of padding only
    with pytest.raises(ValueError):
        vocab_shard(V, 3, 0)
