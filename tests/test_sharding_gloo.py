"""Multi-rank host logic on CPU ranks (gloo, world size 2): token shards,
global RoPE offsets, the Cache-DiT sums exchange, and a rank that dies
before the exchange.  The compute steps are the fp64 oracle here; on GPUs
the same functions call the CUDA library."""
import multiprocessing as mp
import os
import socket
import traceback

import numpy as np
import pytest
import torch

from dit_block_pass_b200.sharding import shard_range


def test_shard_range_covers_and_balances():
    for n in (0, 1, 7, 124992, 126192):
        for world in (1, 2, 3, 8):
            spans = [shard_range(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_sums(orc):
    from parity import bits

    def sums_fn(prev, cur):
        out = [orc.cachedit_sums(bits(prev[b]), bits(cur[b])) for b in range(prev.shape[0])]
        return torch.tensor(out, dtype=torch.float64)
    return sums_fn


def _oracle_decide(orc):
    def decide_fn(sums, threshold):
        R, B, _ = sums.shape
        rel, reuse = [], []
        for b in range(B):
            num = den = 0.0
            for r in range(R):           # rank order
                num += float(sums[r, b, 0])
                den += float(sums[r, b, 1])
            q, u = orc.cachedit_decide(num, den, threshold)
            rel.append(q)
            reuse.append(u)
        return torch.tensor(rel, dtype=torch.float64), torch.tensor(reuse, dtype=torch.uint8)
    return decide_fn


POLICY_SIGMAS = [0.02, 0.03, 0.1, 0.02, 0.03, 0.02, 0.02, 0.2, 0.01]


def _worker(rank, world, port, mode, q):
    try:
        import sys
        root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
        sys.path.insert(0, root)
        sys.path.insert(0, os.path.join(root, "tests"))
        import datetime

        import torch.distributed as dist

        import oracle
        from dit_block_pass_b200 import sharding
        from dit_block_pass_b200 import workloads as W
        os.environ["MASTER_ADDR"] = "127.0.0.1"
        os.environ["MASTER_PORT"] = str(port)
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=20))
        orc = oracle.default()
        wl = W.Workload("shard", B=2, T=3, Hg=5, Wg=7, D=256, H=2, hd=128, F=8,
                        pairs=(22, 21, 21), sigma_cache=(0.03, 0.1))
        B, N, D = wl.B, wl.N, wl.D
        a, b = sharding.shard_range(N, rank, world)
        if mode == "die":
            if rank == 1:
                os._exit(3)          # leaves between steps, before the exchange
            prev, cur = (t.view(B, N, D) for t in W.cache_pair(wl))
            try:
                sharding.cachedit_residual_diff_sharded(
                    prev[:, a:b], cur[:, a:b], 0.04, sums_fn=_oracle_sums(orc),
                    decide_fn=_oracle_decide(orc))
                q.put((rank, "no error"))
            except Exception as e:          # the survivor learns of it on the host
                q.put((rank, "error:" + type(e).__name__))
            return
        if mode == "policy":
            # a run of steps: each rank decides from the all-gathered sums
            # with the library's reuse rule (host code)
            from dit_block_pass_b200 import CachePolicy
            pol = CachePolicy(0.04, 0, 2)
            decisions, rels = [], []
            for t, sig in enumerate(POLICY_SIGMAS):
                wt = W.Workload("shard", B=2, T=3, Hg=5, Wg=7, D=256, H=2, hd=128, F=8,
                                pairs=(22, 21, 21), sigma_cache=(sig, sig / 2), seed=t)
                prev, cur = (x.view(B, N, D) for x in W.cache_pair(wt))
                rel, _ = sharding.cachedit_residual_diff_sharded(
                    prev[:, a:b].contiguous(), cur[:, a:b].contiguous(), 0.04,
                    sums_fn=_oracle_sums(orc), decide_fn=_oracle_decide(orc))
                r = float(rel.max())
                rels.append(r)
                decisions.append(pol.decide(r if t > 0 else None))
            q.put((rank, "policy", decisions, rels))
            dist.barrier()
            dist.destroy_process_group()
            return
        # Cache-DiT over shards == over the whole clip, identical on every rank
        prev, cur = (t.view(B, N, D) for t in W.cache_pair(wl))
        rel, reuse = sharding.cachedit_residual_diff_sharded(
            prev[:, a:b].contiguous(), cur[:, a:b].contiguous(), 0.04,
            sums_fn=_oracle_sums(orc), decide_fn=_oracle_decide(orc))
        from parity import bits
        ref_rel, ref_reuse = orc.cachedit_residual_diff(bits(prev), bits(cur), 0.04)
        # QK on a shard with the global offset == the same rows of the full clip
        qkv = W.token_rows(wl, W.S_QKV, 3 * D)
        wq, wk = W.norm_weights(wl)

        def op(q_, k_, w_q, w_k, heads, pairs, grid=None, pos_offset=0, theta=1e4, eps=1e-6):
            n = q_.shape[1]
            pos = orc.grid_positions(*grid, pos_offset, n)
            return orc.qk_rmsnorm_rope3d(bits(q_[0]), w_q.double().numpy(), heads, wl.hd, pos,
                                         pairs, theta, eps)

        shard_out = sharding.qk_rmsnorm_rope3d_shard(
            qkv[a:b, :D].reshape(1, b - a, D), None, wq, None, wl.H, wl.pairs,
            (wl.T, wl.Hg, wl.Wg), a, op=lambda *x, **k: q.put((rank, "qk", a, b, op(*x, **k))))
        del shard_out
        gathered = [torch.empty(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, rel)
        q.put((rank, "cache", rel.numpy(), reuse.numpy(), ref_rel, ref_reuse,
               torch.stack(gathered).numpy()))
        dist.barrier()
        dist.destroy_process_group()
    except Exception:
        q.put((rank, "exception", traceback.format_exc()))


def _run(world, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = []
    import queue
    # drain before joining: a child does not exit while its queued data is unread
    deadline = 120.0
    import time
    t0 = time.time()
    while time.time() - t0 < deadline:
        try:
            out.append(q.get(timeout=1.0))
        except queue.Empty:
            if not any(p.is_alive() for p in procs):
                break
    for p in procs:
        p.join(timeout=5)
        if p.is_alive():
            p.kill()
    return out


def test_two_rank_shards_match_the_whole_clip():
    import oracle
    orc = oracle.default()
    out = _run(2, "ok")
    errs = [o for o in out if o[1] == "exception"]
    assert not errs, errs[0][2]
    cache = [o for o in out if o[1] == "cache"]
    assert len(cache) == 2
    for _, _, rel, reuse, ref_rel, ref_reuse, allrel in cache:
        assert np.allclose(rel, ref_rel, rtol=1e-13, atol=0)
        assert np.array_equal(reuse, ref_reuse)
        assert np.array_equal(allrel[0], allrel[1])       # bit-identical on every rank
    # QK shards with global offsets reassemble the full-clip result
    from dit_block_pass_b200 import workloads as W
    from parity import bits
    wl = W.Workload("shard", B=2, T=3, Hg=5, Wg=7, D=256, H=2, hd=128, F=8, pairs=(22, 21, 21))
    qkv = W.token_rows(wl, W.S_QKV, 3 * wl.D)
    wq, _ = W.norm_weights(wl)
    full = orc.qk_rmsnorm_rope3d(bits(qkv[:wl.N, :wl.D]), wq.double().numpy(), wl.H, wl.hd,
                                 orc.grid_positions(wl.T, wl.Hg, wl.Wg, 0, wl.N), wl.pairs,
                                 wl.theta, wl.eps)
    parts = sorted((o[2], o[3], o[4]) for o in out if o[1] == "qk")
    assert [p[:2] for p in parts] == [(0, 53), (53, 105)]
    assert np.array_equal(np.concatenate([p[2] for p in parts]), full)


def test_a_rank_that_leaves_before_the_exchange_is_reported():
    out = _run(2, "die")
    survivors = [o for o in out if o[0] == 0]
    assert survivors, out
    assert survivors[0][1].startswith("error:"), survivors


def test_two_ranks_take_the_same_reuse_decisions():
    """Over a run of steps, both ranks decide from the all-gathered sums with
    the library's reuse rule, agree step by step, and match the oracle's rule
    applied to the whole clip's relative differences."""
    import oracle
    from dit_block_pass_b200 import workloads as W
    from parity import bits
    out = _run(2, "policy")
    errs = [o for o in out if o[1] == "exception"]
    assert not errs, errs[0][2]
    runs = [o for o in out if o[1] == "policy"]
    assert len(runs) == 2
    assert runs[0][2] == runs[1][2] and runs[0][3] == runs[1][3]
    orc = oracle.default()
    whole = []
    for t, sig in enumerate(POLICY_SIGMAS):
        wt = W.Workload("shard", B=2, T=3, Hg=5, Wg=7, D=256, H=2, hd=128, F=8,
                        pairs=(22, 21, 21), sigma_cache=(sig, sig / 2), seed=t)
        prev, cur = W.cache_pair(wt)
        rel, _ = orc.cachedit_residual_diff(bits(prev).reshape(2, wt.N, 256),
                                            bits(cur).reshape(2, wt.N, 256), 0.04)
        whole.append(float(rel.max()))
    assert np.allclose(runs[0][3], whole, rtol=1e-12, atol=0)
    expect = oracle.cache_policy(whole, 0.04, 0, 2)
    assert runs[0][2] == expect
    assert any(expect) and not all(expect[1:])
