"""Host logic of the context-parallel forward (keys sharded across ranks).

The shard planner must cover every key exactly once in rank order and report
how many keys follow each shard; the exchange must deliver every rank's
partial in rank order.  Two gloo ranks run here on the CPU: each computes the
partial of its shard with the CPU oracle (non-causal and unbiased, where a
shard's partial is plain attention over its keys), the ranks all-gather the
partials through ``gather_partials``, and the LSE merge of what arrives must
equal the oracle on all keys.  The GPU path (partials from the kernel, merge
in the combine kernel, positions through k_after) is checked against the
oracle in the GPU parity tests.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from exact_attention_forward_flash_b200.context_parallel import (  # noqa: E402
    shard_bounds, shard_seqused)


@pytest.mark.parametrize("k_len", [0, 1, 127, 128, 129, 1000, 4096, 131072])
@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_shards_cover_the_keys_once_in_rank_order(k_len, world):
    pos = 0
    sizes = []
    for r in range(world):
        start, length, after = shard_bounds(k_len, world, r)
        assert start == pos and length >= 0
        assert after == k_len - start - length
        if start + length < k_len:
            assert length % 128 == 0  # only the last non-empty shard is ragged
        pos += length
        sizes.append(-(-length // 128))
    assert pos == k_len
    assert max(sizes) - min(sizes) <= 1


def test_shard_bounds_rejects_bad_arguments():
    with pytest.raises(ValueError):
        shard_bounds(10, 2, 2)
    with pytest.raises(ValueError):
        shard_bounds(-1, 2, 0)


def test_shard_seqused_splits_valid_keys():
    # padded length 1000 in shards [0,384) [384,768) [768,1000); valid 0, 500, 1000
    used = [0, 500, 1000]
    parts = [shard_seqused(used, s, n) for s, n in ((0, 384), (384, 384), (768, 232))]
    assert parts[0] == ([0, 384, 384], [0, 116, 616])
    assert parts[1] == ([0, 116, 384], [0, 0, 232])
    assert parts[2] == ([0, 0, 232], [0, 0, 0])
    for b in range(3):
        assert sum(p[0][b] for p in parts) == used[b]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    g = torch.Generator().manual_seed(7)
    B, Sq, Sk, Hq, Hkv, D = 2, 3, 300, 4, 2, 8
    q = torch.randn(B, Sq, Hq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Sk, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Sk, Hkv, D, generator=g, dtype=torch.float64)
    return q, k, v


def _packed(o, lse):
    """oracle (O [B,Sq,Hq,D], LSE [B,Hq,Sq]) -> packed (token, head) rows"""
    B, Sq, Hq, D = o.shape
    return (torch.from_numpy(np.ascontiguousarray(o)).reshape(B * Sq * Hq, D),
            torch.from_numpy(np.ascontiguousarray(lse.transpose(0, 2, 1))).reshape(-1))


def _rank_main(rank, world, port, out_q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from exact_attention_forward_flash_b200.context_parallel import gather_partials
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v = _problem()
        start, length, _ = shard_bounds(k.shape[1], world, rank, align=64)
        o, lse = oracle.attention(q.numpy(), k[:, start:start + length].numpy(),
                                  v[:, start:start + length].numpy(), softmax_scale=0.3)
        o_p, l_p = _packed(o, lse)
        o_all, l_all = gather_partials(o_p, l_p)
        out_q.put((rank, o_all.numpy(), l_all.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_partials_that_merge_to_the_full_result():
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q_)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q_.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v = _problem()
    ref_o, ref_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), softmax_scale=0.3)
    ref_o, ref_l = _packed(ref_o, ref_l)
    for _, o_all, l_all in res:
        assert o_all.shape[0] == world
        # LSE merge of the gathered partials (rank order must not matter)
        m = l_all.max(axis=0)
        w = np.exp(l_all - m)
        lse = m + np.log(w.sum(axis=0))
        o = (np.exp(l_all - lse)[:, :, None] * o_all).sum(axis=0)
        np.testing.assert_allclose(lse, ref_l.numpy(), rtol=0, atol=1e-12)
        np.testing.assert_allclose(o, ref_o.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_array_equal(res[0][1], res[1][1])


# ---------------------------------------------------------------------------
# fa_fwd_context_parallel itself over two gloo ranks, with its two device
# steps (the shard partial, the merge) done by the oracle on CPU tensors
# ---------------------------------------------------------------------------
def _cp_problem():
    g = torch.Generator().manual_seed(11)
    B, Sq, Sk, Hq, Hkv, D, R = 2, 5, 300, 4, 2, 8, 128
    q = torch.randn(B, Sq, Hq, D, generator=g, dtype=torch.float64)
    k = torch.randn(B, Sk, Hkv, D, generator=g, dtype=torch.float64)
    v = torch.randn(B, Sk, Hkv, D, generator=g, dtype=torch.float64)
    rb = torch.randn(B, Sq, Hq, R, generator=g, dtype=torch.float64)
    return q, k, v, rb


def _oracle_shard_partial(q, k, v, *, k_after=None, causal=False, softmax_scale=None,
                          seqused_k=None, rel_bias=None, window=None, softcap=0.0,
                          num_splits=0):
    """Stand-in for the kernel's shard partial: the oracle over a sequence
    made of the shard's keys followed by k_after unused keys, restricted to
    the shard (bottom-right alignment needs only the keys after the shard)."""
    import oracle
    after = int(k_after[0])
    assert all(int(a) == after for a in k_after)
    B, Sk, Hkv, D = k.shape
    pad = torch.zeros(B, after, Hkv, D, dtype=k.dtype)
    o, lse = oracle.attention(q.numpy(), torch.cat([k, pad], 1).numpy(),
                              torch.cat([v, pad], 1).numpy(), causal=causal,
                              softmax_scale=softmax_scale, rel_bias=rel_bias.numpy(),
                              kv_range=(0, Sk))
    return _packed(o, lse)


def _oracle_combine(o_all, l_all, B, Sq, Hq, *, dtype=None, out=None, lse=None):
    """Stand-in for the merge kernel: the oracle's LSE merge."""
    import oracle
    o, l = oracle.lse_combine(o_all.numpy(), l_all.numpy())
    D = o.shape[1]
    return (torch.from_numpy(o).reshape(B, Sq, Hq, D),
            torch.from_numpy(l).reshape(B, Sq, Hq).permute(0, 2, 1).contiguous())


def _cp_rank_main(rank, world, port, out_q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from exact_attention_forward_flash_b200 import context_parallel as cp
    cp.fa_fwd_shard_partial = _oracle_shard_partial
    cp.fa_combine_partials = _oracle_combine
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, rb = _cp_problem()
        start, length, after = cp.shard_bounds(k.shape[1], world, rank)
        k_after = torch.full((q.shape[0],), after, dtype=torch.int32)
        o, lse = cp.fa_fwd_context_parallel(q, k[:, start:start + length].contiguous(),
                                            v[:, start:start + length].contiguous(),
                                            k_after=k_after, causal=True, softmax_scale=0.3,
                                            rel_bias=rb)
        out_q.put((rank, o.numpy(), lse.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_the_context_parallel_forward():
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q_ = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_rank_main, args=(r, world, port, q_)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q_.get(timeout=180) for _ in procs), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    q, k, v, rb = _cp_problem()
    ref_o, ref_l = oracle.attention(q.numpy(), k.numpy(), v.numpy(), causal=True,
                                    softmax_scale=0.3, rel_bias=rb.numpy())
    for _, o, lse in res:
        np.testing.assert_allclose(o, ref_o, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_l, rtol=0, atol=1e-12)


def test_single_process_context_parallel_needs_no_process_group():
    from exact_attention_forward_flash_b200 import context_parallel as cp
    o = torch.arange(6.0).reshape(3, 2)
    l = torch.zeros(3)
    o_all, l_all = cp.gather_partials(o, l)
    assert o_all.shape == (1, 3, 2) and torch.equal(o_all[0], o) and l_all.shape == (1, 3)


# ---------------------------------------------------------------------------
# property checks of the planner over random sizes
# ---------------------------------------------------------------------------
from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=300, deadline=None)
@given(k_len=st.integers(0, 1 << 20), world=st.integers(1, 64),
       align=st.sampled_from([1, 8, 64, 128, 256]))
def test_shard_bounds_properties(k_len, world, align):
    shards = [shard_bounds(k_len, world, r, align=align) for r in range(world)]
    pos = 0
    for start, length, after in shards:
        assert start == pos and length >= 0 and after == k_len - start - length
        pos += length
    assert pos == k_len
    blocks = [-(-n // align) for _, n, _ in shards]
    assert max(blocks) - min(blocks) <= 1
    # only the last non-empty shard may hold a partial block
    nonempty = [n for _, n, _ in shards if n]
    assert all(n % align == 0 for n in nonempty[:-1])


@settings(max_examples=300, deadline=None)
@given(data=st.data())
def test_shard_seqused_properties(data):
    world = data.draw(st.integers(1, 9))
    padded = data.draw(st.integers(0, 5000))
    used = data.draw(st.lists(st.integers(0, padded), min_size=1, max_size=6))
    total_used = [0] * len(used)
    for r in range(world):
        start, length, _ = shard_bounds(padded, world, r)
        loc, after = shard_seqused(used, start, length)
        for b, n in enumerate(used):
            assert 0 <= loc[b] <= length and after[b] >= 0
            # valid keys before, in and after the shard add up to all of them
            before = min(max(n, 0), start)
            assert before + loc[b] + after[b] == n
            total_used[b] += loc[b]
    assert total_used == used
