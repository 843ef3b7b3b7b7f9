"""GPU parity of the context-parallel forward against the CPU fp64 oracle.

The key shards of one problem are processed one after another on cuda:0, as
the ranks of a context-parallel job would each process theirs: every shard's
fp32 partial comes from the kernel with the shard's k_after, the stacked
partials are merged by the combine kernel, and the result must equal the
oracle over ALL keys (causal diagonal, window and relative bias included,
which depend on the keys' positions in the whole sequence).  The shards never
wait on one another, so running them in turn on one GPU is safe.  The last
test runs the whole path, exchange included, through a one-rank NCCL group.
"""
import socket

import numpy as np
import pytest
import torch

import fa_inputs
import oracle
import exact_attention_forward_flash_b200 as fa
from exact_attention_forward_flash_b200.context_parallel import (
    fa_fwd_context_parallel, shard_bounds, shard_seqused)
from parity_util import compare

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    fa.load_library()
    yield
    assert fa.check_device_error() == 0, "a kernel wait timed out"


def sharded(p, world, num_splits=1, window=None, softcap=0.0, align=128):
    """Partials of every shard of p's keys (rank order), merged on the GPU."""
    g = p.to(DEV)
    B, Sq, Hq, _ = p.q.shape
    Sk = p.k.shape[1]
    o_parts, l_parts = [], []
    for r in range(world):
        start, length, after = shard_bounds(Sk, world, r, align=align)
        if p.seqused_k is not None:
            used, aft = shard_seqused(p.seqused_k.tolist(), start, length)
            su = torch.tensor(used, dtype=torch.int32, device=DEV)
        else:
            su, aft = None, [after] * B
        ka = torch.tensor(aft, dtype=torch.int32, device=DEV)
        ks = g.k[:, start:start + length].contiguous()
        vs = g.v[:, start:start + length].contiguous()
        o, l = fa.fa_fwd_shard_partial(g.q, ks, vs, k_after=ka, causal=p.causal,
                                       softmax_scale=p.softmax_scale, seqused_k=su,
                                       rel_bias=g.rel_bias, window=window, softcap=softcap,
                                       num_splits=num_splits)
        o_parts.append(o)
        l_parts.append(l)
    out, lse = fa.fa_combine_partials(torch.stack(o_parts), torch.stack(l_parts), B, Sq, Hq,
                                      dtype=p.q.dtype)
    torch.cuda.synchronize()
    return out, lse


def ref(p, window=(-1, -1), softcap=0.0):
    return oracle.attention(p.q, p.k, p.v, causal=p.causal, softmax_scale=p.softmax_scale,
                            seqused_k=p.seqused_k, rel_bias=p.rel_bias, window=window,
                            softcap=softcap)


@pytest.mark.parametrize("world", [1, 2, 4, 7])
@pytest.mark.parametrize("ns", [1, 3])
def test_decode_shards_merge_to_the_full_result(world, ns):
    p = fa_inputs.random_dense(70 + world, 3, 1, 1000, 8, 2, 128)
    out, lse = sharded(p, world, num_splits=ns)
    ro, rl = ref(p)
    compare(out, lse, ro, rl, what=f"cp decode world={world} ns={ns}")


@pytest.mark.parametrize("D", [16, 64, 72, 128, 256])
def test_causal_bias_seqused_shards(D):
    # several query rows, causal bottom-right diagonal, 128-wide bias and
    # padded keys: every rule that reads a key's global position
    p = fa_inputs.random_dense(80 + D, 2, 37, 900, 8, 2, D, causal=True, seqused=[700, 900],
                               pad_value=1e4, bias_extent=128)
    out, lse = sharded(p, 3, num_splits=2)
    ro, rl = ref(p)
    compare(out, lse, ro, rl, what=f"cp causal bias seqused D={D}")


@pytest.mark.parametrize("D", [64, 128])
def test_fp16_gqa_shards_with_local_splits(D):
    p = fa_inputs.random_dense(95 + D, 2, 17, 2500, 16, 2, D, dtype=torch.float16, causal=True,
                               bias_extent=256)
    out, lse = sharded(p, 3, num_splits=4)
    ro, rl = ref(p)
    compare(out, lse, ro, rl, what=f"cp fp16 D={D}")


def test_window_softcap_shards():
    p = fa_inputs.random_dense(90, 2, 64, 2000, 8, 2, 128, causal=True, q_std=3.0)
    out, lse = sharded(p, 4, num_splits=2, window=(500, 0), softcap=8.0)
    ro, rl = ref(p, window=(500, 0), softcap=8.0)
    compare(out, lse, ro, rl, what="cp window softcap")


def test_empty_shards_contribute_nothing():
    # 200 keys over 4 ranks: shards of 128, 72, 0 and 0 keys
    p = fa_inputs.random_dense(91, 2, 3, 200, 4, 2, 128, causal=True)
    assert shard_bounds(200, 4, 3)[1] == 0
    out, lse = sharded(p, 4)
    ro, rl = ref(p)
    compare(out, lse, ro, rl, what="cp empty shards")


def test_shard_with_no_keys_writes_zero_and_minus_inf():
    p = fa_inputs.random_dense(92, 2, 5, 0, 4, 2, 128)
    g = p.to(DEV)
    o, l = fa.fa_fwd_shard_partial(g.q, g.k, g.v)
    torch.cuda.synchronize()
    assert (o == 0).all() and torch.isneginf(l).all()


def test_merge_is_invariant_to_the_order_of_partials():
    p = fa_inputs.random_dense(93, 2, 1, 1500, 8, 2, 128)
    g = p.to(DEV)
    parts = []
    for r in range(3):
        s, n, a = shard_bounds(1500, 3, r)
        ka = torch.full((2,), a, dtype=torch.int32, device=DEV)
        parts.append(fa.fa_fwd_shard_partial(g.q, g.k[:, s:s + n].contiguous(),
                                             g.v[:, s:s + n].contiguous(), k_after=ka))
    o1, l1 = fa.fa_combine_partials(torch.stack([x[0] for x in parts]),
                                    torch.stack([x[1] for x in parts]), 2, 1, 8)
    rev = parts[::-1]
    o2, l2 = fa.fa_combine_partials(torch.stack([x[0] for x in rev]),
                                    torch.stack([x[1] for x in rev]), 2, 1, 8)
    torch.cuda.synchronize()
    assert (o1.float() - o2.float()).abs().max().item() <= 2 ** -8
    assert (l1 - l2).abs().max().item() <= 1e-5


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_context_parallel_through_a_one_rank_nccl_group():
    import datetime
    import torch.distributed as dist
    p = fa_inputs.random_dense(94, 2, 9, 1100, 8, 2, 128, causal=True, bias_extent=128)
    g = p.to(DEV)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        ka = torch.zeros(2, dtype=torch.int32, device=DEV)
        out, lse = fa_fwd_context_parallel(g.q, g.k, g.v, k_after=ka, causal=True,
                                           softmax_scale=p.softmax_scale, rel_bias=g.rel_bias)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ro, rl = ref(p)
    compare(out, lse, ro, rl, what="cp one-rank nccl")
    # one shard holding every key: the same rows as the plain forward
    o2, l2 = fa.fa_fwd(g.q, g.k, g.v, causal=True, softmax_scale=p.softmax_scale,
                       rel_bias=g.rel_bias)
    torch.cuda.synchronize()
    assert (out.float() - o2.float()).abs().max().item() <= 2 ** -7
    np.testing.assert_allclose(lse.cpu().numpy(), l2.cpu().numpy(), rtol=0, atol=1e-4)
