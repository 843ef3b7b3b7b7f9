"""Pins for the CPU oracle: facts fixed by the pages and by the mathematics.

Each check is chosen so that a plausible mistake in the oracle (a dropped
term, a sign or index error, a transposed operand, a wrong mask direction,
scaling the bias) fails at least one of them.  None of them re-calls the
oracle's own routine to produce an expected value.
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle
import fa_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _one_hot_v(n_keys, D, Hkv=1, B=None):
    """v_j = e_j, so an output row equals its attention row."""
    v = np.zeros((n_keys, Hkv, D), dtype=np.float32)
    for j in range(n_keys):
        v[j, :, j] = 1.0
    return v


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------

def test_single_key_returns_its_value_and_score():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((1, 3, 2, 8)).astype(np.float32)
    k = rng.standard_normal((1, 1, 2, 8)).astype(np.float32)
    v = rng.standard_normal((1, 1, 2, 8)).astype(np.float32)
    o, lse = oracle.attention(q, k, v, softmax_scale=0.3)
    for h in range(2):
        for i in range(3):
            np.testing.assert_array_equal(o[0, i, h], v[0, 0, h].astype(np.float64))
            s0 = 0.3 * float(np.dot(q[0, i, h].astype(np.float64), k[0, 0, h].astype(np.float64)))
            assert lse[0, h, i] == pytest.approx(s0, abs=1e-12)


def test_constant_values_give_that_constant():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((2, 5, 4, 16)).astype(np.float32) * 3
    k = rng.standard_normal((2, 7, 2, 16)).astype(np.float32)
    c = rng.standard_normal(16).astype(np.float32)
    v = np.broadcast_to(c, (2, 7, 2, 16)).copy()
    for causal in (False, True):
        o, _ = oracle.attention(q, k, v, causal=causal)
        np.testing.assert_allclose(o, np.broadcast_to(c.astype(np.float64), o.shape), rtol=0, atol=1e-13)


def test_zero_query_gives_mean_of_admissible_values():
    """q = 0 makes every score 0: O is the mean of V over the admissible keys
    and LSE = ln(count).  The count encodes causal bottom-right alignment
    (row i admits i + (k_len - q_len) + 1 keys) and seqused_k."""
    rng = np.random.default_rng(2)
    B, Sq, Sk, H, D = 2, 4, 9, 2, 8
    q = np.zeros((B, Sq, H, D), np.float32)
    k = rng.standard_normal((B, Sk, H, D)).astype(np.float32)
    v = rng.standard_normal((B, Sk, H, D)).astype(np.float32)
    used = [9, 6]
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal=causal, seqused_k=used)
        for b in range(B):
            for i in range(Sq):
                n = used[b]
                if causal:
                    n = min(n, i + (used[b] - Sq) + 1)
                for h in range(H):
                    mean = v[b, :n, h].astype(np.float64).mean(axis=0)
                    np.testing.assert_allclose(o[b, i, h], mean, atol=1e-14)
                    assert lse[b, h, i] == pytest.approx(math.log(n), abs=1e-14)


def test_rows_are_stochastic_and_masked_keys_get_zero_weight():
    """With one-hot values the output row is the probability row: it sums to
    1, is nonnegative, and is exactly 0 on causally masked keys (j > i + delta)
    and on keys beyond seqused_k."""
    rng = np.random.default_rng(3)
    Sq, Sk, D = 5, 12, 16
    q = rng.standard_normal((1, Sq, 1, D)).astype(np.float32)
    k = rng.standard_normal((1, Sk, 1, D)).astype(np.float32)
    v = _one_hot_v(Sk, D)[None]
    o, _ = oracle.attention(q, k, v, causal=True, seqused_k=[10])
    delta = 10 - Sq
    for i in range(Sq):
        p = o[0, i, 0]
        assert abs(p.sum() - 1.0) < 1e-15
        assert (p >= 0).all()
        for j in range(Sk):
            if j > i + delta or j >= 10:
                assert p[j] == 0.0
            else:
                assert p[j] > 0.0


def test_probabilities_follow_exp_of_scores_high_precision():
    """Brute force in 50-digit decimal arithmetic: the whole score matrix is
    built first, masked entries dropped, and softmax taken without any max
    shift.  Covers every flag combination on tiny shapes."""
    getcontext().prec = 50
    rng = np.random.default_rng(4)
    for case in range(16):
        causal = bool(case & 1)
        use_bias = bool(case & 2)
        gqa = bool(case & 4)
        varlen = bool(case & 8)
        Hkv = 1 if gqa else 2
        Hq = 2
        D = 4
        q_lens = [3, 1] if varlen else [3, 3]
        k_lens = [5, 2] if varlen else [5, 5]
        R = 3
        cu_q = np.cumsum([0] + q_lens).astype(np.int32)
        cu_k = np.cumsum([0] + k_lens).astype(np.int32)
        q = (rng.standard_normal((cu_q[-1], Hq, D)) * 0.7).astype(np.float32)
        k = (rng.standard_normal((cu_k[-1], Hkv, D)) * 0.7).astype(np.float32)
        v = rng.standard_normal((cu_k[-1], Hkv, D)).astype(np.float32)
        rb = rng.standard_normal((cu_q[-1], Hq, R)).astype(np.float32) if use_bias else None
        scale = 0.8
        o, lse = oracle.attention(q, k, v, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
                                  causal=causal, softmax_scale=scale, rel_bias=rb)
        for b in range(2):
            ql, kl = q_lens[b], k_lens[b]
            for h in range(Hq):
                kh = h // (Hq // Hkv)
                # full score matrix, None where masked
                S = [[None] * kl for _ in range(ql)]
                for i in range(ql):
                    for j in range(kl):
                        d = i + (kl - ql) - j
                        if causal and d < 0:
                            continue
                        dot = sum(Decimal(float(q[cu_q[b] + i, h, t])) * Decimal(float(k[cu_k[b] + j, kh, t]))
                                  for t in range(D))
                        s = Decimal(scale) * dot
                        if rb is not None and 0 <= d < R:
                            s += Decimal(float(rb[cu_q[b] + i, h, d]))
                        S[i][j] = s
                for i in range(ql):
                    e = [x.exp() if x is not None else Decimal(0) for x in S[i]]
                    Z = sum(e)
                    row = cu_q[b] + i
                    if Z == 0:
                        assert lse[h, row] == -math.inf
                        assert (o[row, h] == 0).all()
                        continue
                    assert lse[h, row] == pytest.approx(float(Z.ln()), abs=1e-13)
                    for t in range(D):
                        ref = sum(e[j] * Decimal(float(v[cu_k[b] + j, kh, t])) for j in range(kl)) / Z
                        assert o[row, h, t] == pytest.approx(float(ref), abs=1e-13)


# --------------------------------------------------------------------------
# the relative-bias contract, hand-built from the page's rule
# --------------------------------------------------------------------------

def _bias_case(case):
    ql, kl, R = case["q_len"], case["k_len"], case["rel_extent"]
    D = 256
    assert kl <= D
    q = np.zeros((ql, 1, D), np.float32)
    k = np.zeros((kl, 1, D), np.float32)
    v = _one_hot_v(kl, D)
    rb = np.zeros((ql, 1, R), np.float32)
    if "bias_all" in case:
        rb[:] = case["bias_all"]
    for dstr, val in case.get("bias", {}).items():
        rb[:, 0, int(dstr)] = val
    o, lse = oracle.attention(q, k, v, cu_seqlens_q=[0, ql], cu_seqlens_k=[0, kl],
                              causal=case["causal"], rel_bias=rb)
    return o[:, 0, :kl], lse[0], rb


def test_rel_bias_contract_golden_cases():
    with open(os.path.join(GOLDEN, "rel_bias_contract.json")) as f:
        spec = json.load(f)
    for case in spec["cases"]:
        P, lse, rb = _bias_case(case)
        ql, kl, R = case["q_len"], case["k_len"], case["rel_extent"]
        delta = kl - ql
        dom = case["dominant"]
        rows = case.get("check_rows", range(ql))
        for i in rows:
            want = dom[str(i)] if isinstance(dom, dict) else dom[i]
            p = P[i]
            admissible = [j for j in range(kl) if not (case["causal"] and i + delta - j < 0)]
            if want == "all":
                np.testing.assert_allclose(p[admissible], 1.0 / len(admissible), atol=1e-12)
                continue
            # the dominant keys share (almost) all the weight equally
            assert p[want].sum() > 1 - 1e-9, (case["name"], i, p)
            np.testing.assert_allclose(p[want], 1.0 / len(want), atol=1e-9)
            # closed form: weight of key j is exp(bias(d_j)) / sum
            w = []
            for j in admissible:
                d = i + delta - j
                w.append(math.exp(rb[i, 0, d]) if 0 <= d < R else 1.0)
            Z = math.fsum(w)
            for j, wj in zip(admissible, w):
                assert p[j] == pytest.approx(wj / Z, rel=1e-12, abs=1e-300)
            assert lse[i] == pytest.approx(math.log(Z), abs=1e-12)


def test_bias_is_added_unscaled_and_shifts_lse():
    """A bias c on every admissible key (causal, all d < rel_extent) leaves O
    unchanged and moves LSE by exactly c -- not by c * scale."""
    rng = np.random.default_rng(5)
    ql = kl = 6
    D, R, c = 8, 128, 1.75
    q = rng.standard_normal((ql, 2, D)).astype(np.float32)
    k = rng.standard_normal((kl, 2, D)).astype(np.float32)
    v = rng.standard_normal((kl, 2, D)).astype(np.float32)
    rb = np.full((ql, 2, R), c, np.float32)
    kw = dict(cu_seqlens_q=[0, ql], cu_seqlens_k=[0, kl], causal=True, softmax_scale=0.25)
    o0, l0 = oracle.attention(q, k, v, **kw)
    o1, l1 = oracle.attention(q, k, v, rel_bias=rb, **kw)
    np.testing.assert_allclose(o1, o0, atol=1e-14)
    np.testing.assert_allclose(l1 - l0, c, atol=1e-13)


def test_rel_extent_boundary():
    """d = rel_extent - 1 is biased, d = rel_extent is not."""
    R = 4
    ql = kl = 7
    D = 8
    q = np.zeros((ql, 1, D), np.float32)
    k = np.zeros((kl, 1, D), np.float32)
    v = _one_hot_v(kl, D)
    rb = np.zeros((ql, 1, R), np.float32)
    rb[:, 0, R - 1] = 5.0
    o, _ = oracle.attention(q, k, v, cu_seqlens_q=[0, ql], cu_seqlens_k=[0, kl],
                            causal=True, rel_bias=rb)
    i = 6
    p = o[i, 0]
    j_biased = i - (R - 1)           # d = R - 1
    j_unbiased = i - R               # d = R
    assert p[j_biased] == pytest.approx(math.exp(5.0) / (math.exp(5.0) + 6))
    assert p[j_unbiased] == pytest.approx(1.0 / (math.exp(5.0) + 6))


# --------------------------------------------------------------------------
# structural invariants
# --------------------------------------------------------------------------

def test_fully_masked_rows_are_zero_with_minus_inf_lse():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((1, 5, 1, 8)).astype(np.float32)
    k = rng.standard_normal((1, 3, 1, 8)).astype(np.float32)
    v = rng.standard_normal((1, 3, 1, 8)).astype(np.float32)
    o, lse = oracle.attention(q, k, v, causal=True)
    # delta = -2: rows 0 and 1 see no key
    for i in (0, 1):
        assert (o[0, i, 0] == 0).all() and lse[0, 0, i] == -math.inf
    for i in (2, 3, 4):
        assert np.isfinite(lse[0, 0, i])
    o, lse = oracle.attention(q, k, v, seqused_k=[0])
    assert (o == 0).all() and (lse == -math.inf).all()


def test_varlen_equals_per_sequence_dense():
    p = fa_inputs.random_varlen(7, [3, 0, 5], [4, 2, 5], Hq=4, Hkv=2, D=16,
                                causal=True, bias_extent=128)
    o, lse = oracle.attention(p.q, p.k, p.v, cu_seqlens_q=p.cu_seqlens_q,
                              cu_seqlens_k=p.cu_seqlens_k, causal=True,
                              rel_bias=p.rel_bias)
    cq, ck = p.cu_seqlens_q.tolist(), p.cu_seqlens_k.tolist()
    for b in range(3):
        if cq[b + 1] == cq[b]:
            continue
        qb = p.q[cq[b]:cq[b + 1]][None]
        kb = p.k[ck[b]:ck[b + 1]][None]
        vb = p.v[ck[b]:ck[b + 1]][None]
        rbb = p.rel_bias[cq[b]:cq[b + 1]][None]
        od, ld = oracle.attention(qb, kb, vb, causal=True, rel_bias=rbb)
        np.testing.assert_array_equal(o[cq[b]:cq[b + 1]], od[0])
        np.testing.assert_array_equal(lse[:, cq[b]:cq[b + 1]], ld[0])


def test_gqa_reads_kv_head_h_div_group():
    """Query head h uses K/V head h // (Hq/Hkv): equal to MHA with each K/V
    head repeated for its group of consecutive query heads."""
    p = fa_inputs.random_dense(8, 1, 6, 9, Hq=6, Hkv=2, D=8, causal=True)
    o, lse = oracle.attention(p.q, p.k, p.v, causal=True)
    k_rep = p.k.repeat_interleave(3, dim=2)
    v_rep = p.v.repeat_interleave(3, dim=2)
    o2, lse2 = oracle.attention(p.q, k_rep, v_rep, causal=True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    # and a different grouping (h % Hkv) would differ
    k_tile = p.k.repeat(1, 1, 3, 1)
    v_tile = p.v.repeat(1, 1, 3, 1)
    o3, _ = oracle.attention(p.q, k_tile, v_tile, causal=True)
    assert np.abs(o3 - o).max() > 1e-3


def test_seqused_ignores_padded_rows():
    p = fa_inputs.random_dense(9, 2, 5, 11, Hq=4, Hkv=1, D=16, seqused=[7, 11],
                               pad_value=1e4)
    o, lse = oracle.attention(p.q, p.k, p.v, seqused_k=p.seqused_k)
    for b, u in enumerate([7, 11]):
        ob, lb = oracle.attention(p.q[b:b + 1], p.k[b:b + 1, :u], p.v[b:b + 1, :u])
        np.testing.assert_array_equal(o[b], ob[0])
        np.testing.assert_array_equal(lse[b], lb[0])
    assert np.isfinite(o).all() and np.abs(o).max() < 10


def test_split_partials_combine_to_unsplit():
    p = fa_inputs.random_dense(10, 2, 3, 40, Hq=4, Hkv=2, D=8, causal=True,
                               bias_extent=128)
    o, lse = oracle.attention(p.q, p.k, p.v, causal=True, rel_bias=p.rel_bias)
    bounds = [0, 7, 16, 16, 33, 40]
    parts_o, parts_l = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        po, pl = oracle.attention(p.q, p.k, p.v, causal=True, rel_bias=p.rel_bias,
                                  kv_range=(lo, hi))
        parts_o.append(po.reshape(-1, 8))
        # lse [B,Hq,Sq] -> row order of out [B,Sq,Hq]
        parts_l.append(pl.transpose(0, 2, 1).reshape(-1))
    co, cl = oracle.lse_combine(np.stack(parts_o), np.stack(parts_l))
    np.testing.assert_allclose(co, o.reshape(-1, 8), atol=1e-13)
    np.testing.assert_allclose(cl, lse.transpose(0, 2, 1).reshape(-1), atol=1e-13)
    # the empty split (16, 16) has lse -inf and no weight
    assert (parts_l[2] == -math.inf).all()


def test_rows_entry_matches_full_entry():
    p = fa_inputs.random_varlen(11, [4, 6], [5, 6], Hq=4, Hkv=2, D=8,
                                causal=True, bias_extent=128)
    o, lse = oracle.attention(p.q, p.k, p.v, cu_seqlens_q=p.cu_seqlens_q,
                              cu_seqlens_k=p.cu_seqlens_k, causal=True,
                              rel_bias=p.rel_bias)
    rows = np.array([[0, 0, 0], [0, 3, 3], [1, 1, 5], [1, 2, 0]])
    ro, rl = oracle.attention_rows(p.q, p.k, p.v, rows, cu_seqlens_q=p.cu_seqlens_q,
                                   cu_seqlens_k=p.cu_seqlens_k, causal=True,
                                   rel_bias=p.rel_bias)
    cq = p.cu_seqlens_q.tolist()
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(ro[n], o[cq[b] + i, h])
        assert rl[n] == lse[h, cq[b] + i]


def test_default_scale_is_inverse_sqrt_head_dim():
    p = fa_inputs.random_dense(12, 1, 3, 4, Hq=1, Hkv=1, D=64)
    o0, l0 = oracle.attention(p.q, p.k, p.v)
    o1, l1 = oracle.attention(p.q, p.k, p.v, softmax_scale=0.125)
    np.testing.assert_array_equal(o0, o1)
    np.testing.assert_array_equal(l0, l1)


def test_workload_shapes_match_their_descriptions():
    p = fa_inputs.make("dense_257")
    assert tuple(p.q.shape) == (1, 257, 8, 128) and p.q.dtype == torch.bfloat16
    p = fa_inputs.make("varlen_gqa_bias")
    lens = p.meta["lens"]
    assert len(lens) == 4 and all(512 <= L <= 4096 for L in lens)
    assert tuple(p.rel_bias.shape) == (sum(lens), 32, 256)
    assert p.causal and p.Hq == 32 and p.Hkv == 8
    p = fa_inputs.make("encoder_d256_seqused")
    assert p.seqused_k.tolist() == [968, 968]
    # 1e4 rounded to bf16
    pad = float(torch.tensor(1e4).to(torch.bfloat16))
    assert float(p.k[0, 968:].float().min()) == pad and float(p.v[1, 968:].float().max()) == pad
    p = fa_inputs.make("tabpfn_d16")
    assert tuple(p.q.shape) == (1, 30000, 8, 16) and p.q.dtype == torch.float16
    p = fa_inputs.make("vision_d72")
    assert tuple(p.k.shape) == (32, 729, 16, 72) and not p.causal


# --------------------------------------------------------------------------
# score and mask modifiers (readings of the pages' "mask/score modifiers"):
# sliding window by distance d = i + (k_len - q_len) - j, soft-cap before bias
# --------------------------------------------------------------------------
@pytest.mark.parametrize("q_len,k_len,left,right,causal", [
    (6, 6, 2, 1, False),    # window both sides
    (5, 9, 3, -1, False),   # left bound only, k longer (delta = 4)
    (7, 4, -1, 2, False),   # right bound only, k shorter (delta = -3)
    (6, 8, 1, 5, True),     # causal caps the right side at 0
    (8, 8, 0, 0, False),    # the diagonal key alone
])
def test_window_weights_are_uniform_over_the_admissible_band(q_len, k_len, left, right, causal):
    # q = 0: every admissible key has score 0, so with one-hot values each
    # output row is 1/count on the admissible keys and LSE = ln(count)
    D = max(k_len, 1)
    q = np.zeros((q_len, 1, D), dtype=np.float32)
    k = np.random.default_rng(5).standard_normal((k_len, 1, D)).astype(np.float32)
    v = _one_hot_v(k_len, D)
    cu_q = np.array([0, q_len], dtype=np.int32)
    cu_k = np.array([0, k_len], dtype=np.int32)
    out, lse = oracle.attention(q, k, v, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
                                causal=causal, window=(left, right))
    delta = k_len - q_len
    for i in range(q_len):
        ok = []
        for j in range(k_len):
            d = i + delta - j
            if causal and d < 0:
                continue
            if left >= 0 and d > left:
                continue
            if right >= 0 and -d > right:
                continue
            ok.append(j)
        want = np.zeros(D)
        for j in ok:
            want[j] = 1.0 / len(ok)
        np.testing.assert_allclose(out[i, 0], want, atol=1e-15)
        if ok:
            assert lse[0, i] == pytest.approx(math.log(len(ok)), abs=1e-14)
        else:
            assert lse[0, i] == -math.inf


def test_softcap_single_key_closed_form_and_order_with_bias():
    # D = 1, q = 2, k = 3, scale 1: raw score 6; one key, so LSE is the score
    q = np.full((1, 1, 1), 2.0, dtype=np.float32)
    k = np.full((1, 1, 1), 3.0, dtype=np.float32)
    v = np.full((1, 1, 1), 0.75, dtype=np.float32)
    cu = np.array([0, 1], dtype=np.int32)
    for cap in (4.0, 10.0, 0.5):
        out, lse = oracle.attention(q, k, v, cu_seqlens_q=cu, cu_seqlens_k=cu,
                                    softmax_scale=1.0, softcap=cap)
        assert out[0, 0, 0] == pytest.approx(0.75, abs=1e-15)
        assert lse[0, 0] == pytest.approx(cap * math.tanh(6.0 / cap), abs=1e-13)
    # the bias (distance 0) is added after the cap, unscaled
    rb = np.full((1, 1, 128), 0.0, dtype=np.float32)
    rb[0, 0, 0] = -1.25
    out, lse = oracle.attention(q, k, v, cu_seqlens_q=cu, cu_seqlens_k=cu,
                                softmax_scale=1.0, softcap=4.0, rel_bias=rb)
    assert lse[0, 0] == pytest.approx(4.0 * math.tanh(1.5) - 1.25, abs=1e-13)


def test_softcap_saturates_and_vanishes_in_the_limit():
    # raw scores +1e6 and -1e6 cap to +c and -c: weights 1/(1 + e^{-2c})
    q = np.full((1, 1, 2), 1.0, dtype=np.float32)
    k = np.array([[[1e6, 0.0]], [[-1e6, 0.0]]], dtype=np.float32)
    v = _one_hot_v(2, 2)
    cu_q = np.array([0, 1], dtype=np.int32)
    cu_k = np.array([0, 2], dtype=np.int32)
    c = 1.5
    out, lse = oracle.attention(q, k, v, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
                                softmax_scale=1.0, softcap=c)
    w1 = 1.0 / (1.0 + math.exp(-2 * c))
    np.testing.assert_allclose(out[0, 0], [w1, 1.0 - w1], atol=1e-15)
    assert lse[0, 0] == pytest.approx(c + math.log1p(math.exp(-2 * c)), abs=1e-13)
    # a cap far above the scores leaves them as they are
    k2 = np.array([[[0.5, 0.0]], [[-0.25, 0.0]]], dtype=np.float32)
    out, lse = oracle.attention(q, k2, v, cu_seqlens_q=cu_q, cu_seqlens_k=cu_k,
                                softmax_scale=1.0, softcap=1e9)
    z = math.exp(0.5) + math.exp(-0.25)
    np.testing.assert_allclose(out[0, 0], [math.exp(0.5) / z, math.exp(-0.25) / z], atol=1e-12)
    assert lse[0, 0] == pytest.approx(math.log(z), abs=1e-12)


def _dtanh(x):
    """tanh in decimal arithmetic from its exponential definition."""
    e = (2 * x).exp()
    return (e - 1) / (e + 1)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("window", [(-1, -1), (1, -1), (2, 0), (-1, 1), (0, 0)])
@pytest.mark.parametrize("softcap", [0.0, 1.5])
def test_dense_modifiers_seqused_and_ranges_high_precision(causal, window, softcap):
    """Brute force in 50-digit decimals on the dense entry: seqused_k sets each
    sequence's k_len (and so the diagonal), keys are dropped by the causal,
    left and right distance bounds, the cap maps s to c*tanh(s/c) before the
    bias is added, and a key range returns the softmax over its keys only.
    Shapes have Sq != Sk, GQA, and rows that every key misses."""
    getcontext().prec = 50
    rng = np.random.default_rng(100 + 10 * causal + 3 * window[0] + window[1] + int(softcap))
    B, Sq, Sk, Hq, Hkv, D, R = 2, 3, 6, 4, 2, 4, 4
    seqused = [4, 6]
    scale = 0.9
    q = (rng.standard_normal((B, Sq, Hq, D)) * 0.8).astype(np.float32)
    k = (rng.standard_normal((B, Sk, Hkv, D)) * 0.8).astype(np.float32)
    v = rng.standard_normal((B, Sk, Hkv, D)).astype(np.float32)
    k[0, 4:] = 1e4  # padding past seqused_k must never be read
    v[0, 4:] = 1e4
    rb = rng.standard_normal((B * Sq, Hq, R)).astype(np.float32)
    cap = Decimal(softcap)
    left, right = window
    for kv_range in (None, (1, 4)):
        kw = dict(seqused_k=np.array(seqused, np.int32), causal=causal, softmax_scale=scale,
                  rel_bias=rb, window=window, softcap=softcap)
        if kv_range is not None:
            kw["kv_range"] = kv_range
        o, lse = oracle.attention(q, k, v, **kw)
        lo, hi = kv_range if kv_range is not None else (0, Sk)
        for b in range(B):
            kl = seqused[b]
            for h in range(Hq):
                kh = h // (Hq // Hkv)
                for i in range(Sq):
                    e = {}
                    for j in range(max(lo, 0), min(hi, kl)):
                        d = i + kl - Sq - j
                        if (causal and d < 0) or (left >= 0 and d > left) or \
                                (right >= 0 and -d > right):
                            continue
                        s = Decimal(scale) * sum(Decimal(float(q[b, i, h, t])) *
                                                 Decimal(float(k[b, j, kh, t])) for t in range(D))
                        if softcap > 0:
                            s = cap * _dtanh(s / cap)
                        if 0 <= d < R:
                            s += Decimal(float(rb[b * Sq + i, h, d]))
                        e[j] = s.exp()
                    if not e:
                        assert lse[b, h, i] == -math.inf and (o[b, i, h] == 0).all()
                        continue
                    Z = sum(e.values())
                    assert lse[b, h, i] == pytest.approx(float(Z.ln()), abs=1e-13)
                    for t in range(D):
                        ref = sum(w * Decimal(float(v[b, j, kh, t])) for j, w in e.items()) / Z
                        assert o[b, i, h, t] == pytest.approx(float(ref), abs=1e-12)


def test_lse_merge_closed_form_and_degenerate_partials():
    """The merge of key-range partials against its closed form in decimals:
    LSE = ln(sum_s e^{LSE_s}), O = sum_s e^{LSE_s} O_s / e^{LSE}.  Partials of
    magnitude 1000 (e^1000 overflows a double, so the merge must shift by the
    max), a -inf partial that must carry no weight, and a row that every
    partial misses (O = 0, LSE = -inf, no NaN)."""
    getcontext().prec = 50
    rng = np.random.default_rng(7)
    S, D = 3, 5
    lse_parts = np.array([[1000.0, -3.0, 0.5, -math.inf, -math.inf],
                          [1001.5, -2.0, -math.inf, 2.0, -math.inf],
                          [999.25, -7.5, 0.25, -math.inf, -math.inf]])
    o_parts = rng.standard_normal((S, 5, D))
    co, cl = oracle.lse_combine(o_parts, lse_parts)
    for r in range(5):
        live = [s for s in range(S) if lse_parts[s, r] != -math.inf]
        if not live:
            assert cl[r] == -math.inf and (co[r] == 0).all()
            continue
        w = {s: Decimal(float(lse_parts[s, r])).exp() for s in live}
        Z = sum(w.values())
        assert cl[r] == pytest.approx(float(Z.ln()), abs=1e-12)
        for t in range(D):
            ref = sum(w[s] * Decimal(float(o_parts[s, r, t])) for s in live) / Z
            # at |LSE| ~ 1000 one ulp of a double is 1.1e-13, and the weights
            # exp(LSE_s - LSE) inherit it as a relative error
            assert co[r, t] == pytest.approx(float(ref), abs=1e-12)
    # a single live partial passes through unchanged
    assert cl[3] == 2.0 and (co[3] == o_parts[1, 3]).all()
    assert np.isfinite(co).all()
