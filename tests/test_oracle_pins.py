"""Pins of the CPU oracle to things other than itself (CPU only).

Each test checks one oracle function against a library routine (numpy einsum,
torch's scaled_dot_product_attention), a closed form, an invariant, or brute
force on tiny inputs, chosen so that a plausible slip in the oracle (a dropped
head in the score sum, an off-by-one in the causal rule, a reversed tie-break,
a wrong KV-head mapping, a transposed pool index, a wrong scale) fails at least
one of them.

Definitions followed: block scoring and top-k ("Day-0 Inference Adaptation of
Ultra-Large-Scale MoE Models on Domestic AI Accelerators", section 4.1; page 1
"Operatorizing Index Selection"), exact attention over the selected positions
and its agreement with masked full attention (page 3 section IV).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from long_context_indexer_b200.workloads import grid_values


def _gen(seed):
    return torch.Generator().manual_seed(seed)


# ---------------------------------------------------------------- A0 compress

def test_block_compress_closed_forms():
    bs, T = 8, 20  # blocks [0,8) [8,16) [16,20): the last one is partial
    ramp = torch.arange(T, dtype=torch.float32).reshape(1, T, 1, 1).repeat(2, 1, 3, 4)
    kc = oracle.block_compress(ramp, bs)
    assert kc.shape == (2, 3, 3, 4)
    # mean of t over [j*bs, min(T,(j+1)*bs)) is the midpoint of the range
    expect = torch.tensor([3.5, 11.5, 17.5], dtype=torch.float64)
    assert torch.equal(kc[0, :, 0, 0], expect)
    assert torch.equal(kc[1, :, 2, 3], expect)
    const = torch.full((1, 16, 2, 5), 0.3125)
    assert torch.equal(oracle.block_compress(const, 4), torch.full((1, 4, 2, 5), 0.3125,
                                                                   dtype=torch.float64))


def test_block_compress_matches_numpy_mean():
    x = grid_values((2, 64, 3, 16), _gen(1), torch.float32)
    got = oracle.block_compress(x, 16).numpy()
    ref = x.double().numpy().reshape(2, 4, 16, 3, 16).mean(axis=2)
    np.testing.assert_array_equal(got, ref)


def test_block_compress_bf16_is_exact_widening():
    x = grid_values((1, 32, 2, 8), _gen(2), torch.bfloat16)
    a = oracle.block_compress(x, 8)
    b = oracle.block_compress(x.float(), 8)
    assert torch.equal(a, b)


# ---------------------------------------------------------------- A1 scores

def _score_case(seed=3, B=2, S=5, H=3, D=8, NB=6, bs=4, dtype=torch.float32):
    g = _gen(seed)
    q_c = grid_values((B, S, H, D), g, dtype)
    k_c = grid_values((B, NB, H, D), g, dtype)
    ctx = torch.tensor([NB * bs, NB * bs - 3], dtype=torch.int32)[:B]
    q0 = torch.tensor([0, 9], dtype=torch.int32)[:B]
    return q_c, k_c, ctx, q0, bs


def test_block_scores_match_einsum_and_causal_mask():
    q_c, k_c, ctx, q0, bs = _score_case()
    B, S, H, D = q_c.shape
    NB = k_c.shape[1]
    got = oracle.block_scores(q_c, k_c, bs, ctx, q0).reshape(B, S, NB)
    full = np.einsum("bshd,bjhd->bsj", q_c.double().numpy(), k_c.double().numpy())
    for b in range(B):
        for s in range(S):
            p = int(q0[b]) + s
            last = min(p, int(ctx[b]) - 1)
            vis = min(NB, last // bs + 1) if last >= 0 else 0
            row = got[b, s].numpy()
            np.testing.assert_array_equal(row[:vis], full[b, s, :vis])
            assert np.all(np.isneginf(row[vis:]))


def test_scores_on_the_grid_are_exact_in_fp32():
    # Multiples of 1/16 in [-2, 2]: fp32 accumulation in any order equals fp64.
    g = _gen(4)
    q = grid_values((64, 1024), g, torch.float32)
    k = grid_values((128, 1024), g, torch.float32)
    qd, kd = q.double(), k.double()
    exact = qd @ kd.T
    assert torch.equal((q @ k.T).double(), exact)
    assert torch.equal((q.flip(1) @ k.flip(1).T).double(), exact)
    extreme = torch.full((1, 1024), 2.0)
    assert float((extreme @ extreme.T).item()) == 4096.0
    q4 = q.reshape(1, 64, 8, 128)
    k4 = k.reshape(1, 128, 8, 128)
    ora = oracle.block_scores(q4, k4, 1, torch.tensor([128]), torch.tensor([10**6 - 64]))
    assert torch.equal(ora, exact)


def test_visibility_boundaries():
    bs, NB = 16, 8
    q_c = torch.ones((1, 1, 1, 4))
    k_c = torch.ones((1, NB, 1, 4))
    for p, ctx, vis in [(0, 128, 1), (15, 128, 1), (16, 128, 2), (31, 128, 2), (32, 128, 3),
                        (127, 128, 8), (500, 128, 8), (40, 20, 2), (5, 0, 0)]:
        sc = oracle.block_scores(q_c, k_c, bs, torch.tensor([ctx]), torch.tensor([p]))[0]
        n_vis = int(torch.isfinite(sc).sum())
        assert n_vis == vis, (p, ctx, n_vis, vis)
        assert torch.isfinite(sc[:vis]).all()


# ---------------------------------------------------------------- A2 top-k

def _brute_force_ids(scores_row: np.ndarray, vis: int, topk: int):
    """Rank of each visible block = how many visible blocks beat it."""
    out = [-1] * topk
    for j in range(vis):
        rank = 0
        for i in range(vis):
            if scores_row[i] > scores_row[j] or (scores_row[i] == scores_row[j] and i < j):
                rank += 1
        if rank < topk:
            out[rank] = j
    return out


@pytest.mark.parametrize("seed,lo,hi,topk", [(5, -1, 1, 3), (6, -32, 32, 4), (7, 0, 1, 7),
                                             (8, -2, 2, 20)])
def test_index_select_equals_brute_force_ranking(seed, lo, hi, topk):
    g = _gen(seed)
    B, S, H, D, NB, bs = 2, 7, 2, 4, 10, 3
    q_c = grid_values((B, S, H, D), g, torch.float32, lo, hi)
    k_c = grid_values((B, NB, H, D), g, torch.float32, lo, hi)
    ctx = torch.tensor([30, 17], dtype=torch.int32)
    q0 = torch.tensor([1, 12], dtype=torch.int32)
    ids = oracle.index_select(q_c, k_c, bs, ctx, q0, topk).reshape(B, S, topk)
    sc = np.einsum("bshd,bjhd->bsj", q_c.double().numpy(), k_c.double().numpy())
    for b in range(B):
        for s in range(S):
            last = min(int(q0[b]) + s, int(ctx[b]) - 1)
            vis = min(NB, last // bs + 1)
            assert ids[b, s].tolist() == _brute_force_ids(sc[b, s], vis, topk)


def test_index_select_ties_break_to_lower_id():
    q_c = torch.zeros((1, 3, 2, 8))
    k_c = grid_values((1, 12, 2, 8), _gen(9), torch.float32)
    ids = oracle.index_select(q_c, k_c, 4, torch.tensor([48]), torch.tensor([3]), 5)
    # positions 3, 4, 5 see 1, 2, 2 blocks; all scores are 0
    assert ids.tolist() == [[0, -1, -1, -1, -1], [0, 1, -1, -1, -1], [0, 1, -1, -1, -1]]
    ids = oracle.index_select(q_c, k_c, 4, torch.tensor([48]), torch.tensor([47]), 5)
    assert ids[0].tolist() == [0, 1, 2, 3, 4]


def test_index_select_ramp_picks_newest_blocks():
    NB, bs = 16, 4
    q_c = torch.zeros((1, 1, 2, 4))
    q_c[..., 1, 2] = 1.0
    k_c = torch.zeros((1, NB, 2, 4))
    k_c[0, :, 1, 2] = torch.arange(NB) / 16.0  # score of block j = j/16
    for p, expect in [(63, [15, 14, 13]), (9, [2, 1, 0]), (4, [1, 0, -1]), (3, [0, -1, -1])]:
        ids = oracle.index_select(q_c, k_c, bs, torch.tensor([64]), torch.tensor([p]), 3)
        assert ids[0].tolist() == expect, p


def test_index_select_topk_at_least_vis_returns_all_visible_in_rank_order():
    g = _gen(10)
    q_c = grid_values((1, 1, 1, 16), g, torch.float32)
    k_c = grid_values((1, 6, 1, 16), g, torch.float32)
    sc = (k_c[0, :, 0] @ q_c[0, 0, 0]).double()
    order = sorted(range(6), key=lambda j: (-float(sc[j]), j))
    ids = oracle.index_select(q_c, k_c, 8, torch.tensor([48]), torch.tensor([47]), 9)
    assert ids[0].tolist() == order + [-1, -1, -1]


# ---------------------------------------------------------------- A3+A4 attention

def _attn_case(seed=11, B=2, S=3, H_q=4, H_kv=2, hd=8, bs=4, NB=6, spare=3,
               dtype=torch.float64):
    g = _gen(seed)
    P = B * NB + spare
    perm = torch.randperm(P, generator=g).to(torch.int32)
    table = perm[: B * NB].reshape(B, NB)
    k_pool = torch.randn((P, H_kv, bs, hd), generator=g, dtype=torch.float64).to(dtype)
    v_pool = torch.randn((P, H_kv, bs, hd), generator=g, dtype=torch.float64).to(dtype)
    q = torch.randn((B, S, H_q, hd), generator=g, dtype=torch.float64).to(dtype)
    ctx = torch.tensor([NB * bs, NB * bs - 5], dtype=torch.int32)[:B]
    q0 = torch.tensor([NB * bs - S, 9], dtype=torch.int32)[:B]
    return q, k_pool, v_pool, table, ctx, q0


def _logical_kv(pool, table, b, g):
    """Token-major K or V of sequence b, kv head g: [NB*bs, hd] (test's own gather)."""
    return torch.cat([pool[int(table[b, j]), g] for j in range(table.shape[1])], 0)


def _sdpa_row(q_row, k_pool, v_pool, table, b, mask, scale, H_kv):
    """Library attention of one query row [H_q, hd] over the logical cache."""
    H_q, hd = q_row.shape
    G = H_q // H_kv
    K = torch.stack([_logical_kv(k_pool, table, b, g) for g in range(H_kv)])  # [H_kv,T,hd]
    V = torch.stack([_logical_kv(v_pool, table, b, g) for g in range(H_kv)])
    K = K.repeat_interleave(G, dim=0)  # query head h reads kv head h // G
    V = V.repeat_interleave(G, dim=0)
    out = F.scaled_dot_product_attention(q_row[:, None, :].double(), K.double(), V.double(),
                                         attn_mask=mask[None, None, :], scale=scale)
    return out[:, 0, :]


def _block_mask(ids_row, bs, NB, last):
    t = torch.arange(NB * bs)
    sel = torch.zeros(NB, dtype=torch.bool)
    for j in ids_row:
        if j >= 0:
            sel[j] = True
    return sel[t // bs] & (t <= last)


@pytest.mark.parametrize("H_q,H_kv", [(4, 2), (4, 1), (3, 3)])
def test_sparse_attn_matches_sdpa_with_block_mask(H_q, H_kv):
    q, k_pool, v_pool, table, ctx, q0 = _attn_case(H_q=H_q, H_kv=H_kv)
    B, S, _, hd = q.shape
    NB, bs = table.shape[1], k_pool.shape[2]
    g = _gen(12)
    topk = 3
    ids = torch.stack([torch.randperm(NB, generator=g)[:topk] for _ in range(B * S)]).to(torch.int32)
    ids[1, 2] = -1
    scale = 0.37
    got = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, scale)
    for r in range(B * S):
        b, s = divmod(r, S)
        last = min(int(q0[b]) + s, int(ctx[b]) - 1)
        mask = _block_mask(ids[r].tolist(), bs, NB, last)
        if not mask.any():
            assert torch.equal(got[r], torch.zeros_like(got[r]))
            continue
        ref = _sdpa_row(q[b, s], k_pool, v_pool, table, b, mask, scale, H_kv)
        torch.testing.assert_close(got[r], ref, rtol=1e-12, atol=1e-12)


def test_query_past_the_context_attends_only_cached_tokens():
    # last = min(p, ctx - 1): a query positioned beyond the end of its cache
    # attends to tokens up to ctx - 1 only, also inside a selected block whose
    # later slots lie past the context.
    q, k_pool, v_pool, table, _, _ = _attn_case(seed=17, S=3)
    B, S, H_q, hd = q.shape
    NB, bs, H_kv = table.shape[1], k_pool.shape[2], k_pool.shape[1]
    ctx = torch.tensor([NB * bs - 3, 10], dtype=torch.int32)
    q0 = torch.tensor([NB * bs + 5, 30], dtype=torch.int32)
    ids = torch.arange(NB, dtype=torch.int32).repeat(B * S, 1)
    scale = 0.3
    got = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, scale)
    for r in range(B * S):
        b, s = divmod(r, S)
        mask = _block_mask(ids[r].tolist(), bs, NB, int(ctx[b]) - 1)
        ref = _sdpa_row(q[b, s], k_pool, v_pool, table, b, mask, scale, H_kv)
        torch.testing.assert_close(got[r], ref, rtol=1e-12, atol=1e-12)


def test_sparse_attn_equals_dense_masked():
    q, k_pool, v_pool, table, ctx, q0 = _attn_case(seed=13, S=5)
    B, S = q.shape[:2]
    g = _gen(14)
    ids = torch.stack([torch.randperm(6, generator=g)[:4] for _ in range(B * S)]).to(torch.int32)
    a = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, 0.5)
    d = oracle.dense_masked(q, k_pool, v_pool, table, ids, ctx, q0, 0.5)
    torch.testing.assert_close(a, d, rtol=1e-13, atol=1e-13)


def test_full_selection_is_causal_attention():
    # topk >= vis: every visible block is selected, so the result is plain
    # causal attention (a prefill of T tokens attending to themselves).
    g = _gen(15)
    T, bs, H, hd = 24, 4, 2, 8
    NB = T // bs
    q = torch.randn((1, T, H, hd), generator=g, dtype=torch.float64)
    kv = torch.randn((2, T, H, hd), generator=g, dtype=torch.float64)
    # page the logical cache with a reversed table
    table = torch.arange(NB - 1, -1, -1, dtype=torch.int32)[None]
    k_pool = torch.empty((NB, H, bs, hd), dtype=torch.float64)
    v_pool = torch.empty_like(k_pool)
    for j in range(NB):
        k_pool[int(table[0, j])] = kv[0, j * bs:(j + 1) * bs].transpose(0, 1)
        v_pool[int(table[0, j])] = kv[1, j * bs:(j + 1) * bs].transpose(0, 1)
    ctx, q0 = torch.tensor([T]), torch.tensor([0])
    ids = oracle.index_select(torch.zeros((1, T, 1, 4)), torch.zeros((1, NB, 1, 4)), bs, ctx, q0, NB)
    got = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, 1 / math.sqrt(hd))
    ref = F.scaled_dot_product_attention(q[0].transpose(0, 1), kv[0].transpose(0, 1),
                                         kv[1].transpose(0, 1), is_causal=True)
    torch.testing.assert_close(got, ref.transpose(0, 1), rtol=1e-12, atol=1e-12)


def test_attention_closed_forms():
    H, hd, bs, NB = 2, 4, 4, 3
    table = torch.tensor([[2, 0, 1]], dtype=torch.int32)
    ctx, q0 = torch.tensor([12]), torch.tensor([11])
    g = _gen(16)
    q = torch.randn((1, 1, H, hd), generator=g, dtype=torch.float64)
    k_pool = torch.randn((NB, 1, bs, hd), generator=g, dtype=torch.float64)
    ids = torch.tensor([[2, 0]], dtype=torch.int32)
    # constant V: output is that constant
    v_const = torch.full((NB, 1, bs, hd), 0.75, dtype=torch.float64)
    out = oracle.sparse_attn(q, k_pool, v_const, table, ids, ctx, q0, 0.5)
    torch.testing.assert_close(out, torch.full_like(out, 0.75), rtol=0, atol=1e-15)
    # identical keys: uniform weights, output = mean of V over the selected tokens
    v = torch.randn((NB, 1, bs, hd), generator=g, dtype=torch.float64)
    k_same = torch.ones((NB, 1, bs, hd), dtype=torch.float64)
    out = oracle.sparse_attn(q, k_same, v, table, ids, ctx, q0, 0.5)
    sel = torch.cat([v[int(table[0, 2]), 0], v[int(table[0, 0]), 0]])  # blocks 2 and 0
    torch.testing.assert_close(out[0, 0], sel.mean(0), rtol=1e-13, atol=1e-13)


def test_attention_hand_worked_example():
    # One head, hd=2, scale 1, q = (ln 3, 0); tokens 0 and 1 of block 0 with
    # keys (0,0) and (1,0): logits 0 and ln 3, weights 1/4 and 3/4. Values
    # (4,0) and (0,4) give out = (1, 3). Token 2 (key (9,9)) lies beyond the
    # query position p = 1 and must not take part.
    q = torch.tensor([[[[math.log(3.0), 0.0]]]], dtype=torch.float64)
    k_pool = torch.tensor([[[[0.0, 0.0], [1.0, 0.0], [9.0, 9.0], [9.0, 9.0]]]], dtype=torch.float64)
    v_pool = torch.tensor([[[[4.0, 0.0], [0.0, 4.0], [100.0, 100.0], [7.0, 7.0]]]], dtype=torch.float64)
    out = oracle.sparse_attn(q, k_pool, v_pool, torch.tensor([[0]]), torch.tensor([[0]]),
                             torch.tensor([4]), torch.tensor([1]), 1.0)
    torch.testing.assert_close(out[0, 0], torch.tensor([1.0, 3.0], dtype=torch.float64),
                               rtol=0, atol=1e-14)


def test_single_visible_token_and_empty_set():
    q, k_pool, v_pool, table, _, _ = _attn_case(seed=17, B=1, S=1)
    ctx, q0 = torch.tensor([24]), torch.tensor([0])
    ids = torch.tensor([[0, -1, -1]], dtype=torch.int32)
    out = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, 0.3)
    page = int(table[0, 0])
    for h in range(4):
        assert torch.equal(out[0, h], v_pool[page, h // 2, 0])
    none = torch.full((1, 3), -1, dtype=torch.int32)
    assert torch.equal(oracle.sparse_attn(q, k_pool, v_pool, table, none, ctx, q0, 0.3),
                       torch.zeros((1, 4, 8), dtype=torch.float64))
    # a selected block entirely after the query position contributes nothing
    late = torch.tensor([[3, -1, -1]], dtype=torch.int32)
    assert torch.equal(oracle.sparse_attn(q, k_pool, v_pool, table, late, ctx, q0, 0.3),
                       torch.zeros((1, 4, 8), dtype=torch.float64))


def test_page_permutation_and_id_order_invariance():
    q, k_pool, v_pool, table, ctx, q0 = _attn_case(seed=18)
    B, S = q.shape[:2]
    g = _gen(19)
    ids = torch.stack([torch.randperm(6, generator=g)[:4] for _ in range(B * S)]).to(torch.int32)
    base = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, 0.4)
    P = k_pool.shape[0]
    perm = torch.randperm(P, generator=g)  # new page of old page i is perm[i]
    k2 = torch.empty_like(k_pool)
    v2 = torch.empty_like(v_pool)
    k2[perm] = k_pool
    v2[perm] = v_pool
    t2 = perm[table.long()].to(torch.int32)
    assert torch.equal(oracle.sparse_attn(q, k2, v2, t2, ids, ctx, q0, 0.4), base)
    shuffled = ids[:, torch.randperm(4, generator=g)]
    torch.testing.assert_close(oracle.sparse_attn(q, k_pool, v_pool, table, shuffled, ctx, q0, 0.4),
                               base, rtol=1e-13, atol=1e-13)


def test_bf16_inputs_are_widened_exactly():
    q, k_pool, v_pool, table, ctx, q0 = _attn_case(seed=20, dtype=torch.bfloat16)
    ids = torch.tensor([[0, 2, 4]] * 6, dtype=torch.int32)
    a = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, 0.5)
    b = oracle.sparse_attn(q.double(), k_pool.double(), v_pool.double(), table, ids, ctx, q0, 0.5)
    assert torch.equal(a, b)


def test_row_subset_matches_full_call():
    q, k_pool, v_pool, table, ctx, q0 = _attn_case(seed=21, S=4)
    ids = torch.tensor([[1, 3, 5]] * 8, dtype=torch.int32)
    full = oracle.sparse_attn(q, k_pool, v_pool, table, ids, ctx, q0, 0.5)
    part = oracle.sparse_attn(q, k_pool, v_pool, table, ids[[6, 1]], ctx, q0, 0.5, rows=[6, 1])
    assert torch.equal(part, full[[6, 1]])


def test_oracle_rejects_out_of_range_ids():
    q, k_pool, v_pool, table, ctx, q0 = _attn_case(seed=22, B=1, S=1)
    with pytest.raises(ValueError):
        oracle.sparse_attn(q, k_pool, v_pool, table, torch.tensor([[6, -1, -1]]), ctx, q0, 0.5)
    with pytest.raises(ValueError):
        oracle.sparse_attn(q, k_pool, v_pool, table, torch.tensor([[-2, -1, -1]]), ctx, q0, 0.5)


# ---------------------------------------------------------------- N4 gated state scan
# ("Day-0 Adaptation for Trillion-Parameter MoE Models", section III: the state
# is scaled by the chunk's gate, extended by k^T v over the chunk, and read out
# by q for every token of the chunk.)

def _scan_inputs(B, T, H, dk, dv, C, seed, gate_lo=0.5):
    g = _gen(seed)
    q = torch.randn((B, T, H, dk), generator=g, dtype=torch.float64)
    k = torch.randn((B, T, H, dk), generator=g, dtype=torch.float64)
    v = torch.randn((B, T, H, dv), generator=g, dtype=torch.float64)
    nchunks = (T + C - 1) // C
    gate = gate_lo + (1 - gate_lo) * torch.rand((B, H, nchunks), generator=g, dtype=torch.float64)
    s0 = torch.randn((B, H, dk, dv), generator=g, dtype=torch.float64)
    return q, k, v, gate, s0


def test_state_scan_token_chunks_equal_the_gated_recurrence_closed_form():
    """C = 1: o_t = prod_{r<=t} g_r q_t S0 + sum_{s<=t} prod_{s<r<=t} g_r (q_t.k_s) v_s."""
    B, T, H, dk, dv = 2, 9, 3, 4, 5
    q, k, v, gate, s0 = _scan_inputs(B, T, H, dk, dv, 1, 31)
    out, st = oracle.gated_state_scan(q, k, v, gate, s0, 1)
    qn, kn, vn, gn, sn = (x.numpy() for x in (q, k, v, gate, s0))
    for b in range(B):
        for h in range(H):
            g = gn[b, h]
            for t in range(T):
                dec0 = np.prod(g[: t + 1])
                expect = dec0 * qn[b, t, h] @ sn[b, h]
                for s in range(t + 1):
                    expect = expect + np.prod(g[s + 1: t + 1]) * (qn[b, t, h] @ kn[b, s, h]) * vn[b, s, h]
                np.testing.assert_allclose(out[b, t, h].numpy(), expect, rtol=1e-12, atol=1e-12)


def test_state_scan_ungated_is_chunk_masked_linear_attention():
    """gate = 1, S0 = 0: out = ((Q K^T) masked to s < end of t's chunk) V, by
    matmul, with a partial last chunk and dk != dv."""
    B, T, H, dk, dv, C = 1, 11, 2, 6, 3, 4
    q, k, v, _, _ = _scan_inputs(B, T, H, dk, dv, C, 32)
    nchunks = (T + C - 1) // C
    out, _ = oracle.gated_state_scan(q, k, v, torch.ones((B, H, nchunks), dtype=torch.float64),
                                     torch.zeros((B, H, dk, dv), dtype=torch.float64), C)
    t = np.arange(T)
    end = (t // C + 1) * C
    mask = (t[None, :] < end[:, None]).astype(np.float64)       # [t, s]
    for h in range(H):
        qh, kh, vh = q[0, :, h].numpy(), k[0, :, h].numpy(), v[0, :, h].numpy()
        expect = ((qh @ kh.T) * mask) @ vh
        np.testing.assert_allclose(out[0, :, h].numpy(), expect, rtol=1e-12, atol=1e-12)


def test_state_scan_final_state_closed_form_and_input_untouched():
    """S_final = prod_c g_c S0 + sum_s prod_{c > chunk(s)} g_c k_s^T v_s."""
    B, T, H, dk, dv, C = 2, 13, 2, 4, 3, 5
    q, k, v, gate, s0 = _scan_inputs(B, T, H, dk, dv, C, 33)
    s0_copy = s0.clone()
    _, st = oracle.gated_state_scan(q, k, v, gate, s0, C)
    assert torch.equal(s0, s0_copy)
    gn = gate.numpy()
    for b in range(B):
        for h in range(H):
            expect = np.prod(gn[b, h]) * s0[b, h].numpy()
            for s in range(T):
                c = s // C
                expect = expect + np.prod(gn[b, h, c + 1:]) * np.outer(k[b, s, h].numpy(),
                                                                        v[b, s, h].numpy())
            np.testing.assert_allclose(st[b, h].numpy(), expect, rtol=1e-12, atol=1e-12)


def test_state_scan_zero_gate_forgets_earlier_chunks():
    """gate = 0: every chunk reads out q_t (K_c^T V_c) of its own chunk only."""
    B, T, H, dk, dv, C = 1, 8, 1, 3, 4, 4
    q, k, v, _, s0 = _scan_inputs(B, T, H, dk, dv, C, 34)
    out, st = oracle.gated_state_scan(q, k, v, torch.zeros((B, H, 2), dtype=torch.float64), s0, C)
    for c in range(2):
        kc, vc = k[0, c * C:(c + 1) * C, 0].numpy(), v[0, c * C:(c + 1) * C, 0].numpy()
        expect = q[0, c * C:(c + 1) * C, 0].numpy() @ (kc.T @ vc)
        np.testing.assert_allclose(out[0, c * C:(c + 1) * C, 0].numpy(), expect, rtol=1e-12,
                                   atol=1e-12)
    np.testing.assert_allclose(st[0, 0].numpy(), k[0, 4:, 0].numpy().T @ v[0, 4:, 0].numpy(),
                               rtol=1e-12, atol=1e-12)


def test_state_scan_bf16_inputs_are_widened_exactly():
    B, T, H, dk, dv, C = 1, 6, 2, 8, 8, 3
    q, k, v, gate, s0 = _scan_inputs(B, T, H, dk, dv, C, 35)
    qb, kb, vb = (x.to(torch.bfloat16) for x in (q, k, v))
    o1, s1 = oracle.gated_state_scan(qb, kb, vb, gate, s0, C)
    o2, s2 = oracle.gated_state_scan(qb.double(), kb.double(), vb.double(), gate, s0, C)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)
