"""Pins of the fp64 oracle against things other than itself.

Each test checks the oracle against a value the mathematics fixes: a library
routine that implements the same formula (torch fp64 scaled_dot_product_attention
over an independently gathered dense KV), hand-derived closed forms
(tests/golden), invariants of softmax attention, and brute force on tiny integer
inputs.  Together they catch a dropped term, a wrong sign, a transposed operand,
a wrong GQA head index, a wrong page/slot index or a read past kv_len.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from prefix_aware_decode_b200 import workload as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def dense_gather(w, b):
    """Independent numpy gather of request b's K/V: [Hkv][n][D] as float64."""
    n = int(w.kv_lens[b])
    pages = w.block_table[b, : -(-n // w.P)]
    k = wl.bf16_bits_to_f32(w.k_pool[pages])  # [np][Hkv][P][D]
    v = wl.bf16_bits_to_f32(w.v_pool[pages])
    k = k.transpose(1, 0, 2, 3).reshape(w.Hkv, -1, w.D)[:, :n].astype(np.float64)
    v = v.transpose(1, 0, 2, 3).reshape(w.Hkv, -1, w.D)[:, :n].astype(np.float64)
    return k, v


def sdpa_reference(w, b):
    """torch fp64 SDPA with an explicit GQA repeat (kv head h // G); lse by torch.logsumexp."""
    k, v = dense_gather(w, b)
    G = w.Hq // w.Hkv
    q = torch.from_numpy(wl.bf16_bits_to_f32(w.q[b]).astype(np.float64))  # [Hq][D]
    K = torch.from_numpy(k).repeat_interleave(G, dim=0)  # [Hq][n][D]
    V = torch.from_numpy(v).repeat_interleave(G, dim=0)
    out = torch.nn.functional.scaled_dot_product_attention(q[:, None, :], K, V)[:, 0, :]
    logits = torch.einsum("hd,hnd->hn", q, K) / math.sqrt(w.D)
    lse = torch.logsumexp(logits, dim=-1)
    return out.numpy(), lse.numpy()


# ------------------------------------------------------------------ golden closed forms

def test_golden_dense_cases():
    cases = json.load(open(GOLDEN))["dense"]
    for c in cases:
        out, lse = oracle.attend_dense(c["q"], c["K"], c["V"])
        np.testing.assert_allclose(out, c["out"], rtol=0, atol=1e-15, err_msg=c["name"])
        assert abs(lse - c["lse"]) <= 1e-14, c["name"]


def test_golden_paged_case():
    g = json.load(open(GOLDEN))["paged"]
    P, Hkv, D = g["P"], g["Hkv"], g["D"]
    nan = np.float32("nan")
    kp = np.full((g["num_pages"], Hkv, P, D), nan, dtype=np.float32)
    vp = np.full((g["num_pages"], Hkv, P, D), nan, dtype=np.float32)
    bt = np.array(g["block_table"], dtype=np.int32)
    for t, (kr, vr) in enumerate(zip(g["tokens"]["K"], g["tokens"]["V"])):
        page = bt[0, t // P]
        kp[page, 0, t % P] = kr
        vp[page, 0, t % P] = vr
    out, lse = oracle.attend_paged(to_bf16_bits(np.array(g["q"])), to_bf16_bits(kp), to_bf16_bits(vp), bt,
                                   np.array(g["kv_lens"], dtype=np.int32))
    np.testing.assert_allclose(out, np.array(g["out"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, np.array(g["lse"]), rtol=0, atol=1e-14)


# ------------------------------------------------------------------ library routine

@pytest.mark.parametrize("config", [1, 2])
def test_paged_matches_torch_sdpa(config):
    w = wl.make_config(config, scale=1.0 if config == 1 else 0.125)
    out, lse = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
    for b in range(w.B):
        ro, rl = sdpa_reference(w, b)
        np.testing.assert_allclose(out[b], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)
    assert np.isfinite(out).all()


def test_paged_subset_config3_shape():
    w = wl.make_config(3, scale=0.125)
    qs = np.array([0, w.B // 2, w.B - 1], dtype=np.int32)
    out, lse = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens, queries=qs)
    for i, b in enumerate(qs):
        ro, rl = sdpa_reference(w, b)
        np.testing.assert_allclose(out[i], ro, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[i], rl, rtol=0, atol=1e-12)


def test_paged_random_forest_gqa_variants():
    for G, D in [(1, 64), (2, 128), (8, 64)]:
        roots = wl.random_tree(seed=11 + G, n_queries=6, depth=2)
        w = wl.build_workload("rand", roots, Hq=2 * G, Hkv=2, D=D, seed=77 + G)
        out, lse = oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, w.kv_lens)
        for b in range(w.B):
            ro, rl = sdpa_reference(w, b)
            np.testing.assert_allclose(out[b], ro, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b], rl, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ invariants

def rng(seed):
    return np.random.default_rng(seed)


def test_weights_sum_to_one():
    r = rng(1)
    for n in (1, 7, 300):
        q = r.standard_normal(64)
        K = r.standard_normal((n, 64)) * 3
        out, _ = oracle.attend_dense(q, K, np.ones((n, 64)))
        np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def test_single_key_returns_v_exactly():
    r = rng(2)
    q, k, v = r.standard_normal(128), r.standard_normal((1, 128)), r.standard_normal((1, 128))
    out, lse = oracle.attend_dense(q, k, v)
    assert np.array_equal(out, v[0])
    assert abs(lse - float(q @ k[0]) / math.sqrt(128)) < 1e-12


def test_identical_keys_give_mean_and_log_n():
    r = rng(3)
    n, D = 37, 64
    q, k = r.standard_normal(D), r.standard_normal(D)
    V = r.standard_normal((n, D))
    out, lse = oracle.attend_dense(q, np.tile(k, (n, 1)), V)
    np.testing.assert_allclose(out, V.mean(axis=0), rtol=0, atol=1e-12)
    assert abs(lse - (float(q @ k) / math.sqrt(D) + math.log(n))) < 1e-12


def test_merge_of_any_split_equals_unsplit():
    r = rng(4)
    D = 128
    for trial in range(20):
        n = int(r.integers(2, 400))
        q = r.standard_normal(D)
        K = r.standard_normal((n, D)) * 2
        V = r.standard_normal((n, D))
        full, lfull = oracle.attend_dense(q, K, V)
        perm = r.permutation(n)
        cuts = np.sort(r.choice(np.arange(1, n), size=min(n - 1, int(r.integers(1, 6))), replace=False))
        parts = np.split(perm, cuts)
        os_, ls_ = [], []
        for p in parts:
            o, l = oracle.attend_dense(q, K[p], V[p])
            os_.append(o)
            ls_.append(l)
        # an empty part (lse = -inf) must not change the merge
        os_.append(np.zeros(D))
        ls_.append(-np.inf)
        m, lm = oracle.merge(np.array(os_), np.array(ls_))
        np.testing.assert_allclose(m, full, rtol=0, atol=1e-12)
        assert abs(lm - lfull) < 1e-12


def test_merge_two_single_key_parts_closed_form():
    # two one-key parts: merge must equal sigma(delta) v1 + (1 - sigma(delta)) v2
    v1, v2 = np.array([1.0, -2.0, 0.5]), np.array([3.0, 1.0, -1.0])
    l1, l2 = 0.25, -1.75
    m, lm = oracle.merge(np.stack([v1, v2]), np.array([l1, l2]))
    s = 1.0 / (1.0 + math.exp(-(l1 - l2)))
    np.testing.assert_allclose(m, s * v1 + (1 - s) * v2, rtol=0, atol=1e-15)
    assert abs(lm - (l1 + math.log1p(math.exp(l2 - l1)))) < 1e-15


def test_brute_force_two_keys_integer_inputs():
    # D = 4, entries in {-2..2}: out = sigma(delta) v1 + (1 - sigma(delta)) v2, delta = s q.(k1 - k2)
    r = rng(5)
    for _ in range(200):
        q, k1, k2, v1, v2 = (r.integers(-2, 3, size=4).astype(np.float64) for _ in range(5))
        out, lse = oracle.attend_dense(q, np.stack([k1, k2]), np.stack([v1, v2]))
        s = 0.5
        delta = s * float(q @ (k1 - k2))
        sig = 1.0 / (1.0 + math.exp(-delta))
        np.testing.assert_allclose(out, sig * v1 + (1 - sig) * v2, rtol=0, atol=1e-14)
        a, b = s * float(q @ k1), s * float(q @ k2)
        assert abs(lse - (max(a, b) + math.log1p(math.exp(-abs(a - b))))) < 1e-14


def test_permuting_keys_changes_nothing():
    r = rng(6)
    q, K, V = r.standard_normal(64), r.standard_normal((50, 64)), r.standard_normal((50, 64))
    a, la = oracle.attend_dense(q, K, V)
    p = r.permutation(50)
    b, lb = oracle.attend_dense(q, K[p], V[p])
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-13)
    assert abs(la - lb) < 1e-12


def test_key_with_logit_larger_by_50_dominates():
    r = rng(7)
    D = 64
    q = r.standard_normal(D)
    q /= np.linalg.norm(q)
    K = r.standard_normal((20, D)) * 0.1
    V = r.standard_normal((20, D))
    # push key 5's logit 50 above every other one
    logits = K @ q / math.sqrt(D)
    K[5] += q * (logits.max() - logits[5] + 50.0) * math.sqrt(D)
    out, _ = oracle.attend_dense(q, K, V)
    np.testing.assert_allclose(out, V[5], rtol=0, atol=1e-12)


def test_shifting_all_keys_shifts_lse_only():
    r = rng(8)
    D = 64
    q, K, V, u = r.standard_normal(D), r.standard_normal((40, D)), r.standard_normal((40, D)), r.standard_normal(D)
    a, la = oracle.attend_dense(q, K, V)
    b, lb = oracle.attend_dense(q, K + u, V)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    assert abs((lb - la) - float(q @ u) / math.sqrt(D)) < 1e-12


def test_explicit_scale_argument():
    r = rng(9)
    q, K, V = r.standard_normal(16), r.standard_normal((9, 16)), r.standard_normal((9, 16))
    a, la = oracle.attend_dense(q, K, V, scale=0.3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(K)[None], torch.from_numpy(V)[None], scale=0.3)
    np.testing.assert_allclose(a, ref[0, 0].numpy(), rtol=0, atol=1e-13)


def test_paged_rejects_bad_inputs():
    w = wl.make_config(1)
    bt = w.block_table.copy()
    bt[0, 0] = w.num_pages  # out of range
    with pytest.raises(ValueError):
        oracle.attend_paged(w.q, w.k_pool, w.v_pool, bt, w.kv_lens)
    kl = w.kv_lens.copy()
    kl[1] = 0
    with pytest.raises(ValueError):
        oracle.attend_paged(w.q, w.k_pool, w.v_pool, w.block_table, kl)


# ------------------------------------------------------------- session chunk append (attend_rows)

def _session_chunk_case(seed, G, D, ctx, chunk):
    """One session request whose last `chunk` tokens are new rows (causal), and
    two other requests sharing its first pages; rows at positions ctx..ctx+chunk-1."""
    roots = [wl.Node(32, [wl.Node(ctx + chunk - 32), wl.Node(21)]), wl.Node(40)]
    w = wl.build_workload("chunk", roots, Hq=2 * G, Hkv=2, D=D, seed=seed)
    (match,) = np.nonzero(w.kv_lens == ctx + chunk)
    assert len(match) == 1
    b = int(match[0])
    rng = np.random.default_rng(seed)
    qr = to_bf16_bits(rng.normal(size=(chunk, w.Hq, w.D)))
    return w, b, qr


@pytest.mark.parametrize("G,D,ctx,chunk", [(1, 64, 37, 5), (4, 128, 64, 16), (8, 64, 100, 19), (2, 128, 32, 1)])
def test_attend_rows_matches_causal_sdpa(G, D, ctx, chunk):
    w, b, qr = _session_chunk_case(7 + G + D, G, D, ctx, chunk)
    pos = np.arange(ctx, ctx + chunk)
    out, lse = oracle.attend_rows(qr, np.full(chunk, b), pos, w.k_pool, w.v_pool, w.block_table)
    k, v = dense_gather(w, b)  # [Hkv][ctx+chunk][D]
    K = torch.from_numpy(k).repeat_interleave(G, dim=0)  # [Hq][n][D]
    V = torch.from_numpy(v).repeat_interleave(G, dim=0)
    q = torch.from_numpy(wl.bf16_bits_to_f32(qr).astype(np.float64)).permute(1, 0, 2)  # [Hq][C][D]
    n = ctx + chunk
    allowed = torch.arange(n)[None, :] <= torch.from_numpy(pos)[:, None]  # [C][n]: key t <= row position
    ref = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=allowed)  # [Hq][C][D]
    logits = torch.einsum("hcd,hnd->hcn", q, K) / math.sqrt(D)
    ref_lse = torch.logsumexp(logits.masked_fill(~allowed, float("-inf")), dim=-1)  # [Hq][C]
    np.testing.assert_allclose(out, ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse.permute(1, 0).numpy(), rtol=0, atol=1e-12)


def test_attend_rows_last_row_is_decode_and_context_order_does_not_matter():
    G, D, ctx, chunk = 4, 64, 96, 6
    w, b, qr = _session_chunk_case(99, G, D, ctx, chunk)
    pos = np.arange(ctx, ctx + chunk)
    out, lse = oracle.attend_rows(qr, np.full(chunk, b), pos, w.k_pool, w.v_pool, w.block_table)
    # the last row attends over the whole request: the decode attention of a
    # batch whose query for request b is that row
    qd = w.q.copy()
    qd[b] = qr[-1]
    do, dl = oracle.attend_paged(qd, w.k_pool, w.v_pool, w.block_table, w.kv_lens, queries=[b])
    np.testing.assert_allclose(out[-1], do[0], rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse[-1], dl[0], rtol=0, atol=1e-13)
    # swapping two full context pages of the request changes no row (every row
    # sees the whole context; attention does not depend on the order of keys)
    bt2 = w.block_table.copy()
    bt2[b, [1, 3]] = bt2[b, [3, 1]]
    o2, l2 = oracle.attend_rows(qr, np.full(chunk, b), pos, w.k_pool, w.v_pool, bt2)
    np.testing.assert_allclose(o2, out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l2, lse, rtol=0, atol=1e-13)
    # while a row earlier in the chunk sees fewer keys than the one after it
    assert np.abs(out[0] - out[1]).max() > 1e-6
