"""Pins for the float64 oracle against things other than itself: closed forms, the pages' worked
examples (tests/golden), textbook special cases, library routines, invariants and an
independently written dense formulation. CPU only."""
import json
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- rotary

def test_rope_single_pair_is_plane_rotation():
    # hd = 2: one pair with frequency base^0 = 1, so position p rotates by p radians. For one pair
    # the half-split form of the "2. RoPE" section (q*cos + rotate_half(q)*sin) and the adjacent-pair
    # form coincide: (x0, x1) -> (x0 cos p - x1 sin p, x0 sin p + x1 cos p).
    p = np.array([0, 1, 2, 7, 100, 4097], dtype=np.int32)
    x = np.zeros((len(p), 2, 2))
    x[:, 0, 0] = 1.0          # head 0: e0
    x[:, 1, 1] = 1.0          # head 1: e1
    y = oracle.rope(x, p)
    np.testing.assert_allclose(y[:, 0, 0], np.cos(p), atol=1e-15)
    np.testing.assert_allclose(y[:, 0, 1], np.sin(p), atol=1e-15)
    np.testing.assert_allclose(y[:, 1, 0], -np.sin(p), atol=1e-15)
    np.testing.assert_allclose(y[:, 1, 1], np.cos(p), atol=1e-15)


def test_rope_frequencies_base_10000_hd8():
    # inv_freq = 1 / 10000^(2i/8) for i = 0..3 is exactly 1, 1/10, 1/100, 1/1000 and pair i is
    # (x[2i], x[2i+1]).
    freqs = [1.0, 0.1, 0.01, 0.001]
    p = 37
    for i, f in enumerate(freqs):
        x = np.zeros((1, 1, 8))
        x[0, 0, 2 * i] = 1.0
        y = oracle.rope(x, np.array([p], dtype=np.int32))[0, 0]
        expect = np.zeros(8)
        expect[2 * i] = np.cos(p * f)
        expect[2 * i + 1] = np.sin(p * f)
        np.testing.assert_allclose(y, expect, atol=1e-13)


def test_rope_position_zero_is_identity_and_norm_preserved():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 3, 64))
    y0 = oracle.rope(x, np.zeros(6, dtype=np.int32))
    np.testing.assert_array_equal(y0, x)
    y = oracle.rope(x, rng.integers(0, 70000, 6).astype(np.int32))
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


@pytest.mark.parametrize("hd", [16, 64, 128])
def test_rope_relative_position_invariance(hd):
    # q_m . k_n depends only on m - n ("2. RoPE" section).
    rng = np.random.default_rng(hd)
    q = rng.standard_normal((1, 1, hd))
    k = rng.standard_normal((1, 1, hd))
    for m, n in [(5, 3), (100, 0), (2047, 1000)]:
        ref = None
        for delta in [0, 1, 17, 4096, 60000]:
            qm = oracle.rope(q, np.array([m + delta], dtype=np.int32))
            kn = oracle.rope(k, np.array([n + delta], dtype=np.int32))
            d = float(np.sum(qm * kn))
            if ref is None:
                ref = d
            assert abs(d - ref) < 1e-10 * max(1.0, abs(ref))


def test_paired_staggered_rope_equals_slot_rope_for_one_pair():
    # H = 2: the paired table gives head h of token t the phase 2t + h, and the interleave puts it
    # at slot 2t + h. So paired staggered RoPE followed by the interleave equals the interleave
    # followed by plain RoPE at the slot index.
    rng = np.random.default_rng(11)
    T, hd = 9, 32
    x = rng.standard_normal((T, 2, hd))
    a = oracle.interleave(oracle.rope(x, np.arange(T, dtype=np.int32), paired=True, stagger=True))
    b = oracle.rope(oracle.interleave(x), np.arange(2 * T, dtype=np.int32))
    np.testing.assert_allclose(a, b, atol=1e-12)


def test_paired_unstaggered_gives_both_heads_phase_2t():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((5, 4, 16))
    pos = np.arange(5, dtype=np.int32)
    a = oracle.rope(x, pos, paired=True, stagger=False)
    b = oracle.rope(x, 2 * pos)
    np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------------------- interleave

def test_interleave_worked_example():
    g = _gold("interleave_example.json")
    T, H = g["T"], g["H"]
    labels = {}
    x = np.zeros((T, H, 1))
    for h in range(H):
        for t in range(T):
            code = 100 * (h + 1) + (t + 1)
            x[t, h, 0] = code
            labels[code] = g["before"][h][t]
    y = oracle.interleave(x)  # [2T][H/2][1]
    got = [labels[int(c)] for c in y.reshape(-1)]
    assert got == g["after"]


def test_interleave_index_map_example():
    g = _gold("index_map_example.json")
    T, H = g["T"], g["H"]
    x = np.zeros((T, H, 1))
    for t in range(T):
        for h in range(H):
            x[t, h, 0] = 10 * t + h
    y = oracle.interleave(x)
    for e in g["map"]:
        assert y[e["slot"], e["head"], 0] == 10 * e["t"] + e["h"]


@pytest.mark.parametrize("T,H,d", [(1, 2, 1), (7, 6, 5), (33, 12, 64), (4, 32, 128)])
def test_interleave_is_a_view(T, H, d):
    # The explicit copy loop equals reinterpreting [T][H][d] as [2T][H/2][d] (the page's delayed
    # reshape), bit for bit; de-interleave inverts it.
    x = np.random.default_rng(T * H + d).standard_normal((T, H, d))
    y = oracle.interleave(x)
    np.testing.assert_array_equal(y, x.reshape(2 * T, H // 2, d))
    np.testing.assert_array_equal(oracle.deinterleave(y), x)


# ----------------------------------------------------------------------------- attention

def _dense_attention(q, k, v, cu, causal, window, scale):
    """Independent dense formulation: per document, a full score matrix, a boolean mask built from
    a lower-triangular matrix and a band, and a row softmax."""
    S, H, hd = q.shape
    Hkv = k.shape[1]
    G = H // Hkv
    o = np.zeros_like(q)
    lse = np.zeros((S, H))
    for b in range(len(cu) - 1):
        lo, hi = cu[b], cu[b + 1]
        n = hi - lo
        if n == 0:
            continue
        mask = np.ones((n, n), dtype=bool)
        if causal:
            mask &= np.tril(np.ones((n, n), dtype=bool))
        if window > 0:
            ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
            mask &= (ii - jj) < window
        for h in range(H):
            Q = q[lo:hi, h, :]
            K = k[lo:hi, h // G, :]
            V = v[lo:hi, h // G, :]
            Sm = np.where(mask, (Q @ K.T) * scale, -np.inf)
            mx = Sm.max(axis=1, keepdims=True)
            P = np.exp(Sm - mx)
            den = P.sum(axis=1, keepdims=True)
            o[lo:hi, h, :] = (P / den) @ V
            lse[lo:hi, h] = mx[:, 0] + np.log(den[:, 0])
    return o, lse


CASES = [
    # doc lens, H, Hkv, hd, causal, window
    ((5,), 1, 1, 4, True, 0),
    ((16,), 4, 2, 8, True, 0),
    ((3, 1, 9, 4), 2, 2, 8, True, 3),
    ((7, 0, 6), 4, 1, 6, True, 1),
    ((11, 5), 2, 2, 4, False, 0),
    ((16, 2), 4, 4, 8, True, 100),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("integer_valued", [False, True])
def test_loops_match_dense_formulation(case, integer_valued):
    lens, H, Hkv, hd, causal, window = case
    rng = np.random.default_rng(len(lens) * 100 + H * 10 + hd)
    S = sum(lens)
    if integer_valued:
        q = rng.integers(-3, 4, (S, H, hd)).astype(np.float64)
        k = rng.integers(-3, 4, (S, Hkv, hd)).astype(np.float64)
        v = rng.integers(-3, 4, (S, Hkv, hd)).astype(np.float64)
    else:
        q, k, v = (rng.standard_normal((S, n, hd)) for n in (H, Hkv, Hkv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    scale = 1.0 / np.sqrt(hd)
    o, lse = oracle.attention_slots(q, k, v, cu, causal, window, scale)
    od, lsed = _dense_attention(q, k, v, cu, causal, window, scale)
    np.testing.assert_allclose(o, od, atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lsed, atol=1e-12, rtol=0)


@pytest.mark.parametrize("case", CASES[:4])
def test_paired_matches_dense_on_reshaped_sequence(case):
    lens, H, Hkv, hd, causal, window = case
    H, Hkv = 2 * H, 2 * Hkv
    rng = np.random.default_rng(7 + H)
    T = sum(lens)
    q, k, v = (rng.standard_normal((T, n, hd)) for n in (H, Hkv, Hkv))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse = oracle.attn_fwd(q, k, v, cu, causal, window, paired=True)
    od, lsed = _dense_attention(q.reshape(2 * T, H // 2, hd), k.reshape(2 * T, Hkv // 2, hd),
                                v.reshape(2 * T, Hkv // 2, hd), 2 * cu.astype(np.int64), causal,
                                window, 1.0 / np.sqrt(hd))
    np.testing.assert_allclose(o, od.reshape(T, H, hd), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, lsed.reshape(T, H), atol=1e-12, rtol=0)


def test_matches_torch_sdpa_float64():
    torch = pytest.importorskip("torch")
    F = torch.nn.functional
    rng = np.random.default_rng(3)
    S, H, hd = 24, 4, 16
    q, k, v = (rng.standard_normal((S, H, hd)) for _ in range(3))
    for window in (0, 5):
        i = np.arange(S)[:, None]
        j = np.arange(S)[None, :]
        allowed = (j <= i) & ((i - j < window) if window > 0 else True)
        tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2)[None] for a in (q, k, v))
        ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(allowed))
        ref = ref[0].permute(1, 0, 2).numpy()
        o, _ = oracle.attention_slots(q, k, v, np.array([0, S]), True, window)
        np.testing.assert_allclose(o, ref, atol=1e-12, rtol=0)


def test_softmax_rows_sum_to_one():
    # V = 1 everywhere: each output is the sum of the row's softmax weights.
    rng = np.random.default_rng(4)
    S, H, hd = 40, 4, 8
    q = rng.standard_normal((S, H, hd)) * 3
    k = rng.standard_normal((S, 2, hd)) * 3
    v = np.ones((S, 2, hd))
    for window in (0, 7):
        o, _ = oracle.attention_slots(q, k, v, np.array([0, 13, 40]), True, window)
        assert np.max(np.abs(o - 1.0)) < 1e-12


def test_lse_is_log_of_visible_count_when_keys_are_zero():
    S, H, hd = 30, 2, 4
    rng = np.random.default_rng(8)
    q = rng.standard_normal((S, H, hd))
    k = np.zeros((S, H, hd))
    v = rng.standard_normal((S, H, hd))
    cu = [0, 11, 30]
    for window in (0, 4):
        _, lse = oracle.attention_slots(q, k, v, np.array(cu), True, window)
        for b in range(2):
            for i in range(cu[b], cu[b + 1]):
                n = i - cu[b] + 1
                if window > 0:
                    n = min(n, window)
                np.testing.assert_allclose(lse[i], np.log(n), atol=1e-14)


def test_tril_examples():
    # Single head, K = 0 (equal logits), V one-hot by position: the output row is uniform over the
    # visible keys, so its support is the mask row.
    g = _gold("tril_examples.json")
    for n_str, mask in g["masks"].items():
        n = int(n_str)
        q = np.random.default_rng(n).standard_normal((n, 1, n))
        k = np.zeros((n, 1, n))
        v = np.eye(n).reshape(n, 1, n)
        o, _ = oracle.attention_slots(q, k, v, np.array([0, n]), True, 0)
        support = (o[:, 0, :] > 0).astype(int)
        assert support.tolist() == mask
        np.testing.assert_allclose(o[:, 0, :].sum(axis=1), 1.0, atol=1e-14)


def test_pages_paired_mask_example():
    # Paired, two heads, K = 0 and V one-hot over (head, position): the query row at position 4 is
    # uniform over exactly the keys the page says it sees.
    g = _gold("mask_example.json")
    T, H = g["T"], g["H"]
    hd = H * T
    q = np.random.default_rng(1).standard_normal((T, H, hd))
    k = np.zeros((T, H, hd))
    v = np.zeros((T, H, hd))
    for h in range(H):
        for t in range(T):
            v[t, h, h * T + t] = 1.0
    o, _ = oracle.attn_fwd(q, k, v, np.array([0, T], dtype=np.int32), causal=True, paired=True)
    t = g["query_position"] - 1
    for qh in range(H):
        vis = g["visible"][f"head{qh + 1}"]
        expect = np.zeros(hd)
        n = sum(len(p) for p in vis.values())
        for kh_name, positions in vis.items():
            kh = int(kh_name[-1]) - 1
            for p in positions:
                expect[kh * T + (p - 1)] = 1.0 / n
        np.testing.assert_allclose(o[t, qh], expect, atol=1e-15)


def test_window_covering_everything_equals_no_window():
    rng = np.random.default_rng(9)
    q, k, v = (rng.standard_normal((20, 2, 8)) for _ in range(3))
    cu = np.array([0, 8, 20])
    a = oracle.attention_slots(q, k, v, cu, True, 0)
    b = oracle.attention_slots(q, k, v, cu, True, 12)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_window_one_returns_own_value():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((12, 4, 8))
    k = rng.standard_normal((12, 2, 8))
    v = rng.standard_normal((12, 2, 8))
    o, lse = oracle.attention_slots(q, k, v, np.array([0, 5, 12]), True, 1)
    for h in range(4):
        np.testing.assert_allclose(o[:, h, :], v[:, h // 2, :], atol=1e-15)
        np.testing.assert_allclose(lse[:, h], np.sum(q[:, h] * k[:, h // 2], axis=-1) / np.sqrt(8),
                                   atol=1e-13)


def test_gqa_equals_mha_with_repeated_kv():
    # "4. GQA & FlashAttention": K/V heads repeated with repeat_interleave(H/Hkv) give the same
    # result as grouped sharing.
    rng = np.random.default_rng(12)
    q = rng.standard_normal((18, 8, 8))
    k = rng.standard_normal((18, 2, 8))
    v = rng.standard_normal((18, 2, 8))
    cu = np.array([0, 6, 18])
    a = oracle.attention_slots(q, k, v, cu, True, 4)
    b = oracle.attention_slots(q, np.repeat(k, 4, axis=1), np.repeat(v, 4, axis=1), cu, True, 4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_global_and_per_document_positions_agree():
    rng = np.random.default_rng(13)
    lens = [5, 9, 3]
    T, H, hd = sum(lens), 4, 16
    q, k, v = (rng.standard_normal((T, H, hd)) for _ in range(3))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    glob = np.arange(T, dtype=np.int32)
    local = np.concatenate([np.arange(n) for n in lens]).astype(np.int32)
    for paired in (False, True):
        outs = []
        for pos in (glob, local):
            qr = oracle.rope(q, pos, paired=paired, stagger=paired)
            kr = oracle.rope(k, pos, paired=paired, stagger=paired)
            outs.append(oracle.attn_fwd(qr, kr, v, cu, True, 3, paired=paired))
        np.testing.assert_allclose(outs[0][0], outs[1][0], atol=1e-10)
        np.testing.assert_allclose(outs[0][1], outs[1][1], atol=1e-10)


@pytest.mark.parametrize("paired", [False, True])
def test_rows_variant_equals_full(paired):
    rng = np.random.default_rng(14)
    lens = [13, 1, 30, 6]
    T, H, Hkv, hd = sum(lens), 4, 2, 8
    q = rng.standard_normal((T, H, hd))
    k = rng.standard_normal((T, Hkv, hd))
    v = rng.standard_normal((T, Hkv, hd))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, lse = oracle.attn_fwd(q, k, v, cu, True, 5, paired=paired)
    rows = rng.choice(T * H, 40, replace=False)
    orow, lrow = oracle.attn_rows(q, k, v, cu, rows, True, 5, paired=paired)
    np.testing.assert_array_equal(orow, o.reshape(T * H, hd)[rows])
    np.testing.assert_array_equal(lrow, lse.reshape(-1)[rows])


def test_oracle_rejects_bad_arguments():
    q = np.zeros((4, 3, 8))
    with pytest.raises(ValueError):
        oracle.attn_fwd(q, q, q, np.array([0, 4], dtype=np.int32), paired=True)  # odd heads
    with pytest.raises(ValueError):
        oracle.attention_slots(q, q, q, np.array([0, 3, 2]))  # decreasing cu


# ----------------------------------------------------------------------------- bf16 storage

def test_round_bf16_ties_and_neighbours():
    # bfloat16 keeps 8 significant bits: the neighbours of 1 are 1 - 2^-8 and 1 + 2^-7.
    cases = [
        (1.0, 1.0),
        (1 + 2.0 ** -8, 1.0),                      # tie -> even (1.0)
        (1 + 3 * 2.0 ** -8, 1 + 2.0 ** -6),        # tie -> even (mantissa ...10)
        (1 + 2.0 ** -8 + 2.0 ** -30, 1 + 2.0 ** -7),
        (-(1 + 2.0 ** -8 + 2.0 ** -30), -(1 + 2.0 ** -7)),
        (3.4e38, np.inf),                          # past the midpoint above the largest bf16
        (0.0, 0.0),
    ]
    got = oracle.round_bf16(np.array([c[0] for c in cases]))
    assert got.tolist() == [c[1] for c in cases]


def test_round_bf16_matches_torch_on_float32_values():
    torch = pytest.importorskip("torch")
    x = np.random.default_rng(21).standard_normal(100000).astype(np.float32) * 10.0
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(x.astype(np.float64)), ref)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("paired,stagger", [(False, False), (True, False), (True, True)])
def test_rope_stored_is_the_rotation_rounded_once(dtype, paired, stagger):
    # The stored RoPE output is a value of the buffer's dtype within half a unit in its last
    # place of the unrounded rotation (float32 table values), and position 0 (phase 0: cos 1,
    # sin 0) leaves an input that is already in the dtype unchanged.
    torch = pytest.importorskip("torch")
    tdt, bits = (torch.bfloat16, 8) if dtype == "bf16" else (torch.float32, 24)
    rng = np.random.default_rng(31)
    x = torch.from_numpy(rng.standard_normal((64, 4, 32)).astype(np.float32)).to(tdt)
    x = x.to(torch.float64).numpy()
    pos = rng.integers(0, 5000, 64).astype(np.int32)
    pos[:4] = 0
    y = oracle.rope_stored(x, pos, dtype, paired, stagger)
    # values of the dtype
    np.testing.assert_array_equal(torch.from_numpy(y).to(tdt).to(torch.float64).numpy(), y)
    # within half an ulp of the unrounded rotation
    u = oracle.rope(x, pos, paired, stagger, table_f32=True)
    half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(u), 2.0 ** -120))) - bits)
    assert np.all(np.abs(y - u) <= half_ulp)
    # phase 0: tokens at position 0 (every head unless the odd heads are staggered)
    heads = slice(None) if not stagger else slice(0, None, 2)
    np.testing.assert_array_equal(y[:4, heads], x[:4, heads])


def test_float32_tables_only_perturb_by_float32_rounding():
    # Rounding cos / sin to float32 changes each rotated element by at most
    # 2^-24 (|x_2i| + |x_2i+1|) (one float32 half-ulp on each factor of magnitude <= 1).
    rng = np.random.default_rng(22)
    x = rng.standard_normal((200, 4, 64))
    pos = rng.integers(0, 70000, 200).astype(np.int32)
    for paired in (False, True):
        a = oracle.rope(x, pos, paired, paired)
        b = oracle.rope(x, pos, paired, paired, table_f32=True)
        pair = np.abs(x.reshape(200, 4, 32, 2)).sum(-1).repeat(2, axis=-1)
        assert np.all(np.abs(a - b) <= 2.0 ** -24 * pair * 1.0001)
        assert np.any(a != b)


# ------------------------------------------------------------------------------ QK RMS-norm
# "Training an LLM from scratch (part 2)", section "1. RMSNorm": y = x / sqrt(E[x^2] + eps) * gamma
# over the last axis; the paired-head page's rotary kernel applies it to each head row of q and k.

def test_rms_norm_matches_torch_float64():
    import torch

    rng = np.random.default_rng(11)
    x = rng.standard_normal((7, 5, 64)) * rng.uniform(0.1, 9.0, (7, 5, 1))
    g = rng.uniform(0.5, 2.0, 64)
    for gamma, eps in ((None, 1e-6), (g, 1e-6), (g, 0.3)):
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (64,),
                                           None if gamma is None else torch.from_numpy(gamma), eps)
        np.testing.assert_allclose(oracle.rms_norm(x, gamma, eps), ref.numpy(), rtol=1e-14, atol=0)


def test_rms_norm_gives_unit_rms_rows_and_keeps_direction():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((6, 4, 32)) * np.arange(1, 25).reshape(6, 4, 1)  # rows of every scale
    y = oracle.rms_norm(x, eps=0.0)
    np.testing.assert_allclose(np.sqrt((y ** 2).mean(-1)), 1.0, rtol=1e-14)  # each row on its own
    cos = (x * y).sum(-1) / np.linalg.norm(x, axis=-1) / np.linalg.norm(y, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-14)
    # with eps the mean square is ms / (ms + eps)
    ms = (x ** 2).mean(-1)
    y = oracle.rms_norm(x, eps=0.5)
    np.testing.assert_allclose((y ** 2).mean(-1), ms / (ms + 0.5), rtol=1e-13)


def test_rms_norm_scale_and_sign_invariance_and_weights():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((3, 2, 16))
    g = rng.uniform(-2.0, 2.0, 16)
    base = oracle.rms_norm(x, eps=0.0)
    np.testing.assert_allclose(oracle.rms_norm(37.5 * x, eps=0.0), base, rtol=1e-14)
    np.testing.assert_allclose(oracle.rms_norm(-x, eps=0.0), -base, rtol=1e-14)
    np.testing.assert_allclose(oracle.rms_norm(x, g, eps=0.0), base * g, rtol=1e-14)
    # a constant row c becomes c / sqrt(c^2 + eps)
    c = np.full((1, 1, 8), -3.0)
    np.testing.assert_allclose(oracle.rms_norm(c, eps=7.0), -3.0 / 4.0, rtol=1e-15)


def test_norm_then_rope_keeps_the_normalised_length():
    # the rotation is orthogonal: after the norm each head row has length sqrt(hd) (eps = 0)
    rng = np.random.default_rng(14)
    x = rng.standard_normal((9, 6, 128)) * 5.0
    pos = rng.integers(0, 1000, 9).astype(np.int32)
    y = oracle.rope(oracle.rms_norm(x, eps=0.0), pos, paired=True, stagger=True)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.sqrt(128.0), rtol=1e-13)


def test_norm_rope_stored_skips_rotation_outside_the_table():
    rng = np.random.default_rng(15)
    x = synth_bf16(rng.standard_normal((4, 2, 16)))
    pos = np.array([0, -1, 5, 99], dtype=np.int32)
    y = oracle.norm_rope_stored(x, pos, "bf16", eps=1e-6, tab_rows=10)
    n = oracle.round_bf16(oracle.rms_norm(x, eps=1e-6))
    np.testing.assert_array_equal(y[1], n[1])   # position -1: normalised, not rotated
    np.testing.assert_array_equal(y[3], n[3])   # position 99 >= 10 rows
    np.testing.assert_array_equal(y[0], n[0])   # position 0: rotation by 0
    assert not np.array_equal(y[2], n[2])       # position 5: rotated


def synth_bf16(x):
    return oracle.round_bf16(x)


# ------------------------------------------------------------------------------ value embedding
# "modded-nanogpt Paired Head Attention record", section "3. the paired branch of the forward pass":
# v = v + aux_v (reshaped to v's shape on the paired path) before the varlen attention call.

def test_add_stored_matches_torch_bf16_and_f32_addition():
    import torch

    rng = np.random.default_rng(21)
    a = torch.from_numpy(rng.standard_normal(20000).astype(np.float32) * 3).to(torch.bfloat16)
    b = torch.from_numpy(rng.standard_normal(20000).astype(np.float32)).to(torch.bfloat16)
    got = oracle.add_stored(a.double().numpy(), b.double().numpy(), "bf16")
    np.testing.assert_array_equal(got, (a + b).double().numpy())
    af, bf = a.float() * 1.7, b.float() / 3
    got = oracle.add_stored(af.double().numpy(), bf.double().numpy(), "f32")
    np.testing.assert_array_equal(got, (af + bf).double().numpy())


def test_value_embedding_shifts_output_by_its_weighted_mean():
    # attention is linear in v: O(q, k, v + aux) = O(q, k, v) + O(q, k, aux) (float64, no rounding)
    rng = np.random.default_rng(22)
    q, k, v, a = (rng.standard_normal((50, 4, 8)) for _ in range(4))
    cu = np.array([0, 20, 50], dtype=np.int32)
    o1, _ = oracle.attn_fwd(q, k, v + a, cu, True, 7, True)
    o2, _ = oracle.attn_fwd(q, k, v, cu, True, 7, True)
    o3, _ = oracle.attn_fwd(q, k, a, cu, True, 7, True)
    np.testing.assert_allclose(o1, o2 + o3, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------ backward
# Gradients of the attention (and of RoPE) with respect to their inputs, for an upstream gradient
# dO; pinned to finite differences of the forward oracle and to torch's float64 autograd.

def _loss_grad_fd(f, x, g, eps=1e-6):
    """Central differences of <f(x), g> with respect to every element of x."""
    out = np.empty_like(x)
    flat, of = x.reshape(-1), out.reshape(-1)
    for n in range(flat.size):
        old = flat[n]
        flat[n] = old + eps
        up = float((f(x) * g).sum())
        flat[n] = old - eps
        dn = float((f(x) * g).sum())
        flat[n] = old
        of[n] = (up - dn) / (2 * eps)
    return out


@pytest.mark.parametrize("case", [
    # T per doc, H, Hkv, hd, causal, window, paired
    ((5, 7), 2, 2, 4, True, 0, False),
    ((6, 3), 4, 2, 4, True, 2, False),
    ((4, 5), 4, 2, 4, True, 3, True),
    ((6,), 2, 1, 4, False, 0, False),
])
def test_attention_backward_matches_finite_differences(case):
    lens, H, Hkv, hd, causal, window, paired = case
    rng = np.random.default_rng(sum(lens) + H + window)
    T = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q, k, v, g = (rng.standard_normal((T, h, hd)) for h in (H, Hkv, Hkv, H))
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, cu, causal, window, paired)
    fwd = lambda qq, kk, vv: oracle.attn_fwd(qq, kk, vv, cu, causal, window, paired)[0]
    np.testing.assert_allclose(dq, _loss_grad_fd(lambda x: fwd(x, k, v), q.copy(), g), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _loss_grad_fd(lambda x: fwd(q, x, v), k.copy(), g), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _loss_grad_fd(lambda x: fwd(q, k, x), v.copy(), g), rtol=1e-6, atol=1e-8)


def test_attention_backward_matches_torch_autograd_float64():
    import torch

    rng = np.random.default_rng(31)
    T, H, Hkv, hd, window = 40, 4, 2, 8, 9
    cu = np.array([0, 17, 40], dtype=np.int32)
    q, k, v, g = (rng.standard_normal((T, h, hd)) for h in (H, Hkv, Hkv, H))
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, cu, True, window, False)
    tq, tk, tv = (torch.tensor(x, requires_grad=True) for x in (q, k, v))
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    doc = torch.from_numpy(np.searchsorted(cu[1:], np.arange(T), side="right"))
    mask = (doc[:, None] == doc[None, :]) & (j <= i) & (i - j < window)
    kk = tk.repeat_interleave(H // Hkv, dim=1)
    vv = tv.repeat_interleave(H // Hkv, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(
        tq.transpose(0, 1), kk.transpose(0, 1), vv.transpose(0, 1), attn_mask=mask).transpose(0, 1)
    (o * torch.from_numpy(g)).sum().backward()
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dk, tk.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dv, tv.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_paired_backward_equals_standard_backward_on_interleaved_tensors():
    rng = np.random.default_rng(32)
    lens, H, Hkv, hd = (9, 6), 4, 2, 4
    T = sum(lens)
    cu = np.array([0, 9, 15], dtype=np.int32)
    q, k, v, g = (rng.standard_normal((T, h, hd)) for h in (H, Hkv, Hkv, H))
    dq, dk, dv = oracle.attn_bwd(q, k, v, g, cu, True, 5, True)
    il = oracle.interleave
    dqs, dks, dvs = oracle.attn_bwd(il(q), il(k), il(v), il(g), 2 * cu, True, 5, False)
    np.testing.assert_array_equal(dq, oracle.deinterleave(dqs))
    np.testing.assert_array_equal(dk, oracle.deinterleave(dks))
    np.testing.assert_array_equal(dv, oracle.deinterleave(dvs))


@pytest.mark.parametrize("paired,stagger", [(False, False), (True, True)])
def test_rope_backward_is_adjoint_and_inverse(paired, stagger):
    rng = np.random.default_rng(33)
    x, y = rng.standard_normal((2, 7, 6, 16))
    pos = rng.integers(0, 3000, 7).astype(np.int32)
    rx = oracle.rope(x, pos, paired, stagger)
    bty = oracle.rope_bwd(y, pos, paired, stagger)
    assert abs(float((rx * y).sum() - (x * bty).sum())) < 1e-11   # <R x, y> = <x, R^T y>
    np.testing.assert_allclose(oracle.rope_bwd(rx, pos, paired, stagger), x, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------------- e4m3 (FP8)
# The FP8 path consumes e4m3 codes with per-tensor float32 scales ("modded-nanogpt Paired Head
# Attention record", section "5. interactions with other mechanisms": the packed FP8 QKV
# projection). The oracle's decode and encode are pinned to torch's float8_e4m3fn (an independent
# implementation of the same OCP format), to closed-form codes, and to invariants of the scales.

def test_decode_e4m3_all_codes_match_torch():
    import torch

    codes = np.arange(256, dtype=np.uint8)
    got = oracle.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.array_equal(np.signbit(got[ok]), np.signbit(ref[ok]))


def test_decode_e4m3_closed_forms():
    cases = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
             0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0}
    got = oracle.decode_e4m3(np.array(list(cases), dtype=np.uint8))
    np.testing.assert_array_equal(got, np.array(list(cases.values())))
    assert np.isnan(oracle.decode_e4m3(np.array([0x7F, 0xFF], dtype=np.uint8))).all()


def test_encode_e4m3_matches_torch_on_float32_values():
    import torch

    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(50000) * 100.0,                 # normals, some past 448
        rng.standard_normal(20000) * 2.0 ** -8,             # subnormal range
        rng.uniform(440.0, 500.0, 5000),                    # around the largest finite value
    ]).astype(np.float32)
    # exact ties: midpoints between neighbouring finite codes (both even and odd lower codes)
    vals = oracle.decode_e4m3(np.arange(0, 126, dtype=np.uint8))
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    x = np.concatenate([x, mids, -mids, np.float32([464.0, -464.0, 0.0, -0.0])])
    got = oracle.encode_e4m3(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_encode_e4m3_round_trips_every_finite_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    assert np.array_equal(oracle.encode_e4m3(oracle.decode_e4m3(codes)), codes)


def test_attn_fwd_fp8_scales_enter_as_the_definition_says():
    rng = np.random.default_rng(9)
    T, H, hd = 40, 2, 16
    q8, k8, v8 = (oracle.encode_e4m3(rng.standard_normal((T, H, hd)) * 3.0) for _ in range(3))
    cu = np.array([0, 17, 40], dtype=np.int32)
    o1, l1 = oracle.attn_fwd_fp8(q8, k8, v8, 1.0, 1.0, 1.0, cu, True, 5, False, 0.25)
    # v's scale multiplies O and leaves the LSE alone
    o2, l2 = oracle.attn_fwd_fp8(q8, k8, v8, 1.0, 1.0, 2.5, cu, True, 5, False, 0.25)
    np.testing.assert_allclose(o2, 2.5 * o1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(l2, l1, rtol=0, atol=1e-13)
    # q's and k's scales multiply the logits: the same as folding them into the softmax scale
    o3, l3 = oracle.attn_fwd_fp8(q8, k8, v8, 0.5, 3.0, 1.0, cu, True, 5, False, 0.25)
    o4, l4 = oracle.attn_fwd(oracle.decode_e4m3(q8), oracle.decode_e4m3(k8),
                             oracle.decode_e4m3(v8), cu, True, 5, False, 0.25 * 1.5)
    np.testing.assert_allclose(o3, o4, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l3, l4, rtol=1e-12, atol=1e-12)
    # and with unit scales the values are the decoded codes themselves
    o5, l5 = oracle.attn_fwd(oracle.decode_e4m3(q8), oracle.decode_e4m3(k8),
                             oracle.decode_e4m3(v8), cu, True, 5, False, 0.25)
    np.testing.assert_array_equal(o1, o5)
    np.testing.assert_array_equal(l1, l5)
