"""Pins for the CPU oracle: each check ties a piece of the oracle to something other than itself
(closed forms, brute force, library routines, invariants), so that a dropped term, a wrong sign or
index, or a transposed operand in the oracle fails here.  No GPU is needed.

Passages: "Qwen3.8-Flash-Next architecture" (flozi.net), section "Der Weg eines Tokens durch das
Modell", item 2 (pooling of four keys, RoPE after pooling, four indexer query heads on one key
head, 512 blocks = 2048 tokens plus the incomplete last block, attention over the selected tokens
with GQA).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------------- helpers
def np_bf16_rne(x: np.ndarray) -> np.ndarray:
    """Independent double -> bf16 rounding for the normal range: round the float64 bit pattern to
    8 significant bits with an integer add (ties to even), then drop to the bf16 bit pattern."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    b = x.view(np.uint64)
    lsb = (b >> np.uint64(45)) & np.uint64(1)
    b2 = (b + np.uint64((1 << 44) - 1) + lsb) & ~np.uint64((1 << 45) - 1)
    y = b2.view(np.float64).astype(np.float32)
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def rand_bits(rng, shape, scale=1.0):
    return np_bf16_rne(rng.standard_normal(shape) * scale)


def f64(bits):
    return O.bf16_to_f64(bits)


def ulp_bf16(x):
    """Spacing of bf16 values around |x| (normal range)."""
    x = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -120)
    return 2.0 ** (np.floor(np.log2(x)) - 7)


# ----------------------------------------------------------------------------------- bf16
def test_bf16_rounding_matches_integer_rne():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200000) * np.exp2(rng.integers(-100, 100, 200000))
    assert np.array_equal(O.bf16_round(x), np_bf16_rne(x))


def test_bf16_rounding_exact_ties_go_to_even():
    rng = np.random.default_rng(1)
    base = f64(rand_bits(rng, 5000))
    half = ulp_bf16(base) / 2
    ties = base + half                     # exactly half-way between two bf16 values
    got = f64(O.bf16_round(ties))
    lo, hi = base, base + 2 * half
    lo_bits = np_bf16_rne(lo)
    expect = np.where((lo_bits & 1) == 0, lo, hi)
    # when |base| sits at a binade edge the neighbour spacing differs; skip those
    ok = np.abs(np.log2(np.abs(base)) % 1) > 1e-9
    assert np.array_equal(got[ok], expect[ok])


def test_bf16_rounding_matches_torch_for_float32_values():
    rng = np.random.default_rng(2)
    f = (rng.standard_normal(100000) * 3).astype(np.float32)
    t = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_round(f.astype(np.float64)), t)


def test_bf16_special_values():
    vals = np.array([0.0, -0.0, np.inf, -np.inf, 3.5e38, -3.5e38, 1e-45, 2.0 ** -133, 2.0 ** -134 * 1.5])
    got = O.bf16_round(vals)
    assert got[0] == 0x0000 and got[1] == 0x8000
    assert got[2] == 0x7F80 and got[3] == 0xFF80
    assert got[4] == 0x7F80 and got[5] == 0xFF80     # above the largest finite bf16 after rounding
    assert got[7] == 0x0001                          # smallest subnormal
    assert got[8] == 0x0002 or got[8] == 0x0001
    assert O.bf16_round(np.array([np.nan]))[0] & 0x7F80 == 0x7F80


# ----------------------------------------------------------------------------------- pooling
@pytest.mark.parametrize("L", [4, 37, 1024])
def test_pool_is_mean_of_four(L):
    rng = np.random.default_rng(L)
    ki = rand_bits(rng, (2, L, 64), 1 / 8)
    kp = O.pool_block_keys(ki, blk=4)
    nb = L // 4
    assert kp.shape == (2, nb, 64)
    expect = np_bf16_rne(f64(ki[:, : nb * 4]).reshape(2, nb, 4, 64).mean(axis=2))
    assert np.array_equal(kp, expect)


def test_pool_block_size_is_a_parameter():
    rng = np.random.default_rng(3)
    ki = rand_bits(rng, (1, 48, 8))
    kp = O.pool_block_keys(ki, blk=8)
    expect = np_bf16_rne(f64(ki).reshape(1, 6, 8, 8).mean(axis=2))
    assert np.array_equal(kp, expect)


# ----------------------------------------------------------------------------------- RoPE
def test_rope_position_zero_is_identity():
    rng = np.random.default_rng(4)
    ki = rand_bits(rng, (1, 64, 64), 1 / 8)
    a = O.pool_block_keys(ki, rope_theta=10000.0, pos0=0)
    b = O.pool_block_keys(ki, rope_theta=0.0)
    assert np.array_equal(a[:, 0], b[:, 0])
    x = rand_bits(rng, (5, 4, 64))
    assert np.array_equal(O.rope_rows(x, np.zeros(5), 10000.0), x)


def test_rope_basis_vectors_follow_half_split_closed_form():
    Di, theta = 64, 10000.0
    pos = np.array([0, 1, 7, 123, 4095, 262143], dtype=np.int64)
    for i in [0, 1, 5, 31]:
        x = np.zeros((pos.size, 1, Di), dtype=np.uint16)
        x[:, 0, i] = 0x3F80                      # 1.0
        y = f64(O.rope_rows(x, pos, theta))[:, 0]
        ang = pos * theta ** (-2.0 * i / Di)
        # component i carries cos, component i + Di/2 carries sin; nothing else moves
        assert np.all(np.abs(y[:, i] - np.cos(ang)) <= ulp_bf16(np.cos(ang)) / 2 + 1e-30)
        assert np.all(np.abs(y[:, i + Di // 2] - np.sin(ang)) <= ulp_bf16(np.sin(ang)) / 2 + 1e-30)
        mask = np.ones(Di, bool)
        mask[[i, i + Di // 2]] = False
        assert np.all(y[:, mask] == 0)


def test_rope_keys_rotate_at_block_start_complex_form():
    """Pooled key b is the mean rotated at pos0 + 4b, written here as a complex multiply."""
    rng = np.random.default_rng(5)
    Di, theta, pos0 = 64, 500000.0, 1000
    ki = rand_bits(rng, (1, 40, Di), 1 / 8)
    kp = f64(O.pool_block_keys(ki, rope_theta=theta, pos0=pos0))[0]
    m = f64(ki).reshape(10, 4, Di).mean(axis=1)
    z = m[:, : Di // 2] + 1j * m[:, Di // 2:]
    freq = theta ** (-2.0 * np.arange(Di // 2) / Di)
    pos = pos0 + 4 * np.arange(10)
    zr = z * np.exp(1j * pos[:, None] * freq[None, :])
    expect = np.concatenate([zr.real, zr.imag], axis=1)
    assert np.all(np.abs(kp - expect) <= ulp_bf16(expect) / 2 * (1 + 1e-9) + 1e-30)


# ---- YaRN-scaled RoPE ("YaRN: Efficient Context Window Extension of Large Language Models",
# Peng et al. 2023, sections 3.2 and 3.4).  Pinned by the properties that define it rather than by
# its formula: pairs that turn many times over the original context keep their frequency, pairs
# that turn less than once are position-interpolated by the factor, the ramp in between is
# monotone, the magnitude factor scales norms, and relative-position dependence survives.
YARN = dict(factor=8.0, orig_ctx=4096, alpha=1.0, beta=32.0, mscale=1.0)


def _yarn_pair_classes(Di=64, theta=10000.0, orig_ctx=4096):
    f = theta ** (-2.0 * np.arange(Di // 2) / Di)
    turns = orig_ctx * f / (2 * math.pi)
    return np.nonzero(turns > 32.0)[0], np.nonzero(turns < 1.0)[0]


def test_yarn_factor_one_is_plain_rope():
    rng = np.random.default_rng(31)
    x = rand_bits(rng, (6, 2, 64))
    pos = np.array([0, 3, 77, 4096, 100000, 1048575])
    assert np.array_equal(O.rope_rows(x, pos, 10000.0, yarn=dict(factor=1.0, orig_ctx=4096)),
                          O.rope_rows(x, pos, 10000.0))
    ki = rand_bits(rng, (1, 64, 64), 1 / 8)
    assert np.array_equal(O.pool_block_keys(ki, rope_theta=10000.0, pos0=40, yarn=dict(factor=1.0, orig_ctx=4096)),
                          O.pool_block_keys(ki, rope_theta=10000.0, pos0=40))


def test_yarn_keeps_fast_pairs_and_interpolates_slow_pairs():
    """A fast pair rotates exactly as plain RoPE; a slow pair at position p rotates as plain RoPE at
    position p / factor (position interpolation), bit for bit."""
    rng = np.random.default_rng(32)
    Di, theta = 64, 10000.0
    fast, slow = _yarn_pair_classes(Di, theta, YARN["orig_ctx"])
    assert len(fast) >= 8 and len(slow) >= 6
    x = rand_bits(rng, (4, 3, Di))
    pos = np.array([8, 4096, 65536, 1048568])          # multiples of the factor
    y = O.rope_rows(x, pos, theta, yarn=YARN)
    plain = O.rope_rows(x, pos, theta)
    interp = O.rope_rows(x, pos // 8, theta)
    for i in fast:
        assert np.array_equal(y[..., i], plain[..., i]) and np.array_equal(y[..., i + Di // 2], plain[..., i + Di // 2])
    for i in slow:
        assert np.array_equal(y[..., i], interp[..., i]) and np.array_equal(y[..., i + Di // 2], interp[..., i + Di // 2])


def test_yarn_ramp_is_monotone_between_interpolation_and_extrapolation():
    """The angle per position of each pair, read off a rotated basis vector at a small position,
    is squeezed between the interpolated and the plain frequency and their ratio rises with the
    pair's frequency."""
    Di, theta, p = 64, 10000.0, 1     # angles below pi: no wrap-around
    f = theta ** (-2.0 * np.arange(Di // 2) / Di)
    ratios = []
    for i in range(Di // 2):
        x = np.zeros((1, 1, Di), dtype=np.uint16)
        x[0, 0, i] = 0x3F80
        y = f64(O.rope_rows(x, np.array([p]), theta, yarn=YARN))[0, 0]
        ang = math.atan2(y[i + Di // 2], y[i]) / p
        ratios.append(ang / f[i])
    ratios = np.array(ratios)
    assert np.all(ratios >= 1 / 8 - 1e-2) and np.all(ratios <= 1 + 1e-2)
    assert np.all(np.diff(ratios[::-1]) >= -1e-2)    # from the slowest pair up: non-decreasing
    assert ratios[0] > 0.99 and ratios[-1] < 0.13


def test_yarn_magnitude_factor_scales_norms_and_keeps_relative_positions():
    rng = np.random.default_rng(33)
    q = rand_bits(rng, (1, 1, 64))
    k = rand_bits(rng, (1, 1, 64))
    y = dict(YARN, mscale=1.5)
    r = f64(O.rope_rows(q, np.array([12345]), 10000.0, yarn=y))
    assert abs(np.linalg.norm(r) - 1.5 * np.linalg.norm(f64(q))) <= 1e-2 * np.linalg.norm(f64(q))
    dots = []
    for shift in [0, 96, 40000]:
        a = f64(O.rope_rows(q, np.array([50 + shift]), 10000.0, yarn=YARN)).ravel()
        b = f64(O.rope_rows(k, np.array([18 + shift]), 10000.0, yarn=YARN)).ravel()
        dots.append(a @ b)
    assert np.ptp(dots) <= 2e-2 * np.linalg.norm(f64(q)) * np.linalg.norm(f64(k))


def test_yarn_pooled_keys_match_yarn_rotated_means():
    """Pooling with YaRN is the YaRN rotation of the block means at the block start."""
    rng = np.random.default_rng(34)
    ki = rand_bits(rng, (1, 48, 64), 1 / 8)
    kp = O.pool_block_keys(ki, rope_theta=10000.0, pos0=800, yarn=YARN)
    means = O.pool_block_keys(ki)                          # the means, rounded once
    # rotate the exact means: compare in value with one bf16 rounding of slack on each side
    m = f64(ki).reshape(12, 4, 64).mean(axis=1)
    rot = f64(O.rope_rows(O.bf16_round(m)[:, None, :], 800 + 4 * np.arange(12), 10000.0, yarn=YARN))[:, 0]
    got = f64(kp)[0]
    # two roundings on the right (the mean, then the rotated value) against one on the left: the
    # mean's rounding error moves within its rotation pair, so bound by the pair's magnitude
    norm = np.hypot(m[:, :32], m[:, 32:])
    tol = np.concatenate([1.5 * ulp_bf16(norm)] * 2, axis=1)
    assert np.all(np.abs(got - rot) <= tol + 1e-30)
    assert means.shape == kp.shape


def test_rope_preserves_norm_and_depends_on_relative_position():
    rng = np.random.default_rng(6)
    Di, theta = 64, 10000.0
    q = rand_bits(rng, (1, 1, Di))
    k = rand_bits(rng, (1, 1, Di))
    nq = np.linalg.norm(f64(q))
    for p in [3, 77, 9000]:
        r = f64(O.rope_rows(q, np.array([p]), theta))
        assert abs(np.linalg.norm(r) - nq) <= 1e-2 * nq
    dots = []
    for shift in [0, 100, 5000]:
        a = f64(O.rope_rows(q, np.array([50 + shift]), theta)).ravel()
        b = f64(O.rope_rows(k, np.array([20 + shift]), theta)).ravel()
        dots.append(a @ b)
    scale = np.linalg.norm(f64(q)) * np.linalg.norm(f64(k))
    assert np.ptp(dots) <= 2e-2 * scale
    # and it does depend on the offset itself
    a = f64(O.rope_rows(q, np.array([50]), theta)).ravel()
    b = f64(O.rope_rows(k, np.array([40]), theta)).ravel()
    assert abs(a @ b - dots[0]) > 1e-3 * scale


# ----------------------------------------------------------------------------------- scores
def test_linear_scores_are_one_matmul():
    rng = np.random.default_rng(7)
    Hi, Di, NB = 4, 64, 300
    qi = rand_bits(rng, (Hi, Di), 1 / 8)
    kp = rand_bits(rng, (NB, Di), 1 / 16)
    w = rng.uniform(0.5, 2.0, Hi).astype(np.float32)
    s = O.index_scores(qi, kp, 250, head_w=w, mode=O.LINEAR)
    qsum = (w.astype(np.float64)[:, None] * f64(qi)).sum(axis=0)
    expect = (f64(kp)[:250] @ qsum).astype(np.float32)
    assert s.shape == (250,)
    assert np.allclose(s, expect, rtol=2e-7, atol=1e-9)


def test_relu_scores_brute_force():
    rng = np.random.default_rng(8)
    Hi, Di, NB = 3, 8, 20
    qi = rand_bits(rng, (Hi, Di))
    kp = rand_bits(rng, (NB, Di))
    w = np.array([1.0, 0.5, 2.0], dtype=np.float32)
    s = O.index_scores(qi, kp, NB, head_w=w, mode=O.RELU_SUM)
    qf, kf = f64(qi).tolist(), f64(kp).tolist()
    for b in range(NB):
        acc = 0.0
        for h in range(Hi):
            dot = 0.0
            for d in range(Di):
                dot += qf[h][d] * kf[b][d]
            acc += float(w[h]) * (dot if dot > 0 else 0.0)
        assert s[b] == np.float32(acc)
    # ReLU matters: some head dot products are negative, so LINEAR differs
    assert not np.array_equal(s, O.index_scores(qi, kp, NB, head_w=w, mode=O.LINEAR))


def test_scores_use_only_the_visible_blocks():
    rng = np.random.default_rng(9)
    qi = rand_bits(rng, (4, 64))
    kp = rand_bits(rng, (100, 64))
    full = O.index_scores(qi, kp, 100)
    part = O.index_scores(qi, kp, 37)
    assert np.array_equal(full[:37], part)
    assert O.index_scores(qi, kp, 0).size == 0


# ----------------------------------------------------------------------------------- top-k
def brute_topk(s, k):
    order = sorted(range(len(s)), key=lambda i: (-float(s[i]), i))
    chosen = sorted(order[:k])
    return chosen + [-1] * (k - len(chosen))


@pytest.mark.parametrize("n,k,levels", [(0, 4, 0), (3, 8, 0), (8, 8, 0), (50, 1, 0), (200, 17, 0),
                                        (200, 17, 5), (1000, 64, 3), (513, 512, 2)])
def test_topk_brute_force(n, k, levels):
    rng = np.random.default_rng(n * 31 + k)
    s = rng.standard_normal(n).astype(np.float32)
    if levels:
        s = np.floor(s * levels).astype(np.float32) / levels      # many exact ties
    s = np.maximum(s, 0)                                          # ReLU-style zeros
    idx, (sk, sk1) = O.select_topk(s, k)
    assert idx.tolist() == brute_topk(s, k)
    srt = sorted(s.tolist(), reverse=True)
    assert sk == (srt[k - 1] if n >= k else -math.inf)
    assert sk1 == (srt[k] if n > k else -math.inf)


def test_each_sequence_selects_with_its_own_pooled_keys():
    """One selection per token from the single shared key head, over the token's own sequence: in a
    batch of two, every row's list is the brute-force top-k of the scores of that row's indexer
    query against its own sequence's pooled keys alone (the two sequences' lists differ)."""
    x = small_prefill(23, B=2, T=64)
    kp = O.pool_block_keys(x["ki"])
    k = 3
    rows = [(b, t) for b in range(2) for t in range(64)]
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, rows, topk=k)
    for r, (b, t) in enumerate(rows):
        s = O.index_scores(x["qi"][b, t], kp[b], t // 4)
        assert res["idx"][r].tolist() == brute_topk(s, k), (b, t)
    assert not np.array_equal(res["idx"][:64], res["idx"][64:])


# ----------------------------------------------------------------------------------- attention
def small_prefill(seed, B=1, T=45, Hq=4, Hkv=2, D=32, Hi=2, Di=16, blk=4):
    rng = np.random.default_rng(seed)
    return dict(q=rand_bits(rng, (B, T, Hq, D), D ** -0.5), k=rand_bits(rng, (B, T, Hkv, D), D ** -0.5),
                v=rand_bits(rng, (B, T, Hkv, D), D ** -0.5), qi=rand_bits(rng, (B, T, Hi, Di), Di ** -0.5),
                ki=rand_bits(rng, (B, T, Di), Di ** -0.5))


def test_full_budget_equals_dense_causal_attention_sdpa():
    """k >= every visible block: QSA is dense causal attention (torch SDPA in fp64 as the pin)."""
    x = small_prefill(10, B=2)
    B, T, Hq, D = x["q"].shape
    Hkv = x["k"].shape[2]
    kp = O.pool_block_keys(x["ki"])
    rows = [(b, t) for b in range(B) for t in range(T)]
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, rows, topk=T // 4 + 1)
    q = torch.from_numpy(f64(x["q"])).permute(0, 2, 1, 3)
    k = torch.from_numpy(f64(x["k"])).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    v = torch.from_numpy(f64(x["v"])).permute(0, 2, 1, 3).repeat_interleave(Hq // Hkv, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).permute(0, 2, 1, 3).numpy()
    got = f64(res["out"]).reshape(B, T, Hq, D)
    assert np.all(np.abs(got - ref) <= ulp_bf16(ref) / 2 * (1 + 1e-6) + 1e-12)
    logits = (q @ k.transpose(-1, -2)) / math.sqrt(D)
    logits = logits.masked_fill(torch.ones(T, T, dtype=torch.bool).triu(1), -math.inf)
    lse_ref = torch.logsumexp(logits, dim=-1).permute(0, 2, 1).numpy()
    assert np.allclose(res["lse"].reshape(B, T, Hq), lse_ref, rtol=1e-6, atol=1e-6)


def test_attention_textbook_loop_one_row():
    x = small_prefill(11, T=30, Hq=2, Hkv=1, D=8)
    kp = O.pool_block_keys(x["ki"])
    t = 29
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, t)], topk=3)
    sel = [b for b in res["idx"][0].tolist() if b >= 0]
    toks = [4 * b + j for b in sel for j in range(4)] + list(range(4 * (t // 4), t + 1))
    q, k, v = f64(x["q"])[0, t], f64(x["k"])[0], f64(x["v"])[0]
    for h in range(2):
        z = [sum(q[h][d] * k[j][0][d] for d in range(8)) / math.sqrt(8) for j in toks]
        m = max(z)
        p = [math.exp(a - m) for a in z]
        o = [sum(p[i] * v[toks[i]][0][d] for i in range(len(toks))) / sum(p) for d in range(8)]
        assert np.array_equal(res["out"][0, h], np_bf16_rne(np.array(o)))
        assert abs(res["lse"][0, h] - (m + math.log(sum(p)))) < 1e-6


def test_token_count_closed_form_via_lse():
    """With all keys zero every logit is 0, so lse = log|S(t)|; |S(t)| = 4 min(t//4, k) + t%4 + 1."""
    x = small_prefill(12, T=61, Hq=1, Hkv=1, D=16)
    x["k"][:] = 0
    kp = O.pool_block_keys(x["ki"])
    for k in [1, 2, 5, 20]:
        res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, t) for t in range(61)], topk=k)
        n = np.rint(np.exp(res["lse"][:, 0].astype(np.float64))).astype(int)
        expect = [4 * min(t // 4, k) + t % 4 + 1 for t in range(61)]
        assert n.tolist() == expect


def test_golden_budget_512_blocks_is_2048_tokens_plus_own_block():
    with open(os.path.join(GOLDEN, "qsa_budget.json")) as f:
        g = json.load(f)
    blk, k = g["block_tokens"], g["selected_blocks"]
    assert blk * k == g["selected_tokens"]
    T = 2300
    x = small_prefill(13, T=T, Hq=1, Hkv=1, D=16, Hi=4, Di=16)
    x["k"][:] = 0
    kp = O.pool_block_keys(x["ki"], blk=blk)
    rows = [(0, t) for t in (2100, 2101, 2102, 2103, 2299)]
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, rows, topk=k, blk=blk)
    n = np.rint(np.exp(res["lse"][:, 0].astype(np.float64))).astype(int)
    for (_, t), c in zip(rows, n):
        own = t % blk + 1                      # the possibly incomplete own block
        assert c == g["selected_tokens"] + own
        assert g["own_block_min"] <= own <= g["own_block_max"]
    assert np.all(res["idx"] >= 0) and np.all(np.diff(res["idx"], axis=1) > 0)


def test_unselected_tokens_do_not_matter():
    x = small_prefill(14, T=80)
    kp = O.pool_block_keys(x["ki"])
    t = 77
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, t)], topk=5)
    sel = set(4 * b + j for b in res["idx"][0] if b >= 0 for j in range(4)) | set(range(4 * (t // 4), t + 1))
    k2, v2 = x["k"].copy(), x["v"].copy()
    for j in range(80):
        if j not in sel:
            k2[0, j] = 0x7FC0                   # NaN
            v2[0, j] = 0x7FC0
    res2 = O.prefill_rows(x["q"], k2, v2, x["qi"], kp, [(0, t)], topk=5, idx_in=res["idx"])
    assert np.array_equal(res["out"], res2["out"]) and np.array_equal(res["lse"], res2["lse"])
    # and a selected token does matter
    j = sorted(sel)[0]
    v3 = x["v"].copy()
    v3[0, j] = np_bf16_rne(f64(v3[0, j]) + 1.0)
    res3 = O.prefill_rows(x["q"], x["k"], v3, x["qi"], kp, [(0, t)], topk=5, idx_in=res["idx"])
    assert not np.array_equal(res["out"], res3["out"])


def test_index_order_does_not_matter():
    x = small_prefill(15, T=120)
    kp = O.pool_block_keys(x["ki"])
    rows = [(0, t) for t in range(100, 120)]
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, rows, topk=9)
    perm = np.random.default_rng(0).permuted(res["idx"], axis=1)
    res2 = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, rows, topk=9, idx_in=perm)
    a, b = f64(res["out"]), f64(res2["out"])
    assert np.all(np.abs(a - b) <= ulp_bf16(a))


def test_constant_values_and_first_token():
    x = small_prefill(16, T=40)
    x["v"][:] = 0x3F40                           # 0.75 everywhere
    kp = O.pool_block_keys(x["ki"])
    res = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, t) for t in range(40)], topk=3)
    assert np.all(res["out"] == 0x3F40)
    y = small_prefill(17, T=8)
    kp = O.pool_block_keys(y["ki"])
    r0 = O.prefill_rows(y["q"], y["k"], y["v"], y["qi"], kp, [(0, 0)], topk=2)
    Hq, Hkv = 4, 2
    for h in range(Hq):
        assert np.array_equal(r0["out"][0, h], y["v"][0, 0, h // (Hq // Hkv)])
        z = f64(y["q"][0, 0, h]) @ f64(y["k"][0, 0, h // 2]) / math.sqrt(32)
        assert abs(r0["lse"][0, h] - z) < 1e-6
    assert np.all(r0["idx"] == -1)


def test_gqa_head_mapping():
    """Query head h reads KV head h // (Hq/Hkv): changing KV head 1 moves heads 2, 3 only."""
    x = small_prefill(18, T=24)
    kp = O.pool_block_keys(x["ki"])
    rows = [(0, 23)]
    a = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, rows, topk=2)
    v2 = x["v"].copy()
    v2[0, :, 1] = np_bf16_rne(f64(v2[0, :, 1]) * 2)
    b = O.prefill_rows(x["q"], x["k"], v2, x["qi"], kp, rows, topk=2)
    assert np.array_equal(a["out"][0, :2], b["out"][0, :2])
    assert not np.array_equal(a["out"][0, 2:], b["out"][0, 2:])


# ----------------------------------------------------------------------------------- decode
def test_decode_equals_last_prefill_row():
    x = small_prefill(19, B=3, T=64)
    kp = O.pool_block_keys(x["ki"])
    seqlens = np.array([64, 37, 9], dtype=np.int32)
    kc, vc = x["k"].copy(), x["v"].copy()
    for b, L in enumerate(seqlens):
        kc[b, L:] = 0x7FC0                        # cache slots past the sequence are garbage
        vc[b, L:] = 0x7FC0
    qd = np.stack([x["q"][b, L - 1] for b, L in enumerate(seqlens)])
    qid = np.stack([x["qi"][b, L - 1] for b, L in enumerate(seqlens)])
    d = O.decode(qd, kc, vc, qid, kp, seqlens, topk=6)
    for b, L in enumerate(seqlens):
        p = O.prefill_rows(x["q"][b:b + 1, :L], x["k"][b:b + 1, :L], x["v"][b:b + 1, :L], x["qi"][b:b + 1, :L],
                           kp[b:b + 1, : L // 4], [(0, L - 1)], topk=6)
        assert np.array_equal(d["idx"][b], p["idx"][0])
        assert np.array_equal(d["out"][b], p["out"][0])
        assert np.array_equal(d["lse"][b], p["lse"][0])


def test_decode_with_rope_matches_prefill_with_rope():
    x = small_prefill(20, T=50, Hi=4, Di=16)
    theta = 10000.0
    kp = O.pool_block_keys(x["ki"], rope_theta=theta)
    d = O.decode(x["q"][:, 49], x["k"], x["v"], x["qi"][:, 49], kp, np.array([50]), topk=4, rope_theta=theta)
    p = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, 49)], topk=4, rope_theta=theta)
    assert np.array_equal(d["idx"], p["idx"]) and np.array_equal(d["out"], p["out"])
    # RoPE changes the selection somewhere
    kp0 = O.pool_block_keys(x["ki"])
    p0 = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp0, [(0, t) for t in range(20, 50)], topk=4)
    pr = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, t) for t in range(20, 50)], topk=4,
                        rope_theta=theta)
    assert not np.array_equal(p0["idx"], pr["idx"])


def test_chunked_prefill_position_offset():
    """Query rows given as a chunk starting at q_pos0 see the same result as in the full prefill."""
    x = small_prefill(21, T=64)
    kp = O.pool_block_keys(x["ki"])
    full = O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, t) for t in range(40, 64)], topk=5)
    part = O.prefill_rows(x["q"][:, 40:], x["k"], x["v"], x["qi"][:, 40:], kp, [(0, t) for t in range(24)],
                          topk=5, q_pos0=40)
    assert np.array_equal(full["idx"], part["idx"]) and np.array_equal(full["out"], part["out"])


def test_out_of_range_index_is_rejected():
    x = small_prefill(22, T=20)
    kp = O.pool_block_keys(x["ki"])
    bad = np.array([[1, 7, -1]], dtype=np.int32)         # 7 > own block of t=10
    with pytest.raises(ValueError):
        O.prefill_rows(x["q"], x["k"], x["v"], x["qi"], kp, [(0, 10)], topk=3, idx_in=bad)
