"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a worked
example, a closed form, a library routine that computes a special case, a
pure-Python brute force (``tests/brute.py``) or an invariant.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle as O
from tests import brute

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# bf16 storage rounding
# ---------------------------------------------------------------------------
def test_bf16_round_matches_torch_on_float32_values():
    # float32 -> bf16 in torch rounds to nearest, ties to even.  For inputs that
    # are exact float32 values the oracle's single fp64 rounding must agree.
    rng = np.random.default_rng(123)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e30).astype(np.float32),
        (rng.standard_normal(5000) * 1e-38).astype(np.float32),   # bf16 subnormals
        np.float32([0.0, -0.0, 1.0, -1.0, 3.3895314e38, 1e-45]),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_and_single_rounding():
    e = 2.0 ** -8
    assert O.bf16_round(1.0 + e) == 1.0                     # tie -> even (1.0)
    assert O.bf16_round(1.0 + 3 * e) == 1.0 + 4 * e         # tie -> even (1 + 2^-6)
    # Just above a tie: a single rounding from fp64 goes up; rounding through
    # float32 first would land exactly on the tie and go down.
    assert O.bf16_round(1.0 + e + 2.0 ** -40) == 1.0 + 2 * e
    assert O.bf16_round(-(1.0 + e + 2.0 ** -40)) == -(1.0 + 2 * e)
    # subnormal range: spacing 2^-133
    assert O.bf16_round(2.0 ** -134) == 0.0                 # tie between 0 and 1 step -> 0
    assert O.bf16_round(3 * 2.0 ** -134) == 2.0 ** -132     # tie between 1 and 2 steps -> 2
    assert O.bf16_round(2.0 ** -130) == 2.0 ** -130
    assert np.isinf(O.bf16_round(3.4e38))
    bits = O.f64_to_bf16_bits(np.array([1.0, -2.0, 0.5]))
    np.testing.assert_array_equal(bits, np.array([0x3F80, 0xC000, 0x3F00], np.uint16))
    np.testing.assert_array_equal(O.bf16_bits_to_f64(bits), [1.0, -2.0, 0.5])


# ---------------------------------------------------------------------------
# Step 1: chunk pooling
# ---------------------------------------------------------------------------
def _read_pool_golden():
    rows, expect, kv = [], [], {}
    with open(os.path.join(GOLDEN, "chunk_pool_worked_example.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            if k == "row":
                rows.append([float(t) for t in v])
            elif k == "expect":
                expect.append([float(t) for t in v])
            else:
                kv[k] = int(v[0])
    return kv, np.array(rows), np.array(expect)


def test_chunk_pool_worked_example():
    kv, rows, expect = _read_pool_golden()
    assert rows.shape == (kv["padded_len"], kv["H"])
    # padded layout: the document starts at row 0; rows beyond len are padding
    pooled, off = O.chunk_pool(rows, [0], [kv["len"]], 4)
    np.testing.assert_array_equal(off, [0, 2])
    np.testing.assert_array_equal(pooled, expect)


def test_chunk_pool_special_cases():
    rng = np.random.default_rng(5)
    x = O.bf16_round(rng.standard_normal((12, 6)))
    # len 1: the single row itself
    p, _ = O.chunk_pool(x, [3], [1])
    np.testing.assert_array_equal(p, x[3:4])
    # len = 4k with rows that are exact in a quarter: exact quarters
    y = np.arange(8 * 2, dtype=np.float64).reshape(8, 2)
    p, _ = O.chunk_pool(y, [0], [8])
    np.testing.assert_array_equal(p, [[3.0, 4.0], [11.0, 12.0]])
    # all rows equal -> the same vector in every group (len 7: groups of 4 and 3)
    z = np.tile(x[0], (7, 1))
    p, _ = O.chunk_pool(z, [0], [7])
    np.testing.assert_array_equal(p, np.tile(x[0], (2, 1)))
    # chunk = 1 is the identity
    p, _ = O.chunk_pool(x, [0], [12], chunk=1)
    np.testing.assert_array_equal(p, x)
    # empty document: no vectors
    p, off = O.chunk_pool(x, [0, 0], [0, 5])
    np.testing.assert_array_equal(off, [0, 0, 2])


def test_pooled_counts_bounds():
    lens = np.arange(0, 1025)
    c = O.pooled_counts(lens)
    np.testing.assert_array_equal(c, [math.ceil(v / 4) for v in lens])
    assert c.max() == 256


@pytest.mark.parametrize("chunk", [1, 2, 4, 8])
def test_chunk_pool_vs_bruteforce_padded_mask(chunk):
    rng = np.random.default_rng(11 + chunk)
    lens = [0, 1, 2, 3, 4, 5, 8, 9, 13]
    H, Lmax = 3, 16
    padded = rng.standard_normal((len(lens), Lmax, H))
    # packed copy of the valid rows with a row offset per document
    tok_off = np.concatenate([[0], np.cumsum(lens)])
    packed = np.concatenate([padded[d, :lens[d]] for d in range(len(lens))])
    pooled, off = O.chunk_pool(packed, tok_off, lens, chunk, round_out=False)
    for d, n in enumerate(lens):
        mask = [1] * n + [0] * (Lmax - n)
        want = brute.pool_padded(padded[d].tolist(), mask, chunk)
        got = pooled[off[d]:off[d + 1]]
        assert len(want) == got.shape[0]
        if want:
            np.testing.assert_allclose(got, np.array(want), rtol=0, atol=1e-12)
    # the padded layout (row stride Lmax) gives the same result
    pooled2, _ = O.chunk_pool(padded.reshape(-1, H), np.arange(len(lens)) * Lmax, lens, chunk,
                              round_out=False)
    np.testing.assert_array_equal(pooled2, pooled)


# ---------------------------------------------------------------------------
# Step 2: projections
# ---------------------------------------------------------------------------
def test_linear_vs_bruteforce_nonsquare():
    rng = np.random.default_rng(2)
    x = O.bf16_round(rng.standard_normal((5, 7)))
    w = O.bf16_round(rng.standard_normal((3, 7)) * 0.1)
    r = O.bf16_round(rng.standard_normal((5, 3)))
    want = np.array(brute.matvec_rows(x.tolist(), w.tolist()))
    np.testing.assert_allclose(O.linear(x, w, round_out=False), want, atol=1e-12, rtol=0)
    np.testing.assert_allclose(O.linear(x, w, residual=r, round_out=False), want + r,
                               atol=1e-12, rtol=0)
    # rounded once, after the residual add
    np.testing.assert_array_equal(O.linear(x, w, residual=r), O.bf16_round(want + r))


def test_linear_identity_weight():
    rng = np.random.default_rng(3)
    x = O.bf16_round(rng.standard_normal((4, 6)))
    np.testing.assert_array_equal(O.linear(x, np.eye(6)), x)


# ---------------------------------------------------------------------------
# Step 3: merged attention
# ---------------------------------------------------------------------------
def _rand_attn(rng, Lq, Nc, n_q, n_kv, D, kscale=1.0):
    q = rng.standard_normal((Lq, n_q, D))
    ks = rng.standard_normal((Lq, n_kv, D)) * kscale
    vs = rng.standard_normal((Lq, n_kv, D))
    kc = rng.standard_normal((Nc, n_kv, D)) * kscale
    vc = rng.standard_normal((Nc, n_kv, D))
    return q, ks, vs, kc, vc


@pytest.mark.parametrize("Lq,Nc,n_q,n_kv,D", [
    (1, 0, 1, 1, 4), (1, 3, 2, 1, 8), (5, 3, 2, 1, 8), (4, 2, 4, 2, 3), (3, 1, 2, 2, 5), (5, 0, 2, 1, 8)])
def test_attention_vs_bruteforce_concat(Lq, Nc, n_q, n_kv, D):
    rng = np.random.default_rng(100 + Lq * 7 + Nc)
    q, ks, vs, kc, vc = _rand_attn(rng, Lq, Nc, n_q, n_kv, D)
    scale = 1.0 / math.sqrt(D)
    o, lse = O.merged_attention_doc(q, ks, vs, kc, vc, scale, round_out=False)
    bo, blse = brute.attention_concat(q.tolist(), ks.tolist(), vs.tolist(), kc.tolist(),
                                      vc.tolist(), scale)
    np.testing.assert_allclose(o, np.array(bo), atol=1e-12, rtol=0)
    np.testing.assert_allclose(lse, np.array(blse), atol=1e-12, rtol=0)


def _sdpa(q, k, v, mask, scale):
    # torch SDPA in float64 on CPU: [heads][rows][D] layout
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=None if mask is None else torch.from_numpy(mask), scale=scale).numpy()


def test_attention_no_cross_equals_causal_sdpa():
    rng = np.random.default_rng(7)
    Lq, n_q, n_kv, D = 9, 4, 2, 16
    q, ks, vs, kc, vc = _rand_attn(rng, Lq, 0, n_q, n_kv, D)
    scale = 0.25
    o, _ = O.merged_attention_doc(q, ks, vs, kc, vc, scale, round_out=False)
    G = n_q // n_kv
    for h in range(n_q):
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, h][None]), torch.from_numpy(ks[:, h // G][None]),
            torch.from_numpy(vs[:, h // G][None]), is_causal=True, scale=scale).numpy()[0]
        np.testing.assert_allclose(o[:, h], ref, atol=1e-12, rtol=0)


def test_attention_with_cross_equals_masked_sdpa():
    rng = np.random.default_rng(8)
    Lq, Nc, n_q, n_kv, D = 7, 5, 2, 1, 16
    q, ks, vs, kc, vc = _rand_attn(rng, Lq, Nc, n_q, n_kv, D)
    scale = 1.0 / 4
    o, _ = O.merged_attention_doc(q, ks, vs, kc, vc, scale, round_out=False)
    mask = np.concatenate([np.tril(np.ones((Lq, Lq), bool)), np.ones((Lq, Nc), bool)], 1)
    k = np.concatenate([ks[:, 0], kc[:, 0]])
    v = np.concatenate([vs[:, 0], vc[:, 0]])
    for h in range(n_q):
        ref = _sdpa(q[:, h][None], k[None], v[None], mask, scale)[0]
        np.testing.assert_allclose(o[:, h], ref, atol=1e-12, rtol=0)


def test_attention_zero_keys_closed_form():
    rng = np.random.default_rng(9)
    Lq, Nc, n_q, n_kv, D = 6, 4, 2, 1, 5
    q, ks, vs, kc, vc = _rand_attn(rng, Lq, Nc, n_q, n_kv, D, kscale=0.0)
    o, lse = O.merged_attention_doc(q, ks, vs, kc, vc, 0.3, round_out=False)
    for i in range(Lq):
        want = (vs[: i + 1, 0].sum(0) + vc[:, 0].sum(0)) / (i + 1 + Nc)
        for h in range(n_q):
            np.testing.assert_allclose(o[i, h], want, atol=1e-13, rtol=0)
            assert abs(lse[i, h] - math.log(i + 1 + Nc)) < 1e-13


def test_attention_two_segment_lse_merge():
    rng = np.random.default_rng(10)
    Lq, Nc, n_q, n_kv, D = 6, 5, 4, 2, 8
    q, ks, vs, kc, vc = _rand_attn(rng, Lq, Nc, n_q, n_kv, D)
    scale = 0.4
    o, lse = O.merged_attention_doc(q, ks, vs, kc, vc, scale, round_out=False)
    o1, lse1 = O.merged_attention_doc(q, ks, vs, kc[:0], vc[:0], scale, round_out=False)
    G = n_q // n_kv
    for h in range(n_q):
        g = h // G
        # cross-only: a plain unmasked softmax over the cross keys (library)
        qt = torch.from_numpy(q[:, h])
        logits = qt @ torch.from_numpy(kc[:, g]).T * scale
        lse2 = torch.logsumexp(logits, dim=1).numpy()
        o2 = _sdpa(q[:, h][None], kc[:, g][None], vc[:, g][None], None, scale)[0]
        a, b = np.exp(lse1[:, h])[:, None], np.exp(lse2)[:, None]
        np.testing.assert_allclose(o[:, h], (a * o1[:, h] + b * o2) / (a + b), atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[:, h], np.logaddexp(lse1[:, h], lse2), atol=1e-12, rtol=0)


def test_attention_invariants():
    rng = np.random.default_rng(12)
    Lq, Nc, n_q, n_kv, D = 6, 5, 4, 1, 8
    q, ks, vs, kc, vc = _rand_attn(rng, Lq, Nc, n_q, n_kv, D)
    o, lse = O.merged_attention_doc(q, ks, vs, kc, vc, 0.35, round_out=False)
    # permuting the cross vectors changes nothing
    p = rng.permutation(Nc)
    o2, lse2 = O.merged_attention_doc(q, ks, vs, kc[p], vc[p], 0.35, round_out=False)
    np.testing.assert_allclose(o2, o, atol=1e-12, rtol=0)
    # causality: perturbing self rows j > i leaves rows <= i unchanged
    ks2, vs2 = ks.copy(), vs.copy()
    ks2[3:] += 5.0
    vs2[3:] -= 2.0
    o3, _ = O.merged_attention_doc(q, ks2, vs2, kc, vc, 0.35, round_out=False)
    np.testing.assert_allclose(o3[:3], o[:3], atol=1e-12, rtol=0)
    assert np.abs(o3[3:] - o[3:]).max() > 1e-3
    # MHA (n_kv = n_q) is the per-head computation
    qm, ksm, vsm, kcm, vcm = _rand_attn(rng, Lq, Nc, 3, 3, D)
    om, _ = O.merged_attention_doc(qm, ksm, vsm, kcm, vcm, 0.2, round_out=False)
    for h in range(3):
        oh, _ = O.merged_attention_doc(qm[:, h:h + 1], ksm[:, h:h + 1], vsm[:, h:h + 1],
                                       kcm[:, h:h + 1], vcm[:, h:h + 1], 0.2, round_out=False)
        np.testing.assert_allclose(om[:, h], oh[:, 0], atol=1e-12, rtol=0)


def test_attention_batch_composition():
    rng = np.random.default_rng(13)
    n_q, n_kv, D = 2, 1, 4
    lq = [3, 1, 4]
    nc = [2, 0, 5]
    docs = [_rand_attn(rng, a, b, n_q, n_kv, D) for a, b in zip(lq, nc)]
    q_off = np.concatenate([[0], np.cumsum(lq)])
    p_off = np.concatenate([[0], np.cumsum(nc)])
    cat = [np.concatenate([d[i] for d in docs]) for i in range(5)]
    o, lse = O.merged_attention(*cat, q_off, p_off, 0.5, round_out=False)
    for d in range(3):
        od, ld = O.merged_attention_doc(*docs[d], 0.5, round_out=False)
        np.testing.assert_array_equal(o[q_off[d]:q_off[d + 1]], od)
    # reversed document order gives the same per-document results
    order = [2, 1, 0]
    cat_r = [np.concatenate([docs[d][i] for d in order]) for i in range(5)]
    q_r = np.concatenate([[0], np.cumsum([lq[d] for d in order])])
    p_r = np.concatenate([[0], np.cumsum([nc[d] for d in order])])
    o_r, _ = O.merged_attention(*cat_r, q_r, p_r, 0.5, round_out=False)
    for k, d in enumerate(order):
        np.testing.assert_array_equal(o_r[q_r[k]:q_r[k + 1]], o[q_off[d]:q_off[d + 1]])


# ---------------------------------------------------------------------------
# Step 4: readout
# ---------------------------------------------------------------------------
def test_readout_identity_softmax_equals_sigmoid():
    import scipy.special
    for m in [0.0, 1e-8, -1e-8, 1.0, -1.0, 30.0, -30.0, 100.0, -100.0]:
        y, n = 0.3 + m, 0.3
        s = O.sigmoid(np.array([y - n]))[0]
        assert abs(s - brute.softmax2_first(y, n)) <= 1e-15 * max(1.0, s) + 1e-300
        assert abs(s - scipy.special.expit(y - n)) <= 1e-15 * max(1e-300, s) + 1e-300
    big = O.sigmoid(np.array([-1000.0, 1000.0]))
    assert big[0] == 0.0 and big[1] == 1.0 and np.all(np.isfinite(big))
    ms = np.linspace(-40, 40, 801)
    assert np.all(np.diff(O.sigmoid(ms)) >= 0)


def test_readout_values():
    rng = np.random.default_rng(14)
    x = O.bf16_round(rng.standard_normal((3, 10)))
    wy = O.bf16_round(rng.standard_normal(10) * 0.02)
    wn = O.bf16_round(rng.standard_normal(10) * 0.02)
    y, n, m, s = O.yes_no_score(x, wy, wn)
    for i in range(3):
        by = sum(x[i, k] * wy[k] for k in range(10))
        bn = sum(x[i, k] * wn[k] for k in range(10))
        assert abs(y[i] - by) < 1e-14 and abs(n[i] - bn) < 1e-14
        assert abs(s[i] - brute.softmax2_first(by, bn)) < 1e-15
    # identical yes/no rows give exactly one half
    _, _, m2, s2 = O.yes_no_score(x, wy, wy)
    np.testing.assert_array_equal(m2, 0.0)
    np.testing.assert_array_equal(s2, 0.5)


# ---------------------------------------------------------------------------
# End to end (the oracle's own chain)
# ---------------------------------------------------------------------------
def _tiny_stack(rng, H=16, D=8, n_q=2, n_kv=1, Lq=3, L=2, length=9):
    enc = O.bf16_round(rng.standard_normal((length, H)))
    x0 = O.bf16_round(rng.standard_normal((Lq, H)))
    w_qkv = O.bf16_round(rng.standard_normal((L, (n_q + 2 * n_kv) * D, H)) * 0.2)
    w_o = O.bf16_round(rng.standard_normal((L, H, n_q * D)) * 0.2)
    w_kv = O.bf16_round(rng.standard_normal((L, 2 * n_kv * D, H)) * 0.2)
    wy = O.bf16_round(rng.standard_normal(H) * 0.2)
    wn = O.bf16_round(rng.standard_normal(H) * 0.2)
    return enc, x0, w_qkv, w_o, w_kv, wy, wn


def test_end_to_end_zero_weights_closed_form():
    rng = np.random.default_rng(15)
    enc, x0, w_qkv, w_o, w_kv, wy, wn = _tiny_stack(rng)
    zero = [np.zeros_like(w_qkv), np.zeros_like(w_o), np.zeros_like(w_kv)]
    y, n, m, s = O.forward_doc(enc, x0, *zero, wy, wn, 2, 1, 8, 0.35)
    x_last = x0[-1]
    assert abs(y - x_last @ wy) < 1e-14 and abs(n - x_last @ wn) < 1e-14
    assert abs(s - 1.0 / (1.0 + math.exp(-(x_last @ (wy - wn))))) < 1e-14
    # with only the output projection zeroed the attention runs but adds nothing
    y2, _, _, s2 = O.forward_doc(enc, x0, w_qkv, np.zeros_like(w_o), w_kv, wy, wn, 2, 1, 8, 0.35)
    assert y2 == y and s2 == s
    # rows before the final one do not reach the score when nothing mixes rows
    x0b = x0.copy()
    x0b[0] += 3.0
    assert O.forward_doc(enc, x0b, *zero, wy, wn, 2, 1, 8, 0.35) == (y, n, m, s)


def _brute_chain(enc, x0, w_qkv, w_o, w_kv, wy, wn, n_q, n_kv, D, scale):
    """Pure-Python chain of the brute-force pieces with the oracle's bf16 rounding
    points, for one document whose encoder rows are all valid.  Returns (yes, no)."""
    rnd = lambda a: O.bf16_round(np.array(a)).tolist()
    pooled = rnd(brute.pool_padded(enc.tolist(), [1] * len(enc), 4))
    X = x0.tolist()
    for l in range(len(w_qkv)):
        kv = rnd(brute.matvec_rows(pooled, w_kv[l].tolist()))
        qkv = rnd(brute.matvec_rows(X, w_qkv[l].tolist()))
        q = [[r[h * D:(h + 1) * D] for h in range(n_q)] for r in qkv]
        ks = [[r[(n_q + g) * D:(n_q + g + 1) * D] for g in range(n_kv)] for r in qkv]
        vs = [[r[(n_q + n_kv + g) * D:(n_q + n_kv + g + 1) * D] for g in range(n_kv)] for r in qkv]
        kc = [[r[g * D:(g + 1) * D] for g in range(n_kv)] for r in kv]
        vc = [[r[(n_kv + g) * D:(n_kv + g + 1) * D] for g in range(n_kv)] for r in kv]
        o, _ = brute.attention_concat(q, ks, vs, kc, vc, scale)
        o = rnd([sum(r, []) for r in o])
        proj = brute.matvec_rows(o, w_o[l].tolist())
        X = rnd([[a + b for a, b in zip(pr, xr)] for pr, xr in zip(proj, X)])
    by = sum(a * b for a, b in zip(X[-1], wy))
    bn = sum(a * b for a, b in zip(X[-1], wn))
    return by, bn


def test_end_to_end_vs_bruteforce_chain():
    rng = np.random.default_rng(16)
    H, D, n_q, n_kv, Lq, L = 16, 8, 2, 1, 3, 2
    enc, x0, w_qkv, w_o, w_kv, wy, wn = _tiny_stack(rng, H, D, n_q, n_kv, Lq, L, length=9)
    scale = 1.0 / math.sqrt(D)
    got = O.forward_doc(enc, x0, w_qkv, w_o, w_kv, wy, wn, n_q, n_kv, D, scale)
    by, bn = _brute_chain(enc, x0, w_qkv, w_o, w_kv, wy, wn, n_q, n_kv, D, scale)
    assert abs(got[0] - by) < 1e-12 and abs(got[1] - bn) < 1e-12
    assert abs(got[3] - brute.softmax2_first(by, bn)) < 1e-13


def _bits(a):
    """float values -> bf16 bit patterns (the synthetic inputs' storage form)."""
    import synthetic
    return synthetic.f32_to_bf16_bits(np.asarray(a, np.float32))


def test_forward_query_slices_documents_and_uses_the_standard_scale():
    """forward_query on a hand-built three-document query (1, 6 and 9 encoder rows,
    every row distinct) against forward_doc on slices written out here, at the
    standard scaled-dot-product scale 1/sqrt(256) = 1/16 ("What this is": a scaled
    dot-product attention), and against the pure-Python chain for one document.
    Documents are packed one after another with no padding rows between them
    ("Frozen inference contract": right padding, so a document's valid tokens are
    its first rows)."""
    import synthetic
    rng = np.random.default_rng(33)
    H, D, n_q, n_kv, Lq, L = 16, 256, 2, 1, 3, 1
    lens = np.array([1, 6, 9], dtype=np.int32)
    # row t holds distinct values: a random draw plus an offset that grows with t
    enc_f = rng.standard_normal((16, H)).astype(np.float32) + 0.5 * np.arange(16, dtype=np.float32)[:, None]
    x0_f = rng.standard_normal((Lq, H)).astype(np.float32)
    w = synthetic.Weights(
        w_qkv=_bits(rng.standard_normal((L, (n_q + 2 * n_kv) * D, H)) * 0.2),
        w_o=_bits(rng.standard_normal((L, H, n_q * D)) * 0.2),
        w_kv_cross=_bits(rng.standard_normal((L, 2 * n_kv * D, H)) * 0.2),
        w_yes=_bits(rng.standard_normal(H) * 0.2), w_no=_bits(rng.standard_normal(H) * 0.2))
    q = synthetic.Query("pin", H, n_q, n_kv, D, L, lens, np.array([0, 1, 7, 16], dtype=np.int64), _bits(enc_f),
                        Lq, _bits(x0_f), w)
    got = O.forward_query(q)
    enc = O.bf16_bits_to_f64(q.enc)
    x0 = O.bf16_bits_to_f64(q.x0)
    ws = [O.bf16_bits_to_f64(a) for a in (w.w_qkv, w.w_o, w.w_kv_cross, w.w_yes, w.w_no)]
    slices = {0: enc[0:1], 1: enc[1:7], 2: enc[7:16]}
    for d, rows in slices.items():
        want = O.forward_doc(rows, x0, *ws, n_q, n_kv, D, 1.0 / 16)
        assert [float(g[d]) for g in got] == list(want), d
    # the middle document through the pure-Python chain
    by, bn = _brute_chain(slices[1], x0, *ws, n_q, n_kv, D, 1.0 / 16)
    assert abs(got[0][1] - by) < 1e-10 and abs(got[1][1] - bn) < 1e-10
    # the three documents' scores are distinct, so a wrong slice cannot go unnoticed
    assert len({float(s) for s in got[3]}) == 3


def test_forward_query_doc_independence():
    import synthetic
    qy = synthetic.make_query("tiny", layers=1, hidden=64)
    all_scores = O.forward_query(qy)[3]
    # each document alone gives the same score as inside the batch
    for d in range(qy.n_docs):
        s = O.forward_query(qy, docs=[d])[3]
        assert s[0] == all_scores[d]


# ---------------------------------------------------------------------------
# Rotary position embedding of the decoder's self Q and K
# ---------------------------------------------------------------------------
def test_rope_matches_complex_rotation():
    """Each pair (x[i], x[i + D/2]) read as the complex number x[i] + j x[i + D/2] is
    multiplied by exp(j * pos * theta^(-2i/D)) (numpy complex arithmetic)."""
    rng = np.random.default_rng(21)
    D, theta = 16, 10000.0
    x = rng.standard_normal((5, 3, D))
    pos = [0, 1, 7, 100, 511]
    got = O.apply_rope(x, pos, theta, round_out=False)
    z = x[..., : D // 2] + 1j * x[..., D // 2:]
    freq = np.array([theta ** (-(2 * i) / D) for i in range(D // 2)])
    rot = np.exp(1j * np.outer(pos, freq))[:, None, :]
    want = z * rot
    np.testing.assert_allclose(got[..., : D // 2], want.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got[..., D // 2:], want.imag, rtol=0, atol=1e-12)


def test_rope_special_cases():
    rng = np.random.default_rng(22)
    x = rng.standard_normal((4, 2, 8))
    # position 0 is the identity; the rotation keeps every pair's length
    np.testing.assert_array_equal(O.apply_rope(x, [0] * 4, 500.0, round_out=False), x)
    y = O.apply_rope(x, [3, 9, 27, 81], 500.0, round_out=False)
    np.testing.assert_allclose(y[..., :4] ** 2 + y[..., 4:] ** 2, x[..., :4] ** 2 + x[..., 4:] ** 2, rtol=1e-13)
    # D = 2: one pair at frequency 1, so position p rotates (1, 0) to (cos p, sin p)
    e = np.array([[[1.0, 0.0]]])
    np.testing.assert_allclose(O.apply_rope(e, [2], 1e4, round_out=False)[0, 0], [math.cos(2), math.sin(2)],
                               atol=1e-15)
    # composing two shifts is one shift by the sum (rotation angles add)
    a = O.apply_rope(O.apply_rope(x, [5] * 4, 500.0, round_out=False), [6] * 4, 500.0, round_out=False)
    np.testing.assert_allclose(a, O.apply_rope(x, [11] * 4, 500.0, round_out=False), atol=1e-12)


def test_rope_scores_depend_on_relative_position_only():
    """q_m . k_n after rotation depends on m - n only (the point of the embedding)."""
    rng = np.random.default_rng(23)
    D = 32
    q = rng.standard_normal((1, 1, D))
    k = rng.standard_normal((1, 1, D))
    dots = []
    for m, n in [(10, 3), (17, 10), (507, 500)]:
        qm = O.apply_rope(q, [m], 1e4, round_out=False)[0, 0]
        kn = O.apply_rope(k, [n], 1e4, round_out=False)[0, 0]
        dots.append(float(qm @ kn))
    np.testing.assert_allclose(dots, dots[0], rtol=0, atol=1e-11)
    # and a different offset gives a different score
    q0 = O.apply_rope(q, [4], 1e4, round_out=False)[0, 0]
    k0 = O.apply_rope(k, [0], 1e4, round_out=False)[0, 0]
    assert abs(float(q0 @ k0) - dots[0]) > 1e-6


def test_decoder_layer_rope_rotates_self_qk_only():
    """With RoPE the layer equals the plain layer run on rotated Q/K weights' outputs:
    checked by rotating the oracle's own projections and comparing attention inputs."""
    import synthetic
    qy = synthetic.make_query("tiny", layers=1, hidden=64, n_docs=1)
    w = qy.weights
    enc = O.bf16_bits_to_f64(qy.enc)
    x0 = O.bf16_bits_to_f64(qy.x0)
    pooled, _ = O.chunk_pool(enc, [0], [enc.shape[0]], 4)
    args = (O.bf16_bits_to_f64(w.w_qkv[0]), O.bf16_bits_to_f64(w.w_o[0]), O.bf16_bits_to_f64(w.w_kv_cross[0]),
            qy.n_q, qy.n_kv, qy.head_dim, 1 / 16)
    tr = {}
    O.decoder_layer(x0, pooled, *args, trace=tr, rope_theta=1e4)
    tr0 = {}
    O.decoder_layer(x0, pooled, *args, trace=tr0)
    D, nq, nkv, Lq = qy.head_dim, qy.n_q, qy.n_kv, x0.shape[0]
    qkv_rot, qkv = tr["layers"][0]["qkv"], tr0["layers"][0]["qkv"]
    want = O.apply_rope(qkv[:, :(nq + nkv) * D].reshape(Lq, nq + nkv, D), np.arange(Lq), 1e4).reshape(Lq, -1)
    np.testing.assert_array_equal(qkv_rot[:, :(nq + nkv) * D], want)
    np.testing.assert_array_equal(qkv_rot[:, (nq + nkv) * D:], qkv[:, (nq + nkv) * D:])   # V untouched
    np.testing.assert_array_equal(tr["layers"][0]["kv_cross"], tr0["layers"][0]["kv_cross"])  # cross untouched
