"""Pins of the CPU oracle against facts that do not come from the oracle itself.

The pages print no worked example of the chunked-SGMV pair, so the oracle is
pinned by (a) the IEEE codecs of torch and numpy, (b) a float64 brute force
written token-major (the oracle is segment-major), (c) closed forms with
one-hot inputs whose result is a single entry of A or B, (d) the library
matmul in the single-adapter, identity-permutation case (the fast_lora case of
the ms-swift page, section "Compatibility checks"), and (e) invariants:
linearity in x, relabelling of tokens, splitting a segment, zero scaling,
empty segments and the write set.  Each pin is chosen so that a dropped term,
a swapped index or a transposed operand in the oracle breaks at least one.
"""
import numpy as np
import pytest

import oracle
from scatter_gemm_b200.workloads import (CONFIGS, NAN_BITS, from_bits, make_base_weight,
                                         make_problem, to_bits)

# ----------------------------------------------------------------------------
# helpers: an independent float64 brute force, token-major
# ----------------------------------------------------------------------------


def dense_reference(p, in_r64=None, x_bits=None):
    """Returns (shrink64 [tok, S*rs] NaN where unwritten, delta64 [tok, ld_base]).

    Loops over ORIGINAL tokens t, finds the sorted position i with the inverse
    permutation and the segment with a search; the per-token update is the
    dense product A_a x_t followed by B_a h scaled (sgl-kernel-xpu page,
    section "Summary").  `in_r64` replaces the rank activations fed to the
    expand (default: the problem's in_r)."""
    xb = p.x if x_bits is None else x_bits
    X = from_bits(xb, p.dtype).astype(np.float64)[:, : p.K]
    A = from_bits(p.A, p.dtype).astype(np.float64)
    Bm = from_bits(p.B, p.dtype).astype(np.float64)
    R = from_bits(p.in_r, p.dtype).astype(np.float64) if in_r64 is None else in_r64
    inv = np.empty(p.tok, dtype=np.int64)
    inv[p.permutation] = np.arange(p.tok)
    sh = np.full((p.tok, p.S * p.rs), np.nan)
    delta = np.zeros((p.tok, p.ld_base))
    off = p.slice_offsets
    for t in range(p.tok):
        i = inv[t]
        s = int(np.searchsorted(p.seg_indptr, i, side="right")) - 1
        if s < 0 or s >= p.nseg or i >= p.seg_indptr[-1]:
            continue
        a = int(p.weight_indices[s])
        for q in range(p.S):
            sh[i, q * p.rs: q * p.rs + p.r] = A[a, q * p.rs: q * p.rs + p.r, :] @ X[t]
            if p.scalings[a] == 0.0:
                continue
            cols = np.arange(off[q], off[q + 1])
            Bq = Bm[a, cols - off[0], : p.r]
            h = R[i, q * p.rs: q * p.rs + p.r]
            delta[t, cols] = float(p.scalings[a]) * (Bq @ h)
    return sh, delta


def unit_roundoff(dtype):
    return 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11


def tiny_problem(seed, dtype="bf16", **over):
    kw = dict(tok=13, K=37, slices=[5, 3], L=3, r=3, rs=4, nseg=4, recipe="random",
              scaling="uniform", dtype=dtype, col_lead=2, ld_pad=3)
    kw.update(over)
    return make_problem("tiny", seed=seed, **kw)


# ----------------------------------------------------------------------------
# (a) element codecs
# ----------------------------------------------------------------------------


def test_bf16_decode_every_pattern_matches_torch():
    L = oracle.lib()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = from_bits(bits, "bf16")
    got = np.array([L.oracle_decode(int(b), 0) for b in bits], dtype=np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def test_fp16_decode_every_pattern_matches_numpy():
    L = oracle.lib()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    want = bits.view(np.float16).astype(np.float32)
    got = np.array([L.oracle_decode(int(b), 1) for b in bits], dtype=np.float32)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


def _encode_cases(rng):
    raw = rng.integers(0, 2 ** 32, size=30000, dtype=np.uint64).astype(np.uint32)
    vals = raw.view(np.float32)
    # exact ties between neighbouring bf16 values and between fp16 values
    m = rng.integers(0, 2 ** 7, size=2000).astype(np.float32)
    e = rng.integers(-20, 20, size=2000).astype(np.float32)
    ties16 = ((1.0 + (m + 0.5) / 2 ** 7) * np.exp2(e)).astype(np.float32)
    m2 = rng.integers(0, 2 ** 10, size=2000).astype(np.float32)
    e2 = rng.integers(-24, 15, size=2000).astype(np.float32)
    ties_h = ((1.0 + (m2 + 0.5) / 2 ** 10) * np.exp2(e2)).astype(np.float32)
    special = np.array([0.0, -0.0, np.inf, -np.inf, np.nan, 65504.0, 65520.0, 65519.0,
                        6.1e-5, 5.96e-8, 2.98e-8, 1e-40, -1e-40, 3.3895e38, 3.4e38],
                       dtype=np.float32)
    small = rng.standard_normal(5000).astype(np.float32) * np.float32(1e-6)
    return np.concatenate([vals, ties16, -ties16, ties_h, -ties_h, special, small])


def test_bf16_encode_matches_torch():
    L = oracle.lib()
    vals = _encode_cases(np.random.default_rng(1))
    want = to_bits(vals, "bf16")
    got = np.array([L.oracle_encode(float(v), 0) for v in vals], dtype=np.uint16)
    wf, gf = from_bits(want, "bf16"), from_bits(got, "bf16")
    nan = np.isnan(wf)
    assert np.array_equal(np.isnan(gf), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_fp16_encode_matches_numpy():
    L = oracle.lib()
    vals = _encode_cases(np.random.default_rng(2))
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([L.oracle_encode(float(v), 1) for v in vals], dtype=np.uint16)
    nan = np.isnan(want.view(np.float16))
    assert np.array_equal(np.isnan(got.view(np.float16)), nan)
    assert np.array_equal(got[~nan], want[~nan])


def test_encode_f64_rounds_once():
    """1 + 2^-8 + 2^-40 lies just above the bf16 tie between 1 and 1 + 2^-7:
    one rounding gives 1 + 2^-7 (0x3F81); rounding through fp32 first would
    drop the 2^-40 and tie to even (0x3F80)."""
    L = oracle.lib()
    d = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert L.oracle_encode_f64(d, 0) == 0x3F81
    assert L.oracle_encode(float(np.float32(d)), 0) == 0x3F80
    d16 = 1.0 + 2.0 ** -11 + 2.0 ** -40
    assert L.oracle_encode_f64(d16, 1) == 0x3C01


# ----------------------------------------------------------------------------
# (b) brute force on tiny inputs
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_shrink_matches_token_major_brute_force(seed, dtype):
    p = tiny_problem(seed, dtype, lead=2, trail=1)
    sh64, _ = dense_reference(p)
    got64 = oracle.shrink_problem(p, mode=oracle.F64)
    written = ~np.isnan(sh64)
    assert np.array_equal(~np.isnan(got64), written)
    np.testing.assert_allclose(got64[written], sh64[written], rtol=1e-12, atol=1e-12)

    got = oracle.shrink_problem(p, mode=oracle.F32)
    gotf = from_bits(got, dtype).astype(np.float64)
    X = np.abs(from_bits(p.x, dtype).astype(np.float64)[:, : p.K])
    A = np.abs(from_bits(p.A, dtype).astype(np.float64))
    u = unit_roundoff(dtype)
    for i in np.argwhere(written.any(axis=1)).ravel():
        s = int(np.searchsorted(p.seg_indptr, i, side="right")) - 1
        a = p.weight_indices[s]
        mag = A[a] @ X[p.permutation[i]]
        cols = np.flatnonzero(written[i])
        bound = u * np.abs(sh64[i, cols]) + 2 * p.K * 2.0 ** -24 * mag[cols] + 1e-30
        assert np.all(np.abs(gotf[i, cols] - sh64[i, cols]) <= bound)
    # nothing outside the written set changed from its sentinel
    assert np.all(got[~written] == 0x7FFF)


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_expand_matches_token_major_brute_force(seed, dtype):
    p = tiny_problem(seed, dtype, lead=1, trail=2)
    _, delta = dense_reference(p)
    base64 = from_bits(p.base, dtype).astype(np.float64)
    got64 = oracle.expand_problem(p, mode=oracle.F64)
    np.testing.assert_allclose(got64, base64 + delta, rtol=1e-12, atol=1e-12)

    got = from_bits(oracle.expand_problem(p, mode=oracle.F32), dtype).astype(np.float64)
    want = base64 + delta
    u = unit_roundoff(dtype)
    R = np.abs(from_bits(p.in_r, dtype).astype(np.float64))
    Bm = np.abs(from_bits(p.B, dtype).astype(np.float64))
    inv = np.empty(p.tok, dtype=np.int64)
    inv[p.permutation] = np.arange(p.tok)
    for t in range(p.tok):
        i = inv[t]
        s = int(np.searchsorted(p.seg_indptr, i, side="right")) - 1
        if s < 0 or s >= p.nseg or i >= p.seg_indptr[-1]:
            assert np.array_equal(got[t], base64[t])
            continue
        a = p.weight_indices[s]
        for q in range(p.S):
            cols = np.arange(p.slice_offsets[q], p.slice_offsets[q + 1])
            mag = Bm[a, cols - p.slice_offsets[0], : p.r] @ R[i, q * p.rs: q * p.rs + p.r]
            mag = p.scalings[a] * mag
            bound = (u * np.abs(want[t, cols])
                     + 2 * (p.r + 2) * 2.0 ** -24 * (mag + np.abs(base64[t, cols])) + 1e-30)
            assert np.all(np.abs(got[t, cols] - want[t, cols]) <= bound)


# ----------------------------------------------------------------------------
# (c) closed forms: one-hot inputs pick single entries (bit exact)
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_shrink_one_hot_x_picks_column_of_A(dtype):
    """x_t = e_{k(t)}  =>  out_r[i, q*rs+j] = A[a, q*rs+j, k(perm[i])] exactly."""
    p = tiny_problem(7, dtype, K=29)
    rng = np.random.default_rng(7)
    k_of = rng.integers(0, p.K, size=p.tok)
    xf = np.zeros((p.tok, p.ld_x), dtype=np.float32)
    xf[np.arange(p.tok), k_of] = 1.0
    got = oracle.shrink_problem(p, x=to_bits(xf, dtype))
    for s in range(p.nseg):
        a = p.weight_indices[s]
        for i in range(p.seg_indptr[s], p.seg_indptr[s + 1]):
            t = p.permutation[i]
            for q in range(p.S):
                for j in range(p.r):
                    assert got[i, q * p.rs + j] == p.A[a, q * p.rs + j, k_of[t]]
            for q in range(p.S):
                assert np.all(got[i, q * p.rs + p.r:(q + 1) * p.rs] == 0x7FFF)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_expand_one_hot_rank_picks_column_of_B(dtype):
    """in_r[i, q*rs + j(q)] = 1, other valid ranks 0, base = 0, scaling = 2
    =>  base[perm[i], c] = 2 * B[a, c - off[0], j(q)] exactly, c in slice q."""
    p = tiny_problem(8, dtype, scaling=2.0)
    rng = np.random.default_rng(8)
    j_of = rng.integers(0, p.r, size=(p.tok, p.S))
    rf = np.full((p.tok, p.ld_r), np.nan, dtype=np.float32)
    for q in range(p.S):
        rf[:, q * p.rs: q * p.rs + p.r] = 0.0
        rf[np.arange(p.tok), q * p.rs + j_of[:, q]] = 1.0
    base0 = np.zeros_like(p.base)
    got = oracle.expand_problem(p, in_r=to_bits(rf, dtype), base=base0)
    Bf = from_bits(p.B, dtype)
    off = p.slice_offsets
    for s in range(p.nseg):
        a = p.weight_indices[s]
        for i in range(p.seg_indptr[s], p.seg_indptr[s + 1]):
            t = p.permutation[i]
            assert np.all(got[t, : off[0]] == 0)
            assert np.all(got[t, off[-1]:] == 0)
            for q in range(p.S):
                for c in range(off[q], off[q + 1]):
                    want = to_bits(np.array([2.0 * Bf[a, c - off[0], j_of[i, q]]]), dtype)[0]
                    assert got[t, c] == want


# ----------------------------------------------------------------------------
# (d) library special case: one adapter, one segment, identity permutation
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_single_adapter_identity_permutation_is_a_matmul(dtype):
    p = tiny_problem(9, dtype, tok=21, K=64, L=1, nseg=1, slices=[24, 8], r=4, rs=4,
                     scaling=0.5, col_lead=0, ld_pad=0)
    p.permutation = np.arange(p.tok, dtype=np.int32)
    p.weight_indices = np.zeros(1, dtype=np.int32)
    X = from_bits(p.x, dtype).astype(np.float64)
    A = from_bits(p.A[0], dtype).astype(np.float64)
    got = oracle.shrink_problem(p, mode=oracle.F64)
    np.testing.assert_allclose(got, X @ A.T, rtol=1e-12, atol=1e-13)

    R = from_bits(p.in_r, dtype).astype(np.float64)
    base = from_bits(p.base, dtype).astype(np.float64)
    Bm = from_bits(p.B[0], dtype).astype(np.float64)
    want = base.copy()
    want[:, 0:24] += 0.5 * (R[:, 0:4] @ Bm[0:24].T)
    want[:, 24:32] += 0.5 * (R[:, 4:8] @ Bm[24:32].T)
    got_e = oracle.expand_problem(p, mode=oracle.F64)
    np.testing.assert_allclose(got_e, want, rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------
# (e) invariants
# ----------------------------------------------------------------------------


def test_zero_scaling_leaves_base_bit_identical():
    p = tiny_problem(10, "bf16")
    sc = p.scalings.copy()
    sc[p.weight_indices[1]] = 0.0
    got = oracle.expand_problem(p, scalings=sc)
    z = np.zeros_like(sc)
    assert np.array_equal(oracle.expand_problem(p, scalings=z), p.base)
    # rows of the zero-scaled adapter are unchanged bit for bit
    for s in range(p.nseg):
        if sc[p.weight_indices[s]] != 0.0:
            continue
        for i in range(p.seg_indptr[s], p.seg_indptr[s + 1]):
            assert np.array_equal(got[p.permutation[i]], p.base[p.permutation[i]])


def test_empty_segments_and_outside_rows_write_nothing():
    p = tiny_problem(11, "bf16", lead=3, trail=4)
    p.seg_indptr = np.array([3, 3, 8, 8, p.seg_indptr[-1]], dtype=np.int32)
    sh = oracle.shrink_problem(p)
    written_rows = np.flatnonzero((sh != 0x7FFF).any(axis=1))
    assert np.array_equal(written_rows, np.arange(3, p.seg_indptr[-1]))
    ex = oracle.expand_problem(p)
    changed = np.flatnonzero((ex != p.base).any(axis=1))
    assert set(changed) <= set(p.permutation[3: p.seg_indptr[-1]])
    untouched = np.concatenate([p.permutation[:3], p.permutation[p.seg_indptr[-1]:]])
    assert np.array_equal(ex[untouched], p.base[untouched])


def test_shrink_is_linear_in_x():
    """x1 and x2 have disjoint column support, so x1 + x2 is exact in bf16."""
    p = tiny_problem(12, "bf16", K=40)
    xf = from_bits(p.x, "bf16")
    mask = (np.arange(p.ld_x) % 2 == 0)
    x1, x2 = xf * mask, xf * ~mask
    s1 = oracle.shrink_problem(p, mode=oracle.F64, x=to_bits(x1, "bf16"))
    s2 = oracle.shrink_problem(p, mode=oracle.F64, x=to_bits(x2, "bf16"))
    s12 = oracle.shrink_problem(p, mode=oracle.F64, x=to_bits(x1 + x2, "bf16"))
    w = ~np.isnan(s12)
    np.testing.assert_allclose(s12[w], (s1 + s2)[w], rtol=1e-12, atol=1e-13)
    s4 = oracle.shrink_problem(p, mode=oracle.F64, x=to_bits(4.0 * xf, "bf16"))
    assert np.array_equal(s4[w], 4.0 * s12[w])


def test_relabelling_tokens_permutes_results_exactly():
    p = tiny_problem(13, "fp16", lead=1)
    sh, ex = oracle.shrink_problem(p), oracle.expand_problem(p)
    sigma = np.random.default_rng(13).permutation(p.tok)
    q = tiny_problem(13, "fp16", lead=1)
    q.x = np.empty_like(p.x)
    q.x[sigma] = p.x
    q.base = np.empty_like(p.base)
    q.base[sigma] = p.base
    q.permutation = sigma[p.permutation].astype(np.int32)
    assert np.array_equal(oracle.shrink_problem(q), sh)
    exq = oracle.expand_problem(q)
    assert np.array_equal(exq[sigma], ex)


def test_splitting_a_segment_changes_nothing():
    p = tiny_problem(14, "bf16", nseg=2, tok=20)
    sh, ex = oracle.shrink_problem(p), oracle.expand_problem(p)
    lo, hi = p.seg_indptr[0], p.seg_indptr[1]
    assert hi - lo >= 2
    mid = (lo + hi) // 2
    p.seg_indptr = np.array([lo, mid, hi, p.seg_indptr[2]], dtype=np.int32)
    p.weight_indices = np.array([p.weight_indices[0]] * 2 + [p.weight_indices[1]],
                                dtype=np.int32)
    p.nseg = 3
    assert np.array_equal(oracle.shrink_problem(p), sh)
    assert np.array_equal(oracle.expand_problem(p), ex)


def test_shrink_then_expand_is_the_dense_lora_update():
    """Composition through sorted-order rank activations equals the per-token
    dense update s_a * B_a A_a x_t (reading: row i of out_r is token perm[i])."""
    p = tiny_problem(15, "bf16", lead=2, trail=2)
    h64 = oracle.shrink_problem(p, mode=oracle.F64)
    h64 = np.nan_to_num(h64, nan=np.nan)  # padding stays NaN: it must never be read
    got = oracle.expand_problem(p, in_r=h64, mode=oracle.F64_IN)
    X = from_bits(p.x, "bf16").astype(np.float64)[:, : p.K]
    A = from_bits(p.A, "bf16").astype(np.float64)
    Bm = from_bits(p.B, "bf16").astype(np.float64)
    want = from_bits(p.base, "bf16").astype(np.float64)
    inv = np.empty(p.tok, dtype=np.int64)
    inv[p.permutation] = np.arange(p.tok)
    off = p.slice_offsets
    for t in range(p.tok):
        i = inv[t]
        if not (p.seg_indptr[0] <= i < p.seg_indptr[-1]):
            continue
        s = int(np.searchsorted(p.seg_indptr, i, side="right")) - 1
        a = p.weight_indices[s]
        for q in range(p.S):
            W = Bm[a, off[q] - off[0]: off[q + 1] - off[0], : p.r] @ A[a, q * p.rs: q * p.rs + p.r]
            want[t, off[q]: off[q + 1]] += p.scalings[a] * (W @ X[t])
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_padding_is_never_read_on_every_workload_shape():
    """A, B and in_r carry NaN in their rank padding; every written output is finite."""
    for name in CONFIGS:
        cfg = CONFIGS[name]
        over = dict(tok=min(cfg["tok"], 70), K=min(cfg["K"], 96),
                    slices=[min(w, 40) + (w % 3) for w in cfg["slices"]],
                    nseg=min(cfg["nseg"], 9))
        p = make_problem(name, seed=3, **over)
        sh = oracle.shrink_problem(p, mode=oracle.F64)
        assert np.isfinite(sh[~np.isnan(sh)]).all()
        w = ~np.isnan(sh)
        for q in range(p.S):
            assert not w[:, q * p.rs + p.r:(q + 1) * p.rs].any()
        ex = oracle.expand_problem(p)
        assert np.isfinite(from_bits(ex, p.dtype)).all()


def test_table_checks_flag_each_kind_of_bad_table():
    tok, nseg, L, S = 10, 3, 4, 2
    si = np.array([0, 4, 7, 10], dtype=np.int32)
    wi = np.array([0, 3, 1], dtype=np.int32)
    pm = np.random.default_rng(0).permutation(tok).astype(np.int32)
    so = np.array([0, 8, 12], dtype=np.int32)
    assert oracle.check_tables(si, wi, pm, so, tok, nseg, L, S, 12) == 0
    assert oracle.check_tables(np.array([0, 5, 4, 10]), wi, pm, so, tok, nseg, L, S, 12) \
        == oracle.BAD_INDPTR
    assert oracle.check_tables(np.array([0, 4, 7, 11]), wi, pm, so, tok, nseg, L, S, 12) \
        == oracle.BAD_INDPTR
    assert oracle.check_tables(si, np.array([0, 4, 1]), pm, so, tok, nseg, L, S, 12) \
        == oracle.BAD_ADAPTER
    bad_pm = pm.copy()
    bad_pm[3] = bad_pm[4]
    assert oracle.check_tables(si, wi, bad_pm, so, tok, nseg, L, S, 12) == oracle.BAD_PERMUTATION
    assert oracle.check_tables(si, wi, pm, np.array([0, 8, 13]), tok, nseg, L, S, 12) \
        == oracle.BAD_SLICES
    assert oracle.check_tables(si, wi, pm, np.array([0, 8, 6]), tok, nseg, L, S, 12) \
        == oracle.BAD_SLICES
    assert oracle.check_tables(np.array([0, 5, 4, 10]), np.array([0, 4, 1]), bad_pm, so,
                               tok, nseg, L, S, 12) == (oracle.BAD_INDPTR | oracle.BAD_ADAPTER
                                                        | oracle.BAD_PERMUTATION)


def test_nan_sentinels_are_nan():
    for dt, bits in NAN_BITS.items():
        assert np.isnan(from_bits(np.array([bits], dtype=np.uint16), dt)[0])


# ----------------------------------------------------------------------------
# embedding variant: the shrink of one-hot rows
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("seed", range(3))
def test_embedding_a_is_the_shrink_of_one_hot_rows(seed):
    """With x_t = e_{id_t}, the shrink's out_r equals the embedding lookup (bit
    exact: each sum has one nonzero term); identity permutation, one slice."""
    rng = np.random.default_rng(seed)
    V, r, rs, L, tok = 37, 5, 8, 3, 23
    p = tiny_problem(seed, "bf16", tok=tok, K=V, slices=[8], r=r, rs=rs, L=L, nseg=4,
                     ld_pad=0, col_lead=0)
    p.permutation = np.arange(p.tok, dtype=np.int32)
    ids = rng.integers(0, V, size=p.tok).astype(np.int32)
    xf = np.zeros((p.tok, p.ld_x), dtype=np.float32)
    xf[np.arange(p.tok), ids] = 1.0
    via_shrink = oracle.shrink_problem(p, x=to_bits(xf, "bf16"))
    A_emb = p.A.reshape(L, rs, V)  # [L, S*rs, K] with S = 1 and K = V
    out = np.full((p.tok, rs), 0x7FFF, dtype=np.uint16)
    assert oracle.embedding_a(ids, A_emb, p.seg_indptr, p.weight_indices, out, rs, p.tok, V, r,
                              rs, p.nseg, L) == 0
    assert np.array_equal(out, via_shrink)
    # and directly: the adapter's column of the id
    for s in range(p.nseg):
        for i in range(p.seg_indptr[s], p.seg_indptr[s + 1]):
            assert np.array_equal(out[i, :r], A_emb[p.weight_indices[s], :r, ids[i]])


def test_embedding_a_rejects_out_of_vocabulary_ids():
    A = np.zeros((1, 4, 10), dtype=np.uint16)
    out = np.zeros((3, 4), dtype=np.uint16)
    assert oracle.embedding_a(np.array([1, 10, 2]), A, np.array([0, 3]), np.array([0]), out, 4,
                              3, 10, 4, 4, 1, 1) == oracle.BAD_DIMS


# ----------------------------------------------------------------------------
# (f) the base projection with the expand folded in
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("seed,dtype", [(40, "bf16"), (41, "fp16"), (42, "bf16")])
def test_base_expand_matches_token_major_brute_force(seed, dtype):
    p = tiny_problem(seed, dtype)
    W = make_base_weight(p, seed, ld_pad=5)
    Wd = from_bits(W[:, : p.K], dtype).astype(np.float64)
    X = from_bits(p.x, dtype).astype(np.float64)[:, : p.K]
    _, delta = dense_reference(p)
    got = oracle.base_expand_problem(p, W, mode=oracle.F64)
    off = p.slice_offsets
    inv = np.empty(p.tok, dtype=np.int64)
    inv[p.permutation] = np.arange(p.tok)
    for t in range(p.tok):
        i = inv[t]
        in_seg = p.seg_indptr[0] <= i < p.seg_indptr[-1]
        for c in range(off[0], off[-1]):
            if in_seg:
                want = X[t] @ Wd[c - off[0]] + delta[t, c]
                assert abs(got[t, c] - want) <= 1e-12 * (1 + abs(want))
            else:
                assert np.isnan(got[t, c])
    # nothing outside the slices' columns
    assert np.isnan(got[:, : off[0]]).all() and np.isnan(got[:, off[-1]:]).all()


def test_base_expand_with_zero_weight_is_the_expand_of_zeros():
    p = tiny_problem(43, "bf16")
    W = np.zeros((int(p.slice_offsets[-1] - p.slice_offsets[0]), p.K), dtype=np.uint16)
    zero_base = np.zeros_like(p.base)
    got = oracle.base_expand_problem(p, W, out=zero_base)
    want = oracle.expand_problem(p, base=zero_base)
    assert np.array_equal(got, want)


def test_base_expand_with_zero_scaling_is_the_rounded_projection():
    p = tiny_problem(44, "bf16", K=64)
    W = make_base_weight(p, 44)
    z = np.zeros_like(p.scalings)
    got = from_bits(oracle.base_expand_problem(p, W, scalings=z), "bf16").astype(np.float64)
    X = from_bits(p.x, "bf16").astype(np.float64)[:, : p.K]
    Wd = from_bits(W, "bf16").astype(np.float64)
    off = p.slice_offsets
    rows = p.permutation[p.seg_indptr[0]: p.seg_indptr[-1]]
    ref = X[rows] @ Wd.T
    mag = np.abs(X[rows]) @ np.abs(Wd).T
    # one rounding to bf16 plus fp32 accumulation over K terms
    lim = unit_roundoff("bf16") * np.abs(ref) + p.K * 2.0 ** -24 * mag + 1e-30
    assert (np.abs(got[rows][:, off[0]: off[-1]] - ref) <= lim).all()


def test_base_expand_scales_only_the_rank_term():
    p = tiny_problem(45, "bf16")
    W = make_base_weight(p, 45)
    s1 = np.ones_like(p.scalings)
    base = oracle.base_expand_problem(p, W, mode=oracle.F64, scalings=np.zeros_like(s1))
    one = oracle.base_expand_problem(p, W, mode=oracle.F64, scalings=s1)
    three = oracle.base_expand_problem(p, W, mode=oracle.F64, scalings=3 * s1)
    w = ~np.isnan(base)
    np.testing.assert_allclose((three - base)[w], 3 * (one - base)[w], rtol=1e-12, atol=1e-12)
