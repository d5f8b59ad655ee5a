"""Pins the fp64 CPU oracle to things other than itself (CPU only).

* hand-derived worked examples (tests/golden/*.json, each with its citation and derivation);
* an independent unrolled closed form on tiny inputs (oracle/brute.py, quadratic form);
* the TopK = M limit against a masked-matrix gated-linear-attention form;
* the one-hot cyclic router limit against the sliding-window closed form;
* TopK against a stable library sort, with constructed ties, signed zeros and saturating logits;
* sigmoid scores against scipy's expit; the router variants (softmax over the row, scores
  normalised over the TopK set) against scipy's softmax/expit and numpy sums, a hand-derived
  example and the quadratic form; selection counts against a bincount of a library sort;
* the invariant that unselected slots keep their bits;
* the backward (gradients of the recurrence) against central finite differences of the forward;
* mutants of the oracle (planted mistakes, compiled on the CPU) must fail these pins.
"""
import ctypes
import json
import math
import os
import subprocess

import numpy as np
import pytest
from scipy.special import expit

from oracle import brute, oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_stream(rng, T, M, Dv, per_slot, fscale=1.0):
    q = rng.standard_normal((T, M)).astype(np.float32)
    k = rng.standard_normal((T, M)).astype(np.float32)
    v = rng.standard_normal((T, Dv)).astype(np.float32)
    lg = rng.standard_normal((T, M)).astype(np.float32)
    shape = (T, M) if per_slot else (T,)
    f = (-np.log1p(np.exp(rng.standard_normal(shape))) * fscale).astype(np.float32)
    return q, k, v, lg, f


def _fwd1(q, k, v, lg, f, K, H0=None):
    """Run the C oracle on one (b,h) stream."""
    out = oracle.forward(q[None, :, None], k[None, :, None], v[None, :, None], lg[None, :, None],
                         f[None, :, None], K, None if H0 is None else H0[None, None], nthreads=1)
    return out["o"][0, :, 0], out["HT"][0, 0], out["idx"][0, :, 0], out["score"][0, :, 0]


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(np.square(b))), 1e-300))


# ----------------------------------------------------------------------------- golden


def test_golden_head_decay():
    g = json.load(open(os.path.join(GOLDEN, "hand_head_decay_M2.json")))
    q, k, v, lg = (np.array(g[n], np.float32) for n in ("q", "k", "v", "logits"))
    f = np.array(g["f"], np.float32)
    o, HT, idx, score = _fwd1(q, k, v, lg, f, g["K"])
    assert np.array_equal(idx, np.array(g["expect_idx"]))
    assert np.allclose(o, np.array(g["expect_o"]), atol=g["tol"], rtol=0)
    assert np.allclose(HT, np.array(g["expect_HT"]), atol=g["tol"], rtol=0)
    assert np.allclose(score, np.array(g["expect_score"]), atol=1e-12)


def test_golden_slot_decay():
    g = json.load(open(os.path.join(GOLDEN, "hand_slot_decay_M3.json")))
    q, k, v, lg = (np.array(g[n], np.float32) for n in ("q", "k", "v", "logits"))
    f = np.full(lg.shape, -1.0, np.float32)
    for t, row in enumerate(g["f_slot_targets"]):
        for i, target in enumerate(row):
            if target is not None:
                f[t, i] = math.log(target) / expit(float(lg[t, i]))
    H0 = np.array(g["H0"], np.float64)
    o, HT, idx, _ = _fwd1(q, k, v, lg, f, g["K"], H0)
    assert np.array_equal(idx, np.array(g["expect_idx"]))
    assert np.allclose(o, np.array(g["expect_o"]), atol=g["tol"], rtol=0)
    assert np.allclose(HT, np.array(g["expect_HT"]), atol=g["tol"], rtol=0)


# ----------------------------------------------------------------------------- TopK


def _topk_rows():
    rng = np.random.default_rng(11)
    rows = [rng.standard_normal(64).astype(np.float32) for _ in range(50)]
    rows += [(np.round(4 * rng.standard_normal(64)) / 4).astype(np.float32) for _ in range(50)]
    rows.append(np.zeros(64, np.float32))                              # all equal -> 0..K-1
    z = np.zeros(64, np.float32)
    z[::2] = -0.0                                                      # signed zeros tie
    rows.append(z)
    big = (20 + rng.standard_normal(64)).astype(np.float32)           # sigmoid saturates here
    rows.append(big)
    near = np.full(64, 1.5, np.float32)
    bump = rng.random(64) < 0.5
    near[bump] = np.nextafter(np.float32(1.5), np.float32(2.0))
    rows.append(near)                                                  # one-ulp differences
    return np.stack(rows)


@pytest.mark.parametrize("K", [1, 5, 16, 63, 64])
def test_topk_matches_stable_library_sort(K):
    rows = _topk_rows()
    idx, score = oracle.route(rows, K)
    assert np.array_equal(idx, brute.topk_stable(rows, K))


def test_topk_tie_rules():
    idx, _ = oracle.route(np.zeros((1, 32), np.float32), 7)
    assert list(idx[0]) == list(range(7))                             # all-equal row
    row = np.array([0.0, -0.0, 0.0, -0.0] + [-1.0] * 28, np.float32)
    idx, _ = oracle.route(row[None], 3)
    assert list(idx[0]) == [0, 1, 2]                                  # -0.0 == +0.0
    row = np.full(32, 30.0, np.float32)
    row[5] = np.nextafter(np.float32(30.0), np.float32(31.0))
    idx, score = oracle.route(row[None], 2)
    assert list(idx[0]) == [5, 0]                                     # order by logit, not score
    assert score[0, 0] == score[0, 1] or abs(score[0, 0] - score[0, 1]) < 1e-12


def test_scores_match_expit():
    rows = _topk_rows()
    idx, score = oracle.route(rows, 16)
    ref = expit(np.take_along_axis(rows.astype(np.float64), idx, axis=1))
    assert np.max(np.abs(score - ref)) < 1e-15


# ----------------------------------------------------------------------------- recurrence


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("K", [1, 3, 8])
@pytest.mark.parametrize("per_slot", [False, True])
def test_recurrence_matches_quadratic_form(seed, K, per_slot):
    rng = np.random.default_rng(100 + seed)
    T, M, Dv = 9, 8, 3
    q, k, v, lg, f = _rand_stream(rng, T, M, Dv, per_slot)
    H0 = rng.standard_normal((M, Dv)) if seed % 2 else None
    o, HT, idx, _ = _fwd1(q, k, v, lg, f, K, H0)
    ob, HTb = brute.quadratic_form(q, k, v, lg, f, K, H0)
    assert _rel(o, ob) < 1e-12
    assert _rel(HT, HTb) < 1e-12
    assert np.array_equal(idx, brute.topk_stable(lg, K))


@pytest.mark.parametrize("per_slot", [False, True])
def test_dense_limit_is_gated_linear_attention(per_slot):
    rng = np.random.default_rng(7)
    T, M, Dv = 12, 6, 4
    q, k, v, lg, f = _rand_stream(rng, T, M, Dv, per_slot, fscale=0.3)
    H0 = rng.standard_normal((M, Dv))
    o, HT, _, _ = _fwd1(q, k, v, lg, f, M, H0)
    od, HTd = brute.dense_masked_form(q, k, v, lg, f, H0)
    assert _rel(o, od) < 1e-10
    assert _rel(HT, HTd) < 1e-10


def test_window_limit_is_sliding_window():
    rng = np.random.default_rng(3)
    T, M, Dv = 40, 8, 5
    q = rng.standard_normal((T, M)).astype(np.float32)
    v = rng.standard_normal((T, Dv)).astype(np.float32)
    k = np.ones((T, M), np.float32)
    lg = np.zeros((T, M), np.float32)
    lg[np.arange(T), np.arange(T) % M] = 10.0
    f = np.full((T,), -1e4, np.float32)
    o, HT, idx, _ = _fwd1(q, k, v, lg, f, 1)
    ow, HTw = brute.window_form(q, v, M)
    assert np.array_equal(idx[:, 0], np.arange(T) % M)
    assert _rel(o, ow) < 1e-12
    assert _rel(HT, HTw) < 1e-12


def test_unselected_rows_keep_bits():
    rng = np.random.default_rng(5)
    T, M, Dv = 30, 16, 4
    q, k, v, lg, f = _rand_stream(rng, T, M, Dv, False)
    lg[:, M // 2:] = -100.0
    H0 = rng.standard_normal((M, Dv))
    _, HT, idx, _ = _fwd1(q, k, v, lg, f, 4, H0)
    assert idx.max() < M // 2
    assert np.array_equal(HT[M // 2:].view(np.uint64), H0[M // 2:].view(np.uint64))


def test_decode_step_is_one_token_forward():
    rng = np.random.default_rng(9)
    B, H, M, Dv, K = 2, 3, 8, 4, 3
    q = rng.standard_normal((B, H, M)).astype(np.float32)
    k = rng.standard_normal((B, H, M)).astype(np.float32)
    v = rng.standard_normal((B, H, Dv)).astype(np.float32)
    lg = rng.standard_normal((B, H, M)).astype(np.float32)
    f = -np.abs(rng.standard_normal((B, H))).astype(np.float32)
    st = rng.standard_normal((B, H, M, Dv))
    out = oracle.decode_step(q, k, v, lg, f, K, st)
    for b in range(B):
        for h in range(H):
            ob, HTb = brute.quadratic_form(q[b, h][None], k[b, h][None], v[b, h][None],
                                           lg[b, h][None], f[b, h][None], K, st[b, h])
            assert _rel(out["o"][b, h][None], ob) < 1e-12
            assert _rel(out["state"][b, h], HTb) < 1e-12


def test_split_sequence_resumes():
    rng = np.random.default_rng(13)
    T, M, Dv = 50, 16, 8
    q, k, v, lg, f = _rand_stream(rng, T, M, Dv, True)
    o, HT, _, _ = _fwd1(q, k, v, lg, f, 4)
    o1, H1, _, _ = _fwd1(q[:17], k[:17], v[:17], lg[:17], f[:17], 4)
    o2, H2, _, _ = _fwd1(q[17:], k[17:], v[17:], lg[17:], f[17:], 4, H1)
    assert np.array_equal(np.concatenate([o1, o2]), o)
    assert np.array_equal(H2, HT)


def test_threads_do_not_change_results():
    rng = np.random.default_rng(21)
    B, T, H, M, Dv = 3, 20, 5, 16, 8
    x = {n: rng.standard_normal(s).astype(np.float32) for n, s in
         dict(q=(B, T, H, M), k=(B, T, H, M), v=(B, T, H, Dv), logits=(B, T, H, M)).items()}
    f = -np.abs(rng.standard_normal((B, T, H))).astype(np.float32)
    a = oracle.forward(x["q"], x["k"], x["v"], x["logits"], f, 4, nthreads=1)
    b = oracle.forward(x["q"], x["k"], x["v"], x["logits"], f, 4, nthreads=4)
    assert np.array_equal(a["o"], b["o"]) and np.array_equal(a["HT"], b["HT"])


# ----------------------------------------------------------------------------- router variants


ROUTER_NAMES = ["sigmoid", "softmax", "sigmoid_norm", "softmax_norm"]


@pytest.mark.parametrize("router", ROUTER_NAMES)
def test_golden_router_variants(router):
    g = json.load(open(os.path.join(GOLDEN, "hand_router_variants_M3.json")))
    q, k, v, lg = (np.array(g[n], np.float32) for n in ("q", "k", "v", "logits"))
    H0 = np.array(g["H0"], np.float64)
    s_hand = g["expect_scores"][router]
    f = np.array([[math.log(g["decay_targets"][0]) / s_hand[0], math.log(g["decay_targets"][1]) / s_hand[1], -1.0]],
                 np.float32)
    out = oracle.forward(q[None, :, None], k[None, :, None], v[None, :, None], lg[None, :, None], f[None, :, None],
                         g["K"], H0[None, None], nthreads=1, router=router, want_counts=True)
    assert np.array_equal(out["idx"][0, :, 0], np.array(g["expect_idx"]))
    assert np.allclose(out["score"][0, 0, 0], s_hand, atol=g["tol"], rtol=0)
    assert np.allclose(out["o"][0, :, 0], g["expect_o"], atol=g["tol"], rtol=0)
    assert np.allclose(out["HT"][0, 0], g["expect_HT"], atol=g["tol"], rtol=0)
    assert np.array_equal(out["counts"][0, 0], g["expect_counts"])
    idx, sc = oracle.route(lg, g["K"], router)
    assert np.allclose(sc[0], s_hand, atol=g["tol"], rtol=0)


@pytest.mark.parametrize("router", ROUTER_NAMES)
@pytest.mark.parametrize("M,K", [(8, 3), (32, 8), (64, 64)])
def test_router_scores_match_library(router, M, K):
    rng = np.random.default_rng(M + K)
    lg = (3 * rng.standard_normal((50, M))).astype(np.float32)
    lg[5] = 0.0                                   # all tied
    idx, sc = oracle.route(lg, K, router)
    sel, ref = brute.router_scores(lg, K, router)
    assert np.array_equal(idx, brute.topk_stable(lg, K))
    assert np.allclose(sc, np.take_along_axis(ref, idx.astype(np.int64), axis=1), rtol=1e-13, atol=0)
    if router.endswith("_norm"):
        assert np.allclose(sc.sum(axis=1), 1.0, rtol=1e-13)


@pytest.mark.parametrize("router", ROUTER_NAMES)
@pytest.mark.parametrize("per_slot", [False, True])
def test_router_variants_match_quadratic_form(router, per_slot):
    rng = np.random.default_rng(7 + per_slot)
    T, M, Dv, K = 9, 6, 3, 2
    q, k, v, lg, f = _rand_stream(rng, T, M, Dv, per_slot)
    H0 = rng.standard_normal((M, Dv))
    out = oracle.forward(q[None, :, None], k[None, :, None], v[None, :, None], lg[None, :, None], f[None, :, None],
                         K, H0[None, None], nthreads=1, router=router)
    o_b, HT_b = brute.quadratic_form(q, k, v, lg, f, K, H0, router=router)
    assert _rel(out["o"][0, :, 0], o_b) <= 1e-12
    assert _rel(out["HT"][0, 0], HT_b) <= 1e-12


def test_selection_counts_match_bincount():
    rng = np.random.default_rng(3)
    B, T, H, M, Dv, K = 2, 40, 3, 16, 4, 5
    x = {n: rng.standard_normal(sh).astype(np.float32) for n, sh in
         dict(q=(B, T, H, M), k=(B, T, H, M), v=(B, T, H, Dv), logits=(B, T, H, M)).items()}
    x["logits"][0, :7] = np.round(x["logits"][0, :7])   # exact ties
    f = -np.abs(rng.standard_normal((B, T, H))).astype(np.float32)
    out = oracle.forward(x["q"], x["k"], x["v"], x["logits"], f, K, want_counts=True)
    for b in range(B):
        for h in range(H):
            assert np.array_equal(out["counts"][b, h], brute.selection_counts(x["logits"][b, :, h], K))
    assert int(out["counts"].sum()) == B * T * H * K


# ----------------------------------------------------------------------------- mutants

# Each mutant plants one plausible mistake in a copy of the oracle source (compiled here, on the
# CPU, into a scratch directory). The pins above must notice every one of them.
MUTANTS = {
    "read_before_write": ("if (J->o) {", "if (0) {", "for (int r = 0; r < K; ++r) {",
                          "if (J->o) { double* o0 = J->o + row * Dv; for (int d = 0; d < Dv; ++d) o0[d] = 0.0;"
                          " for (int i = 0; i < M; ++i) { const double* Si = S + (size_t)i * Dv;"
                          " for (int d = 0; d < Dv; ++d) o0[d] += (double)q[i] * Si[d]; } }\n"
                          "    for (int r = 0; r < K; ++r) {"),
    "tie_to_higher_index": ("return a < b;", "return a > b;", None, None),
    "decay_without_score": ("const double a = exp(s * f);", "const double a = exp(f);", None, None),
    "write_without_one_minus_a": ("const double wk = (1.0 - a) * (double)k[i];",
                                  "const double wk = (double)k[i];", None, None),
    "q_k_swapped_in_read": ("const double qi = (double)q[i];", "const double qi = (double)k[i];",
                            None, None),
    "softmax_over_selected_only": ("for (int j = 0; j < M; ++j) z += exp((double)row[j] - mx);",
                                   "for (int j = 0; j < K; ++j) z += exp((double)row[sel[j]] - mx);", None, None),
    "normalise_by_first_score": ("for (int r = 0; r < K; ++r) sum += s[r];", "sum = s[0];", None, None),
    "counts_by_rank": ("J->counts[(size_t)pair * M + i] += 1;", "J->counts[(size_t)pair * M + r] += 1;",
                       None, None),
    "backward_decay_grad_without_write_term": ("const double da = dap - (double)k[i] * dw;",
                                               "const double da = dap;", None, None),
    "backward_state_grad_not_decayed": ("        Gi[d] *= a;\n", "        Gi[d] *= 1.0;\n", None, None),
    "backward_slot_decay_grad_without_score": ("J->df[row * M + i] = s * dlam;", "J->df[row * M + i] = dlam;",
                                               None, None),
}


def _build_mutant(tmp_path, name):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "rsm_oracle.c")).read()
    a, b, c, d = MUTANTS[name]
    assert a in src
    src = src.replace(a, b, 1)
    if c is not None:
        assert c in src
        src = src.replace(c, d, 1)
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src)
    so = tmp_path / f"mut_{name}.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-o", str(so),
                           str(path), "-lm"])
    return str(so)


def _pins_pass_with(lib_path) -> bool:
    saved = oracle._lib
    try:
        oracle._lib = oracle.bind(ctypes.CDLL(lib_path))
        for fn, args in [(test_golden_head_decay, ()), (test_golden_slot_decay, ()),
                         (test_golden_router_variants, ("softmax",)),
                         (test_golden_router_variants, ("sigmoid_norm",)),
                         (test_selection_counts_match_bincount, ()),
                         (test_backward_matches_finite_differences, (False,)),
                         (test_backward_matches_finite_differences, (True,)),
                         (test_topk_tie_rules, ()), (test_window_limit_is_sliding_window, ()),
                         (test_recurrence_matches_quadratic_form, (1, 3, True)),
                         (test_recurrence_matches_quadratic_form, (2, 3, False))]:
            try:
                fn(*args)
            except AssertionError:
                return False
        return True
    finally:
        oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(tmp_path, name):
    assert not _pins_pass_with(_build_mutant(tmp_path, name))


def test_pins_pass_with_the_real_oracle():
    assert _pins_pass_with(oracle.build())


# ----------------------------------------------------------------------------- backward


def _separated_logits(rng, T, M):
    """Logits whose neighbours differ by at least 0.25, so that a 2^-10 step never changes TopK."""
    base = np.arange(M, dtype=np.float64) * 0.25
    return np.stack([rng.permutation(base) for _ in range(T)]).astype(np.float32) - 0.7


def _fd_case(per_slot, seed):
    rng = np.random.default_rng(seed)
    T, M, Dv, K = 6, 6, 3, 2
    q = rng.standard_normal((1, T, 1, M)).astype(np.float32)
    k = rng.standard_normal((1, T, 1, M)).astype(np.float32)
    v = rng.standard_normal((1, T, 1, Dv)).astype(np.float32)
    lg = _separated_logits(rng, T, M)[None, :, None]
    fs = (1, T, 1, M) if per_slot else (1, T, 1)
    f = (-0.2 - np.abs(rng.standard_normal(fs))).astype(np.float32)
    H0 = rng.standard_normal((1, 1, M, Dv))
    dO = rng.standard_normal((1, T, 1, Dv))
    dHT = rng.standard_normal((1, 1, M, Dv))
    return dict(q=q, k=k, v=v, logits=lg, f=f, H0=H0), dO, dHT, K


def _loss(x, dO, dHT, K):
    out = oracle.forward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, x["H0"], want_idx=False, nthreads=1)
    return float(np.sum(out["o"] * dO) + np.sum(out["HT"] * dHT))


@pytest.mark.parametrize("per_slot", [False, True])
def test_backward_matches_finite_differences(per_slot):
    """Every gradient component against a central difference of the forward oracle, with a step of
    2^-10 that is exact in fp32 and never moves the TopK cut."""
    x, dO, dHT, K = _fd_case(per_slot, 11 + per_slot)
    g = oracle.backward(x["q"], x["k"], x["v"], x["logits"], x["f"], K, dO=dO, dHT=dHT, H0=x["H0"], nthreads=1)
    eps = 2.0 ** -10
    names = {"q": "dq", "k": "dk", "v": "dv", "logits": "dlogits", "f": "df", "H0": "dH0"}
    for name, gname in names.items():
        base = x[name]
        fd = np.zeros(base.shape)
        for idx in np.ndindex(base.shape):
            xp = {n: a.copy() for n, a in x.items()}
            xm = {n: a.copy() for n, a in x.items()}
            xp[name][idx] += eps
            xm[name][idx] -= eps
            fd[idx] = (_loss(xp, dO, dHT, K) - _loss(xm, dO, dHT, K)) / (2 * eps)
        scale = max(np.max(np.abs(fd)), 1e-12)
        assert np.max(np.abs(g[gname] - fd)) <= 2e-5 * scale, (name, np.max(np.abs(g[gname] - fd)), scale)


def test_backward_unselected_logits_and_keys_get_no_gradient():
    rng = np.random.default_rng(5)
    T, M, Dv, K = 9, 8, 4, 3
    q, k, lg = (rng.standard_normal((1, T, 1, M)).astype(np.float32) for _ in range(3))
    v = rng.standard_normal((1, T, 1, Dv)).astype(np.float32)
    f = -np.abs(rng.standard_normal((1, T, 1))).astype(np.float32)
    g = oracle.backward(q, k, v, lg, f, K, dO=rng.standard_normal((1, T, 1, Dv)), nthreads=1)
    sel = np.zeros((T, M), bool)
    np.put_along_axis(sel, brute.topk_stable(lg[0, :, 0], K).astype(np.int64), True, axis=1)
    assert np.all(g["dk"][0, :, 0][~sel] == 0.0) and np.all(g["dlogits"][0, :, 0][~sel] == 0.0)
