"""Pins for the float64 oracle: what the pages and the mathematics fix.

Every check here is independent of the oracle's own code: reductions to the
simpler members of the family coded from their own update rules, closed forms,
invariants of the erase step, exact retrieval, causal linear attention as one
masked matrix product, the pages' chunked algorithm, and library routines.

Sources (page title and section):
* "Kimi3 = GPT2 x 22580" (hubwiz translation of "22580: From GPT2 to Kimi3,
  Explained"): §2 linear attention, §3 DeltaNet / delta rule, §4 chunkwise
  DeltaNet (token loop, Householder form, WY chunk algorithm), §5 Gated
  DeltaNet, §6 KDA.
* Muir review (arXiv:2611.08376): §2.1 GDN-2 update and Muir readout, §2.4
  boundary-pivoted chunkwise kernel.
* ETH DeltaNet-family study (arXiv:2607.07953), section "Gated DeltaNet-2":
  equal erase and write gates reduce GDN-2 to KDA, and further to Gated
  DeltaNet.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import chunked as och

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _l2n(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def rand_inputs(T, dk, dv, B=1, H=1, seed=0, u=(-5.0, -1.0)):
    """float64 inputs [B,T,H,d] with the workload distributions."""
    r = np.random.default_rng(seed)
    silu = lambda x: x * _sig(x)
    d = dict(
        q=_l2n(silu(r.standard_normal((B, T, H, dk)))),
        k=_l2n(silu(r.standard_normal((B, T, H, dk)))),
        v=r.standard_normal((B, T, H, dv)),
        log_alpha=-np.exp(r.uniform(u[0], u[1], (B, T, H, dk))),
        b=2 * _sig(r.standard_normal((B, T, H, dk))),
        w=_sig(r.standard_normal((B, T, H, dv))),
        z=r.standard_normal((B, T, H, dk)),
        g=_sig(r.standard_normal((B, T, H, dv))),
        gamma_stat=np.exp(0.1 * r.standard_normal((H, dk))),
    )
    return d


def neutral_gain(d):
    """gamma_stat = 1, z = 0 (2*sigmoid(0) = 1), g = 1: readout is plain q S."""
    d = dict(d)
    d["gamma_stat"] = np.ones_like(d["gamma_stat"])
    d["z"] = np.zeros_like(d["z"])
    d["g"] = np.ones_like(d["g"])
    return d


def relerr(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-300))


def head(d, key, b_=0, h_=0):
    return d[key][b_, :, h_, :]


# --------------------------------------------------------------------------
# Reductions: GDN-2 -> KDA -> Gated DeltaNet -> DeltaNet
# --------------------------------------------------------------------------

def kda_loop(q, k, v, beta, la, S0):
    """KDA (per-channel decay) delta rule, coded from its own update:
    S <- Diag(alpha) S;  S <- S + beta k^T (v - k S);  o = q S
    ("Kimi3 = GPT2 x 22580" §3 and §6)."""
    S = S0.copy()
    out = []
    for t in range(q.shape[0]):
        S = np.exp(la[t])[:, None] * S
        u = beta[t] * (v[t] - k[t] @ S)
        S = S + np.outer(k[t], u)
        out.append(q[t] @ S)
    return np.array(out), S


@pytest.mark.parametrize("seed", [0, 1])
def test_equal_gates_reduce_to_kda(seed):
    T, dk, dv = 40, 12, 10
    d = rand_inputs(T, dk, dv, seed=seed)
    beta = np.random.default_rng(100 + seed).uniform(0.05, 0.95, T)
    d["b"] = np.repeat(beta[None, :, None, None], dk, axis=3)
    d["w"] = np.repeat(beta[None, :, None, None], dv, axis=3)
    S0 = np.random.default_rng(7).standard_normal((1, dk, dv))
    r = oracle.forward(d, S0=S0)
    qt = head(d, "q") * d["gamma_stat"][0] * 2 * _sig(head(d, "z"))
    o_ref, S_ref = kda_loop(qt, head(d, "k"), head(d, "v"), beta, head(d, "log_alpha"), S0[0])
    assert relerr(r["o_raw"][0], o_ref) < 1e-12
    assert relerr(r["S"][0], S_ref) < 1e-12


def gdn_loop(q, k, v, beta, la_scalar, S0):
    """Gated DeltaNet: one data-dependent scalar decay per token
    ("Kimi3 = GPT2 x 22580" §5): S <- a S; S <- S + beta k^T (v - k S)."""
    S = S0.copy()
    out = []
    for t in range(q.shape[0]):
        S = np.exp(la_scalar[t]) * S
        S = S + np.outer(k[t], beta[t] * (v[t] - k[t] @ S))
        out.append(q[t] @ S)
    return np.array(out), S


def test_scalar_decay_reduces_to_gated_deltanet():
    T, dk, dv = 33, 8, 8
    d = neutral_gain(rand_inputs(T, dk, dv, seed=3))
    rng = np.random.default_rng(5)
    beta = rng.uniform(0.1, 0.9, T)
    la_s = -np.exp(rng.uniform(-4, -1, T))
    d["b"] = np.repeat(beta[None, :, None, None], dk, axis=3)
    d["w"] = np.repeat(beta[None, :, None, None], dv, axis=3)
    d["log_alpha"] = np.repeat(la_s[None, :, None, None], dk, axis=3)
    r = oracle.forward(d)
    o_ref, S_ref = gdn_loop(head(d, "q"), head(d, "k"), head(d, "v"), beta, la_s,
                            np.zeros((dk, dv)))
    assert relerr(r["o_raw"][0], o_ref) < 1e-12
    assert relerr(r["S"][0], S_ref) < 1e-12
    # alpha = 0 clears the memory (§5): the state after such a step holds only
    # that token's write.
    d2 = dict(d)
    la2 = d["log_alpha"].copy()
    la2[:, 20] = -np.inf
    d2["log_alpha"] = la2
    r2 = oracle.forward({k_: (v_[:, :21] if v_.ndim == 4 else v_) for k_, v_ in d2.items()})
    kk, vv = head(d, "k")[20], head(d, "v")[20]
    assert relerr(r2["S"][0], beta[20] * np.outer(kk, vv)) < 1e-12


def deltanet_token_loop(q, k, v, beta):
    """The pages' DeltaNet prefill loop ("Kimi3 = GPT2 x 22580" §4):
    v_old = k S; u = beta (v - v_old); S = S + k^T u; o = q S."""
    S = np.zeros((k.shape[1], v.shape[1]))
    out = []
    for t in range(q.shape[0]):
        v_old = k[t] @ S
        u = beta[t] * (v[t] - v_old)
        S = S + np.outer(k[t], u)
        out.append(q[t] @ S)
    return np.array(out), S


def householder_loop(q, k, v, beta):
    """Generalised Householder form, column convention (§4):
    S_t = S_{t-1} (I - beta k k^T) + beta v k^T;  o_t = S_t q_t.  S is d_v x d_k."""
    dk, dv = k.shape[1], v.shape[1]
    S = np.zeros((dv, dk))
    out = []
    for t in range(q.shape[0]):
        S = S @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        out.append(S @ q[t])
    return np.array(out), S.T


def wy_chunk(Q, K, V, beta, C):
    """DeltaNet chunkwise WY form (§4), restated: inside a chunk the
    corrections satisfy (I + tril(K_beta K^T, -1)) u = V_beta - K_beta S, solved
    here by forward substitution; then o = Q S + tril(Q K^T) u, S += K^T u."""
    L, d = Q.shape
    dv = V.shape[1]
    S = np.zeros((d, dv))
    O = np.zeros((L, dv))
    for c0 in range(0, L, C):
        sl = slice(c0, min(c0 + C, L))
        q, k, v, bt = Q[sl], K[sl], V[sl], beta[sl]
        kb, vb = k * bt[:, None], v * bt[:, None]
        A = np.tril(kb @ k.T, -1)
        rhs = vb - kb @ S
        u = np.zeros_like(rhs)
        for i in range(len(bt)):                   # forward substitution
            u[i] = rhs[i] - A[i, :i] @ u[:i]
        O[sl] = q @ S + np.tril(q @ k.T) @ u
        S = S + k.T @ u
    return O, S


def test_unit_decay_reduces_to_deltanet():
    T, dk, dv = 50, 10, 6
    d = neutral_gain(rand_inputs(T, dk, dv, seed=11))
    beta = np.random.default_rng(2).uniform(0.05, 0.95, T)
    d["b"] = np.repeat(beta[None, :, None, None], dk, axis=3)
    d["w"] = np.repeat(beta[None, :, None, None], dv, axis=3)
    d["log_alpha"] = np.zeros_like(d["log_alpha"])
    r = oracle.forward(d)
    q, k, v = head(d, "q"), head(d, "k"), head(d, "v")
    for ref in (deltanet_token_loop(q, k, v, beta), householder_loop(q, k, v, beta),
                wy_chunk(q, k, v, beta, 16), wy_chunk(q, k, v, beta, 7)):
        assert relerr(r["o_raw"][0], ref[0]) < 1e-12
        assert relerr(r["S"][0], ref[1]) < 1e-12


# --------------------------------------------------------------------------
# Identities
# --------------------------------------------------------------------------

def test_exact_retrieval_with_orthonormal_keys():
    """Unit keys, alpha = 1, b = w = 1: reading with q = k returns the value
    just written (the delta rule replaces it); with orthonormal keys every
    earlier value stays retrievable and a rewrite replaces only its own slot
    ("Kimi3 = GPT2 x 22580" §3)."""
    dk, dv, n = 16, 8, 6
    rng = np.random.default_rng(4)
    Kq, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Kq[:, :n].T                                   # n orthonormal rows
    vals = rng.standard_normal((n, dv))
    newv = rng.standard_normal(dv)
    # tokens: write k_0..k_{n-1}; rewrite k_2 with newv; then read every key
    # with k = 0 (a pure read: no erase, no write).
    ks = np.concatenate([keys, keys[2:3], np.zeros((n, dk))])
    vs = np.concatenate([vals, newv[None], np.zeros((n, dv))])
    qs = np.concatenate([keys, keys[2:3], keys])
    T = len(ks)
    d = dict(q=qs[None, :, None], k=ks[None, :, None], v=vs[None, :, None],
             log_alpha=np.zeros((1, T, 1, dk)), b=np.ones((1, T, 1, dk)),
             w=np.ones((1, T, 1, dv)), z=np.zeros((1, T, 1, dk)),
             g=np.ones((1, T, 1, dv)), gamma_stat=np.ones((1, dk)))
    r = oracle.forward(d, eps=0.0)
    o = r["o_raw"][0]
    for i in range(n):
        assert np.max(np.abs(o[i] - vals[i])) < 1e-12       # right after writing
    assert np.max(np.abs(o[n] - newv)) < 1e-12
    expect = vals.copy()
    expect[2] = newv
    assert np.max(np.abs(o[n + 1:] - expect)) < 1e-12
    # RMSNorm with g = 1 and eps = 0 gives v / rms(v)
    y = r["y"][0][n + 1:]
    assert np.max(np.abs(y - expect / np.sqrt(np.mean(expect ** 2, 1, keepdims=True)))) < 1e-12


def test_zero_erase_is_causal_linear_attention():
    """b = 0, alpha = 1: o = causal (inclusive) (Q_til K^T) (W*V) as one masked
    matrix product ("Kimi3 = GPT2 x 22580" §2 and §4's chunked linear
    attention); gain and write gate placement included."""
    T, dk, dv = 70, 12, 9
    d = rand_inputs(T, dk, dv, seed=21)
    d["b"] = np.zeros_like(d["b"])
    d["log_alpha"] = np.zeros_like(d["log_alpha"])
    r = oracle.forward(d)
    q, k, v, w, z = (head(d, x) for x in ("q", "k", "v", "w", "z"))
    qt = q * d["gamma_stat"][0] * 2 * _sig(z)
    o_ref = np.tril(qt @ k.T) @ (w * v)
    assert relerr(r["o_raw"][0], o_ref) < 1e-12


def test_zero_erase_closed_form_with_decay():
    """b = 0: S_T = Diag(exp(sum log alpha)) S_0 + sum_s Diag(exp(Lambda_T -
    Lambda_s)) k_s^T (w_s*v_s) -- decayed linear attention (Mamba-2 style,
    §5), written out term by term."""
    T, dk, dv = 25, 7, 5
    d = rand_inputs(T, dk, dv, seed=8, u=(-3, 0))
    d["b"] = np.zeros_like(d["b"])
    S0 = np.random.default_rng(1).standard_normal((1, dk, dv))
    r = oracle.forward(d, S0=S0)
    la, k, v, w = (head(d, x) for x in ("log_alpha", "k", "v", "w"))
    lam_T = la.sum(0)
    S = np.exp(lam_T)[:, None] * S0[0]
    for s in range(T):
        S = S + np.exp(la[s + 1:].sum(0))[:, None] * np.outer(k[s], w[s] * v[s])
    assert relerr(r["S"][0], S) < 1e-12


def test_erase_gate_invariants():
    """No write (w = 0), alpha = 1, unit keys.  b = 1 makes the step the
    projection I - k^T k: afterwards k S = 0, and repeating it changes nothing.
    b = 2 makes it a reflection: it keeps the Frobenius norm and repeating it
    restores the state (Muir review §2.1: erase gate range (0, 2))."""
    dk, dv = 9, 4
    rng = np.random.default_rng(12)
    S0 = rng.standard_normal((1, dk, dv))
    k1 = _l2n(rng.standard_normal(dk))
    for bval in (1.0, 2.0):
        T = 2
        d = dict(q=np.tile(k1, (1, T, 1, 1)), k=np.tile(k1, (1, T, 1, 1)),
                 v=rng.standard_normal((1, T, 1, dv)), log_alpha=np.zeros((1, T, 1, dk)),
                 b=np.full((1, T, 1, dk), bval), w=np.zeros((1, T, 1, dv)),
                 z=np.zeros((1, T, 1, dk)), g=np.ones((1, T, 1, dv)),
                 gamma_stat=np.ones((1, dk)))
        one = oracle.forward({k_: (v_[:, :1] if v_.ndim == 4 else v_) for k_, v_ in d.items()}, S0=S0)
        two = oracle.forward(d, S0=S0)
        if bval == 1.0:
            assert np.max(np.abs(k1 @ one["S"][0])) < 1e-13
            assert np.max(np.abs(two["S"][0] - one["S"][0])) < 1e-13
        else:
            assert abs(np.linalg.norm(one["S"][0]) - np.linalg.norm(S0[0])) < 1e-12
            assert np.max(np.abs(two["S"][0] - S0[0])) < 1e-12


def test_rmsnorm_mean_of_squares():
    """y = g * o / sqrt(mean(o^2) + eps) per head over d_v (Muir review §2.1):
    with g = 1 the mean of y^2 is mean(o^2) / (mean(o^2) + eps)."""
    T, dk, dv = 12, 8, 8
    d = rand_inputs(T, dk, dv, seed=31)
    d["g"] = np.ones_like(d["g"])
    for eps in (1e-6, 0.5):
        r = oracle.forward(d, eps=eps)
        ms_o = np.mean(r["o_raw"][0] ** 2, 1)
        ms_y = np.mean(r["y"][0] ** 2, 1)
        assert np.max(np.abs(ms_y - ms_o / (ms_o + eps))) < 1e-13


def test_readout_gain_limits_of_the_dynamic_modulation():
    """The dynamic readout modulation 2 sigmoid(z) spans (0, 2) (Muir review
    §2.1): z -> +inf doubles the z = 0 readout, z -> -inf silences it, and the
    state never sees z."""
    T, dk, dv = 9, 8, 6
    d = rand_inputs(T, dk, dv, seed=41)
    base = oracle.forward(dict(d, z=np.zeros_like(d["z"])))
    hi = oracle.forward(dict(d, z=np.full_like(d["z"], 40.0)))
    lo = oracle.forward(dict(d, z=np.full_like(d["z"], -40.0)))
    scale = np.max(np.abs(base["o_raw"]))
    assert np.max(np.abs(hi["o_raw"] - 2.0 * base["o_raw"])) <= 1e-14 * scale
    assert np.max(np.abs(lo["o_raw"])) <= 1e-15 * scale
    assert np.max(np.abs(lo["y"])) <= 1e-6          # g * 0 / sqrt(0 + eps)
    for r in (hi, lo, oracle.forward(d)):
        assert np.array_equal(r["S"], base["S"])


def test_static_gain_scales_query_channels_and_never_the_state():
    """gamma_stat multiplies the query channel-wise (Muir review §2.1, a
    query-only gain): with a one-hot profile e_i and z = 0 the readout of
    token t is q_ti times row i of the state after token t (read after write),
    the state is the same for every profile, and a uniform profile c scales
    o_raw by c and leaves y as it is (RMSNorm, exactly when eps = 0)."""
    T, dk, dv, i = 6, 8, 5, 3
    d = rand_inputs(T, dk, dv, seed=43)
    d["z"] = np.zeros_like(d["z"])
    one_hot = np.zeros_like(d["gamma_stat"])
    one_hot[0, i] = 1.0
    r = oracle.forward(dict(d, gamma_stat=one_hot))
    for t in range(T):
        prefix = {k: (v[:, :t + 1] if v.ndim == 4 else v) for k, v in d.items()}
        S_t = oracle.forward(prefix)["S"][0]                 # state after token t
        want = d["q"][0, t, 0, i] * S_t[i]
        assert np.max(np.abs(r["o_raw"][0, t] - want)) <= 1e-13 * max(np.max(np.abs(S_t)), 1e-300)
    base = oracle.forward(d)
    assert np.array_equal(r["S"], base["S"])
    c = 3.5
    scaled = oracle.forward(dict(d, gamma_stat=c * d["gamma_stat"]))
    assert np.array_equal(scaled["S"], base["S"])
    assert relerr(scaled["o_raw"], c * base["o_raw"]) <= 1e-14
    # with eps = 0 RMSNorm removes the scale exactly
    y0, y0c = oracle.forward(d, eps=0.0)["y"], oracle.forward(dict(d, gamma_stat=c * d["gamma_stat"]), eps=0.0)["y"]
    assert relerr(y0c, y0) <= 1e-13


def test_golden_readback_squared_norm():
    """A single association S = k^T v read with the same unnormalised key
    returns |k|^2 v ("Kimi3 = GPT2 x 22580" §3)."""
    with open(os.path.join(GOLDEN, "readback_squared_norm.json")) as f:
        case = json.load(f)
    k = np.array(case["k"], dtype=np.float64)
    v = np.array(case["v"], dtype=np.float64)
    dk, dv = len(k), len(v)
    d = dict(q=k[None, None, None], k=k[None, None, None], v=v[None, None, None],
             log_alpha=np.zeros((1, 1, 1, dk)), b=np.full((1, 1, 1, dk), 0.7),
             w=np.ones((1, 1, 1, dv)), z=np.zeros((1, 1, 1, dk)),
             g=np.ones((1, 1, 1, dv)), gamma_stat=np.ones((1, dk)))
    r = oracle.forward(d)
    assert np.max(np.abs(r["o_raw"][0, 0] - np.array(case["o_expected"]))) < 1e-12


# --------------------------------------------------------------------------
# The chunked algorithm (Muir review §2.4) against the token recurrence
# --------------------------------------------------------------------------

@pytest.mark.parametrize("T,C", [(64, 64), (50, 16), (37, 8), (29, 1), (100, 64), (70, 32)])
def test_chunked_form_matches_recurrence(T, C):
    dk, dv = 12, 10
    d = rand_inputs(T, dk, dv, seed=T * 7 + C)
    S0 = np.random.default_rng(C).standard_normal((1, dk, dv)) * 0.3
    r = oracle.forward(d, S0=S0)
    y, o, S = och.chunked_head(*(head(d, x) for x in ("q", "k", "v", "b", "w", "z", "g", "log_alpha")),
                               d["gamma_stat"][0], S0[0], C)
    assert relerr(o, r["o_raw"][0]) < 1e-10
    assert relerr(S, r["S"][0]) < 1e-10
    assert relerr(y, r["y"][0]) < 1e-10


def test_chunked_form_fast_decay_has_no_division():
    """Per-token decays between exp(-exp(2)) and exp(-exp(3.2)): a chunk of 64
    spans a cumulative decay below exp(-745), which underflows float64 to 0,
    so a form that divides by it breaks.  The pivoted form stays finite and
    exact."""
    T, dk, dv = 64, 8, 8
    d = rand_inputs(T, dk, dv, seed=99, u=(2.0, 3.2))
    r = oracle.forward(d)
    lam = np.cumsum(head(d, "log_alpha"), 0)
    assert np.min(lam) < -745 and np.exp(np.min(lam)) == 0.0
    with np.errstate(over="raise", divide="raise", invalid="raise"):
        y, o, S = och.chunked_head(*(head(d, x) for x in ("q", "k", "v", "b", "w", "z", "g", "log_alpha")),
                                   d["gamma_stat"][0], None, 64)
    assert relerr(o, r["o_raw"][0]) < 1e-10
    assert relerr(S, r["S"][0]) < 1e-10


def test_dc_inverse_matches_library_inverse():
    rng = np.random.default_rng(3)
    for n in (1, 5, 8, 13, 64):
        Tm = np.eye(n) + np.tril(rng.standard_normal((n, n)) * 0.3, -1)
        assert relerr(och.unit_lower_inverse(Tm), np.linalg.inv(Tm)) < 1e-12


def test_pivot_products_match_pairwise_sum():
    rng = np.random.default_rng(6)
    n, dd = 40, 6
    A, Bm = rng.standard_normal((n, dd)), rng.standard_normal((n, dd))
    lam = np.cumsum(-np.exp(rng.uniform(-3, 1, (n, dd))), 0)
    for strict in (True, False):
        P = och.pivot_products(A, Bm, lam, strict)
        ref = np.zeros((n, n))
        for t in range(n):
            for s in range(t + (0 if strict else 1)):
                ref[t, s] = np.sum(A[t] * Bm[s] * np.exp(lam[t] - lam[s]))
        assert relerr(P, ref) < 1e-12


def test_split_run_carries_state():
    """fwd(T) equals fwd(first half) then fwd(second half) with S carried (the
    state is the cache, "Kimi3 = GPT2 x 22580" §3)."""
    T, dk, dv = 60, 8, 8
    d = rand_inputs(T, dk, dv, B=2, H=2, seed=17)
    full = oracle.forward(d)
    first = oracle.forward({k_: (v_[:, :25] if v_.ndim == 4 else v_) for k_, v_ in d.items()})
    second = oracle.forward({k_: (v_[:, 25:] if v_.ndim == 4 else v_) for k_, v_ in d.items()},
                            S0=first["S"])
    assert relerr(np.concatenate([first["y"], second["y"]], 1), full["y"]) < 1e-12
    assert relerr(second["S"], full["S"]) < 1e-12


def test_threading_does_not_change_results():
    d = rand_inputs(30, 16, 40, B=1, H=3, seed=2)
    a = oracle.forward(d, n_threads=1)
    b = oracle.forward(d, n_threads=5)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["S"], b["S"])


def test_head_selection_and_full_layout():
    d = rand_inputs(9, 8, 8, B=2, H=3, seed=5)
    full = oracle.forward_full(d)
    sel = oracle.forward(d, heads=[(1, 2), (0, 1)])
    assert np.array_equal(sel["y"][0], full["y"][1, :, 2])
    assert np.array_equal(sel["S"][1], full["S"][0, 1])


# --------------------------------------------------------------------------
# Key/query preprocessing (Muir review §2.1: SiLU, then l2 normalisation per
# head; values untouched), pinned by what fixes it rather than by retyping it
# --------------------------------------------------------------------------

def test_preprocess_qk_is_unit_norm_along_the_head_channels():
    rng = np.random.Generator(np.random.PCG64(5))
    x = rng.standard_normal((3, 7, 2, 64)) * 3.0
    y = oracle.preprocess_qk(x)
    assert np.allclose(np.linalg.norm(y, axis=-1), 1.0, atol=1e-12)
    # normalised over the last axis only: scaling one token row leaves the others alone
    x2 = x.copy()
    x2[1, 3, 0] *= 5.0
    y2 = oracle.preprocess_qk(x2)
    mask = np.ones(x.shape[:-1], bool)
    mask[1, 3, 0] = False
    assert np.array_equal(y2[mask], y[mask])


def test_preprocess_qk_direction_is_silu():
    """Parallel to x * logistic(x), the logistic taken from scipy."""
    from scipy.special import expit
    rng = np.random.Generator(np.random.PCG64(6))
    x = rng.standard_normal((5, 32)) * 4.0
    s = x * expit(x)
    y = oracle.preprocess_qk(x)
    cos = np.sum(y * s, axis=-1) / np.linalg.norm(s, axis=-1)
    assert np.allclose(cos, 1.0, atol=1e-12)
    # SiLU is not odd: a row and its negation do not map to opposite rows
    assert not np.allclose(oracle.preprocess_qk(-x), -y)


def test_preprocess_qk_special_rows():
    e = np.zeros((3, 8))
    e[0, 2] = 1.5                     # one positive channel -> that unit vector
    e[1, 5] = -2.0                    # one negative channel: SiLU < 0 -> minus that unit vector
    y = oracle.preprocess_qk(e)       # row 2 all zero: stays zero (the norm floor)
    assert np.allclose(y[0], np.eye(8)[2]) and np.allclose(y[1], -np.eye(8)[5])
    assert np.array_equal(y[2], np.zeros(8))


def test_forward_qk_raw_applies_the_preprocessing_first():
    """The raw-input forward equals the forward on preprocessed q and k, and a
    plain forward on the raw tensors differs (the flag is not ignored)."""
    import synth
    inp = synth.generate(synth.GdnShape(B=1, T=40, H=2, dk=32, dv=16, dtype="f32", seed=3))
    rng = np.random.Generator(np.random.PCG64(7))
    raw = dict(inp)
    raw["q"] = rng.standard_normal(inp["q"].shape)
    raw["k"] = rng.standard_normal(inp["k"].shape)
    pre = dict(raw)
    pre["q"], pre["k"] = oracle.preprocess_qk(raw["q"]), oracle.preprocess_qk(raw["k"])
    a = oracle.forward(raw, qk_raw=True)
    b = oracle.forward(pre)
    assert np.array_equal(a["y"], b["y"]) and np.array_equal(a["S"], b["S"])
    assert not np.allclose(oracle.forward(raw)["y"], a["y"])


# --------------------------------------------------------------------------
# Gradient oracle (oracle.backward): its forward is the C recurrence's, and
# its gradients are the central finite differences of that forward.
# --------------------------------------------------------------------------

def _bwd_case(T, dk, dv, seed, H=2):
    import synth
    inp = synth.generate(synth.GdnShape(B=1, T=T, H=H, dk=dk, dv=dv, dtype="f32", u_low=-4, u_high=0, seed=seed))
    rng = np.random.Generator(np.random.PCG64(seed + 1))
    inp = {key: np.asarray(val, dtype=np.float64) for key, val in inp.items()}
    dy = rng.standard_normal((1, T, H, dv))
    dS = rng.standard_normal((H, dk, dv))
    S0 = rng.standard_normal((H, dk, dv)) * 0.5
    return inp, dy, dS, S0


def test_backward_oracle_forward_is_the_c_recurrence():
    from oracle import backward as ob
    inp, dy, dS, S0 = _bwd_case(37, 16, 8, 31)
    r = ob.backward(inp, dy, dS_out=dS, S0=S0)
    c = oracle.forward(inp, S0=S0)
    assert np.max(np.abs(r["y"] - c["y"])) <= 1e-12 * np.max(np.abs(c["y"]))
    assert np.max(np.abs(r["S"] - c["S"])) <= 1e-12 * np.max(np.abs(c["S"]))


def test_backward_oracle_matches_central_differences():
    """Every coordinate of every input, the static profile and the initial
    state, on a tiny case: (L(x + h) - L(x - h)) / 2h against the gradient."""
    import torch
    from oracle import backward as ob
    T, dk, dv, H = 6, 5, 4, 1
    inp, dy, dS, S0 = _bwd_case(T, dk, dv, 41, H=H)
    inp["gamma_stat"] = np.exp(0.3 * np.random.Generator(np.random.PCG64(5)).standard_normal((H, dk)))
    g = ob.backward(inp, dy, dS_out=dS, S0=S0)

    def loss(x):
        args = [torch.as_tensor(x[key][0].transpose(1, 0, 2)) for key in ob.TOKEN_KEYS]   # [H, T, d]
        y, S = ob.forward_torch(*args, torch.as_tensor(x["gamma_stat"]), torch.as_tensor(x["S0"]), 1e-6)
        return float((y.numpy() * dy[0].transpose(1, 0, 2)).sum() + (S.numpy() * dS).sum())

    base = dict(inp, S0=S0)
    h = 1e-6
    for key in list(ob.TOKEN_KEYS) + ["gamma_stat", "S0"]:
        grad = g["dS_in"] if key == "S0" else g["d" + key]
        if key in ob.TOKEN_KEYS:
            grad = grad[:, :, None, :].transpose(2, 1, 0, 3)     # [n, T, d] -> [1, T, H, d]
        fd = np.zeros_like(base[key])
        for idx in np.ndindex(*base[key].shape):
            xp = {kk: vv.copy() for kk, vv in base.items()}
            xm = {kk: vv.copy() for kk, vv in base.items()}
            xp[key][idx] += h
            xm[key][idx] -= h
            fd[idx] = (loss(xp) - loss(xm)) / (2 * h)
        scale = max(np.max(np.abs(fd)), 1e-12)
        assert np.max(np.abs(fd - grad.reshape(fd.shape))) <= 1e-6 * scale, key
