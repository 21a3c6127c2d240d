"""The chunked prefill's algebra, checked on the CPU in fp64 against the oracle's token loop.

For a chunk of C tokens entered with state S0, with G_j the inclusive prefix sum of g over the
chunk, a_j = exp(G_j) and D_j = exp(G_C - G_j), the token recurrence unrolls to
    L_jm = beta_j e^{G_j - G_m} (k_j . k_m)   (m < j),   T = (I + L)^-1,
    Z = S0 K^T,   R = beta (V - a Z),   W = R T^T,   S_C = a_C S0 + (W D) K.
The decays of L are a diagonal similarity, so the tensor-core kernel uses the decay-free
inverse T~ = (I + diag(beta) K~)^-1 (K~ the strictly lower part of K K^T) and
    M1_jm = beta_j D_j T~_mj,   M2_jm = -a_j M1_jm = -a_C beta_j T~_mj,
    Y = V^T M1 + S0 K^T M2,   S_C = a_C S0 + Y K,
with T~ built from 16 x 16 blocks: the diagonal blocks by forward substitution, the blocks below
them as two halves of 32 (T = [[A, 0], [C, B]], C = -B L_21 A). Tokens past the prompt are
padded as g = 0, beta = 0, k = 0, v = 0. This file restates both forms in numpy (sharing nothing
with the kernel or with the oracle), so that a wrong sign, index or decay factor in either
derivation fails here without a GPU; the GPU tests then compare the kernel with the oracle.
"""
import numpy as np
import pytest

import oracle


def _prompt(P, d_k, d_v, seed, g_const=None):
    rng = np.random.default_rng(seed)
    k = rng.standard_normal((P, d_k))
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((P, d_v))
    g = -np.log1p(np.exp(rng.standard_normal(P))) if g_const is None else np.full(P, g_const)
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal(P)))
    return k, v, g, beta


def _block_inverse(L, bs=16):
    """(I + L)^-1 for strictly lower-triangular L, by blocks as the kernel does."""
    n = L.shape[0]
    nb = n // bs
    T = np.zeros_like(L)
    for b in range(nb):                                   # diagonal blocks, column by column
        o = b * bs
        for m in range(bs):
            x = np.zeros(bs)
            x[m] = 1.0
            for ii in range(bs - 1):                      # right-looking: x[ii] final, update below
                x[ii + 1:] -= L[o + ii + 1:o + bs, o + ii] * x[ii]
            T[o:o + bs, o + m] = x
    for dl in range(1, nb):                               # off-diagonal blocks by distance
        for a in range(nb - dl):
            b = a + dl
            Q = L[b * bs:(b + 1) * bs, a * bs:b * bs] @ T[a * bs:b * bs, a * bs:(a + 1) * bs]
            T[b * bs:(b + 1) * bs, a * bs:(a + 1) * bs] = -T[b * bs:(b + 1) * bs, b * bs:(b + 1) * bs] @ Q
    return T


def _chunked_prefill(k, v, g, beta, C=64):
    P, d_k = k.shape
    d_v = v.shape[1]
    n = max(1, -(-P // C)) if P else 0
    pad = n * C - P
    k = np.vstack([k, np.zeros((pad, d_k))])
    v = np.vstack([v, np.zeros((pad, d_v))])
    g = np.concatenate([g, np.zeros(pad)])
    beta = np.concatenate([beta, np.zeros(pad)])
    S = np.zeros((d_v, d_k))
    for c in range(n):
        sl = slice(c * C, (c + 1) * C)
        K, V, gc, bc = k[sl], v[sl], g[sl], beta[sl]
        G = np.cumsum(gc)
        a = np.exp(G)
        D = np.exp(G[-1] - G)
        A = K @ K.T
        L = np.tril(bc[:, None] * np.exp(G[:, None] - G[None, :]) * A, -1)
        T = _block_inverse(L)
        Z = S @ K.T                                       # [d_v, C]
        R = bc[None, :] * (V.T - a[None, :] * Z)          # [d_v, C]
        W = R @ T.T
        S = a[-1] * S + (W * D[None, :]) @ K
    return S


def test_block_inverse_is_the_inverse():
    rng = np.random.default_rng(5)
    K = rng.standard_normal((64, 32))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    G = np.cumsum(-np.log1p(np.exp(rng.standard_normal(64))))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal(64)))
    L = np.tril(b[:, None] * np.exp(G[:, None] - G[None, :]) * (K @ K.T), -1)
    T = _block_inverse(L)
    assert np.allclose(T, np.linalg.inv(np.eye(64) + L), rtol=0, atol=1e-12)
    assert np.allclose(np.tril(T), T) and np.allclose(np.diag(T), 1.0)


@pytest.mark.parametrize("P", [1, 15, 63, 64, 65, 200])
def test_chunked_form_is_the_token_recurrence(P):
    k, v, g, beta = _prompt(P, 16, 24, seed=P)
    S_ref = oracle.prefill(k, v, g, beta)
    S = _chunked_prefill(k, v, g, beta)
    assert np.max(np.abs(S - S_ref)) <= 1e-12 * max(1.0, np.max(np.abs(S_ref)))


def test_chunked_form_weak_decay():
    """alpha close to 1: every chunk's contribution survives, so a wrong decay factor shows."""
    k, v, g, beta = _prompt(300, 16, 16, seed=11, g_const=-0.01)
    S_ref = oracle.prefill(k, v, g, beta)
    assert np.max(np.abs(_chunked_prefill(k, v, g, beta) - S_ref)) <= 1e-11


def test_chunk_length_does_not_matter():
    k, v, g, beta = _prompt(96, 16, 16, seed=3)
    assert np.allclose(_chunked_prefill(k, v, g, beta, C=16), _chunked_prefill(k, v, g, beta, C=32),
                       rtol=0, atol=1e-12)


def test_planted_mistakes_are_caught():
    """The comparison is sharp enough: a chunked form with the decay of R taken at the previous
    token, or with L's decay reversed, misses the token recurrence by far more than rounding."""
    k, v, g, beta = _prompt(130, 16, 16, seed=7)
    S_ref = oracle.prefill(k, v, g, beta)
    ok = _chunked_prefill(k, v, g, beta)

    def variant(flip):
        C = 64
        P = k.shape[0]
        n = -(-P // C)
        pad = n * C - P
        kk = np.vstack([k, np.zeros((pad, 16))])
        vv = np.vstack([v, np.zeros((pad, 16))])
        gg = np.concatenate([g, np.zeros(pad)])
        bb = np.concatenate([beta, np.zeros(pad)])
        S = np.zeros((16, 16))
        for c in range(n):
            sl = slice(c * C, (c + 1) * C)
            K, V, gc, bc = kk[sl], vv[sl], gg[sl], bb[sl]
            G = np.cumsum(gc)
            Gx = G - gc if flip == "exclusive" else G
            sign = -1.0 if flip == "reversed" else 1.0
            L = np.tril(bc[:, None] * np.exp(sign * (G[:, None] - G[None, :])) * (K @ K.T), -1)
            T = np.linalg.inv(np.eye(C) + L)
            R = bc[None, :] * (V.T - np.exp(Gx)[None, :] * (S @ K.T))
            S = np.exp(G[-1]) * S + ((R @ T.T) * np.exp(G[-1] - G)[None, :]) @ K
        return S

    assert np.max(np.abs(ok - S_ref)) <= 1e-12
    for flip in ("exclusive", "reversed"):
        assert np.max(np.abs(variant(flip) - S_ref)) > 1e-3


def _block_inverse_halves(L, bs=16):
    """(I + L)^-1 for strictly lower-triangular 64 x 64 L as the kernel builds it: the four
    diagonal blocks by forward substitution, each half's lower block (T_10 = -T_11 L_10 T_00,
    T_32 = -T_33 L_32 T_22), then X = L_(23)(01) A and C = -B X for the lower-left quarter."""
    T = np.zeros_like(L)
    for b in range(4):
        o = b * bs
        blk = np.eye(bs) + L[o:o + bs, o:o + bs]
        for m in range(bs):                               # forward substitution, one column
            x = np.zeros(bs)
            x[m] = 1.0
            for i in range(bs):
                x[i] -= blk[i, :i] @ x[:i]
            T[o:o + bs, o + m] = x
    sl = [slice(16 * i, 16 * (i + 1)) for i in range(4)]
    for h in (0, 2):
        T[sl[h + 1], sl[h]] = -T[sl[h + 1], sl[h + 1]] @ (L[sl[h + 1], sl[h]] @ T[sl[h], sl[h]])
    A, B = T[:32, :32], T[32:, 32:]
    T[32:, :32] = -B @ (L[32:, :32] @ A)
    return T


def _decay_free_prefill(k, v, g, beta, C=64, mistake=None):
    P, d_k = k.shape
    d_v = v.shape[1]
    n = max(1, -(-P // C)) if P else 0
    pad = n * C - P
    k = np.vstack([k, np.zeros((pad, d_k))])
    v = np.vstack([v, np.zeros((pad, d_v))])
    g = np.concatenate([g, np.zeros(pad)])
    beta = np.concatenate([beta, np.zeros(pad)])
    S = np.zeros((d_v, d_k))
    for c in range(n):
        sl = slice(c * C, (c + 1) * C)
        K, V, gc, bc = k[sl], v[sl], g[sl], beta[sl]
        G = np.cumsum(gc)
        a, D, aC = np.exp(G), np.exp(G[-1] - G), np.exp(G[-1])
        Lt = np.tril(bc[:, None] * (K @ K.T), -1)
        Tt = _block_inverse_halves(Lt) if C == 64 else np.linalg.inv(np.eye(C) + Lt)
        M1 = (bc * (1.0 if mistake == "no_D" else D))[:, None] * Tt.T   # M1[j, m]
        M2 = -a[:, None] * M1                                           # = -a_C beta_j T~_mj
        if mistake == "a_j_for_a_C":
            M2 = -(a * bc)[:, None] * Tt.T
        Y = V.T @ M1 + S @ (K.T @ M2)
        S = aC * S + Y @ K
    return S


def test_block_inverse_by_halves_is_the_inverse():
    rng = np.random.default_rng(6)
    K = rng.standard_normal((64, 32))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal(64)))
    L = np.tril(b[:, None] * (K @ K.T), -1)
    T = _block_inverse_halves(L)
    assert np.allclose(T, np.linalg.inv(np.eye(64) + L), rtol=0, atol=1e-12)


def test_decays_are_a_diagonal_similarity():
    """(I + L)^-1 = E T~ E^-1 with E = diag(e^{G}) and T~ the decay-free inverse."""
    rng = np.random.default_rng(8)
    K = rng.standard_normal((64, 16))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    G = np.cumsum(-np.log1p(np.exp(rng.standard_normal(64))) * 0.1)
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal(64)))
    L = np.tril(b[:, None] * np.exp(G[:, None] - G[None, :]) * (K @ K.T), -1)
    Tt = np.linalg.inv(np.eye(64) + np.tril(b[:, None] * (K @ K.T), -1))
    E = np.diag(np.exp(G))
    assert np.allclose(np.linalg.inv(np.eye(64) + L), E @ Tt @ np.linalg.inv(E), rtol=0, atol=1e-10)


@pytest.mark.parametrize("P", [1, 15, 63, 64, 65, 200])
def test_decay_free_form_is_the_token_recurrence(P):
    k, v, g, beta = _prompt(P, 16, 24, seed=100 + P)
    S_ref = oracle.prefill(k, v, g, beta)
    S = _decay_free_prefill(k, v, g, beta)
    assert np.max(np.abs(S - S_ref)) <= 1e-12 * max(1.0, np.max(np.abs(S_ref)))


def test_decay_free_form_weak_and_strong_decay():
    for g_const in (-0.01, -3.0):
        k, v, g, beta = _prompt(300, 16, 16, seed=12, g_const=g_const)
        S_ref = oracle.prefill(k, v, g, beta)
        assert np.max(np.abs(_decay_free_prefill(k, v, g, beta) - S_ref)) <= 1e-11


def test_decay_free_planted_mistakes_are_caught():
    """M1 without its decay D, or M2 scaled by a_j beta_j instead of a_C beta_j, misses the token
    recurrence by far more than rounding."""
    k, v, g, beta = _prompt(130, 16, 16, seed=9)
    S_ref = oracle.prefill(k, v, g, beta)
    assert np.max(np.abs(_decay_free_prefill(k, v, g, beta) - S_ref)) <= 1e-12
    for mistake in ("no_D", "a_j_for_a_C"):
        assert np.max(np.abs(_decay_free_prefill(k, v, g, beta, mistake=mistake) - S_ref)) > 1e-3
