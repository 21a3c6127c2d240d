"""The chunked prefill's algebra, checked on the CPU in fp64 against the oracle's token loop.

The tensor-core prefill kernel computes the prompt state chunk by chunk. For a chunk of C tokens
entered with state S0, with G_j the inclusive prefix sum of g over the chunk, a_j = exp(G_j):
    L_jm = beta_j e^{G_j - G_m} (k_j . k_m)   (m < j),   T = (I + L)^-1,
    Z = S0 K^T,   R = beta (V - a Z),   W = R T^T,   S_C = a_C S0 + (W D) K,
with D = diag(e^{G_C - G_j}), and it builds T from 16 x 16 blocks: the diagonal blocks by forward
substitution, then T_ba = -T_bb sum_{a <= c < b} L_bc T_ca by block distance. Tokens past the
prompt are padded as g = 0, beta = 0, k = 0, v = 0. This file restates those formulas in numpy
(sharing nothing with the kernel or with the oracle), so that a wrong sign, index or decay factor
in the derivation fails here without a GPU; the GPU tests then compare the kernel with the oracle.
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
