"""fp64 restatement of the chunkwise parallel form (test helper, numpy only).

"KDA cheat sheet", Chunkwise parallel form (eqs. 3-4): within a chunk the
channel-wise cumulative decay Gamma and the pseudo-values from the UT
transform give ``O = (Gamma*Q) S + Tril[(Q*Gamma)(K/Gamma)^T] Vtilde``, with
the diagonal kept because each output reads the post-update state. The page
leaves the UT transform to another paper, so it is re-derived here from the
recurrence (eq. 1 of "Kimi K3: Bounded Decay and Delta Memory"). Write the
state inside a chunk as ``S_t = Diag(gamma_t) X_t`` (gamma_t the inclusive
product of alpha over the chunk so far) and ``u_t = beta_t delta_t``. Then

    X_t = X_{t-1} + (k_t / gamma_t) u_t^T
    (I + A_kk) U = Diag(beta) V - Diag(beta) (K*Gamma) S_0,
        A_kk[t,i] = beta_t <gamma_t*k_t, k_i/gamma_i>   (i < t)
    U = Ut - W S_0,  Ut = T Diag(beta) V,  W = T Diag(beta) (K*Gamma),  T = (I+A_kk)^-1
    O = (Q*Gamma) S_0 + A_qk U,   A_qk[t,i] = <gamma_t*q_t, k_i/gamma_i>  (i <= t)
    S_C = Diag(gamma_C) S_0 + (K * gamma_C/Gamma)^T U

Decay ratios are formed as exp(G_t - G_i) from the chunk-local cumulative
log-decay G, which is exact in fp64 for any chunk length. This helper checks
the algebra that the GPU prefill uses against the token-by-token oracle; it
is not the oracle.
"""
import numpy as np


def chunkwise_head(q, k, v, alpha, beta, S0, C):
    """One head. q, k, alpha [T,K]; v [T,V]; beta [T]; S0 [K,V]. Returns (o [T,V], S [K,V])."""
    T = q.shape[0]
    S = np.array(S0, dtype=np.float64, copy=True)
    o = np.zeros((T, v.shape[1]))
    for start in range(0, T, C):
        sl = slice(start, min(start + C, T))
        n = sl.stop - sl.start
        Q, Kc, Vc, b = q[sl], k[sl], v[sl], beta[sl]
        G = np.cumsum(np.log(alpha[sl]), axis=0)          # [n,K], inclusive
        Gam = np.exp(G)
        diff = G[:, None, :] - G[None, :, :]               # G_t - G_i, [t,i,K]
        lower_incl = np.tril(np.ones((n, n), dtype=bool))
        ratio = np.where(lower_incl[:, :, None], np.exp(np.minimum(diff, 0.0)), 0.0)
        A_qk = np.einsum("tc,ic,tic->ti", Q, Kc, ratio)
        A_kk = b[:, None] * np.einsum("tc,ic,tic->ti", Kc, Kc, ratio)
        A_kk = np.tril(A_kk, -1)
        Tinv = np.linalg.inv(np.eye(n) + A_kk)
        W = Tinv @ (b[:, None] * Kc * Gam)
        Ut = Tinv @ (b[:, None] * Vc)
        U = Ut - W @ S
        o[sl] = (Q * Gam) @ S + A_qk @ U
        tail = np.exp(G[-1][None, :] - G)                 # gamma_C / gamma_i, [n,K]
        S = np.exp(G[-1])[:, None] * S + (Kc * tail).T @ U
    return o, S


def chunkwise_scan(q, k, v, alpha, beta, S0, C):
    """[B,T,H,*] inputs, S0 [B,H,K,V] or None. Returns (o, final_state) in fp64."""
    q, k, v, alpha, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta))
    B, T, H, K = q.shape
    V = v.shape[-1]
    o = np.zeros((B, T, H, V))
    sf = np.zeros((B, H, K, V))
    for b_ in range(B):
        for h in range(H):
            s0 = np.zeros((K, V)) if S0 is None else np.asarray(S0[b_, h], dtype=np.float64)
            o[b_, :, h], sf[b_, h] = chunkwise_head(q[b_, :, h], k[b_, :, h], v[b_, :, h],
                                                    alpha[b_, :, h], beta[b_, :, h], s0, C)
    return o, sf


def block_factored_a(q, k, G, pairwise_diag=False, blk=16, dtype=np.float32):
    """A_qk[t,i] = sum_c q_tc k_ic exp(G_tc - G_ic) (i <= t) of one chunk, formed the way the chunked
    kernels form it, in `dtype` arithmetic: 16-token blocks a, b with the block-boundary references
    s_a (cumulative log-decay before block a) and r_b (after block b), as
    (q * exp(G - G_s_a)) * exp(G_s_a - G_r_b) . (k * exp(G_r_b - G))  for a > b,
    and for the diagonal blocks either the same split with exp(G_s_a - G_r_a) -- the reciprocal of the
    block's whole decay -- or pairwise (``pairwise_diag``). Returns (A_qk, largest factor applied off the
    diagonal blocks). G is the inclusive cumulative log-decay [n, K] in fp64."""
    n, K = q.shape
    G = np.asarray(G, dtype=np.float64)
    nb = (n + blk - 1) // blk
    Gs = [np.zeros(K) if a == 0 else G[blk * a - 1] for a in range(nb)]
    Gr = [G[min(blk * (a + 1), n) - 1] for a in range(nb)]
    A = np.zeros((n, n), dtype=dtype)
    worst = 0.0
    with np.errstate(over="ignore", invalid="ignore", under="ignore"):
        for a in range(nb):
            ta = slice(blk * a, min(blk * (a + 1), n))
            E = np.exp(G[ta] - Gs[a])
            for b in range(a + 1):
                tb = slice(blk * b, min(blk * (b + 1), n))
                if a == b and pairwise_diag:
                    d = G[ta][:, None, :] - G[tb][None, :, :]
                    ratio = np.where(np.tril(np.ones((d.shape[0], d.shape[1]), bool))[:, :, None],
                                     np.exp(np.minimum(d, 0.0)), 0.0).astype(dtype)
                    A[ta, tb] = np.einsum("tc,ic,tic->ti", q[ta].astype(dtype), k[tb].astype(dtype), ratio)
                    continue
                F = np.exp(Gr[b] - G[tb])
                D = np.exp(Gs[a] - Gr[b])
                if a > b:
                    worst = max(worst, float(E.max()), float(F.max()), float(D.max()))
                lhs = (q[ta] * E).astype(dtype) * D.astype(dtype)[None, :]
                blockA = lhs @ (k[tb] * F).astype(dtype).T
                if a == b:
                    blockA = np.tril(blockA)
                A[ta, tb] = blockA
    return A, worst
