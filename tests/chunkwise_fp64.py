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


def chunkwise_backward_head(q, k, v, alpha, beta, S0, d_o, d_sf, C):
    """Gradients of one head's scan through the chunkwise form (the derivation a chunked backward kernel
    follows), in fp64. Inputs as for ``chunkwise_head`` plus d_o [T,V] = dL/do and d_sf [K,V] = dL/dS_T.
    Returns dq, dk, dv, dalpha, dbeta, dS0.

    Per chunk, with G the chunk-local inclusive cumulative log-decay, R[t,i,c] = exp(G_tc - G_ic) (i <= t),
    M_q = sum_c q k R (lower, diagonal kept), M_k = sum_c k k R (strictly lower), A_kk = Diag(beta) M_k,
    T = (I + A_kk)^-1, TB = T Diag(beta), W = TB (K*Gamma), Ut = TB V, U = Ut - W S0,
    O = (Q*Gamma) S0 + M_q U, S_C = Diag(gamma_C) S0 + (K*gamma_C/Gamma)^T U, the adjoints are
        dU = M_q^T dO + (K*gamma_C/Gamma) dS_C,  dS0 = (Q*Gamma)^T dO + Diag(gamma_C) dS_C - W^T dU,
        dTB = dU V^T - dU S0^T (K*Gamma)^T,  dT = dTB Diag(beta),  dA_kk = -T^T dT T^T (strictly lower),
    and the bilinear forms M_q, M_k and the Gamma factors give dq, dk and dG; dlog(alpha) is the reverse
    cumulative sum of dG within the chunk. Chunks are walked backwards from the last, each chunk's dS0 being
    the previous chunk's dS_C; the chunk-start states come from a forward pass."""
    T_, K = q.shape
    Vd = v.shape[1]
    la = np.log(alpha)
    starts = list(range(0, T_, C))
    S = np.array(S0, dtype=np.float64, copy=True)
    S_start = []
    for start in starts:  # forward: the state at every chunk start
        S_start.append(S.copy())
        sl = slice(start, min(start + C, T_))
        _, S = chunkwise_head(q[sl], k[sl], v[sl], alpha[sl], beta[sl], S, C)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dla, dbeta = np.zeros_like(la), np.zeros_like(beta)
    dS = np.array(d_sf, dtype=np.float64, copy=True)
    for ci in range(len(starts) - 1, -1, -1):
        sl = slice(starts[ci], min(starts[ci] + C, T_))
        n = sl.stop - sl.start
        Q, Kc, Vc, b, S0c, dO = q[sl], k[sl], v[sl], beta[sl], S_start[ci], d_o[sl]
        G = np.cumsum(la[sl], axis=0)
        Gam = np.exp(G)
        diff = G[:, None, :] - G[None, :, :]
        low_incl = np.tril(np.ones((n, n), dtype=bool))
        low = np.tril(np.ones((n, n), dtype=bool), -1)
        R = np.where(low_incl[:, :, None], np.exp(np.minimum(diff, 0.0)), 0.0)
        Mq = np.einsum("tc,ic,tic->ti", Q, Kc, R)
        Mk = np.where(low, np.einsum("tc,ic,tic->ti", Kc, Kc, R), 0.0)
        A = b[:, None] * Mk
        Tm = np.linalg.inv(np.eye(n) + A)
        TB = Tm * b[None, :]
        KG = Kc * Gam
        W = TB @ KG
        Ut = TB @ Vc
        U = Ut - W @ S0c
        QG = Q * Gam
        gC = np.exp(G[-1])
        KT = Kc * np.exp(G[-1][None, :] - G)
        # adjoints
        dU = Mq.T @ dO + KT @ dS
        dMq = np.where(low_incl, dO @ U.T, 0.0)
        dQG = dO @ S0c.T
        dS0 = QG.T @ dO + gC[:, None] * dS - W.T @ dU
        dKT = U @ dS.T
        dgC = np.sum(dS * S0c, axis=1)
        dW = -dU @ S0c.T
        dTB = dU @ Vc.T + dW @ KG.T
        dv[sl] += TB.T @ dU
        dKG = TB.T @ dW
        dT = dTB * b[None, :]
        dbeta[sl] += np.sum(dTB * Tm, axis=0)
        dA = np.where(low, -Tm.T @ dT @ Tm.T, 0.0)
        dbeta[sl] += np.sum(dA * Mk, axis=1)
        dMk = dA * b[:, None]
        dG = np.zeros_like(G)
        # M_q[t,i] = sum_c Q_tc K_ic R_tic
        Pq = dMq[:, :, None] * Q[:, None, :] * Kc[None, :, :] * R
        dq[sl] += np.einsum("ti,ic,tic->tc", dMq, Kc, R)
        dk[sl] += np.einsum("ti,tc,tic->ic", dMq, Q, R)
        dG += Pq.sum(axis=1) - Pq.sum(axis=0)
        # M_k[t,i] = sum_c K_tc K_ic R_tic (strictly lower)
        Pk = dMk[:, :, None] * Kc[:, None, :] * Kc[None, :, :] * R
        dk[sl] += np.einsum("ti,ic,tic->tc", dMk, Kc, R) + np.einsum("ti,tc,tic->ic", dMk, Kc, R)
        dG += Pk.sum(axis=1) - Pk.sum(axis=0)
        # the Gamma factors
        dq[sl] += dQG * Gam
        dG += dQG * QG
        dk[sl] += dKG * Gam
        dG += dKG * KG
        dk[sl] += dKT * np.exp(G[-1][None, :] - G)
        dG -= dKT * KT
        dG[-1] += np.sum(dKT * KT, axis=0) + dgC * gC
        dla[sl] += np.cumsum(dG[::-1], axis=0)[::-1]
        dS = dS0
    return dq, dk, dv, dla / alpha, dbeta, dS


def chunkwise_backward(q, k, v, alpha, beta, S0, d_o, d_sf, C):
    """[B,T,H,*] inputs (S0, d_sf [B,H,K,V] or None). Returns a dict of fp64 gradients keyed like
    ``oracle.scan_backward``: q, k, v, alpha, beta, initial_state."""
    q, k, v, alpha, beta, d_o = (np.asarray(x, dtype=np.float64) for x in (q, k, v, alpha, beta, d_o))
    B, T, H, K = q.shape
    V = v.shape[-1]
    out = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta", beta))}
    out["initial_state"] = np.zeros((B, H, K, V))
    for b_ in range(B):
        for h in range(H):
            s0 = np.zeros((K, V)) if S0 is None else np.asarray(S0[b_, h], dtype=np.float64)
            dsf = np.zeros((K, V)) if d_sf is None else np.asarray(d_sf[b_, h], dtype=np.float64)
            r = chunkwise_backward_head(q[b_, :, h], k[b_, :, h], v[b_, :, h], alpha[b_, :, h], beta[b_, :, h],
                                        s0, d_o[b_, :, h], dsf, C)
            for name, g in zip(("q", "k", "v", "alpha", "beta"), r[:5]):
                out[name][b_, :, h] = g
            out["initial_state"][b_, h] = r[5]
    return out


def chunkwise_backward_split(q, k, v, alpha, beta, S0, d_o, d_sf, C):
    """``chunkwise_backward_head`` rearranged into the three passes a chunked backward runs as kernels:
    (1) per chunk, in parallel, the state-independent operands (the forward's, plus dO); (2) one reverse
    recurrence over chunks carrying dS, which needs only dU = A_qk^T dO + (K*gamma_C/Gamma) dS_C and
    dS0 = (Q*Gamma)^T dO + Diag(gamma_C) dS_C - W^T dU, i.e. the affine map
    dS0 = (Q*Gamma - A_qk W)^T dO + (Diag(gamma_C) - W^T (K*gamma_C/Gamma)) dS_C, and emits dU per chunk;
    (3) per chunk, in parallel, every other gradient from dU and the chunk-start state S0.
    One head, inputs as for ``chunkwise_backward_head``; same outputs."""
    T_, K = q.shape
    la = np.log(alpha)
    starts = list(range(0, T_, C))
    # forward states at chunk starts (the forward's recurrence)
    S = np.array(S0, dtype=np.float64, copy=True)
    S_start = []
    for start in starts:
        S_start.append(S.copy())
        sl = slice(start, min(start + C, T_))
        _, S = chunkwise_head(q[sl], k[sl], v[sl], alpha[sl], beta[sl], S, C)
    # pass 1: state-independent operands per chunk
    ops = []
    for start in starts:
        sl = slice(start, min(start + C, T_))
        n = sl.stop - sl.start
        Q, Kc, b = q[sl], k[sl], beta[sl]
        G = np.cumsum(la[sl], axis=0)
        Gam = np.exp(G)
        diff = G[:, None, :] - G[None, :, :]
        low_incl = np.tril(np.ones((n, n), dtype=bool))
        low = np.tril(np.ones((n, n), dtype=bool), -1)
        R = np.where(low_incl[:, :, None], np.exp(np.minimum(diff, 0.0)), 0.0)
        Mq = np.einsum("tc,ic,tic->ti", Q, Kc, R)
        Mk = np.where(low, np.einsum("tc,ic,tic->ti", Kc, Kc, R), 0.0)
        Tm = np.linalg.inv(np.eye(n) + b[:, None] * Mk)
        TB = Tm * b[None, :]
        W = TB @ (Kc * Gam)
        KT = Kc * np.exp(G[-1][None, :] - G)
        ops.append(dict(sl=sl, n=n, G=G, Gam=Gam, R=R, Mq=Mq, Mk=Mk, Tm=Tm, TB=TB, W=W, KT=KT, QG=Q * Gam,
                        gC=np.exp(G[-1])))
    # pass 2: reverse recurrence over dS, emitting dU and dS_C per chunk
    dS = np.array(d_sf, dtype=np.float64, copy=True)
    dU_all, dSC_all = [None] * len(starts), [None] * len(starts)
    for ci in range(len(starts) - 1, -1, -1):
        o = ops[ci]
        dO = d_o[o["sl"]]
        dU = o["Mq"].T @ dO + o["KT"] @ dS
        dU_all[ci], dSC_all[ci] = dU, dS
        dS = o["QG"].T @ dO + o["gC"][:, None] * dS - o["W"].T @ dU
    # pass 3: the remaining gradients per chunk, from dU, dS_C and S0
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dla, dbeta = np.zeros_like(la), np.zeros_like(beta)
    for ci, o in enumerate(ops):
        sl, n = o["sl"], o["n"]
        Q, Kc, Vc, b, S0c, dO = q[sl], k[sl], v[sl], beta[sl], S_start[ci], d_o[sl]
        dU, dSC = dU_all[ci], dSC_all[ci]
        G, Gam, R, Mq, Mk, Tm, TB, KT, gC = (o[x] for x in ("G", "Gam", "R", "Mq", "Mk", "Tm", "TB", "KT", "gC"))
        KG = Kc * Gam
        U = TB @ Vc - o["W"] @ S0c
        low_incl = np.tril(np.ones((n, n), dtype=bool))
        low = np.tril(np.ones((n, n), dtype=bool), -1)
        dMq = np.where(low_incl, dO @ U.T, 0.0)
        dQG = dO @ S0c.T
        dKT = U @ dSC.T
        dgC = np.sum(dSC * S0c, axis=1)
        dW = -dU @ S0c.T
        dTB = dU @ Vc.T + dW @ KG.T
        dv[sl] = TB.T @ dU
        dKG = TB.T @ dW
        dA = np.where(low, -Tm.T @ (dTB * b[None, :]) @ Tm.T, 0.0)
        dbeta[sl] = np.sum(dTB * Tm, axis=0) + np.sum(dA * Mk, axis=1)
        dMk = dA * b[:, None]
        Pq = dMq[:, :, None] * Q[:, None, :] * Kc[None, :, :] * R
        Pk = dMk[:, :, None] * Kc[:, None, :] * Kc[None, :, :] * R
        dq[sl] = np.einsum("ti,ic,tic->tc", dMq, Kc, R) + dQG * Gam
        dk[sl] = (np.einsum("ti,tc,tic->ic", dMq, Q, R) + np.einsum("ti,ic,tic->tc", dMk, Kc, R)
                  + np.einsum("ti,tc,tic->ic", dMk, Kc, R) + dKG * Gam + dKT * np.exp(G[-1][None, :] - G))
        dG = (Pq.sum(axis=1) - Pq.sum(axis=0) + Pk.sum(axis=1) - Pk.sum(axis=0) + dQG * o["QG"] + dKG * KG
              - dKT * KT)
        dG[-1] += np.sum(dKT * KT, axis=0) + dgC * gC
        dla[sl] = np.cumsum(dG[::-1], axis=0)[::-1]
    return dq, dk, dv, dla / alpha, dbeta, dS
