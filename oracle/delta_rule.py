"""Gated delta rule, sequential and chunked (oracle; test infrastructure).

"Anthology of the SOTA, theory-128", section "The account": the state update
is S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T; the write
replaces what the state returns for key k_t with v_t, and alpha_t forgets
uniformly.  The output read is o_t = S_t^T q_t over L2-normalised q and k (the
task statement; the same page names "the key normalization" as part of the
layer).  FP64 throughout.

Readings where the pages are silent:
  * normalisation: q_hat = q / sqrt(||q||^2 + eps), same for k, per (token,
    head) over d_k, eps = 1e-6;
  * no 1/sqrt(d_k) factor on q (the output is S_t^T q_t as written);
  * the correction reads the *undecayed* S_{t-1} (literal form above), not
    alpha_t S_{t-1}.  The other common reading, where the correction reads
    the decayed state (S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1}
    + beta_t k_t v_t^T), is available as ``decayed_read=True`` on the
    sequential form; the two agree when alpha_t = 1;
  * S is d_k x d_v; S_0 = 0 unless given.

Shapes: q, k [B, T, H, dk]; v [B, T, H, dv]; log_alpha, beta [B, T, H];
S0 [B, H, dk, dv] or None.  Returns (o [B, T, H, dv], S_T [B, H, dk, dv]).
"""
import numpy as np

EPS = 1e-6


def l2_normalize(x, eps=EPS):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def _prep(q, k, v, log_alpha, beta, S0, normalize):
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if normalize:
        q = l2_normalize(q)
        k = l2_normalize(k)
    la = np.asarray(log_alpha, dtype=np.float64)
    be = np.asarray(beta, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if S0 is None:
        S0 = np.zeros((B, H, dk, dv))
    S0 = np.asarray(S0, dtype=np.float64)
    return q, k, v, la, be, S0, B, T, H, dk, dv


def delta_rule_sequential(q, k, v, log_alpha, beta, S0=None, normalize=True, decayed_read=False):
    """The literal per-token recurrence, one token at a time.  With
    ``decayed_read`` the correction reads alpha_t S_{t-1} instead of S_{t-1}."""
    q, k, v, la, be, S0, B, T, H, dk, dv = _prep(q, k, v, log_alpha, beta, S0, normalize)
    S = S0.reshape(B * H, dk, dv).copy()
    o = np.empty((B, T, H, dv))
    qf = q.transpose(1, 0, 2, 3).reshape(T, B * H, dk)
    kf = k.transpose(1, 0, 2, 3).reshape(T, B * H, dk)
    vf = v.transpose(1, 0, 2, 3).reshape(T, B * H, dv)
    af = np.exp(la).transpose(1, 0, 2).reshape(T, B * H)
    bf = be.transpose(1, 0, 2).reshape(T, B * H)
    of = np.empty((T, B * H, dv))
    for t in range(T):
        kt = kf[t]
        S_read = S * af[t][:, None, None] if decayed_read else S
        r = np.matmul(kt[:, None, :], S_read)[:, 0, :]            # S_{t-1}^T k_t (or of alpha_t S_{t-1})
        S *= af[t][:, None, None]                                 # alpha_t S_{t-1}
        S += (bf[t][:, None] * kt)[:, :, None] * (vf[t] - r)[:, None, :]
        of[t] = np.matmul(qf[t][:, None, :], S)[:, 0, :]          # S_t^T q_t
    o[:] = of.reshape(T, B, H, dv).transpose(1, 0, 2, 3)
    return o, S.reshape(B, H, dk, dv)


def delta_rule_chunked(q, k, v, log_alpha, beta, S0=None, chunk=64, normalize=True):
    """The same recurrence evaluated chunk by chunk (UT / WY form).

    With u_t = beta_t (v_t - S_{t-1}^T k_t), S_t = alpha_t S_{t-1} + k_t u_t^T.
    Inside a chunk with entry state S0, G_t = sum_{s<=t} log alpha_s (G_0 = 0):
      L_ts  = beta_t exp(G_{t-1} - G_s) (k_t . k_s)        (s < t)
      U     = (I + L)^{-1} [diag(beta) V - diag(beta exp(G_{t-1})) K S0]
      O     = diag(exp(G_t)) Q S0 + (Gamma o Q K^T) U,  Gamma_ts = exp(G_t - G_s), s <= t
      S_out = exp(G_C) S0 + K^T diag(exp(G_C - G_s)) U
    Every exponent is <= 0.  A final partial chunk uses its own length.
    """
    q, k, v, la, be, S0, B, T, H, dk, dv = _prep(q, k, v, log_alpha, beta, S0, normalize)
    o = np.empty((B, T, H, dv))
    S_T = np.empty((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = S0[b, h].copy()
            for t0 in range(0, T, chunk):
                t1 = min(T, t0 + chunk)
                Q = q[b, t0:t1, h]
                K = k[b, t0:t1, h]
                V = v[b, t0:t1, h]
                bt = be[b, t0:t1, h]
                G = np.cumsum(la[b, t0:t1, h])
                Gm1 = np.concatenate([[0.0], G[:-1]])
                C = t1 - t0
                low = np.tril(np.ones((C, C), dtype=bool), -1)
                lowd = np.tril(np.ones((C, C), dtype=bool), 0)
                dG_ex = np.where(low, Gm1[:, None] - G[None, :], -np.inf)
                L = np.where(low, bt[:, None] * np.exp(dG_ex) * (K @ K.T), 0.0)
                Tm = np.eye(C) + L
                rhs = bt[:, None] * V - (bt * np.exp(Gm1))[:, None] * (K @ S)
                U = np.linalg.solve(Tm, rhs)
                dG = np.where(lowd, G[:, None] - G[None, :], -np.inf)
                Gam = np.where(lowd, np.exp(dG), 0.0)
                o[b, t0:t1, h] = np.exp(G)[:, None] * (Q @ S) + (Gam * (Q @ K.T)) @ U
                S = np.exp(G[-1]) * S + K.T @ (np.exp(G[-1] - G)[:, None] * U)
            S_T[b, h] = S
    return o, S_T
