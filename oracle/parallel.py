"""Brute-force O(T^2) parallel form of causal linear attention, float64 numpy.

TEST INFRASTRUCTURE: a second, independent statement of what the recurrent
oracle (la_ref.c) computes, used only by tests/ to pin it.  It shares no code
with la_ref.c or with the CUDA library.

Sources:
  - tensortonic "CS336 L04 linear attention duality": the same outputs can be
    computed "in parallel" from the whole sequence (the page points at prefix
    sums and batched matmuls).
  - Jamie-Stirling/RetNet issue 21, the paragraph after the retention listing:
    the EMA scan computes (Q K^T * D) V, where D is the causal decay mask.
    With per-step factors g_t the mask entry is D[t, s] = prod_{s<r<=t} g_r
    for s <= t and 0 above the diagonal; here it is exp(L_t - L_s) with
    L_t = sum_{r<=t} log g_r, so no factor exceeds 1 (RWKV-LM discussion 189:
    the exponentially weighted parameterisation).
  - flash-linear-attention issue 268: the cache term (carried state S_0) and
    the key-sum term (carried z_0) of the normalised output QKV / QK1.

Per sequence (b, h):
    y_t  = sum_{s<=t} D[t,s] (q_t . k_s) v_s + exp(L_t) q_t^T S_0
    den_t = sum_{s<=t} D[t,s] (q_t . k_s)     + exp(L_t) q_t . z_0
    S_T  = sum_s exp(L_T - L_s) k_s v_s^T + exp(L_T) S_0
    z_T  = sum_s exp(L_T - L_s) k_s       + exp(L_T) z_0
"""
import numpy as np


def _log_decay(decay_kind, log_g, b, h, T):
    if decay_kind == 0:
        return np.zeros(T)
    if decay_kind == 1:
        return np.full(T, float(log_g[h]))
    return np.asarray(log_g[b, h], dtype=np.float64)


def parallel_forward(q, k, v, decay_kind=0, log_g=None, normalize=False,
                     init_state=None, init_z=None):
    """q, k: [B,H,T,Dk]; v: [B,H,T,Dv]; float64.  Returns (y, S_T, z_T)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    y = np.zeros((B, H, T, Dv))
    S_T = np.zeros((B, H, Dk, Dv))
    z_T = np.zeros((B, H, Dk))
    for b in range(B):
        for h in range(H):
            S0 = np.zeros((Dk, Dv)) if init_state is None else init_state[b, h]
            z0 = np.zeros(Dk) if init_z is None else init_z[b, h]
            ell = _log_decay(decay_kind, log_g, b, h, T)
            L = np.cumsum(ell)
            causal = np.tril(np.ones((T, T), dtype=bool))
            D = np.zeros((T, T))
            diff = L[:, None] - L[None, :]
            D[causal] = np.exp(diff[causal])
            A = (q[b, h] @ k[b, h].T) * D
            num = A @ v[b, h] + np.exp(L)[:, None] * (q[b, h] @ S0)
            if normalize:
                den = A.sum(axis=1) + np.exp(L) * (q[b, h] @ z0)
                y[b, h] = num / den[:, None]
            else:
                y[b, h] = num
            LT = L[-1] if T > 0 else 0.0
            w = np.exp(LT - L)
            S_T[b, h] = (k[b, h] * w[:, None]).T @ v[b, h] + np.exp(LT) * S0
            z_T[b, h] = (k[b, h] * w[:, None]).sum(axis=0) + np.exp(LT) * z0
    return y, S_T, z_T


def parallel_reverse(q, k, v, decay_kind=0, log_g=None, normalize=False,
                     init_state=None, init_z=None):
    """Anti-causal parallel form of the reverse scan (S_t = g_t S_{t+1} + k_t
    v_t^T), float64, stated independently of the recurrent oracle.  With
    R_t = sum_{r>=t} log g_r (suffix sums) the weight of token s >= t in y_t
    is prod_{r=t}^{s-1} g_r = exp(R_t - R_s), and the state entering from
    beyond the end reaches token t with exp(R_t):
        y_t   = sum_{s>=t} exp(R_t - R_s) (q_t . k_s) v_s + exp(R_t) q_t^T S_0
        den_t = sum_{s>=t} exp(R_t - R_s) (q_t . k_s)     + exp(R_t) q_t . z_0
        S_1   = sum_s exp(R_1 - R_s) k_s v_s^T + exp(R_1) S_0   (z_1 likewise)
    Returns (y, S_1, z_1)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, T, Dk = q.shape
    Dv = v.shape[-1]
    y = np.zeros((B, H, T, Dv))
    S_1 = np.zeros((B, H, Dk, Dv))
    z_1 = np.zeros((B, H, Dk))
    for b in range(B):
        for h in range(H):
            S0 = np.zeros((Dk, Dv)) if init_state is None else init_state[b, h]
            z0 = np.zeros(Dk) if init_z is None else init_z[b, h]
            ell = _log_decay(decay_kind, log_g, b, h, T)
            R = np.cumsum(ell[::-1])[::-1]
            anti = np.triu(np.ones((T, T), dtype=bool))
            D = np.zeros((T, T))
            diff = R[:, None] - R[None, :]
            D[anti] = np.exp(diff[anti])
            A = (q[b, h] @ k[b, h].T) * D
            num = A @ v[b, h] + np.exp(R)[:, None] * (q[b, h] @ S0)
            if normalize:
                den = A.sum(axis=1) + np.exp(R) * (q[b, h] @ z0)
                y[b, h] = num / den[:, None]
            else:
                y[b, h] = num
            R1 = R[0] if T > 0 else 0.0
            w = np.exp(R1 - R)
            S_1[b, h] = (k[b, h] * w[:, None]).T @ v[b, h] + np.exp(R1) * S0
            z_1[b, h] = (k[b, h] * w[:, None]).sum(axis=0) + np.exp(R1) * z0
    return y, S_1, z_1
