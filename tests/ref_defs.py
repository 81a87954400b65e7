"""Independent numpy-float64 statements of the WKV definitions, used to pin the oracle.

These are NOT the oracle's recurrences retyped: they evaluate the unrolled
O(T^2) sums (WKV-4) and the unrolled state sums with explicit decay products
(WKV-6) term by term, the way the definitions read before any recurrence is
derived, and they are only meant for tiny inputs.

  * WKV-4 ("RWKV: Reinventing RNNs for the Transformer Era", eq. 14 as referenced
    in the temporal-structure section):
      wkv_t = (sum_{i<t} e^{-(t-1-i)w + k_i} v_i + e^{u+k_t} v_t)
            / (sum_{i<t} e^{-(t-1-i)w + k_i}     + e^{u+k_t})
    plus, with a carried state (num0, den0) = (a e^p, b e^p), the extra terms
    e^{-t w} num0 and e^{-t w} den0.  Every term of one t is scaled by the same
    e^{-m} (m = the largest exponent), which leaves the ratio unchanged.
  * WKV-6 ("RWKV-5/6 (Eagle and Finch)", sections 4.1.2 and 4.2.2):
      o_t = r_t ( prod_{m<t} diag(w_m) s0
                  + sum_{tau<t} prod_{m=tau+1}^{t-1} diag(w_m) k_tau^T v_tau
                  + diag(u) k_t^T v_t )
      sT  = prod_{m<T} diag(w_m) s0 + sum_{tau<T} prod_{m=tau+1}^{T-1} diag(w_m) k_tau^T v_tau
"""
import numpy as np


def wkv4_sums(w, u, k, v, s0=None):
    """Returns (y [B,T,C], num_T [B,C], den_T [B,C]) with num/den in absolute scale."""
    w = np.asarray(w, np.float64)
    u = np.asarray(u, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, T, C = k.shape
    y = np.empty((B, T, C))
    num_end = np.zeros((B, C))
    den_end = np.zeros((B, C))
    for b in range(B):
        for c in range(C):
            if s0 is not None:
                a0, b0, p0 = (float(s0[b, 0, c]), float(s0[b, 1, c]), float(s0[b, 2, c]))
            else:
                a0, b0, p0 = 0.0, 0.0, -np.inf
            for t in range(T + 1):
                # exponents and values of every term present at time t
                expo = [-(t - 1 - i) * w[c] + k[b, i, c] for i in range(t)]
                vals = [v[b, i, c] for i in range(t)]
                if a0 != 0.0 or b0 != 0.0:
                    expo.append(p0 - t * w[c])
                    vals.append(None)           # the carried state
                if t < T:
                    expo.append(u[c] + k[b, t, c])
                    vals.append(v[b, t, c])
                m = max(expo)
                num = 0.0
                den = 0.0
                for e, val in zip(expo, vals):
                    f = np.exp(e - m)
                    if val is None:
                        num += f * a0
                        den += f * b0
                    else:
                        num += f * val
                        den += f
                if t < T:
                    y[b, t, c] = num / den
                else:
                    # state after the last token: all past terms, no bonus term
                    num_end[b, c] = num * np.exp(m) if np.isfinite(m) else 0.0
                    den_end[b, c] = den * np.exp(m) if np.isfinite(m) else 0.0
    return y, num_end, den_end


def wkv4_def(w, u, k, v, s0=None):
    return wkv4_sums(w, u, k, v, s0)[0]


def wkv6_def(r, k, v, w, u, s0=None):
    """Unrolled-sum WKV-6.  Shapes as the ABI: [B,T,H,N], u [H,N], s0 [B,H,N,N]."""
    r, k, v, w = (np.asarray(x, np.float64) for x in (r, k, v, w))
    u = np.asarray(u, np.float64)
    B, T, H, N = r.shape
    y = np.empty((B, T, H, N))
    sT = np.empty((B, H, N, N))
    for b in range(B):
        for h in range(H):
            s_init = np.zeros((N, N)) if s0 is None else np.asarray(s0[b, h], np.float64)

            def state_before(t):
                # prod_{m<t} diag(w_m) s0 + sum_{tau<t} prod_{m=tau+1}^{t-1} diag(w_m) k^T v
                d0 = np.ones(N)
                for m in range(t):
                    d0 = d0 * w[b, m, h]
                S = d0[:, None] * s_init
                for tau in range(t):
                    d = np.ones(N)
                    for m in range(tau + 1, t):
                        d = d * w[b, m, h]
                    S = S + (d * k[b, tau, h])[:, None] * v[b, tau, h][None, :]
                return S

            for t in range(T):
                S = state_before(t)
                bonus = (u[h] * k[b, t, h])[:, None] * v[b, t, h][None, :]
                y[b, t, h] = r[b, t, h] @ (S + bonus)
            sT[b, h] = state_before(T)
    return y, sT


def causal_linear_attention(R, K, V, u, s0):
    """Single head with no decay (w = 1): textbook masked matmul form.

    O = (strict_lower(R K^T) + diag(R diag(u) K^T)) V + R s0 ;  sT = s0 + K^T V.
    """
    R, K, V = (np.asarray(x, np.float64) for x in (R, K, V))
    scores = R @ K.T
    A = np.tril(scores, k=-1) + np.diag(np.einsum("ti,i,ti->t", R, u, K))
    return A @ V + R @ s0, s0 + K.T @ V
