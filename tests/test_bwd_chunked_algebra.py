"""The chunked gradient algebra of the GPU gradient kernels, restated in numpy float64.

The kernels in ssd_bwd.cu evaluate the scan's reverse-mode derivative chunk by
chunk.  They never recompute the forward output: the one sum that needs it,
<gy_k, y_k - D x_k>, is rebuilt from a dC term and the pair terms.  Their
state passes carry the state and the adjoint across chunks.  This test
restates exactly that decomposition on the CPU and checks it against the
oracle's position-by-position adjoint (a separate derivation, in C).  A wrong
sign, index or decay in the decomposition fails here without a GPU.  The
GPU parity tests then compare the kernels with the same oracle.

Notation (scan order inside a chunk of Q positions k = 0 .. Q-1):
  cs_k = A sum_{j <= k} dt_j, cl = cs_{Q-1}
  E[k][s] = (C_k . B_s) exp(cs_k - cs_s) for s <= k,  F[k][s] = (x_k . gy_s) exp(cs_s - cs_k) for s >= k
  Sin, Gin: the state entering the chunk from the left, the adjoint entering from the right
"""
import numpy as np
import pytest

import oracle


def _chunked_bwd(x, dt, A, B, C, D, gy, direction, Q):
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    nc = L // Q
    per = H // G
    order = np.arange(L) if direction > 0 else np.arange(L)[::-1]      # scan position -> token
    gx = np.zeros_like(x)
    gdt = np.zeros_like(dt)
    gA = np.zeros(H)
    gD = np.zeros(H)
    gBh = np.zeros((b, L, H, N))
    gCh = np.zeros((b, L, H, N))
    for bi in range(b):
        for h in range(H):
            g = h // per
            tok = [order[c * Q:(c + 1) * Q] for c in range(nc)]
            X = [x[bi, t, h] for t in tok]
            GY = [gy[bi, t, h] for t in tok]
            DT = [dt[bi, t, h] for t in tok]
            Bc = [B[bi, t, g] for t in tok]
            Cc = [C[bi, t, g] for t in tok]
            cs = [A[h] * np.cumsum(d) for d in DT]
            cl = [c_[-1] for c_ in cs]
            # step 1: each chunk's own state sum and adjoint sum
            sf = [(np.exp(cl[c] - cs[c]) * DT[c])[:, None, None] * X[c][:, :, None] * Bc[c][:, None, :] for c in range(nc)]
            sf = [s_.sum(0) for s_ in sf]
            sg = [(np.exp(cs[c])[:, None, None] * GY[c][:, :, None] * Cc[c][:, None, :]).sum(0) for c in range(nc)]
            # step 2: the passes over chunks
            Sin = [np.zeros((P, N)) for _ in range(nc)]
            for c in range(1, nc):
                Sin[c] = np.exp(cl[c - 1]) * Sin[c - 1] + sf[c - 1]
            Gin = [np.zeros((P, N)) for _ in range(nc)]
            for c in range(nc - 2, -1, -1):
                Gin[c] = np.exp(cl[c + 1]) * Gin[c + 1] + sg[c + 1]
            gcs = np.zeros(L)
            u_all = np.zeros(L)
            for c in range(nc):
                k_idx = np.arange(Q)
                low = k_idx[None, :] <= k_idx[:, None]                     # s <= k
                E = (Cc[c] @ Bc[c].T) * np.exp(cs[c][:, None] - cs[c][None, :]) * low
                F = (X[c] @ GY[c].T) * np.exp(cs[c][None, :] - cs[c][:, None]) * low.T
                el = np.exp(cl[c] - cs[c])
                ek = np.exp(cs[c])
                # (k, p) outputs: the adjoint times B, dx, u
                gb = E.T @ GY[c]                                         # sum_{s >= k} E[s][k] gy_s
                go = Bc[c] @ Gin[c].T                                    # sum_n B_k[n] Gin[p][n]
                g_ = el[:, None] * go + gb
                gx[bi, tok[c], h] = DT[c][:, None] * g_ + (0.0 if D is None else D[h]) * GY[c]
                u = (X[c] * g_).sum(1)
                # (k, n) outputs: this head's dB and dC parts
                co = GY[c] @ Sin[c]                                      # sum_p gy_k[p] Sin[p][n]
                bo = X[c] @ Gin[c]
                gbv = F @ Cc[c]                                          # sum_{s >= k} F[k][s] C_s
                gcv = (F.T * DT[c][None, :]) @ Bc[c]                     # sum_{s <= k} F[s][k] dt_s B_s
                gBh[bi, tok[c], h] = DT[c][:, None] * (el[:, None] * bo + gbv)
                gCh[bi, tok[c], h] = ek[:, None] * co + gcv
                # <gy_k, y_k - D x_k> without y: exp(cs_k) C_k . co_k + sum_{s <= k} E[k][s] dt_s x_s . gy_k,
                # with x_s . gy_k = F[s][k] exp(cs_s - cs_k)
                xg_sk = F.T * np.exp(cs[c][None, :] - cs[c][:, None]) * low       # [k][s] = x_s . gy_k (s <= k)
                r1 = ek * (Cc[c] * co).sum(1) + (E * DT[c][None, :] * xg_sk).sum(1)
                r2 = np.diag(F)                                         # x_k . gy_k
                pos = c * Q + np.arange(Q)
                gcs[pos] = r1 - DT[c] * u
                u_all[pos] = u
                gD[h] += r2.sum()
            # step 4: suffix sums of gcs in scan order give ddt and dA
            suf = np.cumsum(gcs[::-1])[::-1]
            dts = dt[bi, order, h]
            gdt[bi, order, h] = u_all + A[h] * suf
            gA[h] += (dts * suf).sum()
    gB = gBh.reshape(b, L, G, per, N).sum(3)
    gC = gCh.reshape(b, L, G, per, N).sum(3)
    return {"x": gx, "dt": gdt, "A": gA, "B": gB, "C": gC, "D": None if D is None else gD}


@pytest.mark.parametrize("direction", [1, -1])
@pytest.mark.parametrize("dims,Q", [((2, 96, 2, 4, 8, 1), 32), ((1, 64, 4, 3, 5, 2), 16), ((1, 48, 2, 2, 3, 1), 48)])
def test_chunked_gradients_equal_the_adjoint(dims, Q, direction):
    b, L, H, P, N, G = dims
    rng = np.random.default_rng(100 + L + Q)
    x = rng.standard_normal((b, L, H, P))
    dt = np.log1p(np.exp(rng.standard_normal((b, L, H)) - 2.0))
    A = -np.exp(rng.uniform(0.0, np.log(8.0), H))
    B = rng.standard_normal((b, L, G, N)) / np.sqrt(N)
    C = rng.standard_normal((b, L, G, N)) / np.sqrt(N)
    D = rng.uniform(0.0, 1.0, H)
    gy = rng.standard_normal((b, L, H, P))
    ref = oracle.ssd_scan_bwd_f64(x, dt, A, B, C, D, direction, gy)
    got = _chunked_bwd(x, dt, A, B, C, D, gy, direction, Q)
    for k in ("x", "dt", "A", "B", "C", "D"):
        assert oracle.rel_err(got[k], ref[k]) <= 1e-11, k
