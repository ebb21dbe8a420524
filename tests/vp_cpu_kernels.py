"""CPU stand-in for the library's vocabulary-parallel kernels (test infrastructure only).

It produces and consumes the exchange format the header documents (per token, base-2
tempered units: m_s, l_s, m_t, l_t, a, e, x_label) from the definitions, in float64 NumPy on
top of the oracle's logit and gradient routines, so that the collective plumbing of
``full_vocab_kl_b200.vocab_parallel`` can run on gloo ranks without a GPU.
"""

import math

import numpy as np
import torch

import oracle

LOG2E = 1.0 / math.log(2.0)
LN2 = math.log(2.0)


def _np(t):
    return t.detach().cpu().numpy()


class CpuKernels:
    def state(self, h_s, W_s, h_t, W_t, labels, beta, tau, vocab_offset, ignore_index, workspace=None):
        lab = _np(labels)
        N, V = lab.shape[0], W_s.shape[0]
        st = np.zeros((7, N))
        rows = np.flatnonzero(lab != ignore_index)
        if len(rows):
            xs = oracle.tempered_logits(_np(h_s)[rows], _np(W_s), tau) * LOG2E
            xt = oracle.tempered_logits(_np(h_t)[rows], _np(W_t), tau) * LOG2E
            ms, mt = xs.max(1), xt.max(1)
            ps, pt = np.exp2(xs - ms[:, None]), np.exp2(xt - mt[:, None])
            st[0, rows], st[1, rows], st[2, rows], st[3, rows] = ms, ps.sum(1), mt, pt.sum(1)
            if beta == 1.0:
                st[4, rows] = (ps * (xs - xt)).sum(1)
            elif beta == 0.0:
                st[4, rows] = (pt * (xt - xs)).sum(1)
            st[5, rows] = (ps * (xs - ms[:, None])).sum(1)
            col = lab[rows] - vocab_offset
            inside = (col >= 0) & (col < V)
            xl = np.full(len(rows), np.nan)
            xl[inside] = xs[np.flatnonzero(inside), col[inside]]
            st[6, rows] = xl
        return torch.from_numpy(st.astype(np.float32)), None

    def combine(self, states, labels, beta, ignore_index, side):
        # masked rows hold zero states (l = 0); their values are computed and then discarded
        with np.errstate(divide="ignore", invalid="ignore"):
            return self._combine(states, labels, beta, ignore_index, side)

    def _combine(self, states, labels, beta, ignore_index, side):
        S = _np(states).astype(np.float64)
        lab = _np(labels)
        N = lab.shape[0]
        valid = lab != ignore_index
        out = {k: np.zeros(N) for k in ("loss_tok", "lse_s", "lse_t", "aux", "entropy_s", "logp_label")}
        M_s, M_t = S[:, 0].max(0), S[:, 2].max(0)
        ws, wt = np.exp2(S[:, 0] - M_s), np.exp2(S[:, 2] - M_t)
        ls, lt = (S[:, 1] * ws).sum(0), (S[:, 3] * wt).sum(0)
        L2s, L2t = M_s + np.log2(ls), M_t + np.log2(lt)
        e = ((S[:, 5] + (S[:, 0] - M_s) * S[:, 1]) * ws).sum(0)
        xl = np.full(N, np.nan)
        for k in range(S.shape[0] - 1, -1, -1):
            have = ~np.isnan(S[k, 6])
            xl[have] = S[k, 6][have]
        if beta == 1.0:
            kl = LN2 * ((S[:, 4] * ws).sum(0) / ls - L2s + L2t)
        elif beta == 0.0:
            kl = LN2 * ((S[:, 4] * wt).sum(0) / lt - L2t + L2s)
        else:
            kl = np.zeros(N)
        vals = {"loss_tok": kl, "aux": kl, "lse_s": LN2 * L2s, "lse_t": LN2 * L2t,
                "entropy_s": LN2 * (np.log2(ls) - e / ls), "logp_label": LN2 * (xl - L2s)}
        for k, v in vals.items():
            out[k][valid] = v[valid]
        res = {k: torch.from_numpy(v.astype(np.float32)) for k, v in out.items()
               if side or k not in ("entropy_s", "logp_label")}
        nv = int(valid.sum())
        res["loss_mean"] = torch.tensor(float(out["loss_tok"].sum() / nv) if nv else 0.0)
        res["n_valid"] = torch.tensor(nv)
        return res

    def jsd_partial(self, h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, ignore_index, workspace=None):
        lab = _np(labels)
        part = np.zeros((2, lab.shape[0]))
        rows = np.flatnonzero(lab != ignore_index)
        logS = oracle.tempered_logits(_np(h_s)[rows], _np(W_s), tau) - _np(lse_s)[rows][:, None]
        logT = oracle.tempered_logits(_np(h_t)[rows], _np(W_t), tau) - _np(lse_t)[rows][:, None]
        logM = np.logaddexp(math.log1p(-beta) + logS, math.log(beta) + logT)
        ks = (np.exp(logS) * (logS - logM)).sum(1)
        kt = (np.exp(logT) * (logT - logM)).sum(1)
        part[0, rows] = beta * kt + (1.0 - beta) * ks
        part[1, rows] = ks
        return torch.from_numpy(part.astype(np.float32))

    def jsd_combine(self, parts, labels, ignore_index):
        P = _np(parts).astype(np.float64)
        lab = _np(labels)
        valid = lab != ignore_index
        loss = np.where(valid, P[:, 0].sum(0), 0.0)
        aux = np.where(valid, P[:, 1].sum(0), 0.0)
        nv = int(valid.sum())
        return {"loss_tok": torch.from_numpy(loss.astype(np.float32)),
                "aux": torch.from_numpy(aux.astype(np.float32)),
                "loss_mean": torch.tensor(float(loss.sum() / nv) if nv else 0.0), "n_valid": torch.tensor(nv)}

    def backward(self, h_s, W_s, h_t, W_t, labels, beta, tau, lse_s, lse_t, aux, grad_out, ignore_index,
                 workspace=None):
        lab = _np(labels)
        hs = _np(h_s).astype(np.float64)
        rows = np.flatnonzero(lab != ignore_index)
        dh = np.zeros_like(hs)
        dW = np.zeros((W_s.shape[0], hs.shape[1]))
        if len(rows):
            logS = oracle.tempered_logits(hs[rows], _np(W_s), tau) - _np(lse_s)[rows][:, None]
            logT = oracle.tempered_logits(_np(h_t)[rows], _np(W_t), tau) - _np(lse_t)[rows][:, None]
            a = _np(aux)[rows].astype(np.float64)
            G = float(grad_out) / (len(rows) * tau) * oracle.dloss_du_student(logS, logT, beta, a, a)
            dh[rows] = G @ _np(W_s).astype(np.float64)
            dW = G.T @ hs[rows]
        return torch.from_numpy(dh), torch.from_numpy(dW)
