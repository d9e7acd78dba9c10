"""The two stages of a context-parallel prefill rank written with the oracle's
functions (test-side stand-in for libhca's hybrid_cp_compress / hybrid_cp_attend),
so that the partitioning and exchange logic of the CP driver can run on CPU
gloo ranks and be compared with the oracle's whole-sequence layer."""
import numpy as np
import torch

from oracle import hca_oracle as O


class OracleCPStages:
    def __init__(self, L, W64, d_c, B=1, eps=1e-6, theta=10000.0):
        self.L, self.W, self.d_c, self.B, self.eps, self.theta = L, W64, d_c, B, eps, theta
        self.m = L.m
        self.csa = L.kind == "csa"

    def halo(self, t0):
        if t0 <= 0:
            return 0
        need = max(self.L.w - 1, self.m if (self.csa and self.L.overlap) else 0)
        return min(t0, need)

    def compress(self, H, t0, n_loc):
        L, W, m = self.L, self.W, self.m
        h = self.halo(t0)
        hb = m if (self.csa and L.overlap and t0 > 0) else 0
        kv, kI = [], []
        for b in range(H.shape[0]):
            Hc = H[b, h - hb:].double().numpy()
            P = lambda nm: O.project(Hc, W[nm])
            if self.csa:
                ent = O.compress_prefill(P("W_aKV"), P("W_aZ"), W["B_a"], m, P("W_bKV"), P("W_bZ"), W["B_b"])
                entI = O.compress_prefill(P("W_IaKV"), P("W_IaZ"), W["B_Ia"], m, P("W_IbKV"), P("W_IbZ"), W["B_Ib"])
                entI = entI[hb // m:]
                kI.append(O.entry_epilogue(entI, m, first_entry=t0 // m, eps=self.eps, rd=L.rd_I, theta=self.theta))
            else:
                ent = O.compress_prefill(P("W_KVc"), P("W_Zc"), W["B"], m)
            ent = ent[hb // m:]
            kv.append(O.entry_epilogue(ent, m, first_entry=t0 // m, eps=self.eps, rd=L.rd, theta=self.theta))
        t = lambda xs: torch.from_numpy(np.stack(xs))
        return t(kv), (t(kI) if self.csa else None), None

    def attend(self, H, t0, n_loc, kv, kI, kIs):
        L, W = self.L, self.W
        h = self.halo(t0)
        c = L.c
        out = np.zeros((H.shape[0], n_loc, L.n_h, c))
        for b in range(H.shape[0]):
            Hb = H[b].double().numpy()
            own = Hb[h:]
            pos = t0 + np.arange(n_loc)
            win = O.rope(O.rmsnorm(O.project(Hb, W["W_KV"]), eps=self.eps), t0 - h + np.arange(h + n_loc), L.rd,
                         self.theta)
            cQ = O.rmsnorm(O.project(own, W["W_DQ"]), eps=self.eps)
            q = O.rope(O.rmsnorm(O.project(cQ, W["W_UQ"]).reshape(n_loc, L.n_h, c), eps=self.eps), pos[:, None],
                       L.rd, self.theta)
            kvb = kv[b].double().numpy()
            if self.csa:
                qI = O.rope(O.project(cQ, W["W_IUQ"]).reshape(n_loc, L.n_hI, L.c_I), pos[:, None], L.rd_I, self.theta)
                wI = O.project(own, W["W_w"]) * (L.c_I ** -0.5 * L.n_hI ** -0.5)
                KI = kI[b].double().numpy()
            for j, t in enumerate(pos):
                V = O.visible_entries(int(t), self.m)
                if self.csa:
                    idx = O.topk_select(O.index_scores(qI[j], wI[j], KI, V), L.k)
                    comp = kvb[idx[idx >= 0]]
                else:
                    comp = kvb[:V]
                wp = O.window_positions(int(t), L.w)
                rows = np.concatenate([win[wp - (t0 - h)], comp], axis=0) if L.w else comp
                out[b, j] = O.attend_output(q[j], rows, W["sink"], c ** -0.5, int(t), L.rd, self.theta)
        return torch.from_numpy(out)
