"""A CPU stand-in of one rank's ``post_weight_pruning_b200.Sweep`` for the host-loop tests.

It takes the same steps and exposes the same exchanged buffers as the library's stepwise
sweep -- the level-1 histogram of key bits [30:18] with the rank's removal count appended,
the predicted and re-read level-2 histograms of key bits [17:0] with their 512-bin
summaries, the per-column counts of tied entries -- so ``sharded.global_sweep`` and its
collectives run unchanged over gloo ranks on CPU.  The arithmetic is numpy (fp64 updates,
fp32 score keys, as the kernels key their scores); Thanos, unstructured budget only.  It is
test infrastructure and does not import the oracle."""
import math

import numpy as np
import torch

LO_BITS = 18
N1 = 1 << (31 - LO_BITS)
N2 = 1 << LO_BITS
NS = N2 >> 9


class NumpySweep:
    def __init__(self, W_local, H, c_total, world, rank, *, sparsity=0.5, block=8, damp=0.01):
        self.W = np.array(W_local, dtype=np.float64)
        self.c, self.b = self.W.shape
        self.H = np.array(H, dtype=np.float64)
        self.c_total, self.world, self.rank = int(c_total), int(world), int(rank)
        self.s, self.B, self.damp = float(sparsity), int(block), float(damp)
        self.nblk = -(-self.b // self.B)
        self.level1 = torch.zeros(N1 + 1, dtype=torch.int32)
        self.level2 = torch.zeros(2 * (N2 + NS), dtype=torch.int32)
        self.ties = torch.zeros(128, dtype=torch.int32)
        self.ties_all = torch.zeros((world, 128), dtype=torch.int32)

    # the level-2 buffer: predicted histogram and summary, then the re-read ones
    def _h2(self, which):
        v = self.level2.numpy()
        o = 0 if which == "pred" else N2 + NS
        return v[o:o + N2], v[o + N2:o + N2 + NS]

    def _keys(self, j):
        S = np.abs(self.W[:, j:]) * np.sqrt(self.g[j:])[None, :]
        return S.astype(np.float32).view(np.uint32) & np.uint32(0x7FFFFFFF)

    def step(self, name, t=0):
        getattr(self, "_" + name)(t)

    def _setup(self, t):
        lam = self.damp * float(np.mean(np.diag(self.H)))
        Hinv = np.linalg.inv(self.H + lam * np.eye(self.b))
        self.U = np.linalg.cholesky(0.5 * (Hinv + Hinv.T)).T
        self.g = 0.5 * np.diag(self.H)
        self.mask = np.zeros((self.c, self.b), dtype=bool)
        self.zstar = int(math.floor(self.s * self.c_total * self.b))
        self.pruned = 0
        self.b1, self.b1_valid = 0, False

    def _score(self, t):
        j = t * self.B
        self.keys = self._keys(j)
        v = self.level1.numpy()
        v[:N1] = np.bincount((self.keys >> LO_BITS).ravel(), minlength=N1).astype(np.int32)
        v[N1] = self.pruned
        if self.b1_valid:                         # the previous block's bin, counted as it goes
            h2, hs = self._h2("pred")
            lo = self.keys[(self.keys >> LO_BITS) == self.b1] & np.uint32(N2 - 1)
            h2[:] = np.bincount(lo, minlength=N2)
            hs[:] = h2.reshape(NS, -1).sum(axis=1)

    def _pick_bin(self, t):
        j = t * self.B
        v = self.level1.numpy()
        r = self.zstar - int(v[N1])
        self.take = max(0, min(r, self.c_total * (self.b - j)))
        self.mode = self.take > 0
        if self.mode:
            cum = np.cumsum(v[:N1].astype(np.int64))
            b1 = int(np.searchsorted(cum, self.take))
            self.l2_ready = self.b1_valid and self.b1 == b1
            self.count_less = int(cum[b1 - 1]) if b1 > 0 else 0
            self.b1, self.b1_valid = b1, True
        v[:] = 0

    def _reread(self, t):
        if self.mode and not self.l2_ready:
            h2, hs = self._h2("reread")
            lo = self.keys[(self.keys >> LO_BITS) == self.b1] & np.uint32(N2 - 1)
            h2[:] = np.bincount(lo, minlength=N2)
            hs[:] = h2.reshape(NS, -1).sum(axis=1)

    def _pick_key(self, t):
        if not self.mode:
            return
        h2, _ = self._h2("pred" if self.l2_ready else "reread")
        cum = np.cumsum(h2.astype(np.int64))
        lo = int(np.searchsorted(cum, self.take - self.count_less))
        before = int(cum[lo - 1]) if lo > 0 else 0
        self.T = np.uint32((self.b1 << LO_BITS) | lo)
        self.m = self.take - self.count_less - before
        self.tie_scan = self.m < int(h2[lo])

    def _count_ties(self, t):
        v = self.ties.numpy()
        v[:] = 0
        if self.mode and self.tie_scan:
            nJ = min(self.B, self.b - t * self.B)
            v[:nJ] = (self.keys[:, :nJ] == self.T).sum(axis=0)

    def _cut_ties(self, t):
        self.pstar = math.inf
        if not (self.mode and self.tie_scan):
            return
        nJ = min(self.B, self.b - t * self.B)
        allc = self.ties_all.numpy().astype(np.int64)
        cum = 0
        for qq in range(nJ):
            cq = int(allc[:, qq].sum())
            if cum + cq >= self.m:
                need = self.m - cum - int(allc[:self.rank, qq].sum())
                mine = int(allc[self.rank, qq])
                if need <= 0:
                    self.pstar = qq * self.c - 1
                elif need >= mine:
                    self.pstar = qq * self.c + self.c - 1
                else:
                    rows = np.flatnonzero(self.keys[:, qq] == self.T)
                    self.pstar = qq * self.c + int(rows[need - 1])
                return
            cum += cq

    def _solve(self, t):
        self.level2.zero_()
        j = t * self.B
        j1 = min(self.b, j + self.B)
        nJ = j1 - j
        if not self.mode:
            return
        kb = self.keys[:, :nJ]
        pos = np.arange(nJ)[None, :] * self.c + np.arange(self.c)[:, None]
        sel = (kb < self.T) | ((kb == self.T) & (pos <= self.pstar))
        K = self.U[j:j1, j:j1].T @ self.U[j:j1, j:]
        for k in range(self.c):
            Q = np.flatnonzero(sel[k])
            if Q.size == 0:
                continue
            z = np.linalg.solve(K[np.ix_(Q, Q)], self.W[k, j + Q])
            self.W[k, j:] -= z @ K[Q, :]
            self.W[k, j + Q] = 0.0
        self.mask[:, j:j1] = sel
        self.pruned += int(sel.sum())

    def _finish(self, t):
        pass
