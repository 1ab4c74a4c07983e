"""Host-side bookkeeping of the oracle's hybrid KV cache (numpy only).

TEST INFRASTRUCTURE ONLY.  This file decides which position lives in which
segment of the cache; every number it stores comes from the oracle's own
quantizer (``hyq_oracle.c`` via :func:`oracle.pack`) or is an input copied
verbatim.

Segments per unit (b, kv head), following the three token classes of the
aifromscratch.in explainer ("How It Works"):
  * quantized majority: packed INT4 codes + fp16 (scale, zero) for every
    position that has left the local window, [0, T - W);
  * vertical-line tokens: FP16 K/V rows of the selected positions, in
    ascending position order;
  * local window: FP16 K/V of the last W positions in a ring, slot = p % W.

Readings where the pages are silent:
  * every token is packed when it leaves the window, VL or not, so codes
    exist for all of [0, T - W);
  * re-selection from the cache keeps FP16 rows only for positions selected
    again; newly selected positions have no FP16 source left and stay INT4
    ("unpromoted"); dropped positions fall back to their codes.

Staged promotion (optional, ``stage`` > 0; the pages say nothing about it):
the FP16 rows of the ``stage`` most recently quantized positions, [T - W -
stage, T - W), are also kept in a ring (slot = p % stage), filled from the
prompt and by every append with the row leaving the window.  A cache-mode
re-selection then promotes a newly selected position from that ring when it
lies in the staged range and is newer than every position kept from the
previous set (promoted rows follow the kept rows, which then only move to
lower slots); other new positions stay unpromoted.  With re-selection every
64 tokens every staged position is newer than the whole previous set.
"""
from __future__ import annotations

import numpy as np

from . import D, ROW_BYTES, pack


class OracleCache:
    def __init__(self, B, Hq, Hkv, cap, vl_cap, W=128, stage=0):
        assert Hq % Hkv == 0
        vl_cap = max(int(vl_cap), 1)
        self.B, self.Hq, self.Hkv, self.cap, self.vl_cap, self.W = B, Hq, Hkv, cap, vl_cap, W
        U = B * Hkv
        self.stage = int(stage)
        self.stage_k = np.zeros((U, max(self.stage, 1), D), np.uint16)
        self.stage_v = np.zeros((U, max(self.stage, 1), D), np.uint16)
        self.k_codes = np.zeros((U, cap, ROW_BYTES), np.uint8)
        self.v_codes = np.zeros((U, cap, ROW_BYTES), np.uint8)
        self.k_sz = np.zeros((U, cap, 8), np.uint16)
        self.v_sz = np.zeros((U, cap, 8), np.uint16)
        self.win_k = np.zeros((U, W, D), np.uint16)
        self.win_v = np.zeros((U, W, D), np.uint16)
        self.vl_k = np.zeros((U, vl_cap, D), np.uint16)
        self.vl_v = np.zeros((U, vl_cap, D), np.uint16)
        self.vl_pos = np.full((U, vl_cap), -1, np.int32)
        self.vl_count = np.zeros(U, np.int32)
        self.seq_len = np.zeros(B, np.int32)

    # ------------------------------------------------------------ prompt
    def load_prompt(self, K, V, seq_len, units=None):
        """K, V: [B][Hkv][>=T][128] fp16 (as uint16 bits or float16).
        Packs [0, T-W) and fills the window with [max(0, T-W), T).  With
        `units`, only those (b * Hkv + h) units are filled."""
        K = np.asarray(K).view(np.uint16)
        V = np.asarray(V).view(np.uint16)
        seq_len = np.asarray(seq_len, np.int32)
        keep = None if units is None else set(int(u) for u in units)
        for b in range(self.B):
            T = int(seq_len[b])
            assert 0 <= T <= self.cap
            self.seq_len[b] = T
            n_old = max(0, T - self.W)
            for h in range(self.Hkv):
                u = b * self.Hkv + h
                if keep is not None and u not in keep:
                    continue
                if n_old:
                    c, s, bad = pack(K[b, h, :n_old])
                    assert bad == 0
                    self.k_codes[u, :n_old], self.k_sz[u, :n_old] = c, s
                    c, s, bad = pack(V[b, h, :n_old])
                    assert bad == 0
                    self.v_codes[u, :n_old], self.v_sz[u, :n_old] = c, s
                for p in range(n_old, T):
                    self.win_k[u, p % self.W] = K[b, h, p]
                    self.win_v[u, p % self.W] = V[b, h, p]
                for p in range(max(0, n_old - self.stage), n_old):
                    self.stage_k[u, p % self.stage] = K[b, h, p]
                    self.stage_v[u, p % self.stage] = V[b, h, p]
                self.vl_count[u] = 0
                self.vl_pos[u] = -1

    def staged(self, b, p):
        """Whether position p of batch b has its FP16 rows in the staging ring."""
        n_old = int(self.seq_len[b]) - self.W
        return self.stage > 0 and max(0, n_old - self.stage) <= p < n_old

    # ------------------------------------------------------------ VL set
    def apply_vl(self, pos, K_full=None, V_full=None, units=None):
        """pos: [B][Hkv][k] ascending.  With K_full/V_full (prefill mode) the
        FP16 rows come from them; without (cache mode) only positions already
        held in FP16 stay FP16.  Returns the number of unpromoted positions."""
        pos = np.asarray(pos, np.int32)
        k = pos.shape[-1]
        assert k <= self.vl_cap
        unpromoted = 0
        if K_full is not None:
            K_full = np.asarray(K_full).view(np.uint16)
            V_full = np.asarray(V_full).view(np.uint16)
        keep = None if units is None else set(int(u) for u in units)
        for b in range(self.B):
            for h in range(self.Hkv):
                u = b * self.Hkv + h
                if keep is not None and u not in keep:
                    continue
                new = [int(p) for p in pos[b, h]]
                if K_full is not None:
                    rows_k = [K_full[b, h, p] for p in new]
                    rows_v = [V_full[b, h, p] for p in new]
                    kept = new
                else:
                    old = {int(self.vl_pos[u, i]): i for i in range(self.vl_count[u])}
                    last_kept = max([p for p in new if p in old], default=-1)
                    kept, rows_k, rows_v = [], [], []
                    for p in new:
                        if p in old:
                            src_k, src_v = self.vl_k[u, old[p]], self.vl_v[u, old[p]]
                        elif self.staged(b, p) and p > last_kept:
                            src_k, src_v = self.stage_k[u, p % self.stage], self.stage_v[u, p % self.stage]
                        else:
                            continue
                        kept.append(p)
                        rows_k.append(src_k.copy())
                        rows_v.append(src_v.copy())
                    unpromoted += len(new) - len(kept)
                self.vl_pos[u] = -1
                for i, p in enumerate(kept):
                    self.vl_pos[u, i] = p
                    self.vl_k[u, i] = rows_k[i]
                    self.vl_v[u, i] = rows_v[i]
                self.vl_count[u] = len(kept)
        return unpromoted

    # ------------------------------------------------------------ decode
    def append(self, k_new, v_new):
        """k_new, v_new: [B][Hkv][128] fp16.  The row leaving the window
        (position T - W) is packed first, then the new token takes its slot."""
        k_new = np.asarray(k_new).view(np.uint16)
        v_new = np.asarray(v_new).view(np.uint16)
        for b in range(self.B):
            T = int(self.seq_len[b])
            assert T + 1 <= self.cap
            slot = T % self.W
            for h in range(self.Hkv):
                u = b * self.Hkv + h
                if T >= self.W:
                    p_out = T - self.W
                    if self.stage:
                        self.stage_k[u, p_out % self.stage] = self.win_k[u, slot]
                        self.stage_v[u, p_out % self.stage] = self.win_v[u, slot]
                    c, s, bad = pack(self.win_k[u, slot])
                    assert bad == 0
                    self.k_codes[u, p_out], self.k_sz[u, p_out] = c[0], s[0]
                    c, s, bad = pack(self.win_v[u, slot])
                    assert bad == 0
                    self.v_codes[u, p_out], self.v_sz[u, p_out] = c[0], s[0]
                self.win_k[u, slot] = k_new[b, h]
                self.win_v[u, slot] = v_new[b, h]
            self.seq_len[b] = T + 1
