"""The expert-parallel layer's stages restated on the host with the oracle
(test infrastructure): the same interface as EpMoeLayer (route_and_pack,
experts, shared_and_combine, update_bias), numpy and torch CPU tensors
instead of the CUDA library, and the dispatch row format written out
independently from its documented layout:

  codes uint8 [d] | scales fp32 [d/128] | local expert of each slot int32
  [K] (-1: elsewhere) | gate of each slot fp32 [K] | source token int32 |
  zero padding to a multiple of 16 bytes.

Rank q owns routed experts [q E, (q+1) E), E = N_r / P; a token goes once to
each rank owning one of its experts, rows destination-major with tokens
ascending; the receiver's partial output of a row is the sum of its local
experts' outputs weighted by the gates (slot order), the source adds the
shared expert's output and the partial outputs (rank order), FP64 here, then
one bf16 rounding."""
from __future__ import annotations

import numpy as np
import torch

import oracle


def row_bytes(d, K):
    return (d + 4 * (d // 128) + 8 * K + 4 + 15) // 16 * 16


class OracleEpStages:
    def __init__(self, cfg, rank, n_ranks, router_w, bias, experts, x_bits, offset=None):
        self.cfg, self.rank, self.P = cfg, rank, n_ranks
        self.E = cfg.n_routed // n_ranks
        self.router_w, self.bias = router_w, np.asarray(bias, np.float32).copy()
        self.experts_w = experts   # e -> oracle-quantised weights
        self.x = x_bits            # uint16 [T, d]
        self.offset = offset
        self.device = torch.device("cpu")
        self.row_bytes = row_bytes(cfg.d, cfg.topk)

        class _S:  # the shape fields ep_forward reads
            pass
        self.shape = _S()
        self.shape.T, self.shape.d = x_bits.shape

    def route_and_pack(self, x, logit_offset=None):
        cfg, K, d = self.cfg, self.cfg.topk, self.cfg.d
        r = oracle.route(self.x, self.router_w, self.bias, cfg.n_groups, cfg.topk_groups, K,
                         logit_offset=self.offset)
        self.r = r
        self.counts = torch.from_numpy(r["counts"].astype(np.int32))
        q, s = oracle.quant_act_1x128(self.x)
        self.xq, self.xs = q, s
        dest = r["topk_idx"] // self.E            # [T, K] destination ranks
        rows = []
        self.send_row = np.full((self.x.shape[0], self.P), -1, np.int64)
        for p in range(self.P):
            for t in range(self.x.shape[0]):
                if not np.any(dest[t] == p):
                    continue
                self.send_row[t, p] = len(rows)
                buf = bytearray(self.row_bytes)
                buf[0:d] = q[t].tobytes()
                buf[d:d + 4 * (d // 128)] = s[t].astype("<f4").tobytes()
                o = d + 4 * (d // 128)
                slots = np.where(dest[t] == p, r["topk_idx"][t] - p * self.E, -1)
                gates = np.where(dest[t] == p, r["topk_gate"][t], 0.0).astype("<f4")
                buf[o:o + 4 * K] = slots.astype("<i4").tobytes()
                buf[o + 4 * K:o + 8 * K] = gates.tobytes()
                buf[o + 8 * K:o + 8 * K + 4] = np.int32(t).astype("<i4").tobytes()
                rows.append(np.frombuffer(bytes(buf), np.uint8))
        counts = [int(np.sum(np.any(dest == p, axis=1))) for p in range(self.P)]
        send = np.stack(rows) if rows else np.zeros((1, self.row_bytes), np.uint8)
        return torch.from_numpy(send.copy()), counts

    def experts(self, recv_buf, n_recv):
        cfg, K, d = self.cfg, self.cfg.topk, self.cfg.d
        rb = recv_buf.numpy()
        out = np.zeros((n_recv, d), np.float64)
        o0 = d + 4 * (d // 128)
        for j in range(n_recv):
            row = rb[j]
            codes = row[:d][None, :]
            scales = row[d:o0].view("<f4")[None, :]
            slots = row[o0:o0 + 4 * K].view("<i4")
            gates = row[o0 + 4 * K:o0 + 8 * K].view("<f4")
            for k in range(K):
                if slots[k] < 0:
                    continue
                e = self.rank * self.E + int(slots[k])
                out[j] += float(gates[k]) * oracle.swiglu_expert(codes, scales,
                                                                 *self.experts_w(e))[0]
        return torch.from_numpy(out)

    def shared_and_combine(self, x, back_recv):
        cfg = self.cfg
        y = oracle.swiglu_expert(self.xq, self.xs, *self.experts_w(cfg.n_routed)).copy()
        br = back_recv.numpy()
        for t in range(self.x.shape[0]):
            for p in range(self.P):
                if self.send_row[t, p] >= 0:
                    y[t] += br[self.send_row[t, p]]
        return torch.from_numpy(oracle.f64_to_bf16_bits(y).view(np.int16))

    def update_bias(self, global_counts, total_tokens):
        self.bias = oracle.update_bias(global_counts.numpy(), self.bias, total_tokens,
                                       self.cfg.topk, self.cfg.gamma)
