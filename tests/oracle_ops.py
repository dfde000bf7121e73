"""Stand-in for the library calls the entry-range sharded decoder makes,
computed by the oracle on CPU tensors (TEST INFRASTRUCTURE). It lets the
sharding logic (ranges, local ids, key exchange, selection from the union,
window on the first shard, log-sum-exp merge) run on CPU ranks and be checked
against the unsharded oracle. Caches hold one sequence in one page.

Keys follow the library's contract: a 64-bit value whose high half orders by
score and whose low half is the complement of the global id, so larger keys
are higher scores and, on equal scores, lower ids; 0 is empty."""
import math

import numpy as np
import torch

import oracle


class KvCache:
    def __init__(self, codes, scales, kidx, page_table, seq_len, page_size):
        self.codes, self.scales, self.kidx = codes, scales, kidx
        self.page_table, self.seq_len = page_table, seq_len
        self.page_size = int(page_size)


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _n(kv):
    return int(kv.seq_len[0])


def workspace(nbytes, device):
    return None


def csa2_index_full_workspace_size(nq, n_max):
    return 0


def csa2_sparse_attn_workspace_size(nq, h, k, w_max):
    return 0


def csa2_append_fp4(x_bf16, seq, pos, kv):
    codes, scales = oracle.quantize_rows(_bits(x_bf16))
    p = pos.numpy()
    kv.codes.numpy()[p] = codes
    kv.scales.numpy()[p] = scales


def csa2_index_full(qidx, w, q_per_seq, q_limit, n_max, kv, k, p, topk, pool, ws):
    assert q_limit is None
    n = _n(kv)
    for qi in range(qidx.shape[0]):
        tk, pl = oracle.index_full(qidx[qi].numpy(), w[qi].numpy(), kv.kidx.numpy()[:max(n, 1)],
                                   np.zeros(1, np.int32), max(n, 1), n, k, p)
        topk[qi] = torch.from_numpy(tk)
        if p > 0:
            pool[qi] = torch.from_numpy(pl)


def _score_key(s):
    b = int(np.array([s + 0.0], np.float32).view(np.uint32)[0])
    return (~b & 0xFFFFFFFF) if b & 0x80000000 else (b | 0x80000000)


def csa2_score_ids(qidx, w, q_per_seq, ids, kv, id_offset, keys):
    kidx = kv.kidx.numpy()
    out = np.zeros(ids.shape, np.uint64)
    for qi in range(ids.shape[0]):
        q, wq = qidx[qi].numpy(), w[qi].numpy()
        for j, i in enumerate(ids[qi].tolist()):
            if i < 0:
                continue
            s = oracle.index_score(q, wq, kidx[i])
            out[qi, j] = (_score_key(s) << 32) | (~(i + id_offset) & 0xFFFFFFFF)
    keys.copy_(torch.from_numpy(out.view(np.int64)))


def csa2_select_keys(keys, k, ids):
    kk = keys.numpy().view(np.uint64)
    res = np.full((kk.shape[0], k), -1, np.int32)
    for qi in range(kk.shape[0]):
        live = np.sort(kk[qi][kk[qi] != 0])[::-1][:k]
        res[qi, :live.size] = (~(live & np.uint64(0xFFFFFFFF)) & np.uint64(0xFFFFFFFF)).astype(np.int64)
    ids.copy_(torch.from_numpy(res))


def csa2_sparse_attn_partial(q_bf16, q_per_seq, kv, topk, swa, swa_seq_stride, swa_begin, swa_end, w_max,
                             softmax_scale, o_f32, lse, ws):
    n = max(_n(kv), 1)
    for qi in range(q_bf16.shape[0]):
        b = qi // q_per_seq
        rows = None
        if swa_begin is not None:
            wb, we = int(swa_begin[qi]), int(swa_end[qi])
            ring = swa.shape[1]
            rows = swa[b].numpy()[(wb + np.arange(we - wb)) % ring]
        o, l = oracle.sparse_attn(_bits(q_bf16[qi]), kv.codes.numpy()[:n], kv.scales.numpy()[:n],
                                  np.zeros(1, np.int32), n, topk[qi].numpy(), rows, softmax_scale)
        o_f32[qi] = torch.from_numpy(o)
        lse[qi] = torch.from_numpy(l)


def csa2_attn_merge(o_parts, lse_parts, o_bf16, lse):
    op = o_parts.double().numpy()
    lp = lse_parts.double().numpy()
    m = lp.max(axis=0)
    wts = np.where(np.isfinite(lp), np.exp(lp - np.where(np.isfinite(m), m, 0.0)), 0.0)
    tot = wts.sum(axis=0)
    o = (wts[..., None] * op).sum(axis=0) / np.where(tot > 0, tot, 1.0)[..., None]
    o_bf16.copy_(torch.from_numpy(o))
    if lse is not None:
        lse.copy_(torch.from_numpy(np.where(tot > 0, m + np.log(np.where(tot > 0, tot, 1.0)), -math.inf)))
