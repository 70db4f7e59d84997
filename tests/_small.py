"""Small seeded problems for oracle pins and tiny parity cases."""
from dataclasses import dataclass

import numpy as np
import torch

TAG = 1 << 30


def bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(b):
    return torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()


@dataclass
class Small:
    q: np.ndarray
    k_raw: np.ndarray
    v_raw: np.ndarray
    pt_raw: np.ndarray
    k_cmp: np.ndarray
    v_cmp: np.ndarray
    pt_cmp: np.ndarray
    req: np.ndarray
    pos: np.ndarray
    topk: np.ndarray
    sink: np.ndarray
    scale: float
    W: int
    ratio: int


def small_problem(seed=0, B=2, S=40, H=4, d=16, W=9, ratio=4, K=5, ps=4, qscale=1.0):
    rng = np.random.default_rng(seed)
    N = B * S
    pos = np.tile(np.arange(S, dtype=np.int32), B)
    req = np.repeat(np.arange(B, dtype=np.int32), S)
    q = bf16_bits(qscale * rng.standard_normal((N, H, d)))
    cols = -(-S // ps)
    P = 2 * B * cols
    k_raw = bf16_bits(rng.standard_normal((P, ps, d)))
    v_raw = bf16_bits(rng.standard_normal((P, ps, d)))
    pt_raw = rng.permutation(P)[: B * cols].reshape(B, cols).astype(np.int32)
    G = max(1, S // max(ratio, 1))
    ccols = -(-G // ps)
    Pc = 2 * B * ccols
    k_cmp = bf16_bits(rng.standard_normal((Pc, ps, d)))
    v_cmp = bf16_bits(rng.standard_normal((Pc, ps, d)))
    pt_cmp = rng.permutation(Pc)[: B * ccols].reshape(B, ccols).astype(np.int32)
    topk = np.full((N, K), -1, dtype=np.int32)
    for i, p in enumerate(pos):
        nc = (p + 1) // max(ratio, 1) if ratio else 0
        take = min(K, nc)
        if take:
            topk[i, :take] = rng.choice(nc, take, replace=False)
    sink = rng.standard_normal(H).astype(np.float32)
    return Small(q, k_raw, v_raw, pt_raw, k_cmp, v_cmp, pt_cmp, req, pos, topk, sink,
                 1.0 / np.sqrt(d), W, ratio)


def gather_rows(pr: Small, b, keys):
    """K and V rows (FP64) of the given keys of request b, by page table."""
    ks, vs = [], []
    for key in keys:
        key = int(key)
        if key & TAG:
            t = key & (TAG - 1)
            pool_k, pool_v, pt = pr.k_raw, pr.v_raw, pr.pt_raw
        else:
            t = key
            pool_k, pool_v, pt = pr.k_cmp, pr.v_cmp, pr.pt_cmp
        ps = pool_k.shape[1]
        page = pt[b, t // ps]
        ks.append(pool_k[page, t % ps])
        vs.append(pool_v[page, t % ps])
    d = pr.k_raw.shape[2]
    if not ks:
        return np.zeros((0, d)), np.zeros((0, d))
    return bits_to_f64(np.stack(ks)), bits_to_f64(np.stack(vs))


def run_oracle(oracle, pr: Small, indptr, indices, rows=None, include_sink=True, sink=None):
    return oracle.sparse_sink_attn(
        pr.q, pr.k_raw, pr.v_raw, pr.pt_raw, pr.req, indptr, indices,
        pr.sink if sink is None else sink, pr.scale,
        k_cmp=pr.k_cmp, v_cmp=pr.v_cmp, pt_cmp=pr.pt_cmp, rows=rows,
        include_sink=include_sink, threads=2)
