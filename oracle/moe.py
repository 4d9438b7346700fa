"""Grouped MoE GEMM of LUT3 expert weights with MXFP8 activations: the
token-to-expert alignment and the gathered product.

Test infrastructure only (see ``oracle/__init__.py``).

The vLLM PR 62759 write-up's native grouped GEMM (its sections on gathering A
and on expert parallelism): token rows are gathered through
``sorted_token_ids``, the output of ``moe_align_block_size``, which lists the
(token, choice) pairs of each expert contiguously with each expert's run
padded to a multiple of the M block; the kernel takes one expert per M block,
fills the A rows of padding entries with zeros, and a block whose expert is
not on this rank (a negative id) writes zeros for its valid rows.

Readings taken where the page is silent:

* Pair p = t * top_k + j (token t, choice j) goes to expert topk_ids[t, j].
  The sorted ids hold p; the padding value is P = T * top_k (the number of
  pairs, one past the last valid id). Within an expert the pairs are listed in
  ascending p here; any order is as valid (each output row depends on its own
  pair only), and the device may list them in another order.
* Experts are visited in ascending id; an expert with no pairs gets no block.
  expert_ids[b] = expert_map[e] for the expert e whose run holds block b
  (the identity without a map; a negative entry marks an expert that is not
  local).
* Y[p, :] = A[p // top_k, :] . W_e for the local expert e of pair p (MXFP8
  dequantised activations times the exact LUT3 decode, FP64), Y[p, :] = 0 for
  a pair of a non-local expert. The weighted sum over a token's top_k choices
  comes after this GEMM, outside it, as in the page's kernel.
"""

import numpy as np

from . import lut3, mxfp8


def align(topk_ids, num_experts, block):
    """moe_align_block_size: (sorted_ids int32 [total], expert_ids int32
    [total / block] (global ids), total) for topk_ids int [T, top_k]."""
    ids = np.asarray(topk_ids).reshape(-1)
    P = ids.size
    if np.any(ids < 0) or np.any(ids >= num_experts):
        raise ValueError("expert ids out of range")
    sorted_ids, expert_ids = [], []
    for e in range(num_experts):
        pairs = np.flatnonzero(ids == e).tolist()  # ascending p
        if not pairs:
            continue
        padded = -(-len(pairs) // block) * block
        sorted_ids.extend(pairs + [P] * (padded - len(pairs)))
        expert_ids.extend([e] * (padded // block))
    return np.array(sorted_ids, dtype=np.int32), np.array(expert_ids, dtype=np.int32), len(sorted_ids)


def max_padded(P, num_experts, block):
    """Largest total align can return for P pairs: each of at most min(P, E)
    non-empty runs adds fewer than `block` padding entries, and the total is a
    multiple of `block`."""
    return (P + min(P, num_experts) * (block - 1)) // block * block


def _local(e, expert_map):
    return int(e) if expert_map is None else int(expert_map[e])


def grouped_matmul(codes, scales, top_k, sorted_ids, expert_ids, total, block, experts, expert_map=None):
    """The gathered form: Y float64 [P, N] from the aligned lists. experts[i] =
    (idx, codebooks, exponents) of local expert i; expert_ids hold global ids
    (mapped through expert_map here)."""
    Xq = mxfp8.dequant(codes, scales)
    P = Xq.shape[0] * top_k
    N = experts[0][0].shape[1]
    Y = np.full((P, N), np.nan)
    for b in range(total // block):
        e = _local(expert_ids[b], expert_map)
        W = lut3.dequant(*experts[e]) if e >= 0 else None
        for p in sorted_ids[b * block:(b + 1) * block]:
            if p >= P:
                continue  # padding
            Y[p] = 0.0 if W is None else Xq[p // top_k] @ W
    return Y


def routed_matmul(codes, scales, topk_ids, experts, expert_map=None):
    """The definition, pair by pair without any sorting: Y[t * top_k + j] =
    A[t] . W_{topk_ids[t, j]} (zeros for a non-local expert)."""
    Xq = mxfp8.dequant(codes, scales)
    T, top_k = np.asarray(topk_ids).shape
    N = experts[0][0].shape[1]
    Ws = {}
    Y = np.zeros((T * top_k, N))
    for t in range(T):
        for j in range(top_k):
            e = _local(topk_ids[t][j], expert_map)
            if e < 0:
                continue
            if e not in Ws:
                Ws[e] = lut3.dequant(*experts[e])
            Y[t * top_k + j] = Xq[t] @ Ws[e]
    return Y
