"""CPU oracle of the token Compressor -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this module.  It shares no code with the CUDA library and the library
never calls it.

Source: aclnnCompressor (CANN ops-transformer), 接口功能 and 计算公式 steps 1-5,
the C128A form (coff = 1, no overlap between neighbouring groups) in
compressor(), and the C4A form (coff = 2, cmp_ratio = 4, each group's eight
rows reaching into the next group) in compressor_c4a():

  1. [kv_state, score_state] = X @ [W^KV, W^Gate]   (W given as [coff*D, H] rows,
     so the product with a weight is X @ W^T)
  2. score'_i = score_state[rows of group i] + Ape,  groups of cmp_ratio
     consecutive rows (i = 1 .. s / cmp_ratio)
  3. S'_i = softmax(score'_i)
  4. (S_H)_i = S'_i (Hadamard) kv_state[rows of group i]
  5. C_i = [1]_{1 x cmp_ratio} @ (S_H)_i

Readings of the page (its parameter tables arrived garbled):
  * the softmax of step 3 runs over the cmp_ratio rows of a group, separately
    for every one of the D channels: step 5 sums exactly those rows with a
    ones vector, so each output channel is a convex combination of the
    group's kv_state values of that channel;
  * Ape is [cmp_ratio, D] (the page's [cmp_ratio, coff*D] with coff = 1): row r
    of Ape is added to the score of the r-th token of every group;
  * x, W^KV and W^Gate are bf16, Ape is float32, the output cmpKv [T /
    cmp_ratio, D] is bf16 (rounded once at the end);
  * the stateless case: the T rows are whole groups of one prefill chunk
    (T % cmp_ratio == 0); the state cache, start_pos and cu_seqlens
    bookkeeping of the page is not modelled.

Precision: float64 throughout (bf16 inputs are exact in float64; each product
of two bf16 values is exact; the sums and the exponentials carry float64
rounding only), so the oracle's result is the exact value of the formula to
about 1e-15 relative, and the bf16 output of the device is compared with it
within a tolerance derived from binary32 accumulation and one bf16 rounding.

Pinned by tests/test_oracle_compressor.py (C4A: the eight-row mean when
W^Gate = 0 and Ape = 0, selection of an a row or a b row by a dominant Ape
entry, the last group's four rows, locality, convexity, per-channel shift
invariance): hand-worked examples
(tests/golden/compressor_examples.txt), the group mean when W^Gate = 0 and
Ape = 0, row selection by a dominant Ape entry, invariance under a
per-channel shift of the scores, sensitivity to a per-row shift,
equivariance under a permutation of a group's rows, locality of each group,
convexity, and a mutation check that plants plausible mistakes.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> their exact values: a bf16 number is the
    binary32 number whose upper 16 bits these are."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def states(x: np.ndarray, w_kv: np.ndarray, w_gate: np.ndarray):
    """Step 1: kv_state = X @ W^KV^T and score_state = X @ W^Gate^T (float64)."""
    X = bf16_to_f64(x)
    return X @ bf16_to_f64(w_kv).T, X @ bf16_to_f64(w_gate).T


def group_softmax(score: np.ndarray, ape: np.ndarray, ratio: int) -> np.ndarray:
    """Steps 2-3: add Ape to each group of `ratio` consecutive rows and take the
    softmax over the rows of the group, channel by channel.  Returns [G, ratio, D]."""
    T, D = score.shape
    s = score.reshape(T // ratio, ratio, D) + np.asarray(ape, dtype=np.float64)[None, :, :]
    s = s - s.max(axis=1, keepdims=True)            # exact shift: softmax is unchanged by it
    e = np.exp(s)
    return e / e.sum(axis=1, keepdims=True)


def compress_states(kv: np.ndarray, score: np.ndarray, ape: np.ndarray, ratio: int) -> np.ndarray:
    """Steps 2-5 from the two states: [T, D] each -> C [T / ratio, D]."""
    T, D = kv.shape
    p = group_softmax(score, ape, ratio)                         # steps 2, 3
    sh = p * kv.reshape(T // ratio, ratio, D)                    # step 4
    return np.ones(ratio) @ sh                                   # step 5: [1]_{1 x ratio} @ (S_H)_i


def compressor(x: np.ndarray, w_kv: np.ndarray, w_gate: np.ndarray, ape: np.ndarray, ratio: int,
               groups: Optional[Sequence[int]] = None) -> np.ndarray:
    """The C128A-form Compressor in float64.

    x: bf16 bits [T, H]; w_kv, w_gate: bf16 bits [D, H]; ape: float32 [ratio, D].
    Returns C [T / ratio, D] (float64, before the output rounding), or only the
    listed groups' rows (in the listed order) when `groups` is given."""
    x = np.asarray(x)
    T, H = x.shape
    if T % ratio:
        raise ValueError("T must be a multiple of cmp_ratio")
    if groups is not None:
        rows = np.concatenate([np.arange(g * ratio, (g + 1) * ratio) for g in groups]) if len(groups) else \
            np.zeros(0, dtype=np.int64)
        x = x[rows]
    kv, score = states(x, w_kv, w_gate)
    return compress_states(kv, score, ape, ratio)


def compressor_c4a(x: np.ndarray, w_kv: np.ndarray, w_gate: np.ndarray, ape: np.ndarray,
                   groups: Optional[Sequence[int]] = None) -> np.ndarray:
    """The C4A-form Compressor (coff = 2, cmp_ratio = 4) in float64, by the
    page's steps (计算公式, C4A lines), group by group:

      1. [kv^a, score^a] = X @ [W^aKV, W^aGate], [kv^b, score^b] = X @ [W^bKV, W^bGate]
      2. score'_i = [score^a[rows 4(i-1)+1 .. 4i] ; score^b[rows 4i+1 .. 4(i+1)]] + Ape
      3. S'_i = softmax(score'_i)
      4. (S_H)_i = S'_i (Hadamard) [kv^a[rows 4(i-1)+1 .. 4i] ; kv^b[rows 4i+1 .. 4(i+1)]]
      5. C_i = [1]_{1 x 8} @ (S_H)_i

    Readings: W^KV and W^Gate are [2D, H] (the page's [coff*D, H]) with the a
    weights in rows [0, D) and the b weights in rows [D, 2D); Ape is
    [4, 2D] (the page's [cmp_ratio, coff*D]): columns [0, D) are added to the
    a rows (row r to the r-th token of the group's own four) and columns
    [D, 2D) to the b rows (row r to the r-th token of the next four); ";"
    stacks rows, so a group spans eight rows, its own four tokens through the
    a projections and the next group's four through the b projections.  The
    last group of the chunk has no next four tokens: those rows do not exist,
    and its softmax and sum run over its own four a rows.

    x: bf16 bits [T, H] (T a multiple of 4); w_kv, w_gate: bf16 bits [2D, H];
    ape: float32 [4, 2D].  Returns C [T / 4, D] (float64), or the listed
    groups' rows in the listed order."""
    x = np.asarray(x)
    T, H = x.shape
    if T % 4:
        raise ValueError("T must be a multiple of 4")
    D = np.asarray(w_kv).shape[0] // 2
    a_kv, b_kv = np.asarray(w_kv)[:D], np.asarray(w_kv)[D:]
    a_gate, b_gate = np.asarray(w_gate)[:D], np.asarray(w_gate)[D:]
    ape = np.asarray(ape, dtype=np.float64)
    G = T // 4
    out = []
    for i in (range(G) if groups is None else groups):
        own, nxt = x[4 * i:4 * i + 4], x[4 * i + 4:4 * i + 8]          # nxt is empty for the last group
        kv_a, score_a = states(own, a_kv, a_gate)                        # step 1, the rows group i uses
        kv_b, score_b = states(nxt, b_kv, b_gate)
        score = np.vstack([score_a + ape[:, :D], score_b + ape[:len(nxt), D:]])     # step 2
        kv = np.vstack([kv_a, kv_b])
        e = np.exp(score - score.max(axis=0, keepdims=True))             # step 3 (an exact shift)
        p = e / e.sum(axis=0, keepdims=True)
        out.append(np.ones(len(score)) @ (p * kv))                       # steps 4, 5
    return np.array(out).reshape(-1, D)


def abs_states(x: np.ndarray, w_kv: np.ndarray, w_gate: np.ndarray, groups: Sequence[int], ratio: int):
    """|X| @ |W|^T for the listed groups' rows: the sums of absolute products
    that bound the rounding error of any order of binary32 accumulation."""
    rows = np.concatenate([np.arange(g * ratio, (g + 1) * ratio) for g in groups])
    X = np.abs(bf16_to_f64(np.asarray(x)[rows]))
    return X @ np.abs(bf16_to_f64(w_kv)).T, X @ np.abs(bf16_to_f64(w_gate)).T
