"""Conditional-rescale statistics of the causal prefill -- TEST / ANALYSIS
INFRASTRUCTURE ONLY (like the rest of ``oracle/``; the product library never
loads it).

The conditional rescale ("FlashAttention-4", samanvya.dev: the running
maximum is moved, and the accumulated output rescaled, only when a block's
maximum exceeds it by more than a threshold) decides per block of keys
whether any row of a group must rescale.  The decisions are a deterministic
function of the scores, so they can be counted here exactly, without a
counter inside the kernel.  The rule follows the prefill kernel's layout:

  * query tiles of 128 rows, decided in groups of 32 rows (one warp);
  * key blocks of 128 keys visited in ascending order, causal: tile t sees
    blocks 0..t (block t partly masked);
  * scores in log2 units, s = (q . k) * scale * log2(e), from the bf16 inputs
    with fp32 products and sums (the tensor core's precision);
  * at a tile's first block the reference is that block's row maximum; at
    each later block, "grew" = some row's block maximum exceeds its
    reference, "rescaled" = some row's exceeds it by more than 8; when
    rescaled, every row of the group takes max(reference, block maximum).

``python -m oracle.rescale_stats [workload]`` prints the counts as one JSON
line (default workload gqa4k).
"""
from __future__ import annotations

import json
import math
import sys

import numpy as np


def rescale_counts(q, k, scale, threshold=8.0, tile=128, group=32, block=128):
    """Counts for one head: q [N, d], k [N, d] (float32 arrays of bf16
    values), causal.  Returns (decisions, grew, rescaled)."""
    N = q.shape[0]
    s = (q @ k.T) * np.float32(scale * math.log2(math.e))       # fp32
    rows = np.arange(N)[:, None]
    s = np.where(np.arange(N)[None, :] <= rows, s, -np.inf)
    nb = (N + block - 1) // block
    # row maxima per key block: [N, nb]
    pad = nb * block - N
    sp = np.pad(s, ((0, 0), (0, pad)), constant_values=-np.inf) if pad else s
    bmax = sp.reshape(N, nb, block).max(axis=2)
    dec = grew = resc = 0
    for t in range((N + tile - 1) // tile):
        r0 = t * tile
        last_row = min(r0 + tile, N) - 1
        hi = last_row // block + 1
        for g0 in range(r0, min(r0 + tile, N), group):
            rws = slice(g0, min(g0 + group, N))
            m_ref = bmax[rws, 0].copy()
            for j in range(1, hi):
                mb = bmax[rws, j]
                dec += 1
                if np.any(mb > m_ref):
                    grew += 1
                if np.any(mb > m_ref + threshold):
                    resc += 1
                    m_ref = np.maximum(m_ref, mb)
    return dec, grew, resc


def main(argv):
    sys.path.insert(0, ".")
    import workloads
    name = argv[1] if len(argv) > 1 else "gqa4k"
    inp = workloads.make(name, seed=0)
    assert inp.causal and inp.window == 0, "causal, no window"
    B, N, Hq, d = inp.q.shape
    Hkv = inp.k.shape[2]
    group = Hq // Hkv
    tot = np.zeros(3, dtype=np.int64)
    for b in range(B):
        for h in range(Hq):
            q = inp.q[b, :, h, :].float().numpy()
            k = inp.k[b, :, h // group, :].float().numpy()
            tot += np.array(rescale_counts(q, k, inp.scale))
    dec, grew, resc = (int(x) for x in tot)
    print(json.dumps({
        "workload": name, "threshold_log2": 8, "decisions": dec, "max_grew": grew,
        "rescaled": resc, "skipped_fraction": round(1.0 - resc / max(dec, 1), 5),
        "rescales_vs_unconditional": round(grew / max(resc, 1), 2),
        "how": "host count of the prefill kernel's per-warp decision rule on the workload's "
               "scores (32-row groups, 128-key blocks, ascending, causal)"}))


if __name__ == "__main__":
    main(sys.argv)
