"""Host model of the align/sort kernels' partition arithmetic (no GPU).

`csrc/sort.cuh` splits the flat slots into parts (one per CTA of the cluster
sort, one for the single-CTA sort), each part into 32 warp chunks, counts per
(warp, expert), turns the counts into absolute positions by prefixes over the
warps, the CTAs before this one and the experts' padded segments, and places
every slot at its position plus its rank among equal experts of its 32-slot
step. This model repeats that arithmetic step for step in numpy, with the
same chunk formulas and clamps, and checks that it reproduces the oracle's
stable sort on many sizes, including parts and chunks that come out empty or
ragged. It checks the scheme; the kernels themselves are compared with the
oracle on the GPU (tests/test_gpu_kernels.py).
"""
import numpy as np
import pytest

import oracle


def _model_sort(ids, E, bm, parts):
    N = ids.size
    flat = ids.reshape(-1)
    part = (N + parts - 1) // parts
    ranges = []  # (part, warp, f0, f1)
    for r in range(parts):
        p0 = min(r * part, N)
        p1 = min(p0 + part, N)
        chunk = (p1 - p0 + 31) // 32
        for w in range(32):
            f0 = min(p0 + w * chunk, p1)
            f1 = min(f0 + chunk, p1)
            ranges.append((r, w, f0, f1))
    # 1. counts per (part, warp, expert), in 32-slot steps
    cnt = np.zeros((parts, 32, E), np.int64)
    for r, w, f0, f1 in ranges:
        for b in range(f0, f1, 32):
            for e in flat[b:min(b + 32, f1)]:
                cnt[r, w, e] += 1
    # 2. prefixes: over warps inside a part, over the parts before, over padded segments
    tot = cnt.sum(axis=(0, 1))
    pad = (tot + bm - 1) // bm * bm
    seg_start = np.concatenate([[0], np.cumsum(pad)[:-1]])
    cta_tot = cnt.sum(axis=1)                                        # [parts, E]
    before_cta = np.cumsum(cta_tot, axis=0) - cta_tot                # exclusive over parts
    before_warp = np.cumsum(cnt, axis=1) - cnt                       # exclusive over warps
    pos0 = seg_start[None, None, :] + before_cta[:, None, :] + before_warp
    # 3. placement: entry + rank among equal experts of the 32-slot step, then advance
    n_pad = int(pad.sum())
    out = np.full(n_pad, -7, np.int64)
    nxt = pos0.copy()
    for r, w, f0, f1 in ranges:
        for b in range(f0, f1, 32):
            step = flat[b:min(b + 32, f1)]
            for lane, e in enumerate(step):
                rank = int(np.sum(step[:lane] == e))
                out[nxt[r, w, e] + rank] = b + lane
            for e in np.unique(step):
                nxt[r, w, e] += int(np.sum(step == e))
    # padding: sentinel N after each segment's slots; block owners
    block_expert = np.full(n_pad // bm, -7, np.int64)
    for e in range(E):
        out[seg_start[e] + tot[e]:seg_start[e] + pad[e]] = N
        block_expert[seg_start[e] // bm:(seg_start[e] + pad[e]) // bm] = e
    return out, block_expert, tot, np.concatenate([seg_start, [n_pad]]), n_pad


CASES = [(1, 1, 1, 16), (3, 1, 512, 256), (5, 3, 7, 64), (33, 2, 16, 16), (100, 6, 64, 32), (511, 8, 256, 128),
         (512, 8, 512, 64), (1000, 4, 16, 32), (4095, 1, 33, 16), (2000, 7, 100, 128)]


@pytest.mark.parametrize("T,k,E,bm", CASES)
@pytest.mark.parametrize("parts", [1, 8])
def test_partitioned_sort_reproduces_the_oracle(T, k, E, bm, parts):
    rng = np.random.default_rng(T * 31 + E + parts)
    p = 1.0 / np.arange(1, E + 1) ** 1.2
    ids = rng.choice(E, size=(T, k), p=p / p.sum()).astype(np.int32)
    srt, be, cnt, off, n = _model_sort(ids, E, bm, parts)
    ref = oracle.align_sort(ids, E, bm)
    assert n == ref["num_padded"]
    assert np.array_equal(srt, ref["sorted_ids"])
    assert np.array_equal(be, ref["block_expert"])
    assert np.array_equal(cnt, ref["expert_counts"])
    assert np.array_equal(off, ref["expert_offsets"])
