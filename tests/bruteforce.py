"""Brute-force decode attention in plain Python floats, for tiny inputs.

A second, deliberately different route to the same result as the oracle: it
walks every logical position, turns it into a slot through the block table
(slot = physical block * block_size + row) and reads the cache row by slot;
the softmax is exp(s) / sum(exp(s)) with no max subtraction (fine for the
small scores of tiny tests) and sums use math.fsum.
"""
import math


def brute_decode(q, key_cache, value_cache, block_tables, context_lens, sm_scale, n_kv):
    S = len(q)
    n_q = len(q[0])
    d = len(q[0][0])
    bs = len(key_cache[0])
    group = n_q // n_kv
    out = [[[0.0] * d for _ in range(n_q)] for _ in range(S)]
    for s in range(S):
        L = int(context_lens[s])
        slots = []
        for p in range(L):
            slots.append(int(block_tables[s][p // bs]) * bs + p % bs)
        for h in range(n_q):
            kv = h // group
            scores = []
            for slot in slots:
                krow = key_cache[slot // bs][slot % bs][kv]
                scores.append(sm_scale * math.fsum(float(q[s][h][i]) * float(krow[i]) for i in range(d)))
            ex = [math.exp(x) for x in scores]
            z = math.fsum(ex)
            for i in range(d):
                acc = []
                for w, slot in zip(ex, slots):
                    acc.append(w * float(value_cache[slot // bs][slot % bs][kv][i]))
                out[s][h][i] = math.fsum(acc) / z if L else 0.0
    return out
