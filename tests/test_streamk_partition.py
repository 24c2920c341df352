"""Host-side check of the stream-K decode's partition against the workspace
the library sizes for it (no GPU).

The stream-K decodes (csrc/sparse_decode_streamk.cuh and its warp-group
form) give worker w of W the entries [floor(w X / W), floor((w + 1) X / W))
of the batch's padded extended selections (E entries per (request, kv head)
pair, X = pairs * E), with W = min(workers resident in one wave, 2048,
X / 16).  Every (pair, split) segment a worker streams writes one partial
slot k = w - (first worker of that (pair, split)); the merge reads slots
0 .. (last worker - first worker).  Here the partition is walked for many
shapes, worker counts and split boundaries, and the largest slot index any
(pair, split) reaches must fit the slots that
qsa_sparse_decode_workspace_bytes reserves (the stream-K layout: split
boundaries [B, S+1] int32, then lse [pairs, S, K, M] and o [pairs, S, K,
M, D] float32, each 256-byte aligned)."""
import random

from sparse_attention_decode_compress_b200 import _lib


def _al(x):
    return -(-x // 256) * 256


def _range_begin(w, X, W):
    return w * X // W


def _worker_of(x, X, W):
    return ((x + 1) * W - 1) // X


def _workers(X, w_hw):
    return max(1, min(w_hw, 2048, X // 16))


def _max_slots(pairs, E, W, S, rng):
    """Largest number of workers that share one (pair, split): over up to 200
    pairs, each with random split boundaries and with all of its E entries
    in one split (the longest a split can be)."""
    X = pairs * E
    worst = 0
    for P in rng.sample(range(pairs), min(pairs, 200)):
        nE = rng.randint(0, E)
        cuts = sorted(rng.randint(0, nE) for _ in range(S - 1))
        for eb in ([0] + cuts + [nE], [0, E]):
            for s in range(len(eb) - 1):
                if eb[s + 1] <= eb[s]:
                    continue
                wf = _worker_of(P * E + eb[s], X, W)
                wl = _worker_of(P * E + eb[s + 1] - 1, X, W)
                worst = max(worst, wl - wf + 1)
    return worst


def test_partition_tiles_the_entries():
    rng = random.Random(3)
    for _ in range(300):
        X = rng.randint(1, 200000)
        W = _workers(X, rng.choice([12, 592, 740, 1184, 1776, 5000]))
        assert _range_begin(0, X, W) == 0 and _range_begin(W, X, W) == X
        for w in rng.sample(range(W), min(W, 40)):
            a, b = _range_begin(w, X, W), _range_begin(w + 1, X, W)
            assert a <= b
            if b > a:
                assert _worker_of(a, X, W) == w and _worker_of(b - 1, X, W) == w


def test_workspace_holds_every_partial_slot():
    lib = _lib.load()
    rng = random.Random(5)
    # worker counts of the launches: one warp per worker (148 SMs x 12), or
    # groups of 2, 3 or 4 warps (8, 5 or 4 groups per SM), and small GPUs
    w_hw_choices = [1776, 1184, 740, 592, 96, 12]
    for _ in range(400):
        B = rng.choice([1, 2, 3, 17, 64, 128, 256, 1000])
        Hkv = rng.choice([1, 2, 4, 8])
        G = rng.choice([1, 2, 4, 8])
        T = rng.choice([1, 1, 2, 4]) if G * 4 <= 32 else 1
        topk = rng.choice([4, 64, 300, 512, 2048, 4096])
        S = rng.choice([1, 2, 3, 4, 7, 16])
        D = rng.choice([64, 128])
        Hq, M = G * Hkv, G * T
        E = topk + (2 if T > 1 else 0)
        pairs = B * Hkv
        need_k = max(_max_slots(pairs, E, _workers(pairs * E, w_hw), S, rng)
                     for w_hw in w_hw_choices)
        need = (_al(B * (S + 1) * 4) + _al(pairs * S * need_k * M * 4) +
                _al(pairs * S * need_k * M * D * 4))
        got = lib.qsa_sparse_decode_workspace_bytes(B, T, Hq, Hkv, D, topk, S)
        assert got >= need, (B, Hkv, G, T, topk, S, D, need_k, got, need)
