"""Small random paged-cache cases for tests (numpy RNG, seeded).

Builds a pool with a random physical placement of every sequence's pages,
NaN in every slot that holds no token, and random N(0,1) BF16 values
elsewhere.  Holds no attention arithmetic.
"""
import numpy as np

T, G, H, D = 16, 8, 32, 64
NAN = 0x7FC0


def bf16_bits(x):
    """float array -> BF16 bit patterns, round to nearest even."""
    f = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    rnd = ((f >> 16) & 1) + 0x7FFF
    return ((f + rnd) >> 16).astype(np.uint16)


def bf16_to_f64(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def make_case(lens, seed=0, num_layers=1, spare_pages=3, max_blocks=None):
    """lens: lengths after the append (decode attends to all of them).
    Returns dict(pool, bt, seq_lens, q, k_new, v_new) with the new token's
    K/V already stored in the pool and also returned as k_new / v_new."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lens, np.int32)
    B = lens.size
    need = [(int(l) + T - 1) // T for l in lens]
    mb = max(1, max(need)) if max_blocks is None else max_blocks
    n_pages = num_layers * sum(need) + spare_pages
    perm = rng.permutation(n_pages).astype(np.int32)
    bt = np.full((num_layers, B, mb), -1, np.int32)
    cur = 0
    for l in range(num_layers):
        for b in range(B):
            bt[l, b, :need[b]] = perm[cur:cur + need[b]]
            cur += need[b]
    pool = np.full((n_pages, 2, G, T, D), NAN, np.uint16)
    for l in range(num_layers):
        for b in range(B):
            for t in range(int(lens[b])):
                p = bt[l, b, t // T]
                pool[p, :, :, t % T, :] = bf16_bits(rng.standard_normal((2, G, D)))
    q = bf16_bits(rng.standard_normal((B, H, D)))
    k_new = np.zeros((B, G, D), np.uint16)
    v_new = np.zeros((B, G, D), np.uint16)
    for b in range(B):
        if lens[b] > 0:
            t = int(lens[b]) - 1
            p = bt[0, b, t // T]
            k_new[b] = pool[p, 0, :, t % T, :]
            v_new[b] = pool[p, 1, :, t % T, :]
    return dict(pool=pool, bt=bt, seq_lens=lens, q=q, k_new=k_new, v_new=v_new)


def contiguous_kv(case, layer=0):
    """Numpy fancy-index gather of K and V per sequence: list of
    (K [G, L, D], V [G, L, D]) float64 arrays."""
    out = []
    for b, L in enumerate(case["seq_lens"]):
        t = np.arange(int(L))
        pages = case["bt"][layer, b, t // T]
        K = case["pool"][pages, 0, :, t % T, :]   # [L, G, D]
        V = case["pool"][pages, 1, :, t % T, :]
        out.append((bf16_to_f64(K).transpose(1, 0, 2), bf16_to_f64(V).transpose(1, 0, 2)))
    return out


# Hand-worked append-race cases: (name, block-table rows [batch][max_blocks],
# lengths after the append, race under pkv_append, race under the fused
# call), over a pool of APPEND_CASE_PAGES pages.  Sequence b writes slot
# (L-1) % 16 of page row[(L-1) // 16]; the fused call also reads slots
# t % 16 of pages row[t // 16] for t < L.
APPEND_CASE_PAGES = 8
APPEND_CONFLICT_CASES = [
    # (0,4) and (3,3): distinct pages, each read only by its writer
    ("distinct pages", [[0, 1], [2, 3]], [5, 20], False, False),
    # both write (5,2)
    ("same slot", [[5, 0], [5, 1]], [3, 3], True, True),
    # writes (5,3) and (5,5); sequence 1 reads slots 0..5 of page 5
    ("same page, other slots", [[5, 0], [5, 1]], [4, 6], False, True),
    # page 7 is a prefix both read in full; the writes go to pages 1 and 2
    ("shared read-only prefix", [[7, 1], [7, 2]], [20, 18], False, False),
    # sequence 1 (L = 0) names page 4 but reads and writes nothing
    ("idle slot names the page", [[4, 0], [4, 0]], [11, 0], False, False),
    # page 3 named twice: the write (3,3) at t = 19 lands on t = 3 of the same context
    ("page named twice by one table", [[3, 3], [0, 1]], [20, 2], False, True),
    # sequence 1's page is outside the pool: no write; sequence 2 writes (2,0)
    ("invalid page is no write", [[6, 0], [99, 0], [2, 0]], [9, 1, 1], False, False),
    # both name page 99, outside the pool: neither writes
    ("two writes outside the pool", [[99, 0], [99, 0]], [1, 1], False, False),
    # three writers, two of them on (1,15); the third on (1,0) is read by both
    ("three writers", [[1, 0], [0, 1], [2, 1]], [16, 32, 17], True, True),
]


# Hand-worked fill-race cases: (name, block-table rows [batch][max_blocks],
# tokens per sequence, start positions, race), over APPEND_CASE_PAGES pages.
# Token i of sequence b goes to slot (start+i) % 16 of page row[(start+i) // 16].
FILL_CONFLICT_CASES = [
    ("disjoint pages", [[0, 1], [2, 3]], [20, 16], [0, 0], False),
    # both write slots 2..3 of page 5
    ("overlapping positions on one page", [[5, 0], [5, 1]], [4, 2], [0, 2], True),
    # slots 0..3 and 4..7 of page 5
    ("one page, disjoint slots", [[5, 0], [5, 1]], [4, 4], [0, 4], False),
    # positions 0 and 16 both land on slot 0 of page 3
    ("page named twice by one table", [[3, 3]], [17], [0], True),
    ("page named twice, positions apart", [[3, 3]], [8], [12], False),
    # both name page 99, outside the pool: neither writes
    ("writes outside the pool", [[99, 0], [99, 0]], [3, 3], [0, 0], False),
    # sequence 1 starts beyond its table: skipped, so its overlap does not count
    ("skipped sequence", [[4, 0], [4, 1]], [5, 5], [0, 30], False),
    ("empty sequences", [[2, 0], [2, 0], [2, 1]], [0, 0, 3], [0, 0, 0], False),
]


def shared_prefix_case(seed=71, prefix_pages=3, tails=(5, 37, 16, 130, 1)):
    """Sequences whose first prefix_pages pages are the same physical pages
    (a common prompt prefix), each with its own tail pages; and the same
    batch with the prefix copied into private pages."""
    rng = np.random.default_rng(seed)
    B = len(tails)
    lens = np.array([16 * prefix_pages + t for t in tails], np.int32)
    need = (lens + 15) // 16
    own = need - prefix_pages
    P_shared = prefix_pages + int(own.sum()) + 2
    mb = int(need.max())
    bt = np.full((1, B, mb), -1, np.int32)
    perm = rng.permutation(P_shared).astype(np.int32)
    bt[0, :, :prefix_pages] = perm[:prefix_pages]
    cur = prefix_pages
    for b in range(B):
        bt[0, b, prefix_pages:need[b]] = perm[cur:cur + own[b]]
        cur += own[b]
    pool = np.full((P_shared, 2, 8, 16, 64), NAN, np.uint16)
    for p in perm[:prefix_pages]:
        pool[p] = bf16_bits(rng.standard_normal((2, 8, 16, 64)))
    for b in range(B):
        for t in range(16 * prefix_pages, int(lens[b])):
            pool[bt[0, b, t // 16], :, :, t % 16, :] = bf16_bits(rng.standard_normal((2, 8, 64)))
    q = bf16_bits(rng.standard_normal((B, 32, 64)))
    k_new = np.stack([pool[bt[0, b, (lens[b] - 1) // 16], 0, :, (lens[b] - 1) % 16] for b in range(B)])
    v_new = np.stack([pool[bt[0, b, (lens[b] - 1) // 16], 1, :, (lens[b] - 1) % 16] for b in range(B)])
    shared = dict(pool=pool, bt=bt, seq_lens=lens, q=q, k_new=k_new, v_new=v_new)
    # private copies of the prefix pages for every sequence but the first
    extra = (B - 1) * prefix_pages
    pool2 = np.concatenate([pool, np.full((extra, 2, 8, 16, 64), NAN, np.uint16)])
    bt2 = bt.copy()
    nxt = P_shared
    for b in range(1, B):
        for j in range(prefix_pages):
            pool2[nxt] = pool[bt[0, b, j]]
            bt2[0, b, j] = nxt
            nxt += 1
    private = dict(shared, pool=pool2, bt=bt2)
    return shared, private
