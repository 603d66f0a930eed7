"""CPU replicas of the CUDA kernels' index arithmetic (no GPU needed).

The decode kernels compute every shared- and global-memory index from a few
integer formulas; these tests restate those formulas in Python and check,
over random and adversarial shapes, that every index stays inside its buffer
and that the work partitions cover every item exactly once. They are the
bounds evidence for the kernels (a device memory checker is not available
on the GPU pool), and they run again whenever the formulas change:

* the gate's split of the pooled-key positions over CTAs and the per-row
  count of gate pieces that tells the last CTA of a row to select it
  (gate_phase in sparse_decode.cu);
* the decode's fixed parts of a row when rows fit the grid, and their slots;
* the two-ended span of list positions when rows outnumber the CTAs: front
  pieces (one claim in flight, an eighth of what is left, at least a chunk)
  and help from the back, under random interleavings of the atomic adds --
  every position taken once, the row counted as fully taken once, runs
  within the slots reserved per row;
* the fused step's workspace layout (step_workspace_layout, step_geometry)
  and shared-memory layout (make_layout) for every supported shape;
* select_row (gate_core.cuh), thread by thread: every key, histogram, bucket
  and output index in bounds, and the list equal to a sort.
"""
import random

import numpy as np
import pytest

# ---------------------------------------------------------------- constants of sparse_decode.cu

SMEM_LIMIT = 232448
CONSUMER_WARPS = 8
MAX_STAGES = 8
MAX_GATE_STAGES = 8
INFO_WORDS = MAX_STAGES + 4
STAGE_INFO_WORDS = 8
GATE_SCRATCH = 16384
GATE_CHUNK = 32768
MIN_GATE_POSITIONS = 32
MAX_SEL_ROWS = 32
SELECT_HEAD = 32
POOL_THREADS = 96


def step_geometry(B, Hkv, NBmax, blk, kmax, num_sms):
    """step_geometry: gate CTAs, CTAs per row, claim chunk, slots per (row, head)."""
    rows = B * Hkv
    if rows <= num_sms:
        per_row = num_sms // rows
        cap = (NBmax + MIN_GATE_POSITIONS - 1) // MIN_GATE_POSITIONS
        cpr = max(1, min(per_row, cap))
        gate_ctas = rows * cpr
    else:
        cpr, gate_ctas = 0, num_sms
    base = 2 if blk == 64 else 1
    chunk = max(base, (kmax + 63) // 64)
    nslots = max((kmax + chunk - 1) // chunk + 2, min(kmax, cpr))
    return gate_ctas, cpr, chunk, nslots


# ---------------------------------------------------------------- gate partition

def gate_pieces(rows, NBmax, G1):
    """For every CTA of the gate: the rows it counts in, and the positions it holds."""
    V1 = rows * NBmax
    count = [0] * rows
    owned = np.zeros(V1, np.int32)
    for c in range(G1):
        h0, h1 = c * V1 // G1, (c + 1) * V1 // G1
        owned[h0:h1] += 1
        r_stop = (h1 + NBmax - 1) // NBmax
        for r in range(h0 // NBmax, r_stop):
            assert 0 <= r < rows
            rs = r * NBmax
            i0 = h0 - rs if h0 > rs else 0
            i1 = min(h1 - rs, NBmax)
            assert 0 <= i0 <= i1 <= NBmax
            count[r] += 1
    return count, owned


@pytest.mark.parametrize("seed", range(6))
def test_gate_ranges_cover_positions_once_and_counts_match(seed):
    rng = random.Random(seed)
    for _ in range(150):
        rows = rng.randint(1, 400)
        NBmax = rng.randint(1, 700)
        G1 = rng.choice([1, 2, 37, 148, 300, rows, rows * rng.randint(1, 4)])
        count, owned = gate_pieces(rows, NBmax, G1)
        assert np.all(owned == 1)  # every pooled-key position scored by exactly one CTA
        V1 = rows * NBmax
        for r in range(rows):
            rs = r * NBmax
            cf = ((rs + 1) * G1 - 1) // V1
            cl = ((rs + NBmax) * G1 - 1) // V1
            assert count[r] == cl - cf + 1  # the kernel's count target for "last CTA of the row"


def gate_row(i, B, Hkv, gate_cpr):
    """The gate's row order: row i when rows fit the grid, else head-major (i = kvh * B + b)."""
    return i if gate_cpr > 0 else (i % B) * Hkv + i // B


@pytest.mark.parametrize("seed", range(4))
def test_gate_order_is_a_permutation_and_ctas_mostly_share_one_head(seed):
    """With more rows than CTAs, the gate visits rows head-major: every row once, its gate
    index giving the positions [i * NBmax, (i + 1) * NBmax) the count target uses, and the
    batches of consecutive indices a CTA gates mostly one head (one W_q bulk copy)."""
    rng = random.Random(seed)
    for _ in range(100):
        Hkv = rng.choice([1, 2, 4, 8])
        B = rng.randint(1, 300)
        rows = B * Hkv
        order = [gate_row(i, B, Hkv, 0) for i in range(rows)]
        assert sorted(order) == list(range(rows))
        assert [gate_row(i, B, Hkv, 1) for i in range(rows)] == list(range(rows))
        NBmax, G1 = rng.randint(1, 600), 148
        if rows <= G1:
            continue
        V1 = rows * NBmax
        mixed = 0
        for c in range(G1):
            h0, h1 = c * V1 // G1, (c + 1) * V1 // G1
            first, stop = h0 // NBmax, (h1 + NBmax - 1) // NBmax
            for b0 in range(first, stop, 8):  # batches of up to 8 rows
                heads = {gate_row(i, B, Hkv, 0) % Hkv for i in range(b0, min(stop, b0 + 8))}
                mixed += len(heads) > 1
        # a batch spans two heads only where the CTA's range crosses a head boundary
        assert mixed <= Hkv - 1 + G1 * max(0, (8 * Hkv) // B), (B, Hkv, mixed)


# ---------------------------------------------------------------- decode: fixed parts when rows fit

@pytest.mark.parametrize("cpr", [1, 2, 3, 7, 18, 32, 148])
def test_fixed_parts_take_each_position_once_with_distinct_slots(cpr):
    for nsel in range(0, 200):
        taken = []
        slots = set()
        for part in range(cpr):
            a0 = part * nsel // cpr
            a1 = (part + 1) * nsel // cpr
            if a0 < a1:
                taken.extend(range(a0, a1))
                slot = part if nsel >= cpr else a0
                assert slot not in slots
                slots.add(slot)
        assert taken == list(range(nsel))
        # the merge reads slots [0, nslots) with nslots = the number of non-empty parts
        assert slots == set(range(min(nsel, cpr)))


def test_fixed_part_slots_fit_the_workspace():
    rng = random.Random(3)
    for _ in range(400):
        blk = rng.choice([64, 128])
        NBmax = rng.randint(1, 16384)
        kmax = rng.randint(1, NBmax)
        B, Hkv = rng.randint(1, 64), rng.randint(1, 8)
        gate_ctas, cpr, chunk, nslots = step_geometry(B, Hkv, NBmax, blk, kmax, 148)
        if cpr:
            assert min(kmax, cpr) <= nslots  # fixed slots of the non-empty parts


# ---------------------------------------------------------------- decode: span claims when rows outnumber CTAs

class Row:
    def __init__(self, nsel, kept):
        self.front, self.back = kept, nsel
        self.nslots = 0
        self.counted = 1 if kept == nsel else 0  # the selecting CTA counts a row it kept entirely

    def add_front(self, n):
        old = (self.front, self.back)
        self.front += n
        return old

    def add_back(self, t):
        old = (self.front, self.back)
        self.back -= t
        return old


def front_run(row, nsel, a0, a1, chunk, taken):
    """The producer's run from the front: the held piece, then one claim in flight (a generator:
    every atomic add on the row is one step)."""
    row.nslots += 1
    n1 = max(chunk, (nsel - a1) // 8)
    c1 = row.add_front(n1)
    yield
    while True:
        taken.extend(range(a0, a1))
        f0, b0 = c1
        e0, e1 = f0, min(f0 + n1, b0)
        if f0 < b0 and f0 + n1 >= b0:
            row.counted += 1
        if e0 >= e1:
            return
        a0, a1 = e0, e1
        n1 = max(chunk, (b0 - a1) // 8)
        c1 = row.add_front(n1)
        yield


def visit_front(row, nsel, chunk, taken):
    f0, b0 = row.add_front(chunk)
    if f0 < b0 and f0 + chunk >= b0:
        row.counted += 1
    yield
    a0, a1 = f0, min(f0 + chunk, b0)
    if a0 < a1:
        yield from front_run(row, nsel, a0, a1, chunk, taken)


def helper(rows, nsels, chunk, fair, taken):
    """Help from the back: the row with the most left, half of it, at most a fair share."""
    while True:
        left = [max(0, r.back - r.front) for r in rows]
        best = max(left)
        if best < 2 * chunk:
            return
        k = left.index(best)
        t = max(chunk, min(best // 2, fair))
        f0, b0 = rows[k].add_back(t)
        if f0 < b0 and b0 - t <= f0:
            rows[k].counted += 1
        yield
        a0, a1 = max(b0 - t, f0), b0
        if a0 < a1:
            rows[k].nslots += 1
            taken[k].extend(range(a0, a1))
        yield


@pytest.mark.parametrize("seed", range(8))
def test_span_claims_take_every_position_once(seed):
    rng = random.Random(seed)
    for _ in range(60):
        nrows = rng.randint(1, 12)
        kmax = rng.choice([1, 2, 5, 8, 64, 103, 300])
        blk = rng.choice([64, 128])
        chunk = max(2 if blk == 64 else 1, (kmax + 63) // 64)
        nslots = (kmax + chunk - 1) // chunk + 2
        nsels = [rng.randint(0, kmax) for _ in range(nrows)]
        rows, taken, agents = [], [], []
        for k, ns in enumerate(nsels):
            kept = min(chunk, ns) if ns > 0 and rng.random() < 0.8 else 0  # listed by its selector, or not
            rows.append(Row(ns, kept))
            taken.append([])
            if kept:
                agents.append(front_run(rows[k], ns, 0, kept, chunk, taken[k]))
            for _ in range(rng.randint(0 if kept else 1, 2)):  # other CTAs working the row from the front
                agents.append(visit_front(rows[k], ns, chunk, taken[k]))
        fair = max(1, nrows * kmax // rng.randint(1, 20))
        for _ in range(rng.randint(0, 6)):
            agents.append(helper(rows, nsels, chunk, fair, taken))
        while agents:  # random interleaving of the atomic adds
            a = rng.choice(agents)
            try:
                next(a)
            except StopIteration:
                agents.remove(a)
        for k, ns in enumerate(nsels):
            assert sorted(taken[k]) == list(range(ns)), (k, ns)  # every position exactly once
            assert rows[k].front >= rows[k].back                 # the span is exhausted
            assert rows[k].counted == 1                          # counted as fully taken once
            assert rows[k].nslots <= nslots                      # runs fit the reserved slots


# ---------------------------------------------------------------- workspace and shared-memory layouts

def workspace_layout(B, Hq, Hkv, D, dg, blk, Lmax, kmax, num_sms):
    NBmax = (Lmax + blk - 1) // blk
    rows = B * Hkv
    S = step_geometry(B, Hkv, NBmax, blk, kmax, num_sms)[3]
    up = lambda x: (x + 255) // 256 * 256
    w = {"launch_ctr": (0, 8), "rows_taken": (8, 8), "row_cnt": (256, rows * 4)}
    w["row_state"] = (up(256 + rows * 4), rows * 32)
    counters_end = up(w["row_state"][0] + rows * 32)
    w["keys"] = (counters_end, rows * NBmax * 4)
    w["o_part"] = (up(counters_end + rows * NBmax * 4), B * Hq * S * D * 4)
    w["lse_part"] = (up(w["o_part"][0] + B * Hq * S * D * 4), B * Hq * S * 4)
    total = up(w["lse_part"][0] + B * Hq * S * 4)
    return w, counters_end, total, S


def test_workspace_regions_are_disjoint_aligned_and_hold_every_index():
    rng = random.Random(5)
    for _ in range(300):
        blk = rng.choice([64, 128])
        Hkv = rng.randint(1, 8)
        G = rng.randint(1, 8)
        B = rng.randint(1, 200)
        Lmax = rng.randint(1, 16384 * blk // 8)
        NBmax = (Lmax + blk - 1) // blk
        kmax = rng.randint(1, NBmax)
        D = rng.choice([64, 128])
        w, counters_end, total, S = workspace_layout(B, Hkv * G, Hkv, D, 128, blk, Lmax, kmax, 148)
        spans = sorted(w.values())
        for (a, n), (b, _) in zip(spans, spans[1:]):
            assert a + n <= b
        assert spans[-1][0] + spans[-1][1] <= total
        for name in ("row_state", "keys", "o_part", "lse_part"):
            assert w[name][0] % 16 == 0
        assert w["row_state"][0] + w["row_state"][1] <= counters_end  # zeroed with the counters
        # largest slot write: head (B*Hq - 1), slot S - 1, d = D - 1
        last = ((B * Hkv * G - 1) * S + S - 1) * D + D - 1
        assert w["o_part"][0] + 4 * last < w["o_part"][0] + w["o_part"][1] + 4


def struct_sizes(D, G):
    pool = (POOL_THREADS // (D // 8)) * D * 4 + D * 4
    # count, publish, own_len, early_count; early_ids[MAX_STAGES]; thr_valid, thr_bstar; the threshold
    # bins (20 bytes); row, nsel, len; head (the kernel asserts the same size)
    sel_list = 4 * 4 + 4 * MAX_STAGES + 4 * 2 + 20 + 4 * MAX_SEL_ROWS * 3 + 4 * MAX_SEL_ROWS * SELECT_HEAD
    assert sel_list == 4556
    return pool, sel_list


def make_layout(D, blk, G, with_refresh):
    tile = blk * D * 2
    stage = (2 * tile + G * D * 2 + 1023) // 1024 * 1024
    merge = max(CONSUMER_WARPS * G * D * 4 + 2 * CONSUMER_WARPS * G * 4, GATE_SCRATCH if with_refresh else 0)
    info = (INFO_WORDS + MAX_STAGES * STAGE_INFO_WORDS) * 4
    bars = (2 * MAX_STAGES + 4 + MAX_GATE_STAGES) * 8  # full/empty, consumers, gate stages, helpers, W_q, threshold
    pool, sel_list = struct_sizes(D, G)
    refresh = pool + 16 if with_refresh else 0
    sel = sel_list if with_refresh else 0
    tail = merge + info + bars + refresh + sel + 64
    nst = min(MAX_STAGES, (SMEM_LIMIT - 1024 - tail) // stage)
    merge_off = nst * stage
    info_off = (merge_off + merge + 15) // 16 * 16
    bar_off = (info_off + info + 15) // 16 * 16
    refresh_off = bar_off + bars
    sel_off = (refresh_off + refresh + 15) // 16 * 16
    total = sel_off + sel + 1024
    return dict(stage=stage, nst=nst, merge_off=merge_off, merge=merge, info_off=info_off, info=info,
                bar_off=bar_off, bars=bars, refresh_off=refresh_off, refresh=refresh, sel_off=sel_off, sel=sel,
                total=total)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("blk", [64, 128])
@pytest.mark.parametrize("G", range(1, 9))
def test_shared_memory_layout_fits(D, blk, G):
    for with_refresh in (False, True):
        l = make_layout(D, blk, G, with_refresh)
        assert l["nst"] >= 2
        assert l["total"] <= SMEM_LIMIT
        # every region ends before the next starts; the q of a stage fits after its K and V tiles
        assert l["merge_off"] + l["merge"] <= l["info_off"]
        assert l["info_off"] + l["info"] <= l["bar_off"]
        assert l["bar_off"] + l["bars"] <= l["refresh_off"]
        assert l["refresh_off"] + l["refresh"] <= l["sel_off"]
        assert 2 * blk * D * 2 + G * D * 2 <= l["stage"]
        # the warp states of the flush, or the merge weights [G][slots] (slots <= 66)
        assert CONSUMER_WARPS * G * D + 2 * CONSUMER_WARPS * G <= l["merge"] // 4
        assert G * 66 <= l["merge"] // 4
        if with_refresh:
            ring = l["nst"] * l["stage"]
            for NBmax in (1, 32, 512, 1024, 4096, 16384):
                keys = (NBmax * 4 + 1023) // 1024 * 1024
                n_gate = (ring - keys) // GATE_CHUNK
                assert n_gate >= 1  # at least one pooled-key copy in flight
                n_gate = min(n_gate, MAX_GATE_STAGES)
                keys_off = ring - keys  # the order keys end the ring; pooled-key copies start at 0
                assert keys_off % 1024 == 0 and n_gate * GATE_CHUNK <= keys_off
                # one CTA per row: decode stages issued during the selection stay clear of the keys
                n_early = min(keys_off // l["stage"], l["nst"] - 1)
                assert 0 <= n_early <= MAX_STAGES - 1 and n_early * l["stage"] <= keys_off
                for dg in (64, 128):
                    # rows that fit the grid: W_q (dg x D fp32, one bulk copy) first fills the
                    # last wq gate stages, used only when at least one stage stays free for keys
                    wq_bytes = dg * D * 4
                    wq = -(-wq_bytes // GATE_CHUNK)
                    assert wq_bytes % 16 == 0 and wq_bytes < (1 << 20)  # bulk size, mbarrier tx count
                    if n_gate > wq:
                        start = keys + (n_gate - wq) * GATE_CHUNK
                        assert start % 16 == 0 and start + wq_bytes <= keys + n_gate * GATE_CHUNK


# ---------------------------------------------------------------- select_row, thread by thread

BINS, BUCKET = 2048, 64


def order_key(f):
    f = np.float32(f)
    if f == 0:
        f = np.float32(0.0)
    u = int(np.array(f, np.float32).view(np.uint32))
    if (u & 0x7fffffff) > 0x7f800000:
        return 0
    return (~u & 0xffffffff) if (u & 0x80000000) else (u | 0x80000000)


def key_value(k):
    bits = (k & 0x7fffffff) if (k & 0x80000000) else (~k & 0xffffffff)
    return np.array(bits, np.uint32).view(np.float32)[()]


def clz(x):
    return 32 - int(x).bit_length() if x else 32


class Bins:
    def __init__(self, lo, hi):
        self.lo = lo
        with np.errstate(all="ignore"):
            self.flo = key_value(lo)
            fhi = key_value(hi)
            w = np.float32(fhi - self.flo)
            self.scale = np.float32(np.float32(BINS) / w)
            self.by_value = bool(np.isfinite(self.flo) and np.isfinite(fhi) and np.isfinite(w) and w > 0
                                 and np.isfinite(self.scale))
        d = (hi - lo) & 0xffffffff
        self.shift = max(0, 32 - clz(d) - 11)

    def __call__(self, k):
        if self.by_value:
            with np.errstate(all="ignore"):
                x = np.float32(np.float32(key_value(k) - self.flo) * self.scale)
            return min(BINS - 1, int(x))
        return ((k - self.lo) & 0xffffffff) >> self.shift


def select_row(keys, NB, kmax, T, on_threshold=None):
    """select_row with T threads: every read of keys / hist / bucket and write of out is checked.
    on_threshold(bins, bstar) is called once, when the first histogram has fixed the threshold bin."""
    def K(i):
        assert 0 <= i < NB - 1 <= len(keys), ("keys", i)
        return keys[i]
    out = [None] * kmax

    def W(p, v):
        assert 0 <= p < kmax, ("out", p)
        out[p] = v
    kb = min(kmax, NB)
    for p in range(max(kb, 0), kmax):
        W(p, -1)
    if NB == 0:
        return out
    ncand, m = NB - 1, kb - 1
    if m >= ncand:
        for j in range(NB):
            W(j, j)
        return out
    if m == 0:
        W(0, NB - 1)
        return out
    per = (ncand + T - 1) // T
    kbp = (BINS + T - 1) // T
    rng_ = [(min(ncand, t * per), min(ncand, min(ncand, t * per) + per)) for t in range(T)]

    def binq(t, q):
        return BINS - 1 - (t * kbp + q)
    lo = min(K(i) for i in range(ncand))
    hi = max(K(i) for i in range(ncand))
    rem = m
    while True:
        if lo == hi:
            cnt = [sum(K(i) == lo for i in range(*rng_[t])) for t in range(T)]
            ex = np.concatenate([[0], np.cumsum(cnt)[:-1]])
            iT = None
            for t in range(T):
                if ex[t] < rem <= ex[t] + cnt[t]:
                    seen = ex[t]
                    for i in range(*rng_[t]):
                        if K(i) == lo:
                            seen += 1
                            if seen == rem:
                                iT = i
            kT = lo
            break
        b = Bins(lo, hi)
        hist = [0] * BINS
        for i in range(ncand):
            k = K(i)
            if lo <= k <= hi:
                h = b(k)
                assert 0 <= h < BINS, ("hist", h)
                hist[h] += 1
        mine = [sum(hist[binq(t, q)] for q in range(kbp) if binq(t, q) >= 0) for t in range(T)]
        ex = np.concatenate([[0], np.cumsum(mine)[:-1]])
        found = None
        for t in range(T):
            if ex[t] < rem <= ex[t] + mine[t]:
                run, q = ex[t], 0
                while q < kbp and binq(t, q) >= 0:
                    c = hist[binq(t, q)]
                    if run + c >= rem:
                        found = (binq(t, q), c, run)
                        break
                    run += c
                    q += 1
        assert found is not None
        bstar, bcount, above = found
        rem -= above
        if on_threshold is not None:
            on_threshold(b, bstar)
            on_threshold = None
        assert 1 <= rem <= bcount
        if bcount <= BUCKET:
            bucket = [(K(i), i) for i in range(ncand) if lo <= K(i) <= hi and b(K(i)) == bstar]
            assert len(bucket) == bcount <= BUCKET  # the bucket arrays hold BUCKET entries
            ranks = [sum((ok > mk) or (ok == mk and oi < mi) for ok, oi in bucket) for mk, mi in bucket]
            sel = [e for e, r in zip(bucket, ranks) if r == rem - 1]
            assert len(sel) == 1
            kT, iT = sel[0]
            break
        ks = [K(i) for i in range(ncand) if lo <= K(i) <= hi and b(K(i)) == bstar]
        nlo, nhi = min(ks), max(ks)
        assert (nlo, nhi) != (lo, hi)  # every step narrows the range
        lo, hi = nlo, nhi

    def kept(i):
        return K(i) > kT or (K(i) == kT and i <= iT)
    nsel = []
    for t in range(T):
        c0, c1 = rng_[t]
        ln = c1 - c0
        off = (t % 32) % ln if ln > 0 else 0  # the rotated start of the counting pass
        n = 0
        for _ in range(ln):
            n += kept(c0 + off)
            off += 1
            if off == ln:
                off = 0
        nsel.append(n)
    pos = np.concatenate([[0], np.cumsum(nsel)[:-1]])
    for t in range(T):
        p = int(pos[t])
        if nsel[t]:
            for i in range(*rng_[t]):
                if kept(i):
                    W(p, i)
                    p += 1
    W(m, NB - 1)
    return out


def sorted_selection(keys, NB, kmax):
    kb = min(kmax, NB)
    if NB == 0:
        return [-1] * kmax
    idx = sorted(range(NB - 1), key=lambda i: (-keys[i], i))[:kb - 1]
    return sorted(idx) + [NB - 1] + [-1] * (kmax - kb)


SCORE_FAMILIES = {
    "normal": lambda rng, n: rng.standard_normal(n) * 0.06,
    "all_equal": lambda rng, n: np.full(n, 0.25),
    "clustered": lambda rng, n: 0.5 + rng.integers(0, 40, n) * 1e-7,
    "few": lambda rng, n: rng.choice([0.1, 0.2, 0.3, -0.2], n),
    "zeros": lambda rng, n: rng.choice([0.0, -0.0, 1e-30, -1e-30], n),
    "wide": lambda rng, n: rng.standard_normal(n) * 10.0 ** rng.integers(-20, 20, n),
    "geometric": lambda rng, n: rng.choice([-1.0, 1.0], n) * 2.0 ** -rng.integers(0, 120, n),
    "ulps": lambda rng, n: np.where(rng.random(n) < 0.02, 1e30, 1.0 + rng.integers(0, 3 * n, n) * 2.0 ** -23),
    "inf_nan": lambda rng, n: rng.choice([np.inf, -np.inf, np.nan, 1.0, -3e38, 3e38, 0.5], n),
}


@pytest.mark.parametrize("NB,kmax", [(33, 8), (64, 8), (512, 64), (512, 2), (1024, 103), (1025, 300), (4096, 64)])
def test_early_stages_take_only_kept_blocks_and_the_rest_completes_the_list(NB, kmax):
    """The fused step (one CTA per row) issues its first decode stages from the candidates whose
    bin lies above the first histogram's threshold bin, in index order, before the selection has
    finished; its producer later walks the finished list and skips those blocks. Every such block
    must be kept, never the open last block, and the stages issued plus the ones walked must be the
    kept list exactly once each."""
    rng = np.random.default_rng(NB * 7 + kmax)
    for name, gen in SCORE_FAMILIES.items():
        with np.errstate(all="ignore"):
            f = gen(rng, NB - 1).astype(np.float32)
        keys = [order_key(x) for x in f] + [0]
        for n_early in (1, 5, 7):
            early = []

            def hook(b, bstar):
                for i in range(NB - 1):  # the producer warp's ascending scan, 32 candidates a ballot
                    if len(early) < n_early and b(keys[i]) > bstar:
                        early.append(i)
            out = select_row(keys, NB, kmax, 384, hook)
            kept = [j for j in out if j >= 0]
            assert kept == sorted_selection(keys, NB, kmax)[:len(kept)], name
            assert len(early) <= n_early and early == sorted(set(early))
            assert all(j in kept and j != NB - 1 for j in early), (name, early)
            walked = [j for k, j in enumerate(kept) if not (k + 1 < len(kept) and j in early)]
            assert sorted(early + walked) == kept and walked[-1] == NB - 1, name


@pytest.mark.parametrize("NB,kmax,T", [(1, 8, 256), (2, 1, 256), (2, 8, 384), (33, 8, 384), (512, 64, 384),
                                       (513, 100, 256), (1024, 103, 384), (1025, 300, 384), (2049, 512, 256)])
def test_select_row_indices_in_bounds_and_list_exact(NB, kmax, T):
    rng = np.random.default_rng(NB * 31 + kmax)
    for name, gen in SCORE_FAMILIES.items():
        with np.errstate(all="ignore"):
            f = gen(rng, max(NB - 1, 0)).astype(np.float32)
        keys = [order_key(x) for x in f] + [0]  # NB - 1 candidates (the last block has no key)
        assert select_row(keys, NB, kmax, T) == sorted_selection(keys, NB, kmax), name
