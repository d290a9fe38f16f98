"""CPU checks of the attention kernels' synchronisation protocols (tests/pipeline_model.py).

Each model follows one kernel's role loops: the barriers each role waits on and arrives at (with the phase counters
the kernel keeps), the TMA copies, the tensor-pipe operations, and the TMEM / shared-memory regions each step reads
or writes. Thread counts are scaled down: a warpgroup arriving with all its threads is one arrival. Thousands of
random interleavings with random stalls must finish without a deadlock, a barrier phase passed with the wrong number
of completions, a region reused while a copy or tensor operation may still touch it, or a value read that another
step has overwritten. Planted mistakes, including the partial-row-sum race that an earlier version of the sparse
kernel had, must be caught.
"""
import random

import pytest

from tests.pipeline_model import Model


# --------------------------------------------------------------------------------------------------- dense step

def dense_model(m, n_items, T, with_mass, chunk_tiles, bugs=()):
    """attn_dense_kernel: one query block per item, T key tiles (single-buffered K, double-buffered V); with the mass
    phase (with_mass True), T more Q K^T tiles whose block sums are reduced through V buffer 0; with one-pass masses
    (with_mass "one_pass"), each forward tile's block sums stored to the workspace (W{g}) and reduced by both groups
    after the row sums are known, with the row factors in shared memory (F) between the PART and PART2 barriers."""
    one_pass = with_mass == "one_pass"
    two_pass = bool(with_mass) and not one_pass
    for b in ("Q_FULL", "Q_EMPTY", "K_FULL", "K_EMPTY", "S_FULL", "PV_DONE", "MMA_DONE",
              "V_FULL0", "V_FULL1", "V_EMPTY0", "V_EMPTY1"):
        m.bar(b)
    for b in ("S_FREE", "P_FULL", "O_FREE", "SUM_X", "PART", "PART2", "MASS_DONE"):
        m.bar(b, 2)  # both softmax warpgroups
    mass_tiles = T if two_pass else 0

    def qk_producer():
        nq = nk = 0
        for _ in range(n_items):
            yield ("wait", "Q_EMPTY", nq - 1)
            yield ("expect", "Q_FULL", 1)
            yield ("tma", "Q_FULL", 1, "Q")
            nq += 1
            for _ in range(T + mass_tiles):
                yield ("wait", "K_EMPTY", nk - 1)
                yield ("expect", "K_FULL", 1)
                yield ("tma", "K_FULL", 1, "K")
                nk += 1

    def v_producer():
        nv = 0
        for it in range(n_items):
            for _ in range(T):
                vb = nv & 1
                yield ("wait", f"V_EMPTY{vb}", (nv >> 1) - 1)
                yield ("expect", f"V_FULL{vb}", 1)
                yield ("tma", f"V_FULL{vb}", 1, f"V{vb}")
                nv += 1
            if two_pass:
                yield ("wait", "MASS_DONE", it)

    def mma():
        c = {"nq": 0, "n_qk": 0, "nk": 0, "n_pv": 0, "items": 0}

        def issue_pv(t):
            vb = c["n_pv"] & 1
            yield ("wait", "P_FULL", c["n_pv"])
            yield ("wait", f"V_FULL{vb}", c["n_pv"] >> 1)
            if t == 0:
                yield ("wait", "O_FREE", c["items"] - 1)
            yield ("mma", ["Ph0", "Ph1", f"V{vb}"], ["O"])
            yield ("commit", f"V_EMPTY{vb}")
            yield ("commit", "PV_DONE")
            c["n_pv"] += 1

        for _ in range(n_items):
            yield ("wait", "Q_FULL", c["nq"])
            c["nq"] += 1
            for t in range(T + mass_tiles):
                yield ("wait", "K_FULL", c["nk"])
                if c["n_qk"] > 0 and "no_s_free_wait" not in bugs:
                    yield ("wait", "S_FREE", c["n_qk"] - 1)
                yield ("mma", ["Q", "K"], ["S"])
                yield ("commit", "S_FULL")
                yield ("commit", "K_EMPTY")
                c["nk"] += 1
                c["n_qk"] += 1
                if t == T + mass_tiles - 1:
                    yield ("commit", "Q_EMPTY")
                if 1 <= t <= T:
                    yield from issue_pv(t - 1)
            if mass_tiles == 0:
                yield from issue_pv(T - 1)
            c["items"] += 1
        yield ("commit", "MMA_DONE")
        yield ("wait", "MMA_DONE", 0)

    def softmax(g):
        n_s = n_pv = n_chunks = 0
        for it in range(n_items):
            for t in range(T):
                yield ("wait", "S_FULL", n_s)
                n_s += 1
                yield ("read", "S")  # both halves: its own, and the other's for the row max
                yield ("arrive", "S_FREE")
                if t > 0 and "no_pv_wait_before_p" not in bugs:
                    yield ("wait", "PV_DONE", n_pv)
                    n_pv += 1
                    yield ("read", "O")  # rescale of this group's half of O
                    yield ("write", "O")
                yield ("put", f"Ph{g}", ("p", it, t))
                if one_pass:
                    yield ("put", f"W{g}", ("sums", it, t))  # this tile's block sums of its rows
                yield ("arrive", "P_FULL")
            if "no_pv_wait_before_p" in bugs:
                n_pv += T - 1
            yield ("wait", "PV_DONE", n_pv)
            n_pv += 1
            yield ("put", f"XSh{g}", ("sum", it))  # one exchange buffer for every item
            yield ("arrive", "SUM_X")
            yield ("wait", "SUM_X", it)
            yield ("read", "pad")  # the read of the other group's sums may come well after the wait
            yield ("get", f"XSh{g ^ 1}", ("sum", it))
            yield ("read", "O")
            yield ("arrive", "O_FREE")
            if one_pass:
                if g == 0:
                    yield ("put", "F", ("factors", it))
                yield ("arrive", "PART")
                if "no_part_wait" not in bugs:
                    yield ("wait", "PART", it)
                yield ("get", "F", ("factors", it))
                yield ("get", "W0", ("sums", it, T - 1))  # the reduction reads both groups' stored sums
                yield ("get", "W1", ("sums", it, T - 1))
                yield ("arrive", "PART2")
                if "no_part2_wait" not in bugs:
                    yield ("wait", "PART2", it)
            if two_pass:
                for t0 in range(0, T, chunk_tiles):
                    for _ in range(t0, min(T, t0 + chunk_tiles)):
                        yield ("wait", "S_FULL", n_s)
                        n_s += 1
                        yield ("read", "S")
                        yield ("arrive", "S_FREE")
                        yield ("write", "V0")  # per-warp partial block sums
                    yield ("arrive", "PART")
                    yield ("wait", "PART", n_chunks)
                    yield ("read", "V0")
                    yield ("arrive", "PART2")
                    yield ("wait", "PART2", n_chunks)
                    n_chunks += 1
                yield ("arrive", "MASS_DONE")

    m.roles = {"qk_producer": qk_producer(), "v_producer": v_producer(), "mma": mma(),
               "softmax0": softmax(0), "softmax1": softmax(1)}


# -------------------------------------------------------------------------------------------------- sparse step

def sparse_model(m, counts, bugs=(), seed=0):
    """attn_sparse_kernel: items read ahead through a four-entry ring, Q double-buffered in shared memory (read by every
    Q K^T of its item, released after the last), K in a 3-stage ring, V in a 2-stage ring whose last slot of an item
    takes the item's O for the TMA store, two S buffers and two P buffers in TMEM, a data-dependent rescale of O, and
    an epilogue deferred until the next item's first tile (row sums exchanged through shared memory)."""
    rng = random.Random(seed)
    RING, KST = 4, 3
    for i in range(RING):
        m.bar(f"IT_FULL{i}")
        m.bar(f"IT_EMPTY{i}", 5)  # Q/K producer, V producer, MMA issuer, two softmax warpgroups
    for i in range(2):
        for b in ("Q_FULL", "Q_EMPTY", "V_FULL", "V_EMPTY", "S_FULL", "PV_DONE"):
            m.bar(f"{b}{i}")
        m.bar(f"P_FULL{i}", 2)
        m.bar(f"STAGED{i}", 2)
    for i in range(KST):
        m.bar(f"K_FULL{i}"), m.bar(f"K_EMPTY{i}")
    for b in ("MMA_DONE", "STORE_DONE"):
        m.bar(b)
    for b in ("SUM_X", "O_FREE"):
        m.bar(b, 2)
    n_items = len(counts)
    rescale = {(g, n): rng.random() < 0.4 for g in (0, 1) for n in range(sum(counts) + 2)}

    def next_item(r):
        yield ("wait", f"IT_FULL{r % RING}", r // RING)
        yield ("arrive", f"IT_EMPTY{r % RING}")

    def reader():
        for r in range(n_items + 1):  # the last record marks the end of the stream
            yield ("wait", f"IT_EMPTY{r % RING}", r // RING - 1)
            yield ("arrive", f"IT_FULL{r % RING}")

    def qk_producer():
        nq = nk = 0
        for r in range(n_items + 1):
            yield from next_item(r)
            if r == n_items:
                return
            qs = nq & 1
            yield ("wait", f"Q_EMPTY{qs}", (nq >> 1) - 1)
            yield ("expect", f"Q_FULL{qs}", 1)
            yield ("tma", f"Q_FULL{qs}", 1, f"Q{qs}")
            nq += 1
            for _ in range(counts[r]):
                ks = nk % KST
                yield ("wait", f"K_EMPTY{ks}", nk // KST - 1)
                yield ("expect", f"K_FULL{ks}", 1)
                yield ("tma", f"K_FULL{ks}", 1, f"K{ks}")
                nk += 1

    def v_producer():
        nv, n_store = 0, 0
        empty, staged, fin = [0, 0], [0, 0], [False, False]

        def flush(sl):
            nonlocal n_store
            yield ("wait", f"STAGED{sl}", staged[sl])
            staged[sl] += 1
            yield ("store", "STORE_DONE", f"V{sl}")
            yield ("wait", "STORE_DONE", n_store)
            n_store += 1
            fin[sl] = False

        for r in range(n_items + 1):
            yield from next_item(r)
            if r == n_items:
                break
            for t in range(counts[r]):
                vs = nv & 1
                if nv >= 2:
                    if fin[vs]:
                        yield from flush(vs)
                    else:
                        yield ("wait", f"V_EMPTY{vs}", empty[vs])
                        empty[vs] += 1
                yield ("expect", f"V_FULL{vs}", 1)
                yield ("tma", f"V_FULL{vs}", 1, f"V{vs}")
                fin[vs] = t == counts[r] - 1
                nv += 1
        for k in range(2):
            if fin[(nv + k) & 1]:
                yield from flush((nv + k) & 1)

    def mma():
        nq = n = items = 0
        pend = {}

        def issue_pv():
            b = pend["n"] & 1
            yield ("wait", f"P_FULL{b}", pend["n"] >> 1)
            yield ("wait", f"V_FULL{b}", pend["n"] >> 1)
            if pend["first"] and pend["item"] > 0 and "no_o_free_wait" not in bugs:
                yield ("wait", "O_FREE", pend["item"] - 1)
            yield ("mma", [f"P{b}h0", f"P{b}h1", f"V{b}"], ["O"])
            if not pend["last"]:
                yield ("commit", f"V_EMPTY{b}")
            yield ("commit", f"PV_DONE{b}")
            pend.clear()

        for r in range(n_items + 1):
            yield from next_item(r)
            if r == n_items:
                break
            qs = nq & 1
            yield ("wait", f"Q_FULL{qs}", nq >> 1)
            nq += 1
            for t in range(counts[r]):
                ks, b = n % KST, n & 1
                yield ("wait", f"K_FULL{ks}", n // KST)
                yield ("mma", [f"Q{qs}", f"K{ks}"], [f"S{b}"])
                yield ("commit", f"S_FULL{b}")
                yield ("commit", f"K_EMPTY{ks}")
                if t == counts[r] - 1 and "early_q_release" not in bugs:
                    yield ("commit", f"Q_EMPTY{qs}")
                if t == 0 and "early_q_release" in bugs:
                    yield ("commit", f"Q_EMPTY{qs}")
                if pend:
                    yield from issue_pv()
                pend.update(n=n, first=t == 0, last=t == counts[r] - 1, item=items)
                n += 1
            items += 1
        if pend:
            yield from issue_pv()
        yield ("commit", "MMA_DONE")
        yield ("wait", "MMA_DONE", 0)

    def softmax(g):
        n = n_epi = 0
        pend, nl = False, 0

        def epilogue():
            nonlocal n_epi
            bl = nl & 1
            if "no_epilogue_pv_wait" not in bugs:
                yield ("wait", f"PV_DONE{bl}", nl >> 1)
            yield ("put", f"X{g}", ("sum", n_epi))  # partial row sums in shared memory
            yield ("arrive", "SUM_X")
            yield ("wait", "SUM_X", n_epi)
            yield ("read", "pad")  # the read of the other group's sums may come well after the wait
            yield ("get", f"X{g ^ 1}", ("sum", n_epi))
            yield ("read", "O")
            yield ("arrive", "O_FREE")
            yield ("write", f"V{bl}")  # O staged for the TMA store
            yield ("arrive", f"STAGED{bl}")
            n_epi += 1

        for r in range(n_items + 1):
            yield from next_item(r)
            if r == n_items:
                break
            for t in range(counts[r]):
                b = n & 1
                yield ("wait", f"S_FULL{b}", n >> 1)
                yield ("read", f"S{b}")
                if t > 0 and rescale[(g, n)]:
                    if "no_rescale_wait" not in bugs:
                        yield ("wait", f"PV_DONE{b ^ 1}", (n - 1) >> 1)
                    yield ("read", "O")
                    yield ("write", "O")
                yield ("put", f"P{b}h{g}", ("p", n))
                yield ("arrive", f"P_FULL{b}")
                if t == 0 and pend:
                    yield from epilogue()
                    pend = False
                n += 1
            pend, nl = True, n - 1
        if pend:
            yield from epilogue()

    m.roles = {"reader": reader(), "qk_producer": qk_producer(), "v_producer": v_producer(), "mma": mma(),
               "softmax0": softmax(0), "softmax1": softmax(1)}


# -------------------------------------------------------------------------------------------------------- tests

def _dense_cases():
    return [(n_items, T, mass, chunk) for n_items in (1, 3) for T in (1, 2, 5) for mass in (False, True, "one_pass")
            for chunk in (1, 2)]


@pytest.mark.parametrize("n_items,T,with_mass,chunk", _dense_cases())
def test_dense_protocol(n_items, T, with_mass, chunk):
    for seed in range(12):
        m = Model(seed * 31 + T, pipe_overlap=bool(seed & 1))
        dense_model(m, n_items, T, with_mass, chunk)
        m.run()
        assert not m.errors, m.errors[:3]


def test_sparse_protocol():
    rng = random.Random(5)
    for seed in range(300):
        counts = [rng.choice([1, 1, 1, 2, 3, 5]) for _ in range(rng.randint(1, 8))]
        m = Model(seed, pipe_overlap=bool(seed & 1))
        sparse_model(m, counts, seed=seed)
        m.run()
        assert not m.errors, (counts, m.errors[:3])


@pytest.mark.parametrize("bug,mode", [("no_s_free_wait", True), ("no_pv_wait_before_p", True),
                                      ("no_part_wait", "one_pass"), ("no_part2_wait", "one_pass")])
def test_dense_planted_mistakes_are_caught(bug, mode):
    caught = 0
    for seed in range(40):
        m = Model(seed)
        dense_model(m, 3, 3, mode, 2, bugs=(bug,))
        m.run()
        caught += bool(m.errors)
    assert caught > 0


@pytest.mark.parametrize("bug", ["no_o_free_wait", "no_epilogue_pv_wait", "no_rescale_wait", "early_q_release"])
def test_sparse_planted_mistakes_are_caught(bug):
    rng = random.Random(2)
    caught = 0
    for seed in range(120):
        counts = [rng.choice([1, 1, 2, 3]) for _ in range(rng.randint(2, 8))]
        m = Model(seed, pipe_overlap=bool(seed & 1))
        sparse_model(m, counts, bugs=(bug,), seed=seed)
        m.run()
        caught += bool(m.errors)
    assert caught > 0
