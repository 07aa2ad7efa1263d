"""The engine's copy / dequant plan (lst_plan_reads), on the host: for every schedule the engine
runs (SFT 2L reads, DPO 3L reads, with and without reuse, over consecutive steps), each read
computes from a slot and a weight scratch that hold its layer, a copy never lands in the slot the
previous read computes from, and every wait names the right read. No GPU needed."""
import pytest

lst = pytest.importorskip("layer_streamed_qlora_streaming_b200")

SLOT, COPY, WAIT, LOADED, WSLOT, DEQ, WWAIT, WFILLED = range(8)


def reads(L, dpo):
    return (list(range(L)) if dpo else []) + list(range(L)) + list(range(L - 1, -1, -1))


def check_step(layers, rows, held0, wheld0, reuse, nf4, pre_slot=-1):
    """Replay the plan on two slots / two scratches and check every invariant; returns the number
    of copies and dequants. pre_slot: the slot a previous step copied this step's first read into."""
    held = list(held0) if reuse else [-1, -1]
    wheld = list(wheld0) if reuse else [-1, -1]
    if not reuse and pre_slot >= 0:
        held[pre_slot] = layers[0]
    last_use, loaded, wlast, wfill = [-1, -1], [-1, -1], [-1, -1], [-1, -1]
    copies = deqs = 0
    for n, (j, row) in enumerate(zip(layers, rows)):
        s = row[SLOT]
        assert s in (0, 1)
        if row[COPY]:
            copies += 1
            if n > 0:
                assert s != rows[n - 1][SLOT], "a copy must not land in the slot the previous read uses"
            assert row[WAIT] == last_use[s]
            held[s] = j
            loaded[s] = n
        else:
            assert (reuse or (n == 0 and s == pre_slot)) and held[s] == j, \
                "a read without a copy must find its layer in the slot"
        assert held[s] == j
        assert row[LOADED] == loaded[s]
        last_use[s] = n
        if not nf4:
            assert row[DEQ] == 0
            continue
        w = row[WSLOT]
        assert w in (0, 1)
        if row[DEQ]:
            deqs += 1
            if n > 0:
                assert w != rows[n - 1][WSLOT], "a dequant must not overwrite the scratch in use"
            assert row[WWAIT] == wlast[w]
            wheld[w] = j
            wfill[w] = n
        else:
            assert reuse and wheld[w] == j
        assert wheld[w] == j
        assert row[WFILLED] == wfill[w]
        wlast[w] = n
    return copies, deqs, tuple(held), tuple(wheld)


@pytest.mark.parametrize("L", [1, 2, 3, 4, 7, 32])
@pytest.mark.parametrize("dpo", [False, True])
@pytest.mark.parametrize("reuse", [False, True])
@pytest.mark.parametrize("nf4", [False, True])
def test_plan_invariants_over_consecutive_steps(L, dpo, reuse, nf4):
    layers = reads(L, dpo)
    R = len(layers)
    held, wheld = (-1, -1), (-1, -1)
    counts = []
    for step in range(3):
        rows, h2, w2 = lst.plan_reads(layers, reuse, nf4, held, wheld)
        copies, deqs, h3, w3 = check_step(layers, rows.tolist(), held, wheld, reuse, nf4)
        assert (h3, w3 if nf4 else w2) == (h2, w2)
        counts.append((copies, deqs))
        held, wheld = h2, w2
    if not reuse:
        assert all(c == (R, R if nf4 else 0) for c in counts)      # every read fetches
    elif L == 1:
        assert [c[0] for c in counts] == [1, 0, 0]                # one layer: fetched once, kept
    elif L >= 3:
        # first step: the two layers at the forward/backward turn are kept; later steps also keep
        # the two layers the previous step ended with (layers 0 and 1 begin the next step)
        assert [c[0] for c in counts] == [R - 2, R - 4, R - 4]
        if nf4:
            assert [c[1] for c in counts] == [R - 2, R - 4, R - 4]


def test_canonical_schedule_alternates_and_waits_two_back():
    rows, _, _ = lst.plan_reads(reads(5, False), False, True)
    for n, r in enumerate(rows.tolist()):
        assert r[SLOT] == n % 2 and r[COPY] == 1 and r[WAIT] == (n - 2 if n >= 2 else -1) and r[LOADED] == n
        assert r[WSLOT] == n % 2 and r[DEQ] == 1 and r[WWAIT] == (n - 2 if n >= 2 else -1)


def test_plan_rejects_bad_arguments():
    with pytest.raises(lst.LstError):
        lst.plan_reads([], True, True)
    with pytest.raises(lst.LstError):
        lst.plan_reads([0, -1], True, True)


@pytest.mark.parametrize("L", [1, 2, 3, 32])
@pytest.mark.parametrize("dpo", [False, True])
@pytest.mark.parametrize("nf4", [False, True])
def test_prefetch_copies_the_next_first_read_after_the_last_read_of_its_slot(L, dpo, nf4):
    """Reuse off with prefetch: every step still copies R blobs (R - 1 of its own reads plus the next
    step's first read); that copy goes into the slot the step's last read does not use and waits
    only for the read before it; the next step computes its first read from that slot uncopied."""
    layers = reads(L, dpo)
    R = len(layers)
    held, wheld, pre = (-1, -1), (-1, -1), -1
    for step in range(3):
        rows, h2, w2, (pslot, pwait) = lst.plan_reads(layers, False, nf4, held, wheld, prefetch=pre)
        rows = rows.tolist()
        copies, deqs, h3, _ = check_step(layers, rows, held, wheld, False, nf4, pre_slot=pre)
        assert copies == (R if pre < 0 else R - 1)
        assert deqs == (R if nf4 else 0)                           # dequant is not carried over
        if pre >= 0:
            assert rows[0][SLOT] == pre and rows[0][COPY] == 0 and rows[0][LOADED] == -1
        assert pslot == 1 - rows[-1][SLOT]
        assert pwait == max(n for n in range(R) if rows[n][SLOT] == pslot) == R - 2
        assert h2[pslot] == layers[0] and h2[1 - pslot] == h3[1 - pslot]
        held, wheld, pre = h2, w2, pslot
    # with reuse on there is nothing to prefetch
    _, _, _, p = lst.plan_reads(layers, True, nf4, (-1, -1), (-1, -1), prefetch=-1)
    assert p == (-1, -1)
    with pytest.raises(lst.LstError):
        lst.plan_reads(layers, False, nf4, prefetch=2)
