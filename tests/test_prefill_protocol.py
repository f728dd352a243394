"""A randomised model of the barrier protocol of the persistent prefill
kernel (``csrc/paged_prefill.cu``), run on the CPU.

Roles are generators that wait and arrive exactly as the kernel's warps do:
the K and V load warps (Q tiles into two buffers, K/V tiles into two stages),
the S-issuing and the P V-issuing MMA warps, and eight softmax warps (with a
random lazy rescale of O and the per-item epilogue).  S goes through three
tensor-memory buffers; P overwrites S in its buffer; one O accumulator.  The
K-load warp takes every item (empty ones included) and publishes its index in
a four-slot ring, which the eleven other warps read before they start the
item.  mbarriers complete a phase when their expected arrivals are in; a wait
is the parity test the hardware does.  tcgen05 work runs on one in-order pipe,
a commit arrives once everything its thread issued before it is done; TMA
loads land in any order.

Checked on every schedule: no deadlock; every parity wait releases exactly on
the phase it means (a wait that could be satisfied by an older or a newer
phase is a bug even when the schedule happens to be benign); no buffer (Q, K
and V stages, S buffers in tensor memory, O) is rewritten while an
asynchronous reader is pending, or read before its writer completed.  Each
synchronisation the kernel relies on, removed or pointed at the wrong tile,
makes some schedule fail.
"""

import random

import pytest

pytestmark = pytest.mark.filterwarnings("ignore")

NS = 3  # S buffers in tensor memory


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.arrivals, self.done = name, count, 0, 0

    def arrive(self):
        self.arrivals += 1
        assert self.arrivals <= self.count, f"{self.name}: too many arrivals"
        if self.arrivals == self.count:
            self.arrivals, self.done = 0, self.done + 1


def run_model(ntiles_per_item, seed, drop=None):
    """ntiles_per_item: K/V tiles of each item of one CTA (0 = an empty item,
    skipped by every role).  drop: name of one synchronisation to remove (or,
    for "rescale" / "epilogue", to point at the tile before the right one)."""
    rnd = random.Random(seed)
    bars = {}

    def bar(name, count=1):
        bars[name] = Bar(name, count)

    for i in range(2):
        for nm in ("q", "qfree", "k", "kfree", "v", "vfree"):
            bar(f"{nm}{i}")
    for i in range(NS):
        bar(f"s{i}")
        bar(f"pfree{i}")
        bar(f"p{i}", 8)
    for i in range(4):
        bar(f"item{i}")
        bar(f"itemfree{i}", 11)
    ring = {}
    pipe, loads = [], []
    pending = {}          # resource -> list of async ops reading (or writing) it
    s_ops = {}            # global tile -> S op
    st = {"pv_item": -1, "o_readers": 0, "s_readers": {}}

    def wait(name, phase):
        b = bars[name]
        while (b.done & 1) == (phase & 1):
            assert b.done <= phase, f"{name}: phase {phase} overtaken ({b.done} done)"
            yield
        assert b.done == phase + 1, f"{name}: released with {b.done} phases done, meant phase {phase}"

    def busy(res):
        return [op for op in pending.get(res, []) if not op["done"]]

    def read(op, *res):
        for r in res:
            pending.setdefault(r, []).append(op)

    items = list(ntiles_per_item)

    def publish(k):
        """The K-load warp takes item k (len(items): the end) and publishes its
        index in slot k % 4, once the eleven readers have read what the slot
        held four items back."""
        if k >= 4 and drop != "itemfree":
            yield from wait(f"itemfree{k % 4}", (k - 4) >> 2)
        ring[k % 4] = k
        bars[f"item{k % 4}"].arrive()
        yield

    def read_items():
        """Another warp's view of the item sequence: item k's tile count, then
        None at the end."""
        for k in range(len(items) + 1):
            yield from wait(f"item{k % 4}", k >> 2)
            assert ring[k % 4] == k, "a warp read another item's index"
            bars[f"itemfree{k % 4}"].arrive()
            yield ("item", items[k] if k < len(items) else None)

    def walk(gen):
        """The next item's tile count as read from the ring (waits pass
        through); None at the end."""
        for x in gen:
            if isinstance(x, tuple):
                return x[1]
            yield x
        return None

    def producer(kind):
        n = jt = 0
        src = None if kind == "K" else read_items()
        for k in range(len(items) + 1):
            if kind == "K":
                yield from publish(k)
                nt = items[k] if k < len(items) else None
            else:
                nt = yield from walk(src)
            if nt is None:
                break
            if nt == 0:
                continue
            if kind == "K":
                qb = n & 1
                if n >= 2 and drop != "qfree":
                    yield from wait(f"qfree{qb}", (n - 2) >> 1)
                assert not busy(f"Q{qb}"), "Q buffer rewritten while S reads it"
                loads.append((f"q{qb}", {"done": False}))
            for _ in range(nt):
                b = jt & 1
                if jt >= 2:
                    yield from wait(f"{kind.lower()}free{b}", (jt - 2) >> 1)
                assert not busy(f"{kind}{b}"), f"{kind} stage rewritten while read"
                loads.append((f"{kind.lower()}{b}", {"done": False}))
                jt += 1
                yield
            n += 1

    def s_issuer():
        n = jt = 0
        src = read_items()
        while True:
            nt = yield from walk(src)
            if nt is None:
                break
            if nt == 0:
                continue
            qb = n & 1
            yield from wait(f"q{qb}", n >> 1)
            for j in range(nt):
                b, ks = jt % NS, jt & 1
                if jt >= NS and drop != "pfree":
                    yield from wait(f"pfree{b}", jt // NS - 1)
                yield from wait(f"k{ks}", jt >> 1)
                assert not busy(f"S{b}"), "S buffer rewritten while P V reads P"
                assert st["s_readers"].get(b, 0) == 0, "S buffer rewritten while the softmax reads it"
                op = {"done": False, "tile": jt}
                read(op, f"Q{qb}", f"K{ks}")
                s_ops[jt] = op
                pipe.extend([("op", op), ("commit", f"s{b}"), ("commit", f"kfree{ks}")])
                if j == nt - 1:
                    pipe.append(("commit", f"qfree{qb}"))
                jt += 1
                yield
            n += 1

    def pv_issuer():
        n = jt = 0
        src = read_items()
        while True:
            nt = yield from walk(src)
            if nt is None:
                break
            if nt == 0:
                continue
            for j in range(nt):
                b, vs = jt % NS, jt & 1
                yield from wait(f"v{vs}", jt >> 1)
                yield from wait(f"p{b}", jt // NS)
                assert st["o_readers"] == 0, "P V writes O while a softmax warp reads it"
                op = {"done": False, "tile": jt}
                read(op, f"V{vs}", f"S{b}", "O")
                st["pv_item"] = max(st["pv_item"], n)
                pipe.extend([("op", op), ("commit", f"vfree{vs}"), ("commit", f"pfree{b}")])
                jt += 1
                yield
            n += 1

    def softmax():
        n = jt = 0
        src = read_items()
        while True:
            nt = yield from walk(src)
            if nt is None:
                break
            if nt == 0:
                continue
            for j in range(nt):
                b = jt % NS
                yield from wait(f"s{b}", jt // NS)
                assert s_ops[jt]["done"], "S read before its MMA completed"
                st["s_readers"][b] = st["s_readers"].get(b, 0) + 1
                yield
                st["s_readers"][b] -= 1
                if j == nt - 1 and rnd.random() < 0.5:
                    # the item's last tile reaches past the context: this warp
                    # zeroes the tail rows of the V stage before arriving on P
                    vs = jt & 1
                    yield from wait(f"v{vs}", jt >> 1)
                    assert not busy(f"V{vs}"), "V stage zeroed while a P V reads it"
                    assert not any(name == f"v{vs}" for name, _ in loads), "V stage zeroed under a landing load"
                if j > 0 and rnd.random() < 0.3:
                    jp = jt - 1 if drop != "rescale" else jt - 2
                    if jp >= 0:
                        yield from wait(f"pfree{jp % NS}", jp // NS)
                    assert not busy("O"), "O rescaled while a P V is pending"
                    st["o_readers"] += 1
                    yield
                    st["o_readers"] -= 1
                yield
                bars[f"p{b}"].arrive()
                jt += 1
            jl = jt - 1 if drop != "epilogue" else jt - 2
            if jl >= 0:
                yield from wait(f"pfree{jl % NS}", jl // NS)
            assert not busy("O"), "epilogue reads O with a P V pending"
            st["o_readers"] += 1
            yield
            assert st["pv_item"] <= n, "next item's P V issued while O is read out"
            st["o_readers"] -= 1
            yield
            n += 1

    roles = [producer("K"), producer("V"), s_issuer(), pv_issuer()] + [softmax() for _ in range(8)]
    alive = list(range(len(roles)))
    for _ in range(400000):
        if not (alive or pipe or loads):
            return
        r = rnd.random()
        if pipe and r < 0.15:
            kind, x = pipe.pop(0)
            if kind == "op":
                x["done"] = True
            else:
                bars[x].arrive()
            continue
        if loads and r < 0.3:
            name, op = loads.pop(rnd.randrange(len(loads)))
            op["done"] = True
            bars[name].arrive()
            continue
        if alive:
            k = rnd.choice(alive)
            try:
                next(roles[k])
            except StopIteration:
                alive.remove(k)
    raise AssertionError("deadlock")


def _items(seed):
    rnd = random.Random(seed)
    return [rnd.choice([0, 1, 1, 2, 3, 5, 8]) for _ in range(rnd.randint(1, 9))]


def test_protocol_holds_on_random_schedules():
    for seed in range(300):
        run_model(_items(seed), seed)


@pytest.mark.parametrize("drop", ["qfree", "pfree", "itemfree", "rescale", "epilogue"])
def test_each_synchronisation_is_needed(drop):
    """Removing the Q-buffer release, the S-buffer release (P V done) or the
    item ring's release, or pointing the rescale's or the epilogue's wait at
    the tile before the one it must wait for, breaks some schedule."""
    failures = 0
    for seed in range(300):
        try:
            run_model(_items(seed), seed, drop=drop)
        except AssertionError:
            failures += 1
    assert failures > 0
