"""Discrete model of a CTA's synchronisation protocol, shared by the protocol tests: mbarriers
with the hardware's parity rule, arrival counts and TMA transaction counts; MMAs executed in
issue order per issuing thread and interleaved at random across threads; commits that
arrive once everything their thread issued before them has completed; TMA loads completing
at random times; and reads of named memory regions checked against the data they must see.
Roles are generators that yield ("wait", barrier, phase), ("until", predicate) or None (a
plain step).  Bulk store groups (TMA stores committed as a group) read their sources when
they execute, in any order."""
import random


class Violation(Exception):
    pass


class Barrier:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.pending, self.tx, self.phase = count, 0, 0

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        if self.pending < 0:
            raise Violation(f"{self.name}: more arrivals than its count")
        self._maybe_complete()

    def tx_done(self):
        self.tx -= 1
        self._maybe_complete()

    def ready(self, k):
        """A wait for the completion of phase k (parity k & 1)."""
        if self.phase >= k + 2:
            raise Violation(f"{self.name}: phase {k} overrun (count {self.phase})")
        return (self.phase & 1) != (k & 1)


class Sim:
    def __init__(self, seed, abort_after=None):
        self.rng = random.Random(seed)
        # abort injection: after this many scheduler steps a role's bounded wait gives up;
        # from then on every abortable wait returns False (the CTA abort flag)
        self.abort_after, self.aborted, self.steps = abort_after, False, 0
        self.bars, self.mem, self.queues, self.tma = {}, {}, {}, []
        self.bulk, self.bulk_seq = [], 0  # bulk store groups: (seq, reads, who, owner)
        self.bulk_issued = {}  # per owner: sequence numbers of its groups, in issue order

    def bar(self, name, count):
        self.bars[name] = Barrier(name, count)

    # data ------------------------------------------------------------------------------
    def write(self, region, label):
        self.mem[region] = label

    def read(self, region, want, who):
        if self.aborted:
            return  # after an abort the outputs are undefined; only teardown is checked
        got = self.mem.get(region)
        if got != want:
            raise Violation(f"{who} read {region}: saw {got}, expected {want}")

    # asynchronous work ---------------------------------------------------------------------
    def mma(self, thread, reads, writes, who):
        """An MMA group: checks its reads and performs its writes when it executes."""
        self.queues.setdefault(thread, []).append(("mma", reads, writes, who))

    def commit(self, thread, barrier):
        self.queues.setdefault(thread, []).append(("commit", barrier))

    def tma_load(self, barrier, region, label):
        self.tma.append((barrier, region, label))

    def bulk_group(self, reads, who, owner=None):
        """A committed group of bulk (TMA) stores or reduces, issued by thread `owner`: it
        reads its source regions when it executes; groups execute in any order."""
        self.bulk_seq += 1
        self.bulk.append((self.bulk_seq, reads, who, owner))
        self.bulk_issued.setdefault(owner, []).append(self.bulk_seq)

    def bulk_read_done_but(self, k, owner=None):
        """cp.async.bulk.wait_group.read k by thread `owner` (bulk groups are per thread):
        every group of that thread but its k most recent has read its source."""
        mine = [seq for seq, _, _, o in self.bulk if o == owner]
        issued = self.bulk_issued.get(owner, [])
        recent = set(issued[-k:]) if k > 0 else set()
        return all(seq in recent for seq in mine)

    def _step_async(self):
        choices = [q for q in self.queues.values() if q]
        if self.tma:
            choices.append(self.tma)
        if self.bulk:
            choices.append(self.bulk)
        if not choices:
            return False
        q = self.rng.choice(choices)
        if q is self.bulk:
            _, reads, who, _ = self.bulk.pop(self.rng.randrange(len(self.bulk)))
            for region, want in reads:
                self.read(region, want, who)
        elif q is self.tma:
            barrier, region, label = self.tma.pop(self.rng.randrange(len(self.tma)))
            self.write(region, label)
            self.bars[barrier].tx_done()
        else:
            op = q.pop(0)
            if op[0] == "mma":
                _, reads, writes, who = op
                for region, want in reads:
                    self.read(region, want, who)
                for region, label in writes:
                    self.write(region, label)
            else:
                self.bars[op[1]].arrive()
        return True

    def run(self, roles):
        """roles: generators yielding ("wait", barrier, phase) (a bounded wait: the value sent
        back is False once the CTA has aborted), ("drain", barrier, phase) (a wait for the
        role's own asynchronous work, which must complete), ("until", predicate) or None
        (a plain step).  When the last role returns -- the kernel's final block barrier,
        after which tensor memory is freed -- no MMA, TMA load or bulk store may be in
        flight."""
        state = {name: None for name in roles}  # pending wait of each role
        live = dict(roles)
        idle = 0

        def ready(w):
            if w is None:
                return True
            if w[0] == "until":
                return w[1]()
            if w[0] == "wait" and self.aborted:
                return True
            return self.bars[w[1]].ready(w[2])

        sent = {name: None for name in roles}
        while live or any(self.queues.values()) or self.tma or self.bulk:
            self.steps += 1
            if self.abort_after is not None and self.steps >= self.abort_after:
                self.aborted = True
            runnable = [n for n in live if ready(state[n])]
            pending = any(self.queues.values()) or self.tma or self.bulk
            options = runnable + (["async"] if pending else [])
            if not options:
                waits = {n: state[n] for n in live}
                raise Violation(f"deadlock: {waits}")
            pick = self.rng.choice(options)
            if pick == "async":
                self._step_async()
                continue
            w = state[pick]
            if w is not None and w[0] in ("wait", "drain") and w[0] == "wait":
                value = not (self.aborted and not self.bars[w[1]].ready(w[2]))
            else:
                value = True
            try:
                req = live[pick].send(value if sent[pick] is not None else None)
                sent[pick] = True
                if req is None:
                    state[pick] = None
                elif req[0] in ("wait", "drain"):
                    state[pick] = (req[0], req[1], req[2])
                else:
                    state[pick] = ("until", req[1])
            except StopIteration:
                del live[pick]
                state.pop(pick)
                if not live and (any(self.queues.values()) or self.tma or self.bulk):
                    raise Violation("the CTA finished with asynchronous work in flight")
            idle += 1
            if idle > 10_000_000:
                raise Violation("no termination")
