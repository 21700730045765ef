"""Randomised models of the barrier protocols of the persistent forward kernel, the
persistent dq/dk/dv kernel, the dbias kernel and the pair-weighted averaging GEMM kernel
(pba_fwd.cuh, pba_bwd.cuh, pba_pwa.cuh): every role (TMA producer, MMA
issuers, softmax / element-wise warps, epilogue warpgroup) is a generator that waits on
mbarrier phases exactly as the kernel does; TMA copies and MMAs complete asynchronously in a
random order (MMAs of one issuer in issue order).  The models check that the protocol never
deadlocks, that every parity wait is exact (never two phases behind or one ahead), and that
no buffer (K/V/Q/bias stages, TMEM S/P/O, P/dS tiles, dK/dV and dQ accumulators) is
overwritten while a reader still needs it.  Test infrastructure only."""
import random


class Bar:
    def __init__(self, name, count):
        self.name, self.count = name, count
        self.arr, self.tx, self.ph = 0, 0, 0   # ph = completed phases

    def _check(self):
        if self.arr == self.count and self.tx == 0:
            self.arr = 0
            self.ph += 1

    def arrive(self, n=1):
        self.arr += n
        assert self.arr <= self.count, (self.name, "too many arrivals")
        self._check()

    def arrive_tx(self, nbytes):
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0
        self._check()

    def test(self, n):
        # waiting for completion of phase number n (parity n & 1)
        assert n <= self.ph + 1, (self.name, "waiting for a phase more than one ahead", n, self.ph)
        assert self.ph <= n + 1, (self.name, "parity alias: barrier two phases past the wait", n, self.ph)
        return self.ph == n + 1



class FwdSim:
    def __init__(self, nJ, nbs, KVS, BS, seed, row_mask=False, plant=None):
        self.rng = random.Random(seed)
        self.plant = plant
        self.nJ, self.nbs, self.KVS, self.BS = nJ, nbs, KVS, BS
        self.row_mask = row_mask
        self.items = len(nbs)
        # global step list: (item, j, s)
        self.steps = [(n, j, s) for n, nb in enumerate(nbs) for j in range(nJ) for s in range(nb)]
        self.K = len(self.steps)
        self.tiles = [(n, j) for n in range(self.items) for j in range(nJ)]
        B = Bar
        self.q_full, self.q_empty = B("q_full", 1), B("q_empty", 1)
        self.k_full = [B("k_full%d" % i, 1) for i in range(KVS)]
        self.k_empty = [B("k_empty%d" % i, 1) for i in range(KVS)]
        self.v_full = [B("v_full%d" % i, 1) for i in range(KVS)]
        self.v_empty = [B("v_empty%d" % i, 1) for i in range(KVS)]
        self.bias_full = [B("bias_full%d" % i, 1) for i in range(BS)]
        self.bias_ready = [B("bias_ready%d" % i, 1) for i in range(BS)]
        self.bias_empty = [B("bias_empty%d" % i, 1) for i in range(BS)]
        self.s_full, self.s_free = B("s_full", 1), B("s_free", 1)
        self.p_full, self.p_free = B("p_full", 1), B("p_free", 1)
        self.ofinal = B("ofinal", 1)
        self.tma, self.mq_qk, self.mq_pv = [], [], []
        self.q_item = None; self.q_readers = 0
        self.k_stage = [None] * KVS; self.k_readers = [0] * KVS
        self.v_stage = [None] * KVS; self.v_readers = [0] * KVS
        self.words = [None] * KVS; self.words_readers = [0] * KVS
        self.bias_tile = [None] * BS; self.bias_state = ["free"] * BS; self.bias_left = [0] * BS
        self.S_step = None; self.S_reading = False; self.S_pend = 0
        self.P_step = None; self.P_pend = 0
        self.O_item = {}       # slot -> item whose products it holds
        self.O_pend = {}       # slot -> PVs in flight
        self.O_reading = set()
        self.done_items = []

    def step_async(self):
        ch = []
        if self.tma: ch.append("tma")
        if self.mq_qk: ch.append("qk")
        if self.mq_pv: ch.append("pv")
        if not ch: return
        c = self.rng.choice(ch)
        if c == "tma":
            bar, n, fn = self.tma.pop(self.rng.randrange(len(self.tma)))
            fn(); bar.complete_tx(n)
        else:
            q = self.mq_qk if c == "qk" else self.mq_pv
            kind, x = q.pop(0)
            if kind == "mma": x()
            else: x.arrive()

    def producer(self):
        KVS, BS = self.KVS, self.BS
        kg = 0; jg = 0
        def load_bias(jg, tile):
            bs = jg % BS
            if jg >= BS:
                while not self.bias_empty[bs].test(jg // BS - 1): yield
            assert self.bias_state[bs] in ("free", "folded") and self.bias_left[bs] == 0
            self.bias_state[bs] = "loading"; self.bias_tile[bs] = tile
            self.bias_full[bs].arrive_tx(1)
            self.tma.append((self.bias_full[bs], 1, lambda bs=bs: self.bias_state.__setitem__(bs, "landed")))
            yield
        def load_k(k):
            st, use = k % KVS, k // KVS
            if use >= 1:
                while not self.k_empty[st].test(use - 1): yield
            assert self.k_readers[st] == 0
            self.k_stage[st] = None
            self.k_full[st].arrive_tx(1)
            self.tma.append((self.k_full[st], 1, lambda st=st, k=k: self.k_stage.__setitem__(st, k)))
            yield
        def load_v(k):
            st, use = k % KVS, k // KVS
            if use >= 1:
                while not self.v_empty[st].test(use - 1): yield
            assert self.v_readers[st] == 0 and self.words_readers[st] == 0
            self.v_stage[st] = None; self.words[st] = k
            self.v_full[st].arrive_tx(1)
            self.tma.append((self.v_full[st], 1, lambda st=st, k=k: self.v_stage.__setitem__(st, k)))
            yield
        for n, nb in enumerate(self.nbs):
            Kn = self.nJ * nb
            k0 = kg
            yield from load_bias(jg, (n, 0))
            yield from load_k(k0)
            # the item's Q tiles: the previous item's Q K^T products must be done
            if n >= 1 and self.plant != "no_q_empty_wait":
                while not self.q_empty.test(n - 1): yield
            assert self.q_readers == 0, "Q refilled while a Q K^T reads it"
            self.q_item = None
            self.q_full.arrive_tx(1)
            self.tma.append((self.q_full, 1, lambda n=n: setattr(self, "q_item", n)))
            yield
            for kl in range(Kn):
                if kl + 1 < Kn: yield from load_k(k0 + kl + 1)
                yield from load_v(k0 + kl)
                if kl + 1 < Kn and (kl + 1) % nb == 0:
                    yield from load_bias(jg + (kl + 1) // nb, (n, (kl + 1) // nb))
            kg += Kn; jg += self.nJ

    def fold(self):
        for jg, tile in enumerate(self.tiles):
            bs = jg % self.BS
            while not self.bias_full[bs].test(jg // self.BS): yield
            assert self.bias_state[bs] == "landed" and self.bias_tile[bs] == tile
            self.bias_state[bs] = "folded"; self.bias_left[bs] = self.nbs[tile[0]]
            yield
            self.bias_ready[bs].arrive()

    def issuer_qk(self):
        kg = 0
        for n, nb in enumerate(self.nbs):
            Kn = self.nJ * nb
            while not self.q_full.test(n): yield
            for kl in range(Kn):
                k = kg + kl; st = k % self.KVS
                if k > 0:
                    while not self.s_free.test(k - 1): yield
                while not self.k_full[st].test(k // self.KVS): yield
                assert self.k_stage[st] == k and self.q_item == n
                self.q_readers += 1; self.k_readers[st] += 1; self.S_pend += 1
                def ex(st=st, k=k, n=n):
                    assert not self.S_reading
                    assert self.k_stage[st] == k and self.q_item == n
                    self.q_readers -= 1; self.k_readers[st] -= 1; self.S_pend -= 1
                    self.S_step = k
                self.mq_qk.append(("mma", ex))
                self.mq_qk.append(("commit", self.s_full))
                self.mq_qk.append(("commit", self.k_empty[st]))
                if kl == Kn - 1:
                    self.mq_qk.append(("commit", self.q_empty))
                yield
            kg += Kn

    def issuer_pv(self):
        kg = 0
        for n, nb in enumerate(self.nbs):
            Kn = self.nJ * nb
            for kl in range(Kn):
                k = kg + kl; st = k % self.KVS; s = kl % nb
                while not self.p_full.test(k): yield
                while not self.v_full[st].test(k // self.KVS): yield
                assert self.v_stage[st] == k
                if kl < nb:   # first tile: the slot starts over
                    assert s not in self.O_reading, "O overwritten while the epilogue reads it"
                    self.O_item[s] = n
                assert self.O_item[s] == n
                self.v_readers[st] += 1; self.P_pend += 1; self.O_pend[s] = self.O_pend.get(s, 0) + 1
                def ex(st=st, k=k, s=s, n=n):
                    assert self.P_step == k and self.v_stage[st] == k and self.O_item[s] == n
                    assert s not in self.O_reading
                    self.v_readers[st] -= 1; self.P_pend -= 1; self.O_pend[s] -= 1
                self.mq_pv.append(("mma", ex))
                self.mq_pv.append(("commit", self.p_free))
                self.mq_pv.append(("commit", self.v_empty[st]))
                yield
            self.mq_pv.append(("commit", self.ofinal))
            kg += Kn

    def softmax(self):
        kg = 0; jg = 0
        for n, nb in enumerate(self.nbs):
            for j in range(self.nJ):
                bs = (jg + j) % self.BS
                for s in range(nb):
                    k = kg + j * nb + s; st = k % self.KVS
                    while not self.s_full.test(k): yield
                    if s == 0:
                        while not self.bias_ready[bs].test((jg + j) // self.BS): yield
                    if self.row_mask:
                        while not self.v_full[st].test(k // self.KVS): yield
                        assert self.words[st] == k
                        self.words_readers[st] += 1
                    assert self.S_step == k and self.S_pend == 0
                    self.S_reading = True
                    yield
                    self.S_reading = False
                    self.s_free.arrive()
                    assert self.bias_tile[bs] == (n, j) and self.bias_state[bs] == "folded"
                    yield
                    self.bias_left[bs] -= 1
                    if s == nb - 1:
                        assert self.bias_left[bs] == 0
                        self.bias_empty[bs].arrive()
                    if k > 0:
                        while not self.p_free.test(k - 1): yield
                    assert self.P_pend == 0
                    assert self.O_pend.get(s, 0) == 0
                    self.P_step = k
                    yield
                    if self.row_mask:
                        assert self.words[st] == k
                        self.words_readers[st] -= 1
                    self.p_full.arrive()
            # epilogue of item n
            while not self.ofinal.test(n): yield
            assert all(self.O_pend.get(s, 0) == 0 for s in range(nb))
            assert all(self.O_item.get(s) == n for s in range(nb))
            self.O_reading = set(range(nb))
            yield
            self.O_reading = set()
            self.done_items.append(n)
            kg += self.nJ * nb; jg += self.nJ

    def run(self):
        live = {"prod": self.producer(), "fold": self.fold(), "qk": self.issuer_qk(),
                "pv": self.issuer_pv(), "smx": self.softmax()}
        idle = 0
        while live or self.tma or self.mq_qk or self.mq_pv:
            opts = list(live) + (["async"] * 2 if (self.tma or self.mq_qk or self.mq_pv) else [])
            c = self.rng.choice(opts)
            if c == "async":
                self.step_async(); idle = 0; continue
            try: next(live[c])
            except StopIteration: del live[c]
            idle += 1
            if idle > 200000: raise RuntimeError("deadlock: live=%s" % list(live))
        assert self.done_items == list(range(self.items))



class BwdSim:
    """The persistent dq/dk/dv kernel (pba_bwd.cuh): a producer (K/V per item; Q, dOa and row
    statistics per step; a bias tile per step), one element-wise role (S/dP -> P/dS), the
    dQ / dK-dV epilogue warpgroup, and three MMA issuers, each in issue order: one for the
    dV products, one for the dK products, and one that issues S/dP of step t and then the
    dQ products of step t - 1."""

    def __init__(self, M, nI, QS, BS, KVB, DKB, seed, plant=None):
        self.rng = random.Random(seed)
        self.plant = plant
        self.M, self.QS, self.BS, self.KVB, self.DKB = M, QS, BS, KVB, DKB
        self.nis = nI if isinstance(nI, list) else [nI] * M
        self.steps = [(m, i) for m in range(M) for i in range(self.nis[m])]
        self.T = len(self.steps)
        B = Bar
        self.kv_full = [B("kv_full%d" % x, 1) for x in range(KVB)]
        self.kv_empty = [B("kv_empty%d" % x, 1) for x in range(KVB)]          # dQ issuer
        self.q_full = [B("q_full%d" % x, 1) for x in range(QS)]
        self.q_empty = [B("q_empty%d" % x, 3) for x in range(QS)]             # dV, dK commits + EW
        self.bias_full = [B("bias_full%d" % x, 1) for x in range(BS)]
        self.bias_empty = [B("bias_empty%d" % x, 1) for x in range(BS)]
        self.sd_full, self.sd_free = B("sd_full", 1), B("sd_free", 1)
        self.ps_full, self.ps_free = B("ps_full", 1), B("ps_free", 3)        # dV, dK, dQ commits
        self.dq_full = [B("dq_full%d" % x, 1) for x in range(2)]
        self.dq_free = [B("dq_free%d" % x, 1) for x in range(2)]
        self.dkv_full = [B("dkv_full%d" % x, 2) for x in range(DKB)]          # dV, dK commits
        self.dkv_free = [B("dkv_free%d" % x, 1) for x in range(DKB)]
        self.tma = []
        self.mq = {"dv": [], "dk": [], "sdq": []}   # one in-order queue per issuer
        # resource state
        self.kv_item = [None] * KVB; self.kv_readers = [0] * KVB; self.words_item = [None] * KVB
        self.q_step = [None] * QS; self.q_readers = [0] * QS
        self.bias_step = [None] * BS
        self.sd_step = None; self.sd_reading = False; self.sd_pending = 0
        self.ps_step = None; self.ps_pending = 0
        self.dq_step = [None, None]; self.dq_pending = [0, 0]
        self.acc_item = {"dv": [None] * DKB, "dk": [None] * DKB}
        self.acc_steps = {"dv": [0] * DKB, "dk": [0] * DKB}
        self.dkv_pending = [0] * DKB
        self.dkv_reading = [False] * DKB
        self.epi_done = []
        self.dq_flushed = []

    def step_async(self):
        opts = ["tma"] if self.tma else []
        opts += [k for k, q in self.mq.items() if q]
        if not opts: return
        c = self.rng.choice(opts)
        if c == "tma":
            bar, n, fn = self.tma.pop(self.rng.randrange(len(self.tma)))
            fn(); bar.complete_tx(n)
        else:
            kind, x = self.mq[c].pop(0)
            if kind == "mma": x()
            else: x.arrive()

    def producer(self):
        for m in range(self.M):
            x = m % self.KVB
            if m >= self.KVB:
                while not self.kv_empty[x].test(m // self.KVB - 1): yield
            assert self.kv_readers[x] == 0, "K/V stage refilled while MMAs read it"
            self.words_item[x] = m
            self.kv_item[x] = None
            self.kv_full[x].arrive_tx(1)
            self.tma.append((self.kv_full[x], 1, lambda x=x, m=m: self.kv_item.__setitem__(x, m)))
            yield
            for i in range(self.nis[m]):
                t = sum(self.nis[:m]) + i
                st, bs = t % self.QS, t % self.BS
                if t >= self.QS:
                    while not self.q_empty[st].test(t // self.QS - 1): yield
                assert self.q_readers[st] == 0, "Q/dOa stage refilled while it is read"
                self.q_step[st] = None
                self.q_full[st].arrive_tx(1)
                self.tma.append((self.q_full[st], 1, lambda st=st, t=t: self.q_step.__setitem__(st, t)))
                yield
                if t >= self.BS:
                    while not self.bias_empty[bs].test(t // self.BS - 1): yield
                self.bias_step[bs] = None
                self.bias_full[bs].arrive_tx(1)
                self.tma.append((self.bias_full[bs], 1, lambda bs=bs, t=t: self.bias_step.__setitem__(bs, t)))
                yield

    def issuer_sdq(self):
        # S/dP of step t, then the dQ products of step t - 1; with one K/V stage, a step that
        # starts an item issues the previous item's last dQ first (that dQ frees the stage)
        T = self.T
        for t in range(T + 1):
            dq_first = self.KVB == 1 and t < T and self.steps[t][1] == 0 and self.plant != "sdp_before_dq"
            for part in (("dq", "sdp") if dq_first else ("sdp", "dq")):
                if part == "sdp":
                    yield from self._sdp(t)
                else:
                    yield from self._dq(t)

    def _sdp(self, t):
        T = self.T
        if True:
            if t < T:
                m = self.steps[t][0]
                st, x = t % self.QS, m % self.KVB
                if self.steps[t][1] == 0:
                    while not self.kv_full[x].test(m // self.KVB): yield
                while not self.q_full[st].test(t // self.QS): yield
                if t > 0:
                    while not self.sd_free.test(t - 1): yield
                assert self.q_step[st] == t and self.kv_item[x] == m
                self.q_readers[st] += 1; self.kv_readers[x] += 1; self.sd_pending += 1
                def ex_s(t=t, st=st, x=x, m=m):
                    assert not self.sd_reading, "S/dP overwritten while the EW reads them"
                    assert self.q_step[st] == t and self.kv_item[x] == m
                    self.q_readers[st] -= 1; self.kv_readers[x] -= 1; self.sd_pending -= 1
                    self.sd_step = t
                self.mq["sdq"].append(("mma", ex_s))
                self.mq["sdq"].append(("commit", self.sd_full))
                yield

    def _dq(self, t):
        if True:
            if t >= 1:
                tq = t - 1
                m, i = self.steps[tq]
                x = m % self.KVB
                while not self.ps_full.test(tq): yield
                if tq >= 2:
                    while not self.dq_free[tq & 1].test((tq >> 1) - 1): yield
                assert self.ps_step == tq and self.kv_item[x] == m
                self.ps_pending += 1; self.kv_readers[x] += 1; self.dq_pending[tq & 1] += 1
                def ex_q(tq=tq, x=x, m=m):
                    assert self.ps_step == tq and self.kv_item[x] == m
                    self.ps_pending -= 1; self.kv_readers[x] -= 1; self.dq_pending[tq & 1] -= 1
                    self.dq_step[tq & 1] = tq
                q = self.mq["sdq"]
                q.append(("mma", ex_q))
                q.append(("commit", self.ps_free))
                q.append(("commit", self.dq_full[tq & 1]))
                if i == self.nis[m] - 1 and self.plant != "no_kv_empty_commit":
                    q.append(("commit", self.kv_empty[x]))
                yield

    def issuer_dkv(self, kind):
        T = self.T
        for t in range(T):
            (m, i), st = self.steps[t], t % self.QS
            d = m % self.DKB
            while not self.ps_full.test(t): yield
            if i == 0 and m >= self.DKB and self.plant != "no_dkv_free_wait":
                while not self.dkv_free[d].test(m // self.DKB - 1): yield
            assert self.ps_step == t and self.q_step[st] == t
            assert self.sd_step is not None and self.sd_step >= t, "products before S/dP of the step"
            if i == 0:
                assert not self.dkv_reading[d], "dK/dV accumulator reset while the epilogue reads it"
                self.acc_item[kind][d] = m; self.acc_steps[kind][d] = 0
            assert self.acc_item[kind][d] == m, "dK/dV buffer reused before its epilogue"
            self.ps_pending += 1; self.q_readers[st] += 1; self.dkv_pending[d] += 1
            def ex(t=t, st=st, d=d, m=m):
                assert self.ps_step == t and self.q_step[st] == t
                assert self.acc_item[kind][d] == m and not self.dkv_reading[d]
                self.ps_pending -= 1; self.q_readers[st] -= 1; self.dkv_pending[d] -= 1
                self.acc_steps[kind][d] += 1
            q = self.mq[kind]
            q.append(("mma", ex))
            q.append(("commit", self.ps_free))
            q.append(("commit", self.q_empty[st]))
            if i == self.nis[m] - 1:
                q.append(("commit", self.dkv_full[d]))
            yield

    def ew(self):
        T = self.T
        for t in range(T):
            (m, i), st, bs = self.steps[t], t % self.QS, t % self.BS
            if i == 0:
                while not self.kv_full[m % self.KVB].test(m // self.KVB): yield
                assert self.words_item[m % self.KVB] == m
            while not self.sd_full.test(t): yield
            while not self.q_full[st].test(t // self.QS): yield
            while not self.bias_full[bs].test(t // self.BS): yield
            assert self.sd_step == t and self.sd_pending == 0 and self.bias_step[bs] == t and self.q_step[st] == t
            self.sd_reading = True; self.q_readers[st] += 1   # row stats of the Q stage
            yield
            assert self.q_step[st] == t, "row stats changed under the element-wise warps"
            self.sd_reading = False; self.q_readers[st] -= 1
            self.sd_free.arrive(); self.bias_empty[bs].arrive(); self.q_empty[st].arrive()
            if t > 0 and self.plant != "no_ps_free_wait":
                while not self.ps_free.test(t - 1): yield
            assert self.ps_pending == 0, "P/dS overwritten while MMAs read them"
            self.ps_step = t
            yield
            self.ps_full.arrive()

    def epi(self):
        T = self.T
        for t in range(T):
            m, i = self.steps[t]
            while not self.dq_full[t & 1].test(t >> 1): yield
            assert self.dq_step[t & 1] == t and self.dq_pending[t & 1] == 0
            self.dq_flushed.append(t)
            yield
            self.dq_free[t & 1].arrive()
            if i == self.nis[m] - 1:
                d = m % self.DKB
                while not self.dkv_full[d].test(m // self.DKB): yield
                assert self.dkv_pending[d] == 0
                for kind in ("dv", "dk"):
                    assert self.acc_item[kind][d] == m and self.acc_steps[kind][d] == self.nis[m]
                self.epi_done.append(m)
                self.dkv_reading[d] = True
                yield
                assert all(self.acc_item[kind][d] == m for kind in ("dv", "dk")), "dK/dV changed under the epilogue"
                self.dkv_reading[d] = False
                self.dkv_free[d].arrive()

    def run(self):
        live = {"prod": self.producer(), "sdq": self.issuer_sdq(), "dv": self.issuer_dkv("dv"),
                "dk": self.issuer_dkv("dk"), "ew": self.ew(), "epi": self.epi()}
        idle = 0
        while live or self.tma or any(self.mq.values()):
            busy = self.tma or any(self.mq.values())
            opts = list(live) + (["async"] * 2 if busy else [])
            c = self.rng.choice(opts)
            if c == "async":
                self.step_async(); idle = 0; continue
            try: next(live[c])
            except StopIteration: del live[c]
            idle += 1
            if idle > 200000: raise RuntimeError("deadlock: live=%s" % list(live))
        assert self.epi_done == list(range(self.M)) and self.dq_flushed == list(range(self.T))


class DbiasSim:
    """The dbias kernel (pba_bwd.cuh): one producer fills NS stages (Q, dOa, K and V tiles, row
    statistics and mask words of one broadcast row each) after the bias tile; one MMA issuer
    computes S and dP of row n into TMEM buffer n & 1 and releases the stage by a commit; nwg
    element-wise warpgroups (a key range each, 128 arrivals each) read the TMEM buffer,
    the stage's row statistics and mask words, and release both."""

    def __init__(self, nb, NS, seed, plant=None, nwg=3):
        self.rng = random.Random(seed)
        self.plant = plant
        self.nb, self.NS, self.nwg = nb, NS, nwg
        B = Bar
        self.bias = B("bias", 1)
        self.full = [B("full%d" % x, 1) for x in range(NS)]
        # MMA commit + every element-wise thread
        self.empty = [B("empty%d" % x, 1 + 128 * nwg) for x in range(NS)]
        self.sd_full = [B("sd_full%d" % x, 1) for x in range(2)]
        self.sd_free = [B("sd_free%d" % x, 128 * nwg) for x in range(2)]
        self.tma, self.mq = [], []
        self.stage_row = [None] * NS; self.stage_readers = [0] * NS; self.mask_row = [None] * NS
        self.tm_row = [None, None]; self.tm_readers = [0, 0]; self.tm_pending = [0, 0]
        self.summed = [[] for _ in range(nwg)]

    def step_async(self):
        opts = (["tma"] if self.tma else []) + (["mma"] if self.mq else [])
        if not opts: return
        if self.rng.choice(opts) == "tma":
            bar, n, fn = self.tma.pop(self.rng.randrange(len(self.tma)))
            fn(); bar.complete_tx(n)
        else:
            kind, x = self.mq.pop(0)
            if kind == "mma": x()
            else: x.arrive()

    def producer(self):
        self.bias.arrive_tx(1)
        self.tma.append((self.bias, 1, lambda: None))
        yield
        for n in range(self.nb):
            st = n % self.NS
            if n >= self.NS and self.plant != "no_empty_wait":
                while not self.empty[st].test(n // self.NS - 1): yield
            assert self.stage_readers[st] == 0, "stage refilled while it is read"
            self.mask_row[st] = n          # plain shared stores, ordered by the arrive below
            self.stage_row[st] = None
            self.full[st].arrive_tx(1)
            self.tma.append((self.full[st], 1, lambda st=st, n=n: self.stage_row.__setitem__(st, n)))
            yield

    def issuer(self):
        for n in range(self.nb):
            st, x = n % self.NS, n & 1
            while not self.full[st].test(n // self.NS): yield
            if n >= 2 and self.plant != "no_sd_free_wait":
                while not self.sd_free[x].test((n >> 1) - 1): yield
            assert self.stage_row[st] == n
            self.stage_readers[st] += 1; self.tm_pending[x] += 1
            def ex(st=st, x=x, n=n):
                assert self.stage_row[st] == n, "stage changed under the MMA"
                assert self.tm_readers[x] == 0, "S/dP overwritten while the element-wise warps read them"
                self.stage_readers[st] -= 1; self.tm_pending[x] -= 1
                self.tm_row[x] = n
            self.mq.append(("mma", ex))
            self.mq.append(("commit", self.sd_full[x]))
            self.mq.append(("commit", self.empty[st]))
            yield

    def ew(self, e):
        while not self.bias.test(0): yield
        for n in range(self.nb):
            st, x = n % self.NS, n & 1
            while not self.sd_full[x].test(n >> 1): yield
            while not self.full[st].test(n // self.NS): yield
            assert self.tm_row[x] == n and self.tm_pending[x] == 0
            assert self.stage_row[st] == n and self.mask_row[st] == n
            self.tm_readers[x] += 1; self.stage_readers[st] += 1
            yield
            assert self.tm_row[x] == n and self.stage_row[st] == n and self.mask_row[st] == n, \
                "inputs changed under the element-wise warps"
            self.tm_readers[x] -= 1; self.stage_readers[st] -= 1
            self.summed[e].append(n)
            self.sd_free[x].arrive(128); self.empty[st].arrive(128)

    def run(self):
        live = {"prod": self.producer(), "mma": self.issuer()}
        for e in range(self.nwg):
            live["ew%d" % e] = self.ew(e)
        idle = 0
        while live or self.tma or self.mq:
            opts = list(live) + (["async"] * 2 if (self.tma or self.mq) else [])
            c = self.rng.choice(opts)
            if c == "async":
                self.step_async(); idle = 0; continue
            try: next(live[c])
            except StopIteration: del live[c]
            idle += 1
            if idle > 200000: raise RuntimeError("deadlock: live=%s" % list(live))
        assert self.summed == [list(range(self.nb))] * self.nwg


class PwaGemmSim:
    """The pair-weighted averaging GEMM and dW kernels (pba_pwa.cuh, one protocol): one producer
    fills NS stages (GEMM: a 64-deep block of w and the chunk's value tiles; dW: one row's dOa
    and V tiles) over the nK reduction stages; one MMA
    issuer accumulates every stage into one TMEM accumulator, releases each stage by a commit
    and signals the epilogue by a last commit; the epilogue reads the accumulator once."""

    def __init__(self, nK, NS, seed, plant=None):
        self.rng = random.Random(seed)
        self.plant = plant
        self.nK, self.NS = nK, NS
        self.full = [Bar("full%d" % x, 1) for x in range(NS)]
        self.empty = [Bar("empty%d" % x, 1) for x in range(NS)]
        self.done = Bar("done", 1)
        self.tma, self.mq = [], []
        self.stage = [None] * NS; self.readers = [0] * NS
        self.acc = []          # reduction stages added to the accumulator, in order
        self.read = None

    def step_async(self):
        opts = (["tma"] if self.tma else []) + (["mma"] if self.mq else [])
        if not opts: return
        if self.rng.choice(opts) == "tma":
            bar, n, fn = self.tma.pop(self.rng.randrange(len(self.tma)))
            fn(); bar.complete_tx(n)
        else:
            kind, x = self.mq.pop(0)
            if kind == "mma": x()
            else: x.arrive()

    def producer(self):
        for r in range(self.nK):
            st = r % self.NS
            if r >= self.NS and self.plant != "no_empty_wait":
                while not self.empty[st].test(r // self.NS - 1): yield
            assert self.readers[st] == 0, "stage refilled while the MMA reads it"
            self.stage[st] = None
            self.full[st].arrive_tx(1)
            self.tma.append((self.full[st], 1, lambda st=st, r=r: self.stage.__setitem__(st, r)))
            yield

    def issuer(self):
        for r in range(self.nK):
            st = r % self.NS
            while not self.full[st].test(r // self.NS): yield
            assert self.stage[st] == r
            self.readers[st] += 1
            def ex(st=st, r=r):
                assert self.stage[st] == r, "stage changed under the MMA"
                self.readers[st] -= 1
                self.acc.append(r)
            self.mq.append(("mma", ex))
            self.mq.append(("commit", self.empty[st]))
            yield
        if self.plant != "early_done":
            self.mq.append(("commit", self.done))
        else:
            self.mq.insert(0, ("commit", self.done))

    def epilogue(self):
        while not self.done.test(0): yield
        self.read = list(self.acc)

    def run(self):
        live = {"prod": self.producer(), "mma": self.issuer(), "epi": self.epilogue()}
        idle = 0
        while live or self.tma or self.mq:
            opts = list(live) + (["async"] * 2 if (self.tma or self.mq) else [])
            c = self.rng.choice(opts)
            if c == "async":
                self.step_async(); idle = 0; continue
            try: next(live[c])
            except StopIteration: del live[c]
            idle += 1
            if idle > 200000: raise RuntimeError("deadlock: live=%s" % list(live))
        assert self.read == list(range(self.nK)), "the epilogue read an unfinished accumulator"
