"""Randomised model of the CTA protocol of attn_fwd_pp_kernel<D, MIXED>
(csrc/attn_pp.cuh), test infrastructure for the CPU suite.

The kernel's 20 warps are modelled as cooperating generators: the producer
(Q tiles, the NVFP4 K/V ring, the bf16 tile queue and the raw K, V and Q
streams), the Q K^T issuer, the P V issuer and the 16 softmax warps (two
query tiles x two key halves x four TMEM lane quadrants).  Every wait, arrive
and commit of the kernel appears here in the kernel's order; the tensor pipe
executes issued operations in order at random times and copies land at random
times.  A run fails on mbarrier parity aliasing (a wait more than one phase
ahead or behind), on deadlock, and on a data hazard on any buffer (ring
stages, Q, S, P, the bf16 tiles and P buffer, O rescaled against P V,
epilogue staging, scale factors).
"""
import random
import sys


class Err(Exception):
    pass


class Bar:
    def __init__(s, name, count):
        s.name, s.count, s.pend, s.done = name, count, 0, 0

    def arrive(s):
        s.pend += 1
        if s.pend == s.count:
            s.done += 1
            s.pend = 0


def test(bar, n, who):
    """Non-blocking test of phase number n (parity semantics, aliasing check)."""
    # a parity wait is only valid when the barrier is in phase n or has just
    # completed it: further behind or ahead, the parity names another phase
    if bar.done >= n + 2:
        raise Err(f"{who}: aliasing on {bar.name}: wants phase {n}, completed {bar.done}")
    if bar.done < n:
        raise Err(f"{who}: waits ahead on {bar.name}: wants phase {n}, completed {bar.done}")
    return bar.done >= n + 1


class Sim:
    def __init__(s, seed, B=1, H=2, T=5, causal=True, G=2, cta=0, mixed=True, pmask=0.3):
        s.rng = random.Random(seed)
        s.B, s.H, s.T, s.causal, s.G, s.cta, s.mixed = B, H, T, causal, G, cta, mixed
        s.S = 3 if mixed else 4
        s.QB = 1 if mixed else 2
        s.mask = {}
        for bh in range(B * H):
            for t in range(T):
                for u in range(T):
                    s.mask[(bh, t, u)] = 1 if (mixed and s.rng.random() < pmask) else 0
        nbh = B * H
        s.nitems = nbh * ((T + 1) // 2)
        s.nrounds = (s.nitems + G - 1) // G
        # barriers
        Bn = Bar
        s.q_full = [Bn(f"q_full{i}", 1) for i in range(s.QB)]
        s.q_empty = [Bn(f"q_empty{i}", 1) for i in range(s.QB)]
        s.kv_full = [Bn(f"kv_full{i}", 1) for i in range(s.S)]
        s.kv_empty = [Bn(f"kv_empty{i}", 2) for i in range(s.S)]
        s.s_full = [Bn(f"s_full{i}", 1) for i in range(2)]
        s.s_free = [Bn(f"s_free{i}", 8) for i in range(2)]
        s.p_full = [Bn(f"p_full{i}", 8) for i in range(2)]
        s.o_done = [Bn(f"o_done{i}", 1) for i in range(2)]
        s.xbar = [[Bn(f"xbar{x}{q}", 2) for q in range(4)] for x in range(2)]
        s.kb_full, s.kb_empty = Bn("kb_full", 1), Bn("kb_empty", 1)
        s.vb_full, s.vb_empty = Bn("vb_full", 1), Bn("vb_empty", 1)
        s.qb_full, s.qb_empty = Bn("qb_full", 1), Bn("qb_empty", 1)
        s.pb_grant = [Bn("pb_grant0", 1), Bn("pb_grant1", 1)]
        s.abort = False
        # async
        s.tma = []    # [(bar, [(buf, key, tag)])]
        s.pipe = []   # in-order tensor ops
        # buffer state
        s.buf = {}    # buffer key -> tag
        s.xch = {}    # (slot, x, h, r) -> (value tag)
        s.executed = set()   # executed reader ops: ('qk', it, x, u), ('pv', it, x, u), ('cpk', it, u), ('cpv', it, u)
        s.o_state = [None, None]   # per tile: (it, u_last_accumulated)
        s.o_rescaled = {}          # (x, it, u, q, h) rescale done
        s.epi_done = {}            # (x, it) -> set of (q, h) done with the epilogue
        s.staging = {}             # (x, q, h) -> busy
        s.pv_count = [0, 0]        # PV executed per tile
        s.last_pv_exec = None
        s.bf16_pv_exec = 0
        s.done_roles = 0
        s.log = []

    # -------------------------------------------------------------- schedule
    def item_index(s, j):
        c = (s.G - 1 - s.cta) if (j & 1) else s.cta
        i = j * s.G + c
        return i if i < s.nitems else -1

    def item(s, i):
        nbh = s.B * s.H
        npairs = (s.T + 1) // 2
        r = i // nbh
        bh = i - r * nbh
        pair = npairs - 1 - r if s.causal else r
        tA, tB = 2 * pair, 2 * pair + 1
        hasB = tB < s.T
        nuA = min(tA + 1, s.T) if s.causal else s.T
        nuB = (min(tB + 1, s.T) if s.causal else s.T) if hasB else 0
        return dict(bh=bh, pair=pair, nuA=nuA, nuB=nuB, nu=max(nuA, nuB), hasB=hasB)

    def items(s):
        out = []
        for j in range(s.nrounds):
            i = s.item_index(j)
            if i >= 0:
                out.append(s.item(i))
        return out

    def bf16(s, I, x, u):
        if not s.mixed:
            return False
        if u >= (I['nuB'] if x else I['nuA']):
            return False
        return s.mask[(I['bh'], 2 * I['pair'] + x, u)] == 1

    # -------------------------------------------------------------- helpers
    def wait(s, bar, n, who):
        while True:
            if s.abort:
                raise Err(f"{who}: abort")
            if test(bar, n, who):
                return
            yield f"{who} wait {bar.name}#{n}"

    def commit(s, bar):
        s.pipe.append(('commit', bar))

    # -------------------------------------------------------------- producer
    def producer(s):
        its = s.items()
        # streams as lists of ops (each op: (cond_fn, action_fn)); polled in turn
        # Q stream
        qops = []
        for it, I in enumerate(its):
            qops.append(('q', it, I))
        rops = []
        rg = 0
        for it, I in enumerate(its):
            for u in range(I['nu']):
                rops.append(('r', it, I, u, rg))
                rg += 1
        ktiles = [(it, I, u) for it, I in enumerate(its) for u in range(I['nu'])
                  if s.bf16(I, 0, u) or s.bf16(I, 1, u)]
        # ring index of each tile: a bf16 stream may use a tile only once the ring
        # has published it (loaded it)
        ridx = {}
        g = 0
        for it, I in enumerate(its):
            for u in range(I['nu']):
                ridx[(it, u)] = g
                g += 1
        events = [(it, I, u, x) for it, I in enumerate(its) for u in range(I['nu']) for x in (0, 1)
                  if s.bf16(I, x, u)]
        qi = ri = ki = vi = ei = 0
        nrl = 0  # raw-Q reloads issued
        qhold = None
        while qi < len(qops) or ri < len(rops) or ki < len(ktiles) or vi < len(ktiles) or ei < len(events):
            prog = False
            if qi < len(qops):
                _, it, I = qops[qi]
                qs = it % s.QB
                if it < s.QB or test(s.q_empty[qs], it // s.QB - 1, 'prod q'):
                    # hazard: every QK reading the old content executed
                    if it >= s.QB:
                        old = it - s.QB
                        Io = its[old]
                        for x in range(2 if Io['hasB'] else 1):
                            for u in range(Io['nuB'] if x else Io['nuA']):
                                if not s.bf16(Io, x, u) and ('qk', old, x, u) not in s.executed:
                                    raise Err(f"Q buffer {qs} reloaded before QK{(old, x, u)} executed")
                    s.tma.append((s.q_full[qs], [(('q', qs), ('Q', it))]))
                    qi += 1
                    prog = True
            if ri < len(rops):
                _, it, I, u, g = rops[ri]
                st = g % s.S
                if g < s.S or test(s.kv_empty[st], g // s.S - 1, 'prod ring'):
                    if g >= s.S:
                        ot = s.buf.get(('stage', st))
                        if ot is not None:
                            oit, ou = ot[1], ot[2]
                            Io = its[oit]
                            need = [('cpv', oit, ou)]
                            for x in range(2):
                                if ou < (Io['nuB'] if x else Io['nuA']) and not s.bf16(Io, x, ou):
                                    need += [('qk', oit, x, ou), ('pv', oit, x, ou)]
                            for n_ in need:
                                if n_ not in s.executed:
                                    raise Err(f"stage {st} reloaded before {n_} executed")
                    s.tma.append((s.kv_full[st], [(('stage', st), ('KV', it, u))]))
                    ri += 1
                    prog = True
            if s.mixed:
                if ki < len(ktiles) and ridx[(ktiles[ki][0], ktiles[ki][2])] < ri and (ki == 0 or test(s.kb_empty, ki - 1, 'prod kb')):
                    it, I, u = ktiles[ki]
                    if ki > 0:
                        oit, oI, ou = ktiles[ki - 1]
                        for x in range(2):
                            if s.bf16(oI, x, ou) and ('qk', oit, x, ou) not in s.executed:
                                raise Err("kb reloaded early")
                    s.tma.append((s.kb_full, [(('kb',), ('K', it, u))]))
                    ki += 1
                    prog = True
                if vi < len(ktiles) and ridx[(ktiles[vi][0], ktiles[vi][2])] < ri and (vi == 0 or test(s.vb_empty, vi - 1, 'prod vb')):
                    it, I, u = ktiles[vi]
                    if vi > 0:
                        oit, oI, ou = ktiles[vi - 1]
                        for x in range(2):
                            if s.bf16(oI, x, ou) and ('pv', oit, x, ou) not in s.executed:
                                raise Err("vb reloaded early")
                    s.tma.append((s.vb_full, [(('vb',), ('V', it, u))]))
                    vi += 1
                    prog = True
                if ei < len(events) and ridx[(events[ei][0], events[ei][2])] < ri:
                    it, I, u, x = events[ei]
                    want = (it, x)
                    go = want == qhold
                    if not go and (nrl == 0 or test(s.qb_empty, nrl - 1, 'prod qb')):
                        for e in events[:ei]:
                            if ('qk', e[0], e[3], e[2]) not in s.executed:
                                raise Err("qb reloaded early")
                        s.tma.append((s.qb_full, [(('qb',), ('QB', it, x))]))
                        qhold = want
                        nrl += 1
                        go = True
                    if go:
                        ei += 1
                        prog = True
            if s.abort:
                raise Err("producer abort")
            yield "producer poll" if not prog else "producer issued"
        # drain: each TMA barrier's last issued phase
        for qs in range(s.QB):
            c = len([1 for op in qops if op[1] % s.QB == qs])
            if c:
                yield from s.wait(s.q_full[qs], c - 1, 'drain q')
        for st in range(s.S):
            c = len([1 for op in rops if op[4] % s.S == st])
            if c:
                yield from s.wait(s.kv_full[st], c - 1, 'drain kv')
        if s.mixed:
            if ki:
                yield from s.wait(s.kb_full, ki - 1, 'drain kb')
            if vi:
                yield from s.wait(s.vb_full, vi - 1, 'drain vb')
            if nrl:
                yield from s.wait(s.qb_full, nrl - 1, 'drain qb')
        s.done_roles += 1

    # -------------------------------------------------------------- issuers
    def issuer_qk(s):
        its = s.items()
        g0 = 0
        kv_waited = -1
        last = None  # (x, idx) of the previous S reader
        nS = [0, 0]
        bk = bq = 0
        qhold = None
        S = s.S
        nreload = 0
        for it, I in enumerate(its):
            qs = it % s.QB
            yield from s.wait(s.q_full[qs], it // s.QB, 'qk q_full')
            for x in range(2 if I['hasB'] else 1):
                s.pipe.append(('cpq', qs, x, it))
            for u in range(I['nu']):
                gt = g0 + u
                st = gt % S
                yield from s.wait(s.kv_full[st], gt // S, 'qk kv_full')
                s.pipe.append(('cpk', st, it, u))
                sfk_done = True
                for x in (0, 1):
                    if u >= (I['nuB'] if x else I['nuA']):
                        continue
                    if last is not None:
                        yield from s.wait(s.s_free[last[0]], last[1], 'qk s_free')
                    bA, bB = s.bf16(I, 0, u), s.bf16(I, 1, u)
                    if (bB if x else bA):
                        if x == 0 or not bA:
                            yield from s.wait(s.kb_full, bk, 'qk kb_full')
                        want = (it, x)
                        if want != qhold:
                            if qhold is not None:
                                s.commit(s.qb_empty)  # the raw Q buffer may be reloaded after the Q K^T so far
                            yield from s.wait(s.qb_full, bq, 'qk qb_full')
                            bq += 1
                            qhold = want
                        s.pipe.append(('qkb', it, x, u))
                        if x == 1 or not bB:
                            s.commit(s.kb_empty)
                            bk += 1
                    else:
                        if not sfk_done:
                            s.pipe.append(('cpk', st, it, u))
                            sfk_done = True
                        s.pipe.append(('qkf', qs, st, it, x, u))
                    s.commit(s.s_full[x])
                    last = (x, nS[x])
                    nS[x] += 1
                s.commit(s.kv_empty[st])
            s.commit(s.q_empty[qs])
            g0 += I['nu']
        s.done_roles += 1

    def issuer_pv(s):
        its = s.items()
        g0 = 0
        nP = [0, 0]
        bv = 0
        S = s.S
        first = True  # no bf16 block seen yet
        for it, I in enumerate(its):
            for u in range(I['nu']):
                gt = g0 + u
                st = gt % S
                yield from s.wait(s.kv_full[st], gt // S, 'pv kv_full')
                s.pipe.append(('cpv', st, it, u))
                for x in (0, 1):
                    if u >= (I['nuB'] if x else I['nuA']):
                        continue
                    bA, bB = s.bf16(I, 0, u), s.bf16(I, 1, u)
                    if (bB if x else bA):
                        # hand the bf16 P buffer to this block once the P V issued so far complete
                        if first:
                            s.pb_grant[x].arrive()
                            first = False
                        else:
                            s.commit(s.pb_grant[x])
                    yield from s.wait(s.p_full[x], nP[x], 'pv p_full')
                    if (bB if x else bA):
                        if x == 0 or not bA:
                            yield from s.wait(s.vb_full, bv, 'pv vb_full')
                        s.pipe.append(('pvb', it, x, u))
                        if x == 1 or not bB:
                            s.commit(s.vb_empty)
                            bv += 1
                    else:
                        s.pipe.append(('pvf', st, it, x, u))
                    s.commit(s.o_done[x])
                    nP[x] += 1
                s.commit(s.kv_empty[st])
            g0 += I['nu']
        s.done_roles += 1

    # -------------------------------------------------------------- softmax
    def softmax(s, x, h, q):
        who = f"sm{x}{h}{q}"
        its = s.items()
        k = 0
        nb = 0  # this tile's bf16 blocks so far
        xp = 0

        def exchange(val):
            nonlocal xp
            s.xch[(xp & 1, x, h, q)] = val
            s.xbar[x][q].arrive()
            yield from s.wait(s.xbar[x][q], xp, who + ' xbar')
            other = s.xch.get((xp & 1, x, h ^ 1, q))
            if other != val:
                raise Err(f"{who}: exchange read {other}, expected {val}")
            xp += 1

        for it, I in enumerate(its):
            nux = I['nuB'] if x else I['nuA']
            for u in range(nux):
                bA, bB = s.bf16(I, 0, u), s.bf16(I, 1, u)
                bfx = bB if x else bA
                yield from s.wait(s.s_full[x], k, who + ' s_full')
                tag = s.buf.get(('S',))
                if tag != ('S', it, x, u):
                    raise Err(f"{who}: read S {tag}, expected {(it, x, u)}")
                if not bfx:
                    s.s_reads[(it, x, u)] = s.s_reads.get((it, x, u), 0) + 1
                    s.s_free[x].arrive()
                yield "sm compute"
                yield from exchange(('max', it, x, u))
                yield "sm compute"
                if k > 0:
                    yield from s.wait(s.o_done[x], k - 1, who + ' o_done')
                # O must hold this tile's accumulation through u-1, with no PV pending
                if u > 0:
                    if s.o_state[x] != (it, u - 1):
                        raise Err(f"{who}: rescale with O state {s.o_state[x]}, expected {(it, u - 1)}")
                if bfx:
                    yield from s.wait(s.pb_grant[x], nb, who + ' pb_grant')
                    nb += 1
                    if s.pb_pending:
                        raise Err(f"{who}: writes bf16 P while a bf16 PV is pending")
                    # S is re-read while P is written, then released
                    tag = s.buf.get(('S',))
                    if tag != ('S', it, x, u):
                        raise Err(f"{who}: re-read S {tag}, expected {(it, x, u)}")
                    s.buf[('pb', h, q)] = ('PB', it, x, u)
                    s.s_reads[(it, x, u)] = s.s_reads.get((it, x, u), 0) + 1
                    s.s_free[x].arrive()
                    if u == 0 and h == 1:
                        # l <- 0: both halves of quadrant q finished the previous epilogue
                        pass
                else:
                    if s.pf_pending[x]:
                        raise Err(f"{who}: writes NVFP4 P while its PV is pending")
                    if s.staging.get((x, q, 0)) or s.staging.get((x, q, 1)):
                        raise Err(f"{who}: writes P over an epilogue staging area")
                    s.buf[('p', x, h, q)] = ('P', it, x, u)
                s.o_rescaled[(x, it, u, h, q)] = True
                s.p_full[x].arrive()
                k += 1
            if nux == 0:
                continue
            yield from s.wait(s.o_done[x], k - 1, who + ' o_done(epi)')
            if s.o_state[x] != (it, nux - 1):
                raise Err(f"{who}: epilogue sees O {s.o_state[x]}, expected {(it, nux - 1)}")
            if s.mixed:
                yield from exchange(('lb', it, x))
            s.staging[(x, q, h)] = True
            yield "epilogue"
            yield "epilogue"
            if s.o_state[x] != (it, nux - 1):
                raise Err(f"{who}: O changed during the epilogue")
            s.staging[(x, q, h)] = False
            s.epi_done.setdefault((x, it), set()).add((h, q))
        s.done_roles += 1

    # -------------------------------------------------------------- async engine
    def step_async(s):
        opts = []
        if s.tma:
            opts.append('tma')
        if s.pipe:
            opts.append('pipe')
        if not opts:
            return False
        what = s.rng.choice(opts)
        if what == 'tma':
            idx = s.rng.randrange(len(s.tma))
            bar, writes = s.tma.pop(idx)
            for key, tag in writes:
                s.buf[key] = tag
            bar.arrive()
            return True
        op = s.pipe.pop(0)
        kind = op[0]
        its = s.items_cache
        if kind == 'commit':
            op[1].arrive()
        elif kind == 'cpq':
            _, qs, x, it = op
            if s.buf.get(('q', qs)) != ('Q', it):
                raise Err(f"cpq reads Q buffer {s.buf.get(('q', qs))}, expected item {it}")
            s.buf[('sfq', x)] = ('SFQ', it)
        elif kind == 'cpk':
            _, st, it, u = op
            if s.buf.get(('stage', st)) != ('KV', it, u):
                raise Err(f"cpk reads stage {st}: {s.buf.get(('stage', st))}, expected {(it, u)}")
            s.buf[('sfk',)] = ('SFK', it, u)
            s.executed.add(('cpk', it, u))
        elif kind == 'cpv':
            _, st, it, u = op
            if s.buf.get(('stage', st)) != ('KV', it, u):
                raise Err(f"cpv reads stage {st}: {s.buf.get(('stage', st))}, expected {(it, u)}")
            s.buf[('sfv',)] = ('SFV', it, u)
            s.executed.add(('cpv', it, u))
        elif kind in ('qkf', 'qkb'):
            if kind == 'qkf':
                _, qs, st, it, x, u = op
                if s.buf.get(('q', qs)) != ('Q', it):
                    raise Err(f"QK reads Q {s.buf.get(('q', qs))}, expected {it}")
                if s.buf.get(('stage', st)) != ('KV', it, u):
                    raise Err(f"QK reads stage {s.buf.get(('stage', st))}, expected {(it, u)}")
                if s.buf.get(('sfk',)) != ('SFK', it, u) or s.buf.get(('sfq', x)) != ('SFQ', it):
                    raise Err("QK scale factors stale")
            else:
                _, it, x, u = op
                if s.buf.get(('qb',)) != ('QB', it, x):
                    raise Err(f"bf16 QK reads qb {s.buf.get(('qb',))}, expected {(it, x)}")
                if s.buf.get(('kb',)) != ('K', it, u):
                    raise Err(f"bf16 QK reads kb {s.buf.get(('kb',))}, expected {(it, u)}")
            # S overwrite: the previous S fully read
            prev = s.buf.get(('S',))
            if prev is not None and s.s_reads.get(prev[1:], 0) != 8:
                raise Err(f"QK overwrites S {prev} read by {s.s_reads.get(prev[1:], 0)}/8 warps")
            s.buf[('S',)] = ('S', it, x, u)
            s.executed.add(('qk', it, x, u))
        elif kind in ('pvf', 'pvb'):
            if kind == 'pvf':
                _, st, it, x, u = op
                if s.buf.get(('stage', st)) != ('KV', it, u) or s.buf.get(('sfv',)) != ('SFV', it, u):
                    raise Err(f"PV reads stage/SFV stale {s.buf.get(('stage', st))} {s.buf.get(('sfv',))} {(it, u)}")
                for h in range(2):
                    for q in range(4):
                        if s.buf.get(('p', x, h, q)) != ('P', it, x, u):
                            raise Err(f"PV reads P part {(h, q)} = {s.buf.get(('p', x, h, q))}, expected {(it, x, u)}")
            else:
                _, it, x, u = op
                if s.buf.get(('vb',)) != ('V', it, u):
                    raise Err(f"bf16 PV reads vb {s.buf.get(('vb',))}, expected {(it, u)}")
                for h in range(2):
                    for q in range(4):
                        if s.buf.get(('pb', h, q)) != ('PB', it, x, u):
                            raise Err(f"bf16 PV reads pb part {s.buf.get(('pb', h, q))}, expected {(it, x, u)}")
            # accumulator state
            if u == 0:
                if it > 0:
                    # the last item of this tile role must have been fully read out
                    prev_it = max((pi for (xx, pi) in s.epi_done if xx == x), default=None)
                    for pit in range(it):
                        I = s.items_cache[pit]
                        nux = I['nuB'] if x else I['nuA']
                        if nux > 0 and len(s.epi_done.get((x, pit), ())) != 8:
                            raise Err(f"PV({it},{x},0) overwrites O before item {pit}'s epilogue finished")
            else:
                if s.o_state[x] != (it, u - 1):
                    raise Err(f"PV({it},{x},{u}) accumulates onto O state {s.o_state[x]}")
                for h in range(2):
                    for q in range(4):
                        if not s.o_rescaled.get((x, it, u, h, q)):
                            raise Err(f"PV({it},{x},{u}) before the rescale of {(h, q)}")
            s.o_state[x] = (it, u)
            s.executed.add(('pv', it, x, u))
        else:
            raise Err(f"unknown op {op}")
        return True

    @property
    def pb_pending(s):
        return any(o[0] == 'pvb' for o in s.pipe)

    @property
    def pf_pending(s):
        return [any(o[0] == 'pvf' and o[3] == x for o in s.pipe) for x in range(2)]

    def run(s, max_steps=2_000_000):
        s.items_cache = s.items()
        s.s_reads = {}
        roles = [s.producer(), s.issuer_qk(), s.issuer_pv()] + [s.softmax(x, h, q) for x in range(2) for h in range(2) for q in range(4)]
        names = ['prod', 'iqk', 'ipv'] + [f'sm{x}{h}{q}' for x in range(2) for h in range(2) for q in range(4)]
        alive = list(range(len(roles)))
        last = {i: None for i in alive}
        stall = 0
        for step in range(max_steps):
            if not alive and not s.tma and not s.pipe:
                return step
            # choose between a role step and an async event
            if (s.tma or s.pipe) and (not alive or s.rng.random() < 0.35):
                s.step_async()
                stall = 0
                continue
            if not alive:
                continue
            i = s.rng.choice(alive)
            try:
                msg = next(roles[i])
            except StopIteration:
                alive.remove(i)
                stall = 0
                continue
            if msg is not None and ' wait ' in msg or msg == 'producer poll':
                stall += 1
            else:
                stall = 0
            if stall > 5000 and not s.tma and not s.pipe:
                raise Err(f"deadlock: alive={[names[a] for a in alive]} last={msg}")
        raise Err("step limit")


def main():
    n = int(sys.argv[1]) if len(sys.argv) > 1 else 300
    rng = random.Random(12345)
    for t in range(n):
        mixed = rng.random() < 0.7
        T = rng.randint(1, 7)
        H = rng.randint(1, 3)
        G = rng.randint(1, 4)
        cfg = dict(seed=t, B=1, H=H, T=T, causal=rng.random() < 0.6, G=G, cta=rng.randrange(G), mixed=mixed,
                   pmask=rng.choice([0.0, 0.1, 0.3, 0.7, 1.0]))
        sim = Sim(**cfg)
        try:
            steps = sim.run()
        except Err as e:
            print("FAIL", cfg, e)
            return 1
    print(f"{n} randomised runs: no deadlock, aliasing or hazard")
    return 0


if __name__ == "__main__":
    sys.exit(main())
