"""Model check of the single-CTA GEMM kernel's K-block hand-off (CPU only).

Four roles share two barrier rings in ``csrc/bsgemm_kernel.cuh``:
- the TMA producer fills stage s and completes ``full[s]``; before refilling it,
  it waits for ``empty[s]``;
- two MMA issuers take the K-blocks in turn (issuer i the blocks of parity i).
  Each walks every stage and, for its own blocks, waits for ``full[s]`` and then
  for TMEM buffer b (``tmem_empty[b]``), issues the MMAs, commits
  ``tmem_full[b]`` after the block's last stage and ``empty[s]`` after each
  stage. At g = 64 a stage holds two K-blocks, one per issuer, so ``empty[s]``
  needs both issuers' commits; where the K tail leaves a stage without its
  second half, issuer 1 commits without MMAs. At g = 256 a K-block spans two
  stages;
- the promotion warps wait for ``tmem_full[b]``, read the partial and arrive on
  ``tmem_empty[b]``.

Every wait is a parity wait: waiting for phase k passes when the barrier's
completed-phase count c has (c & 1) != (k & 1). That answer is only right when
c == k + 1. A barrier one phase behind (c == k - 1) or two ahead (c == k + 2)
gives the same answer, which is aliasing. The model runs the roles with these
barriers as counters. A commit completes once its issuer's earlier MMAs have
(each issuer's commits in order, the two issuers' in any order), and the TMA
completions come in any order. Random schedules are run over random work
lists: whole tiles, split-K pieces and stream-K ranges, with a partial last
K-block. The checks:
- no wait passes at a count other than k + 1, no arrival lands in another
  phase than the one it is meant for, and the roles never deadlock;
- no stage is overwritten while MMAs read it or before they have used it;
- no TMEM buffer is rewritten before the promotion has read it;
- no MMA reads a stage before its copy landed, and no promotion reads an
  unfinished partial.
The stage and buffer counts are those the kernel derives from the tile width
and operand layout. Planted protocol mistakes show the model catches each
kind of fault.
"""
import random

import pytest

BK = 128                       # K bytes per stage
BUDGET = 227 * 1024 - 1024 - 512
EPI_STAGING = 8 * 32 * 128     # per-warp TMA-store staging of the data-parallel tiles


def stages(bnq: int, q_mn: bool, tma_store: bool = False) -> int:
    """Pipeline stages beside the epilogue staging: 32 KB for data-parallel
    tiles (tma_store), the BF16 [bnq][128] tile for swap-AB tiles."""
    q_rows = 128 if (q_mn and bnq < 128) else bnq
    staging = EPI_STAGING if tma_store else bnq * 128 * 2
    return min(8, (BUDGET - staging) // (BM_BYTES + q_rows * BK))


BM_BYTES = 128 * BK


def bufs(bnq: int) -> int:
    return 2 if bnq >= 256 else 4 if bnq >= 128 else 8


def work_list(rng, gran, K):
    """K-block ranges [kb0, kb1) of a CTA's work items, as the scheduler hands
    them out: whole tiles, split pieces and stream-K ranges (at g = 64 they start
    on even K-blocks, a unit being one 128-deep stage)."""
    Kb = -(-K // gran)
    items = []
    for _ in range(rng.randint(1, 4)):
        kind = rng.choice(("tile", "piece"))
        if kind == "tile" or Kb == 1:
            items.append((0, Kb))
        else:
            a, b = sorted(rng.sample(range(Kb + 1), 2))
            if gran == 64:
                a -= a & 1
                b = b + (b & 1) if b < Kb else Kb
                b = min(b, Kb)
                if a == b:
                    continue
            items.append((a, b))
    return items or [(0, Kb)]


class Bar:
    __slots__ = ("c",)

    def __init__(self):
        self.c = 0

    def passes(self, k):
        return (self.c & 1) != (k & 1)


class CountBar(Bar):
    """A barrier whose phase completes after `need` arrivals; an arrival meant
    for another phase than the current one is an error."""
    __slots__ = ("need", "got")

    def __init__(self, need):
        super().__init__()
        self.need, self.got = need, 0

    def add(self, phase, errors, what):
        if phase != self.c:
            errors.append(f"{what}: arrival for phase {phase} landed during phase {self.c}")
            return
        self.got += 1
        if self.got == self.need:
            self.c += 1
            self.got = 0


def programs(gran, K, items, S, mutation=None):
    """The producer's stage slots and each issuer's steps, as the kernel runs
    them. A step: (slot, wait_full, wait_block, mma, commit_block, commit_slot);
    wait_block / commit_block name the K-block whose TMEM buffer is claimed /
    committed, or None. Issuer x % 2 takes K-block x."""
    shared = (gran != BK or S % 2 == 1) and mutation != "skip_foreign_stage_wait"
    by_kb = mutation == "issuer_by_kb"
    nst = -(-K // BK)
    nslots = 0
    steps = ([], [])
    x = 0
    for kb0, kb1 in items:
        if gran >= BK:
            st0, st1 = kb0 * (gran // BK), kb1 * (gran // BK)
        else:
            st0, st1 = kb0 // 2, (kb1 + 1) // 2
        nslots += min(st1, nst) - st0
    slot = 0
    for kb0, kb1 in items:
        for kb in range(kb0, kb1):
            owner = (kb if by_kb else x) & 1
            if gran >= BK:
                for j in range(gran // BK):
                    k0 = kb * gran + j * BK
                    if k0 >= K:
                        break
                    last = j == gran // BK - 1 or k0 + BK >= K
                    steps[owner].append((slot, True, x if j == 0 else None, True, x if last else None, slot))
                    if shared:
                        steps[1 - owner].append((slot, True, None, False, None, slot))
                    slot += 1
            else:
                k0 = kb * gran
                t0 = kb & 1
                last_in_stage = t0 == 1 or k0 + gran >= K
                steps[owner].append((slot, True, x, True, x, slot))
                if t0 == 0 and last_in_stage and mutation != "tail_no_release":
                    steps[1 - owner].append((slot, True, None, False, None, slot))
                if last_in_stage:
                    slot += 1
            x += 1
    assert slot == nslots
    return nslots, steps, x


def simulate(S, B, gran, K, items, rng, mutation=None):
    shared = (gran != BK or S % 2 == 1) and mutation != "skip_foreign_stage_wait"
    stage_users = 1 if (mutation == "one_stage_user" or not shared) else 2
    full = [Bar() for _ in range(S)]
    empty = [CountBar(stage_users) for _ in range(S)]
    tfull = [Bar() for _ in range(B)]
    tempty = [Bar() for _ in range(B)]
    errors = []

    def check(bar, k, what):
        if bar.c != k + 1:
            errors.append(f"{what}: waited for phase {k}, count was {bar.c}")

    nslots, steps, nblocks = programs(gran, K, items, S, mutation)
    readers = [0] * nslots          # MMA groups that read each slot
    for prog in steps:
        for st in prog:
            if st[3]:
                readers[st[0]] += 1
    reads_done = [0] * nslots       # ... of which completed

    p_it = 0                        # producer: stage slots filled
    landing = []                    # TMA copies in flight (slots)
    landed = set()
    m_i = [0, 0]                    # each issuer: next step
    m_sub = [0, 0]                  # 0 = before its waits, 1 = full passed
    inflight = ([], [])             # each issuer's commits not yet complete, in issue order
    promo = 0
    blocks_done = set()
    slow = {r for r in ("prod", "land", "mma0", "mma1", "done0", "done1", "promo") if rng.random() < 0.3}
    guard = 0
    def running():
        return (promo < nblocks or p_it < nslots or landing or inflight[0] or inflight[1] or
                m_i != [len(steps[0]), len(steps[1])])

    while running() and not errors:
        guard += 1
        if guard > 300000:
            errors.append("no progress")
            break
        acts = []
        if p_it < nslots:
            k = p_it // S - (0 if mutation == "producer_phase" else 1)
            if k < 0 or empty[p_it % S].passes(k):
                acts.append(("prod",))
        if landing:
            acts.append(("land",))
        for i in (0, 1):
            if m_i[i] < len(steps[i]):
                slot, wf, wb, _, _, _ = steps[i][m_i[i]]
                if m_sub[i] == 0 and wf:
                    if full[slot % S].passes(slot // S):
                        acts.append(("m_full", i))
                else:
                    ok = True
                    if wb is not None and mutation != "skip_tmem_wait":
                        k = wb // B - (0 if mutation == "tmem_phase" else 1)
                        ok = k < 0 or tempty[wb % B].passes(k)
                    if ok:
                        acts.append(("m_issue", i))
            if inflight[i]:
                acts.append(("m_done", i))
        k = promo // B - (1 if mutation == "promo_phase" else 0)
        if promo < nblocks and (k < 0 or tfull[promo % B].passes(k)):
            acts.append(("promo",))
        if not acts:
            errors.append(f"deadlock: producer {p_it}/{nslots}, issuers {m_i}, promotion {promo}/{nblocks}")
            break

        def role(a):
            return {"m_full": f"mma{a[-1]}", "m_issue": f"mma{a[-1]}", "m_done": f"done{a[-1]}"}.get(a[0], a[0])
        a = rng.choices(acts, [0.03 if role(x) in slow else 1.0 for x in acts])[0]
        if a[0] == "prod":
            if p_it // S - 1 >= 0 and mutation is None:
                check(empty[p_it % S], p_it // S - 1, f"producer slot {p_it}")
            old = p_it - S
            if old >= 0 and reads_done[old] < readers[old]:
                errors.append(f"producer slot {p_it}: stage {p_it % S} overwritten while slot {old} is read")
            landing.append(p_it)
            p_it += 1
        elif a[0] == "land":
            slot = landing.pop(rng.randrange(len(landing)))
            landed.add(slot)
            full[slot % S].c += 1
        elif a[0] == "m_full":
            i = a[1]
            slot = steps[i][m_i[i]][0]
            check(full[slot % S], slot // S, f"issuer {i} step {m_i[i]} (full)")
            m_sub[i] = 1
        elif a[0] == "m_issue":
            i = a[1]
            slot, wf, wb, mma, cb, cs = steps[i][m_i[i]]
            if wb is not None:
                if wb // B - 1 >= 0 and mutation is None:
                    check(tempty[wb % B], wb // B - 1, f"issuer {i} step {m_i[i]} (tmem_empty)")
                if promo < wb - B + 1:
                    errors.append(f"issuer {i}: buffer {wb % B} rewritten before block {wb - B} was promoted")
            if mma and slot not in landed:
                errors.append(f"issuer {i}: stage slot {slot} read before its copy landed")
            if mutation == "early_release" and cs is not None and mma:
                empty[cs % S].add(cs // S, errors, f"issuer {i} early release, slot {cs}")
                cs = None
            inflight[i].append((slot if mma else None, cb, cs))
            m_i[i] += 1
            m_sub[i] = 0
        elif a[0] == "m_done":
            i = a[1]
            rs, cb, cs = inflight[i].pop(0)
            if rs is not None:
                reads_done[rs] += 1
            if cb is not None:
                tfull[cb % B].c += 1
                blocks_done.add(cb)
            if cs is not None:
                empty[cs % S].add(cs // S, errors, f"issuer {i} commit, slot {cs}")
        else:
            if mutation is None:
                check(tfull[promo % B], promo // B, f"promotion block {promo}")
            if promo not in blocks_done:
                errors.append(f"promotion block {promo}: read an unfinished partial")
            tempty[promo % B].c += 1
            promo += 1
    if not errors and (m_i != [len(steps[0]), len(steps[1])] or p_it != nslots):
        errors.append("roles finished out of step")
    return errors


# (tile width, MN-major Q, TMA-store staging): swap-AB tiles (16..128 wide) keep
# every stage, data-parallel tiles (128, 256) give 32 KB to the epilogue staging
CONFIGS = ([(bnq, q_mn, False) for bnq in (16, 32, 64, 128) for q_mn in (False, True)] +
           [(bnq, q_mn, True) for bnq in (128, 256) for q_mn in (False, True)])


def test_odd_ring_shares_its_stages():
    """The grouped 128-wide tiles have no staging and 7 stages, an odd ring: at
    g = 128 both issuers then wait for and release every stage."""
    S = min(8, BUDGET // (BM_BYTES + 128 * BK))
    assert S == 7
    rng = random.Random(7)
    for _ in range(80):
        K = rng.choice([BK, 3 * BK, 9 * BK + 64, 17 * BK])
        items = work_list(rng, 128, K)
        errors = simulate(S, bufs(128), 128, K, items, rng)
        assert not errors, (S, K, items, errors[0])


@pytest.mark.parametrize("gran", [64, 128, 256])
@pytest.mark.parametrize("bnq,q_mn,tma_store", CONFIGS)
def test_handoff_never_aliases_or_deadlocks(bnq, q_mn, tma_store, gran):
    S, B = stages(bnq, q_mn, tma_store), bufs(bnq)
    rng = random.Random(1000 * bnq + 10 * gran + q_mn + 5 * tma_store)
    for _ in range(60):
        K = rng.choice([BK, 2 * BK, 3 * BK, 5 * BK + 16, 7 * BK, 9 * BK + 64, 17 * BK])
        items = work_list(rng, gran, K)
        errors = simulate(S, B, gran, K, items, rng)
        assert not errors, (S, B, gran, K, items, errors[0])


def test_stage_counts_match_the_kernel_budget():
    """The 256-wide data-parallel tile keeps 4 stages beside its 32 KB of
    epilogue staging; the 128-wide one 6; swap-AB 128 keeps 6 beside its 32 KB
    BF16 tile; the narrow swap tiles 8."""
    assert stages(256, False, True) == 4 and stages(256, True, True) == 4
    assert stages(128, False, True) == 6
    assert stages(128, False, False) == 6 and stages(64, False, False) == 8
    assert stages(16, False, False) == 8 and stages(16, True, False) == 6   # MN-major Q: 128-wide atoms


MUTATIONS = [
    "producer_phase",   # the producer waits for the stage's current phase, not the previous one
    "tmem_phase",       # an issuer waits for the buffer's current phase
    "skip_tmem_wait",   # an issuer does not wait for the promotion to free the buffer
    "early_release",    # the stage is released when the MMAs are issued, not when they finish
    "promo_phase",      # the promotion waits for the previous phase of tmem_full
    "one_stage_user",   # g != 128: a stage is released by one issuer's commit, not both
    "tail_no_release",  # g = 64: the other issuer does not release a stage the K tail left half empty
    "issuer_by_kb",     # the issuer is picked by the K-block's parity within its work item
    "skip_foreign_stage_wait",  # g != 128: an issuer skips the stages of the other's blocks
]

# (tile width, MN-major Q, g) where each mistake can show: the issuer and
# stage-sharing mistakes need g != 128, and a buffer that changes owner
# aliases soonest with two buffers
MUTATION_CONFIGS = {
    "one_stage_user": ((256, False, 64), (128, False, 256)),
    "tail_no_release": ((256, False, 64), (16, True, 64)),
    "issuer_by_kb": ((256, False, 64),),
    "skip_foreign_stage_wait": ((128, False, 256), (256, False, 64)),
}


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_model_catches_planted_protocol_mistakes(mutation):
    """Each planted mistake is caught: as a deadlock, a wait passing at the
    wrong phase, or a stage or buffer used out of turn."""
    rng = random.Random(sum(map(ord, mutation)))
    for bnq, q_mn, gran in MUTATION_CONFIGS.get(mutation, ((256, False, 128), (128, True, 64), (64, False, 256))):
        S, B = stages(bnq, q_mn, bnq >= 128), bufs(bnq)
        caught = False
        for _ in range(300):
            K = rng.choice([5 * BK, 9 * BK, 17 * BK, 9 * BK + 64])
            items = work_list(rng, gran, K)
            if simulate(S, B, gran, K, items, rng, mutation):
                caught = True
                break
        assert caught, (mutation, bnq, q_mn, gran)


# ---------------------------------------------------------------- CTA pairs
# ``csrc/bsgemm_pair.cuh``: both CTAs' producers wait their own empty[s] and
# load their halves of stage s; both copies complete on the even CTA's full[s],
# whose phase also needs the even producer's arrive (with the byte count). The
# even CTA's two MMA issuers follow the single-CTA kernel's rules (issuer x % 2
# takes K-block x; stages shared where they change hands) and commit to both
# CTAs' tmem_full[b] and empty[s]. Each CTA's promotion warps wait their own
# tmem_full[b] and arrive on the even CTA's tmem_empty[b], whose phase needs
# both CTAs' arrivals.
PAIR_STAGES = min(8, (BUDGET - EPI_STAGING) // (2 * 128 * BK))   # 32 KB per stage beside the staging: 6
PAIR_BUFS = 2


class PhaseBar:
    """A barrier whose phase completes when every expected contribution of that
    phase has arrived; a contribution meant for another phase is an error."""
    __slots__ = ("c", "need", "got")

    def __init__(self, need):
        self.c, self.need, self.got = 0, set(need), set()

    def passes(self, k):
        return (self.c & 1) != (k & 1)

    def add(self, who, phase, errors, what):
        if phase != self.c:
            errors.append(f"{what}: contribution for phase {phase} arrived during phase {self.c}")
            return
        self.got.add(who)
        if self.got >= self.need:
            self.c += 1
            self.got = set()


def simulate_pair(gran, K, tiles, rng, mutation=None):
    S, B = PAIR_STAGES, PAIR_BUFS
    errors = []

    def check(bar, k, what):
        if bar.c != k + 1:
            errors.append(f"{what}: waited for phase {k}, count was {bar.c}")

    Kb = -(-K // gran)
    items = [(0, Kb)] * tiles
    nslots, steps, nblocks = programs(gran, K, items, S)
    shared = gran != BK or S % 2 == 1
    full = [PhaseBar({"arrive", "land0", "land1"}) for _ in range(S)]
    empty = [[CountBar(2 if shared else 1) for _ in range(S)] for _ in range(2)]
    tfull = [[Bar() for _ in range(B)] for _ in range(2)]
    tempty = [PhaseBar({0, 1} if mutation != "tmem_empty_one_cta" else {0}) for _ in range(B)]
    readers = [0] * nslots
    for prog in steps:
        for st in prog:
            if st[3]:
                readers[st[0]] += 1
    reads_done = [0] * nslots

    p_it = [0, 0]
    landing = []
    landed = [set(), set()]
    m_i = [0, 0]
    m_sub = [0, 0]
    inflight = ([], [])
    promo = [0, 0]
    blocks_done = set()
    slow = {r for r in ("prod0", "prod1", "land", "mma0", "mma1", "done0", "done1", "promo0", "promo1")
            if rng.random() < 0.3}

    def running():
        return (min(promo) < nblocks or p_it != [nslots, nslots] or landing or inflight[0] or inflight[1]
                or m_i != [len(steps[0]), len(steps[1])])

    guard = 0
    while running() and not errors:
        guard += 1
        if guard > 400000:
            errors.append("no progress")
            break
        acts = []
        for r in (0, 1):
            if p_it[r] < nslots:
                it = p_it[r]
                k = it // S - 1
                if k < 0 or (r == 1 and mutation == "odd_skips_stage_wait") or empty[r][it % S].passes(k):
                    acts.append(("prod", r))
        if landing:
            acts.append(("land",))
        for i in (0, 1):
            if m_i[i] < len(steps[i]):
                slot, wf, wb, _, _, _ = steps[i][m_i[i]]
                if m_sub[i] == 0 and wf:
                    if full[slot % S].passes(slot // S):
                        acts.append(("m_full", i))
                elif wb is None or wb // B - 1 < 0 or tempty[wb % B].passes(wb // B - 1):
                    acts.append(("m_issue", i))
            if inflight[i]:
                acts.append(("m_done", i))
        for r in (0, 1):
            if promo[r] < nblocks and tfull[r][promo[r] % B].passes(promo[r] // B):
                acts.append(("promo", r))
        if not acts:
            errors.append(f"deadlock: producers {p_it}/{nslots}, issuers {m_i}, promotion {promo}")
            break

        def role(a):
            return {"prod": f"prod{a[-1]}", "promo": f"promo{a[-1]}", "m_full": f"mma{a[-1]}",
                    "m_issue": f"mma{a[-1]}", "m_done": f"done{a[-1]}"}.get(a[0], a[0])
        a = rng.choices(acts, [0.03 if role(x) in slow else 1.0 for x in acts])[0]
        if a[0] == "prod":
            r = a[1]
            it = p_it[r]
            old = it - S
            if old >= 0 and reads_done[old] < readers[old]:
                errors.append(f"producer {r} slot {it}: stage {it % S} overwritten while slot {old} is read")
            if r == 0:
                full[it % S].add("arrive", it // S, errors, f"even producer slot {it}")
            landing.append((r, it))
            p_it[r] += 1
        elif a[0] == "land":
            r, it = landing.pop(rng.randrange(len(landing)))
            landed[r].add(it)
            full[it % S].add(f"land{r}", it // S, errors, f"copy of CTA {r} slot {it}")
        elif a[0] == "m_full":
            i = a[1]
            slot = steps[i][m_i[i]][0]
            check(full[slot % S], slot // S, f"issuer {i} step {m_i[i]} (full)")
            m_sub[i] = 1
        elif a[0] == "m_issue":
            i = a[1]
            slot, wf, wb, mma, cb, cs = steps[i][m_i[i]]
            if wb is not None:
                if wb // B - 1 >= 0:
                    check(tempty[wb % B], wb // B - 1, f"issuer {i} step {m_i[i]} (tmem_empty)")
                if min(promo) < wb - B + 1:
                    errors.append(f"issuer {i}: buffer {wb % B} rewritten before block {wb - B} "
                                  f"was promoted in both CTAs")
            if mma and (slot not in landed[0] or slot not in landed[1]):
                errors.append(f"issuer {i}: stage slot {slot} read before both copies landed")
            if mutation == "early_release" and cs is not None and mma:
                for r in (0, 1):
                    empty[r][cs % S].add(cs // S, errors, f"issuer {i} early release, slot {cs}")
                cs = None
            inflight[i].append((slot if mma else None, cb, cs))
            m_i[i] += 1
            m_sub[i] = 0
        elif a[0] == "m_done":
            i = a[1]
            rs, cb, cs = inflight[i].pop(0)
            if rs is not None:
                reads_done[rs] += 1
            if cb is not None:
                for r in ((0,) if mutation == "tmem_full_even_only" else (0, 1)):
                    tfull[r][cb % B].c += 1
                blocks_done.add(cb)
            if cs is not None:
                for r in (0, 1):
                    empty[r][cs % S].add(cs // S, errors, f"issuer {i} commit to CTA {r}, slot {cs}")
        else:
            r = a[1]
            blk = promo[r]
            check(tfull[r][blk % B], blk // B, f"promotion of CTA {r}, block {blk}")
            if blk not in blocks_done:
                errors.append(f"promotion of CTA {r}, block {blk}: read an unfinished partial")
            if mutation == "tmem_empty_one_cta" and r == 1:
                pass            # the planted mistake: the odd CTA's arrival is not counted
            else:
                tempty[blk % B].add(r, blk // B, errors, f"promotion of CTA {r}, block {blk}")
            promo[r] += 1
    return errors


@pytest.mark.parametrize("gran", [64, 128, 256])
def test_pair_handoff_never_aliases_or_deadlocks(gran):
    rng = random.Random(77 + gran)
    for _ in range(150):
        K = rng.choice([BK, 2 * BK, 3 * BK, 5 * BK + 16, 9 * BK + 64, 17 * BK])
        errors = simulate_pair(gran, K, rng.randint(1, 3), rng)
        assert not errors, (gran, K, errors[0])


PAIR_MUTATIONS = ["odd_skips_stage_wait", "tmem_full_even_only", "tmem_empty_one_cta", "early_release"]


@pytest.mark.parametrize("mutation", PAIR_MUTATIONS)
def test_pair_model_catches_planted_mistakes(mutation):
    rng = random.Random(len(mutation))
    for gran in (64, 128, 256):
        caught = any(simulate_pair(gran, rng.choice([9 * BK, 17 * BK]), rng.randint(1, 3), rng, mutation)
                     for _ in range(300))
        assert caught, (mutation, gran)
