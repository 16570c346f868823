"""Model check of the single-CTA GEMM kernel's K-block hand-off (CPU only).

Three roles share two barrier rings in ``csrc/bsgemm_kernel.cuh``:
- the TMA producer fills stage s and completes ``full[s]``; before refilling it,
  it waits for ``empty[s]``;
- the MMA warp waits for ``full[s]`` and then for TMEM buffer b (``tmem_empty[b]``).
  It issues the K-block's MMAs and commits ``tmem_full[b]`` after the block's last
  stage and ``empty[s]`` after each stage. At g = 64 a stage holds two K-blocks;
  at g = 256 a K-block spans two stages;
- the promotion warps wait for ``tmem_full[b]``, read the partial and arrive on
  ``tmem_empty[b]``.

Every wait is a parity wait: waiting for phase k passes when the barrier's
completed-phase count c has (c & 1) != (k & 1). That answer is only right when
c == k + 1. A barrier one phase behind (c == k - 1) or two ahead (c == k + 2)
gives the same answer, which is aliasing. The model runs the three roles with
these barriers as counters. The MMA completions are asynchronous, in issue
order, and the TMA completions come in any order. Random schedules are run
over random work lists: whole tiles, split-K pieces and stream-K ranges, with
a partial last K-block. The checks:
- no wait passes at a count other than k + 1, and the roles never deadlock;
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


def simulate(S, B, gran, K, items, rng, mutation=None):
    full = [Bar() for _ in range(S)]
    empty = [Bar() for _ in range(S)]
    tfull = [Bar() for _ in range(B)]
    tempty = [Bar() for _ in range(B)]
    errors = []

    def check(bar, k, what):
        if bar.c != k + 1:
            errors.append(f"{what}: waited for phase {k}, count was {bar.c}")

    nst = -(-K // BK)

    # producer program: the stage slots it fills, in order
    prod = []
    for kb0, kb1 in items:
        if gran >= BK:
            st0, st1 = kb0 * (gran // BK), kb1 * (gran // BK)
        else:
            st0, st1 = kb0 // 2, (kb1 + 1) // 2
        prod += [None] * (min(st1, nst) - st0)

    # MMA program: a list of steps (wait_full, wait_tmem, commit_tmem_full, commit_empty)
    mma = []
    for kb0, kb1 in items:
        for kb in range(kb0, kb1):
            if gran >= BK:
                for j in range(gran // BK):
                    k0 = kb * gran + j * BK
                    if k0 >= K:
                        break
                    last = j == gran // BK - 1 or k0 + BK >= K
                    mma.append((True, j == 0, last, True))
            else:
                k0 = kb * gran
                t0 = kb & 1
                mma.append((t0 == 0, True, True, t0 == 1 or k0 + gran >= K))
    nblocks = sum(kb1 - kb0 for kb0, kb1 in items)

    p_it = 0                       # producer: stage slots filled
    landing = []                   # TMA copies in flight (stage indices)
    m_i = 0                        # MMA: next step
    m_st = 0                       # MMA: stage slots consumed
    m_blk = 0                      # MMA: K-blocks started
    m_sub = 0                      # MMA: 0 = before its waits, 1 = full passed
    inflight = []                  # MMA commits not yet complete, in issue order
    promo = 0
    reading = [0] * S              # MMA groups in flight that read each stage
    stage_done = 0                 # stage slots whose reads are complete
    blocks_done = 0                # K-blocks whose MMAs are complete
    landed = set()                 # stage slots whose copies landed
    # adversarial pacing: some roles run far slower than the others in this run
    slow = {r for r in ("prod", "land", "mma", "m_done", "promo") if rng.random() < 0.3}
    guard = 0
    while promo < nblocks and not errors:
        guard += 1
        if guard > 200000:
            errors.append("no progress")
            break
        acts = []
        if p_it < len(prod):
            k = p_it // S - (0 if mutation == "producer_phase" else 1)
            if k < 0 or empty[p_it % S].passes(k):
                acts.append("prod")
        if landing:
            acts.append("land")
        if m_i < len(mma):
            wf, wt, _, _ = mma[m_i]
            s = m_st % S
            if m_sub == 0 and wf:
                if full[s].passes(m_st // S):
                    acts.append("m_full")
            else:
                b, k = m_blk % B, m_blk // B - (0 if mutation == "tmem_phase" else 1)
                if not wt or k < 0 or mutation == "skip_tmem_wait" or tempty[b].passes(k):
                    acts.append("m_issue")
        if inflight:
            acts.append("m_done")
        b, k = promo % B, promo // B - (1 if mutation == "promo_phase" else 0)
        if k < 0 or tfull[b].passes(k):
            acts.append("promo")
        if not acts:
            errors.append(f"deadlock: producer {p_it}/{len(prod)}, mma {m_i}/{len(mma)}, promotion {promo}")
            break
        role = {"m_full": "mma", "m_issue": "mma"}
        weights = [0.03 if role.get(x, x) in slow else 1.0 for x in acts]
        a = rng.choices(acts, weights)[0]
        if a == "prod":
            if p_it // S - 1 >= 0 and mutation is None:
                check(empty[p_it % S], p_it // S - 1, f"producer slot {p_it}")
            if reading[p_it % S] or stage_done < p_it - S + 1:
                errors.append(f"producer slot {p_it}: stage {p_it % S} overwritten while in use")
            landing.append(p_it)
            p_it += 1
        elif a == "land":
            slot = landing.pop(rng.randrange(len(landing)))
            landed.add(slot)
            full[slot % S].c += 1
        elif a == "m_full":
            check(full[m_st % S], m_st // S, f"mma step {m_i} (full)")
            m_sub = 1
        elif a == "m_issue":
            wf, wt, ctf, cem = mma[m_i]
            if wt and m_blk // B - 1 >= 0 and mutation is None:
                check(tempty[m_blk % B], m_blk // B - 1, f"mma step {m_i} (tmem_empty)")
            if m_st not in landed:
                errors.append(f"mma step {m_i}: stage slot {m_st} read before its copy landed")
            if wt and promo < m_blk - B + 1:
                errors.append(f"mma step {m_i}: buffer {m_blk % B} rewritten before block "
                              f"{m_blk - B} was promoted")
            reading[m_st % S] += 1
            if mutation == "early_release" and cem:
                empty[m_st % S].c += 1
                stage_done += 1
                cem_late = False
            else:
                cem_late = cem
            inflight.append((m_blk % B if ctf else None, m_st % S if cem_late else None, m_st % S))
            if ctf:
                m_blk += 1
            if cem:
                m_st += 1
            m_i += 1
            m_sub = 0
        elif a == "m_done":
            tb, es, rs = inflight.pop(0)
            reading[rs] -= 1
            if tb is not None:
                tfull[tb].c += 1
                blocks_done += 1
            if es is not None:
                empty[es].c += 1
                stage_done += 1
        else:
            if mutation is None:
                check(tfull[promo % B], promo // B, f"promotion block {promo}")
            if blocks_done < promo + 1:
                errors.append(f"promotion block {promo}: read an unfinished partial")
            tempty[promo % B].c += 1
            promo += 1
    if not errors and (m_i != len(mma) or p_it != len(prod)):
        errors.append("roles finished out of step")
    return errors


# (tile width, MN-major Q, TMA-store staging): swap-AB tiles (16..128 wide) keep
# every stage, data-parallel tiles (128, 256) give 32 KB to the epilogue staging
CONFIGS = ([(bnq, q_mn, False) for bnq in (16, 32, 64, 128) for q_mn in (False, True)] +
           [(bnq, q_mn, True) for bnq in (128, 256) for q_mn in (False, True)])


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
    "tmem_phase",       # the MMA waits for the buffer's current phase
    "skip_tmem_wait",   # the MMA does not wait for the promotion to free the buffer
    "early_release",    # the stage is released when the MMAs are issued, not when they finish
    "promo_phase",      # the promotion waits for the previous phase of tmem_full
]


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_model_catches_planted_protocol_mistakes(mutation):
    """Each planted mistake is caught: as a deadlock, a wait passing at the
    wrong phase, or a stage or buffer used out of turn."""
    rng = random.Random(hash(mutation) & 0xFFFF)
    for bnq, q_mn, gran in ((256, False, 128), (128, True, 64), (64, False, 256)):
        S, B = stages(bnq, q_mn, bnq >= 128), bufs(bnq)
        caught = False
        for _ in range(300):
            K = rng.choice([5 * BK, 9 * BK, 17 * BK])
            items = work_list(rng, gran, K)
            if simulate(S, B, gran, K, items, rng, mutation):
                caught = True
                break
        assert caught, (mutation, bnq, q_mn, gran)


# ---------------------------------------------------------------- CTA pairs
# ``csrc/bsgemm_pair.cuh``: both CTAs' producers wait their own empty[s] and
# load their halves of stage s; both copies complete on the even CTA's full[s],
# whose phase also needs the even producer's arrive (with the byte count). The
# even CTA's MMA warp waits full[s] and its tmem_empty[b], issues the pair MMAs
# and commits to both CTAs' tmem_full[b] and empty[s]. Each CTA's promotion warps
# wait their own tmem_full[b] and arrive on the even CTA's tmem_empty[b], whose
# phase needs both CTAs' arrivals.
PAIR_STAGES = min(8, BUDGET // (2 * 128 * BK))   # 16 KB of A and 16 KB of B per stage: 7
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

    nst = -(-K // BK)
    Kb = -(-K // gran)
    items = [(0, Kb)] * tiles
    full = [PhaseBar({"arrive", "land0", "land1"}) for _ in range(S)]
    empty = [[Bar() for _ in range(S)] for _ in range(2)]
    tfull = [[Bar() for _ in range(B)] for _ in range(2)]
    tempty = [PhaseBar({0, 1} if mutation != "tmem_empty_one_cta" else {0}) for _ in range(B)]
    mma = []
    for kb0, kb1 in items:
        for kb in range(kb0, kb1):
            if gran >= BK:
                for j in range(gran // BK):
                    k0 = kb * gran + j * BK
                    if k0 >= K:
                        break
                    mma.append((True, j == 0, j == gran // BK - 1 or k0 + BK >= K, True))
            else:
                k0 = kb * gran
                mma.append(((kb & 1) == 0, True, True, (kb & 1) == 1 or k0 + gran >= K))
    nprod = nst * tiles
    nblocks = Kb * tiles

    p_it = [0, 0]
    landing = []
    landed = [set(), set()]
    m_i = m_st = m_blk = m_sub = 0
    inflight = []
    promo = [0, 0]
    reading = [0] * S
    stage_done = 0
    blocks_done = 0
    slow = {r for r in ("prod0", "prod1", "land", "mma", "m_done", "promo0", "promo1") if rng.random() < 0.3}
    guard = 0
    while min(promo) < nblocks and not errors:
        guard += 1
        if guard > 400000:
            errors.append("no progress")
            break
        acts = []
        for r in (0, 1):
            if p_it[r] < nprod:
                it = p_it[r]
                k = it // S - 1
                if k < 0 or (r == 1 and mutation == "odd_skips_stage_wait") or empty[r][it % S].passes(k):
                    acts.append(("prod", r))
        if landing:
            acts.append(("land",))
        if m_i < len(mma):
            wf, wt, _, _ = mma[m_i]
            if m_sub == 0 and wf:
                if full[m_st % S].passes(m_st // S):
                    acts.append(("m_full",))
            else:
                b, k = m_blk % B, m_blk // B - 1
                if not wt or k < 0 or tempty[b].passes(k):
                    acts.append(("m_issue",))
        if inflight:
            acts.append(("m_done",))
        for r in (0, 1):
            if promo[r] < nblocks and tfull[r][promo[r] % B].passes(promo[r] // B):
                acts.append(("promo", r))
        if not acts:
            errors.append(f"deadlock: producers {p_it}/{nprod}, mma {m_i}/{len(mma)}, promotion {promo}")
            break

        def role(a):
            return {"prod": f"prod{a[1] if len(a) > 1 else ''}", "promo": f"promo{a[1] if len(a) > 1 else ''}",
                    "m_full": "mma", "m_issue": "mma"}.get(a[0], a[0])
        a = rng.choices(acts, [0.03 if role(x) in slow else 1.0 for x in acts])[0]
        if a[0] == "prod":
            r = a[1]
            it = p_it[r]
            if (reading[it % S] or stage_done < it - S + 1):
                errors.append(f"producer {r} slot {it}: stage {it % S} overwritten while in use")
            if r == 0:
                full[it % S].add("arrive", it // S, errors, f"even producer slot {it}")
            landing.append((r, it))
            p_it[r] += 1
        elif a[0] == "land":
            r, it = landing.pop(rng.randrange(len(landing)))
            landed[r].add(it)
            full[it % S].add(f"land{r}", it // S, errors, f"copy of CTA {r} slot {it}")
        elif a[0] == "m_full":
            check(full[m_st % S], m_st // S, f"mma step {m_i} (full)")
            m_sub = 1
        elif a[0] == "m_issue":
            wf, wt, ctf, cem = mma[m_i]
            if wt and m_blk // B - 1 >= 0:
                check(tempty[m_blk % B], m_blk // B - 1, f"mma step {m_i} (tmem_empty)")
            if m_st not in landed[0] or m_st not in landed[1]:
                errors.append(f"mma step {m_i}: stage slot {m_st} read before both copies landed")
            if wt and min(promo) < m_blk - B + 1:
                errors.append(f"mma step {m_i}: buffer {m_blk % B} rewritten before block "
                              f"{m_blk - B} was promoted in both CTAs")
            reading[m_st % S] += 1
            if mutation == "early_release" and cem:
                for r in (0, 1):
                    empty[r][m_st % S].c += 1
                stage_done += 1
                cem = False
            inflight.append((m_blk % B if ctf else None, m_st % S if cem else None, m_st % S))
            if ctf:
                m_blk += 1
            if mma[m_i][3]:
                m_st += 1
            m_i += 1
            m_sub = 0
        elif a[0] == "m_done":
            tb, es, rs = inflight.pop(0)
            reading[rs] -= 1
            if tb is not None:
                for r in ((0,) if mutation == "tmem_full_even_only" else (0, 1)):
                    tfull[r][tb].c += 1
                blocks_done += 1
            if es is not None:
                for r in (0, 1):
                    empty[r][es].c += 1
                stage_done += 1
        else:
            r = a[1]
            blk = promo[r]
            check(tfull[r][blk % B], blk // B, f"promotion of CTA {r}, block {blk}")
            if blocks_done < blk + 1:
                errors.append(f"promotion of CTA {r}, block {blk}: read an unfinished partial")
            if mutation == "tmem_empty_one_cta" and r == 1:
                pass            # the planted mistake: the odd CTA's arrival is not counted
            else:
                tempty[blk % B].add(r, blk // B, errors, f"promotion of CTA {r}, block {blk}")
            promo[r] += 1
    if not errors and (m_i != len(mma) or p_it != [nprod, nprod]):
        errors.append("roles finished out of step")
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
