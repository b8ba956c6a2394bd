"""The mbarrier / TMA / tcgen05 hand-offs of the tensor-core prefill kernels, checked as models (CPU only).

Each model below transcribes, per warp role, the waits, arrivals, copies, tensor-core ops, commits and buffer
accesses of one CTA of a kernel in `trainable_block_sparse_v2_b200/csrc/`, in program order.  The model
checker in `pipeline_model.py` runs them under many random schedules (see its docstring for what it
reports).  Each model is run as written and with planted mistakes (a dropped wait, a dropped named barrier, a
single-buffered exchange); the planted mistakes must be reported, which pins the checker itself.
"""
import pytest

from pipeline_model import PipelineModel, ProtocolError

RING = 3


def drained(m: PipelineModel, name: str, ops, skip: bool = False):
    """an issuing role's ops, then its drain: a commit on a barrier of its own and the wait for it, after which
    none of its tensor-core ops is in flight (the kernels drain every issuer before the CTA frees its TMEM)"""
    m.bar(f"drain.{name}", 1)
    yield from ops
    if not skip:
        yield ("commit", f"drain.{name}")
        yield ("wait", f"drain.{name}", 0)


# --------------------------------------------------------------------------------------------------------------
# attn_tc_kernel (csrc/attn_tc.cu): 128-row tile, U union blocks in NP = ceil(U / 2) steps of 128 keys.
# Warp 0: Q once (shared memory, the A operand of every S MMA), then K per step (3-slot ring); warp 10: V per
# step (a VR-slot ring: 2 at d 128, 3 at d 64); warp 1: S(p) = Q K^T into S buffer p % 3, after PV(p - 3)
# completed; warp 11: O += P(v) V; warps 2-9: softmax, two per TMEM lane quarter, each on 64 keys, P written
# over the first 64 columns of its S buffer.  Warps 1 and 11 issue tensor-core ops independently: nothing
# orders one's ops after the other's except the mbarriers.
# --------------------------------------------------------------------------------------------------------------
NS = 3


def attn_tc_model(m: PipelineModel, U: int, rescale_steps=(), parts: int = 2, mistake: str = "", VR: int = 2):
    NP = (U + 1) // 2
    m.bar("q_full", 1)
    for i in range(RING):
        for n in ("k_full", "k_empty"):
            m.bar(f"{n}{i}", 1)
    for i in range(VR):
        for n in ("v_full", "v_empty"):
            m.bar(f"{n}{i}", 1)
    for i in range(NS):
        m.bar(f"s_full{i}", 1)
        m.bar(f"p_full{i}", 128 * parts)
        m.bar(f"o_done{i}", 1)
    rd = 8 // parts  # 16-column chunks of S read per part
    wr = 4 // parts  # 16-column chunks of P written per part

    def k_producer():
        yield ("arrive_tx", "q_full", 1, 1)
        yield ("tma", "q_full", 1, [("Q", "Q")])
        for p in range(NP):
            s, k = p % RING, p // RING
            if k >= 1 and mistake != "k producer skips k_empty":
                yield ("wait", f"k_empty{s}", k - 1)
            yield ("arrive_tx", f"k_full{s}", 1, 1)
            yield ("tma", f"k_full{s}", 1, [(f"K{s}", ("K", p))])
        # the producer's drain before the CTA ends: every copy it issued has landed
        yield ("wait", "q_full", 0)
        for s in range(min(RING, NP)):
            yield ("wait", f"k_full{s}", (NP - 1 - s) // RING)

    def v_producer():
        for p in range(NP):
            s, k = p % VR, p // VR
            if k >= 1 and mistake != "v producer skips v_empty":
                yield ("wait", f"v_empty{s}", k - 1)
            yield ("arrive_tx", f"v_full{s}", 1, 1)
            yield ("tma", f"v_full{s}", 1, [(f"V{s}", ("V", p))])
        for s in range(min(VR, NP)):
            yield ("wait", f"v_full{s}", (NP - 1 - s) // VR)

    def s_issuer():
        yield ("wait", "q_full", 0)
        for p in range(NP):
            s, sb = p % RING, p % NS
            if p >= NS and mistake != "S issuer skips o_done":
                yield ("wait", f"o_done{sb}", (p - NS) // NS)
            yield ("wait", f"k_full{s}", p // RING)
            yield ("mma", [("Q", "Q"), (f"K{s}", ("K", p))],
                   [(f"S{sb}.q{q}.c{c}", ("S", p)) for q in range(4) for c in range(8)], f"S{p}")
            yield ("commit", f"s_full{sb}")
            yield ("commit", f"k_empty{s}")

    def pv_issuer():
        for v in range(NP):
            pv, sv = v % NS, v % VR
            if mistake != "PV issuer skips p_full":
                yield ("wait", f"p_full{pv}", v // NS)
            yield ("wait", f"v_full{sv}", v // VR)
            reads = [(f"S{pv}.q{q}.c{c}", ("P", v)) for q in range(4) for c in range(4)]
            reads += [(f"V{sv}", ("V", v))]
            if v > 0:
                reads += [(f"O.q{q}.h{k}", ("O", v - 1)) for q in range(4) for k in range(parts)]
            yield ("mma", reads, [(f"O.q{q}.h{k}", ("O", v)) for q in range(4) for k in range(parts)], f"PV{v}")
            yield ("commit", f"o_done{pv}")
            yield ("commit", f"v_empty{sv}")

    def softmax(warp):
        q4, part = warp & 3, (warp - 2) >> 2
        nb = 1 + q4
        for p in range(NP):
            sb = p % NS
            xm = p & 1 if mistake != "single-buffered max exchange" else 0
            yield ("wait", f"s_full{sb}", p // NS)
            for c in range(rd * part, rd * part + rd):
                yield ("read", f"S{sb}.q{q4}.c{c}", ("S", p))
            yield ("write", f"xm{xm}.q{q4}.h{part}", ("m", p))
            if mistake != "no barrier before P":
                yield ("nbar", nb, parts)
            for k in range(parts):
                yield ("read", f"xm{xm}.q{q4}.h{k}", ("m", p))
            if p in rescale_steps and p >= 1:  # every part of a quarter takes the same decision
                if mistake != "rescale without o_done":
                    yield ("wait", f"o_done{(p - 1) % NS}", (p - 1) // NS)
                yield ("read", f"O.q{q4}.h{part}", ("O", p - 1))
                yield ("write", f"O.q{q4}.h{part}", ("O", p - 1))
            for c in range(wr * part, wr * part + wr):
                yield ("write", f"S{sb}.q{q4}.c{c}", ("P", p))
            yield ("arrive", f"p_full{sb}", 32)
        if mistake != "no barrier before the sums":
            yield ("nbar", nb, parts)
        yield ("write", f"xm0.q{q4}.h{part}", ("l",))
        yield ("nbar", nb, parts)
        for k in range(parts):
            yield ("read", f"xm0.q{q4}.h{k}", ("l",))
        if NP > 0:
            yield ("wait", f"o_done{(NP - 1) % NS}", (NP - 1) // NS)
            yield ("read", f"O.q{q4}.h{part}", ("O", NP - 1))

    m.role("k_producer", k_producer())
    m.role("v_producer", v_producer())
    m.role("s_issuer", drained(m, "s_issuer", s_issuer()))
    m.role("pv_issuer", drained(m, "pv_issuer", pv_issuer(), skip=mistake == "PV issuer skips its drain"))
    for w in range(2, 2 + 4 * parts):
        m.role(f"softmax{w}", softmax(w))


# --------------------------------------------------------------------------------------------------------------
# score_tc_kernel (csrc/score_tc.cu): two 128-row Q tiles against 128-kernel stages, stages 0..ntiles-1 for the
# LSE pass and ntiles..2 ntiles-1 for the block maxima.  Warp 0: both Q tiles, then the kernel stages (3-slot
# ring); warp 1: S(tile) = Q(tile) kern^T per stage; warps 2-17: TMEM readers, four per lane quarter, 32
# columns each (pass 2 also reads the column before its first: the previous part's last, or for part 0 the
# stage's last); the four LSE parts meet in shared memory; pass 2 writes the group scores over the Q staging
# area; then reader warp w selects token w - 2.
# --------------------------------------------------------------------------------------------------------------
def score_tc_model(m: PipelineModel, ntiles: int, mistake: str = "", parts: int = 4):
    nq = 2 * ntiles
    nreaders = 4 * parts
    m.bar("q_full", 1)
    m.bar("q_tmem", 128)
    for i in range(RING):
        m.bar(f"k_full{i}", 1)
        m.bar(f"k_empty{i}", 1)
    for t in range(2):
        m.bar(f"s_full{t}", 1)
        m.bar(f"s_empty{t}", 32 * nreaders)

    def producer():
        yield ("arrive_tx", "q_full", 1, 2)
        yield ("tma", "q_full", 1, [("area", "Q")])
        yield ("tma", "q_full", 1, [("area2", "Q")])
        for q in range(nq):
            s, k = q % RING, q // RING
            if k >= 1:
                yield ("wait", f"k_empty{s}", k - 1)
            yield ("arrive_tx", f"k_full{s}", 1, 1)
            yield ("tma", f"k_full{s}", 1, [(f"kern{s}", ("kern", q))])
        # the producer's drain before the CTA ends: every copy it issued has landed
        yield ("wait", "q_full", 0)
        for s in range(min(RING, nq)):
            yield ("wait", f"k_full{s}", (nq - 1 - s) // RING)

    def issuer():
        yield ("wait", "q_tmem", 0)
        for q in range(nq):
            s = q % RING
            yield ("wait", f"k_full{s}", q // RING)
            for tile in range(2):
                if q >= 1 and mistake != "issuer skips s_empty":
                    yield ("wait", f"s_empty{tile}", q - 1)
                yield ("mma", [(f"QT{tile}.q{x}", "Q") for x in range(4)] + [(f"kern{s}", ("kern", q))],
                       [(f"S{tile}.q{x}.p{h}", ("S", q)) for x in range(4) for h in range(parts)], f"S{tile}.{q}")
                yield ("commit", f"s_full{tile}")
            yield ("commit", f"k_empty{s}")

    def reader(w):
        q4, part = w & 3, (w - 2) >> 2
        yield ("wait", "q_full", 0)
        if part == 0:
            yield ("read", "area", "Q")
            yield ("read", "area2", "Q")
            yield ("write", f"QT0.q{q4}", "Q")
            yield ("write", f"QT1.q{q4}", "Q")
            yield ("arrive", "q_tmem", 32)
        for q in range(nq):
            for tile in range(2):
                yield ("wait", f"s_full{tile}", q)
                yield ("read", f"S{tile}.q{q4}.p{part}", ("S", q))
                if q >= ntiles:
                    yield ("read", f"S{tile}.q{q4}.p{(part - 1) % parts}", ("S", q))
                yield ("arrive", f"s_empty{tile}", 32)
                if q >= ntiles:  # group scores over the Q staging area
                    yield ("write", "area", "S")
                    for tok in (8 * tile + 2 * q4, 8 * tile + 2 * q4 + 1):
                        yield ("write", f"Ssm.t{tok}.s{q}.p{part}", "S")  # this stage's blocks of the part
            if q == ntiles - 1:
                yield ("write", f"hm.q{q4}.p{part}", "m")
                if mistake != "no barrier in the LSE exchange":
                    yield ("nbar", 1, nreaders)
                for k in range(parts):
                    yield ("read", f"hm.q{q4}.p{k}", "m")
        if mistake != "no barrier before the select":
            yield ("nbar", 1, nreaders)
        ts = w - 2
        for q in range(ntiles, nq):
            for h in range(parts):
                yield ("read", f"Ssm.t{ts}.s{q}.p{h}", "S")

    m.role("producer", producer())
    m.role("issuer", drained(m, "issuer", issuer()))
    for w in range(2, 2 + nreaders):
        m.role(f"reader{w}", reader(w))


# --------------------------------------------------------------------------------------------------------------
def _run(model, seeds, *args, **kw):
    for seed in seeds:
        m = PipelineModel(seed)
        model(m, *args, **kw)
        m.run()


@pytest.mark.parametrize("VR", [2, 3])
@pytest.mark.parametrize("U", [1, 2, 3, 4, 5, 7, 12, 33])
def test_attn_tc_protocol(U, VR):
    for seed in range(40):
        NP = (U + 1) // 2
        rescale = {p for p in range(NP) if (seed * 7 + p) % 3 == 0}
        m = PipelineModel(seed)
        attn_tc_model(m, U, rescale, VR=VR)
        m.run()


@pytest.mark.parametrize("ntiles", [1, 2, 3, 5])
def test_score_tc_protocol(ntiles):
    _run(score_tc_model, range(40), ntiles)


def _caught(model, seeds, *args, **kw):
    try:
        _run(model, seeds, *args, **kw)
    except ProtocolError:
        return True
    return False


@pytest.mark.parametrize("mistake,U", [
    ("k producer skips k_empty", 9), ("v producer skips v_empty", 9), ("S issuer skips o_done", 9),
    ("PV issuer skips p_full", 5),
    ("single-buffered max exchange", 5), ("no barrier before P", 3), ("rescale without o_done", 5),
    ("no barrier before the sums", 5), ("PV issuer skips its drain", 5),
])
def test_attn_tc_planted_mistakes_are_caught(mistake, U):
    NP = (U + 1) // 2
    assert _caught(attn_tc_model, range(300), U, set(range(1, NP)), mistake=mistake), mistake


@pytest.mark.parametrize("mistake", ["issuer skips s_empty", "no barrier in the LSE exchange",
                                     "no barrier before the select"])
def test_score_tc_planted_mistakes_are_caught(mistake):
    assert _caught(score_tc_model, range(300), 3, mistake=mistake), mistake


def test_checker_reports_a_deadlock_and_a_wrong_phase():
    m = PipelineModel(0)
    m.bar("b", 1)
    m.role("a", [("wait", "b", 0)])
    with pytest.raises(ProtocolError, match="deadlock"):
        m.run()
    m = PipelineModel(0)
    m.bar("b", 1)
    m.role("a", [("arrive", "b", 1), ("arrive", "b", 1), ("arrive", "b", 1), ("wait", "b", 0)])
    with pytest.raises(ProtocolError, match="phase 0 returned with 3"):
        m.run()


# --------------------------------------------------------------------------------------------------------------
# bwd_dq_tc_kernel (csrc/attn_bwd_tc.cu): one 128-row tile over U union blocks.  Warp 0: Q and dO once, K per
# step (3-slot ring); warp 10: V per step; warp 1: S(p) = Q K^T into buffer p & 1 once dQ(p - 2) is done; warp
# 11: dP(p) = dO V^T into buffer p & 1 once dS(p - 2) was signalled; warp 12: dQ += dS(p) K (the three issuers'
# ops unordered relative to each other; K(p) freed by S(p)'s and dQ(p)'s commits); warps 2-9: dS, two per lane
# quarter (half 0: keys 0-31, half 1: keys 32-63); dS goes
# back over the first 32 columns of its S buffer after both halves' loads (named barrier per quarter).
# --------------------------------------------------------------------------------------------------------------
def bwd_dq_model(m: PipelineModel, U: int, mistake: str = ""):
    m.bar("qd_full", 1)
    m.bar("qd_tmem", 128)
    for i in range(RING):
        for n in ("k_full", "v_full", "v_empty"):
            m.bar(f"{n}{i}", 1)
        m.bar(f"k_empty{i}", 1 if mistake == "k_empty waits for one issuer" else 2)
    for i in range(2):
        m.bar(f"s_full{i}", 2)
        m.bar(f"ds_full{i}", 256)
        m.bar(f"dq_done{i}", 1)

    def warp0():
        yield ("arrive_tx", "qd_full", 1, 2)
        yield ("tma", "qd_full", 1, [("Qs", "Q")])
        yield ("tma", "qd_full", 1, [("dOs", "dO")])
        for p in range(U):
            s, k = p % RING, p // RING
            if k >= 1 and mistake != "K producer skips k_empty":
                yield ("wait", f"k_empty{s}", k - 1)
            yield ("arrive_tx", f"k_full{s}", 1, 1)
            yield ("tma", f"k_full{s}", 1, [(f"K{s}", ("K", p))])

    def warp10():
        for p in range(U):
            s, k = p % RING, p // RING
            if k >= 1:
                yield ("wait", f"v_empty{s}", k - 1)
            yield ("arrive_tx", f"v_full{s}", 1, 1)
            yield ("tma", f"v_full{s}", 1, [(f"V{s}", ("V", p))])

    def s_issuer():
        yield ("wait", "qd_tmem", 0)
        for p in range(U):
            s, sb = p % RING, p & 1
            if p >= 2 and mistake != "S issuer skips dq_done":
                yield ("wait", f"dq_done{sb}", (p - 2) >> 1)
            yield ("wait", f"k_full{s}", p // RING)
            yield ("mma", [(f"QT.q{q}", "Q") for q in range(4)] + [(f"K{s}", ("K", p))],
                   [(f"S{sb}.q{q}.{c}", ("S", p)) for q in range(4) for c in ("a", "b", "hi")], f"S{p}")
            yield ("commit", f"s_full{sb}")
            yield ("commit", f"k_empty{s}")

    def dp_issuer():
        yield ("wait", "qd_tmem", 0)
        for p in range(U):
            s, sb = p % RING, p & 1
            if p >= 2 and mistake != "dP issuer skips ds_full":
                yield ("wait", f"ds_full{sb}", (p - 2) >> 1)
            yield ("wait", f"v_full{s}", p // RING)
            yield ("mma", [(f"dOT.q{q}", "dO") for q in range(4)] + [(f"V{s}", ("V", p))],
                   [(f"DP{sb}.q{q}.{c}", ("DP", p)) for q in range(4) for c in ("lo", "hi")], f"DP{p}")
            yield ("commit", f"s_full{sb}")
            yield ("commit", f"v_empty{s}")

    def dq_issuer():
        for v in range(U):
            db, s = v & 1, v % RING
            if mistake != "issuer skips ds_full":
                yield ("wait", f"ds_full{db}", v >> 1)
            yield ("wait", f"k_full{s}", v // RING)
            reads = [(f"S{db}.q{q}.{c}", ("dS", v)) for q in range(4) for c in ("a", "b")]
            reads += [(f"K{s}", ("K", v))] + ([("dQ", ("dQ", v - 1))] if v > 0 else [])
            yield ("mma", reads, [("dQ", ("dQ", v))], f"dQ{v}")
            yield ("commit", f"dq_done{db}")
            yield ("commit", f"k_empty{s}")

    def ds_warp(w):
        q4, half = w & 3, (w - 2) >> 2
        yield ("wait", "qd_full", 0)
        if half == 0:
            yield ("read", "Qs", "Q")
            yield ("read", "dOs", "dO")
            yield ("write", f"QT.q{q4}", "Q")
            yield ("write", f"dOT.q{q4}", "dO")
            yield ("arrive", "qd_tmem", 32)
        for p in range(U):
            sb = p & 1
            yield ("wait", f"s_full{sb}", p >> 1)
            if half == 0:
                yield ("read", f"S{sb}.q{q4}.a", ("S", p))
                yield ("read", f"S{sb}.q{q4}.b", ("S", p))
                yield ("read", f"DP{sb}.q{q4}.lo", ("DP", p))
            else:
                yield ("read", f"S{sb}.q{q4}.hi", ("S", p))
                yield ("read", f"DP{sb}.q{q4}.hi", ("DP", p))
            if mistake != "no pair barrier":
                yield ("nbar", 1 + q4, 2)
            yield ("write", f"S{sb}.q{q4}.{'a' if half == 0 else 'b'}", ("dS", p))
            yield ("arrive", f"ds_full{sb}", 32)
        if U > 0:
            if mistake != "no final dq_done wait":
                yield ("wait", f"dq_done{(U - 1) & 1}", (U - 1) >> 1)
            yield ("read", "dQ", ("dQ", U - 1))

    m.role("warp0", warp0())
    m.role("warp10", warp10())
    m.role("s_issuer", drained(m, "s_issuer", s_issuer()))
    m.role("dp_issuer", drained(m, "dp_issuer", dp_issuer()))
    m.role("dq_issuer", drained(m, "dq_issuer", dq_issuer(), skip=mistake == "dQ issuer skips its drain"))
    for w in range(2, 10):
        m.role(f"ds{w}", ds_warp(w))


# --------------------------------------------------------------------------------------------------------------
# bwd_dkdv_tc_kernel (csrc/attn_bwd_tc.cu): work items (one 64-key block and up to 256 of its listed tokens),
# each in 8-token tiles.  Warp 0: the item's K and V, then per tile the token ids (shared memory) and the Q / dO
# rows (TMA, 2 buffers); warp 1: S, dP per tile into buffers tile & 1; warp 6: dV^T += dO^T P and dK^T += Q^T dS
# (the two issuers' ops unordered relative to each other; a Q / dO buffer is freed by both issuers' commits, K / V
# by warp 1's); warps 2-5: P and dS into shared-memory tiles (one row per thread), and after each item the
# flush of dV^T / dK^T from TMEM.
# --------------------------------------------------------------------------------------------------------------
def bwd_dkdv_model(m: PipelineModel, items, mistake: str = ""):
    m.bar("kv_full", 1)
    m.bar("kv_free", 1)
    for i in range(2):
        m.bar(f"qd_full{i}", 1)
        m.bar(f"qd_free{i}", 1 if mistake == "qd_free waits for one issuer" else 2)
        m.bar(f"s_full{i}", 1)
    m.bar("pd_full", 128)
    m.bar("pd_free", 1)
    m.bar("acc_done", 1)
    m.bar("acc_free", 128)
    Q4 = range(4)

    def producer():
        n_tile = 0
        for n_item, ntiles in enumerate(items):
            if n_item >= 1 and mistake != "producer skips kv_free":
                yield ("wait", "kv_free", n_item - 1)
            yield ("arrive_tx", "kv_full", 1, 1)
            yield ("tma", "kv_full", 1, [("KV", ("KV", n_item))])
            for _ in range(ntiles):
                qb, use = n_tile & 1, n_tile >> 1
                if use >= 1 and mistake != "producer skips qd_free":
                    yield ("wait", f"qd_free{qb}", use - 1)
                yield ("write", f"tok{qb}", ("tok", n_tile))
                yield ("arrive_tx", f"qd_full{qb}", 1, 1)
                yield ("tma", f"qd_full{qb}", 1, [(f"QdO{qb}", ("QdO", n_tile))])
                n_tile += 1

    def s_issuer():
        n_tile = 0
        for n_item, ntiles in enumerate(items):
            yield ("wait", "kv_full", n_item)
            for i in range(ntiles):
                ctr = n_tile + i
                b = ctr & 1
                # S buffer b held S(ctr - 2): QdO(ctr) is loaded only after both issuers freed buffer b for
                # tile ctr - 2, and dVdK(ctr - 2) ran on P(ctr - 2), written after the warps read S(ctr - 2)
                yield ("wait", f"qd_full{b}", ctr >> 1)
                yield ("mma", [(f"QdO{b}", ("QdO", ctr)), ("KV", ("KV", n_item))],
                       [(f"S{b}.q{q}", ("S", ctr)) for q in Q4] + [(f"DP{b}.q{q}", ("DP", ctr)) for q in Q4], f"S{ctr}")
                yield ("commit", f"s_full{b}")
                yield ("commit", f"qd_free{b}")
            n_tile += ntiles
            yield ("commit", "kv_free")

    def acc_issuer():
        n_tile = 0
        for n_item, ntiles in enumerate(items):
            if n_item >= 1 and mistake != "issuer skips acc_free":
                yield ("wait", "acc_free", n_item - 1)
            for i in range(ntiles):
                ctr = n_tile + i
                yield ("wait", f"qd_full{ctr & 1}", ctr >> 1)
                yield ("wait", "pd_full", ctr)
                reads = [(f"QdO{ctr & 1}", ("QdO", ctr))] + [(f"P.q{q}", ("P", ctr)) for q in Q4]
                if i > 0:
                    reads += [(f"acc.q{q}", ("acc", n_item, i - 1)) for q in Q4]
                yield ("mma", reads, [(f"acc.q{q}", ("acc", n_item, i)) for q in Q4], f"dVdK{ctr}")
                yield ("commit", "pd_free")
                yield ("commit", f"qd_free{ctr & 1}")
            n_tile += ntiles
            yield ("commit", "acc_done")

    def warps(q4):
        n_tile = 0
        for n_item, ntiles in enumerate(items):
            for _ in range(ntiles):
                b = n_tile & 1
                yield ("wait", f"qd_full{b}", n_tile >> 1)
                yield ("wait", f"s_full{b}", n_tile >> 1)
                yield ("read", f"tok{b}", ("tok", n_tile))
                yield ("read", f"S{b}.q{q4}", ("S", n_tile))
                yield ("read", f"DP{b}.q{q4}", ("DP", n_tile))
                if n_tile >= 1 and mistake != "warps skip pd_free":
                    yield ("wait", "pd_free", n_tile - 1)
                yield ("write", f"P.q{q4}", ("P", n_tile))
                yield ("arrive", "pd_full", 32)
                n_tile += 1
            if mistake != "warps skip acc_done":
                yield ("wait", "acc_done", n_item)
            if ntiles > 0:
                yield ("read", f"acc.q{q4}", ("acc", n_item, ntiles - 1))
            yield ("arrive", "acc_free", 32)

    m.role("producer", producer())
    m.role("s_issuer", drained(m, "s_issuer", s_issuer(), skip=mistake == "S issuer skips its drain"))
    m.role("acc_issuer", drained(m, "acc_issuer", acc_issuer()))
    for q4 in Q4:
        m.role(f"warp{2 + q4}", warps(q4))


@pytest.mark.parametrize("U", [0, 1, 2, 3, 4, 7, 12])
def test_bwd_dq_protocol(U):
    _run(bwd_dq_model, range(60), U)


@pytest.mark.parametrize("items", [[1], [0], [3, 0, 2], [5, 1, 0, 4], [2, 2, 2, 2, 2], [0, 0, 1]])
def test_bwd_dkdv_protocol(items):
    _run(bwd_dkdv_model, range(60), items)


@pytest.mark.parametrize("mistake", ["K producer skips k_empty", "issuer skips ds_full", "no pair barrier",
                                     "no final dq_done wait", "S issuer skips dq_done", "dP issuer skips ds_full",
                                     "k_empty waits for one issuer", "dQ issuer skips its drain"])
def test_bwd_dq_planted_mistakes_are_caught(mistake):
    assert _caught(bwd_dq_model, range(300), 7, mistake=mistake), mistake


@pytest.mark.parametrize("mistake", ["producer skips kv_free", "producer skips qd_free", "issuer skips acc_free",
                                     "warps skip pd_free", "warps skip acc_done", "qd_free waits for one issuer",
                                     "S issuer skips its drain"])
def test_bwd_dkdv_planted_mistakes_are_caught(mistake):
    # acc_free matters only where empty items let the issuer commit acc_done twice without a P tile between
    assert _caught(bwd_dkdv_model, range(300), [3, 0, 0, 2, 4], mistake=mistake), mistake
