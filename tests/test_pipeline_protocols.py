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


# --------------------------------------------------------------------------------------------------------------
# attn_tc_kernel (csrc/attn_tc.cu): 128-row tile, U union blocks in NP = ceil(U / 2) steps of 128 keys.
# Warp 0: Q once, then K per step (3-slot ring); warp 10: V per step (Q is staged in the last V slot);
# warp 1: S(p) = Q K^T into S buffer p & 1, then O += P(p - 1) V; warps 2-9: softmax, two per TMEM lane
# quarter, each on 64 keys, P written over the first 64 columns of its S buffer.
# --------------------------------------------------------------------------------------------------------------
def attn_tc_model(m: PipelineModel, U: int, rescale_steps=(), parts: int = 2, mistake: str = ""):
    NP = (U + 1) // 2
    m.bar("q_full", 1)
    m.bar("q_tmem", 128)
    for i in range(RING):
        for n in ("k_full", "k_empty", "v_full", "v_empty"):
            m.bar(f"{n}{i}", 1)
    for i in range(2):
        m.bar(f"s_full{i}", 1)
        m.bar(f"p_full{i}", 128 * parts)
        m.bar(f"o_done{i}", 1)
    vq = f"V{RING - 1}"
    rd = 8 // parts  # 16-column chunks of S read per part
    wr = 4 // parts  # 16-column chunks of P written per part

    def k_producer():
        yield ("arrive_tx", "q_full", 1, 1)
        yield ("tma", "q_full", 1, [(vq, "Q")])
        for p in range(NP):
            s, k = p % RING, p // RING
            if k >= 1 and mistake != "k producer skips k_empty":
                yield ("wait", f"k_empty{s}", k - 1)
            yield ("arrive_tx", f"k_full{s}", 1, 1)
            yield ("tma", f"k_full{s}", 1, [(f"K{s}", ("K", p))])

    def v_producer():
        for p in range(NP):
            s, k = p % RING, p // RING
            if k >= 1:
                yield ("wait", f"v_empty{s}", k - 1)
            if p == RING - 1 and mistake != "V fill ignores q_tmem":
                yield ("wait", "q_tmem", 0)
            yield ("arrive_tx", f"v_full{s}", 1, 1)
            yield ("tma", f"v_full{s}", 1, [(f"V{s}", ("V", p))])

    def issuer():
        yield ("wait", "q_tmem", 0)
        for p in range(NP + 1):
            if p < NP:
                s, sb = p % RING, p & 1
                yield ("wait", f"k_full{s}", p // RING)
                yield ("mma", [(f"QT.q{q}", "Q") for q in range(4)] + [(f"K{s}", ("K", p))],
                       [(f"S{sb}.q{q}.c{c}", ("S", p)) for q in range(4) for c in range(8)], f"S{p}")
                yield ("commit", f"s_full{sb}")
                yield ("commit", f"k_empty{s}")
            if p >= 1:
                v = p - 1
                if mistake != "issuer skips p_full":
                    yield ("wait", f"p_full{v & 1}", v >> 1)
                yield ("wait", f"v_full{v % RING}", v // RING)
                reads = [(f"S{v & 1}.q{q}.c{c}", ("P", v)) for q in range(4) for c in range(4)]
                reads += [(f"V{v % RING}", ("V", v))]
                if v > 0:
                    reads += [(f"O.q{q}.h{k}", ("O", v - 1)) for q in range(4) for k in range(parts)]
                yield ("mma", reads, [(f"O.q{q}.h{k}", ("O", v)) for q in range(4) for k in range(parts)], f"PV{v}")
                yield ("commit", f"o_done{v & 1}")
                yield ("commit", f"v_empty{v % RING}")

    def softmax(warp):
        q4, part = warp & 3, (warp - 2) >> 2
        nb = 1 + q4
        yield ("wait", "q_full", 0)
        if part == 0:
            yield ("read", vq, "Q")
            yield ("write", f"QT.q{q4}", "Q")
            yield ("arrive", "q_tmem", 32)
        for p in range(NP):
            sb = p & 1
            xm = p & 1 if mistake != "single-buffered max exchange" else 0
            yield ("wait", f"s_full{sb}", p >> 1)
            for c in range(rd * part, rd * part + rd):
                yield ("read", f"S{sb}.q{q4}.c{c}", ("S", p))
            yield ("write", f"xm{xm}.q{q4}.h{part}", ("m", p))
            if mistake != "no barrier before P":
                yield ("nbar", nb, parts)
            for k in range(parts):
                yield ("read", f"xm{xm}.q{q4}.h{k}", ("m", p))
            if p in rescale_steps and p >= 1:  # every part of a quarter takes the same decision
                if mistake != "rescale without o_done":
                    yield ("wait", f"o_done{(p - 1) & 1}", (p - 1) >> 1)
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
            yield ("wait", f"o_done{(NP - 1) & 1}", (NP - 1) >> 1)
            yield ("read", f"O.q{q4}.h{part}", ("O", NP - 1))

    m.role("k_producer", k_producer())
    m.role("v_producer", v_producer())
    m.role("issuer", issuer())
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
    m.role("issuer", issuer())
    for w in range(2, 2 + nreaders):
        m.role(f"reader{w}", reader(w))


# --------------------------------------------------------------------------------------------------------------
def _run(model, seeds, *args, **kw):
    for seed in seeds:
        m = PipelineModel(seed)
        model(m, *args, **kw)
        m.run()


@pytest.mark.parametrize("U", [1, 2, 3, 4, 5, 7, 12, 33])
def test_attn_tc_protocol(U):
    for seed in range(40):
        NP = (U + 1) // 2
        rescale = {p for p in range(NP) if (seed * 7 + p) % 3 == 0}
        m = PipelineModel(seed)
        attn_tc_model(m, U, rescale)
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
    ("k producer skips k_empty", 9), ("V fill ignores q_tmem", 9), ("issuer skips p_full", 5),
    ("single-buffered max exchange", 5), ("no barrier before P", 3), ("rescale without o_done", 5),
    ("no barrier before the sums", 5),
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
