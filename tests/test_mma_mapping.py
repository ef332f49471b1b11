"""The batch-1 tensor-core GEMV's operand mapping, checked on the CPU.

The kernel feeds mma.sync m16n8k16 straight from the packed codes: lane
t = 4g + r holds chunk r of row g of a 128-weight block, word j of that chunk
is MMA j's A fragment (row g: the word's first K segment, row g + 8: its
second), and B column 2h + s holds segment s of the activations restricted to
group h of the block.  This test restates that scheme (from the packed-layout
text of include/qnt.h and the m16n8k16 fragment layout of the PTX ISA), runs
the four MMAs of a block as fp64 matrix products and checks that
D[g][2h] + D[g+8][2h+1], summed over the block's MMAs, is row g's dot product
over group h.  A wrong mask, segment, activation position or fragment index
fails it."""
import numpy as np
import pytest

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1(c):
    v = E2M1[c & 7]
    return -v if c & 8 else v


def nibble_weight(fmt, p, j):
    """Chunk weight held by nibble p of word j (include/qnt.h, packed layout)."""
    if fmt == "int4":
        return 16 * (p % 2) + 4 * j + 2 * ((p // 2) % 2) + p // 4
    return 8 * j + p


def pack_block(fmt, q):
    """q: [8 rows][128] codes of one block -> 512 bytes as 128 little-endian words."""
    words = np.zeros(128, dtype=np.uint32)
    for i in range(8):
        for c in range(4):
            pos = 4 * i + (c ^ ((i // 2) % 4))          # 16-byte chunk slot of row i, chunk c
            for j in range(4):
                w = 0
                for p in range(8):
                    w |= int(q[i, 32 * c + nibble_weight(fmt, p, j)]) << (4 * p)
                words[4 * pos + j] = w
    return words


def half_pair(bits32):
    lo, hi = bits32 & 0xFFFF, bits32 >> 16
    return [float(np.array([lo], dtype=np.uint16).view(np.float16)[0]),
            float(np.array([hi], dtype=np.uint16).view(np.float16)[0])]


def a_fragments(fmt, w):
    """The kernel's four A registers from one code word, as value pairs."""
    if fmt == "int4":
        w8 = w >> 8
        regs = [w & 0x000F000F, w8 & 0x000F000F, w & 0x00F000F0, w8 & 0x00F000F0]
        return [half_pair(r) for r in regs]     # fp16 subnormals q 2^-24 (16 q 2^-24 for bits 4..7)
    # cvt.rn.f16x2.e2m1x2 of byte b: low nibble -> low half
    return [[e2m1((w >> (8 * b)) & 15), e2m1((w >> (8 * b + 4)) & 15)] for b in range(4)]


def b_entries(fmt, x, G):
    """Activation image of one block: entry (s, r) = 4 MMAs x (b0, b1) value pairs.

    Offset o of a chunk meets B half hf, segment s of MMA j where
    o = 16 hf + 4j + 2s + e (INT4; half hf = 1 carries x / 16) or
    o = 8j + 4hf + 2s + e (FP4 family)."""
    ent = np.zeros((2, 4, 4, 2, 2))             # [s][r][j][hf][e]
    for r in range(4):
        for o in range(32):
            e = o % 2
            if fmt == "int4":
                hf, j, s = o // 16, (o % 16) // 4, (o // 2) % 2
                val = x[32 * r + o] / (16.0 if hf else 1.0)
            else:
                j, hf, s = o // 8, (o // 4) % 2, (o // 2) % 2
                val = x[32 * r + o]
            ent[s, r, j, hf, e] = val
    return ent


def razer_patch(w, pairs, sv):
    """The kernel's RaZeR step: nibbles equal to 0b1000 (decoded -0), found with
    t = (w & 0x77777777) + 0x77777777, spec = w & ~t & 0x88888888, take sv."""
    t = ((w & 0x77777777) + 0x77777777) & 0xFFFFFFFF
    spec = w & ~t & 0x88888888
    out = [list(p) for p in pairs]
    for b in range(4):
        if spec & (0x8 << (8 * b)):
            out[b][0] = sv
        if spec & (0x80 << (8 * b)):
            out[b][1] = sv
    return out


def emulate_block(fmt, q, x, G, sv=None, part=None):
    """Run the block's four MMAs with the kernel's lane assignments; return the
    per-lane sums D[g][2r] + D[g+8][2r+1] (lane 4g + r).  sv[g][h]: RaZeR special
    value of row g, group h; part: AFPQ "pos" / "neg" operand (max(h, 0) / h - that)."""
    GPB = 128 // G
    words = pack_block(fmt, q)
    ent = b_entries(fmt, x, G)
    acc = np.zeros((16, 8))
    for j in range(4):
        A = np.zeros((16, 16))
        B = np.zeros((16, 8))
        for t in range(32):
            g, r = t // 4, t % 4
            # A: chunk r of row g, word j
            w = int(words[4 * (4 * g + (r ^ ((g // 2) % 4))) + j])
            a = a_fragments(fmt, w)
            if sv is not None:
                a = razer_patch(w, a, sv[g][r // (4 // GPB)])   # the group of this lane's chunk
            if part is not None:
                a = [[max(v, 0.0) if part == "pos" else v - max(v, 0.0) for v in pr] for pr in a]
            A[g, 2 * r:2 * r + 2] = a[0]
            A[g + 8, 2 * r:2 * r + 2] = a[1]
            A[g, 2 * r + 8:2 * r + 10] = a[2]
            A[g + 8, 2 * r + 8:2 * r + 10] = a[3]
            # B: column n = t / 4 = 2h + s; only lanes whose chunk r lies in group h load
            n, hB, sB = t // 4, t // 8, (t // 4) % 2
            if hB < GPB and r // (4 // GPB) == hB:
                B[2 * r:2 * r + 2, n] = ent[sB, r, j, 0]
                B[2 * r + 8:2 * r + 10, n] = ent[sB, r, j, 1]
        acc += A @ B
    return np.array([acc[t // 4, 2 * (t % 4)] + acc[t // 4 + 8, 2 * (t % 4) + 1] for t in range(32)])


@pytest.mark.parametrize("fmt", ["int4", "fp4"])
@pytest.mark.parametrize("G", [128, 64, 32])
def test_block_mma_gives_row_group_dot_products(fmt, G):
    rng = np.random.default_rng(G + (0 if fmt == "int4" else 1))
    q = rng.integers(0, 16, size=(8, 128))
    x = rng.standard_normal(128)
    lanes = emulate_block(fmt, q, x, G)
    GPB = 128 // G
    scale = 2.0 ** -24 if fmt == "int4" else 1.0      # INT4 codes enter as fp16 subnormals
    for g in range(8):
        for h in range(4):
            got = lanes[4 * g + h]
            if h >= GPB:
                assert got == 0.0                     # columns of absent groups stay zero
                continue
            ks = range(h * G, (h + 1) * G)
            dq = [q[g, k] * scale if fmt == "int4" else e2m1(int(q[g, k])) for k in ks]
            want = float(np.dot(dq, x[list(ks)]))
            assert got == pytest.approx(want, rel=1e-12, abs=1e-30)


def test_codes_reach_each_weight_once():
    # every (row, weight) of a block enters exactly one A element of exactly one MMA
    for fmt in ("int4", "fp4"):
        seen = np.zeros((8, 128), dtype=int)
        for c in range(4):
            for j in range(4):
                for p in range(8):
                    seen[:, 32 * c + nibble_weight(fmt, p, j)] += 1
        assert (seen == 1).all()


@pytest.mark.parametrize("G", [128, 64, 32])
def test_razer_special_values_follow_the_chunk_group(G):
    rng = np.random.default_rng(100 + G)
    q = rng.integers(0, 16, size=(8, 128))
    q[:, ::5] = 8                                        # plenty of -0 codes in every group
    x = rng.standard_normal(128)
    GPB = 128 // G
    sv = [[float(rng.choice([5.0, -5.0, 8.0, -8.0])) for _ in range(GPB)] for _ in range(8)]
    lanes = emulate_block("razer", q, x, G, sv=sv)
    for g in range(8):
        for h in range(GPB):
            ks = range(h * G, (h + 1) * G)
            dq = [sv[g][h] if q[g, k] == 8 else e2m1(int(q[g, k])) for k in ks]
            assert lanes[4 * g + h] == pytest.approx(float(np.dot(dq, x[list(ks)])), rel=1e-12)


@pytest.mark.parametrize("G", [128, 32])
def test_afpq_positive_and_negative_parts(G):
    rng = np.random.default_rng(200 + G)
    q = rng.integers(0, 16, size=(8, 128))
    x = rng.standard_normal(128)
    pos = emulate_block("afpq", q, x, G, part="pos")
    neg = emulate_block("afpq", q, x, G, part="neg")
    for g in range(8):
        for h in range(128 // G):
            ks = list(range(h * G, (h + 1) * G))
            vals = np.array([e2m1(int(q[g, k])) for k in ks])
            assert pos[4 * g + h] == pytest.approx(float(np.dot(np.maximum(vals, 0), x[ks])), rel=1e-12, abs=1e-15)
            assert neg[4 * g + h] == pytest.approx(float(np.dot(np.minimum(vals, 0), x[ks])), rel=1e-12, abs=1e-15)


def test_activation_image_offsets_agree_between_builder_and_reader():
    """The builder stores the pair for (block b, chunk r, segment s, MMA j, half hf)
    at byte 256 b + 128 (j >> 1) + 16 (4 s + r) + 8 (j & 1) + 4 hf; a lane reading
    entry (s, r) loads 16 bytes at 256 b + 16 (4 s + r) and 16 at + 128, and takes
    register 2 j + hf of the eight as MMA j's b0 (hf = 0) / b1 (hf = 1)."""
    def written(b, r, s, j, hf):
        return 256 * b + 128 * (j >> 1) + 16 * (4 * s + r) + 8 * (j & 1) + 4 * hf

    def read(b, r, s, reg):
        base = 256 * b + 16 * (4 * s + r) + (128 if reg >= 4 else 0)
        return base + 4 * (reg % 4)

    offsets = set()
    for b in range(3):
        for r in range(4):
            for s in range(2):
                for j in range(4):
                    for hf in range(2):
                        off = written(b, r, s, j, hf)
                        assert off == read(b, r, s, 2 * j + hf)
                        offsets.add(off)
    assert sorted(offsets) == list(range(0, 3 * 256, 4))      # 256 bytes per block, no overlap


# ------------------------------------------------------------------ several blocks per set of accumulators
def emulate_set(fmt, qs, xs, G, q, NQ):
    """The kernel's set scheme: a set of S = 4 / GPB blocks (q + NQ i, i < S),
    one accumulator D_i per block, all fed the same B registers.  Lane t = 4g + r
    takes B column pair hp = t / 8, i.e. block q + NQ (hp / GPB), group hp % GPB,
    and loads its entry only if its chunk r lies in that group (G = 128: every
    lane).  The epilogue of lane 4g + r reads D_{r / GPB}[g][2r] +
    D_{r / GPB}[g+8][2r+1]: row g's dot product over block q + NQ (r / GPB),
    group r % GPB.  qs / xs map a block index to its codes / activations."""
    GPB = 128 // G
    S = 4 // GPB
    ents = {b: b_entries(fmt, xs[b], G) for b in xs}
    acc = [np.zeros((16, 8)) for _ in range(S)]
    for i in range(S):
        words = pack_block(fmt, qs[q + NQ * i])
        for j in range(4):
            A = np.zeros((16, 8 * 2))
            B = np.zeros((16, 8))
            for t in range(32):
                g, r = t // 4, t % 4
                w = int(words[4 * (4 * g + (r ^ ((g // 2) % 4))) + j])
                a = a_fragments(fmt, w)
                A[g, 2 * r:2 * r + 2] = a[0]
                A[g + 8, 2 * r:2 * r + 2] = a[1]
                A[g, 2 * r + 8:2 * r + 10] = a[2]
                A[g + 8, 2 * r + 8:2 * r + 10] = a[3]
                n, hp, sB = t // 4, t // 8, (t // 4) % 2
                if (r * GPB) // 4 == hp % GPB:
                    bb = q + NQ * (hp // GPB)
                    B[2 * r:2 * r + 2, n] = ents[bb][sB, r, j, 0]
                    B[2 * r + 8:2 * r + 10, n] = ents[bb][sB, r, j, 1]
            acc[i] += A @ B
    return np.array([acc[(t % 4) // GPB][t // 4, 2 * (t % 4)] + acc[(t % 4) // GPB][t // 4 + 8, 2 * (t % 4) + 1]
                     for t in range(32)])


@pytest.mark.parametrize("fmt", ["int4", "fp4"])
@pytest.mark.parametrize("G", [128, 64, 32])
def test_set_of_blocks_gives_every_lane_a_row_group_dot_product(fmt, G):
    rng = np.random.default_rng(300 + G + (0 if fmt == "int4" else 7))
    GPB = 128 // G
    S, RB = 4 // GPB, 16
    NQ = RB // S
    qs = {b: rng.integers(0, 16, size=(8, 128)) for b in range(RB)}
    xs = {b: rng.standard_normal(128) for b in range(RB)}
    scale = 2.0 ** -24 if fmt == "int4" else 1.0
    covered = set()
    for q in range(NQ):
        lanes = emulate_set(fmt, qs, xs, G, q, NQ)
        for t in range(32):
            g, r = t // 4, t % 4
            blk, h = q + NQ * (r // GPB), r % GPB
            ks = range(h * G, (h + 1) * G)
            dq = [qs[blk][g, k] * scale if fmt == "int4" else e2m1(int(qs[blk][g, k])) for k in ks]
            want = float(np.dot(dq, xs[blk][list(ks)]))
            assert lanes[t] == pytest.approx(want, rel=1e-12, abs=1e-30), (q, t)
            covered.add((g, blk, h))
    assert len(covered) == 8 * RB * GPB          # every (row, block, group) of the item exactly once
