"""CPU checks of the integer identities and lane mappings the quadratic loss pass relies on
(zero_order_forward_b200/csrc/zo_loss.cu), restated here from their definitions:

- the masked multiply that gathers the sign nibbles of probes t and t + 4 from a word whose
  byte q holds element q's 8 probe signs;
- the shuffle rounds that hand each lane of a pair its own and its partner's word of each of
  its octets (two and four octets per pass), and the word rotation of the quad form.
"""
import random

WORDS = 4  # a Philox block: four 32-bit words, word q = the 4 elements of quad lane q


def test_multiply_gathers_two_probe_nibbles():
    rng = random.Random(1)
    for _ in range(20000):
        w = rng.getrandbits(32)
        for t in range(4):
            p = (((w >> t) & 0x11111111) * 0x01020408) & 0xFFFFFFFF
            for probe, shift in ((t, 24), (t + 4, 28)):
                nib = sum(((w >> (8 * q + probe)) & 1) << q for q in range(4))
                assert (p >> shift) & 0xF == nib
                # the table offset 2048 * nibble, as the kernel forms it
                off = ((p >> (shift - 11)) & 0x7800)
                assert off == nib << 11


def _pair_four_octets(blocks):
    """NOCT 4: blocks[o] is octet o's block (list of 4 words) for one vector step of a quad;
    lane q generates octet q.  Returns, per lane, (wo[2], wp[2])."""
    out = []
    for lane in range(4):
        q, h = lane, lane & 1
        sw = ((q & 1) << 1) | (q >> 1)
        R = []
        for r in range(4):
            c = r >> 1
            src = sw ^ c                       # the lane read in round r
            word = 2 * ((src & 1) ^ c) + (r & 1)  # what that lane sends in round r
            R.append(blocks[src][word])
        x = sw & 1
        e0, o0 = (R[2], R[3]) if x else (R[0], R[1])
        e1, o1 = (R[0], R[1]) if x else (R[2], R[3])
        wo = [o0 if h else e0, o1 if h else e1]
        wp = [e0 if h else o0, e1 if h else o1]
        out.append((wo, wp))
    return out


def test_pair_exchange_four_octets_delivers_own_and_partner_words():
    blocks = [[(o << 8) | w for w in range(WORDS)] for o in range(4)]  # tag = (octet, word)
    for lane, (wo, wp) in enumerate(_pair_four_octets(blocks)):
        h = lane & 1
        for j in range(2):
            octet = 2 * h + j
            assert wo[j] == (octet << 8) | lane          # own vector: word q of the octet
            assert wp[j] == (octet << 8) | (lane ^ 1)    # partner's vector


def test_pair_exchange_two_octets_delivers_both_vectors():
    # lane q generates (vector q >> 1, octet q & 1); tag = (vector, octet, word)
    blocks = {(k, o): [(k << 16) | (o << 8) | w for w in range(WORDS)] for k in range(2) for o in range(2)}
    for lane in range(4):
        q, h = lane, lane & 1
        R = []
        for r in range(4):
            c = r >> 1
            src = q ^ (2 * c)
            word = 2 * ((src >> 1) ^ c) + (r & 1)
            R.append(blocks[(src >> 1, src & 1)][word])
        x = q >> 1
        e0, o0 = (R[2], R[3]) if x else (R[0], R[1])
        e1, o1 = (R[0], R[1]) if x else (R[2], R[3])
        wo = [o0 if h else e0, o1 if h else e1]
        wp = [e0 if h else o0, e1 if h else o1]
        for k in range(2):
            assert wo[k] == (k << 16) | (h << 8) | lane
            assert wp[k] == (k << 16) | (h << 8) | (lane ^ 1)


def test_quad_word_rotation():
    # after the two conditional swaps, w[r] is word q ^ r, the vector of quad lane q ^ r
    for q in range(4):
        w = list(range(WORDS))
        if q & 1:
            w = [w[1], w[0], w[3], w[2]]
        if q & 2:
            w = [w[2], w[3], w[0], w[1]]
        assert w == [q ^ r for r in range(4)]
    # round r reads the table column of lane q ^ r: distinct across the quad in every round
    for r in range(4):
        assert sorted(q ^ r for q in range(4)) == [0, 1, 2, 3]


def test_probe_to_accumulator_mapping_covers_every_probe_once():
    # lane class c (= lane mod G) accumulates local octets j < LO as probes 8 (LO c + j) + t
    for noct, G in ((2, 2), (4, 2), (8, 4)):
        LO = noct // G
        seen = sorted(8 * (LO * c + j) + t for c in range(G) for j in range(LO) for t in range(8))
        assert seen == list(range(8 * noct))
