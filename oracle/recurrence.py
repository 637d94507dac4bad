"""Second formulation of the trellis states, pure Python -- TEST INFRASTRUCTURE.

The C oracle reads each weight's state as a cyclic 16-bit window of the tile's
bit string.  This module builds the same states the other way, as a shift
register: s_i = ((s_{i-1} << K) | chunk_i) & 0xFFFF, where chunk_i is weight
i's own K bits and s_{-1} is the last 16 bits of the stream (the tail-biting
closure: the code's end feeds its start).  It follows the bitshift-trellis
description of the EXL3 GEMM kernel article (section "Viterbi编码内核剖析") and
the ExLlamaV3 overview (a QTIP-style tail-biting trellis with K bits per
weight).  Agreement of the two formulations pins the window arithmetic.
Pure-Python loops: use on small inputs only.
"""


def stream_bits(tile_words):
    """The tile's bit string, most significant bit of word 0 first."""
    bits = []
    for w in tile_words:
        w = int(w)
        for b in range(15, -1, -1):
            bits.append((w >> b) & 1)
    return bits


def tile_states(tile_words, K):
    bits = stream_bits(tile_words)
    assert len(bits) == 256 * K
    s = 0
    for b in bits[-16:]:
        s = (s << 1) | b
    out = []
    for i in range(256):
        chunk = 0
        for b in bits[i * K:(i + 1) * K]:
            chunk = (chunk << 1) | b
        s = ((s << K) | chunk) & 0xFFFF
        out.append(s)
    return out
