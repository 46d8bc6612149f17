"""The library's INT4 storage format, unpacked into plain index order for the
parity tests (test infrastructure; not part of the oracle, which has no notion
of byte layout).

include/lserve.h (lserve_quantize_pages_int4) declares where each code and
parameter sits; this module follows that prose and nothing else.  A byte holds
two codes: nibble n of a 32-bit word is bits 4n..4n+3 of the word, i.e. byte
n // 2 of the (little-endian) word, its high half when n is odd.

  kq    one row of d/2 bytes per token: four chunks of d/8 bytes; word w of chunk
        t holds nibbles n = j + 4e of channels 16 (r/2) + 8 (r%2) + 2t + e,
        r = 4w + j
  vq    one page of 64 * d/2 bytes: four slices of 16 tokens, each 32 chunks of
        d/4 bytes; word m of chunk 4g + t holds nibbles n = j + 4e of channel
        16m + g + 8 (j%2), token 16 slice + 2t + 8 (j/2) + e
  kpar  [2, d]: s, then lo, each four chunks of d/4 entries; entry i of chunk t
        is channel 16 (i/4) + 8 ((i/2)%2) + 2t + i%2
  vpar  [64, 2]: (s, lo) per token

Pinned by tests/golden/int4_layout.json (positions worked out by hand from the
same prose) and by the bijection checks in test_oracle_quant.py.
"""
import numpy as np


def key_nibble_positions(d):
    """pos[c] = nibble index (2 * byte + high) of channel c inside a key row."""
    pos = np.full(d, -1, np.int64)
    chunk = d // 8
    for t in range(4):
        for w in range(chunk // 4):
            for j in range(4):
                r = 4 * w + j
                for e in range(2):
                    c = 16 * (r // 2) + 8 * (r % 2) + 2 * t + e
                    n = j + 4 * e
                    pos[c] = 2 * (t * chunk + 4 * w + n // 2) + n % 2
    return pos


def value_nibble_positions(d):
    """pos[u, c] = nibble index of (token u, channel c) inside a page of values."""
    pos = np.full((64, d), -1, np.int64)
    chunk = d // 4
    for sl in range(4):
        for g in range(8):
            for t in range(4):
                base = (sl * 32 + 4 * g + t) * chunk
                for m in range(d // 16):
                    for j in range(4):
                        for e in range(2):
                            c = 16 * m + g + 8 * (j % 2)
                            u = 16 * sl + 2 * t + 8 * (j // 2) + e
                            n = j + 4 * e
                            pos[u, c] = 2 * (base + 4 * m + n // 2) + n % 2
    return pos


def key_param_channels(d):
    """chan[idx] = channel whose step / offset sits at index idx of a kpar row."""
    q = d // 4
    return np.array([16 * (i // 4) + 8 * ((i // 2) % 2) + 2 * t + i % 2 for t in range(4) for i in range(q)],
                    np.int64)


def _nibbles(packed):
    packed = np.asarray(packed, np.uint8)
    nib = np.empty(packed.shape[:-1] + (2 * packed.shape[-1],), np.uint8)
    nib[..., 0::2] = packed & 15
    nib[..., 1::2] = packed >> 4
    return nib


def unpack_keys(kq, d):
    """kq uint8 [..., 64, d/2] -> codes [..., 64, d]."""
    return _nibbles(kq)[..., key_nibble_positions(d)]


def unpack_values(vq, d):
    """vq uint8 [..., 64 * d/2] (or [..., 64, d/2]) -> codes [..., 64, d]."""
    vq = np.asarray(vq, np.uint8)
    flat = vq.reshape(vq.shape[:-2] + (-1,)) if vq.ndim >= 2 and vq.shape[-2] == 64 and vq.shape[-1] == d // 2 \
        else vq
    return _nibbles(flat)[..., value_nibble_positions(d)]


def unpack_key_params(kpar):
    """kpar float32 [..., 2, d] -> (step, lo), each [..., d] in channel order."""
    kpar = np.asarray(kpar, np.float32)
    d = kpar.shape[-1]
    out = np.empty_like(kpar)
    out[..., key_param_channels(d)] = kpar
    return out[..., 0, :], out[..., 1, :]


def unpack_value_params(vpar):
    """vpar float32 [..., 64, 2] -> (step, lo), each [..., 64]."""
    vpar = np.asarray(vpar, np.float32)
    return vpar[..., 0], vpar[..., 1]
