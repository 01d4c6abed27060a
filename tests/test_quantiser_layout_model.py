"""Host restatement of the FP8 quantiser's transposed-V store indexing (fp8_quantize_kernel:
one block per 32-token tile and head; a 16-token chunk goes out as one 16-byte store when its
tokens lie in one segment and its first key is 16-byte aligned, the other tokens as bytes), checked
on random packs: every key of every segment is written exactly once, the 16-byte stores are
aligned and inside the row, and nothing lands outside the segment's own keys (the keys between
segments are never written). The layout: segment s starts at key 16*ceil(cu[s]/16) + 16*s."""
import numpy as np
import pytest

TILE = 32


def vt_keys(cu):
    T, B = int(cu[-1]), len(cu) - 1
    return 16 * ((T + 15) // 16) + 16 * B


def key_offsets(cu):
    """Per token: key - token (16*ceil(beg/16) + 16*s - beg of its segment s)."""
    T, B = int(cu[-1]), len(cu) - 1
    off = np.zeros(T, dtype=np.int64)
    for t in range(T):
        s = int(np.searchsorted(cu, t, side="right")) - 1  # last s with cu[s] <= t
        s = min(s, B - 1)
        beg = int(cu[s])
        off[t] = 16 * ((beg + 15) // 16) + 16 * s - beg
    return off


def writes(cu):
    """(vector store starts, byte keys) of one channel row, as the kernel issues them."""
    T, K = int(cu[-1]), vt_keys(cu)
    off = key_offsets(cu)
    vec, byte = [], []
    for t0 in range(0, T, TILE):
        s_off = [off[t0 + i] if t0 + i < T else 0 for i in range(TILE)]
        for ch in range(TILE // 16):
            tf = t0 + 16 * ch
            key0 = tf + s_off[16 * ch]
            is_vec = (tf + 15 < T and s_off[16 * ch] == s_off[16 * ch + 15] and key0 % 16 == 0
                      and key0 >= 0 and key0 + 16 <= K)
            if is_vec:
                vec.append(key0)
            else:
                for i in range(16):
                    t = tf + i
                    key = t + s_off[16 * ch + i]
                    if t < T and 0 <= key < K:
                        byte.append(key)
    return vec, byte


def _packs():
    rng = np.random.default_rng(11)
    out = [[5, 250, 3, 700, 9], [1, 127, 128, 129, 300, 0, 513, 17], [128], [0, 0, 300, 0, 129, 0], [16] * 9,
           [33, 31, 64, 1, 15, 17]]
    for _ in range(20):
        out.append([int(x) for x in rng.integers(0, 200, int(rng.integers(1, 30)))])
    out.append([int(x) for x in rng.integers(0, 40, 5000)])  # more segments than the scheduler stages
    return out


@pytest.mark.parametrize("segs", _packs(), ids=lambda s: f"B{len(s)}_T{sum(s)}")
def test_transposed_v_keys_written_once_and_only_inside_segments(segs):
    cu = np.concatenate([[0], np.cumsum(segs)]).astype(np.int64)
    if cu[-1] == 0:
        return
    K = vt_keys(cu)
    vec, byte = writes(cu)
    count = np.zeros(K, dtype=np.int64)
    for k0 in vec:
        assert k0 % 16 == 0 and 0 <= k0 and k0 + 16 <= K
        count[k0:k0 + 16] += 1
    for k in byte:
        count[k] += 1
    want = np.zeros(K, dtype=np.int64)
    for s in range(len(segs)):
        k0 = 16 * ((cu[s] + 15) // 16) + 16 * s
        want[k0:k0 + segs[s]] = 1
    assert np.array_equal(count, want)


def test_vector_stores_need_a_segment_start_on_16_tokens():
    """Chunks are 16-token aligned, so a segment's keys go out as 16-byte stores only when
    it starts on a multiple of 16 tokens (then token -> key is a shift by a multiple of 16);
    otherwise every key of it is a byte store."""
    vec, byte = writes(np.array([0, 16, 1040], dtype=np.int64))
    assert 16 * len(vec) == 1040 and not byte
    vec, byte = writes(np.array([0, 5, 1029], dtype=np.int64))
    assert not vec and len(byte) == 1029
