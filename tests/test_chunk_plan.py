"""The separation loop's geometry as the library computes it on the host (mrf_chunk_plan, the
function mrf_separate_audio uses) against the oracle's chunk plan: "Mel-Band RoFormer —
architecture, inference hot path & RTX 3050 feasibility", section "Verified inference hot path"
(8 s chunks, stride 0.9 chunk, reflect padding by the border, tail padding by reflection past
half a chunk, zeros below).  Host only, no GPU."""
import pytest

from oracle import signal

SR = 44100
CHUNK = 8 * SR
STRIDE = int(CHUNK * 0.9)
BORDER = CHUNK - STRIDE


def lengths():
    base = [2, 100, SR, int(1.7 * SR), 2 * BORDER - 1, 2 * BORDER, 2 * BORDER + 1, CHUNK - 1, CHUNK, CHUNK + 1,
            5 * SR, 9 * SR, 16 * SR, 20 * SR, 60 * SR, 120 * SR, 600 * SR]
    # lengths whose padded tail sits at or around half a chunk and a full chunk
    for k in (1, 2, 5):
        for tail in (CHUNK // 2 - 1, CHUNK // 2, CHUNK // 2 + 1, CHUNK - 1, CHUNK):
            base.append(k * STRIDE + tail - 2 * BORDER)
    return sorted(set(x for x in base if x >= 2))


@pytest.mark.parametrize("L", lengths())
def test_chunk_plan_matches_the_oracle(L):
    from axial_band_split_b200 import mrf
    got = mrf.chunk_plan(SR, L)
    chunk, border, Lp, chunks, _ = signal.chunk_plan(L, SR)
    assert got["chunk"] == chunk and got["border"] == border and got["padded_length"] == Lp
    assert len(got["off"]) == len(chunks)
    modes = {None: 0, "reflect": 1, "zeros": 2}
    for i, (off, n, mode) in enumerate(chunks):
        assert (got["off"][i], got["valid"][i], got["mode"][i]) == (off, n, modes[mode]), (i, off, n, mode)


def test_chunk_plan_rejects_bad_arguments():
    from axial_band_split_b200 import mrf
    with pytest.raises(mrf.MrfError):
        mrf.chunk_plan(0, 1000)
    with pytest.raises(mrf.MrfError):
        mrf.chunk_plan(SR, 1)


@pytest.mark.parametrize("seconds", [2.0, 4.0, 11.0, 16.0, 13.35])
@pytest.mark.parametrize("L", [5 * SR, 60 * SR, 61 * SR + 12345])
def test_chunk_plan_other_chunk_lengths_match_the_oracle(seconds, L):
    # the chunk-length sweep's geometry: every quantity scales with the chunk
    from axial_band_split_b200 import mrf
    c = int(seconds * SR)
    got = mrf.chunk_plan(SR, L, c)
    chunk, border, Lp, chunks, _ = signal.chunk_plan(L, SR, c)
    assert got["chunk"] == chunk == c and got["border"] == border and got["padded_length"] == Lp
    modes = {None: 0, "reflect": 1, "zeros": 2}
    assert [(int(o), int(n), int(m)) for o, n, m in zip(got["off"], got["valid"], got["mode"])] == \
        [(off, n, modes[mode]) for off, n, mode in chunks]


def test_chunk_plan_rejects_tiny_chunks():
    from axial_band_split_b200 import mrf
    with pytest.raises(mrf.MrfError):
        mrf.chunk_plan(SR, 1000, 5)
