"""Host-side cutting of pipelined host calls into row blocks (no GPU): every
row of every call lands in exactly one block, in order; small calls and
calls that are not 2-D stay whole."""
import pytest
import torch

import w4a8_integer_gemm_b200 as q


class _Layer:
    pass


def _call(M, K, N):
    return (torch.zeros(M, K, dtype=torch.float16), _Layer(), torch.zeros(M, N, dtype=torch.float16))


def _covered(calls, pieces):
    """Per call, the row ranges its blocks cover, from the blocks' storage."""
    out = []
    for x, _, y in calls:
        rows = []
        for px, _, py in pieces:
            if px.untyped_storage().data_ptr() == x.untyped_storage().data_ptr():
                r0 = (px.data_ptr() - x.data_ptr()) // (x.shape[1] * 2)
                assert (py.data_ptr() - y.data_ptr()) // (y.shape[1] * 2) == r0
                assert px.shape[0] == py.shape[0]
                rows.append((r0, r0 + px.shape[0]))
        out.append(rows)
    return out


@pytest.mark.parametrize("chunk_rows", [None, 1, 128, 1000, 1 << 20])
def test_blocks_cover_every_row_once(chunk_rows):
    calls = [_call(2500, 4096, 4096), _call(7, 1024, 512), _call(8192, 8192, 8192), _call(1, 64, 64)]
    pieces = q._host_pieces(calls, chunk_rows)
    for (x, _, _), rows in zip(calls, _covered(calls, pieces)):
        assert rows[0][0] == 0 and rows[-1][1] == x.shape[0]
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
        if chunk_rows is not None:
            assert all(r1 - r0 <= chunk_rows for r0, r1 in rows)
    assert all(p[1] is c[1] for p in pieces for c in calls if p[0].untyped_storage().data_ptr() == c[0].untyped_storage().data_ptr())


def test_default_blocks_are_about_16_mb():
    # K = N = 8192: 1024 rows of 16 KB each way per block
    pieces = q._host_pieces([_call(8192, 8192, 8192)], None)
    assert [p[0].shape[0] for p in pieces] == [1024] * 8
    # the wider side sets the block: N = 28672 -> 256 rows (14 MB of Y)
    pieces = q._host_pieces([_call(1000, 4096, 28672)], None)
    assert [p[0].shape[0] for p in pieces] == [256, 256, 256, 232]
    # never fewer than 128 rows per block
    pieces = q._host_pieces([_call(300, 4096, 1 << 17)], None)
    assert [p[0].shape[0] for p in pieces] == [128, 128, 44]


def test_small_and_odd_calls_stay_whole():
    small = _call(100, 8192, 8192)
    flat = (torch.zeros(3 * 4096, dtype=torch.float16), _Layer(), torch.zeros(3, 4096, dtype=torch.float16))
    pieces = q._host_pieces([small, flat], None)
    assert len(pieces) == 2 and pieces[0][0] is small[0] and pieces[1][0] is flat[0]


def test_chunk_rows_must_be_positive():
    with pytest.raises(ValueError):
        q.w4a8_linear_host_many([_call(4, 64, 64)], chunk_rows=0)
